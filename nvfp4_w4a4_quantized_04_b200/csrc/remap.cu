// Lossless MXFP4 -> NVFP4 weight remap (sm_100a).
//
// "DeepSeek-V4.1-Flash-NVFP4", format section: MXFP4 holds 32-element blocks
// with a power-of-two (UE8M0) scale, NVFP4 16-element blocks with a finer
// scale, so the weights remap block by block without loss; the repository's
// conversion script does the "E2M1 -> E4M3" remap.  The E2M1 codes are kept;
// each 32-block with scale 2^e becomes two 16-blocks with the E4M3 scale
// 2^(e-g), where s_g = 2^g is the per-tensor FP32 global.  E4M3 holds
// exactly 2^-9 .. 2^8, so g = e_max - 8 and a tensor whose exponent spread
// exceeds 17 cannot be remapped losslessly (reported, not trapped).
//
// Pass 1 (reads codes + exponents, writes the code copy): per tensor, the
// largest and smallest exponent over blocks that are not all +-0, and the
// 0xFF check.  Pass 2 (reads exponents only): the scale bytes and s_g.
#include <cuda_runtime.h>
#include <stdint.h>

#include "common.cuh"

namespace nvfp4 {

// ws[2t] = max(u+1), ws[2t+1] = max(256-u) over non-zero blocks of tensor t
// (0 = no such block), via atomicMax on zero-initialised words.
__global__ void __launch_bounds__(256) remap_scan_kernel(
    const uint8_t *__restrict__ q_mx, const uint8_t *__restrict__ e8, int64_t blocks_per_tensor,
    int64_t chunk, uint8_t *__restrict__ q_nv, uint32_t *__restrict__ ws, int32_t *dev_status) {
  const int64_t t = blockIdx.y;
  const int64_t b0 = (int64_t)blockIdx.x * chunk;
  const int64_t b1 = min(blocks_per_tensor, b0 + chunk);
  const uint4 *qt = reinterpret_cast<const uint4 *>(q_mx) + t * blocks_per_tensor;
  uint4 *qo = reinterpret_cast<uint4 *>(q_nv) + t * blocks_per_tensor;
  const uint8_t *et = e8 + t * blocks_per_tensor;
  uint32_t hi = 0, lo = 0;
  bool bad = false;
  const bool copy = qo != qt;
  auto visit = [&](uint4 c, uint32_t u) {
    if (u == 0xFFu) { bad = true; return; }
    const uint32_t nz = (c.x | c.y | c.z | c.w) & 0x77777777u;   // magnitude bits
    if (nz) {
      hi = max(hi, u + 1u);
      lo = max(lo, 256u - u);
    }
  };
  // four blocks (64 bytes of codes) in flight per thread
  int64_t b = b0 + threadIdx.x;
  const int64_t st = blockDim.x;
  for (; b + 3 * st < b1; b += 4 * st) {
    const uint4 c0 = __ldg(qt + b), c1 = __ldg(qt + b + st), c2 = __ldg(qt + b + 2 * st), c3 = __ldg(qt + b + 3 * st);
    const uint32_t u0 = et[b], u1 = et[b + st], u2 = et[b + 2 * st], u3 = et[b + 3 * st];
    if (copy) { qo[b] = c0; qo[b + st] = c1; qo[b + 2 * st] = c2; qo[b + 3 * st] = c3; }
    visit(c0, u0); visit(c1, u1); visit(c2, u2); visit(c3, u3);
  }
  for (; b < b1; b += st) {
    const uint4 c = __ldg(qt + b);
    if (copy) qo[b] = c;
    visit(c, et[b]);
  }
#pragma unroll
  for (int d = 16; d > 0; d >>= 1) {
    hi = max(hi, __shfl_xor_sync(0xffffffffu, hi, d));
    lo = max(lo, __shfl_xor_sync(0xffffffffu, lo, d));
  }
  if ((threadIdx.x & 31) == 0 && hi) {
    atomicMax(&ws[2 * t], hi);
    atomicMax(&ws[2 * t + 1], lo);
  }
  if (bad) report(dev_status, NVFP4_ERR_NOT_REPRESENTABLE);
}

// E4M3 byte of 2^p, p in [-9, 8].
__device__ __forceinline__ uint32_t e4m3_pow2(int p) {
  return p >= -6 ? (uint32_t)((p + 7) << 3) : (1u << (p + 9));
}

template <bool kTiled>
__global__ void __launch_bounds__(256) remap_scale_kernel(
    const uint8_t *__restrict__ e8, int64_t rows, int64_t K, int64_t n_tensors,
    const uint32_t *__restrict__ ws, uint8_t *__restrict__ sf, float *__restrict__ gs,
    int32_t *dev_status) {
  const uint64_t nb32_row = (uint64_t)(K >> 5);
  const uint64_t per_tensor = (uint64_t)rows * nb32_row;
  const uint64_t total = (uint64_t)n_tensors * per_tensor;
  const uint64_t nsf = (uint64_t)(K >> 4);
  const uint64_t stride = (uint64_t)gridDim.x * blockDim.x;
  const bool small = total < 0xFFFFFFF0ull;
  for (uint64_t i = (uint64_t)blockIdx.x * blockDim.x + threadIdx.x; i < total; i += stride) {
    uint64_t t, within, r, jb;
    if (small) {
      const uint32_t i32 = (uint32_t)i, t32 = i32 / (uint32_t)per_tensor;
      const uint32_t w32 = i32 - t32 * (uint32_t)per_tensor, r32 = w32 / (uint32_t)nb32_row;
      t = t32; within = w32; r = r32; jb = w32 - r32 * (uint32_t)nb32_row;
    } else {
      t = i / per_tensor; within = i - t * per_tensor; r = within / nb32_row; jb = within - r * nb32_row;
    }
    const uint32_t hi = ws[2 * t], lo = ws[2 * t + 1];
    const int g = hi ? (int)hi - 1 - 127 - 8 : 0;
    if (within == 0) {
      gs[t] = ldexpf(1.0f, g);   // 2^g exactly, g in [-135, 119] (subnormal below -126)
      if (hi) {
        const int emin = 256 - (int)lo - 127;
        if (emin - g < -9) report(dev_status, NVFP4_ERR_NOT_REPRESENTABLE);
      }
    }
    const int e = (int)e8[i] - 127;
    const int p = max(-9, min(8, e - g));
    const uint32_t S = e4m3_pow2(p);
    const uint64_t row = t * (uint64_t)rows + r, j = 2 * jb;
    if (kTiled) {
      // scales j and j+1 share one 4-scale group: two adjacent bytes
      *reinterpret_cast<uint16_t *>(sf + sf_tiled_offset(row, j, nsf)) = (uint16_t)(S | (S << 8));
    } else {
      *reinterpret_cast<uint16_t *>(sf + row * nsf + j) = (uint16_t)(S | (S << 8));
    }
  }
}

}  // namespace nvfp4

using namespace nvfp4;

extern "C" nvfp4_status mxfp4_to_nvfp4(const uint8_t *q_mx, const uint8_t *ue8m0, int64_t n_tensors,
                                       int64_t rows, int64_t K, uint8_t *q_nv, uint8_t *sf_nv,
                                       nvfp4_sf_layout sf_layout, float *global_scale,
                                       void *workspace, int32_t *dev_status, cudaStream_t stream) {
  if (n_tensors < 0 || rows < 0 || K <= 0) return NVFP4_ERR_INVALID_ARG;
  if (K % 32 != 0) return NVFP4_ERR_UNSUPPORTED_SHAPE;
  if (sf_layout != NVFP4_SF_ROWMAJOR && sf_layout != NVFP4_SF_MMA_TILED) return NVFP4_ERR_INVALID_ARG;
  if (sf_layout == NVFP4_SF_MMA_TILED && (K % 64 != 0 || rows % 128 != 0)) return NVFP4_ERR_UNSUPPORTED_SHAPE;
  if (n_tensors > kMaxGroups * 16) return NVFP4_ERR_UNSUPPORTED_SHAPE;
  if (n_tensors == 0 || rows == 0) return NVFP4_OK;
  if (!q_mx || !ue8m0 || !q_nv || !sf_nv || !global_scale || !workspace) return NVFP4_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(q_mx) | reinterpret_cast<uintptr_t>(q_nv) |
       reinterpret_cast<uintptr_t>(workspace)) & 15u) return NVFP4_ERR_INVALID_ARG;
  if (sf_layout == NVFP4_SF_ROWMAJOR && (reinterpret_cast<uintptr_t>(sf_nv) & 1u)) return NVFP4_ERR_INVALID_ARG;
  uint32_t *ws = reinterpret_cast<uint32_t *>(workspace);
  if (cudaMemsetAsync(ws, 0, sizeof(uint32_t) * 2 * n_tensors, stream) != cudaSuccess) return NVFP4_ERR_CUDA;
  const int64_t bpt = rows * (K / 32);
  const int64_t chunk = 8192;
  dim3 grid1((unsigned)((bpt + chunk - 1) / chunk), (unsigned)n_tensors);
  if (grid1.y > 65535) return NVFP4_ERR_UNSUPPORTED_SHAPE;
  remap_scan_kernel<<<grid1, 256, 0, stream>>>(q_mx, ue8m0, bpt, chunk, q_nv, ws, dev_status);
  if (cudaGetLastError() != cudaSuccess) return NVFP4_ERR_CUDA;
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int64_t total = n_tensors * bpt;
  int64_t blocks = (total + 255) / 256;
  if (blocks > (int64_t)sms * 8) blocks = (int64_t)sms * 8;
  if (sf_layout == NVFP4_SF_MMA_TILED)
    remap_scale_kernel<true><<<(unsigned)blocks, 256, 0, stream>>>(ue8m0, rows, K, n_tensors, ws, sf_nv, global_scale, dev_status);
  else
    remap_scale_kernel<false><<<(unsigned)blocks, 256, 0, stream>>>(ue8m0, rows, K, n_tensors, ws, sf_nv, global_scale, dev_status);
  return cudaGetLastError() == cudaSuccess ? NVFP4_OK : NVFP4_ERR_CUDA;
}
