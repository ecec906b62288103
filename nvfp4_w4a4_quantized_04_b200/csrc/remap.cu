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
// 0xFF check.  Pass 2 (reads exponents only): the scale bytes and s_g, a warp
// per 512-byte scale atom in the tensor-core layout.
#include <cuda_runtime.h>
#include <stdint.h>

#include "common.cuh"
#include "host_util.cuh"

namespace nvfp4 {

// ws[2t] = max(u+1), ws[2t+1] = max(256-u) over non-zero blocks of tensor t
// (0 = no such block), via atomicMax on zero-initialised words; or one such
// pair per CTA of the tensor (partials), reduced by the scale pass.  A CTA takes
// kScanChunk consecutive blocks of one tensor, eight per thread (128 bytes of
// codes in flight per thread); CTAs are short and not persistent.
constexpr int kScanUnroll = 8;
constexpr int64_t kScanChunk = 256 * kScanUnroll;

__global__ void __launch_bounds__(256) remap_scan_kernel(
    const uint8_t *__restrict__ q_mx, const uint8_t *__restrict__ e8, int64_t blocks_per_tensor,
    uint8_t *__restrict__ q_nv, uint32_t *__restrict__ ws, bool partials, int32_t *dev_status) {
  const int64_t t = blockIdx.y;
  const int64_t b0 = (int64_t)blockIdx.x * kScanChunk;
  const int64_t b1 = min(blocks_per_tensor, b0 + kScanChunk);
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
  const int64_t st = blockDim.x;
  int64_t b = b0 + threadIdx.x;
  if (b0 + kScanChunk <= blocks_per_tensor) {
    uint4 c[kScanUnroll];
    uint32_t u[kScanUnroll];
#pragma unroll
    for (int k = 0; k < kScanUnroll; ++k) c[k] = __ldg(qt + b + k * st);
#pragma unroll
    for (int k = 0; k < kScanUnroll; ++k) u[k] = et[b + k * st];
    if (copy) {
#pragma unroll
      for (int k = 0; k < kScanUnroll; ++k) qo[b + k * st] = c[k];
    }
#pragma unroll
    for (int k = 0; k < kScanUnroll; ++k) visit(c[k], u[k]);
  } else {
    for (; b < b1; b += st) {
      const uint4 c = __ldg(qt + b);
      if (copy) qo[b] = c;
      visit(c, et[b]);
    }
  }
#pragma unroll
  for (int d = 16; d > 0; d >>= 1) {
    hi = max(hi, __shfl_xor_sync(0xffffffffu, hi, d));
    lo = max(lo, __shfl_xor_sync(0xffffffffu, lo, d));
  }
  // one pair of atomics per CTA: the words of a tensor are shared by all of
  // its CTAs, so same-address atomics are what this pass must keep few
  __shared__ uint32_t red[2][8];
  if ((threadIdx.x & 31) == 0) {
    red[0][threadIdx.x >> 5] = hi;
    red[1][threadIdx.x >> 5] = lo;
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    for (int w = 1; w < (int)(blockDim.x >> 5); ++w) {
      hi = max(hi, red[0][w]);
      lo = max(lo, red[1][w]);
    }
    if (partials) {
      // this CTA's own pair of words: every pair is written, so nothing needs
      // clearing first, and the scale pass reduces a tensor's pairs
      const int64_t slot = t * gridDim.x + blockIdx.x;
      ws[2 * slot] = hi;
      ws[2 * slot + 1] = lo;
    } else if (hi) {
      atomicMax(&ws[2 * t], hi);
      atomicMax(&ws[2 * t + 1], lo);
    }
  }
  if (bad) report(dev_status, NVFP4_ERR_NOT_REPRESENTABLE);
}

// E4M3 byte of 2^p, p in [-9, 8].
__device__ __forceinline__ uint32_t e4m3_pow2(int p) {
  return p >= -6 ? (uint32_t)((p + 7) << 3) : (1u << (p + 9));
}

// Tensor-core scale layout: a warp writes 512-byte atoms (row block, group of
// four 16-element scales), up to kAtomRun consecutive groups of one row block
// per work unit, so the 32-byte sectors of UE8M0 bytes it reads (16 groups of
// a row) come from L2 once and are reused from L1.  In an atom, lane l covers
// rows l, l+32, l+64 and l+96 of the row block: for each it reads the two
// UE8M0 bytes of the group's 64 elements and writes the four scale bytes
// (each 32-block's byte twice) as one 16-byte line.  Lane 0 of a tensor's
// first unit also writes s_g and checks the exponent spread.
constexpr int64_t kAtomRun = 16;

// The tensor's exponent words: one pair (npart == 0), or the max over its
// npart per-CTA pairs.
__device__ __forceinline__ int remap_global_exp(const uint32_t *__restrict__ ws, int64_t t, int npart, uint32_t &hi,
                                                uint32_t &lo) {
  if (npart == 0) {
    hi = ws[2 * t];
    lo = ws[2 * t + 1];
  } else {
    hi = 0;
    lo = 0;
    for (int i = 0; i < npart; ++i) {
      hi = max(hi, ws[2 * (t * npart + i)]);
      lo = max(lo, ws[2 * (t * npart + i) + 1]);
    }
  }
  return hi ? (int)hi - 1 - 127 - 8 : 0;
}

__global__ void __launch_bounds__(256) remap_scale_atoms_kernel(
    const uint8_t *__restrict__ e8, int64_t rows, int64_t K, int64_t n_tensors,
    const uint32_t *__restrict__ ws, int npart, uint8_t *__restrict__ sf, float *__restrict__ gs, bool vec,
    int32_t *dev_status) {
  const int lane = threadIdx.x & 31;
  const int64_t rb_per_t = rows >> 7, kg_per_row = K >> 6, nb32 = K >> 5;
  const int64_t runs_per_rb = (kg_per_row + kAtomRun - 1) / kAtomRun;
  const int64_t units_per_t = rb_per_t * runs_per_rb;
  const int64_t total = n_tensors * units_per_t;
  const int64_t nwarps = ((int64_t)gridDim.x * blockDim.x) >> 5;
  for (int64_t u = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5; u < total; u += nwarps) {
    const int64_t t = u / units_per_t, w = u - t * units_per_t;
    const int64_t rb = w / runs_per_rb, kg0 = (w - rb * runs_per_rb) * kAtomRun;
    const int64_t kg1 = min(kg_per_row, kg0 + kAtomRun);
    uint32_t hi, lo;
    const int g = remap_global_exp(ws, t, npart, hi, lo);
    if (w == 0 && lane == 0) {
      gs[t] = ldexpf(1.0f, g);   // 2^g exactly, g in [-135, 119] (subnormal below -126)
      if (hi && (256 - (int)lo - 127) - g < -9) report(dev_status, NVFP4_ERR_NOT_REPRESENTABLE);
    }
    const uint8_t *rows0 = e8 + (t * rows + rb * 128 + lane) * nb32;
    uint8_t *atom = sf + (t * rb_per_t + rb) * kg_per_row * 512 + lane * 16;
    const int kr = (int)(kg1 - kg0);
    // the run's UE8M0 bytes of this lane's four rows, loaded up front: one or
    // two 16-byte loads per row when they are aligned and the run is 8 or 16
    // groups long (then they end inside the run), single bytes otherwise
    uint32_t ew[4][8];
#pragma unroll
    for (int qd = 0; qd < 4; ++qd) {
      const uint8_t *er = rows0 + qd * 32 * nb32 + 2 * kg0;
      if (vec && (kr == 8 || kr == 16)) {
        const uint4 a = __ldg(reinterpret_cast<const uint4 *>(er));
        const uint4 b = kr == 16 ? __ldg(reinterpret_cast<const uint4 *>(er) + 1) : make_uint4(0, 0, 0, 0);
        ew[qd][0] = a.x; ew[qd][1] = a.y; ew[qd][2] = a.z; ew[qd][3] = a.w;
        ew[qd][4] = b.x; ew[qd][5] = b.y; ew[qd][6] = b.z; ew[qd][7] = b.w;
      } else {
#pragma unroll
        for (int w8 = 0; w8 < 8; ++w8) {
          uint32_t v = 0;
#pragma unroll
          for (int by = 0; by < 4; ++by)
            if (4 * w8 + by < 2 * kr) v |= (uint32_t)er[4 * w8 + by] << (8 * by);
          ew[qd][w8] = v;
        }
      }
    }
#pragma unroll
    for (int i = 0; i < (int)kAtomRun; ++i) {
      if (i < kr) {
        uint32_t words[4];
#pragma unroll
        for (int qd = 0; qd < 4; ++qd) {
          const uint32_t pair = ew[qd][i >> 1] >> (16 * (i & 1));     // UE8M0 bytes of blocks 2(kg0+i), +1
          const uint32_t S0 = e4m3_pow2(max(-9, min(8, (int)(pair & 0xFFu) - 127 - g)));
          const uint32_t S1 = e4m3_pow2(max(-9, min(8, (int)((pair >> 8) & 0xFFu) - 127 - g)));
          words[qd] = S0 * 0x0101u | S1 * 0x01010000u;
        }
        *reinterpret_cast<uint4 *>(atom + (kg0 + i) * 512) = make_uint4(words[0], words[1], words[2], words[3]);
      }
    }
  }
}

// Row-major scale layout: MX block i (over all tensors) gives scales 2i and
// 2i+1, written as one 2-byte store.
__global__ void __launch_bounds__(256) remap_scale_rows_kernel(
    const uint8_t *__restrict__ e8, int64_t per_tensor, int64_t n_tensors, const uint32_t *__restrict__ ws,
    int npart, uint8_t *__restrict__ sf, float *__restrict__ gs, int32_t *dev_status) {
  const uint64_t total = (uint64_t)n_tensors * (uint64_t)per_tensor;
  const uint64_t stride = (uint64_t)gridDim.x * blockDim.x;
  for (uint64_t i = (uint64_t)blockIdx.x * blockDim.x + threadIdx.x; i < total; i += stride) {
    const uint64_t t = i / (uint64_t)per_tensor, within = i - t * (uint64_t)per_tensor;
    uint32_t hi, lo;
    const int g = remap_global_exp(ws, (int64_t)t, npart, hi, lo);
    if (within == 0) {
      gs[t] = ldexpf(1.0f, g);   // 2^g exactly, g in [-135, 119] (subnormal below -126)
      if (hi && (256 - (int)lo - 127) - g < -9) report(dev_status, NVFP4_ERR_NOT_REPRESENTABLE);
    }
    const uint32_t S = e4m3_pow2(max(-9, min(8, (int)e8[i] - 127 - g)));
    *reinterpret_cast<uint16_t *>(sf + 2 * i) = (uint16_t)(S | (S << 8));
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
  const int64_t bpt = rows * (K / 32);
  const int64_t xblocks = (bpt + kScanChunk - 1) / kScanChunk;
  if (xblocks > 0x7FFFFFFF) return NVFP4_ERR_UNSUPPORTED_SHAPE;
  dim3 grid1((unsigned)xblocks, (unsigned)n_tensors);
  if (grid1.y > 65535) return NVFP4_ERR_UNSUPPORTED_SHAPE;
  // Up to kMaxPartials scan CTAs per tensor: each writes its own pair of
  // words (8 bytes per CTA, within nvfp4_workspace_size(n_tensors)) and the
  // scale pass reduces them, so no clearing launch is needed.  More CTAs per
  // tensor: atomics on one zero-initialised pair per tensor.
  constexpr int64_t kMaxPartials = 64;
  const int npart = xblocks <= kMaxPartials ? (int)xblocks : 0;
  if (npart == 0 && cudaMemsetAsync(ws, 0, sizeof(uint32_t) * 2 * n_tensors, stream) != cudaSuccess)
    return NVFP4_ERR_CUDA;
  remap_scan_kernel<<<grid1, 256, 0, stream>>>(q_mx, ue8m0, bpt, q_nv, ws, npart != 0, dev_status);
  if (cudaGetLastError() != cudaSuccess) return NVFP4_ERR_CUDA;
  const int sms = host::sm_count();
  if (sf_layout == NVFP4_SF_MMA_TILED) {
    const int64_t units = n_tensors * (rows / 128) * ((K / 64 + kAtomRun - 1) / kAtomRun);
    int64_t blocks = (units + 7) / 8;                      // a warp per unit, 8 warps per CTA
    if (blocks > (int64_t)sms * 8) blocks = (int64_t)sms * 8;
    // 16-byte exponent loads need 16-byte aligned rows of exponents
    const bool vec = (reinterpret_cast<uintptr_t>(ue8m0) & 15u) == 0 && (K / 32) % 16 == 0;
    remap_scale_atoms_kernel<<<(unsigned)blocks, 256, 0, stream>>>(ue8m0, rows, K, n_tensors, ws, npart, sf_nv,
                                                                   global_scale, vec, dev_status);
  } else {
    const int64_t total = n_tensors * bpt;
    int64_t blocks = (total + 255) / 256;
    if (blocks > (int64_t)sms * 8) blocks = (int64_t)sms * 8;
    remap_scale_rows_kernel<<<(unsigned)blocks, 256, 0, stream>>>(ue8m0, bpt, n_tensors, ws, npart, sf_nv,
                                                                   global_scale, dev_status);
  }
  return cudaGetLastError() == cudaSuccess ? NVFP4_OK : NVFP4_ERR_CUDA;
}
