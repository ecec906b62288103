// MXFP4 encoder (sm_100a): bf16 rows -> E2M1 codes with one UE8M0
// (power-of-two) scale per 32 elements.
//
// "DeepSeek-V4.1-Flash-NVFP4", format table of the format section: MXFP4
// blocks are 32 elements wide with a UE8M0 scale; its which-layers section
// converts an FP8 table to MXFP4 this way (lossy).  The page gives no rule
// for the exponent; the one used is the OCP Microscaling v1.0 conversion:
// E = floor(log2 amax) - 2 (2 is the exponent of 6, the largest E2M1
// magnitude), clamped to the UE8M0 range, and code_k = e2m1_rne_satfinite(
// x_k * 2^-E).  For a bf16 amax with biased exponent field eb the byte is
// u = E + 127 = max(eb - 2, 0) (a zero or subnormal amax gives 0), and 2^-E
// is the fp32 normal with exponent field 254 - u, so the multiply is exact
// unless the product is below the fp32 normal range, where it rounds to a
// value that encodes as (signed) zero either way.
//
// HBM-bound (2 bytes read, 0.53 written per element): one thread per
// 32-element block, 64 bytes of loads in flight per thread, a 16-byte code
// store per thread (warp-contiguous) and one scale byte.
#include <cuda_runtime.h>
#include <stdint.h>

#include "common.cuh"
#include "host_util.cuh"

namespace nvfp4 {
namespace {

__device__ __forceinline__ void load64(const uint16_t *p, bool v8, uint4 (&v)[4]) {
  if (v8) {
#pragma unroll
    for (int h = 0; h < 2; ++h)
      asm volatile("ld.global.nc.L1::no_allocate.v8.b32 {%0,%1,%2,%3,%4,%5,%6,%7}, [%8];"
                   : "=r"(v[2 * h].x), "=r"(v[2 * h].y), "=r"(v[2 * h].z), "=r"(v[2 * h].w),
                     "=r"(v[2 * h + 1].x), "=r"(v[2 * h + 1].y), "=r"(v[2 * h + 1].z), "=r"(v[2 * h + 1].w)
                   : "l"(p + 16 * h));
  } else {
#pragma unroll
    for (int k = 0; k < 4; ++k)
      asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
                   : "=r"(v[k].x), "=r"(v[k].y), "=r"(v[k].z), "=r"(v[k].w) : "l"(p + 8 * k));
  }
}

// Eight bf16 (one uint4) times the power of two `s` -> one word of eight E2M1
// codes, element 2i in the low nibble of byte i.
__device__ __forceinline__ uint32_t scale_encode8(uint4 v, float s) {
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
  float f[8];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    f[2 * i] = __fmul_rn(__uint_as_float(w[i] << 16), s);
    f[2 * i + 1] = __fmul_rn(__uint_as_float(w[i] & 0xFFFF0000u), s);
  }
  return f32x8_to_e2m1x8(f);
}

// Same byte split as the tensor-core scale atoms of the NVFP4 layout, with
// one scale per 32 elements: 128-row blocks, groups of 4 scales (128
// elements), 512-byte atoms.
__device__ __forceinline__ uint64_t mx_tiled_offset(uint32_t r, uint32_t b, uint32_t nb) {
  return ((uint64_t)(r >> 7) * (nb >> 2) + (b >> 2)) * 512 + (r & 31) * 16 + ((r & 127) >> 5) * 4 + (b & 3);
}

template <bool kTiled>
__global__ void __launch_bounds__(256) mxfp4_quantize_kernel(
    const uint16_t *__restrict__ x, int64_t ld_x, uint32_t nb, uint32_t total, uint32_t fd_m,
    uint32_t fd_l, uint8_t *__restrict__ q, uint8_t *__restrict__ e8, int32_t *dev_status) {
  const bool v8 = ((reinterpret_cast<uintptr_t>(x) & 31u) == 0) && ((ld_x & 15) == 0);
  bool bad = false;
  const uint32_t stride = gridDim.x * blockDim.x;
  for (uint32_t i = blockIdx.x * blockDim.x + threadIdx.x; i < total; i += stride) {
    // i / nb by a multiply-high (Granlund-Montgomery constants from the host)
    const uint32_t r = (uint32_t)(((uint64_t)__umulhi(i, fd_m) + i) >> fd_l);
    const uint32_t b = i - r * nb;
    uint4 v[4];
    load64(x + (int64_t)r * ld_x + (int64_t)b * 32, v8, v);
    uint32_t m = 0;
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      m = __vmaxu2(m, v[k].x & 0x7FFF7FFFu);
      m = __vmaxu2(m, v[k].y & 0x7FFF7FFFu);
      m = __vmaxu2(m, v[k].z & 0x7FFF7FFFu);
      m = __vmaxu2(m, v[k].w & 0x7FFF7FFFu);
    }
    m = max(m & 0xFFFFu, m >> 16);
    uint32_t u;
    uint4 codes;
    if (m >= 0x7F80u) {                       // NaN or inf in the block
      bad = true;
      u = 0xFFu;
      codes = make_uint4(0, 0, 0, 0);
    } else {
      const uint32_t eb = m >> 7;             // biased exponent field of the amax
      u = eb > 2u ? eb - 2u : 0u;
      const float s = __uint_as_float((254u - u) << 23);   // 2^-E, E = u - 127
      codes = make_uint4(scale_encode8(v[0], s), scale_encode8(v[1], s), scale_encode8(v[2], s),
                         scale_encode8(v[3], s));
    }
    *reinterpret_cast<uint4 *>(q + (uint64_t)i * 16) = codes;
    e8[kTiled ? mx_tiled_offset(r, b, nb) : (uint64_t)i] = (uint8_t)u;
  }
  if (bad) report(dev_status, NVFP4_ERR_NONFINITE);
}

}  // namespace
}  // namespace nvfp4

using namespace nvfp4;

extern "C" nvfp4_status mxfp4_quantize(const void *x, int64_t rows, int64_t K, int64_t ld_x, uint8_t *q,
                                       uint8_t *ue8m0, nvfp4_sf_layout sf_layout, int32_t *dev_status,
                                       cudaStream_t stream) {
  if (rows < 0 || K <= 0 || ld_x < K) return NVFP4_ERR_INVALID_ARG;
  if (K % 32 != 0 || ld_x % 8 != 0) return NVFP4_ERR_UNSUPPORTED_SHAPE;
  if (sf_layout != NVFP4_SF_ROWMAJOR && sf_layout != NVFP4_SF_MMA_TILED) return NVFP4_ERR_INVALID_ARG;
  if (sf_layout == NVFP4_SF_MMA_TILED && K % 128 != 0) return NVFP4_ERR_UNSUPPORTED_SHAPE;
  if (rows == 0) return NVFP4_OK;
  if (!x || !q || !ue8m0) return NVFP4_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(x) & 15u) || (reinterpret_cast<uintptr_t>(q) & 15u)) return NVFP4_ERR_INVALID_ARG;
  const uint64_t nb = (uint64_t)(K / 32);
  const uint64_t total = (uint64_t)rows * nb;
  if (total >= (1ull << 31)) return NVFP4_ERR_UNSUPPORTED_SHAPE;
  // Granlund-Montgomery (1994) constants for division by nb
  uint32_t l = 0;
  while (l < 32 && (1ull << l) < nb) ++l;
  const uint32_t m = (uint32_t)((((1ull << 32) * ((1ull << l) - nb)) / nb) + 1);
  // one wave of resident 256-thread blocks (8 per SM) at most
  uint64_t grid = (total + 255) / 256;
  const uint64_t cap = (uint64_t)host::sm_count() * 8;
  if (grid > cap) grid = cap;
  const uint16_t *xb = reinterpret_cast<const uint16_t *>(x);
  if (sf_layout == NVFP4_SF_MMA_TILED)
    mxfp4_quantize_kernel<true><<<(unsigned)grid, 256, 0, stream>>>(xb, ld_x, (uint32_t)nb, (uint32_t)total, m, l,
                                                                    q, ue8m0, dev_status);
  else
    mxfp4_quantize_kernel<false><<<(unsigned)grid, 256, 0, stream>>>(xb, ld_x, (uint32_t)nb, (uint32_t)total, m, l,
                                                                     q, ue8m0, dev_status);
  return cudaGetLastError() == cudaSuccess ? NVFP4_OK : NVFP4_ERR_CUDA;
}
