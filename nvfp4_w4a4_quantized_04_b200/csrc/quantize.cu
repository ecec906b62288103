// NVFP4 quantize / dequantize / SwiGLU-requantize / KV kernels (sm_100a).
//
// Two-level scaling as the "Qwen3.8-Flash-Next-NVFP4" page's W4A4 section
// describes it: a per-tensor (or per expert group) FP32 global scale, one
// FP8 E4M3 scale per 16 elements along the last dimension, E2M1 values
// packed two per byte ("DeepSeek-V4.1-Flash-NVFP4", format section).
//
// The activation path is HBM-bound (about 2.5 bytes moved per element), so
// the kernels here are plain streaming kernels: 16-byte vector loads, one
// thread pair per 16-element block, warp-contiguous stores, grids sized in
// multiples of the SM count with grid-stride loops.
#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <stdint.h>

#include <mutex>

#include "common.cuh"
#include "host_util.cuh"

namespace nvfp4 {

__device__ __forceinline__ uint4 ldg_nc_v4(const void *p) {
  uint4 v;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "l"(p));
  return v;
}

// max of |bf16| over the 8 halves of a uint4, as 16-bit magnitude bits
// (NaN patterns compare above inf, so a non-finite element shows up as >= 0x7F80).
__device__ __forceinline__ uint32_t absmax8_bits(uint4 v, uint32_t m) {
  m = __vmaxu2(m, v.x & 0x7FFF7FFFu);
  m = __vmaxu2(m, v.y & 0x7FFF7FFFu);
  m = __vmaxu2(m, v.z & 0x7FFF7FFFu);
  m = __vmaxu2(m, v.w & 0x7FFF7FFFu);
  return m;
}

__device__ __forceinline__ uint32_t halves_max(uint32_t m) { return max(m & 0xFFFFu, m >> 16); }

__device__ __forceinline__ uint32_t warp_max(uint32_t m) {
#pragma unroll
  for (int d = 16; d > 0; d >>= 1) m = max(m, __shfl_xor_sync(0xffffffffu, m, d));
  return m;
}

// ---------------------------------------------------------------- pass 1: amax
// Each warp owns a contiguous range of result rows; it keeps a running max
// while the rows stay in one group and flushes one atomicMax per group run.
__global__ void __launch_bounds__(256) amax_rows_kernel(
    const uint16_t *__restrict__ x, int64_t ld_x, int64_t K, int64_t rows,
    const int32_t *__restrict__ row_index, const int32_t *__restrict__ group_offsets, int G,
    uint32_t *__restrict__ amax_bits) {
  extern __shared__ int32_t smem[];
  int32_t *off = smem;
  if (group_offsets) {
    for (int i = threadIdx.x; i <= G; i += blockDim.x) off[i] = group_offsets[i];
    __syncthreads();
  }
  const int lane = threadIdx.x & 31;
  const int64_t warp = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int64_t nwarps = ((int64_t)gridDim.x * blockDim.x) >> 5;
  const int64_t per = (rows + nwarps - 1) / nwarps;
  const int64_t r0 = warp * per, r1 = min(rows, r0 + per);
  if (r0 >= r1) return;
  const int64_t nvec = K >> 3;
  int g = group_offsets ? upper_group(off, G, r0) : 0;
  uint32_t m = 0;
  for (int64_t r = r0; r < r1; ++r) {
    if (group_offsets) {
      int gn = g;
      while (gn + 1 < G && off[gn + 1] <= r) ++gn;
      if (gn != g) {
        uint32_t mm = warp_max(halves_max(m));
        if (lane == 0 && mm) atomicMax(&amax_bits[g], mm << 16);
        m = 0;
        g = gn;
      }
    }
    const int64_t src = row_index ? (int64_t)row_index[r] : r;
    const uint16_t *row = x + src * ld_x;
    int64_t c = lane;
#pragma unroll 1
    for (; c + 96 < nvec; c += 128) {
      uint4 a = ldg_nc_v4(row + 8 * c), b = ldg_nc_v4(row + 8 * (c + 32));
      uint4 d = ldg_nc_v4(row + 8 * (c + 64)), e = ldg_nc_v4(row + 8 * (c + 96));
      m = absmax8_bits(a, m); m = absmax8_bits(b, m);
      m = absmax8_bits(d, m); m = absmax8_bits(e, m);
    }
    for (; c < nvec; c += 32) m = absmax8_bits(ldg_nc_v4(row + 8 * c), m);
  }
  uint32_t mm = warp_max(halves_max(m));
  if (lane == 0 && mm) atomicMax(&amax_bits[g], mm << 16);
}

// One 16-element bf16 block: a 32-byte load when v8 (32-byte aligned), else two 16-byte loads.
__device__ __forceinline__ void load_block(const uint16_t *p, bool v8, uint4 &a, uint4 &b) {
  if (v8) {
    asm volatile("ld.global.nc.L1::no_allocate.v8.b32 {%0,%1,%2,%3,%4,%5,%6,%7}, [%8];"
                 : "=r"(a.x), "=r"(a.y), "=r"(a.z), "=r"(a.w), "=r"(b.x), "=r"(b.y), "=r"(b.z), "=r"(b.w)
                 : "l"(p));
  } else {
    a = ldg_nc_v4(p);
    b = ldg_nc_v4(p + 8);
  }
}

// Dense contiguous tensor: flat grid-stride over 16-element blocks (32 bytes,
// one 32-byte load when x is 32-byte aligned).  Four blocks, 128 bytes, are in
// flight per thread and at least four CTAs of 256 threads fit on an SM, so
// each SM keeps 128 KB of loads outstanding; the grid is one resident wave.
template <bool kV8>
__global__ void __launch_bounds__(256, 4) amax_flat_kernel(const uint16_t *__restrict__ x, int64_t nblk,
                                                           uint32_t *__restrict__ amax_bits) {
  const int64_t tid = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  const int64_t stride = (int64_t)gridDim.x * blockDim.x;
  uint32_t m = 0;
  int64_t i = tid;
  for (; i + 3 * stride < nblk; i += 4 * stride) {
    uint4 a[4], b[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) load_block(x + (uint64_t)(i + k * stride) * 16, kV8, a[k], b[k]);
#pragma unroll
    for (int k = 0; k < 4; ++k) m = absmax8_bits(b[k], absmax8_bits(a[k], m));
  }
  for (; i < nblk; i += stride) {
    uint4 a, b;
    load_block(x + (uint64_t)i * 16, kV8, a, b);
    m = absmax8_bits(b, absmax8_bits(a, m));
  }
  m = warp_max(halves_max(m));
  __shared__ uint32_t red[8];
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = m;
  __syncthreads();
  if (threadIdx.x == 0) {
    uint32_t b = 0;
    for (int w = 0; w < (int)(blockDim.x >> 5); ++w) b = max(b, red[w]);
    if (b) atomicMax(amax_bits, b << 16);
  }
}

// s_g from the bit pattern of a non-negative amax: amax / 2688 in one IEEE
// division (2688 = 6 * 448, so the block holding the amax gets the E4M3 scale
// 448), 1 for an amax of 0, NaN (reported) for inf or NaN.
__device__ __forceinline__ float gs_from_amax_bits(uint32_t b, int32_t *dev_status) {
  if (b >= 0x7F800000u) {
    report(dev_status, NVFP4_ERR_NONFINITE);
    return __uint_as_float(0x7FC00000u);
  }
  const float a = __uint_as_float(b);
  return (a == 0.0f) ? 1.0f : __fdiv_rn(a, 2688.0f);
}

// Global scales from the amax (FROM_AMAX; AMAX_GIVEN reads the amax from gs
// itself) or a check of the given ones (GIVEN).  Returns the group's s_g.
__device__ __forceinline__ float finalize_one(const uint32_t *__restrict__ amax_bits, int g, int mode, float *gs,
                                              int32_t *dev_status) {
  if (mode == NVFP4_GS_GIVEN) {
    const float s = gs[g];
    if (!(s > 0.0f) || !isfinite(s)) report(dev_status, NVFP4_ERR_INVALID_ARG);
    return s;
  }
  const uint32_t b = mode == NVFP4_GS_AMAX_GIVEN ? (__float_as_uint(gs[g]) & 0x7FFFFFFFu) : amax_bits[g];
  const float s = gs_from_amax_bits(b, dev_status);
  gs[g] = s;
  return s;
}

// nvfp4_global_scale_from_amax: a = |amax[i]| (times the margin, one IEEE
// multiply, unless it is 1), then the rule above.
__global__ void gs_from_amax_kernel(const float *__restrict__ amax, int n, float margin, float *__restrict__ gs,
                                    int32_t *dev_status) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= n) return;
  float a = fabsf(amax[i]);
  if (margin != 1.0f) a = __fmul_rn(a, margin);
  gs[i] = gs_from_amax_bits(__float_as_uint(a) & 0x7FFFFFFFu, dev_status);
}

__global__ void finalize_scales_kernel(const uint32_t *__restrict__ amax_bits, int G, int mode,
                                       float *__restrict__ gs, int32_t *dev_status) {
  const int g = blockIdx.x * blockDim.x + threadIdx.x;
  if (g < G) finalize_one(amax_bits, g, mode, gs, dev_status);
}

// ---------------------------------------------------------------- pass 2: encode
// Per 16-element block: the block amax in integer SIMD, one IEEE division
// for the scale and one IEEE reciprocal, the 16 products as eight packed
// f32x2 multiplies, eight e2m1x2 conversions and one 8-byte store.

// bf16 pair (element 2i in bits 0..15) -> fp32 pair (element 2i in the low word).
__device__ __forceinline__ uint64_t bf16x2_to_f32x2(uint32_t w) {
  return ((uint64_t)(w & 0xFFFF0000u) << 32) | (uint64_t)(w << 16);
}

__device__ __forceinline__ uint64_t mul_f32x2(uint64_t x, uint64_t rr) {
  uint64_t d;
  asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(x), "l"(rr));
  return d;
}

// Four fp32 pairs -> one word of eight E2M1 codes (element 2i in the low nibble
// of byte i), round to nearest even, saturating at +-6.
__device__ __forceinline__ uint32_t e2m1x8_from_pairs(uint64_t p0, uint64_t p1, uint64_t p2, uint64_t p3) {
  uint32_t out;
  asm("{\n.reg .b8 b0, b1, b2, b3;\n.reg .f32 l0, h0, l1, h1, l2, h2, l3, h3;\n"
      "mov.b64 {l0, h0}, %1;\nmov.b64 {l1, h1}, %2;\nmov.b64 {l2, h2}, %3;\nmov.b64 {l3, h3}, %4;\n"
      "cvt.rn.satfinite.e2m1x2.f32 b0, h0, l0;\ncvt.rn.satfinite.e2m1x2.f32 b1, h1, l1;\n"
      "cvt.rn.satfinite.e2m1x2.f32 b2, h2, l2;\ncvt.rn.satfinite.e2m1x2.f32 b3, h3, l3;\n"
      "mov.b32 %0, {b0, b1, b2, b3};\n}"
      : "=r"(out) : "l"(p0), "l"(p1), "l"(p2), "l"(p3));
  return out;
}

// E4M3 byte -> fp32 through the hardware E4M3 -> f16 conversion (every E4M3
// value is an f16 normal, so both steps are exact).
__device__ __forceinline__ float e4m3_to_f32_hw(uint32_t s) {
  float f;
  asm("{\n.reg .b16 b, l, h;\n.reg .b32 w;\ncvt.u16.u32 b, %1;\ncvt.rn.f16x2.e4m3x2 w, b;\n"
      "mov.b32 {l, h}, w;\ncvt.f32.f16 %0, l;\n}" : "=f"(f) : "r"(s));
  return f;
}

__device__ __forceinline__ uint64_t sanitize_pair(uint64_t d) {
  float lo = __uint_as_float((uint32_t)d), hi = __uint_as_float((uint32_t)(d >> 32));
  lo = isnan(lo) ? 0.0f : lo;
  hi = isnan(hi) ? 0.0f : hi;
  return ((uint64_t)__float_as_uint(hi) << 32) | __float_as_uint(lo);
}

__device__ __forceinline__ uint32_t block_amax_bits(const uint4 &va, const uint4 &vb) {
  return halves_max(absmax8_bits(vb, absmax8_bits(va, 0)));
}

// The block math (the definition in include/nvfp4.h) on a block already in
// fp32 pairs with its amax a_b: S = e4m3(a_b / (6 s_g)), r = 1/(S s_g) (0 when
// that product is 0), codes = e2m1(x r).
__device__ __forceinline__ uint2 encode_f32x16(const uint64_t (&xf)[8], float a_b, float s_g, float t_g,
                                               uint32_t &S) {
  S = f32_to_e4m3_satfinite(__fdiv_rn(a_b, t_g));
  const float e = __fmul_rn(e4m3_to_f32_hw(S), s_g);
  const float r = (e == 0.0f) ? 0.0f : __frcp_rn(e);
  const uint64_t rr = ((uint64_t)__float_as_uint(r) << 32) | __float_as_uint(r);
  uint64_t prod[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) prod[i] = mul_f32x2(xf[i], rr);
  if (isinf(r)) {                     // 0 * inf: the NaN encodes as +0
#pragma unroll
    for (int i = 0; i < 8; ++i) prod[i] = sanitize_pair(prod[i]);
  }
  return make_uint2(e2m1x8_from_pairs(prod[0], prod[1], prod[2], prod[3]),
                    e2m1x8_from_pairs(prod[4], prod[5], prod[6], prod[7]));
}

// Same, from the raw bf16 block; flags a non-finite element.
__device__ __forceinline__ uint2 encode_block16(const uint4 &va, const uint4 &vb, float s_g, float t_g,
                                                uint32_t &S, bool &bad) {
  const uint32_t m = block_amax_bits(va, vb);
  if (m >= 0x7F80u) bad = true;
  const uint64_t xf[8] = {bf16x2_to_f32x2(va.x), bf16x2_to_f32x2(va.y), bf16x2_to_f32x2(va.z),
                          bf16x2_to_f32x2(va.w), bf16x2_to_f32x2(vb.x), bf16x2_to_f32x2(vb.y),
                          bf16x2_to_f32x2(vb.z), bf16x2_to_f32x2(vb.w)};
  return encode_f32x16(xf, __uint_as_float(m << 16), s_g, t_g, S);
}

// Row part and block part of the MMA-tiled scale offset (they add up to
// sf_tiled_offset(r, j, nsf)).
__device__ __forceinline__ uint64_t sf_row_part(uint32_t r, uint32_t nsf) {
  return (uint64_t)(r >> 7) * (nsf >> 2) * 512 + (r & 31) * 16 + ((r & 127) >> 5) * 4;
}
__device__ __forceinline__ uint32_t sf_blk_part(uint32_t j) { return (j >> 2) * 512 + (j & 3); }

// n / d for 32-bit n by a multiply-high, with the constants of Granlund and
// Montgomery, "Division by invariant integers using multiplication" (1994):
// l = ceil(log2 d), m = floor(2^32 (2^l - d) / d) + 1, q = (mulhi(n, m) + n) >> l.
struct FastDiv { uint32_t d, m, l; };
FastDiv make_fastdiv(uint32_t d) {
  uint32_t l = 0;
  while (l < 32 && (1ull << l) < d) ++l;
  const uint64_t m = (((1ull << 32) * ((1ull << l) - d)) / d) + 1;
  return FastDiv{d, (uint32_t)m, l};
}
__device__ __forceinline__ uint32_t fast_div(uint32_t n, const FastDiv &f) {
  return (uint32_t)(((uint64_t)__umulhi(n, f.m) + n) >> f.l);
}

// Gathered long rows (row_index, K >= 2048): one warp per result row, the
// row's group and source row looked up once, up to 8 blocks (256 bytes) in
// flight per lane; warps stride over rows so the grid streams through the
// input together.  Only real rows are written (a slot's padding rows are not).
template <bool kTiled>
__global__ void __launch_bounds__(256) quantize_rows_kernel(
    const uint16_t *__restrict__ x, int64_t ld_x, int64_t K64, int64_t rows,
    const int32_t *__restrict__ row_index, const int32_t *__restrict__ group_offsets, int G,
    const float *__restrict__ gs, uint8_t *__restrict__ q, uint8_t *__restrict__ sf, int32_t *dev_status) {
  extern __shared__ int32_t smem[];
  int32_t *off = smem, *slot = smem + (G + 1), *scratch = smem + 2 * (G + 1);
  if (group_offsets && !load_groups(group_offsets, G, off, slot, scratch, rows, true)) {
    if (threadIdx.x == 0) report(dev_status, NVFP4_ERR_INDEX);
    return;
  }
  const int lane = threadIdx.x & 31;
  const uint32_t K = (uint32_t)K64, nblk = K >> 4;
  const uint32_t warp = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const uint32_t nwarps = (gridDim.x * blockDim.x) >> 5;
  const bool v8 = ((reinterpret_cast<uintptr_t>(x) & 31u) == 0) && ((ld_x & 15) == 0);
  bool bad = false;
  constexpr int B = 8;
  for (uint32_t r = warp; r < (uint32_t)rows; r += nwarps) {
    uint32_t p = r;
    int g = 0;
    if (group_offsets) {
      g = upper_group(off, G, r);
      p = (uint32_t)slot[g] + (r - (uint32_t)off[g]);
    }
    const int64_t src = row_index ? (int64_t)row_index[r] : (int64_t)r;
    const float s_g = gs[g];
    const float t_g = __fmul_rn(6.0f, s_g);
    const uint16_t *xr = x + src * ld_x;
    uint8_t *qr = q + (uint64_t)p * (K >> 1);
    const uint64_t rsf = kTiled ? sf_row_part(p, nblk) : (uint64_t)p * nblk;
    for (uint32_t j0 = 0; j0 < nblk; j0 += 32 * B) {
      uint4 va[B], vb[B];
#pragma unroll
      for (int k = 0; k < B; ++k) {
        const uint32_t j = j0 + k * 32 + lane;
        va[k] = make_uint4(0, 0, 0, 0);
        vb[k] = make_uint4(0, 0, 0, 0);
        if (j < nblk) load_block(xr + (uint64_t)j * 16, v8, va[k], vb[k]);
      }
#pragma unroll
      for (int k = 0; k < B; ++k) {
        const uint32_t j = j0 + k * 32 + lane;
        if (j < nblk) {
          uint32_t S;
          const uint2 codes = encode_block16(va[k], vb[k], s_g, t_g, S, bad);
          *reinterpret_cast<uint2 *>(qr + (uint64_t)j * 8) = codes;
          sf[rsf + (kTiled ? sf_blk_part(j) : j)] = (uint8_t)S;
        }
      }
    }
  }
  if (bad) report(dev_status, NVFP4_ERR_NONFINITE);
}

__device__ __forceinline__ uint32_t ld_acquire_u32(const uint32_t *p) {
  uint32_t v;
  asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}

// One-launch dynamic quantize of a whole ungrouped tensor (FROM_AMAX, no row
// index), the first phase of quantize_kernel<kTiled, true>: every CTA reduces
// its grid-stride share of max|x| into words[0] (atomicMax on the fp32 bit
// pattern, as the amax pass does), counts itself in words[1], and waits until
// all gridDim.x CTAs have (the launch is cooperative, so every CTA is
// resident; the wait is bounded and reports NVFP4_ERR_TIMEOUT, after which the
// CTA writes nothing).  Then each CTA derives s_g from the amax with the
// finalisation's arithmetic; CTA 0 stores it to gs[0].  words[0..1] are zero
// at launch (the host clears them).  Returns false when the CTA must stop.
__device__ __forceinline__ bool fused_global_scale(const uint16_t *__restrict__ x, int64_t ld_x, uint32_t nblk,
                                                   uint32_t total, const FastDiv &fd, uint32_t *words,
                                                   float *gs, float &s_g, int32_t *dev_status) {
  __shared__ uint32_t red[8];
  __shared__ int s_ok;
  const bool v8 = ((reinterpret_cast<uintptr_t>(x) & 31u) == 0) && ((ld_x & 15) == 0);
  // 64-bit indices: total is below 2^32, but b + 4 * nthr need not be
  const uint64_t nthr = (uint64_t)gridDim.x * blockDim.x;
  uint64_t b = (uint64_t)blockIdx.x * blockDim.x + threadIdx.x;
  uint32_t m = 0;
  for (; b + 3 * nthr < total; b += 4 * nthr) {
    uint4 a[4], c[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const uint32_t bb = (uint32_t)(b + k * nthr), r = fast_div(bb, fd);
      load_block(x + (int64_t)r * ld_x + (uint64_t)(bb - r * nblk) * 16, v8, a[k], c[k]);
    }
#pragma unroll
    for (int k = 0; k < 4; ++k) m = absmax8_bits(c[k], absmax8_bits(a[k], m));
  }
  for (; b < total; b += nthr) {
    uint4 a, c;
    const uint32_t bb = (uint32_t)b, r = fast_div(bb, fd);
    load_block(x + (int64_t)r * ld_x + (uint64_t)(bb - r * nblk) * 16, v8, a, c);
    m = absmax8_bits(c, absmax8_bits(a, m));
  }
  m = warp_max(halves_max(m));
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = m;
  __syncthreads();
  if (threadIdx.x == 0) {
    uint32_t bm = 0;
    for (int w = 0; w < (int)(blockDim.x >> 5); ++w) bm = max(bm, red[w]);
    if (bm) atomicMax(&words[0], bm << 16);
    __threadfence();
    atomicAdd(&words[1], 1u);
    int ok = 1;
    const long long t0 = clock64();
    while (ld_acquire_u32(&words[1]) < gridDim.x) {
      if (clock64() - t0 > 4000000000LL) {                   // about 2 s
        ok = 0;
        report(dev_status, NVFP4_ERR_TIMEOUT);
        break;
      }
    }
    s_ok = ok;
  }
  __syncthreads();
  if (!s_ok) return false;
  const uint32_t amax_bits = ld_acquire_u32(&words[0]);
  s_g = gs_from_amax_bits(amax_bits, blockIdx.x == 0 ? dev_status : nullptr);
  if (blockIdx.x == 0 && threadIdx.x == 0) gs[0] = s_g;
  return true;
}

// General form: one thread per 16-element block of the real rows (routed
// order), 64-block chunks, each warp a contiguous run of chunks so every
// lane's row (and the row's group) only moves forward.  The block -> (row,
// block) split is a multiply-high division; only real rows are written.
// kFused: an ungrouped tensor whose global scale comes from its amax, in one
// cooperative launch (fused_global_scale first, then the encode).
template <bool kTiled, bool kFused = false>
__global__ void __launch_bounds__(256) quantize_kernel(
    const uint16_t *__restrict__ x, int64_t ld_x, int64_t K64, int64_t rows,
    const int32_t *__restrict__ row_index, const int32_t *__restrict__ group_offsets, int G,
    float *gs, uint8_t *__restrict__ q, uint8_t *__restrict__ sf, FastDiv fd, uint32_t *fuse_words,
    int32_t *dev_status) {
  extern __shared__ int32_t smem[];
  int32_t *off = smem, *slot = smem + (G + 1), *scratch = smem + 2 * (G + 1);
  if (!kFused && group_offsets && !load_groups(group_offsets, G, off, slot, scratch, rows, true)) {
    if (threadIdx.x == 0) report(dev_status, NVFP4_ERR_INDEX);
    return;
  }
  const int lane = threadIdx.x & 31;
  const uint32_t K = (uint32_t)K64, nblk = K >> 4;
  const uint32_t total = (uint32_t)rows * nblk;              // < 2^32 (host check)
  float fused_sg = 0.0f;
  if constexpr (kFused) {
    if (!fused_global_scale(x, ld_x, nblk, total, fd, fuse_words, gs, fused_sg, dev_status)) return;
  }
  constexpr int U = 2;                                       // 32-block steps per chunk
  const uint32_t nchunks = (total + 32 * U - 1) / (32 * U);
  const uint32_t warp = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const uint32_t nwarps = (gridDim.x * blockDim.x) >> 5;
  // Ungrouped tensors: chunks are dealt round-robin, so all warps work on one
  // narrow band of rows at a time and the scale bytes of a 32-byte sector
  // (rows r, r+1, r+32, ..., r+97 in the tiled layout) are written close
  // together in time; the sector is complete before L2 evicts it.  Contiguous
  // ranges per warp left rows r and r+32 far apart in time when rows are long,
  // and the partial sectors cost a read-modify-write in DRAM.  Grouped calls
  // keep contiguous ranges, so a warp's group index walks forward one group at
  // a time (their rows are short and their ranges a few rows long).
  uint32_t c_begin, c_end, c_step;
  if (!group_offsets) {
    c_begin = warp;
    c_end = nchunks;
    c_step = nwarps;
  } else {
    const uint32_t per = (nchunks + nwarps - 1) / nwarps;
    c_begin = min(nchunks, warp * per);
    c_end = min(nchunks, c_begin + per);
    c_step = 1;
  }
  if (c_begin >= c_end) return;
  const bool v8 = ((reinterpret_cast<uintptr_t>(x) & 31u) == 0) && ((ld_x & 15) == 0);
  int g = group_offsets ? upper_group(off, G, fast_div(c_begin * (32 * U), fd)) : 0;
  uint32_t cached_r = 0xFFFFFFFFu, p = 0;
  int64_t src = 0;
  uint64_t rsf = 0;
  float s_g = kFused ? fused_sg : gs[g], t_g = __fmul_rn(6.0f, s_g);
  bool bad = false;
  for (uint32_t ci = c_begin; ci < c_end; ci += c_step) {
    // Ungrouped tensors are walked from the end: the amax pass just streamed
    // x from front to back, so its tail is what L2 still holds.
    const uint32_t c = group_offsets ? ci : nchunks - 1 - ci;
    uint4 va[U], vb[U];
    uint32_t pp[U], jj[U];
    uint64_t rs[U];
    bool inr[U];
    float sg[U], tg[U];
#pragma unroll
    for (int k = 0; k < U; ++k) {
      const uint32_t b = c * (32 * U) + k * 32 + lane;
      inr[k] = b < total;
      uint32_t r = 0, j = 0;
      if (inr[k]) {
        r = fast_div(b, fd);
        j = b - r * nblk;
        if (r != cached_r) {
          cached_r = r;
          if (group_offsets) {
            const int g0 = g;
            while (g + 1 < G && off[g + 1] <= (int32_t)r) ++g;
            p = (uint32_t)slot[g] + (r - (uint32_t)off[g]);
            if (g != g0) { s_g = gs[g]; t_g = __fmul_rn(6.0f, s_g); }
          } else {
            p = r;
          }
          src = row_index ? (int64_t)row_index[r] : (int64_t)r;
          rsf = kTiled ? sf_row_part(p, nblk) : (uint64_t)p * nblk;
        }
      }
      pp[k] = p;
      jj[k] = j;
      rs[k] = rsf;
      sg[k] = s_g;
      tg[k] = t_g;
      va[k] = make_uint4(0, 0, 0, 0);
      vb[k] = make_uint4(0, 0, 0, 0);
      if (inr[k]) load_block(x + src * ld_x + (uint64_t)j * 16, v8, va[k], vb[k]);
    }
#pragma unroll
    for (int k = 0; k < U; ++k) {
      if (inr[k]) {
        uint32_t S;
        const uint2 codes = encode_block16(va[k], vb[k], sg[k], tg[k], S, bad);
        *reinterpret_cast<uint2 *>(q + (uint64_t)pp[k] * (K >> 1) + (uint64_t)jj[k] * 8) = codes;
        sf[rs[k] + (kTiled ? sf_blk_part(jj[k]) : jj[k])] = (uint8_t)S;
      }
    }
  }
  if (bad) report(dev_status, NVFP4_ERR_NONFINITE);
}

// ---------------------------------------------------------------- MoE dispatch quantize
// Token-major form of the gathered per-expert quantize.  A token routed to k
// experts appears in k routed rows with the same 16-element blocks; only the
// global scale differs.  So each token row is read once: the block amaxes and
// the fp32 form of the block are taken once and each of the token's k copies
// is encoded with its expert's s_g and written to its packed row.
// slot[t*k + c] is the routed row of the token's c-th choice (-1: not routed);
// a lane per choice holds its expert's packed row and global scale.

// Pass 1: the rows are cut into 2048-element pieces, one per warp, eight
// consecutive pieces per CTA (a CTA covers one or more whole tokens when a row
// holds 1, 2, 4 or 8 pieces).  Each lane keeps four 32-byte loads in flight;
// the warp's max|x| goes to shared memory, and after one barrier a thread per
// (token, choice) pair of the CTA raises the expert's amax.  A token whose
// pieces straddle two CTAs is raised by both, which atomicMax makes harmless.
// CTAs are short and not persistent, so the last wave is small.
constexpr int kAmaxWarps = 8;
constexpr int kAmaxPieceBlocks = 128;                      // 16-element blocks per piece (2048 elements)

__global__ void __launch_bounds__(kAmaxWarps * 32) moe_amax_kernel(
    const uint16_t *__restrict__ x, int64_t ld_x, int64_t K, int64_t tokens, const int32_t *__restrict__ slot,
    int topk, const int32_t *__restrict__ group_offsets, int G, uint32_t *__restrict__ amax_bits,
    int32_t *dev_status) {
  extern __shared__ int32_t smem[];
  int32_t *off = smem;
  __shared__ uint32_t piece_max[kAmaxWarps];
  for (int i = threadIdx.x; i <= G; i += blockDim.x) off[i] = group_offsets[i];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t nblk = (uint32_t)(K >> 4);
  const int64_t pieces = (nblk + kAmaxPieceBlocks - 1) / kAmaxPieceBlocks;
  const bool v8 = ((reinterpret_cast<uintptr_t>(x) & 31u) == 0) && ((ld_x & 15) == 0);
  const int64_t u0 = (int64_t)blockIdx.x * kAmaxWarps;     // first piece of the CTA
  const int64_t u = u0 + warp;
  uint32_t m = 0;
  if (u < tokens * pieces) {
    const int64_t t = u / pieces;
    const uint32_t j0 = (uint32_t)(u - t * pieces) * kAmaxPieceBlocks;
    const uint16_t *row = x + t * ld_x;
    constexpr int kLoads = kAmaxPieceBlocks / 32;           // 32-byte loads per lane
    uint4 va[kLoads], vb[kLoads];
#pragma unroll
    for (int k = 0; k < kLoads; ++k) {
      const uint32_t j = j0 + k * 32 + lane;
      va[k] = make_uint4(0, 0, 0, 0);
      vb[k] = make_uint4(0, 0, 0, 0);
      if (j < nblk) load_block(row + (uint64_t)j * 16, v8, va[k], vb[k]);
    }
#pragma unroll
    for (int k = 0; k < kLoads; ++k) m = absmax8_bits(vb[k], absmax8_bits(va[k], m));
  }
  m = warp_max(halves_max(m));
  if (lane == 0) piece_max[warp] = m;
  __syncthreads();
  // tokens touched by this CTA: t_first .. t_last
  const int64_t u_last = min(u0 + kAmaxWarps, tokens * pieces) - 1;
  if (u_last < u0) return;
  const int64_t t_first = u0 / pieces, t_last = u_last / pieces;
  const int64_t i = threadIdx.x / topk, c = threadIdx.x - i * topk;
  if (t_first + i > t_last) return;
  const int64_t t = t_first + i;
  // max over this CTA's pieces of token t
  const int64_t a = max(t * pieces, u0) - u0, b = min((t + 1) * pieces, u_last + 1) - u0;
  uint32_t mm = 0;
  for (int64_t w = a; w < b; ++w) mm = max(mm, piece_max[w]);
  const int32_t r = slot[t * topk + c];
  if (r >= off[G]) report(dev_status, NVFP4_ERR_INDEX);
  else if (r >= 0 && mm) atomicMax(&amax_bits[upper_group(off, G, r)], mm << 16);
}

// Per-group constants of the dispatch encode, computed once per call with the
// same IEEE operations the per-block path would use: rtab[g][S] = 1/(S*s_g)
// (0 when that product is 0) for every E4M3 byte S < 128, and
// ytab[g] = RN(1/(6*s_g)).  One block per group; thread 0 first settles the
// group's s_g (finalize_one), which the block then reads from shared memory.
__global__ void finalize_tables_kernel(const uint32_t *__restrict__ amax_bits, int mode, float *gs,
                                       float *__restrict__ rtab, float *__restrict__ ytab, int32_t *dev_status) {
  __shared__ float s_sg;
  const int g = blockIdx.x;
  const uint32_t S = threadIdx.x;
  if (S == 0) s_sg = finalize_one(amax_bits, g, mode, gs, dev_status);
  __syncthreads();
  const float s_g = s_sg;
  const float e = __fmul_rn(e4m3_to_f32_hw(S), s_g);
  rtab[g * 128 + S] = (e == 0.0f) ? 0.0f : __frcp_rn(e);
  if (S == 0) ytab[g] = __frcp_rn(__fmul_rn(6.0f, s_g));
}

// S = e4m3_rne_satfinite(RN(a_b / t_g)) without the division in the common
// case.  q = RN(a_b * y) with y = RN(1/t_g) is within 3 * 2^-24 (relative) of
// the exact quotient, and so is RN(a_b / t_g); the bracket [q(1-2^-21),
// q(1+2^-21)], each end rounded, holds RN(a_b / t_g) (below the fp32 normal
// range both ends and the quotient encode to 0).  E4M3 rounding is monotone, so
// when both ends give the same byte that byte is the IEEE path's S; otherwise
// (a quotient within 2^-21 of an E4M3 rounding boundary, or y = inf) the
// division is done.
__device__ __forceinline__ uint32_t block_scale_fast(float a_b, float t_g, float y, bool exact) {
  const float q = __fmul_rn(a_b, y);
  const uint32_t lo = f32_to_e4m3_satfinite(__fmul_rn(q, 0.99999952316284180f));   // 1 - 2^-21
  const uint32_t hi = f32_to_e4m3_satfinite(__fmul_rn(q, 1.00000047683715820f));   // 1 + 2^-21
  if (lo == hi && !exact) return lo;
  return f32_to_e4m3_satfinite(__fdiv_rn(a_b, t_g));
}

// Both ends of the bracket of block_scale_fast in one packed multiply and one
// two-way E4M3 conversion: returns the byte of q(1-2^-21) and sets `same` when
// q(1+2^-21) rounds to the same byte.  Each end is rounded exactly as
// f32_to_e4m3_satfinite rounds it alone.
__device__ __forceinline__ uint32_t bracket_e4m3(float q, bool &same) {
  const uint64_t qq = ((uint64_t)__float_as_uint(q) << 32) | __float_as_uint(q);
  const uint64_t ends = mul_f32x2(qq, 0x3F8000043F7FFFF8ull);    // (1 - 2^-21, 1 + 2^-21)
  uint16_t d;
  asm("{\n.reg .f32 l, h;\nmov.b64 {l, h}, %1;\ncvt.rn.satfinite.e4m3x2.f32 %0, h, l;\n}" : "=h"(d) : "l"(ends));
  const uint32_t lo = d & 0xFFu;
  same = lo == (uint32_t)(d >> 8);
  return lo;
}

// Codes of a block in fp32 pairs for a given r (a NaN product 0 * inf encodes as +0).
__device__ __forceinline__ uint2 encode_codes(const uint64_t (&xf)[8], float r) {
  const uint64_t rr = ((uint64_t)__float_as_uint(r) << 32) | __float_as_uint(r);
  uint64_t prod[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) prod[i] = mul_f32x2(xf[i], rr);
  if (isinf(r)) {
#pragma unroll
    for (int i = 0; i < 8; ++i) prod[i] = sanitize_pair(prod[i]);
  }
  return make_uint2(e2m1x8_from_pairs(prod[0], prod[1], prod[2], prod[3]),
                    e2m1x8_from_pairs(prod[4], prod[5], prod[6], prod[7]));
}

// Pass 2: a warp takes 64 consecutive 16-element blocks of one token row (two
// per lane, so the token's routing is warp-uniform), holds them as fp32 pairs
// and encodes them once per routed copy, with the scale byte from
// block_scale_fast and r from the group's table.  The block loads are issued
// before the routing lookups so the two latencies overlap.  Lane c resolves
// choice c (packed row, expert, s_g, 1/(6 s_g)) into the warp's 16-byte slot
// c in shared memory, which the copy loop reads back as one broadcast load
// per copy.
template <bool kTiled>
__global__ void __launch_bounds__(256, 3) moe_encode_blocks_kernel(
    const uint16_t *__restrict__ x, int64_t ld_x, int64_t K64, int64_t tokens, const int32_t *__restrict__ slot,
    int topk, const int32_t *__restrict__ group_offsets, int G, const float *__restrict__ gs,
    const float *__restrict__ rtab, const float *__restrict__ ytab, uint8_t *__restrict__ q,
    uint8_t *__restrict__ sf, int32_t *dev_status) {
  extern __shared__ int32_t smem[];
  int32_t *off = smem, *pslot = smem + (G + 1), *scratch = smem + 2 * (G + 1);
  if (!load_groups(group_offsets, G, off, pslot, scratch, tokens * topk, false)) {
    if (threadIdx.x == 0) report(dev_status, NVFP4_ERR_INDEX);
    return;
  }
  const int lane = threadIdx.x & 31;
  const uint32_t K = (uint32_t)K64, nblk = K >> 4;
  const uint32_t cpr = (nblk + 63) >> 6;                     // 64-block chunks per row
  const uint64_t nwork = (uint64_t)tokens * cpr;
  const uint64_t nwarps = ((uint64_t)gridDim.x * blockDim.x) >> 5;
  const bool v8 = ((reinterpret_cast<uintptr_t>(x) & 31u) == 0) && ((ld_x & 15) == 0);
  __shared__ int4 s_choice[8][32];                           // [warp][choice]: row, expert, s_g, y
  int4 *my_choices = s_choice[threadIdx.x >> 5];
  bool bad = false;
  for (uint64_t w = ((uint64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5; w < nwork; w += nwarps) {
    const uint64_t t = w / cpr;
    const uint32_t j0 = (uint32_t)(w - t * cpr) * 64 + lane, j1 = j0 + 32;
    const uint16_t *xr = x + t * ld_x;
    uint4 a0 = make_uint4(0, 0, 0, 0), b0 = a0, a1 = a0, b1 = a0;
    if (j0 < nblk) load_block(xr + (uint64_t)j0 * 16, v8, a0, b0);
    if (j1 < nblk) load_block(xr + (uint64_t)j1 * 16, v8, a1, b1);
    int32_t my_p = -1, my_e = 0;
    float my_sg = 1.0f, my_y = 0.0f;
    if (lane < topk) {
      const int32_t r = slot[t * topk + lane];
      if (r >= 0 && r < off[G]) {
        const int e = upper_group(off, G, r);
        my_p = pslot[e] + (r - off[e]);
        my_e = e;
        my_sg = gs[e];
        my_y = ytab[e];
      }
    }
    __syncwarp();                                            // the previous row's copies have read the slots
    if (lane < topk) my_choices[lane] = make_int4(my_p, my_e, __float_as_int(my_sg), __float_as_int(my_y));
    __syncwarp();
    const uint32_t m0 = block_amax_bits(a0, b0), m1 = block_amax_bits(a1, b1);
    if (max(m0, m1) >= 0x7F80u) bad = true;
    const float am0 = __uint_as_float(m0 << 16), am1 = __uint_as_float(m1 << 16);
    const uint64_t x0[8] = {bf16x2_to_f32x2(a0.x), bf16x2_to_f32x2(a0.y), bf16x2_to_f32x2(a0.z),
                            bf16x2_to_f32x2(a0.w), bf16x2_to_f32x2(b0.x), bf16x2_to_f32x2(b0.y),
                            bf16x2_to_f32x2(b0.z), bf16x2_to_f32x2(b0.w)};
    const uint64_t x1[8] = {bf16x2_to_f32x2(a1.x), bf16x2_to_f32x2(a1.y), bf16x2_to_f32x2(a1.z),
                            bf16x2_to_f32x2(a1.w), bf16x2_to_f32x2(b1.x), bf16x2_to_f32x2(b1.y),
                            bf16x2_to_f32x2(b1.z), bf16x2_to_f32x2(b1.w)};
    const uint32_t jb0 = kTiled ? sf_blk_part(j0) : j0, jb1 = kTiled ? sf_blk_part(j1) : j1;
    for (int c = 0; c < topk; ++c) {
      const int4 ch = my_choices[c];
      const int32_t p = ch.x;
      if (p < 0) continue;
      const int32_t e = ch.y;
      const float s_g = __int_as_float(ch.z);
      const float y = __int_as_float(ch.w);
      const float t_g = __fmul_rn(6.0f, s_g);
      const bool exact = !(y <= 3.402823466e38f);             // y = inf (or NaN): always divide
      const float *rt = rtab + (int64_t)e * 128;
      uint8_t *qr = q + (uint64_t)p * (K >> 1);
      const uint64_t rsf = kTiled ? sf_row_part((uint32_t)p, nblk) : (uint64_t)p * nblk;
      if (j1 < nblk) {
        // both blocks (every chunk of a row whose K is a multiple of 1024):
        // straight-line code, so the two blocks' chains interleave
        const uint64_t qv = mul_f32x2(((uint64_t)__float_as_uint(am1) << 32) | __float_as_uint(am0),
                                      ((uint64_t)__float_as_uint(y) << 32) | __float_as_uint(y));
        bool same0, same1;
        uint32_t S0 = bracket_e4m3(__uint_as_float((uint32_t)qv), same0);
        uint32_t S1 = bracket_e4m3(__uint_as_float((uint32_t)(qv >> 32)), same1);
        if (!same0 || exact) S0 = f32_to_e4m3_satfinite(__fdiv_rn(am0, t_g));
        if (!same1 || exact) S1 = f32_to_e4m3_satfinite(__fdiv_rn(am1, t_g));
        const float r0 = __ldg(rt + S0), r1 = __ldg(rt + S1);
        const uint2 c0 = encode_codes(x0, r0), c1 = encode_codes(x1, r1);
        *reinterpret_cast<uint2 *>(qr + (uint64_t)j0 * 8) = c0;
        *reinterpret_cast<uint2 *>(qr + (uint64_t)j1 * 8) = c1;
        sf[rsf + jb0] = (uint8_t)S0;
        sf[rsf + jb1] = (uint8_t)S1;
      } else if (j0 < nblk) {
        const uint32_t S = block_scale_fast(am0, t_g, y, exact);
        *reinterpret_cast<uint2 *>(qr + (uint64_t)j0 * 8) = encode_codes(x0, __ldg(rt + S));
        sf[rsf + jb0] = (uint8_t)S;
      }
    }
  }
  if (bad) report(dev_status, NVFP4_ERR_NONFINITE);
}

// ---------------------------------------------------------------- element-wise codecs
// The two conversions of the encode path on their own, for any fp32 input:
// E2M1 through e2m1x8_from_pairs (the code step of every quantize kernel; a
// NaN input encodes as +0, as the product 0 * inf does there), E4M3 through
// f32_to_e4m3_satfinite (the block-scale step; NaN gives 0x7F).
__global__ void e2m1_encode_kernel(const float4 *__restrict__ x, int64_t n8, uint32_t *__restrict__ q) {
  const int64_t stride = (int64_t)gridDim.x * blockDim.x;
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n8; i += stride) {
    const float4 a = x[2 * i], b = x[2 * i + 1];
    auto pair = [](float lo, float hi) {
      return sanitize_pair(((uint64_t)__float_as_uint(hi) << 32) | __float_as_uint(lo));
    };
    q[i] = e2m1x8_from_pairs(pair(a.x, a.y), pair(a.z, a.w), pair(b.x, b.y), pair(b.z, b.w));
  }
}

__global__ void e4m3_encode_kernel(const float4 *__restrict__ x, int64_t n4, uint32_t *__restrict__ out) {
  const int64_t stride = (int64_t)gridDim.x * blockDim.x;
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n4; i += stride) {
    const float4 v = x[i];
    auto enc = [](float f) { return isnan(f) ? 0x7Fu : f32_to_e4m3_satfinite(f); };
    out[i] = enc(v.x) | (enc(v.y) << 8) | (enc(v.z) << 16) | (enc(v.w) << 24);
  }
}

// ---------------------------------------------------------------- dequantize
// (code * S) in f16 is exact (at most 6 significant bits, |.| <= 2688), so the
// hardware E2M1 -> f16 conversion times the f16 scale gives the exact product;
// one fp32 multiply by s_g then rounds once, as the definition asks.
__device__ __forceinline__ uint64_t dq_pair(uint32_t byte, uint32_t S2h, uint64_t gg) {
  uint32_t h;
  asm("{\n.reg .b8 b;\ncvt.u8.u32 b, %1;\ncvt.rn.f16x2.e2m1x2 %0, b;\n}" : "=r"(h) : "r"(byte));
  asm("mul.rn.f16x2 %0, %0, %1;" : "+r"(h) : "r"(S2h));
  float lo, hi;
  asm("{\n.reg .f16 l, u;\nmov.b32 {l, u}, %2;\ncvt.f32.f16 %0, l;\ncvt.f32.f16 %1, u;\n}" : "=f"(lo), "=f"(hi) : "r"(h));
  const uint64_t x = ((uint64_t)__float_as_uint(hi) << 32) | __float_as_uint(lo);
  uint64_t d;
  asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(x), "l"(gg));
  return d;
}

template <bool kTiled, bool kBf16>
__global__ void __launch_bounds__(256) dequantize_kernel(
    const uint8_t *__restrict__ q, const uint8_t *__restrict__ sf, const float *__restrict__ gs,
    const int32_t *__restrict__ group_offsets, int G, int64_t rows, int64_t K, void *__restrict__ y) {
  extern __shared__ int32_t smem[];
  int32_t *off = smem, *slot = smem + (G + 1), *scratch = smem + 2 * (G + 1);
  if (group_offsets && !load_groups(group_offsets, G, off, slot, scratch, rows, true)) return;   // nothing written
  // one thread per 8 elements (a thread pair per 16-element block), so a warp
  // writes 512 (bf16) or 1024 (fp32) contiguous bytes per step
  const uint64_t nhalf = (uint64_t)(K >> 3);
  const uint64_t total = (uint64_t)rows * nhalf;
  const uint64_t stride = (uint64_t)gridDim.x * blockDim.x;
  const uint64_t nblk = (uint64_t)(K >> 4);
  const bool small = total < 0xFFFFFFF0ull;
  for (uint64_t h = (uint64_t)blockIdx.x * blockDim.x + threadIdx.x; h < total; h += stride) {
    uint64_t r, c;
    if (small) { const uint32_t r32 = (uint32_t)h / (uint32_t)nhalf; r = r32; c = (uint32_t)h - r32 * (uint32_t)nhalf; }
    else { r = h / nhalf; c = h - r * nhalf; }
    const uint64_t j = c >> 1;
    int g = 0;
    uint64_t p = r;
    if (group_offsets) {
      g = upper_group(off, G, (int64_t)r);
      p = (uint64_t)slot[g] + (r - (uint64_t)off[g]);
    }
    const float s_g = gs[g];
    const uint32_t sb = kTiled ? sf[sf_tiled_offset(p, j, nblk)] : sf[p * nblk + j];
    uint32_t S2h;
    {
      const uint16_t pair = (uint16_t)(sb | (sb << 8));
      asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(S2h) : "h"(pair));
    }
    const uint64_t gg = ((uint64_t)__float_as_uint(s_g) << 32) | __float_as_uint(s_g);
    const uint32_t cw = *reinterpret_cast<const uint32_t *>(q + p * (K >> 1) + c * 4);
    uint64_t d[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) d[i] = dq_pair((cw >> (8 * i)) & 0xFFu, S2h, gg);
    if (kBf16) {
      uint32_t hw[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        __nv_bfloat162 t = __floats2bfloat162_rn(__uint_as_float((uint32_t)d[i]), __uint_as_float((uint32_t)(d[i] >> 32)));
        hw[i] = *reinterpret_cast<uint32_t *>(&t);
      }
      *reinterpret_cast<uint4 *>(reinterpret_cast<uint16_t *>(y) + r * K + c * 8) = make_uint4(hw[0], hw[1], hw[2], hw[3]);
    } else {
      uint4 *dst = reinterpret_cast<uint4 *>(reinterpret_cast<float *>(y) + r * K + c * 8);
      dst[0] = make_uint4((uint32_t)d[0], (uint32_t)(d[0] >> 32), (uint32_t)d[1], (uint32_t)(d[1] >> 32));
      dst[1] = make_uint4((uint32_t)d[2], (uint32_t)(d[2] >> 32), (uint32_t)d[3], (uint32_t)(d[3] >> 32));
    }
  }
}

// Ungrouped tensors (the KV cache, dense activations): a flat walk over the
// 16-element blocks.  Lane l of a warp takes blocks c0 + l + 32 i, i < kU, so
// each warp store instruction writes 1 KB (bf16) or 2 KB (fp32) of contiguous
// output, and all kU blocks' code words and scale bytes are loaded before the
// first is decoded: 8 blocks x 9 bytes stay in flight per lane.  (One thread
// per 8 elements with one 4-byte load at a time kept too few reads in flight
// to cover HBM latency: 0.69 of the copy rate on the KV cache.)
template <bool kTiled, bool kBf16>
__global__ void __launch_bounds__(256) dequantize_flat_kernel(
    const uint8_t *__restrict__ q, const uint8_t *__restrict__ sf, const float *__restrict__ gs, int64_t rows,
    int64_t K, void *__restrict__ y) {
  constexpr int kU = 8;
  const int lane = threadIdx.x & 31;
  const uint64_t nblk = (uint64_t)(K >> 4);
  const uint64_t nb = (uint64_t)rows * nblk;
  const uint64_t nwarps = ((uint64_t)gridDim.x * blockDim.x) >> 5;
  const float s_g = gs[0];
  const uint64_t gg = ((uint64_t)__float_as_uint(s_g) << 32) | __float_as_uint(s_g);
  for (uint64_t c0 = (((uint64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5) * (32 * kU); c0 < nb;
       c0 += nwarps * (32 * kU)) {
    uint2 cw[kU];
    uint32_t sb[kU];
#pragma unroll
    for (int i = 0; i < kU; ++i) {
      const uint64_t b = c0 + (uint64_t)(32 * i + lane);
      cw[i] = make_uint2(0, 0);
      sb[i] = 0;
      if (b < nb) {
        cw[i] = __ldg(reinterpret_cast<const uint2 *>(q) + b);
        if (kTiled) {
          const uint64_t r = b / nblk;
          sb[i] = __ldg(sf + sf_tiled_offset((int64_t)r, (int64_t)(b - r * nblk), (int64_t)nblk));
        } else {
          sb[i] = __ldg(sf + b);
        }
      }
    }
#pragma unroll
    for (int i = 0; i < kU; ++i) {
      const uint64_t b = c0 + (uint64_t)(32 * i + lane);
      if (b >= nb) continue;
      uint32_t S2h;
      {
        const uint16_t pair = (uint16_t)(sb[i] | (sb[i] << 8));
        asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(S2h) : "h"(pair));
      }
      uint64_t d[8];
#pragma unroll
      for (int k = 0; k < 4; ++k) d[k] = dq_pair((cw[i].x >> (8 * k)) & 0xFFu, S2h, gg);
#pragma unroll
      for (int k = 0; k < 4; ++k) d[4 + k] = dq_pair((cw[i].y >> (8 * k)) & 0xFFu, S2h, gg);
      if (kBf16) {
        uint32_t hw[8];
#pragma unroll
        for (int k = 0; k < 8; ++k) {
          __nv_bfloat162 t =
              __floats2bfloat162_rn(__uint_as_float((uint32_t)d[k]), __uint_as_float((uint32_t)(d[k] >> 32)));
          hw[k] = *reinterpret_cast<uint32_t *>(&t);
        }
        uint16_t *dst = reinterpret_cast<uint16_t *>(y) + b * 16;
        asm volatile("st.global.v8.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8};" ::"l"(dst), "r"(hw[0]), "r"(hw[1]),
                     "r"(hw[2]), "r"(hw[3]), "r"(hw[4]), "r"(hw[5]), "r"(hw[6]), "r"(hw[7])
                     : "memory");
      } else {
        float *dst = reinterpret_cast<float *>(y) + b * 16;
#pragma unroll
        for (int k = 0; k < 2; ++k)
          asm volatile("st.global.v8.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8};" ::"l"(dst + 8 * k),
                       "r"((uint32_t)d[4 * k]), "r"((uint32_t)(d[4 * k] >> 32)), "r"((uint32_t)d[4 * k + 1]),
                       "r"((uint32_t)(d[4 * k + 1] >> 32)), "r"((uint32_t)d[4 * k + 2]),
                       "r"((uint32_t)(d[4 * k + 2] >> 32)), "r"((uint32_t)d[4 * k + 3]),
                       "r"((uint32_t)(d[4 * k + 3] >> 32))
                       : "memory");
      }
    }
  }
}

// ---------------------------------------------------------------- SwiGLU + amax
// h[r, j] = bf16(silu(g) * u), g = y[r, j], u = y[r, I + j]; per-group amax of h.
template <bool kBf16In>
__global__ void __launch_bounds__(256) swiglu_amax_kernel(
    const void *__restrict__ y, int64_t rows, int64_t I, const int32_t *__restrict__ group_offsets,
    int G, uint16_t *__restrict__ h, uint32_t *__restrict__ amax_bits) {
  extern __shared__ int32_t smem[];
  int32_t *off = smem;
  if (group_offsets) {
    for (int i = threadIdx.x; i <= G; i += blockDim.x) off[i] = group_offsets[i];
    __syncthreads();
  }
  const int lane = threadIdx.x & 31;
  const int64_t warp = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int64_t nwarps = ((int64_t)gridDim.x * blockDim.x) >> 5;
  const int64_t per = (rows + nwarps - 1) / nwarps;
  const int64_t r0 = warp * per, r1 = min(rows, r0 + per);
  if (r0 >= r1) return;
  const int64_t nvec = I >> 3;
  int g = group_offsets ? upper_group(off, G, r0) : 0;
  uint32_t m = 0;
  for (int64_t r = r0; r < r1; ++r) {
    if (group_offsets) {
      int gn = g;
      while (gn + 1 < G && off[gn + 1] <= r) ++gn;
      if (gn != g) {
        uint32_t mm = warp_max(halves_max(m));
        if (lane == 0 && mm) atomicMax(&amax_bits[g], mm << 16);
        m = 0;
        g = gn;
      }
    }
    for (int64_t c = lane; c < nvec; c += 32) {
      float gv[8], uv[8];
      if (kBf16In) {
        const uint16_t *yr = reinterpret_cast<const uint16_t *>(y) + r * 2 * I;
        uint4 a = ldg_nc_v4(yr + 8 * c), b = ldg_nc_v4(yr + I + 8 * c);
        const uint32_t wa[4] = {a.x, a.y, a.z, a.w}, wb[4] = {b.x, b.y, b.z, b.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          gv[2 * i] = bf16_bits_to_f32(wa[i] & 0xFFFFu); gv[2 * i + 1] = bf16_bits_to_f32(wa[i] >> 16);
          uv[2 * i] = bf16_bits_to_f32(wb[i] & 0xFFFFu); uv[2 * i + 1] = bf16_bits_to_f32(wb[i] >> 16);
        }
      } else {
        const float *yr = reinterpret_cast<const float *>(y) + r * 2 * I;
        const float4 *ga = reinterpret_cast<const float4 *>(yr + 8 * c);
        const float4 *ua = reinterpret_cast<const float4 *>(yr + I + 8 * c);
        float4 g0 = __ldg(ga), g1 = __ldg(ga + 1), u0 = __ldg(ua), u1 = __ldg(ua + 1);
        gv[0] = g0.x; gv[1] = g0.y; gv[2] = g0.z; gv[3] = g0.w;
        gv[4] = g1.x; gv[5] = g1.y; gv[6] = g1.z; gv[7] = g1.w;
        uv[0] = u0.x; uv[1] = u0.y; uv[2] = u0.z; uv[3] = u0.w;
        uv[4] = u1.x; uv[5] = u1.y; uv[6] = u1.z; uv[7] = u1.w;
      }
      uint32_t hw[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        float s0 = __fdiv_rn(gv[2 * i], __fadd_rn(1.0f, expf(-gv[2 * i])));
        float s1 = __fdiv_rn(gv[2 * i + 1], __fadd_rn(1.0f, expf(-gv[2 * i + 1])));
        __nv_bfloat162 t = __floats2bfloat162_rn(__fmul_rn(s0, uv[2 * i]), __fmul_rn(s1, uv[2 * i + 1]));
        hw[i] = *reinterpret_cast<uint32_t *>(&t);
        m = __vmaxu2(m, hw[i] & 0x7FFF7FFFu);
      }
      *reinterpret_cast<uint4 *>(h + r * I + 8 * c) = make_uint4(hw[0], hw[1], hw[2], hw[3]);
    }
  }
  uint32_t mm = warp_max(halves_max(m));
  if (lane == 0 && mm) atomicMax(&amax_bits[g], mm << 16);
}

}  // namespace nvfp4

// ====================================================================== host side
using namespace nvfp4;

namespace {

// Workspace: amax / exponent-range words (2 per group) and room for kernel
// bookkeeping, then the per-group encode tables of the dispatch quantize
// (128 reciprocals + 1 per group).
size_t workspace_words_bytes(int num_groups) {
  return (sizeof(uint32_t) * 2 * (size_t)num_groups + 256 + 255) / 256 * 256;
}
float *workspace_tables(void *workspace, int num_groups) {
  return reinterpret_cast<float *>(reinterpret_cast<uint8_t *>(workspace) + workspace_words_bytes(num_groups));
}

int num_sms() { return host::sm_count(); }

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

int64_t grid_for(int64_t work_items, int threads, int per_sm) {
  int64_t need = (work_items + threads - 1) / threads;
  int64_t cap = (int64_t)num_sms() * per_sm;
  if (need < 1) need = 1;
  return need < cap ? need : cap;
}

// Grid for a grid-stride kernel: at most one wave of resident blocks, so no
// block starts late with a full share of the work.
template <typename Kernel>
int64_t grid_resident(Kernel kernel, int64_t work_items, int threads, size_t smem) {
  return grid_for(work_items, threads, host::blocks_per_sm(reinterpret_cast<const void *>(kernel), threads, smem));
}

nvfp4_status launch_status() {
  return cudaGetLastError() == cudaSuccess ? NVFP4_OK : NVFP4_ERR_CUDA;
}

// amax pass + global-scale finalisation, shared by quantize and KV paths.
nvfp4_status run_global_scales(const uint16_t *x, int64_t rows, int64_t K, int64_t ld_x,
                               const int32_t *row_index, const int32_t *group_offsets, int G,
                               nvfp4_gs_mode gs_mode, float *global_scale, void *workspace,
                               int32_t *dev_status, cudaStream_t stream) {
  uint32_t *amax_bits = reinterpret_cast<uint32_t *>(workspace);
  if (gs_mode == NVFP4_GS_FROM_AMAX) {
    if (cudaMemsetAsync(amax_bits, 0, sizeof(uint32_t) * G, stream) != cudaSuccess) return NVFP4_ERR_CUDA;
    if (rows > 0) {
      if (!group_offsets && !row_index && ld_x == K) {
        const int64_t nblk = rows * K / 16;
        if ((reinterpret_cast<uintptr_t>(x) & 31u) == 0) {
          const unsigned grid = (unsigned)grid_resident(amax_flat_kernel<true>, (nblk + 3) / 4, 256, 0);
          amax_flat_kernel<true><<<grid, 256, 0, stream>>>(x, nblk, amax_bits);
        } else {
          const unsigned grid = (unsigned)grid_resident(amax_flat_kernel<false>, (nblk + 3) / 4, 256, 0);
          amax_flat_kernel<false><<<grid, 256, 0, stream>>>(x, nblk, amax_bits);
        }
      } else {
        size_t sm = group_offsets ? sizeof(int32_t) * (G + 1) : 0;
        int64_t warps_needed = rows;
        amax_rows_kernel<<<(unsigned)grid_for(warps_needed * 32, 256, 8), 256, sm, stream>>>(
            x, ld_x, K, rows, row_index, group_offsets, G, amax_bits);
      }
      if (cudaGetLastError() != cudaSuccess) return NVFP4_ERR_CUDA;
    }
  }
  finalize_scales_kernel<<<(G + 127) / 128, 128, 0, stream>>>(amax_bits, G, (int)gs_mode, global_scale, dev_status);
  return launch_status();
}

nvfp4_status run_encode(const uint16_t *x, int64_t rows, int64_t K, int64_t ld_x,
                        const int32_t *row_index, const int32_t *group_offsets, int G,
                        const float *gs, uint8_t *q, uint8_t *sf, nvfp4_sf_layout layout,
                        int32_t *dev_status, cudaStream_t stream) {
  const bool tiled = layout == NVFP4_SF_MMA_TILED;
  if (rows == 0) return NVFP4_OK;
  const size_t sm = group_offsets ? sizeof(int32_t) * (2 * (G + 1) + 8) : 0;
  if (row_index && K >= 2048) {
    // one warp per result row
    if (tiled) {
      const unsigned grid = (unsigned)grid_resident(quantize_rows_kernel<true>, rows * 32, 256, sm);
      quantize_rows_kernel<true><<<grid, 256, sm, stream>>>(x, ld_x, K, rows, row_index, group_offsets, G, gs, q, sf, dev_status);
    } else {
      const unsigned grid = (unsigned)grid_resident(quantize_rows_kernel<false>, rows * 32, 256, sm);
      quantize_rows_kernel<false><<<grid, 256, sm, stream>>>(x, ld_x, K, rows, row_index, group_offsets, G, gs, q, sf, dev_status);
    }
    return launch_status();
  }
  const int64_t nblk = K / 16;
  const FastDiv fd = make_fastdiv((uint32_t)nblk);
  // the block index is 32-bit: one launch covers fewer than 2^32 - 64 blocks;
  // a larger ungrouped tensor goes in pieces of whole 128-row tiles
  const int64_t max_rows = ((int64_t)0xFFFFFFC0ll / nblk) / 128 * 128;
  if (rows > max_rows && (group_offsets || row_index)) return NVFP4_ERR_UNSUPPORTED_SHAPE;
  for (int64_t r0 = 0; r0 < rows; r0 += max_rows) {
    const int64_t n = rows - r0 < max_rows ? rows - r0 : max_rows;
    const uint16_t *xp = x + r0 * ld_x;
    uint8_t *qp = q + r0 * (K / 2);
    uint8_t *sp = sf + (tiled ? (r0 / 128) * (nblk / 4) * 512 : r0 * nblk);
    const int64_t work = (n * nblk + 1) / 2;
    if (tiled) {
      const unsigned grid = (unsigned)grid_resident(quantize_kernel<true>, work, 256, sm);
      quantize_kernel<true><<<grid, 256, sm, stream>>>(xp, ld_x, K, n, row_index, group_offsets, G, const_cast<float *>(gs), qp, sp, fd, nullptr, dev_status);
    } else {
      const unsigned grid = (unsigned)grid_resident(quantize_kernel<false>, work, 256, sm);
      quantize_kernel<false><<<grid, 256, sm, stream>>>(xp, ld_x, K, n, row_index, group_offsets, G, const_cast<float *>(gs), qp, sp, fd, nullptr, dev_status);
    }
    if (cudaGetLastError() != cudaSuccess) return NVFP4_ERR_CUDA;
  }
  return NVFP4_OK;
}

// The dynamic quantize of an ungrouped tensor in one cooperative launch
// (quantize_kernel<tiled, true>): the amax pass, the global scale and the
// encode without the two extra launches and their gaps.  The grid is at most
// one resident wave, so every CTA can wait for the others.  *launched is false
// (and nothing was enqueued but the clearing of the two workspace words) when
// the runtime refuses the cooperative launch; the caller then runs the
// separate passes.
nvfp4_status run_fused_dense(const uint16_t *x, int64_t rows, int64_t K, int64_t ld_x, float *global_scale,
                             uint8_t *q, uint8_t *sf, nvfp4_sf_layout layout, void *workspace,
                             int32_t *dev_status, cudaStream_t stream, bool *launched) {
  *launched = false;
  const bool tiled = layout == NVFP4_SF_MMA_TILED;
  const int64_t nblk = K / 16, total = rows * nblk;
  uint32_t *words = reinterpret_cast<uint32_t *>(workspace);
  if (cudaMemsetAsync(words, 0, 2 * sizeof(uint32_t), stream) != cudaSuccess) return NVFP4_ERR_CUDA;
  auto kern = tiled ? quantize_kernel<true, true> : quantize_kernel<false, true>;
  const int per_sm = host::blocks_per_sm(reinterpret_cast<const void *>(kern), 256, 0);
  const int64_t nchunks = (total + 63) / 64;
  int64_t grid = (int64_t)per_sm * num_sms();
  if ((nchunks + 7) / 8 < grid) grid = (nchunks + 7) / 8;    // at least one 64-block chunk per warp
  if (grid < 1) grid = 1;
  const FastDiv fd = make_fastdiv((uint32_t)nblk);
  const uint16_t *a_x = x;
  int64_t a_ld = ld_x, a_k = K, a_rows = rows;
  const int32_t *a_ri = nullptr, *a_go = nullptr;
  int a_g = 1;
  float *a_gs = global_scale;
  uint8_t *a_q = q, *a_sf = sf;
  FastDiv a_fd = fd;
  uint32_t *a_w = words;
  int32_t *a_st = dev_status;
  void *args[] = {&a_x, &a_ld, &a_k, &a_rows, &a_ri, &a_go, &a_g, &a_gs, &a_q, &a_sf, &a_fd, &a_w, &a_st};
  const cudaError_t e = cudaLaunchCooperativeKernel(reinterpret_cast<const void *>(kern), dim3((unsigned)grid),
                                                    dim3(256), args, 0, stream);
  if (e != cudaSuccess) {
    (void)cudaGetLastError();
    return NVFP4_OK;
  }
  *launched = true;
  return NVFP4_OK;
}

}  // namespace

extern "C" {

const char *nvfp4_status_string(int status) {
  switch (status) {
    case NVFP4_OK: return "ok";
    case NVFP4_ERR_INVALID_ARG: return "invalid argument";
    case NVFP4_ERR_UNSUPPORTED_SHAPE: return "unsupported shape";
    case NVFP4_ERR_CUDA: return "CUDA error";
    case NVFP4_ERR_NONFINITE: return "non-finite input";
    case NVFP4_ERR_NOT_REPRESENTABLE: return "not representable";
    case NVFP4_ERR_TIMEOUT: return "bounded wait timed out";
    case NVFP4_ERR_INDEX: return "index out of range";
    default: return "unknown status";
  }
}

size_t nvfp4_workspace_size(int num_groups) {
  if (num_groups < 1) num_groups = 1;
  size_t bytes = workspace_words_bytes(num_groups) + sizeof(float) * 129 * (size_t)num_groups;
  return (bytes + 255) / 256 * 256;
}

int64_t nvfp4_padded_rows_bound(int64_t rows, int num_groups) {
  if (num_groups < 1) num_groups = 1;
  int64_t b = rows + 127 * (int64_t)num_groups;
  return (b + 127) / 128 * 128;
}

nvfp4_status nvfp4_quantize(const void *x, int64_t rows, int64_t K, int64_t ld_x,
                            const int32_t *row_index, const int32_t *group_offsets, int num_groups,
                            nvfp4_gs_mode gs_mode, float *global_scale, uint8_t *q, uint8_t *sf,
                            nvfp4_sf_layout sf_layout, void *workspace, int32_t *dev_status,
                            cudaStream_t stream) {
  if (rows < 0 || K <= 0 || ld_x < K) return NVFP4_ERR_INVALID_ARG;
  if (K % 16 != 0 || ld_x % 8 != 0) return NVFP4_ERR_UNSUPPORTED_SHAPE;
  if (sf_layout != NVFP4_SF_ROWMAJOR && sf_layout != NVFP4_SF_MMA_TILED) return NVFP4_ERR_INVALID_ARG;
  if (sf_layout == NVFP4_SF_MMA_TILED && K % 64 != 0) return NVFP4_ERR_UNSUPPORTED_SHAPE;
  if (gs_mode != NVFP4_GS_FROM_AMAX && gs_mode != NVFP4_GS_GIVEN && gs_mode != NVFP4_GS_AMAX_GIVEN)
    return NVFP4_ERR_INVALID_ARG;
  const int G = group_offsets ? num_groups : 1;
  if (G < 1 || G > kMaxGroups) return NVFP4_ERR_UNSUPPORTED_SHAPE;
  if (!global_scale || !workspace || !aligned16(workspace)) return NVFP4_ERR_INVALID_ARG;
  if (rows > 0 && (!x || !q || !sf || !aligned16(x) || !aligned16(q))) return NVFP4_ERR_INVALID_ARG;
  if (rows > ((int64_t)1 << 31)) return NVFP4_ERR_UNSUPPORTED_SHAPE;
  const uint16_t *xb = reinterpret_cast<const uint16_t *>(x);
  if (gs_mode == NVFP4_GS_FROM_AMAX && !group_offsets && !row_index && rows > 0 &&
      rows * (K / 16) <= (int64_t)0xFFFFFFC0ll) {
    bool launched = false;
    const nvfp4_status fs = run_fused_dense(xb, rows, K, ld_x, global_scale, q, sf, sf_layout, workspace,
                                            dev_status, stream, &launched);
    if (fs != NVFP4_OK || launched) return fs;
  }
  nvfp4_status st = run_global_scales(xb, rows, K, ld_x, row_index, group_offsets, G, gs_mode,
                                      global_scale, workspace, dev_status, stream);
  if (st != NVFP4_OK) return st;
  return run_encode(xb, rows, K, ld_x, row_index, group_offsets, G, global_scale, q, sf, sf_layout,
                    dev_status, stream);
}

nvfp4_status nvfp4_moe_quantize(const void *x, int64_t tokens, int64_t K, int64_t ld_x, const int32_t *slot,
                                int topk, const int32_t *group_offsets, int num_groups, nvfp4_gs_mode gs_mode,
                                float *global_scale, uint8_t *q, uint8_t *sf, nvfp4_sf_layout sf_layout,
                                void *workspace, int32_t *dev_status, cudaStream_t stream) {
  if (tokens < 0 || K <= 0 || ld_x < K || topk < 1 || topk > 32) return NVFP4_ERR_INVALID_ARG;
  if (K % 16 != 0 || ld_x % 8 != 0) return NVFP4_ERR_UNSUPPORTED_SHAPE;
  if (sf_layout != NVFP4_SF_ROWMAJOR && sf_layout != NVFP4_SF_MMA_TILED) return NVFP4_ERR_INVALID_ARG;
  if (sf_layout == NVFP4_SF_MMA_TILED && K % 64 != 0) return NVFP4_ERR_UNSUPPORTED_SHAPE;
  if (gs_mode != NVFP4_GS_FROM_AMAX && gs_mode != NVFP4_GS_GIVEN && gs_mode != NVFP4_GS_AMAX_GIVEN)
    return NVFP4_ERR_INVALID_ARG;
  const int G = num_groups;
  if (!group_offsets || G < 1 || G > kMaxGroups) return NVFP4_ERR_INVALID_ARG;
  if (!global_scale || !workspace || !aligned16(workspace)) return NVFP4_ERR_INVALID_ARG;
  if (tokens > 0 && (!x || !slot || !q || !sf || !aligned16(x) || !aligned16(q))) return NVFP4_ERR_INVALID_ARG;
  if (tokens * topk > ((int64_t)1 << 31)) return NVFP4_ERR_UNSUPPORTED_SHAPE;
  const uint16_t *xb = reinterpret_cast<const uint16_t *>(x);
  uint32_t *amax_bits = reinterpret_cast<uint32_t *>(workspace);
  const int64_t pieces = tokens * ((K / 16 + kAmaxPieceBlocks - 1) / kAmaxPieceBlocks);   // amax pass pieces
  if ((pieces + kAmaxWarps - 1) / kAmaxWarps > 0x7FFFFFFF) return NVFP4_ERR_UNSUPPORTED_SHAPE;
  if (gs_mode == NVFP4_GS_FROM_AMAX) {
    if (cudaMemsetAsync(amax_bits, 0, sizeof(uint32_t) * G, stream) != cudaSuccess) return NVFP4_ERR_CUDA;
    if (tokens > 0) {
      const size_t sm = sizeof(int32_t) * (G + 1);
      const unsigned grid = (unsigned)((pieces + kAmaxWarps - 1) / kAmaxWarps);
      moe_amax_kernel<<<grid, kAmaxWarps * 32, sm, stream>>>(xb, ld_x, K, tokens, slot, topk, group_offsets, G,
                                                             amax_bits, dev_status);
      if (cudaGetLastError() != cudaSuccess) return NVFP4_ERR_CUDA;
    }
  }
  float *rtab = workspace_tables(workspace, G), *ytab = rtab + (size_t)G * 128;
  finalize_tables_kernel<<<G, 128, 0, stream>>>(amax_bits, (int)gs_mode, global_scale, rtab, ytab, dev_status);
  if (cudaGetLastError() != cudaSuccess) return NVFP4_ERR_CUDA;
  if (tokens == 0) return NVFP4_OK;
  const size_t sm = sizeof(int32_t) * (2 * (G + 1) + 8);
  const int64_t work = tokens * ((K / 16 + 63) / 64) * 32;       // one warp per 64 blocks of a row
  if (sf_layout == NVFP4_SF_MMA_TILED) {
    const unsigned grid = (unsigned)grid_resident(moe_encode_blocks_kernel<true>, work, 256, sm);
    moe_encode_blocks_kernel<true><<<grid, 256, sm, stream>>>(xb, ld_x, K, tokens, slot, topk, group_offsets, G,
                                                              global_scale, rtab, ytab, q, sf, dev_status);
  } else {
    const unsigned grid = (unsigned)grid_resident(moe_encode_blocks_kernel<false>, work, 256, sm);
    moe_encode_blocks_kernel<false><<<grid, 256, sm, stream>>>(xb, ld_x, K, tokens, slot, topk, group_offsets, G,
                                                               global_scale, rtab, ytab, q, sf, dev_status);
  }
  return launch_status();
}

nvfp4_status nvfp4_global_scale_from_amax(const float *amax, int64_t n, float margin, float *global_scale,
                                          int32_t *dev_status, cudaStream_t stream) {
  if (n < 0 || !(margin > 0.0f) || !isfinite(margin)) return NVFP4_ERR_INVALID_ARG;
  if (n > ((int64_t)1 << 30)) return NVFP4_ERR_UNSUPPORTED_SHAPE;
  if (n == 0) return NVFP4_OK;
  if (!amax || !global_scale) return NVFP4_ERR_INVALID_ARG;
  gs_from_amax_kernel<<<(unsigned)((n + 255) / 256), 256, 0, stream>>>(amax, (int)n, margin, global_scale,
                                                                      dev_status);
  return launch_status();
}

nvfp4_status nvfp4_e2m1_encode(const float *x, int64_t n, uint8_t *q, cudaStream_t stream) {
  if (n < 0) return NVFP4_ERR_INVALID_ARG;
  if (n % 8 != 0) return NVFP4_ERR_UNSUPPORTED_SHAPE;
  if (n == 0) return NVFP4_OK;
  if (!x || !q || !aligned16(x) || !aligned16(q)) return NVFP4_ERR_INVALID_ARG;
  const int64_t n8 = n / 8;
  e2m1_encode_kernel<<<(unsigned)grid_for(n8, 256, 8), 256, 0, stream>>>(reinterpret_cast<const float4 *>(x), n8,
                                                                        reinterpret_cast<uint32_t *>(q));
  return launch_status();
}

nvfp4_status nvfp4_e4m3_encode(const float *x, int64_t n, uint8_t *out, cudaStream_t stream) {
  if (n < 0) return NVFP4_ERR_INVALID_ARG;
  if (n % 4 != 0) return NVFP4_ERR_UNSUPPORTED_SHAPE;
  if (n == 0) return NVFP4_OK;
  if (!x || !out || !aligned16(x) || !aligned16(out)) return NVFP4_ERR_INVALID_ARG;
  const int64_t n4 = n / 4;
  e4m3_encode_kernel<<<(unsigned)grid_for(n4, 256, 8), 256, 0, stream>>>(reinterpret_cast<const float4 *>(x), n4,
                                                                        reinterpret_cast<uint32_t *>(out));
  return launch_status();
}

nvfp4_status nvfp4_dequantize(const uint8_t *q, const uint8_t *sf, nvfp4_sf_layout sf_layout,
                              const float *global_scale, const int32_t *group_offsets, int num_groups,
                              int64_t rows, int64_t K, void *y, nvfp4_out_dtype out_dtype,
                              cudaStream_t stream) {
  if (rows < 0 || K <= 0 || K % 16 != 0) return NVFP4_ERR_UNSUPPORTED_SHAPE;
  if (sf_layout == NVFP4_SF_MMA_TILED && K % 64 != 0) return NVFP4_ERR_UNSUPPORTED_SHAPE;
  if (sf_layout != NVFP4_SF_ROWMAJOR && sf_layout != NVFP4_SF_MMA_TILED) return NVFP4_ERR_INVALID_ARG;
  if (out_dtype != NVFP4_OUT_F32 && out_dtype != NVFP4_OUT_BF16) return NVFP4_ERR_INVALID_ARG;
  const int G = group_offsets ? num_groups : 1;
  if (G < 1 || G > kMaxGroups) return NVFP4_ERR_UNSUPPORTED_SHAPE;
  if (rows == 0) return NVFP4_OK;
  if (!q || !sf || !global_scale || !y || !aligned16(q) || !aligned16(y)) return NVFP4_ERR_INVALID_ARG;
  const bool tiled = sf_layout == NVFP4_SF_MMA_TILED, bf = out_dtype == NVFP4_OUT_BF16;
  if (!group_offsets && ((reinterpret_cast<uintptr_t>(y) & 31u) == 0)) {
    // 32-byte output stores need a 32-byte aligned y (rows of K % 16 == 0 elements keep it)
    const int64_t warps = (rows * (K / 16) + 255) / 256;
#define NVFP4_DQF(T, B)                                                                                        \
  dequantize_flat_kernel<T, B><<<(unsigned)grid_resident(dequantize_flat_kernel<T, B>, warps * 32, 256, 0), 256, 0, \
                                 stream>>>(q, sf, global_scale, rows, K, y)
    if (tiled && bf) NVFP4_DQF(true, true);
    else if (tiled) NVFP4_DQF(true, false);
    else if (bf) NVFP4_DQF(false, true);
    else NVFP4_DQF(false, false);
#undef NVFP4_DQF
    return launch_status();
  }
  const int64_t work = rows * (K / 8);
  const unsigned grid = (unsigned)grid_for(work, 256, 8);
  const size_t sm = group_offsets ? sizeof(int32_t) * (2 * (G + 1) + 8) : 0;
#define NVFP4_DQ(T, B) dequantize_kernel<T, B><<<grid, 256, sm, stream>>>(q, sf, global_scale, group_offsets, G, rows, K, y)
  if (tiled && bf) NVFP4_DQ(true, true);
  else if (tiled) NVFP4_DQ(true, false);
  else if (bf) NVFP4_DQ(false, true);
  else NVFP4_DQ(false, false);
#undef NVFP4_DQ
  return launch_status();
}

nvfp4_status nvfp4_swiglu_quantize(const void *y, nvfp4_out_dtype y_dtype, int64_t rows, int64_t I,
                                   const int32_t *group_offsets, int num_groups, float *global_scale,
                                   uint8_t *q, uint8_t *sf, nvfp4_sf_layout sf_layout, void *h,
                                   void *workspace, int32_t *dev_status, cudaStream_t stream) {
  if (rows < 0 || I <= 0 || I % 16 != 0) return NVFP4_ERR_UNSUPPORTED_SHAPE;
  if (sf_layout == NVFP4_SF_MMA_TILED && I % 64 != 0) return NVFP4_ERR_UNSUPPORTED_SHAPE;
  if (y_dtype != NVFP4_OUT_F32 && y_dtype != NVFP4_OUT_BF16) return NVFP4_ERR_INVALID_ARG;
  const int G = group_offsets ? num_groups : 1;
  if (G < 1 || G > kMaxGroups) return NVFP4_ERR_UNSUPPORTED_SHAPE;
  if (!global_scale || !workspace || !aligned16(workspace)) return NVFP4_ERR_INVALID_ARG;
  if (rows > 0 && (!y || !q || !sf || !h || !aligned16(y) || !aligned16(q) || !aligned16(h)))
    return NVFP4_ERR_INVALID_ARG;
  uint32_t *amax_bits = reinterpret_cast<uint32_t *>(workspace);
  if (cudaMemsetAsync(amax_bits, 0, sizeof(uint32_t) * G, stream) != cudaSuccess) return NVFP4_ERR_CUDA;
  if (rows > 0) {
    const size_t sm = group_offsets ? sizeof(int32_t) * (G + 1) : 0;
    if (y_dtype == NVFP4_OUT_BF16) {
      const unsigned grid = (unsigned)grid_resident(swiglu_amax_kernel<true>, rows * 32, 256, sm);
      swiglu_amax_kernel<true><<<grid, 256, sm, stream>>>(y, rows, I, group_offsets, G, (uint16_t *)h, amax_bits);
    } else {
      const unsigned grid = (unsigned)grid_resident(swiglu_amax_kernel<false>, rows * 32, 256, sm);
      swiglu_amax_kernel<false><<<grid, 256, sm, stream>>>(y, rows, I, group_offsets, G, (uint16_t *)h, amax_bits);
    }
    if (cudaGetLastError() != cudaSuccess) return NVFP4_ERR_CUDA;
  }
  finalize_scales_kernel<<<(G + 127) / 128, 128, 0, stream>>>(amax_bits, G, (int)NVFP4_GS_FROM_AMAX, global_scale,
                                                              dev_status);
  if (cudaGetLastError() != cudaSuccess) return NVFP4_ERR_CUDA;
  return run_encode(reinterpret_cast<const uint16_t *>(h), rows, I, I, nullptr, group_offsets, G,
                    global_scale, q, sf, sf_layout, dev_status, stream);
}

nvfp4_status nvfp4_kv_quantize(const void *k, const void *v, int64_t tokens, int64_t heads,
                               int64_t head_dim, nvfp4_gs_mode gs_mode, float *k_gs, float *v_gs,
                               uint8_t *k_q, uint8_t *k_sf, uint8_t *v_q, uint8_t *v_sf,
                               void *workspace, int32_t *dev_status, cudaStream_t stream) {
  if (tokens < 0 || heads <= 0 || head_dim <= 0) return NVFP4_ERR_INVALID_ARG;
  const int64_t rows = tokens * heads;
  nvfp4_status st = nvfp4_quantize(k, rows, head_dim, head_dim, nullptr, nullptr, 1, gs_mode, k_gs,
                                   k_q, k_sf, NVFP4_SF_ROWMAJOR, workspace, dev_status, stream);
  if (st != NVFP4_OK) return st;
  return nvfp4_quantize(v, rows, head_dim, head_dim, nullptr, nullptr, 1, gs_mode, v_gs, v_q, v_sf,
                        NVFP4_SF_ROWMAJOR, reinterpret_cast<char *>(workspace) + 16, dev_status, stream);
}

nvfp4_status nvfp4_kv_dequantize(const uint8_t *k_q, const uint8_t *k_sf, const float *k_gs,
                                 const uint8_t *v_q, const uint8_t *v_sf, const float *v_gs,
                                 int64_t tokens, int64_t heads, int64_t head_dim, void *k_out,
                                 void *v_out, cudaStream_t stream) {
  if (tokens < 0 || heads <= 0 || head_dim <= 0) return NVFP4_ERR_INVALID_ARG;
  const int64_t rows = tokens * heads;
  nvfp4_status st = nvfp4_dequantize(k_q, k_sf, NVFP4_SF_ROWMAJOR, k_gs, nullptr, 1, rows, head_dim,
                                     k_out, NVFP4_OUT_BF16, stream);
  if (st != NVFP4_OK) return st;
  return nvfp4_dequantize(v_q, v_sf, NVFP4_SF_ROWMAJOR, v_gs, nullptr, 1, rows, head_dim, v_out,
                          NVFP4_OUT_BF16, stream);
}

}  // extern "C"

// ======================================================= allocation-free variant
// Scratch of nvfp4_quantize_noalloc: the per-group amax words (the same layout
// nvfp4_quantize keeps in the caller's workspace), one copy per device.
static __device__ __align__(256) uint32_t g_noalloc_scratch[2 * NVFP4_NOALLOC_MAX_GROUPS + 64];

namespace {
std::mutex g_noalloc_mu;
void *g_noalloc_ptr[64] = {};       // per device ordinal, filled by the first call on that device
}  // namespace

extern "C" nvfp4_status nvfp4_quantize_noalloc(const void *x, int64_t rows, int64_t K, int64_t ld_x,
                                               const int32_t *row_index, const int32_t *group_offsets,
                                               int num_groups, nvfp4_gs_mode gs_mode, float *global_scale,
                                               uint8_t *q, uint8_t *sf, nvfp4_sf_layout sf_layout,
                                               int32_t *dev_status, cudaStream_t stream) {
  const int G = group_offsets ? num_groups : 1;
  if (G < 1) return NVFP4_ERR_UNSUPPORTED_SHAPE;
  if (G > NVFP4_NOALLOC_MAX_GROUPS) return NVFP4_ERR_UNSUPPORTED_SHAPE;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return NVFP4_ERR_CUDA;
  void *scratch;
  {
    std::lock_guard<std::mutex> lock(g_noalloc_mu);
    if (!g_noalloc_ptr[dev]) {
      // host code cannot use the array's name as a device address: ask the
      // runtime for this device's address of it, once
      void *ptr = nullptr;
      if (cudaGetSymbolAddress(&ptr, g_noalloc_scratch) != cudaSuccess || !ptr) return NVFP4_ERR_CUDA;
      g_noalloc_ptr[dev] = ptr;
    }
    scratch = g_noalloc_ptr[dev];
  }
  return nvfp4_quantize(x, rows, K, ld_x, row_index, group_offsets, num_groups, gs_mode, global_scale, q, sf,
                        sf_layout, scratch, dev_status, stream);
}
