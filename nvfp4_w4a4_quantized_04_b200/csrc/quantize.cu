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

// Dense contiguous tensor: flat grid-stride over 16-byte vectors.
__global__ void __launch_bounds__(256) amax_flat_kernel(const uint4 *__restrict__ x, int64_t nvec,
                                                        uint32_t *__restrict__ amax_bits) {
  const int64_t tid = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  const int64_t stride = (int64_t)gridDim.x * blockDim.x;
  uint32_t m = 0;
  int64_t i = tid;
  for (; i + 3 * stride < nvec; i += 4 * stride) {
    uint4 a = ldg_nc_v4(x + i), b = ldg_nc_v4(x + i + stride);
    uint4 c = ldg_nc_v4(x + i + 2 * stride), d = ldg_nc_v4(x + i + 3 * stride);
    m = absmax8_bits(a, m); m = absmax8_bits(b, m);
    m = absmax8_bits(c, m); m = absmax8_bits(d, m);
  }
  for (; i < nvec; i += stride) m = absmax8_bits(ldg_nc_v4(x + i), m);
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

// Global scales from the amax (FROM_AMAX; AMAX_GIVEN reads the amax from gs
// itself) or a check of the given ones (GIVEN).
__global__ void finalize_scales_kernel(const uint32_t *__restrict__ amax_bits, int G, int mode,
                                       float *__restrict__ gs, int32_t *dev_status) {
  int g = blockIdx.x * blockDim.x + threadIdx.x;
  if (g >= G) return;
  if (mode == NVFP4_GS_GIVEN) {
    float s = gs[g];
    if (!(s > 0.0f) || !isfinite(s)) report(dev_status, NVFP4_ERR_INVALID_ARG);
    return;
  }
  uint32_t b = mode == NVFP4_GS_AMAX_GIVEN ? (__float_as_uint(gs[g]) & 0x7FFFFFFFu) : amax_bits[g];
  if (b >= 0x7F800000u) {
    gs[g] = __uint_as_float(0x7FC00000u);
    report(dev_status, NVFP4_ERR_NONFINITE);
    return;
  }
  float a = __uint_as_float(b);
  gs[g] = (a == 0.0f) ? 1.0f : __fdiv_rn(a, 2688.0f);   // 2688 = 6 * 448
}

// ---------------------------------------------------------------- pass 2: encode
// One thread per 16-element block: one 32-byte load (two 16-byte loads when
// the row stride is not 32-byte aligned), the block amax in integer SIMD,
// one IEEE division for the scale and one IEEE reciprocal per block, the
// 16 products as eight packed f32x2 multiplies, eight e2m1x2 conversions and
// one 8-byte store.  A warp covers 32 consecutive blocks per step; warps
// stride over 64-block chunks so the whole grid streams through memory
// together.  Rows only move forward per lane, so the row -> (group, source
// row) lookup walks forward from the last group.
__device__ __forceinline__ uint2 load_block(const uint16_t *p, bool v8, uint4 &a, uint4 &b) {
  if (v8) {
    asm volatile("ld.global.nc.L1::no_allocate.v8.b32 {%0,%1,%2,%3,%4,%5,%6,%7}, [%8];"
                 : "=r"(a.x), "=r"(a.y), "=r"(a.z), "=r"(a.w), "=r"(b.x), "=r"(b.y), "=r"(b.z), "=r"(b.w)
                 : "l"(p));
  } else {
    a = ldg_nc_v4(p);
    b = ldg_nc_v4(p + 8);
  }
  return make_uint2(0, 0);
}

// bf16 pair (lo in bits 0..15) times r, both products rounded to nearest even.
__device__ __forceinline__ uint64_t mul_pair(uint32_t w, uint64_t rr) {
  const uint64_t x = ((uint64_t)(w & 0xFFFF0000u) << 32) | (uint64_t)(w << 16);
  uint64_t d;
  asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(x), "l"(rr));
  return d;
}

__device__ __forceinline__ uint32_t e2m1x4_from_pairs(uint64_t p0, uint64_t p1) {
  uint32_t out;
  asm("{\n.reg .b8 b0, b1;\n.reg .f32 l0, h0, l1, h1;\n"
      "mov.b64 {l0, h0}, %1;\nmov.b64 {l1, h1}, %2;\n"
      "cvt.rn.satfinite.e2m1x2.f32 b0, h0, l0;\n"
      "cvt.rn.satfinite.e2m1x2.f32 b1, h1, l1;\n"
      "mov.b32 %0, {b0, b1, b0, b1};\n}"
      : "=r"(out) : "l"(p0), "l"(p1));
  return out & 0xFFFFu;
}

__device__ __forceinline__ uint64_t sanitize_pair(uint64_t d) {
  float lo = __uint_as_float((uint32_t)d), hi = __uint_as_float((uint32_t)(d >> 32));
  lo = isnan(lo) ? 0.0f : lo;
  hi = isnan(hi) ? 0.0f : hi;
  return ((uint64_t)__float_as_uint(hi) << 32) | __float_as_uint(lo);
}

// The 16-element block math (see the definition in include/nvfp4.h): block
// amax, S = e4m3(a_b / (6 s_g)), r = 1/(S s_g), codes = e2m1(x r).  Returns
// the 8 packed code bytes and S; flags non-finite input.
__device__ __forceinline__ uint2 encode_block16(const uint4 &va, const uint4 &vb, float s_g, float t_g, bool real,
                                                uint32_t &S, bool &bad) {
  const uint32_t m = halves_max(absmax8_bits(vb, absmax8_bits(va, 0)));
  if (real && m >= 0x7F80u) bad = true;
  S = 0;
  if (real) S = f32_to_e4m3_satfinite(__fdiv_rn(__uint_as_float(m << 16), t_g));
  const float e = __fmul_rn(e4m3_to_f32(S), s_g);
  const float r = (e == 0.0f) ? 0.0f : __frcp_rn(e);
  const uint64_t rr = ((uint64_t)__float_as_uint(r) << 32) | __float_as_uint(r);
  const uint32_t w[8] = {va.x, va.y, va.z, va.w, vb.x, vb.y, vb.z, vb.w};
  uint64_t prod[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) prod[i] = mul_pair(w[i], rr);
  if (isinf(r)) {                     // 0 * inf: the NaN encodes as +0
#pragma unroll
    for (int i = 0; i < 8; ++i) prod[i] = sanitize_pair(prod[i]);
  }
  uint2 codes;
  codes.x = e2m1x4_from_pairs(prod[0], prod[1]) | (e2m1x4_from_pairs(prod[2], prod[3]) << 16);
  codes.y = e2m1x4_from_pairs(prod[4], prod[5]) | (e2m1x4_from_pairs(prod[6], prod[7]) << 16);
  return codes;
}

// Gathered long rows (row_index, K >= 2048): one warp per output row, the row's group and source
// row looked up once, up to 8 blocks (256 bytes) in flight per lane; warps
// stride over rows so the grid streams through the input together.
template <bool kTiled>
__global__ void __launch_bounds__(256) quantize_rows_kernel(
    const uint16_t *__restrict__ x, int64_t ld_x, int64_t K64, int64_t rows,
    const int32_t *__restrict__ row_index, const int32_t *__restrict__ group_offsets, int G,
    int64_t P, const float *__restrict__ gs, uint8_t *__restrict__ q, uint8_t *__restrict__ sf,
    int32_t *dev_status) {
  extern __shared__ int32_t smem[];
  int32_t *off = smem, *slot = smem + (G + 1), *scratch = smem + 2 * (G + 1);
  if (group_offsets) load_groups(group_offsets, G, off, slot, scratch);
  const int lane = threadIdx.x & 31;
  const uint32_t K = (uint32_t)K64, nblk = K >> 4;
  const uint32_t p_end = group_offsets ? (uint32_t)slot[G] : (uint32_t)P;
  const uint32_t warp = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const uint32_t nwarps = (gridDim.x * blockDim.x) >> 5;
  const bool v8 = ((reinterpret_cast<uintptr_t>(x) & 31u) == 0) && ((ld_x & 15) == 0);
  int g = 0;
  bool bad = false;
  constexpr int B = 8;
  for (uint32_t p = warp; p < p_end; p += nwarps) {
    bool real;
    int64_t src;
    if (group_offsets) {
      if (g + 8 < G && (uint32_t)slot[g + 8] <= p) g = upper_group(slot, G, p);
      while (g + 1 < G && (uint32_t)slot[g + 1] <= p) ++g;
      const uint32_t local = p - (uint32_t)slot[g];
      real = local < (uint32_t)(off[g + 1] - off[g]);
      src = (int64_t)off[g] + local;
    } else {
      real = p < (uint64_t)rows;
      src = p;
    }
    if (real && row_index) src = row_index[src];
    const float s_g = real ? gs[g] : 1.0f;
    const float t_g = __fmul_rn(6.0f, s_g);
    const uint16_t *xr = x + src * ld_x;
    uint8_t *qr = q + (uint64_t)p * (K >> 1);
    for (uint32_t j0 = 0; j0 < nblk; j0 += 32 * B) {
      uint4 va[B], vb[B];
#pragma unroll
      for (int k = 0; k < B; ++k) {
        const uint32_t j = j0 + k * 32 + lane;
        va[k] = make_uint4(0, 0, 0, 0);
        vb[k] = make_uint4(0, 0, 0, 0);
        if (real && j < nblk) load_block(xr + (uint64_t)j * 16, v8, va[k], vb[k]);
      }
#pragma unroll
      for (int k = 0; k < B; ++k) {
        const uint32_t j = j0 + k * 32 + lane;
        uint32_t S;
        const uint2 codes = encode_block16(va[k], vb[k], s_g, t_g, real && j < nblk, S, bad);
        if (j < nblk) {
          *reinterpret_cast<uint2 *>(qr + (uint64_t)j * 8) = codes;
          if (kTiled) sf[sf_tiled_offset(p, j, nblk)] = (uint8_t)S;
          else sf[(uint64_t)p * nblk + j] = (uint8_t)S;
        }
      }
    }
  }
  if (bad) report(dev_status, NVFP4_ERR_NONFINITE);
}

template <bool kTiled>
__global__ void __launch_bounds__(256) quantize_kernel(
    const uint16_t *__restrict__ x, int64_t ld_x, int64_t K64, int64_t rows,
    const int32_t *__restrict__ row_index, const int32_t *__restrict__ group_offsets, int G,
    int64_t P, const float *__restrict__ gs, uint8_t *__restrict__ q, uint8_t *__restrict__ sf,
    int32_t *dev_status) {
  extern __shared__ int32_t smem[];
  int32_t *off = smem, *slot = smem + (G + 1), *scratch = smem + 2 * (G + 1);
  if (group_offsets) load_groups(group_offsets, G, off, slot, scratch);
  const int lane = threadIdx.x & 31;
  const uint32_t K = (uint32_t)K64, nblk = K >> 4;
  const uint32_t p_end = group_offsets ? (uint32_t)slot[G] : (uint32_t)P;
  const uint64_t total = (uint64_t)p_end * nblk;             // blocks, row-major
  constexpr int U = 2;                                       // 32-block steps per chunk
  const uint64_t nchunks = (total + 32 * U - 1) / (32 * U);
  const uint64_t warp = ((uint64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const uint64_t nwarps = ((uint64_t)gridDim.x * blockDim.x) >> 5;
  const bool small = total < 0xFFFFFFF0ull;
  const bool v8 = ((reinterpret_cast<uintptr_t>(x) & 31u) == 0) && ((ld_x & 15) == 0);
  int g = 0;
  uint32_t cached_p = 0xFFFFFFFFu;
  int64_t cached_src = -1;
  bool cached_real = false;
  float s_g = 1.0f, t_g = 6.0f;
  int g_for_scale = -1;
  bool bad = false;
  for (uint64_t c = warp; c < nchunks; c += nwarps) {
    uint4 va[U], vb[U];
    uint32_t pp[U], jj[U];
    bool real[U], inr[U];
    float sg[U], tg[U];
#pragma unroll
    for (int k = 0; k < U; ++k) {
      const uint64_t b = c * (32 * U) + k * 32 + lane;
      inr[k] = b < total;
      uint32_t p = 0, j = 0;
      if (inr[k]) {
        if (small) { p = (uint32_t)b / nblk; j = (uint32_t)b - p * nblk; }
        else { p = (uint32_t)(b / nblk); j = (uint32_t)(b - (uint64_t)p * nblk); }
        if (p != cached_p) {
          cached_p = p;
          if (group_offsets) {
            if (g + 8 < G && (uint32_t)slot[g + 8] <= p) g = upper_group(slot, G, p);
            while (g + 1 < G && (uint32_t)slot[g + 1] <= p) ++g;
            const uint32_t local = p - (uint32_t)slot[g];
            cached_real = local < (uint32_t)(off[g + 1] - off[g]);
            cached_src = (int64_t)off[g] + local;
          } else {
            cached_real = p < (uint64_t)rows;
            cached_src = p;
          }
          if (cached_real && row_index) cached_src = row_index[cached_src];
          if (g != g_for_scale) {
            g_for_scale = g;
            s_g = gs[g];
            t_g = __fmul_rn(6.0f, s_g);
          }
        }
      }
      pp[k] = p;
      jj[k] = j;
      real[k] = inr[k] && cached_real;
      sg[k] = s_g;
      tg[k] = t_g;
      va[k] = make_uint4(0, 0, 0, 0);
      vb[k] = make_uint4(0, 0, 0, 0);
      if (real[k]) load_block(x + cached_src * ld_x + (uint64_t)j * 16, v8, va[k], vb[k]);
    }
#pragma unroll
    for (int k = 0; k < U; ++k) {
      uint32_t S;
      const uint2 codes = encode_block16(va[k], vb[k], sg[k], tg[k], real[k], S, bad);
      if (inr[k]) {
        *reinterpret_cast<uint2 *>(q + (uint64_t)pp[k] * (K >> 1) + (uint64_t)jj[k] * 8) = codes;
        if (kTiled) sf[sf_tiled_offset(pp[k], jj[k], nblk)] = (uint8_t)S;
        else sf[(uint64_t)pp[k] * nblk + jj[k]] = (uint8_t)S;
      }
    }
  }
  if (bad) report(dev_status, NVFP4_ERR_NONFINITE);
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
  if (group_offsets) load_groups(group_offsets, G, off, slot, scratch);
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

int g_num_sms = 0;

int num_sms() {
  if (g_num_sms == 0) {
    int dev = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&g_num_sms, cudaDevAttrMultiProcessorCount, dev);
    if (g_num_sms <= 0) g_num_sms = 148;
  }
  return g_num_sms;
}

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

int64_t grid_for(int64_t work_items, int threads, int per_sm) {
  int64_t need = (work_items + threads - 1) / threads;
  int64_t cap = (int64_t)num_sms() * per_sm;
  if (need < 1) need = 1;
  return need < cap ? need : cap;
}

// Grid for a grid-stride kernel: at most one wave of resident blocks, so no
// block starts late with a full share of the work.
struct OccEntry { const void *fn; int threads; size_t smem; int per_sm; };
OccEntry g_occ[64];
int g_occ_n = 0;

template <typename Kernel>
int64_t grid_resident(Kernel kernel, int64_t work_items, int threads, size_t smem) {
  const void *fn = reinterpret_cast<const void *>(kernel);
  int per_sm = 0;
  for (int i = 0; i < g_occ_n; ++i)
    if (g_occ[i].fn == fn && g_occ[i].threads == threads && g_occ[i].smem == smem) per_sm = g_occ[i].per_sm;
  if (per_sm == 0) {
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kernel, threads, smem) != cudaSuccess || per_sm < 1)
      per_sm = 1;
    if (g_occ_n < 64) g_occ[g_occ_n++] = OccEntry{fn, threads, smem, per_sm};
  }
  return grid_for(work_items, threads, per_sm);
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
        int64_t nvec = rows * K / 8;
        amax_flat_kernel<<<(unsigned)grid_for(nvec / 4, 256, 8), 256, 0, stream>>>(
            reinterpret_cast<const uint4 *>(x), nvec, amax_bits);
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
  int64_t P;
  if (group_offsets) P = nvfp4_padded_rows_bound(rows, G);
  else P = tiled ? (rows + 127) / 128 * 128 : rows;
  if (P == 0) return NVFP4_OK;
  const int64_t blocks = P * (K / 16);
  const size_t sm = group_offsets ? sizeof(int32_t) * (2 * (G + 1) + 8) : 0;
  if (row_index && K >= 2048 && P <= 0xFFFFFFFFll) {
    // one warp per output row
    if (tiled) {
      const unsigned grid = (unsigned)grid_resident(quantize_rows_kernel<true>, P * 32, 256, sm);
      quantize_rows_kernel<true><<<grid, 256, sm, stream>>>(x, ld_x, K, rows, row_index, group_offsets, G, P, gs, q, sf, dev_status);
    } else {
      const unsigned grid = (unsigned)grid_resident(quantize_rows_kernel<false>, P * 32, 256, sm);
      quantize_rows_kernel<false><<<grid, 256, sm, stream>>>(x, ld_x, K, rows, row_index, group_offsets, G, P, gs, q, sf, dev_status);
    }
    return launch_status();
  }
  if (tiled) {
    const unsigned grid = (unsigned)grid_resident(quantize_kernel<true>, (blocks + 1) / 2, 256, sm);
    quantize_kernel<true><<<grid, 256, sm, stream>>>(x, ld_x, K, rows, row_index, group_offsets, G, P, gs, q, sf, dev_status);
  } else {
    const unsigned grid = (unsigned)grid_resident(quantize_kernel<false>, (blocks + 1) / 2, 256, sm);
    quantize_kernel<false><<<grid, 256, sm, stream>>>(x, ld_x, K, rows, row_index, group_offsets, G, P, gs, q, sf, dev_status);
  }
  return launch_status();
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
  // amax / exponent-range words (2 per group) plus room for kernel bookkeeping
  size_t bytes = sizeof(uint32_t) * 2 * (size_t)num_groups + 256;
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
  nvfp4_status st = run_global_scales(xb, rows, K, ld_x, row_index, group_offsets, G, gs_mode,
                                      global_scale, workspace, dev_status, stream);
  if (st != NVFP4_OK) return st;
  return run_encode(xb, rows, K, ld_x, row_index, group_offsets, G, global_scale, q, sf, sf_layout,
                    dev_status, stream);
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
