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

// Global scales from the amax (FROM_AMAX) or a check of the given ones.
__global__ void finalize_scales_kernel(const uint32_t *__restrict__ amax_bits, int G, int given,
                                       float *__restrict__ gs, int32_t *dev_status) {
  int g = blockIdx.x * blockDim.x + threadIdx.x;
  if (g >= G) return;
  if (given) {
    float s = gs[g];
    if (!(s > 0.0f) || !isfinite(s)) report(dev_status, NVFP4_ERR_INVALID_ARG);
    return;
  }
  uint32_t b = amax_bits[g];
  if (b >= 0x7F800000u) {
    gs[g] = __uint_as_float(0x7FC00000u);
    report(dev_status, NVFP4_ERR_NONFINITE);
    return;
  }
  float a = __uint_as_float(b);
  gs[g] = (a == 0.0f) ? 1.0f : __fdiv_rn(a, 2688.0f);   // 2688 = 6 * 448
}

// ---------------------------------------------------------------- pass 2: encode
// One thread pair per 16-element block (8 elements = one 16-byte load per
// thread); a warp covers 16 consecutive blocks per chunk and owns a
// contiguous range of chunks, so its output-row -> expert-group lookup only
// ever moves forward and is kept across iterations.  The index space is the
// padded output rows, so slot padding is zero-filled by the same pass.
struct EncodeItem {
  uint4 v;
  uint32_t p, j;
  int g;
  bool in_range, real;
};

template <bool kTiled>
__device__ __forceinline__ void encode_finish(const EncodeItem &it, int half, uint32_t nblk, uint32_t K,
                                              const float *__restrict__ gs, uint8_t *__restrict__ q,
                                              uint8_t *__restrict__ sf, bool &bad) {
  uint32_t m = halves_max(absmax8_bits(it.v, 0));
  m = max(m, __shfl_xor_sync(0xffffffffu, m, 1));
  if (it.real && m >= 0x7F80u) bad = true;
  const float s_g = it.real ? gs[it.g] : 1.0f;
  const float a_b = __uint_as_float(m << 16);
  uint32_t S = 0;
  if (it.real) S = f32_to_e4m3_satfinite(__fdiv_rn(a_b, __fmul_rn(6.0f, s_g)));
  const float e = __fmul_rn(e4m3_to_f32(S), s_g);
  const float r = (e == 0.0f) ? 0.0f : __frcp_rn(e);
  float f[8];
  const uint32_t w[4] = {it.v.x, it.v.y, it.v.z, it.v.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float lo = __fmul_rn(bf16_bits_to_f32(w[i] & 0xFFFFu), r);
    const float hi = __fmul_rn(bf16_bits_to_f32(w[i] >> 16), r);
    f[2 * i] = isnan(lo) ? 0.0f : lo;
    f[2 * i + 1] = isnan(hi) ? 0.0f : hi;
  }
  const uint32_t codes = f32x8_to_e2m1x8(f);
  if (it.in_range) {
    *reinterpret_cast<uint32_t *>(q + (uint64_t)it.p * (K >> 1) + it.j * 8 + half * 4) = codes;
    if (half == 0) {
      if (kTiled) sf[sf_tiled_offset(it.p, it.j, nblk)] = (uint8_t)S;
      else sf[(uint64_t)it.p * nblk + it.j] = (uint8_t)S;
    }
  }
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
  const int lane = threadIdx.x & 31, half = lane & 1;
  const uint32_t K = (uint32_t)K64, nblk = K >> 4;
  const uint32_t nsl = (nblk + 15) >> 4;                     // 16-block slices per row
  const uint32_t p_end = group_offsets ? (uint32_t)slot[G] : (uint32_t)P;
  const uint64_t units = (uint64_t)p_end * nsl;              // (row, slice) work units, row-major
  constexpr int U = 4;                                       // consecutive units per warp step
  const uint64_t nchunks = (units + U - 1) / U;
  const uint64_t warp = ((uint64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const uint64_t nwarps = ((uint64_t)gridDim.x * blockDim.x) >> 5;
  const bool small = units < 0xFFFFFFF0ull;
  // Warps stride over 4-unit chunks (2 KB of input per warp step, all warps
  // moving through memory together).  Rows only move forward per lane, so the
  // row -> (group, source row) lookup walks forward from the last group.
  int g = 0;
  uint32_t cached_p = 0xFFFFFFFFu;
  int64_t cached_src = -1;
  bool cached_real = false;
  bool bad = false;
  for (uint64_t c = warp; c < nchunks; c += nwarps) {
    EncodeItem it[U];
    int64_t src[U];
#pragma unroll
    for (int k = 0; k < U; ++k) {
      const uint64_t unit = c * U + k;
      uint32_t p = 0, sl = 0;
      if (unit < units) {
        if (small) { p = (uint32_t)unit / nsl; sl = (uint32_t)unit - p * nsl; }
        else { p = (uint32_t)(unit / nsl); sl = (uint32_t)(unit - (uint64_t)p * nsl); }
      }
      const uint32_t j = sl * 16 + (lane >> 1);
      it[k].in_range = unit < units && j < nblk;
      it[k].p = p;
      it[k].j = j;
      if (unit < units && p != cached_p) {
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
      }
      it[k].g = g;
      it[k].real = it[k].in_range && cached_real;
      src[k] = cached_src;
    }
#pragma unroll
    for (int k = 0; k < U; ++k) {
      it[k].v = make_uint4(0, 0, 0, 0);
      if (it[k].real) it[k].v = ldg_nc_v4(x + src[k] * ld_x + it[k].j * 16 + half * 8);
    }
#pragma unroll
    for (int k = 0; k < U; ++k) encode_finish<kTiled>(it[k], half, nblk, K, gs, q, sf, bad);
  }
  if (bad) report(dev_status, NVFP4_ERR_NONFINITE);
}

// ---------------------------------------------------------------- dequantize
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
  for (uint64_t h = (uint64_t)blockIdx.x * blockDim.x + threadIdx.x; h < total; h += stride) {
    const uint64_t r = h / nhalf, c = h - r * nhalf;
    const uint64_t j = c >> 1;
    int g = 0;
    uint64_t p = r;
    if (group_offsets) {
      g = upper_group(off, G, (int64_t)r);
      p = (uint64_t)slot[g] + (r - (uint64_t)off[g]);
    }
    const float s_g = gs[g];
    const float Sv = e4m3_to_f32(kTiled ? sf[sf_tiled_offset(p, j, nblk)] : sf[p * nblk + j]);
    const uint32_t cw = *reinterpret_cast<const uint32_t *>(q + p * (K >> 1) + c * 4);
    float out[8];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const uint32_t byte = (cw >> (8 * i)) & 0xFFu;
      out[2 * i] = __fmul_rn(__fmul_rn(e2m1_to_f32(byte & 15u), Sv), s_g);
      out[2 * i + 1] = __fmul_rn(__fmul_rn(e2m1_to_f32(byte >> 4), Sv), s_g);
    }
    if (kBf16) {
      uint32_t hw[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        __nv_bfloat162 t = __floats2bfloat162_rn(out[2 * i], out[2 * i + 1]);
        hw[i] = *reinterpret_cast<uint32_t *>(&t);
      }
      *reinterpret_cast<uint4 *>(reinterpret_cast<uint16_t *>(y) + r * K + c * 8) = make_uint4(hw[0], hw[1], hw[2], hw[3]);
    } else {
      float4 *dst = reinterpret_cast<float4 *>(reinterpret_cast<float *>(y) + r * K + c * 8);
      dst[0] = make_float4(out[0], out[1], out[2], out[3]);
      dst[1] = make_float4(out[4], out[5], out[6], out[7]);
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

nvfp4_status launch_status() {
  return cudaGetLastError() == cudaSuccess ? NVFP4_OK : NVFP4_ERR_CUDA;
}

// amax pass + global-scale finalisation, shared by quantize and KV paths.
nvfp4_status run_global_scales(const uint16_t *x, int64_t rows, int64_t K, int64_t ld_x,
                               const int32_t *row_index, const int32_t *group_offsets, int G,
                               nvfp4_gs_mode gs_mode, float *global_scale, void *workspace,
                               int32_t *dev_status, cudaStream_t stream) {
  uint32_t *amax_bits = reinterpret_cast<uint32_t *>(workspace);
  const int given = gs_mode == NVFP4_GS_GIVEN;
  if (!given) {
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
  finalize_scales_kernel<<<(G + 127) / 128, 128, 0, stream>>>(amax_bits, G, given, global_scale, dev_status);
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
  const int64_t pairs = P * (K / 16);
  const size_t sm = group_offsets ? sizeof(int32_t) * (2 * (G + 1) + 8) : 0;
  const unsigned grid = (unsigned)grid_for(pairs * 2, 256, 8);
  if (tiled)
    quantize_kernel<true><<<grid, 256, sm, stream>>>(x, ld_x, K, rows, row_index, group_offsets, G, P, gs, q, sf, dev_status);
  else
    quantize_kernel<false><<<grid, 256, sm, stream>>>(x, ld_x, K, rows, row_index, group_offsets, G, P, gs, q, sf, dev_status);
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
  if (gs_mode != NVFP4_GS_FROM_AMAX && gs_mode != NVFP4_GS_GIVEN) return NVFP4_ERR_INVALID_ARG;
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
    const unsigned grid = (unsigned)grid_for(rows * 32, 256, 8);
    if (y_dtype == NVFP4_OUT_BF16)
      swiglu_amax_kernel<true><<<grid, 256, sm, stream>>>(y, rows, I, group_offsets, G, (uint16_t *)h, amax_bits);
    else
      swiglu_amax_kernel<false><<<grid, 256, sm, stream>>>(y, rows, I, group_offsets, G, (uint16_t *)h, amax_bits);
    if (cudaGetLastError() != cudaSuccess) return NVFP4_ERR_CUDA;
  }
  finalize_scales_kernel<<<(G + 127) / 128, 128, 0, stream>>>(amax_bits, G, 0, global_scale, dev_status);
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
