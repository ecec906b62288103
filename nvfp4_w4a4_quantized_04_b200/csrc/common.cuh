// Shared device helpers of the NVFP4 CUDA library (sm_100a only).
#pragma once

#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <stdint.h>

#include "nvfp4.h"

#if defined(__CUDA_ARCH__) && (__CUDA_ARCH__ < 1000)
#error "this library targets sm_100a only"
#endif

namespace nvfp4 {

constexpr int kSlotAlign = 128;       // rows per expert slot granule (MMA tile rows)
constexpr int kMaxGroups = 4096;      // largest num_groups / num_experts accepted

// First data error wins; nothing traps.
__device__ __forceinline__ void report(int32_t *dev_status, int code) {
  if (dev_status) atomicCAS(dev_status, 0, code);
}

__device__ __forceinline__ float bf16_bits_to_f32(uint32_t b16) {
  return __uint_as_float(b16 << 16);
}

// E4M3 byte -> fp32, exact (bias 7, subnormals m * 2^-9; 0x7F is never produced).
__device__ __forceinline__ float e4m3_to_f32(uint32_t s) {
  uint32_t e = (s >> 3) & 15u, m = s & 7u;
  float v = (e == 0) ? __uint2float_rn(m) * 0.001953125f
                     : __uint_as_float(((e + 120u) << 23) | (m << 20));
  return (s & 0x80u) ? -v : v;
}

// fp32 -> E4M3, round to nearest even, saturating finite values to 448
// (hardware conversion; result in the low byte).
__device__ __forceinline__ uint32_t f32_to_e4m3_satfinite(float v) {
  uint16_t out;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(out) : "f"(0.0f), "f"(v));
  return out & 0xFFu;
}

// Four pairs of fp32 -> four bytes of packed E2M1 (element 2i in the low
// nibble of byte i), round to nearest even, saturating at +-6.
__device__ __forceinline__ uint32_t f32x8_to_e2m1x8(const float *v) {
  uint32_t out;
  asm("{\n"
      ".reg .b8 b0, b1, b2, b3;\n"
      "cvt.rn.satfinite.e2m1x2.f32 b0, %2, %1;\n"
      "cvt.rn.satfinite.e2m1x2.f32 b1, %4, %3;\n"
      "cvt.rn.satfinite.e2m1x2.f32 b2, %6, %5;\n"
      "cvt.rn.satfinite.e2m1x2.f32 b3, %8, %7;\n"
      "mov.b32 %0, {b0, b1, b2, b3};\n"
      "}"
      : "=r"(out)
      : "f"(v[0]), "f"(v[1]), "f"(v[2]), "f"(v[3]), "f"(v[4]), "f"(v[5]), "f"(v[6]), "f"(v[7]));
  return out;
}

// E2M1 code (4 bits) -> fp32, exact.
__device__ __forceinline__ float e2m1_to_f32(uint32_t c) {
  // magnitudes 0, .5, 1, 1.5, 2, 3, 4, 6 as bf16-style exponent/mantissa
  const uint32_t mag = c & 7u;
  float v;
  if (mag < 2) v = 0.5f * (float)mag;
  else {
    uint32_t e = (mag >> 1) - 1u;       // 0,1,2 for mags 2..7
    uint32_t m = mag & 1u;              // mantissa bit
    v = __uint_as_float(((127u + e) << 23) | (m << 22));
  }
  return (c & 8u) ? -v : v;
}

// Offset of scale (r, j) in the MMA-tiled layout for a matrix with K/16 = nsf
// scales per row (nsf % 4 == 0).
__device__ __host__ __forceinline__ int64_t sf_tiled_offset(int64_t r, int64_t j, int64_t nsf) {
  return ((r >> 7) * (nsf >> 2) + (j >> 2)) * 512 + (r & 31) * 16 + ((r & 127) >> 5) * 4 + (j & 3);
}

// Block-wide: off[0..G] = group_offsets and slot[0..G] = exclusive prefix sums
// of the 128-aligned group sizes (the slot starts), both in smem.  `scratch`
// holds blockDim.x/32 ints.  blockDim.x must be a multiple of 32.
// Returns false (uniformly over the block, tables not built) unless the
// offsets start at 0, never decrease and end at `total` (exact) or at most at
// `total`: every output row a kernel writes is derived from them.
__device__ inline bool load_groups(const int32_t *__restrict__ group_offsets, int G,
                                   int32_t *off, int32_t *slot, int32_t *scratch, int64_t total, bool exact) {
  for (int i = threadIdx.x; i <= G; i += blockDim.x) off[i] = group_offsets[i];
  __syncthreads();
  bool bad = false;
  for (int i = threadIdx.x; i < G; i += blockDim.x) bad |= off[i + 1] < off[i];
  if (threadIdx.x == 0) bad |= off[0] != 0 || (exact ? (int64_t)off[G] != total : (int64_t)off[G] > total);
  if (__syncthreads_or(bad)) return false;
  const int nt = blockDim.x, t = threadIdx.x;
  const int per = (G + nt - 1) / nt;
  const int g0 = min(G, t * per), g1 = min(G, g0 + per);
  int32_t local = 0;
  for (int g = g0; g < g1; ++g) {
    int32_t c = off[g + 1] - off[g];
    local += (c + kSlotAlign - 1) / kSlotAlign * kSlotAlign;
  }
  // inclusive warp scan of the per-thread sums
  const int lane = t & 31, warp = t >> 5;
  int32_t incl = local;
#pragma unroll
  for (int d = 1; d < 32; d <<= 1) {
    int32_t n = __shfl_up_sync(0xffffffffu, incl, d);
    if (lane >= d) incl += n;
  }
  if (lane == 31) scratch[warp] = incl;
  __syncthreads();
  if (t == 0) {
    int32_t acc = 0;
    for (int w = 0; w < nt / 32; ++w) { int32_t v = scratch[w]; scratch[w] = acc; acc += v; }
  }
  __syncthreads();
  int32_t run = scratch[warp] + incl - local;   // exclusive prefix of this thread
  for (int g = g0; g < g1; ++g) {
    slot[g] = run;
    int32_t c = off[g + 1] - off[g];
    run += (c + kSlotAlign - 1) / kSlotAlign * kSlotAlign;
  }
  if (g1 == G && g0 < g1) slot[G] = run;
  if (G == 0 && t == 0) slot[0] = 0;
  __syncthreads();
  return true;
}

// Largest g in [0, G) with a[g] <= x (a non-decreasing, a[0] <= x).
__device__ __forceinline__ int upper_group(const int32_t *a, int G, int64_t x) {
  int lo = 0, hi = G - 1;
  while (lo < hi) {
    int mid = (lo + hi + 1) >> 1;
    if ((int64_t)a[mid] <= x) lo = mid; else hi = mid - 1;
  }
  return lo;
}

}  // namespace nvfp4
