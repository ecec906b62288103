// MoE plumbing around the expert GEMMs (sm_100a): routing -> expert-grouped
// row order, and the weighted combine of the top-k expert outputs.
//
// The routed experts of the "Qwen3.8-Flash-Next-NVFP4" page take each token to
// its top-10 of 512 experts; the grouped GEMM wants the routed rows of each
// expert contiguous.  nvfp4_moe_route builds that order deterministically
// (tokens ascending inside every expert group) with a counting sort:
//   1. count: one CTA per 256-token chunk, a shared-memory histogram of the
//      chunk's choices -> counts[chunk][expert];
//   2. scan: exclusive prefix sums over chunks (per expert) and over experts
//      -> every chunk's first row in every expert group, and the offsets;
//   3. place: per chunk, one 256-bit mask per expert marks the chunk's tokens
//      that chose it; a token's rank among earlier tokens of the chunk is a
//      popcount, so the placement needs no ordering between threads.
// nvfp4_moe_combine is a streaming kernel (HBM-bound): out[t] = sum_j
// w[t,j] * y[slot[t,j]], accumulated in fp32 in choice order.
#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <stdint.h>

#include "common.cuh"
#include "host_util.cuh"

namespace nvfp4 {
namespace moe {

constexpr int kChunk = 256;          // tokens per route CTA (= threads)
constexpr int kMaxExperts = 2048;    // 2048 experts x 8 mask words x 4 B = 64 KB of smem
constexpr int kMaxTopk = 32;

__global__ void __launch_bounds__(kChunk) route_count_kernel(const int32_t *__restrict__ ids, int64_t T, int k,
                                                             int E, int32_t *__restrict__ counts,
                                                             int32_t *dev_status) {
  extern __shared__ int32_t hist[];
  for (int e = threadIdx.x; e < E; e += kChunk) hist[e] = 0;
  __syncthreads();
  const int64_t t = (int64_t)blockIdx.x * kChunk + threadIdx.x;
  if (t < T) {
    for (int j = 0; j < k; ++j) {
      const int e = ids[t * k + j];
      if (e < 0 || e >= E) { report(dev_status, NVFP4_ERR_INDEX); continue; }
      atomicAdd(&hist[e], 1);
    }
  }
  __syncthreads();
  for (int e = threadIdx.x; e < E; e += kChunk) counts[(int64_t)blockIdx.x * E + e] = hist[e];
}

// One CTA: counts[c][e] -> first row of chunk c in group e (in place) and
// offsets[E+1].
__global__ void __launch_bounds__(1024) route_scan_kernel(int32_t *__restrict__ counts, int64_t n_chunks, int E,
                                                          int32_t *__restrict__ offsets) {
  __shared__ int32_t warp_sums[32];
  __shared__ int32_t carry;
  if (threadIdx.x == 0) carry = 0;
  __syncthreads();
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  for (int e0 = 0; e0 < E; e0 += 1024) {
    const int e = e0 + threadIdx.x;
    int32_t total = 0;
    if (e < E) {
      for (int64_t c = 0; c < n_chunks; ++c) {
        const int32_t v = counts[c * E + e];
        counts[c * E + e] = total;          // exclusive within the expert, fixed up below
        total += v;
      }
    }
    // exclusive scan of the expert totals across the block (plus the carry of earlier passes)
    int32_t incl = total;
#pragma unroll
    for (int d = 1; d < 32; d <<= 1) {
      const int32_t n = __shfl_up_sync(0xffffffffu, incl, d);
      if (lane >= d) incl += n;
    }
    if (lane == 31) warp_sums[warp] = incl;
    __syncthreads();
    if (threadIdx.x == 0) {
      int32_t acc = carry;
      for (int w = 0; w < 32; ++w) { const int32_t v = warp_sums[w]; warp_sums[w] = acc; acc += v; }
      carry = acc;
    }
    __syncthreads();
    const int32_t base = warp_sums[warp] + incl - total;
    if (e < E) {
      offsets[e] = base;
      for (int64_t c = 0; c < n_chunks; ++c) counts[c * E + e] += base;
    }
    __syncthreads();
  }
  if (threadIdx.x == 0) offsets[E] = carry;
}

__global__ void __launch_bounds__(kChunk) route_place_kernel(const int32_t *__restrict__ ids, int64_t T, int k,
                                                             int E, const int32_t *__restrict__ chunk_base,
                                                             int32_t *__restrict__ row_index,
                                                             int32_t *__restrict__ slot) {
  extern __shared__ uint32_t masks[];       // [E][8]: bit t%32 of word t/32 = token t of the chunk chose e
  for (int i = threadIdx.x; i < E * 8; i += kChunk) masks[i] = 0;
  __syncthreads();
  const int64_t t = (int64_t)blockIdx.x * kChunk + threadIdx.x;
  const int w = threadIdx.x >> 5;
  const uint32_t bit = 1u << (threadIdx.x & 31);
  if (t < T) {
    for (int j = 0; j < k; ++j) {
      const int e = ids[t * k + j];
      if (e >= 0 && e < E) atomicOr(&masks[e * 8 + w], bit);
    }
  }
  __syncthreads();
  if (t < T) {
    for (int j = 0; j < k; ++j) {
      const int e = ids[t * k + j];
      if (e < 0 || e >= E) { slot[t * k + j] = -1; continue; }
      int rank = __popc(masks[e * 8 + w] & (bit - 1u));
      for (int ww = 0; ww < w; ++ww) rank += __popc(masks[e * 8 + ww]);
      const int32_t row = chunk_base[(int64_t)blockIdx.x * E + e] + rank;
      row_index[row] = (int32_t)t;
      slot[t * k + j] = row;
    }
  }
}

__device__ __forceinline__ void load8(const void *y, bool bf16, int64_t idx, float (&v)[8]) {
  if (bf16) {
    const uint4 u = __ldg(reinterpret_cast<const uint4 *>(reinterpret_cast<const uint16_t *>(y) + idx));
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      v[2 * i] = __uint_as_float(w[i] << 16);
      v[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
    }
  } else {
    const float4 *p = reinterpret_cast<const float4 *>(reinterpret_cast<const float *>(y) + idx);
    const float4 a = __ldg(p), b = __ldg(p + 1);
    v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w; v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
  }
}

// One thread per (token, 8 columns): k loads of 16/32 bytes in flight.
template <bool kBf16In, bool kBf16Out>
__global__ void __launch_bounds__(256) combine_kernel(const void *__restrict__ y, int64_t rows,
                                                      const int32_t *__restrict__ slot,
                                                      const float *__restrict__ w, int64_t T, int k, int64_t H,
                                                      void *__restrict__ out, int32_t *dev_status) {
  const int64_t ncg = H >> 3;
  const int64_t total = T * ncg;
  const int64_t stride = (int64_t)gridDim.x * blockDim.x;
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < total; i += stride) {
    const int64_t t = i / ncg, c = (i - t * ncg) * 8;
    float acc[8] = {0, 0, 0, 0, 0, 0, 0, 0};
    for (int j = 0; j < k; ++j) {
      const int32_t r = __ldg(slot + t * k + j);
      if (r < 0) continue;
      if (r >= rows) {                      // never read past y: skip and report
        if (c == 0) report(dev_status, NVFP4_ERR_INDEX);
        continue;
      }
      const float wj = __ldg(w + t * k + j);
      float v[8];
      load8(y, kBf16In, (int64_t)r * H + c, v);
#pragma unroll
      for (int q = 0; q < 8; ++q) acc[q] = fmaf(wj, v[q], acc[q]);
    }
    if (kBf16Out) {
      uint32_t hw[4];
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        __nv_bfloat162 b2 = __floats2bfloat162_rn(acc[2 * q], acc[2 * q + 1]);
        hw[q] = *reinterpret_cast<uint32_t *>(&b2);
      }
      *reinterpret_cast<uint4 *>(reinterpret_cast<uint16_t *>(out) + t * H + c) = make_uint4(hw[0], hw[1], hw[2], hw[3]);
    } else {
      float4 *o = reinterpret_cast<float4 *>(reinterpret_cast<float *>(out) + t * H + c);
      o[0] = make_float4(acc[0], acc[1], acc[2], acc[3]);
      o[1] = make_float4(acc[4], acc[5], acc[6], acc[7]);
    }
  }
}

}  // namespace moe
}  // namespace nvfp4

using namespace nvfp4;

extern "C" size_t nvfp4_moe_route_workspace_size(int64_t tokens, int num_experts) {
  if (tokens < 0) tokens = 0;
  if (num_experts < 1) num_experts = 1;
  const int64_t n_chunks = (tokens + moe::kChunk - 1) / moe::kChunk;
  size_t bytes = sizeof(int32_t) * (size_t)(n_chunks > 0 ? n_chunks : 1) * (size_t)num_experts;
  return (bytes + 255) / 256 * 256;
}

extern "C" nvfp4_status nvfp4_moe_route(const int32_t *topk_ids, int64_t tokens, int topk, int num_experts,
                                        int32_t *expert_offsets, int32_t *row_index, int32_t *slot,
                                        void *workspace, int32_t *dev_status, cudaStream_t stream) {
  if (tokens < 0 || topk < 1 || topk > moe::kMaxTopk) return NVFP4_ERR_INVALID_ARG;
  if (num_experts < 1 || num_experts > moe::kMaxExperts) return NVFP4_ERR_UNSUPPORTED_SHAPE;
  if (tokens * topk > ((int64_t)1 << 31) - 1) return NVFP4_ERR_UNSUPPORTED_SHAPE;
  if (!expert_offsets || !workspace) return NVFP4_ERR_INVALID_ARG;
  if (tokens > 0 && (!topk_ids || !row_index || !slot)) return NVFP4_ERR_INVALID_ARG;
  int32_t *counts = reinterpret_cast<int32_t *>(workspace);
  const int64_t n_chunks = (tokens + moe::kChunk - 1) / moe::kChunk;
  if (n_chunks > 0) {
    moe::route_count_kernel<<<(unsigned)n_chunks, moe::kChunk, sizeof(int32_t) * num_experts, stream>>>(
        topk_ids, tokens, topk, num_experts, counts, dev_status);
    if (cudaGetLastError() != cudaSuccess) return NVFP4_ERR_CUDA;
  }
  moe::route_scan_kernel<<<1, 1024, 0, stream>>>(counts, n_chunks, num_experts, expert_offsets);
  if (cudaGetLastError() != cudaSuccess) return NVFP4_ERR_CUDA;
  if (n_chunks > 0) {
    const size_t sm = sizeof(uint32_t) * 8 * (size_t)num_experts;
    if (sm > 48 * 1024 &&
        !host::set_max_dynamic_smem(reinterpret_cast<const void *>(moe::route_place_kernel), (int)sm))
      return NVFP4_ERR_CUDA;
    moe::route_place_kernel<<<(unsigned)n_chunks, moe::kChunk, sm, stream>>>(topk_ids, tokens, topk, num_experts,
                                                                              counts, row_index, slot);
    if (cudaGetLastError() != cudaSuccess) return NVFP4_ERR_CUDA;
  }
  return NVFP4_OK;
}

extern "C" nvfp4_status nvfp4_moe_combine(const void *y, nvfp4_out_dtype y_dtype, int64_t rows, const int32_t *slot,
                                          const float *weights, int64_t tokens, int topk, int64_t H, void *out,
                                          nvfp4_out_dtype out_dtype, int32_t *dev_status, cudaStream_t stream) {
  if (tokens < 0 || rows < 0 || topk < 1 || topk > moe::kMaxTopk || H <= 0) return NVFP4_ERR_INVALID_ARG;
  if (H % 8 != 0) return NVFP4_ERR_UNSUPPORTED_SHAPE;
  if ((y_dtype != NVFP4_OUT_F32 && y_dtype != NVFP4_OUT_BF16) ||
      (out_dtype != NVFP4_OUT_F32 && out_dtype != NVFP4_OUT_BF16))
    return NVFP4_ERR_INVALID_ARG;
  if (tokens == 0) return NVFP4_OK;
  if ((rows > 0 && !y) || !slot || !weights || !out) return NVFP4_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(y) | reinterpret_cast<uintptr_t>(out)) & 15u) return NVFP4_ERR_INVALID_ARG;
  const int sms = host::sm_count();
  const int64_t work = tokens * (H / 8);
  int64_t blocks = (work + 255) / 256;
  if (blocks > (int64_t)sms * 8) blocks = (int64_t)sms * 8;
  const bool bi = y_dtype == NVFP4_OUT_BF16, bo = out_dtype == NVFP4_OUT_BF16;
#define NVFP4_CB(A, B) moe::combine_kernel<A, B><<<(unsigned)blocks, 256, 0, stream>>>(y, rows, slot, weights, tokens, topk, H, out, dev_status)
  if (bi && bo) NVFP4_CB(true, true);
  else if (bi) NVFP4_CB(true, false);
  else if (bo) NVFP4_CB(false, true);
  else NVFP4_CB(false, false);
#undef NVFP4_CB
  return cudaGetLastError() == cudaSuccess ? NVFP4_OK : NVFP4_ERR_CUDA;
}
