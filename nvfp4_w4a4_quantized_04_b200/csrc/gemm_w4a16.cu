// Weight-only NVFP4 grouped GEMM, bf16 activations (W4A16), sm_100a.
//
// The "DeepSeek-V4.1-Flash-NVFP4" page lists the MTP layer's experts as
// W4A16_NVFP4: the weights are NVFP4 (E2M1 codes, E4M3 scale per 16, FP32
// global) and the activations stay bf16.  For every routed expert e:
//   Y_e = X_e (s_g[e] * W_e)^T,   W_e[n, k] = e2m1(code) * e4m3(S[n, k/16]),
// accumulated in fp32.  With the SwiGLU epilogue the weight is a fused gate_up
// [2I, K] (gate rows 0..I-1, up rows I..2I-1) and the output is
// h = bf16(silu(g) * u).
//
// Built for decode-sized expert groups (a few tokens per expert), where the
// weight bytes dominate: a warp owns 32 weight rows x 8 tokens and runs
// mma.sync m16n8k16 (bf16 in, fp32 accumulate) over K, every weight byte read
// once per 8 tokens.  The 16-element K slices of the instruction are mapped to
// memory so that each lane's A elements are 16 consecutive codes of a row (one
// 8-byte load, one E4M3 scale) and its B elements 16 consecutive bf16 of a
// token; the same permutation on both sides leaves the dot products unchanged.
// E2M1 -> bf16 and the product with the scale in bf16 are exact (at most 6
// significant bits); s_g multiplies the accumulated sum once.
#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <stdint.h>

#include "common.cuh"

namespace nvfp4 {
namespace w4a16 {

constexpr int kTokChunk = 8;       // tokens per warp tile (MMA N)
constexpr int kRows = 32;          // weight rows per warp: two MMA tiles of 16 sharing the B fragment
constexpr int kThreads = 256;

// Two E2M1 codes (one byte, element 2i in the low nibble) times a bf16x2 scale
// -> one bf16x2 register (low half = even element), exact.
__device__ __forceinline__ uint32_t e2m1x2_bf16x2(uint32_t byte, uint32_t s2) {
  uint32_t h, r;
  asm("{\n.reg .b8 b;\n.reg .f16 l, u;\n.reg .f32 fl, fu;\ncvt.u8.u32 b, %1;\ncvt.rn.f16x2.e2m1x2 %0, b;\n}"
      : "=r"(h) : "r"(byte));
  asm("{\n.reg .f16 l, u;\n.reg .f32 fl, fu;\nmov.b32 {l, u}, %1;\ncvt.f32.f16 fl, l;\ncvt.f32.f16 fu, u;\n"
      "cvt.rn.bf16x2.f32 %0, fu, fl;\n}" : "=r"(r) : "r"(h));
  asm("mul.rn.bf16x2 %0, %0, %1;" : "+r"(r) : "r"(s2));
  return r;
}

// E4M3 byte -> bf16 in both halves (exact: every E4M3 value is a bf16).
__device__ __forceinline__ uint32_t e4m3_bf16x2(uint32_t s) {
  uint32_t h, r;
  asm("{\n.reg .b16 b;\ncvt.u16.u32 b, %1;\ncvt.rn.f16x2.e4m3x2 %0, b;\n}" : "=r"(h) : "r"(s & 0xFFu));
  asm("{\n.reg .f16 l, u;\n.reg .f32 fl;\nmov.b32 {l, u}, %1;\ncvt.f32.f16 fl, l;\ncvt.rn.bf16x2.f32 %0, fl, fl;\n}"
      : "=r"(r) : "r"(h));
  return r;
}

__device__ __forceinline__ void mma_bf16(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                         uint32_t b0, uint32_t b1) {
  asm volatile("mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
               "{%0,%1,%2,%3};"
               : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
               : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// One 64-element K chunk of a 16-row weight tile against the B fragment:
// lane (g = lane/4, t = lane%4) holds codes 16t..16t+15 of the chunk for rows
// g and g+8 (wlo, whi) with their scales (slo, shi).
__device__ __forceinline__ void chunk_mma(float (&d)[4], uint2 wlo, uint2 whi, uint32_t slo, uint32_t shi,
                                          const uint32_t (&b)[8]) {
  const uint32_t s_lo = e4m3_bf16x2(slo), s_hi = e4m3_bf16x2(shi);
  const uint32_t lo[2] = {wlo.x, wlo.y}, hi[2] = {whi.x, whi.y};
#pragma unroll
  for (int s = 0; s < 4; ++s) {
    // k-step s: elements 4s..4s+3 of the lane's 16 = bytes 2s, 2s+1
    const uint32_t wl = lo[s >> 1] >> (16 * (s & 1)), wh = hi[s >> 1] >> (16 * (s & 1));
    mma_bf16(d, e2m1x2_bf16x2(wl & 0xFFu, s_lo), e2m1x2_bf16x2(wh & 0xFFu, s_hi),
             e2m1x2_bf16x2((wl >> 8) & 0xFFu, s_lo), e2m1x2_bf16x2((wh >> 8) & 0xFFu, s_hi), b[2 * s], b[2 * s + 1]);
  }
}

// Work item = (expert, 16-row block (gate rows with SwiGLU), 8-token chunk).
template <bool kSwiglu, bool kBf16Out>
__global__ void __launch_bounds__(kThreads) w4a16_kernel(
    const uint16_t *__restrict__ x, int64_t ld_x, int64_t x_rows, const int32_t *__restrict__ row_index,
    const uint8_t *__restrict__ wq, const uint8_t *__restrict__ wsf, const float *__restrict__ w_gs,
    const int32_t *__restrict__ expert_offsets, int E, int64_t M_total, int N, int K, void *__restrict__ y,
    int32_t *dev_status) {
  extern __shared__ int32_t smem[];
  int32_t *off = smem, *items = smem + (E + 1);       // items[e] = first work item of expert e
  const int rows_out = kSwiglu ? N / 2 : N;
  const int row_blocks = rows_out / kRows;
  __shared__ int32_t scratch[kThreads / 32];
  for (int i = threadIdx.x; i <= E; i += blockDim.x)
    off[i] = expert_offsets ? expert_offsets[i] : (i == 0 ? 0 : (int32_t)M_total);
  __syncthreads();
  {
    // items[e] = exclusive prefix sum of row_blocks * chunks(e): block-wide scan
    const int per = (E + kThreads - 1) / kThreads;
    const int e0 = min(E, (int)threadIdx.x * per), e1 = min(E, e0 + per);
    int32_t local = 0;
    for (int e = e0; e < e1; ++e) local += row_blocks * ((off[e + 1] - off[e] + kTokChunk - 1) / kTokChunk);
    const int ln = threadIdx.x & 31, wp = threadIdx.x >> 5;
    int32_t incl = local;
#pragma unroll
    for (int dd = 1; dd < 32; dd <<= 1) {
      const int32_t v = __shfl_up_sync(0xffffffffu, incl, dd);
      if (ln >= dd) incl += v;
    }
    if (ln == 31) scratch[wp] = incl;
    __syncthreads();
    if (threadIdx.x == 0) {
      int32_t a = 0;
      for (int w = 0; w < kThreads / 32; ++w) { const int32_t v = scratch[w]; scratch[w] = a; a += v; }
    }
    __syncthreads();
    int32_t run = scratch[wp] + incl - local;
    for (int e = e0; e < e1; ++e) {
      items[e] = run;
      run += row_blocks * ((off[e + 1] - off[e] + kTokChunk - 1) / kTokChunk);
    }
    if (e1 == E && e0 < e1) items[E] = run;
  }
  __syncthreads();
  const int lane = threadIdx.x & 31, g = lane >> 2, t = lane & 3;
  const int64_t warp = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int64_t nwarps = ((int64_t)gridDim.x * blockDim.x) >> 5;
  const int64_t total = items[E];
  const int64_t row_bytes = K / 2, sf_bytes = K / 16;
  const int nchunks = K / 64;
  bool bad_index = false;
  for (int64_t it = warp; it < total; it += nwarps) {
    const int e = upper_group(items, E, it);
    const int64_t local = it - items[e];
    const int rb = (int)(local % row_blocks);
    const int chunk = (int)(local / row_blocks);
    const int32_t r0 = off[e] + chunk * kTokChunk;
    const int ntok = min(kTokChunk, off[e + 1] - r0);
    // B rows: token g of the chunk (a missing token reads a valid row; its column is not stored)
    int64_t src = r0 + min(g, ntok - 1);
    if (row_index) {
      src = row_index[src];
      if (src < 0 || src >= x_rows) { src = 0; bad_index = true; }
    }
    const uint16_t *xr = x + src * ld_x + 16 * t;
    const int64_t n0 = (int64_t)e * N + (int64_t)rb * kRows;
    // lane rows g, g+8 (tile 0) and g+16, g+24 (tile 1); with SwiGLU the
    // matching up rows N/2 further
    const uint8_t *qrow = wq + (n0 + g) * row_bytes + 8 * t;
    const uint8_t *frow = wsf + (n0 + g) * sf_bytes + t;
    const int64_t up = (int64_t)(N / 2) * row_bytes, upf = (int64_t)(N / 2) * sf_bytes;
    constexpr int NW = kSwiglu ? 8 : 4;               // weight rows per lane
    float d[NW / 2][4] = {};
    auto load = [&](int c, uint4 &x0, uint4 &x1, uint2 (&w)[NW], uint32_t (&sc)[NW]) {
      x0 = __ldg(reinterpret_cast<const uint4 *>(xr + 64 * c));
      x1 = __ldg(reinterpret_cast<const uint4 *>(xr + 64 * c + 8));
#pragma unroll
      for (int i = 0; i < NW; ++i) {
        const int64_t ro = (int64_t)(i & 3) * 8;           // rows g, g+8, g+16, g+24
        const int64_t qo = ro * row_bytes + (i >= 4 ? up : 0), fo = ro * sf_bytes + (i >= 4 ? upf : 0);
        w[i] = __ldg(reinterpret_cast<const uint2 *>(qrow + qo + 32 * c));
        sc[i] = __ldg(frow + fo + 4 * c);
      }
    };
    uint4 x0, x1;
    uint2 w[NW];
    uint32_t sc[NW];
    load(0, x0, x1, w, sc);
    for (int c = 0; c < nchunks; ++c) {
      uint4 nx0 = x0, nx1 = x1;
      uint2 nw[NW];
      uint32_t nsc[NW];
#pragma unroll
      for (int i = 0; i < NW; ++i) { nw[i] = w[i]; nsc[i] = sc[i]; }
      if (c + 1 < nchunks) load(c + 1, nx0, nx1, nw, nsc);     // next chunk in flight during this one
      const uint32_t b[8] = {x0.x, x0.y, x0.z, x0.w, x1.x, x1.y, x1.z, x1.w};
#pragma unroll
      for (int m = 0; m < NW / 2; ++m) chunk_mma(d[m], w[2 * m], w[2 * m + 1], sc[2 * m], sc[2 * m + 1], b);
      x0 = nx0; x1 = nx1;
#pragma unroll
      for (int i = 0; i < NW; ++i) { w[i] = nw[i]; sc[i] = nsc[i]; }
    }
    // tile m (0, 1): d[m][0..1] row 16m+g, d[m][2..3] row 16m+g+8, tokens 2t, 2t+1;
    // with SwiGLU d[2+m] holds the matching up rows
    const float gs = w_gs[e];
#pragma unroll
    for (int m = 0; m < 2; ++m) {
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int tok = 2 * t + (i & 1);
        const int row = rb * kRows + 16 * m + g + 8 * (i >> 1);
        if (tok < ntok) {
          const float gv = __fmul_rn(d[m][i], gs);
          float v = gv;
          if constexpr (kSwiglu) v = __fmul_rn(__fdividef(gv, 1.0f + __expf(-gv)), __fmul_rn(d[2 + m][i], gs));
          const int64_t o = (int64_t)(r0 + tok) * rows_out + row;
          if (kBf16Out) reinterpret_cast<__nv_bfloat16 *>(y)[o] = __float2bfloat16_rn(v);
          else reinterpret_cast<float *>(y)[o] = v;
        }
      }
    }
  }
  if (bad_index) report(dev_status, NVFP4_ERR_INDEX);
}

}  // namespace w4a16
}  // namespace nvfp4

using namespace nvfp4;

extern "C" nvfp4_status nvfp4_grouped_gemm_w4a16(const void *x, int64_t ld_x, int64_t x_rows, const int32_t *row_index,
                                                 const uint8_t *b_q, const uint8_t *b_sf, const float *b_gs,
                                                 const int32_t *expert_offsets, int num_experts, int64_t M_total,
                                                 int64_t N, int64_t K, void *y, nvfp4_out_dtype out_dtype,
                                                 nvfp4_epilogue epi, int32_t *dev_status, cudaStream_t stream) {
  if (epi != NVFP4_EPI_NONE && epi != NVFP4_EPI_SWIGLU) return NVFP4_ERR_INVALID_ARG;
  if (out_dtype != NVFP4_OUT_F32 && out_dtype != NVFP4_OUT_BF16) return NVFP4_ERR_INVALID_ARG;
  const bool swiglu = epi == NVFP4_EPI_SWIGLU;
  const int E = expert_offsets ? num_experts : 1;
  if (E < 1 || E > kMaxGroups) return NVFP4_ERR_UNSUPPORTED_SHAPE;
  if (M_total < 0 || N <= 0 || K <= 0 || ld_x < K || x_rows < 0) return NVFP4_ERR_INVALID_ARG;
  if (!row_index && x_rows < M_total) return NVFP4_ERR_INVALID_ARG;
  if (K % 64 != 0 || ld_x % 8 != 0 || N % (swiglu ? 64 : 32) != 0) return NVFP4_ERR_UNSUPPORTED_SHAPE;
  if ((int64_t)E * N > ((int64_t)1 << 31) - 1 || M_total > ((int64_t)1 << 31) - 1 || N > (1 << 30))
    return NVFP4_ERR_UNSUPPORTED_SHAPE;
  if (M_total == 0) return NVFP4_OK;
  if (!x || x_rows == 0 || !b_q || !b_sf || !b_gs || !y) return NVFP4_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(x) | reinterpret_cast<uintptr_t>(b_q)) & 15u) return NVFP4_ERR_INVALID_ARG;
  if (reinterpret_cast<uintptr_t>(b_sf) & 1u) return NVFP4_ERR_INVALID_ARG;
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const size_t sm = sizeof(int32_t) * 2 * (size_t)(E + 1);
  const int blocks = sms * 8;
  const uint16_t *xb = reinterpret_cast<const uint16_t *>(x);
#define NVFP4_W4(S, B)                                                                                      \
  w4a16::w4a16_kernel<S, B><<<blocks, w4a16::kThreads, sm, stream>>>(xb, ld_x, x_rows, row_index, b_q, b_sf, b_gs, \
                                                                     expert_offsets, E, M_total, (int)N, (int)K, y, \
                                                                     dev_status)
  if (sm > 48 * 1024) return NVFP4_ERR_UNSUPPORTED_SHAPE;
  const bool bo = out_dtype == NVFP4_OUT_BF16;
  if (swiglu && bo) NVFP4_W4(true, true);
  else if (swiglu) NVFP4_W4(true, false);
  else if (bo) NVFP4_W4(false, true);
  else NVFP4_W4(false, false);
#undef NVFP4_W4
  return cudaGetLastError() == cudaSuccess ? NVFP4_OK : NVFP4_ERR_CUDA;
}
