// Weight-only NVFP4 grouped GEMM with 16-bit activations (W4A16), sm_100a:
// the warp-MMA kernel for small groups (the decode regime).
//
// The "DeepSeek-V4.1-Flash-NVFP4" page lists the MTP layer's experts as
// W4A16_NVFP4: the weights are NVFP4 (E2M1 codes, E4M3 scale per 16, FP32
// global) and the activations stay 16-bit.  For every routed expert e:
//   Y_e = X_e (s_g[e] * W_e)^T,   W_e[n, k] = e2m1(code) * e4m3(S[n, k/16]),
// accumulated in fp32.  With the SwiGLU epilogue the weight is a fused gate_up
// [2I, K] (gate rows 0..I-1, up rows I..2I-1) and the output is
// h = silu(g) * u.
//
// Built for decode-sized expert groups (a few tokens per expert), where the
// weight bytes dominate and the kernel must stream them at HBM rate.  Here the
// contraction runs as mma.sync: a tcgen05 MMA with N = 16 tokens and K = 16
// f16 elements costs about 108 cycles per instruction (measured), which caps a
// tensor-memory kernel at about 2.7 TB/s of weights when groups hold 1-3
// tokens, while this kernel, bound by the E2M1 -> f16 conversions, streams
// about 4 TB/s.  Larger groups go to the tcgen05 kernel (gemm_w4a16.cu).
//  * Tensor-core operands in f16.  E2M1 -> f16 is one hardware conversion per
//    two codes, and e2m1 * e4m3 is exact in f16 (at most 6 significant bits,
//    |.| in [2^-10, 2688]), so each weight element costs one conversion and
//    one f16x2 multiply per pair.  The bf16 activations are converted once per
//    call by a prep kernel: each routed row is scaled by a power of two 2^-k
//    that puts its max |x| in [2^14, 2^15), then rounded to f16.  Every
//    element within 2^29 of the row's max is exact; smaller ones land on f16's
//    subnormal grid (error below 2^-25 of the row max).  The epilogue
//    multiplies by 2^k again, which is exact.
//  * Pipeline.  One producer warp streams, per 256-element K stage, the
//    128-row weight tile and its scales by TMA (128-byte swizzle) and the
//    item's activation rows (4 KB per 8 tokens, pre-arranged by the prep
//    kernel in fragment order) by bulk copies, into a 7-stage ring of 26 KB
//    stages.
//    Sixteen consumer warps run mma.sync m16n8k16 (f16 in, fp32 accumulate):
//    warp w owns weight rows 16 (w%8) .. +16 (x 8 tokens) and the K half w/8
//    of every stage; the two halves are added through shared memory at the
//    end of the item.  Two warps per row tile hide the latency of the
//    conversion -> multiply -> MMA chain.
//  * K permutation.  Within a stage, lane t of a quad holds K range
//    [64t, 64t+64) of its rows: MMA slice s takes physical K 64t + 4s + {0..3},
//    the same on both operands, which leaves the dot products unchanged and
//    gives each lane two 16-byte weight loads and one scale word per row.
//  * Work item = (expert, 128-row weight block, up to two 8-token chunks):
//    the converted weight fragments feed one MMA per chunk.  An expert with
//    more than 16 tokens re-reads its weight block per item, and those reads
//    follow each other so they hit L2.
//  * Every mbarrier wait is bounded (NVFP4_ERR_TIMEOUT, then all roles leave).
#include "gemm_common.cuh"
#include "host_util.cuh"

#include <cuda_fp16.h>

#include <type_traits>

namespace nvfp4 {
namespace w4a16_mma {

using gemm::kWaitBudgetCycles;
using gemm::mbar_arrive;
using gemm::mbar_arrive_expect_tx;
using gemm::mbar_init;
using gemm::mbar_try_wait;
using gemm::mbar_wait;
using gemm::smem_u32;

constexpr int kTok = 8;                      // tokens per chunk (MMA N)
constexpr int kChunks = 2;                   // chunks per item: both share one weight conversion
constexpr int kConsumers = 16;               // consumer warps: 8 row tiles x 2 K halves
constexpr int kThreads = (kConsumers + 1) * 32;
constexpr int kStages = 7;
constexpr int kWBytes = 128 * 128;           // 128 rows x 256 codes
constexpr int kSBytes = 128 * 16;            // 128 rows x 16 scales
constexpr int kXChunk = kTok * 256 * 2;      // 8 tokens x 256 f16
constexpr int kStageBytes = kWBytes + kSBytes + kChunks * kXChunk;
constexpr int OFF_BAR = kStages * kStageBytes;
constexpr int OFF_MISC = OFF_BAR + 2 * kStages * 8;
constexpr int OFF_RED = OFF_MISC + 16;       // K-half partial sums: 8 warps x 32 lanes x 8 floats
constexpr int OFF_TABLES = OFF_RED + 8 * 32 * 32;
constexpr int kMaxExperts = 1024;
constexpr int TABLE_BYTES = 3 * (kMaxExperts + 1) * 4 + 32 * 4;
constexpr int SMEM_BYTES = OFF_TABLES + TABLE_BYTES + 1024;
static_assert(SMEM_BYTES <= 232448, "shared memory budget");

// Block-wide exclusive prefix sums over e < E of f(e), into out[0..E].
template <typename F>
__device__ void block_prefix(int E, int32_t *out, int32_t *scratch, F f) {
  const int nt = blockDim.x, t = threadIdx.x, lane = t & 31, warp = t >> 5;
  const int per = (E + nt - 1) / nt;
  const int e0 = min(E, t * per), e1 = min(E, e0 + per);
  int32_t local = 0;
  for (int e = e0; e < e1; ++e) local += f(e);
  int32_t incl = local;
#pragma unroll
  for (int d = 1; d < 32; d <<= 1) {
    const int32_t v = __shfl_up_sync(0xffffffffu, incl, d);
    if (lane >= d) incl += v;
  }
  if (lane == 31) scratch[warp] = incl;
  __syncthreads();
  if (t == 0) {
    int32_t a = 0;
    for (int w = 0; w < nt / 32; ++w) { const int32_t v = scratch[w]; scratch[w] = a; a += v; }
  }
  __syncthreads();
  int32_t run = scratch[warp] + incl - local;
  for (int e = e0; e < e1; ++e) { out[e] = run; run += f(e); }
  if (e1 == E && e0 < e1) out[E] = run;
  if (E == 0 && t == 0) out[0] = 0;
  __syncthreads();
}

// ------------------------------------------------------------------ prep
// Activation layout in the workspace: the tokens of expert e form
// ceil(n_e/8) chunks of 8 rows, chunk index C = cslot[e] + c.  For chunk C and
// K stage st the 4 KB block at ((C * nst + st) * 2048) halves holds, at
// 16-byte piece (i * 32 + L), token g = L/4 at K = 256 st + 64 (L%4) + 8 i ..
// +8: lane L of a consumer warp reads its pieces i = 0..7 with conflict-free
// 16-byte shared loads.  xscale[C * 8 + g] = 2^k of that token.
__global__ void __launch_bounds__(256) w4a16_prep_kernel(
    const uint16_t *__restrict__ x, int64_t ld_x, int64_t x_rows, const int32_t *__restrict__ row_index,
    const int32_t *__restrict__ offsets, int E, int64_t M_total, int K, uint16_t *__restrict__ x16,
    float *__restrict__ xscale, int32_t *dev_status) {
  extern __shared__ int32_t smem[];
  int32_t *off = smem, *cslot = smem + (E + 1), *scratch = smem + 2 * (E + 1);
  for (int i = threadIdx.x; i <= E; i += blockDim.x)
    off[i] = offsets ? offsets[i] : (i == 0 ? 0 : (int32_t)M_total);
  __syncthreads();
  block_prefix(E, cslot, scratch, [&](int e) { return (off[e + 1] - off[e] + kTok - 1) / kTok; });
  const int lane = threadIdx.x & 31;
  const int nst = K / 256;
  const int64_t nwarps = ((int64_t)gridDim.x * blockDim.x) >> 5;
  bool bad_index = false, bad_value = false;
  for (int64_t r = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5; r < M_total; r += nwarps) {
    const int e = upper_group(off, E, r);
    const int i = (int)(r - off[e]);
    const int64_t C = cslot[e] + i / kTok;
    const int g = i % kTok;
    int64_t src = row_index ? (int64_t)row_index[r] : r;
    if (src < 0 || src >= x_rows) { src = 0; bad_index = true; }
    const uint16_t *xr = x + src * ld_x;
    uint32_t m = 0;
    for (int k = lane * 8; k < K; k += 256) {
      const uint4 v = __ldg(reinterpret_cast<const uint4 *>(xr + k));
      m = __vmaxu2(m, v.x & 0x7FFF7FFFu);
      m = __vmaxu2(m, v.y & 0x7FFF7FFFu);
      m = __vmaxu2(m, v.z & 0x7FFF7FFFu);
      m = __vmaxu2(m, v.w & 0x7FFF7FFFu);
    }
    m = max(m & 0xFFFFu, m >> 16);
#pragma unroll
    for (int d = 16; d > 0; d >>= 1) m = max(m, __shfl_xor_sync(0xffffffffu, m, d));
    if (m >= 0x7F80u) bad_value = true;
    // k = floor(log2 max) - 14, kept where 2^k and 2^-k are fp32 normals
    int k = (m == 0 || m >= 0x7F80u) ? 0 : (int)(m >> 7) - 127 - 14;
    k = max(-126, min(k, 113));
    const float sc = __uint_as_float((uint32_t)(127 - k) << 23);
    if (lane == 0) xscale[C * kTok + g] = __uint_as_float((uint32_t)(127 + k) << 23);
    uint16_t *dst = x16 + C * (int64_t)nst * 2048;
    for (int p = lane; p < K / 8; p += 32) {
      const int st = p >> 5, rest = p & 31, t = rest >> 3, i8 = rest & 7;
      const int kk = st * 256 + 64 * t + 8 * i8;
      const uint4 v = __ldg(reinterpret_cast<const uint4 *>(xr + kk));
      const uint32_t w[4] = {v.x, v.y, v.z, v.w};
      uint32_t o[4];
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const float lo = __fmul_rn(__uint_as_float(w[j] << 16), sc);
        const float hi = __fmul_rn(__uint_as_float(w[j] & 0xFFFF0000u), sc);
        const __half2 h = __floats2half2_rn(lo, hi);
        o[j] = *reinterpret_cast<const uint32_t *>(&h);
      }
      *reinterpret_cast<uint4 *>(dst + (int64_t)st * 2048 + (i8 * 32 + g * 4 + t) * 8) =
          make_uint4(o[0], o[1], o[2], o[3]);
    }
  }
  if (bad_index) report(dev_status, NVFP4_ERR_INDEX);
  if (bad_value) report(dev_status, NVFP4_ERR_NONFINITE);
}

// ------------------------------------------------------------------ GEMM
// Two E4M3 bytes (low 16 bits) -> f16x2 (low half = low byte), exact.
__device__ __forceinline__ uint32_t e4m3x2_f16x2(uint32_t two) {
  uint32_t h;
  asm("{\n.reg .b16 b;\ncvt.u16.u32 b, %1;\ncvt.rn.f16x2.e4m3x2 %0, b;\n}" : "=r"(h) : "r"(two & 0xFFFFu));
  return h;
}

// The four bytes of a word (8 codes) -> four f16x2 (byte j -> o[j]), exact.
__device__ __forceinline__ void e2m1x8_f16x2(uint32_t w, uint32_t (&o)[4]) {
  asm("{\n.reg .b8 b0, b1, b2, b3;\nmov.b32 {b0, b1, b2, b3}, %4;\n"
      "cvt.rn.f16x2.e2m1x2 %0, b0;\ncvt.rn.f16x2.e2m1x2 %1, b1;\n"
      "cvt.rn.f16x2.e2m1x2 %2, b2;\ncvt.rn.f16x2.e2m1x2 %3, b3;\n}"
      : "=r"(o[0]), "=r"(o[1]), "=r"(o[2]), "=r"(o[3]) : "r"(w));
}

__device__ __forceinline__ uint32_t hmul2(uint32_t a, uint32_t b) {
  uint32_t d;
  asm("mul.rn.f16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
  return d;
}

__device__ __forceinline__ void mma_f16(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                        uint32_t b0, uint32_t b1) {
  asm volatile("mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
               "{%0,%1,%2,%3};"
               : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
               : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// The four block scales of a lane's 64 K elements, each broadcast to both halves.
__device__ __forceinline__ void scales4(uint32_t word, uint32_t (&s)[4]) {
  const uint32_t lo = e4m3x2_f16x2(word), hi = e4m3x2_f16x2(word >> 16);
  s[0] = __byte_perm(lo, 0, 0x1010);
  s[1] = __byte_perm(lo, 0, 0x3232);
  s[2] = __byte_perm(hi, 0, 0x1010);
  s[3] = __byte_perm(hi, 0, 0x3232);
}

struct Item { int e, rb, c, nc; };      // expert, weight block, first chunk, chunks (1 or 2)

__device__ __forceinline__ int chunks_of(const int32_t *off, int e) { return (off[e + 1] - off[e] + kTok - 1) / kTok; }
__device__ __forceinline__ int groups_of(const int32_t *off, int e) { return (chunks_of(off, e) + kChunks - 1) / kChunks; }

__device__ __forceinline__ Item decode_item(int64_t it, const int32_t *items, const int32_t *off, int E) {
  Item I;
  I.e = upper_group(items, E, it);
  const int ng = groups_of(off, I.e);
  const int rem = (int)(it - items[I.e]);
  I.rb = rem / ng;                        // weight block major: the groups of one block follow each other
  I.c = (rem % ng) * kChunks;
  I.nc = min(kChunks, chunks_of(off, I.e) - I.c);
  return I;
}

template <bool kSwiglu, bool kBf16Out>
__global__ void __launch_bounds__(kThreads, 1) w4a16_kernel(
    const __grid_constant__ CUtensorMap tmap_w, const __grid_constant__ CUtensorMap tmap_s,
    const uint16_t *__restrict__ x16, const float *__restrict__ xscale, const float *__restrict__ w_gs,
    const int32_t *__restrict__ offsets, int E, int64_t M_total, int N, int K, void *__restrict__ y,
    int32_t *dev_status) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
  const uint32_t sbase = smem_u32(smem);
  const uint32_t bar_full = sbase + OFF_BAR, bar_empty = bar_full + 8 * kStages;
  volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + OFF_MISC);
  volatile int *stop_word = reinterpret_cast<volatile int *>(smem + OFF_MISC + 4);
  int32_t *off = reinterpret_cast<int32_t *>(smem + OFF_TABLES);
  int32_t *cslot = off + (kMaxExperts + 1), *items = cslot + (kMaxExperts + 1), *scratch = items + (kMaxExperts + 1);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int rows_out = kSwiglu ? N / 2 : N;
  const int row_blocks = kSwiglu ? rows_out / 64 : N / 128;
  const int nst = K / 256;

  if (threadIdx.x == 0) {
    *abort_flag = 0;
    for (int s = 0; s < kStages; ++s) {
      mbar_init(bar_full + 8 * s, 1);
      mbar_init(bar_empty + 8 * s, kConsumers);
    }
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  for (int i = threadIdx.x; i <= E; i += blockDim.x)
    off[i] = offsets ? offsets[i] : (i == 0 ? 0 : (int32_t)M_total);
  __syncthreads();
  block_prefix(E, cslot, scratch, [&](int e) { return (off[e + 1] - off[e] + kTok - 1) / kTok; });
  block_prefix(E, items, scratch, [&](int e) { return row_blocks * groups_of(off, e); });
  const int64_t total = items[E];

  if (warp == kConsumers) {
    // ================================================================ producer
    if (lane == 0) {
      const uint64_t pol = gemm::policy_evict_first();
      int stage = 0;
      uint32_t phase = 0;
      bool armed[kStages] = {};
      uint32_t armed_parity[kStages] = {};
      bool ok = true;
      for (int64_t it = blockIdx.x; it < total && ok; it += gridDim.x) {
        const Item I = decode_item(it, items, off, E);
        const int64_t C = cslot[I.e] + I.c;
        const uint32_t bytes = kWBytes + kSBytes + I.nc * kXChunk;
        const int32_t row0 = I.e * N + I.rb * (kSwiglu ? 64 : 128);
        const int32_t uprow0 = row0 + N / 2;
        for (int st = 0; st < nst; ++st) {
          if (!mbar_wait(bar_empty + 8 * stage, phase ^ 1, abort_flag, dev_status)) { ok = false; break; }
          const uint32_t fb = bar_full + 8 * stage;
          mbar_arrive_expect_tx(fb, bytes);
          armed[stage] = true;
          armed_parity[stage] = phase;
          const uint32_t base = sbase + stage * kStageBytes;
          if (kSwiglu) {
            gemm::tma_load_2d(base, &tmap_w, st * 128, row0, fb, pol);
            gemm::tma_load_2d(base + kWBytes / 2, &tmap_w, st * 128, uprow0, fb, pol);
            gemm::tma_load_2d(base + kWBytes, &tmap_s, st * 16, row0, fb, pol);
            gemm::tma_load_2d(base + kWBytes + kSBytes / 2, &tmap_s, st * 16, uprow0, fb, pol);
          } else {
            gemm::tma_load_2d(base, &tmap_w, st * 128, row0, fb, pol);
            gemm::tma_load_2d(base + kWBytes, &tmap_s, st * 16, row0, fb, pol);
          }
          for (int cc = 0; cc < I.nc; ++cc)
            gemm::bulk_load(base + kWBytes + kSBytes + cc * kXChunk, x16 + ((C + cc) * nst + st) * 2048, kXChunk, fb);
          if (++stage == kStages) { stage = 0; phase ^= 1; }
        }
      }
      // every armed stage's copies land before the CTA exits
      for (int s = 0; s < kStages; ++s) {
        if (!armed[s]) continue;
        const long long t0 = clock64();
        while (!mbar_try_wait(bar_full + 8 * s, armed_parity[s]) && clock64() - t0 < kWaitBudgetCycles) {}
      }
    }
  } else {
    // ================================================================ consumers
    const int g = lane >> 2, t = lane & 3;
    const int tile = warp & 7, half = warp >> 3;                      // row tile, K half of each stage
    const int rowA = kSwiglu ? 8 * tile + g : 16 * tile + g;          // MMA rows g and g + 8
    const int rowB = kSwiglu ? 64 + 8 * tile + g : 16 * tile + 8 + g;
    // the lane's 16 code bytes of this half: 16-byte chunk 2t + half of the row (128-byte swizzle)
    const uint32_t offA = rowA * 128 + (((2 * t + half) ^ (rowA & 7)) << 4);
    const uint32_t offB = rowB * 128 + (((2 * t + half) ^ (rowB & 7)) << 4);
    float *red = reinterpret_cast<float *>(smem + OFF_RED) + (tile * 32 + lane) * 8;
    int stage = 0;
    uint32_t phase = 0;
    for (int64_t it = blockIdx.x; it < total; it += gridDim.x) {
      const Item I = decode_item(it, items, off, E);
      float d[kChunks][4] = {};
      // the K loop, compiled once per chunk count (I.nc is warp-uniform)
      auto kloop = [&](auto nc_tag) {
      constexpr bool two = decltype(nc_tag)::value == 2;
      for (int st = 0; st < nst; ++st) {
        if (!gemm::mbar_wait_warp(bar_full + 8 * stage, phase, abort_flag, dev_status)) break;
        const uint8_t *base = smem + stage * kStageBytes;
        const uint4 wa = *reinterpret_cast<const uint4 *>(base + offA);
        const uint4 wb = *reinterpret_cast<const uint4 *>(base + offB);
        // scales of K blocks 4t + 2 half .. +1 (two bytes of the lane's word)
        const uint32_t sa = *reinterpret_cast<const uint16_t *>(base + kWBytes + rowA * 16 + 4 * t + 2 * half);
        const uint32_t sb = *reinterpret_cast<const uint16_t *>(base + kWBytes + rowB * 16 + 4 * t + 2 * half);
        const uint8_t *xb = base + kWBytes + kSBytes;
        uint4 xp[kChunks][4];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          xp[0][i] = *reinterpret_cast<const uint4 *>(xb + ((4 * half + i) * 32 + lane) * 16);
          if constexpr (two) xp[1][i] = *reinterpret_cast<const uint4 *>(xb + kXChunk + ((4 * half + i) * 32 + lane) * 16);
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(bar_empty + 8 * stage);     // release: the loads above are ordered before it
        if (++stage == kStages) { stage = 0; phase ^= 1; }
        const uint32_t hA = e4m3x2_f16x2(sa), hB = e4m3x2_f16x2(sb);
        const uint32_t sA[2] = {__byte_perm(hA, 0, 0x1010), __byte_perm(hA, 0, 0x3232)};
        const uint32_t sB[2] = {__byte_perm(hB, 0, 0x1010), __byte_perm(hB, 0, 0x3232)};
        const uint32_t wA[4] = {wa.x, wa.y, wa.z, wa.w};
        const uint32_t wB[4] = {wb.x, wb.y, wb.z, wb.w};
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          // word j = slices 8 half + 2j, +1 (physical K 64t + 4 (8 half + 2j) .. +7):
          // bytes 0, 1 feed the first slice, bytes 2, 3 the second
          uint32_t fa[4], fb[4];
          e2m1x8_f16x2(wA[j], fa);
          e2m1x8_f16x2(wB[j], fb);
          const uint32_t sa2 = sA[j >> 1], sb2 = sB[j >> 1];
          const uint32_t a0 = hmul2(fa[0], sa2), a1 = hmul2(fb[0], sb2), a2 = hmul2(fa[1], sa2), a3 = hmul2(fb[1], sb2);
          const uint32_t c0 = hmul2(fa[2], sa2), c1 = hmul2(fb[2], sb2), c2 = hmul2(fa[3], sa2), c3 = hmul2(fb[3], sb2);
          mma_f16(d[0], a0, a1, a2, a3, xp[0][j].x, xp[0][j].y);
          mma_f16(d[0], c0, c1, c2, c3, xp[0][j].z, xp[0][j].w);
          if constexpr (two) {
            mma_f16(d[1], a0, a1, a2, a3, xp[1][j].x, xp[1][j].y);
            mma_f16(d[1], c0, c1, c2, c3, xp[1][j].z, xp[1][j].w);
          }
        }
      }
      };
      if (I.nc == 2) kloop(std::integral_constant<int, 2>{});
      else kloop(std::integral_constant<int, 1>{});
      // The second K half hands its partial sums to the first.  Every consumer
      // warp reaches both barriers of every item it starts (a wait that gave
      // up only ends the stage loop), and the decision to stop is read from
      // one shared word after the second barrier, so all warps leave together.
      if (half == 1) {
        reinterpret_cast<float4 *>(red)[0] = make_float4(d[0][0], d[0][1], d[0][2], d[0][3]);
        reinterpret_cast<float4 *>(red)[1] = make_float4(d[1][0], d[1][1], d[1][2], d[1][3]);
      }
      asm volatile("bar.sync 1, %0;" :: "n"(kConsumers * 32) : "memory");
      if (half == 0) {
        const float4 p0 = reinterpret_cast<const float4 *>(red)[0], p1 = reinterpret_cast<const float4 *>(red)[1];
        d[0][0] += p0.x; d[0][1] += p0.y; d[0][2] += p0.z; d[0][3] += p0.w;
        d[1][0] += p1.x; d[1][1] += p1.y; d[1][2] += p1.z; d[1][3] += p1.w;
      }
      if (warp == 0 && lane == 0) *stop_word = *abort_flag;
      asm volatile("bar.sync 1, %0;" :: "n"(kConsumers * 32) : "memory");
      if (*stop_word) break;
      if (half == 1) continue;
      // per chunk: d[cc][0], d[cc][1]: row A, tokens 2t, 2t+1; d[cc][2], d[cc][3]: row B
      const float gs = w_gs[I.e];
#pragma unroll
      for (int cc = 0; cc < kChunks; ++cc) {
        if (cc >= I.nc) break;
        const int32_t r0 = off[I.e] + (I.c + cc) * kTok;
        const int ntok = min(kTok, off[I.e + 1] - r0);
        const int64_t C = cslot[I.e] + I.c + cc;
#pragma unroll
        for (int j = 0; j < 2; ++j) {
          const int tok = 2 * t + j;
          if (tok >= ntok) continue;
          const float xs = xscale[C * kTok + tok];
          const float va = __fmul_rn(__fmul_rn(d[cc][j], gs), xs);
          const float vb = __fmul_rn(__fmul_rn(d[cc][2 + j], gs), xs);
          if constexpr (kSwiglu) {
            const float h = __fmul_rn(__fdividef(va, 1.0f + __expf(-va)), vb);
            const int64_t o = (int64_t)(r0 + tok) * rows_out + I.rb * 64 + 8 * tile + g;
            if (kBf16Out) reinterpret_cast<__nv_bfloat16 *>(y)[o] = __float2bfloat16_rn(h);
            else reinterpret_cast<float *>(y)[o] = h;
          } else {
            const int64_t o = (int64_t)(r0 + tok) * rows_out + I.rb * 128 + 16 * tile + g;
            if (kBf16Out) {
              reinterpret_cast<__nv_bfloat16 *>(y)[o] = __float2bfloat16_rn(va);
              reinterpret_cast<__nv_bfloat16 *>(y)[o + 8] = __float2bfloat16_rn(vb);
            } else {
              reinterpret_cast<float *>(y)[o] = va;
              reinterpret_cast<float *>(y)[o + 8] = vb;
            }
          }
        }
      }
    }
  }
  __syncthreads();
}

}  // namespace w4a16_mma
}  // namespace nvfp4

// ====================================================================== host side
namespace nvfp4 {
namespace w4a16_mma {

namespace {

// 2-D uint8 view [rows, row_bytes] with a {16 bytes, box_rows} box, no swizzle
// (row-major E4M3 scales: 16 per 256-element K stage).
bool make_map_scales16(CUtensorMap *map, const void *base, uint64_t rows, uint64_t row_bytes, uint32_t box_rows) {
  cuuint64_t dims[2] = {row_bytes, rows};
  cuuint64_t strides[1] = {row_bytes};
  cuuint32_t box[2] = {16, box_rows};
  return gemm::encode_u8_map(map, 2, base, dims, strides, box, CU_TENSOR_MAP_SWIZZLE_NONE);
}

// Upper bound on the 8-token chunks of all experts: sum ceil(n_e / 8).
int64_t chunks_bound(int64_t M_total, int E) { return (M_total + 7 * (int64_t)E) / 8 + 1; }

size_t x16_bytes(int64_t M_total, int E, int64_t K) {
  return ((size_t)chunks_bound(M_total, E) * 8 * (size_t)K * 2 + 255) / 256 * 256;
}

}  // namespace

size_t workspace_bytes(int64_t M_total, int E, int64_t K) {
  return x16_bytes(M_total, E, K) + (size_t)chunks_bound(M_total, E) * 8 * sizeof(float) + 256;
}

// Arguments are validated by nvfp4_grouped_gemm_w4a16.
nvfp4_status launch(const void *x, int64_t ld_x, int64_t x_rows, const int32_t *row_index, const uint8_t *b_q,
                    const uint8_t *b_sf, const float *b_gs, const int32_t *expert_offsets, int E, int64_t M_total,
                    int64_t N, int64_t K, void *y, nvfp4_out_dtype out_dtype, bool swiglu, void *workspace,
                    int32_t *dev_status, cudaStream_t stream) {
  uint16_t *x16 = reinterpret_cast<uint16_t *>(workspace);
  float *xscale = reinterpret_cast<float *>(reinterpret_cast<uint8_t *>(workspace) + x16_bytes(M_total, E, K));
  const int sms = host::sm_count();
  // prep: the routed rows, as scaled f16 in fragment order
  {
    const size_t sm = sizeof(int32_t) * (2 * (size_t)(E + 1) + 8);
    int64_t grid = (M_total + 7) / 8;
    if (grid > (int64_t)sms * 8) grid = (int64_t)sms * 8;
    w4a16_prep_kernel<<<(unsigned)grid, 256, sm, stream>>>(reinterpret_cast<const uint16_t *>(x), ld_x, x_rows,
                                                           row_index, expert_offsets, E, M_total, (int)K, x16, xscale,
                                                           dev_status);
    if (cudaGetLastError() != cudaSuccess) return NVFP4_ERR_CUDA;
  }
  CUtensorMap tw, ts;
  const uint32_t box_rows = swiglu ? 64 : 128;
  if (!gemm::make_map(&tw, b_q, (uint64_t)E * N, (uint64_t)K / 2, box_rows)) return NVFP4_ERR_CUDA;
  if (!make_map_scales16(&ts, b_sf, (uint64_t)E * N, (uint64_t)K / 16, box_rows)) return NVFP4_ERR_CUDA;
  const int variant = (swiglu ? 2 : 0) + (out_dtype == NVFP4_OUT_BF16 ? 1 : 0);
  auto kern = variant == 3 ? w4a16_kernel<true, true>
            : variant == 2 ? w4a16_kernel<true, false>
            : variant == 1 ? w4a16_kernel<false, true> : w4a16_kernel<false, false>;
  if (!host::set_max_dynamic_smem(reinterpret_cast<const void *>(kern), SMEM_BYTES)) return NVFP4_ERR_CUDA;
  kern<<<sms, kThreads, SMEM_BYTES, stream>>>(tw, ts, x16, xscale, b_gs, expert_offsets, E, M_total, (int)N, (int)K,
                                              y, dev_status);
  return cudaGetLastError() == cudaSuccess ? NVFP4_OK : NVFP4_ERR_CUDA;
}

}  // namespace w4a16_mma
}  // namespace nvfp4
