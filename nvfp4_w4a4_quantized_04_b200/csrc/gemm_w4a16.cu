// Weight-only NVFP4 grouped GEMM with 16-bit activations (W4A16), sm_100a.
//
// The "DeepSeek-V4.1-Flash-NVFP4" page lists the MTP layer's experts as
// W4A16_NVFP4: the weights are NVFP4 (E2M1 codes, E4M3 scale per 16, FP32
// global) and the activations stay 16-bit.  For every routed expert e:
//   Y_e = X_e (s_g[e] * W_e)^T,   W_e[n, k] = e2m1(code) * e4m3(S[n, k/16]),
// accumulated in fp32.  With the SwiGLU epilogue the weight is a fused gate_up
// [2I, K] (gate rows 0..I-1, up rows I..2I-1) and the output is
// h = silu(g) * u.
//
// This is the kernel for groups of more than a few tokens: one weight
// conversion and one run of MMAs serve up to 64 tokens.  (Each tcgen05 MMA
// with N = 16 and K = 16 costs about 108 cycles, so with groups of 1-3 tokens
// this kernel tops out near 2.7 TB/s of weights; the warp-MMA kernel of
// gemm_w4a16_mma.cu serves that regime.)
//  * Operands in f16 on the 5th-generation tensor cores (tcgen05.mma
//    kind::f16, fp32 accumulation in tensor memory).  E2M1 -> f16 is one
//    hardware conversion per two codes, and e2m1 * e4m3 is exact in f16 (at
//    most 6 significant bits, |.| in [2^-10, 2688]).  The bf16 activations are
//    converted once per call by a prep kernel: each routed row is scaled by a
//    power of two 2^-k that puts its max |x| in [2^14, 2^15), then rounded to
//    f16.  Every element within 2^29 of the row's max is exact; smaller ones
//    land on f16's subnormal grid (error below 2^-25 of the row max).  The
//    epilogue multiplies by 2^k again, which is exact.
//  * The weights are the MMA's A operand, read from tensor memory: eight
//    converter warps turn a 256-element K stage of 128 weight rows into f16
//    (two warps per TMEM lane quadrant, one K half each) and write it with
//    tcgen05.st into one of three A buffers (128 columns each).  The tokens
//    are the B operand, read from shared memory: the prep kernel lays the
//    routed rows out in 16-row groups per K stage and 64-element K sub-tile,
//    in the tensor core's 128-byte-swizzled K-major layout, the groups of
//    one sub-tile next to each other, so four bulk copies bring an item's
//    (up to 4) groups of a stage in.
//  * Pipeline.  One producer warp streams per stage the 128-row weight tile
//    and its row-major scales by TMA (128-byte swizzle) and the item's tokens
//    by bulk copies into a four-stage ring; one thread issues the 16 MMAs of a
//    stage (M = 128 weight rows, N = 16..64 tokens, K = 16 each); four
//    epilogue warps read the double-buffered accumulator.
//  * Work item = (expert, 128-row weight block, 64-token chunk).  An expert
//    with more than 64 tokens re-reads its weight block per chunk, and those
//    items follow each other so the re-reads hit L2.
//  * Every mbarrier wait is bounded (NVFP4_ERR_TIMEOUT, then all roles leave).
#include "gemm_common.cuh"
#include "host_util.cuh"

#include <cuda_fp16.h>

#include <atomic>

namespace nvfp4 {
namespace w4a16 {

using gemm::kWaitBudgetCycles;
using gemm::mbar_arrive;
using gemm::mbar_arrive_expect_tx;
using gemm::mbar_init;
using gemm::mbar_try_wait;
using gemm::mbar_wait;
using gemm::mbar_wait_warp;
using gemm::smem_u32;
using gemm::tc_fence_after;
using gemm::tc_fence_before;

constexpr int kGrp = 16;                     // rows of a token group (the MMA's N step)
constexpr int kTok = 64;                     // tokens per item: up to 4 groups
constexpr int kStages = 4;
constexpr int kWBytes = 128 * 128;           // 128 rows x 256 codes
constexpr int kSBytes = 128 * 16;            // 128 rows x 16 scales
constexpr int kGrpBytes = kGrp * 128;        // one group's rows of one 64-element K sub-tile (2 KB)
constexpr int kSubBytes = kTok * 128;        // shared-memory room for one K sub-tile of an item (8 KB)
constexpr int kXBytes = 4 * kSubBytes;       // four K sub-tiles per 256-element stage
constexpr int kStageBytes = kWBytes + kSBytes + kXBytes;
constexpr int kABufs = 3;                    // f16 weight stages in tensor memory
constexpr uint32_t kACols = 128;             // 256 f16 per row = 128 columns
constexpr uint32_t kAccCol = kABufs * kACols;  // accumulators: 2 x 64 columns after the A buffers
constexpr uint32_t kTmemCols = 512;
static_assert(kAccCol + 2 * kTok <= kTmemCols, "tensor memory budget");
constexpr int kConverters = 8;               // warps 6.., kConverters / 4 per TMEM lane quadrant
constexpr int kConvSplit = kConverters / 4;  // K pieces of a stage per weight row
constexpr int kConvCodes = 256 / kConvSplit; // codes per converter thread per stage
static_assert(kConverters % 4 == 0 && kConvCodes % 64 == 0, "whole 32-column stores per converter");
constexpr int W_PRODUCER = 0, W_MMA = 1, W_CONV0 = 6;   // warps 2..5: epilogue
constexpr int kWarps = W_CONV0 + kConverters;
constexpr int kThreads = kWarps * 32;
constexpr int OFF_BAR = kStages * kStageBytes;
// full[S], empty[S], a_full[3], a_free[3], acc_full[2], acc_empty[2], drain
constexpr int NUM_BARS = 2 * kStages + 2 * kABufs + 2 + 2 + 1;
constexpr int OFF_MISC = OFF_BAR + NUM_BARS * 8;
constexpr int OFF_TABLES = OFF_MISC + 16;
constexpr int kMaxExperts = 1024;
constexpr int TABLE_BYTES = 3 * (kMaxExperts + 1) * 4 + 32 * 4;
constexpr int SMEM_BYTES = OFF_TABLES + TABLE_BYTES + 1024;
static_assert(SMEM_BYTES <= 232448, "shared memory budget");
static_assert(kStageBytes % 1024 == 0 && kWBytes % 1024 == 0, "128-byte swizzle atoms");

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
// ceil(n_e/16) groups of 16 rows, group index G = gslot[e] + i/16 of Gt in
// all.  For K stage st and 64-element K sub-tile k, the 2 KB block at byte
// ((st * 4 + k) * Gt + G) * 2048 holds group G's 16 rows of 128 bytes in the
// tensor core's 128-byte-swizzled K-major layout: row g's 16-byte piece j
// (K = 256 st + 64 k + 8 j .. +8) sits at g * 128 + (j ^ (g & 7)) * 16.  The
// groups of one sub-tile lie next to each other, so the (up to 4) groups of an
// item form one contiguous run per sub-tile.  xscale[G * 16 + g] = 2^k of that
// token.  Padding rows of a group are not written: the MMA reads them, the
// epilogue never stores the columns they feed.
__global__ void __launch_bounds__(256) w4a16_prep_kernel(
    const uint16_t *__restrict__ x, int64_t ld_x, int64_t x_rows, const int32_t *__restrict__ row_index,
    const int32_t *__restrict__ offsets, int E, int64_t M_total, int K, uint16_t *__restrict__ x16,
    float *__restrict__ xscale, int32_t *dev_status) {
  extern __shared__ int32_t smem[];
  int32_t *off = smem, *gslot = smem + (E + 1), *scratch = smem + 2 * (E + 1);
  for (int i = threadIdx.x; i <= E; i += blockDim.x)
    off[i] = offsets ? offsets[i] : (i == 0 ? 0 : (int32_t)M_total);
  __syncthreads();
  block_prefix(E, gslot, scratch, [&](int e) { return (off[e + 1] - off[e] + kGrp - 1) / kGrp; });
  const int64_t Gt = gslot[E];
  const int lane = threadIdx.x & 31;
  const int64_t nwarps = ((int64_t)gridDim.x * blockDim.x) >> 5;
  bool bad_index = false, bad_value = false;
  for (int64_t r = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5; r < M_total; r += nwarps) {
    const int e = upper_group(off, E, r);
    const int i = (int)(r - off[e]);
    const int64_t G = gslot[e] + i / kGrp;
    const int g = i % kGrp;
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
    if (lane == 0) xscale[G * kGrp + g] = __uint_as_float((uint32_t)(127 + k) << 23);
    uint8_t *dst = reinterpret_cast<uint8_t *>(x16) + G * (int64_t)kGrpBytes + g * 128;
    for (int p = lane; p < K / 8; p += 32) {
      const int st = p >> 5, rest = p & 31, ks = rest >> 3, j = rest & 7;
      const uint4 v = __ldg(reinterpret_cast<const uint4 *>(xr + (int64_t)p * 8));
      const uint32_t w[4] = {v.x, v.y, v.z, v.w};
      uint32_t o[4];
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const float lo = __fmul_rn(__uint_as_float(w[q] << 16), sc);
        const float hi = __fmul_rn(__uint_as_float(w[q] & 0xFFFF0000u), sc);
        const __half2 h = __floats2half2_rn(lo, hi);
        o[q] = *reinterpret_cast<const uint32_t *>(&h);
      }
      *reinterpret_cast<uint4 *>(dst + (int64_t)(st * 4 + ks) * Gt * kGrpBytes + ((j ^ (g & 7)) << 4)) =
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

// The four bytes of a word (8 codes) -> four f16x2 (byte j -> o[j], its low
// nibble in the low half), exact.
__device__ __forceinline__ void e2m1x8_f16x2(uint32_t w, uint32_t *o) {
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

// 32 consecutive 32-bit tensor-memory columns of this warp's lane quadrant.
__device__ __forceinline__ void tc_st_x32(uint32_t taddr, const uint32_t *v) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,"
      "%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};"
      :: "r"(taddr), "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7]),
         "r"(v[8]), "r"(v[9]), "r"(v[10]), "r"(v[11]), "r"(v[12]), "r"(v[13]), "r"(v[14]), "r"(v[15]),
         "r"(v[16]), "r"(v[17]), "r"(v[18]), "r"(v[19]), "r"(v[20]), "r"(v[21]), "r"(v[22]), "r"(v[23]),
         "r"(v[24]), "r"(v[25]), "r"(v[26]), "r"(v[27]), "r"(v[28]), "r"(v[29]), "r"(v[30]), "r"(v[31])
      : "memory");
}

__device__ __forceinline__ void tc_ld_x16(uint32_t taddr, uint32_t *r) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
      : "r"(taddr));
}

// D (fp32, tensor memory) += A (f16, tensor memory, M = 128 lanes x K = 16 in
// 8 columns) x B (f16, shared memory descriptor)^T.
__device__ __forceinline__ void tc_mma_f16_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc, uint32_t idesc,
                                              uint32_t accumulate) {
  asm volatile(
      "{\n.reg .pred p;\nsetp.ne.b32 p, %4, 0;\n"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n}"
      :: "r"(d_tmem), "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// Instruction descriptor, kind::f16: fp32 D, f16 A and B, both K-major,
// M = 128, N = n.
__device__ __forceinline__ uint32_t idesc_f16(uint32_t m, uint32_t n) {
  return (1u << 4) | ((n >> 3) << 17) | ((m >> 4) << 24);
}

struct Item { int e, rb, c; };           // expert, weight block, 64-token chunk

__device__ __forceinline__ int chunks_of(const int32_t *off, int e) { return (off[e + 1] - off[e] + kTok - 1) / kTok; }
__device__ __forceinline__ int groups_of(const int32_t *off, int e) { return (off[e + 1] - off[e] + kGrp - 1) / kGrp; }

__device__ __forceinline__ Item decode_item(int64_t it, const int32_t *items, const int32_t *off, int E) {
  Item I;
  I.e = upper_group(items, E, it);
  const int nc = chunks_of(off, I.e);
  const int rem = (int)(it - items[I.e]);
  I.rb = rem / nc;                       // weight block major: the chunks of one block follow each other
  I.c = rem % nc;
  return I;
}

// TMEM lane (within the 128 weight rows of an item) -> row of the item's
// shared-memory weight tile.  SwiGLU: the tile holds 64 gate rows then the 64
// matching up rows; lane 32q + l takes gate row 16q + l (l < 16) or up row
// 16q + l - 16, so a gate lane and its up lane sit 16 lanes apart in one
// quadrant.  Otherwise lane = row.
template <bool kSwiglu>
__device__ __forceinline__ int smem_row_of_lane(int q, int l) {
  if constexpr (kSwiglu) return l < 16 ? 16 * q + l : 64 + 16 * q + (l - 16);
  return 32 * q + l;
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
  const uint32_t bar_a_full = bar_empty + 8 * kStages, bar_a_free = bar_a_full + 8 * kABufs;
  const uint32_t bar_acc_full = bar_a_free + 8 * kABufs, bar_acc_empty = bar_acc_full + 16;
  const uint32_t bar_drain = bar_acc_empty + 16;
  volatile uint32_t *tmem_holder = reinterpret_cast<volatile uint32_t *>(smem + OFF_MISC);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + OFF_MISC + 4);
  int32_t *off = reinterpret_cast<int32_t *>(smem + OFF_TABLES);
  int32_t *gslot = off + (kMaxExperts + 1), *items = gslot + (kMaxExperts + 1), *scratch = items + (kMaxExperts + 1);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int rows_out = kSwiglu ? N / 2 : N;
  const int row_blocks = kSwiglu ? rows_out / 64 : N / 128;
  const int nst = K / 256;

  if (threadIdx.x == 0) {
    *abort_flag = 0;
    for (int s = 0; s < kStages; ++s) {
      mbar_init(bar_full + 8 * s, 1);
      mbar_init(bar_empty + 8 * s, 1);
    }
    for (int a = 0; a < kABufs; ++a) {
      mbar_init(bar_a_full + 8 * a, kConverters * 32);
      mbar_init(bar_a_free + 8 * a, 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(bar_acc_full + 8 * b, 1);
      mbar_init(bar_acc_empty + 8 * b, 128);
    }
    mbar_init(bar_drain, 1);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == W_MMA) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;"
                 :: "r"(smem_u32((const void *)tmem_holder)), "r"(kTmemCols) : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  for (int i = threadIdx.x; i <= E; i += blockDim.x)
    off[i] = offsets ? offsets[i] : (i == 0 ? 0 : (int32_t)M_total);
  __syncthreads();
  block_prefix(E, gslot, scratch, [&](int e) { return groups_of(off, e); });
  block_prefix(E, items, scratch, [&](int e) { return row_blocks * chunks_of(off, e); });
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_holder;
  const int64_t total = items[E];
  const int64_t Gt = gslot[E];

  if (warp == W_PRODUCER) {
    // ================================================================ producer
    if (lane == 0) {
      gemm::prefetch_tensormap(&tmap_w);
      gemm::prefetch_tensormap(&tmap_s);
      const uint64_t pol = gemm::policy_evict_first();
      int stage = 0;
      uint32_t phase = 0;
      bool armed[kStages] = {};
      uint32_t armed_parity[kStages] = {};
      bool ok = true;
      for (int64_t it = blockIdx.x; it < total && ok; it += gridDim.x) {
        const Item I = decode_item(it, items, off, E);
        const int ntok = min(kTok, off[I.e + 1] - off[I.e] - I.c * kTok);
        const int ng = (ntok + kGrp - 1) / kGrp;
        const int64_t G0 = gslot[I.e] + 4 * I.c;
        const int32_t row0 = I.e * N + I.rb * (kSwiglu ? 64 : 128);
        const int32_t uprow0 = row0 + N / 2;
        for (int st = 0; st < nst; ++st) {
          if (!mbar_wait(bar_empty + 8 * stage, phase ^ 1, abort_flag, dev_status)) { ok = false; break; }
          const uint32_t fb = bar_full + 8 * stage;
          mbar_arrive_expect_tx(fb, kWBytes + kSBytes + 4 * ng * kGrpBytes);
          armed[stage] = true;
          armed_parity[stage] = phase;
          const uint32_t base = sbase + stage * kStageBytes;
          for (int k = 0; k < 4; ++k)
            gemm::bulk_load(base + kWBytes + kSBytes + k * kSubBytes,
                            reinterpret_cast<const uint8_t *>(x16) + ((int64_t)(st * 4 + k) * Gt + G0) * kGrpBytes,
                            ng * kGrpBytes, fb);
          if (kSwiglu) {
            gemm::tma_load_2d(base, &tmap_w, st * 128, row0, fb, pol);
            gemm::tma_load_2d(base + kWBytes / 2, &tmap_w, st * 128, uprow0, fb, pol);
            gemm::tma_load_2d(base + kWBytes, &tmap_s, st * 16, row0, fb, pol);
            gemm::tma_load_2d(base + kWBytes + kSBytes / 2, &tmap_s, st * 16, uprow0, fb, pol);
          } else {
            gemm::tma_load_2d(base, &tmap_w, st * 128, row0, fb, pol);
            gemm::tma_load_2d(base + kWBytes, &tmap_s, st * 16, row0, fb, pol);
          }
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
  } else if (warp >= W_CONV0) {
    // ================================================================ weight converters
    // Thread (quadrant q, lane l, K piece h) converts kConvCodes codes of one
    // weight row per stage into kConvCodes / 2 f16x2 columns of A buffer
    // kst % 3, lane 32q + l.
    const int q = warp & 3, h = (warp - W_CONV0) >> 2;
    const uint32_t lane_base = (uint32_t)(32 * q) << 16;
    const int R = smem_row_of_lane<kSwiglu>(q, lane);
    uint32_t kst = 0;
    bool ok = true;
    for (int64_t it = blockIdx.x; it < total && ok; it += gridDim.x) {
      for (int st = 0; st < nst; ++st, ++kst) {
        const uint32_t s = kst % kStages, a = kst % kABufs;
        if (!mbar_wait_warp(bar_full + 8 * s, (kst / kStages) & 1, abort_flag, dev_status)) { ok = false; break; }
        if (kst >= (uint32_t)kABufs &&
            !mbar_wait_warp(bar_a_free + 8 * a, ((kst / kABufs) - 1) & 1, abort_flag, dev_status)) {
          ok = false; break;
        }
        tc_fence_after();
        const uint8_t *base = smem + s * kStageBytes;
        constexpr int kChunks16 = kConvCodes / 32;          // 16-byte code chunks per thread
        uint32_t scw[kChunks16 / 2];                        // this piece's scale bytes, 4 per word
#pragma unroll
        for (int i = 0; i < kChunks16 / 2; ++i)
          scw[i] = *reinterpret_cast<const uint32_t *>(base + kWBytes + R * 16 + h * (kConvCodes / 16) + 4 * i);
#pragma unroll
        for (int half32 = 0; half32 < kChunks16 / 2; ++half32) {
          uint32_t v[32];
#pragma unroll
          for (int jj = 0; jj < 2; ++jj) {
            const int jc = 2 * half32 + jj;                 // 16-byte chunk of this piece: 32 codes, 2 blocks
            const int j = kChunks16 * h + jc;               // chunk of the 128-byte row
            const uint4 c = *reinterpret_cast<const uint4 *>(base + R * 128 + ((j ^ (R & 7)) << 4));
            const uint32_t sw = scw[jc >> 1];
            const uint32_t b0 = (sw >> (16 * (jc & 1))) & 0xFFu, b1 = (sw >> (16 * (jc & 1) + 8)) & 0xFFu;
            const uint32_t S0 = e4m3x2_f16x2(b0 | (b0 << 8)), S1 = e4m3x2_f16x2(b1 | (b1 << 8));
            uint32_t o[16];
            e2m1x8_f16x2(c.x, o);
            e2m1x8_f16x2(c.y, o + 4);
            e2m1x8_f16x2(c.z, o + 8);
            e2m1x8_f16x2(c.w, o + 12);
#pragma unroll
            for (int t = 0; t < 8; ++t) v[16 * jj + t] = hmul2(o[t], S0);
#pragma unroll
            for (int t = 8; t < 16; ++t) v[16 * jj + t] = hmul2(o[t], S1);
          }
          tc_st_x32(tmem_base + lane_base + a * kACols + (kConvCodes / 2) * h + 32 * half32, v);
        }
        asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
        tc_fence_before();
        mbar_arrive(bar_a_full + 8 * a);
      }
    }
  } else if (warp == W_MMA) {
    // ================================================================ MMA issuer
    uint32_t kst = 0, titer = 0;
    bool ok = true;
    for (int64_t it = blockIdx.x; it < total && ok; it += gridDim.x, ++titer) {
      const Item I = decode_item(it, items, off, E);
      const int ntok = min(kTok, off[I.e + 1] - off[I.e] - I.c * kTok);
      const uint32_t idesc = idesc_f16(128, (uint32_t)((ntok + kGrp - 1) / kGrp) * kGrp);
      const uint32_t ab = titer & 1;
      const uint32_t t_acc = tmem_base + kAccCol + ab * kTok;
      if (!mbar_wait_warp(bar_acc_empty + 8 * ab, ((titer >> 1) & 1) ^ 1, abort_flag, dev_status)) { ok = false; break; }
      tc_fence_after();
      for (int st = 0; st < nst; ++st, ++kst) {
        const uint32_t s = kst % kStages, a = kst % kABufs;
        if (!mbar_wait_warp(bar_full + 8 * s, (kst / kStages) & 1, abort_flag, dev_status)) { ok = false; break; }
        if (!mbar_wait_warp(bar_a_full + 8 * a, (kst / kABufs) & 1, abort_flag, dev_status)) { ok = false; break; }
        tc_fence_after();
        if (lane == 0) {
          const uint32_t xb = sbase + s * kStageBytes + kWBytes + kSBytes;
#pragma unroll
          for (int kk = 0; kk < 16; ++kk) {
            // K sub-tile kk/4 (8 KB apart), +32 bytes of K per MMA inside the 128-byte rows
            const uint64_t bd = gemm::desc_sw128(xb + (kk >> 2) * kSubBytes) + 2 * (kk & 3);
            tc_mma_f16_ts(t_acc, tmem_base + a * kACols + 8 * kk, bd, idesc, (st > 0 || kk > 0) ? 1u : 0u);
          }
          gemm::tc_commit(bar_empty + 8 * s);
          gemm::tc_commit(bar_a_free + 8 * a);
        }
        __syncwarp();
      }
      if (!ok) break;
      if (lane == 0) gemm::tc_commit(bar_acc_full + 8 * ab);
      __syncwarp();
    }
    if (lane == 0) {
      gemm::tc_commit(bar_drain);
      const long long t0 = clock64();
      while (!mbar_try_wait(bar_drain, 0) && clock64() - t0 < kWaitBudgetCycles) {}
    }
    __syncwarp();
  } else {
    // ================================================================ epilogue (warps 2..5)
    const int q = warp & 3;
    const uint32_t lane_base = (uint32_t)(32 * q) << 16;
    uint32_t titer = 0;
    for (int64_t it = blockIdx.x; it < total; it += gridDim.x, ++titer) {
      const Item I = decode_item(it, items, off, E);
      const uint32_t ab = titer & 1;
      if (!mbar_wait_warp(bar_acc_full + 8 * ab, (titer >> 1) & 1, abort_flag, dev_status)) break;
      tc_fence_after();
      const int32_t r0 = off[I.e] + I.c * kTok;
      const int ntok = min(kTok, off[I.e + 1] - r0);
      uint32_t r[kTok];
#pragma unroll
      for (int c0 = 0; c0 < kTok; c0 += kGrp)
        if (c0 < ntok) tc_ld_x16(tmem_base + lane_base + kAccCol + ab * kTok + c0, r + c0);
      asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
      tc_fence_before();
      mbar_arrive(bar_acc_empty + 8 * ab);
      const float *xs_item = xscale + (gslot[I.e] + 4 * I.c) * (int64_t)kGrp;
      const float gs = w_gs[I.e];
#pragma unroll
      for (int tok = 0; tok < kTok; ++tok) {
        if (tok >= ((ntok + kGrp - 1) / kGrp) * kGrp) break;
        const float xs = tok < ntok ? xs_item[tok] : 0.0f;
        const float v = __fmul_rn(__fmul_rn(__uint_as_float(r[tok]), gs), xs);
        if constexpr (kSwiglu) {
          // lane l < 16 holds gate row 16q + l, lane l + 16 the matching up row
          const float other = __shfl_xor_sync(0xffffffffu, v, 16);
          if (lane < 16 && tok < ntok) {
            const float hv = __fmul_rn(__fdividef(v, 1.0f + __expf(-v)), other);
            const int64_t o = (int64_t)(r0 + tok) * rows_out + I.rb * 64 + 16 * q + lane;
            if (kBf16Out) reinterpret_cast<__nv_bfloat16 *>(y)[o] = __float2bfloat16_rn(hv);
            else reinterpret_cast<float *>(y)[o] = hv;
          }
        } else {
          if (tok < ntok) {
            const int64_t o = (int64_t)(r0 + tok) * rows_out + I.rb * 128 + 32 * q + lane;
            if (kBf16Out) reinterpret_cast<__nv_bfloat16 *>(y)[o] = __float2bfloat16_rn(v);
            else reinterpret_cast<float *>(y)[o] = v;
          }
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == W_MMA) {
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" :: "r"(tmem_base), "r"(kTmemCols) : "memory");
  }
}

}  // namespace w4a16
}  // namespace nvfp4

// ====================================================================== host side
namespace nvfp4 {
namespace w4a16_mma {
size_t workspace_bytes(int64_t M_total, int E, int64_t K);
nvfp4_status launch(const void *x, int64_t ld_x, int64_t x_rows, const int32_t *row_index, const uint8_t *b_q,
                    const uint8_t *b_sf, const float *b_gs, const int32_t *expert_offsets, int E, int64_t M_total,
                    int64_t N, int64_t K, void *y, nvfp4_out_dtype out_dtype, bool swiglu, void *workspace,
                    int32_t *dev_status, cudaStream_t stream);
}  // namespace w4a16_mma
}  // namespace nvfp4

using namespace nvfp4;

namespace {

// 2-D uint8 view [rows, row_bytes] with a {16 bytes, box_rows} box, no swizzle
// (row-major E4M3 scales: 16 per 256-element K stage).
bool make_map_scales16(CUtensorMap *map, const void *base, uint64_t rows, uint64_t row_bytes, uint32_t box_rows) {
  cuuint64_t dims[2] = {row_bytes, rows};
  cuuint64_t strides[1] = {row_bytes};
  cuuint32_t box[2] = {16, box_rows};
  return gemm::encode_u8_map(map, 2, base, dims, strides, box, CU_TENSOR_MAP_SWIZZLE_NONE);
}

// Upper bound on the 16-row token groups of all experts: sum ceil(n_e / 16).
int64_t groups_bound(int64_t M_total, int E) { return (M_total + (w4a16::kGrp - 1) * (int64_t)E) / w4a16::kGrp + 1; }

// f16 activations of the tcgen05 kernel: per group and 256-element K stage, 8 KB.
size_t x16_bytes(int64_t M_total, int E, int64_t K) {
  return ((size_t)groups_bound(M_total, E) * (size_t)(K / 256) * 4 * w4a16::kGrpBytes + 255) / 256 * 256;
}

size_t tc_workspace_bytes(int64_t M_total, int E, int64_t K) {
  return x16_bytes(M_total, E, K) + (size_t)groups_bound(M_total, E) * w4a16::kGrp * sizeof(float) + 256;
}

// 0 automatic: the warp-MMA kernel when the groups average at most 16 routed
// rows, the tcgen05 kernel otherwise; 1 the warp-MMA kernel; 2 the tcgen05 one.
std::atomic<int> g_w4a16_kernel{0};
constexpr int64_t kWarpMmaMaxRowsPerExpert = 16;

nvfp4_status launch_tc(const void *x, int64_t ld_x, int64_t x_rows, const int32_t *row_index, const uint8_t *b_q,
                       const uint8_t *b_sf, const float *b_gs, const int32_t *expert_offsets, int E, int64_t M_total,
                       int64_t N, int64_t K, void *y, nvfp4_out_dtype out_dtype, bool swiglu, void *workspace,
                       int32_t *dev_status, cudaStream_t stream) {
  uint16_t *x16 = reinterpret_cast<uint16_t *>(workspace);
  float *xscale = reinterpret_cast<float *>(reinterpret_cast<uint8_t *>(workspace) + x16_bytes(M_total, E, K));
  const int sms = host::sm_count();
  // prep: the routed rows, as scaled f16 in the tensor core's swizzled K-major layout
  {
    const size_t sm = sizeof(int32_t) * (2 * (size_t)(E + 1) + 8);
    int64_t grid = (M_total + 7) / 8;
    if (grid > (int64_t)sms * 8) grid = (int64_t)sms * 8;
    w4a16::w4a16_prep_kernel<<<(unsigned)grid, 256, sm, stream>>>(
        reinterpret_cast<const uint16_t *>(x), ld_x, x_rows, row_index, expert_offsets, E, M_total, (int)K, x16, xscale,
        dev_status);
    if (cudaGetLastError() != cudaSuccess) return NVFP4_ERR_CUDA;
  }
  CUtensorMap tw, ts;
  const uint32_t box_rows = swiglu ? 64 : 128;
  if (!gemm::make_map(&tw, b_q, (uint64_t)E * N, (uint64_t)K / 2, box_rows)) return NVFP4_ERR_CUDA;
  if (!make_map_scales16(&ts, b_sf, (uint64_t)E * N, (uint64_t)K / 16, box_rows)) return NVFP4_ERR_CUDA;
  const int variant = (swiglu ? 2 : 0) + (out_dtype == NVFP4_OUT_BF16 ? 1 : 0);
  auto kern = variant == 3 ? w4a16::w4a16_kernel<true, true>
            : variant == 2 ? w4a16::w4a16_kernel<true, false>
            : variant == 1 ? w4a16::w4a16_kernel<false, true> : w4a16::w4a16_kernel<false, false>;
  if (!host::set_max_dynamic_smem(reinterpret_cast<const void *>(kern), w4a16::SMEM_BYTES)) return NVFP4_ERR_CUDA;
  kern<<<sms, w4a16::kThreads, w4a16::SMEM_BYTES, stream>>>(tw, ts, x16, xscale, b_gs, expert_offsets, E, M_total,
                                                            (int)N, (int)K, y, dev_status);
  return cudaGetLastError() == cudaSuccess ? NVFP4_OK : NVFP4_ERR_CUDA;
}

}  // namespace

extern "C" size_t nvfp4_w4a16_workspace_size(int64_t M_total, int num_experts, int64_t K) {
  if (M_total < 0 || K <= 0) return 0;
  const int E = num_experts < 1 ? 1 : num_experts;
  const size_t a = tc_workspace_bytes(M_total, E, K), b = w4a16_mma::workspace_bytes(M_total, E, K);
  return a > b ? a : b;
}

extern "C" nvfp4_status nvfp4_w4a16_select_kernel(int mode) {
  if (mode < 0 || mode > 2) return NVFP4_ERR_INVALID_ARG;
  g_w4a16_kernel = mode;
  return NVFP4_OK;
}

extern "C" nvfp4_status nvfp4_grouped_gemm_w4a16(const void *x, int64_t ld_x, int64_t x_rows, const int32_t *row_index,
                                                 const uint8_t *b_q, const uint8_t *b_sf, const float *b_gs,
                                                 const int32_t *expert_offsets, int num_experts, int64_t M_total,
                                                 int64_t N, int64_t K, void *y, nvfp4_out_dtype out_dtype,
                                                 nvfp4_epilogue epi, void *workspace, int32_t *dev_status,
                                                 cudaStream_t stream) {
  if (epi != NVFP4_EPI_NONE && epi != NVFP4_EPI_SWIGLU) return NVFP4_ERR_INVALID_ARG;
  if (out_dtype != NVFP4_OUT_F32 && out_dtype != NVFP4_OUT_BF16) return NVFP4_ERR_INVALID_ARG;
  const bool swiglu = epi == NVFP4_EPI_SWIGLU;
  const int E = expert_offsets ? num_experts : 1;
  if (E < 1 || E > w4a16::kMaxExperts) return NVFP4_ERR_UNSUPPORTED_SHAPE;
  if (M_total < 0 || N <= 0 || K <= 0 || ld_x < K || x_rows < 0) return NVFP4_ERR_INVALID_ARG;
  if (!row_index && x_rows < M_total) return NVFP4_ERR_INVALID_ARG;
  if (K % 256 != 0 || ld_x % 8 != 0 || N % 128 != 0) return NVFP4_ERR_UNSUPPORTED_SHAPE;
  if ((int64_t)E * N > ((int64_t)1 << 31) - 1 || M_total > ((int64_t)1 << 30) || K > (1 << 24))
    return NVFP4_ERR_UNSUPPORTED_SHAPE;
  if (M_total == 0) return NVFP4_OK;
  if (!x || x_rows == 0 || !b_q || !b_sf || !b_gs || !y || !workspace) return NVFP4_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(x) | reinterpret_cast<uintptr_t>(b_q) | reinterpret_cast<uintptr_t>(b_sf) |
       reinterpret_cast<uintptr_t>(workspace)) & 15u)
    return NVFP4_ERR_INVALID_ARG;
  const int mode = g_w4a16_kernel.load();
  const bool warp_mma = mode == 1 || (mode == 0 && M_total <= kWarpMmaMaxRowsPerExpert * (int64_t)E);
  if (warp_mma)
    return w4a16_mma::launch(x, ld_x, x_rows, row_index, b_q, b_sf, b_gs, expert_offsets, E, M_total, N, K, y,
                             out_dtype, swiglu, workspace, dev_status, stream);
  return launch_tc(x, ld_x, x_rows, row_index, b_q, b_sf, b_gs, expert_offsets, E, M_total, N, K, y, out_dtype, swiglu,
                   workspace, dev_status, stream);
}
