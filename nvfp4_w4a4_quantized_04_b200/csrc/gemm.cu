// Block-scaled FP4 x FP4 grouped GEMM on the 5th-generation tensor cores (sm_100a).
//
// What it computes: for every routed expert e, Y_e = (a_gs[e] * b_gs[e]) *
// X_e W_e^T with X_e the expert's packed NVFP4 activations and W_e its packed
// NVFP4 weights, FP32 accumulation -- the W4A4 routed-expert projections of the
// "Qwen3.8-Flash-Next-NVFP4" page (gate_up_proj / down_proj) on the native
// 4-bit tensor-core path that the "DeepSeek-V4.1-Flash-NVFP4" page's
// "why NVFP4" section describes.
//
// Design (B200):
//  * tcgen05.mma.cta_group::1.kind::mxf4nvf4.block_scale.scale_vec::4X: E2M1
//    operands straight from shared memory, E4M3 scales per 16 elements from
//    tensor memory, FP32 accumulator in tensor memory.
//  * Swap-AB: the MMA's M side (128) walks weight rows, the N side (16..192,
//    step 16) walks the tokens of one expert, so a group of m tokens costs
//    roundup(m,16) MMA columns instead of a 128-row tile.  Experts with more
//    than 192 tokens are cut into equal chunks on 64-row boundaries.
//  * Operands are staged by TMA (128-byte swizzle, K-major, 256 elements of K
//    per stage): the weight tile by one 128-row box, the token tile by at most
//    two boxes (128/64/32 rows); the per-16 scales arrive by bulk copy in the
//    tensor-core atom layout (512-byte atoms of 128 rows x 4 scales).
//  * Scale factors reach tensor memory through four helper warps (ld.shared +
//    tcgen05.st, one lane quadrant each, double-buffered), not tcgen05.cp
//    from the MMA thread: on B200 each scale copy costs the MMA issuer about
//    as much as an MMA, and the MoE tiles need 8-12 of them per K stage.
//  * Persistent grid (one CTA per SM), warp-specialised: warp 0 loads weights
//    and scales, warp 10 loads tokens, warp 1 issues MMAs, warps 6..9 write
//    scales to tensor memory, warps 2..5 drain the accumulator (tcgen05.ld)
//    and store Y.  A 4-stage mbarrier ring links loads and MMA; the two
//    accumulators (2 x 192 columns) are double-buffered so the epilogue of one
//    tile overlaps the main loop of the next.
//  * Every mbarrier wait is bounded: past the budget the kernel records
//    NVFP4_ERR_TIMEOUT, every role leaves its loop, outstanding copies and
//    MMAs are drained (again bounded) and tensor memory is freed.
//  * No cluster multicast anywhere.
#include <cuda.h>
#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <cudaTypedefs.h>
#include <stdint.h>

#include "common.cuh"

namespace nvfp4 {
namespace gemm {

constexpr int BM = 128;                 // weight rows per tile (MMA M)
constexpr int BN = 192;                 // max tokens per tile (MMA N)
constexpr int BK = 256;                 // K elements per stage = 128 bytes of codes
constexpr int STAGES = 4;
constexpr int W_STAGE = BM * 128;       // 16 KB
constexpr int X_STAGE = BN * 128;       // 24 KB
constexpr int SFW_STAGE = 2048;         // 128 rows x 16 scales (4 atoms)
constexpr int SFX_STAGE = 4096;         // up to 2 row blocks x 4 atoms
constexpr int OFF_W = 0;
constexpr int OFF_X = OFF_W + STAGES * W_STAGE;
constexpr int OFF_SFW = OFF_X + STAGES * X_STAGE;
constexpr int OFF_SFX = OFF_SFW + STAGES * SFW_STAGE;
constexpr int EPI_WARP_BYTES = 32 * 32 * 4;                   // 32 tokens x 32 columns, fp32
constexpr int OFF_EPI = OFF_SFX + STAGES * SFX_STAGE;        // epilogue staging, one slab per warp
constexpr int OFF_BAR = OFF_EPI + 4 * EPI_WARP_BYTES;        // 8-byte mbarriers
// full[S], empty[S], sf_full[2], acc_full[2], acc_empty[2], drain
constexpr int NUM_BARS = 2 * STAGES + 2 + 2 + 2 + 1;
constexpr int OFF_MISC = OFF_BAR + NUM_BARS * 8;              // tmem base, abort flag
constexpr int OFF_GROUPS = OFF_MISC + 16;                     // off / slot / tile arrays
constexpr int kMaxExperts = 1024;
constexpr int NUM_WARPS = 11;
constexpr int NUM_THREADS = NUM_WARPS * 32;
constexpr int SMEM_BYTES = OFF_GROUPS + 3 * (kMaxExperts + 1) * 4 + 2 * NUM_WARPS * 4 + 1024;  // + scan scratch, +1024 for alignment
constexpr uint32_t TMEM_COLS = 512;
constexpr uint32_t TMEM_ACC_STRIDE = BN;       // accumulator b at column b*192
constexpr uint32_t TMEM_SF = 2 * BN;           // scale buffers at 384 and 448
constexpr uint32_t TMEM_SF_STRIDE = 64;        // per buffer: W scales 16 cols, token scales 32 cols
constexpr long long kWaitBudgetCycles = 4000000000LL;   // ~2 s at 2 GHz

// warp roles (warps 2..5: epilogue, lane quadrants 2,3,0,1)
constexpr int W_PRODUCER = 0;     // weights + scales
constexpr int W_MMA = 1;
constexpr int W_SF0 = 6;          // 6..9: scale factors smem -> tensor memory (quadrants 2,3,0,1)
constexpr int W_XLOAD = 10;       // token tiles

static_assert(SMEM_BYTES <= 232448, "shared memory budget");
static_assert(TMEM_SF + 2 * TMEM_SF_STRIDE <= TMEM_COLS, "tensor memory budget");

// ------------------------------------------------------------------ PTX wrappers
__device__ __forceinline__ uint32_t smem_u32(const void *p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" :: "r"(bar), "r"(count) : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
  asm volatile("{ .reg .b64 st; mbarrier.arrive.shared::cta.b64 st, [%0]; }" :: "r"(bar) : "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint32_t bar, uint32_t bytes) {
  asm volatile("{ .reg .b64 st; mbarrier.arrive.expect_tx.shared::cta.b64 st, [%0], %1; }"
               :: "r"(bar), "r"(bytes) : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile("{ .reg .pred p; mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2; selp.u32 %0, 1, 0, p; }"
               : "=r"(ok) : "r"(bar), "r"(parity) : "memory");
  return ok != 0;
}

// Bounded wait.  Returns false (and raises the CTA abort flag plus a
// TIMEOUT status) if the phase did not complete within the budget, or if
// another role has already aborted.
__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity, volatile int *abort_flag,
                                          int32_t *dev_status) {
  if (mbar_try_wait(bar, parity)) return true;
  const long long t0 = clock64();
  while (true) {
    if (mbar_try_wait(bar, parity)) return true;
    if (*abort_flag) return false;
    if (clock64() - t0 > kWaitBudgetCycles) {
      *abort_flag = 1;
      report(dev_status, NVFP4_ERR_TIMEOUT);
      return false;
    }
  }
}

// Warp-wide bounded wait: every lane waits, the verdict is made uniform so
// that no .sync.aligned tcgen05 instruction ever runs on a partial warp.
__device__ __forceinline__ bool mbar_wait_warp(uint32_t bar, uint32_t parity, volatile int *abort_flag,
                                               int32_t *dev_status) {
  const bool ok = mbar_wait(bar, parity, abort_flag, dev_status);
  return __all_sync(0xffffffffu, ok) != 0;
}

__device__ __forceinline__ void tma_load_2d(uint32_t dst, const CUtensorMap *map, int32_t x, int32_t y,
                                            uint32_t bar, uint64_t policy) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes.L2::cache_hint"
      " [%0], [%1, {%2, %3}], [%4], %5;"
      :: "r"(dst), "l"(map), "r"(x), "r"(y), "r"(bar), "l"(policy) : "memory");
}

__device__ __forceinline__ void bulk_load(uint32_t dst, const void *src, uint32_t bytes, uint32_t bar) {
  asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
               :: "r"(dst), "l"(src), "r"(bytes), "r"(bar) : "memory");
}

__device__ __forceinline__ uint64_t policy_evict_first() {
  uint64_t p;
  asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(p));
  return p;
}
__device__ __forceinline__ uint64_t policy_evict_last() {
  uint64_t p;
  asm volatile("createpolicy.fractional.L2::evict_last.b64 %0, 1.0;" : "=l"(p));
  return p;
}

__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

// K-major operand tile, 128-byte swizzle: rows of 128 bytes, 8-row atoms
// 1024 bytes apart (stride byte offset), version 1 descriptor.
__device__ __forceinline__ uint64_t desc_sw128(uint32_t addr) {
  return (uint64_t)((addr & 0x3FFFFu) >> 4) | ((uint64_t)1 << 16) | ((uint64_t)(1024 >> 4) << 32) |
         ((uint64_t)1 << 46) | ((uint64_t)2 << 61);
}

__device__ __forceinline__ void tc_mma(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                       uint32_t sfa_tmem, uint32_t sfb_tmem, uint32_t accumulate) {
  asm volatile(
      "{\n.reg .pred p;\nsetp.ne.b32 p, %4, 0;\n"
      "tcgen05.mma.cta_group::1.kind::mxf4nvf4.block_scale.scale_vec::4X [%0], %1, %2, %3, [%5], [%6], p;\n}"
      :: "r"(d_tmem), "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate), "r"(sfa_tmem), "r"(sfb_tmem)
      : "memory");
}

__device__ __forceinline__ void tc_commit(uint32_t bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];"
               :: "r"(bar) : "memory");
}

__device__ __forceinline__ void tc_ld32_nowait(uint32_t taddr, uint32_t *r) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
      "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
        "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]),
        "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr));
}

// Instruction descriptor, kind::mxf4nvf4: E2M1 x E2M1, K-major both,
// UE4M3 scales, M = 128, N = n (multiple of 16).
__device__ __forceinline__ uint32_t idesc_mxf4nvf4(uint32_t n) {
  return (1u << 7) | (1u << 10) | ((n >> 3) << 17) | ((uint32_t)(BM >> 4) << 24);
}

__device__ __forceinline__ void tc_st_x4(uint32_t taddr, uint4 v) {
  asm volatile("tcgen05.st.sync.aligned.32x32b.x4.b32 [%0], {%1, %2, %3, %4};"
               :: "r"(taddr), "r"(v.x), "r"(v.y), "r"(v.z), "r"(v.w) : "memory");
}

__device__ __forceinline__ void tc_wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

__device__ __forceinline__ uint4 lds128(uint32_t addr) {
  uint4 v;
  asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(addr));
  return v;
}

// ------------------------------------------------------------------ tile map
// Tiles are (expert, 128-row weight block, token chunk), weight-block-major
// inside an expert so that the chunks of one weight block run on adjacent
// CTAs.  An expert with m tokens is cut into ceil(m/192) chunks of equal size
// rounded up to 64, so every chunk starts on a 64-row boundary of the expert's
// 128-aligned slot: its scale atoms start at row (start & ~127) and the MMA
// reads them from tensor-memory column offset (start & 127)/32 (0 or 2).
struct Tile {
  int e;          // expert
  int w_row0;     // first weight row (over E*N rows)
  int n_col0;     // first output column
  int x_row0;     // first activation row (slot space)
  int y_row0;     // first output row
  int n_valid;    // tokens in this tile (1..192)
};

__device__ __forceinline__ int chunks_of(int m) { return (m + BN - 1) / BN; }

// With the SwiGLU epilogue the fused gate_up weight is stored in 32-row
// groups (16 gate rows, then the 16 matching up rows), so a 128-row weight
// tile covers the 64 h columns starting at n_col0 = 64*mt.
template <bool kSwiglu>
__device__ __forceinline__ Tile decode_tile(int t, const int32_t *s_off, const int32_t *s_slot,
                                            const int32_t *s_tile, int E, int N) {
  Tile T;
  const int e = upper_group(s_tile, E, t);
  const int m_e = s_off[e + 1] - s_off[e];
  const int nch = chunks_of(m_e);
  const int csz = ((m_e + nch - 1) / nch + 63) & ~63;
  const int local = t - s_tile[e];
  const int mt = local / nch, ch = local - mt * nch;
  const int start = ch * csz;
  T.e = e;
  T.n_col0 = kSwiglu ? mt * (BM / 2) : mt * BM;
  T.w_row0 = e * N + mt * BM;
  T.x_row0 = s_slot[e] + start;
  T.y_row0 = s_off[e] + start;
  T.n_valid = min(csz, m_e - start);
  return T;
}

// ------------------------------------------------------------------ kernel
template <bool kSwiglu, bool kBf16Out>
__global__ void __launch_bounds__(NUM_THREADS, 1) grouped_gemm_kernel(
    const __grid_constant__ CUtensorMap tmap_w,
    const __grid_constant__ CUtensorMap tmap_x128,
    const __grid_constant__ CUtensorMap tmap_x64, const __grid_constant__ CUtensorMap tmap_x32,
    const uint8_t *__restrict__ w_sf, const uint8_t *__restrict__ x_sf,
    const float *__restrict__ w_gs, const float *__restrict__ x_gs,
    const int32_t *__restrict__ expert_offsets, int E, int M_total, int N, int K,
    void *__restrict__ y, float *__restrict__ amax_out, int32_t *dev_status) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
  const uint32_t sbase = smem_u32(smem);
  const uint32_t bar_full = sbase + OFF_BAR;              // [STAGES], count 2 (two producer threads)
  const uint32_t bar_empty = bar_full + 8 * STAGES;       // [STAGES], count 1 (MMA commit)
  const uint32_t bar_sf_full = bar_empty + 8 * STAGES;    // [2], count 128 (scale warps)
  const uint32_t bar_acc_full = bar_sf_full + 16;         // [2], count 1 (MMA commit)
  const uint32_t bar_acc_empty = bar_acc_full + 16;       // [2], count 128 (epilogue threads)
  const uint32_t bar_drain = bar_acc_empty + 16;
  volatile uint32_t *tmem_holder = reinterpret_cast<volatile uint32_t *>(smem + OFF_MISC);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + OFF_MISC + 4);
  int32_t *s_off = reinterpret_cast<int32_t *>(smem + OFF_GROUPS);
  int32_t *s_slot = s_off + (kMaxExperts + 1);
  int32_t *s_tile = s_slot + (kMaxExperts + 1);
  int32_t *s_scratch = s_tile + (kMaxExperts + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int n_mtiles = N / BM;
  const int ksteps = K / BK;

  // ---- per-CTA set-up: expert table, barriers, tensor memory
  if (expert_offsets) {
    for (int i = threadIdx.x; i <= E; i += NUM_THREADS) s_off[i] = expert_offsets[i];
  } else if (threadIdx.x == 0) {
    s_off[0] = 0;
    s_off[1] = M_total;
  }
  if (threadIdx.x == 0) {
    *abort_flag = 0;
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(bar_full + 8 * s, 2);
      mbar_init(bar_empty + 8 * s, 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(bar_sf_full + 8 * b, 128);
      mbar_init(bar_acc_full + 8 * b, 1);
      mbar_init(bar_acc_empty + 8 * b, 128);
    }
    mbar_init(bar_drain, 1);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == W_MMA) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;"
                 :: "r"(smem_u32((const void *)tmem_holder)), "r"(TMEM_COLS) : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  __syncthreads();
  {
    // slot starts (128-aligned groups) and tile starts: block-wide exclusive scans
    const int per = (E + NUM_THREADS - 1) / NUM_THREADS;
    const int e0 = min(E, (int)threadIdx.x * per), e1 = min(E, e0 + per);
    int32_t ls = 0, lt = 0;
    for (int e = e0; e < e1; ++e) {
      const int32_t m = s_off[e + 1] - s_off[e];
      ls += (m + kSlotAlign - 1) / kSlotAlign * kSlotAlign;
      lt += n_mtiles * chunks_of(m);
    }
    int32_t is = ls, it = lt;
#pragma unroll
    for (int d = 1; d < 32; d <<= 1) {
      const int32_t a = __shfl_up_sync(0xffffffffu, is, d), b = __shfl_up_sync(0xffffffffu, it, d);
      if (lane >= d) { is += a; it += b; }
    }
    if (lane == 31) { s_scratch[warp] = is; s_scratch[NUM_WARPS + warp] = it; }
    __syncthreads();
    if (threadIdx.x == 0) {
      int32_t as = 0, at = 0;
      for (int w = 0; w < NUM_WARPS; ++w) {
        const int32_t vs = s_scratch[w], vt = s_scratch[NUM_WARPS + w];
        s_scratch[w] = as; s_scratch[NUM_WARPS + w] = at;
        as += vs; at += vt;
      }
    }
    __syncthreads();
    int32_t rs = s_scratch[warp] + is - ls, rt = s_scratch[NUM_WARPS + warp] + it - lt;
    for (int e = e0; e < e1; ++e) {
      const int32_t m = s_off[e + 1] - s_off[e];
      s_slot[e] = rs;
      s_tile[e] = rt;
      rs += (m + kSlotAlign - 1) / kSlotAlign * kSlotAlign;
      rt += n_mtiles * chunks_of(m);
    }
    if (e1 == E && e0 < e1) { s_slot[E] = rs; s_tile[E] = rt; }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_holder;
  const int total_tiles = s_tile[E];
  const int64_t sf_row_stride = (int64_t)(K / 64) * 512;   // bytes per 128-row block of scales

  if (warp == W_PRODUCER || warp == W_XLOAD) {
    // ================================================================ TMA producers
    // warp 0 lane 0: weight tile and all scale blocks; warp 10 lane 0: the
    // token tile boxes.  Each arms the stage's full barrier with its own
    // bytes, so the two issue streams (about 65 ns per copy instruction) run
    // in parallel.
    if (lane == 0) {
      const bool is_w = warp == W_PRODUCER;
      const uint64_t pol = is_w ? policy_evict_first() : policy_evict_last();
      int stage = 0;
      uint32_t phase = 0;
      bool armed[STAGES] = {};
      uint32_t armed_parity[STAGES] = {};
      bool ok = true;
      for (int t = blockIdx.x; t < total_tiles && ok; t += gridDim.x) {
        const Tile T = decode_tile<kSwiglu>(t, s_off, s_slot, s_tile, E, N);
        const int rows_ld = (T.n_valid + 31) & ~31;
        const int xr0 = T.x_row0 & ~127;                               // first scale row block
        const int nrb = ((T.x_row0 & 127) + T.n_valid + 127) >> 7;     // 1 or 2
        const uint32_t bytes = is_w ? (uint32_t)(W_STAGE + SFW_STAGE + nrb * 2048)
                                    : (uint32_t)(rows_ld * 128);
        const uint8_t *sfw_tile = w_sf + (int64_t)(T.w_row0 >> 7) * sf_row_stride;
        const uint8_t *sfx_tile = x_sf + (int64_t)(xr0 >> 7) * sf_row_stride;
        for (int ks = 0; ks < ksteps; ++ks) {
          if (!mbar_wait(bar_empty + 8 * stage, phase ^ 1, abort_flag, dev_status)) { ok = false; break; }
          const uint32_t fb = bar_full + 8 * stage;
          mbar_arrive_expect_tx(fb, bytes);
          armed[stage] = true;
          armed_parity[stage] = phase;
          if (is_w) {
            tma_load_2d(sbase + OFF_W + stage * W_STAGE, &tmap_w, ks * 128, T.w_row0, fb, pol);
            bulk_load(sbase + OFF_SFW + stage * SFW_STAGE, sfw_tile + ks * 2048, 2048, fb);
            for (int rb = 0; rb < nrb; ++rb)
              bulk_load(sbase + OFF_SFX + stage * SFX_STAGE + rb * 2048, sfx_tile + rb * sf_row_stride + ks * 2048,
                        2048, fb);
          } else {
            uint32_t dst = sbase + OFF_X + stage * X_STAGE;
            int row = T.x_row0, left = rows_ld;
            if (left >= 128) { tma_load_2d(dst, &tmap_x128, ks * 128, row, fb, pol); dst += 16384; row += 128; left -= 128; }
            if (left >= 64) { tma_load_2d(dst, &tmap_x64, ks * 128, row, fb, pol); dst += 8192; row += 64; left -= 64; }
            if (left >= 32) { tma_load_2d(dst, &tmap_x32, ks * 128, row, fb, pol); }
          }
          if (++stage == STAGES) { stage = 0; phase ^= 1; }
        }
      }
      // Drain: every armed stage's copies must have landed before the CTA exits.
      for (int s = 0; s < STAGES; ++s) {
        if (!armed[s]) continue;
        const long long t0 = clock64();
        while (!mbar_try_wait(bar_full + 8 * s, armed_parity[s]) && clock64() - t0 < kWaitBudgetCycles) {}
      }
    }
  } else if (warp >= W_SF0 && warp < W_SF0 + 4) {
    // ================================================================ scale factors -> TMEM
    // Each warp writes its lane quadrant: lane l of every quadrant gets the 16
    // bytes of atom row l (the scales of rows l, l+32, l+64, l+96), i.e. the
    // replicated 32x128b layout the block-scaled MMA reads.
    const uint32_t lane_base = (uint32_t)((warp & 3) * 32) << 16;
    int stage = 0;
    uint32_t phase = 0;
    uint32_t kiter = 0;                 // global k-step counter (selects the scale buffer)
    bool ok = true;
    for (int t = blockIdx.x; t < total_tiles && ok; t += gridDim.x) {
      const Tile T = decode_tile<kSwiglu>(t, s_off, s_slot, s_tile, E, N);
      const int nrb = ((T.x_row0 & 127) + T.n_valid + 127) >> 7;
      for (int ks = 0; ks < ksteps; ++ks, ++kiter) {
        const uint32_t sb = kiter & 1;
        // buffer sb was last read by the MMAs of k-step kiter-2: wait for them
        if (kiter >= 2) {
          const uint32_t prev = kiter - 2;
          if (!mbar_wait_warp(bar_empty + 8 * (prev % STAGES), (prev / STAGES) & 1, abort_flag, dev_status)) {
            ok = false; break;
          }
        }
        if (!mbar_wait_warp(bar_full + 8 * stage, phase, abort_flag, dev_status)) { ok = false; break; }
        tc_fence_after();
        const uint32_t tcol = tmem_base + lane_base + TMEM_SF + sb * TMEM_SF_STRIDE;
        const uint32_t sfw_addr = sbase + OFF_SFW + stage * SFW_STAGE + lane * 16;
        const uint32_t sfx_addr = sbase + OFF_SFX + stage * SFX_STAGE + lane * 16;
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) tc_st_x4(tcol + kk * 4, lds128(sfw_addr + kk * 512));
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) tc_st_x4(tcol + 16 + kk * 8, lds128(sfx_addr + kk * 512));
        if (nrb > 1) {
#pragma unroll
          for (int kk = 0; kk < 4; ++kk) tc_st_x4(tcol + 16 + kk * 8 + 4, lds128(sfx_addr + 2048 + kk * 512));
        }
        tc_wait_st();
        tc_fence_before();
        mbar_arrive(bar_sf_full + 8 * sb);
        if (++stage == STAGES) { stage = 0; phase ^= 1; }
      }
    }
  } else if (warp == W_MMA) {
    // ================================================================ MMA issuer
    int stage = 0;
    uint32_t phase = 0;
    uint32_t kiter = 0, titer = 0;
    bool ok = true;
    for (int t = blockIdx.x; t < total_tiles && ok; t += gridDim.x, ++titer) {
      const Tile T = decode_tile<kSwiglu>(t, s_off, s_slot, s_tile, E, N);
      const uint32_t n_mma = (T.n_valid + 15) & ~15;
      const uint32_t idesc = idesc_mxf4nvf4(n_mma);
      const uint32_t xoff = (uint32_t)(T.x_row0 & 127) >> 5;      // 0 or 2 columns
      const uint32_t ab = titer & 1;
      const uint32_t t_acc = tmem_base + ab * TMEM_ACC_STRIDE;
      if (!mbar_wait_warp(bar_acc_empty + 8 * ab, ((titer >> 1) & 1) ^ 1, abort_flag, dev_status)) { ok = false; break; }
      tc_fence_after();
      for (int ks = 0; ks < ksteps; ++ks, ++kiter) {
        const uint32_t sb = kiter & 1;
        if (!mbar_wait_warp(bar_full + 8 * stage, phase, abort_flag, dev_status)) { ok = false; break; }
        if (!mbar_wait_warp(bar_sf_full + 8 * sb, (kiter >> 1) & 1, abort_flag, dev_status)) { ok = false; break; }
        tc_fence_after();
        if (lane == 0) {
          const uint32_t t_sf = tmem_base + TMEM_SF + sb * TMEM_SF_STRIDE;
          const uint64_t dw = desc_sw128(sbase + OFF_W + stage * W_STAGE);
          const uint64_t dx = desc_sw128(sbase + OFF_X + stage * X_STAGE);
#pragma unroll
          for (int kk = 0; kk < 4; ++kk) {
            // +32 bytes of K per MMA: +2 in the descriptor's 16-byte address field
            tc_mma(t_acc, dw + 2 * kk, dx + 2 * kk, idesc, t_sf + kk * 4, t_sf + 16 + kk * 8 + xoff,
                   (ks > 0 || kk > 0) ? 1u : 0u);
          }
          tc_commit(bar_empty + 8 * stage);
        }
        __syncwarp();
        if (++stage == STAGES) { stage = 0; phase ^= 1; }
      }
      if (!ok) break;
      if (lane == 0) tc_commit(bar_acc_full + 8 * ab);
      __syncwarp();
    }
    // Drain: all MMAs this thread issued complete before TMEM is freed.
    if (lane == 0) {
      tc_commit(bar_drain);
      const long long t0 = clock64();
      while (!mbar_try_wait(bar_drain, 0) && clock64() - t0 < kWaitBudgetCycles) {}
    }
    __syncwarp();
  } else {
    // ================================================================ epilogue
    const int quad = warp & 3;                    // TMEM lane quadrant of this warp
    const uint32_t lane_base = (uint32_t)(quad * 32) << 16;
    const uint32_t epi = sbase + OFF_EPI + (warp - 2) * EPI_WARP_BYTES;
    uint32_t titer = 0;
    for (int t = blockIdx.x; t < total_tiles; t += gridDim.x, ++titer) {
      const Tile T = decode_tile<kSwiglu>(t, s_off, s_slot, s_tile, E, N);
      const uint32_t ab = titer & 1;
      if (!mbar_wait_warp(bar_acc_full + 8 * ab, (titer >> 1) & 1, abort_flag, dev_status)) break;
      tc_fence_after();
      const float alpha = __fmul_rn(x_gs[T.e], w_gs[T.e]);
      const uint32_t tacc = tmem_base + lane_base + ab * TMEM_ACC_STRIDE;
      uint32_t hmax = 0;                           // SwiGLU: max |h| bits of this lane
      for (int c0 = 0; c0 < T.n_valid; c0 += 64) {
        uint32_t r[64];
        tc_ld32_nowait(tacc + (uint32_t)c0, r);
        if (c0 + 32 < T.n_valid) tc_ld32_nowait(tacc + (uint32_t)c0 + 32, r + 32);
        asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
        if (c0 + 64 >= T.n_valid) {
          // the whole accumulator has been read: hand it back to the MMA warp
          tc_fence_before();
          mbar_arrive(bar_acc_empty + 8 * ab);
        }
        if (kSwiglu) {
          // TMEM lane l of quadrant q holds h column 16q + (l & 15): the gate
          // row for l < 16, the matching up row for l >= 16.  One xor-16
          // shuffle per token pair gives each lane both operands; the gate
          // lane finishes tokens 0..15 of the 32, the up lane tokens 16..31.
          // h = bf16(silu(g) * u) with g, u = alpha*acc in fp32 (silu through
          // the fast exp and divide intrinsics: a few fp32 ulps, far below the
          // bf16 rounding of h).  The 32x16 h block is staged in shared memory
          // (the two token halves 576 bytes apart, so the halves' stores hit
          // disjoint banks) and written as 32-byte row segments.
          const bool gate_lane = lane < 16;
          const uint32_t half = gate_lane ? 0u : 576u;
#pragma unroll
          for (int sub = 0; sub < 2; ++sub) {
            const int tok0 = c0 + sub * 32;
            if (tok0 >= T.n_valid) break;
            const int rows_here = min(32, T.n_valid - tok0);
            const int my0 = gate_lane ? 0 : 16;
#pragma unroll
            for (int j = 0; j < 16; ++j) {
              const uint32_t mine = gate_lane ? r[sub * 32 + 16 + j] : r[sub * 32 + j];
              const uint32_t other = __shfl_xor_sync(0xffffffffu, mine, 16);
              const float gv = __fmul_rn(__uint_as_float(gate_lane ? r[sub * 32 + j] : other), alpha);
              const float uv = __fmul_rn(__uint_as_float(gate_lane ? other : r[sub * 32 + 16 + j]), alpha);
              const float sv = __fdividef(gv, 1.0f + __expf(-gv));
              const __nv_bfloat16 hv = __float2bfloat16_rn(__fmul_rn(sv, uv));
              const uint16_t hb = *reinterpret_cast<const uint16_t *>(&hv);
              if (my0 + j < rows_here) hmax = max(hmax, (uint32_t)(hb & 0x7FFFu));
              asm volatile("st.shared.b16 [%0], %1;" :: "r"(epi + half + j * 32 + (lane & 15) * 2), "h"(hb) : "memory");
            }
            __syncwarp();
            const int NH = N / 2;
            __nv_bfloat16 *hbase = reinterpret_cast<__nv_bfloat16 *>(y) + (int64_t)(T.y_row0 + tok0) * NH +
                                   T.n_col0 + quad * 16;
#pragma unroll
            for (int it = 0; it < 2; ++it) {
              const int row = it * 16 + (lane >> 1), chunk = lane & 1;
              if (row < rows_here) {
                const uint4 v = lds128(epi + (row >> 4) * 576 + (row & 15) * 32 + chunk * 16);
                *reinterpret_cast<uint4 *>(hbase + (int64_t)row * NH + chunk * 8) = v;
              }
            }
            __syncwarp();
          }
          continue;
        }
        // Stage each 32-token x 32-column block in shared memory (this lane
        // owns one weight column), then write whole 64/128-byte row segments
        // of Y with 16-byte vector stores.
#pragma unroll
        for (int sub = 0; sub < 2; ++sub) {
          const int tok0 = c0 + sub * 32;
          if (tok0 >= T.n_valid) break;
          const int rows_here = min(32, T.n_valid - tok0);
          if (kBf16Out) {
#pragma unroll
            for (int i = 0; i < 32; ++i) {
              const __nv_bfloat16 hv = __float2bfloat16_rn(__fmul_rn(__uint_as_float(r[sub * 32 + i]), alpha));
              asm volatile("st.shared.b16 [%0], %1;" :: "r"(epi + i * 64 + lane * 2),
                           "h"(*reinterpret_cast<const uint16_t *>(&hv)) : "memory");
            }
            __syncwarp();
            __nv_bfloat16 *ybase = reinterpret_cast<__nv_bfloat16 *>(y) + (int64_t)(T.y_row0 + tok0) * N + T.n_col0 + quad * 32;
#pragma unroll
            for (int it = 0; it < 4; ++it) {
              const int row = it * 8 + (lane >> 2), chunk = lane & 3;
              if (row < rows_here) {
                const uint4 v = lds128(epi + row * 64 + chunk * 16);
                *reinterpret_cast<uint4 *>(ybase + (int64_t)row * N + chunk * 8) = v;
              }
            }
          } else {
#pragma unroll
            for (int i = 0; i < 32; ++i) {
              const float fv = __fmul_rn(__uint_as_float(r[sub * 32 + i]), alpha);
              asm volatile("st.shared.b32 [%0], %1;" :: "r"(epi + i * 128 + lane * 4), "f"(fv) : "memory");
            }
            __syncwarp();
            float *ybase = reinterpret_cast<float *>(y) + (int64_t)(T.y_row0 + tok0) * N + T.n_col0 + quad * 32;
#pragma unroll
            for (int it = 0; it < 8; ++it) {
              const int row = it * 4 + (lane >> 3), chunk = lane & 7;
              if (row < rows_here) {
                const uint4 v = lds128(epi + row * 128 + chunk * 16);
                *reinterpret_cast<uint4 *>(ybase + (int64_t)row * N + chunk * 4) = v;
              }
            }
          }
          __syncwarp();
        }
      }
      if (kSwiglu) {
#pragma unroll
        for (int d = 16; d > 0; d >>= 1) hmax = max(hmax, __shfl_xor_sync(0xffffffffu, hmax, d));
        if (lane == 0 && hmax) atomicMax(reinterpret_cast<uint32_t *>(amax_out) + T.e, hmax << 16);
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == W_MMA) {
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" :: "r"(tmem_base), "r"(TMEM_COLS) : "memory");
  }
}

}  // namespace gemm
}  // namespace nvfp4

// ====================================================================== host side
using namespace nvfp4;

namespace {

PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;

bool get_encoder() {
  if (g_encode) return true;
  void *fn = nullptr;
  cudaDriverEntryPointQueryResult qres;
  if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &qres) != cudaSuccess ||
      qres != cudaDriverEntryPointSuccess || !fn)
    return false;
  g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
  return true;
}

// 2-D uint8 view [rows, row_bytes] with a {128 bytes, box_rows} box, 128-byte swizzle.
bool make_map(CUtensorMap *map, const void *base, uint64_t rows, uint64_t row_bytes, uint32_t box_rows) {
  cuuint64_t dims[2] = {row_bytes, rows};
  cuuint64_t strides[1] = {row_bytes};
  cuuint32_t box[2] = {128, box_rows};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = g_encode(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void *>(base), dims, strides, box, estr,
                        CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                        CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

int g_sms = 0;
bool g_attr_set[3] = {false, false, false};

}  // namespace

extern "C" nvfp4_status nvfp4_grouped_gemm(const uint8_t *a_q, const uint8_t *a_sf, const float *a_gs,
                                           const uint8_t *b_q, const uint8_t *b_sf, const float *b_gs,
                                           const int32_t *expert_offsets, int num_experts, int64_t M_total,
                                           int64_t N, int64_t K, void *y, nvfp4_out_dtype out_dtype,
                                           nvfp4_epilogue epi, float *amax_out, void *workspace,
                                           int32_t *dev_status, cudaStream_t stream) {
  (void)workspace;
  if (epi != NVFP4_EPI_NONE && epi != NVFP4_EPI_SWIGLU) return NVFP4_ERR_INVALID_ARG;
  if (out_dtype != NVFP4_OUT_F32 && out_dtype != NVFP4_OUT_BF16) return NVFP4_ERR_INVALID_ARG;
  const bool swiglu = epi == NVFP4_EPI_SWIGLU;
  if (swiglu && (out_dtype != NVFP4_OUT_BF16 || !amax_out)) return NVFP4_ERR_INVALID_ARG;
  const int E = expert_offsets ? num_experts : 1;
  if (E < 1 || E > gemm::kMaxExperts) return NVFP4_ERR_UNSUPPORTED_SHAPE;
  if (M_total < 0 || N <= 0 || K <= 0) return NVFP4_ERR_INVALID_ARG;
  if (N % 128 != 0 || K % 256 != 0) return NVFP4_ERR_UNSUPPORTED_SHAPE;
  if ((int64_t)E * N > ((int64_t)1 << 31) - 1 || M_total > ((int64_t)1 << 30)) return NVFP4_ERR_UNSUPPORTED_SHAPE;
  if (M_total == 0) return NVFP4_OK;
  if (!a_q || !a_sf || !a_gs || !b_q || !b_sf || !b_gs || !y) return NVFP4_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(a_q) | reinterpret_cast<uintptr_t>(b_q) | reinterpret_cast<uintptr_t>(a_sf) |
       reinterpret_cast<uintptr_t>(b_sf) | reinterpret_cast<uintptr_t>(y)) & 15u)
    return NVFP4_ERR_INVALID_ARG;
  if (!get_encoder()) return NVFP4_ERR_CUDA;
  const int64_t x_rows = nvfp4_padded_rows_bound(M_total, E);
  CUtensorMap tw, tx128, tx64, tx32;
  if (!make_map(&tw, b_q, (uint64_t)E * N, (uint64_t)K / 2, 128)) return NVFP4_ERR_CUDA;
  if (!make_map(&tx128, a_q, (uint64_t)x_rows, (uint64_t)K / 2, 128)) return NVFP4_ERR_CUDA;
  if (!make_map(&tx64, a_q, (uint64_t)x_rows, (uint64_t)K / 2, 64)) return NVFP4_ERR_CUDA;
  if (!make_map(&tx32, a_q, (uint64_t)x_rows, (uint64_t)K / 2, 32)) return NVFP4_ERR_CUDA;
  if (g_sms == 0) {
    int dev = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&g_sms, cudaDevAttrMultiProcessorCount, dev);
    if (g_sms <= 0) g_sms = 148;
  }
  const int variant = swiglu ? 2 : (out_dtype == NVFP4_OUT_BF16 ? 1 : 0);
  auto kern = variant == 2 ? gemm::grouped_gemm_kernel<true, true>
                           : (variant == 1 ? gemm::grouped_gemm_kernel<false, true> : gemm::grouped_gemm_kernel<false, false>);
  if (!g_attr_set[variant]) {
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, gemm::SMEM_BYTES) != cudaSuccess)
      return NVFP4_ERR_CUDA;
    g_attr_set[variant] = true;
  }
  kern<<<g_sms, gemm::NUM_THREADS, gemm::SMEM_BYTES, stream>>>(tw, tx128, tx64, tx32, b_sf, a_sf, b_gs, a_gs,
                                                               expert_offsets, E, (int)M_total, (int)N, (int)K, y,
                                                               amax_out, dev_status);
  return cudaGetLastError() == cudaSuccess ? NVFP4_OK : NVFP4_ERR_CUDA;
}
