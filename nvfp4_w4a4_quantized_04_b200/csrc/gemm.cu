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
//    and store Y.  Two mbarrier rings (4 weight stages, 4 token stages) link
//    loads and MMA; the two
//    accumulators (2 x 192 columns) are double-buffered so the epilogue of one
//    tile overlaps the main loop of the next.
//  * Every mbarrier wait is bounded: past the budget the kernel records
//    NVFP4_ERR_TIMEOUT, every role leaves its loop, outstanding copies and
//    MMAs are drained (again bounded) and tensor memory is freed.
//  * No cluster multicast anywhere.
#include <atomic>

#include "gemm_common.cuh"
#include "host_util.cuh"

namespace nvfp4 {
namespace gemm {

// Ring layout of the one-CTA kernel: the weight ring (tile + scales) and the
// token ring (tile + scales) have separate full/empty barriers.
constexpr int W_STAGES = 4;
constexpr int X_STAGES = 4;
constexpr int X_STAGE = BN * 128;       // 24 KB
constexpr int OFF_W = 0;
constexpr int OFF_X = OFF_W + W_STAGES * W_STAGE;
constexpr int OFF_SFW = OFF_X + X_STAGES * X_STAGE;
constexpr int OFF_SFX = OFF_SFW + W_STAGES * SFW_STAGE;
constexpr int OFF_EPI = OFF_SFX + X_STAGES * SFX_STAGE;      // epilogue staging, one slab per warp
constexpr int OFF_BAR = OFF_EPI + 4 * EPI_WARP_BYTES;        // 8-byte mbarriers
// wfull[WS], wempty[WS], xfull[XS], xempty[XS], sf_full[2], acc_full[2], acc_empty[2], drain
constexpr int NUM_BARS = 2 * W_STAGES + 2 * X_STAGES + 2 + 2 + 2 + 1;
constexpr int OFF_MISC = OFF_BAR + NUM_BARS * 8;              // tmem base, abort flag
constexpr int OFF_GROUPS = OFF_MISC + 16;                     // off / slot / tile arrays
constexpr int SMEM_BYTES = OFF_GROUPS + GROUP_TABLE_BYTES + 1024;   // +1024 for alignment
static_assert(SMEM_BYTES <= 232448, "shared memory budget");

// ------------------------------------------------------------------ kernel
// kMx: MXFP4 operands (kind::mxf4, one UE8M0 scale per 32 elements, no
// global scales); otherwise NVFP4 (kind::mxf4nvf4, E4M3 per 16 elements).
template <bool kSwiglu, bool kBf16Out, bool kQuantH = false, bool kMx = false>
__global__ void __launch_bounds__(NUM_THREADS, 1) grouped_gemm_kernel(
    const __grid_constant__ CUtensorMap tmap_w,
    const __grid_constant__ CUtensorMap tmap_x128,
    const __grid_constant__ CUtensorMap tmap_x64, const __grid_constant__ CUtensorMap tmap_x32,
    const uint8_t *__restrict__ w_sf, const uint8_t *__restrict__ x_sf,
    const float *__restrict__ w_gs, const float *__restrict__ x_gs,
    const int32_t *__restrict__ expert_offsets, int E, int M_total, int N, int K,
    void *__restrict__ y, float *__restrict__ amax_out, int32_t *dev_status, HQuantOut hq) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
  const uint32_t sbase = smem_u32(smem);
  const uint32_t bar_wfull = sbase + OFF_BAR;             // [W_STAGES], count 1 (weight producer)
  const uint32_t bar_wempty = bar_wfull + 8 * W_STAGES;   // [W_STAGES], count 1 (MMA commit)
  const uint32_t bar_xfull = bar_wempty + 8 * W_STAGES;   // [X_STAGES], count 1 (token producer)
  const uint32_t bar_xempty = bar_xfull + 8 * X_STAGES;   // [X_STAGES], count 1 (MMA commit)
  const uint32_t bar_sf_full = bar_xempty + 8 * X_STAGES; // [2], count 128 (scale warps)
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

  // ---- per-CTA set-up: barriers, tensor memory, expert tables
  if (threadIdx.x == 0) {
    *abort_flag = 0;
    for (int s = 0; s < W_STAGES; ++s) {
      mbar_init(bar_wfull + 8 * s, 1);
      mbar_init(bar_wempty + 8 * s, 1);
    }
    for (int s = 0; s < X_STAGES; ++s) {
      mbar_init(bar_xfull + 8 * s, 1);
      mbar_init(bar_xempty + 8 * s, 1);
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
  build_tile_tables(expert_offsets, E, M_total, n_mtiles, s_off, s_slot, s_tile, s_scratch, dev_status);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_holder;
  const int total_tiles = s_tile[E];
  // bytes per 128-row block of scales, and scale bytes per K stage of one row block
  const int64_t sf_row_stride = (int64_t)(K / (kMx ? 128 : 64)) * 512;
  constexpr uint32_t kSfStage = kMx ? 1024u : 2048u;

  if (warp == W_PRODUCER || warp == W_XLOAD) {
    // ================================================================ TMA producers
    // warp 0 lane 0: the weight ring (weight tile + weight scales); warp 10
    // lane 0: the token ring (token scales + token tile boxes).  The two
    // issue streams (about 65 ns per copy instruction) run in parallel.
    if (lane == 0) {
      const bool is_w = warp == W_PRODUCER;
      const uint64_t pol = is_w ? policy_evict_first() : policy_evict_last();
      const int nstages = is_w ? W_STAGES : X_STAGES;
      const uint32_t bar_full = is_w ? bar_wfull : bar_xfull, bar_empty = is_w ? bar_wempty : bar_xempty;
      int stage = 0;
      uint32_t phase = 0;
      constexpr int kMaxStages = W_STAGES > X_STAGES ? W_STAGES : X_STAGES;
      bool armed[kMaxStages] = {};
      uint32_t armed_parity[kMaxStages] = {};
      bool ok = true;
      for (int t = blockIdx.x; t < total_tiles && ok; t += gridDim.x) {
        const Tile T = decode_tile<kSwiglu>(t, s_off, s_slot, s_tile, E, N, BM, 0);
        const int rows_ld = (T.n_valid + 31) & ~31;
        const int xr0 = T.x_row0 & ~127;                               // first scale row block
        const int nrb = ((T.x_row0 & 127) + T.n_valid + 127) >> 7;     // 1 or 2
        const uint32_t bytes = is_w ? (uint32_t)(W_STAGE + kSfStage) : (uint32_t)(rows_ld * 128 + nrb * kSfStage);
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
            bulk_load(sbase + OFF_SFW + stage * SFW_STAGE, sfw_tile + ks * kSfStage, kSfStage, fb);
          } else {
            for (int rb = 0; rb < nrb; ++rb)
              bulk_load(sbase + OFF_SFX + stage * SFX_STAGE + rb * 2048, sfx_tile + rb * sf_row_stride + ks * kSfStage,
                        kSfStage, fb);
            uint32_t dst = sbase + OFF_X + stage * X_STAGE;
            int row = T.x_row0, left = rows_ld;
            if (left >= 128) { tma_load_2d(dst, &tmap_x128, ks * 128, row, fb, pol); dst += 16384; row += 128; left -= 128; }
            if (left >= 64) { tma_load_2d(dst, &tmap_x64, ks * 128, row, fb, pol); dst += 8192; row += 64; left -= 64; }
            if (left >= 32) { tma_load_2d(dst, &tmap_x32, ks * 128, row, fb, pol); }
          }
          if (++stage == nstages) { stage = 0; phase ^= 1; }
        }
      }
      // Drain: every armed stage's copies must have landed before the CTA exits.
      for (int s = 0; s < nstages; ++s) {
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
    uint32_t kiter = 0;                 // global k-step counter: ring stages, phases, scale buffer
    bool ok = true;
    for (int t = blockIdx.x; t < total_tiles && ok; t += gridDim.x) {
      const Tile T = decode_tile<kSwiglu>(t, s_off, s_slot, s_tile, E, N, BM, 0);
      const int nrb = ((T.x_row0 & 127) + T.n_valid + 127) >> 7;
      for (int ks = 0; ks < ksteps; ++ks, ++kiter) {
        const uint32_t sb = kiter & 1;
        // buffer sb was last read by the MMAs of k-step kiter-2: wait for them
        if (kiter >= 2) {
          const uint32_t prev = kiter - 2;
          if (!mbar_wait_warp(bar_wempty + 8 * (prev % W_STAGES), (prev / W_STAGES) & 1, abort_flag, dev_status)) {
            ok = false; break;
          }
        }
        const uint32_t sw = kiter % W_STAGES, sx = kiter % X_STAGES;
        if (!mbar_wait_warp(bar_wfull + 8 * sw, (kiter / W_STAGES) & 1, abort_flag, dev_status)) { ok = false; break; }
        if (!mbar_wait_warp(bar_xfull + 8 * sx, (kiter / X_STAGES) & 1, abort_flag, dev_status)) { ok = false; break; }
        tc_fence_after();
        const uint32_t tcol = tmem_base + lane_base + TMEM_SF + sb * TMEM_SF_STRIDE;
        if constexpr (kMx)
          sf_stage_to_tmem_mx(tcol, sbase + OFF_SFW + sw * SFW_STAGE + lane * 16,
                              sbase + OFF_SFX + sx * SFX_STAGE + lane * 16, nrb);
        else
          sf_stage_to_tmem(tcol, sbase + OFF_SFW + sw * SFW_STAGE + lane * 16, sbase + OFF_SFX + sx * SFX_STAGE + lane * 16,
                           nrb);
        tc_fence_before();
        mbar_arrive(bar_sf_full + 8 * sb);
      }
    }
  } else if (warp == W_MMA) {
    // ================================================================ MMA issuer
    uint32_t kiter = 0, titer = 0;
    bool ok = true;
    for (int t = blockIdx.x; t < total_tiles && ok; t += gridDim.x, ++titer) {
      const Tile T = decode_tile<kSwiglu>(t, s_off, s_slot, s_tile, E, N, BM, 0);
      const uint32_t n_mma = (T.n_valid + 15) & ~15;
      const uint32_t idesc = kMx ? idesc_mxf4_ue8m0(BM, n_mma) : idesc_mxf4nvf4(BM, n_mma);
      const uint32_t xoff = (uint32_t)(T.x_row0 & 127) >> 5;      // 0 or 2 columns
      const uint32_t ab = titer & 1;
      const uint32_t t_acc = tmem_base + ab * TMEM_ACC_STRIDE;
      if (!mbar_wait_warp(bar_acc_empty + 8 * ab, ((titer >> 1) & 1) ^ 1, abort_flag, dev_status)) { ok = false; break; }
      tc_fence_after();
      for (int ks = 0; ks < ksteps; ++ks, ++kiter) {
        const uint32_t sb = kiter & 1;
        const uint32_t sw = kiter % W_STAGES, sx = kiter % X_STAGES;
        if (!mbar_wait_warp(bar_wfull + 8 * sw, (kiter / W_STAGES) & 1, abort_flag, dev_status)) { ok = false; break; }
        if (!mbar_wait_warp(bar_xfull + 8 * sx, (kiter / X_STAGES) & 1, abort_flag, dev_status)) { ok = false; break; }
        if (!mbar_wait_warp(bar_sf_full + 8 * sb, (kiter >> 1) & 1, abort_flag, dev_status)) { ok = false; break; }
        tc_fence_after();
        if (lane == 0) {
          const uint32_t t_sf = tmem_base + TMEM_SF + sb * TMEM_SF_STRIDE;
          const uint64_t dw = desc_sw128(sbase + OFF_W + sw * W_STAGE);
          const uint64_t dx = desc_sw128(sbase + OFF_X + sx * X_STAGE);
#pragma unroll
          for (int kk = 0; kk < 4; ++kk) {
            // +32 bytes of K per MMA: +2 in the descriptor's 16-byte address field
            if constexpr (kMx)
              tc_mma_mx(t_acc, dw + 2 * kk, dx + 2 * kk, idesc, t_sf + kk * 4, t_sf + 16 + kk * 8 + xoff,
                        (ks > 0 || kk > 0) ? 1u : 0u);
            else
              tc_mma(t_acc, dw + 2 * kk, dx + 2 * kk, idesc, t_sf + kk * 4, t_sf + 16 + kk * 8 + xoff,
                     (ks > 0 || kk > 0) ? 1u : 0u);
          }
          tc_commit(bar_wempty + 8 * sw);
          tc_commit(bar_xempty + 8 * sx);
        }
        __syncwarp();
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
      const Tile T = decode_tile<kSwiglu>(t, s_off, s_slot, s_tile, E, N, BM, 0);
      const uint32_t ab = titer & 1;
      if (!mbar_wait_warp(bar_acc_full + 8 * ab, (titer >> 1) & 1, abort_flag, dev_status)) break;
      tc_fence_after();
      const float alpha = kMx ? 1.0f : __fmul_rn(x_gs[T.e], w_gs[T.e]);
      epilogue_tile<kSwiglu, kBf16Out, kQuantH>(T, tmem_base + lane_base + ab * TMEM_ACC_STRIDE, alpha, epi, quad,
                                                lane, N, y, amax_out, bar_acc_empty + 8 * ab, false, hq, dev_status);
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

// 0 automatic (two weight blocks per tile for bf16 outputs with N % 256 == 0
// and K >= 1024; else the deep 512-element ring when the groups average at
// most 16 rows; else 512-element stages when K % 512 == 0; else one CTA per
// tile with 256-element stages), 1 one CTA per tile with 256-element stages,
// 2 CTA pairs, 3 the deep 512-element ring whenever K % 512 == 0, 4 two
// weight blocks per tile whenever N % 256 == 0 and the output is bf16 (else
// as 0); the MXFP4 GEMM follows the same rule
std::atomic<int> g_gemm_kernel{0};

}  // namespace

// Decode-sized groups: the experts average at most 16 routed rows.
bool small_groups(int64_t M_total, int E) { return M_total <= gemm::kDeepRingMaxRowsPerExpert * (int64_t)E; }

// The deep ring of the one-block kernel (64-token tiles, three slots) in mode
// 3, and in mode 0 for small groups.
bool deep_ring(int64_t M_total, int E) {
  const int mode = g_gemm_kernel.load();
  return mode == 3 || (mode == 0 && small_groups(M_total, E));
}

// The two-weight-block kernel (gemm_w2.cu) serves NVFP4 operands with a bf16
// output (plain, SwiGLU h or NVFP4 h) and N % 256 == 0: always in mode 4, and
// in mode 0 when K >= 1024 (its single accumulator pair drains between tiles,
// which a K loop of at least four stages hides behind the ring's loads), for
// decode-sized groups as well as large ones.
bool use_w2(int64_t N, int64_t K, bool bf16_out) {
  if (N % 256 != 0 || !bf16_out) return false;
  const int mode = g_gemm_kernel.load();
  return mode == 4 || (mode == 0 && K >= 1024);
}

// One CTA per SM, but no more CTAs than tiles can exist: each expert has at
// most ceil(m_e / BN) <= m_e / BN + 1 token chunks per 128-row weight block.
int persistent_grid(int64_t M_total, int E, int64_t N) {
  const int64_t bound = (N / gemm::BM) * ((M_total + gemm::BN - 1) / gemm::BN + E);
  const int sms = host::sm_count();
  return (int)(bound < sms ? bound : sms);
}

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
  // the SwiGLU epilogue raises amax_out[e] with integer atomics: start from 0
  if (swiglu && cudaMemsetAsync(amax_out, 0, sizeof(float) * (size_t)E, stream) != cudaSuccess) return NVFP4_ERR_CUDA;
  if (M_total == 0) return NVFP4_OK;
  if (!a_q || !a_sf || !a_gs || !b_q || !b_sf || !b_gs || !y) return NVFP4_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(a_q) | reinterpret_cast<uintptr_t>(b_q) | reinterpret_cast<uintptr_t>(a_sf) |
       reinterpret_cast<uintptr_t>(b_sf) | reinterpret_cast<uintptr_t>(y)) & 15u)
    return NVFP4_ERR_INVALID_ARG;
  if (use_w2(N, K, out_dtype == NVFP4_OUT_BF16))
    return gemm::launch_grouped_gemm_w2(a_q, a_sf, a_gs, b_q, b_sf, b_gs, expert_offsets, E, M_total, N, K, y, swiglu,
                                        amax_out, nullptr, false, small_groups(M_total, E), dev_status, stream);
  if (g_gemm_kernel == 2)
    return gemm::launch_grouped_gemm_pair(a_q, a_sf, a_gs, b_q, b_sf, b_gs, expert_offsets, E, M_total, N, K, y,
                                          out_dtype, swiglu, amax_out, dev_status, stream);
  if ((g_gemm_kernel == 0 || g_gemm_kernel == 3) && K % 512 == 0)
    return gemm::launch_grouped_gemm_k512(a_q, a_sf, a_gs, b_q, b_sf, b_gs, expert_offsets, E, M_total, N, K, y,
                                          out_dtype, swiglu, amax_out, nullptr, false, deep_ring(M_total, E), dev_status, stream);
  const int64_t x_rows = nvfp4_padded_rows_bound(M_total, E);
  CUtensorMap tw, tx128, tx64, tx32;
  if (!gemm::make_map(&tw, b_q, (uint64_t)E * N, (uint64_t)K / 2, 128)) return NVFP4_ERR_CUDA;
  if (!gemm::make_map(&tx128, a_q, (uint64_t)x_rows, (uint64_t)K / 2, 128)) return NVFP4_ERR_CUDA;
  if (!gemm::make_map(&tx64, a_q, (uint64_t)x_rows, (uint64_t)K / 2, 64)) return NVFP4_ERR_CUDA;
  if (!gemm::make_map(&tx32, a_q, (uint64_t)x_rows, (uint64_t)K / 2, 32)) return NVFP4_ERR_CUDA;
  const int variant = swiglu ? 2 : (out_dtype == NVFP4_OUT_BF16 ? 1 : 0);
  auto kern = variant == 2 ? gemm::grouped_gemm_kernel<true, true>
                           : (variant == 1 ? gemm::grouped_gemm_kernel<false, true> : gemm::grouped_gemm_kernel<false, false>);
  if (!host::set_max_dynamic_smem(reinterpret_cast<const void *>(kern), gemm::SMEM_BYTES)) return NVFP4_ERR_CUDA;
  kern<<<persistent_grid(M_total, E, N), gemm::NUM_THREADS, gemm::SMEM_BYTES, stream>>>(tw, tx128, tx64, tx32, b_sf, a_sf, b_gs, a_gs,
                                                               expert_offsets, E, (int)M_total, (int)N, (int)K, y,
                                                               amax_out, dev_status, gemm::HQuantOut{});
  return cudaGetLastError() == cudaSuccess ? NVFP4_OK : NVFP4_ERR_CUDA;
}

extern "C" nvfp4_status nvfp4_gemm_set_wait_budget(int64_t cycles) {
  if (cycles < 0) return NVFP4_ERR_INVALID_ARG;
  const long long v = cycles == 0 ? gemm::kWaitBudgetCycles : (long long)cycles;
  if (cudaMemcpyToSymbol(gemm::c_wait_budget, &v, sizeof(v)) != cudaSuccess) return NVFP4_ERR_CUDA;
  if (gemm::set_wait_budget_k512(v) != NVFP4_OK) return NVFP4_ERR_CUDA;
  return gemm::set_wait_budget_w2(v);
}

extern "C" nvfp4_status nvfp4_gemm_select_kernel(int mode) {
  if (mode < 0 || mode > 4) return NVFP4_ERR_INVALID_ARG;
  g_gemm_kernel = mode;
  return NVFP4_OK;
}

extern "C" nvfp4_status nvfp4_grouped_gemm_swiglu_nvfp4(const uint8_t *a_q, const uint8_t *a_sf, const float *a_gs,
                                                      const uint8_t *b_q, const uint8_t *b_sf, const float *b_gs,
                                                      const int32_t *expert_offsets, int num_experts, int64_t M_total,
                                                      int64_t N, int64_t K, const float *h_gs, uint8_t *h_q,
                                                      uint8_t *h_sf, void *workspace, int32_t *dev_status,
                                                      cudaStream_t stream) {
  (void)workspace;
  const int E = expert_offsets ? num_experts : 1;
  if (E < 1 || E > gemm::kMaxExperts) return NVFP4_ERR_UNSUPPORTED_SHAPE;
  if (M_total < 0 || N <= 0 || K <= 0) return NVFP4_ERR_INVALID_ARG;
  if (N % 128 != 0 || K % 256 != 0) return NVFP4_ERR_UNSUPPORTED_SHAPE;
  if ((int64_t)E * N > ((int64_t)1 << 31) - 1 || M_total > ((int64_t)1 << 30)) return NVFP4_ERR_UNSUPPORTED_SHAPE;
  if (M_total == 0) return NVFP4_OK;
  if (!a_q || !a_sf || !a_gs || !b_q || !b_sf || !b_gs || !h_gs || !h_q || !h_sf) return NVFP4_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(a_q) | reinterpret_cast<uintptr_t>(b_q) | reinterpret_cast<uintptr_t>(a_sf) |
       reinterpret_cast<uintptr_t>(b_sf) | reinterpret_cast<uintptr_t>(h_q)) & 15u)
    return NVFP4_ERR_INVALID_ARG;
  gemm::HQuantOut hq;
  hq.gs = h_gs;
  hq.q = h_q;
  hq.sf = h_sf;
  if (use_w2(N, K, true))
    return gemm::launch_grouped_gemm_w2(a_q, a_sf, a_gs, b_q, b_sf, b_gs, expert_offsets, E, M_total, N, K, nullptr,
                                        true, nullptr, &hq, false, small_groups(M_total, E), dev_status, stream);
  if ((g_gemm_kernel == 0 || g_gemm_kernel == 3) && K % 512 == 0)
    return gemm::launch_grouped_gemm_k512(a_q, a_sf, a_gs, b_q, b_sf, b_gs, expert_offsets, E, M_total, N, K, nullptr,
                                          NVFP4_OUT_BF16, true, nullptr, &hq, false, deep_ring(M_total, E), dev_status, stream);
  const int64_t x_rows = nvfp4_padded_rows_bound(M_total, E);
  CUtensorMap tw, tx128, tx64, tx32;
  if (!gemm::make_map(&tw, b_q, (uint64_t)E * N, (uint64_t)K / 2, 128)) return NVFP4_ERR_CUDA;
  if (!gemm::make_map(&tx128, a_q, (uint64_t)x_rows, (uint64_t)K / 2, 128)) return NVFP4_ERR_CUDA;
  if (!gemm::make_map(&tx64, a_q, (uint64_t)x_rows, (uint64_t)K / 2, 64)) return NVFP4_ERR_CUDA;
  if (!gemm::make_map(&tx32, a_q, (uint64_t)x_rows, (uint64_t)K / 2, 32)) return NVFP4_ERR_CUDA;
  auto kern = gemm::grouped_gemm_kernel<true, true, true>;
  if (!host::set_max_dynamic_smem(reinterpret_cast<const void *>(kern), gemm::SMEM_BYTES)) return NVFP4_ERR_CUDA;
  kern<<<persistent_grid(M_total, E, N), gemm::NUM_THREADS, gemm::SMEM_BYTES, stream>>>(tw, tx128, tx64, tx32, b_sf, a_sf, b_gs, a_gs,
                                                               expert_offsets, E, (int)M_total, (int)N, (int)K, nullptr,
                                                               nullptr, dev_status, hq);
  return cudaGetLastError() == cudaSuccess ? NVFP4_OK : NVFP4_ERR_CUDA;
}

// MXFP4 x MXFP4 grouped GEMM (kind::mxf4): the same persistent pipeline with
// UE8M0 scales per 32 elements and no global scales.
extern "C" nvfp4_status mxfp4_grouped_gemm(const uint8_t *a_q, const uint8_t *a_sf, const uint8_t *b_q,
                                           const uint8_t *b_sf, const int32_t *expert_offsets, int num_experts,
                                           int64_t M_total, int64_t N, int64_t K, void *y,
                                           nvfp4_out_dtype out_dtype, void *workspace, int32_t *dev_status,
                                           cudaStream_t stream) {
  (void)workspace;
  if (out_dtype != NVFP4_OUT_F32 && out_dtype != NVFP4_OUT_BF16) return NVFP4_ERR_INVALID_ARG;
  const int E = expert_offsets ? num_experts : 1;
  if (E < 1 || E > gemm::kMaxExperts) return NVFP4_ERR_UNSUPPORTED_SHAPE;
  if (M_total < 0 || N <= 0 || K <= 0) return NVFP4_ERR_INVALID_ARG;
  if (N % 128 != 0 || K % 256 != 0) return NVFP4_ERR_UNSUPPORTED_SHAPE;
  if ((int64_t)E * N > ((int64_t)1 << 31) - 1 || M_total > ((int64_t)1 << 30)) return NVFP4_ERR_UNSUPPORTED_SHAPE;
  if (M_total == 0) return NVFP4_OK;
  if (!a_q || !a_sf || !b_q || !b_sf || !y) return NVFP4_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(a_q) | reinterpret_cast<uintptr_t>(b_q) | reinterpret_cast<uintptr_t>(a_sf) |
       reinterpret_cast<uintptr_t>(b_sf) | reinterpret_cast<uintptr_t>(y)) & 15u)
    return NVFP4_ERR_INVALID_ARG;
  if (use_w2(N, K, out_dtype == NVFP4_OUT_BF16))
    return gemm::launch_grouped_gemm_w2(a_q, a_sf, nullptr, b_q, b_sf, nullptr, expert_offsets, E, M_total, N, K, y,
                                        false, nullptr, nullptr, true, small_groups(M_total, E), dev_status, stream);
  if ((g_gemm_kernel == 0 || g_gemm_kernel == 3) && K % 512 == 0)
    return gemm::launch_grouped_gemm_k512(a_q, a_sf, nullptr, b_q, b_sf, nullptr, expert_offsets, E, M_total, N, K, y,
                                          out_dtype, false, nullptr, nullptr, true, deep_ring(M_total, E), dev_status, stream);
  const int64_t x_rows = nvfp4_padded_rows_bound(M_total, E);
  CUtensorMap tw, tx128, tx64, tx32;
  if (!gemm::make_map(&tw, b_q, (uint64_t)E * N, (uint64_t)K / 2, 128)) return NVFP4_ERR_CUDA;
  if (!gemm::make_map(&tx128, a_q, (uint64_t)x_rows, (uint64_t)K / 2, 128)) return NVFP4_ERR_CUDA;
  if (!gemm::make_map(&tx64, a_q, (uint64_t)x_rows, (uint64_t)K / 2, 64)) return NVFP4_ERR_CUDA;
  if (!gemm::make_map(&tx32, a_q, (uint64_t)x_rows, (uint64_t)K / 2, 32)) return NVFP4_ERR_CUDA;
  const int variant = out_dtype == NVFP4_OUT_BF16 ? 5 : 4;
  auto kern = variant == 5 ? gemm::grouped_gemm_kernel<false, true, false, true>
                           : gemm::grouped_gemm_kernel<false, false, false, true>;
  if (!host::set_max_dynamic_smem(reinterpret_cast<const void *>(kern), gemm::SMEM_BYTES)) return NVFP4_ERR_CUDA;
  kern<<<persistent_grid(M_total, E, N), gemm::NUM_THREADS, gemm::SMEM_BYTES, stream>>>(tw, tx128, tx64, tx32, b_sf, a_sf, nullptr, nullptr,
                                                               expert_offsets, E, (int)M_total, (int)N, (int)K, y,
                                                               nullptr, dev_status, gemm::HQuantOut{});
  return cudaGetLastError() == cudaSuccess ? NVFP4_OK : NVFP4_ERR_CUDA;
}
