// Block-scaled FP4 x FP4 grouped GEMM on CTA pairs (tcgen05 cta_group::2, sm_100a).
//
// Same computation as the one-CTA kernel in gemm.cu -- for every routed expert
// e, Y_e = (a_gs[e] * b_gs[e]) * X_e W_e^T on the native 4-bit tensor-core
// path ("DeepSeek-V4.1-Flash-NVFP4", "why NVFP4"; the routed experts'
// gate_up_proj / down_proj of "Qwen3.8-Flash-Next-NVFP4", W4A4) -- with the
// tile spread over the two SMs of a cluster:
//  * One MMA covers 256 weight rows (M, 128 in each CTA's shared and tensor
//    memory) x up to 192 tokens (N).  The token tile is split N/2 + N/2
//    between the two CTAs, so every CTA streams its 128 weight rows but only
//    half of the token rows: the token tiles, re-read from L2 for every weight
//    block, move half the bytes per unit of work, and one MMA instruction does
//    twice the work.
//  * Weight and token tiles and their scales, of both CTAs, are counted on
//    the leader CTA's full barriers (cta_group::2 tensor copies); only the
//    leader issues MMAs, and its commits reach the empty / accumulator
//    barriers of both CTAs (tcgen05.commit multicast).  No load uses cluster
//    multicast.
//  * Each CTA's tensor memory holds the scales of its own 128 weight rows and
//    of all N tokens (the layout of the one-CTA kernel).  The leader's four
//    scale warps copy them from both CTAs' shared memory with
//    tcgen05.cp.cta_group::2 (one K chunk each) and commit to sf_full: the
//    peer CTA's own tensor-memory stores were measured at ~2000 cycles per
//    stage while the pair's MMAs run, the copies at a few hundred.  The
//    epilogue warps of both CTAs drain their own accumulators and release
//    them to the leader.
//  * Every wait is bounded; a timeout raises the abort flag of both CTAs.
#include <mutex>

#include "gemm_common.cuh"
#include "host_util.cuh"

namespace nvfp4 {
namespace gemm {
namespace pair {

constexpr int W_STAGES = 6;
constexpr int X_STAGES = 5;
constexpr int XH_ROWS = BN / 2;                             // token rows per CTA
constexpr int X_STAGE = XH_ROWS * 128;                      // 12 KB
constexpr int OFF_W = 0;
constexpr int OFF_X = OFF_W + W_STAGES * W_STAGE;
constexpr int OFF_SFW = OFF_X + X_STAGES * X_STAGE;
constexpr int OFF_SFX = OFF_SFW + W_STAGES * SFW_STAGE;
constexpr int OFF_EPI = OFF_SFX + X_STAGES * SFX_STAGE;
constexpr int OFF_BAR = OFF_EPI + 4 * EPI_WARP_BYTES;
// wfull[WS], wempty[WS], xfull[XS], xempty[XS], sf_full[2], acc_full[2], acc_empty[2], drain
constexpr int NUM_BARS = 2 * W_STAGES + 2 * X_STAGES + 2 + 2 + 2 + 1;
constexpr int OFF_MISC = OFF_BAR + NUM_BARS * 8;            // tmem base, abort flag
constexpr int OFF_GROUPS = OFF_MISC + 16;
constexpr int SMEM_BYTES = OFF_GROUPS + GROUP_TABLE_BYTES + 1024;
static_assert(SMEM_BYTES <= 232448, "shared memory budget");
static_assert(OFF_X % 1024 == 0 && X_STAGE % 1024 == 0 && W_STAGE % 1024 == 0, "128-byte swizzle atoms");
constexpr long long kAbortSettleCycles = 200000;            // ~0.1 ms for copies in flight after an abort

template <bool kSwiglu, bool kBf16Out>
__global__ void __launch_bounds__(NUM_THREADS, 1) grouped_gemm_pair_kernel(
    const __grid_constant__ CUtensorMap tmap_w, const __grid_constant__ CUtensorMap tmap_x96,
    const __grid_constant__ CUtensorMap tmap_x64, const __grid_constant__ CUtensorMap tmap_x32,
    const __grid_constant__ CUtensorMap tmap_sfx, const __grid_constant__ CUtensorMap tmap_sfw,
    const float *__restrict__ w_gs, const float *__restrict__ x_gs, const int32_t *__restrict__ expert_offsets,
    int E, int M_total, int N, int K, void *__restrict__ y, float *__restrict__ amax_out, int32_t *dev_status) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
  const uint32_t sbase = smem_u32(smem);
  const uint32_t bar_wfull = sbase + OFF_BAR;                // leader: both CTAs' weight tiles + scales
  const uint32_t bar_wempty = bar_wfull + 8 * W_STAGES;      // MMA commit (multicast to both CTAs)
  const uint32_t bar_xfull = bar_wempty + 8 * W_STAGES;      // leader: both CTAs' token tiles + scales
  const uint32_t bar_xempty = bar_xfull + 8 * X_STAGES;      // MMA commit (multicast)
  const uint32_t bar_sf_full = bar_xempty + 8 * X_STAGES;    // leader: [2], scale-copy commits (4)
  const uint32_t bar_acc_full = bar_sf_full + 16;            // [2], MMA commit (multicast)
  const uint32_t bar_acc_empty = bar_acc_full + 16;          // leader: [2], epilogue threads of both CTAs (256)
  const uint32_t bar_drain = bar_acc_empty + 16;
  volatile uint32_t *tmem_holder = reinterpret_cast<volatile uint32_t *>(smem + OFF_MISC);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + OFF_MISC + 4);
  int32_t *s_off = reinterpret_cast<int32_t *>(smem + OFF_GROUPS);
  int32_t *s_slot = s_off + (kMaxExperts + 1);
  int32_t *s_tile = s_slot + (kMaxExperts + 1);
  int32_t *s_scratch = s_tile + (kMaxExperts + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();                   // 0: leader, issues the MMAs
  const bool leader = rank == 0;
  const int pair_id = (int)cluster_id_x(), npairs = (int)nclusters_x();
  const int n_mtiles = N / (2 * BM);
  const int ksteps = K / BK;
  const uint32_t peer_abort = mapa_shared(smem_u32((const void *)abort_flag), rank ^ 1u);
  const uint32_t lead_wfull = mapa_shared(bar_wfull, 0), lead_xfull = mapa_shared(bar_xfull, 0);
  const uint32_t lead_acc_empty = mapa_shared(bar_acc_empty, 0);

  // ---- set-up: barriers, tensor memory of the pair, expert tables
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
      mbar_init(bar_sf_full + 8 * b, 4);
      mbar_init(bar_acc_full + 8 * b, 1);
      mbar_init(bar_acc_empty + 8 * b, 256);
    }
    mbar_init(bar_drain, 1);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == W_MMA) {
    asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;"
                 :: "r"(smem_u32((const void *)tmem_holder)), "r"(TMEM_COLS) : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
  }
  build_tile_tables(expert_offsets, E, M_total, n_mtiles, s_off, s_slot, s_tile, s_scratch, dev_status);
  tc_fence_before();
  __syncthreads();
  cluster_sync_all();              // both CTAs' barriers exist before any remote arrive or pair copy
  tc_fence_after();
  const uint32_t tmem_base = *tmem_holder;
  const int total_tiles = s_tile[E];

  if (warp == W_PRODUCER || warp == W_XLOAD) {
    // ================================================================ TMA producers
    // warp 0 lane 0: this CTA's 128 weight rows and their scales; warp 10
    // lane 0: this CTA's half of the token rows and the token scales of the
    // whole tile.  All counted on the leader's wfull / xfull, which the
    // leader arms with the bytes of both CTAs.
    if (lane == 0) {
      const bool is_w = warp == W_PRODUCER;
      const uint64_t pol = is_w ? policy_evict_first() : policy_evict_last();
      const int nstages = is_w ? W_STAGES : X_STAGES;
      const uint32_t bar_empty = is_w ? bar_wempty : bar_xempty;
      const uint32_t bar_full_local = is_w ? bar_wfull : bar_xfull;
      const uint32_t lead_full = is_w ? lead_wfull : lead_xfull;
      int stage = 0;
      uint32_t phase = 0;
      bool armed[W_STAGES] = {};
      uint32_t armed_parity[W_STAGES] = {};
      bool ok = true;
      for (int t = pair_id; t < total_tiles && ok; t += npairs) {
        const Tile T = decode_tile<kSwiglu>(t, s_off, s_slot, s_tile, E, N, 2 * BM, (int)rank);
        const int half = ((T.n_valid + 15) & ~15) >> 1;            // token rows per CTA (8..96)
        const int xbox = half <= 32 ? 32 : (half <= 64 ? 64 : 96);
        const CUtensorMap *xmap = xbox == 32 ? &tmap_x32 : (xbox == 64 ? &tmap_x64 : &tmap_x96);
        const uint32_t tile_bytes = is_w ? (uint32_t)(W_STAGE + SFW_STAGE) : (uint32_t)(xbox * 128 + SFX_STAGE);
        const int xrb = T.x_row0 >> 7;                                 // first scale row block
        for (int ks = 0; ks < ksteps; ++ks) {
          if (!mbar_wait<true>(bar_empty + 8 * stage, phase ^ 1, abort_flag, dev_status, peer_abort)) { ok = false; break; }
          if (leader) mbar_arrive_expect_tx(bar_full_local + 8 * stage, 2 * tile_bytes);
          armed[stage] = true;
          armed_parity[stage] = phase;
          if (is_w) {
            tma_load_2d_pair(sbase + OFF_W + stage * W_STAGE, &tmap_w, ks * 128, T.w_row0, lead_full + 8 * stage, pol);
            tma_load_3d_pair(sbase + OFF_SFW + stage * SFW_STAGE, &tmap_sfw, 0, ks * 8, T.w_row0 >> 7,
                             lead_full + 8 * stage, pol);
          } else {
            tma_load_3d_pair(sbase + OFF_SFX + stage * SFX_STAGE, &tmap_sfx, 0, ks * 8, xrb, lead_full + 8 * stage, pol);
            tma_load_2d_pair(sbase + OFF_X + stage * X_STAGE, xmap, ks * 128, T.x_row0 + (int)rank * half,
                             lead_full + 8 * stage, pol);
          }
          if (++stage == nstages) { stage = 0; phase ^= 1; }
        }
      }
      // Drain (leader): both CTAs' copies counted on an armed stage must have
      // landed before the pair exits.
      for (int s = 0; s < nstages && leader; ++s) {
        if (!armed[s]) continue;
        const long long t0 = clock64();
        while (!mbar_try_wait(bar_full_local + 8 * s, armed_parity[s]) && clock64() - t0 < kWaitBudgetCycles) {}
      }
    }
  } else if (warp >= W_SF0 && warp < W_SF0 + 4) {
    // ================================================================ scale factors -> TMEM
    // Leader only: warp 6+kk copies K chunk kk of the stage's scales (weight
    // scales of 128 rows, token scales of one or two 128-row blocks) into
    // scale buffer kiter & 1 of both CTAs, then commits to sf_full.  The
    // buffer was last read by the MMAs of k-step kiter-2: wait for them.
    uint32_t kiter = 0;
    bool ok = true;
    const int kk = warp - W_SF0;
    for (int t = pair_id; t < total_tiles && ok && leader; t += npairs) {
      const Tile T = decode_tile<kSwiglu>(t, s_off, s_slot, s_tile, E, N, 2 * BM, 0);
      const int nrb = ((T.x_row0 & 127) + T.n_valid + 127) >> 7;
      for (int ks = 0; ks < ksteps; ++ks, ++kiter) {
        const uint32_t sb = kiter & 1;
        if (kiter >= 2) {
          const uint32_t prev = kiter - 2;
          if (!mbar_wait_warp<true>(bar_wempty + 8 * (prev % W_STAGES), (prev / W_STAGES) & 1, abort_flag,
                                    dev_status, peer_abort)) {
            ok = false; break;
          }
        }
        const uint32_t sw = kiter % W_STAGES, sx = kiter % X_STAGES;
        if (!mbar_wait_warp<true>(bar_wfull + 8 * sw, (kiter / W_STAGES) & 1, abort_flag, dev_status, peer_abort)) {
          ok = false; break;
        }
        if (!mbar_wait_warp<true>(bar_xfull + 8 * sx, (kiter / X_STAGES) & 1, abort_flag, dev_status, peer_abort)) {
          ok = false; break;
        }
        tc_fence_after();
        if (lane == 0) {
          const uint32_t t_sf = tmem_base + TMEM_SF + sb * TMEM_SF_STRIDE;
          const uint32_t sfw = sbase + OFF_SFW + sw * SFW_STAGE, sfx = sbase + OFF_SFX + sx * SFX_STAGE;
          tc_cp_sf_pair(t_sf + kk * 4, desc_sf_atom(sfw + kk * 512));
          tc_cp_sf_pair(t_sf + 16 + kk * 8, desc_sf_atom(sfx + kk * 512));
          if (nrb > 1) tc_cp_sf_pair(t_sf + 16 + kk * 8 + 4, desc_sf_atom(sfx + 2048 + kk * 512));
          tc_commit_pair(bar_sf_full + 8 * sb);
        }
        __syncwarp();
      }
    }
  } else if (warp == W_MMA) {
    // ================================================================ MMA issuer (leader only)
    if (leader) {
      uint32_t kiter = 0, titer = 0;
      bool ok = true;
      for (int t = pair_id; t < total_tiles && ok; t += npairs, ++titer) {
        const Tile T = decode_tile<kSwiglu>(t, s_off, s_slot, s_tile, E, N, 2 * BM, 0);
        const uint32_t n_mma = (T.n_valid + 15) & ~15;
        const uint32_t idesc = idesc_mxf4nvf4(2 * BM, n_mma);
        const uint32_t xoff = (uint32_t)(T.x_row0 & 127) >> 5;      // 0 or 2 columns
        const uint32_t ab = titer & 1;
        const uint32_t t_acc = tmem_base + ab * TMEM_ACC_STRIDE;
        if (!mbar_wait_warp<true>(bar_acc_empty + 8 * ab, ((titer >> 1) & 1) ^ 1, abort_flag, dev_status,
                                  peer_abort)) {
          ok = false; break;
        }
        tc_fence_after();
        for (int ks = 0; ks < ksteps; ++ks, ++kiter) {
          const uint32_t sb = kiter & 1;
          const uint32_t sw = kiter % W_STAGES, sx = kiter % X_STAGES;
          if (!mbar_wait_warp<true>(bar_wfull + 8 * sw, (kiter / W_STAGES) & 1, abort_flag, dev_status, peer_abort)) {
            ok = false; break;
          }
          if (!mbar_wait_warp<true>(bar_xfull + 8 * sx, (kiter / X_STAGES) & 1, abort_flag, dev_status, peer_abort)) {
            ok = false; break;
          }
          if (!mbar_wait_warp<true>(bar_sf_full + 8 * sb, (kiter >> 1) & 1, abort_flag, dev_status, peer_abort)) {
            ok = false; break;
          }
          tc_fence_after();
          if (lane == 0) {
            const uint32_t t_sf = tmem_base + TMEM_SF + sb * TMEM_SF_STRIDE;
            const uint64_t dw = desc_sw128(sbase + OFF_W + sw * W_STAGE);
            const uint64_t dx = desc_sw128(sbase + OFF_X + sx * X_STAGE);
#pragma unroll
            for (int kk = 0; kk < 4; ++kk) {
              // +32 bytes of K per MMA: +2 in the descriptor's 16-byte address field
              tc_mma_pair(t_acc, dw + 2 * kk, dx + 2 * kk, idesc, t_sf + kk * 4, t_sf + 16 + kk * 8 + xoff,
                          (ks > 0 || kk > 0) ? 1u : 0u);
            }
            tc_commit_pair_both(bar_wempty + 8 * sw);
            tc_commit_pair_both(bar_xempty + 8 * sx);
          }
          __syncwarp();
        }
        if (!ok) break;
        if (lane == 0) tc_commit_pair_both(bar_acc_full + 8 * ab);
        __syncwarp();
      }
      // Drain: all MMAs of the pair complete before tensor memory is freed.
      if (lane == 0) {
        tc_commit_pair(bar_drain);
        const long long t0 = clock64();
        while (!mbar_try_wait(bar_drain, 0) && clock64() - t0 < kWaitBudgetCycles) {}
      }
      __syncwarp();
    }
  } else {
    // ================================================================ epilogue (both CTAs)
    const int quad = warp & 3;                    // TMEM lane quadrant of this warp
    const uint32_t lane_base = (uint32_t)(quad * 32) << 16;
    const uint32_t epi = sbase + OFF_EPI + (warp - 2) * EPI_WARP_BYTES;
    uint32_t titer = 0;
    for (int t = pair_id; t < total_tiles; t += npairs, ++titer) {
      const Tile T = decode_tile<kSwiglu>(t, s_off, s_slot, s_tile, E, N, 2 * BM, (int)rank);
      const uint32_t ab = titer & 1;
      if (!mbar_wait_warp<true>(bar_acc_full + 8 * ab, (titer >> 1) & 1, abort_flag, dev_status, peer_abort)) break;
      tc_fence_after();
      const float alpha = __fmul_rn(x_gs[T.e], w_gs[T.e]);
      epilogue_tile<kSwiglu, kBf16Out>(T, tmem_base + lane_base + ab * TMEM_ACC_STRIDE, alpha, epi, quad, lane, N, y,
                                       amax_out, leader ? bar_acc_empty + 8 * ab : lead_acc_empty + 8 * ab, !leader);
    }
  }

  tc_fence_before();
  __syncthreads();
  if (*abort_flag) {
    // after a timeout, let copies still in flight into this CTA land first
    const long long t0 = clock64();
    while (clock64() - t0 < kAbortSettleCycles) {}
  }
  cluster_sync_all();              // neither CTA frees tensor memory or exits while the pair still works
  tc_fence_after();
  if (warp == W_MMA) {
    asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" :: "r"(tmem_base), "r"(TMEM_COLS) : "memory");
  }
}

}  // namespace pair

// ====================================================================== host side
namespace {
// Resident CTA pairs per variant and device, from the occupancy query (0 = not asked yet).
std::mutex g_pair_mu;
int g_pair_clusters[host::kMaxDevices][3] = {};
}  // namespace

nvfp4_status launch_grouped_gemm_pair(const uint8_t *a_q, const uint8_t *a_sf, const float *a_gs,
                                      const uint8_t *b_q, const uint8_t *b_sf, const float *b_gs,
                                      const int32_t *expert_offsets, int E, int64_t M_total, int64_t N, int64_t K,
                                      void *y, nvfp4_out_dtype out_dtype, bool swiglu, float *amax_out,
                                      int32_t *dev_status, cudaStream_t stream) {
  if (N % (2 * BM) != 0) return NVFP4_ERR_UNSUPPORTED_SHAPE;
  const int64_t x_rows = nvfp4_padded_rows_bound(M_total, E);
  CUtensorMap tw, tx96, tx64, tx32, tsfx;
  if (!make_map(&tw, b_q, (uint64_t)E * N, (uint64_t)K / 2, 128)) return NVFP4_ERR_CUDA;
  if (!make_map(&tx96, a_q, (uint64_t)x_rows, (uint64_t)K / 2, 96)) return NVFP4_ERR_CUDA;
  if (!make_map(&tx64, a_q, (uint64_t)x_rows, (uint64_t)K / 2, 64)) return NVFP4_ERR_CUDA;
  if (!make_map(&tx32, a_q, (uint64_t)x_rows, (uint64_t)K / 2, 32)) return NVFP4_ERR_CUDA;
  if (!make_map_sfx(&tsfx, a_sf, (uint64_t)x_rows / 128, (uint64_t)K)) return NVFP4_ERR_CUDA;
  CUtensorMap tsfw;
  if (!make_map_sfw(&tsfw, b_sf, (uint64_t)E * N / 128, (uint64_t)K)) return NVFP4_ERR_CUDA;
  const int variant = swiglu ? 2 : (out_dtype == NVFP4_OUT_BF16 ? 1 : 0);
  auto kern = variant == 2 ? pair::grouped_gemm_pair_kernel<true, true>
                           : (variant == 1 ? pair::grouped_gemm_pair_kernel<false, true>
                                           : pair::grouped_gemm_pair_kernel<false, false>);
  if (!host::set_max_dynamic_smem(reinterpret_cast<const void *>(kern), pair::SMEM_BYTES)) return NVFP4_ERR_CUDA;
  const int dev = host::current_device();
  if (dev < 0) return NVFP4_ERR_CUDA;
  cudaLaunchConfig_t cfg = {};
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.blockDim = dim3(NUM_THREADS, 1, 1);
  cfg.dynamicSmemBytes = pair::SMEM_BYTES;
  cfg.stream = stream;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  int clusters;
  {
    std::lock_guard<std::mutex> lock(g_pair_mu);
    clusters = g_pair_clusters[dev][variant];
  }
  if (clusters == 0) {
    const int sms = host::sm_count();
    cfg.gridDim = dim3(2 * (sms / 2 > 0 ? sms / 2 : 1), 1, 1);
    int n = 0;
    if (cudaOccupancyMaxActiveClusters(&n, kern, &cfg) != cudaSuccess || n < 1) {
      (void)cudaGetLastError();
      n = sms / 2 > 0 ? sms / 2 : 1;
    }
    clusters = n;
    std::lock_guard<std::mutex> lock(g_pair_mu);
    g_pair_clusters[dev][variant] = n;
  }
  cfg.gridDim = dim3(2 * clusters, 1, 1);
  const cudaError_t err = cudaLaunchKernelEx(&cfg, kern, tw, tx96, tx64, tx32, tsfx, tsfw, b_gs, a_gs, expert_offsets,
                                             E, (int)M_total, (int)N, (int)K, y, amax_out, dev_status);
  return err == cudaSuccess ? NVFP4_OK : NVFP4_ERR_CUDA;
}

}  // namespace gemm
}  // namespace nvfp4
