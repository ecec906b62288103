// Block-scaled FP4 x FP4 grouped GEMM, two weight blocks per tile (sm_100a).
//
// The same computation as the one-CTA kernels (gemm.cu, gemm_k512.cu): for
// every routed expert e, Y_e = (a_gs[e] * b_gs[e]) * X_e W_e^T on the
// 5th-generation tensor cores, the W4A4 routed-expert projections of the
// "Qwen3.8-Flash-Next-NVFP4" page (gate_up_proj / down_proj) on the native
// 4-bit path of the "DeepSeek-V4.1-Flash-NVFP4" page's "why NVFP4" section.
// Same MMA (kind::mxf4nvf4, swap-AB: weight rows on M, up to 192 tokens on N),
// scale path, epilogue and bounded waits.
//
// What differs: a tile is 256 weight rows (two 128-row blocks) x one token
// chunk.  Each 256-element K stage holds both weight blocks (one 256-row TMA
// box, 32 KB) and the token tile once (up to 24 KB), and every K step issues
// two MMAs, one per block, into two accumulators that read the same token
// operand.  Per byte of weights a stage carries half the token bytes of the
// one-block kernels, and three stages fit in shared memory: 96 KB of weights
// in flight per SM instead of 64 KB.  (A probe ring of copies without the math
// streamed 4.8 TB/s of weights with the one-block kernel's two 80 KB slots and
// 5.5 TB/s with three slots of 32 KB of weights and 24 KB of tokens, the bytes
// of this kernel's slots.)  The price is tensor memory: two 192-column
// accumulators and the two scale buffers fill all 512 columns, so the
// accumulators are not double buffered.  Eight epilogue warps (two per lane
// quadrant, one per block) drain them, and the MMAs of the next tile wait for
// that; the ring keeps loading meanwhile.  So the kernel serves K >= 1024 (four
// or more stages per tile), where a tile's main loop is longer than its drain.
// Outputs are bf16 (or SwiGLU h, or NVFP4 h).
#include "gemm_common.cuh"
#include "host_util.cuh"

namespace nvfp4 {
namespace gemm {
namespace w2 {

constexpr int W2_STAGE = 2 * W_STAGE;              // 256 rows x 128 B = 32 KB
constexpr int SFW2_STAGE = 2 * SFW_STAGE;          // two 128-row blocks x 2 KB
constexpr int EPI2_WARP_BYTES = 2048;              // bf16 staging of 32 tokens x 32 columns
constexpr int kEpiWarps = 8;
constexpr int kWarps = 15;
constexpr int kThreads = kWarps * 32;
constexpr int GROUP_BYTES = 3 * (kMaxExperts + 1) * 4 + 2 * kWarps * 4;   // off / slot / tile + scan scratch
constexpr uint32_t kSfStride = 64;                 // per scale buffer: weight blocks 0 and 1 (16 + 16), tokens (32)

// The ring and tensor-memory layout for tiles of at most kCap tokens in
// kSlots slots.  (192, 3) is the general kernel.  (64, 4), for decode-sized
// groups, has 8 KB token boxes, so a fourth slot fits (128 KB of weights in
// flight per SM), and its accumulator pairs take 128 columns each, so two of
// them fit beside the scale buffers: the epilogue of a tile overlaps the next
// tile's MMAs.  A 64-token tile starts on a 64-row boundary and stays inside
// one 128-row block of token scales.
template <int kCap, int kSlots>
struct W2Ring {
  static constexpr int kAccBufs = (4 * kCap + 2 * (int)kSfStride <= (int)TMEM_COLS) ? 2 : 1;
  static constexpr int X_STAGE = kCap * 128;
  static constexpr int SFX_BYTES = kCap <= 64 ? SFW_STAGE : SFX_STAGE;
  static constexpr int OFF_W = 0;
  static constexpr int OFF_X = OFF_W + kSlots * W2_STAGE;
  static constexpr int OFF_SFW = OFF_X + kSlots * X_STAGE;
  static constexpr int OFF_SFX = OFF_SFW + kSlots * SFW2_STAGE;
  static constexpr int OFF_EPI = OFF_SFX + kSlots * SFX_BYTES;
  static constexpr int OFF_BAR = OFF_EPI + kEpiWarps * EPI2_WARP_BYTES;
  // wfull, wempty, xfull, xempty, sfw_data, sfx_data [kSlots]; sf_full[2], sf_free[2],
  // acc_full[kAccBufs], acc_empty[kAccBufs], drain
  static constexpr int NUM_BARS = 6 * kSlots + 2 + 2 + 2 * kAccBufs + 1;
  static constexpr int OFF_MISC = OFF_BAR + NUM_BARS * 8;
  static constexpr int OFF_GROUPS = OFF_MISC + 16;
  static constexpr int SMEM_BYTES = OFF_GROUPS + GROUP_BYTES + 1024;
  // tensor memory: accumulator pair b at columns 2 kCap b (block 0) and
  // 2 kCap b + kCap (block 1), then the two scale buffers
  static constexpr uint32_t kAccPair = 2 * kCap;
  static constexpr uint32_t kSf = kAccBufs * 2 * kCap;
  static_assert(kSf + 2 * kSfStride <= TMEM_COLS, "tensor memory budget");
  static_assert(SMEM_BYTES <= 232448, "shared memory budget");
  static_assert(OFF_X % 1024 == 0 && X_STAGE % 1024 == 0 && W2_STAGE % 1024 == 0, "128-byte swizzle atoms");
};

// warps: 0 weight producer, 1 MMA, 2..5 epilogue of block 0, 6..9 scales,
// 10 token producer, 11..14 epilogue of block 1
constexpr int W_EPI_B = 11;

// kMx: MXFP4 operands (kind::mxf4, one UE8M0 scale per 32 elements, no global
// scales; a K stage holds two 512-byte scale atoms per row block instead of
// four); otherwise NVFP4 (kind::mxf4nvf4, E4M3 per 16 elements).
template <bool kSwiglu, bool kQuantH, int kCap, int kSlots, bool kMx = false>
__global__ void __launch_bounds__(kThreads, 1) grouped_gemm_w2_kernel(
    const __grid_constant__ CUtensorMap tmap_w, const __grid_constant__ CUtensorMap tmap_x32,
    const __grid_constant__ CUtensorMap tmap_x64, const __grid_constant__ CUtensorMap tmap_x128,
    const __grid_constant__ CUtensorMap tmap_x192,
    const uint8_t *__restrict__ w_sf, const uint8_t *__restrict__ x_sf,
    const float *__restrict__ w_gs, const float *__restrict__ x_gs,
    const int32_t *__restrict__ expert_offsets, int E, int M_total, int N, int K,
    void *__restrict__ y, float *__restrict__ amax_out, int32_t *dev_status, HQuantOut hq) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
  const uint32_t sbase = smem_u32(smem);
  using R = W2Ring<kCap, kSlots>;
  constexpr int kStages = kSlots;
  constexpr int kAccBufs = R::kAccBufs;
  const uint32_t bar_wfull = sbase + R::OFF_BAR;
  const uint32_t bar_wempty = bar_wfull + 8 * kStages;
  const uint32_t bar_xfull = bar_wempty + 8 * kStages;
  const uint32_t bar_xempty = bar_xfull + 8 * kStages;
  const uint32_t bar_sfw_data = bar_xempty + 8 * kStages;
  const uint32_t bar_sfx_data = bar_sfw_data + 8 * kStages;
  const uint32_t bar_sf_full = bar_sfx_data + 8 * kStages;   // [2], count 128 (scale warps)
  const uint32_t bar_sf_free = bar_sf_full + 16;              // [2], count 1 (MMA commit)
  const uint32_t bar_acc_full = bar_sf_free + 16;             // [kAccBufs], count 1 (MMA commit)
  const uint32_t bar_acc_empty = bar_acc_full + 8 * kAccBufs; // [kAccBufs], count 256 (both blocks' epilogues)
  const uint32_t bar_drain = bar_acc_empty + 8 * kAccBufs;
  volatile uint32_t *tmem_holder = reinterpret_cast<volatile uint32_t *>(smem + R::OFF_MISC);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + R::OFF_MISC + 4);
  int32_t *s_off = reinterpret_cast<int32_t *>(smem + R::OFF_GROUPS);
  int32_t *s_slot = s_off + (kMaxExperts + 1);
  int32_t *s_tile = s_slot + (kMaxExperts + 1);
  int32_t *s_scratch = s_tile + (kMaxExperts + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int n_mtiles = N / (2 * BM);
  const int ksteps = K / BK;

  if (threadIdx.x == 0) {
    *abort_flag = 0;
    for (int s = 0; s < kStages; ++s) {
      mbar_init(bar_wfull + 8 * s, 1);
      mbar_init(bar_wempty + 8 * s, 1);
      mbar_init(bar_xfull + 8 * s, 1);
      mbar_init(bar_xempty + 8 * s, 1);
      mbar_init(bar_sfw_data + 8 * s, 1);
      mbar_init(bar_sfx_data + 8 * s, 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(bar_sf_full + 8 * b, 128);
      mbar_init(bar_sf_free + 8 * b, 1);
    }
    for (int b = 0; b < kAccBufs; ++b) {
      mbar_init(bar_acc_full + 8 * b, 1);
      mbar_init(bar_acc_empty + 8 * b, 32 * kEpiWarps);
    }
    mbar_init(bar_drain, 1);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == W_MMA) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;"
                 :: "r"(smem_u32((const void *)tmem_holder)), "r"(TMEM_COLS) : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  // tiles of 256 weight rows (wrows = 2 * BM): decode_tile's w_row0 and n_col0
  // are those of the first block; the second block follows 128 rows later
  build_tile_tables<kCap, kThreads>(expert_offsets, E, M_total, n_mtiles, s_off, s_slot, s_tile, s_scratch, dev_status);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_holder;
  const int total_tiles = s_tile[E];
  const int64_t sf_row_stride = (int64_t)(K / (kMx ? 128 : 64)) * 512;   // bytes per 128-row block of scales
  constexpr uint32_t kSfStage = kMx ? 1024u : 2048u;                     // one row block's scales of a K stage

  if (warp == W_PRODUCER || warp == W_XLOAD) {
    // ================================================================ TMA producers
    if (lane == 0) {
      const bool is_w = warp == W_PRODUCER;
      if (is_w) {
        prefetch_tensormap(&tmap_w);
      } else {
        prefetch_tensormap(&tmap_x32);
        prefetch_tensormap(&tmap_x64);
        prefetch_tensormap(&tmap_x128);
        prefetch_tensormap(&tmap_x192);
      }
      // weights at normal L2 priority (evict_first measured 3 % slower: more
      // of the weight sectors were fetched from DRAM twice), tokens evict_last
      const uint64_t pol = is_w ? policy_evict_normal() : policy_evict_last();
      const uint32_t bar_full = is_w ? bar_wfull : bar_xfull, bar_empty = is_w ? bar_wempty : bar_xempty;
      const uint32_t bar_sfd = is_w ? bar_sfw_data : bar_sfx_data;
      int stage = 0;
      uint32_t phase = 0;
      bool armed[kStages] = {};
      uint32_t armed_parity[kStages] = {};
      bool ok = true;
      for (int t = blockIdx.x; t < total_tiles && ok; t += gridDim.x) {
        const Tile T = decode_tile<kSwiglu, kCap>(t, s_off, s_slot, s_tile, E, N, 2 * BM, 0);
        const int xr0 = T.x_row0 & ~127;
        const int nrb = ((T.x_row0 & 127) + T.n_valid + 127) >> 7;
        const int xbox = T.n_valid <= 32 ? 32 : T.n_valid <= 64 ? 64 : T.n_valid <= 128 ? 128 : 192;
        const CUtensorMap *xmap = xbox == 32 ? &tmap_x32 : xbox == 64 ? &tmap_x64 : xbox == 128 ? &tmap_x128 : &tmap_x192;
        const uint32_t bytes = is_w ? (uint32_t)W2_STAGE : (uint32_t)(xbox * 128);
        const uint32_t sf_bytes = is_w ? 2 * kSfStage : (uint32_t)nrb * kSfStage;
        const uint8_t *sfw_tile = w_sf + (int64_t)(T.w_row0 >> 7) * sf_row_stride;
        const uint8_t *sfx_tile = x_sf + (int64_t)(xr0 >> 7) * sf_row_stride;
        for (int ks = 0; ks < ksteps; ++ks) {
          if (!mbar_wait(bar_empty + 8 * stage, phase ^ 1, abort_flag, dev_status)) { ok = false; break; }
          const uint32_t fb = bar_full + 8 * stage, sb = bar_sfd + 8 * stage;
          // the scale bytes first, on their own barrier, then the large copy
          mbar_arrive_expect_tx(sb, sf_bytes);
          mbar_arrive_expect_tx(fb, bytes);
          armed[stage] = true;
          armed_parity[stage] = phase;
          if (is_w) {
            bulk_load(sbase + R::OFF_SFW + stage * SFW2_STAGE, sfw_tile + ks * kSfStage, kSfStage, sb);
            bulk_load(sbase + R::OFF_SFW + stage * SFW2_STAGE + kSfStage, sfw_tile + sf_row_stride + ks * kSfStage,
                      kSfStage, sb);
            tma_load_2d(sbase + R::OFF_W + stage * W2_STAGE, &tmap_w, ks * 128, T.w_row0, fb, pol);
          } else {
            for (int rb = 0; rb < nrb; ++rb)
              bulk_load(sbase + R::OFF_SFX + stage * R::SFX_BYTES + rb * kSfStage,
                        sfx_tile + rb * sf_row_stride + ks * kSfStage, kSfStage, sb);
            tma_load_2d(sbase + R::OFF_X + stage * R::X_STAGE, xmap, ks * 128, T.x_row0, fb, pol);
          }
          if (++stage == kStages) { stage = 0; phase ^= 1; }
        }
      }
      // every armed stage's copies land before the CTA exits (bounded)
      for (int s = 0; s < kStages; ++s) {
        if (!armed[s]) continue;
        long long t0 = clock64();
        while (!mbar_try_wait(bar_full + 8 * s, armed_parity[s]) && clock64() - t0 < kWaitBudgetCycles) {}
        t0 = clock64();
        while (!mbar_try_wait(bar_sfd + 8 * s, armed_parity[s]) && clock64() - t0 < kWaitBudgetCycles) {}
      }
    }
  } else if (warp >= W_SF0 && warp < W_SF0 + 4) {
    // ================================================================ scale factors -> TMEM
    // lane l of quadrant q gets atom row l (rows l, l+32, l+64, l+96) of each
    // scale atom: weight block 0 at columns 0..15 of the buffer, block 1 at
    // 16..31, the token rows of one or two 128-row blocks at 32 + 8 kk (+4).
    const uint32_t lane_base = (uint32_t)((warp & 3) * 32) << 16;
    uint32_t kst = 0;
    bool ok = true;
    for (int t = blockIdx.x; t < total_tiles && ok; t += gridDim.x) {
      const Tile T = decode_tile<kSwiglu, kCap>(t, s_off, s_slot, s_tile, E, N, 2 * BM, 0);
      const int nrb = ((T.x_row0 & 127) + T.n_valid + 127) >> 7;
      for (int ks = 0; ks < ksteps && ok; ++ks, ++kst) {
        const uint32_t s = kst % kStages, par = (kst / kStages) & 1, sb = kst & 1;
        if (!mbar_wait_warp(bar_sfw_data + 8 * s, par, abort_flag, dev_status)) { ok = false; break; }
        if (!mbar_wait_warp(bar_sfx_data + 8 * s, par, abort_flag, dev_status)) { ok = false; break; }
        if (kst >= 2 &&
            !mbar_wait_warp(bar_sf_free + 8 * sb, ((kst - 2) >> 1) & 1, abort_flag, dev_status)) {
          ok = false; break;
        }
        tc_fence_after();
        const uint32_t tcol = tmem_base + lane_base + R::kSf + sb * kSfStride;
        const uint32_t sfw = sbase + R::OFF_SFW + s * SFW2_STAGE + lane * 16;
        const uint32_t sfx = sbase + R::OFF_SFX + s * R::SFX_BYTES + lane * 16;
        if constexpr (kMx) {
          // an MX atom covers two MMAs (128 elements): each MMA gets its own 4
          // columns with its two scales in bytes 0 and 1 of the row's word
#pragma unroll
          for (int a = 0; a < 2; ++a) {
            const uint4 w0 = lds128(sfw + a * 512), w1 = lds128(sfw + kSfStage + a * 512);
            const uint4 x0 = lds128(sfx + a * 512);
            tc_st_x4(tcol + (2 * a) * 4, lo16x4(w0));
            tc_st_x4(tcol + (2 * a + 1) * 4, hi16x4(w0));
            tc_st_x4(tcol + 16 + (2 * a) * 4, lo16x4(w1));
            tc_st_x4(tcol + 16 + (2 * a + 1) * 4, hi16x4(w1));
            tc_st_x4(tcol + 32 + (2 * a) * 8, lo16x4(x0));
            tc_st_x4(tcol + 32 + (2 * a + 1) * 8, hi16x4(x0));
            if (nrb > 1) {
              const uint4 x1 = lds128(sfx + kSfStage + a * 512);
              tc_st_x4(tcol + 32 + (2 * a) * 8 + 4, lo16x4(x1));
              tc_st_x4(tcol + 32 + (2 * a + 1) * 8 + 4, hi16x4(x1));
            }
          }
        } else {
#pragma unroll
          for (int kk = 0; kk < 4; ++kk) tc_st_x4(tcol + kk * 4, lds128(sfw + kk * 512));
#pragma unroll
          for (int kk = 0; kk < 4; ++kk) tc_st_x4(tcol + 16 + kk * 4, lds128(sfw + kSfStage + kk * 512));
#pragma unroll
          for (int kk = 0; kk < 4; ++kk) tc_st_x4(tcol + 32 + kk * 8, lds128(sfx + kk * 512));
          if (nrb > 1) {
#pragma unroll
            for (int kk = 0; kk < 4; ++kk) tc_st_x4(tcol + 32 + kk * 8 + 4, lds128(sfx + kSfStage + kk * 512));
          }
        }
        tc_wait_st();
        tc_fence_before();
        mbar_arrive(bar_sf_full + 8 * sb);
      }
    }
  } else if (warp == W_MMA) {
    // ================================================================ MMA issuer
    uint32_t kst = 0, titer = 0;
    bool ok = true;
    for (int t = blockIdx.x; t < total_tiles && ok; t += gridDim.x, ++titer) {
      const Tile T = decode_tile<kSwiglu, kCap>(t, s_off, s_slot, s_tile, E, N, 2 * BM, 0);
      const uint32_t n_mma = (T.n_valid + 15) & ~15;
      const uint32_t idesc = kMx ? idesc_mxf4_ue8m0(BM, n_mma) : idesc_mxf4nvf4(BM, n_mma);
      const uint32_t xoff = (uint32_t)(T.x_row0 & 127) >> 5;
      // accumulator pair ab: the epilogue of the tile kAccBufs back must have read it
      const uint32_t ab = titer % kAccBufs;
      const uint32_t t_acc = tmem_base + ab * R::kAccPair;
      if (!mbar_wait_warp(bar_acc_empty + 8 * ab, ((titer / kAccBufs) & 1) ^ 1, abort_flag, dev_status)) {
        ok = false; break;
      }
      tc_fence_after();
      for (int ks = 0; ks < ksteps && ok; ++ks, ++kst) {
        const uint32_t s = kst % kStages, par = (kst / kStages) & 1, sb = kst & 1;
        if (!mbar_wait_warp(bar_wfull + 8 * s, par, abort_flag, dev_status)) { ok = false; break; }
        if (!mbar_wait_warp(bar_xfull + 8 * s, par, abort_flag, dev_status)) { ok = false; break; }
        if (!mbar_wait_warp(bar_sf_full + 8 * sb, (kst >> 1) & 1, abort_flag, dev_status)) {
          ok = false; break;
        }
        tc_fence_after();
        if (lane == 0) {
          const uint32_t t_sf = tmem_base + R::kSf + sb * kSfStride;
          const uint64_t dw0 = desc_sw128(sbase + R::OFF_W + s * W2_STAGE);
          const uint64_t dw1 = desc_sw128(sbase + R::OFF_W + s * W2_STAGE + W_STAGE);
          const uint64_t dx = desc_sw128(sbase + R::OFF_X + s * R::X_STAGE);
#pragma unroll
          for (int kk = 0; kk < 4; ++kk) {
            const uint32_t acc = (ks > 0 || kk > 0) ? 1u : 0u;
            // +32 bytes of K per MMA: +2 in the descriptor's 16-byte address field
            if constexpr (kMx) {
              tc_mma_mx(t_acc, dw0 + 2 * kk, dx + 2 * kk, idesc, t_sf + kk * 4, t_sf + 32 + kk * 8 + xoff, acc);
              tc_mma_mx(t_acc + kCap, dw1 + 2 * kk, dx + 2 * kk, idesc, t_sf + 16 + kk * 4,
                        t_sf + 32 + kk * 8 + xoff, acc);
            } else {
              tc_mma(t_acc, dw0 + 2 * kk, dx + 2 * kk, idesc, t_sf + kk * 4, t_sf + 32 + kk * 8 + xoff, acc);
              tc_mma(t_acc + kCap, dw1 + 2 * kk, dx + 2 * kk, idesc, t_sf + 16 + kk * 4, t_sf + 32 + kk * 8 + xoff,
                     acc);
            }
          }
          tc_commit(bar_sf_free + 8 * sb);
          tc_commit(bar_wempty + 8 * s);
          tc_commit(bar_xempty + 8 * s);
        }
        __syncwarp();
      }
      if (!ok) break;
      if (lane == 0) tc_commit(bar_acc_full + 8 * ab);
      __syncwarp();
    }
    if (lane == 0) {
      tc_commit(bar_drain);
      const long long t0 = clock64();
      while (!mbar_try_wait(bar_drain, 0) && clock64() - t0 < kWaitBudgetCycles) {}
    }
    __syncwarp();
  } else {
    // ================================================================ epilogue (warps 2..5 and 11..14)
    const int block = warp >= W_EPI_B ? 1 : 0;
    const int quad = warp & 3;
    const uint32_t lane_base = (uint32_t)(quad * 32) << 16;
    const uint32_t epi = sbase + R::OFF_EPI + (block * 4 + (warp - (block ? W_EPI_B : 2))) * EPI2_WARP_BYTES;
    uint32_t titer = 0;
    for (int t = blockIdx.x; t < total_tiles; t += gridDim.x, ++titer) {
      Tile T = decode_tile<kSwiglu, kCap>(t, s_off, s_slot, s_tile, E, N, 2 * BM, 0);
      if (block) {
        T.w_row0 += BM;
        T.n_col0 += kSwiglu ? BM / 2 : BM;
      }
      const uint32_t ab = titer % kAccBufs;
      if (!mbar_wait_warp(bar_acc_full + 8 * ab, (titer / kAccBufs) & 1, abort_flag, dev_status)) break;
      tc_fence_after();
      const float alpha = kMx ? 1.0f : __fmul_rn(x_gs[T.e], w_gs[T.e]);
      epilogue_tile<kSwiglu, true, kQuantH>(T, tmem_base + lane_base + ab * R::kAccPair + (block ? kCap : 0), alpha,
                                            epi, quad, lane, N, y, amax_out, bar_acc_empty + 8 * ab, false, hq,
                                            dev_status);
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == W_MMA) {
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" :: "r"(tmem_base), "r"(TMEM_COLS) : "memory");
  }
}

}  // namespace w2

nvfp4_status set_wait_budget_w2(long long cycles) {
  return cudaMemcpyToSymbol(c_wait_budget, &cycles, sizeof(cycles)) == cudaSuccess ? NVFP4_OK : NVFP4_ERR_CUDA;
}

template <int kCap, int kSlots, bool kMx>
nvfp4_status launch_ring(const CUtensorMap &tw, const CUtensorMap &tx32, const CUtensorMap &tx64,
                         const CUtensorMap &tx128, const CUtensorMap &tx192, const uint8_t *b_sf, const uint8_t *a_sf,
                         const float *b_gs, const float *a_gs, const int32_t *expert_offsets, int E, int64_t M_total,
                         int64_t N, int64_t K, void *y, bool swiglu, float *amax_out, const HQuantOut *hq,
                         int32_t *dev_status, cudaStream_t stream) {
  using R = w2::W2Ring<kCap, kSlots>;
  auto kern = kMx ? w2::grouped_gemm_w2_kernel<false, false, kCap, kSlots, true>
             : hq ? w2::grouped_gemm_w2_kernel<true, true, kCap, kSlots>
                  : swiglu ? w2::grouped_gemm_w2_kernel<true, false, kCap, kSlots>
                           : w2::grouped_gemm_w2_kernel<false, false, kCap, kSlots>;
  if (!host::set_max_dynamic_smem(reinterpret_cast<const void *>(kern), R::SMEM_BYTES)) return NVFP4_ERR_CUDA;
  // no more CTAs than tiles: each expert has at most m_e / kCap + 1 token chunks per weight-block pair
  const int64_t tile_bound = (N / (2 * BM)) * ((M_total + kCap - 1) / kCap + E);
  const int grid = (int)(tile_bound < host::sm_count() ? tile_bound : host::sm_count());
  kern<<<grid, w2::kThreads, R::SMEM_BYTES, stream>>>(tw, tx32, tx64, tx128, tx192, b_sf, a_sf, b_gs, a_gs,
                                                      expert_offsets, E, (int)M_total, (int)N, (int)K, y, amax_out,
                                                      dev_status, hq ? *hq : HQuantOut{});
  return cudaGetLastError() == cudaSuccess ? NVFP4_OK : NVFP4_ERR_CUDA;
}

// Arguments are validated by the callers; N % 256 == 0, K % 256 == 0, bf16
// output (or SwiGLU h, or NVFP4 h when hq is given; MXFP4 operands, mx, only
// with a plain output and without global scales).
nvfp4_status launch_grouped_gemm_w2(const uint8_t *a_q, const uint8_t *a_sf, const float *a_gs, const uint8_t *b_q,
                                    const uint8_t *b_sf, const float *b_gs, const int32_t *expert_offsets, int E,
                                    int64_t M_total, int64_t N, int64_t K, void *y, bool swiglu, float *amax_out,
                                    const HQuantOut *hq, bool mx, bool deep, int32_t *dev_status,
                                    cudaStream_t stream) {
  const int64_t x_rows = nvfp4_padded_rows_bound(M_total, E);
  CUtensorMap tw, tx32, tx64, tx128, tx192;
  if (!make_map(&tw, b_q, (uint64_t)E * N, (uint64_t)K / 2, 2 * BM)) return NVFP4_ERR_CUDA;
  if (!make_map(&tx32, a_q, (uint64_t)x_rows, (uint64_t)K / 2, 32)) return NVFP4_ERR_CUDA;
  if (!make_map(&tx64, a_q, (uint64_t)x_rows, (uint64_t)K / 2, 64)) return NVFP4_ERR_CUDA;
  if (!make_map(&tx128, a_q, (uint64_t)x_rows, (uint64_t)K / 2, 128)) return NVFP4_ERR_CUDA;
  if (!make_map(&tx192, a_q, (uint64_t)x_rows, (uint64_t)K / 2, 192)) return NVFP4_ERR_CUDA;
  if (mx && (swiglu || hq)) return NVFP4_ERR_UNSUPPORTED_SHAPE;
  if (deep) {
    auto launch = mx ? launch_ring<64, 4, true> : launch_ring<64, 4, false>;
    return launch(tw, tx32, tx64, tx128, tx192, b_sf, a_sf, b_gs, a_gs, expert_offsets, E, M_total, N, K, y, swiglu,
                  amax_out, hq, dev_status, stream);
  }
  auto launch = mx ? launch_ring<BN, 3, true> : launch_ring<BN, 3, false>;
  return launch(tw, tx32, tx64, tx128, tx192, b_sf, a_sf, b_gs, a_gs, expert_offsets, E, M_total, N, K, y, swiglu,
                amax_out, hq, dev_status, stream);
}

}  // namespace gemm
}  // namespace nvfp4
