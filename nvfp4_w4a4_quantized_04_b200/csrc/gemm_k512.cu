// Block-scaled FP4 x FP4 grouped GEMM, 512-element K stages (sm_100a).
//
// The same computation as grouped_gemm_kernel (gemm.cu): for every routed
// expert e, Y_e = (a_gs[e] * b_gs[e]) * X_e W_e^T on the 5th-generation tensor
// cores, the W4A4 routed-expert projections of the "Qwen3.8-Flash-Next-NVFP4"
// page (gate_up_proj / down_proj) on the native 4-bit path the
// "DeepSeek-V4.1-Flash-NVFP4" page's "why NVFP4" section describes.  Same warp
// roles, MMA, scale path, epilogues, persistent tile order and bounded waits.
//
// What differs: a ring slot holds 512 elements of K (two 128-byte K chunks)
// instead of 256, loaded by one 3-D TMA box per operand ({128 bytes, rows, 2
// chunks}, 128-byte swizzle), so a slot's bytes double while the copy
// instructions and barrier rounds per slot stay the same.  Two slots per ring
// keep the bytes in flight of the 256-element kernel's four.  The scales still
// go to tensor memory per 256-element half, through two buffers that the MMA
// releases half by half (sf_free).  The token box is 32, 64, 128 or 192 rows,
// the smallest that holds the tile's tokens.  Measured against the 256-element
// kernel, bit-identical: 2.5-3 % faster on the 512-expert MoE shapes and 8-12 %
// on decode (1-3 tokens per expert), where a stage is mostly weight bytes.
// Used when K % 512 == 0 (nvfp4_gemm_select_kernel mode 0), for NVFP4 and for
// MXFP4 operands (kind::mxf4, UE8M0 scales per 32 elements, no global scales).
#include "gemm_common.cuh"
#include "host_util.cuh"

namespace nvfp4 {
namespace gemm {
namespace {

// Ring layout for tiles of at most kCap tokens with kSlots slots of 512
// elements of K.  (192, 2) is the general kernel; (64, 3) serves groups of a
// few tokens (decode), where the smaller token slots leave room for a third
// weight slot: 96 KB of weights in flight per SM instead of 64 KB, which a
// private probe measured as 1.076 -> 0.980 ms on the 384-expert decode layer.
template <int kCap, int kSlots>
struct Ring {
  static constexpr int W_STAGE2 = 2 * W_STAGE;                  // 32 KB
  static constexpr int X_STAGE2 = 2 * kCap * 128;               // two K halves of up to kCap token rows
  static constexpr int SFW_STAGE2 = 4096;                       // 128 weight rows x 32 scales
  static constexpr int SFX_STAGE2 = kCap > 64 ? 8192 : 4096;    // one or two 128-row blocks x 4 KB
  static constexpr int OFF_W = 0;
  static constexpr int OFF_X = OFF_W + kSlots * W_STAGE2;
  static constexpr int OFF_SFW = OFF_X + kSlots * X_STAGE2;
  static constexpr int OFF_SFX = OFF_SFW + kSlots * SFW_STAGE2;
  static constexpr int OFF_EPI = OFF_SFX + kSlots * SFX_STAGE2;
  static constexpr int OFF_BAR = OFF_EPI + 4 * EPI_WARP_BYTES;
  // wfull[S], wempty[S], xfull[S], xempty[S], sf_full[2], sf_free[2], acc_full[2], acc_empty[2], drain,
  // sfw_data[S], sfx_data[S]
  static constexpr int NUM_BARS = 4 * kSlots + 2 + 2 + 2 + 2 + 1 + 2 * kSlots;
  static constexpr int OFF_MISC = OFF_BAR + NUM_BARS * 8;
  static constexpr int OFF_GROUPS = OFF_MISC + 16;
  static constexpr int SMEM_BYTES = OFF_GROUPS + GROUP_TABLE_BYTES + 1024;
  static_assert(SMEM_BYTES <= 232448, "shared memory budget");
  static_assert(OFF_X % 1024 == 0 && X_STAGE2 % 1024 == 0, "128-byte swizzle atoms");
  static_assert(kSlots <= 8, "armed-slot bookkeeping");
};
using RingWide = Ring<192, 2>;
using RingDeep = Ring<64, 3>;

// Rows of the token box: the smallest of 32, 64, 128, 192 that holds the tile.
__device__ __forceinline__ int token_box_rows(int n_valid) {
  return n_valid <= 32 ? 32 : n_valid <= 64 ? 64 : n_valid <= 128 ? 128 : 192;
}

// Scales of one 256-element half into tensor memory (the 256-element kernel's
// sf_stage_to_tmem with the second token row block 4 KB further on).
__device__ __forceinline__ void sf_half_to_tmem(uint32_t tcol, uint32_t sfw_addr, uint32_t sfx_addr, int nrb) {
#pragma unroll
  for (int kk = 0; kk < 4; ++kk) tc_st_x4(tcol + kk * 4, lds128(sfw_addr + kk * 512));
#pragma unroll
  for (int kk = 0; kk < 4; ++kk) tc_st_x4(tcol + 16 + kk * 8, lds128(sfx_addr + kk * 512));
  if (nrb > 1) {
#pragma unroll
    for (int kk = 0; kk < 4; ++kk) tc_st_x4(tcol + 16 + kk * 8 + 4, lds128(sfx_addr + 4096 + kk * 512));
  }
  tc_wait_st();
}

// MXFP4 form: a 512-byte atom holds 4 UE8M0 scales per row = 128 elements =
// two MMAs, so a 256-element half has two atoms per row block; each MMA gets
// its own 4 tensor-memory columns with its two scales in bytes 0 and 1 (the
// 256-element kernel's sf_stage_to_tmem_mx, second row block 4 KB on).
__device__ __forceinline__ void sf_half_to_tmem_mx(uint32_t tcol, uint32_t sfw_addr, uint32_t sfx_addr, int nrb) {
#pragma unroll
  for (int a = 0; a < 2; ++a) {
    const uint4 w = lds128(sfw_addr + a * 512);
    tc_st_x4(tcol + (2 * a) * 4, lo16x4(w));
    tc_st_x4(tcol + (2 * a + 1) * 4, hi16x4(w));
  }
#pragma unroll
  for (int a = 0; a < 2; ++a) {
    const uint4 x = lds128(sfx_addr + a * 512);
    tc_st_x4(tcol + 16 + (2 * a) * 8, lo16x4(x));
    tc_st_x4(tcol + 16 + (2 * a + 1) * 8, hi16x4(x));
  }
  if (nrb > 1) {
#pragma unroll
    for (int a = 0; a < 2; ++a) {
      const uint4 x = lds128(sfx_addr + 4096 + a * 512);
      tc_st_x4(tcol + 16 + (2 * a) * 8 + 4, lo16x4(x));
      tc_st_x4(tcol + 16 + (2 * a + 1) * 8 + 4, hi16x4(x));
    }
  }
  tc_wait_st();
}

// kMx: MXFP4 operands (kind::mxf4, one UE8M0 scale per 32 elements, no global
// scales); otherwise NVFP4 (kind::mxf4nvf4, E4M3 per 16 elements).  kCap and
// kSlots pick the ring layout (Ring above).
template <bool kSwiglu, bool kBf16Out, bool kQuantH, bool kMx, int kCap = 192, int kSlots = 2>
__global__ void __launch_bounds__(NUM_THREADS, 1) grouped_gemm_k512_kernel(
    const __grid_constant__ CUtensorMap tmap_w, const __grid_constant__ CUtensorMap tmap_x32,
    const __grid_constant__ CUtensorMap tmap_x64, const __grid_constant__ CUtensorMap tmap_x128,
    const __grid_constant__ CUtensorMap tmap_x192,
    const uint8_t *__restrict__ w_sf, const uint8_t *__restrict__ x_sf,
    const float *__restrict__ w_gs, const float *__restrict__ x_gs,
    const int32_t *__restrict__ expert_offsets, int E, int M_total, int N, int K,
    void *__restrict__ y, float *__restrict__ amax_out, int32_t *dev_status, HQuantOut hq) {
  using R = Ring<kCap, kSlots>;
  constexpr int S_W = kSlots, S_X = kSlots;
  constexpr int W_STAGE2 = R::W_STAGE2, X_STAGE2 = R::X_STAGE2, SFW_STAGE2 = R::SFW_STAGE2,
                SFX_STAGE2 = R::SFX_STAGE2;
  constexpr int OFF_W = R::OFF_W, OFF_X = R::OFF_X, OFF_SFW = R::OFF_SFW, OFF_SFX = R::OFF_SFX,
                OFF_EPI = R::OFF_EPI, OFF_BAR = R::OFF_BAR, OFF_MISC = R::OFF_MISC, OFF_GROUPS = R::OFF_GROUPS;
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
  const uint32_t sbase = smem_u32(smem);
  const uint32_t bar_wfull = sbase + OFF_BAR;
  const uint32_t bar_wempty = bar_wfull + 8 * S_W;
  const uint32_t bar_xfull = bar_wempty + 8 * S_W;
  const uint32_t bar_xempty = bar_xfull + 8 * S_X;
  const uint32_t bar_sf_full = bar_xempty + 8 * S_X;     // [2], count 128
  const uint32_t bar_sf_free = bar_sf_full + 16;         // [2], count 1 (MMA commit)
  const uint32_t bar_acc_full = bar_sf_free + 16;
  const uint32_t bar_acc_empty = bar_acc_full + 16;
  const uint32_t bar_drain = bar_acc_empty + 16;
  // A slot's scale bytes land on barriers of their own (weight and token
  // scales, one per producer), so the scale warps can stage them into tensor
  // memory while the slot's large weight and token copies are still arriving.
  const uint32_t bar_sfw_data = bar_drain + 8;            // [S_W], count 1
  const uint32_t bar_sfx_data = bar_sfw_data + 8 * S_W;   // [S_X], count 1
  volatile uint32_t *tmem_holder = reinterpret_cast<volatile uint32_t *>(smem + OFF_MISC);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + OFF_MISC + 4);
  int32_t *s_off = reinterpret_cast<int32_t *>(smem + OFF_GROUPS);
  int32_t *s_slot = s_off + (kMaxExperts + 1);
  int32_t *s_tile = s_slot + (kMaxExperts + 1);
  int32_t *s_scratch = s_tile + (kMaxExperts + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int n_mtiles = N / BM;
  const int ksteps = K / 512;

  if (threadIdx.x == 0) {
    *abort_flag = 0;
    for (int s = 0; s < S_W; ++s) {
      mbar_init(bar_wfull + 8 * s, 1);
      mbar_init(bar_wempty + 8 * s, 1);
      mbar_init(bar_sfw_data + 8 * s, 1);
    }
    for (int s = 0; s < S_X; ++s) {
      mbar_init(bar_xfull + 8 * s, 1);
      mbar_init(bar_xempty + 8 * s, 1);
      mbar_init(bar_sfx_data + 8 * s, 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(bar_sf_full + 8 * b, 128);
      mbar_init(bar_sf_free + 8 * b, 1);
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
  build_tile_tables<kCap>(expert_offsets, E, M_total, n_mtiles, s_off, s_slot, s_tile, s_scratch, dev_status);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_holder;
  const int total_tiles = s_tile[E];
  // bytes per 128-row block of scales, and per 256-element half of one row block
  const int64_t sf_row_stride = (int64_t)(K / (kMx ? 128 : 64)) * 512;
  constexpr uint32_t kHalfSf = kMx ? 1024u : 2048u;

  if (warp == W_PRODUCER || warp == W_XLOAD) {
    if (lane == 0) {
      const bool is_w = warp == W_PRODUCER;
      // bring the tensor maps into the TMA unit's descriptor cache up front
      if (is_w) {
        prefetch_tensormap(&tmap_w);
      } else {
        prefetch_tensormap(&tmap_x32);
        prefetch_tensormap(&tmap_x64);
        prefetch_tensormap(&tmap_x128);
        prefetch_tensormap(&tmap_x192);
      }
      const uint64_t pol = is_w ? policy_evict_first() : policy_evict_last();
      const uint32_t bar_full = is_w ? bar_wfull : bar_xfull, bar_empty = is_w ? bar_wempty : bar_xempty;
      const uint32_t bar_sfd = is_w ? bar_sfw_data : bar_sfx_data;
      int stage = 0;
      uint32_t phase = 0;
      bool armed[S_W] = {}; uint32_t armed_parity[S_W] = {};
      bool ok = true;
      for (int t = blockIdx.x; t < total_tiles && ok; t += gridDim.x) {
        const Tile T = decode_tile<kSwiglu, kCap>(t, s_off, s_slot, s_tile, E, N, BM, 0);
        const int xr0 = T.x_row0 & ~127;
        const int nrb = ((T.x_row0 & 127) + T.n_valid + 127) >> 7;
        const int xbox = token_box_rows(T.n_valid);
        const CUtensorMap *xmap = xbox == 32 ? &tmap_x32 : xbox == 64 ? &tmap_x64 : xbox == 128 ? &tmap_x128 : &tmap_x192;
        const uint32_t bytes = is_w ? (uint32_t)W_STAGE2 : (uint32_t)(2 * xbox * 128);
        const uint32_t sf_bytes = is_w ? 2 * kHalfSf : (uint32_t)nrb * 2 * kHalfSf;
        const uint8_t *sfw_tile = w_sf + (int64_t)(T.w_row0 >> 7) * sf_row_stride;
        const uint8_t *sfx_tile = x_sf + (int64_t)(xr0 >> 7) * sf_row_stride;
        for (int ks = 0; ks < ksteps; ++ks) {
          if (!mbar_wait(bar_empty + 8 * stage, phase ^ 1, abort_flag, dev_status)) { ok = false; break; }
          const uint32_t fb = bar_full + 8 * stage, sb = bar_sfd + 8 * stage;
          // the scale bytes first, on their own barrier, then the large copy
          mbar_arrive_expect_tx(sb, sf_bytes);
          mbar_arrive_expect_tx(fb, bytes);
          armed[stage] = true; armed_parity[stage] = phase;
          if (is_w) {
            bulk_load(sbase + OFF_SFW + stage * SFW_STAGE2, sfw_tile + ks * 2 * kHalfSf, 2 * kHalfSf, sb);
            tma_load_3d(sbase + OFF_W + stage * W_STAGE2, &tmap_w, 0, T.w_row0, 2 * ks, fb, pol);
          } else {
            for (int rb = 0; rb < nrb; ++rb)
              bulk_load(sbase + OFF_SFX + stage * SFX_STAGE2 + rb * 4096, sfx_tile + rb * sf_row_stride + ks * 2 * kHalfSf,
                        2 * kHalfSf, sb);
            tma_load_3d(sbase + OFF_X + stage * X_STAGE2, xmap, 0, T.x_row0, 2 * ks, fb, pol);
          }
          if (++stage == S_W) { stage = 0; phase ^= 1; }
        }
      }
      for (int s = 0; s < S_W; ++s) {
        if (!armed[s]) continue;
        long long t0 = clock64();
        while (!mbar_try_wait(bar_full + 8 * s, armed_parity[s]) && clock64() - t0 < kWaitBudgetCycles) {}
        t0 = clock64();
        while (!mbar_try_wait(bar_sfd + 8 * s, armed_parity[s]) && clock64() - t0 < kWaitBudgetCycles) {}
      }
    }
  } else if (warp >= W_SF0 && warp < W_SF0 + 4) {
    const uint32_t lane_base = (uint32_t)((warp & 3) * 32) << 16;
    uint32_t kst = 0, hk = 0;
    bool ok = true;
    for (int t = blockIdx.x; t < total_tiles && ok; t += gridDim.x) {
      const Tile T = decode_tile<kSwiglu, kCap>(t, s_off, s_slot, s_tile, E, N, BM, 0);
      const int nrb = ((T.x_row0 & 127) + T.n_valid + 127) >> 7;
      for (int ks = 0; ks < ksteps && ok; ++ks, ++kst) {
        const uint32_t s2 = kst % S_W, par = (kst / S_W) & 1;
        if (!mbar_wait_warp(bar_sfw_data + 8 * s2, par, abort_flag, dev_status)) { ok = false; break; }
        if (!mbar_wait_warp(bar_sfx_data + 8 * s2, par, abort_flag, dev_status)) { ok = false; break; }
        for (int h = 0; h < 2; ++h, ++hk) {
          const uint32_t sb = hk & 1;
          if (hk >= 2 && !mbar_wait_warp(bar_sf_free + 8 * sb, ((hk - 2) >> 1) & 1, abort_flag, dev_status)) {
            ok = false; break;
          }
          tc_fence_after();
          const uint32_t tcol = tmem_base + lane_base + TMEM_SF + sb * TMEM_SF_STRIDE;
          if constexpr (kMx)
            sf_half_to_tmem_mx(tcol, sbase + OFF_SFW + s2 * SFW_STAGE2 + h * kHalfSf + lane * 16,
                               sbase + OFF_SFX + s2 * SFX_STAGE2 + h * kHalfSf + lane * 16, nrb);
          else
            sf_half_to_tmem(tcol, sbase + OFF_SFW + s2 * SFW_STAGE2 + h * kHalfSf + lane * 16,
                            sbase + OFF_SFX + s2 * SFX_STAGE2 + h * kHalfSf + lane * 16, nrb);
          tc_fence_before();
          mbar_arrive(bar_sf_full + 8 * sb);
        }
      }
    }
  } else if (warp == W_MMA) {
    uint32_t kst = 0, hk = 0, titer = 0;
    bool ok = true;
    for (int t = blockIdx.x; t < total_tiles && ok; t += gridDim.x, ++titer) {
      const Tile T = decode_tile<kSwiglu, kCap>(t, s_off, s_slot, s_tile, E, N, BM, 0);
      const uint32_t n_mma = (T.n_valid + 15) & ~15;
      const uint32_t idesc = kMx ? idesc_mxf4_ue8m0(BM, n_mma) : idesc_mxf4nvf4(BM, n_mma);
      const uint32_t x_half = (uint32_t)token_box_rows(T.n_valid) * 128;   // bytes of one K half of the token tile
      const uint32_t xoff = (uint32_t)(T.x_row0 & 127) >> 5;
      const uint32_t ab = titer & 1;
      const uint32_t t_acc = tmem_base + ab * TMEM_ACC_STRIDE;
      if (!mbar_wait_warp(bar_acc_empty + 8 * ab, ((titer >> 1) & 1) ^ 1, abort_flag, dev_status)) { ok = false; break; }
      tc_fence_after();
      for (int ks = 0; ks < ksteps && ok; ++ks, ++kst) {
        const uint32_t s2 = kst % S_W, par = (kst / S_W) & 1;
        if (!mbar_wait_warp(bar_wfull + 8 * s2, par, abort_flag, dev_status)) { ok = false; break; }
        if (!mbar_wait_warp(bar_xfull + 8 * s2, par, abort_flag, dev_status)) { ok = false; break; }
        for (int h = 0; h < 2; ++h, ++hk) {
          const uint32_t sb = hk & 1;
          if (!mbar_wait_warp(bar_sf_full + 8 * sb, (hk >> 1) & 1, abort_flag, dev_status)) { ok = false; break; }
          tc_fence_after();
          if (lane == 0) {
            const uint32_t t_sf = tmem_base + TMEM_SF + sb * TMEM_SF_STRIDE;
            const uint64_t dw = desc_sw128(sbase + OFF_W + s2 * W_STAGE2 + h * W_STAGE);
            const uint64_t dx = desc_sw128(sbase + OFF_X + s2 * X_STAGE2 + h * x_half);
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)
              if constexpr (kMx)
                tc_mma_mx(t_acc, dw + 2 * kk, dx + 2 * kk, idesc, t_sf + kk * 4, t_sf + 16 + kk * 8 + xoff,
                          (ks > 0 || h > 0 || kk > 0) ? 1u : 0u);
              else
                tc_mma(t_acc, dw + 2 * kk, dx + 2 * kk, idesc, t_sf + kk * 4, t_sf + 16 + kk * 8 + xoff,
                       (ks > 0 || h > 0 || kk > 0) ? 1u : 0u);
            tc_commit(bar_sf_free + 8 * sb);
          }
          __syncwarp();
        }
        if (!ok) break;
        if (lane == 0) { tc_commit(bar_wempty + 8 * s2); tc_commit(bar_xempty + 8 * s2); }
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
    const int quad = warp & 3;
    const uint32_t lane_base = (uint32_t)(quad * 32) << 16;
    const uint32_t epi = sbase + OFF_EPI + (warp - 2) * EPI_WARP_BYTES;
    uint32_t titer = 0;
    for (int t = blockIdx.x; t < total_tiles; t += gridDim.x, ++titer) {
      const Tile T = decode_tile<kSwiglu, kCap>(t, s_off, s_slot, s_tile, E, N, BM, 0);
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

}  // namespace

// 3-D view {128 bytes, rows, K/256 chunks} of packed rows, boxes of {128, box_rows, 2}: the
// box lands as two K-chunk tiles [2][box_rows][128 B], each in the 128-byte-swizzled K-major layout.
bool make_map_k512(CUtensorMap *map, const void *base, uint64_t rows, uint64_t row_bytes, uint32_t box_rows) {
  cuuint64_t dims[3] = {128, rows, row_bytes / 128};
  cuuint64_t strides[2] = {row_bytes, 128};
  cuuint32_t box[3] = {128, box_rows, 2};
  return encode_u8_map(map, 3, base, dims, strides, box, CU_TENSOR_MAP_SWIZZLE_128B);
}

nvfp4_status set_wait_budget_k512(long long cycles) {
  return cudaMemcpyToSymbol(c_wait_budget, &cycles, sizeof(cycles)) == cudaSuccess ? NVFP4_OK : NVFP4_ERR_CUDA;
}

namespace {

template <int kCap, int kSlots>
nvfp4_status launch_ring(const CUtensorMap &tw, const CUtensorMap &tx32, const CUtensorMap &tx64,
                         const CUtensorMap &tx128, const CUtensorMap &tx192, const uint8_t *a_sf, const float *a_gs,
                         const uint8_t *b_sf, const float *b_gs, const int32_t *expert_offsets, int E,
                         int64_t M_total, int64_t N, int64_t K, void *y, int variant, float *amax_out,
                         const HQuantOut *hq, int32_t *dev_status, cudaStream_t stream) {
  using R = Ring<kCap, kSlots>;
  auto kern = variant == 5   ? grouped_gemm_k512_kernel<false, true, false, true, kCap, kSlots>
              : variant == 4 ? grouped_gemm_k512_kernel<false, false, false, true, kCap, kSlots>
              : variant == 3 ? grouped_gemm_k512_kernel<true, true, true, false, kCap, kSlots>
              : variant == 2 ? grouped_gemm_k512_kernel<true, true, false, false, kCap, kSlots>
              : variant == 1 ? grouped_gemm_k512_kernel<false, true, false, false, kCap, kSlots>
                             : grouped_gemm_k512_kernel<false, false, false, false, kCap, kSlots>;
  if (!host::set_max_dynamic_smem(reinterpret_cast<const void *>(kern), R::SMEM_BYTES)) return NVFP4_ERR_CUDA;
  // persistent: one CTA per SM, but no more CTAs than tiles can exist (each
  // expert has at most ceil(m_e / kCap) <= m_e / kCap + 1 token chunks)
  const int64_t tile_bound = (N / BM) * ((M_total + kCap - 1) / kCap + E);
  const int grid = (int)(tile_bound < host::sm_count() ? tile_bound : host::sm_count());
  kern<<<grid, NUM_THREADS, R::SMEM_BYTES, stream>>>(tw, tx32, tx64, tx128, tx192, b_sf, a_sf, b_gs, a_gs,
                                                                 expert_offsets, E, (int)M_total, (int)N, (int)K, y,
                                                                 amax_out, dev_status, hq ? *hq : HQuantOut{});
  return cudaGetLastError() == cudaSuccess ? NVFP4_OK : NVFP4_ERR_CUDA;
}

}  // namespace

// Arguments are validated by the callers (nvfp4_grouped_gemm and
// nvfp4_grouped_gemm_swiglu_nvfp4); K % 512 == 0 here.  deep selects the
// 64-token, three-slot ring.
nvfp4_status launch_grouped_gemm_k512(const uint8_t *a_q, const uint8_t *a_sf, const float *a_gs,
                                      const uint8_t *b_q, const uint8_t *b_sf, const float *b_gs,
                                      const int32_t *expert_offsets, int E, int64_t M_total, int64_t N, int64_t K,
                                      void *y, nvfp4_out_dtype out_dtype, bool swiglu, float *amax_out,
                                      const HQuantOut *hq, bool mx, bool deep, int32_t *dev_status,
                                      cudaStream_t stream) {
  const int64_t x_rows = nvfp4_padded_rows_bound(M_total, E);
  CUtensorMap tw, tx32, tx64, tx128, tx192;
  if (!make_map_k512(&tw, b_q, (uint64_t)E * N, (uint64_t)K / 2, 128)) return NVFP4_ERR_CUDA;
  if (!make_map_k512(&tx32, a_q, (uint64_t)x_rows, (uint64_t)K / 2, 32)) return NVFP4_ERR_CUDA;
  if (!make_map_k512(&tx64, a_q, (uint64_t)x_rows, (uint64_t)K / 2, 64)) return NVFP4_ERR_CUDA;
  if (!make_map_k512(&tx128, a_q, (uint64_t)x_rows, (uint64_t)K / 2, 128)) return NVFP4_ERR_CUDA;
  if (!make_map_k512(&tx192, a_q, (uint64_t)x_rows, (uint64_t)K / 2, 192)) return NVFP4_ERR_CUDA;
  const bool bf = out_dtype == NVFP4_OUT_BF16;
  const int variant = mx ? (bf ? 5 : 4) : hq ? 3 : swiglu ? 2 : (bf ? 1 : 0);
  if (deep)
    return launch_ring<64, 3>(tw, tx32, tx64, tx128, tx192, a_sf, a_gs, b_sf, b_gs, expert_offsets, E, M_total, N,
                              K, y, variant, amax_out, hq, dev_status, stream);
  return launch_ring<192, 2>(tw, tx32, tx64, tx128, tx192, a_sf, a_gs, b_sf, b_gs, expert_offsets, E, M_total, N, K,
                             y, variant, amax_out, hq, dev_status, stream);
}

}  // namespace gemm
}  // namespace nvfp4
