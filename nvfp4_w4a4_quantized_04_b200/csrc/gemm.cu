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
//  * Swap-AB: the MMA's M side (128) walks weight rows, the N side (16..256,
//    step 16) walks the tokens of one expert, so a group of m tokens costs
//    roundup(m,16) MMA columns instead of a 128-row tile.
//  * Operands are staged by TMA (128-byte swizzle, K-major, 256 elements of K
//    per stage); the per-16 scales arrive by bulk copy in the tensor-core atom
//    layout (512-byte atoms of 128 rows x 4 scales) and are moved to tensor
//    memory with tcgen05.cp (32x128b, replicated to the four lane quadrants).
//  * Persistent grid (one CTA per SM), warp-specialised: warp 0 issues TMA,
//    warp 1 issues MMAs, warps 2..5 drain the accumulator (tcgen05.ld) and
//    store Y.  A 4-stage mbarrier ring links TMA and MMA; two barriers hand
//    the accumulator between MMA and epilogue.
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
constexpr int BN = 256;                 // max tokens per tile (MMA N)
constexpr int BK = 256;                 // K elements per stage = 128 bytes of codes
constexpr int STAGES = 4;
constexpr int W_STAGE = BM * 128;       // 16 KB
constexpr int X_STAGE = BN * 128;       // 32 KB
constexpr int SFW_STAGE = 2048;         // 128 rows x 16 scales (4 atoms)
constexpr int SFX_STAGE = 4096;         // 256 rows x 16 scales (2 x 4 atoms)
constexpr int OFF_W = 0;
constexpr int OFF_X = OFF_W + STAGES * W_STAGE;
constexpr int OFF_SFW = OFF_X + STAGES * X_STAGE;
constexpr int OFF_SFX = OFF_SFW + STAGES * SFW_STAGE;
constexpr int OFF_BAR = OFF_SFX + STAGES * SFX_STAGE;        // 8-byte mbarriers
constexpr int NUM_BARS = 2 * STAGES + 3;                      // full, empty, acc_full, acc_empty, drain
constexpr int OFF_MISC = OFF_BAR + NUM_BARS * 8;              // tmem base, abort flag
constexpr int OFF_GROUPS = OFF_MISC + 16;                     // off / slot / tile arrays
constexpr int kMaxExperts = 768;
constexpr int SMEM_BYTES = OFF_GROUPS + 3 * (kMaxExperts + 1) * 4 + 64 + 1024;  // +1024 for alignment
constexpr int NUM_THREADS = 192;
constexpr uint32_t TMEM_COLS = 512;
constexpr uint32_t TMEM_SFW = 256;      // column of the weight scales (4 kk x 4 columns)
constexpr uint32_t TMEM_SFX = 288;      // column of the token scales (4 kk x 8 columns)
constexpr long long kWaitBudgetCycles = 4000000000LL;   // ~2 s at 2 GHz

static_assert(SMEM_BYTES <= 232448, "shared memory budget");

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

// Scale atom for tcgen05.cp: 32 rows x 16 bytes, no swizzle, 8-row core
// matrices 128 bytes apart.
__device__ __forceinline__ uint64_t desc_sf(uint32_t addr) {
  return (uint64_t)((addr & 0x3FFFFu) >> 4) | ((uint64_t)(128 >> 4) << 32) | ((uint64_t)1 << 46);
}

__device__ __forceinline__ void tc_cp_sf(uint32_t taddr, uint64_t desc) {
  asm volatile("tcgen05.cp.cta_group::1.32x128b.warpx4 [%0], %1;" :: "r"(taddr), "l"(desc) : "memory");
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

__device__ __forceinline__ void tc_ld32(uint32_t taddr, uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
      "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
        "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]),
        "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr));
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

// Instruction descriptor, kind::mxf4nvf4: E2M1 x E2M1, K-major both,
// UE4M3 scales, M = 128, N = n (multiple of 16).
__device__ __forceinline__ uint32_t idesc_mxf4nvf4(uint32_t n) {
  return (1u << 7) | (1u << 10) | ((n >> 3) << 17) | ((uint32_t)(BM >> 4) << 24);
}

// ------------------------------------------------------------------ tile map
struct Tile {
  int e;          // expert
  int w_row0;     // first weight row (over E*N rows)
  int n_col0;     // first output column
  int x_row0;     // first activation row (slot space)
  int y_row0;     // first output row
  int n_valid;    // tokens in this tile (1..256)
};

__device__ __forceinline__ Tile decode_tile(int t, const int32_t *s_off, const int32_t *s_slot,
                                            const int32_t *s_tile, int E, int n_mtiles, int N) {
  Tile T;
  const int e = upper_group(s_tile, E, t);
  const int m_e = s_off[e + 1] - s_off[e];
  const int nch = (m_e + BN - 1) / BN;
  const int local = t - s_tile[e];
  const int mt = local / nch, ch = local - mt * nch;
  T.e = e;
  T.n_col0 = mt * BM;
  T.w_row0 = e * N + mt * BM;
  T.x_row0 = s_slot[e] + ch * BN;
  T.y_row0 = s_off[e] + ch * BN;
  T.n_valid = min(BN, m_e - ch * BN);
  (void)n_mtiles;
  return T;
}

// ------------------------------------------------------------------ kernel
template <bool kBf16Out>
__global__ void __launch_bounds__(NUM_THREADS, 1) grouped_gemm_kernel(
    const __grid_constant__ CUtensorMap tmap_w, const __grid_constant__ CUtensorMap tmap_x,
    const uint8_t *__restrict__ w_sf, const uint8_t *__restrict__ x_sf,
    const float *__restrict__ w_gs, const float *__restrict__ x_gs,
    const int32_t *__restrict__ expert_offsets, int E, int M_total, int N, int K,
    void *__restrict__ y, int32_t *dev_status) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
  const uint32_t sbase = smem_u32(smem);
  const uint32_t bar_full = sbase + OFF_BAR;
  const uint32_t bar_empty = bar_full + 8 * STAGES;
  const uint32_t bar_acc_full = bar_empty + 8 * STAGES;
  const uint32_t bar_acc_empty = bar_acc_full + 8;
  const uint32_t bar_drain = bar_acc_empty + 8;
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
      mbar_init(bar_full + 8 * s, 1);
      mbar_init(bar_empty + 8 * s, 1);
    }
    mbar_init(bar_acc_full, 1);
    mbar_init(bar_acc_empty, 128);
    mbar_init(bar_drain, 1);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;"
                 :: "r"(smem_u32((const void *)tmem_holder)), "r"(TMEM_COLS) : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  __syncthreads();
  // slot starts (128-aligned groups) and tile starts, one thread (E <= 768)
  if (threadIdx.x == 0) {
    int32_t slot = 0, tiles = 0;
    for (int e = 0; e < E; ++e) {
      const int32_t m = s_off[e + 1] - s_off[e];
      s_slot[e] = slot;
      s_tile[e] = tiles;
      slot += (m + kSlotAlign - 1) / kSlotAlign * kSlotAlign;
      tiles += n_mtiles * ((m + BN - 1) / BN);
    }
    s_slot[E] = slot;
    s_tile[E] = tiles;
  }
  (void)s_scratch;
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_holder;
  const int total_tiles = s_tile[E];

  if (warp == 0) {
    // ================================================================ TMA producer
    if (lane == 0) {
      const uint64_t pol_w = policy_evict_first();
      const uint64_t pol_x = policy_evict_last();
      const int64_t sf_row_stride = (int64_t)(K / 64) * 512;   // bytes per 128-row block of scales
      int stage = 0;
      uint32_t phase = 0;
      bool armed[STAGES] = {};
      uint32_t armed_parity[STAGES] = {};
      bool ok = true;
      for (int t = blockIdx.x; t < total_tiles && ok; t += gridDim.x) {
        const Tile T = decode_tile(t, s_off, s_slot, s_tile, E, n_mtiles, N);
        const int rows_ld = (T.n_valid + 31) & ~31;
        const int nrb = (T.n_valid + 127) >> 7;
        const uint32_t bytes = W_STAGE + rows_ld * 128 + SFW_STAGE + nrb * 2048;
        const uint8_t *sfw_tile = w_sf + (int64_t)(T.w_row0 >> 7) * sf_row_stride;
        const uint8_t *sfx_tile = x_sf + (int64_t)(T.x_row0 >> 7) * sf_row_stride;
        for (int ks = 0; ks < ksteps; ++ks) {
          if (!mbar_wait(bar_empty + 8 * stage, phase ^ 1, abort_flag, dev_status)) { ok = false; break; }
          const uint32_t fb = bar_full + 8 * stage;
          mbar_arrive_expect_tx(fb, bytes);
          armed[stage] = true;
          armed_parity[stage] = phase;
          tma_load_2d(sbase + OFF_W + stage * W_STAGE, &tmap_w, ks * 128, T.w_row0, fb, pol_w);
          for (int i = 0; i < rows_ld / 32; ++i)
            tma_load_2d(sbase + OFF_X + stage * X_STAGE + i * 4096, &tmap_x, ks * 128, T.x_row0 + 32 * i, fb, pol_x);
          bulk_load(sbase + OFF_SFW + stage * SFW_STAGE, sfw_tile + ks * 2048, 2048, fb);
          for (int rb = 0; rb < nrb; ++rb)
            bulk_load(sbase + OFF_SFX + stage * SFX_STAGE + rb * 2048, sfx_tile + rb * sf_row_stride + ks * 2048,
                      2048, fb);
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
  } else if (warp == 1) {
    // ================================================================ MMA issuer
    int stage = 0;
    uint32_t phase = 0, acc_phase = 0;
    bool ok = true;
    const uint32_t t_acc = tmem_base;
    const uint32_t t_sfw = tmem_base + TMEM_SFW;
    const uint32_t t_sfx = tmem_base + TMEM_SFX;
    for (int t = blockIdx.x; t < total_tiles && ok; t += gridDim.x) {
      const Tile T = decode_tile(t, s_off, s_slot, s_tile, E, n_mtiles, N);
      const uint32_t n_mma = (T.n_valid + 15) & ~15;
      const int nrb = (T.n_valid + 127) >> 7;
      const uint32_t idesc = idesc_mxf4nvf4(n_mma);
      if (!mbar_wait_warp(bar_acc_empty, acc_phase ^ 1, abort_flag, dev_status)) { ok = false; break; }
      tc_fence_after();
      for (int ks = 0; ks < ksteps; ++ks) {
        if (!mbar_wait_warp(bar_full + 8 * stage, phase, abort_flag, dev_status)) { ok = false; break; }
        tc_fence_after();
        if (lane == 0) {
          const uint32_t w_addr = sbase + OFF_W + stage * W_STAGE;
          const uint32_t x_addr = sbase + OFF_X + stage * X_STAGE;
          const uint32_t sfw_addr = sbase + OFF_SFW + stage * SFW_STAGE;
          const uint32_t sfx_addr = sbase + OFF_SFX + stage * SFX_STAGE;
#pragma unroll
          for (int kk = 0; kk < 4; ++kk) {
            tc_cp_sf(t_sfw + kk * 4, desc_sf(sfw_addr + kk * 512));
            for (int rb = 0; rb < nrb; ++rb) tc_cp_sf(t_sfx + kk * 8 + rb * 4, desc_sf(sfx_addr + rb * 2048 + kk * 512));
          }
#pragma unroll
          for (int kk = 0; kk < 4; ++kk) {
            tc_mma(t_acc, desc_sw128(w_addr + kk * 32), desc_sw128(x_addr + kk * 32), idesc, t_sfw + kk * 4,
                   t_sfx + kk * 8, (ks > 0 || kk > 0) ? 1u : 0u);
          }
          tc_commit(bar_empty + 8 * stage);
        }
        __syncwarp();
        if (++stage == STAGES) { stage = 0; phase ^= 1; }
      }
      if (!ok) break;
      if (lane == 0) tc_commit(bar_acc_full);
      __syncwarp();
      acc_phase ^= 1;
    }
    // Drain: all MMAs / copies this thread issued complete before TMEM is freed.
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
    uint32_t acc_phase = 0;
    for (int t = blockIdx.x; t < total_tiles; t += gridDim.x) {
      const Tile T = decode_tile(t, s_off, s_slot, s_tile, E, n_mtiles, N);
      if (!mbar_wait_warp(bar_acc_full, acc_phase, abort_flag, dev_status)) break;
      tc_fence_after();
      const float alpha = __fmul_rn(x_gs[T.e], w_gs[T.e]);
      const int n_col = T.n_col0 + quad * 32 + lane;
      for (int c0 = 0; c0 < T.n_valid; c0 += 32) {
        uint32_t r[32];
        tc_ld32(tmem_base + lane_base + (uint32_t)c0, r);
        const int lim = min(32, T.n_valid - c0);
        if (kBf16Out) {
          __nv_bfloat16 *yp = reinterpret_cast<__nv_bfloat16 *>(y) + (int64_t)(T.y_row0 + c0) * N + n_col;
#pragma unroll
          for (int i = 0; i < 32; ++i)
            if (i < lim) yp[(int64_t)i * N] = __float2bfloat16_rn(__fmul_rn(__uint_as_float(r[i]), alpha));
        } else {
          float *yp = reinterpret_cast<float *>(y) + (int64_t)(T.y_row0 + c0) * N + n_col;
#pragma unroll
          for (int i = 0; i < 32; ++i)
            if (i < lim) yp[(int64_t)i * N] = __fmul_rn(__uint_as_float(r[i]), alpha);
        }
      }
      tc_fence_before();
      mbar_arrive(bar_acc_empty);
      acc_phase ^= 1;
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) {
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
bool g_attr_set[2] = {false, false};

}  // namespace

extern "C" nvfp4_status nvfp4_grouped_gemm(const uint8_t *a_q, const uint8_t *a_sf, const float *a_gs,
                                           const uint8_t *b_q, const uint8_t *b_sf, const float *b_gs,
                                           const int32_t *expert_offsets, int num_experts, int64_t M_total,
                                           int64_t N, int64_t K, void *y, nvfp4_out_dtype out_dtype,
                                           nvfp4_epilogue epi, void *workspace, int32_t *dev_status,
                                           cudaStream_t stream) {
  (void)workspace;
  if (epi != NVFP4_EPI_NONE) return NVFP4_ERR_INVALID_ARG;
  if (out_dtype != NVFP4_OUT_F32 && out_dtype != NVFP4_OUT_BF16) return NVFP4_ERR_INVALID_ARG;
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
  CUtensorMap tw, tx;
  if (!make_map(&tw, b_q, (uint64_t)E * N, (uint64_t)K / 2, 128)) return NVFP4_ERR_CUDA;
  if (!make_map(&tx, a_q, (uint64_t)x_rows, (uint64_t)K / 2, 32)) return NVFP4_ERR_CUDA;
  if (g_sms == 0) {
    int dev = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&g_sms, cudaDevAttrMultiProcessorCount, dev);
    if (g_sms <= 0) g_sms = 148;
  }
  const int bf = out_dtype == NVFP4_OUT_BF16;
  auto kern = bf ? gemm::grouped_gemm_kernel<true> : gemm::grouped_gemm_kernel<false>;
  if (!g_attr_set[bf]) {
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, gemm::SMEM_BYTES) != cudaSuccess)
      return NVFP4_ERR_CUDA;
    g_attr_set[bf] = true;
  }
  kern<<<g_sms, gemm::NUM_THREADS, gemm::SMEM_BYTES, stream>>>(tw, tx, b_sf, a_sf, b_gs, a_gs, expert_offsets, E,
                                                               (int)M_total, (int)N, (int)K, y, dev_status);
  return cudaGetLastError() == cudaSuccess ? NVFP4_OK : NVFP4_ERR_CUDA;
}
