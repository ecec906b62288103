// Shared pieces of the block-scaled FP4 grouped GEMM kernels (sm_100a): the
// tile constants, PTX wrappers for mbarriers, TMA and the tcgen05 tensor-core
// instructions, the expert/tile tables, the scale-factor copy into tensor
// memory and the accumulator epilogue.  Included by gemm.cu (one CTA per
// tile) and gemm_pair.cu (a CTA pair per tile, cta_group::2).
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <cudaTypedefs.h>
#include <stdint.h>

#include <mutex>

#include "common.cuh"

namespace nvfp4 {
namespace gemm {

constexpr int BM = 128;                 // weight rows per CTA (MMA M of one CTA)
constexpr int BN = 192;                 // max tokens per tile (MMA N)
constexpr int BK = 256;                 // K elements per stage = 128 bytes of codes
constexpr int W_STAGE = BM * 128;       // 16 KB
constexpr int SFW_STAGE = 2048;         // 128 rows x 16 scales (4 atoms)
constexpr int SFX_STAGE = 4096;         // up to 2 row blocks x 4 atoms
constexpr int EPI_WARP_BYTES = 32 * 32 * 4;                   // 32 tokens x 32 columns, fp32
constexpr int kMaxExperts = 1024;
constexpr int NUM_WARPS = 11;
constexpr int NUM_THREADS = NUM_WARPS * 32;
constexpr int GROUP_TABLE_BYTES = 3 * (kMaxExperts + 1) * 4 + 2 * NUM_WARPS * 4;   // off / slot / tile + scan scratch
constexpr uint32_t TMEM_COLS = 512;
constexpr uint32_t TMEM_ACC_STRIDE = BN;       // accumulator b at column b*192
constexpr uint32_t TMEM_SF = 2 * BN;           // scale buffers at 384 and 448
constexpr uint32_t TMEM_SF_STRIDE = 64;        // per buffer: W scales 16 cols, token scales 32 cols
constexpr long long kWaitBudgetCycles = 4000000000LL;   // ~2 s at 2 GHz
// Budget of the main-loop waits (mbar_wait), one copy per translation unit.
// Only a test lowers it (nvfp4_gemm_set_wait_budget, one-CTA kernel) to force
// the timeout path; the drains at the end of a kernel always use
// kWaitBudgetCycles, so no copy or MMA is ever left in flight.
static __constant__ long long c_wait_budget = kWaitBudgetCycles;

// warp roles (warps 2..5: epilogue, lane quadrants 2,3,0,1)
constexpr int W_PRODUCER = 0;     // weight tiles + weight scales
constexpr int W_MMA = 1;
constexpr int W_SF0 = 6;          // 6..9: scale factors smem -> tensor memory (quadrants 2,3,0,1)
constexpr int W_XLOAD = 10;       // token tiles + token scales

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

// Non-blocking form: returns at once whether the phase has completed.
__device__ __forceinline__ bool mbar_test_wait(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile("{ .reg .pred p; mbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2; selp.u32 %0, 1, 0, p; }"
               : "=r"(ok) : "r"(bar), "r"(parity) : "memory");
  return ok != 0;
}

// Same, with cluster-scope acquire: for barriers that the peer CTA of a pair
// arrives on remotely.
__device__ __forceinline__ bool mbar_try_wait_cluster(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{ .reg .pred p; mbarrier.try_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2; selp.u32 %0, 1, 0, p; }"
      : "=r"(ok) : "r"(bar), "r"(parity) : "memory");
  return ok != 0;
}

// Store to a 32-bit word of another CTA of the cluster (address from mapa).
__device__ __forceinline__ void st_cluster_u32(uint32_t addr, uint32_t v) {
  asm volatile("st.shared::cluster.u32 [%0], %1;" :: "r"(addr), "r"(v) : "memory");
}

// Bounded wait.  Returns false (and raises the CTA abort flag plus a
// TIMEOUT status) if the phase did not complete within the budget, or if
// another role has already aborted.  peer_abort (a cluster address, 0 for
// none) receives the abort flag too, so a paired CTA leaves its loops as well.
template <bool kCluster = false>
__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity, volatile int *abort_flag,
                                          int32_t *dev_status, uint32_t peer_abort = 0) {
  // try_wait may suspend the thread inside the instruction until the phase
  // completes, so a lowered (test) budget polls with test_wait instead
  const bool poll = !kCluster && c_wait_budget < kWaitBudgetCycles;
  auto try_once = [&]() {
    if (poll) return mbar_test_wait(bar, parity);
    return kCluster ? mbar_try_wait_cluster(bar, parity) : mbar_try_wait(bar, parity);
  };
  if (try_once()) return true;
  const long long t0 = clock64();
  while (true) {
    if (try_once()) return true;
    if (*abort_flag) return false;
    if (clock64() - t0 > c_wait_budget) {
      *abort_flag = 1;
      if (peer_abort) st_cluster_u32(peer_abort, 1u);
      report(dev_status, NVFP4_ERR_TIMEOUT);
      return false;
    }
  }
}

// Warp-wide bounded wait: every lane waits, the result is made uniform so
// that no .sync.aligned tcgen05 instruction ever runs on a partial warp.
template <bool kCluster = false>
__device__ __forceinline__ bool mbar_wait_warp(uint32_t bar, uint32_t parity, volatile int *abort_flag,
                                               int32_t *dev_status, uint32_t peer_abort = 0) {
  const bool ok = mbar_wait<kCluster>(bar, parity, abort_flag, dev_status, peer_abort);
  return __all_sync(0xffffffffu, ok) != 0;
}

__device__ __forceinline__ void tma_load_2d(uint32_t dst, const CUtensorMap *map, int32_t x, int32_t y,
                                            uint32_t bar, uint64_t policy) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes.L2::cache_hint"
      " [%0], [%1, {%2, %3}], [%4], %5;"
      :: "r"(dst), "l"(map), "r"(x), "r"(y), "r"(bar), "l"(policy) : "memory");
}

// Fetch a tensor map (a __grid_constant__ kernel parameter) into the TMA
// descriptor cache ahead of its first copy.
__device__ __forceinline__ void prefetch_tensormap(const CUtensorMap *map) {
  asm volatile("prefetch.tensormap [%0];" :: "l"(reinterpret_cast<uint64_t>(map)) : "memory");
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
__device__ __forceinline__ uint64_t policy_evict_normal() {
  uint64_t p;
  asm volatile("createpolicy.fractional.L2::evict_normal.b64 %0, 1.0;" : "=l"(p));
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

// MXFP4 x MXFP4: UE8M0 scales, two per row per MMA (K = 64 in 32-element blocks),
// read from bytes 0 and 1 of the row's tensor-memory word (scale id 0).
__device__ __forceinline__ void tc_mma_mx(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                          uint32_t sfa_tmem, uint32_t sfb_tmem, uint32_t accumulate) {
  asm volatile(
      "{\n.reg .pred p;\nsetp.ne.b32 p, %4, 0;\n"
      "tcgen05.mma.cta_group::1.kind::mxf4.block_scale.scale_vec::2X [%0], %1, %2, %3, [%5], [%6], p;\n}"
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
// UE4M3 scales, M = m (128, or 256 for a CTA pair), N = n (multiple of 16).
__device__ __forceinline__ uint32_t idesc_mxf4nvf4(uint32_t m, uint32_t n) {
  return (1u << 7) | (1u << 10) | ((n >> 3) << 17) | ((m >> 4) << 24);
}

// Same fields with the scale type set to UE8M0 (bit 23), for kind::mxf4.
__device__ __forceinline__ uint32_t idesc_mxf4_ue8m0(uint32_t m, uint32_t n) {
  return idesc_mxf4nvf4(m, n) | (1u << 23);
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

// 3-D tiled TMA load (no swizzle): the token scales of two 128-row blocks in
// one copy.
__device__ __forceinline__ void tma_load_3d(uint32_t dst, const CUtensorMap *map, int32_t x, int32_t y, int32_t z,
                                            uint32_t bar, uint64_t policy) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes.L2::cache_hint"
      " [%0], [%1, {%2, %3, %4}], [%5], %6;"
      :: "r"(dst), "l"(map), "r"(x), "r"(y), "r"(z), "r"(bar), "l"(policy) : "memory");
}

// ------------------------------------------------------------------ CTA pair (cta_group::2)
__device__ __forceinline__ uint32_t cluster_ctarank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}
__device__ __forceinline__ uint32_t cluster_id_x() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%clusterid.x;" : "=r"(r));
  return r;
}
__device__ __forceinline__ uint32_t nclusters_x() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%nclusterid.x;" : "=r"(r));
  return r;
}

// Shared address of the same variable in CTA `rank` of the cluster.
__device__ __forceinline__ uint32_t mapa_shared(uint32_t addr, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(addr), "r"(rank));
  return r;
}

// Arrive on an mbarrier of another CTA of the cluster (release at cluster scope).
__device__ __forceinline__ void mbar_arrive_remote(uint32_t cluster_addr) {
  asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" :: "r"(cluster_addr) : "memory");
}

// Whole-cluster barrier (every thread of both CTAs).
__device__ __forceinline__ void cluster_sync_all() {
  asm volatile("barrier.cluster.arrive.release.aligned;\nbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}

// Tile load whose completion is counted on the mbarrier of the pair's leader
// CTA (`bar` is a cluster address); the data lands in this CTA's shared memory.
__device__ __forceinline__ void tma_load_2d_pair(uint32_t dst, const CUtensorMap *map, int32_t x, int32_t y,
                                                 uint32_t bar, uint64_t policy) {
  asm volatile(
      "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.tile.mbarrier::complete_tx::bytes.L2::cache_hint"
      " [%0], [%1, {%2, %3}], [%4], %5;"
      :: "r"(dst), "l"(map), "r"(x), "r"(y), "r"(bar), "l"(policy) : "memory");
}

// 3-D tiled TMA load counted on the pair leader's mbarrier (cluster address).
__device__ __forceinline__ void tma_load_3d_pair(uint32_t dst, const CUtensorMap *map, int32_t x, int32_t y, int32_t z,
                                                 uint32_t bar, uint64_t policy) {
  asm volatile(
      "cp.async.bulk.tensor.3d.cta_group::2.shared::cluster.global.tile.mbarrier::complete_tx::bytes.L2::cache_hint"
      " [%0], [%1, {%2, %3, %4}], [%5], %6;"
      :: "r"(dst), "l"(map), "r"(x), "r"(y), "r"(z), "r"(bar), "l"(policy) : "memory");
}

// Shared-memory descriptor of one 512-byte scale atom for tcgen05.cp: 32 rows
// x 16 bytes, no swizzle, 8-row core matrices 128 bytes apart.
__device__ __forceinline__ uint64_t desc_sf_atom(uint32_t addr) {
  return (uint64_t)((addr & 0x3FFFFu) >> 4) | ((uint64_t)(128 >> 4) << 32) | ((uint64_t)1 << 46);
}

// Scale atom -> tensor memory of both CTAs of the pair (each from its own
// shared memory), replicated to the four lane quadrants (32x128b.warpx4).
__device__ __forceinline__ void tc_cp_sf_pair(uint32_t taddr, uint64_t desc) {
  asm volatile("tcgen05.cp.cta_group::2.32x128b.warpx4 [%0], %1;" :: "r"(taddr), "l"(desc) : "memory");
}

// One MMA over the pair: M = 256 (128 weight rows from each CTA's shared
// memory and tensor memory), N tokens split N/2 + N/2 across the two CTAs.
__device__ __forceinline__ void tc_mma_pair(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                            uint32_t sfa_tmem, uint32_t sfb_tmem, uint32_t accumulate) {
  asm volatile(
      "{\n.reg .pred p;\nsetp.ne.b32 p, %4, 0;\n"
      "tcgen05.mma.cta_group::2.kind::mxf4nvf4.block_scale.scale_vec::4X [%0], %1, %2, %3, [%5], [%6], p;\n}"
      :: "r"(d_tmem), "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate), "r"(sfa_tmem), "r"(sfb_tmem)
      : "memory");
}

// Commit of the pair's MMAs to the mbarrier at `bar` in both CTAs (mask 0b11).
__device__ __forceinline__ void tc_commit_pair_both(uint32_t bar) {
  asm volatile(
      "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64 [%0], %1;"
      :: "r"(bar), "h"((uint16_t)3) : "memory");
}

// Commit of the pair's MMAs to one local mbarrier.
__device__ __forceinline__ void tc_commit_pair(uint32_t bar) {
  asm volatile("tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.b64 [%0];"
               :: "r"(bar) : "memory");
}

// ------------------------------------------------------------------ tile map
// Tiles are (expert, weight block, token chunk), weight-block-major inside an
// expert so that the chunks of one weight block run at the same time.  An
// expert with m tokens is cut into ceil(m/192) chunks of equal size rounded up
// to 64, so every chunk starts on a 64-row boundary of the expert's 128-aligned
// slot: its scale atoms start at row (start & ~127) and the MMA reads them
// from tensor-memory column offset (start & 127)/32 (0 or 2).
struct Tile {
  int e;          // expert
  int w_row0;     // first weight row of this CTA (over E*N rows)
  int n_col0;     // first output column of this CTA
  int x_row0;     // first activation row of the tile (slot space)
  int y_row0;     // first output row
  int n_valid;    // tokens in this tile (1..192)
};

// kCap: the most tokens one tile takes (192, or 64 for the deep-ring kernel
// of decode-sized groups); chunks start on 64-row boundaries either way.
template <int kCap = BN>
__device__ __forceinline__ int chunks_of(int m) { return (m + kCap - 1) / kCap; }

// Tile t of a grid whose weight blocks are `wrows` rows (128 for one CTA, 256
// for a pair); `sub` is the CTA's 128-row half of the block.  With the SwiGLU
// epilogue the fused gate_up weight is stored in 32-row groups (16 gate rows,
// then the 16 matching up rows), so 128 weight rows give 64 h columns.
template <bool kSwiglu, int kCap = BN>
__device__ __forceinline__ Tile decode_tile(int t, const int32_t *s_off, const int32_t *s_slot,
                                            const int32_t *s_tile, int E, int N, int wrows, int sub) {
  static_assert(kCap % 64 == 0 && kCap <= BN, "tiles start on 64-row boundaries and fit the accumulator");
  Tile T;
  const int e = upper_group(s_tile, E, t);
  const int m_e = s_off[e + 1] - s_off[e];
  const int nch = chunks_of<kCap>(m_e);
  const int csz = ((m_e + nch - 1) / nch + 63) & ~63;
  const int local = t - s_tile[e];
  const int mt = local / nch, ch = local - mt * nch;
  const int start = ch * csz;
  const int row_in_e = mt * wrows + sub * BM;
  T.e = e;
  T.n_col0 = kSwiglu ? row_in_e / 2 : row_in_e;
  T.w_row0 = e * N + row_in_e;
  T.x_row0 = s_slot[e] + start;
  T.y_row0 = s_off[e] + start;
  T.n_valid = min(csz, m_e - start);
  return T;
}

// Block-wide: s_off = expert offsets ({0, M_total} without offsets), s_slot =
// 128-aligned slot starts, s_tile = first tile of each expert (n_mtiles weight
// blocks x chunks per expert).  Every thread of the block (kThreadsT threads)
// calls it; s_scratch holds 2 * kThreadsT / 32 ints.
// Every tile's rows, and so every output row the epilogue stores, come from
// the offsets: unless they start at 0, never decrease and end at M_total, the
// call reports NVFP4_ERR_INDEX and leaves s_tile[E] = 0, so the kernel runs no
// tile (no copy, no MMA, no store).
template <int kCap = BN, int kThreadsT = NUM_THREADS>
__device__ inline void build_tile_tables(const int32_t *__restrict__ expert_offsets, int E, int M_total,
                                         int n_mtiles, int32_t *s_off, int32_t *s_slot, int32_t *s_tile,
                                         int32_t *s_scratch, int32_t *dev_status) {
  if (expert_offsets) {
    for (int i = threadIdx.x; i <= E; i += kThreadsT) s_off[i] = expert_offsets[i];
  } else if (threadIdx.x == 0) {
    s_off[0] = 0;
    s_off[1] = M_total;
  }
  __syncthreads();
  bool bad = false;
  for (int i = threadIdx.x; i < E; i += kThreadsT) bad |= s_off[i + 1] < s_off[i];
  if (threadIdx.x == 0) bad |= s_off[0] != 0 || s_off[E] != M_total;
  if (__syncthreads_or(bad)) {
    if (threadIdx.x == 0) {
      s_tile[E] = 0;
      report(dev_status, NVFP4_ERR_INDEX);
    }
    __syncthreads();
    return;
  }
  constexpr int kWarpsT = kThreadsT / 32;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int per = (E + kThreadsT - 1) / kThreadsT;
  const int e0 = min(E, (int)threadIdx.x * per), e1 = min(E, e0 + per);
  int32_t ls = 0, lt = 0;
  for (int e = e0; e < e1; ++e) {
    const int32_t m = s_off[e + 1] - s_off[e];
    ls += (m + kSlotAlign - 1) / kSlotAlign * kSlotAlign;
    lt += n_mtiles * chunks_of<kCap>(m);
  }
  int32_t is = ls, it = lt;
#pragma unroll
  for (int d = 1; d < 32; d <<= 1) {
    const int32_t a = __shfl_up_sync(0xffffffffu, is, d), b = __shfl_up_sync(0xffffffffu, it, d);
    if (lane >= d) { is += a; it += b; }
  }
  if (lane == 31) { s_scratch[warp] = is; s_scratch[kWarpsT + warp] = it; }
  __syncthreads();
  if (threadIdx.x == 0) {
    int32_t as = 0, at = 0;
    for (int w = 0; w < kWarpsT; ++w) {
      const int32_t vs = s_scratch[w], vt = s_scratch[kWarpsT + w];
      s_scratch[w] = as; s_scratch[kWarpsT + w] = at;
      as += vs; at += vt;
    }
  }
  __syncthreads();
  int32_t rs = s_scratch[warp] + is - ls, rt = s_scratch[kWarpsT + warp] + it - lt;
  for (int e = e0; e < e1; ++e) {
    const int32_t m = s_off[e + 1] - s_off[e];
    s_slot[e] = rs;
    s_tile[e] = rt;
    rs += (m + kSlotAlign - 1) / kSlotAlign * kSlotAlign;
    rt += n_mtiles * chunks_of<kCap>(m);
  }
  if (e1 == E && e0 < e1) { s_slot[E] = rs; s_tile[E] = rt; }
  __syncthreads();
}

// One K stage of scale factors into tensor memory, written by one warp for its
// lane quadrant: lane l gets the 16 bytes of atom row l (the scales of rows l,
// l+32, l+64, l+96), i.e. the replicated 32x128b layout the block-scaled MMA
// reads.  Weight scales go to columns 0..15 of the buffer, token scales of one
// or two 128-row blocks to columns 16 + 8*kk + 4*rb.
__device__ __forceinline__ void sf_stage_to_tmem(uint32_t tcol, uint32_t sfw_addr, uint32_t sfx_addr, int nrb) {
#pragma unroll
  for (int kk = 0; kk < 4; ++kk) tc_st_x4(tcol + kk * 4, lds128(sfw_addr + kk * 512));
#pragma unroll
  for (int kk = 0; kk < 4; ++kk) tc_st_x4(tcol + 16 + kk * 8, lds128(sfx_addr + kk * 512));
  if (nrb > 1) {
#pragma unroll
    for (int kk = 0; kk < 4; ++kk) tc_st_x4(tcol + 16 + kk * 8 + 4, lds128(sfx_addr + 2048 + kk * 512));
  }
  tc_wait_st();
}

// MXFP4 form of the same: a 512-byte atom now holds 4 UE8M0 scales per row =
// 128 elements = two MMAs, so one K stage has two atoms per row block.  Each
// MMA gets its own 4 columns (the NVFP4 column map) with its two scales in
// bytes 0 and 1 of the row's word: the low half-word of the atom word for the
// first MMA of the pair, the high half-word for the second.
__device__ __forceinline__ uint4 lo16x4(uint4 v) {
  return make_uint4(v.x & 0xFFFFu, v.y & 0xFFFFu, v.z & 0xFFFFu, v.w & 0xFFFFu);
}
__device__ __forceinline__ uint4 hi16x4(uint4 v) { return make_uint4(v.x >> 16, v.y >> 16, v.z >> 16, v.w >> 16); }

__device__ __forceinline__ void sf_stage_to_tmem_mx(uint32_t tcol, uint32_t sfw_addr, uint32_t sfx_addr, int nrb) {
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
      const uint4 x = lds128(sfx_addr + 2048 + a * 512);
      tc_st_x4(tcol + 16 + (2 * a) * 8 + 4, lo16x4(x));
      tc_st_x4(tcol + 16 + (2 * a + 1) * 8 + 4, hi16x4(x));
    }
  }
  tc_wait_st();
}

// One 16-element block of bf16 values encoded with a given global s_g
// (t_g = 6 s_g): the block amax, S = e4m3(a_b / t_g), e = S * s_g,
// r = 1/e (0 when e is 0), codes = e2m1(x * r), each step one IEEE
// round-to-nearest-even fp32 operation; a NaN product (0 * inf) encodes as +0.
__device__ __forceinline__ uint2 encode16_given(const uint4 &va, const uint4 &vb, float s_g, float t_g, uint32_t &S,
                                                bool &nonfinite) {
  const uint32_t w[8] = {va.x, va.y, va.z, va.w, vb.x, vb.y, vb.z, vb.w};
  uint32_t m2 = 0;
#pragma unroll
  for (int i = 0; i < 8; ++i) m2 = __vmaxu2(m2, w[i] & 0x7FFF7FFFu);
  const uint32_t m = max(m2 & 0xFFFFu, m2 >> 16);
  nonfinite = m >= 0x7F80u;
  S = f32_to_e4m3_satfinite(__fdiv_rn(__uint_as_float(m << 16), t_g));
  const float e = __fmul_rn(e4m3_to_f32(S), s_g);
  const float r = (e == 0.0f) ? 0.0f : __frcp_rn(e);
  uint32_t out[2];
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    float v[8];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const uint32_t x = w[4 * h + i];
      v[2 * i] = __fmul_rn(__uint_as_float(x << 16), r);
      v[2 * i + 1] = __fmul_rn(__uint_as_float(x & 0xFFFF0000u), r);
    }
#pragma unroll
    for (int i = 0; i < 8; ++i) v[i] = isnan(v[i]) ? 0.0f : v[i];
    out[h] = f32x8_to_e2m1x8(v);
  }
  return make_uint2(out[0], out[1]);
}

// NVFP4 output of the SwiGLU epilogue (h quantized with a given global per
// expert): codes [slot rows, I/2] and MMA-tiled scales in the activation slot
// layout of the gate_up input.
struct HQuantOut {
  const float *gs = nullptr;    // [E] given global scale of h
  uint8_t *q = nullptr;
  uint8_t *sf = nullptr;
};

// Epilogue of one tile for the calling warp (lane quadrant `quad`, 32
// accumulator rows = 32 weight rows of this CTA): tcgen05.ld the accumulator
// 64 columns (tokens) at a time, scale by alpha = a_gs[e] * b_gs[e], and store
// Y (fp32 or bf16) or, with the SwiGLU epilogue, h = bf16(silu(g) * u) plus
// the expert's max |h|.  Once the last columns are in registers the
// accumulator is handed back by an arrive on `acc_empty` (in the pair's leader
// CTA when release_remote).
// With kQuantH (SwiGLU only) h is not stored: each 16-column block of a
// token (one warp's 16 columns) is quantized on the spot with the expert's
// given global, exactly as nvfp4_quantize in GIVEN mode would quantize the
// bf16 h, and the codes and the E4M3 scale are written to hq.
template <bool kSwiglu, bool kBf16Out, bool kQuantH = false>
__device__ __forceinline__ void epilogue_tile(const Tile &T, uint32_t tacc, float alpha, uint32_t epi, int quad,
                                              int lane, int N, void *__restrict__ y, float *__restrict__ amax_out,
                                              uint32_t acc_empty, bool release_remote,
                                              const HQuantOut &hq = HQuantOut{}, int32_t *dev_status = nullptr) {
  uint32_t hmax2 = 0;                          // SwiGLU: max |h| bits of this lane, two bf16 lanes
  float q_sg = 1.0f, q_tg = 6.0f;
  bool q_bad = false, q_gs_bad = false;
  if constexpr (kQuantH) {
    q_sg = hq.gs[T.e];
    q_tg = __fmul_rn(6.0f, q_sg);
    if (!(q_sg > 0.0f) || !isfinite(q_sg)) q_gs_bad = true;
  }
  for (int c0 = 0; c0 < T.n_valid; c0 += 64) {
    uint32_t r[64];
    tc_ld32_nowait(tacc + (uint32_t)c0, r);
    if (c0 + 32 < T.n_valid) tc_ld32_nowait(tacc + (uint32_t)c0 + 32, r + 32);
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
    if (c0 + 64 >= T.n_valid) {
      // the whole accumulator has been read: hand it back to the MMA warp
      tc_fence_before();
      if (release_remote) mbar_arrive_remote(acc_empty);
      else mbar_arrive(acc_empty);
    }
    if constexpr (kSwiglu) {
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
#pragma unroll
        for (int j = 0; j < 16; ++j) {
          const uint32_t mine = gate_lane ? r[sub * 32 + 16 + j] : r[sub * 32 + j];
          const uint32_t other = __shfl_xor_sync(0xffffffffu, mine, 16);
          const float gv = __fmul_rn(__uint_as_float(gate_lane ? r[sub * 32 + j] : other), alpha);
          const float uv = __fmul_rn(__uint_as_float(gate_lane ? other : r[sub * 32 + 16 + j]), alpha);
          const float sv = __fdividef(gv, 1.0f + __expf(-gv));
          const __nv_bfloat16 hv = __float2bfloat16_rn(__fmul_rn(sv, uv));
          const uint16_t hb = *reinterpret_cast<const uint16_t *>(&hv);
          asm volatile("st.shared.b16 [%0], %1;" :: "r"(epi + half + j * 32 + (lane & 15) * 2), "h"(hb) : "memory");
        }
        __syncwarp();
        if constexpr (kQuantH) {
          // lane L encodes token row L of this sub: its 16 columns are one block
          if (lane < rows_here) {
            const uint32_t ra = epi + (lane >> 4) * 576 + (lane & 15) * 32;
            const uint4 va = lds128(ra), vb = lds128(ra + 16);
            uint32_t S;
            bool nonfinite;
            const uint2 codes = encode16_given(va, vb, q_sg, q_tg, S, nonfinite);
            q_bad |= nonfinite;
            const int NH = N / 2;
            const int64_t p = (int64_t)T.x_row0 + tok0 + lane;             // slot row of this token
            const int col0 = T.n_col0 + quad * 16;
            *reinterpret_cast<uint2 *>(hq.q + p * (NH / 2) + col0 / 2) = codes;
            hq.sf[sf_tiled_offset(p, col0 / 16, NH / 16)] = (uint8_t)S;
          }
          __syncwarp();
          continue;
        }
        const int NH = N / 2;
        __nv_bfloat16 *hbase = reinterpret_cast<__nv_bfloat16 *>(y) + (int64_t)(T.y_row0 + tok0) * NH +
                               T.n_col0 + quad * 16;
#pragma unroll
        for (int it = 0; it < 2; ++it) {
          const int row = it * 16 + (lane >> 1), chunk = lane & 1;
          if (row < rows_here) {
            const uint4 v = lds128(epi + (row >> 4) * 576 + (row & 15) * 32 + chunk * 16);
            *reinterpret_cast<uint4 *>(hbase + (int64_t)row * NH + chunk * 8) = v;
            // the expert's max |h|, over the real rows only, from the bf16 bits stored
            hmax2 = __vmaxu2(__vmaxu2(hmax2, v.x & 0x7FFF7FFFu), __vmaxu2(v.y & 0x7FFF7FFFu, v.z & 0x7FFF7FFFu));
            hmax2 = __vmaxu2(hmax2, v.w & 0x7FFF7FFFu);
          }
        }
        __syncwarp();
      }
    } else {
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
  }
  if constexpr (kQuantH) {
    if (q_gs_bad) report(dev_status, NVFP4_ERR_INVALID_ARG);
    if (q_bad) report(dev_status, NVFP4_ERR_NONFINITE);
  } else if (kSwiglu) {
    uint32_t hmax = max(hmax2 & 0xFFFFu, hmax2 >> 16);
#pragma unroll
    for (int d = 16; d > 0; d >>= 1) hmax = max(hmax, __shfl_xor_sync(0xffffffffu, hmax, d));
    if (lane == 0 && hmax) atomicMax(reinterpret_cast<uint32_t *>(amax_out) + T.e, hmax << 16);
  }
}

}  // namespace gemm
}  // namespace nvfp4

// ====================================================================== host helpers
namespace nvfp4 {
namespace gemm {

inline PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  if (!fn) {
    void *p = nullptr;
    cudaDriverEntryPointQueryResult qres;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &qres) == cudaSuccess &&
        qres == cudaDriverEntryPointSuccess && p)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  }
  return fn;
}

// A uint8 tensor map of rank 2 or 3, from a process-wide cache keyed by its
// arguments.  Encoding is several microseconds of host work per map, which
// would otherwise dominate the call of a small GEMM.  A map holds only an
// address and a shape, never ownership, so an entry stays valid for whatever
// buffer later sits at the same address.
inline bool encode_u8_map(CUtensorMap *map, int rank, const void *base, const cuuint64_t *dims,
                          const cuuint64_t *strides, const cuuint32_t *box, CUtensorMapSwizzle swizzle) {
  struct Entry {
    bool used;
    int rank, swizzle;
    const void *base;
    cuuint64_t dims[3], strides[2];
    cuuint32_t box[3];
    CUtensorMap map;
  };
  static std::mutex mu;
  static Entry cache[64];
  static int next = 0;
  auto same = [&](const Entry &e) {
    if (!e.used || e.rank != rank || e.swizzle != (int)swizzle || e.base != base) return false;
    for (int i = 0; i < rank; ++i)
      if (e.dims[i] != dims[i] || e.box[i] != box[i] || (i < rank - 1 && e.strides[i] != strides[i])) return false;
    return true;
  };
  {
    std::lock_guard<std::mutex> lock(mu);
    for (const Entry &e : cache)
      if (same(e)) { *map = e.map; return true; }
  }
  auto enc = tensor_map_encoder();
  if (!enc) return false;
  cuuint32_t estr[3] = {1, 1, 1};
  if (enc(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, (cuuint32_t)rank, const_cast<void *>(base), dims, strides, box, estr,
          CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
          CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
    return false;
  std::lock_guard<std::mutex> lock(mu);
  Entry &e = cache[next];
  next = (next + 1) % 64;
  e.used = true;
  e.rank = rank;
  e.swizzle = (int)swizzle;
  e.base = base;
  for (int i = 0; i < rank; ++i) {
    e.dims[i] = dims[i];
    e.box[i] = box[i];
    if (i < rank - 1) e.strides[i] = strides[i];
  }
  e.map = *map;
  return true;
}

// 2-D uint8 view [rows, row_bytes] with a {128 bytes, box_rows} box, 128-byte swizzle.
inline bool make_map(CUtensorMap *map, const void *base, uint64_t rows, uint64_t row_bytes, uint32_t box_rows) {
  cuuint64_t dims[2] = {row_bytes, rows};
  cuuint64_t strides[1] = {row_bytes};
  cuuint32_t box[2] = {128, box_rows};
  return encode_u8_map(map, 2, base, dims, strides, box, CU_TENSOR_MAP_SWIZZLE_128B);
}

// Token scales in the MMA-tiled layout viewed as [row block][K/32][256 bytes]:
// one {256, 8, 2} box is the 2 KB of one K stage for two consecutive 128-row
// blocks (a block past the end reads as zeros).
inline bool make_map_sfx(CUtensorMap *map, const void *base, uint64_t row_blocks, uint64_t K) {
  cuuint64_t dims[3] = {256, K / 32, row_blocks};
  cuuint64_t strides[2] = {256, K * 8};
  cuuint32_t box[3] = {256, 8, 2};
  return encode_u8_map(map, 3, base, dims, strides, box, CU_TENSOR_MAP_SWIZZLE_NONE);
}

// Weight scales in the MMA-tiled layout viewed as [row block][K/32][256 bytes]:
// one {256, 8, 1} box is the 2 KB of one K stage of one 128-row block.
inline bool make_map_sfw(CUtensorMap *map, const void *base, uint64_t row_blocks, uint64_t K) {
  cuuint64_t dims[3] = {256, K / 32, row_blocks};
  cuuint64_t strides[2] = {256, K * 8};
  cuuint32_t box[3] = {256, 8, 1};
  return encode_u8_map(map, 3, base, dims, strides, box, CU_TENSOR_MAP_SWIZZLE_NONE);
}

// The 512-element-stage kernel's launch (gemm_k512.cu), K % 512 == 0;
// hq != nullptr selects the SwiGLU epilogue that writes NVFP4 h; mx selects
// MXFP4 operands (no global scales: a_gs and b_gs are not read); deep selects
// the ring of three slots for tiles of at most 64 tokens (few tokens per
// expert) instead of two slots for up to 192.
nvfp4_status launch_grouped_gemm_k512(const uint8_t *a_q, const uint8_t *a_sf, const float *a_gs,
                                      const uint8_t *b_q, const uint8_t *b_sf, const float *b_gs,
                                      const int32_t *expert_offsets, int E, int64_t M_total, int64_t N, int64_t K,
                                      void *y, nvfp4_out_dtype out_dtype, bool swiglu, float *amax_out,
                                      const HQuantOut *hq, bool mx, bool deep, int32_t *dev_status,
                                      cudaStream_t stream);
// Rows per expert on average at or below which the automatic choice takes the
// deep ring (the decode regime: 640 routed rows over 384 experts).
constexpr int64_t kDeepRingMaxRowsPerExpert = 16;
// Its copy of the main-loop wait budget (see c_wait_budget).
nvfp4_status set_wait_budget_k512(long long cycles);

// The two-weight-block kernel's launch (gemm_w2.cu): N % 256 == 0, bf16
// output (SwiGLU h when swiglu, NVFP4 h when hq != nullptr), NVFP4 operands;
// mx selects MXFP4 operands (plain output, a_gs and b_gs not read); deep
// selects tiles of at most 64 tokens in four slots with double-buffered
// accumulators (decode-sized groups) instead of 192 tokens in three slots.
nvfp4_status launch_grouped_gemm_w2(const uint8_t *a_q, const uint8_t *a_sf, const float *a_gs, const uint8_t *b_q,
                                    const uint8_t *b_sf, const float *b_gs, const int32_t *expert_offsets, int E,
                                    int64_t M_total, int64_t N, int64_t K, void *y, bool swiglu, float *amax_out,
                                    const HQuantOut *hq, bool mx, bool deep, int32_t *dev_status,
                                    cudaStream_t stream);
nvfp4_status set_wait_budget_w2(long long cycles);

// The pair kernel's launch (gemm_pair.cu).  Requires N % 256 == 0.
nvfp4_status launch_grouped_gemm_pair(const uint8_t *a_q, const uint8_t *a_sf, const float *a_gs,
                                      const uint8_t *b_q, const uint8_t *b_sf, const float *b_gs,
                                      const int32_t *expert_offsets, int E, int64_t M_total, int64_t N, int64_t K,
                                      void *y, nvfp4_out_dtype out_dtype, bool swiglu, float *amax_out,
                                      int32_t *dev_status, cudaStream_t stream);

}  // namespace gemm
}  // namespace nvfp4
