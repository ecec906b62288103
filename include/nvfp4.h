/*
 * nvfp4.h -- C ABI of the NVFP4 W4A4 routed-expert hot path for B200 (sm_100a).
 *
 * What the operations compute comes from these pages (cited by title and
 * section):
 *  [P1] "Qwen3.8-Flash-Next-NVFP4 ..." (lpnh.cn/news/2736522), section on the
 *       W4A4 two-level scaling: every 16 elements along the last dimension
 *       share one FP8 E4M3 block scale, each tensor has one FP32 global
 *       scale, 4.5 effective bits; weights are quantized statically,
 *       activations dynamically with the same per-16 rule; only the routed
 *       experts' gate_up_proj / down_proj are quantized.
 *  [P2] "DeepSeek-V4.1-Flash-NVFP4 ..." (kwkr.cn/news/613851), sections on the
 *       format (E2M1 values {0,0.5,1,1.5,2,3,4,6}, two per byte, group 16;
 *       MXFP4 32-element UE8M0 blocks remapped losslessly block by block) and
 *       on why NVFP4 (Blackwell tensor cores take 4-bit operands natively).
 *  [P3] "Qwen3.8-2.4T-A95B-NVFP4 ..." (hnwysp.cn/news/107543): NVFP4 KV cache.
 *
 * Conventions shared by every entry point
 *  - All tensor pointers are DEVICE pointers owned by the caller.  The
 *    library allocates nothing; scratch space is a caller-supplied
 *    `workspace` of at least nvfp4_workspace_size() bytes (device memory).
 *  - Every call is asynchronous on `stream` and never synchronises the host
 *    or copies device data to the host.
 *  - Return value: argument/shape/launch errors found on the host.
 *    Data-dependent errors are written by the kernels to the optional device
 *    word `dev_status` (int32): the first error wins (compare-and-swap from
 *    NVFP4_OK), and nothing traps.  The caller zeroes it before use.
 *  - Pointers to packed tensors must be 16-byte aligned.
 *  - Number formats: E2M1 codes packed two per byte, element 2j in bits
 *    [3:0] and element 2j+1 in bits [7:4]; block scales are E4M3 bytes; the
 *    global scale s_g is the fp32 dequantisation multiplier, so an element
 *    decodes to (e2m1(code) * e4m3(S)) * s_g.
 *  - Scale-factor layouts (nvfp4_sf_layout):
 *      ROWMAJOR:  sf[r * (K/16) + j] for row r, block j.
 *      MMA_TILED: the tensor-core operand layout.  Rows are grouped in
 *        128-row blocks and scales in groups of 4 (64 elements); each
 *        (row-block, 4-group) pair is a 512-byte atom, atoms ordered
 *        row-block-major, and inside an atom the scale of row r, block j is
 *        at (r%32)*16 + ((r%128)/32)*4 + (j%4).  Requires K % 64 == 0; the
 *        tensor holds roundup(rows,128) rows.
 *  - Grouped (MoE) row placement: with `group_offsets` (int32 [G+1], raw
 *    prefix sums of the rows of each expert group, on the device), packed
 *    rows of group g start at the 128-aligned slot
 *    slot[g] = sum_{h<g} roundup(rows_h, 128); rows of a slot past the
 *    group's rows are left unwritten (the grouped GEMM reads them as padding
 *    MMA rows whose outputs it never stores).  Size packed buffers with
 *    nvfp4_padded_rows_bound().
 */
#ifndef NVFP4_H_
#define NVFP4_H_

#include <stddef.h>
#include <stdint.h>
#include <cuda_runtime.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    NVFP4_OK = 0,
    NVFP4_ERR_INVALID_ARG = 1,       /* null / misaligned pointer, bad enum */
    NVFP4_ERR_UNSUPPORTED_SHAPE = 2, /* shape outside the documented limits */
    NVFP4_ERR_CUDA = 3,              /* a launch or runtime call failed */
    /* data-dependent errors, written to *dev_status by the kernels */
    NVFP4_ERR_NONFINITE = 16,        /* an input element (or amax) is NaN or inf */
    NVFP4_ERR_NOT_REPRESENTABLE = 17,/* MXFP4 exponent byte 0xFF or spread > 17 */
    NVFP4_ERR_TIMEOUT = 18,          /* a bounded wait inside a kernel gave up */
    NVFP4_ERR_INDEX = 19             /* an index input (expert id) is out of range */
} nvfp4_status;

typedef enum { NVFP4_SF_ROWMAJOR = 0, NVFP4_SF_MMA_TILED = 1 } nvfp4_sf_layout;
/* FROM_AMAX: s_g from the amax of the input (an extra read pass).
 * GIVEN: s_g supplied (calibrated input scale, static KV scale).
 * AMAX_GIVEN: global_scale holds the group amax on entry (e.g. produced by
 *   the SwiGLU GEMM epilogue); it is replaced by s_g = amax/2688 (1 if 0). */
typedef enum { NVFP4_GS_FROM_AMAX = 0, NVFP4_GS_GIVEN = 1, NVFP4_GS_AMAX_GIVEN = 2 } nvfp4_gs_mode;
typedef enum { NVFP4_OUT_F32 = 0, NVFP4_OUT_BF16 = 1 } nvfp4_out_dtype;
/* NONE: y = alpha * A B^T.  SWIGLU: the weight is a fused gate_up [2I, K]
 * per expert stored gate/up interleaved in 32-row groups: packed rows
 * 32j..32j+15 are gate rows 16j..16j+15 and packed rows 32j+16..32j+31 the
 * up rows 16j..16j+15 (quantize the rows in that order, e.g. through the
 * row_index of nvfp4_quantize: a row permutation commutes with NVFP4
 * quantization, whose block scales are row-local and whose global scale is
 * per expert).  The epilogue writes h = bf16(silu(g) * u) with
 * g = alpha*acc_gate, u = alpha*acc_up kept in fp32 (no bf16 rounding of the
 * gate_up output in between; silu through the fast exp/divide intrinsics),
 * y is bf16 [M_total, N/2], and amax_out[e]
 * receives max |h| of expert e (fp32 bit pattern via integer max; the call
 * clears amax_out first). */
typedef enum { NVFP4_EPI_NONE = 0, NVFP4_EPI_SWIGLU = 1 } nvfp4_epilogue;

/* Human-readable name of a status code (static string). */
const char *nvfp4_status_string(int status);

/* Bytes of device workspace needed by any call below for up to `num_groups`
 * groups / experts / tensors (num_groups >= 1). */
size_t nvfp4_workspace_size(int num_groups);

/* Upper bound on packed rows when `rows` gathered rows are split into
 * `num_groups` 128-aligned slots (= rows + 127*num_groups, rounded to 128). */
int64_t nvfp4_padded_rows_bound(int64_t rows, int num_groups);

/*
 * nvfp4_quantize -- dynamic (or static) NVFP4 quantisation of bf16 rows.
 * [P1 two-level scaling: per-16 E4M3 block scale + FP32 global; activations
 *  quantized on the fly; P2 format: E2M1 codes packed two per byte.]
 *
 *   x           bf16 [*, ld_x]; ld_x >= K, in elements, ld_x % 8 == 0.
 *   rows, K     rows of the (gathered) result and row length; K % 16 == 0,
 *               K % 64 == 0 for MMA_TILED; rows >= 0 (0 is a no-op).
 *   row_index   nullable int32 [rows]: result row r is x[row_index[r]].
 *   group_offsets, num_groups
 *               nullable int32 [num_groups+1] device prefix sums over result
 *               rows (offsets[0] == 0, offsets[G] == rows).  Each group has
 *               its own global scale and its own 128-aligned slot in q/sf.
 *               NULL: one group, rows written contiguously (padded to 128 rows
 *               only for MMA_TILED).  Padding rows (a slot's rows past its
 *               group, a tile's rows past `rows`) are not written: the
 *               grouped GEMM never stores the columns they feed.
 *   gs_mode, global_scale
 *               fp32 [max(1,num_groups)] device.  FROM_AMAX: written with
 *               s_g = amax/2688 (2688 = 6*448: the block holding the amax gets
 *               scale 448), or 1 for an all-zero group.  GIVEN: read (a
 *               calibrated input scale or a static KV scale), must be > 0.
 *               AMAX_GIVEN: holds the group amax on entry, replaced by s_g as
 *               in FROM_AMAX (no amax pass over x).
 *   q           uint8 [packed rows, K/2]; sf uint8 scales in `sf_layout`.
 *   workspace   >= nvfp4_workspace_size(num_groups) bytes.
 *   dev_status  nullable int32: NVFP4_ERR_NONFINITE when an input element of a
 *               group is NaN/inf (that group's outputs are unspecified).
 * Launches: FROM_AMAX without row_index and group_offsets runs as one
 * cooperative launch (amax, global scale, encode; its CTAs wait for each other
 * with a bounded wait, NVFP4_ERR_TIMEOUT if it ever ran out), after clearing
 * two words of the workspace; if the runtime refuses a cooperative launch, or
 * rows * K/16 >= 2^32 - 64, the separate passes run instead.  Other calls run
 * an amax pass (FROM_AMAX), a scale finalisation and the encode.
 * Arithmetic (each step one IEEE fp32 round-to-nearest-even operation):
 *   block amax a_b; S = e4m3_rne_satfinite(a_b / (6*s_g));
 *   r = 1/(S*s_g) (0 when S*s_g == 0); code_i = e2m1_rne_satfinite(x_i * r).
 */
nvfp4_status nvfp4_quantize(const void *x, int64_t rows, int64_t K, int64_t ld_x,
                            const int32_t *row_index, const int32_t *group_offsets,
                            int num_groups, nvfp4_gs_mode gs_mode, float *global_scale,
                            uint8_t *q, uint8_t *sf, nvfp4_sf_layout sf_layout,
                            void *workspace, int32_t *dev_status, cudaStream_t stream);

/*
 * nvfp4_moe_quantize -- the routed-expert activation quantize in token order.
 * [P1: routed experts' inputs are quantized to NVFP4 on the fly, one global
 *  scale per expert group as in nvfp4_quantize.]
 * Same result, byte for byte in every routed row, as nvfp4_quantize with
 * rows = group_offsets[num_groups] and row_index[slot[t*topk + c]] = t, but
 * each token row of x is read once: its 16-element block amaxes are formed
 * once and its topk copies are encoded with their experts' global scales.
 *   x           bf16 [tokens, ld_x], ld_x >= K, ld_x % 8 == 0.
 *   slot        int32 [tokens, topk] device: routed row of each (token,
 *               choice), as nvfp4_moe_route writes it; -1 = not routed.  The
 *               non-negative entries must be distinct and cover
 *               [0, group_offsets[num_groups]); an entry beyond that range is
 *               skipped and reported as NVFP4_ERR_INDEX.  1 <= topk <= 32.
 *   group_offsets, num_groups   int32 [num_groups+1] prefix sums over routed
 *               rows (required); each group has its own 128-aligned slot in
 *               q/sf as in nvfp4_quantize.  Padding rows of a slot are left
 *               unwritten (the grouped GEMM never stores their columns).
 *   gs_mode, global_scale, q, sf, sf_layout, workspace, dev_status
 *               as in nvfp4_quantize (FROM_AMAX takes the amax per expert over
 *               the tokens routed to it).
 */
nvfp4_status nvfp4_moe_quantize(const void *x, int64_t tokens, int64_t K, int64_t ld_x, const int32_t *slot,
                                int topk, const int32_t *group_offsets, int num_groups, nvfp4_gs_mode gs_mode,
                                float *global_scale, uint8_t *q, uint8_t *sf, nvfp4_sf_layout sf_layout,
                                void *workspace, int32_t *dev_status, cudaStream_t stream);

/*
 * nvfp4_dequantize -- y = (e2m1(code) * e4m3(S)) * s_g, rounded once to the
 * output type.  [P1: quantized tensors are dequantized with their scales.]
 *   q, sf, sf_layout  packed input (grouped slots when group_offsets != NULL).
 *   global_scale      fp32 [max(1,num_groups)].
 *   y                 [rows, K] fp32 or bf16, rows in unpadded order.
 */
nvfp4_status nvfp4_dequantize(const uint8_t *q, const uint8_t *sf, nvfp4_sf_layout sf_layout,
                              const float *global_scale, const int32_t *group_offsets,
                              int num_groups, int64_t rows, int64_t K, void *y,
                              nvfp4_out_dtype out_dtype, cudaStream_t stream);

/*
 * nvfp4_global_scale_from_amax -- the global-scale rule on its own, for a
 * calibration pass that fixes a static scale (the checkpoints' input_scale)
 * from observed amaxes.  [P1 two-level scaling: one FP32 global scale per
 * tensor; calibrated activation scales.]
 *   global_scale[i] = a_i / 2688 (1 when a_i == 0), a_i = |amax[i]| * margin:
 *   the multiply is one IEEE fp32 round-to-nearest-even operation and is
 *   skipped when margin == 1, the division is one IEEE operation -- with
 *   margin 1 exactly the s_g that FROM_AMAX mode derives from that amax.
 *   amax          fp32 [n] device (max |x| per tensor or group); may alias
 *                 global_scale.
 *   n             >= 0 (0 is a no-op), at most 2^30.
 *   margin        finite and > 0, else NVFP4_ERR_INVALID_ARG (> 1 leaves
 *                 headroom for activations larger than the calibration saw).
 *   global_scale  fp32 [n] device, written.
 *   dev_status    nullable: NVFP4_ERR_NONFINITE when some a_i is NaN or inf
 *                 (that entry is written as NaN).
 */
nvfp4_status nvfp4_global_scale_from_amax(const float *amax, int64_t n, float margin, float *global_scale,
                                          int32_t *dev_status, cudaStream_t stream);

/*
 * nvfp4_e2m1_encode -- the element-wise FP32 -> E2M1 step of every quantize
 * call on its own.  [P2: the E2M1 value set {0, 0.5, 1, 1.5, 2, 3, 4, 6} with
 *  a sign bit, two codes per byte.]  Round to nearest, ties to the even
 * mantissa bit; magnitudes above 6 (and +-inf) saturate to 6; the sign is
 * kept, so -0 and small negatives give 0x8; NaN gives +0 (the quantize
 * kernels' rule for the product 0 * inf).
 *   x   fp32 [n] device, 16-byte aligned; n % 8 == 0 (else UNSUPPORTED_SHAPE).
 *   q   uint8 [n/2] device, 16-byte aligned: element 2i in bits [3:0] of byte
 *       i, element 2i+1 in bits [7:4].
 */
nvfp4_status nvfp4_e2m1_encode(const float *x, int64_t n, uint8_t *q, cudaStream_t stream);

/*
 * nvfp4_e4m3_encode -- the element-wise FP32 -> E4M3 step of the block
 * scales on its own.  [P1: the per-16 block scale is an FP8 E4M3 value, at
 *  most 448.]  Round to nearest even, subnormals kept (2^-9 is the smallest),
 * magnitudes from 464 up (and +-inf) saturate to +-448 (0x7E / 0xFE); NaN
 * gives 0x7F.
 *   x    fp32 [n] device, 16-byte aligned; n % 4 == 0 (else UNSUPPORTED_SHAPE).
 *   out  uint8 [n] device, 16-byte aligned.
 */
nvfp4_status nvfp4_e4m3_encode(const float *x, int64_t n, uint8_t *out, cudaStream_t stream);

/*
 * mxfp4_to_nvfp4 -- lossless block-by-block MXFP4 -> NVFP4 weight remap.
 * [P2: MXFP4 uses 32-element blocks with UE8M0 (power-of-two) scales, NVFP4
 *  16-element blocks with a finer scale; because the finer format can express
 *  every MXFP4 block exactly, the page converts the weights one block at a time
 *  with no change to any dequantized value (its conversion script performs an
 *  E2M1->E4M3 scale remap).]
 *   n_tensors tensors of [rows, K] laid back to back (K % 32 == 0).
 *   q_mx uint8 [n*rows, K/2]; ue8m0 uint8 [n*rows, K/32].
 *   q_nv uint8 [n*rows, K/2] (codes copied unchanged; may equal q_mx);
 *   sf_nv scales in sf_layout (MMA_TILED needs rows % 128 == 0, K % 64 == 0);
 *   global_scale fp32 [n]: s_g = 2^g with g = e_max - 8 over the blocks that
 *   are not all +-0 (g = 0 if none); every 32-block of exponent e gets the
 *   E4M3 scale 2^clamp(e-g, -9, 8) on both halves.
 *   workspace >= nvfp4_workspace_size(n_tensors).
 *   dev_status: NVFP4_ERR_NOT_REPRESENTABLE when a byte is 0xFF or a tensor's
 *   exponent spread exceeds 17 (E4M3 holds exactly 2^-9 .. 2^8).
 */
nvfp4_status mxfp4_to_nvfp4(const uint8_t *q_mx, const uint8_t *ue8m0, int64_t n_tensors,
                            int64_t rows, int64_t K, uint8_t *q_nv, uint8_t *sf_nv,
                            nvfp4_sf_layout sf_layout, float *global_scale, void *workspace,
                            int32_t *dev_status, cudaStream_t stream);

/*
 * mxfp4_quantize -- MXFP4 encode: E2M1 codes with one UE8M0 (power-of-two)
 * scale per 32 elements.
 * [P2, format table: MXFP4 = 32-element blocks with UE8M0 scales; P2,
 *  which-layers section: an FP8 table is converted to MXFP4, a lossy step.
 *  The page gives no exponent rule; this follows the OCP Microscaling v1.0
 *  conversion.]
 *   x        bf16 [rows, ld_x], ld_x >= K, ld_x % 8 == 0, 16-byte aligned.
 *            (bf16 holds every FP8 E4M3 value exactly, so an FP8 source is
 *            encoded by passing its values widened to bf16.)
 *   rows, K  K % 32 == 0 (K % 128 == 0 for MMA_TILED); rows * K/32 < 2^31;
 *            rows == 0 is a no-op.
 *   q        uint8 [rows, K/2], 16-byte aligned, same nibble order as NVFP4.
 *   ue8m0    uint8 scales, ROWMAJOR [rows, K/32] or MMA_TILED (the NVFP4 atom
 *            layout with one scale per 32 elements: 128-row blocks, 4 scales =
 *            128 elements per 512-byte atom; the tensor holds roundup(rows,128)
 *            rows, padding rows not written).
 *   dev_status  NVFP4_ERR_NONFINITE when a block holds a NaN or inf (that
 *            block gets byte 0xFF and zero codes).
 * Per 32-block with amax a: E = floor(log2 a) - 2 clamped to [-127, 127]
 * (byte E + 127; an all-zero block gets 0), codes = e2m1_rne_satfinite(x * 2^-E).
 */
nvfp4_status mxfp4_quantize(const void *x, int64_t rows, int64_t K, int64_t ld_x, uint8_t *q,
                            uint8_t *ue8m0, nvfp4_sf_layout sf_layout, int32_t *dev_status,
                            cudaStream_t stream);

/*
 * nvfp4_grouped_gemm -- Y_e = (a_gs[e] * b_gs[e]) * A_e B_e^T for every expert e,
 * block-scaled FP4 x FP4 on the tcgen05 tensor cores, fp32 accumulation.
 * [P2 "why NVFP4": Blackwell tensor cores multiply 4-bit operands natively;
 *  P1: routed experts' gate_up_proj / down_proj in W4A4.]
 *   a_q, a_sf   packed activations in 128-aligned expert slots (the output of
 *               nvfp4_quantize with group_offsets), MMA_TILED scales.
 *   a_gs        fp32 [E] activation global scales.
 *   b_q, b_sf   packed weights [E, N, K/2], MMA_TILED scales over E*N rows.
 *   b_gs        fp32 [E] weight global scales.
 *   expert_offsets  nullable int32 [E+1] device prefix sums of routed rows
 *               (offsets[E] == M_total).  NULL means one dense GEMM (E = 1).
 *   M_total, N, K   Y is [M_total, N]; N % 128 == 0, K % 256 == 0.
 *   y, out_dtype    fp32 or bf16 [M_total, N], rows in routed (unpadded) order.
 *   epi, amax_out   NVFP4_EPI_NONE (amax_out unused), or NVFP4_EPI_SWIGLU: y is
 *                   bf16 h [M_total, N/2] (out_dtype must be BF16), amax_out
 *                   fp32 [E] (cleared and written by the call), N/2 % 64 == 0.
 *   workspace   >= nvfp4_workspace_size(E); dev_status: NVFP4_ERR_TIMEOUT if a
 *               pipeline wait gave up (the output is then incomplete).
 */
nvfp4_status nvfp4_grouped_gemm(const uint8_t *a_q, const uint8_t *a_sf, const float *a_gs,
                                const uint8_t *b_q, const uint8_t *b_sf, const float *b_gs,
                                const int32_t *expert_offsets, int num_experts,
                                int64_t M_total, int64_t N, int64_t K, void *y,
                                nvfp4_out_dtype out_dtype, nvfp4_epilogue epi, float *amax_out,
                                void *workspace, int32_t *dev_status, cudaStream_t stream);

/*
 * nvfp4_grouped_gemm_swiglu_nvfp4 -- the gate_up grouped GEMM with the SwiGLU
 * epilogue emitting NVFP4 h directly, for a down projection whose input
 * global scale is given (calibrated).
 * [P1: activation scales from calibration, the checkpoints' input_scale;
 *  the same two-level NVFP4 block encoding as nvfp4_quantize.]
 * h = bf16(silu(g) * u) exactly as with NVFP4_EPI_SWIGLU, then every 16
 * columns of a routed row are quantized with the expert's h_gs[e]: the bytes
 * nvfp4_quantize would write for that bf16 h in GIVEN mode, grouped by
 * expert, MMA_TILED.  h itself never reaches memory.
 *   a_*, b_*, expert_offsets, num_experts, M_total, N, K  as nvfp4_grouped_gemm
 *               (b is the gate/up-interleaved fused weight of NVFP4_EPI_SWIGLU).
 *   h_gs        fp32 [E], > 0 and finite (else NVFP4_ERR_INVALID_ARG in dev_status).
 *   h_q, h_sf   uint8 [nvfp4_padded_rows_bound(M_total, E), N/4] codes and their
 *               MMA-tiled scales, in the expert slots of the gate_up input;
 *               padding rows are not written.  16-byte aligned h_q.
 *   dev_status  also NVFP4_ERR_NONFINITE (non-finite h), NVFP4_ERR_TIMEOUT.
 */
nvfp4_status nvfp4_grouped_gemm_swiglu_nvfp4(const uint8_t *a_q, const uint8_t *a_sf, const float *a_gs,
                                             const uint8_t *b_q, const uint8_t *b_sf, const float *b_gs,
                                             const int32_t *expert_offsets, int num_experts, int64_t M_total,
                                             int64_t N, int64_t K, const float *h_gs, uint8_t *h_q, uint8_t *h_sf,
                                             void *workspace, int32_t *dev_status, cudaStream_t stream);

/*
 * mxfp4_grouped_gemm -- Y_e = A_e B_e^T for every expert e with MXFP4 operands
 * (E2M1 codes, one UE8M0 scale per 32 elements, no global scale) on the
 * tcgen05 tensor cores (kind::mxf4, block-scaled), fp32 accumulation.
 * [P2, format table: MXFP4 blocks of 32 with power-of-two scales, the
 *  checkpoint's source format before the NVFP4 remap; this is the direct
 *  MXFP4 GEMM to set against the remap-then-NVFP4 route.]
 *   a_q, a_sf   activations in 128-aligned expert slots (as for
 *               nvfp4_grouped_gemm), scales from mxfp4_quantize in MMA_TILED
 *               layout over nvfp4_padded_rows_bound(M_total, E) rows.
 *   b_q, b_sf   weights [E, N, K/2], MMA_TILED UE8M0 scales over E*N rows.
 *   expert_offsets, num_experts, M_total, N, K, y, out_dtype, workspace,
 *   dev_status  as for nvfp4_grouped_gemm (N % 128 == 0, K % 256 == 0; no
 *               epilogue option).
 */
nvfp4_status mxfp4_grouped_gemm(const uint8_t *a_q, const uint8_t *a_sf, const uint8_t *b_q,
                                const uint8_t *b_sf, const int32_t *expert_offsets, int num_experts,
                                int64_t M_total, int64_t N, int64_t K, void *y,
                                nvfp4_out_dtype out_dtype, void *workspace, int32_t *dev_status,
                                cudaStream_t stream);

/*
 * nvfp4_grouped_gemm_w4a16 -- weight-only NVFP4 grouped GEMM with bf16
 * activations: Y_e = X_e (b_gs[e] * W_e)^T for every expert e, fp32 accumulate.
 * [P5: the MTP layer's experts are W4A16_NVFP4 -- NVFP4 weights, 16-bit
 *  activations; P1/P2: the weight format and its dequantisation.]
 * Two kernels (nvfp4_w4a16_select_kernel): a warp-MMA one for decode-sized
 * groups and a tcgen05 one (dequantized weights as the A operand in tensor
 * memory) for larger groups.  The tensor-core operands are f16: the weights exactly (e2m1 * e4m3 fits f16),
 * the activations after a per-row power-of-two scaling 2^-k that puts the row's
 * max |x| in [2^14, 2^15) -- exact for every element within 2^29 of the row
 * max, smaller ones rounded to f16's subnormal grid (error < 2^-25 * max|x|);
 * the epilogue multiplies by 2^k again.
 *   x, ld_x, x_rows  bf16 [x_rows, ld_x] activations (ld_x >= K, % 8 == 0,
 *               16-byte aligned).
 *   row_index   nullable int32 [M_total]: routed row r reads x[row_index[r]]
 *               (an entry outside [0, x_rows) reads row 0 and reports
 *               NVFP4_ERR_INDEX); NULL: row r reads x[r] (x_rows >= M_total).
 *   b_q, b_sf, b_gs  packed weights [E, N, K/2], ROW-MAJOR E4M3 scales
 *               [E*N, K/16] (16-byte aligned), fp32 global per expert.
 *   expert_offsets, num_experts  int32 [E+1] prefix sums over routed rows
 *               (NULL: one dense GEMM); num_experts <= 1024.
 *   M_total, N, K    K % 256 == 0; N % 128 == 0.
 *   y, out_dtype     fp32 or bf16 [M_total, N] (routed order); with
 *               NVFP4_EPI_SWIGLU the weight is a fused gate_up [2I, K] (gate
 *               rows first) and y is h = silu(g) * u, [M_total, N/2].
 *   workspace   >= nvfp4_w4a16_workspace_size(M_total, num_experts, K) bytes,
 *               16-byte aligned (the scaled f16 activations and their scales).
 *   dev_status  NVFP4_ERR_INDEX, NVFP4_ERR_NONFINITE (a non-finite activation
 *               row), NVFP4_ERR_TIMEOUT.
 */
size_t nvfp4_w4a16_workspace_size(int64_t M_total, int num_experts, int64_t K);
/*
 * nvfp4_w4a16_select_kernel -- which kernel nvfp4_grouped_gemm_w4a16 runs
 * (process-wide; a tuning and testing switch, not part of the pages' method):
 *   0  automatic (default): the warp-MMA kernel (mma.sync, 16 tokens per
 *      weight pass) when the experts average at most 16 routed rows
 *      (M_total <= 16 * num_experts), the tcgen05 kernel otherwise;
 *   1  the warp-MMA kernel;  2  the tcgen05 kernel (dequantized weights as the
 *      MMA's A operand in tensor memory, up to 64 tokens per weight pass).
 * Both compute the same products; sums may differ in rounding order.
 * Returns NVFP4_ERR_INVALID_ARG for another mode.
 */
nvfp4_status nvfp4_w4a16_select_kernel(int mode);
nvfp4_status nvfp4_grouped_gemm_w4a16(const void *x, int64_t ld_x, int64_t x_rows, const int32_t *row_index,
                                      const uint8_t *b_q, const uint8_t *b_sf, const float *b_gs,
                                      const int32_t *expert_offsets, int num_experts, int64_t M_total,
                                      int64_t N, int64_t K, void *y, nvfp4_out_dtype out_dtype,
                                      nvfp4_epilogue epi, void *workspace, int32_t *dev_status,
                                      cudaStream_t stream);

/*
 * nvfp4_gemm_select_kernel -- which grouped GEMM kernel nvfp4_grouped_gemm runs
 * (process-wide; a tuning and testing switch, not part of the pages' method):
 *   0  automatic (default): for a bf16 output with N % 256 == 0 and
 *      K >= 1024, the kernel of mode 4; otherwise one CTA per 128-row weight
 *      tile, with 512-element K stages when K % 512 == 0 (tiles of at most 64
 *      tokens in a ring of three slots when the experts average at most 16
 *      routed rows, M_total <= 16 * num_experts; of at most 192 tokens in two
 *      slots otherwise) and 256-element stages when not;
 *   1  one CTA per tile, 256-element K stages;  2  CTA pairs (tcgen05
 *      cta_group::2, 256 weight rows per tile; N % 256 != 0 is then
 *      NVFP4_ERR_UNSUPPORTED_SHAPE);  3  the three-slot, 64-token ring
 *      whenever K % 512 == 0 (256-element stages otherwise);  4  two
 *      128-row weight blocks per tile sharing one token tile, three
 *      256-element K stages, whenever N % 256 == 0 and the output is bf16
 *      (plain Y, SwiGLU h, or NVFP4 h from nvfp4_grouped_gemm_swiglu_nvfp4);
 *      other calls run as in mode 0.
 *      The modes apply to nvfp4_grouped_gemm_swiglu_nvfp4 too, and modes 0
 *      and 4 to mxfp4_grouped_gemm (its other modes run as mode 0).
 * All give the same Y up to the fp32 accumulation order inside a tile.
 * Returns NVFP4_ERR_INVALID_ARG for another mode.
 */
nvfp4_status nvfp4_gemm_select_kernel(int mode);

/*
 * nvfp4_gemm_set_wait_budget -- a testing switch for the failure path of the
 * one-CTA grouped GEMM kernels (nvfp4_gemm_select_kernel modes 0, 1, 3 and
 * 4; not part of the pages' method).  Every wait of the kernel's main loop on a ring,
 * scale or accumulator barrier gives up after this many SM clock cycles: it
 * raises the CTA's abort flag, writes NVFP4_ERR_TIMEOUT to dev_status, and
 * every role leaves its loop.  The closing waits for copies and MMAs still in
 * flight keep the full budget, so the kernel ends cleanly and the context
 * stays usable.  cycles = 0 restores the default (4e9 cycles, about 2 s); a
 * test sets 1 to force the timeout.  Process-wide, synchronous; call it
 * between launches.  Returns NVFP4_ERR_INVALID_ARG for cycles < 0.
 */
nvfp4_status nvfp4_gemm_set_wait_budget(int64_t cycles);

/*
 * nvfp4_swiglu_quantize -- the step between the two expert projections:
 * h = bf16(silu(g) * u) with g = y[:, :I] (gate rows of the fused gate_up
 * weight come first) and u = y[:, I:], then h is NVFP4-quantized per expert
 * group exactly as nvfp4_quantize(FROM_AMAX) would quantize it.
 *   y        fp32 or bf16 [rows, 2I] (the gate_up GEMM output, routed order).
 *   h        nullable bf16 [rows, I]: also store h.
 *   group_offsets / num_groups / global_scale / q / sf / sf_layout: as in
 *   nvfp4_quantize (global scales are always computed from the amax of h).
 *   silu(g) = g / (1 + exp(-g)) in fp32 with the device expf.
 */
nvfp4_status nvfp4_swiglu_quantize(const void *y, nvfp4_out_dtype y_dtype, int64_t rows,
                                   int64_t I, const int32_t *group_offsets, int num_groups,
                                   float *global_scale, uint8_t *q, uint8_t *sf,
                                   nvfp4_sf_layout sf_layout, void *h, void *workspace,
                                   int32_t *dev_status, cudaStream_t stream);

/*
 * nvfp4_kv_quantize -- NVFP4 KV-cache write for one attention layer: K and V
 * (bf16 [tokens, heads, head_dim] each) quantized in groups of 16 along
 * head_dim, one global scale per tensor.  [P3: --kv-cache-dtype nvfp4.]
 * Same arithmetic as nvfp4_quantize with rows = tokens*heads and
 * K = head_dim; k_gs / v_gs are fp32 [1] each, written (FROM_AMAX) or read
 * (GIVEN, the serving case).  Scales are ROWMAJOR.
 *   workspace >= nvfp4_workspace_size(2).
 */
nvfp4_status nvfp4_kv_quantize(const void *k, const void *v, int64_t tokens, int64_t heads,
                               int64_t head_dim, nvfp4_gs_mode gs_mode, float *k_gs, float *v_gs,
                               uint8_t *k_q, uint8_t *k_sf, uint8_t *v_q, uint8_t *v_sf,
                               void *workspace, int32_t *dev_status, cudaStream_t stream);

/* nvfp4_kv_dequantize -- the attention-side read: both tensors back to bf16. */
nvfp4_status nvfp4_kv_dequantize(const uint8_t *k_q, const uint8_t *k_sf, const float *k_gs,
                                 const uint8_t *v_q, const uint8_t *v_sf, const float *v_gs,
                                 int64_t tokens, int64_t heads, int64_t head_dim,
                                 void *k_out, void *v_out, cudaStream_t stream);

/*
 * nvfp4_moe_route -- routed (token, choice) pairs -> expert-grouped row order.
 * [P1 results section: each token goes to its top-10 of 512 routed experts;
 *  the grouped GEMM consumes the routed rows of one expert contiguously.]
 *   topk_ids        int32 [tokens, topk] expert ids (the router's choices;
 *                   a token lists an expert at most once).
 *   expert_offsets  int32 [num_experts+1] out: prefix sums of the per-expert
 *                   row counts (the `group_offsets` / `expert_offsets` of the
 *                   calls above).
 *   row_index       int32 [tokens*topk] out: token id of every routed row;
 *                   rows of an expert are in ascending token id.
 *   slot            int32 [tokens, topk] out: routed row of each choice
 *                   (-1 for an out-of-range id).
 *   workspace       >= nvfp4_moe_route_workspace_size(tokens, num_experts).
 *   num_experts <= 2048, topk <= 32.  Deterministic (no order-dependent
 *   atomics decide any output).  dev_status: NVFP4_ERR_INDEX for an id
 *   outside [0, num_experts) (that pair is dropped).
 */
size_t nvfp4_moe_route_workspace_size(int64_t tokens, int num_experts);
nvfp4_status nvfp4_moe_route(const int32_t *topk_ids, int64_t tokens, int topk, int num_experts,
                             int32_t *expert_offsets, int32_t *row_index, int32_t *slot,
                             void *workspace, int32_t *dev_status, cudaStream_t stream);

/*
 * nvfp4_moe_combine -- out[t, :] = sum_j weights[t, j] * y[slot[t, j], :],
 * accumulated in fp32 in choice order (the weighted sum of a token's expert
 * outputs after the down projection).
 *   y, rows  fp32 or bf16 [rows, H] (the down GEMM output); H % 8 == 0.
 *   slot     int32 [tokens, topk] from nvfp4_moe_route: -1 entries are
 *            skipped; an entry >= rows is skipped and reported as
 *            NVFP4_ERR_INDEX in dev_status (nullable), never read.
 *   weights  fp32 [tokens, topk] routing weights.
 *   out      fp32 or bf16 [tokens, H].
 */
nvfp4_status nvfp4_moe_combine(const void *y, nvfp4_out_dtype y_dtype, int64_t rows, const int32_t *slot,
                               const float *weights, int64_t tokens, int topk, int64_t H, void *out,
                               nvfp4_out_dtype out_dtype, int32_t *dev_status, cudaStream_t stream);

/*
 * nvfp4_quantize_noalloc -- nvfp4_quantize without a caller workspace.
 *
 * For callers that cannot hand the library a scratch buffer: code that must
 * not call cudaMalloc or a caching allocator at this point (a host runtime
 * whose device memory is owned and budgeted by another component, an
 * allocator-free plug-in or interposer, a hot path that has to stay free of
 * allocation-related synchronisation).  This entry point is not described by
 * the pages; it exists for those callers.
 *
 * Same arguments, arithmetic and results as nvfp4_quantize, minus `workspace`.
 * The scratch (per-group amax words) lives in one static device array inside
 * the library, sized for NVFP4_NOALLOC_MAX_GROUPS groups (8.25 KB on every GPU
 * that loads the library, held until process exit).  num_groups (or 1 without
 * group_offsets) above NVFP4_NOALLOC_MAX_GROUPS returns
 * NVFP4_ERR_UNSUPPORTED_SHAPE.  Nothing is allocated or freed: the first call
 * on a device looks up that device's address of the array (a runtime symbol
 * query, no allocation) and caches it, so make that first call before any
 * stream capture on the device.  Every call shares the array and clears the
 * words it needs before use; calls that can overlap on the GPU (different
 * streams, or a second call enqueued before the first finished on another
 * stream) race on it and must be serialised by the caller.
 */
#define NVFP4_NOALLOC_MAX_GROUPS 1024
nvfp4_status nvfp4_quantize_noalloc(const void *x, int64_t rows, int64_t K, int64_t ld_x,
                                    const int32_t *row_index, const int32_t *group_offsets,
                                    int num_groups, nvfp4_gs_mode gs_mode, float *global_scale,
                                    uint8_t *q, uint8_t *sf, nvfp4_sf_layout sf_layout,
                                    int32_t *dev_status, cudaStream_t stream);

#ifdef __cplusplus
}
#endif
#endif /* NVFP4_H_ */
