/*
 * NVFP4 reference oracle -- TEST INFRASTRUCTURE ONLY.
 *
 * A plain, scalar, CPU implementation of what the NVFP4 W4A4 hot path
 * computes.  It is used only by the tests, by the package smoke check and by
 * the CPU-baseline leg of the bench; the product path never calls it.  It
 * shares no code, header or table with the CUDA library.
 *
 * Sources (the pages are cited by page title and section):
 *  [P1] "Qwen3.8-Flash-Next-NVFP4 ..." (lpnh.cn/news/2736522), section
 *       "核心W4A4 双级缩放机制拆解" (the two-level scaling mechanism): 16-element
 *       blocks along the last dimension with an FP8 E4M3 scale (scale_bits
 *       [4,3]), one FP32 global scale per tensor, 4.5 effective bits, largest
 *       audited block scale 448.0, weights static / activations dynamic.
 *  [P2] "DeepSeek-V4.1-Flash-NVFP4 ..." (kwkr.cn/news/613851), section
 *       "二、NVFP4 格式拆解" (the format): E2M1 = 1 sign, 2 exponent, 1 mantissa
 *       bit, magnitudes {0,0.5,1,1.5,2,3,4,6} (FP4_TABLE), two values per byte
 *       (float4_e2m1fn_x2), group size 16; the MXFP4 -> NVFP4 table (32-element
 *       blocks with power-of-two UE8M0 scales vs 16-element blocks), lossless
 *       block-by-block remap; section "四、量化是如何完成的" (blocks verified).
 *  [P3] "Qwen3.8-2.4T-A95B-NVFP4 ..." (hnwysp.cn/news/107543), section "为什么值得开
 *       NVFP4 KV 缓存": NVFP4 KV cache, group size 16.
 *
 * Readings taken where the pages are silent:
 *  - global scale s_g = amax / (6 * 448); s_g = 1 for an all-zero tensor;
 *  - every fp32 step is one IEEE round-to-nearest-even operation;
 *  - E4M3 block scale: round-to-nearest-even, saturate to 448, subnormals kept;
 *  - E2M1: round-to-nearest-even (ties to the even mantissa bit), saturate to
 *    6 (also for +-inf), sign kept (a negative value rounding to 0 gives -0),
 *    NaN encodes as +0;
 *  - element 2j in bits [3:0] and element 2j+1 in bits [7:4] of byte j;
 *  - remap: g = e_max - 8 over the blocks that are not all zero;
 *  - MXFP4 encode: the OCP MX v1.0 exponent rule E = floor(log2 amax) - 2,
 *    clamped to the UE8M0 range, byte 0 for an all-zero block, 0xFF for a
 *    block with a non-finite element.
 *
 * Compiled with -O2 -ffp-contract=off and no fast-math, so every float
 * expression below is evaluated as written.
 */
#include <math.h>
#include <stdint.h>
#include <stddef.h>
#include <string.h>
#include <stdlib.h>

#define ORC_OK 0
#define ORC_ERR_NONFINITE 16
#define ORC_ERR_NOT_REPRESENTABLE 17

/* ------------------------------------------------------------------ */
/* bf16 <-> fp32                                                       */
/* ------------------------------------------------------------------ */
static float bf16_to_f32(uint16_t b) {
    uint32_t u = ((uint32_t)b) << 16;
    float f;
    memcpy(&f, &u, 4);
    return f;
}

static uint16_t f32_to_bf16_rne(float f) {
    uint32_t u;
    memcpy(&u, &f, 4);
    if ((u & 0x7F800000u) == 0x7F800000u && (u & 0x007FFFFFu)) return (uint16_t)((u >> 16) | 0x40u);
    uint32_t r = u + 0x7FFFu + ((u >> 16) & 1u);
    return (uint16_t)(r >> 16);
}

/* ------------------------------------------------------------------ */
/* E2M1 (FP4) codec  [P2, the format section]                          */
/* ------------------------------------------------------------------ */

/* The eight magnitudes printed on the page, indexed by the 3 low code bits
 * (exponent bits [2:1], mantissa bit [0]). */
static const double E2M1_MAG[8] = {0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0};

double orc_e2m1_decode(uint8_t code) {
    double m = E2M1_MAG[code & 7];
    return (code & 8) ? -m : m;
}

/* Round-to-nearest-even onto the E2M1 grid, saturating at 6.
 * Midpoints between neighbours go to the neighbour whose mantissa bit is 0:
 *   0.25 -> 0, 0.75 -> 1.0, 1.25 -> 1.0, 1.75 -> 2.0, 2.5 -> 2.0, 3.5 -> 4.0, 5 -> 4.0. */
uint8_t orc_e2m1_encode(float v) {
    if (isnan(v)) return 0;
    uint8_t sign = signbit(v) ? 8 : 0;
    float a = fabsf(v);
    uint8_t mag;
    if (a <= 0.25f)      mag = 0;   /* tie 0.25 -> 0 (even) */
    else if (a < 0.75f)  mag = 1;   /* 0.5 */
    else if (a <= 1.25f) mag = 2;   /* 1.0; ties 0.75 and 1.25 -> 1.0 (even) */
    else if (a < 1.75f)  mag = 3;   /* 1.5 */
    else if (a <= 2.5f)  mag = 4;   /* 2.0; ties 1.75 and 2.5 -> 2.0 */
    else if (a < 3.5f)   mag = 5;   /* 3.0 */
    else if (a <= 5.0f)  mag = 6;   /* 4.0; ties 3.5 and 5 -> 4.0 */
    else                 mag = 7;   /* 6.0, saturating (inf included) */
    return (uint8_t)(sign | mag);
}

/* ------------------------------------------------------------------ */
/* FP8 E4M3 (fn) codec  [P1: scale_bits [4,3], max scale 448]          */
/* ------------------------------------------------------------------ */

/* bias 7; exponent field 0 is subnormal (m * 2^-9); 0x7F / 0xFF are NaN. */
double orc_e4m3_decode(uint8_t code) {
    int s = code >> 7, e = (code >> 3) & 15, m = code & 7;
    double v;
    if (e == 15 && m == 7) return NAN;
    if (e == 0) v = ldexp((double)m, -9);
    else v = ldexp(1.0 + m / 8.0, e - 7);
    return s ? -v : v;
}

/* Round half to even of a non-negative double that is a multiple of 1/2^k
 * (exact inputs only: callers pass values whose fraction is exact). */
static double round_half_even(double x) {
    double f = floor(x);
    double d = x - f;
    if (d > 0.5) return f + 1.0;
    if (d < 0.5) return f;
    return (fmod(f, 2.0) == 0.0) ? f : f + 1.0;
}

/* Round-to-nearest-even to E4M3, saturating finite values to +-448. */
uint8_t orc_e4m3_encode(float v) {
    if (isnan(v)) return 0x7F;
    uint8_t sign = signbit(v) ? 0x80 : 0;
    double a = fabs((double)v);
    if (a >= 448.0) return (uint8_t)(sign | 0x7E);
    if (a < ldexp(1.0, -6)) {
        /* subnormal range: multiples of 2^-9 */
        double m = round_half_even(a * 512.0);   /* exact scaling by a power of two */
        if (m >= 8.0) return (uint8_t)(sign | 0x08); /* rounds up to 2^-6 */
        return (uint8_t)(sign | (uint8_t)m);
    }
    int e;
    double fr = frexp(a, &e);          /* a = fr * 2^e, fr in [0.5, 1) */
    int E = e - 1;                     /* a = (2*fr) * 2^E, 2*fr in [1, 2) */
    double mant = (2.0 * fr - 1.0) * 8.0; /* exact: fp32 has 24 bits */
    double m = round_half_even(mant);
    if (m >= 8.0) { m = 0.0; E += 1; }
    int field = E + 7;
    if (field > 15 || (field == 15 && m >= 7.0)) return (uint8_t)(sign | 0x7E);
    return (uint8_t)(sign | (field << 3) | (int)m);
}

/* ------------------------------------------------------------------ */
/* Quantize  [P1 two-level scaling; P2 format]                          */
/* ------------------------------------------------------------------ */

/* s_g from the amax: the block holding the amax gets the scale 448. */
float orc_global_scale_from_amax(float amax) {
    if (amax == 0.0f) return 1.0f;
    return amax / 2688.0f;   /* 2688 = 6 * 448 */
}

/* E4M3 scale byte of one 16-element block with block amax a_b. */
uint8_t orc_block_scale(float a_b, float s_g) {
    float t = 6.0f * s_g;
    float sigma = a_b / t;
    return orc_e4m3_encode(sigma);
}

/* Encode one 16-element block given its scale byte S and the global s_g.
 * x: 16 fp32 values; out: 8 packed bytes. */
void orc_encode_block(const float *x, uint8_t S, float s_g, uint8_t *out) {
    float e = (float)orc_e4m3_decode(S) * s_g;
    float r = (e == 0.0f) ? 0.0f : 1.0f / e;
    for (int j = 0; j < 8; ++j) {
        float v0 = x[2 * j] * r;
        float v1 = x[2 * j + 1] * r;
        uint8_t c0 = orc_e2m1_encode(v0);
        uint8_t c1 = orc_e2m1_encode(v1);
        out[j] = (uint8_t)(c0 | (c1 << 4));
    }
}

/* amax of |x| over a set of bf16 rows: rows r in [r0, r1) of the gathered
 * matrix, row r being x[row_index ? row_index[r] : r].  Returns the max as
 * fp32; NaN propagates as NaN, inf as inf. */
static float group_amax(const uint16_t *x, int64_t K, int64_t ld, const int32_t *row_index,
                        int64_t r0, int64_t r1) {
    float amax = 0.0f;
    int nan_seen = 0;
    for (int64_t r = r0; r < r1; ++r) {
        const uint16_t *row = x + (row_index ? (int64_t)row_index[r] : r) * ld;
        for (int64_t k = 0; k < K; ++k) {
            float a = fabsf(bf16_to_f32(row[k]));
            if (isnan(a)) nan_seen = 1;
            else if (a > amax) amax = a;
        }
    }
    return nan_seen ? NAN : amax;
}

/*
 * Quantize bf16 rows to NVFP4.
 *   x: bf16 bits, [*, ld]; rows of the gathered matrix are x[row_index[r]]
 *      (or x[r] when row_index is NULL), r in [0, rows).
 *   group_offsets: NULL (one group = whole matrix) or [num_groups+1] prefix
 *      sums over gathered rows; each group gets its own global scale.
 *   gs_given: 0 = global scale from amax (written to global_scale[g]),
 *             1 = global_scale[g] is read.
 *   q: [rows, K/2] packed codes, sf: [rows, K/16] E4M3 bytes (row-major),
 *   both in gathered row order (no padding).
 * Returns ORC_OK, or ORC_ERR_NONFINITE when some input element of a
 * processed group is NaN or +-inf (outputs of that group are then left
 * unspecified; in the amax mode its global scale is written as NaN).
 */
int orc_quantize(const uint16_t *x, int64_t rows, int64_t K, int64_t ld,
                 const int32_t *row_index, const int32_t *group_offsets, int num_groups,
                 int gs_given, float *global_scale, uint8_t *q, uint8_t *sf) {
    int status = ORC_OK;
    int G = group_offsets ? num_groups : 1;
    for (int g = 0; g < G; ++g) {
        int64_t r0 = group_offsets ? group_offsets[g] : 0;
        int64_t r1 = group_offsets ? group_offsets[g + 1] : rows;
        float s_g;
        if (gs_given) {
            s_g = global_scale[g];
        } else {
            float amax = group_amax(x, K, ld, row_index, r0, r1);
            if (!isfinite(amax)) { status = ORC_ERR_NONFINITE; global_scale[g] = NAN; continue; }
            s_g = orc_global_scale_from_amax(amax);
            global_scale[g] = s_g;
        }
        int bad = 0;
        #pragma omp parallel for schedule(static) reduction(|:bad)
        for (int64_t r = r0; r < r1; ++r) {
            const uint16_t *row = x + (row_index ? (int64_t)row_index[r] : r) * ld;
            for (int64_t b = 0; b < K / 16; ++b) {
                float v[16];
                float a_b = 0.0f;
                for (int i = 0; i < 16; ++i) {
                    v[i] = bf16_to_f32(row[b * 16 + i]);
                    float a = fabsf(v[i]);
                    if (!isfinite(a)) bad = 1;
                    else if (a > a_b) a_b = a;
                }
                uint8_t S = orc_block_scale(a_b, s_g);
                sf[r * (K / 16) + b] = S;
                orc_encode_block(v, S, s_g, q + r * (K / 2) + b * 8);
            }
        }
        if (bad) status = ORC_ERR_NONFINITE;
    }
    return status;
}

/*
 * Dequantize: x_hat = (code * S) * s_g, in fp32 (the first product is exact).
 *   row_gs: per-row global scale (callers expand group scales to rows).
 *   out_f32 (nullable) [rows, K]; out_bf16 (nullable) bits [rows, K], RNE of the fp32 value.
 */
void orc_dequantize(const uint8_t *q, const uint8_t *sf, const float *row_gs,
                    int64_t rows, int64_t K, float *out_f32, uint16_t *out_bf16) {
    #pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < rows; ++r) {
        for (int64_t k = 0; k < K; ++k) {
            uint8_t byte = q[r * (K / 2) + k / 2];
            uint8_t code = (k & 1) ? (byte >> 4) : (byte & 15);
            float S = (float)orc_e4m3_decode(sf[r * (K / 16) + k / 16]);
            float c = (float)orc_e2m1_decode(code);
            float y = (c * S) * row_gs[r];
            if (out_f32) out_f32[r * K + k] = y;
            if (out_bf16) out_bf16[r * K + k] = f32_to_bf16_rne(y);
        }
    }
}

/* Dequantize to fp64 (used to form the GEMM operands): code * S * s_g in
 * fp64, which is exact (at most 2 + 4 + 24 significant bits). */
void orc_dequantize_f64(const uint8_t *q, const uint8_t *sf, const float *row_gs,
                        int64_t rows, int64_t K, double *out) {
    #pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < rows; ++r) {
        for (int64_t k = 0; k < K; ++k) {
            uint8_t byte = q[r * (K / 2) + k / 2];
            uint8_t code = (k & 1) ? (byte >> 4) : (byte & 15);
            out[r * K + k] = orc_e2m1_decode(code) * orc_e4m3_decode(sf[r * (K / 16) + k / 16])
                             * (double)row_gs[r];
        }
    }
}

/* ------------------------------------------------------------------ */
/* MXFP4 -> NVFP4 remap  [P2: format table; lossless block remap]      */
/* ------------------------------------------------------------------ */

/* E4M3 byte holding exactly 2^p, p in [-9, 8]. */
static uint8_t e4m3_pow2(int p) {
    if (p >= -6) return (uint8_t)((p + 7) << 3);
    return (uint8_t)(1 << (p + 9));   /* subnormal: 2^p = 2^(p+9) * 2^-9 */
}

/*
 * n_tensors tensors of [rows, K] laid back to back.  Codes are copied
 * unchanged; every 32-block with exponent byte u (scale 2^(u-127)) becomes
 * two 16-blocks with the E4M3 scale 2^(e - g); s_g = 2^g with g = e_max - 8,
 * e_max over the blocks whose 32 codes are not all +-0 (g = 0 when there is
 * none).  Returns ORC_ERR_NOT_REPRESENTABLE when a byte is 0xFF (NaN) or the
 * spread e_min - g < -9 on some tensor (that tensor's outputs then follow the
 * clamp rule below and are not lossless).
 * Blocks that are all zero get 2^clamp(e-g, -9, 8).
 */
int orc_remap_mxfp4(const uint8_t *q_mx, const uint8_t *e8, int64_t n_tensors, int64_t rows,
                    int64_t K, uint8_t *q_nv, uint8_t *sf_nv, float *global_scale) {
    int status = ORC_OK;
    int64_t nb32 = rows * (K / 32);
    for (int64_t t = 0; t < n_tensors; ++t) {
        const uint8_t *qt = q_mx + t * rows * (K / 2);
        const uint8_t *et = e8 + t * nb32;
        int have = 0, emax = 0, emin = 0;
        for (int64_t b = 0; b < nb32; ++b) {
            if (et[b] == 0xFF) { status = ORC_ERR_NOT_REPRESENTABLE; continue; }
            int allzero = 1;
            for (int j = 0; j < 16; ++j)
                if (qt[b * 16 + j] & 0x77) { allzero = 0; break; }
            if (allzero) continue;
            int e = (int)et[b] - 127;
            if (!have) { emax = emin = e; have = 1; }
            if (e > emax) emax = e;
            if (e < emin) emin = e;
        }
        int g = have ? emax - 8 : 0;
        if (have && emin - g < -9) status = ORC_ERR_NOT_REPRESENTABLE;
        global_scale[t] = (float)ldexp(1.0, g);
        for (int64_t b = 0; b < nb32; ++b) {
            int e = (int)et[b] - 127;
            int p = e - g;
            if (p < -9) p = -9;
            if (p > 8) p = 8;
            uint8_t S = e4m3_pow2(p);
            sf_nv[t * rows * (K / 16) + 2 * b] = S;
            sf_nv[t * rows * (K / 16) + 2 * b + 1] = S;
        }
        memcpy(q_nv + t * rows * (K / 2), qt, (size_t)(rows * (K / 2)));
    }
    return status;
}

/* MXFP4 dequantize in fp64: code * 2^(u-127). */
void orc_dequantize_mxfp4_f64(const uint8_t *q, const uint8_t *e8, int64_t rows, int64_t K,
                              double *out) {
    for (int64_t r = 0; r < rows; ++r)
        for (int64_t k = 0; k < K; ++k) {
            uint8_t byte = q[r * (K / 2) + k / 2];
            uint8_t code = (k & 1) ? (byte >> 4) : (byte & 15);
            out[r * K + k] = ldexp(orc_e2m1_decode(code), (int)e8[r * (K / 32) + k / 32] - 127);
        }
}

/* ------------------------------------------------------------------ */
/* MXFP4 encode  [P2, section 三 (which layers): the FP8 -> MXFP4 step, */
/* one UE8M0 scale per 32 elements, lossy; format table of section 二] */
/* ------------------------------------------------------------------ */

/* The page fixes the block (32 elements) and the scale type (UE8M0, a power
 * of two) but not how the exponent is chosen.  Reading taken: the OCP
 * Microscaling v1.0 conversion.  Per 32-block of a row,
 *   E = floor(log2(amax)) - 2          (2 = exponent of 6, the largest E2M1),
 *   E clamped to [-127, 127]           (UE8M0 byte u = E + 127; 0xFF is NaN),
 *   code_k = e2m1(x_k / 2^E)           (round to nearest even, saturating at 6).
 * An all-zero block takes u = 0 and zero codes (signs kept).  A block holding
 * a NaN or an infinity takes u = 0xFF and all codes 0, and the call returns
 * ORC_ERR_NONFINITE.  The input is bf16, which holds every FP8 E4M3 value
 * exactly, so an FP8 source is covered by passing its values as bf16.
 * x: [rows, ld_x] bf16, K % 32 == 0; q: [rows, K/2]; e8: [rows, K/32]. */
int orc_quantize_mxfp4(const uint16_t *x, int64_t rows, int64_t K, int64_t ld_x,
                       uint8_t *q, uint8_t *e8) {
    int status = ORC_OK;
    for (int64_t r = 0; r < rows; ++r)
        for (int64_t b = 0; b < K / 32; ++b) {
            const uint16_t *xb = x + r * ld_x + b * 32;
            uint8_t *qb = q + r * (K / 2) + b * 16;
            double amax = 0.0;
            int finite = 1;
            for (int k = 0; k < 32; ++k) {
                double v = bf16_to_f32(xb[k]);
                if (!isfinite(v)) finite = 0;
                else if (fabs(v) > amax) amax = fabs(v);
            }
            if (!finite) {
                status = ORC_ERR_NONFINITE;
                e8[r * (K / 32) + b] = 0xFF;
                memset(qb, 0, 16);
                continue;
            }
            int E = -127;
            if (amax > 0.0) {
                int e2;
                frexp(amax, &e2);          /* amax = m * 2^e2, m in [0.5, 1) */
                E = (e2 - 1) - 2;          /* floor(log2 amax) - 2 */
                if (E < -127) E = -127;
                if (E > 127) E = 127;
            }
            e8[r * (K / 32) + b] = (uint8_t)(E + 127);
            for (int k = 0; k < 32; k += 2) {
                uint8_t c0 = orc_e2m1_encode((float)ldexp(bf16_to_f32(xb[k]), -E));
                uint8_t c1 = orc_e2m1_encode((float)ldexp(bf16_to_f32(xb[k + 1]), -E));
                qb[k / 2] = (uint8_t)(c0 | (c1 << 4));
            }
        }
    return status;
}

/* ------------------------------------------------------------------ */
/* SwiGLU between the two projections                                  */
/* ------------------------------------------------------------------ */

/* h[r, j] = bf16( silu(g) * u ), g = y[r, j], u = y[r, I + j]; silu(g) =
 * g / (1 + exp(-g)), evaluated in fp64 and rounded once to bf16. */
void orc_swiglu(const float *y, int64_t rows, int64_t I, uint16_t *h) {
    #pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < rows; ++r)
        for (int64_t j = 0; j < I; ++j) {
            double g = y[r * 2 * I + j], u = y[r * 2 * I + I + j];
            double s = g / (1.0 + exp(-g));
            h[r * I + j] = f32_to_bf16_rne((float)(s * u));
        }
}

/* ------------------------------------------------------------------ */
/* Dot products for sampled GEMM outputs (fp64)                        */
/* ------------------------------------------------------------------ */

/* y = sum_k a[k] * b[k] and sabs = sum_k |a[k] * b[k]| in fp64. */
void orc_dot_f64(const double *a, const double *b, int64_t K, double *y, double *sabs) {
    double s = 0.0, t = 0.0;
    for (int64_t k = 0; k < K; ++k) {
        double p = a[k] * b[k];
        s += p;
        t += fabs(p);
    }
    *y = s;
    *sabs = t;
}

/* Bulk helpers over many values, for exhaustive codec checks. */
void orc_e2m1_encode_array(const float *v, int64_t n, uint8_t *out) {
    #pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < n; ++i) out[i] = orc_e2m1_encode(v[i]);
}

void orc_e4m3_encode_array(const float *v, int64_t n, uint8_t *out) {
    #pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < n; ++i) out[i] = orc_e4m3_encode(v[i]);
}

/* Encode every fp32 bit pattern in [lo, hi) (as uint32) -- lets a test walk
 * all 2^32 inputs without materialising them. */
void orc_e2m1_encode_bits_range(uint64_t lo, uint64_t hi, uint8_t *out) {
    #pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < (int64_t)(hi - lo); ++i) {
        uint32_t u = (uint32_t)(lo + (uint64_t)i);
        float f;
        memcpy(&f, &u, 4);
        out[i] = orc_e2m1_encode(f);
    }
}

void orc_e4m3_encode_bits_range(uint64_t lo, uint64_t hi, uint8_t *out) {
    #pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < (int64_t)(hi - lo); ++i) {
        uint32_t u = (uint32_t)(lo + (uint64_t)i);
        float f;
        memcpy(&f, &u, 4);
        out[i] = orc_e4m3_encode(f);
    }
}

/* ------------------------------------------------------------------ */
/* MoE routing structure and combine (the steps on either side of the  */
/* expert GEMMs; P1 results section: top-10 of 512 routed experts)     */
/* ------------------------------------------------------------------ */

/*
 * Group routed (token, choice) pairs by expert: expert e's rows are the
 * tokens that chose e, in ascending token id; offsets[E+1] are the prefix
 * sums of the counts; slot[t*k + j] is the routed row of token t's j-th
 * choice.  A plain counting sort in token order.
 * A choice whose expert id is outside [0, E) is dropped (reading taken: the
 * pages route each token to experts of the model only, so an id past the
 * table names no expert): it gets slot -1, is not counted in the offsets and
 * gets no routed row, so row_index holds offsets[E] entries and its tail is
 * left untouched.  Returns 0, 1 when some choice was dropped, or 2 for
 * arguments that describe no routing at all (E, k <= 0 or T < 0).
 */
int orc_route(const int32_t *ids, int64_t T, int k, int E, int32_t *offsets, int32_t *row_index,
              int32_t *slot) {
    if (E <= 0 || k <= 0 || T < 0) return 2;
    int dropped = 0;
    for (int e = 0; e <= E; ++e) offsets[e] = 0;
    for (int64_t i = 0; i < T * k; ++i) {
        if (ids[i] < 0 || ids[i] >= E) { dropped = 1; continue; }
        offsets[ids[i] + 1] += 1;
    }
    for (int e = 0; e < E; ++e) offsets[e + 1] += offsets[e];
    int32_t *fill = (int32_t *)malloc(sizeof(int32_t) * (size_t)(unsigned)E);
    if (!fill) return 2;
    for (int e = 0; e < E; ++e) fill[e] = offsets[e];
    for (int64_t t = 0; t < T; ++t)
        for (int j = 0; j < k; ++j) {
            int e = ids[t * k + j];
            if (e < 0 || e >= E) { slot[t * k + j] = -1; continue; }
            int32_t r = fill[e]++;
            row_index[r] = (int32_t)t;
            slot[t * k + j] = r;
        }
    free(fill);
    return dropped;
}

/* out[t, :] = sum_j w[t, j] * y[slot[t, j], :], accumulated in fp64 in
 * choice order, skipping slot -1; also |w*y| summed for the tolerance.  y is fp32. */
void orc_combine(const float *y, const int32_t *slot, const float *w, int64_t T, int k, int64_t H,
                 double *out, double *sabs) {
    #pragma omp parallel for schedule(static)
    for (int64_t t = 0; t < T; ++t)
        for (int64_t c = 0; c < H; ++c) {
            double s = 0.0, a = 0.0;
            for (int j = 0; j < k; ++j) {
                if (slot[t * k + j] < 0) continue;      /* a choice the routing dropped adds nothing */
                double p = (double)w[t * k + j] * (double)y[(int64_t)slot[t * k + j] * H + c];
                s += p;
                a += fabs(p);
            }
            out[t * H + c] = s;
            sabs[t * H + c] = a;
        }
}
