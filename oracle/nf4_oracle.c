/*
 * nf4_oracle.c -- plain, slow, obviously-correct CPU oracle for the NF4 +
 * double-quantization encoding of a frozen QLoRA base weight.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product library links, loads or
 * calls this file; only the tests, the smoke check and the CPU-baseline leg of
 * the benchmark do.  It shares no code, header, table or constant generator
 * with the CUDA library: the codebook here comes from Wichura's AS 241
 * inverse-normal, the library computes its own by bisection on erfc.
 *
 * What the pages fix, and where:
 *   - "QLoRA Guide" (dataaihub.co), section "NF4 vs uniform INT4": NF4 places
 *     its 16 levels at quantiles of the standard normal; quantization is
 *     block-wise so an outlier only spoils its own block.
 *   - "Qlora Expert" (skillsdirectory.com), section "Core Concept": levels at
 *     N(0,1) quantiles; double quantization re-quantizes the per-block fp32
 *     constants to 8 bit; section "Memory Math" / "Hyperparameter Guidance":
 *     the saving is about 0.37 bit per parameter.
 *   - "QLoRA Implementation Details (2025 Edition)" (spritualkrishna.cloud),
 *     section "Step 1: 4-bit Quantization with NF4", "NF4 Math": 64 values
 *     per block.
 *   - "QLoRA: The 4-bit Revolution" (shshell.com), section "2. Double
 *     Quantization": the scaling factors go from 32-bit to 8-bit.
 * Readings taken where the pages are silent:
 *   R1 codebook construction (asymmetric 8 positive / 7 negative quantiles,
 *      offset delta = ((1-1/32)+(1-1/30))/2, normalised by the largest level);
 *   R2 nearest level with ties to the lower index, via fp32 midpoints;
 *   R3 nibble order: element 2j in the high nibble of byte j;
 *   R4 double quantization: groups of 256 block constants, fp32 mean and a
 *      symmetric int8 code of (c - mean) with scale = max|c - mean| / 127;
 *      the group sum is taken in fp64 over a pairwise tree (stride 128..1);
 *   R5 dequantized weight = bf16_rne(L[q] * fmaf(code, scale, mean)).
 *
 * Compile with -ffp-contract=off: every fp32 operation below is meant to be
 * one IEEE-rounded operation, exactly as written.
 */
#include <math.h>
#include <stdint.h>
#include <string.h>

#define NF4_BLOCK 64
#define DQ_GROUP 256

/* ---------------------------------------------------------------------------
 * Inverse standard normal CDF, Wichura (1988), Applied Statistics algorithm
 * AS 241 "PPND16" (rational approximations, about 1e-16 relative accuracy).
 * Returns the x with Phi(x) = p for 0 < p < 1.
 * ------------------------------------------------------------------------- */
double oracle_ppnd16(double p)
{
    double q = p - 0.5;
    double r, val;
    if (fabs(q) <= 0.425) {
        r = 0.180625 - q * q;
        val = q * (((((((r * 2509.0809287301226727 + 33430.575583588128105) * r +
                        67265.770927008700853) * r + 45921.953931549871457) * r +
                      13731.693765509461125) * r + 1971.5909503065514427) * r +
                    133.14166789178437745) * r + 3.387132872796366608) /
              (((((((r * 5226.495278852545925 + 28729.085735721942674) * r +
                    39307.89580009271061) * r + 21213.794301586595867) * r +
                  5394.1960214247511077) * r + 687.1870074920579083) * r +
                42.313330701600911252) * r + 1.0);
        return val;
    }
    r = (q < 0.0) ? p : 1.0 - p;
    r = sqrt(-log(r));
    if (r <= 5.0) {
        r -= 1.6;
        val = (((((((r * 7.7454501427834140764e-4 + 0.0227238449892691845833) * r +
                    0.24178072517745061177) * r + 1.27045825245236838258) * r +
                  3.64784832476320460504) * r + 5.7694972214606914055) * r +
                4.6303378461565452959) * r + 1.42343711074968357734) /
              (((((((r * 1.05075007164441684324e-9 + 5.475938084995344946e-4) * r +
                    0.0151986665636164571966) * r + 0.14810397642748007459) * r +
                  0.68976733498510000455) * r + 1.6763848301838038494) * r +
                2.05319162663775882187) * r + 1.0);
    } else {
        r -= 5.0;
        val = (((((((r * 2.01033439929228813265e-7 + 2.71155556874348757815e-5) * r +
                    0.0012426609473880784386) * r + 0.026532189526576123093) * r +
                  0.29656057182850489123) * r + 1.7848265399172913358) * r +
                5.4637849111641143699) * r + 6.6579046435011037772) /
              (((((((r * 2.04426310338993978564e-15 + 1.4215117583164458887e-7) * r +
                    1.8463183175100546818e-5) * r + 7.868691311456132591e-4) * r +
                  0.0148753612908506148525) * r + 0.13692988092273580531) * r +
                0.59983220655588793769) * r + 1.0);
    }
    return (q < 0.0) ? -val : val;
}

/* ---------------------------------------------------------------------------
 * Reading R1: the 16 NF4 levels.  8 positive quantiles at the first 8 of 9
 * evenly spaced probabilities from delta down to 1/2, 7 negative ones at the
 * first 7 of 8 evenly spaced probabilities, plus an exact zero; sorted and
 * divided (in fp64) by the largest, then rounded once to fp32.  The top and
 * bottom levels are both Phi^-1(delta) before normalisation, so they come out
 * as exactly +1 and -1.
 * ------------------------------------------------------------------------- */
void oracle_nf4_codebook(double out64[16], float out32[16])
{
    const double delta = 0.5 * ((1.0 - 1.0 / 32.0) + (1.0 - 1.0 / 30.0));
    double v[16];
    int n = 0;
    for (int i = 0; i < 7; ++i) {          /* negative side, largest magnitude first */
        double p = delta + (0.5 - delta) * (double)i / 7.0;
        v[n++] = -oracle_ppnd16(p);
    }
    v[n++] = 0.0;
    for (int i = 7; i >= 0; --i) {         /* positive side, ascending */
        double p = delta + (0.5 - delta) * (double)i / 8.0;
        v[n++] = oracle_ppnd16(p);
    }
    /* v is already ascending: -Phi^-1 is increasing in i on the negative side,
     * Phi^-1 is decreasing in i on the positive side and walked backwards. */
    double vmax = v[15];
    for (int i = 0; i < 16; ++i) {
        out64[i] = v[i] / vmax;
        out32[i] = (float)out64[i];
    }
}

/* Reading R2: decision thresholds m_i = fl32((L_i + L_{i+1}) / 2). */
void oracle_nf4_midpoints(const float L[16], float m[15])
{
    for (int i = 0; i < 15; ++i) m[i] = (L[i] + L[i + 1]) * 0.5f;
}

/* Reading R2: the level index of a normalised value is the number of
 * thresholds it lies strictly above (a value exactly on a threshold takes the
 * lower level). */
int oracle_nf4_encode_value(float x, const float m[15])
{
    int q = 0;
    for (int i = 0; i < 15; ++i)
        if (x > m[i]) ++q;
    return q;
}

/* bf16 <-> fp32 from the IEEE-754 definitions (bf16 is the top half of an
 * fp32 word; fp32 -> bf16 rounds to nearest, ties to even). */
float oracle_bf16_to_f32(uint16_t h)
{
    uint32_t u = (uint32_t)h << 16;
    float f;
    memcpy(&f, &u, 4);
    return f;
}

uint16_t oracle_f32_to_bf16(float f)
{
    uint32_t u;
    memcpy(&u, &f, 4);
    if ((u & 0x7fffffffu) > 0x7f800000u) return (uint16_t)((u >> 16) | 0x0040u); /* NaN stays NaN */
    uint32_t lsb = (u >> 16) & 1u;
    u += 0x7fffu + lsb;
    return (uint16_t)(u >> 16);
}

/* ---------------------------------------------------------------------------
 * Block absmax (one fp32 constant per 64 consecutive weights in flattened
 * row-major order).  Exact: a bf16 magnitude is an fp32 value.
 * ------------------------------------------------------------------------- */
void oracle_block_absmax(const uint16_t* W, int64_t nblocks, float* absmax)
{
    for (int64_t b = 0; b < nblocks; ++b) {
        float c = 0.0f;
        for (int j = 0; j < NF4_BLOCK; ++j) {
            float a = fabsf(oracle_bf16_to_f32(W[b * NF4_BLOCK + j]));
            if (a > c) c = a;
        }
        absmax[b] = c;
    }
}

/* ---------------------------------------------------------------------------
 * Reading R4: second-level quantization of the block constants.
 * For the group g of blocks [256 g, 256 g + n_g):
 *   S       = fp64 pairwise sum of the constants (256 slots, empty slots 0,
 *             slot i += slot i + stride for stride = 128, 64, ..., 1)
 *   mean_g  = fl32(S / n_g)
 *   d_b     = fl32(c_b - mean_g)
 *   scale_g = fl32(max_b |d_b| / 127)
 *   code_b  = clamp(rint(fl32(d_b / scale_g)), -127, 127), or 0 if scale_g = 0
 * ------------------------------------------------------------------------- */
void oracle_double_quant(const float* absmax, int64_t nblocks, int8_t* codes, float* scale, float* mean)
{
    int64_t ngroups = (nblocks + DQ_GROUP - 1) / DQ_GROUP;
    for (int64_t g = 0; g < ngroups; ++g) {
        int64_t b0 = g * DQ_GROUP;
        int64_t n = nblocks - b0;
        if (n > DQ_GROUP) n = DQ_GROUP;
        double slot[DQ_GROUP];
        for (int i = 0; i < DQ_GROUP; ++i) slot[i] = (i < n) ? (double)absmax[b0 + i] : 0.0;
        for (int stride = DQ_GROUP / 2; stride >= 1; stride /= 2)
            for (int i = 0; i < stride; ++i) slot[i] = slot[i] + slot[i + stride];
        float mu = (float)(slot[0] / (double)n);
        float dmax = 0.0f;
        for (int64_t i = 0; i < n; ++i) {
            float d = absmax[b0 + i] - mu;
            if (fabsf(d) > dmax) dmax = fabsf(d);
        }
        float sc = dmax / 127.0f;
        for (int64_t i = 0; i < n; ++i) {
            int code = 0;
            if (sc != 0.0f) {
                float d = absmax[b0 + i] - mu;
                float t = rintf(d / sc);
                if (t > 127.0f) t = 127.0f;
                if (t < -127.0f) t = -127.0f;
                code = (int)t;
            }
            codes[b0 + i] = (int8_t)code;
        }
        scale[g] = sc;
        mean[g] = mu;
    }
}

/* ---------------------------------------------------------------------------
 * Quantize + double-quantize a bf16 weight W [N, K] (row-major, K % 64 == 0).
 * Outputs: packed [N, K/2] (reading R3), codes [N*K/64], scale/mean [G].
 * The nibbles are encoded with the true block absmax c_b (quantization
 * happens first, the constants are compressed after).
 * ------------------------------------------------------------------------- */
int oracle_quantize_dq(const uint16_t* W, int64_t N, int64_t K, uint8_t* packed, int8_t* codes,
                       float* scale, float* mean, float* absmax_scratch)
{
    if (N <= 0 || K <= 0 || (K % NF4_BLOCK) != 0) return -1;
    double L64[16];
    float L[16], m[15];
    oracle_nf4_codebook(L64, L);
    oracle_nf4_midpoints(L, m);
    int64_t nblocks = N * K / NF4_BLOCK;
    oracle_block_absmax(W, nblocks, absmax_scratch);
    for (int64_t b = 0; b < nblocks; ++b) {
        float c = absmax_scratch[b];
        for (int j = 0; j < NF4_BLOCK; j += 2) {
            int q[2];
            for (int h = 0; h < 2; ++h) {
                if (c == 0.0f) {
                    q[h] = 7;                        /* the exact-zero level */
                } else {
                    float x = oracle_bf16_to_f32(W[b * NF4_BLOCK + j + h]) / c;
                    q[h] = oracle_nf4_encode_value(x, m);
                }
            }
            packed[(b * NF4_BLOCK + j) / 2] = (uint8_t)((q[0] << 4) | q[1]);
        }
    }
    oracle_double_quant(absmax_scratch, nblocks, codes, scale, mean);
    return 0;
}

/* Reading R5: the block constant recovered from its int8 code. */
float oracle_block_constant(int8_t code, float scale, float mean)
{
    return fmaf((float)code, scale, mean);
}

/* Reading R5: W' = bf16_rne(L[q] * c'_b) for every weight. */
int oracle_dequant(const uint8_t* packed, const int8_t* codes, const float* scale, const float* mean,
                   int64_t N, int64_t K, uint16_t* Wout)
{
    if (N <= 0 || K <= 0 || (K % NF4_BLOCK) != 0) return -1;
    double L64[16];
    float L[16];
    oracle_nf4_codebook(L64, L);
    int64_t nblocks = N * K / NF4_BLOCK;
    for (int64_t b = 0; b < nblocks; ++b) {
        int64_t g = b / DQ_GROUP;
        float cp = oracle_block_constant(codes[b], scale[g], mean[g]);
        for (int j = 0; j < NF4_BLOCK; ++j) {
            int64_t e = b * NF4_BLOCK + j;
            uint8_t byte = packed[e / 2];
            int q = (e % 2 == 0) ? (byte >> 4) : (byte & 0x0f);
            float w = L[q] * cp;
            Wout[e] = oracle_f32_to_bf16(w);
        }
    }
    return 0;
}

/* Dequantize only the listed rows of W' (for sampled parity on large shapes). */
int oracle_dequant_rows(const uint8_t* packed, const int8_t* codes, const float* scale, const float* mean,
                        int64_t N, int64_t K, const int64_t* rows, int64_t nrows, uint16_t* Wout)
{
    if (N <= 0 || K <= 0 || (K % NF4_BLOCK) != 0) return -1;
    double L64[16];
    float L[16];
    oracle_nf4_codebook(L64, L);
    for (int64_t ri = 0; ri < nrows; ++ri) {
        int64_t n = rows[ri];
        if (n < 0 || n >= N) return -2;
        for (int64_t k = 0; k < K; ++k) {
            int64_t e = n * K + k;
            int64_t b = e / NF4_BLOCK;
            int64_t g = b / DQ_GROUP;
            float cp = oracle_block_constant(codes[b], scale[g], mean[g]);
            uint8_t byte = packed[e / 2];
            int q = (e % 2 == 0) ? (byte >> 4) : (byte & 0x0f);
            Wout[ri * K + k] = oracle_f32_to_bf16(L[q] * cp);
        }
    }
    return 0;
}

/* ===========================================================================
 * The FP4 codebook variant ("Qlora Expert", Hyperparameter Guidance: the
 * 4-bit quant type is "nf4" or "fp4"; "QLoRA Guide", FAQs: NF4 vs FP4).
 * The pages give no FP4 values.  Reading: the 4-bit float E2M1 (1 sign,
 * 2 exponent, 1 mantissa bit; magnitudes 0, 0.5, 1, 1.5, 2, 3, 4, 6), the
 * nibble being the E2M1 bit pattern itself (sign in bit 3), normalised to
 * [-1, 1] by dividing by the largest magnitude 6 in fp64 and rounding once
 * to fp32.  Codes 0 and 8 are +0 and -0; the encoder only emits +0.
 * Everything else (blocks of 64, absmax, the double quantization, the
 * dequantized weight bf16_rne(L[q] * c')) is the same as for NF4; only the
 * 16-entry table and the encoder's level order change.
 * ========================================================================= */
#define QUANT_NF4 0
#define QUANT_FP4 1

void oracle_fp4_codebook(double out64[16], float out32[16])
{
    static const double mag[8] = {0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0};
    for (int code = 0; code < 16; ++code) {
        double v = mag[code & 7] / 6.0;
        if (code & 8) v = -v;
        out64[code] = v;
        out32[code] = (float)v;
    }
}

/* The levels of a quant type as nibble-indexed table L, and its distinct
 * levels in ascending order as nibble codes (nlev of them). */
static int codebook_of(int qt, float L[16], int sorted_code[16])
{
    double L64[16];
    if (qt == QUANT_NF4) {
        oracle_nf4_codebook(L64, L);
        for (int i = 0; i < 16; ++i) sorted_code[i] = i;
        return 16;
    }
    if (qt == QUANT_FP4) {
        oracle_fp4_codebook(L64, L);
        int n = 0;
        for (int code = 15; code >= 9; --code) sorted_code[n++] = code;   /* -1 .. -1/12 */
        for (int code = 0; code <= 7; ++code) sorted_code[n++] = code;    /* 0 .. 1 */
        return n;                                                          /* 15: -0 is not emitted */
    }
    return 0;
}

/* The 16-entry table of a quant type (nibble-indexed); returns the number of
 * distinct levels, 0 for an unknown type. */
int oracle_codebook(int qt, float out32[16])
{
    int sc[16];
    return codebook_of(qt, out32, sc);
}

/* Reading R2 for any codebook: thresholds between neighbouring distinct
 * levels m_i = fl32((s_i + s_{i+1}) / 2); the level is the number of
 * thresholds x lies strictly above; its nibble is that level's code. */
int oracle_encode_value_qt(int qt, float x)
{
    float L[16], m[15];
    int sc[16];
    int n = codebook_of(qt, L, sc);
    for (int i = 0; i + 1 < n; ++i) m[i] = (L[sc[i]] + L[sc[i + 1]]) * 0.5f;
    int q = 0;
    for (int i = 0; i + 1 < n; ++i)
        if (x > m[i]) ++q;
    return sc[q];
}

/* Quantize + double-quantize with the given quant type (see oracle_quantize_dq). */
int oracle_quantize_dq_qt(int qt, const uint16_t* W, int64_t N, int64_t K, uint8_t* packed, int8_t* codes,
                          float* scale, float* mean, float* absmax_scratch)
{
    if (N <= 0 || K <= 0 || (K % NF4_BLOCK) != 0) return -1;
    float L[16], m[15];
    int sc[16];
    int n = codebook_of(qt, L, sc);
    if (n == 0) return -3;
    for (int i = 0; i + 1 < n; ++i) m[i] = (L[sc[i]] + L[sc[i + 1]]) * 0.5f;
    int zero_code = -1;
    for (int i = 0; i < n; ++i)
        if (L[sc[i]] == 0.0f) { zero_code = sc[i]; break; }
    int64_t nblocks = N * K / NF4_BLOCK;
    oracle_block_absmax(W, nblocks, absmax_scratch);
    for (int64_t b = 0; b < nblocks; ++b) {
        float c = absmax_scratch[b];
        for (int j = 0; j < NF4_BLOCK; j += 2) {
            int q[2];
            for (int h = 0; h < 2; ++h) {
                if (c == 0.0f) {
                    q[h] = zero_code;
                } else {
                    float x = oracle_bf16_to_f32(W[b * NF4_BLOCK + j + h]) / c;
                    int k = 0;
                    for (int i = 0; i + 1 < n; ++i)
                        if (x > m[i]) ++k;
                    q[h] = sc[k];
                }
            }
            packed[(b * NF4_BLOCK + j) / 2] = (uint8_t)((q[0] << 4) | q[1]);
        }
    }
    oracle_double_quant(absmax_scratch, nblocks, codes, scale, mean);
    return 0;
}

/* W' = bf16_rne(L[q] * c'_b) for the listed rows, with the given quant type
 * (rows = NULL: every row, in order). */
int oracle_dequant_qt(int qt, const uint8_t* packed, const int8_t* codes, const float* scale, const float* mean,
                      int64_t N, int64_t K, const int64_t* rows, int64_t nrows, uint16_t* Wout)
{
    if (N <= 0 || K <= 0 || (K % NF4_BLOCK) != 0) return -1;
    float L[16];
    int sc[16];
    if (codebook_of(qt, L, sc) == 0) return -3;
    if (rows == NULL) nrows = N;
    for (int64_t ri = 0; ri < nrows; ++ri) {
        int64_t n = rows ? rows[ri] : ri;
        if (n < 0 || n >= N) return -2;
        for (int64_t k = 0; k < K; ++k) {
            int64_t e = n * K + k;
            int64_t b = e / NF4_BLOCK;
            int64_t g = b / DQ_GROUP;
            float cp = oracle_block_constant(codes[b], scale[g], mean[g]);
            uint8_t byte = packed[e / 2];
            int q = (e % 2 == 0) ? (byte >> 4) : (byte & 0x0f);
            Wout[ri * K + k] = oracle_f32_to_bf16(L[q] * cp);
        }
    }
    return 0;
}

/* ===========================================================================
 * Dequantize-and-merge ("Qlora Expert", When to Use / Common Pitfalls: a
 * dense model needs dequantize-and-merge, since merging requires
 * dequantization; "QLoRA Implementation Details (2025 Edition)", Step 7:
 * merge for inference).  The dense weight of the trained layer is the
 * dequantized base plus the scaled LoRA product:
 *   W_merged[n, k] = bf16_rne( fmaf(s, d[n, k], w'[n, k]) ),
 *   d[n, k] = sum_j B[n, j] A[j, k]   in fp32, j = 0, 1, ..., r-1, one fmaf
 *             per term starting from 0 (the first term is exact),
 *   w'[n, k] the dequantized weight (bf16, as the forward multiplies with it).
 * A [r, K] and B [N, r] are bf16; rows = NULL merges every row in order.
 * ========================================================================= */
int oracle_dequant_merge(int qt, const uint8_t* packed, const int8_t* codes, const float* scale, const float* mean,
                         int64_t N, int64_t K, const uint16_t* A, const uint16_t* B, int r, float s,
                         const int64_t* rows, int64_t nrows, uint16_t* Wout)
{
    if (r < 1) return -4;
    int rc = oracle_dequant_qt(qt, packed, codes, scale, mean, N, K, rows, nrows, Wout);
    if (rc != 0) return rc;
    if (rows == NULL) nrows = N;
    for (int64_t ri = 0; ri < nrows; ++ri) {
        int64_t n = rows ? rows[ri] : ri;
        for (int64_t k = 0; k < K; ++k) {
            float d = 0.0f;
            for (int j = 0; j < r; ++j)
                d = fmaf(oracle_bf16_to_f32(B[n * r + j]), oracle_bf16_to_f32(A[(int64_t)j * K + k]), d);
            float w = oracle_bf16_to_f32(Wout[ri * K + k]);
            Wout[ri * K + k] = oracle_f32_to_bf16(fmaf(s, d, w));
        }
    }
    return 0;
}

/* ===========================================================================
 * 8-bit AdamW step for the LoRA adapters ("Qlora Expert", Hyperparameter
 * Guidance and Memory Math: paged_adamw_8bit, 8-bit Adam to cut optimizer
 * memory; "QLoRA Implementation Details (2025 Edition)", Step 5: Paged
 * Optimizer).  The paging (unified memory) is driver behaviour and not part
 * of the step.  The pages name the optimizer but give no state encoding.
 * Reading: both moments are stored blockwise like the weights -- blocks of
 * 256 consecutive parameters, one fp32 scale per block, and one 8-bit code
 * per parameter, the code being an FP8 E4M3 number (1 sign, 4 exponent bits
 * with bias 7, 3 mantissa bits, largest finite 448), so that
 *   state value = fl32(e4m3(code) * scale_b),  scale_b = fl32(absmax_b / 448),
 *   code        = e4m3_rne_saturating(fl32(x * inv_b)), inv_b = fl32(448 / absmax_b),
 *                 0 if absmax_b = 0.
 * The update is AdamW with decoupled weight decay, every operation one IEEE
 * fp32 rounding in this order (g, p are bf16 widened exactly):
 *   m  = b1 * m + omb1 * g                 (two products, then the sum)
 *   v  = b2 * v + omb2 * (g * g)
 *   mh = m * rbc1,  vh = v * rbc2
 *   u  = mh / (sqrt(vh) + eps) + wd * p
 *   p  = bf16_rne(p - lr * u)
 * with omb1 = fl32(1 - b1), omb2 = fl32(1 - b2), rbc1 = fl32(1 / (1 - b1^t)),
 * rbc2 = fl32(1 / (1 - b2^t)) computed in double from the fp32 b1, b2 and the
 * step t (the bias corrections and the block scales enter as reciprocals, so
 * that one division and one square root per parameter remain).  The new m, v
 * of a block are then requantized with that block's new absmax.
 * ========================================================================= */
#define ADAM_BLOCK 256
#define E4M3_MAX 448.0f

/* Value of an E4M3 code (the 0x7f / 0xff NaN patterns are never produced). */
float oracle_e4m3_to_f32(uint8_t c)
{
    int s = c >> 7, e = (c >> 3) & 15, m = c & 7;
    double v = (e == 0) ? ldexp((double)m / 8.0, -6) : ldexp(1.0 + (double)m / 8.0, e - 7);
    return (float)(s ? -v : v);
}

/* Nearest E4M3 value of a finite fp32 x, ties to even mantissa, magnitudes
 * above 448 saturating to 448 (no infinities in E4M3). */
uint8_t oracle_f32_to_e4m3(float x)
{
    uint8_t s = (x < 0.0f || (x == 0.0f && signbit(x))) ? 0x80 : 0;
    double a = fabs((double)x);
    if (a >= 448.0) return (uint8_t)(s | 0x7e);                 /* 1.75 * 2^8 */
    int e;
    frexp(a, &e);                                               /* a = f * 2^e, f in [0.5, 1) */
    int ex = e - 1;                                             /* a in [2^ex, 2^(ex+1)) */
    if (ex < -6) ex = -6;                                       /* subnormal range: fixed quantum */
    double quantum = ldexp(1.0, ex - 3);
    double q = a / quantum;                                     /* exact: a power-of-two scaling */
    double r = rint(q);                                         /* ties to even */
    double v = r * quantum;
    if (v >= 448.0) return (uint8_t)(s | 0x7e);
    if (v == 0.0) return s;
    int ve;
    frexp(v, &ve);
    int vex = ve - 1;
    if (vex < -6) {                                             /* subnormal: m * 2^-9 */
        return (uint8_t)(s | (uint8_t)(v / ldexp(1.0, -9)));
    }
    int mant = (int)((v / ldexp(1.0, vex) - 1.0) * 8.0);
    return (uint8_t)(s | (uint8_t)((vex + 7) << 3) | (uint8_t)mant);
}

/* Blockwise quantization of one block of fp32 values into codes + scale. */
static void quant_block8(const float* x, int n, uint8_t* code, float* scale)
{
    float amax = 0.0f;
    for (int i = 0; i < n; ++i)
        if (fabsf(x[i]) > amax) amax = fabsf(x[i]);
    *scale = amax / E4M3_MAX;
    float inv = (amax == 0.0f) ? 0.0f : E4M3_MAX / amax;
    for (int i = 0; i < n; ++i) code[i] = (amax == 0.0f) ? 0 : oracle_f32_to_e4m3(x[i] * inv);
}

/* One AdamW step over n parameters (see the block comment above).  p, g: bf16
 * [n]; m_code, v_code: [n]; m_scale, v_scale: [ceil(n / 256)].  All in-out
 * except g.  Returns 0, or -1 for n <= 0 or step < 1. */
int oracle_adamw8_step(uint16_t* p, const uint16_t* g, int64_t n, uint8_t* m_code, float* m_scale,
                       uint8_t* v_code, float* v_scale, int64_t step, float lr, float b1, float b2, float eps,
                       float wd)
{
    if (n <= 0 || step < 1) return -1;
    const float omb1 = (float)(1.0 - (double)b1), omb2 = (float)(1.0 - (double)b2);
    const float rbc1 = (float)(1.0 / (1.0 - pow((double)b1, (double)step)));
    const float rbc2 = (float)(1.0 / (1.0 - pow((double)b2, (double)step)));
    float mnew[ADAM_BLOCK], vnew[ADAM_BLOCK];
    for (int64_t b0 = 0; b0 < n; b0 += ADAM_BLOCK) {
        int64_t blk = b0 / ADAM_BLOCK;
        int cnt = (int)((n - b0) < ADAM_BLOCK ? (n - b0) : ADAM_BLOCK);
        for (int i = 0; i < cnt; ++i) {
            int64_t e = b0 + i;
            float gf = oracle_bf16_to_f32(g[e]);
            float pf = oracle_bf16_to_f32(p[e]);
            float mo = oracle_e4m3_to_f32(m_code[e]) * m_scale[blk];
            float vo = oracle_e4m3_to_f32(v_code[e]) * v_scale[blk];
            float t1 = b1 * mo, t2 = omb1 * gf;
            float mn = t1 + t2;
            float gg = gf * gf;
            float t3 = b2 * vo, t4 = omb2 * gg;
            float vn = t3 + t4;
            float mh = mn * rbc1, vh = vn * rbc2;
            float den = sqrtf(vh) + eps;
            float u = mh / den;
            float dec = wd * pf;
            u = u + dec;
            float st = lr * u;
            p[e] = oracle_f32_to_bf16(pf - st);
            mnew[i] = mn;
            vnew[i] = vn;
        }
        quant_block8(mnew, cnt, m_code + b0, &m_scale[blk]);
        quant_block8(vnew, cnt, v_code + b0, &v_scale[blk]);
    }
    return 0;
}

/* ===========================================================================
 * LoRA dropout ("Qlora Expert", Implementation Pattern: lora_dropout=0.05;
 * "QLoRA Implementation Details (2025 Edition)", Step 4: lora_dropout=0.1).
 * Reading (the pages give only the rate): dropout on the LoRA branch's input
 * X, the base path unchanged; element (m, k) of X is kept with probability
 * about 1 - p and kept values are scaled by 1 / (1 - p).  The mask comes
 * from the counter-based generator Philox4x64-10 (Salmon, Moraes, Dror and
 * Shaw, "Parallel random numbers: as easy as 1, 2, 3", SC 2011), written
 * here from that definition:
 *   round:  (hi0, lo0) = M0 * c0,  (hi1, lo1) = M1 * c2  (128-bit products)
 *           c = (hi1 ^ c1 ^ k0, lo1, hi0 ^ c3 ^ k1, lo0)
 *   key:    (k0, k1) += (W0, W1) between rounds; 10 rounds.
 * Element e = m K + k uses 16-bit field (e mod 16) of the 256-bit output for
 * counter (e div 16, offset, 0, 0) and key (seed, 0), fields in little-endian
 * order (field 4i + j is bits 16j .. 16j + 15 of output i); it is kept iff
 * field >= t, t = llrint(p * 2^16).
 * ========================================================================= */
static const uint64_t PHILOX_M0 = 0xD2E7470EE14C6C93ull, PHILOX_M1 = 0xCA5A826395121157ull;
static const uint64_t PHILOX_W0 = 0x9E3779B97F4A7C15ull, PHILOX_W1 = 0xBB67AE8584CAA73Bull;

static void mulhilo64(uint64_t a, uint64_t b, uint64_t* hi, uint64_t* lo)
{
    unsigned __int128 p = (unsigned __int128)a * (unsigned __int128)b;
    *hi = (uint64_t)(p >> 64);
    *lo = (uint64_t)p;
}

void oracle_philox4x64(const uint64_t ctr_in[4], const uint64_t key_in[2], uint64_t out[4])
{
    uint64_t c[4] = {ctr_in[0], ctr_in[1], ctr_in[2], ctr_in[3]};
    uint64_t k0 = key_in[0], k1 = key_in[1];
    for (int round = 0; round < 10; ++round) {
        if (round > 0) { k0 += PHILOX_W0; k1 += PHILOX_W1; }
        uint64_t hi0, lo0, hi1, lo1;
        mulhilo64(PHILOX_M0, c[0], &hi0, &lo0);
        mulhilo64(PHILOX_M1, c[2], &hi1, &lo1);
        uint64_t n0 = hi1 ^ c[1] ^ k0, n1 = lo1, n2 = hi0 ^ c[3] ^ k1, n3 = lo0;
        c[0] = n0; c[1] = n1; c[2] = n2; c[3] = n3;
    }
    for (int i = 0; i < 4; ++i) out[i] = c[i];
}

/* Keep mask [M, K] (1 = kept) of the LoRA dropout above. */
int oracle_dropout_mask(uint64_t seed, uint64_t offset, int64_t M, int64_t K, float p, uint8_t* keep)
{
    if (M <= 0 || K <= 0 || !(p >= 0.0f && p < 1.0f)) return -1;
    const uint32_t t = (uint32_t)llrint((double)p * 65536.0);
    const uint64_t key[2] = {seed, 0};
    for (int64_t e16 = 0; e16 * 16 < M * K; ++e16) {
        const uint64_t ctr[4] = {(uint64_t)e16, offset, 0, 0};
        uint64_t o[4];
        oracle_philox4x64(ctr, key, o);
        for (int j = 0; j < 16 && e16 * 16 + j < M * K; ++j) {
            uint32_t field = (uint32_t)((o[j / 4] >> (16 * (j % 4))) & 0xffffu);
            keep[e16 * 16 + j] = (uint8_t)(field >= t);
        }
    }
    return 0;
}
