/*
 * qlora_oracle.c -- plain, slow, single-threaded CPU oracle for the QLoRA
 * NF4 storage format.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path may link, load or
 * call this file; only the tests, the smoke check and the benchmark's
 * CPU-baseline leg do.  It shares no code, header or table with the CUDA
 * library: its NF4 levels come from oracle/nf4_levels.inc, which
 * oracle/make_nf4_levels.py writes.
 *
 * Every step follows the pages in their order, written as scalar loops:
 *
 *   - absmax quantiser, scale = absmax / 7, q = round(w / scale), w^ = q*scale
 *     ("QLoRA", learning-llms.pages.dev/topics/qlora: the absmax equation and
 *     the 8-weight worked block that follows it);
 *   - 64-weight blocks with one absmax each, scales double-quantised to
 *     8 bits (same page, the bullet on 64-weight blocks; "QLoRA", infra.bea.ai,
 *     §1 subsection "Double Quantization");
 *   - each weight stored as the index of the nearest of the 16 NF4 levels
 *     (learning-llms page, the sentence before the absmax equation and the
 *     bullet on NF4);
 *   - two 4-bit codes per byte (learning-llms page, the sentence below the
 *     worked-block table: eight weights become eight half-bytes and a scale);
 *   - dequantisation to bf16 for the matmul (learning-llms page, the bullet on
 *     4-bit storage with bf16 compute).
 *
 * Readings taken where the pages are silent (each one is listed with its
 * reason in the design notes):
 *   R1 codebook: the QLoRA paper's normal-quantile construction.
 *   R2 normalisation: x = fp32(w * fp32(1/absmax)), one reciprocal per block.
 *   R3 nearest level: ties go to the lower code.
 *   R4 zero block: absmax below the smallest normal fp32 (0 or subnormal)
 *      encodes every weight of the block as code 7 (the exact zero level).
 *   R5 nibble order: element 2j in the low nibble of byte j, 2j+1 in the high.
 *   R6 second level ("8-bit"): linear unsigned 8-bit, one fp32 scale per
 *      256 consecutive blocks (blocks numbered in row-major order):
 *      s2 = fp32(m/255), q8 = min(255, rint_even(absmax / s2)), where m is
 *      the group's largest absmax; m below the smallest normal fp32 gives
 *      s2 = 0 and q8 = 0.  Codes come from the fp32 absmax, before this step.
 *   R7 dequant: w^ = bf16_rne(fp32(level[code] * fp32(float(q8) * s2)));
 *      without double quantisation, w^ = bf16_rne(fp32(level[code]*absmax)).
 *   R8 non-finite input: rejected (status 2); outputs unspecified.
 */
#include <math.h>
#include <stdint.h>
#include <string.h>
#include <float.h>

#define ORACLE_OK 0
#define ORACLE_INVALID 1
#define ORACLE_NONFINITE 2

#define BLOCK 64
#define GROUP 256

static const float NF4_LEVEL[16] = {
#include "nf4_levels.inc"
};

/* ---------------------------------------------------------------- helpers */

static uint32_t f32_bits(float f) { uint32_t u; memcpy(&u, &f, 4); return u; }
static float bits_f32(uint32_t u) { float f; memcpy(&f, &u, 4); return f; }

/* IEEE round-to-nearest-even from binary32 to bfloat16 (upper 16 bits). */
static uint16_t f32_to_bf16(float f)
{
    uint32_t u = f32_bits(f);
    if ((u & 0x7fffffffu) > 0x7f800000u)          /* NaN stays NaN (quiet) */
        return (uint16_t)((u >> 16) | 0x0040u);
    uint32_t keep_lsb = (u >> 16) & 1u;
    u += 0x7fffu + keep_lsb;                        /* ties to even */
    return (uint16_t)(u >> 16);
}

static float bf16_to_f32(uint16_t h) { return bits_f32((uint32_t)h << 16); }

void oracle_nf4_levels(float out[16])
{
    for (int c = 0; c < 16; ++c) out[c] = NF4_LEVEL[c];
}

void oracle_f32_to_bf16(const float* in, int64_t n, uint16_t* out)
{
    for (int64_t i = 0; i < n; ++i) out[i] = f32_to_bf16(in[i]);
}

void oracle_bf16_to_f32(const uint16_t* in, int64_t n, float* out)
{
    for (int64_t i = 0; i < n; ++i) out[i] = bf16_to_f32(in[i]);
}

/* -------------------------------------------- symmetric absmax integer grid
 * learning-llms page, the absmax equation: scale = absmax / 7, q = round(w / scale), w^ = q * scale, for a
 * 4-bit grid; the page's listing clamps q to [-8, 7].  Generalised to b bits:
 * scale = absmax / (2^(b-1) - 1), q clamped to [-2^(b-1), 2^(b-1) - 1].
 * round() is round-half-to-even (the listing's torch.round).
 * Returns the scale; q and w_hat are written for all n weights.
 */
float oracle_absmax_int_quantize(const float* w, int64_t n, int bits,
                                 int32_t* q, float* w_hat)
{
    float absmax = 0.0f;
    for (int64_t i = 0; i < n; ++i) {
        float a = fabsf(w[i]);
        if (a > absmax) absmax = a;
    }
    const float qmax = (float)((1 << (bits - 1)) - 1);
    const float qmin = -(float)(1 << (bits - 1));
    float scale = absmax / qmax;
    for (int64_t i = 0; i < n; ++i) {
        float r = (scale > 0.0f) ? nearbyintf(w[i] / scale) : 0.0f;
        if (r > qmax) r = qmax;
        if (r < qmin) r = qmin;
        q[i] = (int32_t)r;
        w_hat[i] = (float)q[i] * scale;
    }
    return scale;
}

/* ------------------------------------------------------- NF4 nearest level
 * The index of the nearest of the 16 levels; the distance is taken in
 * binary64, where the difference of two binary32 numbers of this range is
 * exact.  A strict '<' keeps the lower code on an exact tie (reading R3).
 */
int oracle_nf4_nearest(float x)
{
    int best = 0;
    double best_d = fabs((double)x - (double)NF4_LEVEL[0]);
    for (int c = 1; c < 16; ++c) {
        double d = fabs((double)x - (double)NF4_LEVEL[c]);
        if (d < best_d) { best_d = d; best = c; }
    }
    return best;
}

/* ------------------------------------------------------------ storage sizes
 * Bytes of each array of the format for an [rows, cols] matrix:
 *   codes  rows*cols/2      (two 4-bit codes per byte)
 *   absmax rows*cols/64     (uint8 with double quantisation, else fp32 x4)
 *   group  ceil(blocks/256) fp32 scales (double quantisation only)
 */
int oracle_nf4_sizes(int64_t rows, int64_t cols, int double_quant,
                     int64_t* codes_bytes, int64_t* absmax_bytes,
                     int64_t* group_bytes)
{
    if (rows < 1 || cols < 1 || cols % BLOCK != 0) return ORACLE_INVALID;
    int64_t blocks = rows * cols / BLOCK;
    *codes_bytes = rows * cols / 2;
    if (double_quant) {
        *absmax_bytes = blocks;
        *group_bytes = 4 * ((blocks + GROUP - 1) / GROUP);
    } else {
        *absmax_bytes = 4 * blocks;
        *group_bytes = 0;
    }
    return ORACLE_OK;
}

/* --------------------------------------------------------------- quantise
 * w: [rows, cols] binary32 values, row-major (bf16 inputs are upcast by the
 * caller, which is exact).  cols % 64 == 0.  Block b covers the 64
 * consecutive elements w[64b .. 64b+63] of the row-major array, so a block
 * never crosses a row.
 *
 * Outputs (all caller-allocated):
 *   codes      [rows*cols/2]  packed, element 2j -> low nibble of byte j
 *   absmax_f32 [blocks]       the fp32 block absmax (always written)
 *   q8         [blocks]       double_quant only (may be NULL otherwise)
 *   s2         [groups]       double_quant only (may be NULL otherwise)
 */
int oracle_nf4_quantize(const float* w, int64_t rows, int64_t cols,
                        int double_quant, uint8_t* codes, float* absmax_f32,
                        uint8_t* q8, float* s2)
{
    if (rows < 1 || cols < 1 || cols % BLOCK != 0) return ORACLE_INVALID;
    const int64_t blocks = rows * cols / BLOCK;

    /* Step 1: block absmax, the largest magnitude in each 64-weight block
       (learning-llms page, absmax equation; the bullet on 64-weight blocks). */
    for (int64_t b = 0; b < blocks; ++b) {
        float m = 0.0f;
        for (int i = 0; i < BLOCK; ++i) {
            float v = w[b * BLOCK + i];
            if (!isfinite(v)) return ORACLE_NONFINITE;    /* R8 */
            float a = fabsf(v);
            if (a > m) m = a;
        }
        absmax_f32[b] = m;
    }

    /* Step 2: normalise by the block absmax and take the nearest NF4 level,
       then pack two codes per byte. */
    for (int64_t b = 0; b < blocks; ++b) {
        const float m = absmax_f32[b];
        const int zero_block = !(m >= FLT_MIN);           /* R4 */
        const float inv = zero_block ? 0.0f : 1.0f / m;   /* R2 */
        for (int i = 0; i < BLOCK; i += 2) {
            int c[2];
            for (int h = 0; h < 2; ++h) {
                if (zero_block) {
                    c[h] = 7;
                } else {
                    float x = w[b * BLOCK + i + h] * inv;
                    c[h] = oracle_nf4_nearest(x);
                }
            }
            codes[(b * BLOCK + i) / 2] = (uint8_t)(c[0] | (c[1] << 4));   /* R5 */
        }
    }

    /* Step 3: double quantisation of the block scales (R6). */
    if (double_quant) {
        const int64_t groups = (blocks + GROUP - 1) / GROUP;
        for (int64_t g = 0; g < groups; ++g) {
            int64_t b0 = g * GROUP;
            int64_t b1 = b0 + GROUP < blocks ? b0 + GROUP : blocks;
            float m = 0.0f;
            for (int64_t b = b0; b < b1; ++b)
                if (absmax_f32[b] > m) m = absmax_f32[b];
            if (!(m >= FLT_MIN)) {
                s2[g] = 0.0f;
                for (int64_t b = b0; b < b1; ++b) q8[b] = 0;
                continue;
            }
            const float step = m / 255.0f;
            s2[g] = step;
            for (int64_t b = b0; b < b1; ++b) {
                float r = nearbyintf(absmax_f32[b] / step);
                if (r > 255.0f) r = 255.0f;
                q8[b] = (uint8_t)r;
            }
        }
    }
    return ORACLE_OK;
}

/* ------------------------------------------------------------- dequantise
 * out: [rows*cols] bf16 bit patterns.  Reading R7.
 */
int oracle_nf4_dequantize(const uint8_t* codes, const uint8_t* q8,
                          const float* s2, const float* absmax_f32,
                          int64_t rows, int64_t cols, int double_quant,
                          uint16_t* out)
{
    if (rows < 1 || cols < 1 || cols % BLOCK != 0) return ORACLE_INVALID;
    const int64_t n = rows * cols;
    for (int64_t e = 0; e < n; ++e) {
        const int64_t b = e / BLOCK;
        float scale;
        if (double_quant) scale = (float)q8[b] * s2[b / GROUP];
        else scale = absmax_f32[b];
        const uint8_t byte = codes[e / 2];
        const int code = (e % 2 == 0) ? (byte & 0xF) : (byte >> 4);
        out[e] = f32_to_bf16(NF4_LEVEL[code] * scale);
    }
    return ORACLE_OK;
}

/* Quantise a few whole 256-block groups of a larger matrix: the sampled
 * check for matrices too large to quantise on the CPU in a test.  w holds
 * the source elements of groups g0 .. g0+ngroups-1 only (flattened), and the
 * outputs are indexed the same way. */
int oracle_nf4_quantize_groups(const float* w, int64_t nelem, uint8_t* codes,
                               float* absmax_f32, uint8_t* q8, float* s2)
{
    if (nelem < 1 || nelem % BLOCK != 0) return ORACLE_INVALID;
    return oracle_nf4_quantize(w, 1, nelem, 1, codes, absmax_f32, q8, s2);
}
