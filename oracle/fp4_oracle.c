/*
 * fp4_oracle.c -- plain, slow CPU oracle for block-scaled FP4 quantization.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the test suite, the smoke check and the
 * benchmark's CPU-baseline leg may load this library.  It shares no code,
 * header, table or constant with the CUDA implementation.
 *
 * Build: gcc -std=c11 -O2 -ffp-contract=off -fno-fast-math -fPIC -shared
 * (x86-64 SSE arithmetic: every float operation below is one IEEE-754 binary32
 * operation rounded to nearest-even, with subnormals kept).
 *
 * What it computes, and where the pages say so:
 *   - E2M1 elements {0, .5, 1, 1.5, 2, 3, 4, 6} with a sign bit, rounded to
 *     nearest with ties to the even code ("Ripensare il Bias di Shrinkage nel
 *     Pretraining di LLM in FP4", Problematica and Metodologia 1).
 *   - the uniform UFP4 grid k*s, k in [-7, 7] (same page, Metodologia 2,
 *     "La Ricetta UFP4").
 *   - MXFP4: 32-element blocks, power-of-two (E8M0) scale ("Pre-addestramento
 *     di Modelli Linguistici di Grandi Dimensioni con MXFP4", Metodologia).
 *   - NVFP4: 16-element groups with an 8-bit (E4M3) scale and an FP32 tensor
 *     scale; the double-block variant with an FP32 scale per 128-element outer
 *     block ("TetraJet-v2", section 2.A, Structure).
 *   - deterministic H16/H32 and random-sign Hadamard rotations (MXFP4 page,
 *     Metodologia; shrinkage page, Metodologia 2; TetraJet-v2 2.C).
 *   - stochastic rounding with E[round(x)] = x (TetraJet-v2 2.A), drawn from
 *     Philox4x32-10 (Salmon, Moraes, Dror, Shaw, "Parallel random numbers: as
 *     easy as 1, 2, 3", SC'11).
 *
 * Where the pages are silent the plain readings used are:
 *   - E2M1 code = sign<<3 | magnitude index (index into the sorted grid, which
 *     is the s|ee|m bit pattern); element 2j in the low nibble of byte j.
 *   - MX scale exponent e = floor(log2 amax) - 2, clamped to [-127, 127];
 *     an all-zero block gets e = -127.
 *   - NV: s_t = amax/(6*448) (UFP4: amax/(7*448)), s_b = E4M3_RNE_sat((m/Q)/s_t),
 *     v = x / (s_b*s_t); a zero block scale gives signed zeros.  A tensor or
 *     outer scale that comes out 0 (amax 0, or an amax below 2688 * 2^-149
 *     whose quotient underflows) is replaced by 1, as for an all-zero block.
 *   - double block: s_o = amax128/2688 per 128-element chunk of a line,
 *     then the NV rule with s_t replaced by s_o.
 *   - rotation y = c_n * H_n * (d . x) on each aligned n-block of a line, H_n
 *     Sylvester-ordered, butterfly in binary32 with h = 1, 2, 4, ..., n/2;
 *     c_16 = 0.25, c_32 = binary32 nearest to 1/sqrt(32).
 *   - random signs: bit j of word 0 of Philox(key = seed, ctr = (0,0,0,1)),
 *     bit set means -1; one sign vector per seed.
 *   - SR word for logical element i = r*C + c: word (i mod 4) of
 *     Philox(key = seed, ctr = (lo32(i/4), hi32(i/4), tensor_id, 0));
 *     round up iff (word >> 8) * 2^-24 < (u - lo)/(hi - lo).
 */

#include <math.h>
#include <stdint.h>
#include <stddef.h>
#include <string.h>
#include <stdlib.h>

/* numeric codes of the options; the same numbering as the public C ABI so
 * the tests can pass one set of integers to both sides */
enum { ORC_MXFP4 = 0, ORC_NVFP4 = 1, ORC_UFP4 = 2 };
enum { ORC_RTNE = 0, ORC_SR = 1 };
enum { ORC_ROT_NONE = 0, ORC_ROT_H16 = 1, ORC_ROT_H32 = 2, ORC_ROT_RH16 = 3, ORC_ROT_RH32 = 4 };
enum { ORC_IN_F32 = 0, ORC_IN_BF16 = 1 };

/* ------------------------------------------------------------------------ */
/* Philox4x32-10, from the SC'11 description: ten rounds of a Feistel-like   */
/* bijection built from two 32x32->64 multiplies, the key bumped by the Weyl */
/* constants between rounds.                                                  */
/* ------------------------------------------------------------------------ */

void orc_philox4x32_10(const uint32_t ctr_in[4], const uint32_t key_in[2], uint32_t out[4])
{
    const uint32_t M0 = 0xD2511F53u, M1 = 0xCD9E8D57u;   /* round multipliers */
    const uint32_t W0 = 0x9E3779B9u, W1 = 0xBB67AE85u;   /* key schedule (Weyl) */
    uint32_t c0 = ctr_in[0], c1 = ctr_in[1], c2 = ctr_in[2], c3 = ctr_in[3];
    uint32_t k0 = key_in[0], k1 = key_in[1];
    for (int round = 0; round < 10; ++round) {
        if (round > 0) { k0 += W0; k1 += W1; }
        uint64_t p0 = (uint64_t)M0 * (uint64_t)c0;
        uint64_t p1 = (uint64_t)M1 * (uint64_t)c2;
        uint32_t hi0 = (uint32_t)(p0 >> 32), lo0 = (uint32_t)p0;
        uint32_t hi1 = (uint32_t)(p1 >> 32), lo1 = (uint32_t)p1;
        uint32_t n0 = hi1 ^ c1 ^ k0;
        uint32_t n1 = lo1;
        uint32_t n2 = hi0 ^ c3 ^ k1;
        uint32_t n3 = lo0;
        c0 = n0; c1 = n1; c2 = n2; c3 = n3;
    }
    out[0] = c0; out[1] = c1; out[2] = c2; out[3] = c3;
}

/* the 32-bit random word for logical element index i */
static uint32_t sr_word(uint64_t seed, uint32_t tensor_id, uint64_t i)
{
    uint64_t q = i / 4;
    uint32_t ctr[4] = { (uint32_t)q, (uint32_t)(q >> 32), tensor_id, 0u };
    uint32_t key[2] = { (uint32_t)seed, (uint32_t)(seed >> 32) };
    uint32_t out[4];
    orc_philox4x32_10(ctr, key, out);
    return out[i % 4];
}

/* sign vector of the random-sign Hadamard: +1 or -1 for j < n (n <= 32) */
void orc_rht_signs(uint64_t seed, int n, float* d)
{
    uint32_t ctr[4] = { 0u, 0u, 0u, 1u };
    uint32_t key[2] = { (uint32_t)seed, (uint32_t)(seed >> 32) };
    uint32_t out[4];
    orc_philox4x32_10(ctr, key, out);
    for (int j = 0; j < n; ++j)
        d[j] = ((out[0] >> j) & 1u) ? -1.0f : 1.0f;
}

/* ------------------------------------------------------------------------ */
/* Number formats                                                             */
/* ------------------------------------------------------------------------ */

static const float E2M1_GRID[8] = { 0.0f, 0.5f, 1.0f, 1.5f, 2.0f, 3.0f, 4.0f, 6.0f };
static const float UFP4_GRID[8] = { 0.0f, 1.0f, 2.0f, 3.0f, 4.0f, 5.0f, 6.0f, 7.0f };

double orc_e2m1_value(uint8_t code)
{
    double mag = (double)E2M1_GRID[code & 7u];
    return (code & 8u) ? -mag : mag;
}

double orc_ufp4_value(uint8_t code)
{
    double mag = (double)(code & 7u);
    return (code & 8u) ? -mag : mag;
}

/* E4M3 (no infinities, 0x7F / 0xFF are NaN): bias 7, 3 mantissa bits,
 * subnormals m * 2^-9.  Returns the value of an unsigned code 0..0x7E. */
double orc_e4m3_value(uint8_t code)
{
    int e = (code >> 3) & 0xF, m = code & 7;
    double v;
    if (code == 0x7F || code == 0xFF) return NAN;
    if (e == 0) v = ldexp((double)m, -9);
    else        v = ldexp(1.0 + m / 8.0, e - 7);
    return (code & 0x80) ? -v : v;
}

/* nearest non-negative finite E4M3 value to s >= 0, ties to the even code,
 * values above 448 saturate to 448 (0x7E).  Plain search over all codes. */
uint8_t orc_e4m3_encode(float s)
{
    double x = (double)s;
    uint8_t best = 0;
    double best_d = INFINITY;
    if (x >= 448.0) return 0x7E;          /* satfinite: the largest finite value */
    for (int c = 0; c <= 0x7E; ++c) {
        double d = fabs(orc_e4m3_value((uint8_t)c) - x);
        if (d < best_d || (d == best_d && (c & 1) == 0 && (best & 1) != 0)) {
            best_d = d;
            best = (uint8_t)c;
        }
    }
    return best;
}

/* magnitude index of the grid point nearest to u >= 0 (u already clamped to
 * the top level); on an exact tie the even index wins */
static int nearest_even(const float grid[8], float u)
{
    int best = 0;
    double best_d = INFINITY;
    for (int k = 0; k < 8; ++k) {
        double d = fabs((double)u - (double)grid[k]);
        if (d < best_d || (d == best_d && (k & 1) == 0)) {
            best_d = d;
            best = k;
        }
    }
    return best;
}

int orc_e2m1_rtne_index(float u) { return nearest_even(E2M1_GRID, u > 6.0f ? 6.0f : u); }
int orc_ufp4_rtne_index(float u) { return nearest_even(UFP4_GRID, u > 7.0f ? 7.0f : u); }

/* one element: v = x / S (already scaled), sign from x.  Returns the 4-bit code. */
static uint8_t round_element(float v, const float grid[8], int rounding,
                             uint64_t seed, uint32_t tensor_id, uint64_t i)
{
    uint8_t sign = signbit(v) ? 8u : 0u;
    float top = grid[7];
    float u = fabsf(v);
    if (u > top) u = top;
    int k;
    if (rounding == ORC_RTNE) {
        k = nearest_even(grid, u);
    } else {
        int lo = 0;
        while (lo < 7 && grid[lo + 1] <= u) ++lo;      /* largest level <= u */
        if (lo == 7) {
            k = 7;
        } else {
            float f = (u - grid[lo]) / (grid[lo + 1] - grid[lo]);  /* exact */
            uint32_t r = sr_word(seed, tensor_id, i);
            float t = (float)(r >> 8) * 0x1p-24f;
            k = (t < f) ? lo + 1 : lo;
        }
    }
    return (uint8_t)(sign | (uint8_t)k);
}

/* ------------------------------------------------------------------------ */
/* Rotation                                                                   */
/* ------------------------------------------------------------------------ */

static int rotation_size(int rotation)
{
    switch (rotation) {
    case ORC_ROT_H16: case ORC_ROT_RH16: return 16;
    case ORC_ROT_H32: case ORC_ROT_RH32: return 32;
    default: return 0;
    }
}

/* y = c_n * H_n * (d . x) in place, n in {16, 32}; d == NULL means all +1 */
void orc_rotate_block(float* x, int n, const float* d)
{
    if (d)
        for (int j = 0; j < n; ++j) x[j] = x[j] * d[j];
    for (int h = 1; h < n; h <<= 1)
        for (int j = 0; j < n; ++j)
            if ((j & h) == 0) {
                float a = x[j], b = x[j + h];
                x[j] = a + b;
                x[j + h] = a - b;
            }
    float c = (n == 16) ? 0.25f : (float)(1.0 / sqrt(32.0));
    for (int j = 0; j < n; ++j) x[j] = x[j] * c;
}

float orc_c32(void) { return (float)(1.0 / sqrt(32.0)); }

/* ------------------------------------------------------------------------ */
/* Lines: a line is the run of K elements along the quantization axis.       */
/* axis = 1: line l is input row l (K = C); axis = 0: line l is column l     */
/* (K = R).  Element k of line l is input (r, c) with logical index r*C + c. */
/* ------------------------------------------------------------------------ */

static float load_elem(const void* x, int in_dtype, int64_t off)
{
    if (in_dtype == ORC_IN_BF16) {
        uint32_t b = (uint32_t)((const uint16_t*)x)[off] << 16;
        float f;
        memcpy(&f, &b, 4);
        return f;
    }
    return ((const float*)x)[off];
}

/* load line l, widen to binary32 and apply the rotation */
static void load_rotated_line(const void* x, int in_dtype, int64_t R, int64_t C, int64_t ld,
                              int axis, int rotation, uint64_t seed, int64_t l, float* buf)
{
    int64_t K = axis ? C : R;
    for (int64_t k = 0; k < K; ++k) {
        int64_t r = axis ? l : k, c = axis ? k : l;
        buf[k] = load_elem(x, in_dtype, r * ld + c);
    }
    int n = rotation_size(rotation);
    if (n) {
        float d[32];
        int random = (rotation == ORC_ROT_RH16 || rotation == ORC_ROT_RH32);
        if (random) orc_rht_signs(seed, n, d);
        for (int64_t b = 0; b < K; b += n) orc_rotate_block(buf + b, n, random ? d : NULL);
    }
}

/* max |y| over lines [l0, l1) of the rotated tensor */
float orc_tensor_amax(const void* x, int in_dtype, int64_t R, int64_t C, int64_t ld,
                      int axis, int rotation, uint64_t seed, int64_t l0, int64_t l1)
{
    int64_t K = axis ? C : R;
    float* buf = (float*)malloc(sizeof(float) * (size_t)(K > 0 ? K : 1));
    float amax = 0.0f;
    for (int64_t l = l0; l < l1; ++l) {
        load_rotated_line(x, in_dtype, R, C, ld, axis, rotation, seed, l, buf);
        for (int64_t k = 0; k < K; ++k) {
            float a = fabsf(buf[k]);
            if (a > amax) amax = a;
        }
    }
    free(buf);
    return amax;
}

/* floor(log2(m)) for finite m > 0, exact (frexp gives m = f * 2^e, f in [0.5, 1)) */
static int floor_log2(float m)
{
    int e;
    frexpf(m, &e);
    return e - 1;
}

/* the FP32 tensor scale from the tensor amax: amax / (Q * 448), 1 for amax 0 */
float orc_tensor_scale(float amax, int format)
{
    float q448 = (format == ORC_UFP4) ? 7.0f * 448.0f : 6.0f * 448.0f;
    float s = amax / q448;
    return s > 0.0f ? s : 1.0f;    /* amax 0, or so small the quotient underflows */
}

/* Quantize lines [l0, l1).  Outputs are indexed by line:
 *   codes  [lines, K/2]      packed, element 2j in the low nibble of byte j
 *   scales [lines, K/blk]    E8M0 byte (MX) or E4M3 byte (NV, UFP4), row-major
 *   outer  [lines, K/128]    FP32 outer scales (double block only)
 * tensor_scale is s_t (NV/UFP4 without double block), ignored otherwise.
 * Returns 0 on success, nonzero on an unsupported combination. */
int orc_quantize_lines(const void* x, int in_dtype, int64_t R, int64_t C, int64_t ld,
                       int format, int rounding, int rotation, int axis, int double_block,
                       uint64_t seed, uint32_t tensor_id, float tensor_scale,
                       int64_t l0, int64_t l1,
                       uint8_t* codes, uint8_t* scales, float* outer)
{
    int64_t K = axis ? C : R;
    int blk = (format == ORC_MXFP4) ? 32 : 16;
    int n = rotation_size(rotation);
    if (K % blk) return 1;
    if (n && K % n) return 2;
    if (double_block && (format != ORC_NVFP4 || K % 128)) return 3;
    const float* grid = (format == ORC_UFP4) ? UFP4_GRID : E2M1_GRID;
    float Q = (format == ORC_UFP4) ? 7.0f : 6.0f;

    float* buf = (float*)malloc(sizeof(float) * (size_t)(K > 0 ? K : 1));
    uint8_t* code = (uint8_t*)malloc((size_t)(K > 0 ? K : 1));
    for (int64_t l = l0; l < l1; ++l) {
        int64_t lo = l - l0;   /* output line */
        load_rotated_line(x, in_dtype, R, C, ld, axis, rotation, seed, l, buf);

        /* double block: one FP32 outer scale per 128 elements of the line */
        if (double_block)
            for (int64_t o = 0; o < K / 128; ++o) {
                float m128 = 0.0f;
                for (int j = 0; j < 128; ++j) {
                    float a = fabsf(buf[o * 128 + j]);
                    if (a > m128) m128 = a;
                }
                float s_o = m128 / 2688.0f;
                outer[lo * (K / 128) + o] = s_o > 0.0f ? s_o : 1.0f;   /* as for s_t */
            }

        for (int64_t b = 0; b < K / blk; ++b) {
            float* xb = buf + b * blk;
            float m = 0.0f;
            for (int j = 0; j < blk; ++j) {
                float a = fabsf(xb[j]);
                if (a > m) m = a;
            }
            if (format == ORC_MXFP4) {
                int e = (m > 0.0f) ? floor_log2(m) - 2 : -127;
                if (e < -127) e = -127;
                if (e > 127) e = 127;
                scales[lo * (K / blk) + b] = (uint8_t)(e + 127);
                float inv = ldexpf(1.0f, -e);            /* exact power of two */
                for (int j = 0; j < blk; ++j) {
                    int64_t k = b * blk + j;
                    int64_t r = axis ? l : k, c = axis ? k : l;
                    code[k] = round_element(xb[j] * inv, grid, rounding, seed, tensor_id,
                                            (uint64_t)(r * C + c));
                }
            } else {
                float s_ref = double_block ? outer[lo * (K / 128) + (b * blk) / 128] : tensor_scale;
                float sb = (m / Q) / s_ref;
                uint8_t E = orc_e4m3_encode(sb);
                scales[lo * (K / blk) + b] = E;
                float S = (float)orc_e4m3_value(E) * s_ref;
                for (int j = 0; j < blk; ++j) {
                    int64_t k = b * blk + j;
                    int64_t r = axis ? l : k, c = axis ? k : l;
                    if (E == 0) {
                        code[k] = signbit(xb[j]) ? 8u : 0u;
                    } else {
                        code[k] = round_element(xb[j] / S, grid, rounding, seed, tensor_id,
                                                (uint64_t)(r * C + c));
                    }
                }
            }
        }
        for (int64_t j = 0; j < K / 2; ++j)
            codes[lo * (K / 2) + j] = (uint8_t)(code[2 * j] | (code[2 * j + 1] << 4));
    }
    free(code);
    free(buf);
    return 0;
}

/* Dequantize lines [0, lines) exactly into binary64: value = q * s_b * s_ref,
 * with s_b = 2^(byte-127) (MX), E4M3 (NV/UFP4), s_ref = tensor or outer scale. */
int orc_dequantize(const uint8_t* codes, const uint8_t* scales, const float* outer,
                   float tensor_scale, int64_t lines, int64_t K, int format, int double_block,
                   double* out)
{
    int blk = (format == ORC_MXFP4) ? 32 : 16;
    if (K % blk) return 1;
    for (int64_t l = 0; l < lines; ++l)
        for (int64_t k = 0; k < K; ++k) {
            uint8_t byte = codes[l * (K / 2) + k / 2];
            uint8_t c = (k & 1) ? (uint8_t)(byte >> 4) : (uint8_t)(byte & 0xF);
            double q = (format == ORC_UFP4) ? orc_ufp4_value(c) : orc_e2m1_value(c);
            uint8_t sbyte = scales[l * (K / blk) + k / blk];
            double s;
            if (format == ORC_MXFP4) {
                s = ldexp(1.0, (int)sbyte - 127);
            } else {
                double s_ref = double_block ? (double)outer[l * (K / 128) + k / 128]
                                            : (double)tensor_scale;
                s = orc_e4m3_value(sbyte) * s_ref;
            }
            out[l * K + k] = q * s;
        }
    return 0;
}

/* ------------------------------------------------------------------------ */
/* MXNorm ("MXNorm: Reusing MXFP block scales for efficient tensor            */
/* normalisation", 2. Metodologia): the inverse RMS of a row t is estimated   */
/* from the absolute maxima m_tk of its K blocks of B elements,               */
/*     rho_t = c(p, B) * ((1/K) sum_k m_tk^p)^(-1/p),                          */
/* and the normalised row y = x * rho_t is what the MX cast quantizes.        */
/* Readings (the pages give the formula only): m_tk in binary32 (exact); the  */
/* sum in binary64, pairwise in block order (a range's sum is the sum of its  */
/* two halves, split at the largest power of two below its length); the      */
/* mean, the square root (p = 2) and c / g in binary64, each correctly        */
/* rounded, then one rounding to binary32, saturating at the largest finite   */
/* binary32; an all-zero row gets rho = 1.                                    */
/* ------------------------------------------------------------------------ */

/* pairwise binary64 sum of a[0..n) in index order */
static double pairwise_sum(const double* a, int64_t n)
{
    if (n <= 0) return 0.0;
    if (n == 1) return a[0];
    int64_t h = 1;
    while (h * 2 < n) h *= 2;          /* largest power of two below n */
    return pairwise_sum(a, h) + pairwise_sum(a + h, n - h);
}

double orc_pairwise_sum(const double* a, int64_t n) { return pairwise_sum(a, n); }

/* rho of rows [l0, l1) of a row-major [R, ld] input (C columns), blocks of
 * B elements along the row; also each row's max |x| (rowmax).  Returns 0, or
 * nonzero for a bad shape or p. */
int orc_mxnorm_rho(const void* x, int in_dtype, int64_t R, int64_t C, int64_t ld, int B, int p,
                   double c, int64_t l0, int64_t l1, float* rho, float* rowmax)
{
    if (B <= 0 || C % B || (p != 1 && p != 2)) return 1;
    int64_t K = C / B;
    double* mp = (double*)malloc(sizeof(double) * (size_t)(K > 0 ? K : 1));
    for (int64_t l = l0; l < l1; ++l) {
        float rmax = 0.0f;
        for (int64_t k = 0; k < K; ++k) {
            float m = 0.0f;
            for (int j = 0; j < B; ++j) {
                float a = fabsf(load_elem(x, in_dtype, l * ld + k * B + j));
                if (a > m) m = a;
            }
            if (m > rmax) rmax = m;
            mp[k] = (p == 2) ? (double)m * (double)m : (double)m;
        }
        double S = pairwise_sum(mp, K);
        float r;
        if (S == 0.0) {
            r = 1.0f;
        } else {
            double mean = S / (double)K;
            double g = (p == 2) ? sqrt(mean) : mean;
            double q = c / g;
            r = (q >= (double)3.4028234663852886e38) ? 3.4028234663852886e38f : (float)q;
        }
        rho[l - l0] = r;
        rowmax[l - l0] = rmax;
    }
    (void)R;
    free(mp);
    return 0;
}

/* ------------------------------------------------------------------------ */
/* OutControl's high-precision channels ("TetraJet-v2" 2.C: the top p% of    */
/* activation channels, fixed after a calibration window, kept in FP8 for     */
/* the forward and backward passes).  Readings: FP8 is E4M3 under one FP32    */
/* tensor scale s8 = amax / 448 (1 if that is 0); a value x is coded as       */
/* E4M3_rne_satfinite(x / s8), the division one IEEE binary32 operation, the  */
/* sign kept (-0 -> code 0x80).                                               */
/* ------------------------------------------------------------------------ */

/* E4M3 codes of in[i] / s8 (binary32 division), sign in bit 7 */
void orc_fp8_encode_array(const float* in, int64_t n, float s8, uint8_t* out)
{
    for (int64_t i = 0; i < n; ++i) {
        float v = in[i] / s8;
        uint8_t mag = orc_e4m3_encode(fabsf(v));
        out[i] = (uint8_t)((signbit(v) ? 0x80u : 0u) | mag);
    }
}
