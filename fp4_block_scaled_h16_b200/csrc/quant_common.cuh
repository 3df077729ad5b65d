// quant_common.cuh -- device code shared by the row-axis and column-axis
// quantizer kernels: loads, the rotation on packed binary32 pairs, block
// scales and the element encoders.
//
// Every floating-point step is one IEEE binary32 operation rounded to nearest
// even, in the fixed order of the method (butterfly stages h = 1, 2, 4, ...),
// so the codes match a scalar reference bit for bit; the packed f32x2
// instructions of sm_100a perform two such operations at once.
#pragma once

#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <cstdint>

#include "fp4_device.cuh"
#include "internal.h"

namespace fp4 {

// ------------------------------------------------------------------ packed math
__device__ __forceinline__ float2 add2(float2 a, float2 b) { return __fadd2_rn(a, b); }
// a - b as a + (-b): the same IEEE result, signed zeros included
__device__ __forceinline__ float2 sub2(float2 a, float2 b) { return __fadd2_rn(a, make_float2(-b.x, -b.y)); }
__device__ __forceinline__ float2 mul2(float2 a, float2 b) { return __fmul2_rn(a, b); }

// max(|a|, |b|, |c|)
__device__ __forceinline__ float amax3(float a, float b, float c) {
    float d;
    asm("max.abs.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
    return d;
}

template <int N>
__device__ __forceinline__ float absmax_n(const float* v, float m = 0.0f) {
#pragma unroll
    for (int j = 0; j + 1 < N; j += 2) m = amax3(m, v[j], v[j + 1]);
    if (N & 1) m = fmaxf(m, fabsf(v[N - 1]));
    return m;
}

// ------------------------------------------------------------------ loads
// Raw 16-byte words of one unit, issued before any use so that several units'
// loads are in flight per thread.
template <bool BF16, int U>
struct Raw {
    static constexpr int WORDS = BF16 ? U / 8 : U / 4;   // uint4 per unit
    uint4 w[WORDS];
    __device__ __forceinline__ void load(const void* base, int64_t off) {
        const uint4* p = BF16 ? reinterpret_cast<const uint4*>(static_cast<const uint16_t*>(base) + off)
                              : reinterpret_cast<const uint4*>(static_cast<const float*>(base) + off);
#pragma unroll
        for (int q = 0; q < WORDS; ++q) w[q] = __ldg(p + q);
    }
    __device__ __forceinline__ void zero() {
#pragma unroll
        for (int q = 0; q < WORDS; ++q) w[q] = make_uint4(0u, 0u, 0u, 0u);
    }
    __device__ __forceinline__ void unpack(float* v) const {
#pragma unroll
        for (int q = 0; q < WORDS; ++q) {
            if (BF16) {
                v[8 * q + 0] = bf16_lo(w[q].x); v[8 * q + 1] = bf16_hi(w[q].x);
                v[8 * q + 2] = bf16_lo(w[q].y); v[8 * q + 3] = bf16_hi(w[q].y);
                v[8 * q + 4] = bf16_lo(w[q].z); v[8 * q + 5] = bf16_hi(w[q].z);
                v[8 * q + 6] = bf16_lo(w[q].w); v[8 * q + 7] = bf16_hi(w[q].w);
            } else {
                v[4 * q + 0] = __uint_as_float(w[q].x); v[4 * q + 1] = __uint_as_float(w[q].y);
                v[4 * q + 2] = __uint_as_float(w[q].z); v[4 * q + 3] = __uint_as_float(w[q].w);
            }
        }
    }
};

// ------------------------------------------------------------------ rotation
// y = c_N * H_N * (d . x) on N contiguous values.  Pairs P[i] = (x[i], x[i+N/2])
// let stages h = 1 .. N/4 run as packed operations on both halves at once;
// the last stage (h = N/2) combines the two halves of each pair.
template <int N, bool SIGNS>
__device__ __forceinline__ void rotate_block(float* v, uint32_t sign_mask) {
    constexpr int H = N / 2;
    float2 p[H];
#pragma unroll
    for (int i = 0; i < H; ++i) {
        float a = v[i], b = v[i + H];
        if (SIGNS) {
            a = __uint_as_float(__float_as_uint(a) ^ (((sign_mask >> i) & 1u) << 31));
            b = __uint_as_float(__float_as_uint(b) ^ (((sign_mask >> (i + H)) & 1u) << 31));
        }
        p[i] = make_float2(a, b);
    }
#pragma unroll
    for (int h = 1; h < H; h <<= 1) {
#pragma unroll
        for (int i = 0; i < H; ++i) {
            if ((i & h) == 0) {
                const float2 a = p[i], b = p[i + h];
                p[i] = add2(a, b);
                p[i + h] = sub2(a, b);
            }
        }
    }
    const float c = (N == 16) ? 0.25f : __uint_as_float(0x3E3504F3u);   // binary32(1/sqrt(32))
    const float2 cc = make_float2(c, c);
#pragma unroll
    for (int i = 0; i < H; ++i) {
        const float a = p[i].x, b = p[i].y;
        const float2 r = mul2(make_float2(__fadd_rn(a, b), __fsub_rn(a, b)), cc);
        v[i] = r.x;
        v[i + H] = r.y;
    }
}

// max |y| of a rotated block without materialising y: max_j |RN(c*y_j)| =
// RN(c * max_j |y_j|) (c > 0 and rounding are monotone), and the last stage's
// pair (a + b, a - b) has max(|RN(a+b)|, |RN(a-b)|) = RN(|a| + |b|).
template <int N, bool SIGNS>
__device__ __forceinline__ float rotated_absmax(const float* v, uint32_t sign_mask, float m) {
    constexpr int H = N / 2;
    float2 p[H];
#pragma unroll
    for (int i = 0; i < H; ++i) {
        float a = v[i], b = v[i + H];
        if (SIGNS) {
            a = __uint_as_float(__float_as_uint(a) ^ (((sign_mask >> i) & 1u) << 31));
            b = __uint_as_float(__float_as_uint(b) ^ (((sign_mask >> (i + H)) & 1u) << 31));
        }
        p[i] = make_float2(a, b);
    }
#pragma unroll
    for (int h = 1; h < H; h <<= 1) {
#pragma unroll
        for (int i = 0; i < H; ++i) {
            if ((i & h) == 0) {
                const float2 a = p[i], b = p[i + h];
                p[i] = add2(a, b);
                p[i + h] = sub2(a, b);
            }
        }
    }
    float t = 0.0f;
#pragma unroll
    for (int i = 0; i + 1 < H; i += 2)
        t = amax3(t, __fadd_rn(fabsf(p[i].x), fabsf(p[i].y)), __fadd_rn(fabsf(p[i + 1].x), fabsf(p[i + 1].y)));
    const float c = (N == 16) ? 0.25f : __uint_as_float(0x3E3504F3u);
    return fmaxf(m, __fmul_rn(t, c));
}

template <int U, int ROT, bool SIGNS>
__device__ __forceinline__ float unit_rotated_absmax(const float* v, uint32_t sign_mask, float m) {
    if (ROT == 0) {
        m = absmax_n<U>(v, m);
    } else {
#pragma unroll
        for (int b = 0; b < U / (ROT ? ROT : 16); ++b) m = rotated_absmax<(ROT ? ROT : 16), SIGNS>(v + b * ROT, sign_mask, m);
    }
    return m;
}

template <int U, int ROT, bool SIGNS>
__device__ __forceinline__ void rotate_unit(float* v, uint32_t sign_mask) {
    if (ROT) {
#pragma unroll
        for (int b = 0; b < U / (ROT ? ROT : 16); ++b) rotate_block<(ROT ? ROT : 16), SIGNS>(v + b * ROT, sign_mask);
    }
}

// ------------------------------------------------------------------ scales
// Pair layout of a unit: packed operations act on (v[j], v[j + PS]), with
// PS = 8 under a 16-rotation (the rotation's own pairs) and U/2 otherwise.
template <int U, int ROT>
struct PairLayout {
    static constexpr int PS = (ROT == 16 || U == 16) ? 8 : U / 2;
    static constexpr int N = U / 2;                       // pairs per unit
    static __device__ __forceinline__ int lo(int p) { return PS == 8 ? (p & 7) + ((p >> 3) << 4) : p; }
};

// MX: e = clamp(floor(log2 m) - 2, -127, 127); v <- v * 2^-e (exact); returns e + 127
template <int ROT>
__device__ __forceinline__ uint32_t mx_scale32(float* v, float m) {
    using PL = PairLayout<32, ROT>;
    int e = (m > 0.0f) ? ilogbf(m) - 2 : -127;
    e = max(-127, min(127, e));
    const float inv = (e <= 126) ? __uint_as_float((uint32_t)(127 - e) << 23) : __uint_as_float(0x00400000u);
    const float2 ii = make_float2(inv, inv);
#pragma unroll
    for (int p = 0; p < PL::N; ++p) {
        const int j = PL::lo(p);
        const float2 r = mul2(make_float2(v[j], v[j + PL::PS]), ii);
        v[j] = r.x;
        v[j + PL::PS] = r.y;
    }
    return (uint32_t)(e + 127);
}

// amax / (Q * 448); 1 when that is 0 (amax 0, or so small the quotient underflows)
__device__ __forceinline__ float tensor_scale_of(float amax, int fmt) {
    const float q448 = (fmt == UFP4) ? 3136.0f : 2688.0f;
    const float s = __fdiv_rn(amax, q448);
    return s > 0.0f ? s : 1.0f;
}

// RN(a / d) from y = RN(1/d) by one correction step: q0 = a*y, r = a - d*q0
// (exact, one fused multiply-add), q = RN(q0 + r*y).  This is Markstein's
// correction of a faithful quotient by the exact remainder (P. Markstein,
// "Computation of elementary functions on the IBM RISC System/6000
// processor", IBM J. Res. Dev. 34(1), 1990; "IA-64 and Elementary
// Functions", 2000, ch. 8): with y the correctly rounded reciprocal and q0
// within an ulp of a/d, q is the correctly rounded quotient, as long as no
// step under- or overflows.  Callers keep a, d, 1/d and the quotient in the
// normal range (the range tests below) and fall back to IEEE division
// otherwise; for d = 6 and d = 7 an exhaustive check over every normal
// a >= 2^-122 agrees with IEEE division.
__device__ __forceinline__ float div_rcp(float a, float d, float y) {
    const float q0 = __fmul_rn(a, y);
    return __fmaf_rn(__fmaf_rn(-d, q0, a), y, q0);
}

// per-tensor (or per-chunk) reference scale with its reciprocal, for the block scale
struct ScaleRef {
    float s, y;        // s_ref and RN(1/s_ref)
    bool fast;         // s_ref in [2^-100, 2^100]: the correction step is exact
};
__device__ __forceinline__ ScaleRef make_ref(float s) {
    ScaleRef r;
    r.s = s;
    r.fast = (s >= 0x1p-100f) && (s <= 0x1p100f);
    r.y = r.fast ? __frcp_rn(s) : 0.0f;
    return r;
}

// s_b = E4M3_rne_satfinite((m / Q) / s_ref), both divisions correctly rounded
template <int FMT>
__device__ __forceinline__ uint32_t block_scale_code(float m, const ScaleRef& ref) {
    constexpr float Q = (FMT == UFP4) ? 7.0f : 6.0f;
    constexpr float YQ = (FMT == UFP4) ? 0x1.24924ap-3f : 0x1.555556p-3f;   // RN(1/7), RN(1/6)
    const float n = (m >= 0x1p-122f) ? div_rcp(m, Q, YQ) : __fdiv_rn(m, Q);
    float sb;
    if (ref.fast && n >= 0x1p-100f && __fmul_rn(n, ref.y) < 0x1p100f) sb = div_rcp(n, ref.s, ref.y);
    else sb = __fdiv_rn(n, ref.s);
    return cvt_e4m3(sb);
}

// the codes of NB blocks with maxima m[]: one test for the whole unit decides
// whether every division is in the range where the reciprocal-and-correction
// form is exact (a zero maximum passes: it gives code 0 either way), and the
// common case then runs without branches; otherwise block_scale_code per block
template <int FMT, int NB>
__device__ __forceinline__ void block_scale_codes(const float* m, const ScaleRef& ref, uint32_t* code) {
    constexpr float Q = (FMT == UFP4) ? 7.0f : 6.0f;
    constexpr float YQ = (FMT == UFP4) ? 0x1.24924ap-3f : 0x1.555556p-3f;   // RN(1/7), RN(1/6)
    float n[NB];
    bool fast = ref.fast;
#pragma unroll
    for (int b = 0; b < NB; ++b) {
        n[b] = div_rcp(m[b], Q, YQ);
        const bool in_range = m[b] >= 0x1p-122f && n[b] >= 0x1p-100f && __fmul_rn(n[b], ref.y) < 0x1p100f;
        fast = fast && (m[b] == 0.0f || in_range);
    }
    if (fast) {
#pragma unroll
        for (int b = 0; b < NB; ++b) code[b] = cvt_e4m3(div_rcp(n[b], ref.s, ref.y));
    } else {
#pragma unroll
        for (int b = 0; b < NB; ++b) code[b] = block_scale_code<FMT>(m[b], ref);
    }
}

// S = RN(E * s_ref) and y = RN(1/S) for block scale code E; y = 0 marks a
// block that takes the slow path: IEEE division when S or 1/S is outside the
// normal range, and, for E = 0 (S = 0), x * 0, the signed zeros of the codes.
__device__ __forceinline__ float2 scale_pair(uint32_t E, float s_ref) {
    if (E == 0u) return make_float2(0.0f, 0.0f);
    const float S = __fmul_rn(e4m3_to_f32(E), s_ref);
    const bool fast = S >= 0x1p-125f && S <= 0x1p125f;
    return make_float2(S, fast ? __frcp_rn(S) : 0.0f);
}

// per-CTA table of scale_pair(E, s_t) for every E4M3 code of a tensor scale
struct ScaleTable {
    float2 e[128];
    __device__ __forceinline__ void build(float s_t, int tid, int nthreads) {
        for (int c = tid; c < 128; c += nthreads) e[c] = scale_pair((uint32_t)c, s_t);
    }
};

// v <- v / S per element, S and y per 16-block (SY[b] = (S_b, y_b)), on the
// unit's pair layout: q0 = x*y, r = x - S*q0 (exact), q = q0 + r*y = RN(x/S)
// (Markstein's correction, as in div_rcp) while S and 1/S are normal (r is formed as -(S*q0 - x) so that x = -0
// gives -0); IEEE division otherwise; S = y = 0 -> +-0.
template <int U, int ROT>
__device__ __forceinline__ void nv_divide(float* v, const float2* SY) {
    using PL = PairLayout<U, ROT>;
    bool slow = false;
#pragma unroll
    for (int b = 0; b < U / 16; ++b) slow = slow || SY[b].y == 0.0f;
    if (!slow) {
        // every block of the unit on the exact reciprocal path: no branches.
        // The residual is taken as -(S q0 - x): the same value for x != 0, and
        // for x = -0 it keeps q = -0 (x - S q0 would give +0 and lose the
        // sign that the zero code carries)
#pragma unroll
        for (int p = 0; p < PL::N; ++p) {
            const int j = PL::lo(p), k = j + PL::PS;
            const float2 a = SY[j / 16], b = SY[k / 16];
            const float2 x = make_float2(v[j], v[k]);
            const float2 yy = make_float2(a.y, b.y);
            const float2 q0 = mul2(x, yy);
            const float2 rn = __ffma2_rn(make_float2(a.x, b.x), q0, make_float2(-x.x, -x.y));
            const float2 q = __ffma2_rn(make_float2(-rn.x, -rn.y), yy, q0);
            v[j] = q.x;
            v[k] = q.y;
        }
        return;
    }
#pragma unroll
    for (int p = 0; p < PL::N; ++p) {
        const int j = PL::lo(p), k = j + PL::PS;
        const float2 a = SY[j / 16], b = SY[k / 16];
        const bool slow = (a.y == 0.0f) || (b.y == 0.0f);
        if (!slow) {
            const float2 x = make_float2(v[j], v[k]);
            const float2 yy = make_float2(a.y, b.y);
            const float2 q0 = mul2(x, yy);
            const float2 rn = __ffma2_rn(make_float2(a.x, b.x), q0, make_float2(-x.x, -x.y));   // -(x - S q0)
            const float2 q = __ffma2_rn(make_float2(-rn.x, -rn.y), yy, q0);
            v[j] = q.x;
            v[k] = q.y;
        } else {
            v[j] = a.x != 0.0f ? __fdiv_rn(v[j], a.x) : __fmul_rn(v[j], 0.0f);
            v[k] = b.x != 0.0f ? __fdiv_rn(v[k], b.x) : __fmul_rn(v[k], 0.0f);
        }
    }
}

// ------------------------------------------------------------------ encoders

// Stochastic rounding of |v| onto E2M1 as one exact integer carry.  With lo
// the level below u = min(|v|, 6), w the gap above it and t = (r >> 8) * 2^-24,
// "round up iff t < (u - lo) / w" is "(r >> 8) < F", F = ceil(2^24 (u - lo) / w).
// The levels are multiples of w = 0.5 on [0, 2), of 1 on [2, 4) and of 2 on
// [4, 6], so with X = ceil(2^25 u) (exact: 2^25 u is an integer unless u <
// 1/4, and then only the ceiling matters) and s = 0, 1, 2 the binade shift,
// Y = X >> s holds the index of lo within its binade above bit 24 and F in its
// low 24 bits.  Adding 2^24 - 1 - (r >> 8) = (~r) >> 8 carries into bit 24
// exactly when (r >> 8) < F; adding s << 25 turns the binade's first index (0,
// 2, 2) into the code's (0, 4, 6).  Returns the sum: the magnitude index in
// bits 24-26, zeros above (the sum stays below 2^27).
__device__ __forceinline__ uint32_t sr_e2m1_sum(float v, uint32_t r) {
    const float u = fminf(fabsf(v), 6.0f);
    const uint32_t X = __float2uint_ru(__fmul_rn(u, 0x1p25f));
    const uint32_t s = min(X >> 26, 2u);
    return (X >> s) + ((~r) >> 8) + (s << 25);
}

// the same on the uniform grid k = 0..7 (w = 1): X = ceil(2^24 u) holds floor(u)
// above bit 24 and F below it
__device__ __forceinline__ uint32_t sr_ufp4_sum(float v, uint32_t r) {
    const float u = fminf(fabsf(v), 7.0f);
    return __float2uint_ru(__fmul_rn(u, 0x1p24f)) + ((~r) >> 8);
}

// nibble j (0..7, a compile-time constant after unrolling) of a code word from
// such a sum and the sign bit of the value: magnitude bits from bits 24-26 of
// the sum, sign from bit 31 of x
__device__ __forceinline__ uint32_t sr_nibble(uint32_t sum, float x, int j) {
    const uint32_t mag = (j < 7) ? (sum >> (24 - 4 * j)) : (sum << 4);
    return (mag & (7u << (4 * j))) | ((__float_as_uint(x) >> (28 - 4 * j)) & (8u << (4 * j)));
}

// 8 scaled values -> one word of codes, element j in nibble j
template <int FMT, bool SR>
__device__ __forceinline__ uint32_t encode8(const float* v, const uint32_t* rnd) {
    if (FMT != UFP4 && !SR) {
        // hardware RNE onto E2M1, saturating at +-6; a value rounding to zero
        // keeps its sign (code 8), as the method's codes require
        uint32_t w;
        asm("{\n\t.reg .b8 b0, b1, b2, b3;\n\t"
            "cvt.rn.satfinite.e2m1x2.f32 b0, %2, %1;\n\t"
            "cvt.rn.satfinite.e2m1x2.f32 b1, %4, %3;\n\t"
            "cvt.rn.satfinite.e2m1x2.f32 b2, %6, %5;\n\t"
            "cvt.rn.satfinite.e2m1x2.f32 b3, %8, %7;\n\t"
            "mov.b32 %0, {b0, b1, b2, b3};\n\t}"
            : "=r"(w)
            : "f"(v[0]), "f"(v[1]), "f"(v[2]), "f"(v[3]), "f"(v[4]), "f"(v[5]), "f"(v[6]), "f"(v[7]));
        return w;
    }
    uint32_t w = 0;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
        if (FMT == UFP4 && !SR) {
            // magnitude and sign bit (bit 31 of v moved to bit 3 of the nibble)
            const uint32_t k = (uint32_t)__float2int_rn(fminf(fabsf(v[j]), 7.0f));
            w |= (k | ((__float_as_uint(v[j]) >> 28) & 8u)) << (4 * j);
        } else {
            w |= sr_nibble(FMT == UFP4 ? sr_ufp4_sum(v[j], rnd[j]) : sr_e2m1_sum(v[j], rnd[j]), v[j], j);
        }
    }
    return w;
}

// ------------------------------------------------------------------ division by a constant
// q = n / d for n < 2^32 with a host-computed multiplier (Granlund and
// Montgomery, "Division by invariant integers using multiplication", 1994,
// section 4): m = floor(2^(32+l) / d) - 2^32 + 1, l = ceil(log2 d).
__device__ __forceinline__ uint32_t fast_div(uint32_t n, uint32_t m, uint32_t l) {
    const uint32_t t = __umulhi(m, n);
    return (uint32_t)(((uint64_t)t + n) >> l);
}

}  // namespace fp4
