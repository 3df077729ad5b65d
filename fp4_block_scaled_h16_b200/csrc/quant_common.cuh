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

template <int U, int ROT, bool SIGNS>
__device__ __forceinline__ void rotate_unit(float* v, uint32_t sign_mask) {
    if (ROT) {
#pragma unroll
        for (int b = 0; b < U / (ROT ? ROT : 16); ++b) rotate_block<(ROT ? ROT : 16), SIGNS>(v + b * ROT, sign_mask);
    }
}

// ------------------------------------------------------------------ scales
// MX: e = clamp(floor(log2 m) - 2, -127, 127); v <- v * 2^-e (exact); returns e + 127
__device__ __forceinline__ uint32_t mx_scale32(float* v, float m) {
    int e = (m > 0.0f) ? ilogbf(m) - 2 : -127;
    e = max(-127, min(127, e));
    const float inv = (e <= 126) ? __uint_as_float((uint32_t)(127 - e) << 23) : __uint_as_float(0x00400000u);
    const float2 ii = make_float2(inv, inv);
#pragma unroll
    for (int j = 0; j < 32; j += 2) {
        const float2 r = mul2(make_float2(v[j], v[j + 1]), ii);
        v[j] = r.x;
        v[j + 1] = r.y;
    }
    return (uint32_t)(e + 127);
}

// amax / (Q * 448); 1 when that is 0 (amax 0, or so small the quotient underflows)
__device__ __forceinline__ float tensor_scale_of(float amax, int fmt) {
    const float q448 = (fmt == UFP4) ? 3136.0f : 2688.0f;
    const float s = __fdiv_rn(amax, q448);
    return s > 0.0f ? s : 1.0f;
}

// NV / UFP4 16-block: s_b = E4M3((m / Q) / s_ref); v <- v / (s_b * s_ref).
// Returns the scale byte (0: the block is all signed zeros, v untouched).
template <int FMT>
__device__ __forceinline__ uint32_t nv_scale16(float* v, float m, float s_ref) {
    constexpr float Q = (FMT == UFP4) ? 7.0f : 6.0f;
    const float sb = __fdiv_rn(__fdiv_rn(m, Q), s_ref);
    const uint32_t E = cvt_e4m3(sb);
    if (E == 0u) return 0u;
    const float S = __fmul_rn(e4m3_to_f32(E), s_ref);
    if (S >= 0x1p-125f && S <= 0x1p125f) {
        // q0 = x*y, r = x - S*q0 (exact), q = q0 + r*y: RN(x / S) for this range
        const float y = __frcp_rn(S);
        const float2 yy = make_float2(y, y), ns = make_float2(-S, -S);
#pragma unroll
        for (int j = 0; j < 16; j += 2) {
            const float2 x = make_float2(v[j], v[j + 1]);
            const float2 q0 = mul2(x, yy);
            const float2 r = __ffma2_rn(ns, q0, x);
            const float2 q = __ffma2_rn(r, yy, q0);
            v[j] = q.x;
            v[j + 1] = q.y;
        }
    } else {
#pragma unroll
        for (int j = 0; j < 16; ++j) v[j] = __fdiv_rn(v[j], S);
    }
    return E;
}

// ------------------------------------------------------------------ encoders
__device__ __forceinline__ uint32_t sign_nibbles8(const float* v) {
    uint32_t s = 0;
#pragma unroll
    for (int j = 0; j < 8; ++j) s |= (__float_as_uint(v[j]) >> 31) << (4 * j + 3);
    return s;
}

__device__ __forceinline__ uint32_t sr_e2m1(float u, uint32_t r) {
    u = fminf(u, 6.0f);
    float lo, winv, base;
    if (u < 2.0f) {
        const float t = floorf(__fmul_rn(u, 2.0f));
        base = t; lo = __fmul_rn(t, 0.5f); winv = 2.0f;
    } else if (u < 4.0f) {
        const float t = floorf(u);
        base = __fadd_rn(t, 2.0f); lo = t; winv = 1.0f;
    } else if (u < 6.0f) {
        base = 6.0f; lo = 4.0f; winv = 0.5f;
    } else {
        base = 7.0f; lo = 6.0f; winv = 0.0f;
    }
    const float f = __fmul_rn(__fsub_rn(u, lo), winv);
    const float t = __fmul_rn((float)(r >> 8), 0x1p-24f);
    return (uint32_t)base + (t < f ? 1u : 0u);
}

__device__ __forceinline__ uint32_t sr_ufp4(float u, uint32_t r) {
    u = fminf(u, 7.0f);
    const float t = floorf(u);
    const float f = __fsub_rn(u, t);
    const float th = __fmul_rn((float)(r >> 8), 0x1p-24f);
    return (uint32_t)t + (th < f ? 1u : 0u);
}

// 8 scaled values -> one word of codes, element j in nibble j
template <int FMT, bool SR>
__device__ __forceinline__ uint32_t encode8(const float* v, const uint32_t* rnd) {
    if (FMT != UFP4 && !SR) {
        // hardware RNE onto E2M1, saturating at +-6; a value rounding to zero
        // keeps its sign (code 8), as the method's codes require
        const uint32_t b0 = cvt_e2m1x2(v[0], v[1]);
        const uint32_t b1 = cvt_e2m1x2(v[2], v[3]);
        const uint32_t b2 = cvt_e2m1x2(v[4], v[5]);
        const uint32_t b3 = cvt_e2m1x2(v[6], v[7]);
        return b0 | (b1 << 8) | (b2 << 16) | (b3 << 24);
    }
    uint32_t w = 0;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
        const float u = fabsf(v[j]);
        uint32_t k;
        if (FMT == UFP4) k = SR ? sr_ufp4(u, rnd[j]) : (uint32_t)__float2int_rn(fminf(u, 7.0f));
        else             k = sr_e2m1(u, rnd[j]);
        w |= k << (4 * j);
    }
    return w | sign_nibbles8(v);
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
