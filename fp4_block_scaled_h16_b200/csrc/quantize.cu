// quantize.cu -- fused rotate / amax / scale / round / pack quantizer for
// block-scaled FP4 on sm_100a, and the rotated-tensor amax pass.
//
// Method: "Pre-addestramento di Modelli Linguistici di Grandi Dimensioni con
// MXFP4" (Metodologia: MXFP4, H16/H32, random Hadamard, SR); "Ripensare il
// Bias di Shrinkage nel Pretraining di LLM in FP4" (Metodologia 1-2: E2M1
// RTNE, the uniform UFP4 grid, RHT fused with the quantizer, Efficienza);
// "TetraJet-v2" 2.A (NVFP4 16-groups with E4M3 scales, the 128/16 double
// block, SR, 1x16 groups re-aligned for the transposed weight).
//
// Both kernels are HBM-bound streaming kernels: every element is read once
// (twice for NVFP4/UFP4 with an internal amax: the amax pass, then this one)
// and written as half a byte plus its share of a scale byte.
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <cstdint>

#include "fp4_device.cuh"
#include "internal.h"

namespace fp4 {

// -------------------------------------------------------------------- element rounding

// magnitude index of |v| on the E2M1 grid by stochastic rounding with a
// 24-bit threshold: up iff (r >> 8) * 2^-24 < (u - lo) / (hi - lo)
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

// magnitude index k of |v| on the uniform grid k = 0..7 by stochastic rounding
__device__ __forceinline__ uint32_t sr_ufp4(float u, uint32_t r) {
    u = fminf(u, 7.0f);
    const float t = floorf(u);
    const float f = __fsub_rn(u, t);
    const float th = __fmul_rn((float)(r >> 8), 0x1p-24f);
    return (uint32_t)t + (th < f ? 1u : 0u);
}

__device__ __forceinline__ uint32_t rtne_ufp4(float u) {
    return (uint32_t)__float2int_rn(fminf(u, 7.0f));
}

// sign bits of 8 values at bit 4j+3
__device__ __forceinline__ uint32_t sign_nibbles8(const float* v) {
    uint32_t s = 0;
#pragma unroll
    for (int j = 0; j < 8; ++j) s |= (__float_as_uint(v[j]) >> 31) << (4 * j + 3);
    return s;
}

// 8 scaled values -> one 32-bit word of codes (element j in nibble j)
template <int FMT, bool SR>
__device__ __forceinline__ uint32_t encode8(const float* v, const uint32_t* rnd) {
    uint32_t w = 0;
    if (FMT != UFP4 && !SR) {
        // hardware RNE onto E2M1 of |v| (saturating at 6), sign added after
        const uint32_t b0 = cvt_e2m1x2(fabsf(v[0]), fabsf(v[1]));
        const uint32_t b1 = cvt_e2m1x2(fabsf(v[2]), fabsf(v[3]));
        const uint32_t b2 = cvt_e2m1x2(fabsf(v[4]), fabsf(v[5]));
        const uint32_t b3 = cvt_e2m1x2(fabsf(v[6]), fabsf(v[7]));
        w = b0 | (b1 << 8) | (b2 << 16) | (b3 << 24);
    } else {
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            const float u = fabsf(v[j]);
            uint32_t k;
            if (FMT == UFP4) k = SR ? sr_ufp4(u, rnd[j]) : rtne_ufp4(u);
            else             k = sr_e2m1(u, rnd[j]);
            w |= k << (4 * j);
        }
    }
    return w | sign_nibbles8(v);
}

// -------------------------------------------------------------------- loads

template <bool BF16>
struct Loader;

template <>
struct Loader<true> {
    // 8 contiguous bf16 from a 16-byte aligned address
    static __device__ __forceinline__ void load8(const void* base, int64_t off, float* v) {
        const uint4 q = __ldg(reinterpret_cast<const uint4*>(static_cast<const uint16_t*>(base) + off));
        v[0] = bf16_lo(q.x); v[1] = bf16_hi(q.x); v[2] = bf16_lo(q.y); v[3] = bf16_hi(q.y);
        v[4] = bf16_lo(q.z); v[5] = bf16_hi(q.z); v[6] = bf16_lo(q.w); v[7] = bf16_hi(q.w);
    }
    static __device__ __forceinline__ float load1(const void* base, int64_t off) {
        return __uint_as_float((uint32_t)__ldg(static_cast<const unsigned short*>(base) + off) << 16);
    }
};

template <>
struct Loader<false> {
    static __device__ __forceinline__ void load8(const void* base, int64_t off, float* v) {
        const float4* p = reinterpret_cast<const float4*>(static_cast<const float*>(base) + off);
        const float4 a = __ldg(p), b = __ldg(p + 1);
        v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
        v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
    }
    static __device__ __forceinline__ float load1(const void* base, int64_t off) {
        return __ldg(static_cast<const float*>(base) + off);
    }
};

// rotation of one n-block in registers: signs, butterfly, scale by c_n
template <int N>
__device__ __forceinline__ void rotate(float* v, uint32_t sign_mask) {
    float t[N];
#pragma unroll
    for (int j = 0; j < N; ++j)
        t[j] = __uint_as_float(__float_as_uint(v[j]) ^ (((sign_mask >> j) & 1u) << 31));
    butterfly<N>(t);
    const float c = (N == 16) ? 0.25f : __uint_as_float(0x3E3504F3u);  // binary32(1/sqrt(32))
#pragma unroll
    for (int j = 0; j < N; ++j) v[j] = __fmul_rn(t[j], c);
}

__device__ __forceinline__ float absmax(const float* v, int n) {
    float m = 0.0f;
    for (int j = 0; j < n; ++j) m = fmaxf(m, fabsf(v[j]));
    return m;
}

// -------------------------------------------------------------------- block scaling

// MX: e = clamp(floor(log2 m) - 2, -127, 127); returns the scale byte and
// scales v by 2^-e in place (exact).
__device__ __forceinline__ uint32_t mx_scale(float* v, float m) {
    int e = (m > 0.0f) ? ilogbf(m) - 2 : -127;     // ilogbf: exact floor(log2 m)
    e = max(-127, min(127, e));
    // 2^-e in binary32: normal for e <= 126, the subnormal 2^-127 for e = 127
    const float inv = (e <= 126) ? __uint_as_float((uint32_t)(127 - e) << 23)
                                 : __uint_as_float(0x00400000u);
#pragma unroll
    for (int j = 0; j < 32; ++j) v[j] = __fmul_rn(v[j], inv);
    return (uint32_t)(e + 127);
}

// NV / UFP4 16-block: s_b = E4M3((m / Q) / s_ref); v <- v / (s_b * s_ref).
// Returns the scale byte; zero scale leaves v untouched and sets *zero.
template <int FMT>
__device__ __forceinline__ uint32_t nv_scale(float* v, float m, float s_ref, bool* zero) {
    constexpr float Q = (FMT == UFP4) ? 7.0f : 6.0f;
    const float sb = __fdiv_rn(__fdiv_rn(m, Q), s_ref);
    const uint32_t E = cvt_e4m3(sb);
    *zero = (E == 0u);
    if (E == 0u) return 0u;
    const float S = __fmul_rn(e4m3_to_f32(E), s_ref);
    const float y = __frcp_rn(S);
    // fast exact path while S and 1/S are normal, else per-element division
    const bool fast = (S >= 0x1p-125f) && (S <= 0x1p125f);
    if (fast) {
#pragma unroll
        for (int j = 0; j < 16; ++j) v[j] = div_by(v[j], S, y);
    } else {
#pragma unroll
        for (int j = 0; j < 16; ++j) v[j] = __fdiv_rn(v[j], S);
    }
    return E;
}

// amax / (Q * 448); 1 when that is 0 (amax 0, or an amax so small the
// quotient underflows), as for an all-zero block
__device__ __forceinline__ float tensor_scale_of(float amax, int fmt) {
    const float q448 = (fmt == UFP4) ? 3136.0f : 2688.0f;
    const float s = __fdiv_rn(amax, q448);
    return s > 0.0f ? s : 1.0f;
}

// -------------------------------------------------------------------- axis = 1 kernel
//
// A thread owns a unit of U contiguous elements of one line (U = 32 for MXFP4
// or a 32-rotation, else 16); a warp owns 32 consecutive units.  Double-block
// 128-chunks span 128/U adjacent lanes and are reduced with shuffles.

template <bool BF16, int FMT, bool SR, int ROT, bool DB, bool AMAX_ONLY>
__global__ void __launch_bounds__(256)
quant_rows_kernel(const QuantArgs a) {
    constexpr int U = (FMT == MXFP4 || ROT == 32) ? 32 : 16;
    const int64_t units_per_line = a.K / U;
    const int64_t total = a.L * units_per_line;
    const int lane = threadIdx.x & 31;
    const int64_t warp_global = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const int64_t warp_stride = ((int64_t)gridDim.x * blockDim.x) >> 5;

    float s_t = 1.0f;
    if (!AMAX_ONLY && FMT != MXFP4 && !DB) {
        s_t = tensor_scale_of(*a.amax_in, FMT);
        if (blockIdx.x == 0 && threadIdx.x == 0 && a.tensor_scale_out) *a.tensor_scale_out = s_t;
    }
    float tmax = 0.0f;

    for (int64_t wb = warp_global * 32; wb < total; wb += warp_stride * 32) {
        const int64_t u = wb + lane;
        const bool active = u < total;
        const int64_t l = active ? u / units_per_line : 0;
        const int64_t j = active ? u - l * units_per_line : 0;
        const int64_t off = l * a.ld + j * U;

        float v[U];
        if (active) {
#pragma unroll
            for (int q = 0; q < U / 8; ++q) Loader<BF16>::load8(a.x, off + 8 * q, v + 8 * q);
        } else {
#pragma unroll
            for (int q = 0; q < U; ++q) v[q] = 0.0f;
        }
        if (ROT) {
#pragma unroll
            for (int b = 0; b < U / (ROT ? ROT : 16); ++b) rotate<(ROT ? ROT : 16)>(v + b * ROT, a.sign_mask);
        }
        if (AMAX_ONLY) {
            tmax = fmaxf(tmax, absmax(v, U));
            continue;
        }

        // ---- scales
        uint32_t sbytes[U / 16];
        bool zero[U / 16];
        if (FMT == MXFP4) {
            sbytes[0] = mx_scale(v, absmax(v, 32));
            zero[0] = false;
        } else {
            float s_ref = s_t;
            if (DB) {
                // the 128-chunk of this unit spans G = 128/U adjacent lanes
                constexpr int G = 128 / U;
                float m = absmax(v, U);
#pragma unroll
                for (int s = 1; s < G; s <<= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, s));
                s_ref = tensor_scale_of(m, NVFP4);
                if (active && (lane & (G - 1)) == 0)
                    a.outer[l * (a.K / 128) + (j * U) / 128] = s_ref;
            }
#pragma unroll
            for (int b = 0; b < U / 16; ++b)
                sbytes[b] = nv_scale<FMT>(v + 16 * b, absmax(v + 16 * b, 16), s_ref, &zero[b]);
        }
        if (!active) continue;

        // ---- random words for SR: element i = l * cols + j * U + k (axis 1)
        uint32_t rnd[U];
        if (SR) {
            const uint64_t i0 = (uint64_t)l * (uint64_t)a.cols + (uint64_t)(j * U);
#pragma unroll
            for (int q = 0; q < U / 4; ++q) {
                const uint4 w = sr_words((i0 >> 2) + q, a.tensor_id, a.keys);
                rnd[4 * q] = w.x; rnd[4 * q + 1] = w.y; rnd[4 * q + 2] = w.z; rnd[4 * q + 3] = w.w;
            }
        }

        // ---- codes
        uint32_t words[U / 8];
#pragma unroll
        for (int q = 0; q < U / 8; ++q) {
            const bool z = (FMT != MXFP4) && zero[(8 * q) / 16];
            words[q] = z ? sign_nibbles8(v + 8 * q) : encode8<FMT, SR>(v + 8 * q, rnd + 8 * q);
        }
        uint8_t* dst = a.codes + l * (a.K / 2) + j * (U / 2);
        if (U == 16) {
            *reinterpret_cast<uint2*>(dst) = make_uint2(words[0], words[1]);
        } else {
            *reinterpret_cast<uint4*>(dst) = make_uint4(words[0], words[1], words[U == 32 ? 2 : 0],
                                                        words[U == 32 ? 3 : 0]);
        }
        const int64_t blk = (FMT == MXFP4) ? 32 : 16;
#pragma unroll
        for (int b = 0; b < (FMT == MXFP4 ? 1 : U / 16); ++b)
            a.scales[sf_offset(l, (j * U) / blk + b, a.nb4)] = (uint8_t)sbytes[b];
    }

    if (AMAX_ONLY) {
        const uint32_t bits = __reduce_max_sync(0xffffffffu, __float_as_uint(tmax));
        if (lane == 0 && bits) atomicMax(a.amax_out, bits);
    }
}

// -------------------------------------------------------------------- axis = 0 kernel
//
// A CTA of 4 warps stages a tile of 128 rows x 64 columns in shared memory;
// thread (warp w, lane t) then owns columns 2t, 2t+1 over rows 32w..32w+31,
// i.e. one 32-element piece of two output lines.  Output lines are the input
// columns, so the codes of a line piece are one 16-byte store.

constexpr int T0_ROWS = 128, T0_COLS = 64, T0_THREADS = 128;

template <bool BF16, int FMT, bool SR, int ROT, bool DB, bool AMAX_ONLY>
__global__ void __launch_bounds__(T0_THREADS)
quant_cols_kernel(const QuantArgs a) {
    __shared__ __align__(16) float tile[T0_ROWS][T0_COLS + 4];
    __shared__ float chunk_max[4][T0_COLS];
    const int64_t R = a.rows, C = a.cols;
    const int64_t row0 = (int64_t)blockIdx.y * T0_ROWS, col0 = (int64_t)blockIdx.x * T0_COLS;
    const int tid = threadIdx.x, w = tid >> 5, lane = tid & 31;

    float s_t = 1.0f;
    if (!AMAX_ONLY && FMT != MXFP4 && !DB) {
        s_t = tensor_scale_of(*a.amax_in, FMT);
        if (blockIdx.x == 0 && blockIdx.y == 0 && tid == 0 && a.tensor_scale_out) *a.tensor_scale_out = s_t;
    }

    // ---- stage the tile: 8-element chunks, zero outside [R, C)
    for (int q = tid; q < T0_ROWS * (T0_COLS / 8); q += T0_THREADS) {
        const int r = q / (T0_COLS / 8), c8 = (q % (T0_COLS / 8)) * 8;
        const int64_t gr = row0 + r, gc = col0 + c8;
        float v[8];
        if (gr < R && gc + 8 <= C) {
            Loader<BF16>::load8(a.x, gr * a.ld + gc, v);
        } else {
#pragma unroll
            for (int e = 0; e < 8; ++e)
                v[e] = (gr < R && gc + e < C) ? Loader<BF16>::load1(a.x, gr * a.ld + gc + e) : 0.0f;
        }
        *reinterpret_cast<float4*>(&tile[r][c8]) = make_float4(v[0], v[1], v[2], v[3]);
        *reinterpret_cast<float4*>(&tile[r][c8 + 4]) = make_float4(v[4], v[5], v[6], v[7]);
    }
    __syncthreads();

    const int64_t rbase = row0 + 32 * w;            // first row (= K index) of this piece
    const int nvalid = (int)max((int64_t)0, min((int64_t)32, R - rbase));   // 0, 16 or 32
    float v[2][32];
#pragma unroll
    for (int k = 0; k < 32; ++k) {
        const float2 p = *reinterpret_cast<const float2*>(&tile[32 * w + k][2 * lane]);
        v[0][k] = p.x;
        v[1][k] = p.y;
    }

    if (ROT) {
#pragma unroll
        for (int cc = 0; cc < 2; ++cc)
#pragma unroll
            for (int b = 0; b < 32 / (ROT ? ROT : 16); ++b) rotate<(ROT ? ROT : 16)>(v[cc] + b * ROT, a.sign_mask);
    }
    if (AMAX_ONLY) {
        // rows beyond R are zero-filled and rotate to zero; columns beyond C too
        float m = fmaxf(absmax(v[0], 32), absmax(v[1], 32));
        const uint32_t bits = __reduce_max_sync(0xffffffffu, __float_as_uint(m));
        if (lane == 0 && bits) atomicMax(a.amax_out, bits);
        return;
    }

    float s_ref[2] = {s_t, s_t};
    if (DB) {
        // the 128-row chunk is this CTA's tile: reduce the 4 warps' maxima
#pragma unroll
        for (int cc = 0; cc < 2; ++cc) chunk_max[w][2 * lane + cc] = absmax(v[cc], 32);
        __syncthreads();
#pragma unroll
        for (int cc = 0; cc < 2; ++cc) {
            const int c = 2 * lane + cc;
            const float m = fmaxf(fmaxf(chunk_max[0][c], chunk_max[1][c]), fmaxf(chunk_max[2][c], chunk_max[3][c]));
            s_ref[cc] = tensor_scale_of(m, NVFP4);
            if (w == 0 && col0 + c < C) a.outer[(col0 + c) * (a.K / 128) + row0 / 128] = s_ref[cc];
        }
    }
    if (nvalid == 0) return;

    uint32_t sbytes[2][2];
    bool zero[2][2] = {{false, false}, {false, false}};
#pragma unroll
    for (int cc = 0; cc < 2; ++cc) {
        if (FMT == MXFP4) {
            sbytes[cc][0] = mx_scale(v[cc], absmax(v[cc], 32));
        } else {
#pragma unroll
            for (int b = 0; b < 2; ++b)
                sbytes[cc][b] = nv_scale<FMT>(v[cc] + 16 * b, absmax(v[cc] + 16 * b, 16), s_ref[cc], &zero[cc][b]);
        }
    }
    const int64_t line0 = col0 + 2 * lane;     // even; this thread's lines are line0, line0 + 1
    uint32_t words[2][4];
#pragma unroll
    for (int q = 0; q < 4; ++q) {
        uint32_t rnd[2][8];
        if (SR) {
            // element (r, line): i = r * C + line.  With C % 4 == 0 the two
            // lines of a row share one Philox group (words line0 % 4 and +1).
#pragma unroll
            for (int k = 0; k < 8; ++k) {
                const uint64_t i = (uint64_t)(rbase + 8 * q + k) * (uint64_t)C + (uint64_t)line0;
                const uint4 wds = sr_words(i >> 2, a.tensor_id, a.keys);
                rnd[0][k] = word_of(wds, (int)(i & 3));
                if ((C & 3) == 0) {
                    rnd[1][k] = word_of(wds, (int)(i & 3) + 1);
                } else {
                    const uint64_t i1 = i + 1;
                    rnd[1][k] = word_of(sr_words(i1 >> 2, a.tensor_id, a.keys), (int)(i1 & 3));
                }
            }
        }
#pragma unroll
        for (int cc = 0; cc < 2; ++cc) {
            const bool z = (FMT != MXFP4) && zero[cc][q / 2];
            words[cc][q] = z ? sign_nibbles8(v[cc] + 8 * q) : encode8<FMT, SR>(v[cc] + 8 * q, rnd[cc]);
        }
    }
#pragma unroll
    for (int cc = 0; cc < 2; ++cc) {
        const int64_t line = line0 + cc;
        if (line < C) {
            uint8_t* dst = a.codes + line * (a.K / 2) + rbase / 2;
            if (nvalid == 32) *reinterpret_cast<uint4*>(dst) = make_uint4(words[cc][0], words[cc][1], words[cc][2], words[cc][3]);
            else              *reinterpret_cast<uint2*>(dst) = make_uint2(words[cc][0], words[cc][1]);
            const int64_t blk = (FMT == MXFP4) ? 32 : 16;
            a.scales[sf_offset(line, rbase / blk, a.nb4)] = (uint8_t)sbytes[cc][0];
            if (FMT != MXFP4 && nvalid == 32) a.scales[sf_offset(line, rbase / blk + 1, a.nb4)] = (uint8_t)sbytes[cc][1];
        }
    }
}

// -------------------------------------------------------------------- dispatch

template <bool BF16, int FMT, bool SR, int ROT, bool DB, bool AMAX_ONLY>
static cudaError_t launch_one(const QuantArgs& a, int axis, cudaStream_t s) {
    if (axis == 1) {
        constexpr int U = (FMT == MXFP4 || ROT == 32) ? 32 : 16;
        const int64_t total = a.L * (a.K / U);
        const int64_t warps = (total + 31) / 32;
        int64_t blocks = (warps + 7) / 8;
        const int64_t cap = (int64_t)num_sms() * 8;
        if (blocks > cap) blocks = cap;
        if (blocks < 1) blocks = 1;
        quant_rows_kernel<BF16, FMT, SR, ROT, DB, AMAX_ONLY><<<(unsigned)blocks, 256, 0, s>>>(a);
    } else {
        dim3 grid((unsigned)((a.cols + T0_COLS - 1) / T0_COLS), (unsigned)((a.rows + T0_ROWS - 1) / T0_ROWS));
        quant_cols_kernel<BF16, FMT, SR, ROT, DB, AMAX_ONLY><<<grid, T0_THREADS, 0, s>>>(a);
    }
    return cudaGetLastError();
}

template <bool BF16, int FMT, bool SR, bool DB, bool AMAX_ONLY>
static cudaError_t by_rot(const QuantArgs& a, int rot_n, int axis, cudaStream_t s) {
    switch (rot_n) {
    case 0: return launch_one<BF16, FMT, SR, 0, DB, AMAX_ONLY>(a, axis, s);
    case 16: return launch_one<BF16, FMT, SR, 16, DB, AMAX_ONLY>(a, axis, s);
    default: return launch_one<BF16, FMT, SR, 32, DB, AMAX_ONLY>(a, axis, s);
    }
}

template <bool BF16>
static cudaError_t by_fmt(const QuantArgs& a, int fmt, bool sr, int rot_n, bool db, int axis, cudaStream_t s) {
    if (fmt == MXFP4) return sr ? by_rot<BF16, MXFP4, true, false, false>(a, rot_n, axis, s)
                                : by_rot<BF16, MXFP4, false, false, false>(a, rot_n, axis, s);
    if (fmt == UFP4) return sr ? by_rot<BF16, UFP4, true, false, false>(a, rot_n, axis, s)
                               : by_rot<BF16, UFP4, false, false, false>(a, rot_n, axis, s);
    if (db) return sr ? by_rot<BF16, NVFP4, true, true, false>(a, rot_n, axis, s)
                      : by_rot<BF16, NVFP4, false, true, false>(a, rot_n, axis, s);
    return sr ? by_rot<BF16, NVFP4, true, false, false>(a, rot_n, axis, s)
              : by_rot<BF16, NVFP4, false, false, false>(a, rot_n, axis, s);
}

cudaError_t launch_quantize(const QuantArgs& a, bool bf16, int fmt, bool sr, int rot_n, bool db,
                            int axis, cudaStream_t s) {
    return bf16 ? by_fmt<true>(a, fmt, sr, rot_n, db, axis, s)
                : by_fmt<false>(a, fmt, sr, rot_n, db, axis, s);
}

cudaError_t launch_amax(const QuantArgs& a, bool bf16, int rot_n, int axis, cudaStream_t s) {
    // the amax pass uses the 16-element unit (32 for a 32-rotation)
    return bf16 ? by_rot<true, NVFP4, false, false, true>(a, rot_n, axis, s)
                : by_rot<false, NVFP4, false, false, true>(a, rot_n, axis, s);
}

}  // namespace fp4
