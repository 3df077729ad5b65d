// quantize.cu -- fused rotate / amax / scale / round / pack quantizer for
// block-scaled FP4 on sm_100a, row-axis kernel and the dispatcher.
//
// Method: "Pre-addestramento di Modelli Linguistici di Grandi Dimensioni con
// MXFP4" (Metodologia: MXFP4, H16/H32, random Hadamard, SR); "Ripensare il
// Bias di Shrinkage nel Pretraining di LLM in FP4" (Metodologia 1-2: E2M1
// RTNE, the uniform UFP4 grid, RHT fused with the quantizer, Efficienza);
// "TetraJet-v2" 2.A (NVFP4 16-groups with E4M3 scales, the 128/16 double
// block, SR, 1x16 groups re-aligned for the transposed weight).
//
// These are HBM-bound streaming kernels: every element is read once (twice
// for NVFP4/UFP4 with an internal amax: the amax pass, then this one) and
// written as half a byte plus its share of a scale byte.  To stay below the
// issue budget that bandwidth allows (about a dozen instructions per element),
// the butterfly, scaling and division run on packed f32x2 pairs, block maxima
// use the 3-input abs-max, line indices come from a multiply-shift division,
// and each thread keeps about 128 bytes of loads in flight.
#include <cuda_runtime.h>
#include <cstdint>

#include "quant_common.cuh"

namespace fp4 {

// -------------------------------------------------------------------- axis = 1
// A thread owns units of U contiguous elements of one line (U = 32 for MXFP4
// or a 32-rotation, else 16); a warp takes 32*G consecutive units per pass,
// G units per thread, all loads issued before any arithmetic.  Double-block
// 128-chunks span 128/U adjacent lanes and are reduced with shuffles.

template <bool BF16, int FMT, bool SR, int ROT, bool SIGNS, bool DB, bool AMAX_ONLY>
__global__ void __launch_bounds__(256)
quant_rows_kernel(const QuantArgs a) {
    constexpr int U = (FMT == MXFP4 || ROT == 32) ? 32 : 16;
    constexpr int UNIT_BYTES = U * (BF16 ? 2 : 4);
    constexpr int G = (128 / UNIT_BYTES) > 0 ? 128 / UNIT_BYTES : 1;
    const uint32_t upl = (uint32_t)(a.K / U);
    const uint32_t total = (uint32_t)(a.L * (int64_t)upl);
    const uint32_t lane = threadIdx.x & 31u;
    const uint32_t warp = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const uint32_t nwarps = (gridDim.x * blockDim.x) >> 5;

    float s_t = 1.0f;
    if (!AMAX_ONLY && FMT != MXFP4 && !DB) {
        s_t = tensor_scale_of(*a.amax_in, FMT);
        if (blockIdx.x == 0 && threadIdx.x == 0 && a.tensor_scale_out) *a.tensor_scale_out = s_t;
    }
    float tmax = 0.0f;

    for (uint32_t base = warp * 32u * G; base < total; base += nwarps * 32u * G) {
        Raw<BF16, U> raw[G];
        uint32_t ln[G], jn[G];
#pragma unroll
        for (int k = 0; k < G; ++k) {
            const uint32_t u = base + 32u * k + lane;
            ln[k] = fast_div(u, a.div_m, a.div_l);
            jn[k] = u - ln[k] * upl;
            if (u < total) raw[k].load(a.x, (int64_t)ln[k] * a.ld + (int64_t)jn[k] * U);
            else raw[k].zero();
        }
#pragma unroll
        for (int k = 0; k < G; ++k) {
            const bool active = base + 32u * k + lane < total;
            const int64_t l = ln[k], j = jn[k];
            float v[U];
            raw[k].unpack(v);
            rotate_unit<U, ROT, SIGNS>(v, a.sign_mask);
            if (AMAX_ONLY) {
                tmax = absmax_n<U>(v, tmax);
                continue;
            }

            // ---- scales
            uint32_t sbytes[U / 16];
            if (FMT == MXFP4) {
                sbytes[0] = mx_scale32(v, absmax_n<32>(v));
            } else {
                float s_ref = s_t;
                if (DB) {
                    // the 128-chunk of this unit spans 128/U adjacent lanes
                    constexpr int GL = 128 / U;
                    float m = absmax_n<U>(v);
#pragma unroll
                    for (int s = 1; s < GL; s <<= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, s));
                    s_ref = tensor_scale_of(m, NVFP4);
                    if (active && (lane & (GL - 1)) == 0) a.outer[l * (a.K / 128) + (j * U) / 128] = s_ref;
                }
#pragma unroll
                for (int b = 0; b < U / 16; ++b)
                    sbytes[b] = nv_scale16<FMT>(v + 16 * b, absmax_n<16>(v + 16 * b), s_ref);
            }
            if (!active) continue;

            // ---- random words for SR: element i = l * cols + j * U + e
            uint32_t rnd[U];
            if (SR) {
                const uint64_t i0 = (uint64_t)l * (uint64_t)a.cols + (uint64_t)(j * U);
#pragma unroll
                for (int q = 0; q < U / 4; ++q) {
                    const uint4 w = sr_words((i0 >> 2) + q, a.tensor_id, a.keys);
                    rnd[4 * q] = w.x; rnd[4 * q + 1] = w.y; rnd[4 * q + 2] = w.z; rnd[4 * q + 3] = w.w;
                }
            }

            // ---- codes and scale bytes
            uint32_t words[U / 8];
#pragma unroll
            for (int q = 0; q < U / 8; ++q) {
                const bool z = (FMT != MXFP4) && sbytes[(8 * q) / 16] == 0u;
                words[q] = z ? sign_nibbles8(v + 8 * q) : encode8<FMT, SR>(v + 8 * q, rnd + 8 * q);
            }
            uint8_t* dst = a.codes + l * (a.K / 2) + j * (U / 2);
            if (U == 16) *reinterpret_cast<uint2*>(dst) = make_uint2(words[0], words[1]);
            else *reinterpret_cast<uint4*>(dst) = make_uint4(words[0], words[1], words[U / 8 - 2], words[U / 8 - 1]);
            constexpr int BLK = (FMT == MXFP4) ? 32 : 16;
#pragma unroll
            for (int b = 0; b < (FMT == MXFP4 ? 1 : U / 16); ++b)
                a.scales[sf_offset(l, (j * U) / BLK + b, a.nb4)] = (uint8_t)sbytes[b];
        }
    }

    if (AMAX_ONLY) {
        const uint32_t bits = __reduce_max_sync(0xffffffffu, __float_as_uint(tmax));
        if (lane == 0 && bits) atomicMax(a.amax_out, bits);
    }
}

// -------------------------------------------------------------------- dispatch

namespace {

template <bool BF16, int FMT, bool SR, int ROT, bool SIGNS, bool DB, bool AMAX_ONLY>
cudaError_t launch_rows(const QuantArgs& a, cudaStream_t s) {
    constexpr int U = (FMT == MXFP4 || ROT == 32) ? 32 : 16;
    constexpr int UNIT_BYTES = U * (BF16 ? 2 : 4);
    constexpr int G = (128 / UNIT_BYTES) > 0 ? 128 / UNIT_BYTES : 1;
    const int64_t total = a.L * (a.K / U);
    const int64_t warps = (total + 32 * G - 1) / (32 * G);
    int64_t blocks = (warps + 7) / 8;
    const int64_t cap = (int64_t)num_sms() * 4;
    if (blocks > cap) blocks = cap;
    if (blocks < 1) blocks = 1;
    quant_rows_kernel<BF16, FMT, SR, ROT, SIGNS, DB, AMAX_ONLY><<<(unsigned)blocks, 256, 0, s>>>(a);
    return cudaGetLastError();
}

template <bool BF16, int FMT, bool SR, bool DB, bool AMAX_ONLY>
cudaError_t rows_by_rot(const QuantArgs& a, int rot_n, bool signs, cudaStream_t s) {
    if (rot_n == 0) return launch_rows<BF16, FMT, SR, 0, false, DB, AMAX_ONLY>(a, s);
    if (rot_n == 16) return signs ? launch_rows<BF16, FMT, SR, 16, true, DB, AMAX_ONLY>(a, s)
                                  : launch_rows<BF16, FMT, SR, 16, false, DB, AMAX_ONLY>(a, s);
    return signs ? launch_rows<BF16, FMT, SR, 32, true, DB, AMAX_ONLY>(a, s)
                 : launch_rows<BF16, FMT, SR, 32, false, DB, AMAX_ONLY>(a, s);
}

template <bool BF16>
cudaError_t rows_by_fmt(const QuantArgs& a, int fmt, bool sr, int rot_n, bool signs, bool db, cudaStream_t s) {
    if (fmt == MXFP4) return sr ? rows_by_rot<BF16, MXFP4, true, false, false>(a, rot_n, signs, s)
                                : rows_by_rot<BF16, MXFP4, false, false, false>(a, rot_n, signs, s);
    if (fmt == UFP4) return sr ? rows_by_rot<BF16, UFP4, true, false, false>(a, rot_n, signs, s)
                               : rows_by_rot<BF16, UFP4, false, false, false>(a, rot_n, signs, s);
    if (db) return sr ? rows_by_rot<BF16, NVFP4, true, true, false>(a, rot_n, signs, s)
                      : rows_by_rot<BF16, NVFP4, false, true, false>(a, rot_n, signs, s);
    return sr ? rows_by_rot<BF16, NVFP4, true, false, false>(a, rot_n, signs, s)
              : rows_by_rot<BF16, NVFP4, false, false, false>(a, rot_n, signs, s);
}

// multiplier and shift for fast_div by d >= 1: m = floor(2^(32+l)/d) - 2^32 + 1
void set_divisor(QuantArgs& a, uint32_t d) {
    uint32_t l = 0;
    while (l < 32 && (uint64_t(1) << l) < d) ++l;
    const unsigned __int128 num = (unsigned __int128)1 << (32 + l);
    a.div_m = (uint32_t)((uint64_t)(num / d) - (uint64_t(1) << 32) + 1);
    a.div_l = l;
}

}  // namespace

cudaError_t launch_quantize(QuantArgs a, bool bf16, int fmt, bool sr, int rot_n, bool db, int axis,
                            cudaStream_t s) {
    const bool signs = a.sign_mask != 0u;
    if (axis == 0) return launch_quantize_cols(a, bf16, fmt, sr, rot_n, signs, db, s);
    const int U = (fmt == MXFP4 || rot_n == 32) ? 32 : 16;
    set_divisor(a, (uint32_t)(a.K / U));
    return bf16 ? rows_by_fmt<true>(a, fmt, sr, rot_n, signs, db, s)
                : rows_by_fmt<false>(a, fmt, sr, rot_n, signs, db, s);
}

cudaError_t launch_amax(QuantArgs a, bool bf16, int rot_n, int axis, cudaStream_t s) {
    const bool signs = a.sign_mask != 0u;
    if (axis == 0) return launch_amax_cols(a, bf16, rot_n, signs, s);
    // the amax pass uses the 16-element unit (32 for a 32-rotation)
    set_divisor(a, (uint32_t)(a.K / (rot_n == 32 ? 32 : 16)));
    return bf16 ? rows_by_rot<true, NVFP4, false, false, true>(a, rot_n, signs, s)
                : rows_by_rot<false, NVFP4, false, false, true>(a, rot_n, signs, s);
}

}  // namespace fp4
