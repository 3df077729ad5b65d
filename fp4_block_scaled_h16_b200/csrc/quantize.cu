// quantize.cu -- fused rotate / amax / scale / round / pack quantizer for
// block-scaled FP4 on sm_100a: the dispatcher, and the row-axis kernels for
// bf16 input (f32 input: quantize_rows_f32.cu; column axis: quantize_cols.cu).
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
// and the next pass's loads are in flight while the current one computes.
#include <cuda_runtime.h>
#include <cstdint>

#include "quant_rows.cuh"

namespace fp4 {

extern template cudaError_t launch_rows_quantize<false>(const QuantArgs&, int, bool, int, bool, bool, cudaStream_t);
extern template cudaError_t launch_rows_amax<false>(const QuantArgs&, int, bool, cudaStream_t);
extern template cudaError_t launch_rows_fused<false>(const QuantArgs&, int, bool, int, bool, cudaStream_t);
extern template cudaError_t launch_cols_quantize<true>(const QuantArgs&, int, bool, int, bool, bool, cudaStream_t);
extern template cudaError_t launch_cols_quantize<false>(const QuantArgs&, int, bool, int, bool, bool, cudaStream_t);
extern template cudaError_t launch_cols_amax<true>(const QuantArgs&, int, bool, cudaStream_t);
extern template cudaError_t launch_cols_amax<false>(const QuantArgs&, int, bool, cudaStream_t);
extern template cudaError_t launch_cols_fused<true>(const QuantArgs&, int, bool, int, bool, cudaStream_t);
extern template cudaError_t launch_cols_fused<false>(const QuantArgs&, int, bool, int, bool, cudaStream_t);

namespace {

// multiplier and shift for fast_div by d >= 1: m = floor(2^(32+l)/d) - 2^32 + 1
void set_divisor(QuantArgs& a, uint32_t d) {
    uint32_t l = 0;
    while (l < 32 && (uint64_t(1) << l) < d) ++l;
    const unsigned __int128 num = (unsigned __int128)1 << (32 + l);
    a.div_m = (uint32_t)((uint64_t)(num / d) - (uint64_t(1) << 32) + 1);
    a.div_l = l;
}

int unit_of(int fmt, int rot_n, int64_t K) {
    return (fmt == MXFP4 || rot_n == 32 || K % 32 == 0) ? 32 : 16;
}

}  // namespace

cudaError_t launch_quantize(QuantArgs a, bool bf16, int fmt, bool sr, int rot_n, bool db, int axis,
                            cudaStream_t s) {
    const bool signs = a.sign_mask != 0u;
    if (axis == 0)
        return bf16 ? launch_cols_quantize<true>(a, fmt, sr, rot_n, signs, db, s)
                    : launch_cols_quantize<false>(a, fmt, sr, rot_n, signs, db, s);
    set_divisor(a, (uint32_t)(a.K / unit_of(fmt, rot_n, a.K)));
    return bf16 ? launch_rows_quantize<true>(a, fmt, sr, rot_n, signs, db, s)
                : launch_rows_quantize<false>(a, fmt, sr, rot_n, signs, db, s);
}

cudaError_t launch_quantize_fused(QuantArgs a, bool bf16, int fmt, bool sr, int rot_n, int axis, cudaStream_t s) {
    const bool signs = a.sign_mask != 0u;
    if (axis == 0)
        return bf16 ? launch_cols_fused<true>(a, fmt, sr, rot_n, signs, s)
                    : launch_cols_fused<false>(a, fmt, sr, rot_n, signs, s);
    set_divisor(a, (uint32_t)(a.K / unit_of(fmt, rot_n, a.K)));
    return bf16 ? launch_rows_fused<true>(a, fmt, sr, rot_n, signs, s)
                : launch_rows_fused<false>(a, fmt, sr, rot_n, signs, s);
}

cudaError_t launch_amax(QuantArgs a, bool bf16, int rot_n, int axis, cudaStream_t s) {
    const bool signs = a.sign_mask != 0u;
    if (axis == 0) return bf16 ? launch_cols_amax<true>(a, rot_n, signs, s) : launch_cols_amax<false>(a, rot_n, signs, s);
    set_divisor(a, (uint32_t)(a.K / unit_of(NVFP4, rot_n, a.K)));
    return bf16 ? launch_rows_amax<true>(a, rot_n, signs, s) : launch_rows_amax<false>(a, rot_n, signs, s);
}

}  // namespace fp4
