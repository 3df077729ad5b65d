// quantize_dual.cu -- instantiations of the both-axes quantizer (quant_cols.cuh
// with DUAL): a bf16 tensor quantized along its rows and its columns in one
// cooperative launch; a separate translation unit so that it compiles in
// parallel with the single-axis kernels.
#include "quant_cols.cuh"

namespace fp4 {

cudaError_t launch_both_axes(const QuantArgs& a, const RowOut& ro, int fmt, bool sr_cols, bool sr_rows, int rot_n,
                             cudaStream_t s) {
    return launch_both_axes_impl(a, ro, fmt, sr_cols, sr_rows, rot_n, s);
}

}  // namespace fp4
