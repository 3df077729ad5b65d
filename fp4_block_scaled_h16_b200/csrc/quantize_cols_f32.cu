// quantize_cols_f32.cu -- instantiations of the transposed-axis quantizer
// (quant_cols.cuh) for f32 input; a separate translation unit so that the
// input types compile in parallel.
#include "quant_cols.cuh"

namespace fp4 {

template cudaError_t launch_cols_quantize<false>(const QuantArgs&, int, bool, int, bool, bool, cudaStream_t);
template cudaError_t launch_cols_amax<false>(const QuantArgs&, int, bool, cudaStream_t);
template cudaError_t launch_cols_fused<false>(const QuantArgs&, int, bool, int, bool, cudaStream_t);

}  // namespace fp4
