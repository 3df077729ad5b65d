// quantize_cols_bf16.cu -- instantiations of the transposed-axis quantizer
// (quant_cols.cuh) for bf16 input; a separate translation unit so that the
// input types compile in parallel.
#include "quant_cols.cuh"

namespace fp4 {

template cudaError_t launch_cols_quantize<true>(const QuantArgs&, int, bool, int, bool, bool, cudaStream_t);
template cudaError_t launch_cols_amax<true>(const QuantArgs&, int, bool, cudaStream_t);
template cudaError_t launch_cols_fused<true>(const QuantArgs&, int, bool, int, bool, cudaStream_t);

}  // namespace fp4
