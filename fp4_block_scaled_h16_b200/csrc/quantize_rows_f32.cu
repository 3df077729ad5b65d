// quantize_rows_f32.cu -- the row-axis quantizer kernels for float32 input
// (a separate translation unit so the instantiations compile in parallel).
#include "quant_rows.cuh"

namespace fp4 {

template cudaError_t launch_rows_quantize<false>(const QuantArgs&, int, bool, int, bool, bool, cudaStream_t);
template cudaError_t launch_rows_amax<false>(const QuantArgs&, int, bool, cudaStream_t);
template cudaError_t launch_rows_fused<false>(const QuantArgs&, int, bool, int, bool, cudaStream_t);

}  // namespace fp4
