// rotate.cu -- the Hadamard rotation alone, as a separate streaming kernel:
// y = c_n * H_n * (d . x) on every aligned n-block of each row, written back
// in the input's type.  This is the unfused form of the rotation that the
// quantizer otherwise applies in registers ("Ripensare il Bias di Shrinkage
// nel Pretraining di LLM in FP4", Efficienza: a separate RHT kernel before the
// quantizer costs about 1.4-1.6x the quantization alone, the fused one about
// 1.06-1.07x).  Same binary32 arithmetic as the quantizer's rotation; a bf16
// output is the binary32 result rounded to nearest even.
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <cstdint>

#include "quant_common.cuh"

namespace fp4 {

namespace {

constexpr int ROT_THREADS = 256;

// one n-element block per thread per step, grid-stride over the blocks of the
// [rows, cols] input (row pitch ld, output pitch ldy)
template <bool BF16, int N, bool SIGNS>
__global__ void __launch_bounds__(ROT_THREADS)
rotate_rows_kernel(const void* __restrict__ x, void* __restrict__ y, int64_t rows, int64_t cols, int64_t ld,
                   int64_t ldy, uint32_t sign_mask) {
    const int64_t per_row = cols / N;
    const int64_t total = rows * per_row;
    for (int64_t u = (int64_t)blockIdx.x * ROT_THREADS + threadIdx.x; u < total;
         u += (int64_t)gridDim.x * ROT_THREADS) {
        const int64_t r = u / per_row, c = (u - r * per_row) * N;
        float v[N];
        Raw<BF16, N> w;
        w.load(x, r * ld + c);
        w.unpack(v);
        rotate_block<N, SIGNS>(v, sign_mask);
        if (BF16) {
            uint4* dst = reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(y) + r * ldy + c);
#pragma unroll
            for (int q = 0; q < N / 8; ++q) {
                uint32_t pk[4];
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const __nv_bfloat162 h = __floats2bfloat162_rn(v[8 * q + 2 * e], v[8 * q + 2 * e + 1]);
                    pk[e] = *reinterpret_cast<const uint32_t*>(&h);
                }
                dst[q] = make_uint4(pk[0], pk[1], pk[2], pk[3]);
            }
        } else {
            float4* dst = reinterpret_cast<float4*>(static_cast<float*>(y) + r * ldy + c);
#pragma unroll
            for (int q = 0; q < N / 4; ++q) dst[q] = make_float4(v[4 * q], v[4 * q + 1], v[4 * q + 2], v[4 * q + 3]);
        }
    }
}

template <bool BF16, int N, bool SIGNS>
cudaError_t launch_rot(const void* x, void* y, int64_t rows, int64_t cols, int64_t ld, int64_t ldy,
                       uint32_t sign_mask, cudaStream_t s) {
    const int64_t total = rows * (cols / N);
    int64_t grid = (total + ROT_THREADS - 1) / ROT_THREADS;
    const int64_t cap = (int64_t)num_sms() * 8;      // 8 resident CTAs of 256 threads per SM
    if (grid > cap) grid = cap;
    if (grid < 1) grid = 1;
    rotate_rows_kernel<BF16, N, SIGNS><<<(unsigned)grid, ROT_THREADS, 0, s>>>(x, y, rows, cols, ld, ldy, sign_mask);
    return cudaGetLastError();
}

template <bool BF16>
cudaError_t rot_by_n(const void* x, void* y, int64_t rows, int64_t cols, int64_t ld, int64_t ldy, int n,
                     uint32_t sign_mask, cudaStream_t s) {
    if (n == 16) return sign_mask ? launch_rot<BF16, 16, true>(x, y, rows, cols, ld, ldy, sign_mask, s)
                                  : launch_rot<BF16, 16, false>(x, y, rows, cols, ld, ldy, sign_mask, s);
    return sign_mask ? launch_rot<BF16, 32, true>(x, y, rows, cols, ld, ldy, sign_mask, s)
                     : launch_rot<BF16, 32, false>(x, y, rows, cols, ld, ldy, sign_mask, s);
}

}  // namespace

cudaError_t launch_rotate_rows(const void* x, void* y, bool bf16, int64_t rows, int64_t cols, int64_t ld,
                               int64_t ldy, int n, uint32_t sign_mask, cudaStream_t s) {
    return bf16 ? rot_by_n<true>(x, y, rows, cols, ld, ldy, n, sign_mask, s)
                : rot_by_n<false>(x, y, rows, cols, ld, ldy, n, sign_mask, s);
}

}  // namespace fp4
