// outctl.cu -- OutControl's outlier channels ("TetraJet-v2" 2.C): the top p%
// of the activation channels, chosen once in a calibration window, are kept
// in FP8 for the forward and backward passes while the rest of the tensor is
// FP4.  This file holds the pieces besides the FP4 quantizer (which skips the
// channels through its channel mask) and the split GEMM (gemm_outctl.cu):
//   - the calibration statistic, the per-channel amax max_r |x[r, c]|;
//   - the channel mask (one bit per column) built from the channel list;
//   - the FP8 part: x[:, channels] gathered into [rows, k8] E4M3 codes under
//     one FP32 tensor scale s8 = amax / 448 (1 if that is 0), each code
//     E4M3_rne_satfinite(RN(x / s8)) with the sign kept, columns past the
//     channel count zero; an amax pass and a quantize pass.
// A channel index outside [0, cols) is skipped (its FP8 column reads 0) and
// reported through the device error word as FP4_ERR_INVALID_ARG.
#include <cuda_runtime.h>
#include <cstdint>

#include "internal.h"
#include "fp4_device.cuh"

namespace fp4 {

namespace {

constexpr int OC_THREADS = 256;
constexpr unsigned int ERR_INVALID_ARG = 1u;

__device__ __forceinline__ float load_as_f32(const void* x, bool bf16, int64_t off) {
    if (bf16) return __uint_as_float((uint32_t)__ldg(static_cast<const unsigned short*>(x) + off) << 16);
    return __ldg(static_cast<const float*>(x) + off);
}

// max over rows of |x[r, c]|, 8 columns per thread, a slab of rows per CTA
// row; atomicMax on the binary32 bits (>= 0) of out[] (zeroed by the caller)
__global__ void __launch_bounds__(OC_THREADS)
channel_amax_kernel(const void* __restrict__ x, bool bf16, int64_t rows, int64_t cols, int64_t ld, int64_t rows_per,
                    unsigned int* __restrict__ out) {
    const int64_t c0 = ((int64_t)blockIdx.x * OC_THREADS + threadIdx.x) * 8;
    if (c0 >= cols) return;
    const int64_t r0 = (int64_t)blockIdx.y * rows_per;
    const int64_t r1 = min(rows, r0 + rows_per);
    float m[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
    const int nc = (int)min((int64_t)8, cols - c0);
    for (int64_t r = r0; r < r1; ++r) {
#pragma unroll
        for (int e = 0; e < 8; ++e)
            if (e < nc) m[e] = fmaxf(m[e], fabsf(load_as_f32(x, bf16, r * ld + c0 + e)));
    }
#pragma unroll
    for (int e = 0; e < 8; ++e)
        if (e < nc && __float_as_uint(m[e])) atomicMax(out + c0 + e, __float_as_uint(m[e]));
}

__global__ void build_mask_kernel(const int32_t* __restrict__ ch, int64_t n, int64_t cols, uint32_t* __restrict__ mask,
                                  unsigned int* err) {
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += (int64_t)gridDim.x * blockDim.x) {
        const int32_t c = ch[i];
        if (c < 0 || c >= cols) {
            atomicExch(err, ERR_INVALID_ARG);
            continue;
        }
        atomicOr(mask + (c >> 5), 1u << (c & 31));
    }
}

// FP8 pass 1: amax of the gathered channels.  Rows are spread over the CTAs
// (grid-stride) and a row's channels over the threads, so a thread reads the
// channel list once per row from L1 and forms one 64-bit row offset per row.
__global__ void __launch_bounds__(OC_THREADS)
fp8_amax_kernel(const void* __restrict__ x, bool bf16, int64_t rows, int64_t cols, int64_t ld,
                const int32_t* __restrict__ ch, int64_t n, unsigned int* __restrict__ amax) {
    float m = 0.0f;
    for (int64_t r = blockIdx.x; r < rows; r += gridDim.x) {
        const int64_t base = r * ld;
        for (int64_t j = threadIdx.x; j < n; j += OC_THREADS) {
            const int32_t c = __ldg(ch + j);
            if (c >= 0 && c < cols) m = fmaxf(m, fabsf(load_as_f32(x, bf16, base + c)));
        }
    }
    const uint32_t b = __reduce_max_sync(0xffffffffu, __float_as_uint(m));
    if ((threadIdx.x & 31) == 0 && b) atomicMax(amax, b);
}

// FP8 pass 2: the codes of [rows, k8] (zero past n) and the tensor scale; two
// codes per thread step (one e4m3x2 conversion), k8 even
__global__ void __launch_bounds__(OC_THREADS)
fp8_quantize_kernel(const void* __restrict__ x, bool bf16, int64_t rows, int64_t cols, int64_t ld,
                    const int32_t* __restrict__ ch, int64_t n, int64_t k8, const float* __restrict__ amax,
                    uint8_t* __restrict__ codes, float* __restrict__ scale_out) {
    float s8 = __fdiv_rn(*amax, 448.0f);
    if (!(s8 > 0.0f)) s8 = 1.0f;
    if (blockIdx.x == 0 && threadIdx.x == 0) *scale_out = s8;
    for (int64_t r = blockIdx.x; r < rows; r += gridDim.x) {
        const int64_t base = r * ld;
        for (int64_t j = 2 * threadIdx.x; j < k8; j += 2 * OC_THREADS) {
            float v[2];
#pragma unroll
            for (int e = 0; e < 2; ++e) {
                v[e] = 0.0f;
                if (j + e < n) {
                    const int32_t c = __ldg(ch + j + e);
                    if (c >= 0 && c < cols) v[e] = __fdiv_rn(load_as_f32(x, bf16, base + c), s8);
                }
            }
            uint16_t pk;
            asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(pk) : "f"(v[1]), "f"(v[0]));
            *reinterpret_cast<uint16_t*>(codes + r * k8 + j) = pk;
        }
    }
}

int grid_for(int64_t work, int per_sm) {
    int64_t g = (work + OC_THREADS - 1) / OC_THREADS;
    const int64_t cap = (int64_t)num_sms() * per_sm;
    if (g > cap) g = cap;
    return (int)(g < 1 ? 1 : g);
}

}  // namespace

cudaError_t launch_channel_amax(const void* x, bool bf16, int64_t rows, int64_t cols, int64_t ld, float* out,
                                cudaStream_t s) {
    const int64_t rows_per = 256;
    dim3 grid((unsigned)((cols + 8 * OC_THREADS - 1) / (8 * OC_THREADS)), (unsigned)((rows + rows_per - 1) / rows_per));
    channel_amax_kernel<<<grid, OC_THREADS, 0, s>>>(x, bf16, rows, cols, ld, rows_per,
                                                     reinterpret_cast<unsigned int*>(out));
    return cudaGetLastError();
}

cudaError_t launch_channel_mask(const int32_t* ch, int64_t n, int64_t cols, uint32_t* mask, cudaStream_t s) {
    if (n == 0) return cudaSuccess;
    build_mask_kernel<<<grid_for(n, 1), OC_THREADS, 0, s>>>(ch, n, cols, mask, device_error_word());
    return cudaGetLastError();
}

cudaError_t launch_fp8_gather(const void* x, bool bf16, int64_t rows, int64_t cols, int64_t ld, const int32_t* ch,
                              int64_t n, int64_t k8, unsigned int* amax_word, uint8_t* codes, float* scale,
                              cudaStream_t s) {
    // one CTA per row at a time, at most 8 CTAs per SM
    const int64_t cap = (int64_t)num_sms() * 8;
    const unsigned grid = (unsigned)(rows < cap ? (rows > 0 ? rows : 1) : cap);
    if (n > 0) {
        fp8_amax_kernel<<<grid, OC_THREADS, 0, s>>>(x, bf16, rows, cols, ld, ch, n, amax_word);
        cudaError_t e = cudaGetLastError();
        if (e != cudaSuccess) return e;
    }
    fp8_quantize_kernel<<<grid, OC_THREADS, 0, s>>>(
        x, bf16, rows, cols, ld, ch, n, k8, reinterpret_cast<const float*>(amax_word), codes, scale);
    return cudaGetLastError();
}

}  // namespace fp4
