// ufp4_split.cu -- the UFP4 operands of fp4_gemm rewritten as sums of two E2M1
// operands, so that the block-scaled FP4 tensor cores can take them.
//
// The uniform grid of "Ripensare il Bias di Shrinkage nel Pretraining di LLM in
// FP4" (Metodologia 2: levels k s, k in [-7, 7]) has levels 5 and 7 that E2M1
// lacks, and no tcgen05 MMA kind reads uniform 4-bit codes under 16-element
// E4M3 scales.  Every level is however the sum of two E2M1 values under the
// same block scale:
//     k    0 1 2 3 4 5 6 7
//     a1   0 1 2 3 4 4 6 6       a2 = k - a1 = 1 for k = 5, 7, else 0
// so A B^T = A1 B1^T + A1 B2^T + A2 B1^T + A2 B2^T, exactly: every product of
// grid values is exact and the FP32 accumulation sees the same terms.  The
// four products are one NVFP4 GEMM over K'' = 4 Kp with
//     A'' = [A1 | A2 | A1 | A2],   B'' = [B1 | B1 | B2 | B2]
// (Kp = K rounded up to 256, the padding zero codes under zero scales), which
// this kernel writes into the caller's workspace: each thread turns 32 codes
// (16 bytes, two 16-element blocks) into the four segments' codes and copies
// the two block scales four times, in the tiled scale layout of the result.
#include <cuda_runtime.h>
#include <cstdint>

#include "internal.h"

namespace fp4 {

namespace {

constexpr int SPLIT_THREADS = 256;

// 8 UFP4 codes (sign << 3 | k) -> the E2M1 codes of a1 and a2, nibble-parallel.
// E2M1 codes of the values: 0 -> 0, 1 -> 2 (0b010), 2 -> 4, 3 -> 5, 4 -> 6, 6 -> 7.
__device__ __forceinline__ void split8(uint32_t w, uint32_t& c1, uint32_t& c2) {
    const uint32_t ones = 0x11111111u;
    const uint32_t b0 = w & ones, b1 = (w >> 1) & ones, b2 = (w >> 2) & ones;
    const uint32_t s = w & 0x88888888u;
    // a1 code: bit0 for k in {3, 6, 7}; bit1 for k in {1, 4, 5, 6, 7}; bit2 for k >= 2
    const uint32_t x0 = b1 & (b0 | b2);
    const uint32_t x1 = b2 | (b0 & ~b1);
    const uint32_t x2 = b2 | b1;
    c1 = x0 | (x1 << 1) | (x2 << 2) | s;
    // a2 = 1 (code 0b010) for k in {5, 7}; the sign only where a2 is not zero
    const uint32_t t = b2 & b0;
    c2 = (t << 1) | (s & (t << 3));
}

struct SplitArgs {
    const uint8_t* codes;       // [L, K/2]
    const uint8_t* scales;      // tiled, nb4 groups of 4 blocks per line
    int64_t L, K, nb4;
    int64_t Kp;                 // K rounded up to 256
    uint8_t* out_codes;         // [L, 4 Kp / 2]
    uint8_t* out_scales;        // tiled, out_nb4 = Kp / 16 groups per line
    int64_t out_nb4;
    uint32_t order;             // bit s: segment s takes part 2 (a2) instead of part 1
};

__global__ void __launch_bounds__(SPLIT_THREADS)
ufp4_split_kernel(const SplitArgs a) {
    const int64_t chunks_per_line = a.Kp / 32;             // 32 elements (16 bytes) per chunk
    const int64_t total = a.L * chunks_per_line;
    for (int64_t u = (int64_t)blockIdx.x * SPLIT_THREADS + threadIdx.x; u < total;
         u += (int64_t)gridDim.x * SPLIT_THREADS) {
        const int64_t l = u / chunks_per_line, ch = u - l * chunks_per_line;
        const int64_t k0 = ch * 32;                        // first element of the chunk
        uint4 p1 = make_uint4(0u, 0u, 0u, 0u), p2 = p1;
        uint32_t s0 = 0u, s1 = 0u;
        if (k0 < a.K) {
            // K % 32 may be 16: the second half of the last chunk is padding
            const bool half = k0 + 32 > a.K;
            const uint8_t* src = a.codes + l * (a.K / 2) + k0 / 2;
            uint4 w;
            if (half) {
                const uint2 h = *reinterpret_cast<const uint2*>(src);
                w = make_uint4(h.x, h.y, 0u, 0u);
            } else {
                w = *reinterpret_cast<const uint4*>(src);
            }
            split8(w.x, p1.x, p2.x);
            split8(w.y, p1.y, p2.y);
            split8(w.z, p1.z, p2.z);
            split8(w.w, p1.w, p2.w);
            const int64_t b = k0 / 16;
            s0 = a.scales[sf_offset(l, b, a.nb4)];
            s1 = half ? 0u : a.scales[sf_offset(l, b + 1, a.nb4)];
        }
#pragma unroll
        for (int s = 0; s < 4; ++s) {
            const uint4 v = ((a.order >> s) & 1u) ? p2 : p1;
            *reinterpret_cast<uint4*>(a.out_codes + l * (2 * a.Kp) + s * (a.Kp / 2) + k0 / 2) = v;
            const int64_t ob = s * (a.Kp / 16) + k0 / 16;
            // blocks 2j and 2j + 1 sit side by side in the tiled layout
            *reinterpret_cast<uint16_t*>(a.out_scales + sf_offset(l, ob, a.out_nb4)) = (uint16_t)(s0 | (s1 << 8));
        }
    }
}

}  // namespace

size_t ufp4_split_bytes(int64_t L, int64_t K) {
    const int64_t Kp = (K + 255) / 256 * 256;
    const size_t codes = (size_t)L * (size_t)(2 * Kp);
    const size_t scales = (size_t)((L + 127) / 128 * 128) * (size_t)(4 * Kp / 16);
    return (codes + 1023) / 1024 * 1024 + (scales + 1023) / 1024 * 1024;
}

cudaError_t launch_ufp4_split(const uint8_t* codes, const uint8_t* scales, int64_t L, int64_t K, uint8_t* out,
                              bool b_operand, cudaStream_t s) {
    SplitArgs a{};
    a.codes = codes;
    a.scales = scales;
    a.L = L;
    a.K = K;
    a.nb4 = (K / 16 + 3) / 4;
    a.Kp = (K + 255) / 256 * 256;
    a.out_codes = out;
    a.out_scales = out + ((size_t)L * (size_t)(2 * a.Kp) + 1023) / 1024 * 1024;
    a.out_nb4 = a.Kp / 16;                      // 4 Kp / 16 blocks, 4 per group
    a.order = b_operand ? 0xCu : 0xAu;          // A: [1 2 1 2], B: [1 1 2 2]
    const int64_t total = L * (a.Kp / 32);
    int64_t grid = (total + SPLIT_THREADS - 1) / SPLIT_THREADS;
    const int64_t cap = (int64_t)num_sms() * 8;
    if (grid > cap) grid = cap;
    if (grid < 1) grid = 1;
    ufp4_split_kernel<<<(unsigned)grid, SPLIT_THREADS, 0, s>>>(a);
    return cudaGetLastError();
}

}  // namespace fp4
