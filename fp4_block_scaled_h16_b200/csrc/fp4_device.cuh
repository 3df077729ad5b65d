// fp4_device.cuh -- device-side building blocks of the quantizer: Philox4x32-10,
// the E2M1 / E4M3 conversions of sm_100a and the tiled scale-factor
// addressing.  Written for the CUDA path only.
#pragma once

#include <cstdint>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

namespace fp4 {

// ---------------------------------------------------------------- formats

enum Format : int { MXFP4 = 0, NVFP4 = 1, UFP4 = 2 };

// ---------------------------------------------------------------- Philox4x32-10
// Salmon, Moraes, Dror, Shaw, "Parallel random numbers: as easy as 1, 2, 3"
// (SC'11).  The ten round keys are the same for every thread, so the host
// computes them once (key + r * Weyl constants) and passes them in.
struct PhiloxKeys {
    uint32_t k0[10];
    uint32_t k1[10];
};

__device__ __forceinline__ uint4 philox4x32_10(uint4 c, const PhiloxKeys& keys) {
#pragma unroll
    for (int r = 0; r < 10; ++r) {
        // each 32 x 32 -> 64-bit product as one wide multiply (both halves at once)
        const uint64_t p0 = (uint64_t)0xD2511F53u * c.x;
        const uint64_t p1 = (uint64_t)0xCD9E8D57u * c.z;
        const uint32_t lo0 = (uint32_t)p0, hi0 = (uint32_t)(p0 >> 32);
        const uint32_t lo1 = (uint32_t)p1, hi1 = (uint32_t)(p1 >> 32);
        c = make_uint4(hi1 ^ c.y ^ keys.k0[r], lo1, hi0 ^ c.w ^ keys.k1[r], lo0);
    }
    return c;
}

// stochastic-rounding word of logical element index i (a multiple-of-4 group
// shares one Philox call: counter = (lo32(i/4), hi32(i/4), tensor_id, 0))
__device__ __forceinline__ uint4 sr_words(uint64_t group, uint32_t tensor_id, const PhiloxKeys& k) {
    return philox4x32_10(make_uint4((uint32_t)group, (uint32_t)(group >> 32), tensor_id, 0u), k);
}

__device__ __forceinline__ uint32_t word_of(const uint4& w, int j) {
    return j == 0 ? w.x : (j == 1 ? w.y : (j == 2 ? w.z : w.w));
}

// ---------------------------------------------------------------- conversions

// two binary32 -> packed e2m1x2 byte, round to nearest even, saturating to +-6.
// `lo` lands in bits 0-3, `hi` in bits 4-7.
__device__ __forceinline__ uint32_t cvt_e2m1x2(float lo, float hi) {
    uint32_t out;
    asm("{\n\t.reg .b8 t;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 t, %1, %2;\n\t"
        "cvt.u32.u8 %0, t;\n\t}"
        : "=r"(out) : "f"(hi), "f"(lo));
    return out;
}

// binary32 -> E4M3 byte, round to nearest even, saturating to 448.
__device__ __forceinline__ uint32_t cvt_e4m3(float s) {
    uint16_t out;
    asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(out) : "f"(0.0f), "f"(s));
    return (uint32_t)(out & 0xFFu);
}

// E4M3 byte -> binary32 (exact)
__device__ __forceinline__ float e4m3_to_f32(uint32_t code) {
    uint32_t h2;
    uint16_t in = (uint16_t)(code & 0xFFu);
    asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(h2) : "h"(in));
    return __half2float(__ushort_as_half((unsigned short)(h2 & 0xFFFFu)));
}

__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

// ---------------------------------------------------------------- tiled scales
// byte offset of (line l, block b) in the tcgen05 scale-factor layout:
// 512-byte atoms of 128 lines x 4 blocks, line l at (l%32)*16 + ((l%128)/32)*4.
__device__ __forceinline__ int64_t sf_offset(int64_t l, int64_t b, int64_t nb4) {
    return (((l >> 7) * nb4 + (b >> 2)) << 9) + ((l & 31) << 4) + (((l >> 5) & 3) << 2) + (b & 3);
}

}  // namespace fp4
