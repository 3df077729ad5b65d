// mxnorm.cu -- MXNorm fused with the FP4 cast ("MXNorm: Reusing MXFP block
// scales for efficient tensor normalisation", 2. Metodologia): the inverse RMS
// of every row is estimated from the absolute maxima m_tk of its K blocks,
// the very maxima the block scales of the cast come from,
//     rho_t = c * ((1/K) sum_k m_tk^p)^(-1/p),    p in {1, 2},
// and the normalised row y = RN(x * rho_t) is quantized along the row in the
// same kernel (the norm's gain is folded into the next layer's weight).
//
// Arithmetic, as the oracle: m_tk in binary32; the sum in binary64, pairwise
// in block order (level by level over adjacent pairs, padded with zeros to a
// power of two, which is the same tree); the mean, the square root and c / g
// correctly rounded in binary64, then rounded once to binary32 and saturated
// at the largest finite binary32; an all-zero row gets rho = 1.  The cast is
// the quantizer's own: MXFP4 with its E8M0 block scale, or NVFP4 / UFP4 with
// the E4M3 block scale under the tensor scale of y's amax, which needs the
// whole tensor: those formats run a statistics pass (rho and the amax of y,
// max_t RN(rowmax_t * rho_t)) and then the quantize pass, which reads rho back.
//
// bf16 rows of up to 4096 columns (a multiple of 256) run one warp per row
// (mxnorm_warp_kernel); other rows one CTA of 128
// threads per row at a time (grid-stride over the rows): the row is staged
// in shared memory once, each thread takes blocks tid, tid + 128, ... for the
// maxima and again for the cast.
#include <cuda_runtime.h>
#include <cstdint>

#include "quant_common.cuh"

namespace fp4 {

namespace {

constexpr int MN_THREADS = 128;

struct MxNormArgs {
    const void* x;
    int64_t rows, cols, ld;
    int p;
    double c;
    int K, n2;                 // blocks per row, and K rounded up to a power of two
    uint8_t* codes;
    uint8_t* scales;
    int64_t nb4;
    float* rho;                // [rows]
    float* tensor_scale_out;   // NVFP4 / UFP4
    unsigned int* amax_out;    // statistics pass: atomicMax of the amax of y (binary32 bits)
    const float* amax_in;      // quantize pass: the amax of y
    PhiloxKeys keys;
    uint32_t tensor_id;
};

// PASS 0: MXFP4, rho and the cast in one pass; 1: statistics (rho, amax of y);
// 2: the cast with rho and the amax from pass 1
template <bool BF16, int FMT, bool SR, int PASS>
__global__ void __launch_bounds__(MN_THREADS)
mxnorm_kernel(const MxNormArgs a) {
    constexpr int ES = BF16 ? 2 : 4;
    constexpr int BLK = (FMT == MXFP4) ? 32 : 16;
    extern __shared__ __align__(16) uint8_t mn_smem[];
    double* part = reinterpret_cast<double*>(mn_smem);                  // [n2] m^p, then the tree
    uint8_t* row_buf = mn_smem + (size_t)a.n2 * sizeof(double);         // the staged row
    __shared__ float red_max[MN_THREADS / 32];
    __shared__ float rho_s;
    __shared__ ScaleTable table;
    const int tid = threadIdx.x, lane = tid & 31;
    const int64_t C = a.cols;
    const int K = a.K;

    ScaleRef ref_t = make_ref(1.0f);
    if (PASS == 2) {
        ref_t = make_ref(tensor_scale_of(*a.amax_in, FMT));
        if (blockIdx.x == 0 && tid == 0 && a.tensor_scale_out) *a.tensor_scale_out = ref_t.s;
        table.build(ref_t.s, tid, MN_THREADS);
    }

    for (int64_t row = blockIdx.x; row < a.rows; row += gridDim.x) {
        // ---- stage the row: 16-byte pieces, coalesced
        const uint4* src = reinterpret_cast<const uint4*>(static_cast<const uint8_t*>(a.x) + row * a.ld * ES);
        uint4* dst = reinterpret_cast<uint4*>(row_buf);
        const int pieces = (int)(C * ES / 16);
        for (int i = tid; i < pieces; i += MN_THREADS) dst[i] = __ldg(src + i);
        __syncthreads();

        float rho;
        if (PASS == 2) {
            rho = a.rho[row];
        } else {
            // ---- block maxima, m^p in binary64 (zeros past K), row maximum
            float rmax = 0.0f;
            for (int k = tid; k < a.n2; k += MN_THREADS) {
                double mp = 0.0;
                if (k < K) {
                    float v[BLK];
                    if (BF16) {
                        const uint4* p = reinterpret_cast<const uint4*>(row_buf + (size_t)k * BLK * 2);
#pragma unroll
                        for (int q = 0; q < BLK / 8; ++q) {
                            const uint4 w = p[q];
                            v[8 * q + 0] = bf16_lo(w.x); v[8 * q + 1] = bf16_hi(w.x);
                            v[8 * q + 2] = bf16_lo(w.y); v[8 * q + 3] = bf16_hi(w.y);
                            v[8 * q + 4] = bf16_lo(w.z); v[8 * q + 5] = bf16_hi(w.z);
                            v[8 * q + 6] = bf16_lo(w.w); v[8 * q + 7] = bf16_hi(w.w);
                        }
                    } else {
                        const float4* p = reinterpret_cast<const float4*>(row_buf + (size_t)k * BLK * 4);
#pragma unroll
                        for (int q = 0; q < BLK / 4; ++q) {
                            const float4 w = p[q];
                            v[4 * q] = w.x; v[4 * q + 1] = w.y; v[4 * q + 2] = w.z; v[4 * q + 3] = w.w;
                        }
                    }
                    const float m = absmax_n<BLK>(v);
                    rmax = fmaxf(rmax, m);
                    mp = (a.p == 2) ? __dmul_rn((double)m, (double)m) : (double)m;
                }
                part[k] = mp;
            }
            __syncthreads();
            // ---- pairwise binary64 sum: level w adds the adjacent subtrees [i, i+w) and [i+w, i+2w)
            for (int w = 1; w < a.n2; w <<= 1) {
                for (int i = tid * 2 * w; i < a.n2; i += MN_THREADS * 2 * w) part[i] = __dadd_rn(part[i], part[i + w]);
                __syncthreads();
            }
            const uint32_t mb = __reduce_max_sync(0xffffffffu, __float_as_uint(rmax));
            if (lane == 0) red_max[tid >> 5] = __uint_as_float(mb);
            __syncthreads();
            if (tid == 0) {
                const double S = part[0];
                float r = 1.0f;
                if (S > 0.0) {
                    const double mean = __ddiv_rn(S, (double)K);
                    const double g = (a.p == 2) ? __dsqrt_rn(mean) : mean;
                    const double q = __ddiv_rn(a.c, g);
                    r = (q >= 3.4028234663852886e38) ? 3.4028234663852886e38f : __double2float_rn(q);
                }
                rho_s = r;
                a.rho[row] = r;
                if (PASS == 1) {
                    float rm = 0.0f;
#pragma unroll
                    for (int w = 0; w < MN_THREADS / 32; ++w) rm = fmaxf(rm, red_max[w]);
                    // amax of y: max_j |RN(x_j rho)| = RN(max_j |x_j| rho), rounding being monotone
                    const float ya = __fmul_rn(rm, r);
                    if (__float_as_uint(ya)) atomicMax(a.amax_out, __float_as_uint(ya));
                }
            }
            __syncthreads();
            rho = rho_s;
        }

        if (PASS != 1) {
            // ---- the cast of y = RN(x * rho), block by block
            const float2 rr = make_float2(rho, rho);
            for (int k = tid; k < K; k += MN_THREADS) {
                float v[BLK];
                if (BF16) {
                    const uint4* p = reinterpret_cast<const uint4*>(row_buf + (size_t)k * BLK * 2);
#pragma unroll
                    for (int q = 0; q < BLK / 8; ++q) {
                        const uint4 w = p[q];
                        v[8 * q + 0] = bf16_lo(w.x); v[8 * q + 1] = bf16_hi(w.x);
                        v[8 * q + 2] = bf16_lo(w.y); v[8 * q + 3] = bf16_hi(w.y);
                        v[8 * q + 4] = bf16_lo(w.z); v[8 * q + 5] = bf16_hi(w.z);
                        v[8 * q + 6] = bf16_lo(w.w); v[8 * q + 7] = bf16_hi(w.w);
                    }
                } else {
                    const float4* p = reinterpret_cast<const float4*>(row_buf + (size_t)k * BLK * 4);
#pragma unroll
                    for (int q = 0; q < BLK / 4; ++q) {
                        const float4 w = p[q];
                        v[4 * q] = w.x; v[4 * q + 1] = w.y; v[4 * q + 2] = w.z; v[4 * q + 3] = w.w;
                    }
                }
#pragma unroll
                for (int j = 0; j < BLK; j += 2) {
                    const float2 y = mul2(make_float2(v[j], v[j + 1]), rr);
                    v[j] = y.x;
                    v[j + 1] = y.y;
                }
                uint32_t sb;
                if (FMT == MXFP4) {
                    sb = mx_scale32<0>(v, absmax_n<32>(v));
                } else {
                    const float bm = absmax_n<16>(v);
                    block_scale_codes<FMT, 1>(&bm, ref_t, &sb);
                    const float2 SY = table.e[sb];
                    nv_divide<16, 0>(v, &SY);
                }
                uint32_t rnd[BLK];
                if (SR) {
                    const uint64_t i0 = (uint64_t)row * (uint64_t)C + (uint64_t)k * BLK;   // a multiple of 16
#pragma unroll
                    for (int q = 0; q < BLK / 4; ++q) {
                        const uint4 w = sr_words((i0 >> 2) + q, a.tensor_id, a.keys);
                        rnd[4 * q] = w.x; rnd[4 * q + 1] = w.y; rnd[4 * q + 2] = w.z; rnd[4 * q + 3] = w.w;
                    }
                }
                uint32_t words[BLK / 8];
#pragma unroll
                for (int q = 0; q < BLK / 8; ++q) words[q] = encode8<FMT, SR>(v + 8 * q, rnd + 8 * q);
                uint8_t* out = a.codes + row * (C / 2) + (int64_t)k * (BLK / 2);
                if (BLK == 32) *reinterpret_cast<uint4*>(out) = make_uint4(words[0], words[1], words[BLK / 8 - 2], words[BLK / 8 - 1]);
                else *reinterpret_cast<uint2*>(out) = make_uint2(words[0], words[1]);
                a.scales[sf_offset(row, k, a.nb4)] = (uint8_t)sb;
            }
        }
        __syncthreads();       // the row buffer is reused by the next row
    }
}

// ---------------------------------------------------------------- warp per row
// bf16 rows of at most MNW_MAX_CHUNKS * 256 columns (a multiple of 256): one
// warp per row.  Chunk i (256 elements) gives lane l the 8 elements
// [256 i + 8 l, 256 i + 8 l + 8) as one 16-byte word, so a block is 2 lanes
// (16 elements) or 4 lanes (32), and its maximum comes from a shuffle within
// them.  The pairwise binary64 sum runs as a butterfly inside each chunk,
// where every lane adds the same two subtrees and so holds the chunk's
// subtree sum; lane i keeps chunk i's, and a butterfly over lanes 0-15
// (zeros past the last chunk) adds the chunks: the same tree, node for node,
// as the CTA kernel's zero-padded one, with no barrier.  The row is read
// twice, for the statistics and for the cast (the second read from L1/L2),
// so that few registers leave room for many warps; the cast uses the block
// maxima of the first read, max |y| = RN(max |x| * rho) (rounding is monotone).
constexpr int MNW_WARPS = 8;
constexpr int MNW_MAX_CHUNKS = 16;
constexpr int MNW_UNROLL = 4;                     // chunks whose loads are in flight together

// v <- RN(v / S) for 8 values of one block with (S, RN(1/S)), as nv_divide
__device__ __forceinline__ void divide8(float* v, float2 SY) {
    if (SY.y != 0.0f) {
        const float2 yy = make_float2(SY.y, SY.y), ss = make_float2(SY.x, SY.x);
#pragma unroll
        for (int j = 0; j < 8; j += 2) {
            const float2 x = make_float2(v[j], v[j + 1]);
            const float2 q0 = mul2(x, yy);
            const float2 rn = __ffma2_rn(ss, q0, make_float2(-x.x, -x.y));
            const float2 q = __ffma2_rn(make_float2(-rn.x, -rn.y), yy, q0);
            v[j] = q.x;
            v[j + 1] = q.y;
        }
    } else {
#pragma unroll
        for (int j = 0; j < 8; ++j) v[j] = SY.x != 0.0f ? __fdiv_rn(v[j], SY.x) : __fmul_rn(v[j], 0.0f);
    }
}

__device__ __forceinline__ void unpack8(const uint4& w, float* v) {
    v[0] = bf16_lo(w.x); v[1] = bf16_hi(w.x); v[2] = bf16_lo(w.y); v[3] = bf16_hi(w.y);
    v[4] = bf16_lo(w.z); v[5] = bf16_hi(w.z); v[6] = bf16_lo(w.w); v[7] = bf16_hi(w.w);
}

template <int FMT, bool SR, int PASS>
__global__ void __launch_bounds__(MNW_WARPS * 32, SR ? 3 : 4)   // the Philox words need more registers
mxnorm_warp_kernel(const MxNormArgs a) {
    constexpr int BLK = (FMT == MXFP4) ? 32 : 16;
    constexpr int LPB = BLK / 8;                       // lanes per block
    __shared__ ScaleTable table;
    const int lane = threadIdx.x & 31;
    const int64_t C = a.cols;
    const int nch = (int)(C / 256);
    ScaleRef ref_t = make_ref(1.0f);
    if (PASS == 2) {
        ref_t = make_ref(tensor_scale_of(*a.amax_in, FMT));
        if (blockIdx.x == 0 && threadIdx.x == 0 && a.tensor_scale_out) *a.tensor_scale_out = ref_t.s;
        table.build(ref_t.s, threadIdx.x, MNW_WARPS * 32);
        __syncthreads();
    }
    const int64_t warps = (int64_t)gridDim.x * MNW_WARPS;
    for (int64_t row = (int64_t)blockIdx.x * MNW_WARPS + (threadIdx.x >> 5); row < a.rows; row += warps) {
        const uint4* src = reinterpret_cast<const uint4*>(static_cast<const uint16_t*>(a.x) + row * a.ld) + lane;

        float rho;
        if (PASS == 2) {
            rho = a.rho[row];
        } else {
            double mine = 0.0;                        // lane i: the sum of chunk i
            float rmax = 0.0f;
            for (int i0 = 0; i0 < nch; i0 += MNW_UNROLL) {
                uint4 w[MNW_UNROLL];
#pragma unroll
                for (int u = 0; u < MNW_UNROLL; ++u)
                    if (i0 + u < nch) w[u] = __ldg(src + 32 * (i0 + u));
#pragma unroll
                for (int u = 0; u < MNW_UNROLL; ++u) {
                    if (i0 + u >= nch) break;
                    float v[8];
                    unpack8(w[u], v);
                    float m = absmax_n<8>(v);
#pragma unroll
                    for (int sh = 1; sh < LPB; sh <<= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, sh));
                    rmax = fmaxf(rmax, m);
                    double t = (a.p == 2) ? __dmul_rn((double)m, (double)m) : (double)m;
                    // the chunk's subtree: butterfly over its blocks, in block order
#pragma unroll
                    for (int sh = LPB; sh < 32; sh <<= 1) t = __dadd_rn(t, __shfl_xor_sync(0xffffffffu, t, sh));
                    if (lane == i0 + u) mine = t;
                }
            }
            // the chunk sums, pairwise over 16 lanes (zeros past the last chunk)
#pragma unroll
            for (int sh = 1; sh < MNW_MAX_CHUNKS; sh <<= 1) mine = __dadd_rn(mine, __shfl_xor_sync(0xffffffffu, mine, sh));
            const double S = __shfl_sync(0xffffffffu, mine, 0);
            rho = 1.0f;
            if (S > 0.0) {
                const double mean = __ddiv_rn(S, (double)a.K);
                const double g = (a.p == 2) ? __dsqrt_rn(mean) : mean;
                const double q = __ddiv_rn(a.c, g);
                rho = (q >= 3.4028234663852886e38) ? 3.4028234663852886e38f : __double2float_rn(q);
            }
            if (lane == 0) a.rho[row] = rho;
            if (PASS == 1) {
                // amax of y: RN(max |x| * rho) (rounding is monotone)
                const float rm = __uint_as_float(__reduce_max_sync(0xffffffffu, __float_as_uint(rmax)));
                const float ya = __fmul_rn(rm, rho);
                if (lane == 0 && __float_as_uint(ya)) atomicMax(a.amax_out, __float_as_uint(ya));
                continue;
            }
        }

        // ---- the cast of y = RN(x * rho)
        const float2 rr = make_float2(rho, rho);
        for (int i0 = 0; i0 < nch; i0 += MNW_UNROLL) {
            uint4 w[MNW_UNROLL];
#pragma unroll
            for (int u = 0; u < MNW_UNROLL; ++u)
                if (i0 + u < nch) w[u] = __ldg(src + 32 * (i0 + u));
#pragma unroll
            for (int u = 0; u < MNW_UNROLL; ++u) {
                const int i = i0 + u;
                if (i >= nch) break;
                float v[8];
                unpack8(w[u], v);
                float mx = absmax_n<8>(v);
#pragma unroll
                for (int sh = 1; sh < LPB; sh <<= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, sh));
#pragma unroll
                for (int j = 0; j < 8; j += 2) {
                    const float2 y = mul2(make_float2(v[j], v[j + 1]), rr);
                    v[j] = y.x;
                    v[j + 1] = y.y;
                }
                const float my = __fmul_rn(mx, rho);          // the block's max |y|
                uint32_t sb;
                if (FMT == MXFP4) {
                    int e = (my > 0.0f) ? ilogbf(my) - 2 : -127;
                    e = max(-127, min(127, e));
                    sb = (uint32_t)(e + 127);
                    const float inv = (e <= 126) ? __uint_as_float((uint32_t)(127 - e) << 23) : __uint_as_float(0x00400000u);
#pragma unroll
                    for (int j = 0; j < 8; j += 2) {
                        const float2 t = mul2(make_float2(v[j], v[j + 1]), make_float2(inv, inv));
                        v[j] = t.x;
                        v[j + 1] = t.y;
                    }
                } else {
                    block_scale_codes<FMT, 1>(&my, ref_t, &sb);
                    divide8(v, table.e[sb]);
                }
                uint32_t rnd[8];
                if (SR) {
                    const uint64_t e0 = (uint64_t)row * (uint64_t)C + (uint64_t)(256 * i + 8 * lane);   // a multiple of 8
                    const uint4 w0 = sr_words(e0 >> 2, a.tensor_id, a.keys);
                    const uint4 w1 = sr_words((e0 >> 2) + 1, a.tensor_id, a.keys);
                    rnd[0] = w0.x; rnd[1] = w0.y; rnd[2] = w0.z; rnd[3] = w0.w;
                    rnd[4] = w1.x; rnd[5] = w1.y; rnd[6] = w1.z; rnd[7] = w1.w;
                }
                const uint32_t word = encode8<FMT, SR>(v, rnd);
                *reinterpret_cast<uint32_t*>(a.codes + row * (C / 2) + 128 * i + 4 * lane) = word;
                if ((lane & (LPB - 1)) == 0) a.scales[sf_offset(row, (256 / BLK) * i + lane / LPB, a.nb4)] = (uint8_t)sb;
            }
        }
    }
}

// the warp kernel serves bf16 rows of 256 .. MNW_MAX_CHUNKS * 256 columns (a multiple of 256)
bool mxnorm_warp_fits(bool bf16, int64_t cols, int64_t ld) {
    return bf16 && cols % 256 == 0 && cols >= 256 && cols <= 256 * MNW_MAX_CHUNKS && ld % 8 == 0;
}

template <int FMT, bool SR, int PASS>
cudaError_t launch_mn_warp(const MxNormArgs& a, cudaStream_t s) {
    int64_t grid = (a.rows + MNW_WARPS - 1) / MNW_WARPS;
    const int64_t cap = (int64_t)num_sms() * (SR ? 3 : 4);
    if (grid > cap) grid = cap;
    if (grid < 1) grid = 1;
    mxnorm_warp_kernel<FMT, SR, PASS><<<(unsigned)grid, MNW_WARPS * 32, 0, s>>>(a);
    return cudaGetLastError();
}

template <bool BF16, int FMT, bool SR, int PASS>
cudaError_t launch_mn(const MxNormArgs& a, cudaStream_t s) {
    auto kernel = mxnorm_kernel<BF16, FMT, SR, PASS>;
    const size_t smem = (size_t)a.n2 * sizeof(double) + (size_t)a.cols * (BF16 ? 2 : 4);
    static PerDeviceOnce setup;
    const cudaError_t se = setup.run([&](int) {
        return cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, 160 * 1024);
    });
    if (se != cudaSuccess) return se;
    int64_t grid = (int64_t)num_sms() * 8;
    if (grid > a.rows) grid = a.rows;
    if (grid < 1) grid = 1;
    kernel<<<(unsigned)grid, MN_THREADS, smem, s>>>(a);
    return cudaGetLastError();
}

template <bool BF16, int FMT, bool SR>
cudaError_t mn_by_pass(const MxNormArgs& a, int pass, cudaStream_t s) {
    const bool warp = mxnorm_warp_fits(BF16, a.cols, a.ld);
    if constexpr (FMT == MXFP4) {
        return warp ? launch_mn_warp<MXFP4, SR, 0>(a, s) : launch_mn<BF16, MXFP4, SR, 0>(a, s);
    } else {
        if (pass == 1) return warp ? launch_mn_warp<FMT, false, 1>(a, s) : launch_mn<BF16, FMT, false, 1>(a, s);
        return warp ? launch_mn_warp<FMT, SR, 2>(a, s) : launch_mn<BF16, FMT, SR, 2>(a, s);
    }
}

template <bool BF16>
cudaError_t mn_by_fmt(const MxNormArgs& a, int fmt, bool sr, int pass, cudaStream_t s) {
    if (fmt == UFP4) return sr ? mn_by_pass<BF16, UFP4, true>(a, pass, s) : mn_by_pass<BF16, UFP4, false>(a, pass, s);
    return sr ? mn_by_pass<BF16, NVFP4, true>(a, pass, s) : mn_by_pass<BF16, NVFP4, false>(a, pass, s);
}

}  // namespace

// MXNorm + cast: MXFP4 in one launch; NVFP4 / UFP4 as the statistics pass
// (amax_word must be zeroed on the stream first) then the quantize pass
cudaError_t launch_mxnorm(const void* x, bool bf16, int64_t rows, int64_t cols, int64_t ld, int fmt, bool sr, int p,
                          double c, uint8_t* codes, uint8_t* scales, float* tensor_scale, float* rho,
                          unsigned int* amax_word, const PhiloxKeys& keys, uint32_t tensor_id, cudaStream_t s) {
    MxNormArgs a{};
    a.x = x; a.rows = rows; a.cols = cols; a.ld = ld;
    a.p = p; a.c = c;
    const int blk = fmt == MXFP4 ? 32 : 16;
    a.K = (int)(cols / blk);
    a.n2 = 1;
    while (a.n2 < a.K) a.n2 <<= 1;
    a.codes = codes; a.scales = scales;
    a.nb4 = (a.K + 3) / 4;
    a.rho = rho;
    a.tensor_scale_out = tensor_scale;
    a.amax_out = amax_word;
    a.amax_in = reinterpret_cast<const float*>(amax_word);
    a.keys = keys;
    a.tensor_id = tensor_id;
    if (fmt == MXFP4)
        return bf16 ? (sr ? mn_by_pass<true, MXFP4, true>(a, 0, s) : mn_by_pass<true, MXFP4, false>(a, 0, s))
                    : (sr ? mn_by_pass<false, MXFP4, true>(a, 0, s) : mn_by_pass<false, MXFP4, false>(a, 0, s));
    cudaError_t e = bf16 ? mn_by_fmt<true>(a, fmt, sr, 1, s) : mn_by_fmt<false>(a, fmt, sr, 1, s);
    if (e != cudaSuccess) return e;
    return bf16 ? mn_by_fmt<true>(a, fmt, sr, 2, s) : mn_by_fmt<false>(a, fmt, sr, 2, s);
}

}  // namespace fp4
