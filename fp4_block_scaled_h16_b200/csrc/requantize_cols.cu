// requantize_cols.cu -- fp4_requantize's kernel: the transposed-axis (axis = 0)
// quantizer reading its tile from an already quantized tensor, X^ = the exact
// dequantized values rounded once to binary32 ("TetraJet-v2" 2.A: the backward
// pass estimates with X^, and the 1x16 groups are re-aligned for the
// transposed weight).  Blocks run down the columns of X^ and the output lines
// are its columns; same arithmetic as the other quantizer kernels.
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <cstdint>

#include "quant_common.cuh"

namespace fp4 {

// A CTA of 4 warps stages a 128-row x 64-column tile in shared memory; thread
// (warp w, lane t) owns columns 2t, 2t+1 over rows 32w..32w+31, i.e. one
// 32-element piece of two output lines, stored as 16 contiguous bytes each.
constexpr int T0_ROWS = 128, T0_COLS = 64, T0_THREADS = 128;

// one FP4 code of the source -> its grid value (E2M1 {0, .5, 1, 1.5, 2, 3, 4, 6}
// or the UFP4 level k), sign from bit 3 (code 8 is -0)
__device__ __forceinline__ float fp4_code_value(uint32_t n, bool ufp4) {
    const uint32_t m = n & 7u;
    const float mag = ufp4 ? (float)m : (float)((0xC8643210u >> (4u * m)) & 0xFu) * 0.5f;   // twice the level
    return (n & 8u) ? -mag : mag;
}

// two E2M1 codes (one byte, element 2j in the low nibble) -> their grid values
// as binary16, element 2j in the low half
__device__ __forceinline__ __half2 e2m1x2_to_h2(uint32_t byte) {
    uint32_t r;
    asm("{\n\t.reg .b8 t;\n\tcvt.u8.u32 t, %1;\n\tcvt.rn.f16x2.e2m1x2 %0, t;\n\t}" : "=r"(r) : "r"(byte));
    return *reinterpret_cast<__half2*>(&r);
}

// FP4SRC: the tile is the dequantized source X^ (fp4_requantize) instead of x
// (only FP4SRC = true is instantiated; bf16 / f32 input has its own kernel in
// quant_cols.cuh)
template <bool BF16, int FMT, bool SR, int ROT, bool SIGNS, bool DB, bool AMAX_ONLY, bool FP4SRC = false>
__global__ void __launch_bounds__(T0_THREADS, 4)
requant_cols_kernel(const QuantArgs a) {
    __shared__ __align__(16) float tile[T0_ROWS][T0_COLS + 4];
    __shared__ float chunk_max[4][T0_COLS];
    const int64_t R = a.rows, C = a.cols;
    const int64_t row0 = (int64_t)blockIdx.y * T0_ROWS, col0 = (int64_t)blockIdx.x * T0_COLS;
    const int tid = threadIdx.x, w = tid >> 5, lane = tid & 31;

    __shared__ ScaleTable table;                        // (S, 1/S) per E4M3 code under s_t
    ScaleRef ref_t = make_ref(1.0f);
    if (!AMAX_ONLY && FMT != MXFP4 && !DB) {
        ref_t = make_ref(tensor_scale_of(*a.amax_in, FMT));
        if (blockIdx.x == 0 && blockIdx.y == 0 && tid == 0 && a.tensor_scale_out) *a.tensor_scale_out = ref_t.s;
        table.build(ref_t.s, tid, T0_THREADS);
    }

    if constexpr (FP4SRC) {
        // ---- stage the dequantized tile: one 16-element piece (8 bytes of
        // codes, one block scale) per step, 4 per thread; zero outside [R, C).
        // Element value: RN((q * E) * s_ref), where q * E is exact in binary32
        // (E4M3 E, s_ref the tensor or outer scale); MXFP4: q * 2^(e - 127),
        // exact (E = 1, s_ref = 2^(e - 127)).  C % 16 == 0, so pieces are whole.
        const int sblk = a.src_fmt == MXFP4 ? 32 : 16;
        const bool ufp4 = a.src_fmt == UFP4;
        const float ts = (a.src_fmt != MXFP4 && !a.src_db) ? *a.src_ts : 1.0f;
#pragma unroll
        for (int it = 0; it < (T0_ROWS * T0_COLS / 16) / T0_THREADS; ++it) {
            const int q = tid + it * T0_THREADS;
            const int r = q >> 2, c = (q & 3) * 16;
            const int64_t gr = row0 + r, gc = col0 + c;
            float x[16];
            if (gr < R && gc < C) {
                const uint2 cw = __ldg(reinterpret_cast<const uint2*>(a.src_codes + gr * (C / 2) + gc / 2));
                const uint32_t sb = a.src_scales[sf_offset(gr, gc / sblk, a.src_nb4)];
                float E, s_ref;
                if (a.src_fmt == MXFP4) {
                    E = 1.0f;
                    s_ref = sb ? __uint_as_float(sb << 23) : __uint_as_float(0x00400000u);   // 2^(sb - 127)
                } else {
                    E = e4m3_to_f32(sb);
                    s_ref = a.src_db ? __ldg(a.src_outer + gr * (C / 128) + gc / 128) : ts;
                }
                if (ufp4) {
#pragma unroll
                    for (int k = 0; k < 16; ++k) {
                        const uint32_t n = ((k < 8 ? cw.x : cw.y) >> (4 * (k & 7))) & 0xFu;
                        x[k] = __fmul_rn(__fmul_rn(fp4_code_value(n, true), E), s_ref);
                    }
                } else {
                    // E2M1: codes decoded two at a time; q * E is exact in binary16
                    // (at most 6 significant bits, between 2^-10 and 2688)
                    const __half2 E2 = __float2half2_rn(E);
#pragma unroll
                    for (int b = 0; b < 8; ++b) {
                        const uint32_t byte = ((b < 4 ? cw.x : cw.y) >> (8 * (b & 3))) & 0xFFu;
                        const float2 qe = __half22float2(__hmul2(e2m1x2_to_h2(byte), E2));
                        x[2 * b] = __fmul_rn(qe.x, s_ref);
                        x[2 * b + 1] = __fmul_rn(qe.y, s_ref);
                    }
                }
            } else {
#pragma unroll
                for (int k = 0; k < 16; ++k) x[k] = 0.0f;
            }
#pragma unroll
            for (int k = 0; k < 16; k += 4)
                *reinterpret_cast<float4*>(&tile[r][c + k]) = make_float4(x[k], x[k + 1], x[k + 2], x[k + 3]);
        }
    } else {
    // ---- stage the tile: 16-byte chunks, all loads issued first; zero outside [R, C)
    constexpr int EPC = BF16 ? 8 : 4;                    // elements per 16-byte chunk
    constexpr int CHUNKS = T0_ROWS * (T0_COLS / EPC);
    constexpr int PER_THREAD = CHUNKS / T0_THREADS;
    uint4 raw[PER_THREAD];
#pragma unroll
    for (int it = 0; it < PER_THREAD; ++it) {
        const int q = tid + it * T0_THREADS;
        const int r = q / (T0_COLS / EPC), c = (q % (T0_COLS / EPC)) * EPC;
        const int64_t gr = row0 + r, gc = col0 + c;
        if (gr < R && gc + EPC <= C) {
            const uint4* p = BF16 ? reinterpret_cast<const uint4*>(static_cast<const uint16_t*>(a.x) + gr * a.ld + gc)
                                  : reinterpret_cast<const uint4*>(static_cast<const float*>(a.x) + gr * a.ld + gc);
            raw[it] = __ldg(p);
        } else {
            uint32_t e[4] = {0u, 0u, 0u, 0u};
            for (int k = 0; k < EPC; ++k) {
                if (gr < R && gc + k < C) {
                    const uint32_t bits = BF16 ? (uint32_t)__ldg(static_cast<const unsigned short*>(a.x) + gr * a.ld + gc + k)
                                               : __float_as_uint(__ldg(static_cast<const float*>(a.x) + gr * a.ld + gc + k));
                    if (BF16) e[k / 2] |= bits << (16 * (k & 1));
                    else e[k] = bits;
                }
            }
            raw[it] = make_uint4(e[0], e[1], e[2], e[3]);
        }
    }
#pragma unroll
    for (int it = 0; it < PER_THREAD; ++it) {
        const int q = tid + it * T0_THREADS;
        const int r = q / (T0_COLS / EPC), c = (q % (T0_COLS / EPC)) * EPC;
        if (BF16) {
            *reinterpret_cast<float4*>(&tile[r][c]) = make_float4(bf16_lo(raw[it].x), bf16_hi(raw[it].x),
                                                                  bf16_lo(raw[it].y), bf16_hi(raw[it].y));
            *reinterpret_cast<float4*>(&tile[r][c + 4]) = make_float4(bf16_lo(raw[it].z), bf16_hi(raw[it].z),
                                                                      bf16_lo(raw[it].w), bf16_hi(raw[it].w));
        } else {
            *reinterpret_cast<float4*>(&tile[r][c]) = make_float4(__uint_as_float(raw[it].x), __uint_as_float(raw[it].y),
                                                                  __uint_as_float(raw[it].z), __uint_as_float(raw[it].w));
        }
    }
    }
    __syncthreads();

    const int64_t rbase = row0 + 32 * w;            // first row (= K index) of this piece
    const int nvalid = (int)max((int64_t)0, min((int64_t)32, R - rbase));   // 0, 16 or 32
    float v[2][32];
#pragma unroll
    for (int k = 0; k < 32; ++k) {
        const float2 p = *reinterpret_cast<const float2*>(&tile[32 * w + k][2 * lane]);
        v[0][k] = p.x;
        v[1][k] = p.y;
    }
#pragma unroll
    for (int cc = 0; cc < 2; ++cc) rotate_unit<32, ROT, SIGNS>(v[cc], a.sign_mask);

    if (AMAX_ONLY) {
        // rows beyond R and columns beyond C are zero-filled and rotate to zero
        const float m = absmax_n<32>(v[1], absmax_n<32>(v[0]));
        const uint32_t bits = __reduce_max_sync(0xffffffffu, __float_as_uint(m));
        if (lane == 0 && bits) atomicMax(a.amax_out, bits);
        return;
    }

    ScaleRef s_ref[2] = {ref_t, ref_t};
    if (DB) {
        // the 128-row chunk is this CTA's tile: reduce the 4 warps' maxima
#pragma unroll
        for (int cc = 0; cc < 2; ++cc) chunk_max[w][2 * lane + cc] = absmax_n<32>(v[cc]);
        __syncthreads();
#pragma unroll
        for (int cc = 0; cc < 2; ++cc) {
            const int c = 2 * lane + cc;
            const float m = fmaxf(fmaxf(chunk_max[0][c], chunk_max[1][c]), fmaxf(chunk_max[2][c], chunk_max[3][c]));
            s_ref[cc] = make_ref(tensor_scale_of(m, NVFP4));
            if (w == 0 && col0 + c < C) a.outer[(col0 + c) * (a.K / 128) + row0 / 128] = s_ref[cc].s;
        }
    }
    if (nvalid == 0) return;

    uint32_t sbytes[2][2];
#pragma unroll
    for (int cc = 0; cc < 2; ++cc) {
        if (FMT == MXFP4) {
            sbytes[cc][0] = mx_scale32<ROT>(v[cc], absmax_n<32>(v[cc]));
            sbytes[cc][1] = 1u;
        } else {
            float2 SY[2];
            float bm[2];
#pragma unroll
            for (int b = 0; b < 2; ++b) bm[b] = absmax_n<16>(v[cc] + 16 * b);
            block_scale_codes<FMT, 2>(bm, s_ref[cc], sbytes[cc]);
#pragma unroll
            for (int b = 0; b < 2; ++b) SY[b] = DB ? scale_pair(sbytes[cc][b], s_ref[cc].s) : table.e[sbytes[cc][b]];
            nv_divide<32, ROT>(v[cc], SY);
        }
    }
    const int64_t line0 = col0 + 2 * lane;     // even; this thread's lines are line0, line0 + 1
    uint32_t words[2][4];
#pragma unroll
    for (int q = 0; q < 4; ++q) {
        uint32_t rnd[2][8];
        if (SR) {
            // element (r, line): i = r * C + line.  With C % 4 == 0 the four
            // lines of lanes 2t and 2t+1 share one Philox group per row: each
            // lane of the pair draws every other row and they swap two words.
            if ((C & 3) == 0) {
                const uint32_t par = lane & 1;
#pragma unroll
                for (int m = 0; m < 4; ++m) {
                    const uint64_t row = (uint64_t)(rbase + 8 * q + 2 * m + par);
                    const uint64_t i = row * (uint64_t)C + (uint64_t)(line0 - 2 * par);   // group start
                    const uint4 wds = sr_words(i >> 2, a.tensor_id, a.keys);
                    const uint32_t mine0 = par ? wds.z : wds.x, mine1 = par ? wds.w : wds.y;
                    const uint32_t send0 = par ? wds.x : wds.z, send1 = par ? wds.y : wds.w;
                    const uint32_t recv0 = __shfl_xor_sync(0xffffffffu, send0, 1);
                    const uint32_t recv1 = __shfl_xor_sync(0xffffffffu, send1, 1);
                    // row 2m is the even lane's, row 2m+1 the odd lane's
                    rnd[0][2 * m] = par ? recv0 : mine0;
                    rnd[1][2 * m] = par ? recv1 : mine1;
                    rnd[0][2 * m + 1] = par ? mine0 : recv0;
                    rnd[1][2 * m + 1] = par ? mine1 : recv1;
                }
            } else {
#pragma unroll
                for (int k = 0; k < 8; ++k) {
                    const uint64_t i = (uint64_t)(rbase + 8 * q + k) * (uint64_t)C + (uint64_t)line0;
                    rnd[0][k] = word_of(sr_words(i >> 2, a.tensor_id, a.keys), (int)(i & 3));
                    const uint64_t i1 = i + 1;
                    rnd[1][k] = word_of(sr_words(i1 >> 2, a.tensor_id, a.keys), (int)(i1 & 3));
                }
            }
        }
#pragma unroll
        for (int cc = 0; cc < 2; ++cc) words[cc][q] = encode8<FMT, SR>(v[cc] + 8 * q, rnd[cc]);
    }
    constexpr int BLK = (FMT == MXFP4) ? 32 : 16;
#pragma unroll
    for (int cc = 0; cc < 2; ++cc) {
        const int64_t line = line0 + cc;
        if (line < C) {
            uint8_t* dst = a.codes + line * (a.K / 2) + rbase / 2;
            if (nvalid == 32 && (a.K & 31) == 0) {
                *reinterpret_cast<uint4*>(dst) = make_uint4(words[cc][0], words[cc][1], words[cc][2], words[cc][3]);
            } else {
                // line pitch K/2 is only 8-byte aligned when K % 32 == 16
                reinterpret_cast<uint2*>(dst)[0] = make_uint2(words[cc][0], words[cc][1]);
                if (nvalid == 32) reinterpret_cast<uint2*>(dst)[1] = make_uint2(words[cc][2], words[cc][3]);
            }
            a.scales[sf_offset(line, rbase / BLK, a.nb4)] = (uint8_t)sbytes[cc][0];
            if (FMT != MXFP4 && nvalid == 32) a.scales[sf_offset(line, rbase / BLK + 1, a.nb4)] = (uint8_t)sbytes[cc][1];
        }
    }
}

// -------------------------------------------------------------------- dispatch

namespace {

template <bool BF16, int FMT, bool SR, int ROT, bool SIGNS, bool DB, bool AMAX_ONLY, bool FP4SRC>
cudaError_t launch_cols(const QuantArgs& a, cudaStream_t s) {
    dim3 grid((unsigned)((a.cols + T0_COLS - 1) / T0_COLS), (unsigned)((a.rows + T0_ROWS - 1) / T0_ROWS));
    requant_cols_kernel<BF16, FMT, SR, ROT, SIGNS, DB, AMAX_ONLY, FP4SRC><<<grid, T0_THREADS, 0, s>>>(a);
    return cudaGetLastError();
}

template <bool BF16, int FMT, bool SR, bool DB, bool AMAX_ONLY, bool FP4SRC = false>
cudaError_t cols_by_rot(const QuantArgs& a, int rot_n, bool signs, cudaStream_t s) {
    if (rot_n == 0) return launch_cols<BF16, FMT, SR, 0, false, DB, AMAX_ONLY, FP4SRC>(a, s);
    if (rot_n == 16) return signs ? launch_cols<BF16, FMT, SR, 16, true, DB, AMAX_ONLY, FP4SRC>(a, s)
                                  : launch_cols<BF16, FMT, SR, 16, false, DB, AMAX_ONLY, FP4SRC>(a, s);
    return signs ? launch_cols<BF16, FMT, SR, 32, true, DB, AMAX_ONLY, FP4SRC>(a, s)
                 : launch_cols<BF16, FMT, SR, 32, false, DB, AMAX_ONLY, FP4SRC>(a, s);
}

template <bool BF16, bool FP4SRC = false>
cudaError_t cols_by_fmt(const QuantArgs& a, int fmt, bool sr, int rot_n, bool signs, bool db, cudaStream_t s) {
    if (fmt == MXFP4) return sr ? cols_by_rot<BF16, MXFP4, true, false, false, FP4SRC>(a, rot_n, signs, s)
                                : cols_by_rot<BF16, MXFP4, false, false, false, FP4SRC>(a, rot_n, signs, s);
    if (fmt == UFP4) return sr ? cols_by_rot<BF16, UFP4, true, false, false, FP4SRC>(a, rot_n, signs, s)
                               : cols_by_rot<BF16, UFP4, false, false, false, FP4SRC>(a, rot_n, signs, s);
    if (db) return sr ? cols_by_rot<BF16, NVFP4, true, true, false, FP4SRC>(a, rot_n, signs, s)
                      : cols_by_rot<BF16, NVFP4, false, true, false, FP4SRC>(a, rot_n, signs, s);
    return sr ? cols_by_rot<BF16, NVFP4, true, false, false, FP4SRC>(a, rot_n, signs, s)
              : cols_by_rot<BF16, NVFP4, false, false, false, FP4SRC>(a, rot_n, signs, s);
}

}  // namespace

cudaError_t launch_requantize_cols(const QuantArgs& a, int fmt, bool sr, int rot_n, bool signs, bool db,
                                   cudaStream_t s) {
    return cols_by_fmt<false, true>(a, fmt, sr, rot_n, signs, db, s);
}

cudaError_t launch_requant_amax_cols(const QuantArgs& a, int rot_n, bool signs, cudaStream_t s) {
    return cols_by_rot<false, NVFP4, false, false, true, true>(a, rot_n, signs, s);
}

}  // namespace fp4
