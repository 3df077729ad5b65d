// quant_cols.cuh -- the transposed-axis (axis = 0) quantizer for bf16 / f32
// input: blocks run down the columns of the row-major input and the output
// lines are its columns, as the Dgrad / Wgrad operands need ("TetraJet-v2"
// 2.A: 1x16 groups re-aligned for the transposed weight).  Same arithmetic,
// in the same order, as the row-axis kernel.  Instantiated per input type in
// quantize_cols_bf16.cu / quantize_cols_f32.cu.
//
// Persistent CTAs of four warps stream 128-row x 64-column tiles through a
// ring of shared-memory stages filled by 2-D TMA loads (zero fill past the
// tensor's edges), thread 0 refilling a slot once every warp has copied it
// out.  Lane (q, h) of warp w owns columns 4q .. 4q+3 over rows
// 32w + 16h .. 32w + 16h + 15 of the tile: one 16-element block of four
// output lines.  So
//   - the rotation runs on packed binary32 pairs of two columns, all stages
//     local; the h = 16 stage of a 32-rotation pairs lane q with lane q + 16;
//   - a 32-element MX block is the lane's rows and its partner's (one
//     shuffle for the maximum); a 128-element double-block chunk is the
//     tile's 128 rows (the four warps meet once per tile);
//   - for stochastic rounding, the four columns of one row are one Philox
//     counter (logical index r * cols + c, c a multiple of 4), so each call's
//     four words serve four elements and no lane waits on another.
//
// Modes, as the row axis: quantize with a known tensor amax, the amax alone,
// or both in one cooperative launch (amax pass, bounded grid barrier, quantize
// pass over the same tiles in reverse order).
//
// Both axes (DUAL, bf16, fused only): the same launch also quantizes along the
// rows, from the same tiles, so the tensor crosses HBM once for both layouts.
// The tiles then land with the 128-byte swizzle (16-byte chunk c of tile row r
// at chunk c ^ (r % 8)), so that thread t reading tile row t (two 32-element
// row units, the row quantizer's arithmetic) and the column lanes both read
// shared memory without bank conflicts.  The row part of each tile runs
// before the column part copies the tile out and releases its slot.
//
// Every wait is bounded by the wait limit of fp4_set_wait_limit (ring: 16 x,
// grid barrier: 4 x); whatever way a CTA leaves, thread 0 first waits for
// every tile load it issued.
#pragma once

#include <cuda.h>

#include "quant_common.cuh"
#include "sm100.cuh"

namespace fp4 {

constexpr int QC_THREADS = 128;
constexpr int QC_ROWS = 128, QC_COLS = 64;
constexpr uint32_t QC_DRAIN_LIMIT = 1u << 22;

enum ColMode { QC_QUANT = 0, QC_AMAX = 1, QC_FUSED = 2 };

// ring waits: 16 x the wait limit; grid barrier: 4 x (saturating)
__device__ __forceinline__ uint32_t qc_ring_limit(uint32_t w) { return w >= (1u << 27) ? 0xFFFFFFFFu : w << 4; }
__device__ __forceinline__ uint32_t qc_grid_limit(uint32_t w) { return w >= (1u << 29) ? 0xFFFFFFFFu : w << 2; }

// Four CTAs per SM (128 registers).  (Measured on B200: a fifth CTA for the
// stochastic-rounding variants, at 96 registers with two stages, was no
// faster: they are bound by their instruction count, not by occupancy.)  The
// both-axes variants with stochastic rounding on the columns run three CTAs
// per SM: at 128 registers they spilled, and with up to 168 they are 7%
// faster on the layer's tensors; two CTAs, or a fourth stage, were slower.
// The double-block variants (about 150 bytes of spills at 128 registers) run
// three CTAs per SM as well: 8% faster on a 4096 x 14336 weight.  (MXFP4 with
// stochastic rounding measured slower at three.)
template <bool BF16, bool SR, bool SWZ = false>
struct ColRing {
    static constexpr int ES = BF16 ? 2 : 4;
    static constexpr int BYTES = QC_ROWS * QC_COLS * ES;        // one tile: 16 KB (bf16) / 32 KB (f32)
    static constexpr int STAGES = BF16 ? 3 : 2;
    static constexpr int CTAS = (SWZ && SR) ? 3 : 4;            // the launch bound
    static constexpr int ALIGN = SWZ ? 1024 : 128;              // the 128-byte swizzle wants 1024-byte stages
    static constexpr int SMEM = STAGES * BYTES + ALIGN /*alignment*/ + STAGES * 16 /*barriers*/;
};

struct ColTiles {
    int n_tr, n_tc, total;      // row tiles, column tiles, n_tr * n_tc (< 2^31)
    uint32_t tc_m, tc_l;        // multiply-shift division by n_tc
};

// 8 values of one column (rows 2i, 2i+1 in byte i) -> a word of E2M1 codes,
// round to nearest even, saturating; a value that rounds to zero keeps its sign
__device__ __forceinline__ uint32_t e2m1_rn8(float a0, float a1, float a2, float a3, float a4, float a5, float a6,
                                             float a7) {
    uint32_t w;
    asm("{\n\t.reg .b8 b0, b1, b2, b3;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b0, %2, %1;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b1, %4, %3;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b2, %6, %5;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b3, %8, %7;\n\t"
        "mov.b32 %0, {b0, b1, b2, b3};\n\t}"
        : "=r"(w)
        : "f"(a0), "f"(a1), "f"(a2), "f"(a3), "f"(a4), "f"(a5), "f"(a6), "f"(a7));
    return w;
}

__device__ __forceinline__ float col_of(const float2& p, int c) { return (c & 1) ? p.y : p.x; }

// ALIGN4 (stochastic rounding only): cols % 4 == 0, so the four columns of a
// row are one Philox counter; otherwise they may straddle two
// DUAL / SR1: also quantize along the rows (rounding SR1), see the file comment
template <bool BF16, int FMT, bool SR, int ROT, bool SIGNS, bool DB, int MODE, bool ALIGN4 = true, bool DUAL = false,
          bool SR1 = false>
__global__ void __launch_bounds__(QC_THREADS, (DB ? 3 : ColRing<BF16, SR, DUAL>::CTAS))
quant_cols_kernel(const __grid_constant__ CUtensorMap tmx, const QuantArgs a, const ColTiles ct, const RowOut ro) {
    constexpr bool AMAX_ONLY = MODE == QC_AMAX, FUSED = MODE == QC_FUSED;
    static_assert(!FUSED || (FMT != MXFP4 && !DB), "only a tensor-scaled format has an amax pass");
    static_assert(!DB || (FMT == NVFP4 && MODE == QC_QUANT), "double block: NVFP4 quantize only");
    static_assert(!DUAL || (BF16 && FUSED && ALIGN4), "both axes: bf16, fused launch, cols % 64 == 0");
    using Ring = ColRing<BF16, SR, DUAL>;
    constexpr int STAGES = Ring::STAGES, BYTES = Ring::BYTES;
    constexpr int BLK = (FMT == MXFP4) ? 32 : 16;
    extern __shared__ uint8_t qc_smem_raw[];
    constexpr uint32_t AL = (uint32_t)Ring::ALIGN;
    uint8_t* buf = qc_smem_raw + ((AL - (sm100::smem_u32(qc_smem_raw) & (AL - 1u))) & (AL - 1u));
    uint64_t* full = reinterpret_cast<uint64_t*>(buf + STAGES * BYTES);   // tile landed
    uint64_t* empty = full + STAGES;                                     // every warp has copied it out
    __shared__ ScaleTable table;                        // (S, 1/S) per E4M3 code under s_t
    __shared__ float chunk_max[2][4][QC_COLS];          // double block: 32-row column maxima per warp
    __shared__ float warp_max[QC_THREADS / 32];
    __shared__ ScaleTable table1;                       // DUAL: the row quantization's table
    __shared__ float warp_max1[QC_THREADS / 32];
    __shared__ uint32_t grid_verdict;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int q = lane & 15, h = lane >> 4;
    const int64_t R = a.rows, C = a.cols;

    ScaleRef ref_t = make_ref(1.0f);
    if (MODE == QC_QUANT && FMT != MXFP4 && !DB) {
        ref_t = make_ref(tensor_scale_of(*a.amax_in, FMT));
        if (blockIdx.x == 0 && tid == 0 && a.tensor_scale_out) *a.tensor_scale_out = ref_t.s;
        table.build(ref_t.s, tid, QC_THREADS);
    }
    if (tid == 0) {
        for (int s = 0; s < STAGES; ++s) {
            sm100::mbar_init(&full[s], 1);
            sm100::mbar_init(&empty[s], QC_THREADS / 32);
        }
        sm100::fence_barrier_init();
        sm100::prefetch_tmap(&tmx);
    }
    __syncthreads();

    // this CTA's tiles first, first + stride, ... make one pass; a fused
    // launch streams them twice, the second pass in reverse order
    const int first = blockIdx.x, stride = gridDim.x;
    const int n = first < ct.total ? (ct.total - first + stride - 1) / stride : 0;
    const int nv = FUSED ? 2 * n : n;
    auto tile_of = [&](int v) { return (FUSED && v >= n) ? first + (2 * n - 1 - v) * stride : first + v * stride; };
    uint32_t issued = 0;
    auto issue = [&](int t, int slot) {
        ++issued;
        const int tr = (int)fast_div((uint32_t)t, ct.tc_m, ct.tc_l), tc = t - tr * ct.n_tc;
        sm100::mbar_arrive_expect_tx(&full[slot], (uint32_t)BYTES);
        sm100::tma_load_2d(buf + slot * BYTES, &tmx, tc * QC_COLS, tr * QC_ROWS, &full[slot]);
    };
    if (tid == 0)
        for (int p = 0; p < STAGES - 1; ++p)
            if (p < nv) issue(tile_of(p), p);

    float tmax = 0.0f, tmax1 = 0.0f;
    ScaleRef ref_t1 = make_ref(1.0f);
    bool ok = true;
    for (int it = 0; it < nv; ++it) {
        if (FUSED && it == n) {
            // end of the amax pass: the CTA's maximum, the grid's, then the
            // tensor scale and its table (every thread of the CTA gets here)
            const uint32_t wbits = __reduce_max_sync(0xffffffffu, __float_as_uint(tmax));
            const uint32_t wbits1 = DUAL ? __reduce_max_sync(0xffffffffu, __float_as_uint(tmax1)) : 0u;
            if (lane == 0) {
                warp_max[warp] = __uint_as_float(wbits);
                if (DUAL) warp_max1[warp] = __uint_as_float(wbits1);
            }
            const bool failed = __syncthreads_or(!ok);
            if (tid == 0) {
                float m = 0.0f, m1 = 0.0f;
#pragma unroll
                for (int w = 0; w < QC_THREADS / 32; ++w) {
                    m = fmaxf(m, warp_max[w]);
                    if (DUAL) m1 = fmaxf(m1, warp_max1[w]);
                }
                if (__float_as_uint(m)) atomicMax(a.amax_out, __float_as_uint(m));
                if (DUAL && __float_as_uint(m1)) atomicMax(ro.amax_out, __float_as_uint(m1));
                __threadfence();
                atomicAdd(a.grid_count, 1u);
                bool done = false;
                const uint32_t glimit = qc_grid_limit(a.wait_limit);
                for (uint32_t i = 0; i < glimit; ++i) {
                    if (sm100::ld_acquire_gpu(a.grid_count) >= gridDim.x) { done = true; break; }
                    __nanosleep(32);
                }
                if (!done) atomicExch(a.err, 7u);       // FP4_ERR_TIMEOUT
                warp_max[0] = __uint_as_float(sm100::ld_acquire_gpu(a.amax_out));
                if (DUAL) warp_max1[0] = __uint_as_float(sm100::ld_acquire_gpu(ro.amax_out));
                grid_verdict = (done && !failed) ? 1u : 0u;
            }
            __syncthreads();
            if (!grid_verdict) {
                ok = false;
                break;
            }
            ref_t = make_ref(tensor_scale_of(warp_max[0], FMT));
            if (blockIdx.x == 0 && tid == 0 && a.tensor_scale_out) *a.tensor_scale_out = ref_t.s;
            table.build(ref_t.s, tid, QC_THREADS);
            if (DUAL) {
                ref_t1 = make_ref(tensor_scale_of(warp_max1[0], FMT));
                if (blockIdx.x == 0 && tid == 0 && ro.tensor_scale_out) *ro.tensor_scale_out = ref_t1.s;
                table1.build(ref_t1.s, tid, QC_THREADS);
            }
            __syncthreads();
        }
        const int t = tile_of(it);
        const int slot = it % STAGES;
        // the verdict on a wait is the warp's (a double-block launch meets once
        // per tile, so there every warp carries a failure on to that meeting)
        bool got = __all_sync(0xffffffffu, sm100::mbar_wait(&full[slot], (uint32_t)(it / STAGES) & 1u,
                                                             qc_ring_limit(a.wait_limit), nullptr));
        if (!got) {
            ok = false;
            if (!DB) {
                if (FUSED && it < n) { it = n - 1; continue; }
                break;
            }
        }
        if (DUAL && got) {
            // ---- the row axis: thread t quantizes tile row t, two 32-element units
            const uint8_t* tile = buf + slot * BYTES;
            const int tr = (int)fast_div((uint32_t)t, ct.tc_m, ct.tc_l), tc = t - tr * ct.n_tc;
            const int64_t row = (int64_t)tr * QC_ROWS + tid;
#pragma unroll 1
            for (int u = 0; u < 2; ++u) {
                float v1[32];
#pragma unroll
                for (int k = 0; k < 4; ++k) {
                    // logical chunk 4u + k of row tid sits at chunk (4u + k) ^ (tid % 8)
                    const uint4 w = *reinterpret_cast<const uint4*>(tile + tid * 128 + (((4 * u + k) ^ (tid & 7)) << 4));
                    v1[8 * k + 0] = bf16_lo(w.x); v1[8 * k + 1] = bf16_hi(w.x);
                    v1[8 * k + 2] = bf16_lo(w.y); v1[8 * k + 3] = bf16_hi(w.y);
                    v1[8 * k + 4] = bf16_lo(w.z); v1[8 * k + 5] = bf16_hi(w.z);
                    v1[8 * k + 6] = bf16_lo(w.w); v1[8 * k + 7] = bf16_hi(w.w);
                }
                if (it < n) {
                    // rows past the tensor read as zeros and leave the maximum alone
                    tmax1 = unit_rotated_absmax<32, ROT, SIGNS>(v1, a.sign_mask, tmax1);
                    continue;
                }
                if (row >= R) continue;
                rotate_unit<32, ROT, SIGNS>(v1, a.sign_mask);
                float bm[2] = {absmax_n<16>(v1), absmax_n<16>(v1 + 16)};
                uint32_t sb[2];
                block_scale_codes<FMT, 2>(bm, ref_t1, sb);
                const float2 SY[2] = {table1.e[sb[0]], table1.e[sb[1]]};
                nv_divide<32, ROT>(v1, SY);
                const int64_t c0 = (int64_t)tc * QC_COLS + 32 * u;      // first column of the unit
                uint32_t rnd[32];
                if (SR1) {
                    const uint64_t i0 = (uint64_t)row * (uint64_t)C + (uint64_t)c0;
#pragma unroll
                    for (int k = 0; k < 8; ++k) {
                        const uint4 w = sr_words((i0 >> 2) + k, ro.tensor_id, a.keys);
                        rnd[4 * k] = w.x; rnd[4 * k + 1] = w.y; rnd[4 * k + 2] = w.z; rnd[4 * k + 3] = w.w;
                    }
                }
                uint32_t words[4];
#pragma unroll
                for (int k = 0; k < 4; ++k) words[k] = encode8<FMT, SR1>(v1 + 8 * k, rnd + 8 * k);
                *reinterpret_cast<uint4*>(ro.codes + row * (C / 2) + c0 / 2) = make_uint4(words[0], words[1], words[2], words[3]);
                // blocks 2j' and 2j'+1 sit side by side in the tiled layout
                *reinterpret_cast<uint16_t*>(ro.scales + sf_offset(row, c0 / 16, ro.nb4)) = (uint16_t)(sb[0] | (sb[1] << 8));
            }
        }

        // my 16 rows x 4 columns, out of the slot
        float2 v[16][2];
        if (got) {
            const uint8_t* tile = buf + slot * BYTES;
#pragma unroll
            for (int j = 0; j < 16; ++j) {
                const int rr = 32 * warp + 16 * h + j;
                if (DUAL) {
                    // columns 4q .. 4q+3: half (q % 2) of logical chunk q / 2, which
                    // sits at chunk (q / 2) ^ (rr % 8), and rr % 8 = j % 8
                    const uint2 w = *reinterpret_cast<const uint2*>(tile + rr * 128 + (((q >> 1) ^ (j & 7)) << 4) +
                                                                    ((q & 1) << 3));
                    v[j][0] = make_float2(bf16_lo(w.x), bf16_hi(w.x));
                    v[j][1] = make_float2(bf16_lo(w.y), bf16_hi(w.y));
                } else if (BF16) {
                    const uint2 w = *reinterpret_cast<const uint2*>(tile + (rr * QC_COLS + 4 * q) * 2);
                    v[j][0] = make_float2(bf16_lo(w.x), bf16_hi(w.x));
                    v[j][1] = make_float2(bf16_lo(w.y), bf16_hi(w.y));
                } else {
                    const float4 w = *reinterpret_cast<const float4*>(tile + (rr * QC_COLS + 4 * q) * 4);
                    v[j][0] = make_float2(w.x, w.y);
                    v[j][1] = make_float2(w.z, w.w);
                }
            }
        }
        __syncwarp();
        if (lane == 0) sm100::mbar_arrive(&empty[slot]);
        bool stalled = false;
        if (tid == 0 && it + STAGES - 1 < nv) {
            const int refill = (it + STAGES - 1) % STAGES;
            if (it > 0 && !sm100::mbar_wait(&empty[refill], (uint32_t)((it - 1) / STAGES) & 1u,
                                            qc_ring_limit(a.wait_limit), nullptr))
                stalled = true;
            else
                issue(tile_of(it + STAGES - 1), refill);
        }
        if (__any_sync(0xffffffffu, stalled)) {
            ok = false;
            if (!DB) {
                if (FUSED && it < n) { it = n - 1; continue; }
                break;
            }
        }
        if (!got) {
#pragma unroll
            for (int j = 0; j < 16; ++j) v[j][0] = v[j][1] = make_float2(0.0f, 0.0f);
        }

        // ---- rotation along the column: y = c_n H_n (d . x) per n-block
        if (ROT) {
            if (SIGNS) {
#pragma unroll
                for (int j = 0; j < 16; ++j) {
                    const uint32_t e = (ROT == 32 ? 16u * h : 0u) + j;
                    const uint32_t sb = ((a.sign_mask >> e) & 1u) << 31;
#pragma unroll
                    for (int cp = 0; cp < 2; ++cp)
                        v[j][cp] = make_float2(__uint_as_float(__float_as_uint(v[j][cp].x) ^ sb),
                                               __uint_as_float(__float_as_uint(v[j][cp].y) ^ sb));
                }
            }
#pragma unroll
            for (int hh = 1; hh < 16; hh <<= 1) {
#pragma unroll
                for (int j = 0; j < 16; ++j) {
                    if ((j & hh) == 0) {
#pragma unroll
                        for (int cp = 0; cp < 2; ++cp) {
                            const float2 x0 = v[j][cp], x1 = v[j + hh][cp];
                            v[j][cp] = add2(x0, x1);
                            v[j + hh][cp] = sub2(x0, x1);
                        }
                    }
                }
            }
            if (ROT == 32) {
                // stage h = 16: element j (lane half 0) with element j + 16 (half 1)
#pragma unroll
                for (int j = 0; j < 16; ++j) {
#pragma unroll
                    for (int cp = 0; cp < 2; ++cp) {
                        const float2 o = v[j][cp];
                        const float2 p = make_float2(__shfl_xor_sync(0xffffffffu, o.x, 16),
                                                     __shfl_xor_sync(0xffffffffu, o.y, 16));
                        v[j][cp] = h == 0 ? add2(o, p) : sub2(p, o);
                    }
                }
            }
        }
        const float cn = (ROT == 16) ? 0.25f : __uint_as_float(0x3E3504F3u);   // binary32(1/sqrt(32))

        // ---- column maxima of my 16 rows; with a rotation they are taken before
        // the factor c_n and scaled after: max |RN(c y)| = RN(c max |y|), since
        // c > 0 and rounding are monotone, so the amax pass skips the 64 products
        float m[4];
#pragma unroll
        for (int c = 0; c < 4; ++c) {
            float mm = 0.0f;
#pragma unroll
            for (int j = 0; j + 1 < 16; j += 2) mm = amax3(mm, col_of(v[j][c >> 1], c), col_of(v[j + 1][c >> 1], c));
            m[c] = ROT ? __fmul_rn(mm, cn) : mm;
        }
        if (AMAX_ONLY || (FUSED && it < n)) {
            tmax = fmaxf(tmax, fmaxf(fmaxf(m[0], m[1]), fmaxf(m[2], m[3])));
            continue;
        }
        if (ROT) {
            const float2 cc = make_float2(cn, cn);
#pragma unroll
            for (int j = 0; j < 16; ++j) {
                v[j][0] = mul2(v[j][0], cc);
                v[j][1] = mul2(v[j][1], cc);
            }
        }

        const int tr = (int)fast_div((uint32_t)t, ct.tc_m, ct.tc_l), tc = t - tr * ct.n_tc;
        const int64_t rbase = (int64_t)tr * QC_ROWS + 32 * warp + 16 * h;   // first row (= K index) of my block
        const int64_t line0 = (int64_t)tc * QC_COLS + 4 * q;                  // my first column (= line)

        // ---- scales
        ScaleRef ref[4] = {ref_t, ref_t, ref_t, ref_t};
        if (DB) {
            // the 128-row chunk is the tile: each warp's 32-row maxima, then all four
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                const float m32 = fmaxf(m[c], __shfl_xor_sync(0xffffffffu, m[c], 16));
                if (h == 0) chunk_max[it & 1][warp][4 * q + c] = m32;
            }
            if (__syncthreads_or(!ok)) break;       // a failure of any warp ends the CTA here
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                const float* cm = &chunk_max[it & 1][0][4 * q + c];
                const float m128 = fmaxf(fmaxf(cm[0], cm[QC_COLS]), fmaxf(cm[2 * QC_COLS], cm[3 * QC_COLS]));
                ref[c] = make_ref(tensor_scale_of(m128, NVFP4));
                if (warp == 0 && h == 0 && line0 + c < C && rbase < R)
                    a.outer[(line0 + c) * (a.K / 128) + rbase / 128] = ref[c].s;
            }
        }
        uint32_t E[4];
        if (FMT == MXFP4) {
            float2 inv[2];
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                const float m32 = fmaxf(m[c], __shfl_xor_sync(0xffffffffu, m[c], 16));
                int e = (m32 > 0.0f) ? ilogbf(m32) - 2 : -127;
                e = max(-127, min(127, e));
                E[c] = (uint32_t)(e + 127);
                const float s = (e <= 126) ? __uint_as_float((uint32_t)(127 - e) << 23) : __uint_as_float(0x00400000u);
                if (c & 1) inv[c >> 1].y = s; else inv[c >> 1].x = s;
            }
#pragma unroll
            for (int j = 0; j < 16; ++j) {
                v[j][0] = mul2(v[j][0], inv[0]);
                v[j][1] = mul2(v[j][1], inv[1]);
            }
        } else {
            float2 SY[4];
            bool slow = false;
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                E[c] = block_scale_code<FMT>(m[c], ref[c]);
                SY[c] = DB ? scale_pair(E[c], ref[c].s) : table.e[E[c]];
                slow = slow || SY[c].y == 0.0f;
            }
            // v <- RN(v / S) by the reciprocal and one correction step with the
            // residual -(S q0 - x) (keeps -0), IEEE division where S or 1/S is
            // not normal; S = 0 gives signed zeros
            if (!slow) {
                const float2 y0 = make_float2(SY[0].y, SY[1].y), y1 = make_float2(SY[2].y, SY[3].y);
                const float2 s0 = make_float2(SY[0].x, SY[1].x), s1 = make_float2(SY[2].x, SY[3].x);
#pragma unroll
                for (int j = 0; j < 16; ++j) {
#pragma unroll
                    for (int cp = 0; cp < 2; ++cp) {
                        const float2 x = v[j][cp];
                        const float2 yy = cp ? y1 : y0, ss = cp ? s1 : s0;
                        const float2 q0 = mul2(x, yy);
                        const float2 rn = __ffma2_rn(ss, q0, make_float2(-x.x, -x.y));
                        v[j][cp] = __ffma2_rn(make_float2(-rn.x, -rn.y), yy, q0);
                    }
                }
            } else {
#pragma unroll
                for (int j = 0; j < 16; ++j) {
#pragma unroll
                    for (int c = 0; c < 4; ++c) {
                        const float x = col_of(v[j][c >> 1], c);
                        float r;
                        if (SY[c].y != 0.0f) {
                            const float q0 = __fmul_rn(x, SY[c].y);
                            const float rn = __fmaf_rn(SY[c].x, q0, -x);
                            r = __fmaf_rn(-rn, SY[c].y, q0);
                        } else {
                            r = SY[c].x != 0.0f ? __fdiv_rn(x, SY[c].x) : __fmul_rn(x, 0.0f);
                        }
                        if (c & 1) v[j][c >> 1].y = r; else v[j][c >> 1].x = r;
                    }
                }
            }
        }

        // ---- round and pack: column c's 16 codes in cw[c][0] (rows 0-7), cw[c][1] (8-15)
        uint32_t cw[4][2];
        if (FMT != UFP4 && !SR) {
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                const int cp = c >> 1;
#pragma unroll
                for (int half = 0; half < 2; ++half) {
                    const int j0 = 8 * half;
                    cw[c][half] = e2m1_rn8(col_of(v[j0][cp], c), col_of(v[j0 + 1][cp], c), col_of(v[j0 + 2][cp], c),
                                           col_of(v[j0 + 3][cp], c), col_of(v[j0 + 4][cp], c), col_of(v[j0 + 5][cp], c),
                                           col_of(v[j0 + 6][cp], c), col_of(v[j0 + 7][cp], c));
                }
            }
        } else {
#pragma unroll
            for (int c = 0; c < 4; ++c) cw[c][0] = cw[c][1] = 0u;
            // element (r, c) has logical index r * cols + c; with cols % 4 == 0
            // the four columns of one row are one Philox counter, and two rows'
            // counters are drawn together so that their rounds overlap
            const uint64_t i0 = (uint64_t)rbase * (uint64_t)C + (uint64_t)line0;
#pragma unroll
            for (int j = 0; j < 16; j += 2) {
                uint32_t rw[2][4] = {{0u, 0u, 0u, 0u}, {0u, 0u, 0u, 0u}};
                if (SR) {
                    const uint64_t ia = i0 + (uint64_t)j * (uint64_t)C, ib = ia + (uint64_t)C;
                    if (ALIGN4) {
                        const uint4 wa = sr_words(ia >> 2, a.tensor_id, a.keys);
                        const uint4 wb = sr_words(ib >> 2, a.tensor_id, a.keys);
                        rw[0][0] = wa.x; rw[0][1] = wa.y; rw[0][2] = wa.z; rw[0][3] = wa.w;
                        rw[1][0] = wb.x; rw[1][1] = wb.y; rw[1][2] = wb.z; rw[1][3] = wb.w;
                    } else {
#pragma unroll
                        for (int rr = 0; rr < 2; ++rr) {
                            const uint64_t i = rr ? ib : ia;
                            const uint4 w = sr_words(i >> 2, a.tensor_id, a.keys);
                            const uint4 w2 = sr_words((i >> 2) + 1, a.tensor_id, a.keys);
                            const uint32_t off = (uint32_t)(i & 3);
#pragma unroll
                            for (int c = 0; c < 4; ++c) {
                                const uint32_t k = off + c;
                                rw[rr][c] = word_of(k < 4 ? w : w2, (int)(k & 3));
                            }
                        }
                    }
                }
#pragma unroll
                for (int rr = 0; rr < 2; ++rr) {
#pragma unroll
                    for (int c = 0; c < 4; ++c) {
                        const float x = col_of(v[j + rr][c >> 1], c);
                        const int nb = (j + rr) & 7;
                        if (FMT == UFP4 && !SR) {
                            const uint32_t k = (uint32_t)__float2int_rn(fminf(fabsf(x), 7.0f));
                            cw[c][(j + rr) >> 3] |= (k | ((__float_as_uint(x) >> 28) & 8u)) << (4 * nb);
                        } else {
                            cw[c][(j + rr) >> 3] |= sr_nibble(FMT == UFP4 ? sr_ufp4_sum(x, rw[rr][c])
                                                                          : sr_e2m1_sum(x, rw[rr][c]), x, nb);
                        }
                    }
                }
            }
        }

        // ---- store: 8 bytes of codes and the block scale of each of my lines
        if (rbase < R) {
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                const int64_t line = line0 + c;
                if (line < C) {
                    *reinterpret_cast<uint2*>(a.codes + line * (a.K / 2) + rbase / 2) = make_uint2(cw[c][0], cw[c][1]);
                    if (FMT != MXFP4 || h == 0) a.scales[sf_offset(line, rbase / BLK, a.nb4)] = (uint8_t)E[c];
                }
            }
        }
    }

    // every tile load issued must land before the CTA may exit: the last fill
    // of slot s has phase (issued - 1 - s) / STAGES; earlier fills of the slot
    // were consumed before it was refilled
    if (tid == 0) {
#pragma unroll
        for (int sl = 0; sl < STAGES; ++sl)
            if (issued > (uint32_t)sl)
                sm100::mbar_wait(&full[sl], ((issued - 1u - sl) / STAGES) & 1u, QC_DRAIN_LIMIT, nullptr);
    }
    if (!ok) {
        if (lane == 0) atomicExch(a.err, 7u);         // FP4_ERR_TIMEOUT
        return;
    }
    if (AMAX_ONLY) {
        const uint32_t bits = __reduce_max_sync(0xffffffffu, __float_as_uint(tmax));
        if (lane == 0 && bits) atomicMax(a.amax_out, bits);
    }
}


template <bool BF16, int FMT, bool SR, int ROT, bool SIGNS, bool DB, int MODE, bool ALIGN4>
cudaError_t launch_cols_k(const QuantArgs& a, cudaStream_t s) {
    using Ring = ColRing<BF16, SR>;
    auto kernel = quant_cols_kernel<BF16, FMT, SR, ROT, SIGNS, DB, MODE, ALIGN4>;
    static PerDeviceOnce setup;
    static int resident_on[kOnceDevices];
    int dev = 0;
    const cudaError_t se = setup.run([&](int d) {
        cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, Ring::SMEM);
        if (e == cudaSuccess)
            e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&resident_on[d], kernel, QC_THREADS, Ring::SMEM);
        return e;
    }, &dev);
    if (se != cudaSuccess) return se;
    if (a.rows >= ((int64_t)1 << 31) || a.cols >= ((int64_t)1 << 31)) return cudaErrorInvalidValue;
    ColTiles ct{};
    ct.n_tr = (int)((a.rows + QC_ROWS - 1) / QC_ROWS);
    ct.n_tc = (int)((a.cols + QC_COLS - 1) / QC_COLS);
    const int64_t total = (int64_t)ct.n_tr * ct.n_tc;
    if (total >= ((int64_t)1 << 31) || total == 0) return cudaErrorInvalidValue;
    ct.total = (int)total;
    uint32_t l = 0;
    while (l < 32 && (uint64_t(1) << l) < (uint64_t)ct.n_tc) ++l;
    ct.tc_m = (uint32_t)((uint64_t)(((unsigned __int128)1 << (32 + l)) / (uint64_t)ct.n_tc) - (uint64_t(1) << 32) + 1);
    ct.tc_l = l;
    CUtensorMap tm;
    if (!make_input_map(&tm, a.x, BF16, a.rows, a.cols, a.ld)) return cudaErrorInvalidValue;
    const int resident = resident_on[dev];
    int64_t grid = (int64_t)num_sms() * (resident > 0 ? resident : 1);
    if (grid > total) grid = total;
    if (MODE == QC_FUSED) {
        if (resident < 1) return cudaErrorInvalidConfiguration;
        QuantArgs ka = a;
        ColTiles kct = ct;
        RowOut kro{};
        void* args[] = {&tm, &ka, &kct, &kro};
        return cudaLaunchCooperativeKernel(reinterpret_cast<const void*>(kernel), dim3((unsigned)grid),
                                           dim3(QC_THREADS), args, Ring::SMEM, s);
    }
    kernel<<<(unsigned)grid, QC_THREADS, Ring::SMEM, s>>>(tm, a, ct, RowOut{});
    return cudaGetLastError();
}

// both axes in one cooperative launch (bf16, NVFP4 / UFP4, cols % 64 == 0):
// a describes the column-axis result and carries the shared fields, ro the
// row-axis result; a.amax_out, ro.amax_out and a.grid_count are zeroed words
template <int FMT, bool SR0, bool SR1, int ROT>
cudaError_t launch_dual_k(const QuantArgs& a, const RowOut& ro, cudaStream_t s) {
    using Ring = ColRing<true, SR0, true>;
    auto kernel = quant_cols_kernel<true, FMT, SR0, ROT, false, false, QC_FUSED, true, true, SR1>;
    static PerDeviceOnce setup;
    static int resident_on[kOnceDevices];
    int dev = 0;
    const cudaError_t se = setup.run([&](int d) {
        cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, Ring::SMEM);
        if (e == cudaSuccess)
            e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&resident_on[d], kernel, QC_THREADS, Ring::SMEM);
        return e;
    }, &dev);
    if (se != cudaSuccess) return se;
    if (a.rows >= ((int64_t)1 << 31) || a.cols >= ((int64_t)1 << 31) || a.cols % QC_COLS) return cudaErrorInvalidValue;
    ColTiles ct{};
    ct.n_tr = (int)((a.rows + QC_ROWS - 1) / QC_ROWS);
    ct.n_tc = (int)(a.cols / QC_COLS);
    const int64_t total = (int64_t)ct.n_tr * ct.n_tc;
    if (total >= ((int64_t)1 << 31) || total == 0) return cudaErrorInvalidValue;
    ct.total = (int)total;
    uint32_t l = 0;
    while (l < 32 && (uint64_t(1) << l) < (uint64_t)ct.n_tc) ++l;
    ct.tc_m = (uint32_t)((uint64_t)(((unsigned __int128)1 << (32 + l)) / (uint64_t)ct.n_tc) - (uint64_t(1) << 32) + 1);
    ct.tc_l = l;
    CUtensorMap tm;
    if (!make_input_map(&tm, a.x, true, a.rows, a.cols, a.ld, true)) return cudaErrorInvalidValue;
    const int resident = resident_on[dev];
    if (resident < 1) return cudaErrorInvalidConfiguration;
    int64_t grid = (int64_t)num_sms() * resident;
    if (grid > total) grid = total;
    QuantArgs ka = a;
    ColTiles kct = ct;
    RowOut kro = ro;
    void* args[] = {&tm, &ka, &kct, &kro};
    return cudaLaunchCooperativeKernel(reinterpret_cast<const void*>(kernel), dim3((unsigned)grid), dim3(QC_THREADS),
                                       args, Ring::SMEM, s);
}

template <int FMT, bool SR0, bool SR1>
cudaError_t dual_by_rot(const QuantArgs& a, const RowOut& ro, int rot_n, cudaStream_t s) {
    return rot_n == 16 ? launch_dual_k<FMT, SR0, SR1, 16>(a, ro, s) : launch_dual_k<FMT, SR0, SR1, 0>(a, ro, s);
}

// entry for fp4_quantize_both_axes (quantize_dual.cu): rot_n 0 or 16, no signs
inline cudaError_t launch_both_axes_impl(const QuantArgs& a, const RowOut& ro, int fmt, bool sr_cols, bool sr_rows,
                                         int rot_n, cudaStream_t s) {
    if (fmt == UFP4) {
        if (sr_cols) return sr_rows ? dual_by_rot<UFP4, true, true>(a, ro, rot_n, s) : dual_by_rot<UFP4, true, false>(a, ro, rot_n, s);
        return sr_rows ? dual_by_rot<UFP4, false, true>(a, ro, rot_n, s) : dual_by_rot<UFP4, false, false>(a, ro, rot_n, s);
    }
    if (sr_cols) return sr_rows ? dual_by_rot<NVFP4, true, true>(a, ro, rot_n, s) : dual_by_rot<NVFP4, true, false>(a, ro, rot_n, s);
    return sr_rows ? dual_by_rot<NVFP4, false, true>(a, ro, rot_n, s) : dual_by_rot<NVFP4, false, false>(a, ro, rot_n, s);
}

// stochastic rounding of a tensor whose column count is not a multiple of 4
// takes the instantiation whose Philox counters may straddle two groups
template <bool BF16, int FMT, bool SR, int ROT, bool SIGNS, bool DB, int MODE>
cudaError_t launch_cols(const QuantArgs& a, cudaStream_t s) {
    if (SR && (a.cols & 3) != 0) return launch_cols_k<BF16, FMT, SR, ROT, SIGNS, DB, MODE, false>(a, s);
    return launch_cols_k<BF16, FMT, SR, ROT, SIGNS, DB, MODE, true>(a, s);
}

template <bool BF16, int FMT, bool SR, bool DB, int MODE>
cudaError_t cols_by_rot(const QuantArgs& a, int rot_n, bool signs, cudaStream_t s) {
    if (rot_n == 0) return launch_cols<BF16, FMT, SR, 0, false, DB, MODE>(a, s);
    if (rot_n == 16) return signs ? launch_cols<BF16, FMT, SR, 16, true, DB, MODE>(a, s)
                                  : launch_cols<BF16, FMT, SR, 16, false, DB, MODE>(a, s);
    return signs ? launch_cols<BF16, FMT, SR, 32, true, DB, MODE>(a, s)
                 : launch_cols<BF16, FMT, SR, 32, false, DB, MODE>(a, s);
}

// one input type's entry points (quantize_cols_bf16.cu, quantize_cols_f32.cu)
template <bool BF16>
cudaError_t launch_cols_quantize(const QuantArgs& a, int fmt, bool sr, int rot_n, bool signs, bool db,
                                 cudaStream_t s) {
    if (fmt == MXFP4) return sr ? cols_by_rot<BF16, MXFP4, true, false, QC_QUANT>(a, rot_n, signs, s)
                                : cols_by_rot<BF16, MXFP4, false, false, QC_QUANT>(a, rot_n, signs, s);
    if (fmt == UFP4) return sr ? cols_by_rot<BF16, UFP4, true, false, QC_QUANT>(a, rot_n, signs, s)
                               : cols_by_rot<BF16, UFP4, false, false, QC_QUANT>(a, rot_n, signs, s);
    if (db) return sr ? cols_by_rot<BF16, NVFP4, true, true, QC_QUANT>(a, rot_n, signs, s)
                      : cols_by_rot<BF16, NVFP4, false, true, QC_QUANT>(a, rot_n, signs, s);
    return sr ? cols_by_rot<BF16, NVFP4, true, false, QC_QUANT>(a, rot_n, signs, s)
              : cols_by_rot<BF16, NVFP4, false, false, QC_QUANT>(a, rot_n, signs, s);
}

template <bool BF16>
cudaError_t launch_cols_amax(const QuantArgs& a, int rot_n, bool signs, cudaStream_t s) {
    return cols_by_rot<BF16, NVFP4, false, false, QC_AMAX>(a, rot_n, signs, s);
}

template <bool BF16>
cudaError_t launch_cols_fused(const QuantArgs& a, int fmt, bool sr, int rot_n, bool signs, cudaStream_t s) {
    if (fmt == UFP4) return sr ? cols_by_rot<BF16, UFP4, true, false, QC_FUSED>(a, rot_n, signs, s)
                               : cols_by_rot<BF16, UFP4, false, false, QC_FUSED>(a, rot_n, signs, s);
    return sr ? cols_by_rot<BF16, NVFP4, true, false, QC_FUSED>(a, rot_n, signs, s)
              : cols_by_rot<BF16, NVFP4, false, false, QC_FUSED>(a, rot_n, signs, s);
}

}  // namespace fp4
