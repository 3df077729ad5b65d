// gemm_db.cu -- block-scaled FP4 GEMM for the double-block NVFP4 format
// ("TetraJet-v2" 2.A: a 128-element outer block scaled globally in FP32 over
// 16-element inner blocks scaled locally in E4M3):
//
//   C[i, j] = sum_kc  s_oA[i, kc] * s_oB[j, kc] * P_kc[i, j],
//   P_kc[i, j] = sum_{k in chunk kc} qA[i, k] qB[j, k] sA[i, k/16] sB[j, k/16].
//
// The outer scale changes every 128 elements of K, so it cannot ride in the
// tensor core's E4M3 block scales.  Each 128-K chunk is two block-scaled MMAs
// (tcgen05 kind::mxf4nvf4, 128 x 128 x 64) into one of three TMEM partial
// buffers in rotation; while the tensor core fills one, eight epilogue warps
// (two per TMEM lane quarter, 64 columns each, so that the per-chunk barrier
// and bookkeeping work is shared by twice the arithmetic) promote another:
// acc[i, j] += s_oA[i, kc] * (s_oB[j, kc] * P_kc[i, j]) in registers, on
// packed f32x2 pairs.  The operand pipeline (TMA producer warp, MMA warp,
// 4-stage ring of 256-K stages) is the one of the plain GEMM; one more warp
// stages each tile's B outer scales transposed ([chunk][column]), in groups
// of 64 chunks (any K), into a double-buffered shared area, so the promotion
// reads four of them per 128-bit shared load.  All hand-offs are mbarriers
// with bounded waits.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <cstdint>
#include <mutex>

#include "internal.h"
#include "sm100.cuh"

namespace fp4 {

namespace {

constexpr int BM = 128, BN = 128, BK = 256;
constexpr int STAGES = 4;
constexpr int EPI_WARPS = 8;              // two per TMEM lane quarter, half the columns each
constexpr int COLS = BN / (EPI_WARPS / 4);      // columns one epilogue warp promotes
constexpr int HALF = COLS / 2;                  // columns per TMEM load
constexpr int NUM_THREADS = 32 * (2 + EPI_WARPS + 1);   // producer, MMA, epilogue, outer-scale warp
constexpr int STAGER_WARP = 2 + EPI_WARPS;
constexpr uint32_t TMEM_COLS = 512;
constexpr uint32_t DRAIN_LIMIT = 1u << 22;
constexpr unsigned int ERR_TIMEOUT = 7u;
constexpr int MAX_CHUNKS = 64;                        // chunks of B outer scales per staged group

constexpr uint32_t A_BYTES = BM * BK / 2, B_BYTES = BN * BK / 2;
constexpr uint32_t SFA_BYTES = BM * (BK / 16), SFB_BYTES = BN * (BK / 16);
constexpr uint32_t TX = A_BYTES + B_BYTES + SFA_BYTES + SFB_BYTES;
constexpr uint32_t STAGE_BYTES = (TX + 1023) / 1024 * 1024;
constexpr uint32_t OUTER_BYTES = 2 * MAX_CHUNKS * BN * 4;   // two groups of s_oB, [chunk][column]
constexpr uint32_t SMEM = STAGES * STAGE_BYTES + OUTER_BYTES + 1024 + 256;
constexpr int PBUF = 3;                               // TMEM partial buffers in rotation
constexpr uint32_t SFA_COL = PBUF * BN;               // TMEM: partials at 0, BN, 2 BN, then scales
constexpr uint32_t SFB_COL = SFA_COL + 16;

struct DbParams {
    const uint8_t* a_sf;
    const uint8_t* b_sf;
    const float* a_outer;      // [M, K/128]
    const float* b_outer;      // [N, K/128]
    void* c;
    int64_t ldc;
    int M, N, K;
    int nb4;
    int tiles_m, tiles_n;
    uint32_t wait_limit;
    unsigned int* err;
};

__device__ __forceinline__ void raise_timeout(const DbParams& p, volatile int* abort_flag) {
    *abort_flag = 1;
    atomicExch(p.err, ERR_TIMEOUT);
}

// PAIRED: K / 128 is even, and the promotion warps read the row outer scales
// two chunks at a time (8-byte loads, half the load instructions); otherwise
// one chunk at a time
template <bool OUT_BF16, bool PAIRED>
__global__ void __launch_bounds__(NUM_THREADS, 1)
gemm_db_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB, const DbParams p) {
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw = sm100::smem_u32(smem_raw);
    uint8_t* smem = smem_raw + ((1024u - (raw & 1023u)) & 1023u);
    float* outer_b = reinterpret_cast<float*>(smem + STAGES * STAGE_BYTES);
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + STAGES * STAGE_BYTES + OUTER_BYTES);
    uint64_t* empty = full + STAGES;
    uint64_t* pfull = empty + STAGES;          // partial buffer b holds a finished chunk
    uint64_t* pempty = pfull + PBUF;           // partial buffer b was read by the epilogue
    uint64_t* ofull = pempty + PBUF;           // outer-scale buffer b is staged for a tile
    uint64_t* oempty = ofull + 2;              // the epilogue is done with outer buffer b
    uint64_t* drain = oempty + 2;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; ++s) {
            sm100::mbar_init(&full[s], 1);
            sm100::mbar_init(&empty[s], 1);
        }
        for (int b = 0; b < PBUF; ++b) {
            sm100::mbar_init(&pfull[b], 1);
            sm100::mbar_init(&pempty[b], EPI_WARPS);
        }
        for (int b = 0; b < 2; ++b) {
            sm100::mbar_init(&ofull[b], 32);
            sm100::mbar_init(&oempty[b], EPI_WARPS);
        }
        sm100::mbar_init(drain, 1);
        *abort_flag = 0;
        sm100::fence_barrier_init();
        sm100::prefetch_tmap(&tmA);
        sm100::prefetch_tmap(&tmB);
    }
    if (warp == 1) {
        sm100::tmem_alloc(tmem_slot, TMEM_COLS);
        sm100::tmem_relinquish();
    }
    sm100::tc_fence_before();
    __syncthreads();
    sm100::tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    const int tiles = p.tiles_m * p.tiles_n;
    // stages per tile; with K an odd multiple of 128 the last stage holds one
    // 128-K chunk (its code boxes read zeros past K, half its scale bytes)
    const int kt_count = (p.K + BK - 1) / BK;
    const bool ragged_k = (p.K % BK) != 0;
    const int nkc = p.K / 128;

    if (warp == 0) {
        // ------------------------------------------------------------ producer
        if (sm100::elect_one()) {
            int stage = 0;
            uint32_t phase = 0, fills = 0;
            bool ok = true;
            for (int t = blockIdx.x; t < tiles && ok; t += gridDim.x) {
                int tm_, tn_;
                tile_coords(t, p.tiles_m, p.tiles_n, tm_, tn_);
                const int m0 = tm_ * BM, n0 = tn_ * BN;
                for (int kt = 0; kt < kt_count; ++kt) {
                    if (!sm100::mbar_wait(&empty[stage], phase ^ 1u, p.wait_limit, abort_flag)) {
                        raise_timeout(p, abort_flag);
                        ok = false;
                        break;
                    }
                    uint8_t* st = smem + stage * STAGE_BYTES;
                    const bool half_k = ragged_k && kt == kt_count - 1;
                    const uint32_t sfa = half_k ? SFA_BYTES / 2 : SFA_BYTES, sfb = half_k ? SFB_BYTES / 2 : SFB_BYTES;
                    sm100::mbar_arrive_expect_tx(&full[stage], A_BYTES + B_BYTES + sfa + sfb);
                    sm100::tma_load_2d(st, &tmA, kt * (BK / 2), m0, &full[stage]);
                    sm100::tma_load_2d(st + A_BYTES, &tmB, kt * (BK / 2), n0, &full[stage]);
                    const int kb0 = kt * (BK / 16);
                    sm100::bulk_load(st + A_BYTES + B_BYTES,
                                     p.a_sf + ((int64_t)(m0 / 128) * p.nb4 + kb0 / 4) * 512, sfa, &full[stage]);
                    sm100::bulk_load(st + A_BYTES + B_BYTES + SFA_BYTES,
                                     p.b_sf + ((int64_t)(n0 / 128) * p.nb4 + kb0 / 4) * 512, sfb, &full[stage]);
                    ++fills;
                    if (++stage == STAGES) { stage = 0; phase ^= 1u; }
                }
            }
#pragma unroll
            for (int s = 0; s < STAGES; ++s)
                if (fills > (uint32_t)s)
                    sm100::mbar_wait(&full[s], ((fills - 1u - s) / STAGES) & 1u, DRAIN_LIMIT, nullptr);
        }
        __syncwarp();
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer
        if (sm100::elect_one()) {
            int stage = 0, pb = 0;
            uint32_t phase = 0, pphase = 0u;          // bit b: phase of partial buffer b
            bool ok = true, issued = false;
            const uint32_t idesc = sm100::idesc_block_scaled(BN, false, 0, 0);
            for (int t = blockIdx.x; t < tiles && ok; t += gridDim.x) {
                for (int kt = 0; kt < kt_count && ok; ++kt) {
                    if (!sm100::mbar_wait(&full[stage], phase, p.wait_limit, abort_flag)) {
                        raise_timeout(p, abort_flag);
                        ok = false;
                        break;
                    }
                    sm100::tc_fence_after();
                    const uint32_t st = sm100::smem_u32(smem + stage * STAGE_BYTES);
                    const uint32_t st_sfa = st + A_BYTES + B_BYTES, st_sfb = st_sfa + SFA_BYTES;
                    const int chunks = (ragged_k && kt == kt_count - 1) ? 1 : 2;
#pragma unroll
                    for (int j = 0; j < 4; ++j) {
                        if (j >= 2 * chunks) break;
                        sm100::tc_cp_sf(tmem + SFA_COL + 4 * j, sm100::desc_sf(st_sfa + 512 * j));
                        sm100::tc_cp_sf(tmem + SFB_COL + 4 * j, sm100::desc_sf(st_sfb + 512 * j));
                    }
                    // two 128-K chunks per stage (one in a half stage), each into its own
                    // partial buffer
#pragma unroll
                    for (int h = 0; h < 2; ++h) {
                        if (h >= chunks) break;
                        if (!sm100::mbar_wait(&pempty[pb], ((pphase >> pb) & 1u) ^ 1u, p.wait_limit, abort_flag)) {
                            raise_timeout(p, abort_flag);
                            ok = false;
                            break;
                        }
                        sm100::tc_fence_after();
#pragma unroll
                        for (int q = 0; q < 2; ++q) {
                            const int kk = 2 * h + q;
                            sm100::mma_nvf4(tmem + BN * pb, sm100::desc_sw128(st + 32 * kk),
                                            sm100::desc_sw128(st + A_BYTES + 32 * kk), idesc,
                                            tmem + SFA_COL + 4 * kk, tmem + SFB_COL + 4 * kk, q);
                        }
                        issued = true;
                        sm100::tc_commit(&pfull[pb]);
                        pphase ^= 1u << pb;
                        pb = (pb + 1 == PBUF) ? 0 : pb + 1;
                    }
                    if (!ok) break;
                    sm100::tc_commit(&empty[stage]);
                    if (++stage == STAGES) { stage = 0; phase ^= 1u; }
                }
            }
            if (issued) {
                sm100::tc_commit(drain);
                sm100::mbar_wait(drain, 0, DRAIN_LIMIT, nullptr);
            }
        }
        __syncwarp();
    } else if (warp == STAGER_WARP) {
        // ------------------------------------------------------------ outer-scale stager
        int ob = 0;
        uint32_t ophase = 0u;                         // bit b: phase of outer buffer b
        for (int t = blockIdx.x; t < tiles; t += gridDim.x) {
            int tm_, tn_;
            tile_coords(t, p.tiles_m, p.tiles_n, tm_, tn_);
            const int n0 = tn_ * BN;
            // the tile's B outer scales in groups of up to MAX_CHUNKS chunks,
            // one group per buffer: rows n0 .. n0+127 of [N, K/128] written
            // transposed ([chunk][column]); consecutive lanes take consecutive
            // columns so the shared stores do not collide on a bank
            bool staged = true;
            for (int g0 = 0; g0 < nkc; g0 += MAX_CHUNKS) {
                const int cnt = min(MAX_CHUNKS, nkc - g0);
                int got = 0;
                if (lane == 0)
                    got = sm100::mbar_wait(&oempty[ob], ((ophase >> ob) & 1u) ^ 1u, p.wait_limit, abort_flag) ? 1 : 0;
                if (!__shfl_sync(0xffffffffu, got, 0)) {
                    if (lane == 0) raise_timeout(p, abort_flag);
                    staged = false;
                    break;
                }
                float* dst = outer_b + ob * (MAX_CHUNKS * BN);
                const float* src = p.b_outer + (int64_t)n0 * nkc + g0;
                for (int e = lane; e < BN * cnt; e += 32) {
                    const int kc = e / BN, c = e % BN;
                    dst[e] = __ldg(src + (int64_t)c * nkc + kc);
                }
                __syncwarp();
                sm100::mbar_arrive(&ofull[ob]);          // release: every lane's stores before
                ophase ^= 1u << ob;
                ob ^= 1;
            }
            if (!staged) break;
        }
    } else {
        // ------------------------------------------------------------ promotion + epilogue
        const int q = warp & 3;                 // TMEM lane quarter of this warp
        const int cg = (warp - 2) >> 2;         // column group of this warp
        int pb = 0, ob = 0;
        uint32_t pphase = 0u, ophase = 0u;            // bit b: phase of buffer b
        bool ok = true;
        for (int t = blockIdx.x; t < tiles && ok; t += gridDim.x) {
            int tm_, tn_;
                tile_coords(t, p.tiles_m, p.tiles_n, tm_, tn_);
                const int m0 = tm_ * BM, n0 = tn_ * BN + cg * COLS;
            const int row = m0 + 32 * q + lane;
            const float* outer_tile = outer_b + cg * COLS;     // set per group of chunks below
            float2 acc[COLS / 2];
#pragma unroll
            for (int c = 0; c < COLS / 2; ++c) acc[c] = make_float2(0.0f, 0.0f);
            // the row's outer scales, loaded ahead of their use: in pairs (PAIRED,
            // one pair ahead) or one at a time (three chunks ahead)
            const float* a_outer_row = p.a_outer + (int64_t)row * nkc;
            const float2* a_outer_pairs = reinterpret_cast<const float2*>(a_outer_row);
            float2 sa_cur = make_float2(0.0f, 0.0f), sa_nxt = make_float2(0.0f, 0.0f);
            float sa0 = 0.0f, sa1 = 0.0f, sa2n = 0.0f;
            if (PAIRED) {
                sa_cur = __ldg(a_outer_pairs);
                sa_nxt = nkc > 2 ? __ldg(a_outer_pairs + 1) : sa_cur;
            } else {
                sa0 = __ldg(a_outer_row);
                sa1 = nkc > 1 ? __ldg(a_outer_row + 1) : 0.0f;
                sa2n = nkc > 2 ? __ldg(a_outer_row + 2) : 0.0f;
            }
            // the slice is read in two halves of 16 columns: one half's TMEM load
            // is in flight while the other half is promoted
            const uint32_t tbase = tmem + ((uint32_t)(32 * q) << 16) + cg * COLS;
            uint32_t ra[HALF], rb[HALF];
            if (!__all_sync(0xffffffffu, sm100::mbar_wait(&pfull[pb], (pphase >> pb) & 1u, p.wait_limit, abort_flag))) {
                if (lane == 0) raise_timeout(p, abort_flag);
                ok = false;
            } else {
                sm100::tc_fence_after();
                sm100::tmem_ld32(tbase + BN * pb, ra);
                sm100::tmem_ld_wait_on(ra);
            }
            int kc = 0;
            for (int g0 = 0; g0 < nkc && ok; g0 += MAX_CHUNKS) {
                // the next group of B outer scales (chunks g0 .. gend - 1)
                const int gend = min(nkc, g0 + MAX_CHUNKS);
                if (!__all_sync(0xffffffffu, sm100::mbar_wait(&ofull[ob], (ophase >> ob) & 1u, p.wait_limit, abort_flag))) {
                    if (lane == 0) raise_timeout(p, abort_flag);
                    ok = false;
                    break;
                }
                outer_tile = outer_b + ob * (MAX_CHUNKS * BN) + cg * COLS - g0 * BN;
                for (; kc < gend && ok; ++kc) {
                    const float sa = PAIRED ? ((kc & 1) ? sa_cur.y : sa_cur.x) : sa0;
                    const float2 sa2 = make_float2(sa, sa);
                    const float4* sb = reinterpret_cast<const float4*>(outer_tile + kc * BN);
                    sm100::tmem_ld32(tbase + BN * pb + HALF, rb);
                    // acc += sa * (sB * P) on the first half, packed
#pragma unroll
                    for (int c = 0; c < HALF / 4; ++c) {
                        const float4 w = sb[c];
                        const float2 t0 = __fmul2_rn(make_float2(__uint_as_float(ra[4 * c]), __uint_as_float(ra[4 * c + 1])),
                                                     make_float2(w.x, w.y));
                        const float2 t1 = __fmul2_rn(make_float2(__uint_as_float(ra[4 * c + 2]), __uint_as_float(ra[4 * c + 3])),
                                                     make_float2(w.z, w.w));
                        acc[2 * c] = __ffma2_rn(t0, sa2, acc[2 * c]);
                        acc[2 * c + 1] = __ffma2_rn(t1, sa2, acc[2 * c + 1]);
                    }
                    sm100::tmem_ld_wait_on(rb);
                    sm100::tc_fence_before();
                    __syncwarp();
                    if (lane == 0) sm100::mbar_arrive(&pempty[pb]);     // the tensor core may refill it
                    pphase ^= 1u << pb;
                    pb = (pb + 1 == PBUF) ? 0 : pb + 1;
                    if (PAIRED) {
                        if (kc & 1) {
                            sa_cur = sa_nxt;
                            if (kc + 3 < nkc) sa_nxt = __ldg(a_outer_pairs + (kc + 3) / 2);
                        }
                    } else {
                        sa0 = sa1;
                        sa1 = sa2n;
                        if (kc + 3 < nkc) sa2n = __ldg(a_outer_row + kc + 3);
                    }
                    bool next = false;
                    if (kc + 1 < nkc) {
                        if (__all_sync(0xffffffffu,
                                       sm100::mbar_wait(&pfull[pb], (pphase >> pb) & 1u, p.wait_limit, abort_flag))) {
                            sm100::tc_fence_after();
                            sm100::tmem_ld32(tbase + BN * pb, ra);
                            next = true;
                        } else {
                            if (lane == 0) raise_timeout(p, abort_flag);
                            ok = false;
                        }
                    }
                    // the second half, while the next chunk's first half loads
#pragma unroll
                    for (int c = 0; c < HALF / 4; ++c) {
                        const float4 w = sb[HALF / 4 + c];
                        const float2 t0 = __fmul2_rn(make_float2(__uint_as_float(rb[4 * c]), __uint_as_float(rb[4 * c + 1])),
                                                     make_float2(w.x, w.y));
                        const float2 t1 = __fmul2_rn(make_float2(__uint_as_float(rb[4 * c + 2]), __uint_as_float(rb[4 * c + 3])),
                                                     make_float2(w.z, w.w));
                        acc[HALF / 2 + 2 * c] = __ffma2_rn(t0, sa2, acc[HALF / 2 + 2 * c]);
                        acc[HALF / 2 + 2 * c + 1] = __ffma2_rn(t1, sa2, acc[HALF / 2 + 2 * c + 1]);
                    }
                    if (next) sm100::tmem_ld_wait_on(ra);
                }
                __syncwarp();
                if (lane == 0) sm100::mbar_arrive(&oempty[ob]);          // this group's outer scales are used
                ophase ^= 1u << ob;
                ob ^= 1;
            }
            if (!ok) break;
            // store this warp's part of the tile's row
            if (OUT_BF16) {
                uint4* dst = reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(p.c) + (int64_t)row * p.ldc + n0);
#pragma unroll
                for (int v = 0; v < COLS / 8; ++v) {
                    uint32_t pk[4];
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const __nv_bfloat162 h = __floats2bfloat162_rn(acc[4 * v + e].x, acc[4 * v + e].y);
                        pk[e] = *reinterpret_cast<const uint32_t*>(&h);
                    }
                    dst[v] = make_uint4(pk[0], pk[1], pk[2], pk[3]);
                }
            } else {
                float4* dst = reinterpret_cast<float4*>(static_cast<float*>(p.c) + (int64_t)row * p.ldc + n0);
#pragma unroll
                for (int v = 0; v < COLS / 4; ++v)
                    dst[v] = make_float4(acc[2 * v].x, acc[2 * v].y, acc[2 * v + 1].x, acc[2 * v + 1].y);
            }
        }
    }

    sm100::tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        sm100::tc_fence_after();
        sm100::tmem_dealloc(tmem, TMEM_COLS);
    }
}

template <bool OUT_BF16, bool PAIRED>
cudaError_t run_db(const GemmArgs& g, cudaStream_t s) {
    static PerDeviceOnce setup;
    const cudaError_t attr_err = setup.run([](int) {
        return cudaFuncSetAttribute(gemm_db_kernel<OUT_BF16, PAIRED>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                    (int)SMEM);
    });
    if (attr_err != cudaSuccess) return attr_err;
    CUtensorMap ta, tb;
    if (!make_codes_map(&ta, g.a_codes, g.M, g.K, BM) || !make_codes_map(&tb, g.b_codes, g.N, g.K, BN))
        return cudaErrorInvalidValue;
    DbParams p{};
    p.a_sf = g.a_scales;
    p.b_sf = g.b_scales;
    p.a_outer = g.a_outer;
    p.b_outer = g.b_outer;
    p.c = g.c;
    p.ldc = g.ldc;
    p.M = (int)g.M;
    p.N = (int)g.N;
    p.K = (int)g.K;
    p.nb4 = (int)(g.K / 16 / 4);
    p.tiles_m = (int)(g.M / BM);
    p.tiles_n = (int)(g.N / BN);
    p.wait_limit = g.wait_limit;
    p.err = device_error_word();
    const int tiles = p.tiles_m * p.tiles_n;
    const int grid = tiles < num_sms() ? tiles : num_sms();
    gemm_db_kernel<OUT_BF16, PAIRED><<<grid, NUM_THREADS, SMEM, s>>>(ta, tb, p);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_gemm_db(const GemmArgs& g, cudaStream_t s) {
    if ((g.K / 128) % 2 == 0) return g.out_bf16 ? run_db<true, true>(g, s) : run_db<false, true>(g, s);
    return g.out_bf16 ? run_db<true, false>(g, s) : run_db<false, false>(g, s);
}

}  // namespace fp4
