// gemm_pair.cu -- the block-scaled FP4 GEMM of gemm.cu on CTA pairs: clusters
// of two CTAs on two SMs share each 256 x 256 output tile through tcgen05.mma
// with cta_group::2 (M = 256: rows 0-127 of the tile in the leader's TMEM,
// 128-255 in the peer's), for the Fprop, Dgrad and Wgrad GEMMs of a linear
// layer ("Pre-addestramento di Modelli Linguistici di Grandi Dimensioni con
// MXFP4", Metodologia; NVFP4 16-groups: "TetraJet-v2" 2.A).
//
//   C[i, j] = alpha * sum_k qA[i, k] qB[j, k] sA[i, k / blk] sB[j, k / blk]
//
// Each CTA loads only its own 128 rows of A and its half (128 rows) of the
// tile's B, and the MMA reads B from both CTAs' shared memory.  The operand
// bytes per FLOP are two thirds of those of the single-CTA 128 x 256 tile.
// No load uses cluster multicast: every CTA fetches its own bytes.
//
// Roles (both CTAs, one CTA per SM, persistent over pair tiles):
//   warp 0   TMA producer: 2-D loads of the packed codes (128-byte swizzle)
//            and 3-D loads of the 512-byte scale atoms (its A rows' scales;
//            all 256 columns' B scales, which each CTA's MMA half needs)
//            into a ring of stages.  Every load's bytes are counted on the
//            leader's "full" barrier of the stage (cta_group::2 form), which
//            the leader's producer arms with both CTAs' bytes;
//   warp 1   TMEM (allocated for the pair); in the leader, one thread issues
//            the scale copies and the MMAs of both CTAs and commits each
//            stage's release to both CTAs' "empty" barriers, and each tile's
//            accumulator to both CTAs' "acc_full" barriers;
//   warps 2-9 epilogue of this CTA's 128 rows; after their TMEM loads both
//            CTAs' epilogue warps arrive on the leader's "acc_empty", then
//            scale and convert, write 32-row x 128-byte boxes of C into
//            shared memory (128-byte swizzle, no bank conflicts) and store
//            each with one TMA tiled store, so every row reaches L2 as whole
//            128-byte lines.
// Every wait is bounded.  A wait that runs out sets the device error word to
// FP4_ERR_TIMEOUT and the CTA stops; before either CTA exits, the leader makes
// sure every load issued by either CTA has landed (the peer reports how many
// stages it filled) and that its MMAs are complete, and a cluster barrier
// keeps the peer's shared memory and TMEM alive until then.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <cstdint>

#include "internal.h"
#include "sm100.cuh"

namespace fp4 {

namespace {

constexpr int PM = 256;                  // rows of C per pair tile (128 per CTA)
constexpr int PN = 256;                  // columns of C per pair tile
constexpr int BK = 256;                  // K elements per stage
constexpr int NUM_THREADS = 320;
constexpr int EPI_WARPS = 8;
constexpr uint32_t TMEM_COLS = 512;
constexpr uint32_t DRAIN_LIMIT = 1u << 22;
constexpr unsigned int ERR_TIMEOUT = 7u;   // FP4_ERR_TIMEOUT
constexpr uint32_t SMEM_LIMIT = 232448;    // opt-in shared memory per block
constexpr uint32_t EPI_BUF = 4096;         // per epilogue warp: one 32-row x 128-byte box of C

template <int FMT>
struct PCfg {
    static constexpr int BLK = (FMT == MXFP4) ? 32 : 16;        // elements per scale
    static constexpr int KB = BK / BLK;                          // scale bytes per row per stage
    static constexpr int ATOMS = KB / 4;                         // 512-byte atoms per 128 rows per stage
    static constexpr uint32_t A_BYTES = 128 * BK / 2;            // this CTA's 128 rows of A
    static constexpr uint32_t B_BYTES = 128 * BK / 2;            // this CTA's 128 rows of B
    static constexpr uint32_t SFA_BYTES = 128 * KB;
    static constexpr uint32_t SFB_BYTES = PN * KB;               // the scales of all 256 columns
    static constexpr uint32_t STAGE_BYTES = A_BYTES + B_BYTES + SFA_BYTES + SFB_BYTES;
    static constexpr uint32_t EXTRA = 1024 /*align*/ + EPI_WARPS * EPI_BUF + 256 /*barriers*/;
    static constexpr int FIT = (int)((SMEM_LIMIT - EXTRA) / STAGE_BYTES);
    static constexpr int STAGES = FIT > 6 ? 6 : FIT;             // 5 for both formats
    static constexpr uint32_t SMEM = STAGES * STAGE_BYTES + EXTRA;
    static constexpr uint32_t SFA_COL = PN;                      // TMEM column of the A scales
    static constexpr uint32_t SFB_COL = PN + 4 * ATOMS;          // TMEM column of the B scales
    static_assert(STAGE_BYTES % 1024 == 0, "stages keep the 1024-byte alignment of the swizzle atoms");
    static_assert(SFB_COL + 8 * ATOMS <= TMEM_COLS, "TMEM budget");
    static_assert(2 * STAGES * 8 + 4 * 8 + 12 <= 256, "barrier block");
};

struct PairParams {
    const float* a_ts;
    const float* b_ts;
    int K;
    int tiles_m, tiles_n;    // pair tiles
    // work units: tiles [0, split_base) whole; the tiles after it (a last wave
    // that would keep at most half the pairs busy) as two 256 x 128 halves
    int units, split_base;
    uint32_t wait_limit;
    unsigned int* err;
};

// output block of work unit u: rows m0 .. m0+255, columns n0 .. (256 of them,
// or 128 for a half unit)
__device__ __forceinline__ bool pair_unit(const PairParams& p, int u, int& m0, int& n0) {
    int tm, tn;
    if (u < p.split_base) {
        tile_coords(u, p.tiles_m, p.tiles_n, tm, tn);
        m0 = tm * PM;
        n0 = tn * PN;
        return false;
    }
    const int t = p.split_base + ((u - p.split_base) >> 1);
    tile_coords(t, p.tiles_m, p.tiles_n, tm, tn);
    m0 = tm * PM;
    n0 = tn * PN + ((u - p.split_base) & 1) * (PN / 2);
    return true;
}

__device__ __forceinline__ void raise_timeout(const PairParams& p, volatile int* abort_flag) {
    *abort_flag = 1;
    atomicExch(p.err, ERR_TIMEOUT);
}

// one stage's scale copies and MMAs, issued by the leader for both CTAs;
// NMMA = 256, or 128 for a half unit (each CTA's first 64 rows of B; the
// scales of its 128 columns are the first of the two row blocks copied)
template <int FMT, int NMMA>
__device__ __forceinline__ void mma_stage_pair(uint32_t tmem, uint32_t st, int kt) {
    using G = PCfg<FMT>;
    const uint32_t st_sfa = st + G::A_BYTES + G::B_BYTES;
    const uint32_t st_sfb = st_sfa + G::SFA_BYTES;
#pragma unroll
    for (int j = 0; j < G::ATOMS; ++j) {
        sm100::tc_cp_sf_pair(tmem + G::SFA_COL + 4 * j, sm100::desc_sf(st_sfa + 512 * j));
#pragma unroll
        for (int rb = 0; rb < 2; ++rb)
            sm100::tc_cp_sf_pair(tmem + G::SFB_COL + 8 * j + 4 * rb,
                                 sm100::desc_sf(st_sfb + (rb * G::ATOMS + j) * 512));
    }
#pragma unroll
    for (int kk = 0; kk < BK / 64; ++kk) {
        const uint64_t da = sm100::desc_sw128(st + 32 * kk);
        const uint64_t db = sm100::desc_sw128(st + G::A_BYTES + 32 * kk);
        const uint32_t acc = (kt > 0 || kk > 0) ? 1u : 0u;
        if (FMT == MXFP4) {
            const int j = kk / 2;
            const uint32_t id = sm100::idesc_block_scaled(NMMA, true, (kk & 1) * 2, (kk & 1) * 2, PM);
            sm100::mma_mxf4_pair(tmem, da, db, id, tmem + G::SFA_COL + 4 * j, tmem + G::SFB_COL + 8 * j, acc);
        } else {
            const uint32_t id = sm100::idesc_block_scaled(NMMA, false, 0, 0, PM);
            sm100::mma_nvf4_pair(tmem, da, db, id, tmem + G::SFA_COL + 4 * kk, tmem + G::SFB_COL + 8 * kk, acc);
        }
    }
}

template <int FMT, bool OUT_BF16>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(NUM_THREADS, 1)
gemm_pair_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                 const __grid_constant__ CUtensorMap tmSA, const __grid_constant__ CUtensorMap tmSB,
                 const __grid_constant__ CUtensorMap tmC, const PairParams p) {
    using G = PCfg<FMT>;
    extern __shared__ uint8_t smem_raw[];
    // 1024-byte aligned base; the same offset in both CTAs, which the pair MMA
    // and the multicast commits rely on
    const uint32_t raw = sm100::smem_u32(smem_raw);
    uint8_t* smem = smem_raw + ((1024u - (raw & 1023u)) & 1023u);
    uint8_t* epi_bufs = smem + G::STAGES * G::STAGE_BYTES;      // 1024-byte aligned
    uint64_t* full = reinterpret_cast<uint64_t*>(epi_bufs + EPI_WARPS * EPI_BUF);
    uint64_t* empty = full + G::STAGES;
    uint64_t* acc_full = empty + G::STAGES;
    uint64_t* acc_empty = acc_full + 1;
    uint64_t* drain = acc_empty + 1;
    uint64_t* peer_done = drain + 1;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(peer_done + 1);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
    volatile uint32_t* peer_fills = reinterpret_cast<volatile uint32_t*>(tmem_slot + 2);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t rank = sm100::cluster_rank();
    const int pair = (int)(blockIdx.x >> 1), pairs = (int)(gridDim.x >> 1);
    const int units = p.units;
    const int kt_count = (p.K + BK - 1) / BK;   // a ragged last stage reads zeros past K

    if (threadIdx.x == 0) {
        for (int s = 0; s < G::STAGES; ++s) {
            sm100::mbar_init(&full[s], 1);
            sm100::mbar_init(&empty[s], 1);
        }
        sm100::mbar_init(acc_full, 1);
        sm100::mbar_init(acc_empty, 2 * EPI_WARPS);
        sm100::mbar_init(drain, 1);
        sm100::mbar_init(peer_done, 1);
        *abort_flag = 0;
        *peer_fills = 0;
        sm100::fence_barrier_init();
        sm100::prefetch_tmap(&tmA);
        sm100::prefetch_tmap(&tmB);
        sm100::prefetch_tmap(&tmSA);
        sm100::prefetch_tmap(&tmSB);
        sm100::prefetch_tmap(&tmC);
    }
    if (warp == 1) {
        sm100::tmem_alloc_pair(tmem_slot, TMEM_COLS);
        sm100::tmem_relinquish_pair();
    }
    sm100::tc_fence_before();
    sm100::cluster_sync();        // both CTAs' barriers initialised before any load signals them
    sm100::tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    if (warp == 0) {
        // ------------------------------------------------------------ producer
        if (sm100::elect_one()) {
            int stage = 0;
            uint32_t phase = 0;
            uint32_t fills = 0;           // fill i went to stage i % STAGES, phase i / STAGES
            bool ok = true;
            for (int u = pair; u < units && ok; u += pairs) {
                int m0, nb;                                   // first row and column of the unit
                const bool half_unit = pair_unit(p, u, m0, nb);
                const int ma = m0 + 128 * (int)rank;          // this CTA's rows of A
                // this CTA's rows of B: 128 of a whole tile; for a half unit the
                // MMA reads the first 64 of the box (the rest, past the unit or
                // zero-filled past N, keeps every fill the same size)
                const int nbc = nb + (half_unit ? 64 : 128) * (int)rank;
                for (int kt = 0; kt < kt_count; ++kt) {
                    if (!sm100::mbar_wait(&empty[stage], phase ^ 1u, p.wait_limit, abort_flag)) {
                        raise_timeout(p, abort_flag);
                        ok = false;
                        break;
                    }
                    uint8_t* st = smem + stage * G::STAGE_BYTES;
                    const uint32_t bar = sm100::cluster_addr(&full[stage], 0);
                    if (rank == 0) sm100::mbar_arrive_expect_tx(&full[stage], 2 * G::STAGE_BYTES);
                    sm100::tma_load_2d_pair(st, &tmA, kt * (BK / 2), ma, bar);
                    sm100::tma_load_2d_pair(st + G::A_BYTES, &tmB, kt * (BK / 2), nbc, bar);
                    sm100::tma_load_3d_pair(st + G::A_BYTES + G::B_BYTES, &tmSA, 0, kt * 2 * G::ATOMS, ma / 128, bar);
                    sm100::tma_load_3d_pair(st + G::A_BYTES + G::B_BYTES + G::SFA_BYTES, &tmSB, 0,
                                            kt * 2 * G::ATOMS, nb / 128, bar);
                    ++fills;
                    if (++stage == G::STAGES) { stage = 0; phase ^= 1u; }
                }
            }
            if (rank == 1) {
                // report the fills to the leader, whose barriers count their bytes
                sm100::st_cluster_u32(sm100::cluster_addr(const_cast<uint32_t*>(peer_fills), 0), fills);
                sm100::mbar_arrive_cluster(sm100::cluster_addr(peer_done, 0));
            } else {
                // After a timeout the two producers may have filled different
                // numbers of stages (at most STAGES apart).  Complete the
                // bookkeeping of every fill either CTA issued, then wait for
                // the last phase of every stage: once it completes, every byte
                // either CTA asked for has landed.
                uint32_t pf = fills;
                if (sm100::mbar_wait_cluster(peer_done, 0, DRAIN_LIMIT, nullptr)) pf = *peer_fills;
                else raise_timeout(p, abort_flag);
                const uint32_t lf = fills;
                for (uint32_t i = lf; i < pf; ++i) {          // the peer's half only: expect it
                    const uint32_t s = i % G::STAGES;
                    if (i >= (uint32_t)G::STAGES)
                        sm100::mbar_wait(&full[s], ((i - G::STAGES) / G::STAGES) & 1u, DRAIN_LIMIT, nullptr);
                    sm100::mbar_arrive_expect_tx(&full[s], G::STAGE_BYTES);
                }
                for (uint32_t i = pf; i < lf; ++i) {          // this CTA's half only: the peer's never comes
                    const uint32_t s = i % G::STAGES;
                    if (i >= (uint32_t)G::STAGES)
                        sm100::mbar_wait(&full[s], ((i - G::STAGES) / G::STAGES) & 1u, DRAIN_LIMIT, nullptr);
                    sm100::mbar_complete_tx(&full[s], G::STAGE_BYTES);
                }
                const uint32_t last = lf > pf ? lf : pf;
#pragma unroll
                for (int s = 0; s < G::STAGES; ++s)
                    if (last > (uint32_t)s)
                        sm100::mbar_wait(&full[s], ((last - 1u - s) / G::STAGES) & 1u, DRAIN_LIMIT, nullptr);
            }
        }
        __syncwarp();
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer (leader)
        if (rank == 0 && sm100::elect_one()) {
            int stage = 0;
            uint32_t phase = 0, acc_phase = 0;
            bool ok = true, issued = false;
            for (int u = pair; u < units && ok; u += pairs) {
                const bool half_unit = u >= p.split_base;
                if (!sm100::mbar_wait_cluster(acc_empty, acc_phase ^ 1u, p.wait_limit, abort_flag)) {
                    raise_timeout(p, abort_flag);
                    break;
                }
                sm100::tc_fence_after();
                for (int kt = 0; kt < kt_count; ++kt) {
                    if (!sm100::mbar_wait(&full[stage], phase, p.wait_limit, abort_flag)) {
                        raise_timeout(p, abort_flag);
                        ok = false;
                        break;
                    }
                    sm100::tc_fence_after();
                    const uint32_t st = sm100::smem_u32(smem + stage * G::STAGE_BYTES);
                    if (half_unit) mma_stage_pair<FMT, PN / 2>(tmem, st, kt);
                    else mma_stage_pair<FMT, PN>(tmem, st, kt);
                    issued = true;
                    sm100::tc_commit_pair_both(&empty[stage]);   // both CTAs' stage free once these MMAs are done
                    if (++stage == G::STAGES) { stage = 0; phase ^= 1u; }
                }
                if (!ok) break;
                sm100::tc_commit_pair_both(acc_full);            // both halves of the tile ready
                acc_phase ^= 1u;
            }
            if (issued) {
                sm100::tc_commit_pair_local(drain);
                sm100::mbar_wait(drain, 0, DRAIN_LIMIT, nullptr);
            }
        }
        __syncwarp();
    } else {
        // ------------------------------------------------------------ epilogue (this CTA's 128 rows)
        constexpr int COLS = PN / 2;                    // columns per epilogue warp
        constexpr int BOX_COLS = OUT_BF16 ? 64 : 32;    // 128 bytes of a row
        const int q = warp & 3;                 // TMEM lane quarter this warp may access
        const int half = (warp - 2) >> 2;       // which half of the tile's columns
        uint8_t* buf = epi_bufs + (warp - 2) * EPI_BUF;
        const uint32_t buf_s = sm100::smem_u32(buf);
        float alpha = 1.0f;
        if (FMT == NVFP4) alpha = __fmul_rn(*p.a_ts, *p.b_ts);
        const uint32_t leader_acc_empty = sm100::cluster_addr(acc_empty, 0);
        uint32_t acc_phase = 0;
        for (int u = pair; u < units; u += pairs) {
            int m0, nu;
            const bool half_unit = pair_unit(p, u, m0, nu);
            // a half unit has 128 columns: the second column half's warps only hand over
            const bool idle = half_unit && half == 1;
            int got = 0;
            if (lane == 0) {
                got = sm100::mbar_wait(acc_full, acc_phase, p.wait_limit, abort_flag) ? 1 : 0;
                if (!got) raise_timeout(p, abort_flag);
            }
            if (!__shfl_sync(0xffffffffu, got, 0)) break;
            sm100::tc_fence_after();
            uint32_t r[COLS];
            if (!idle) {
#pragma unroll
                for (int c = 0; c < COLS / 32; ++c) {
                    uint32_t (&rr)[32] = *reinterpret_cast<uint32_t (*)[32]>(&r[32 * c]);
                    sm100::tmem_ld32(tmem + ((uint32_t)(32 * q) << 16) + half * COLS + 32 * c, rr);
                }
                sm100::tmem_ld_wait();
            }
            sm100::tc_fence_before();
            __syncwarp();
            if (lane == 0) sm100::mbar_arrive_cluster(leader_acc_empty);   // the MMA may overwrite it now
            acc_phase ^= 1u;
            if (idle) continue;
            // rows row0 .. row0 + 31 (lane = row), columns n0 .. n0 + COLS - 1
            const int row0 = m0 + 128 * (int)rank + 32 * q;
            const int n0 = nu + half * COLS;
#pragma unroll
            for (int b = 0; b < COLS / BOX_COLS; ++b) {
                if (lane == 0) sm100::bulk_wait_read0();        // the previous box has left the buffer
                __syncwarp();
#pragma unroll
                for (int c = 0; c < 8; ++c) {                    // 16-byte chunk c of this lane's row
                    uint32_t w[4];
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        if (OUT_BF16) {
                            const int i = b * BOX_COLS + 8 * c + 2 * e;
                            const __nv_bfloat162 h = __floats2bfloat162_rn(__fmul_rn(__uint_as_float(r[i]), alpha),
                                                                           __fmul_rn(__uint_as_float(r[i + 1]), alpha));
                            w[e] = *reinterpret_cast<const uint32_t*>(&h);
                        } else {
                            w[e] = __float_as_uint(__fmul_rn(__uint_as_float(r[b * BOX_COLS + 4 * c + e]), alpha));
                        }
                    }
                    // 128-byte swizzle: chunk c of row `lane` sits at chunk c ^ (lane % 8)
                    sm100::st_shared_v4(buf_s + lane * 128 + ((c ^ (lane & 7)) << 4), w[0], w[1], w[2], w[3]);
                }
                sm100::fence_proxy_async_smem();
                __syncwarp();
                if (lane == 0) {
                    sm100::tma_store_2d(&tmC, buf, n0 + b * BOX_COLS, row0);
                    sm100::bulk_commit();
                }
            }
        }
        if (lane == 0) sm100::bulk_wait0();     // this warp's stores are complete before the CTA leaves
        __syncwarp();
    }

    // neither CTA frees its TMEM or leaves while the leader's MMAs or either
    // CTA's loads may still touch it
    sm100::tc_fence_before();
    sm100::cluster_sync();
    if (warp == 1) {
        __syncwarp();
        sm100::tc_fence_after();
        sm100::tmem_dealloc_pair(tmem, TMEM_COLS);
    }
}

// 3-D map over the scale atoms of one operand: [row blocks][atoms along K][512 B]
// seen as [row blocks][2 * atoms][256 B]; a box of `rb` row blocks x
// `halves` 256-byte halves lands as [rb][halves][256] (the MMA's atom order)
bool make_sf_map(CUtensorMap* m, const uint8_t* sf, int64_t row_blocks, int64_t nb4, int halves, int rb) {
    auto fn = encode_fn();
    if (!fn) return false;
    cuuint64_t dims[3] = {256u, (cuuint64_t)(2 * nb4), (cuuint64_t)row_blocks};
    cuuint64_t strides[2] = {256u, (cuuint64_t)(nb4 * 512)};
    cuuint32_t box[3] = {256u, (cuuint32_t)halves, (cuuint32_t)rb};
    cuuint32_t estr[3] = {1u, 1u, 1u};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<uint8_t*>(sf), dims, strides, box, estr,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int FMT, bool OUT_BF16>
cudaError_t run_pair(const GemmArgs& g, cudaStream_t s) {
    using G = PCfg<FMT>;
    static PerDeviceOnce setup;
    static int max_pairs[kOnceDevices] = {};
    int dev = 0;
    const cudaError_t attr_err = setup.run([](int d) {
        cudaError_t e = cudaFuncSetAttribute(gemm_pair_kernel<FMT, OUT_BF16>,
                                             cudaFuncAttributeMaxDynamicSharedMemorySize, (int)G::SMEM);
        if (e != cudaSuccess) return e;
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3(2 * 512);
        cfg.blockDim = dim3(NUM_THREADS);
        cfg.dynamicSmemBytes = G::SMEM;
        int n = 0;
        e = cudaOccupancyMaxActiveClusters(&n, gemm_pair_kernel<FMT, OUT_BF16>, &cfg);
        if (e != cudaSuccess) return e;
        max_pairs[d] = n;
        return n > 0 ? cudaSuccess : cudaErrorInvalidConfiguration;
    }, &dev);
    if (attr_err != cudaSuccess) return attr_err;
    const int64_t nb4 = g.K / G::BLK / 4;
    CUtensorMap ta, tb, tsa, tsb, tc;
    if (!make_codes_map(&ta, g.a_codes, g.M, g.K, 128) || !make_codes_map(&tb, g.b_codes, g.N, g.K, 128) ||
        !make_sf_map(&tsa, g.a_scales, g.M / 128, nb4, 2 * G::ATOMS, 1) ||
        !make_sf_map(&tsb, g.b_scales, g.N / 128, nb4, 2 * G::ATOMS, 2) ||
        !make_c_map(&tc, g.c, OUT_BF16, g.M, g.N, g.ldc))
        return cudaErrorInvalidValue;
    PairParams p{};
    p.a_ts = g.a_ts;
    p.b_ts = g.b_ts;
    p.K = (int)g.K;
    p.tiles_m = (int)(g.M / PM);
    p.tiles_n = (int)(g.N / PN);
    p.wait_limit = g.wait_limit;
    p.err = device_error_word();
    const int tiles = p.tiles_m * p.tiles_n;
    const int pairs = tiles < max_pairs[dev] ? tiles : max_pairs[dev];
    // a last wave that would leave more than half the pairs idle runs as half
    // tiles, so the tail takes about half as long
    const int full_waves = tiles / pairs, tail = tiles - full_waves * pairs;
    const bool split = full_waves > 0 && tail > 0 && 2 * tail <= pairs;
    p.split_base = split ? full_waves * pairs : tiles;
    p.units = split ? p.split_base + 2 * tail : tiles;
    gemm_pair_kernel<FMT, OUT_BF16><<<2 * pairs, NUM_THREADS, G::SMEM, s>>>(ta, tb, tsa, tsb, tc, p);
    return cudaGetLastError();
}

}  // namespace

bool gemm_pair_fits(const GemmArgs& g) {
    return !g.db && g.M % PM == 0 && g.N % PN == 0 && g.M > 0 && g.N > 0 && g.K > 0;
}

cudaError_t launch_gemm_pair(const GemmArgs& g, cudaStream_t s) {
    if (g.fmt == MXFP4) return g.out_bf16 ? run_pair<MXFP4, true>(g, s) : run_pair<MXFP4, false>(g, s);
    return g.out_bf16 ? run_pair<NVFP4, true>(g, s) : run_pair<NVFP4, false>(g, s);
}

}  // namespace fp4
