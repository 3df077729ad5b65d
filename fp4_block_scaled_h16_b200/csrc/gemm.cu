// gemm.cu -- block-scaled FP4 GEMM on the 5th-generation tensor cores of
// sm_100a (tcgen05.mma kind::mxf4 / kind::mxf4nvf4), for the Fprop, Dgrad and
// Wgrad GEMMs of a linear layer on FP4 operands ("Pre-addestramento di
// Modelli Linguistici di Grandi Dimensioni con MXFP4", Metodologia; NVFP4
// 16-groups: "TetraJet-v2" 2.A).
//
//   C[i, j] = alpha * sum_k qA[i, k] qB[j, k] sA[i, k / blk] sB[j, k / blk]
//
// Design (one CTA per SM, persistent over 128 x BN output tiles):
//   warp 0   TMA producer: 2-D tiled loads of the packed codes (128-byte
//            swizzle) and bulk copies of the 512-byte scale-factor atoms into
//            a ring of STAGES shared-memory stages of 256 K-elements each;
//   warp 1   allocates TMEM and issues, from one thread, the smem->TMEM
//            scale-factor copies and four 128 x BN x 64 block-scaled MMAs per
//            stage into an FP32 accumulator in TMEM;
//   warps 2-9 epilogue: two warps per TMEM lane quarter, each owning half of
//            the tile's columns; all of a warp's TMEM loads are issued back to
//            back, the accumulator is released to the MMA warp, and only then
//            are the values scaled by alpha, converted and stored, so the
//            stores overlap the next tile's mainloop.
// Every mbarrier wait is bounded; a wait that runs out sets the device error
// word to FP4_ERR_TIMEOUT, the CTA stops, lets every copy and MMA it issued
// land, frees its TMEM and exits.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <cstdint>
#include <mutex>

#include "internal.h"
#include "sm100.cuh"

namespace fp4 {

namespace {

constexpr int BM = 128;
constexpr int BK = 256;                 // K elements per stage (128 bytes of codes per row)
constexpr int STAGES = 4;
constexpr int NUM_THREADS = 320;
constexpr int EPI_WARPS = 8;
constexpr uint32_t TMEM_COLS = 512;
constexpr uint32_t DRAIN_LIMIT = 1u << 22;
constexpr unsigned int ERR_TIMEOUT = 7u;   // FP4_ERR_TIMEOUT

template <int FMT, int BN>
struct Cfg {
    static constexpr int BLK = (FMT == MXFP4) ? 32 : 16;        // elements per scale
    static constexpr int KB = BK / BLK;                          // scale bytes per row per stage
    static constexpr int ATOMS = KB / 4;                         // 512-byte atoms per 128 rows
    static constexpr uint32_t A_BYTES = BM * BK / 2;
    static constexpr uint32_t B_BYTES = BN * BK / 2;
    static constexpr uint32_t SFA_BYTES = BM * KB;
    static constexpr uint32_t SFB_BYTES = BN * KB;
    static constexpr uint32_t TX = A_BYTES + B_BYTES + SFA_BYTES + SFB_BYTES;
    static constexpr uint32_t STAGE_BYTES = (TX + 1023) / 1024 * 1024;
    static constexpr uint32_t SMEM = STAGES * STAGE_BYTES + 1024 /*align*/ + 256 /*barriers*/;
    static constexpr uint32_t SFA_COL = BN;                      // TMEM column of the A scales
    static constexpr uint32_t SFB_COL = BN + 4 * ATOMS;          // TMEM column of the B scales
    static constexpr uint32_t SFB_COLS_PER_ATOM = 4 * (BN / 128);
    static_assert(SFB_COL + SFB_COLS_PER_ATOM * ATOMS <= TMEM_COLS, "TMEM budget");
};

struct GemmParams {
    const uint8_t* a_sf;
    const uint8_t* b_sf;
    const float* a_ts;
    const float* b_ts;
    void* c;
    int64_t ldc;
    int M, N, K;
    int nb4;          // scale atoms per 128 rows along K
    int tiles_m, tiles_n;
    // work units: tiles [0, split_base) whole; the tiles after it (a last wave
    // that would fill at most half the SMs) as two halves of BN / 2 columns
    int units, split_base;
    uint32_t wait_limit;
    unsigned int* err;
};

__device__ __forceinline__ void raise_timeout(const GemmParams& p, volatile int* abort_flag) {
    *abort_flag = 1;
    atomicExch(p.err, ERR_TIMEOUT);
}

// output block of work unit u: rows m0.., columns n0.. (BN of them, or BN / 2
// for a half unit)
template <int BN>
__device__ __forceinline__ bool unit_geom(const GemmParams& p, int u, int& m0, int& n0) {
    int tm, tn;
    if (u < p.split_base) {
        tile_coords(u, p.tiles_m, p.tiles_n, tm, tn);
        m0 = tm * BM;
        n0 = tn * BN;
        return false;
    }
    const int t = p.split_base + ((u - p.split_base) >> 1);
    tile_coords(t, p.tiles_m, p.tiles_n, tm, tn);
    m0 = tm * BM;
    n0 = tn * BN + ((u - p.split_base) & 1) * (BN / 2);
    return true;
}

// one stage's scale-factor copies and MMAs into the accumulator at `tmem`,
// NMMA columns wide (BN, or BN / 2 for a half unit); a half-K stage (the last
// one when K is an odd multiple of 128) holds the first BK / 2 elements of K
// only: half the scale atoms, and the MMAs over its first two 64-K slices
template <int FMT, int BN, int NMMA>
__device__ __forceinline__ void mma_stage(uint32_t tmem, uint32_t st, int kt, bool half_k) {
    using G = Cfg<FMT, BN>;
    const uint32_t st_sfa = st + G::A_BYTES + G::B_BYTES;
    const uint32_t st_sfb = st_sfa + G::SFA_BYTES;
    const int atoms = half_k ? G::ATOMS / 2 : G::ATOMS;
    const int slices = half_k ? BK / 128 : BK / 64;
#pragma unroll
    for (int j = 0; j < G::ATOMS; ++j) {
        if (j >= atoms) break;
        sm100::tc_cp_sf(tmem + G::SFA_COL + 4 * j, sm100::desc_sf(st_sfa + 512 * j));
#pragma unroll
        for (int rb = 0; rb < NMMA / 128; ++rb)
            sm100::tc_cp_sf(tmem + G::SFB_COL + G::SFB_COLS_PER_ATOM * j + 4 * rb,
                            sm100::desc_sf(st_sfb + (rb * G::ATOMS + j) * 512));
    }
#pragma unroll
    for (int kk = 0; kk < BK / 64; ++kk) {
        if (kk >= slices) break;
        const uint64_t da = sm100::desc_sw128(st + 32 * kk);
        const uint64_t db = sm100::desc_sw128(st + G::A_BYTES + 32 * kk);
        const uint32_t acc = (kt > 0 || kk > 0) ? 1u : 0u;
        if (FMT == MXFP4) {
            // block 32: two scale bytes per MMA, the pair kk % 2 of atom kk / 2
            const int j = kk / 2;
            const uint32_t id = sm100::idesc_block_scaled(NMMA, true, (kk & 1) * 2, (kk & 1) * 2);
            sm100::mma_mxf4(tmem, da, db, id, tmem + G::SFA_COL + 4 * j,
                            tmem + G::SFB_COL + G::SFB_COLS_PER_ATOM * j, acc);
        } else {
            const uint32_t id = sm100::idesc_block_scaled(NMMA, false, 0, 0);
            sm100::mma_nvf4(tmem, da, db, id, tmem + G::SFA_COL + 4 * kk,
                            tmem + G::SFB_COL + G::SFB_COLS_PER_ATOM * kk, acc);
        }
    }
}

template <int FMT, int BN, bool OUT_BF16>
__global__ void __launch_bounds__(NUM_THREADS, 1)
gemm_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
            const __grid_constant__ CUtensorMap tmBh, const GemmParams p) {
    using G = Cfg<FMT, BN>;
    extern __shared__ uint8_t smem_raw[];
    // 1024-byte aligned base (the 128-byte swizzle atoms need it)
    const uint32_t raw = sm100::smem_u32(smem_raw);
    uint8_t* smem = smem_raw + ((1024u - (raw & 1023u)) & 1023u);
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + STAGES * G::STAGE_BYTES);
    uint64_t* empty = full + STAGES;
    uint64_t* acc_full = empty + STAGES;
    uint64_t* acc_empty = acc_full + 1;
    uint64_t* drain = acc_empty + 1;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; ++s) {
            sm100::mbar_init(&full[s], 1);
            sm100::mbar_init(&empty[s], 1);
        }
        sm100::mbar_init(acc_full, 1);
        sm100::mbar_init(acc_empty, EPI_WARPS);
        sm100::mbar_init(drain, 1);
        *abort_flag = 0;
        sm100::fence_barrier_init();
        sm100::prefetch_tmap(&tmA);
        sm100::prefetch_tmap(&tmB);
        if (p.units > p.split_base) sm100::prefetch_tmap(&tmBh);
    }
    if (warp == 1) {
        sm100::tmem_alloc(tmem_slot, TMEM_COLS);
        sm100::tmem_relinquish();
    }
    sm100::tc_fence_before();
    __syncthreads();
    sm100::tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    // stages per unit; with K an odd multiple of 128 the last one is half a
    // stage: its code boxes reach past K (the tensor maps fill zeros there)
    // and it carries half the scale atoms
    const int kt_count = (p.K + BK - 1) / BK;
    const bool ragged_k = (p.K % BK) != 0;

    if (warp == 0) {
        // ------------------------------------------------------------ producer
        if (sm100::elect_one()) {
            int stage = 0;
            uint32_t phase = 0;
            uint32_t fills = 0;           // fill i went to stage i % STAGES, phase i / STAGES
            bool ok = true;
            for (int u = blockIdx.x; u < p.units && ok; u += gridDim.x) {
                int m0, n0;
                const bool half_unit = unit_geom<BN>(p, u, m0, n0);
                for (int kt = 0; kt < kt_count; ++kt) {
                    if (!sm100::mbar_wait(&empty[stage], phase ^ 1u, p.wait_limit, abort_flag)) {
                        raise_timeout(p, abort_flag);
                        ok = false;
                        break;
                    }
                    uint8_t* st = smem + stage * G::STAGE_BYTES;
                    const int kb0 = kt * G::KB;                          // first scale column
                    const uint8_t* sfa = p.a_sf + ((int64_t)(m0 / 128) * p.nb4 + kb0 / 4) * 512;
                    // scale bytes per 128 rows in this stage (half of them in a half-K stage;
                    // the code boxes always count whole, zero-filled past K)
                    const uint32_t sf = (ragged_k && kt == kt_count - 1) ? G::ATOMS * 256 : G::ATOMS * 512;
                    if (BN == 256 && half_unit) {
                        // 128 columns: half of B and of its scales
                        sm100::mbar_arrive_expect_tx(&full[stage], G::A_BYTES + G::B_BYTES / 2 + 2 * sf);
                        sm100::tma_load_2d(st, &tmA, kt * (BK / 2), m0, &full[stage]);
                        sm100::tma_load_2d(st + G::A_BYTES, &tmBh, kt * (BK / 2), n0, &full[stage]);
                        sm100::bulk_load(st + G::A_BYTES + G::B_BYTES, sfa, sf, &full[stage]);
                        const uint8_t* sfb = p.b_sf + ((int64_t)(n0 / 128) * p.nb4 + kb0 / 4) * 512;
                        sm100::bulk_load(st + G::A_BYTES + G::B_BYTES + G::SFA_BYTES, sfb, sf, &full[stage]);
                    } else {
                        sm100::mbar_arrive_expect_tx(&full[stage], G::A_BYTES + G::B_BYTES + (1 + BN / 128) * sf);
                        sm100::tma_load_2d(st, &tmA, kt * (BK / 2), m0, &full[stage]);
                        sm100::tma_load_2d(st + G::A_BYTES, &tmB, kt * (BK / 2), n0, &full[stage]);
                        sm100::bulk_load(st + G::A_BYTES + G::B_BYTES, sfa, sf, &full[stage]);
#pragma unroll
                        for (int rb = 0; rb < BN / 128; ++rb) {
                            const uint8_t* sfb = p.b_sf + ((int64_t)(n0 / 128 + rb) * p.nb4 + kb0 / 4) * 512;
                            sm100::bulk_load(st + G::A_BYTES + G::B_BYTES + G::SFA_BYTES + rb * G::ATOMS * 512,
                                             sfb, sf, &full[stage]);
                        }
                    }
                    ++fills;
                    if (++stage == STAGES) { stage = 0; phase ^= 1u; }
                }
            }
            // drain: every fill issued must land before the CTA may exit; the
            // last fill of stage s had phase (fills - 1 - s) / STAGES
#pragma unroll
            for (int s = 0; s < STAGES; ++s)
                if (fills > (uint32_t)s)
                    sm100::mbar_wait(&full[s], ((fills - 1u - s) / STAGES) & 1u, DRAIN_LIMIT, nullptr);
        }
        __syncwarp();
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer
        if (sm100::elect_one()) {
            int stage = 0;
            uint32_t phase = 0, acc_phase = 0;
            bool ok = true, issued = false;
            for (int u = blockIdx.x; u < p.units && ok; u += gridDim.x) {
                const bool half_unit = u >= p.split_base;
                if (!sm100::mbar_wait(acc_empty, acc_phase ^ 1u, p.wait_limit, abort_flag)) {
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
                    const bool half_k = ragged_k && kt == kt_count - 1;
                    if (BN == 256 && half_unit) mma_stage<FMT, BN, (BN == 256 ? 128 : BN)>(tmem, st, kt, half_k);
                    else mma_stage<FMT, BN, BN>(tmem, st, kt, half_k);
                    issued = true;
                    sm100::tc_commit(&empty[stage]);          // stage free once these MMAs are done
                    if (++stage == STAGES) { stage = 0; phase ^= 1u; }
                }
                if (!ok) break;
                sm100::tc_commit(acc_full);                   // accumulator ready for the epilogue
                acc_phase ^= 1u;
            }
            if (issued) {
                sm100::tc_commit(drain);
                sm100::mbar_wait(drain, 0, DRAIN_LIMIT, nullptr);
            }
        }
        __syncwarp();
    } else {
        // ------------------------------------------------------------ epilogue
        constexpr int COLS = BN / 2;            // columns per epilogue warp
        const int q = warp & 3;                 // TMEM lane quarter this warp may access
        const int half = (warp - 2) >> 2;       // which half of the tile's columns
        float alpha = 1.0f;
        if (FMT == NVFP4) alpha = __fmul_rn(*p.a_ts, *p.b_ts);
        uint32_t acc_phase = 0;
        for (int u = blockIdx.x; u < p.units; u += gridDim.x) {
            int m0, n0;
            const bool half_unit = unit_geom<BN>(p, u, m0, n0);
            n0 += half * COLS;
            // a half unit has BN / 2 columns: the second column half's warps only hand over
            const bool idle = half_unit && half == 1;
            // one lane polls, the warp follows its verdict (the TMEM loads below
            // are warp-collective)
            int got = 0;
            if (lane == 0) {
                got = sm100::mbar_wait(acc_full, acc_phase, p.wait_limit, abort_flag) ? 1 : 0;
                if (!got) raise_timeout(p, abort_flag);
            }
            if (!__shfl_sync(0xffffffffu, got, 0)) break;
            if (idle) {
                __syncwarp();
                if (lane == 0) sm100::mbar_arrive(acc_empty);
                acc_phase ^= 1u;
                continue;
            }
            sm100::tc_fence_after();
            uint32_t r[COLS];
#pragma unroll
            for (int c = 0; c < COLS / 32; ++c) {
                uint32_t (&rr)[32] = *reinterpret_cast<uint32_t (*)[32]>(&r[32 * c]);
                sm100::tmem_ld32(tmem + ((uint32_t)(32 * q) << 16) + half * COLS + 32 * c, rr);
            }
            sm100::tmem_ld_wait();
            sm100::tc_fence_before();
            __syncwarp();
            if (lane == 0) sm100::mbar_arrive(acc_empty);          // the MMA may overwrite it now
            acc_phase ^= 1u;
            const int row = m0 + 32 * q + lane;
            if (OUT_BF16) {
                uint4* dst = reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(p.c) + (int64_t)row * p.ldc + n0);
#pragma unroll
                for (int v = 0; v < COLS / 8; ++v) {
                    uint32_t pk[4];
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const __nv_bfloat162 h = __floats2bfloat162_rn(__fmul_rn(__uint_as_float(r[8 * v + 2 * e]), alpha),
                                                                       __fmul_rn(__uint_as_float(r[8 * v + 2 * e + 1]), alpha));
                        pk[e] = *reinterpret_cast<const uint32_t*>(&h);
                    }
                    dst[v] = make_uint4(pk[0], pk[1], pk[2], pk[3]);
                }
            } else {
                float4* dst = reinterpret_cast<float4*>(static_cast<float*>(p.c) + (int64_t)row * p.ldc + n0);
#pragma unroll
                for (int v = 0; v < COLS / 4; ++v)
                    dst[v] = make_float4(__fmul_rn(__uint_as_float(r[4 * v]), alpha),
                                         __fmul_rn(__uint_as_float(r[4 * v + 1]), alpha),
                                         __fmul_rn(__uint_as_float(r[4 * v + 2]), alpha),
                                         __fmul_rn(__uint_as_float(r[4 * v + 3]), alpha));
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

// ---------------------------------------------------------------- host side

template <int FMT, int BN, bool OUT_BF16>
cudaError_t run(const GemmArgs& g, cudaStream_t s) {
    using G = Cfg<FMT, BN>;
    static PerDeviceOnce setup;
    const cudaError_t attr_err = setup.run([](int) {
        return cudaFuncSetAttribute(gemm_kernel<FMT, BN, OUT_BF16>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                    (int)G::SMEM);
    });
    if (attr_err != cudaSuccess) return attr_err;
    CUtensorMap ta, tb, tbh;
    if (!make_codes_map(&ta, g.a_codes, g.M, g.K, BM) || !make_codes_map(&tb, g.b_codes, g.N, g.K, BN) ||
        !make_codes_map(&tbh, g.b_codes, g.N, g.K, BN / 2))
        return cudaErrorInvalidValue;
    GemmParams p{};
    p.a_sf = g.a_scales;
    p.b_sf = g.b_scales;
    p.a_ts = g.a_ts;
    p.b_ts = g.b_ts;
    p.c = g.c;
    p.ldc = g.ldc;
    p.M = (int)g.M;
    p.N = (int)g.N;
    p.K = (int)g.K;
    p.nb4 = (int)(g.K / G::BLK / 4);
    p.tiles_m = (int)(g.M / BM);
    p.tiles_n = (int)(g.N / BN);
    p.wait_limit = g.wait_limit;
    p.err = device_error_word();
    const int tiles = p.tiles_m * p.tiles_n;
    const int grid = tiles < num_sms() ? tiles : num_sms();
    // a last wave that would leave more than half the SMs idle runs as half
    // tiles (BN = 256 only), so the tail takes about half as long
    const int full_waves = tiles / grid, tail = tiles - full_waves * grid;
    const bool split = BN == 256 && full_waves > 0 && tail > 0 && 2 * tail <= grid;
    p.split_base = split ? full_waves * grid : tiles;
    p.units = split ? p.split_base + 2 * tail : tiles;
    gemm_kernel<FMT, BN, OUT_BF16><<<grid, NUM_THREADS, G::SMEM, s>>>(ta, tb, tbh, p);
    return cudaGetLastError();
}

}  // namespace

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* f = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(f);
    });
    return fn;
}

// 2-D map over packed codes [rows, K/2] bytes, box = 128 bytes x box_rows, 128-byte swizzle
bool make_codes_map(CUtensorMap* m, const uint8_t* codes, int64_t rows, int64_t K, int box_rows) {
    auto fn = encode_fn();
    if (!fn) return false;
    cuuint64_t dims[2] = {(cuuint64_t)(K / 2), (cuuint64_t)rows};
    cuuint64_t strides[1] = {(cuuint64_t)(K / 2)};
    cuuint32_t box[2] = {128u, (cuuint32_t)box_rows};
    cuuint32_t estr[2] = {1u, 1u};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<uint8_t*>(codes), dims, strides, box, estr,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// 2-D map over C [M, N] (row pitch ldc) for the epilogue's tiled stores: box =
// 128 bytes of a row (64 bf16 or 32 fp32) x 32 rows, 128-byte swizzle
bool make_c_map(CUtensorMap* m, void* c, bool bf16, int64_t M, int64_t N, int64_t ldc) {
    auto fn = encode_fn();
    if (!fn) return false;
    const int64_t es = bf16 ? 2 : 4;
    cuuint64_t dims[2] = {(cuuint64_t)N, (cuuint64_t)M};
    cuuint64_t strides[1] = {(cuuint64_t)(ldc * es)};
    cuuint32_t box[2] = {(cuuint32_t)(128 / es), 32u};
    cuuint32_t estr[2] = {1u, 1u};
    return fn(m, bf16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, c, dims, strides, box,
              estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_NONE,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

bool make_input_map(CUtensorMap* m, const void* x, bool bf16, int64_t rows, int64_t cols, int64_t ld, bool swizzle128) {
    auto fn = encode_fn();
    if (!fn) return false;
    const int64_t es = bf16 ? 2 : 4;
    cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
    cuuint64_t strides[1] = {(cuuint64_t)(ld * es)};
    cuuint32_t box[2] = {64u, 128u};
    cuuint32_t estr[2] = {1u, 1u};
    return fn(m, bf16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, const_cast<void*>(x),
              dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
              (swizzle128 && bf16) ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_NONE,
              CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

cudaError_t launch_gemm(const GemmArgs& g, cudaStream_t s) {
    if (g.db) return launch_gemm_db(g, s);
    if (g.pairs && gemm_pair_fits(g)) return launch_gemm_pair(g, s);
    const bool n256 = (g.N % 256) == 0;
    if (g.fmt == MXFP4) {
        if (n256) return g.out_bf16 ? run<MXFP4, 256, true>(g, s) : run<MXFP4, 256, false>(g, s);
        return g.out_bf16 ? run<MXFP4, 128, true>(g, s) : run<MXFP4, 128, false>(g, s);
    }
    if (n256) return g.out_bf16 ? run<NVFP4, 256, true>(g, s) : run<NVFP4, 256, false>(g, s);
    return g.out_bf16 ? run<NVFP4, 128, true>(g, s) : run<NVFP4, 128, false>(g, s);
}

}  // namespace fp4
