// gemm_outctl.cu -- the GEMM of OutControl's split operands ("TetraJet-v2"
// 2.C: the top p% of activation channels in FP8, the rest in FP4):
//
//   C[i, j] = a4 b4 sum_{k < K}  qA[i, k] qB[j, k] sA[i, k/16] sB[j, k/16]
//           + a8 b8 sum_{k < K8} eA[i, k] eB[j, k]
//
// with the NVFP4 parts (the channels zeroed) and the E4M3 parts (the channels
// gathered, under one tensor scale per operand).  Both sums run on the tensor
// cores into two TMEM accumulators of one 128 x 128 tile: the FP4 stages with
// tcgen05 kind::mxf4nvf4 (E4M3 block scales in TMEM), then the FP8 stages with
// kind::f8f6f4.  The epilogue forms a4 b4 acc4 + a8 b8 acc8 once per element
// and rounds the output once.  The pipeline is the plain GEMM's: one CTA per
// SM, persistent over tiles; warp 0 the TMA producer, warp 1 the MMA issuer,
// warps 2-9 the epilogue; every wait bounded, with the same abort protocol.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <cstdint>

#include "internal.h"
#include "sm100.cuh"

namespace fp4 {

namespace {

constexpr int BM = 128, BN = 128, BK = 256, BK8 = 128;   // K per FP4 stage / per FP8 stage
constexpr int STAGES = 5;
constexpr int NUM_THREADS = 320;
constexpr int EPI_WARPS = 8;
constexpr uint32_t TMEM_COLS = 512;
constexpr uint32_t DRAIN_LIMIT = 1u << 22;
constexpr unsigned int ERR_TIMEOUT = 7u;

constexpr uint32_t A_BYTES = BM * 128, B_BYTES = BN * 128;         // 128 bytes of K per row in either format
constexpr uint32_t SF_BYTES = 128 * (BK / 16);                     // one operand's scale bytes per FP4 stage
constexpr uint32_t STAGE_BYTES = (A_BYTES + B_BYTES + 2 * SF_BYTES + 1023) / 1024 * 1024;
constexpr uint32_t SMEM = STAGES * STAGE_BYTES + 1024 + 256;
constexpr uint32_t SFA_COL = BN, SFB_COL = BN + 16, ACC8_COL = 256;   // TMEM columns

struct OcParams {
    const uint8_t* a_sf;
    const uint8_t* b_sf;
    const float* a_ts;
    const float* b_ts;
    const float* a_s8;
    const float* b_s8;
    void* c;
    int64_t ldc;
    int M, N, K, K8;
    int nb4;
    int tiles_m, tiles_n;
    uint32_t wait_limit;
    unsigned int* err;
};

__device__ __forceinline__ void raise_timeout(const OcParams& p, volatile int* abort_flag) {
    *abort_flag = 1;
    atomicExch(p.err, ERR_TIMEOUT);
}

template <bool OUT_BF16>
__global__ void __launch_bounds__(NUM_THREADS, 1)
gemm_outctl_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                   const __grid_constant__ CUtensorMap tmA8, const __grid_constant__ CUtensorMap tmB8,
                   const OcParams p) {
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw = sm100::smem_u32(smem_raw);
    uint8_t* smem = smem_raw + ((1024u - (raw & 1023u)) & 1023u);
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + STAGES * STAGE_BYTES);
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
        if (p.K8 > 0) {
            sm100::prefetch_tmap(&tmA8);
            sm100::prefetch_tmap(&tmB8);
        }
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
    const int kt4 = (p.K + BK - 1) / BK;              // FP4 stages (the last one half when K % 256 == 128)
    const bool ragged_k = (p.K % BK) != 0;
    const int kt8 = p.K8 / BK8;                       // FP8 stages

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
                for (int kt = 0; kt < kt4 + kt8; ++kt) {
                    if (!sm100::mbar_wait(&empty[stage], phase ^ 1u, p.wait_limit, abort_flag)) {
                        raise_timeout(p, abort_flag);
                        ok = false;
                        break;
                    }
                    uint8_t* st = smem + stage * STAGE_BYTES;
                    if (kt < kt4) {
                        const uint32_t sf = (ragged_k && kt == kt4 - 1) ? SF_BYTES / 2 : SF_BYTES;
                        sm100::mbar_arrive_expect_tx(&full[stage], A_BYTES + B_BYTES + 2 * sf);
                        sm100::tma_load_2d(st, &tmA, kt * (BK / 2), m0, &full[stage]);
                        sm100::tma_load_2d(st + A_BYTES, &tmB, kt * (BK / 2), n0, &full[stage]);
                        const int kb0 = kt * (BK / 16);
                        sm100::bulk_load(st + A_BYTES + B_BYTES, p.a_sf + ((int64_t)(m0 / 128) * p.nb4 + kb0 / 4) * 512,
                                         sf, &full[stage]);
                        sm100::bulk_load(st + A_BYTES + B_BYTES + SF_BYTES,
                                         p.b_sf + ((int64_t)(n0 / 128) * p.nb4 + kb0 / 4) * 512, sf, &full[stage]);
                    } else {
                        const int k8 = kt - kt4;
                        sm100::mbar_arrive_expect_tx(&full[stage], A_BYTES + B_BYTES);
                        sm100::tma_load_2d(st, &tmA8, k8 * BK8, m0, &full[stage]);
                        sm100::tma_load_2d(st + A_BYTES, &tmB8, k8 * BK8, n0, &full[stage]);
                    }
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
            int stage = 0;
            uint32_t phase = 0, acc_phase = 0;
            bool ok = true, issued = false;
            const uint32_t id4 = sm100::idesc_block_scaled(BN, false, 0, 0);
            const uint32_t id8 = sm100::idesc_f8_e4m3(BN);
            for (int t = blockIdx.x; t < tiles && ok; t += gridDim.x) {
                if (!sm100::mbar_wait(acc_empty, acc_phase ^ 1u, p.wait_limit, abort_flag)) {
                    raise_timeout(p, abort_flag);
                    break;
                }
                sm100::tc_fence_after();
                for (int kt = 0; kt < kt4 + kt8; ++kt) {
                    if (!sm100::mbar_wait(&full[stage], phase, p.wait_limit, abort_flag)) {
                        raise_timeout(p, abort_flag);
                        ok = false;
                        break;
                    }
                    sm100::tc_fence_after();
                    const uint32_t st = sm100::smem_u32(smem + stage * STAGE_BYTES);
                    if (kt < kt4) {
                        const bool half_k = ragged_k && kt == kt4 - 1;
                        const uint32_t st_sfa = st + A_BYTES + B_BYTES, st_sfb = st_sfa + SF_BYTES;
                        const int atoms = half_k ? 2 : 4;
#pragma unroll
                        for (int j = 0; j < 4; ++j) {
                            if (j >= atoms) break;
                            sm100::tc_cp_sf(tmem + SFA_COL + 4 * j, sm100::desc_sf(st_sfa + 512 * j));
                            sm100::tc_cp_sf(tmem + SFB_COL + 4 * j, sm100::desc_sf(st_sfb + 512 * j));
                        }
#pragma unroll
                        for (int kk = 0; kk < BK / 64; ++kk) {
                            if (kk >= (half_k ? 2 : 4)) break;
                            sm100::mma_nvf4(tmem, sm100::desc_sw128(st + 32 * kk), sm100::desc_sw128(st + A_BYTES + 32 * kk),
                                            id4, tmem + SFA_COL + 4 * kk, tmem + SFB_COL + 4 * kk,
                                            (kt > 0 || kk > 0) ? 1u : 0u);
                        }
                    } else {
                        const int k8 = kt - kt4;
#pragma unroll
                        for (int kk = 0; kk < BK8 / 32; ++kk)
                            sm100::mma_f8(tmem + ACC8_COL, sm100::desc_sw128(st + 32 * kk),
                                          sm100::desc_sw128(st + A_BYTES + 32 * kk), id8, (k8 > 0 || kk > 0) ? 1u : 0u);
                    }
                    issued = true;
                    sm100::tc_commit(&empty[stage]);
                    if (++stage == STAGES) { stage = 0; phase ^= 1u; }
                }
                if (!ok) break;
                sm100::tc_commit(acc_full);
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
        const int q = warp & 3;
        const int half = (warp - 2) >> 2;
        const float a4 = __fmul_rn(*p.a_ts, *p.b_ts);
        const float a8 = p.K8 > 0 ? __fmul_rn(*p.a_s8, *p.b_s8) : 0.0f;
        uint32_t acc_phase = 0;
        for (int t = blockIdx.x; t < tiles; t += gridDim.x) {
            int tm_, tn_;
                tile_coords(t, p.tiles_m, p.tiles_n, tm_, tn_);
                const int m0 = tm_ * BM, n0 = tn_ * BN + half * COLS;
            int got = 0;
            if (lane == 0) {
                got = sm100::mbar_wait(acc_full, acc_phase, p.wait_limit, abort_flag) ? 1 : 0;
                if (!got) raise_timeout(p, abort_flag);
            }
            if (!__shfl_sync(0xffffffffu, got, 0)) break;
            sm100::tc_fence_after();
            uint32_t r4[COLS], r8[COLS];
            const uint32_t lane_base = tmem + ((uint32_t)(32 * q) << 16) + half * COLS;
#pragma unroll
            for (int cch = 0; cch < COLS / 32; ++cch) {
                uint32_t (&rr)[32] = *reinterpret_cast<uint32_t (*)[32]>(&r4[32 * cch]);
                sm100::tmem_ld32(lane_base + 32 * cch, rr);
            }
            if (p.K8 > 0) {
#pragma unroll
                for (int cch = 0; cch < COLS / 32; ++cch) {
                    uint32_t (&rr)[32] = *reinterpret_cast<uint32_t (*)[32]>(&r8[32 * cch]);
                    sm100::tmem_ld32(lane_base + ACC8_COL + 32 * cch, rr);
                }
            }
            sm100::tmem_ld_wait();
            sm100::tc_fence_before();
            __syncwarp();
            if (lane == 0) sm100::mbar_arrive(acc_empty);
            acc_phase ^= 1u;
            float y[COLS];
#pragma unroll
            for (int e = 0; e < COLS; ++e) {
                const float t8 = p.K8 > 0 ? __fmul_rn(a8, __uint_as_float(r8[e])) : 0.0f;
                y[e] = __fmaf_rn(a4, __uint_as_float(r4[e]), t8);
            }
            const int row = m0 + 32 * q + lane;
            if (OUT_BF16) {
                uint4* dst = reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(p.c) + (int64_t)row * p.ldc + n0);
#pragma unroll
                for (int v = 0; v < COLS / 8; ++v) {
                    uint32_t pk[4];
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const __nv_bfloat162 h2 = __floats2bfloat162_rn(y[8 * v + 2 * e], y[8 * v + 2 * e + 1]);
                        pk[e] = *reinterpret_cast<const uint32_t*>(&h2);
                    }
                    dst[v] = make_uint4(pk[0], pk[1], pk[2], pk[3]);
                }
            } else {
                float4* dst = reinterpret_cast<float4*>(static_cast<float*>(p.c) + (int64_t)row * p.ldc + n0);
#pragma unroll
                for (int v = 0; v < COLS / 4; ++v) dst[v] = make_float4(y[4 * v], y[4 * v + 1], y[4 * v + 2], y[4 * v + 3]);
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

template <bool OUT_BF16>
cudaError_t run_oc(const OutctlGemmArgs& g, cudaStream_t s) {
    static PerDeviceOnce setup;
    const cudaError_t attr_err = setup.run([](int) {
        return cudaFuncSetAttribute(gemm_outctl_kernel<OUT_BF16>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                    (int)SMEM);
    });
    if (attr_err != cudaSuccess) return attr_err;
    CUtensorMap ta, tb, ta8, tb8;
    if (!make_codes_map(&ta, g.a_codes, g.M, g.K, BM) || !make_codes_map(&tb, g.b_codes, g.N, g.K, BN))
        return cudaErrorInvalidValue;
    if (g.K8 > 0) {
        // E4M3 codes [rows, K8] bytes: the byte-level map of a code tensor of 2 K8 elements
        if (!make_codes_map(&ta8, g.a8_codes, g.M, 2 * g.K8, BM) || !make_codes_map(&tb8, g.b8_codes, g.N, 2 * g.K8, BN))
            return cudaErrorInvalidValue;
    } else {
        ta8 = ta;
        tb8 = tb;
    }
    OcParams p{};
    p.a_sf = g.a_scales;
    p.b_sf = g.b_scales;
    p.a_ts = g.a_ts;
    p.b_ts = g.b_ts;
    p.a_s8 = g.a8_scale;
    p.b_s8 = g.b8_scale;
    p.c = g.c;
    p.ldc = g.ldc;
    p.M = (int)g.M;
    p.N = (int)g.N;
    p.K = (int)g.K;
    p.K8 = (int)g.K8;
    p.nb4 = (int)(g.K / 16 / 4);
    p.tiles_m = (int)(g.M / BM);
    p.tiles_n = (int)(g.N / BN);
    p.wait_limit = g.wait_limit;
    p.err = device_error_word();
    const int tiles = p.tiles_m * p.tiles_n;
    const int grid = tiles < num_sms() ? tiles : num_sms();
    gemm_outctl_kernel<OUT_BF16><<<grid, NUM_THREADS, SMEM, s>>>(ta, tb, ta8, tb8, p);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_gemm_outctl(const OutctlGemmArgs& g, cudaStream_t s) {
    return g.out_bf16 ? run_oc<true>(g, s) : run_oc<false>(g, s);
}

}  // namespace fp4
