// quant_rows.cuh -- the row-axis (axis = 1) quantizer kernel and its launch
// templates; instantiated per input type in quantize.cu / quantize_rows_f32.cu.
//
// Persistent CTAs stream the input through a ring of shared-memory stages
// filled by bulk asynchronous copies (cp.async.bulk, completion on a "full"
// mbarrier), so the bytes in flight cost no registers: up to STAGES-1 stages
// of 16 KB per CTA are loading while one is computed.  Each warp copies its
// units out to registers at the start of a stage and releases the slot on an
// "empty" mbarrier; thread 0 refills the previous stage's slot, so warps never
// wait for one another.  A stage holds whole lines when a line fits (one copy
// per line) or one segment of a long line.  Thread t of the CTA computes unit
// t of the stage: U = 32 contiguous elements (16 when the line length is only
// a multiple of 16).  Double-block 128-chunks span 128/U adjacent lanes and
// are reduced with shuffles.
//
// Modes: quantize with a known tensor amax; the amax alone (fp4_amax); or
// both in one cooperative launch (fp4_quantize with the internal amax): the
// CTAs run their stages once for the amax, meet at a bounded grid barrier,
// and run them again, in reverse order, to quantize -- the second read of
// the tensor then comes mostly from L2.  Every CTA must be resident for the
// barrier, which the cooperative launch guarantees; work that other streams
// keep on the SMs for more than the barrier's poll budget (4 x the wait limit
// of fp4_set_wait_limit, by default 2^22 sleeps of 32 ns) makes it report
// FP4_ERR_TIMEOUT rather than wait longer.  A ring wait polls at most 16 x the
// wait limit (2^24 by default).  Whatever way a CTA leaves, thread 0 first
// waits (with a fixed bound) for every bulk copy it issued, so no copy lands
// in the shared memory of a CTA that has exited.
#pragma once

#include "quant_common.cuh"
#include "sm100.cuh"

namespace fp4 {

constexpr int RQ_THREADS = 256;
constexpr uint32_t RQ_DRAIN_LIMIT = 1u << 22;       // polls of the exit drain (fixed)

// ring waits: 16 x the wait limit; grid barrier: 4 x (saturating)
__device__ __forceinline__ uint32_t ring_limit(uint32_t w) { return w >= (1u << 27) ? 0xFFFFFFFFu : w << 4; }
__device__ __forceinline__ uint32_t grid_limit(uint32_t w) { return w >= (1u << 29) ? 0xFFFFFFFFu : w << 2; }

// what a launch does: quantize with a known tensor amax, compute the rotated
// tensor's amax only, or both in one launch (amax pass, grid barrier, quantize pass)
enum RowMode { RQ_QUANT = 0, RQ_AMAX = 1, RQ_FUSED = 2 };

// CTAs per SM that registers allow without spills (the SR variants carry a
// Philox word per element)
template <bool SR, int MODE>
constexpr int row_ctas_by_regs() { return MODE == RQ_AMAX ? 4 : (SR ? 2 : 3); }

// A stage holds one U-element unit per thread; the ring has 3 stages (2 when
// the SM's CTAs cannot hold 3), two of them loading while one is computed.
// (Measured on B200: refilling the previous stage's slot from one thread
// beats refilling each slot the moment its last warp has copied it out, and
// a fourth stage adds nothing.)
template <bool BF16, int U, bool SR, int MODE>
struct RowRing {
    static constexpr int BYTES = RQ_THREADS * U * (BF16 ? 2 : 4);
    static constexpr int FIT = (200 * 1024) / (row_ctas_by_regs<SR, MODE>() * BYTES);
    static constexpr int STAGES = FIT < 3 ? 2 : 3;
    static constexpr int SMEM = STAGES * BYTES + STAGES * 16;   // + a full and an empty barrier per stage
};

// CTAs per SM: what registers and shared memory both allow
template <bool BF16, int U, bool SR, int MODE>
constexpr int row_ctas() {
    constexpr int by_smem = (228 * 1024) / (RowRing<BF16, U, SR, MODE>::SMEM + 1024 + 2048);
    constexpr int by_regs = row_ctas_by_regs<SR, MODE>();
    return by_smem < by_regs ? by_smem : by_regs;
}

struct RowStages {
    int total;              // number of stages (< 2^31)
    int lps;                // lines per stage (>= 1) when a line fits, else 0
    int segs;               // segments per line when it does not (else 1)
    int seg_elems;          // elements per segment
    uint32_t seg_m, seg_l;  // multiply-shift division by segs
};

template <bool BF16, int FMT, bool SR, int ROT, bool SIGNS, bool DB, int MODE, int U>
__global__ void __launch_bounds__(RQ_THREADS, (row_ctas<BF16, U, SR, MODE>()))
quant_rows_kernel(const QuantArgs a, const RowStages st) {
    static_assert(U == 16 || U == 32, "unit size");
    constexpr bool AMAX_ONLY = MODE == RQ_AMAX, FUSED = MODE == RQ_FUSED;
    static_assert(!FUSED || (FMT != MXFP4 && !DB), "only a tensor-scaled format has an amax pass");
    constexpr int ES = BF16 ? 2 : 4;
    constexpr int CHUNKS = U * ES / 16;                 // 16-byte chunks per unit
    using Ring = RowRing<BF16, U, SR, MODE>;
    constexpr int RQ_STAGES = Ring::STAGES, RQ_STAGE_BYTES = Ring::BYTES;
    constexpr int WARPS = RQ_THREADS / 32;
    extern __shared__ __align__(128) uint8_t rq_smem[];
    uint8_t* buf = rq_smem;
    uint64_t* full = reinterpret_cast<uint64_t*>(rq_smem + RQ_STAGES * RQ_STAGE_BYTES);  // stage landed
    uint64_t* empty = full + RQ_STAGES;                 // every warp has copied the stage out
    const int tid = threadIdx.x, lane = tid & 31;

    __shared__ ScaleTable table;                        // (S, 1/S) per E4M3 code under s_t
    ScaleRef ref_t = make_ref(1.0f);
    __shared__ float warp_max[RQ_THREADS / 32];          // FUSED: the amax pass's result
    __shared__ uint32_t grid_verdict;
    if (MODE == RQ_QUANT && FMT != MXFP4 && !DB) {
        ref_t = make_ref(tensor_scale_of(*a.amax_in, FMT));
        if (blockIdx.x == 0 && tid == 0 && a.tensor_scale_out) *a.tensor_scale_out = ref_t.s;
        table.build(ref_t.s, tid, RQ_THREADS);
    }
    if (tid == 0) {
        for (int s = 0; s < RQ_STAGES; ++s) {
            sm100::mbar_init(&full[s], 1);
            sm100::mbar_init(&empty[s], WARPS);
        }
        sm100::fence_barrier_init();
    }
    __syncthreads();

    // stage s -> its first line, line count and element range (all below 2^31:
    // the launcher checks the stage count, and K and the lines per stage are
    // bounded by it)
    auto stage_geom = [&](int s, int& l0, int& nl, int& e0, int& ne) {
        if (st.lps) {
            l0 = s * st.lps;
            nl = min(st.lps, (int)(a.L - l0));
            e0 = 0;
            ne = (int)a.K;
        } else {
            l0 = (int)fast_div((uint32_t)s, st.seg_m, st.seg_l);
            nl = 1;
            e0 = (s - l0 * st.segs) * st.seg_elems;
            ne = min(st.seg_elems, (int)(a.K - e0));
        }
    };
    // one thread fills a stage buffer: one bulk copy per line piece.  Fills
    // are issued in pass order, fill v to slot v % STAGES; `issued` counts them
    uint32_t issued = 0;
    auto issue = [&](int s, int slot) {
        ++issued;
        int l0, nl, e0, ne;
        stage_geom(s, l0, nl, e0, ne);
        const uint32_t bytes = (uint32_t)(ne * ES);
        sm100::mbar_arrive_expect_tx(&full[slot], bytes * (uint32_t)nl);
        for (int r = 0; r < nl; ++r) {
            const uint8_t* src = static_cast<const uint8_t*>(a.x) + ((int64_t)(l0 + r) * a.ld + e0) * ES;
            sm100::bulk_load(buf + slot * RQ_STAGE_BYTES + r * bytes, src, bytes, &full[slot]);
        }
    };

    // this CTA's stages first, first + stride, ... (n of them) make one pass;
    // a fused launch streams them twice through the ring, the second pass in
    // reverse order so that the most recently read stages, the likeliest to
    // be still in L2, come first
    const int first = blockIdx.x, stride = gridDim.x;
    const int n = first < st.total ? (st.total - first + stride - 1) / stride : 0;
    const int nv = FUSED ? 2 * n : n;
    auto stage_of = [&](int v) { return (FUSED && v >= n) ? first + (2 * n - 1 - v) * stride : first + v * stride; };
    if (tid == 0)
        for (int p = 0; p < RQ_STAGES - 1; ++p)
            if (p < nv) issue(stage_of(p), p);

    // this thread's unit within a full stage: line my_li of the stage, unit my_ju
    const int full_nl = st.lps ? st.lps : 1;
    const int full_ne = st.lps ? (int)a.K : st.seg_elems;
    const int my_li = st.lps > 1 ? (int)fast_div((uint32_t)tid, a.div_m, a.div_l) : 0;
    const int my_ju = tid - my_li * (full_ne / U);
    const bool my_active = tid < full_nl * (full_ne / U);

    float tmax = 0.0f;
    bool ok = true;
    for (int it = 0; it < nv; ++it) {
        if (FUSED && it == n) {
            // end of the amax pass: the CTA's maximum, then the grid's, then
            // the tensor scale and its table.  Every thread of the CTA gets
            // here (a failed wait of the first pass skips to this point).
            const uint32_t wbits = __reduce_max_sync(0xffffffffu, __float_as_uint(tmax));
            if (lane == 0) warp_max[tid >> 5] = __uint_as_float(wbits);
            const bool failed = __syncthreads_or(!ok);
            if (tid == 0) {
                float m = 0.0f;
#pragma unroll
                for (int w = 0; w < RQ_THREADS / 32; ++w) m = fmaxf(m, warp_max[w]);
                if (__float_as_uint(m)) atomicMax(a.amax_out, __float_as_uint(m));
                __threadfence();
                atomicAdd(a.grid_count, 1u);
                bool done = false;
                const uint32_t glimit = grid_limit(a.wait_limit);
                for (uint32_t i = 0; i < glimit; ++i) {
                    if (sm100::ld_acquire_gpu(a.grid_count) >= gridDim.x) { done = true; break; }
                    __nanosleep(32);
                }
                if (!done) atomicExch(a.err, 7u);       // FP4_ERR_TIMEOUT
                warp_max[0] = __uint_as_float(sm100::ld_acquire_gpu(a.amax_out));
                grid_verdict = (done && !failed) ? 1u : 0u;
            }
            __syncthreads();
            if (!grid_verdict) {
                ok = false;
                break;
            }
            ref_t = make_ref(tensor_scale_of(warp_max[0], FMT));
            if (blockIdx.x == 0 && tid == 0 && a.tensor_scale_out) *a.tensor_scale_out = ref_t.s;
            table.build(ref_t.s, tid, RQ_THREADS);
            __syncthreads();
        }
        const int s = stage_of(it);
        const int slot = it % RQ_STAGES;
        // the verdict on a wait is the warp's; a copy that never lands stops
        // the warp (in the first pass of a fused launch: sends it on to the
        // pass boundary, where the whole CTA meets)
        if (!__all_sync(0xffffffffu,
                        sm100::mbar_wait(&full[slot], (uint32_t)(it / RQ_STAGES) & 1u, ring_limit(a.wait_limit), nullptr))) {
            ok = false;
            if (FUSED && it < n) { it = n - 1; continue; }
            break;
        }
        int l0, nl, e0, ne;
        stage_geom(s, l0, nl, e0, ne);
        const bool active = (nl == full_nl && ne == full_ne) ? my_active : tid < nl * (ne / U);
        const int64_t l = l0 + my_li;
        const int64_t j = e0 / U + my_ju;             // unit index within the line

        // copy the unit out of shared memory (128-bit loads; the 4-way bank
        // conflicts of the 64-byte unit stride still leave shared memory far
        // faster than HBM), then release the slot: the warps run on without
        // waiting for one another, and only the refilling thread waits, for
        // the copies of the previous stage, long done by then
        uint4 w[CHUNKS];
        if (active) {
            const uint4* src = reinterpret_cast<const uint4*>(buf + slot * RQ_STAGE_BYTES + (my_li * ne + my_ju * U) * ES);
#pragma unroll
            for (int q = 0; q < CHUNKS; ++q) w[q] = src[q];
        }
        // the warp's copies are done: release the slot; thread 0 refills the
        // previous stage's slot, which every warp released long ago
        __syncwarp();
        if (lane == 0) sm100::mbar_arrive(&empty[slot]);
        bool stalled = false;
        if (tid == 0 && it + RQ_STAGES - 1 < nv) {
            const int refill = (it + RQ_STAGES - 1) % RQ_STAGES;
            if (it > 0 && !sm100::mbar_wait(&empty[refill], (uint32_t)((it - 1) / RQ_STAGES) & 1u,
                                            ring_limit(a.wait_limit), nullptr))
                stalled = true;
            else
                issue(stage_of(it + RQ_STAGES - 1), refill);
        }
        if (__any_sync(0xffffffffu, stalled)) {
            ok = false;
            if (FUSED && it < n) { it = n - 1; continue; }
            break;
        }

        float v[U];
        if (active) {
#pragma unroll
            for (int q = 0; q < CHUNKS; ++q) {
                if (BF16) {
                    v[8 * q + 0] = bf16_lo(w[q].x); v[8 * q + 1] = bf16_hi(w[q].x);
                    v[8 * q + 2] = bf16_lo(w[q].y); v[8 * q + 3] = bf16_hi(w[q].y);
                    v[8 * q + 4] = bf16_lo(w[q].z); v[8 * q + 5] = bf16_hi(w[q].z);
                    v[8 * q + 6] = bf16_lo(w[q].w); v[8 * q + 7] = bf16_hi(w[q].w);
                } else {
                    v[4 * q + 0] = __uint_as_float(w[q].x); v[4 * q + 1] = __uint_as_float(w[q].y);
                    v[4 * q + 2] = __uint_as_float(w[q].z); v[4 * q + 3] = __uint_as_float(w[q].w);
                }
            }
        } else {
#pragma unroll
            for (int e = 0; e < U; ++e) v[e] = 0.0f;
        }
        if (a.chan_mask && active) {
            // channels taken out of this tensor (OutControl) read as +0
            const int64_t c0 = j * U;
            uint32_t mw = __ldg(a.chan_mask + (c0 >> 5));
            if (U == 16) mw >>= (uint32_t)(c0 & 16);
#pragma unroll
            for (int e = 0; e < U; ++e)
                if ((mw >> e) & 1u) v[e] = 0.0f;
        }
        if (AMAX_ONLY || (FUSED && it < n)) {
            tmax = unit_rotated_absmax<U, ROT, SIGNS>(v, a.sign_mask, tmax);
            continue;
        }
        rotate_unit<U, ROT, SIGNS>(v, a.sign_mask);

        // ---- scales
        uint32_t sbytes[U / 16];
        if (FMT == MXFP4) {
            sbytes[0] = mx_scale32<ROT>(v, absmax_n<32>(v));
        } else {
            ScaleRef ref = ref_t;
            if (DB) {
                // the 128-chunk of this unit spans 128/U adjacent lanes
                constexpr int GL = 128 / U;
                float m = absmax_n<U>(v);
#pragma unroll
                for (int sh = 1; sh < GL; sh <<= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, sh));
                ref = make_ref(tensor_scale_of(m, NVFP4));
                if (active && (lane & (GL - 1)) == 0) a.outer[l * (a.K / 128) + (j * U) / 128] = ref.s;
            }
            float2 SY[U / 16];
            float bm[U / 16];
#pragma unroll
            for (int b = 0; b < U / 16; ++b) bm[b] = absmax_n<16>(v + 16 * b);
            block_scale_codes<FMT, U / 16>(bm, ref, sbytes);
#pragma unroll
            for (int b = 0; b < U / 16; ++b) SY[b] = DB ? scale_pair(sbytes[b], ref.s) : table.e[sbytes[b]];
            nv_divide<U, ROT>(v, SY);
        }
        if (!active) continue;

        // ---- random words for SR: element i = l * cols + j * U + e
        uint32_t rnd[U];
        if (SR) {
            const uint64_t i0 = (uint64_t)l * (uint64_t)a.cols + (uint64_t)(j * U);
#pragma unroll
            for (int q = 0; q < U / 4; ++q) {
                const uint4 w = sr_words((i0 >> 2) + q, a.tensor_id, a.keys);
                rnd[4 * q] = w.x; rnd[4 * q + 1] = w.y; rnd[4 * q + 2] = w.z; rnd[4 * q + 3] = w.w;
            }
        }

        // ---- codes and scale bytes
        uint32_t words[U / 8];
#pragma unroll
        for (int q = 0; q < U / 8; ++q) words[q] = encode8<FMT, SR>(v + 8 * q, rnd + 8 * q);
        uint8_t* dst = a.codes + l * (a.K / 2) + j * (U / 2);
        if (U == 16) *reinterpret_cast<uint2*>(dst) = make_uint2(words[0], words[1]);
        else *reinterpret_cast<uint4*>(dst) = make_uint4(words[0], words[1], words[U / 8 - 2], words[U / 8 - 1]);
        constexpr int BLK = (FMT == MXFP4) ? 32 : 16;
        const int64_t b0 = (j * U) / BLK;
        if (FMT != MXFP4 && U == 32) {
            // blocks 2j' and 2j'+1 sit side by side in the tiled layout
            *reinterpret_cast<uint16_t*>(a.scales + sf_offset(l, b0, a.nb4)) =
                (uint16_t)(sbytes[0] | (sbytes[U / 16 - 1] << 8));
        } else {
            a.scales[sf_offset(l, b0, a.nb4)] = (uint8_t)sbytes[0];
        }
    }

    // every fill issued must land before the CTA may exit (a warp that gave up
    // on a wait leaves fills behind it): the last fill of slot s is fill
    // issued - 1 - ((issued - 1 - s) % STAGES), of phase (issued - 1 - s) / STAGES;
    // all earlier fills of the slot were consumed before it was refilled
    if (tid == 0) {
#pragma unroll
        for (int sl = 0; sl < RQ_STAGES; ++sl)
            if (issued > (uint32_t)sl)
                sm100::mbar_wait(&full[sl], ((issued - 1u - sl) / RQ_STAGES) & 1u, RQ_DRAIN_LIMIT, nullptr);
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

template <bool BF16, int FMT, bool SR, int ROT, bool SIGNS, bool DB, int MODE, int U>
cudaError_t launch_rows(const QuantArgs& a, cudaStream_t s) {
    constexpr int ES = BF16 ? 2 : 4;
    using Ring = RowRing<BF16, U, SR, MODE>;
    auto kernel = quant_rows_kernel<BF16, FMT, SR, ROT, SIGNS, DB, MODE, U>;
    static PerDeviceOnce setup;                  // per instantiation and device
    static int resident_on[kOnceDevices];        // CTAs per SM the launch can keep resident
    int dev = 0;
    const cudaError_t se = setup.run([&](int d) {
        cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, Ring::SMEM);
        if (e == cudaSuccess)
            e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&resident_on[d], kernel, RQ_THREADS, Ring::SMEM);
        return e;
    }, &dev);
    if (se != cudaSuccess) return se;
    const int resident = resident_on[dev];
    // stage, line and element indices inside the kernel are 32-bit
    if (a.L >= ((int64_t)1 << 31) || a.K >= ((int64_t)1 << 31)) return cudaErrorInvalidValue;
    RowStages st{};
    const int64_t line_bytes = a.K * ES;
    int64_t total;
    if (line_bytes <= Ring::BYTES) {
        st.lps = (int)(Ring::BYTES / line_bytes);     // whole lines, one unit per thread at most
        total = (a.L + st.lps - 1) / st.lps;
        st.segs = 1;
        st.seg_elems = (int)a.K;
    } else {
        st.lps = 0;
        st.seg_elems = RQ_THREADS * U;                // a multiple of 128 elements
        st.segs = (int)((a.K + st.seg_elems - 1) / st.seg_elems);
        total = a.L * st.segs;
    }
    if (total >= ((int64_t)1 << 31)) return cudaErrorInvalidValue;
    st.total = (int)total;
    uint32_t l = 0;
    while (l < 32 && (uint64_t(1) << l) < (uint64_t)st.segs) ++l;
    st.seg_m = (uint32_t)((uint64_t)(((unsigned __int128)1 << (32 + l)) / (uint64_t)st.segs) - (uint64_t(1) << 32) + 1);
    st.seg_l = l;
    const int per_sm = resident < row_ctas<BF16, U, SR, MODE>() ? resident : row_ctas<BF16, U, SR, MODE>();
    int64_t grid = (int64_t)num_sms() * (per_sm > 0 ? per_sm : 1);
    if (grid > total) grid = total;
    if (grid < 1) grid = 1;
    if (MODE == RQ_FUSED) {
        // the grid barrier between the passes needs every CTA resident at once
        if (resident < 1) return cudaErrorInvalidConfiguration;
        QuantArgs ka = a;
        RowStages kst = st;
        void* args[] = {&ka, &kst};
        return cudaLaunchCooperativeKernel(reinterpret_cast<const void*>(kernel), dim3((unsigned)grid),
                                           dim3(RQ_THREADS), args, Ring::SMEM, s);
    }
    kernel<<<(unsigned)grid, RQ_THREADS, Ring::SMEM, s>>>(a, st);
    return cudaGetLastError();
}

// unit size: 32 when the line length allows it (always for MXFP4 and 32-rotations)
template <bool BF16, int FMT, bool SR, int ROT, bool SIGNS, bool DB, int MODE>
cudaError_t rows_by_unit(const QuantArgs& a, cudaStream_t s) {
    if (FMT == MXFP4 || ROT == 32 || DB || a.K % 32 == 0)
        return launch_rows<BF16, FMT, SR, ROT, SIGNS, DB, MODE, 32>(a, s);
    return launch_rows<BF16, FMT, SR, ROT, SIGNS, DB, MODE, (FMT == MXFP4 || ROT == 32 || DB) ? 32 : 16>(a, s);
}

template <bool BF16, int FMT, bool SR, bool DB, int MODE>
cudaError_t rows_by_rot(const QuantArgs& a, int rot_n, bool signs, cudaStream_t s) {
    if (rot_n == 0) return rows_by_unit<BF16, FMT, SR, 0, false, DB, MODE>(a, s);
    if (rot_n == 16) return signs ? rows_by_unit<BF16, FMT, SR, 16, true, DB, MODE>(a, s)
                                  : rows_by_unit<BF16, FMT, SR, 16, false, DB, MODE>(a, s);
    return signs ? rows_by_unit<BF16, FMT, SR, 32, true, DB, MODE>(a, s)
                 : rows_by_unit<BF16, FMT, SR, 32, false, DB, MODE>(a, s);
}

template <bool BF16>
cudaError_t rows_by_fmt(const QuantArgs& a, int fmt, bool sr, int rot_n, bool signs, bool db, cudaStream_t s) {
    if (fmt == MXFP4) return sr ? rows_by_rot<BF16, MXFP4, true, false, RQ_QUANT>(a, rot_n, signs, s)
                                : rows_by_rot<BF16, MXFP4, false, false, RQ_QUANT>(a, rot_n, signs, s);
    if (fmt == UFP4) return sr ? rows_by_rot<BF16, UFP4, true, false, RQ_QUANT>(a, rot_n, signs, s)
                               : rows_by_rot<BF16, UFP4, false, false, RQ_QUANT>(a, rot_n, signs, s);
    if (db) return sr ? rows_by_rot<BF16, NVFP4, true, true, RQ_QUANT>(a, rot_n, signs, s)
                      : rows_by_rot<BF16, NVFP4, false, true, RQ_QUANT>(a, rot_n, signs, s);
    return sr ? rows_by_rot<BF16, NVFP4, true, false, RQ_QUANT>(a, rot_n, signs, s)
              : rows_by_rot<BF16, NVFP4, false, false, RQ_QUANT>(a, rot_n, signs, s);
}

// NVFP4 / UFP4 with the tensor amax computed in the same launch
template <bool BF16>
cudaError_t rows_fused_by_fmt(const QuantArgs& a, int fmt, bool sr, int rot_n, bool signs, cudaStream_t s) {
    if (fmt == UFP4) return sr ? rows_by_rot<BF16, UFP4, true, false, RQ_FUSED>(a, rot_n, signs, s)
                               : rows_by_rot<BF16, UFP4, false, false, RQ_FUSED>(a, rot_n, signs, s);
    return sr ? rows_by_rot<BF16, NVFP4, true, false, RQ_FUSED>(a, rot_n, signs, s)
              : rows_by_rot<BF16, NVFP4, false, false, RQ_FUSED>(a, rot_n, signs, s);
}

// one input type's entry points (defined in quantize.cu for bf16, quantize_rows_f32.cu for f32)
template <bool BF16>
cudaError_t launch_rows_quantize(const QuantArgs& a, int fmt, bool sr, int rot_n, bool signs, bool db,
                                 cudaStream_t s) {
    return rows_by_fmt<BF16>(a, fmt, sr, rot_n, signs, db, s);
}

template <bool BF16>
cudaError_t launch_rows_amax(const QuantArgs& a, int rot_n, bool signs, cudaStream_t s) {
    return rows_by_rot<BF16, NVFP4, false, false, RQ_AMAX>(a, rot_n, signs, s);
}

template <bool BF16>
cudaError_t launch_rows_fused(const QuantArgs& a, int fmt, bool sr, int rot_n, bool signs, cudaStream_t s) {
    return rows_fused_by_fmt<BF16>(a, fmt, sr, rot_n, signs, s);
}

}  // namespace fp4
