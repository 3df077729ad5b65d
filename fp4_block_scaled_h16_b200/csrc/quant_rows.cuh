// quant_rows.cuh -- the row-axis (axis = 1) quantizer kernel and its launch
// templates; instantiated per input type in quantize.cu / quantize_rows_f32.cu.
//
// Persistent CTAs stream the input through a ring of shared-memory stages
// filled by bulk asynchronous copies (cp.async.bulk, completion on an
// mbarrier), so the bytes in flight cost no registers: up to STAGES-1 stages
// of 16 KB per CTA are loading while one is computed.  A stage holds whole
// lines when a line fits (one copy per line) or one segment of a long line.
// Thread t of the CTA computes unit t of the stage: U = 32 contiguous
// elements (16 when the line length is only a multiple of 16).  Double-block
// 128-chunks span 128/U adjacent lanes and are reduced with shuffles.
#pragma once

#include "quant_common.cuh"
#include "sm100.cuh"

namespace fp4 {

constexpr int RQ_THREADS = 256;
constexpr uint32_t RQ_WAIT_LIMIT = 1u << 24;

// a stage holds one U-element unit per thread; 3 stages (2 for 32-KB stages)
template <bool BF16, int U>
struct RowRing {
    static constexpr int BYTES = RQ_THREADS * U * (BF16 ? 2 : 4);
    static constexpr int STAGES = BYTES <= 16384 ? 3 : 2;
    static constexpr int SMEM = STAGES * BYTES + STAGES * 8;
};

// CTAs per SM: as many as registers allow without spills (the SR variants
// carry a Philox word per element) and shared memory allows
template <bool BF16, int U, bool SR, bool AMAX_ONLY>
constexpr int row_ctas() {
    constexpr int by_smem = (228 * 1024) / (RowRing<BF16, U>::SMEM + 1024 + 2048);
    constexpr int by_regs = AMAX_ONLY ? 4 : (SR ? 2 : 3);
    return by_smem < by_regs ? by_smem : by_regs;
}

struct RowStages {
    int64_t total;          // number of stages
    int64_t lps;            // lines per stage (>= 1) when a line fits, else 0
    int64_t segs;           // segments per line when it does not (else 1)
    int64_t seg_elems;      // elements per segment
    uint32_t seg_m, seg_l;  // multiply-shift division by segs
};

template <bool BF16, int FMT, bool SR, int ROT, bool SIGNS, bool DB, bool AMAX_ONLY, int U>
__global__ void __launch_bounds__(RQ_THREADS, (row_ctas<BF16, U, SR, AMAX_ONLY>()))
quant_rows_kernel(const QuantArgs a, const RowStages st) {
    static_assert(U == 16 || U == 32, "unit size");
    constexpr int ES = BF16 ? 2 : 4;
    constexpr int CHUNKS = U * ES / 16;                 // 16-byte chunks per unit
    using Ring = RowRing<BF16, U>;
    constexpr int RQ_STAGES = Ring::STAGES, RQ_STAGE_BYTES = Ring::BYTES;
    extern __shared__ __align__(128) uint8_t rq_smem[];
    uint8_t* buf = rq_smem;
    uint64_t* bar = reinterpret_cast<uint64_t*>(rq_smem + RQ_STAGES * RQ_STAGE_BYTES);
    const int tid = threadIdx.x, lane = tid & 31;

    __shared__ ScaleTable table;                        // (S, 1/S) per E4M3 code under s_t
    ScaleRef ref_t = make_ref(1.0f);
    if (!AMAX_ONLY && FMT != MXFP4 && !DB) {
        ref_t = make_ref(tensor_scale_of(*a.amax_in, FMT));
        if (blockIdx.x == 0 && tid == 0 && a.tensor_scale_out) *a.tensor_scale_out = ref_t.s;
        table.build(ref_t.s, tid, RQ_THREADS);
    }
    if (tid == 0) {
        for (int s = 0; s < RQ_STAGES; ++s) sm100::mbar_init(&bar[s], 1);
        sm100::fence_barrier_init();
    }
    __syncthreads();

    // stage s -> its first line, line count and element range
    auto stage_geom = [&](int64_t s, int64_t& l0, int64_t& nl, int64_t& e0, int64_t& ne) {
        if (st.lps) {
            l0 = s * st.lps;
            nl = min(st.lps, a.L - l0);
            e0 = 0;
            ne = a.K;
        } else {
            l0 = fast_div((uint32_t)s, st.seg_m, st.seg_l);
            nl = 1;
            e0 = (s - l0 * st.segs) * st.seg_elems;
            ne = min(st.seg_elems, a.K - e0);
        }
    };
    // one thread fills a stage buffer: one bulk copy per line piece
    auto issue = [&](int64_t s, int slot) {
        int64_t l0, nl, e0, ne;
        stage_geom(s, l0, nl, e0, ne);
        const uint32_t bytes = (uint32_t)(ne * ES);
        sm100::mbar_arrive_expect_tx(&bar[slot], bytes * (uint32_t)nl);
        for (int64_t r = 0; r < nl; ++r) {
            const uint8_t* src = static_cast<const uint8_t*>(a.x) + ((l0 + r) * a.ld + e0) * ES;
            sm100::bulk_load(buf + slot * RQ_STAGE_BYTES + r * bytes, src, bytes, &bar[slot]);
        }
    };

    const int64_t first = blockIdx.x, stride = gridDim.x;
    if (tid == 0)
        for (int p = 0; p < RQ_STAGES - 1; ++p)
            if (first + p * stride < st.total) issue(first + p * stride, p);

    // this thread's unit within a full stage: line my_li of the stage, unit my_ju
    const int64_t full_nl = st.lps ? st.lps : 1;
    const int64_t full_ne = st.lps ? a.K : st.seg_elems;
    const int64_t my_li = st.lps > 1 ? (int64_t)fast_div((uint32_t)tid, a.div_m, a.div_l) : 0;
    const int64_t my_ju = tid - my_li * (full_ne / U);
    const bool my_active = (int64_t)tid < full_nl * (full_ne / U);

    float tmax = 0.0f;
    bool ok = true;
    int it = 0;
    for (int64_t s = first; s < st.total; s += stride, ++it) {
        const int slot = it % RQ_STAGES;
        const bool got = sm100::mbar_wait(&bar[slot], (uint32_t)(it / RQ_STAGES) & 1u, RQ_WAIT_LIMIT, nullptr);
        // one barrier per stage: the verdict is the CTA's, and every thread is
        // done with the previous stage's slot, which is refilled next
        if (__syncthreads_or(!got)) {
            ok = false;                               // a copy that never lands: stop, report
            break;
        }
        if (tid == 0 && s + (RQ_STAGES - 1) * stride < st.total)
            issue(s + (RQ_STAGES - 1) * stride, (it + RQ_STAGES - 1) % RQ_STAGES);

        int64_t l0, nl, e0, ne;
        stage_geom(s, l0, nl, e0, ne);
        const bool active = (nl == full_nl && ne == full_ne) ? my_active : (int64_t)tid < nl * (ne / U);
        const int64_t l = l0 + my_li;
        const int64_t j = e0 / U + my_ju;             // unit index within the line

        // read the unit from shared memory (128-bit loads; the 4-way bank
        // conflicts of the 64-byte unit stride still leave shared memory far
        // faster than HBM)
        float v[U];
        if (active) {
            const uint4* src = reinterpret_cast<const uint4*>(buf + slot * RQ_STAGE_BYTES + (my_li * ne + my_ju * U) * ES);
            uint4 w[CHUNKS];
#pragma unroll
            for (int q = 0; q < CHUNKS; ++q) w[q] = src[q];
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
        if (AMAX_ONLY) {
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
#pragma unroll
            for (int b = 0; b < U / 16; ++b) {
                sbytes[b] = block_scale_code<FMT>(absmax_n<16>(v + 16 * b), ref);
                SY[b] = DB ? scale_pair(sbytes[b], ref.s) : table.e[sbytes[b]];
            }
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

    if (!ok) {
        if (tid == 0) atomicExch(a.err, 7u);          // FP4_ERR_TIMEOUT
        return;
    }
    if (AMAX_ONLY) {
        const uint32_t bits = __reduce_max_sync(0xffffffffu, __float_as_uint(tmax));
        if (lane == 0 && bits) atomicMax(a.amax_out, bits);
    }
}

template <bool BF16, int FMT, bool SR, int ROT, bool SIGNS, bool DB, bool AMAX_ONLY, int U>
cudaError_t launch_rows(const QuantArgs& a, cudaStream_t s) {
    constexpr int ES = BF16 ? 2 : 4;
    using Ring = RowRing<BF16, U>;
    static bool attr_set = false;   // per instantiation
    if (!attr_set) {
        const cudaError_t e = cudaFuncSetAttribute(quant_rows_kernel<BF16, FMT, SR, ROT, SIGNS, DB, AMAX_ONLY, U>,
                                                   cudaFuncAttributeMaxDynamicSharedMemorySize, Ring::SMEM);
        if (e != cudaSuccess) return e;
        attr_set = true;
    }
    RowStages st{};
    const int64_t line_bytes = a.K * ES;
    if (line_bytes <= Ring::BYTES) {
        st.lps = Ring::BYTES / line_bytes;            // whole lines, one unit per thread at most
        st.total = (a.L + st.lps - 1) / st.lps;
        st.segs = 1;
        st.seg_elems = a.K;
    } else {
        st.lps = 0;
        st.seg_elems = (int64_t)RQ_THREADS * U;       // a multiple of 128 elements
        st.segs = (a.K + st.seg_elems - 1) / st.seg_elems;
        st.total = a.L * st.segs;
    }
    if (st.total >= ((int64_t)1 << 31)) return cudaErrorInvalidValue;   // stage indices are 32-bit
    uint32_t l = 0;
    while (l < 32 && (uint64_t(1) << l) < (uint64_t)st.segs) ++l;
    st.seg_m = (uint32_t)((uint64_t)(((unsigned __int128)1 << (32 + l)) / (uint64_t)st.segs) - (uint64_t(1) << 32) + 1);
    st.seg_l = l;
    int64_t grid = (int64_t)num_sms() * row_ctas<BF16, U, SR, AMAX_ONLY>();
    if (grid > st.total) grid = st.total;
    if (grid < 1) grid = 1;
    quant_rows_kernel<BF16, FMT, SR, ROT, SIGNS, DB, AMAX_ONLY, U><<<(unsigned)grid, RQ_THREADS, Ring::SMEM, s>>>(a, st);
    return cudaGetLastError();
}

// unit size: 32 when the line length allows it (always for MXFP4 and 32-rotations)
template <bool BF16, int FMT, bool SR, int ROT, bool SIGNS, bool DB, bool AMAX_ONLY>
cudaError_t rows_by_unit(const QuantArgs& a, cudaStream_t s) {
    if (FMT == MXFP4 || ROT == 32 || DB || a.K % 32 == 0)
        return launch_rows<BF16, FMT, SR, ROT, SIGNS, DB, AMAX_ONLY, 32>(a, s);
    return launch_rows<BF16, FMT, SR, ROT, SIGNS, DB, AMAX_ONLY, (FMT == MXFP4 || ROT == 32 || DB) ? 32 : 16>(a, s);
}

template <bool BF16, int FMT, bool SR, bool DB, bool AMAX_ONLY>
cudaError_t rows_by_rot(const QuantArgs& a, int rot_n, bool signs, cudaStream_t s) {
    if (rot_n == 0) return rows_by_unit<BF16, FMT, SR, 0, false, DB, AMAX_ONLY>(a, s);
    if (rot_n == 16) return signs ? rows_by_unit<BF16, FMT, SR, 16, true, DB, AMAX_ONLY>(a, s)
                                  : rows_by_unit<BF16, FMT, SR, 16, false, DB, AMAX_ONLY>(a, s);
    return signs ? rows_by_unit<BF16, FMT, SR, 32, true, DB, AMAX_ONLY>(a, s)
                 : rows_by_unit<BF16, FMT, SR, 32, false, DB, AMAX_ONLY>(a, s);
}

template <bool BF16>
cudaError_t rows_by_fmt(const QuantArgs& a, int fmt, bool sr, int rot_n, bool signs, bool db, cudaStream_t s) {
    if (fmt == MXFP4) return sr ? rows_by_rot<BF16, MXFP4, true, false, false>(a, rot_n, signs, s)
                                : rows_by_rot<BF16, MXFP4, false, false, false>(a, rot_n, signs, s);
    if (fmt == UFP4) return sr ? rows_by_rot<BF16, UFP4, true, false, false>(a, rot_n, signs, s)
                               : rows_by_rot<BF16, UFP4, false, false, false>(a, rot_n, signs, s);
    if (db) return sr ? rows_by_rot<BF16, NVFP4, true, true, false>(a, rot_n, signs, s)
                      : rows_by_rot<BF16, NVFP4, false, true, false>(a, rot_n, signs, s);
    return sr ? rows_by_rot<BF16, NVFP4, true, false, false>(a, rot_n, signs, s)
              : rows_by_rot<BF16, NVFP4, false, false, false>(a, rot_n, signs, s);
}

// one input type's entry points (defined in quantize.cu for bf16, quantize_rows_f32.cu for f32)
template <bool BF16>
cudaError_t launch_rows_quantize(const QuantArgs& a, int fmt, bool sr, int rot_n, bool signs, bool db,
                                 cudaStream_t s) {
    return rows_by_fmt<BF16>(a, fmt, sr, rot_n, signs, db, s);
}

template <bool BF16>
cudaError_t launch_rows_amax(const QuantArgs& a, int rot_n, bool signs, cudaStream_t s) {
    return rows_by_rot<BF16, NVFP4, false, false, true>(a, rot_n, signs, s);
}

}  // namespace fp4
