// internal.h -- declarations shared by the CUDA translation units of libfp4.so.
#pragma once

#include <cstdint>
#include <mutex>
#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include "fp4_device.cuh"

namespace fp4 {

// arguments of the quantizer and amax kernels (passed by value)
struct QuantArgs {
    const void* x;
    int64_t rows, cols, ld;     // input [rows, ld], `cols` valid columns
    int64_t L, K, nb4;          // lines, elements per line, ceil((K / block) / 4)
    uint8_t* codes;
    uint8_t* scales;
    float* outer;
    float* tensor_scale_out;
    const float* amax_in;       // rotated-tensor amax (NVFP4 / UFP4 without double block)
    unsigned int* amax_out;     // amax pass: atomicMax target (binary32 bits, >= 0)
    unsigned int* grid_count;   // fused launch: arrivals at the grid barrier (zeroed by the host)
    PhiloxKeys keys;
    uint32_t tensor_id;
    uint32_t sign_mask;         // random-sign bits (0: deterministic Hadamard)
    uint32_t div_m, div_l;      // multiply-shift division by the units per line
    unsigned int* err;          // device error word (a bounded wait that ran out)
    uint32_t wait_limit;        // polls of a bounded wait (fp4_set_wait_limit)
    // row axis only: channels (columns) whose bit is set read as +0 (OutControl's
    // FP8 channels, taken out of the FP4 part); NULL for none
    const uint32_t* chan_mask;
    // re-quantization (fp4_requantize): the source is a quantized tensor whose
    // lines are the rows of the logical [rows, cols] input; x is unused
    const uint8_t* src_codes;   // [rows, cols/2]
    const uint8_t* src_scales;  // tiled layout, src_nb4 groups of 4 blocks per line
    const float* src_outer;     // [rows, cols/128] (double block)
    const float* src_ts;        // tensor scale (NVFP4 / UFP4 without double block)
    int src_fmt, src_db;
    int64_t src_nb4;
};

cudaError_t launch_quantize(QuantArgs a, bool bf16, int fmt, bool sr, int rot_n, bool db, int axis,
                            cudaStream_t s);
cudaError_t launch_amax(QuantArgs a, bool bf16, int rot_n, int axis, cudaStream_t s);
// NVFP4 / UFP4, either axis: amax pass, grid barrier and quantize pass in one
// cooperative launch; a.amax_out / a.grid_count point at zeroed words
cudaError_t launch_quantize_fused(QuantArgs a, bool bf16, int fmt, bool sr, int rot_n, int axis, cudaStream_t s);
// the same for axis 0 (quant_cols.cuh), per input type
template <bool BF16>
cudaError_t launch_cols_quantize(const QuantArgs& a, int fmt, bool sr, int rot_n, bool signs, bool db, cudaStream_t s);
template <bool BF16>
cudaError_t launch_cols_amax(const QuantArgs& a, int rot_n, bool signs, cudaStream_t s);
template <bool BF16>
cudaError_t launch_cols_fused(const QuantArgs& a, int fmt, bool sr, int rot_n, bool signs, cudaStream_t s);
// both axes of a bf16 tensor in one cooperative launch (quantize_dual.cu): the
// QuantArgs describe the column-axis result, RowOut the row-axis result
// (rows of `cols` elements)
struct RowOut {
    uint8_t* codes;             // [rows, cols / 2]
    uint8_t* scales;            // tiled layout, nb4 groups of 4 blocks per row
    float* tensor_scale_out;
    unsigned int* amax_out;     // the row-rotated amax (atomicMax target, zeroed by the host)
    int64_t nb4;
    uint32_t tensor_id;         // SR stream of the row quantization
};
cudaError_t launch_both_axes(const QuantArgs& a, const RowOut& ro, int fmt, bool sr_cols, bool sr_rows, int rot_n,
                             cudaStream_t s);
// 2-D TMA map over a [rows, cols] input of row pitch ld, box 64 columns x 128
// rows, zeros past the edges; swizzle128 (bf16 only): the tile lands with the
// 128-byte swizzle, 16-byte chunk c of tile row r at chunk c ^ (r % 8)
bool make_input_map(CUtensorMap* m, const void* x, bool bf16, int64_t rows, int64_t cols, int64_t ld,
                    bool swizzle128 = false);
// the same two along axis 0 of the dequantized source (a.src_*)
cudaError_t launch_requantize_cols(const QuantArgs& a, int fmt, bool sr, int rot_n, bool signs, bool db,
                                   cudaStream_t s);
cudaError_t launch_requant_amax_cols(const QuantArgs& a, int rot_n, bool signs, cudaStream_t s);
// MXNorm fused with the cast (fp4_mxnorm_quantize); amax_word: a zeroed word
// (NVFP4 / UFP4 only)
cudaError_t launch_mxnorm(const void* x, bool bf16, int64_t rows, int64_t cols, int64_t ld, int fmt, bool sr, int p,
                          double c, uint8_t* codes, uint8_t* scales, float* tensor_scale, float* rho,
                          unsigned int* amax_word, const PhiloxKeys& keys, uint32_t tensor_id, cudaStream_t s);
// the rotation alone along the rows (fp4_rotate)
cudaError_t launch_rotate_rows(const void* x, void* y, bool bf16, int64_t rows, int64_t cols, int64_t ld,
                               int64_t ldy, int n, uint32_t sign_mask, cudaStream_t s);

// GEMM
struct GemmArgs {
    const uint8_t* a_codes;
    const uint8_t* a_scales;
    const float* a_outer;
    const float* a_ts;
    const uint8_t* b_codes;
    const uint8_t* b_scales;
    const float* b_outer;
    const float* b_ts;
    int64_t M, N, K;
    void* c;
    int64_t ldc;
    int out_bf16;
    int fmt;
    int db;
    int pairs;        // 1: 256 x 256 tiles on CTA pairs where the shape allows (gemm_pair.cu)
    uint32_t wait_limit;
};
cudaError_t launch_gemm(const GemmArgs& g, cudaStream_t s);
// the CTA-pair GEMM (gemm_pair.cu): M and N multiples of 256, no double block
bool gemm_pair_fits(const GemmArgs& g);
cudaError_t launch_gemm_pair(const GemmArgs& g, cudaStream_t s);

// Output tile t of a tiles_m x tiles_n grid in grouped order: bands of up to
// GEMM_GROUP_M m-tiles, each band walked column by column.  The CTAs of one
// persistent wave then share a compact block of A rows and B columns, so an
// operand larger than L2 is read from DRAM about once instead of once per
// column of tiles.
constexpr int GEMM_GROUP_M = 8;
__host__ __device__ __forceinline__ void tile_coords(int t, int tiles_m, int tiles_n, int& tm, int& tn) {
    const int band = t / (GEMM_GROUP_M * tiles_n);
    const int first_m = band * GEMM_GROUP_M;
    const int gm = (tiles_m - first_m) < GEMM_GROUP_M ? (tiles_m - first_m) : GEMM_GROUP_M;
    const int local = t - band * GEMM_GROUP_M * tiles_n;
    tm = first_m + local % gm;
    tn = local / gm;
}
// OutControl (outctl.cu, gemm_outctl.cu)
cudaError_t launch_channel_amax(const void* x, bool bf16, int64_t rows, int64_t cols, int64_t ld, float* out,
                                cudaStream_t s);
cudaError_t launch_channel_mask(const int32_t* ch, int64_t n, int64_t cols, uint32_t* mask, cudaStream_t s);
cudaError_t launch_fp8_gather(const void* x, bool bf16, int64_t rows, int64_t cols, int64_t ld, const int32_t* ch,
                              int64_t n, int64_t k8, unsigned int* amax_word, uint8_t* codes, float* scale,
                              cudaStream_t s);
struct OutctlGemmArgs {
    const uint8_t* a_codes;
    const uint8_t* a_scales;
    const float* a_ts;
    const uint8_t* b_codes;
    const uint8_t* b_scales;
    const float* b_ts;
    const uint8_t* a8_codes;
    const float* a8_scale;
    const uint8_t* b8_codes;
    const float* b8_scale;
    int64_t M, N, K, K8;
    void* c;
    int64_t ldc;
    int out_bf16;
    uint32_t wait_limit;
};
cudaError_t launch_gemm_outctl(const OutctlGemmArgs& g, cudaStream_t s);
// UFP4 operands as two E2M1 parts (ufp4_split.cu): bytes of one operand's
// split form, and the kernel writing it (codes, then scales at a 1024-byte
// boundary); b_operand selects the segment order [1 1 2 2] instead of [1 2 1 2]
size_t ufp4_split_bytes(int64_t L, int64_t K);
cudaError_t launch_ufp4_split(const uint8_t* codes, const uint8_t* scales, int64_t L, int64_t K, uint8_t* out,
                              bool b_operand, cudaStream_t s);
cudaError_t launch_gemm_db(const GemmArgs& g, cudaStream_t s);
// 2-D TMA map over packed codes [rows, K/2] bytes: box 128 bytes x box_rows, 128-byte swizzle
bool make_codes_map(CUtensorMap* m, const uint8_t* codes, int64_t rows, int64_t K, int box_rows);
// 2-D map over C [M, N] for tiled stores: box 128 bytes x 32 rows, 128-byte swizzle
bool make_c_map(CUtensorMap* m, void* c, bool bf16, int64_t M, int64_t N, int64_t ldc);
// the driver's cuTensorMapEncodeTiled (null when the driver has none)
PFN_cuTensorMapEncodeTiled_v12000 encode_fn();

// One-time setup per device (kernel attributes and occupancy are properties of
// the kernel on one device): run() calls init once for the current device and
// returns its cached status afterwards.
constexpr int kOnceDevices = 64;
struct PerDeviceOnce {
    std::mutex mu;
    bool done[kOnceDevices] = {};
    cudaError_t status[kOnceDevices] = {};
    template <class F>
    cudaError_t run(F&& init, int* dev_out = nullptr) {
        int dev = 0;
        if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kOnceDevices) return cudaErrorInvalidDevice;
        if (dev_out) *dev_out = dev;
        std::lock_guard<std::mutex> lock(mu);
        if (!done[dev]) {
            status[dev] = init(dev);
            done[dev] = true;
        }
        return status[dev];
    }
};

// device state
int num_sms();
unsigned int* device_error_word();   // device address of the error word of the current device

}  // namespace fp4
