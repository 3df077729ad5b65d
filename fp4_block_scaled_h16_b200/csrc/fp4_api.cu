// fp4_api.cu -- the extern "C" entry points of libfp4.so (declared in
// include/fp4.h): argument validation, the host-side Philox key schedule and
// sign mask, and the launches.  The library allocates no device memory.
#include <cuda_runtime.h>
#include <cstdint>
#include <cstring>
#include <mutex>

#include "../../include/fp4.h"
#include "internal.h"

namespace fp4 {

__device__ unsigned int g_error_word;    // FP4_ERR_TIMEOUT etc., set by kernels

namespace {

constexpr int kMaxDevices = 64;
int g_sms[kMaxDevices];
int g_arch_ok[kMaxDevices];               // 0 unknown, 1 sm_100, -1 other
unsigned int* g_err_ptr[kMaxDevices];
std::mutex g_mu;
uint32_t g_wait_limit = 1u << 20;
int g_gemm_pairs = 1;

// Philox4x32-10 on the host, for the random-sign word and the round keys
// (Salmon et al., SC'11: multipliers 0xD2511F53 / 0xCD9E8D57, Weyl key bumps
// 0x9E3779B9 / 0xBB67AE85).
PhiloxKeys make_keys(uint64_t seed) {
    PhiloxKeys k;
    uint32_t a = (uint32_t)seed, b = (uint32_t)(seed >> 32);
    for (int r = 0; r < 10; ++r) {
        k.k0[r] = a;
        k.k1[r] = b;
        a += 0x9E3779B9u;
        b += 0xBB67AE85u;
    }
    return k;
}

uint32_t philox_word0(uint32_t c0, uint32_t c1, uint32_t c2, uint32_t c3, const PhiloxKeys& k) {
    for (int r = 0; r < 10; ++r) {
        const uint64_t p0 = (uint64_t)0xD2511F53u * c0, p1 = (uint64_t)0xCD9E8D57u * c2;
        const uint32_t n0 = (uint32_t)(p1 >> 32) ^ c1 ^ k.k0[r];
        const uint32_t n2 = (uint32_t)(p0 >> 32) ^ c3 ^ k.k1[r];
        c1 = (uint32_t)p1;
        c3 = (uint32_t)p0;
        c0 = n0;
        c2 = n2;
    }
    return c0;
}

int rot_size(int rotation) {
    return (rotation == FP4_ROT_H16 || rotation == FP4_ROT_RH16) ? 16
         : (rotation == FP4_ROT_H32 || rotation == FP4_ROT_RH32) ? 32 : 0;
}

uint32_t sign_mask_of(int rotation, uint64_t seed) {
    if (rotation != FP4_ROT_RH16 && rotation != FP4_ROT_RH32) return 0u;
    const uint32_t w = philox_word0(0u, 0u, 0u, 1u, make_keys(seed));
    return rotation == FP4_ROT_RH16 ? (w & 0xFFFFu) : w;
}

bool aligned16(const void* p) { return ((uintptr_t)p & 15u) == 0; }

// current device is a usable sm_100 GPU; caches the SM count and error word
fp4_status_t device_ready(int* dev_out) {
    int n = 0;
    if (cudaGetDeviceCount(&n) != cudaSuccess || n == 0) {
        cudaGetLastError();
        return FP4_ERR_NO_DEVICE;
    }
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return FP4_ERR_NO_DEVICE;
    std::lock_guard<std::mutex> lock(g_mu);
    if (g_arch_ok[dev] == 0) {
        int major = 0, sms = 0;
        if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
            cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
            return FP4_ERR_CUDA;
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_error_word) != cudaSuccess) return FP4_ERR_CUDA;
        g_err_ptr[dev] = static_cast<unsigned int*>(p);
        g_sms[dev] = sms;
        g_arch_ok[dev] = (major == 10) ? 1 : -1;
    }
    if (g_arch_ok[dev] != 1) return FP4_ERR_NO_DEVICE;
    *dev_out = dev;
    return FP4_OK;
}

}  // namespace

int num_sms() {
    int dev = 0;
    cudaGetDevice(&dev);
    return (dev >= 0 && dev < kMaxDevices && g_sms[dev] > 0) ? g_sms[dev] : 148;
}

unsigned int* device_error_word() {
    int dev = 0;
    cudaGetDevice(&dev);
    return (dev >= 0 && dev < kMaxDevices) ? g_err_ptr[dev] : nullptr;
}

}  // namespace fp4

using namespace fp4;

extern "C" {

const char* fp4_status_string(fp4_status_t s) {
    switch (s) {
    case FP4_OK: return "FP4_OK";
    case FP4_ERR_INVALID_ARG: return "FP4_ERR_INVALID_ARG";
    case FP4_ERR_UNSUPPORTED_SHAPE: return "FP4_ERR_UNSUPPORTED_SHAPE";
    case FP4_ERR_MISALIGNED: return "FP4_ERR_MISALIGNED";
    case FP4_ERR_WORKSPACE: return "FP4_ERR_WORKSPACE";
    case FP4_ERR_NO_DEVICE: return "FP4_ERR_NO_DEVICE";
    case FP4_ERR_CUDA: return "FP4_ERR_CUDA";
    case FP4_ERR_TIMEOUT: return "FP4_ERR_TIMEOUT";
    case FP4_ERR_UNSUPPORTED: return "FP4_ERR_UNSUPPORTED";
    }
    return "FP4_ERR_UNKNOWN";
}

void fp4_set_wait_limit(uint32_t polls) { g_wait_limit = polls ? polls : (1u << 20); }

void fp4_set_gemm_cta_pairs(int enable) { g_gemm_pairs = enable ? 1 : 0; }

size_t fp4_scales_bytes(int64_t lines, int64_t K, fp4_format_t format) {
    if (lines <= 0 || K <= 0) return 0;
    const int64_t blk = (format == FP4_MXFP4) ? 32 : 16;
    const int64_t nb = K / blk;
    return (size_t)(((lines + 127) / 128) * 128) * (size_t)(((nb + 3) / 4) * 4);
}

fp4_status_t fp4_quantize_workspace_size(fp4_format_t format, int double_block, int amax_given,
                                         size_t* bytes) {
    if (!bytes || format < FP4_MXFP4 || format > FP4_UFP4) return FP4_ERR_INVALID_ARG;
    *bytes = (format != FP4_MXFP4 && !double_block && !amax_given) ? 256 : 0;
    return FP4_OK;
}

static fp4_status_t check_input(const void* x, fp4_in_dtype_t in_dtype, int64_t rows, int64_t cols,
                                int64_t ld, fp4_rotation_t rotation, int axis) {
    if (in_dtype != FP4_IN_F32 && in_dtype != FP4_IN_BF16) return FP4_ERR_INVALID_ARG;
    if (rotation < FP4_ROT_NONE || rotation > FP4_ROT_RH32) return FP4_ERR_INVALID_ARG;
    if (axis != 0 && axis != 1) return FP4_ERR_INVALID_ARG;
    if (rows < 0 || cols < 0 || ld < cols) return FP4_ERR_INVALID_ARG;
    if (rows > 0 && cols > 0) {
        if (!x) return FP4_ERR_INVALID_ARG;
        const int64_t es = in_dtype == FP4_IN_BF16 ? 2 : 4;
        if (!aligned16(x) || (ld * es) % 16) return FP4_ERR_MISALIGNED;
    }
    const int64_t K = axis ? cols : rows;
    const int n = rot_size(rotation);
    if (n && K % n) return FP4_ERR_UNSUPPORTED_SHAPE;
    return FP4_OK;
}

fp4_status_t fp4_amax(const void* x, fp4_in_dtype_t in_dtype, int64_t rows, int64_t cols, int64_t ld,
                      fp4_rotation_t rotation, int axis, uint64_t seed, float* amax_out, void* stream) {
    fp4_status_t st = check_input(x, in_dtype, rows, cols, ld, rotation, axis);
    if (st != FP4_OK) return st;
    if (!amax_out) return FP4_ERR_INVALID_ARG;
    if ((uintptr_t)amax_out & 3u) return FP4_ERR_MISALIGNED;
    int dev;
    if ((st = device_ready(&dev)) != FP4_OK) return st;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (cudaMemsetAsync(amax_out, 0, sizeof(float), s) != cudaSuccess) return FP4_ERR_CUDA;
    if (rows == 0 || cols == 0) return FP4_OK;
    QuantArgs a{};
    a.x = x; a.rows = rows; a.cols = cols; a.ld = ld;
    a.L = axis ? rows : cols;
    a.K = axis ? cols : rows;
    a.amax_out = reinterpret_cast<unsigned int*>(amax_out);
    a.sign_mask = sign_mask_of(rotation, seed);
    a.err = device_error_word();
    a.wait_limit = g_wait_limit;
    if (launch_amax(a, in_dtype == FP4_IN_BF16, rot_size(rotation), axis, s) != cudaSuccess) return FP4_ERR_CUDA;
    return FP4_OK;
}

fp4_status_t fp4_rotate(const void* x, fp4_in_dtype_t in_dtype, int64_t rows, int64_t cols, int64_t ld,
                        fp4_rotation_t rotation, int axis, uint64_t seed, void* y, int64_t ldy, void* stream) {
    fp4_status_t st = check_input(x, in_dtype, rows, cols, ld, rotation, axis);
    if (st != FP4_OK) return st;
    if (axis != 1) return FP4_ERR_UNSUPPORTED;
    if (rotation == FP4_ROT_NONE) return FP4_ERR_INVALID_ARG;
    if (ldy < cols) return FP4_ERR_INVALID_ARG;
    if (rows == 0 || cols == 0) return FP4_OK;
    const int64_t es = in_dtype == FP4_IN_BF16 ? 2 : 4;
    if (!y) return FP4_ERR_INVALID_ARG;
    if (!aligned16(y) || (ldy * es) % 16) return FP4_ERR_MISALIGNED;
    int dev;
    if ((st = device_ready(&dev)) != FP4_OK) return st;
    if (launch_rotate_rows(x, y, in_dtype == FP4_IN_BF16, rows, cols, ld, ldy, rot_size(rotation),
                           sign_mask_of(rotation, seed), static_cast<cudaStream_t>(stream)) != cudaSuccess)
        return FP4_ERR_CUDA;
    return FP4_OK;
}

fp4_status_t fp4_quantize(const void* x, fp4_in_dtype_t in_dtype, int64_t rows, int64_t cols, int64_t ld,
                          fp4_format_t format, fp4_rounding_t rounding, fp4_rotation_t rotation, int axis,
                          int double_block, uint64_t seed, uint32_t tensor_id, const float* tensor_amax,
                          uint8_t* codes, uint8_t* scales, float* outer_scales, float* tensor_scale,
                          void* workspace, size_t workspace_bytes, void* stream) {
    fp4_status_t st = check_input(x, in_dtype, rows, cols, ld, rotation, axis);
    if (st != FP4_OK) return st;
    if (format < FP4_MXFP4 || format > FP4_UFP4) return FP4_ERR_INVALID_ARG;
    if (rounding != FP4_RTNE && rounding != FP4_SR) return FP4_ERR_INVALID_ARG;
    if (double_block != 0 && double_block != 1) return FP4_ERR_INVALID_ARG;
    if (double_block && format != FP4_NVFP4) return FP4_ERR_INVALID_ARG;
    const int64_t K = axis ? cols : rows, L = axis ? rows : cols;
    const int64_t blk = (format == FP4_MXFP4) ? 32 : 16;
    if (K % blk) return FP4_ERR_UNSUPPORTED_SHAPE;
    if (double_block && K % 128) return FP4_ERR_UNSUPPORTED_SHAPE;
    const bool needs_ts = format != FP4_MXFP4 && !double_block;
    const bool internal_amax = needs_ts && tensor_amax == nullptr;
    const bool empty = (L == 0 || K == 0);
    if (!empty && (!codes || !scales)) return FP4_ERR_INVALID_ARG;
    if (!empty && double_block && !outer_scales) return FP4_ERR_INVALID_ARG;
    if (needs_ts && !tensor_scale) return FP4_ERR_INVALID_ARG;
    if (codes && !aligned16(codes)) return FP4_ERR_MISALIGNED;
    if ((outer_scales && ((uintptr_t)outer_scales & 3u)) || (tensor_scale && ((uintptr_t)tensor_scale & 3u)) ||
        (tensor_amax && ((uintptr_t)tensor_amax & 3u)))
        return FP4_ERR_MISALIGNED;
    if (internal_amax && !empty) {
        if (!workspace || workspace_bytes < 256) return FP4_ERR_WORKSPACE;
        if (!aligned16(workspace)) return FP4_ERR_MISALIGNED;
    }
    int dev;
    if ((st = device_ready(&dev)) != FP4_OK) return st;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (empty) {
        if (needs_ts) {
            static const float one = 1.0f;
            if (cudaMemcpyAsync(tensor_scale, &one, sizeof(float), cudaMemcpyHostToDevice, s) != cudaSuccess)
                return FP4_ERR_CUDA;
        }
        return FP4_OK;
    }

    QuantArgs a{};
    a.x = x; a.rows = rows; a.cols = cols; a.ld = ld;
    a.L = L; a.K = K;
    a.nb4 = ((K / blk) + 3) / 4;
    a.codes = codes; a.scales = scales; a.outer = outer_scales;
    a.tensor_scale_out = needs_ts ? tensor_scale : nullptr;
    a.keys = make_keys(seed);
    a.tensor_id = tensor_id;
    a.sign_mask = sign_mask_of(rotation, seed);
    a.err = device_error_word();
    a.wait_limit = g_wait_limit;
    const int rn = rot_size(rotation);
    const bool bf16 = in_dtype == FP4_IN_BF16;
    if (internal_amax) {
        // workspace words: 0 the amax (binary32 bits), 1 the grid-barrier count
        if (cudaMemsetAsync(workspace, 0, 2 * sizeof(unsigned int), s) != cudaSuccess) return FP4_ERR_CUDA;
        a.amax_out = static_cast<unsigned int*>(workspace);
        a.grid_count = static_cast<unsigned int*>(workspace) + 1;
        a.amax_in = static_cast<const float*>(workspace);
        // one launch on either axis: amax pass, grid barrier, quantize pass
        if (launch_quantize_fused(a, bf16, format, rounding == FP4_SR, rn, axis, s) != cudaSuccess)
            return FP4_ERR_CUDA;
        return FP4_OK;
    } else {
        a.amax_in = tensor_amax;
    }
    if (launch_quantize(a, bf16, format, rounding == FP4_SR, rn, double_block != 0, axis, s) != cudaSuccess)
        return FP4_ERR_CUDA;
    return FP4_OK;
}

fp4_status_t fp4_quantize_both_axes(const void* x, fp4_in_dtype_t in_dtype, int64_t rows, int64_t cols, int64_t ld,
                                    fp4_format_t format, fp4_rotation_t rotation, uint64_t seed,
                                    fp4_rounding_t rounding_rows, uint32_t tensor_id_rows, uint8_t* codes_rows,
                                    uint8_t* scales_rows, float* tensor_scale_rows, fp4_rounding_t rounding_cols,
                                    uint32_t tensor_id_cols, uint8_t* codes_cols, uint8_t* scales_cols,
                                    float* tensor_scale_cols, void* workspace, size_t workspace_bytes,
                                    void* stream) {
    fp4_status_t st = check_input(x, in_dtype, rows, cols, ld, rotation, 1);
    if (st != FP4_OK) return st;
    if (format < FP4_MXFP4 || format > FP4_UFP4) return FP4_ERR_INVALID_ARG;
    if (rounding_rows != FP4_RTNE && rounding_rows != FP4_SR) return FP4_ERR_INVALID_ARG;
    if (rounding_cols != FP4_RTNE && rounding_cols != FP4_SR) return FP4_ERR_INVALID_ARG;
    if (!tensor_scale_rows || !tensor_scale_cols) return FP4_ERR_INVALID_ARG;
    if (in_dtype != FP4_IN_BF16 || format == FP4_MXFP4) return FP4_ERR_UNSUPPORTED;
    if (rotation != FP4_ROT_NONE && rotation != FP4_ROT_H16) return FP4_ERR_UNSUPPORTED;
    if (rows % 16 || cols % 64) return FP4_ERR_UNSUPPORTED_SHAPE;
    const bool empty = rows == 0 || cols == 0;
    if (!empty && (!codes_rows || !scales_rows || !codes_cols || !scales_cols)) return FP4_ERR_INVALID_ARG;
    if ((codes_rows && !aligned16(codes_rows)) || (codes_cols && !aligned16(codes_cols)) ||
        ((uintptr_t)tensor_scale_rows & 3u) || ((uintptr_t)tensor_scale_cols & 3u))
        return FP4_ERR_MISALIGNED;
    if (!empty) {
        if (!workspace || workspace_bytes < 256) return FP4_ERR_WORKSPACE;
        if (!aligned16(workspace)) return FP4_ERR_MISALIGNED;
    }
    int dev;
    if ((st = device_ready(&dev)) != FP4_OK) return st;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (empty) {
        static const float one = 1.0f;
        if (cudaMemcpyAsync(tensor_scale_rows, &one, sizeof(float), cudaMemcpyHostToDevice, s) != cudaSuccess ||
            cudaMemcpyAsync(tensor_scale_cols, &one, sizeof(float), cudaMemcpyHostToDevice, s) != cudaSuccess)
            return FP4_ERR_CUDA;
        return FP4_OK;
    }
    // workspace words: 0 the column-axis amax, 1 the grid-barrier count, 2 the row-axis amax
    if (cudaMemsetAsync(workspace, 0, 3 * sizeof(unsigned int), s) != cudaSuccess) return FP4_ERR_CUDA;
    unsigned int* words = static_cast<unsigned int*>(workspace);
    QuantArgs a{};
    a.x = x; a.rows = rows; a.cols = cols; a.ld = ld;
    a.L = cols; a.K = rows;
    a.nb4 = ((rows / 16) + 3) / 4;
    a.codes = codes_cols; a.scales = scales_cols;
    a.tensor_scale_out = tensor_scale_cols;
    a.amax_out = words;
    a.grid_count = words + 1;
    a.amax_in = reinterpret_cast<const float*>(words);
    a.keys = make_keys(seed);
    a.tensor_id = tensor_id_cols;
    a.sign_mask = sign_mask_of(rotation, seed);
    a.err = device_error_word();
    a.wait_limit = g_wait_limit;
    RowOut ro{};
    ro.codes = codes_rows; ro.scales = scales_rows;
    ro.tensor_scale_out = tensor_scale_rows;
    ro.amax_out = words + 2;
    ro.nb4 = ((cols / 16) + 3) / 4;
    ro.tensor_id = tensor_id_rows;
    if (launch_both_axes(a, ro, format, rounding_cols == FP4_SR, rounding_rows == FP4_SR, rot_size(rotation), s) !=
        cudaSuccess)
        return FP4_ERR_CUDA;
    return FP4_OK;
}

fp4_status_t fp4_mxnorm_quantize(const void* x, fp4_in_dtype_t in_dtype, int64_t rows, int64_t cols, int64_t ld,
                                 fp4_format_t format, fp4_rounding_t rounding, int p, float c, uint64_t seed,
                                 uint32_t tensor_id, uint8_t* codes, uint8_t* scales, float* tensor_scale,
                                 float* rho, void* workspace, size_t workspace_bytes, void* stream) {
    fp4_status_t st = check_input(x, in_dtype, rows, cols, ld, FP4_ROT_NONE, 1);
    if (st != FP4_OK) return st;
    if (format < FP4_MXFP4 || format > FP4_UFP4) return FP4_ERR_INVALID_ARG;
    if (rounding != FP4_RTNE && rounding != FP4_SR) return FP4_ERR_INVALID_ARG;
    if (p != 1 && p != 2) return FP4_ERR_INVALID_ARG;
    if (!(c > 0.0f) || !(c <= 3.4028234663852886e38f)) return FP4_ERR_INVALID_ARG;   // positive and finite
    const int64_t blk = (format == FP4_MXFP4) ? 32 : 16;
    const bool needs_ts = format != FP4_MXFP4;
    if (rows > 0 && (cols == 0 || cols % blk || cols > 16384)) return FP4_ERR_UNSUPPORTED_SHAPE;
    if (needs_ts && !tensor_scale) return FP4_ERR_INVALID_ARG;
    if (rows > 0 && (!codes || !scales || !rho)) return FP4_ERR_INVALID_ARG;
    if ((codes && !aligned16(codes)) || (rho && ((uintptr_t)rho & 3u)) ||
        (tensor_scale && ((uintptr_t)tensor_scale & 3u)))
        return FP4_ERR_MISALIGNED;
    if (needs_ts && rows > 0) {
        if (!workspace || workspace_bytes < 256) return FP4_ERR_WORKSPACE;
        if (!aligned16(workspace)) return FP4_ERR_MISALIGNED;
    }
    int dev;
    if ((st = device_ready(&dev)) != FP4_OK) return st;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (rows == 0) {
        if (needs_ts) {
            static const float one = 1.0f;
            if (cudaMemcpyAsync(tensor_scale, &one, sizeof(float), cudaMemcpyHostToDevice, s) != cudaSuccess)
                return FP4_ERR_CUDA;
        }
        return FP4_OK;
    }
    unsigned int* amax_word = nullptr;
    if (needs_ts) {
        amax_word = static_cast<unsigned int*>(workspace);
        if (cudaMemsetAsync(amax_word, 0, sizeof(unsigned int), s) != cudaSuccess) return FP4_ERR_CUDA;
    }
    if (launch_mxnorm(x, in_dtype == FP4_IN_BF16, rows, cols, ld, format, rounding == FP4_SR, p, (double)c, codes,
                      scales, needs_ts ? tensor_scale : nullptr, rho, amax_word, make_keys(seed), tensor_id, s) !=
        cudaSuccess)
        return FP4_ERR_CUDA;
    return FP4_OK;
}

fp4_status_t fp4_channel_amax(const void* x, fp4_in_dtype_t in_dtype, int64_t rows, int64_t cols, int64_t ld,
                              float* amax_out, void* stream) {
    fp4_status_t st = check_input(x, in_dtype, rows, cols, ld, FP4_ROT_NONE, 1);
    if (st != FP4_OK) return st;
    if (cols > 0 && !amax_out) return FP4_ERR_INVALID_ARG;
    if (amax_out && ((uintptr_t)amax_out & 3u)) return FP4_ERR_MISALIGNED;
    int dev;
    if ((st = device_ready(&dev)) != FP4_OK) return st;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (cols == 0) return FP4_OK;
    if (cudaMemsetAsync(amax_out, 0, (size_t)cols * sizeof(float), s) != cudaSuccess) return FP4_ERR_CUDA;
    if (rows == 0) return FP4_OK;
    if (launch_channel_amax(x, in_dtype == FP4_IN_BF16, rows, cols, ld, amax_out, s) != cudaSuccess)
        return FP4_ERR_CUDA;
    return FP4_OK;
}

// workspace of fp4_outctl_quantize: [0, 256) the FP4 part's amax and grid
// count, [256, 272) the FP8 part's amax, then the channel mask
static size_t outctl_ws_bytes(int64_t cols) {
    return 272 + (size_t)((cols + 127) / 128) * 16;
}

fp4_status_t fp4_outctl_workspace_size(int64_t cols, size_t* bytes) {
    if (!bytes || cols < 0) return FP4_ERR_INVALID_ARG;
    *bytes = outctl_ws_bytes(cols);
    return FP4_OK;
}

fp4_status_t fp4_outctl_quantize(const void* x, fp4_in_dtype_t in_dtype, int64_t rows, int64_t cols, int64_t ld,
                                 const int32_t* channels, int64_t n_channels, int64_t k8, fp4_rounding_t rounding,
                                 fp4_rotation_t rotation, uint64_t seed, uint32_t tensor_id, uint8_t* codes,
                                 uint8_t* scales, float* tensor_scale, uint8_t* codes8, float* scale8,
                                 void* workspace, size_t workspace_bytes, void* stream) {
    fp4_status_t st = check_input(x, in_dtype, rows, cols, ld, rotation, 1);
    if (st != FP4_OK) return st;
    if (rounding != FP4_RTNE && rounding != FP4_SR) return FP4_ERR_INVALID_ARG;
    if (n_channels < 0 || k8 < 0 || n_channels > k8 || n_channels > cols) return FP4_ERR_INVALID_ARG;
    if (n_channels > 0 && !channels) return FP4_ERR_INVALID_ARG;
    if (cols % 16 || k8 % 128) return FP4_ERR_UNSUPPORTED_SHAPE;
    if (!tensor_scale || !scale8) return FP4_ERR_INVALID_ARG;
    const bool empty = rows == 0 || cols == 0;
    if (!empty && (!codes || !scales)) return FP4_ERR_INVALID_ARG;
    if (rows > 0 && k8 > 0 && !codes8) return FP4_ERR_INVALID_ARG;
    if ((codes && !aligned16(codes)) || (codes8 && !aligned16(codes8)) || ((uintptr_t)tensor_scale & 3u) ||
        ((uintptr_t)scale8 & 3u) || (channels && ((uintptr_t)channels & 3u)))
        return FP4_ERR_MISALIGNED;
    if (!workspace || workspace_bytes < outctl_ws_bytes(cols)) return FP4_ERR_WORKSPACE;
    if (!aligned16(workspace)) return FP4_ERR_MISALIGNED;
    int dev;
    if ((st = device_ready(&dev)) != FP4_OK) return st;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (cudaMemsetAsync(workspace, 0, outctl_ws_bytes(cols), s) != cudaSuccess) return FP4_ERR_CUDA;
    uint8_t* ws = static_cast<uint8_t*>(workspace);
    unsigned int* amax8 = reinterpret_cast<unsigned int*>(ws + 256);
    uint32_t* mask = reinterpret_cast<uint32_t*>(ws + 272);
    const bool bf16 = in_dtype == FP4_IN_BF16;
    if (empty) {
        static const float one = 1.0f;
        if (cudaMemcpyAsync(tensor_scale, &one, sizeof(float), cudaMemcpyHostToDevice, s) != cudaSuccess ||
            cudaMemcpyAsync(scale8, &one, sizeof(float), cudaMemcpyHostToDevice, s) != cudaSuccess)
            return FP4_ERR_CUDA;
        return FP4_OK;
    }
    if (launch_channel_mask(channels, n_channels, cols, mask, s) != cudaSuccess) return FP4_ERR_CUDA;
    // the FP4 part: NVFP4 along the rows with the channels read as +0
    QuantArgs a{};
    a.x = x; a.rows = rows; a.cols = cols; a.ld = ld;
    a.L = rows; a.K = cols;
    a.nb4 = ((cols / 16) + 3) / 4;
    a.codes = codes; a.scales = scales;
    a.tensor_scale_out = tensor_scale;
    a.keys = make_keys(seed);
    a.tensor_id = tensor_id;
    a.sign_mask = sign_mask_of(rotation, seed);
    a.err = device_error_word();
    a.wait_limit = g_wait_limit;
    a.amax_out = reinterpret_cast<unsigned int*>(ws);
    a.grid_count = reinterpret_cast<unsigned int*>(ws) + 1;
    a.amax_in = reinterpret_cast<const float*>(ws);
    a.chan_mask = mask;
    if (launch_quantize_fused(a, bf16, FP4_NVFP4, rounding == FP4_SR, rot_size(rotation), 1, s) != cudaSuccess)
        return FP4_ERR_CUDA;
    // the FP8 part
    if (launch_fp8_gather(x, bf16, rows, cols, ld, channels, n_channels, k8, amax8, codes8, scale8, s) != cudaSuccess)
        return FP4_ERR_CUDA;
    return FP4_OK;
}

fp4_status_t fp4_gemm_outctl(const uint8_t* a_codes, const uint8_t* a_scales, const float* a_tensor_scale,
                             const uint8_t* b_codes, const uint8_t* b_scales, const float* b_tensor_scale,
                             const uint8_t* a8_codes, const float* a8_scale, const uint8_t* b8_codes,
                             const float* b8_scale, int64_t M, int64_t N, int64_t K, int64_t K8, void* c,
                             fp4_out_dtype_t out_dtype, int64_t ldc, void* stream) {
    if (out_dtype != FP4_OUT_F32 && out_dtype != FP4_OUT_BF16) return FP4_ERR_INVALID_ARG;
    if (M < 0 || N < 0 || K < 0 || K8 < 0 || ldc < N) return FP4_ERR_INVALID_ARG;
    if (M == 0 || N == 0) return FP4_OK;
    if (M % 128 || N % 128 || K % 128 || K == 0 || K8 % 128) return FP4_ERR_UNSUPPORTED_SHAPE;
    if (!a_codes || !a_scales || !b_codes || !b_scales || !c || !a_tensor_scale || !b_tensor_scale)
        return FP4_ERR_INVALID_ARG;
    if (K8 > 0 && (!a8_codes || !b8_codes || !a8_scale || !b8_scale)) return FP4_ERR_INVALID_ARG;
    const int64_t es = out_dtype == FP4_OUT_BF16 ? 2 : 4;
    if (!aligned16(a_codes) || !aligned16(b_codes) || !aligned16(a_scales) || !aligned16(b_scales) ||
        !aligned16(c) || (ldc * es) % 16 || (K8 > 0 && (!aligned16(a8_codes) || !aligned16(b8_codes))))
        return FP4_ERR_MISALIGNED;
    int dev;
    fp4_status_t st;
    if ((st = device_ready(&dev)) != FP4_OK) return st;
    OutctlGemmArgs g{};
    g.a_codes = a_codes; g.a_scales = a_scales; g.a_ts = a_tensor_scale;
    g.b_codes = b_codes; g.b_scales = b_scales; g.b_ts = b_tensor_scale;
    g.a8_codes = a8_codes; g.a8_scale = a8_scale; g.b8_codes = b8_codes; g.b8_scale = b8_scale;
    g.M = M; g.N = N; g.K = K; g.K8 = K8; g.c = c; g.ldc = ldc;
    g.out_bf16 = out_dtype == FP4_OUT_BF16;
    g.wait_limit = g_wait_limit;
    if (launch_gemm_outctl(g, static_cast<cudaStream_t>(stream)) != cudaSuccess) return FP4_ERR_CUDA;
    return FP4_OK;
}

fp4_status_t fp4_requantize(const uint8_t* src_codes, const uint8_t* src_scales, const float* src_outer,
                            const float* src_tensor_scale, int64_t lines, int64_t K, fp4_format_t src_format,
                            int src_double_block, fp4_format_t format, fp4_rounding_t rounding,
                            fp4_rotation_t rotation, int double_block, uint64_t seed, uint32_t tensor_id,
                            const float* tensor_amax, uint8_t* codes, uint8_t* scales, float* outer_scales,
                            float* tensor_scale, void* workspace, size_t workspace_bytes, void* stream) {
    // the source: `lines` lines of K elements (the rows of X^ [lines, K])
    if (src_format < FP4_MXFP4 || src_format > FP4_UFP4) return FP4_ERR_INVALID_ARG;
    if (src_double_block != 0 && src_double_block != 1) return FP4_ERR_INVALID_ARG;
    if (src_double_block && src_format != FP4_NVFP4) return FP4_ERR_INVALID_ARG;
    // the result: X^ quantized along axis 0, i.e. K lines of `lines` elements
    if (format < FP4_MXFP4 || format > FP4_UFP4) return FP4_ERR_INVALID_ARG;
    if (rounding != FP4_RTNE && rounding != FP4_SR) return FP4_ERR_INVALID_ARG;
    if (rotation < FP4_ROT_NONE || rotation > FP4_ROT_RH32) return FP4_ERR_INVALID_ARG;
    if (double_block != 0 && double_block != 1) return FP4_ERR_INVALID_ARG;
    if (double_block && format != FP4_NVFP4) return FP4_ERR_INVALID_ARG;
    if (lines < 0 || K < 0) return FP4_ERR_INVALID_ARG;
    const bool empty = (lines == 0 || K == 0);
    const int64_t sblk = (src_format == FP4_MXFP4) ? 32 : 16;
    if (K % 16 || K % sblk || (src_double_block && K % 128)) return FP4_ERR_UNSUPPORTED_SHAPE;
    const int64_t blk = (format == FP4_MXFP4) ? 32 : 16;
    const int rn = rot_size(rotation);
    if (lines % blk || (rn && lines % rn) || (double_block && lines % 128)) return FP4_ERR_UNSUPPORTED_SHAPE;
    const bool src_ts = src_format != FP4_MXFP4 && !src_double_block;
    const bool needs_ts = format != FP4_MXFP4 && !double_block;
    const bool internal_amax = needs_ts && tensor_amax == nullptr;
    if (!empty) {
        if (!src_codes || !src_scales || (src_double_block && !src_outer) || (src_ts && !src_tensor_scale))
            return FP4_ERR_INVALID_ARG;
        if (!codes || !scales || (double_block && !outer_scales)) return FP4_ERR_INVALID_ARG;
        if (!aligned16(src_codes) || !aligned16(codes)) return FP4_ERR_MISALIGNED;
    }
    if (needs_ts && !tensor_scale) return FP4_ERR_INVALID_ARG;
    if ((src_outer && ((uintptr_t)src_outer & 3u)) || (src_tensor_scale && ((uintptr_t)src_tensor_scale & 3u)) ||
        (outer_scales && ((uintptr_t)outer_scales & 3u)) || (tensor_scale && ((uintptr_t)tensor_scale & 3u)) ||
        (tensor_amax && ((uintptr_t)tensor_amax & 3u)))
        return FP4_ERR_MISALIGNED;
    if (internal_amax && !empty) {
        if (!workspace || workspace_bytes < 256) return FP4_ERR_WORKSPACE;
        if (!aligned16(workspace)) return FP4_ERR_MISALIGNED;
    }
    int dev;
    fp4_status_t st;
    if ((st = device_ready(&dev)) != FP4_OK) return st;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (empty) {
        if (needs_ts) {
            static const float one = 1.0f;
            if (cudaMemcpyAsync(tensor_scale, &one, sizeof(float), cudaMemcpyHostToDevice, s) != cudaSuccess)
                return FP4_ERR_CUDA;
        }
        return FP4_OK;
    }
    QuantArgs a{};
    a.x = nullptr; a.rows = lines; a.cols = K; a.ld = K;
    a.L = K; a.K = lines;
    a.nb4 = ((lines / blk) + 3) / 4;
    a.codes = codes; a.scales = scales; a.outer = outer_scales;
    a.tensor_scale_out = needs_ts ? tensor_scale : nullptr;
    a.keys = make_keys(seed);
    a.tensor_id = tensor_id;
    a.sign_mask = sign_mask_of(rotation, seed);
    a.err = device_error_word();
    a.wait_limit = g_wait_limit;
    a.src_codes = src_codes; a.src_scales = src_scales; a.src_outer = src_outer;
    a.src_ts = src_tensor_scale;
    a.src_fmt = src_format; a.src_db = src_double_block;
    a.src_nb4 = ((K / sblk) + 3) / 4;
    if (internal_amax) {
        if (cudaMemsetAsync(workspace, 0, 2 * sizeof(unsigned int), s) != cudaSuccess) return FP4_ERR_CUDA;
        a.amax_out = static_cast<unsigned int*>(workspace);
        if (launch_requant_amax_cols(a, rn, a.sign_mask != 0u, s) != cudaSuccess) return FP4_ERR_CUDA;
        a.amax_in = static_cast<const float*>(workspace);
    } else {
        a.amax_in = tensor_amax;
    }
    if (launch_requantize_cols(a, format, rounding == FP4_SR, rn, a.sign_mask != 0u, double_block != 0, s) !=
        cudaSuccess)
        return FP4_ERR_CUDA;
    return FP4_OK;
}

fp4_status_t fp4_gemm_workspace_size(fp4_format_t format, int double_block, int64_t M, int64_t N, int64_t K,
                                     size_t* bytes) {
    if (!bytes || format < FP4_MXFP4 || format > FP4_UFP4 || M < 0 || N < 0 || K < 0) return FP4_ERR_INVALID_ARG;
    if (double_block != 0 && double_block != 1) return FP4_ERR_INVALID_ARG;
    *bytes = (format == FP4_UFP4 && !double_block && M > 0 && N > 0 && K > 0)
                 ? ufp4_split_bytes(M, K) + ufp4_split_bytes(N, K) : 0;
    return FP4_OK;
}

fp4_status_t fp4_gemm(fp4_format_t format, int double_block,
                      const uint8_t* a_codes, const uint8_t* a_scales, const float* a_outer,
                      const float* a_tensor_scale,
                      const uint8_t* b_codes, const uint8_t* b_scales, const float* b_outer,
                      const float* b_tensor_scale,
                      int64_t M, int64_t N, int64_t K, void* c, fp4_out_dtype_t out_dtype, int64_t ldc,
                      void* workspace, size_t workspace_bytes, void* stream) {
    if (format < FP4_MXFP4 || format > FP4_UFP4) return FP4_ERR_INVALID_ARG;
    if (double_block != 0 && double_block != 1) return FP4_ERR_INVALID_ARG;
    if (double_block && format != FP4_NVFP4) return FP4_ERR_INVALID_ARG;
    if (out_dtype != FP4_OUT_F32 && out_dtype != FP4_OUT_BF16) return FP4_ERR_INVALID_ARG;
    if (M < 0 || N < 0 || K < 0 || ldc < N) return FP4_ERR_INVALID_ARG;
    if (M == 0 || N == 0) return FP4_OK;
    if (M % 128 || N % 128 || K % 128 || K == 0) return FP4_ERR_UNSUPPORTED_SHAPE;
    if (!a_codes || !a_scales || !b_codes || !b_scales || !c) return FP4_ERR_INVALID_ARG;
    if (format != FP4_MXFP4 && !double_block && (!a_tensor_scale || !b_tensor_scale)) return FP4_ERR_INVALID_ARG;
    if (double_block && (!a_outer || !b_outer)) return FP4_ERR_INVALID_ARG;
    const int64_t es = out_dtype == FP4_OUT_BF16 ? 2 : 4;
    if (!aligned16(a_codes) || !aligned16(b_codes) || !aligned16(a_scales) || !aligned16(b_scales) ||
        !aligned16(c) || (ldc * es) % 16 || (double_block && (!aligned16(a_outer) || !aligned16(b_outer))))
        return FP4_ERR_MISALIGNED;
    const size_t split_a = format == FP4_UFP4 ? ufp4_split_bytes(M, K) : 0;
    if (format == FP4_UFP4) {
        if (!workspace || workspace_bytes < split_a + ufp4_split_bytes(N, K)) return FP4_ERR_WORKSPACE;
        if (!aligned16(workspace)) return FP4_ERR_MISALIGNED;
    }
    int dev;
    fp4_status_t st;
    if ((st = device_ready(&dev)) != FP4_OK) return st;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (format == FP4_UFP4) {
        // A B^T = A1 B1^T + A1 B2^T + A2 B1^T + A2 B2^T with A = A1 + A2, B = B1 + B2
        // in E2M1 under the same block scales: one NVFP4 GEMM over 4 Kp
        uint8_t* wa = static_cast<uint8_t*>(workspace);
        uint8_t* wb = wa + split_a;
        if (launch_ufp4_split(a_codes, a_scales, M, K, wa, false, s) != cudaSuccess ||
            launch_ufp4_split(b_codes, b_scales, N, K, wb, true, s) != cudaSuccess)
            return FP4_ERR_CUDA;
        const int64_t Kp = (K + 255) / 256 * 256;
        GemmArgs g{};
        g.a_codes = wa;
        g.a_scales = wa + ((size_t)M * (size_t)(2 * Kp) + 1023) / 1024 * 1024;
        g.a_ts = a_tensor_scale;
        g.b_codes = wb;
        g.b_scales = wb + ((size_t)N * (size_t)(2 * Kp) + 1023) / 1024 * 1024;
        g.b_ts = b_tensor_scale;
        g.M = M; g.N = N; g.K = 4 * Kp; g.c = c; g.ldc = ldc;
        g.out_bf16 = out_dtype == FP4_OUT_BF16;
        g.fmt = FP4_NVFP4;
        g.db = 0;
        g.pairs = g_gemm_pairs;
        g.wait_limit = g_wait_limit;
        if (launch_gemm(g, s) != cudaSuccess) return FP4_ERR_CUDA;
        return FP4_OK;
    }
    GemmArgs g{};
    g.a_codes = a_codes; g.a_scales = a_scales; g.a_outer = a_outer; g.a_ts = a_tensor_scale;
    g.b_codes = b_codes; g.b_scales = b_scales; g.b_outer = b_outer; g.b_ts = b_tensor_scale;
    g.M = M; g.N = N; g.K = K; g.c = c; g.ldc = ldc;
    g.out_bf16 = out_dtype == FP4_OUT_BF16;
    g.fmt = format;
    g.db = double_block;
    g.pairs = g_gemm_pairs;
    g.wait_limit = g_wait_limit;
    if (launch_gemm(g, s) != cudaSuccess) return FP4_ERR_CUDA;
    return FP4_OK;
}

fp4_status_t fp4_last_error(void* stream) {
    int dev;
    fp4_status_t st;
    if ((st = device_ready(&dev)) != FP4_OK) return st;
    if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess) return FP4_ERR_CUDA;
    unsigned int word = 0;
    if (cudaMemcpyFromSymbol(&word, g_error_word, sizeof(word)) != cudaSuccess) return FP4_ERR_CUDA;
    const unsigned int zero = 0;
    if (cudaMemcpyToSymbol(g_error_word, &zero, sizeof(zero)) != cudaSuccess) return FP4_ERR_CUDA;
    return word ? static_cast<fp4_status_t>(word) : FP4_OK;
}

}  // extern "C"
