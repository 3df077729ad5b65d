// quantize_noalloc.cu -- fp4_quantize for callers that cannot allocate device
// memory: the scratch the tensor-scale path needs lives in a static device
// array of this library instead of a caller-provided workspace.
//
// Who needs it: code that runs where cudaMalloc is unavailable or forbidden --
// a plug-in whose host framework owns every device allocation, or a
// real-time loop that may not touch the allocator.  Such callers still own
// their inputs and outputs; only the scratch words (the amax accumulator and
// a grid-barrier count) move into library-owned memory.  The first call on a
// device resolves the array's address (cudaGetSymbolAddress), so it belongs
// before any stream capture.
#include <cuda_runtime.h>
#include <cstdint>
#include <mutex>

#include "../../include/fp4.h"

namespace {

// Two 32-bit words are used (the rotated-tensor amax and a grid-barrier
// count); the array is sized like the workspace fp4_quantize requests, 256
// bytes.  Every GPU that loads the
// library holds one copy until the process exits.
constexpr size_t kScratchBytes = 256;
static __device__ __align__(256) unsigned char g_noalloc_scratch[kScratchBytes];

constexpr int kMaxDevices = 64;
void* g_scratch_addr[kMaxDevices];
std::mutex g_scratch_mu;

// Device address of the scratch array on the current device.  In host code
// the symbol is only a host-side handle, so the address is resolved once per
// device, with that device current, and cached.
fp4_status_t scratch_address(void** out) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
        cudaGetLastError();
        return FP4_ERR_NO_DEVICE;
    }
    std::lock_guard<std::mutex> lock(g_scratch_mu);
    if (!g_scratch_addr[dev]) {
        void* p = nullptr;
        const cudaError_t e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
        if (e != cudaSuccess || !p) {
            cudaGetLastError();
            return FP4_ERR_CUDA;
        }
        g_scratch_addr[dev] = p;
    }
    *out = g_scratch_addr[dev];
    return FP4_OK;
}

}  // namespace

extern "C" fp4_status_t fp4_quantize_noalloc(const void* x, fp4_in_dtype_t in_dtype, int64_t rows,
                                             int64_t cols, int64_t ld, fp4_format_t format,
                                             fp4_rounding_t rounding, fp4_rotation_t rotation, int axis,
                                             uint64_t seed, uint32_t tensor_id, uint8_t* codes,
                                             uint8_t* scales, float* tensor_scale, void* stream) {
    // only the tensor-scale formats need scratch; MXFP4 and the double block
    // take none and are served by fp4_quantize directly
    if (format != FP4_NVFP4 && format != FP4_UFP4) return FP4_ERR_UNSUPPORTED;
    size_t need = 0;
    fp4_status_t st = fp4_quantize_workspace_size(format, 0, 0, &need);
    if (st != FP4_OK) return st;
    if (need > kScratchBytes) return FP4_ERR_WORKSPACE;    // larger than the static array
    // check what fp4_quantize would reject before anything is launched (it
    // checks the input itself and launches nothing on error)
    if (rounding != FP4_RTNE && rounding != FP4_SR) return FP4_ERR_INVALID_ARG;
    if (axis != 0 && axis != 1) return FP4_ERR_INVALID_ARG;
    if (rows < 0 || cols < 0) return FP4_ERR_INVALID_ARG;
    const int64_t K = axis ? cols : rows, L = axis ? rows : cols;
    const bool empty = (K == 0 || L == 0);
    if (!tensor_scale) return FP4_ERR_INVALID_ARG;
    if (!empty && (!codes || !scales)) return FP4_ERR_INVALID_ARG;
    if (K % 16) return FP4_ERR_UNSUPPORTED_SHAPE;
    if ((codes && ((uintptr_t)codes & 15u)) || ((uintptr_t)tensor_scale & 3u)) return FP4_ERR_MISALIGNED;
    void* scratch = nullptr;
    if ((st = scratch_address(&scratch)) != FP4_OK) return st;
    float* amax = static_cast<float*>(scratch);
    if (empty) {
        return fp4_quantize(x, in_dtype, rows, cols, ld, format, rounding, rotation, axis, 0, seed,
                            tensor_id, amax, codes, scales, nullptr, tensor_scale, nullptr, 0, stream);
    }
    // the static array is the workspace of fp4_quantize's internal amax: it
    // clears it on the stream, then accumulates the rotated-tensor amax (and,
    // on the row axis, the grid-barrier count of its one-launch path) there
    return fp4_quantize(x, in_dtype, rows, cols, ld, format, rounding, rotation, axis, 0, seed, tensor_id,
                        nullptr, codes, scales, nullptr, tensor_scale, scratch, kScratchBytes, stream);
}
