// philox_draw.cu -- test infrastructure: draws Philox4x32-10 output groups
// through cuRAND's device API, as an independent check of the CPU oracle's
// Philox (tests/test_gpu_philox_curand.py builds and loads it).
//
// curand_init(seed, subsequence, offset, &state) on a Philox state puts the
// 64-bit subsequence in counter words 2-3 and offset / 4 in counter words 0-1
// under the key (lo32(seed), hi32(seed)); the first curand4() of a state
// whose offset is a multiple of 4 returns the Philox output of that counter.
#include <cuda_runtime.h>
#include <curand_kernel.h>

__global__ void draw_groups(const unsigned long long* seeds, const unsigned long long* subseqs,
                            const unsigned long long* groups, uint4* out, int n) {
    const int i = blockIdx.x * blockDim.x + threadIdx.x;
    if (i >= n) return;
    curandStatePhilox4_32_10_t st;
    curand_init(seeds[i], subseqs[i], 4ull * groups[i], &st);
    out[i] = curand4(&st);
}

// host entry: n draws; out receives 4 words per draw.  Returns a cudaError_t.
extern "C" int philox_draw(const unsigned long long* seeds, const unsigned long long* subseqs,
                           const unsigned long long* groups, unsigned int* out, int n) {
    unsigned long long* d = nullptr;
    uint4* o = nullptr;
    const size_t b = (size_t)n * sizeof(unsigned long long);
    cudaError_t e = cudaMalloc(&d, 3 * b);
    if (e == cudaSuccess) e = cudaMalloc(&o, (size_t)n * sizeof(uint4));
    if (e == cudaSuccess) e = cudaMemcpy(d, seeds, b, cudaMemcpyHostToDevice);
    if (e == cudaSuccess) e = cudaMemcpy(d + n, subseqs, b, cudaMemcpyHostToDevice);
    if (e == cudaSuccess) e = cudaMemcpy(d + 2 * n, groups, b, cudaMemcpyHostToDevice);
    if (e == cudaSuccess) {
        draw_groups<<<(n + 127) / 128, 128>>>(d, d + n, d + 2 * n, o, n);
        e = cudaGetLastError();
    }
    if (e == cudaSuccess) e = cudaMemcpy(out, o, (size_t)n * sizeof(uint4), cudaMemcpyDeviceToHost);
    cudaFree(d);
    cudaFree(o);
    return (int)e;
}
