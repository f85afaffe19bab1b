// Helper kernels for the tuner: deterministic probe data, an L2-sized scribble
// between timed launches, and a device-side byte comparison of two outputs.
#include "mq_device.cuh"
#include "mq_kernels.h"

namespace mq {

__device__ __forceinline__ uint64_t mix64(uint64_t x) {
    // SplitMix64 finalizer (Steele, Lea and Flood, "Fast splittable pseudorandom
    // number generators", OOPSLA 2014)
    x += 0x9E3779B97F4A7C15ull;
    x = (x ^ (x >> 30)) * 0xBF58476D1CE4E5B9ull;
    x = (x ^ (x >> 27)) * 0x94D049BB133111EBull;
    return x ^ (x >> 31);
}

__global__ void fill_random_kernel(void* dst, int dtype, long long n, int head_dim, unsigned long long seed) {
    for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < n; i += (long long)gridDim.x * blockDim.x) {
        const uint64_t r = mix64(seed * 0x100000001B3ull + (uint64_t)i);
        float v = ((float)(r >> 40) * (1.0f / 16777216.0f)) * 4.0f - 2.0f;   // uniform [-2, 2)
        if ((i % head_dim) < 4) v *= 10.0f;
        if (dtype == 0) reinterpret_cast<float*>(dst)[i] = v;
        else if (dtype == 1) reinterpret_cast<__nv_bfloat16*>(dst)[i] = __float2bfloat16_rn(v);
        else reinterpret_cast<__half*>(dst)[i] = __float2half_rn(v);
    }
}

cudaError_t launch_fill_random(void* dst, int dtype, long long n, int head_dim, unsigned long long seed,
                               cudaStream_t st) {
    if (n <= 0) return cudaSuccess;
    const long long blocks = std::min<long long>((n + 255) / 256, 65536);
    fill_random_kernel<<<(unsigned)blocks, 256, 0, st>>>(dst, dtype, n, head_dim, seed);
    return cudaGetLastError();
}

__global__ void scribble_kernel(uint4* dst, long long n16, unsigned v) {
    for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < n16; i += (long long)gridDim.x * blockDim.x)
        dst[i] = make_uint4(v, v + 1, v + 2, (unsigned)i);
}

cudaError_t launch_scribble(void* dst, size_t bytes, unsigned v, cudaStream_t st) {
    const long long n16 = (long long)(bytes / 16);
    if (n16 <= 0) return cudaSuccess;
    scribble_kernel<<<1184, 256, 0, st>>>(reinterpret_cast<uint4*>(dst), n16, v);
    return cudaGetLastError();
}

__global__ void compare_kernel(const uint32_t* a, const uint32_t* b, long long n, unsigned* out) {
    bool diff = false;
    for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < n; i += (long long)gridDim.x * blockDim.x)
        diff |= a[i] != b[i];
    if (__any_sync(0xffffffffu, diff) && (threadIdx.x & 31) == 0) atomicOr(out, 1u);
}

cudaError_t launch_compare(const uint32_t* a, const uint32_t* b, long long n32, unsigned* out, cudaStream_t st) {
    if (n32 <= 0) return cudaSuccess;
    const long long blocks = std::min<long long>((n32 + 255) / 256, 4096);
    compare_kernel<<<(unsigned)blocks, 256, 0, st>>>(a, b, n32, out);
    return cudaGetLastError();
}

}  // namespace mq
