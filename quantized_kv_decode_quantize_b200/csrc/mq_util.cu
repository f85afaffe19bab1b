// Helper kernels for the tuner: deterministic probe data, an L2-sized scribble
// between timed launches, a device-side byte comparison of two outputs, and the
// pieces of the alpha admission rule (a one-format-step perturbation of stored
// pages, the per-point noise it causes, and the check of a candidate against
// alpha times that noise).
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

// ---- storage-resolution noise ----------------------------------------------------
// One step of each stored element's format, in a direction drawn per element from
// SplitMix64 of (seed, element index): an int8 K code or an int4 V code moves by one
// code (towards the inside of its range when the drawn direction would leave it), an
// fp16 scale by one unit in the last place of its magnitude (an infinite or NaN scale
// is left as it is; zero steps up to the smallest subnormal).  Every element of every
// page moves.  The field of a 32-bit word follows from its offset in its record: K
// codes in [0, 8D), V words in [8D, 12D), scales after that.
__device__ __forceinline__ int step_dir(uint64_t seed, uint64_t idx) {
    return (mix64(seed * 0x9E3779B97F4A7C15ull + idx) >> 63) ? 1 : -1;
}

__device__ __forceinline__ int step_code(int v, int d, int lo, int hi) {
    const int w = v + d;
    return (w < lo || w > hi) ? v - d : w;
}

__device__ __forceinline__ uint32_t step_half(uint32_t b, int d) {
    const uint32_t sign = b & 0x8000u, m = b & 0x7FFFu;
    if (m >= 0x7C00u) return b;                       // inf or NaN
    uint32_t n;
    if (d > 0) n = (m + 1 == 0x7C00u) ? m - 1 : m + 1;
    else n = (m == 0) ? 1u : m - 1;
    return sign | n;
}

__global__ void perturb_pages_kernel(const uint32_t* src, uint32_t* dst, long long n_words, int page_words,
                                     int rec_words, int D, unsigned long long seed) {
    for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < n_words;
         i += (long long)gridDim.x * blockDim.x) {
        const uint32_t w = src[i];
        const int wr = (int)(i % page_words) % rec_words;
        const int byte = 4 * wr;
        uint32_t o = 0;
        if (byte < 8 * D) {                            // four int8 K codes
#pragma unroll
            for (int j = 0; j < 4; j++) {
                const int v = (int)(int8_t)((w >> (8 * j)) & 0xFFu);
                o |= (uint32_t)(step_code(v, step_dir(seed, 8ull * i + j), -127, 127) & 0xFF) << (8 * j);
            }
        } else if (byte < 12 * D) {                    // eight int4 V codes
#pragma unroll
            for (int j = 0; j < 8; j++) {
                const int v = (int)((w >> (4 * j)) & 0xFu) - (int)(((w >> (4 * j)) & 0x8u) << 1);
                o |= (uint32_t)(step_code(v, step_dir(seed, 8ull * i + j), -8, 7) & 0xF) << (4 * j);
            }
        } else {                                       // two fp16 scales
            o = step_half(w & 0xFFFFu, step_dir(seed, 8ull * i)) |
                (step_half(w >> 16, step_dir(seed, 8ull * i + 1)) << 16);
        }
        dst[i] = o;
    }
}

cudaError_t launch_perturb_pages(const void* src, void* dst, long long n_pages, int head_dim,
                                 unsigned long long seed, cudaStream_t st) {
    if (n_pages <= 0) return cudaSuccess;
    const int page_words = page_bytes(head_dim) / 4, rec_words = rec_bytes(head_dim) / 4;
    const long long n_words = n_pages * page_words;
    const long long blocks = std::min<long long>((n_words + 255) / 256, 148 * 16);
    perturb_pages_kernel<<<(unsigned)blocks, 256, 0, st>>>(static_cast<const uint32_t*>(src),
                                                            static_cast<uint32_t*>(dst), n_words, page_words,
                                                            rec_words, head_dim, seed);
    return cudaGetLastError();
}

// noise[i] = max(noise[i], |moved[i] - ref[i]|); a NaN on either side counts as an
// infinite movement unless the two bit patterns are equal
__global__ void noise_max_kernel(const float* moved, const float* ref, float* noise, long long n) {
    for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < n; i += (long long)gridDim.x * blockDim.x) {
        const float a = moved[i], b = ref[i];
        float d;
        if (__float_as_uint(a) == __float_as_uint(b)) d = 0.0f;
        else if (a != a || b != b) d = __int_as_float(0x7F800000);
        else d = (float)fabs((double)a - (double)b);
        noise[i] = fmaxf(noise[i], d);
    }
}

cudaError_t launch_noise_max(const float* moved, const float* ref, float* noise, long long n, cudaStream_t st) {
    if (n <= 0) return cudaSuccess;
    const long long blocks = std::min<long long>((n + 255) / 256, 4096);
    noise_max_kernel<<<(unsigned)blocks, 256, 0, st>>>(moved, ref, noise, n);
    return cudaGetLastError();
}

// The alpha rule at every point: |cand - ref| <= alpha * noise.  Sets out[0] when a
// point breaks it and keeps in out[1] the largest |cand - ref| / noise seen, as the
// bits of a non-negative float (0 where the two are bit-identical, +inf where the
// noise is 0 and the point moved, or where a NaN appears on one side only).
__global__ void alpha_check_kernel(const float* cand, const float* ref, const float* noise, long long n, float alpha,
                                   unsigned* out) {
    bool bad = false;
    float worst = 0.0f;
    for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < n; i += (long long)gridDim.x * blockDim.x) {
        const float a = cand[i], b = ref[i];
        if (__float_as_uint(a) == __float_as_uint(b)) continue;
        const double d = (a != a || b != b) ? (double)__int_as_float(0x7F800000) : fabs((double)a - (double)b);
        const double lim = (double)alpha * (double)noise[i];
        bad |= !(d <= lim);
        const double r = noise[i] > 0.0f ? d / (double)noise[i] : (double)__int_as_float(0x7F800000);
        worst = fmaxf(worst, (float)r);
    }
    for (int o = 16; o > 0; o >>= 1) worst = fmaxf(worst, __shfl_xor_sync(0xffffffffu, worst, o));
    const bool any_bad = __any_sync(0xffffffffu, bad);
    if ((threadIdx.x & 31) == 0) {
        if (any_bad) atomicOr(out, 1u);
        if (worst > 0.0f) atomicMax(out + 1, __float_as_uint(worst));
    }
}

cudaError_t launch_alpha_check(const float* cand, const float* ref, const float* noise, long long n, float alpha,
                               unsigned* out, cudaStream_t st) {
    if (n <= 0) return cudaSuccess;
    const long long blocks = std::min<long long>((n + 255) / 256, 4096);
    alpha_check_kernel<<<(unsigned)blocks, 256, 0, st>>>(cand, ref, noise, n, alpha, out);
    return cudaGetLastError();
}

}  // namespace mq
