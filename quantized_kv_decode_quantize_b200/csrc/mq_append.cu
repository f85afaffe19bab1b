// Quantize-on-append (K8/V4) into the paged cache.
//
// The codec is the deep dive's attention_decode_k8v4 codec (blog.123qwe.co.kr on
// magnitudedev/magnitude, section 5: "Key 8-bit, Value 4-bit, group 32, f16
// scale"), with this library's symmetric reading:
//   K per (token, kv-head):        s = fp16_rn(max|x| / 127), code = clamp(rne(x / s), -127, 127)
//   V per (token, kv-head, 32 ch): s = fp16_rn(max|x| / 7),   code = clamp(rne(x / s), -8, 7)
// Both divisions are IEEE fp32 (__fdiv_rn), rounding is to nearest even, and a
// zero scale gives code 0.  One warp handles one (token, kv-head): each lane
// reads D/32 consecutive channels with one vector load, the absmax reductions
// are warp shuffles (exact: max is order-independent), each lane stores its K
// codes with one 4- or 8-byte store, and writes its V codes into the channel-major
// V words of the page (see mq_device.cuh).  A V word holds the codes of eight
// tokens, so its nibble is replaced with two atomic bit operations (clear, then
// set): appends of neighbouring tokens in one launch may touch the same word.
#include "mq_device.cuh"
#include "mq_kernels.h"

namespace mq {

template <typename T>
__device__ __forceinline__ float to_f32(T v);
template <>
__device__ __forceinline__ float to_f32<float>(float v) { return v; }
template <>
__device__ __forceinline__ float to_f32<__nv_bfloat16>(__nv_bfloat16 v) { return __bfloat162float(v); }
template <>
__device__ __forceinline__ float to_f32<__half>(__half v) { return __half2float(v); }

// N consecutive elements starting at p (16-byte or 8-byte aligned) -> floats
template <typename T, int N>
__device__ __forceinline__ void load_vec(const T* p, float (&x)[N]) {
    constexpr int BYTES = N * sizeof(T);
    static_assert(BYTES % 8 == 0, "vector width");
    if constexpr (BYTES % 16 == 0) {
#pragma unroll
        for (int i = 0; i < BYTES / 16; i++) {
            uint4 u = __ldg(reinterpret_cast<const uint4*>(p) + i);
            const T* e = reinterpret_cast<const T*>(&u);
#pragma unroll
            for (int j = 0; j < 16 / (int)sizeof(T); j++) x[i * (16 / sizeof(T)) + j] = to_f32<T>(e[j]);
        }
    } else {
#pragma unroll
        for (int i = 0; i < BYTES / 8; i++) {
            uint2 u = __ldg(reinterpret_cast<const uint2*>(p) + i);
            const T* e = reinterpret_cast<const T*>(&u);
#pragma unroll
            for (int j = 0; j < 8 / (int)sizeof(T); j++) x[i * (8 / sizeof(T)) + j] = to_f32<T>(e[j]);
        }
    }
}

__device__ __forceinline__ int quant_code(float x, float s, float lo, float hi) {
    if (s == 0.0f) return 0;
    float r = rintf(__fdiv_rn(x, s));   // IEEE division, round half to even
    if (r != r) return 0;               // NaN input
    r = fminf(fmaxf(r, lo), hi);
    return static_cast<int>(r);
}

template <int D, typename T>
__global__ void __launch_bounds__(256) append_kernel(AppendParams p) {
    constexpr int CPL = D / 32;          // channels per lane
    constexpr int LPG = 32 / CPL;        // lanes per 32-channel V group
    const int lane = threadIdx.x & 31;
    // a decode launched after this append may start its set-up now; it waits for this
    // grid (griddepcontrol.wait) before it reads any page
    if (threadIdx.x == 0) asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    const long long item = (long long)blockIdx.x * (blockDim.x / 32) + (threadIdx.x >> 5);
    if (item >= (long long)p.n_tokens * p.n_kv_heads) return;
    const int tok = (int)(item / p.n_kv_heads), h = (int)(item % p.n_kv_heads);

    // sequence of this token: last b with cu_new[b] <= tok (binary search)
    int lo = 0, hi = p.n_seqs - 1;
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (__ldg(p.cu_new + mid) <= tok) lo = mid; else hi = mid - 1;
    }
    const int b = lo;
    const long long pos = (long long)__ldg(p.start_pos + b) + (tok - __ldg(p.cu_new + b));
    if (pos < 0 || pos >= (long long)p.max_blocks_per_seq * kPageTokens) {
        if (lane == 0) atomicOr(p.err, kErrBadPosition);
        return;
    }
    const int blk = __ldg(p.block_table + (long long)b * p.max_blocks_per_seq + pos / kPageTokens);
    if (blk < 0 || (long long)blk >= p.n_blocks) {
        if (lane == 0) atomicOr(p.err, kErrBadBlock);
        return;
    }
    const int tau = (int)(pos % kPageTokens);
    uint8_t* page = p.pool + ((long long)blk * p.n_kv_heads + h) * page_bytes(D);

    const size_t vec = ((size_t)tok * p.n_kv_heads + h) * D + (size_t)lane * CPL;
    float xk[CPL], xv[CPL];
    load_vec<T, CPL>(reinterpret_cast<const T*>(p.k) + vec, xk);
    load_vec<T, CPL>(reinterpret_cast<const T*>(p.v) + vec, xv);

    // ---- K: one scale over all D channels ----
    float a = 0.0f;
#pragma unroll
    for (int i = 0; i < CPL; i++) a = fmaxf(a, fabsf(xk[i]));
    a = warp_max(a);
    const __half sk16 = __float2half_rn(__fdiv_rn(a, 127.0f));
    const float sk = __half2float(sk16);
    uint32_t kb[CPL / 4];
#pragma unroll
    for (int w = 0; w < CPL / 4; w++) {
        uint32_t word = 0;
#pragma unroll
        for (int j = 0; j < 4; j++)
            word |= (uint32_t)(quant_code(xk[4 * w + j], sk, -127.0f, 127.0f) & 0xFF) << (8 * j);
        kb[w] = word;
    }
    const int c0 = lane * CPL;
    uint8_t* kdst = page + k_code_byte(D, tau, c0);
    if constexpr (CPL == 4) {
        *reinterpret_cast<uint32_t*>(kdst) = kb[0];
    } else {
        *reinterpret_cast<uint2*>(kdst) = make_uint2(kb[0], kb[1]);
    }
    if (lane == 0) *reinterpret_cast<__half*>(page + k_scale_byte(D, tau)) = sk16;

    // ---- V: one scale per 32-channel group (LPG lanes) ----
    float av = 0.0f;
#pragma unroll
    for (int i = 0; i < CPL; i++) av = fmaxf(av, fabsf(xv[i]));
#pragma unroll
    for (int o = LPG / 2; o > 0; o >>= 1) av = fmaxf(av, __shfl_xor_sync(0xffffffffu, av, o));
    const __half sv16 = __float2half_rn(__fdiv_rn(av, 7.0f));
    const float sv = __half2float(sv16);
    const int bit = v_nibble_bit(tau);
#pragma unroll
    for (int i = 0; i < CPL; i++) {
        const uint32_t n = (uint32_t)quant_code(xv[i], sv, -8.0f, 7.0f) & 0xFu;
        unsigned* w = reinterpret_cast<unsigned*>(page + v_word_byte(D, tau, c0 + i));
        atomicAnd(w, ~(0xFu << bit));
        atomicOr(w, n << bit);
    }
    if (lane % LPG == 0)
        *reinterpret_cast<__half*>(page + v_scale_byte(D, tau, c0 / 32)) = sv16;
}

template <int D>
static cudaError_t launch_append_d(const AppendParams& p, cudaStream_t st) {
    const long long warps = (long long)p.n_tokens * p.n_kv_heads;
    const int wpb = 8;
    const long long blocks = (warps + wpb - 1) / wpb;
    if (blocks > 0x7fffffffLL) return cudaErrorInvalidConfiguration;
    switch (p.dtype) {
        case 0: append_kernel<D, float><<<(unsigned)blocks, wpb * 32, 0, st>>>(p); break;
        case 1: append_kernel<D, __nv_bfloat16><<<(unsigned)blocks, wpb * 32, 0, st>>>(p); break;
        default: append_kernel<D, __half><<<(unsigned)blocks, wpb * 32, 0, st>>>(p); break;
    }
    return cudaGetLastError();
}

cudaError_t launch_append(const AppendParams& p, int head_dim, cudaStream_t st) {
    return head_dim == 128 ? launch_append_d<128>(p, st) : launch_append_d<256>(p, st);
}

}  // namespace mq
