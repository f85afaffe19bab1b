// Quantize-on-append (K8/V4) into the paged cache.
//
// The codec is the deep dive's attention_decode_k8v4 codec (blog.123qwe.co.kr on
// magnitudedev/magnitude, section 5: "Key 8-bit, Value 4-bit, group 32, f16
// scale"), with this library's symmetric reading:
//   K per (token, kv-head):        s = fp16_rn(max|x| / 127), code = clamp(rne(x / s), -127, 127)
//   V per (token, kv-head, 32 ch): s = fp16_rn(max|x| / 7),   code = clamp(rne(x / s), -8, 7)
// Both divisions are IEEE fp32 (x / s is decided by a multiply with 1/s except next to
// a tie, where __fdiv_rn decides: quant_code), rounding is to nearest even, and a zero
// scale gives code 0.
//
// Work split: one warp per (8-position record, kv-head) that a sequence's new tokens
// touch; the grid is (x, sequence, kv-head), sized from the device's SM count, and the
// warps of a (sequence, kv-head) stride over its records.  A token's head vector is read
// with 16-byte loads, one per lane (two per lane for fp32 at head_dim 256): LPT = min(32,
// D x element size / 16) lanes per token, so at head_dim 128 with 2-byte inputs a warp
// quantizes two tokens at once, one per half-warp.  The absmax reductions are shuffles
// within a token's lanes (exact: max is order-independent); each lane stores its K codes
// with one 4- or 8-byte store.  A V word of the page holds one channel's codes for the 8
// tokens of a record (see mq_device.cuh): when the append covers the whole record, the
// warp assembles every word in registers and writes it with a plain store; otherwise
// (the ragged ends of an append, single-token appends) each nibble is replaced with two
// atomic bit operations (clear, then set), since another launch may have written the
// record's other tokens.

#include <algorithm>

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

// code = clamp(rne(x / s)) with x / s the IEEE fp32 quotient.  inv = 1/s and q = x * inv
// (both correctly rounded) put q within |x / s| * 2^-22.4 of that quotient, under 2^-14
// while |x / s| <= 256 (the scales make |x / s| at most ~127.1, and anything past 127.5
// clamps the same way on both sides); so q and the quotient round to the same integer
// unless q lies within 2^-14 of a half-integer, and only such elements (and NaN) take
// the division.
__device__ __forceinline__ int quant_code(float x, float s, float inv, float lo, float hi) {
    if (s == 0.0f) return 0;
    float q = __fmul_rn(x, inv);
    const float h = fabsf(__fsub_rn(__fsub_rn(q, floorf(q)), 0.5f));
    if (!(h > 0x1p-14f)) q = __fdiv_rn(x, s);   // near a tie: the IEEE division decides
    float r = rintf(q);                         // round half to even
    if (r != r) return 0;                       // NaN input
    r = fminf(fmaxf(r, lo), hi);
    return static_cast<int>(r);
}

// Lanes per token: 16 bytes of the token's head vector per lane, at most a warp.
template <int D, typename T>
struct Lanes {
    static constexpr int LPT = (D * (int)sizeof(T) / 16) < 32 ? D * (int)sizeof(T) / 16 : 32;
    static constexpr int TPW = 32 / LPT;   // tokens per warp
    static constexpr int CPL = D / LPT;    // channels per lane
    static constexpr int LPG = 32 / CPL;   // lanes per 32-channel V group
    static_assert(LPT == 16 || LPT == 32, "lanes per token");
};

// One token's codes, quantized by its LPT lanes (lane l: channels CPL * l ..).
template <int CPL>
struct TokenCodes {
    uint32_t kb[CPL / 4];   // this lane's K codes, 4 per word
    __half sk16;            // K scale (every lane)
    uint32_t vn[CPL];       // this lane's V codes as 4-bit two's complement
    __half sv16;            // V scale of this lane's 32-channel group
};

template <int D, typename T>
__device__ __forceinline__ void quantize_token(const AppendParams& p, long long tok, int h, int l,
                                               TokenCodes<Lanes<D, T>::CPL>& out) {
    using LN = Lanes<D, T>;
    constexpr int CPL = LN::CPL, LPG = LN::LPG;
    const size_t vec = ((size_t)tok * p.n_kv_heads + h) * D + (size_t)l * CPL;
    float xk[CPL], xv[CPL];
    load_vec<T, CPL>(reinterpret_cast<const T*>(p.k) + vec, xk);
    load_vec<T, CPL>(reinterpret_cast<const T*>(p.v) + vec, xv);
    // ---- K: one scale over all D channels (the token's LPT lanes) ----
    float a = 0.0f;
#pragma unroll
    for (int i = 0; i < CPL; i++) a = fmaxf(a, fabsf(xk[i]));
#pragma unroll
    for (int o = LN::LPT / 2; o > 0; o >>= 1) a = fmaxf(a, __shfl_xor_sync(0xffffffffu, a, o));
    out.sk16 = __float2half_rn(__fdiv_rn(a, 127.0f));
    const float sk = __half2float(out.sk16), ik = __frcp_rn(sk);
#pragma unroll
    for (int w = 0; w < CPL / 4; w++) {
        uint32_t word = 0;
#pragma unroll
        for (int j = 0; j < 4; j++)
            word |= (uint32_t)(quant_code(xk[4 * w + j], sk, ik, -127.0f, 127.0f) & 0xFF) << (8 * j);
        out.kb[w] = word;
    }
    // ---- V: one scale per 32-channel group (LPG lanes) ----
    float av = 0.0f;
#pragma unroll
    for (int i = 0; i < CPL; i++) av = fmaxf(av, fabsf(xv[i]));
#pragma unroll
    for (int o = LPG / 2; o > 0; o >>= 1) av = fmaxf(av, __shfl_xor_sync(0xffffffffu, av, o));
    out.sv16 = __float2half_rn(__fdiv_rn(av, 7.0f));
    const float sv = __half2float(out.sv16), iv = __frcp_rn(sv);
#pragma unroll
    for (int i = 0; i < CPL; i++) out.vn[i] = (uint32_t)quant_code(xv[i], sv, iv, -8.0f, 7.0f) & 0xFu;
}

// K codes, K scale and V scale of one token at slot tau of a page (lane l of the token).
template <int D, int CPL>
__device__ __forceinline__ void store_token_kscales(uint8_t* page, int tau, int l, const TokenCodes<CPL>& tc) {
    constexpr int LPG = 32 / CPL;
    const int c0 = l * CPL;
    uint8_t* kdst = page + k_code_byte(D, tau, c0);
    static_assert(CPL == 4 || CPL == 8, "channels per lane");
    if constexpr (CPL == 4) {
        *reinterpret_cast<uint32_t*>(kdst) = tc.kb[0];
    } else {
        *reinterpret_cast<uint2*>(kdst) = make_uint2(tc.kb[0], tc.kb[1]);   // within one 16-channel group
    }
    if (l == 0) *reinterpret_cast<__half*>(page + k_scale_byte(D, tau)) = tc.sk16;
    if (l % LPG == 0) *reinterpret_cast<__half*>(page + v_scale_byte(D, tau, c0 / 32)) = tc.sv16;
}

// The kernel is a programmatic dependent launch: the preceding kernel on the stream may
// still run (a decode or merge of the previous step, which may read the pages written
// here).  The new tokens are read and quantized at once; each thread waits for that
// kernel to complete before its first page write.
__device__ __forceinline__ void grid_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

template <int D, typename T>
__global__ void __launch_bounds__(256) append_kernel(AppendParams p) {
    using LN = Lanes<D, T>;
    constexpr int CPL = LN::CPL, TPW = LN::TPW;
    const int lane = threadIdx.x & 31;
    const int sub = lane / LN::LPT, l = lane % LN::LPT;   // this lane's token of the warp's TPW, its lane there
    // a decode launched after this append may start its set-up now; it waits for this
    // grid (griddepcontrol.wait) before it reads any page
    if (threadIdx.x == 0) asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    const int b = blockIdx.y, h = blockIdx.z;
    const int tok0 = __ldg(p.cu_new + b), tok1 = __ldg(p.cu_new + b + 1);
    if (tok0 < 0 || tok1 < tok0 || tok1 > p.n_tokens) {   // inconsistent cu_new: nothing is read
        if (threadIdx.x == 0 && blockIdx.x == 0) atomicOr(p.err, kErrBadSeq);
        return;
    }
    if (tok1 == tok0) return;
    const long long start = __ldg(p.start_pos + b), end = start + (tok1 - tok0);   // positions [start, end)
    const long long limit = (long long)p.max_blocks_per_seq * kPageTokens;
    const long long r_lo = start >= 0 ? start / 8 : -((-start + 7) / 8);             // floor(start / 8)
    const long long r_hi = (end - 1) >= 0 ? (end - 1) / 8 : -((-(end - 1) + 7) / 8);
    const int wpb = blockDim.x / 32;
    // work items: (record, slice); with several slices a record's 8 positions are shared by
    // that many warps (small appends, which would leave most of the GPU idle), each taking
    // its positions through the atomic path
    const int slices = p.slices, per_slice = 8 / slices;
    for (long long item = r_lo * slices + (long long)blockIdx.x * wpb + (threadIdx.x >> 5); item <= r_hi * slices + slices - 1;
         item += (long long)gridDim.x * wpb) {
        const long long r = item >= 0 ? item / slices : -((-item + slices - 1) / slices);
        const int slice = (int)(item - r * slices);
        // a record lies wholly inside or wholly outside [0, limit): limit is a multiple of 16
        if (8 * r < 0 || 8 * r >= limit) {
            if (lane == 0) atomicOr(p.err, kErrBadPosition);
            continue;
        }
        const int blk = __ldg(p.block_table + (long long)b * p.max_blocks_per_seq + (8 * r) / kPageTokens);
        if (blk < 0 || (long long)blk >= p.n_blocks) {
            if (lane == 0) atomicOr(p.err, kErrBadBlock);
            continue;
        }
        uint8_t* page = p.pool + ((long long)blk * p.n_kv_heads + h) * page_bytes(D);
        const int tau0 = (int)((8 * r) % kPageTokens);   // 0 or 8: the record within the page
        long long p0 = 8 * r > start ? 8 * r : start, p1 = 8 * r + 8 < end ? 8 * r + 8 : end;
        if (slices > 1) {
            const long long s0 = 8 * r + slice * per_slice, s1 = s0 + per_slice;
            p0 = p0 > s0 ? p0 : s0;
            p1 = p1 < s1 ? p1 : s1;
            if (p0 >= p1) continue;
        }
        const int c0 = l * CPL;
        if (slices == 1 && p1 - p0 == 8) {
            // the whole record: V words assembled in registers (the TPW tokens of each step
            // in separate lanes, combined below), plain stores
            uint32_t vw[CPL];
#pragma unroll
            for (int i = 0; i < CPL; i++) vw[i] = 0u;
#pragma unroll 2
            for (int t2 = 0; t2 < 8; t2 += TPW) {
                const int tt = t2 + sub;
                TokenCodes<CPL> tc;
                quantize_token<D, T>(p, tok0 + (8 * r + tt - start), h, l, tc);
                if (t2 == 0) grid_wait();
                store_token_kscales<D, CPL>(page, tau0 + tt, l, tc);
                const int bit = v_nibble_bit(tt);
#pragma unroll
                for (int i = 0; i < CPL; i++) vw[i] |= tc.vn[i] << bit;
            }
            if constexpr (TPW == 2) {
#pragma unroll
                for (int i = 0; i < CPL; i++) vw[i] |= __shfl_xor_sync(0xffffffffu, vw[i], 16);
            }
            if (sub == 0) {
#pragma unroll
                for (int i = 0; i < CPL; i++)
                    *reinterpret_cast<uint32_t*>(page + v_word_byte(D, tau0, c0 + i)) = vw[i];
            }
        } else {
            // part of the record: each nibble replaced atomically (TPW positions at a time)
            for (long long q0 = p0; q0 < p1; q0 += TPW) {
                const long long pos = q0 + sub;
                const bool here = pos < p1;
                TokenCodes<CPL> tc;
                // lanes past the record's end quantize the record's first position again
                // (their shuffles must run) and store nothing
                quantize_token<D, T>(p, tok0 + ((here ? pos : p0) - start), h, l, tc);
                if (!here) continue;
                grid_wait();
                const int tau = (int)(pos % kPageTokens);
                store_token_kscales<D, CPL>(page, tau, l, tc);
                const int bit = v_nibble_bit(tau);
#pragma unroll
                for (int i = 0; i < CPL; i++) {
                    unsigned* w = reinterpret_cast<unsigned*>(page + v_word_byte(D, tau, c0 + i));
                    atomicAnd(w, ~(0xFu << bit));
                    atomicOr(w, tc.vn[i] << bit);
                }
            }
        }
    }
}

template <int D>
static cudaError_t launch_append_d(const AppendParams& p, int n_sm, cudaStream_t st) {
    if (p.n_seqs > 65535 || p.n_kv_heads > 65535) return cudaErrorInvalidConfiguration;
    const int wpb = 8;
    // records of one sequence: at most n_tokens / 8 + 2; about 8 CTAs per SM in all.  A small
    // append (its records x 4 within 16 warps per SM) splits every record over 4 warps.
    const long long units = (long long)p.n_seqs * p.n_kv_heads;
    AppendParams q = p;
    q.slices = ((long long)p.n_tokens / 8 + p.n_seqs) * p.n_kv_heads * 4 <= (long long)n_sm * 16 ? 4 : 1;
    const long long per_seq = (((long long)p.n_tokens / 8 + 2) * q.slices + wpb - 1) / wpb;
    const long long fill = ((long long)n_sm * 8 + units - 1) / units;
    const long long gx = std::max<long long>(1, std::min(per_seq, fill));
    const dim3 grid((unsigned)gx, (unsigned)p.n_seqs, (unsigned)p.n_kv_heads);
    cudaLaunchAttribute pdl[1];
    pdl[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    pdl[0].val.programmaticStreamSerializationAllowed = 1;
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = grid;
    cfg.blockDim = dim3(wpb * 32);
    cfg.stream = st;
    cfg.attrs = pdl;
    cfg.numAttrs = 1;
    switch (p.dtype) {
        case 0: return cudaLaunchKernelEx(&cfg, append_kernel<D, float>, q);
        case 1: return cudaLaunchKernelEx(&cfg, append_kernel<D, __nv_bfloat16>, q);
        default: return cudaLaunchKernelEx(&cfg, append_kernel<D, __half>, q);
    }
}

cudaError_t launch_append(const AppendParams& p, int head_dim, int n_sm, cudaStream_t st) {
    return head_dim == 128 ? launch_append_d<128>(p, n_sm, st) : launch_append_d<256>(p, n_sm, st);
}

}  // namespace mq
