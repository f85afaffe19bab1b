// Device-side helpers shared by the mq kernels: page layout, PTX wrappers for
// mbarriers, bulk TMA copies and legacy warp-level MMA, and the error word.
//
// Page layout (one (block, kv-head) page of 16 tokens, head_dim D):
//   [0, 16D)            K codes, int8, permuted for the QK fragments:
//                       16-byte chunk c of lane L = 4g + t sits at (c*32 + L)*16 and
//                       holds channels t*D/4 + 16*(c % (D/64)) .. +15 of token
//                       g + 8*(c / (D/64)).
//   [16D, 16D+32)       K scales, fp16, token order.
//   [16D+32, 24D+32)    V codes, int4 pairs, permuted for the PV fragments:
//                       32-bit word w = 2*q + tp of lane L = 4g + t sits at
//                       ((w/4)*32 + L)*16 + (w%4)*4; its bytes are
//                       [tok A: ch c, c+1][tok A: ch c+2, c+3][tok B: ch c, c+1][tok B: ch c+2, c+3]
//                       with c = 32q + 4g, tok A = 8*tp + 2t, tok B = tok A + 1,
//                       and the even channel of a pair in the low nibble.
//   [24D+32, 25D+32)    V scales, fp16: half index ((t*NG + q)*2 + hi)*2 + par for
//                       token 8*hi + 2t + par and group q (NG = D/32 groups).
#pragma once
#include <cstdint>
#include <cuda_fp16.h>
#include <cuda_bf16.h>

namespace mq {

constexpr int kPageTokens = 16;
constexpr int kChunkPages = 8;                  // tokens per canonical chunk = 128
constexpr int kChunkTokens = kPageTokens * kChunkPages;
constexpr int kMaxSplits = 64;                  // CTA partials per (sequence, kv-head, row block)

__host__ __device__ constexpr int page_bytes(int D) { return 25 * D + 32; }
__host__ __device__ constexpr int k_scale_off(int D) { return 16 * D; }
__host__ __device__ constexpr int v_code_off(int D) { return 16 * D + 32; }
__host__ __device__ constexpr int v_scale_off(int D) { return 24 * D + 32; }

// byte offset of K code (token tau, channel c) inside a page
__host__ __device__ inline int k_code_byte(int D, int tau, int c) {
    const int t = c / (D / 4), o = c % (D / 4);
    const int chunk = (tau / 8) * (D / 64) + o / 16;
    const int lane = 4 * (tau % 8) + t;
    return (chunk * 32 + lane) * 16 + (o % 16);
}

// byte offset (inside a page) of the byte holding V channels (c, c+1) of token
// tau, for c = 32q + 4g' + 2h (h = 0 or 1)
__host__ __device__ inline int v_code_byte(int D, int tau, int c) {
    const int q = c / 32, cg = c % 32, gp = cg / 4, h = (cg % 4) / 2;
    const int t = (tau % 8) / 2, par = tau % 2, tp = tau / 8;
    const int lane = 4 * gp + t, w = 2 * q + tp;
    return v_code_off(D) + ((w / 4) * 32 + lane) * 16 + (w % 4) * 4 + par * 2 + h;
}

__host__ __device__ inline int v_scale_byte(int D, int tau, int q) {
    const int NG = D / 32, t = (tau % 8) / 2, hi = tau / 8, par = tau % 2;
    return v_scale_off(D) + 2 * (((t * NG + q) * 2 + hi) * 2 + par);
}

// ---- device error word (one per device) -----------------------------------
enum : unsigned {
    kErrBadPosition = 1u,   // append position beyond the block table
    kErrBadBlock = 2u,      // block id outside [0, n_blocks)
    kErrBadSeq = 4u,        // seq_len / n_q outside the documented bounds
    kErrTimeout = 8u,       // a bounded wait gave up
    kErrBadRow = 16u,       // a query row beyond total_q
};

#ifdef __CUDACC__
__device__ __forceinline__ uint32_t smem_u32(const void* p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}

__device__ __forceinline__ void mbar_fence_init() {
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint32_t bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes) : "memory");
}

// One test of the phase; the thread may sleep in hardware for up to ~1 ms waiting for
// it (suspend-time hint), so waiting costs no issue slots.
__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{ .reg .pred p; mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3; selp.u32 %0, 1, 0, p; }"
        : "=r"(ok)
        : "r"(bar), "r"(parity), "r"(1000000u)
        : "memory");
    return ok != 0;
}

// Bounded wait: gives up after ~2^31 cycles (about a second) and returns false.
__device__ __forceinline__ bool mbar_wait_bounded(uint32_t bar, uint32_t parity) {
    if (mbar_try_wait(bar, parity)) return true;
    const long long t0 = clock64();
    while (!mbar_try_wait(bar, parity)) {
        if (clock64() - t0 > (1ll << 31)) return false;
    }
    return true;
}

// 1-D bulk copy global -> shared, completion counted on an mbarrier (no multicast).
__device__ __forceinline__ void tma_load_1d(uint32_t dst, const void* src, uint32_t bytes, uint32_t bar,
                                            uint64_t policy) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint [%0], [%1], %2, [%3], %4;" ::"r"(
            dst),
        "l"(src), "r"(bytes), "r"(bar), "l"(policy)
        : "memory");
}

__device__ __forceinline__ uint64_t l2_evict_first_policy() {
    uint64_t p;
    asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(p));
    return p;
}

__device__ __forceinline__ unsigned atom_add_acq_rel_gpu(unsigned* a, unsigned v) {
    unsigned old;
    asm volatile("atom.add.acq_rel.gpu.u32 %0, [%1], %2;" : "=r"(old) : "l"(a), "r"(v) : "memory");
    return old;
}

__device__ __forceinline__ void fence_proxy_async_smem() {
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// shared-memory loads from 32-bit shared-window addresses
__device__ __forceinline__ uint4 ldsa128(uint32_t a) {
    uint4 v;
    asm volatile("ld.shared.v4.u32 {%0,%1,%2,%3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(a));
    return v;
}
__device__ __forceinline__ uint2 ldsa64(uint32_t a) {
    uint2 v;
    asm volatile("ld.shared.v2.u32 {%0,%1}, [%2];" : "=r"(v.x), "=r"(v.y) : "r"(a));
    return v;
}
__device__ __forceinline__ uint32_t ldsa32(uint32_t a) {
    uint32_t v;
    asm volatile("ld.shared.u32 %0, [%1];" : "=r"(v) : "r"(a));
    return v;
}

__device__ __forceinline__ uint4 lds128(const void* p) {
    uint4 v;
    asm volatile("ld.shared.v4.u32 {%0,%1,%2,%3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "r"(smem_u32(p)));
    return v;
}

__device__ __forceinline__ uint2 lds64(const void* p) {
    uint2 v;
    asm volatile("ld.shared.v2.u32 {%0,%1}, [%2];" : "=r"(v.x), "=r"(v.y) : "r"(smem_u32(p)));
    return v;
}

__device__ __forceinline__ uint32_t lds32(const void* p) {
    uint32_t v;
    asm volatile("ld.shared.u32 %0, [%1];" : "=r"(v) : "r"(smem_u32(p)));
    return v;
}

// D = A(16x32, s8) * B(32x8, s8) + C, int32 accumulate
__device__ __forceinline__ void mma_s8s8(int (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
    asm(
        "mma.sync.aligned.m16n8k32.row.col.s32.s8.s8.s32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
        : "+r"(d[0]), "+r"(d[1]), "+r"(d[2]), "+r"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// D = A(16x32, u8) * B(32x8, s8) + C, int32 accumulate
__device__ __forceinline__ void mma_u8s8(int (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
    asm(
        "mma.sync.aligned.m16n8k32.row.col.s32.u8.s8.s32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
        : "+r"(d[0]), "+r"(d[1]), "+r"(d[2]), "+r"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// D = A(16x16, f16) * B(16x8, f16) + D, fp32 accumulate
__device__ __forceinline__ void mma_f16(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                        uint32_t b0, uint32_t b1) {
    asm(
        "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// (x & mask) | magic in one LOP3
__device__ __forceinline__ uint32_t lop_and_or(uint32_t x, uint32_t mask, uint32_t magic) {
    uint32_t d;
    asm("lop3.b32 %0, %1, %2, %3, 0xEA;" : "=r"(d) : "r"(x), "r"(mask), "r"(magic));
    return d;
}

__device__ __forceinline__ uint32_t h2_as_u32(__half2 h) { return *reinterpret_cast<uint32_t*>(&h); }
__device__ __forceinline__ __half2 u32_as_h2(uint32_t u) { return *reinterpret_cast<__half2*>(&u); }

// (x & mask) ^ flip in one LOP3
__device__ __forceinline__ uint32_t lop_and_xor(uint32_t x, uint32_t mask, uint32_t flip) {
    uint32_t d;
    asm("lop3.b32 %0, %1, %2, %3, 0x6A;" : "=r"(d) : "r"(x), "r"(mask), "r"(flip));
    return d;
}

// Two two's-complement 4-bit codes at bit positions (0..3, 16..19) of x -> fp16x2
// holding the exact integer codes.  One LOP3 forms 1024 + (n ^ 8) = 1032 + code in
// each half (0x6400 is 1024; flipping bit 3 turns the two's-complement nibble into
// code + 8), one HSUB2 removes the 1032.
__device__ __forceinline__ uint32_t nib_lo_to_h2(uint32_t x) {
    const uint32_t m = lop_and_xor(x, 0x000F000Fu, 0x64086408u);
    return h2_as_u32(__hsub2(u32_as_h2(m), u32_as_h2(0x64086408u)));   // - 1032
}
// Same for bit positions (4..7, 20..23): 1024 + 16 (code + 8), then /16 - 72.
__device__ __forceinline__ uint32_t nib_hi_to_h2(uint32_t x) {
    const uint32_t m = lop_and_xor(x, 0x00F000F0u, 0x64806480u);
    return h2_as_u32(__hfma2(u32_as_h2(m), u32_as_h2(0x2C002C00u), u32_as_h2(0xD480D480u)));
}

// 2^x with the SFU instruction (ex2.approx.ftz.f32: relative error ~2^-22, subnormal
// results flushed to zero, ex2(-inf) = +0).  Every exponential of the decode kernel
// goes through this one function.
__device__ __forceinline__ float ex2(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

// component i (compile-time after unrolling) of a uint4
__device__ __forceinline__ uint32_t comp(const uint4& v, int i) {
    return i == 0 ? v.x : (i == 1 ? v.y : (i == 2 ? v.z : v.w));
}

__device__ __forceinline__ uint32_t pack_h2(float lo, float hi) {
    return h2_as_u32(__floats2half2_rn(lo, hi));
}

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
    return v;
}
#endif  // __CUDACC__

}  // namespace mq
