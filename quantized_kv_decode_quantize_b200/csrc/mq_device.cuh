// Device-side helpers shared by the mq kernels: page layout, PTX wrappers for
// mbarriers, bulk TMA copies, and the error word.
//
// Page layout (one (block, kv-head) page of 16 tokens, head_dim D): two token-group
// records, tokens 0-7 then 8-15, of rec_bytes(D) = 12.5 D + 16 bytes each.  Within a
// record (token tt = 0..7 of the group):
//   [0, 8D)               K codes, int8, as 8-row x 16-byte blocks: code (tt, c) at
//                         byte (c / 16) * 128 + tt * 16 + c % 16.  Consecutive records
//                         of consecutive pages are then one K-major tensor-core operand
//                         (tokens x channels) whose 8-token groups sit rec_bytes apart.
//   [8D, 12D)             V codes, int4 two's complement, channel-major: one 32-bit
//                         word per channel c at 8D + 4c holding the channel's 8 codes,
//                         token tt at bit 4 * (tt / 2) + 16 * (tt % 2), so that a mask
//                         and a shift give two consecutive tokens as the two halves.
//   [12D, 12D + 16)       K scales, fp16, token order.
//   [12D + 16, 12.5D + 16) V scales, fp16: (tt, group g) at 12D + 16 + 2 * (tt * D/32 + g).
#pragma once
#include <cstdint>
#include <cuda_fp16.h>
#include <cuda_bf16.h>

namespace mq {

constexpr int kPageTokens = 16;
constexpr int kChunkPages = 8;                  // tokens per canonical chunk = 128
constexpr int kChunkTokens = kPageTokens * kChunkPages;
constexpr int kMaxSplits = 64;                  // CTAs per (sequence, kv-head, row block)

__host__ __device__ constexpr int page_bytes(int D) { return 25 * D + 32; }
__host__ __device__ constexpr int rec_bytes(int D) { return 25 * D / 2 + 16; }
__host__ __device__ constexpr int rec_v_off(int D) { return 8 * D; }
__host__ __device__ constexpr int rec_ks_off(int D) { return 12 * D; }
__host__ __device__ constexpr int rec_vs_off(int D) { return 12 * D + 16; }

// byte offset inside a page of K code (token tau, channel c)
__host__ __device__ constexpr int k_code_byte(int D, int tau, int c) {
    return (tau / 8) * rec_bytes(D) + (c / 16) * 128 + (tau % 8) * 16 + c % 16;
}
// byte offset inside a page of the 32-bit V word of channel c for tokens of tau's group,
// and the bit position of tau's code in it
__host__ __device__ constexpr int v_word_byte(int D, int tau, int c) {
    return (tau / 8) * rec_bytes(D) + rec_v_off(D) + 4 * c;
}
__host__ __device__ constexpr int v_nibble_bit(int tau) { return 4 * ((tau % 8) / 2) + 16 * (tau % 2); }
__host__ __device__ constexpr int k_scale_byte(int D, int tau) {
    return (tau / 8) * rec_bytes(D) + rec_ks_off(D) + 2 * (tau % 8);
}
__host__ __device__ constexpr int v_scale_byte(int D, int tau, int g) {
    return (tau / 8) * rec_bytes(D) + rec_vs_off(D) + 2 * ((tau % 8) * (D / 32) + g);
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

// One non-blocking test of the phase.
__device__ __forceinline__ bool mbar_test_wait(uint32_t bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{ .reg .pred p; mbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2; selp.u32 %0, 1, 0, p; }"
        : "=r"(ok)
        : "r"(bar), "r"(parity)
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

// Bounded wait for waits on a pipeline's critical path: spins on the non-blocking test
// (no sleep, so the thread resumes within a few cycles of the phase completing) for
// ~2^16 cycles, then continues as mbar_wait_bounded.
__device__ __forceinline__ bool mbar_wait_spin(uint32_t bar, uint32_t parity) {
    if (mbar_test_wait(bar, parity)) return true;   // the common case: already complete
    const long long t0 = clock64();
    do {
        if (mbar_test_wait(bar, parity)) return true;
    } while (clock64() - t0 < (1ll << 16));
    return mbar_wait_bounded(bar, parity);
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

// A hint that brings [src, src + bytes) into L2 (16-byte multiple); no data moves to the
// SM and nothing waits on it.
__device__ __forceinline__ void bulk_prefetch_l2(const void* src, uint32_t bytes) {
    asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(src), "r"(bytes) : "memory");
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

__device__ __forceinline__ uint32_t h2_as_u32(__half2 h) { return *reinterpret_cast<uint32_t*>(&h); }
__device__ __forceinline__ __half2 u32_as_h2(uint32_t u) { return *reinterpret_cast<__half2*>(&u); }

// (x & mask) ^ flip in one LOP3
__device__ __forceinline__ uint32_t lop_and_xor(uint32_t x, uint32_t mask, uint32_t flip) {
    uint32_t d;
    asm("lop3.b32 %0, %1, %2, %3, 0x6A;" : "=r"(d) : "r"(x), "r"(mask), "r"(flip));
    return d;
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
