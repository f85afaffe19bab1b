// Device helpers shared by the decode kernel (mq_decode_small.cu), the merge kernel
// (mq_decode.cu) and the prefill kernel (mq_prefill.cu).
#pragma once
#include <cfloat>
#include <climits>

#include "mq_device.cuh"
#include "mq_kernels.h"
#include "mq_tc.cuh"

namespace mq {

// ---- merge of two partial results (one binary-tree node) ------------------
__device__ __forceinline__ void merge_coef(float ml, float ll, float mr, float lr, float& m, float& l, float& a,
                                           float& b) {
    m = fmaxf(ml, mr);
    a = (ml == m) ? 1.0f : ex2(__fsub_rn(ml, m));
    b = (mr == m) ? 1.0f : ex2(__fsub_rn(mr, m));
    l = __fadd_rn(__fmul_rn(ll, a), __fmul_rn(lr, b));
}
__device__ __forceinline__ float merge_val(float ol, float orr, float a, float b) {
    return __fadd_rn(__fmul_rn(ol, a), __fmul_rn(orr, b));
}

template <typename T>
__device__ __forceinline__ float ld_f32(const void* base, size_t i);
template <>
__device__ __forceinline__ float ld_f32<float>(const void* base, size_t i) {
    return __ldg(reinterpret_cast<const float*>(base) + i);
}
template <>
__device__ __forceinline__ float ld_f32<__nv_bfloat16>(const void* base, size_t i) {
    return __bfloat162float(reinterpret_cast<const __nv_bfloat16*>(base)[i]);
}
template <>
__device__ __forceinline__ float ld_f32<__half>(const void* base, size_t i) {
    return __half2float(reinterpret_cast<const __half*>(base)[i]);
}

__device__ __forceinline__ float load_q(const DecodeParams& p, size_t i) {
    if (p.q_dtype == 0) return ld_f32<float>(p.q, i);
    if (p.q_dtype == 1) return ld_f32<__nv_bfloat16>(p.q, i);
    return ld_f32<__half>(p.q, i);
}

__device__ __forceinline__ void stsa64(uint32_t a, uint32_t x, uint32_t y) {
    asm volatile("st.shared.v2.u32 [%0], {%1,%2};" ::"r"(a), "r"(x), "r"(y) : "memory");
}
__device__ __forceinline__ void stsa128(uint32_t a, uint32_t x, uint32_t y, uint32_t z, uint32_t w) {
    asm volatile("st.shared.v4.u32 [%0], {%1,%2,%3,%4};" ::"r"(a), "r"(x), "r"(y), "r"(z), "r"(w) : "memory");
}
__device__ __forceinline__ uint32_t ldsa16(uint32_t a) {
    unsigned short v;
    asm volatile("ld.shared.u16 %0, [%1];" : "=h"(v) : "r"(a));
    return v;
}
__device__ __forceinline__ float h_bits_to_f32(uint32_t bits) {
    return __half2float(__ushort_as_half((unsigned short)bits));
}

// Slow path of the decode kernel's waits (out of line), run by the whole warp; `done`
// is this lane's result of the first test.  A timeout raises the CTA's
// abort flag and the device error word.
static __device__ __noinline__ bool wait_slow_warp(uint32_t bar, uint32_t parity, bool spin, bool done,
                                            volatile int* abort_flag, unsigned* err) {
    bool ok = done || (*abort_flag == 0 && (spin ? mbar_wait_spin(bar, parity) : mbar_wait_bounded(bar, parity)));
    ok = __all_sync(0xffffffffu, ok);
    if (!ok && (threadIdx.x & 31) == 0) {
        if (*abort_flag == 0) atomicOr(err, kErrTimeout);
        *abort_flag = 1;
    }
    return ok;
}

// Two 4-bit two's-complement codes (bits 0-3 and 16-19 of x) as an exact fp16 pair.
__device__ __forceinline__ uint32_t code_pair(uint32_t x) {
    const uint32_t biased = lop_and_xor(x, 0x000F000Fu, 0x64086408u);   // fp16 (1024 + code + 8) x 2
    return h2_as_u32(__hsub2(u32_as_h2(biased), u32_as_h2(0x64086408u)));
}
// The same for the codes in bits 4-7 and 20-23, read in place: under exponent 2^6 the
// nibble is the mantissa's bits 4-7 (steps of 1/16 x 16 = 1), so the pair is 64 + code + 8.
__device__ __forceinline__ uint32_t code_pair_hi(uint32_t x) {
    const uint32_t biased = lop_and_xor(x, 0x00F000F0u, 0x54805480u);   // fp16 (64 + code + 8) x 2
    return h2_as_u32(__hsub2(u32_as_h2(biased), u32_as_h2(0x54805480u)));
}


// ---- balanced split counts (a flat grid) -------------------------------------------------
// Where the split count is free (the decode classes), a launch with p.cta_budget > 0 gives
// every unit of sequence b ceil(n_leaves_b / lpc) CTAs of lpc leaves each, lpc the smallest
// power of two (at most 64, the leaves of the longest unit) whose total fits the budget:
// short and long sequences then take work in proportion to their length, and every CTA
// still holds an aligned power-of-two run of leaves (the fixed merge tree).  One warp
// computes it (all 32 lanes call), reading every sequence's length.
struct SeqShape {
    int units, leaves;   // row blocks x kv-heads of the sequence, merge-tree leaves of each
};
__device__ __forceinline__ SeqShape seq_shape(const DecodeParams& p, int b, int rows_per_block) {
    SeqShape sh{0, 0};
    const int L = seq_len_of(p, b), nq = seq_nq_of(p, b);
    if (nq < 1 || nq > p.max_q || nq > L ||
        (long long)L + (long long)p.bt_col * kPageTokens > (long long)p.max_blocks_per_seq * kPageTokens)
        return sh;
    const int n_chunks = (L + kChunkTokens - 1) / kChunkTokens;
    sh.leaves = (n_chunks + p.node_chunks - 1) / p.node_chunks;
    sh.units = p.n_kv_heads * ((p.group * nq + rows_per_block - 1) / rows_per_block);
    return sh;
}
// A flat grid's leaves per CTA (lpc): the smallest power of two (at most 64) for which
// every unit's CTAs, sum over units of ceil(leaves / lpc), fit p.cta_budget.  One warp (all
// 32 lanes call; lane = sequence, in rounds of 32); `first` returns the lane's shape from
// the first round for flat_locate.
__device__ __forceinline__ int flat_lpc(const DecodeParams& p, int rows_per_block, SeqShape& first) {
    const unsigned FULL = 0xffffffffu;
    const int lane = threadIdx.x & 31;
    first = lane < p.n_seqs ? seq_shape(p, lane, rows_per_block) : SeqShape{0, 0};
    long long need[7] = {0, 0, 0, 0, 0, 0, 0};
    for (int b0 = 0; b0 < p.n_seqs; b0 += 32) {
        SeqShape sh = first;
        if (b0 > 0) sh = b0 + lane < p.n_seqs ? seq_shape(p, b0 + lane, rows_per_block) : SeqShape{0, 0};
#pragma unroll
        for (int k = 0; k < 7; k++) need[k] += (long long)sh.units * ((sh.leaves + (1 << k) - 1) >> k);
    }
#pragma unroll
    for (int k = 0; k < 7; k++)
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) need[k] += __shfl_xor_sync(FULL, need[k], o);
    int lpc = 64;
#pragma unroll
    for (int k = 6; k >= 0; k--)
        if (need[k] <= p.cta_budget) lpc = 1 << k;
    return lpc;
}
// CTA `cta` of a flat grid: its sequence b, kv-head hk, row block rb and split sp (CTAs are
// numbered unit by unit, sequences in order, each unit's splits consecutive); false when
// the index is past the launch's work.  One warp, after flat_lpc.
__device__ __forceinline__ bool flat_locate(const DecodeParams& p, int rows_per_block, int lpc, SeqShape first,
                                            int cta, int& b, int& hk, int& rb, int& sp) {
    const unsigned FULL = 0xffffffffu;
    const int lane = threadIdx.x & 31;
    long long base = 0;
    for (int b0 = 0; b0 < p.n_seqs; b0 += 32) {
        SeqShape sh = first;
        if (b0 > 0) sh = b0 + lane < p.n_seqs ? seq_shape(p, b0 + lane, rows_per_block) : SeqShape{0, 0};
        const int per_unit = (sh.leaves + lpc - 1) / lpc;
        const long long cnt = (long long)sh.units * per_unit;
        long long incl = cnt;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const long long v = __shfl_up_sync(FULL, incl, o);
            if (lane >= o) incl += v;
        }
        const long long excl = base + incl - cnt;
        const unsigned who = __ballot_sync(FULL, cnt > 0 && cta >= excl && cta < excl + cnt);
        if (who != 0u) {
            const int src = __ffs(who) - 1;
            const int local = (int)(cta - __shfl_sync(FULL, excl, src));
            const int pu = __shfl_sync(FULL, per_unit, src);
            const int nrb = __shfl_sync(FULL, sh.units, src) / p.n_kv_heads;
            b = b0 + src;
            const int unit = local / pu;
            sp = local % pu;
            hk = unit / nrb;
            rb = unit % nrb;
            return true;
        }
        base += __shfl_sync(FULL, incl, 31);
    }
    return false;
}

// ---- the merge tree over a unit's leaves -----------------------------------------------
// A unit's leaves are runs of node_chunks chunks; the tree over them is fixed: node (k, i)
// covers leaves [i 2^k, (i + 1) 2^k), merges nodes (k - 1, 2i) and (k - 1, 2i + 1), and is
// its left child when the right one starts past the last leaf.  Where the split count is
// free (the classes of up to 8 rows), a CTA holds an aligned power-of-two run of leaves,
// i.e. one node of that tree, which it builds with a binary counter (pending left children
// in slots by level) and publishes as its partial; the merge kernel's tree over the CTAs
// is the same tree's upper part.  TreeStep is what the CTA does when leaf li is complete.
struct TreeStep {
    uint32_t merge_mask;   // slots merged into the new node, in increasing level
    int level;             // the node's level after the carry
    bool push;             // kept in slot `level`; else (the CTA's last leaf) it is the CTA's node
};
__device__ __forceinline__ TreeStep tree_step(int li, int l0, bool last, uint32_t occ, int kmax) {
    TreeStep st{};
    int t = 0, idx = li;
    // carry: a right child whose left sibling (in this CTA) waits in slot t
    while (t < kmax && (idx & 1) && ((idx - 1) << t) >= l0) {
        st.merge_mask |= 1u << t;
        idx >>= 1;
        t++;
    }
    st.level = t;
    st.push = !last;
    // the CTA's last leaf: its right edge, the remaining left children in increasing level
    // (their right parts lie past the sequence's last leaf)
    if (last) st.merge_mask |= occ & ~st.merge_mask;
    return st;
}

// ---- q -> three signed 8-bit limbs of a 23-bit fixed-point value per row ----------------
// Q = rint(q * 2^(22 - E)) with |q| < 2^E the row's absmax bound, |Q| <= 2^22, and
// Q = l2 * 2^16 + l1 * 2^8 + l0 with l0, l1 in [-128, 127] and |l2| <= 65.  Limb k of row
// r is row k * ROWS + r of the NQ x D (K-major) score operand at `qlimb` (rows 3 * ROWS ..
// NQ - 1 are zero padding, written here too).  Row r of the block is query row
// row0 + r = j * group + hq: query token j of the sequence (q row qoff + j), q-head
// hk * group + hq.  Per row, crow_s[r] = softmax scale * log2(e) * 2^(E - 22) (0 for a zero
// row) and lim_s[r] = the first position the row does not see.  Threads tid = 0 ..
// nthr - 1 share the work; the caller orders the writes (fence + barrier) before the MMAs.
template <int D, int ROWS, int NQ>
__device__ __forceinline__ void q_to_limbs(const DecodeParams& p, uint8_t* qlimb, float* crow_s, int* lim_s, int tid,
                                           int nthr, int row0, int rows_here, int qoff, int L, int nq, int hk) {
    constexpr int SL = D / 8;   // 8-channel slices of a row
    const unsigned FULL = 0xffffffffu;
    for (int i = tid; i < (NQ - 3 * ROWS) * D / 16; i += nthr)
        reinterpret_cast<uint4*>(qlimb + (size_t)3 * ROWS * D)[i] = make_uint4(0u, 0u, 0u, 0u);
    for (int it = tid; it < ROWS * SL; it += nthr) {
        const int r = it / SL, sl = it % SL;
        const bool real = r < rows_here;
        const int rr = row0 + r, j = real ? rr / p.group : 0, hq = real ? rr % p.group : 0;
        const long long qrow = (long long)qoff + j;
        const bool qok = real && qrow < p.total_q;
        if (real && !qok && sl == 0) atomicOr(p.err, kErrBadRow);
        const size_t base = ((size_t)qrow * p.n_q_heads + (size_t)hk * p.group + hq) * D + (size_t)8 * sl;
        float qv[8];
        float amax = 0.0f;
#pragma unroll
        for (int e = 0; e < 8; e++) {
            qv[e] = qok ? load_q(p, base + e) : 0.0f;
            amax = fmaxf(amax, fabsf(qv[e]));
        }
#pragma unroll
        for (int o = 1; o < SL; o <<= 1) amax = fmaxf(amax, __shfl_xor_sync(FULL, amax, o));
        int E = 0;
        if (amax > 0.0f) frexpf(amax, &E);   // amax < 2^E
        const bool zero_row = !(amax >= 0x1p-100f);
        const float up = zero_row ? 0.0f : ldexpf(1.0f, 22 - E);
        if (sl == 0) {
            crow_s[r] = zero_row ? 0.0f : ldexpf(p.scale_log2, E - 22);
            lim_s[r] = (real && p.causal) ? (L - nq + j + 1) : L;
        }
        uint32_t w[3][2] = {{0u, 0u}, {0u, 0u}, {0u, 0u}};
#pragma unroll
        for (int e = 0; e < 8; e++) {
            const int Q = (int)rintf(__fmul_rn(qv[e], up));
            const int l0 = ((Q + 128) & 255) - 128;
            const int Q1 = (Q - l0) >> 8;
            const int l1 = ((Q1 + 128) & 255) - 128;
            const int l2 = (Q1 - l1) >> 8;
            w[0][e / 4] |= (uint32_t)(l2 & 255) << (8 * (e % 4));
            w[1][e / 4] |= (uint32_t)(l1 & 255) << (8 * (e % 4));
            w[2][e / 4] |= (uint32_t)(l0 & 255) << (8 * (e % 4));
        }
#pragma unroll
        for (int k = 0; k < 3; k++) {
            const int n = k * ROWS + r;
            const size_t off = (size_t)(n / 8) * (8 * D) + (size_t)(sl / 2) * 128 + (n % 8) * 16 + (sl % 2) * 8;
            *reinterpret_cast<uint2*>(qlimb + off) = make_uint2(w[k][0], w[k][1]);
        }
    }
}

}  // namespace mq
