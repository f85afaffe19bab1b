// Split-K flash-decode over the K8/V4 paged cache, with draft verification.
//
// What it computes (the deep dive on magnitudedev/magnitude at blog.123qwe.co.kr,
// section 5: the decode attention unit attention_decode_k8v4 over the 8-bit-key /
// 4-bit-value cache, and the guarantee that verifying several draft tokens is
// one launch against the cache): for query token j of sequence b (n_b query
// tokens, L_b cached tokens including the drafts) and q-head h,
//     z_t = scale * <q, s_k[t] * kcode_t>,  t = 0 .. L_b - n_b + j
//     out = sum_t softmax(z)_t * (s_v[t, group] * vcode_t),  lse = log sum_t exp z_t
//
// How, on sm_100a:
//  * One CTA takes an aligned block of 128-token chunks of one (sequence, kv-head,
//    row block); every warp of the CTA takes one chunk per round.  Pages (16
//    tokens of one kv-head, 3232 or 6432 bytes) stream into a per-warp shared-memory
//    ring by 1-D bulk TMA copies (cp.async.bulk + mbarrier, L2 evict-first), looked
//    up through the block table.
//  * QK^T on the tensor cores in int8: q is held as a 23-bit fixed-point value per
//    row (q = Q * 2^(E-22), |Q| <= 2^22) split into three 8-bit limbs, so the int8
//    key codes feed mma.m16n8k32 straight from shared memory with no conversion and
//    the int32 products are exact; the limbs are combined once per score in fp32.
//  * P.V on the tensor cores in fp16: the int4 value codes become exact fp16
//    integers with two LOP3 + one HADD2/HFMA2 per pair; the weights
//    p * s_v[token, group] are rounded to fp16 (relative error <= 2^-11 per weight).
//  * Within a chunk one warp keeps an online softmax (running max in log2 units).
//    Chunk results are combined by ONE fixed binary tree over chunk indices
//    (warps of a round, rounds of a CTA, CTAs of a sequence), so the output does
//    not depend on warps per CTA, ring depth or split count.  The last CTA of each
//    (sequence, kv-head, row block) to finish — found with one atomic counter —
//    completes the tree over the CTA partials and writes out and lse; there is no
//    second kernel and no CTA ever waits for another.
#include <cfloat>
#include <climits>

#include "mq_device.cuh"
#include "mq_kernels.h"

namespace mq {

// lazy-max threshold of the online softmax, in log2 units (weights stay <= 2^4)
constexpr float kLazy = 4.0f;

template <int D, int ROWS>
struct Cfg {
    static constexpr int PB = page_bytes(D);
    static constexpr int NG = D / 32;            // V groups (= int8 k-steps of 32 channels)
    static constexpr int KS = D / 32;
    static constexpr int MTQ = (ROWS + 15) / 16; // QK m-tiles (16 query rows each)
    static constexpr int NTP = ROWS / 8;         // PV n-tiles (8 query rows each)
    static constexpr int MTP = D / 16;           // PV m-tiles (16 channels each)
    static constexpr int SLOTS = ROWS / 8;       // query rows owned by a lane: 8k + g
    static constexpr int KCH = D / 32;           // K 16-byte chunks per lane per page
    static constexpr int VCH = D / 64;           // V code chunks per lane per page
    static constexpr int SCH = D / 64;           // V scale chunks per lane per page
    static constexpr bool HI = ROWS > 8;         // rows g+8 of a QK m-tile are real rows
    static constexpr int PART = ROWS * D + 2 * ROWS;                 // floats of one partial
};

struct Smem {
    size_t ring, part, fin, coef, qfrag, flags, mbar, bt, misc, heap, total;
};

// W warps, R ring slots per warp, SD partial entries per warp (entry 0 holds the warp's
// result for the CTA tree; the others are left siblings of its binary counter).
template <int D, int ROWS>
__host__ __device__ inline Smem smem_layout(int W, int R, int SD) {
    using C = Cfg<D, ROWS>;
    Smem s{};
    size_t off = 0;
    auto al = [](size_t x, size_t a) { return (x + a - 1) / a * a; };
    s.ring = off;
    off += (size_t)W * R * C::PB;
    off = al(off, 16);
    s.part = off;
    off += (size_t)W * SD * C::PART * 4;
    s.heap = 0;  // the final merge reuses ring + part
    const size_t heap_bytes = (size_t)2 * kMaxSplits * ROWS * 4 * 4;
    if (off < heap_bytes) off = heap_bytes;
    off = al(off, 16);
    s.fin = off;                      // the final merge's result (outside the heap)
    off += (size_t)C::PART * 4;
    s.coef = off;
    off += (size_t)8 * ROWS * 2 * 4;  // up to 8 merges per phase
    s.qfrag = off;
    off += (size_t)C::MTQ * C::KS * 3 * 32 * 16;
    s.flags = off;
    off += 64 * 4;
    off = al(off, 8);
    s.mbar = off;
    off += (size_t)W * R * 8;
    s.bt = off;
    off += (size_t)W * 4 * kChunkPages * 4;
    s.misc = off;
    off += 64;
    s.total = al(off, 128);
    return s;
}

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

template <int D, int ROWS>
__global__ void __launch_bounds__(256, (D == 128 && ROWS == 8) ? 2 : 1) decode_kernel(const DecodeParams p) {
    using C = Cfg<D, ROWS>;
    extern __shared__ __align__(128) uint8_t smem[];
    const int W = blockDim.x >> 5, warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int g = lane >> 2, t = lane & 3;
    const int R = p.pages_per_stage;
    const Smem S = smem_layout<D, ROWS>(W, R, p.stack_depth);
    const int b = blockIdx.z, hk = blockIdx.y / p.n_rb, rb = blockIdx.y % p.n_rb, sp = blockIdx.x;
    const unsigned FULL = 0xffffffffu;

    // ---- sequence bounds (uniform per CTA) ----
    const int L = __ldg(p.seq_lens + b), nq = __ldg(p.n_q_per_seq + b);
    if (nq < 1 || nq > p.max_q || nq > L || (long long)L > (long long)p.max_blocks_per_seq * kPageTokens) {
        if (sp == 0 && rb == 0 && hk == 0 && threadIdx.x == 0) atomicOr(p.err, kErrBadSeq);
        return;
    }
    const int rows_b = p.group * nq, row0 = rb * ROWS;
    if (row0 >= rows_b) return;
    const int rows_here = min(ROWS, rows_b - row0);
    const int n_pages = (L + kPageTokens - 1) / kPageTokens;
    const int n_chunks = (L + kChunkTokens - 1) / kChunkTokens;
    const int c0 = sp * p.cpc;
    if (c0 >= n_chunks) return;
    const int c1 = min(c0 + p.cpc, n_chunks);
    const int n_splits = (n_chunks + p.cpc - 1) / p.cpc;
    const int n_rounds = (c1 - c0 + W - 1) / W;

    int* misc = reinterpret_cast<int*>(smem + S.misc);
    int* flags = reinterpret_cast<int*>(smem + S.flags);   // [0..W): warp partial empty
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + S.mbar) + warp * R;
    int* bt = reinterpret_cast<int*>(smem + S.bt) + warp * 4 * kChunkPages;
    uint8_t* ring = smem + S.ring + (size_t)warp * R * C::PB;
    float* part = reinterpret_cast<float*>(smem + S.part);
    float* coef = reinterpret_cast<float*>(smem + S.coef);

    // ---- query-row offset of this sequence (sum of n_q of earlier sequences) ----
    if (warp == 0) {
        int s = 0;
        for (int i = lane; i < b; i += 32) s += min(max(__ldg(p.n_q_per_seq + i), 0), p.max_q);
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(FULL, s, o);
        if (lane == 0) misc[0] = s;
    }
    if (lane == 0) {
        for (int s = 0; s < R; s++) mbar_init(smem_u32(&bars[s]), 1);
        mbar_fence_init();
    }
    if (threadIdx.x == 0) misc[1] = 0;
    __syncthreads();
    const int qoff = misc[0];

    // ---- q -> three 8-bit limbs of a 23-bit fixed-point value per row ----------
    // Lane (g, t) owns rows 16*mt + 8*h + g and channels [t*D/4, (t+1)*D/4).  The
    // A fragment of mma.m16n8k32 for k-step ks holds, for row g (h = 0) and g + 8
    // (h = 1), channels t*D/4 + 8*ks + {0..3} (regs 0/1) and + {4..7} (regs 2/3).
    float crow[C::SLOTS];
    int lim[C::SLOTS];
    uint32_t* qfrag_s = reinterpret_cast<uint32_t*>(smem + S.qfrag);
#pragma unroll
    for (int k = 0; k < C::SLOTS; k++) {
        const int mt = k >> 1, h = k & 1;
        const int rl = 8 * k + g;  // local row
        const int r = row0 + rl;
        const bool real = rl < rows_here;
        const int j = real ? r / p.group : 0, hq = real ? r % p.group : 0;
        const long long qrow = (long long)qoff + j;
        const bool qok = real && qrow < p.total_q;
        if (real && !qok && t == 0) atomicOr(p.err, kErrBadRow);
        constexpr int CH = D / 4;
        float amax = 0.0f;
        const size_t base = ((size_t)qrow * p.n_q_heads + (size_t)hk * p.group + hq) * D + (size_t)t * CH;
        // two passes over the lane's channels (max, then limbs) keep few values live
#pragma unroll 8
        for (int c = 0; c < CH; c++) amax = fmaxf(amax, fabsf(qok ? load_q(p, base + c) : 0.0f));
        amax = fmaxf(amax, __shfl_xor_sync(FULL, amax, 1));
        amax = fmaxf(amax, __shfl_xor_sync(FULL, amax, 2));
        int E = 0;
        if (amax > 0.0f) frexpf(amax, &E);  // amax < 2^E
        const bool zero_row = !(amax >= 0x1p-100f);
        const float up = zero_row ? 0.0f : ldexpf(1.0f, 22 - E);
        crow[k] = zero_row ? 0.0f : ldexpf(p.scale_log2, E - 22);
        lim[k] = real ? (L - nq + j + 1) : L;
#pragma unroll
        for (int ks = 0; ks < C::KS; ks++) {
            uint32_t w[3][2];
#pragma unroll
            for (int half = 0; half < 2; half++) {
                uint32_t l2 = 0, l1 = 0, l0 = 0;
#pragma unroll
                for (int i = 0; i < 4; i++) {
                    const float qv = qok ? load_q(p, base + 8 * ks + 4 * half + i) : 0.0f;
                    const int Q = (int)rintf(__fmul_rn(qv, up));
                    l2 |= (uint32_t)((Q >> 16) & 0xFF) << (8 * i);
                    l1 |= (uint32_t)((Q >> 8) & 0xFF) << (8 * i);
                    l0 |= (uint32_t)(Q & 0xFF) << (8 * i);
                }
                w[0][half] = l2;
                w[1][half] = l1;
                w[2][half] = l0;
            }
#pragma unroll
            for (int lb = 0; lb < 3; lb++) {
                if (warp == 0) {
                    uint32_t* f = qfrag_s + ((((size_t)mt * C::KS + ks) * 3 + lb) * 32 + lane) * 4;
                    if constexpr (C::HI) {
                        f[h] = w[lb][0];
                        f[2 + h] = w[lb][1];
                    } else {   // rows g + 8 are padding: keep regs 0 and 2 only, as 64 bits
                        f[0] = w[lb][0];
                        f[1] = w[lb][1];
                    }
                }
            }
        }
    }
    __syncthreads();

    // ---- this warp's chunks: an aligned run [wc0, wc1) of Q = cpc / W chunks ----
    const uint64_t policy = l2_evict_first_policy();
    const int Q = p.cpc / W;
    const int SD = p.stack_depth;                  // partial entries per warp
    const int wc0 = c0 + warp * Q;
    const int my_chunks = max(0, min(wc0 + Q, c1) - wc0);
    const int my_pages = my_chunks > 0 ? min((wc0 + my_chunks) * kChunkPages, n_pages) - wc0 * kChunkPages : 0;
    // Block-table entries of the run: a ring of four chunks' entries in shared memory,
    // fetched two chunks ahead into a register, so that no load is ever waited for.
    constexpr int kUnused = INT_MIN;
    auto bt_fetch = [&](int i) -> int {   // entry of page `lane` of the run's chunk i (lanes < 8)
        int blk = kUnused;
        if (i < my_chunks && lane < kChunkPages) {
            const int lp = (wc0 + i) * kChunkPages + lane;
            if (lp < n_pages) blk = __ldg(p.block_table + (long long)b * p.max_blocks_per_seq + lp);
        }
        return blk;
    };
    auto bt_store = [&](int i, int blk) {
        if (i < my_chunks && lane < kChunkPages) {
            if (blk != kUnused && (blk < 0 || (long long)blk >= p.n_blocks)) {
                atomicOr(p.err, kErrBadBlock);
                blk = -1;
            }
            bt[(i & 3) * kChunkPages + lane] = blk == kUnused ? -1 : blk;
        }
    };
    bt_store(0, bt_fetch(0));
    bt_store(1, bt_fetch(1));
    int bt_next = bt_fetch(2);
    __syncwarp();
    auto issue = [&](int k, int slot) {  // lane 0 only: page k of this warp's run into `slot`
        const int blk = bt[((k / kChunkPages) & 3) * kChunkPages + (k % kChunkPages)];
        const uint8_t* src = p.pool + ((long long)(blk < 0 ? 0 : blk) * p.n_kv_heads + hk) * C::PB;
        mbar_arrive_expect_tx(smem_u32(&bars[slot]), C::PB);
        tma_load_1d(smem_u32(ring + (size_t)slot * C::PB), src, C::PB, smem_u32(&bars[slot]), policy);
    };
    if (lane == 0)
        for (int k = 0; k < R && k < my_pages; k++) issue(k, k);

    // the smallest visibility limit of the real rows of this row block
    const int lim_min = L - nq + row0 / p.group + 1;
    // 32-bit shared-window addresses: ring slot 0 and this lane's q fragments
    const uint32_t ring_s = smem_u32(ring), lane16 = (uint32_t)lane * 16u;
    const uint32_t qf_s = smem_u32(qfrag_s) + lane16;
    float* my_ent = part + (size_t)warp * SD * C::PART;   // this warp's partial entries

    bool aborted = false;
    int k_abort = 0;       // first page not waited for after a timeout
    int k_next = 0;        // next page of this warp to consume
    int slot = 0;          // its ring slot (k_next % R) and mbarrier phase ((k_next / R) & 1)
    uint32_t phase = 0;

    // The run's result, as (O fragments, m and l of the lane's O rows 8n + 2t + e).
    float O[C::MTP][C::NTP][4];
    float mo[C::NTP][2], lo[C::NTP][2];
    int n_ent = 0;            // binary-counter entries in shared memory (warp-uniform)
    uint32_t ent_lvl = 0;     // their levels, 4 bits each

    // entry e (left sibling) (+) registers (right sibling) -> registers
    auto merge_entry = [&](int e) {
        __syncwarp();
        const float* ent = my_ent + (size_t)e * C::PART;
        float ca[C::NTP][2], cb[C::NTP][2];
#pragma unroll
        for (int n = 0; n < C::NTP; n++)
#pragma unroll
            for (int e2 = 0; e2 < 2; e2++) {
                const int r = 8 * n + 2 * t + e2;
                float m, l;
                merge_coef(ent[ROWS * D + r], ent[ROWS * D + ROWS + r], mo[n][e2], lo[n][e2], m, l, ca[n][e2],
                           cb[n][e2]);
                mo[n][e2] = m;
                lo[n][e2] = l;
            }
#pragma unroll
        for (int n = 0; n < C::NTP; n++)
#pragma unroll
            for (int q = 0; q < C::NG; q++) {
                const int ch = 32 * q + 4 * g, r0 = 8 * n + 2 * t;
                const float4 L0 = *reinterpret_cast<const float4*>(ent + (size_t)r0 * D + ch);
                const float4 L1 = *reinterpret_cast<const float4*>(ent + (size_t)(r0 + 1) * D + ch);
                O[2 * q][n][0] = merge_val(L0.x, O[2 * q][n][0], ca[n][0], cb[n][0]);
                O[2 * q][n][2] = merge_val(L0.y, O[2 * q][n][2], ca[n][0], cb[n][0]);
                O[2 * q + 1][n][0] = merge_val(L0.z, O[2 * q + 1][n][0], ca[n][0], cb[n][0]);
                O[2 * q + 1][n][2] = merge_val(L0.w, O[2 * q + 1][n][2], ca[n][0], cb[n][0]);
                O[2 * q][n][1] = merge_val(L1.x, O[2 * q][n][1], ca[n][1], cb[n][1]);
                O[2 * q][n][3] = merge_val(L1.y, O[2 * q][n][3], ca[n][1], cb[n][1]);
                O[2 * q + 1][n][1] = merge_val(L1.z, O[2 * q + 1][n][1], ca[n][1], cb[n][1]);
                O[2 * q + 1][n][3] = merge_val(L1.w, O[2 * q + 1][n][3], ca[n][1], cb[n][1]);
            }
    };
    // registers -> entry e (natural layout: O [ROWS][D], m [ROWS], l [ROWS])
    auto write_entry = [&](int e) {
        float* ent = my_ent + (size_t)e * C::PART;
#pragma unroll
        for (int n = 0; n < C::NTP; n++)
#pragma unroll
            for (int q = 0; q < C::NG; q++) {
                const int ch = 32 * q + 4 * g, r0 = 8 * n + 2 * t;
                *reinterpret_cast<float4*>(ent + (size_t)r0 * D + ch) =
                    make_float4(O[2 * q][n][0], O[2 * q][n][2], O[2 * q + 1][n][0], O[2 * q + 1][n][2]);
                *reinterpret_cast<float4*>(ent + (size_t)(r0 + 1) * D + ch) =
                    make_float4(O[2 * q][n][1], O[2 * q][n][3], O[2 * q + 1][n][1], O[2 * q + 1][n][3]);
            }
        if (g == 0) {
#pragma unroll
            for (int n = 0; n < C::NTP; n++)
#pragma unroll
                for (int e2 = 0; e2 < 2; e2++) {
                    ent[ROWS * D + 8 * n + 2 * t + e2] = mo[n][e2];
                    ent[ROWS * D + ROWS + 8 * n + 2 * t + e2] = lo[n][e2];
                }
        }
        __syncwarp();
    };

    // registers (left sibling) (+) entry (right sibling) -> registers
    auto merge_right = [&](const float* ent) {
        float ca[C::NTP][2], cb[C::NTP][2];
#pragma unroll
        for (int n = 0; n < C::NTP; n++)
#pragma unroll
            for (int e2 = 0; e2 < 2; e2++) {
                const int r = 8 * n + 2 * t + e2;
                float m, l;
                merge_coef(mo[n][e2], lo[n][e2], ent[ROWS * D + r], ent[ROWS * D + ROWS + r], m, l, ca[n][e2],
                           cb[n][e2]);
                mo[n][e2] = m;
                lo[n][e2] = l;
            }
#pragma unroll
        for (int n = 0; n < C::NTP; n++)
#pragma unroll
            for (int q = 0; q < C::NG; q++) {
                const int ch = 32 * q + 4 * g, r0 = 8 * n + 2 * t;
                const float4 R0 = *reinterpret_cast<const float4*>(ent + (size_t)r0 * D + ch);
                const float4 R1 = *reinterpret_cast<const float4*>(ent + (size_t)(r0 + 1) * D + ch);
                O[2 * q][n][0] = merge_val(O[2 * q][n][0], R0.x, ca[n][0], cb[n][0]);
                O[2 * q][n][2] = merge_val(O[2 * q][n][2], R0.y, ca[n][0], cb[n][0]);
                O[2 * q + 1][n][0] = merge_val(O[2 * q + 1][n][0], R0.z, ca[n][0], cb[n][0]);
                O[2 * q + 1][n][2] = merge_val(O[2 * q + 1][n][2], R0.w, ca[n][0], cb[n][0]);
                O[2 * q][n][1] = merge_val(O[2 * q][n][1], R1.x, ca[n][1], cb[n][1]);
                O[2 * q][n][3] = merge_val(O[2 * q][n][3], R1.y, ca[n][1], cb[n][1]);
                O[2 * q + 1][n][1] = merge_val(O[2 * q + 1][n][1], R1.z, ca[n][1], cb[n][1]);
                O[2 * q + 1][n][3] = merge_val(O[2 * q + 1][n][3], R1.w, ca[n][1], cb[n][1]);
            }
    };
    // entry -> registers
    auto load_entry = [&](const float* ent) {
#pragma unroll
        for (int n = 0; n < C::NTP; n++)
#pragma unroll
            for (int e2 = 0; e2 < 2; e2++) {
                mo[n][e2] = ent[ROWS * D + 8 * n + 2 * t + e2];
                lo[n][e2] = ent[ROWS * D + ROWS + 8 * n + 2 * t + e2];
            }
#pragma unroll
        for (int n = 0; n < C::NTP; n++)
#pragma unroll
            for (int q = 0; q < C::NG; q++) {
                const int ch = 32 * q + 4 * g, r0 = 8 * n + 2 * t;
                const float4 R0 = *reinterpret_cast<const float4*>(ent + (size_t)r0 * D + ch);
                const float4 R1 = *reinterpret_cast<const float4*>(ent + (size_t)(r0 + 1) * D + ch);
                O[2 * q][n][0] = R0.x;
                O[2 * q][n][2] = R0.y;
                O[2 * q + 1][n][0] = R0.z;
                O[2 * q + 1][n][2] = R0.w;
                O[2 * q][n][1] = R1.x;
                O[2 * q][n][3] = R1.y;
                O[2 * q + 1][n][1] = R1.z;
                O[2 * q + 1][n][3] = R1.w;
            }
    };

    for (int i = 0; i < my_chunks; i++) {
        if (i >= 1) {
            bt_store(i + 1, bt_next);
            bt_next = bt_fetch(i + 2);
            __syncwarp();
        }
        const int c = wc0 + i;
#pragma unroll
        for (int j = 0; j < C::MTP; j++)
#pragma unroll
            for (int n = 0; n < C::NTP; n++)
#pragma unroll
                for (int e = 0; e < 4; e++) O[j][n][e] = 0.0f;
        float mrun[C::SLOTS], lrun[C::SLOTS];
#pragma unroll
        for (int k = 0; k < C::SLOTS; k++) {
            mrun[k] = -INFINITY;
            lrun[k] = 0.0f;
        }
        const int pages_here = min(kChunkPages, n_pages - c * kChunkPages);
        for (int pi = 0; pi < pages_here; pi++, k_next++) {
            if (!aborted && !mbar_wait_bounded(smem_u32(&bars[slot]), phase)) {
                aborted = true;
                k_abort = k_next;
                if (lane == 0) atomicOr(p.err, kErrTimeout);
            }
            const uint32_t pg = ring_s + (uint32_t)slot * C::PB;   // this page
            const uint32_t pgl = pg + lane16;
            const int lp = c * kChunkPages + pi;
            const bool bad = bt[(i & 3) * kChunkPages + pi] < 0;
            // every token of the page visible to every row: no per-element masking
            const bool full = !bad && (lp + 1) * kPageTokens <= lim_min;

            // ---- scores: int8 QK^T on the tensor cores ----
            const float2 skA = __half22float2(u32_as_h2(ldsa32(pg + k_scale_off(D) + 4 * t)));
            const float2 skB = __half22float2(u32_as_h2(ldsa32(pg + k_scale_off(D) + 16 + 4 * t)));
            float z[C::SLOTS][2][2];
#pragma unroll
            for (int mt = 0; mt < C::MTQ; mt++) {
                // the lane's key chunks: token g (n-tile 0) and token g + 8 (n-tile 1)
                uint4 kc[C::KCH];
#pragma unroll
                for (int ii = 0; ii < C::KCH; ii++) kc[ii] = ldsa128(pgl + ii * 512);
                // int32 chains per limb and n-tile (exact, so any order).  The 8-row class
                // keeps the three limbs apart for ILP; the larger classes, short of
                // registers, shift the top limb in place before the middle one joins it.
                constexpr bool SPLIT3 = ROWS == 8;
                int d2[2][4], d1[SPLIT3 ? 2 : 1][4], d0[2][4];
#pragma unroll
                for (int nt = 0; nt < 2; nt++)
#pragma unroll
                    for (int ii = 0; ii < 4; ii++) {
                        d2[nt][ii] = d0[nt][ii] = 0;
                        if constexpr (SPLIT3) d1[nt][ii] = 0;
                    }
#pragma unroll
                for (int lb = 0; lb < 3; lb++) {
#pragma unroll
                    for (int ks = 0; ks < C::KS; ks++) {
                        uint32_t a[4];
                        const uint32_t f = qf_s + (((mt * C::KS + ks) * 3 + lb) * 512);
                        if constexpr (C::HI) {
                            const uint4 v = ldsa128(f);
                            a[0] = v.x;
                            a[1] = v.y;
                            a[2] = v.z;
                            a[3] = v.w;
                        } else {   // rows g + 8 are padding: their fragment registers are zero
                            const uint2 v = ldsa64(f);
                            a[0] = v.x;
                            a[1] = 0u;
                            a[2] = v.y;
                            a[3] = 0u;
                        }
#pragma unroll
                        for (int nt = 0; nt < 2; nt++) {
                            const uint4 ch = kc[nt * (D / 64) + ks / 2];
                            const uint32_t b0 = (ks & 1) ? ch.z : ch.x;
                            const uint32_t b1 = (ks & 1) ? ch.w : ch.y;
                            if (lb == 0) mma_s8s8(d2[nt], a, b0, b1);
                            else if (lb == 1) {
                                if constexpr (SPLIT3) mma_u8s8(d1[nt], a, b0, b1);
                                else mma_u8s8(d2[nt], a, b0, b1);
                            } else mma_u8s8(d0[nt], a, b0, b1);
                        }
                    }
                    if constexpr (!SPLIT3) {
                        if (lb == 0) {
#pragma unroll
                            for (int nt = 0; nt < 2; nt++)
#pragma unroll
                                for (int ii = 0; ii < 4; ii++)
                                    if (16 * mt + 8 * (ii / 2) < ROWS) d2[nt][ii] <<= 8;
                        }
                    }
                }
#pragma unroll
                for (int nt = 0; nt < 2; nt++)
#pragma unroll
                    for (int h = 0; h < 2; h++) {
                        if (16 * mt + 8 * h < ROWS) {
                            const int k = 2 * mt + h;
#pragma unroll
                            for (int e = 0; e < 2; e++) {
                                int d21;
                                if constexpr (SPLIT3) d21 = (d2[nt][2 * h + e] << 8) + d1[nt][2 * h + e];
                                else d21 = d2[nt][2 * h + e];
                                const float sc = __fmaf_rn((float)d21, 256.0f, (float)d0[nt][2 * h + e]);
                                const float skv = nt == 0 ? (e == 0 ? skA.x : skA.y) : (e == 0 ? skB.x : skB.y);
                                z[k][nt][e] = __fmul_rn(__fmul_rn(sc, crow[k]), skv);
                            }
                        }
                    }
            }

            // ---- online softmax (log2 units) ----
            const int tok0 = lp * kPageTokens + 2 * t;
            float pw[C::SLOTS][2][2], alph[C::SLOTS];
            bool resc = false;
#pragma unroll
            for (int k = 0; k < C::SLOTS; k++) {
                if (!full) {
#pragma unroll
                    for (int nt = 0; nt < 2; nt++)
#pragma unroll
                        for (int e = 0; e < 2; e++) {
                            const bool valid = !bad && (tok0 + 8 * nt + e) < lim[k];
                            z[k][nt][e] = valid ? z[k][nt][e] : -INFINITY;
                        }
                }
                float pm = fmaxf(fmaxf(z[k][0][0], z[k][0][1]), fmaxf(z[k][1][0], z[k][1][1]));
                pm = fmaxf(pm, __shfl_xor_sync(FULL, pm, 1));
                pm = fmaxf(pm, __shfl_xor_sync(FULL, pm, 2));
                // Lazy reference: the row's reference max moves only when a page max
                // exceeds it by more than kLazy (log2 units), so p = 2^(z - m) <= 2^kLazy
                // and a rescale of O is rare.  The first finite page max always moves it
                // (O is still zero then, so that rescale is skipped).
                const float mnew = (pm > __fadd_rn(mrun[k], kLazy)) ? pm : mrun[k];
                alph[k] = (mnew == mrun[k]) ? 1.0f : ex2(__fsub_rn(mrun[k], mnew));
                resc |= (alph[k] != 1.0f) && (mrun[k] != -INFINITY);
#pragma unroll
                for (int nt = 0; nt < 2; nt++)
#pragma unroll
                    for (int e = 0; e < 2; e++) {
                        const float pv = ex2(__fsub_rn(z[k][nt][e], mnew));
                        pw[k][nt][e] = full ? pv : (z[k][nt][e] == -INFINITY ? 0.0f : pv);
                    }
                const float ps = __fadd_rn(__fadd_rn(pw[k][0][0], pw[k][0][1]), __fadd_rn(pw[k][1][0], pw[k][1][1]));
                lrun[k] = __fadd_rn(__fmul_rn(lrun[k], alph[k]), ps);
                mrun[k] = mnew;
            }
            // rescaling by exactly 1 changes nothing, so it is skipped when no row's
            // reference moved (the common case)
            if (__any_sync(FULL, resc)) {
#pragma unroll
                for (int n = 0; n < C::NTP; n++) {
                    const float a0 = __shfl_sync(FULL, alph[n], 8 * t);
                    const float a1 = __shfl_sync(FULL, alph[n], 8 * t + 4);
#pragma unroll
                    for (int j = 0; j < C::MTP; j++) {
                        O[j][n][0] = __fmul_rn(O[j][n][0], a0);
                        O[j][n][1] = __fmul_rn(O[j][n][1], a1);
                        O[j][n][2] = __fmul_rn(O[j][n][2], a0);
                        O[j][n][3] = __fmul_rn(O[j][n][3], a1);
                    }
                }
            }

            // ---- P.V: int4 codes as exact fp16, weights p * s_v in fp16 ----
            uint4 vcw[C::VCH], svw[C::SCH];
#pragma unroll
            for (int ii = 0; ii < C::VCH; ii++) vcw[ii] = ldsa128(pgl + v_code_off(D) + ii * 512);
#pragma unroll
            for (int ii = 0; ii < C::SCH; ii++) svw[ii] = ldsa128(pg + v_scale_off(D) + t * (C::NG * 8) + ii * 16);
#pragma unroll
            for (int q = 0; q < C::NG; q++) {
                const float2 s0 = __half22float2(u32_as_h2(comp(svw[(2 * q) / 4], (2 * q) % 4)));
                const float2 s1 = __half22float2(u32_as_h2(comp(svw[(2 * q + 1) / 4], (2 * q + 1) % 4)));
                const uint32_t x0 = comp(vcw[(2 * q) / 4], (2 * q) % 4);
                const uint32_t x1 = comp(vcw[(2 * q + 1) / 4], (2 * q + 1) % 4);
                const uint32_t y0 = x0 >> 8, y1 = x1 >> 8;
                const uint32_t A0 = nib_lo_to_h2(x0), A1 = nib_hi_to_h2(x0);
                const uint32_t A2 = nib_lo_to_h2(x1), A3 = nib_hi_to_h2(x1);
                const uint32_t B0 = nib_lo_to_h2(y0), B1 = nib_hi_to_h2(y0);
                const uint32_t B2 = nib_lo_to_h2(y1), B3 = nib_hi_to_h2(y1);
#pragma unroll
                for (int n = 0; n < C::NTP; n++) {
                    float w00 = __fmul_rn(pw[n][0][0], s0.x), w01 = __fmul_rn(pw[n][0][1], s0.y);
                    float w10 = __fmul_rn(pw[n][1][0], s1.x), w11 = __fmul_rn(pw[n][1][1], s1.y);
                    if (!full) {  // masked tokens may sit next to unwritten (non-finite) scales
                        w00 = pw[n][0][0] == 0.0f ? 0.0f : w00;
                        w01 = pw[n][0][1] == 0.0f ? 0.0f : w01;
                        w10 = pw[n][1][0] == 0.0f ? 0.0f : w10;
                        w11 = pw[n][1][1] == 0.0f ? 0.0f : w11;
                    }
                    const uint32_t bb0 = pack_h2(w00, w01), bb1 = pack_h2(w10, w11);
                    mma_f16(O[2 * q][n], A0, A1, A2, A3, bb0, bb1);
                    mma_f16(O[2 * q + 1][n], B0, B1, B2, B3, bb0, bb1);
                }
            }
            // every lane has consumed the page (its loads fed the math above): refill
            // the slot.  The reads are complete, so the bulk copy cannot overtake them.
            __syncwarp();
            if (lane == 0 && !aborted && k_next + R < my_pages) issue(k_next + R, slot);
            if (++slot == R) {
                slot = 0;
                phase ^= 1u;
            }
        }
        // ---- chunk result: slot form (rows 8k + g) -> O-row form (rows 8n + 2t + e) ----
        float lrow[C::SLOTS];
#pragma unroll
        for (int k = 0; k < C::SLOTS; k++) {
            float l = lrun[k];
            l = __fadd_rn(l, __shfl_xor_sync(FULL, l, 1));
            l = __fadd_rn(l, __shfl_xor_sync(FULL, l, 2));
            lrow[k] = l;
        }
#pragma unroll
        for (int n = 0; n < C::NTP; n++)
#pragma unroll
            for (int e2 = 0; e2 < 2; e2++) {
                mo[n][e2] = __shfl_sync(FULL, mrun[n], 8 * t + 4 * e2);
                lo[n][e2] = __shfl_sync(FULL, lrow[n], 8 * t + 4 * e2);
            }
        // ---- binary counter over the run's chunks (aligned, so it closes the subtree) ----
        int lvl = 0;
        while (n_ent > 0 && (int)((ent_lvl >> (4 * (n_ent - 1))) & 15u) == lvl) {
            merge_entry(n_ent - 1);
            n_ent--;
            lvl++;
        }
        if (i + 1 < my_chunks) {
            write_entry(n_ent);
            ent_lvl = (ent_lvl & ~(15u << (4 * n_ent))) | ((uint32_t)lvl << (4 * n_ent));
            n_ent++;
        }
    }
    // a run cut short by the end of the sequence: fold what is left, right to left
    for (int e = n_ent - 1; e >= 0; e--) merge_entry(e);

    // ---- tree over the W warp results, in registers: at level s the left warp of
    // each pair merges its right sibling's entry; a warp that is a right sibling at
    // the next level then publishes what it holds to its entry 0 (it may have merged
    // at lower levels even when its sibling at this level is empty) ----
    bool have = my_chunks > 0;
    if (have) write_entry(0);
    if (lane == 0) flags[warp] = have ? 0 : 1;
    __syncthreads();
    for (int s = 1; s < W; s <<= 1) {
        if ((warp & (2 * s - 1)) == 0) {
            if (warp + s < W && flags[warp + s] == 0) {
                const float* rent = part + (size_t)(warp + s) * SD * C::PART;
                if (have) {
                    merge_right(rent);
                } else {
                    load_entry(rent);
                    have = true;
                }
            }
            if ((warp & (4 * s - 1)) == 2 * s && have) {
                write_entry(0);
                if (lane == 0) flags[warp] = 0;
            }
        }
        __syncthreads();
    }
    // any warp that gave up on a wait: drain its copies still in flight, then stop
    if (aborted) {
        for (int k = k_abort; k < my_pages && k < k_abort + R; k++)
            mbar_wait_bounded(smem_u32(&bars[k % R]), (uint32_t)((k / R) & 1));
        misc[1] = 1;
    }
    __syncthreads();
    if (misc[1] == 1) return;

    const size_t pidx = ((size_t)(b * p.n_kv_heads + hk) * p.n_rb + rb);
    // out = O / l and lse for the real rows of this block; (o_src, m_src, l_src) in the
    // natural layout (shared memory)
    auto finalize = [&](const float* o_src, const float* m_src, const float* l_src) {
        for (int i = threadIdx.x; i < rows_here * (D / 4); i += blockDim.x) {
            const int rl = i / (D / 4), c4 = i % (D / 4);
            const int r = row0 + rl, j = r / p.group, hq = r % p.group;
            const long long qrow = (long long)qoff + j;
            if (qrow >= p.total_q) continue;
            const float l = l_src[rl];
            float4 o = reinterpret_cast<const float4*>(o_src + (size_t)rl * D)[c4];
            o.x = __fdiv_rn(o.x, l);
            o.y = __fdiv_rn(o.y, l);
            o.z = __fdiv_rn(o.z, l);
            o.w = __fdiv_rn(o.w, l);
            const size_t orow = (size_t)qrow * p.n_q_heads + (size_t)hk * p.group + hq;
            reinterpret_cast<float4*>(p.out + orow * D)[c4] = o;
            if (c4 == 0 && p.lse != nullptr)
                p.lse[orow] = __fmul_rn(__fadd_rn(m_src[rl], log2f(l)), 0.69314718055994531f);
        }
    };

    if (warp == 0) write_entry(0);   // the CTA's result, natural layout
    __syncthreads();
    if (n_splits == 1) {
        finalize(part, part + ROWS * D, part + ROWS * D + ROWS);
        return;
    }
    // ---- publish this CTA's partial; the last CTA completes the tree ----
    {
        float* go = p.part_o + (pidx * p.split_stride + sp) * (size_t)(ROWS * D);
        float* gml = p.part_ml + (pidx * p.split_stride + sp) * (size_t)(2 * ROWS);
        for (int i = threadIdx.x; i < ROWS * D / 4; i += blockDim.x)
            __stcg(reinterpret_cast<float4*>(go) + i, reinterpret_cast<const float4*>(part)[i]);
        for (int i = threadIdx.x; i < 2 * ROWS; i += blockDim.x) __stcg(gml + i, part[ROWS * D + i]);
    }
    __syncthreads();
    // release: this CTA's partial (written by all threads, ordered by the barrier)
    // happens-before the count; acquire: the last CTA sees every other CTA's partial
    if (threadIdx.x == 0) misc[2] = (atom_add_acq_rel_gpu(p.counters + pidx, 1u) == (unsigned)(n_splits - 1)) ? 1 : 0;
    __syncthreads();
    if (misc[2] == 0) return;

    // Coefficients of every node of the padded tree over the n_splits CTA partials,
    // heap-indexed (node (level, i) at 2^(H-level) + i), per row: m, l, alpha, beta.
    int H = 0;
    while ((1 << H) < n_splits) H++;
    float* hp = reinterpret_cast<float*>(smem + S.heap);
    auto hidx = [&](int level, int i) { return (1 << (H - level)) + i; };
    const float* gml0 = p.part_ml + pidx * p.split_stride * (size_t)(2 * ROWS);
    const float* go0 = p.part_o + pidx * p.split_stride * (size_t)(ROWS * D);
    for (int i = threadIdx.x; i < n_splits * ROWS; i += blockDim.x) {
        const int s = i / ROWS, r = i % ROWS;
        float* nd = hp + ((size_t)hidx(0, s) * ROWS + r) * 4;
        nd[0] = __ldcg(gml0 + (size_t)s * 2 * ROWS + r);
        nd[1] = __ldcg(gml0 + (size_t)s * 2 * ROWS + ROWS + r);
    }
    __syncthreads();
    for (int lv = 1; lv <= H; lv++) {
        const int n_here = (n_splits + (1 << lv) - 1) >> lv;
        for (int i = threadIdx.x; i < n_here * ROWS; i += blockDim.x) {
            const int ni = i / ROWS, r = i % ROWS;
            float* nd = hp + ((size_t)hidx(lv, ni) * ROWS + r) * 4;
            const float* lf = hp + ((size_t)hidx(lv - 1, 2 * ni) * ROWS + r) * 4;
            const bool has_right = (2 * ni + 1) * (1 << (lv - 1)) < n_splits;
            if (has_right) {
                const float* rt = hp + ((size_t)hidx(lv - 1, 2 * ni + 1) * ROWS + r) * 4;
                merge_coef(lf[0], lf[1], rt[0], rt[1], nd[0], nd[1], nd[2], nd[3]);
            } else {
                nd[0] = lf[0];
                nd[1] = lf[1];
                nd[2] = 1.0f;
                nd[3] = 0.0f;
            }
        }
        __syncthreads();
    }
    // Elements: the padded tree evaluated level by level in registers, eight leaves
    // (an aligned level-3 subtree) at a time, their loads all in flight together.
    float* fin = reinterpret_cast<float*>(smem + S.fin);   // final O [ROWS][D], m, l
    const float* root = hp + (size_t)hidx(H, 0) * ROWS * 4;
    const int n_groups = (n_splits + 7) >> 3;
    for (int e4 = threadIdx.x; e4 < ROWS * D / 4; e4 += blockDim.x) {
        const int r = (4 * e4) / D;
        auto node_merge = [&](float4 lf, float4 rt, int level, int idx) {
            const float* nd = hp + ((size_t)hidx(level, idx) * ROWS + r) * 4;
            float4 o;
            o.x = merge_val(lf.x, rt.x, nd[2], nd[3]);
            o.y = merge_val(lf.y, rt.y, nd[2], nd[3]);
            o.z = merge_val(lf.z, rt.z, nd[2], nd[3]);
            o.w = merge_val(lf.w, rt.w, nd[2], nd[3]);
            return o;
        };
        float4 gv[8];
#pragma unroll
        for (int j = 0; j < 8; j++) {
            if (j < n_groups) {
                float4 v[8];
#pragma unroll
                for (int u = 0; u < 8; u++) {
                    const int sidx = 8 * j + u;
                    v[u] = sidx < n_splits ? __ldcg(reinterpret_cast<const float4*>(go0 + (size_t)sidx * ROWS * D) + e4)
                                           : make_float4(0.f, 0.f, 0.f, 0.f);
                }
#pragma unroll
                for (int lv = 1; lv <= 3; lv++) {
#pragma unroll
                    for (int u = 0; u < (8 >> lv); u++) {
                        const int idx = ((8 * j) >> lv) + u;           // node (lv, idx)
                        const bool has_right = (2 * idx + 1) * (1 << (lv - 1)) < n_splits;
                        if (lv <= H) v[u] = has_right ? node_merge(v[2 * u], v[2 * u + 1], lv, idx) : v[2 * u];
                    }
                }
                gv[j] = v[0];
            }
        }
        // levels 4 .. H over the group nodes
#pragma unroll
        for (int lv = 4; lv <= 6; lv++) {
#pragma unroll
            for (int u = 0; u < (64 >> lv); u++) {
                if (lv <= H && u * (1 << lv) < n_splits) {
                    const bool has_right = (2 * u + 1) * (1 << (lv - 1)) < n_splits;
                    gv[u] = has_right ? node_merge(gv[2 * u], gv[2 * u + 1], lv, u) : gv[2 * u];
                }
            }
        }
        reinterpret_cast<float4*>(fin)[e4] = gv[0];
    }
    float* fml = fin + ROWS * D;
    for (int r = threadIdx.x; r < ROWS; r += blockDim.x) {
        fml[r] = root[r * 4 + 0];
        fml[ROWS + r] = root[r * 4 + 1];
    }
    __syncthreads();
    finalize(fin, fml, fml + ROWS);
    if (threadIdx.x == 0) p.counters[pidx] = 0u;
}

size_t decode_smem_bytes(int head_dim, int rows, int warps, int pages_per_stage, int stack_depth) {
#define MQ_SMEM(DD, RR) \
    if (head_dim == DD && rows == RR) return smem_layout<DD, RR>(warps, pages_per_stage, stack_depth).total;
    MQ_SMEM(128, 8) MQ_SMEM(128, 16) MQ_SMEM(128, 32) MQ_SMEM(256, 8) MQ_SMEM(256, 16)
#undef MQ_SMEM
    return 0;
}

template <int D, int ROWS>
static cudaError_t set_smem(size_t smem) {
    return cudaFuncSetAttribute(decode_kernel<D, ROWS>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
}

cudaError_t decode_prepare(int head_dim, int rows, size_t smem) {
    if (head_dim == 128 && rows == 8) return set_smem<128, 8>(smem);
    if (head_dim == 128 && rows == 16) return set_smem<128, 16>(smem);
    if (head_dim == 128 && rows == 32) return set_smem<128, 32>(smem);
    if (head_dim == 256 && rows == 8) return set_smem<256, 8>(smem);
    if (head_dim == 256 && rows == 16) return set_smem<256, 16>(smem);
    return cudaErrorInvalidValue;
}

cudaError_t launch_decode(const DecodeParams& p, int head_dim, int rows, int warps, int max_splits, size_t smem,
                          cudaStream_t st) {
    const dim3 grid((unsigned)max_splits, (unsigned)(p.n_kv_heads * p.n_rb), (unsigned)p.n_seqs);
    const dim3 block((unsigned)(warps * 32));
#define MQ_LAUNCH(DD, RR) \
    if (head_dim == DD && rows == RR) decode_kernel<DD, RR><<<grid, block, smem, st>>>(p); else
    MQ_LAUNCH(128, 8) MQ_LAUNCH(128, 16) MQ_LAUNCH(128, 32) MQ_LAUNCH(256, 8) MQ_LAUNCH(256, 16)
    return cudaErrorInvalidValue;
#undef MQ_LAUNCH
    return cudaGetLastError();
}

}  // namespace mq
