// Split-K flash-decode for blocks of 4 or 8 query rows per kv-head (grouped-query decode:
// GQA 4 with one query token is 4 rows), on the sm_100a tensor cores.
//
// What it computes is mq_decode.cu's (the deep dive on magnitudedev/magnitude at
// blog.123qwe.co.kr, section 5: the decode attention unit attention_decode_k8v4 over the
// 8-bit-key / 4-bit-value cache): for query token j of sequence b and q-head h,
//     z_t = scale * <q, s_k[t] * kcode_t>,  t = 0 .. L_b - n_b + j
//     out = sum_t softmax(z)_t * (s_v[t, group] * vcode_t),  lse = log sum_t exp z_t
//
// How.  One CTA (11 warps; two CTAs per SM for 4 rows of head_dim 128) takes a contiguous range of
// 128-token chunks of one (sequence, kv-head, row block).  Every chunk is a small
// attention problem of its own, solved with the chunk's exact row maxima, and the
// per-chunk results are merged by log-sum-exp in registers:
//  * warp 0 streams the chunk's 8 pages into a shared-memory ring, one 1-D bulk TMA copy
//    per page (block-table lookup, L2 evict-first);
//  * warp 1 issues the score MMAs (kind::i8, M = 128 tokens, q as three signed 8-bit
//    limbs per row along N, exact int32 products in tensor memory);
//  * warps 7-10 (one TMEM lane = one token) form z in fp32, take the chunk's row maxima
//    (redux + one named barrier), and write p = 2^(z - max) <= 1 and the fp16 weights
//    W_g = p * s_v[token, g] to shared memory; each thread keeps its token's share of
//    l = sum_t p_t relative to the running row maxima, summed over the CTA at the end;
//  * warp 2 issues the value MMAs (kind::f16, A = V^T in tensor memory, B = the weights,
//    every group of 32 channels using its own columns) into a fresh accumulator per
//    chunk (two alternate);
//  * warps 3-6 turn the chunk's int4 value codes into V^T in tensor memory as exact fp16
//    values (one channel per lane), and then merge the previous chunk's accumulator into
//    the CTA's running (max, sum, output) held in registers, lane = channel.
// The weights never exceed the fp16 range (p <= 1 and s_v <= 65504), no accumulator is
// ever rescaled in tensor memory, and the chunk steps of the softmax do not wait for one
// another.  The CTA partials of a unit are combined by merge_kernel (mq_decode.cu) over a
// fixed binary tree; a unit that is not split writes out and lse here.  The chunk ranges
// depend only on the shape, the SM count and the configured splits per SM, so the result
// is bit-identical for every ring depth.
#include "mq_decode_common.cuh"

namespace mq {

template <int D, int ROWS>
struct Sm {
    static constexpr int PB = page_bytes(D);
    static constexpr int REC = rec_bytes(D);
    static constexpr int G = D / 32;                        // value groups
    static constexpr int H = D / 128;                       // 128-channel halves (value MMA M tiles)
    static constexpr int NQ = (3 * ROWS + 15) / 16 * 16;    // score MMA N: 3 limbs x rows
    static constexpr int NO = 4 * ROWS;                     // value MMA N per half
    static constexpr int NB = G * ROWS;                     // weight columns: W_0 .. W_{G-1}
    // two CTAs per SM for the 4-row D = 128 class (two independent pipelines per SM,
    // each with half of tensor memory and of the registers), one for the others
    static constexpr int CPS = (D == 128 && ROWS == 4) ? 2 : 1;
    static constexpr int TCOLS = CPS == 2 ? 256 : 512;      // tensor-memory columns per CTA
    static constexpr int NSB = 4;                           // score buffers
    static constexpr int NOB = 2;                           // per-chunk value accumulators
    static constexpr int NVB = 2;                           // V^T buffers
    static constexpr int NWB = 2;                           // weight buffers (shared memory)
    static constexpr int NPB = 2;                           // value-MMA completion barriers
    static constexpr int NML = NWB + NOB;                   // slots of the chunk maxima and sums
    static constexpr int THREADS = 352;                     // 0 TMA, 1 QK, 2 PV, 3-6 values, 7-10 softmax
    static constexpr int T_S = 0;
    static constexpr int T_O = NSB * NQ;
    static constexpr int T_VT = (T_O + NOB * H * NO + 31) / 32 * 32;
    static constexpr int T_END = T_VT + NVB * H * 64;
    static constexpr int WBYTES = kChunkTokens * NB * 2;    // one weight buffer
    static constexpr int LBO_W = NB / 8 * 128;              // its 8-token group stride
    static_assert(ROWS == 4 || ROWS == 8, "row class");
    static_assert(T_END <= TCOLS, "tensor memory budget");
    static_assert(NPB >= NOB && NPB >= NVB && NPB >= NWB, "completion barriers");
};

struct SmallSmem {
    size_t ring, wbuf, qlimb, xch, xm, xl, crow, lim, pgbad, mbar, misc, total;
};

// NS = ring stages (chunks of 8 pages)
template <int D, int ROWS>
__host__ __device__ inline SmallSmem small_layout(int NS) {
    using T = Sm<D, ROWS>;
    SmallSmem s{};
    auto al = [](size_t x, size_t a) { return (x + a - 1) / a * a; };
    size_t off = 0;
    s.ring = off;
    off += (size_t)NS * kChunkPages * T::PB;
    off = al(off, 128);
    s.wbuf = off;
    off += (size_t)T::NWB * T::WBYTES;
    off = al(off, 128);
    s.qlimb = off;
    off += (size_t)T::NQ * D;
    s.xch = off;                                  // [2][ROWS][4 warps] chunk row maxima
    off += (size_t)2 * ROWS * 4 * 4;
    s.xm = off;                                   // [NML][ROWS] chunk row maxima (merged)
    off += (size_t)T::NML * ROWS * 4;
    s.xl = off;                                   // [4 warps][ROWS] the softmax warps' shares of l
    off += (size_t)4 * ROWS * 4;
    s.crow = off;
    off += (size_t)ROWS * 4;
    s.lim = off;
    off += (size_t)ROWS * 4;
    s.pgbad = off;
    off += (size_t)NS * kChunkPages * 4;
    off = al(off, 8);
    s.mbar = off;
    off += (size_t)(2 * NS + 2 * T::NSB + T::NWB + T::NVB + T::NPB + T::NOB + T::NML) * 8;
    s.misc = off;
    off += 64;
    s.total = al(off, 128);
    return s;
}

template <int D, int ROWS>
__global__ void __launch_bounds__(Sm<D, ROWS>::THREADS, Sm<D, ROWS>::CPS) decode_small_kernel(const DecodeParams p) {
    using T = Sm<D, ROWS>;
    extern __shared__ __align__(1024) uint8_t smem[];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int NS = p.stages;
    const SmallSmem S = small_layout<D, ROWS>(NS);
    const int b = blockIdx.z, hk = blockIdx.y / p.n_rb, rb = blockIdx.y % p.n_rb, sp = blockIdx.x;
    const unsigned FULL = 0xffffffffu;

    // ---- sequence bounds (uniform per CTA) ----
    const int L = seq_len_of(p, b), nq = seq_nq_of(p, b);
    if (nq < 1 || nq > p.max_q || nq > L ||
        (long long)L + (long long)p.bt_col * kPageTokens > (long long)p.max_blocks_per_seq * kPageTokens) {
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
    const int n_ck = min(c0 + p.cpc, n_chunks) - c0;
    const int n_splits = (n_chunks + p.cpc - 1) / p.cpc;

    // block-table entries of the first chunk (warp 0, lanes < 8), loaded before the set-up:
    // the table is an input of the launch that no preceding append writes
    int blk_first = 0;
    if (warp == 0) {
        const int lp = c0 * kChunkPages + lane;
        if (lane < kChunkPages && lp < n_pages)
            blk_first = __ldg(p.block_table + (long long)b * p.max_blocks_per_seq + p.bt_col + lp);
    }

    // the dependent merge kernel may be scheduled now; it waits for this grid to complete
    if (threadIdx.x == 0) asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    int* misc = reinterpret_cast<int*>(smem + S.misc);   // 0 qoff, 1 abort, 3 TMEM base
    volatile int* abort_flag = misc + 1;
    float* crow_s = reinterpret_cast<float*>(smem + S.crow);
    int* lim_s = reinterpret_cast<int*>(smem + S.lim);
    int* pgbad = reinterpret_cast<int*>(smem + S.pgbad);
    float* xch = reinterpret_cast<float*>(smem + S.xch);
    float* xm = reinterpret_cast<float*>(smem + S.xm);
    float* xlf = reinterpret_cast<float*>(smem + S.xl);   // [4 softmax warps][ROWS] shares of l
    const uint32_t bar0 = smem_u32(smem + S.mbar);
    auto full_b = [&](int s) { return bar0 + 8u * (uint32_t)s; };
    auto empty_b = [&](int s) { return bar0 + 8u * (uint32_t)(NS + s); };
    const uint32_t sfull_b = bar0 + 8u * (uint32_t)(2 * NS);   // [NSB] score buffer written
    const uint32_t sfree_b = sfull_b + 8 * T::NSB;             // [NSB] score buffer read
    const uint32_t wfull_b = sfree_b + 8 * T::NSB;             // [NWB] weights written
    const uint32_t vfull_b = wfull_b + 8 * T::NWB;             // [NVB] V^T written
    const uint32_t pvdone_b = vfull_b + 8 * T::NVB;            // [NPB] value MMAs of a chunk done
    const uint32_t ofree_b = pvdone_b + 8 * T::NPB;            // [NOB] chunk accumulator read
    const uint32_t mready_b = ofree_b + 8 * T::NOB;            // [NML] chunk maxima and sums written
    auto pv_bar = [&](int j) { return pvdone_b + 8u * (uint32_t)(j % T::NPB); };
    auto pv_par = [&](int j) { return (uint32_t)(j / T::NPB) & 1u; };

    // A bounded wait the whole warp agrees on; a timeout raises the CTA's abort flag (every
    // role then stops taking work) and the device error word.  Every role sleeps in
    // hardware while it waits (mbarrier try_wait): spinning warps took issue slots from
    // the warps that compute (measured: the step was 1 % slower with spinning).
    const bool spin_waits = false;
    auto wait_warp = [&](uint32_t bar, uint32_t parity) -> bool {
        const bool done = mbar_test_wait(bar, parity);
        if (__all_sync(FULL, done)) return true;
        return wait_slow_warp(bar, parity, spin_waits, done, abort_flag, p.err);
    };

    // ---- set-up: barriers, query-row offset, TMEM, q limbs ----
    if (threadIdx.x == 0) {
        for (int s = 0; s < NS; s++) {
            mbar_init(full_b(s), 1);
            mbar_init(empty_b(s), 9);   // QK commit + 4 value warps + 4 softmax warps
        }
        for (int j = 0; j < T::NSB; j++) {
            mbar_init(sfull_b + 8 * j, 1);
            mbar_init(sfree_b + 8 * j, 4);
        }
        for (int j = 0; j < T::NWB; j++) mbar_init(wfull_b + 8 * j, 4);
        for (int j = 0; j < T::NVB; j++) mbar_init(vfull_b + 8 * j, 4);
        for (int j = 0; j < T::NPB; j++) mbar_init(pvdone_b + 8 * j, 1);
        for (int j = 0; j < T::NOB; j++) mbar_init(ofree_b + 8 * j, 4);
        for (int j = 0; j < T::NML; j++) mbar_init(mready_b + 8 * j, 4);
        mbar_fence_init();
        misc[1] = 0;
    }
    if (warp == 0) {
        int s = 0;
        for (int i = lane; i < b; i += 32) s += min(max(seq_nq_of(p, i), 0), p.max_q);
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(FULL, s, o);
        if (lane == 0) misc[0] = s;
    }
    if (warp == 1) {
        tmem_alloc(smem_u32(misc + 3), T::TCOLS);
        tmem_relinquish();
        tc_fence_before();
    }
    __syncthreads();
    const int qoff = misc[0];
    if (warp >= 7) {
        q_to_limbs<D, ROWS, T::NQ>(p, smem + S.qlimb, crow_s, lim_s, threadIdx.x - 224, 128, row0, rows_here, qoff, L,
                                   nq, hk);
        fence_proxy_async_smem();
    }
    // the TMA producer starts at once; the other warps wait for the limbs and TMEM
    if (warp != 0) named_bar_sync(1, T::THREADS - 32);
    tc_fence_after();
    const uint32_t tmem = (uint32_t)misc[3];
    const uint32_t ring = smem_u32(smem + S.ring);

    // the CTA's running result, held by the value warps (lane = channel of each half)
    float Or[T::H][ROWS], Mr[ROWS], lr[ROWS];
#pragma unroll
    for (int r = 0; r < ROWS; r++) {
        Mr[r] = -INFINITY;
        lr[r] = 0.0f;
#pragma unroll
        for (int h = 0; h < T::H; h++) Or[h][r] = 0.0f;
    }

    if (warp == 0) {
        // ================= TMA producer =================
        // The kernel is a programmatic dependent launch: a preceding kernel that allows it
        // (the append of this step) may still be writing pages.  Wait for it to complete
        // before the first page is read; everything before this point reads only the
        // launch's inputs, which no such kernel writes.
        asm volatile("griddepcontrol.wait;" ::: "memory");
        const uint64_t policy = l2_evict_first_policy();
        auto bt_load = [&](int i) -> int {
            const int lp = (c0 + i) * kChunkPages + lane;
            return (i < n_ck && lane < kChunkPages && lp < n_pages)
                       ? __ldg(p.block_table + (long long)b * p.max_blocks_per_seq + p.bt_col + lp)
                       : 0;
        };
        int blk_next = blk_first;
        int issued = 0;
        int s = 0;
        uint32_t ph = 1;   // parity of the empty phase awaited at stage s (the first round does not wait)
        for (int i = 0; i < n_ck; i++) {
            if (i >= NS && !wait_warp(empty_b(s), ph)) break;
            const int c = c0 + i;
            const int npg = min(kChunkPages, n_pages - c * kChunkPages);
            int blk = blk_next;
            bool bad = true;
            if (lane < npg) {
                bad = blk < 0 || (long long)blk >= p.n_blocks;
                if (bad) {
                    atomicOr(p.err, kErrBadBlock);
                    blk = 0;   // read a valid page; its tokens are masked
                }
            }
            if (lane < kChunkPages) pgbad[s * kChunkPages + lane] = bad ? 1 : 0;
            __syncwarp();
            if (lane == 0) mbar_arrive_expect_tx(full_b(s), (uint32_t)(npg * T::PB));
            __syncwarp();
            if (lane < npg)
                tma_load_1d(ring + (uint32_t)((s * kChunkPages + lane) * T::PB),
                            p.pool + ((long long)blk * p.n_kv_heads + hk) * T::PB, T::PB, full_b(s), policy);
            issued = i + 1;
            blk_next = bt_load(i + 1);
            if (++s == NS) {
                s = 0;
                ph ^= 1u;
            }
        }
        // after an abort: let copies still in flight land before the CTA leaves
        if (*abort_flag != 0 && lane == 0)
            for (int k = max(0, issued - NS); k < issued; k++) mbar_wait_bounded(full_b(k % NS), (uint32_t)(k / NS) & 1u);
    } else if (warp == 1) {
        // ================= score MMAs (whole warp; one elected lane issues) =================
        const uint32_t ql = smem_u32(smem + S.qlimb);
        constexpr uint32_t IDQ = instr_desc(2, 1, 1, 0, 0, 128, T::NQ);   // s32 <- s8 x s8, K-major
        const uint64_t dq = smem_desc(ql, 128, 8 * D);
        uint32_t last_bar = 0, last_par = 0;
        int s = 0;
        uint32_t ph = 0;   // ring stage of chunk i and the parity of its fill
        for (int i = 0; i < n_ck; i++) {
            const int sb = i % T::NSB;
            if (!wait_warp(full_b(s), ph)) break;
            if (i >= T::NSB && !wait_warp(sfree_b + 8 * sb, (uint32_t)((i - T::NSB) / T::NSB) & 1u)) break;
            tc_fence_after();
            const uint64_t da = smem_desc(ring + (uint32_t)(s * kChunkPages * T::PB), 128, T::REC);
            const uint32_t dst = tmem + T::T_S + sb * T::NQ;
#pragma unroll
            for (int k = 0; k < D / 32; k++) mma_i8_ss_w(dst, da + 16 * k, dq + 16 * k, IDQ, k > 0 ? 1u : 0u);
            tc_commit_w(sfull_b + 8 * sb);
            tc_commit_w(empty_b(s));
            last_bar = sfull_b + 8 * sb;
            last_par = (uint32_t)(i / T::NSB) & 1u;
            if (++s == NS) {
                s = 0;
                ph ^= 1u;
            }
        }
        // after an abort: the MMAs already issued finish before TMEM is released
        if (lane == 0 && *abort_flag != 0 && last_bar != 0) mbar_wait_bounded(last_bar, last_par);
        __syncwarp();
    } else if (warp == 2) {
        // ================= value MMAs (whole warp; one elected lane issues) =================
        const uint32_t wb0 = smem_u32(smem + S.wbuf);
        constexpr uint32_t IDO = instr_desc(1, 0, 0, 0, 1, 128, T::NO);   // f32 <- f16 x f16, B MN-major
        uint32_t last_bar = 0, last_par = 0;
        for (int j = 0; j < n_ck; j++) {
            const int wb = j % T::NWB, vb = j % T::NVB, ob = j % T::NOB;
            if (!wait_warp(wfull_b + 8 * wb, (uint32_t)(j / T::NWB) & 1u)) break;
            if (!wait_warp(vfull_b + 8 * vb, (uint32_t)(j / T::NVB) & 1u)) break;
            if (j >= T::NOB && !wait_warp(ofree_b + 8 * ob, (uint32_t)((j - T::NOB) / T::NOB) & 1u)) break;
            tc_fence_after();
            // descriptors of the chunk's weight buffer; each k-step adds a constant offset
            // (the 14-bit address field never carries: shared addresses stay below 2^18)
            const uint64_t dw = smem_desc(wb0 + (uint32_t)(wb * T::WBYTES), T::LBO_W, 128);
            const uint32_t vt = tmem + T::T_VT + vb * T::H * 64;
            const uint32_t dst = tmem + T::T_O + ob * T::H * T::NO;
#pragma unroll
            for (int ks = 0; ks < kChunkTokens / 16; ks++) {
                const uint64_t dk = dw + (uint64_t)((ks * 2 * T::LBO_W) >> 4);
#pragma unroll
                for (int h = 0; h < T::H; h++)
                    mma_f16_ts_w(dst + h * T::NO, vt + h * 64 + 8 * ks, dk + (uint64_t)((h * 64 * ROWS) >> 4), IDO,
                                 ks > 0 ? 1u : 0u);
            }
            tc_commit_w(pv_bar(j));
            last_bar = pv_bar(j);
            last_par = pv_par(j);
        }
        if (lane == 0 && *abort_flag != 0 && last_bar != 0) mbar_wait_bounded(last_bar, last_par);
        __syncwarp();
    } else if (warp < 7) {
        // ============ value codes -> V^T in tensor memory; merge of the chunk results ============
        const int q = warp & 3;
        // Chunk j's value accumulator, row maxima and sums of p, merged into the running
        // result by log-sum-exp (merge_coef / merge_val: the merge kernel's arithmetic).
        auto merge_chunk = [&](int j) -> bool {
            if (!wait_warp(pv_bar(j), pv_par(j))) return false;
            const int slot = j % T::NML;
            if (!wait_warp(mready_b + 8 * slot, (uint32_t)(j / T::NML) & 1u)) return false;
            // this chunk's row maxima, read before the accumulator is released (its release
            // lets the softmax reach chunk j + NML, which reuses the slot)
            float mj[ROWS];
#pragma unroll
            for (int r = 0; r < ROWS; r++) mj[r] = xm[slot * ROWS + r];
            tc_fence_after();
            float o[T::H][ROWS];
#pragma unroll
            for (int h = 0; h < T::H; h++) {
                const uint32_t col = T::T_O + (j % T::NOB) * T::H * T::NO + h * T::NO + q * ROWS;
                if constexpr (ROWS == 4) {
                    uint32_t v[4];
                    tmem_ld4(tmem_at(tmem, 32 * q, col), v);
                    tmem_wait_ld();
#pragma unroll
                    for (int r = 0; r < 4; r++) o[h][r] = __uint_as_float(v[r]);
                } else {
                    uint32_t v[8];
                    tmem_ld8(tmem_at(tmem, 32 * q, col), v);
                    tmem_wait_ld();
#pragma unroll
                    for (int r = 0; r < 8; r++) o[h][r] = __uint_as_float(v[r]);
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(ofree_b + 8 * (j % T::NOB));
#pragma unroll
            for (int r = 0; r < ROWS; r++) {
                float m, l, a, bc;
                merge_coef(Mr[r], 0.0f, mj[r], 0.0f, m, l, a, bc);
#pragma unroll
                for (int h = 0; h < T::H; h++) Or[h][r] = merge_val(Or[h][r], o[h][r], a, bc);
                Mr[r] = m;
            }
            return true;
        };
        bool ok = true;
        int s = 0;
        uint32_t ph = 0;   // ring stage of chunk i and the parity of its fill
        for (int i = 0; i < n_ck && ok; i++) {
            const int vb = i % T::NVB;
            // the V^T buffer of chunk i - 2 is free: its value MMAs were waited for when
            // chunk i - 2 was merged (in iteration i - 1)
            if (!wait_warp(full_b(s), ph)) {
                ok = false;
                break;
            }
            tc_fence_after();
            const uint32_t st = ring + (uint32_t)(s * kChunkPages * T::PB) + rec_v_off(D);
#pragma unroll
            for (int h = 0; h < T::H; h++) {
                const uint32_t cw = st + 4u * (uint32_t)(128 * h + 32 * q + lane);
#pragma unroll
                for (int pp = 0; pp < 2; pp++) {
                    uint32_t r[32];
#pragma unroll
                    for (int p4 = 0; p4 < 4; p4++)
#pragma unroll
                        for (int tg = 0; tg < 2; tg++) {
                            const uint32_t w = ldsa32(cw + (uint32_t)((4 * pp + p4) * T::PB + tg * T::REC));
                            // tokens (2k, 2k+1) of the record: bits 4k..4k+3 and 16+4k..
                            r[8 * p4 + 4 * tg + 0] = code_pair(w);
                            r[8 * p4 + 4 * tg + 1] = code_pair(w >> 4);
                            r[8 * p4 + 4 * tg + 2] = code_pair(w >> 8);
                            r[8 * p4 + 4 * tg + 3] = code_pair(w >> 12);
                        }
                    tmem_st32(tmem_at(tmem, 32 * q, T::T_VT + (vb * T::H + h) * 64 + 32 * pp), r);
                }
            }
            tmem_wait_st();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) {
                mbar_arrive(vfull_b + 8 * vb);
                mbar_arrive(empty_b(s));
            }
            if (++s == NS) {
                s = 0;
                ph ^= 1u;
            }
            if (i > 0) ok = merge_chunk(i - 1);
        }
        if (ok) ok = merge_chunk(n_ck - 1);
        tc_fence_before();
    } else {
        // ================= softmax and weights (one TMEM lane = one token) =================
        const int sw = warp - 7, q = warp & 3, t = 32 * q + lane;
        const int tp = t / 16, ttg = (t / 8) & 1, tt = t & 7;
        const uint32_t wb0 = smem_u32(smem + S.wbuf);
        float crow[ROWS];
        int lim[ROWS];
#pragma unroll
        for (int r = 0; r < ROWS; r++) {
            crow[r] = crow_s[r];
            lim[r] = lim_s[r];
        }
        const int lim_min = p.causal ? L - nq + row0 / p.group + 1 : L;   // smallest limit of the real rows
        // The running row maxima over the chunks so far (the same in every softmax warp: they
        // see the same chunk maxima) and this token's share of l = sum_t 2^(z_t - max), kept
        // relative to them; the shares are summed once, after the last chunk.
        float Mrun[ROWS], lt[ROWS];
#pragma unroll
        for (int r = 0; r < ROWS; r++) {
            Mrun[r] = -INFINITY;
            lt[r] = 0.0f;
        }
        // A warp whose wait gave up keeps iterating without work, so that the four warps
        // always meet at their named barrier the same number of times.
        bool ok = true;
        int s = 0;
        uint32_t ph = 0;   // ring stage of chunk i and the parity of its fill
        for (int i = 0; i < n_ck; i++) {
            const int sb = i % T::NSB, wb = i % T::NWB, slot = i % T::NML;
            const int c = c0 + i;
            float sk = 0.0f, sv[T::G];
            bool any_bad = false, my_bad = false;
            float z[ROWS];
            if (ok && wait_warp(full_b(s), ph)) {
                const uint32_t rec = ring + (uint32_t)((s * kChunkPages + tp) * T::PB + ttg * T::REC);
                sk = h_bits_to_f32(ldsa16(rec + rec_ks_off(D) + 2 * tt));
                if constexpr (T::G == 4) {
                    const uint2 v = ldsa64(rec + rec_vs_off(D) + 8 * tt);
                    sv[0] = h_bits_to_f32(v.x & 0xFFFFu);
                    sv[1] = h_bits_to_f32(v.x >> 16);
                    sv[2] = h_bits_to_f32(v.y & 0xFFFFu);
                    sv[3] = h_bits_to_f32(v.y >> 16);
                } else {
                    const uint4 v = ldsa128(rec + rec_vs_off(D) + 16 * tt);
                    const uint32_t u[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
                    for (int k = 0; k < 4; k++) {
                        sv[2 * k] = h_bits_to_f32(u[k] & 0xFFFFu);
                        sv[2 * k + 1] = h_bits_to_f32(u[k] >> 16);
                    }
                }
                const int4 bf0 = *reinterpret_cast<const int4*>(pgbad + s * kChunkPages);
                const int4 bf1 = *reinterpret_cast<const int4*>(pgbad + s * kChunkPages + 4);
                any_bad = (bf0.x | bf0.y | bf0.z | bf0.w | bf1.x | bf1.y | bf1.z | bf1.w) != 0;
                my_bad = pgbad[s * kChunkPages + tp] != 0;
                __syncwarp();
                if (lane == 0) mbar_arrive(empty_b(s));
            } else {
                ok = false;
            }
            if (ok && !wait_warp(sfull_b + 8 * sb, (uint32_t)(i / T::NSB) & 1u)) ok = false;
            const bool clean = (c + 1) * kChunkTokens <= lim_min && !any_bad;
            float* xb = xch + (i & 1) * ROWS * 4;
            if (ok) {
                tc_fence_after();
                // ---- scores: the three limb accumulations of each row -> fp32 ----
                uint32_t a[3 * ROWS];
                const uint32_t col = T::T_S + sb * T::NQ;
                if constexpr (ROWS == 4) {
                    uint32_t v[16];
                    tmem_ld16(tmem_at(tmem, 32 * q, col), v);
                    tmem_wait_ld();
#pragma unroll
                    for (int k = 0; k < 12; k++) a[k] = v[k];
                } else {
                    uint32_t v[16], w[8];
                    tmem_ld16(tmem_at(tmem, 32 * q, col), v);
                    tmem_ld8(tmem_at(tmem, 32 * q, col + 16), w);
                    tmem_wait_ld();
#pragma unroll
                    for (int k = 0; k < 16; k++) a[k] = v[k];
#pragma unroll
                    for (int k = 0; k < 8; k++) a[16 + k] = w[k];
                }
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(sfree_b + 8 * sb);
#pragma unroll
                for (int r = 0; r < ROWS; r++) {
                    const int x = (int)a[r] * 256 + (int)a[ROWS + r];   // exact: |x| < 2^30
                    const float sc = __fmaf_rn((float)x, 256.0f, (float)(int)a[2 * ROWS + r]);
                    z[r] = r < rows_here ? __fmul_rn(__fmul_rn(sc, crow[r]), sk) : -INFINITY;
                }
                // ---- visibility: sequence end, causal drafts, unusable pages ----
                if (!clean) {
                    const int tok = c * kChunkTokens + t;
#pragma unroll
                    for (int r = 0; r < ROWS; r++)
                        if (my_bad || tok >= lim[r]) z[r] = -INFINITY;
                }
                // ---- chunk row maxima over the 128 tokens ----
#pragma unroll
                for (int r = 0; r < ROWS; r++) {
                    const float m = warp_redux_max(z[r]);
                    if (lane == 0) xb[r * 4 + sw] = m;
                }
            }
            named_bar_sync(2, 128);
            if (ok && i >= T::NWB && !wait_warp(pv_bar(i - T::NWB), pv_par(i - T::NWB))) ok = false;
            if (ok) {
                // ---- p = 2^(z - chunk max) <= 1, this token's share of l, weights W_g = p * s_v[g] ----
                float pw[ROWS];
#pragma unroll
                for (int r = 0; r < ROWS; r++) {
                    const float4 v = *reinterpret_cast<const float4*>(xb + r * 4);
                    const float cm = fmaxf(fmaxf(v.x, v.y), fmaxf(v.z, v.w));
                    pw[r] = z[r] == -INFINITY ? 0.0f : ex2(__fsub_rn(z[r], cm));
                    const float mn = fmaxf(Mrun[r], cm);
                    const float al = Mrun[r] == mn ? 1.0f : ex2(__fsub_rn(Mrun[r], mn));
                    const float be = cm == mn ? 1.0f : ex2(__fsub_rn(cm, mn));
                    lt[r] = __fadd_rn(__fmul_rn(lt[r], al), __fmul_rn(pw[r], be));
                    Mrun[r] = mn;
                }
                // the chunk's row maxima for the merge of its value accumulator
                if (sw == 0 && lane < ROWS) {
                    const float4 v = *reinterpret_cast<const float4*>(xb + lane * 4);
                    xm[slot * ROWS + lane] = fmaxf(fmaxf(v.x, v.y), fmaxf(v.z, v.w));
                }
                const uint32_t wrow = wb0 + (uint32_t)(wb * T::WBYTES + (t / 8) * T::LBO_W + (t % 8) * 16);
                float w[T::G][ROWS];
#pragma unroll
                for (int g = 0; g < T::G; g++)
#pragma unroll
                    for (int r = 0; r < ROWS; r++) {
                        // masked tokens may carry unwritten (non-finite) scales
                        w[g][r] = (!clean && pw[r] == 0.0f) ? 0.0f : __fmul_rn(pw[r], sv[g]);
                    }
                if constexpr (ROWS == 4) {
                    // column group cg holds groups 2cg and 2cg + 1, rows 0-3 each
#pragma unroll
                    for (int cg = 0; cg < T::G / 2; cg++)
                        stsa128(wrow + 128u * cg, pack_h2(w[2 * cg][0], w[2 * cg][1]), pack_h2(w[2 * cg][2], w[2 * cg][3]),
                                pack_h2(w[2 * cg + 1][0], w[2 * cg + 1][1]), pack_h2(w[2 * cg + 1][2], w[2 * cg + 1][3]));
                } else {
#pragma unroll
                    for (int g = 0; g < T::G; g++)
                        stsa128(wrow + 128u * g, pack_h2(w[g][0], w[g][1]), pack_h2(w[g][2], w[g][3]),
                                pack_h2(w[g][4], w[g][5]), pack_h2(w[g][6], w[g][7]));
                }
                fence_proxy_async_smem();
                __syncwarp();
                if (lane == 0) {
                    mbar_arrive(wfull_b + 8 * wb);
                    mbar_arrive(mready_b + 8 * slot);
                }
            }
            if (++s == NS) {
                s = 0;
                ph ^= 1u;
            }
        }
        // l per row: the 128 tokens' shares, summed in a fixed order (warp butterfly, then
        // the four warps in index order by the value warps after the final barrier)
#pragma unroll
        for (int r = 0; r < ROWS; r++) {
            float v = lt[r];
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) v = __fadd_rn(v, __shfl_xor_sync(FULL, v, o));
            if (lane == 0) xlf[sw * ROWS + r] = v;
        }
    }

    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, T::TCOLS);
    }
    if (*abort_flag != 0 || warp < 3 || warp >= 7) return;

    // ---- the value warps write the CTA's result from registers (lane = channel) ----
    const int q = warp & 3;
#pragma unroll
    for (int r = 0; r < ROWS; r++)
        lr[r] = __fadd_rn(__fadd_rn(__fadd_rn(xlf[r], xlf[ROWS + r]), xlf[2 * ROWS + r]), xlf[3 * ROWS + r]);
    const size_t pidx = ((size_t)(b * p.n_kv_heads + hk) * p.n_rb + rb);
    if (n_splits == 1) {
        // out = O / l and lse for the real rows of this block
#pragma unroll
        for (int r = 0; r < ROWS; r++) {
            if (r >= rows_here) break;
            const int rr = row0 + r, j = rr / p.group, hq = rr % p.group;
            const long long qrow = (long long)qoff + j;
            if (qrow >= p.total_q) continue;
            const size_t orow = (size_t)qrow * p.n_q_heads + (size_t)hk * p.group + hq;
#pragma unroll
            for (int h = 0; h < T::H; h++) p.out[orow * D + 128 * h + 32 * q + lane] = __fdiv_rn(Or[h][r], lr[r]);
            if (q == 3 && lane == 0 && p.lse != nullptr)
                p.lse[orow] = __fmul_rn(__fadd_rn(Mr[r], log2f(lr[r])), 0.69314718055994531f);
        }
        return;
    }
    // ---- publish this CTA's partial; merge_kernel completes the tree ----
    float* go = p.part_o + (pidx * p.split_stride + sp) * (size_t)(ROWS * D);
    float* gml = p.part_ml + (pidx * p.split_stride + sp) * (size_t)(2 * ROWS);
#pragma unroll
    for (int r = 0; r < ROWS; r++)
#pragma unroll
        for (int h = 0; h < T::H; h++) __stcg(go + r * D + 128 * h + 32 * q + lane, Or[h][r]);
    if (q == 3 && lane < ROWS) {
        float m = Mr[0], l = lr[0];
#pragma unroll
        for (int r = 1; r < ROWS; r++)
            if (lane == r) {
                m = Mr[r];
                l = lr[r];
            }
        __stcg(gml + lane, m);
        __stcg(gml + ROWS + lane, l);
    }
}

size_t small_smem_bytes(int head_dim, int rows, int stages) {
#define MQ_SMEM(DD, RR) \
    if (head_dim == DD && rows == RR) return small_layout<DD, RR>(stages).total;
    MQ_SMEM(128, 4) MQ_SMEM(128, 8) MQ_SMEM(256, 4) MQ_SMEM(256, 8)
#undef MQ_SMEM
    return 0;
}

int small_ctas_per_sm(int head_dim, int rows) { return (head_dim == 128 && rows == 4) ? 2 : 1; }

template <int D, int ROWS>
static cudaError_t small_set_smem(size_t smem) {
    cudaError_t e =
        cudaFuncSetAttribute(decode_small_kernel<D, ROWS>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    // all of the unified L1 / shared-memory array as shared memory, so that two CTAs fit
    return cudaFuncSetAttribute(decode_small_kernel<D, ROWS>, cudaFuncAttributePreferredSharedMemoryCarveout, 100);
}

cudaError_t small_prepare(int head_dim, int rows, size_t smem) {
    if (head_dim == 128 && rows == 4) return small_set_smem<128, 4>(smem);
    if (head_dim == 128 && rows == 8) return small_set_smem<128, 8>(smem);
    if (head_dim == 256 && rows == 4) return small_set_smem<256, 4>(smem);
    if (head_dim == 256 && rows == 8) return small_set_smem<256, 8>(smem);
    return cudaErrorInvalidValue;
}

// The decode kernel of the small row classes, as a programmatic dependent launch.
cudaError_t small_launch(const DecodeParams& p, int head_dim, int rows, dim3 grid, size_t smem, cudaStream_t st) {
    cudaLaunchAttribute pdl[1];
    pdl[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    pdl[0].val.programmaticStreamSerializationAllowed = 1;
    cudaLaunchConfig_t dc{};
    dc.gridDim = grid;
    dc.blockDim = dim3(352);
    dc.dynamicSmemBytes = smem;
    dc.stream = st;
    dc.attrs = pdl;
    dc.numAttrs = 1;
    if (head_dim == 128 && rows == 4) return cudaLaunchKernelEx(&dc, decode_small_kernel<128, 4>, p);
    if (head_dim == 128 && rows == 8) return cudaLaunchKernelEx(&dc, decode_small_kernel<128, 8>, p);
    if (head_dim == 256 && rows == 4) return cudaLaunchKernelEx(&dc, decode_small_kernel<256, 4>, p);
    if (head_dim == 256 && rows == 8) return cudaLaunchKernelEx(&dc, decode_small_kernel<256, 8>, p);
    return cudaErrorInvalidValue;
}

}  // namespace mq
