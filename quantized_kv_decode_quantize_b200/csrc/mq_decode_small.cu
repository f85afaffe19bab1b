// Split-K flash-decode over the K8/V4 paged cache, with draft verification, on the sm_100a
// tensor cores: one warp-specialised kernel for every row class (4, 8, 16 or 32 query rows
// per kv-head; grouped-query decode at GQA 4 with one query token is 4 rows).
//
// What it computes (the deep dive on magnitudedev/magnitude at blog.123qwe.co.kr, section
// 5: the decode attention unit attention_decode_k8v4 over the 8-bit-key / 4-bit-value
// cache, and the guarantee that verifying several draft tokens is one launch against the
// cache): for query token j of sequence b (n_b query tokens, L_b cached tokens including
// the drafts) and q-head h,
//     z_t = scale * <q, s_k[t] * kcode_t>,  t = 0 .. L_b - n_b + j
//     out = sum_t softmax(z)_t * (s_v[t, group] * vcode_t),  lse = log sum_t exp z_t
//
// How.  One CTA (11 warps, 15 with two softmax groups; two CTAs per SM for 4 rows of
// head_dim 128) takes a contiguous range of 128-token chunks of one (sequence, kv-head,
// row block).  Every chunk is a small attention problem of its own, solved with the
// chunk's exact row maxima, and the per-chunk results are merged by log-sum-exp:
//  * warp 0 streams the chunk's 8 pages into a shared-memory ring, one 1-D bulk TMA copy
//    per page (block-table lookup, L2 evict-first);
//  * warp 1 issues the score MMAs (kind::i8, M = 128 tokens, q as three signed 8-bit
//    limbs per row along N, exact int32 products in tensor memory);
//  * the softmax warps (one or two groups of four; one TMEM lane = one token) form z in
//    fp32, take the chunk's row maxima (redux + one named barrier per group), and write
//    p = 2^(z - max) <= 1, the warp's exact integer sums of p per row, and the fp16
//    weights W_g = fp16(p) * s_v[token, g] to shared memory;
//  * warp 2 issues the value MMAs (kind::f16, A = V^T in tensor memory, B = the weights,
//    every group of 32 channels using its own columns) into a fresh accumulator per
//    chunk (two alternate), then keeps the row state, one lane per row: the chunk's
//    maximum and l, the running (M, l), and every log-sum-exp factor the merges use;
//  * warps 3-6 turn the chunk's int4 value codes into V^T in tensor memory as exact fp16
//    values (one channel per lane), then merge the previous chunk's accumulator into the
//    CTA's running output in registers (lane = channel) with warp 2's factors.
// The weights never exceed the fp16 range (p <= 1 and s_v <= 65504), no accumulator is
// ever rescaled in tensor memory, and the chunk steps of the softmax do not wait for one
// another.  The chunks of a merge-tree leaf (node_chunks chunks) fold in order; for the
// classes of up to 8 rows a CTA holds an aligned power-of-two run of leaves and combines
// it into that node of a fixed binary tree (see tree_step; pending children in tensor
// memory), otherwise its range is one leaf.  The CTA's partial goes to the workspace and
// merge_kernel (mq_decode.cu) finishes the tree; a unit of one CTA writes out and lse here.
#include "mq_decode_common.cuh"

namespace mq {

// Levels of the merge-tree node a CTA builds from its leaves: the classes whose split count
// is free (up to 8 rows, where tensor memory has room for the pending children; 64 leaves
// per unit at most); 0 for the others, whose leaf is the CTA's range.
constexpr int tree_levels(int D, int ROWS) { return (ROWS <= 8 && !(D == 256 && ROWS == 8)) ? 6 : 0; }

template <int D, int ROWS, int NSG_>
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
    // buffer depths that fill tensor memory for each class
    static constexpr int NSB = ROWS == 32 ? 1 : ((D == 256 && ROWS == 16) ? 2 : 4);   // score buffers
    static constexpr int NOB = 2;                           // per-chunk value accumulators
    static constexpr int NVB = (D == 256 && ROWS == 16) ? 1 : 2;   // V^T buffers
    static constexpr int NWB = 2;                           // weight buffers (shared memory)
    static constexpr int NPB = 2;                           // value-MMA completion barriers
    static constexpr int NML = NWB + NOB;                   // slots of the merge factors
    static constexpr int KMAX = tree_levels(D, ROWS);
    static constexpr int XS = 1 + KMAX;                     // factor pairs per row and chunk
    // softmax warp groups: a block's rows split over NSG groups of four warps (one warp
    // per TMEM lane quadrant each); rows meet only through the chunk maximum of each row,
    // which a group exchanges on its own named barrier
    static constexpr int NSG = NSG_;
    static constexpr int RPG = ROWS / NSG;                  // rows per group
    static constexpr int THREADS = 224 + 128 * NSG;         // 0 TMA, 1 QK, 2 PV, 3-6 values, 7.. softmax
    static constexpr int T_S = 0;
    static constexpr int T_O = NSB * NQ;
    static constexpr int T_VT = (T_O + NOB * H * NO + 31) / 32 * 32;
    static constexpr int T_STK = T_VT + NVB * H * 64;       // pending left children: KMAX x (H x ROWS)
    static constexpr int T_END = T_STK + KMAX * H * ROWS;
    static constexpr int WBYTES = kChunkTokens * NB * 2;    // one weight buffer
    static constexpr int LBO_W = NB / 8 * 128;              // its 8-token group stride
    static_assert(ROWS == 4 || ROWS == 8 || ROWS == 16 || ROWS == 32, "row class");
    static_assert(NSG == 1 || NSG == 2, "softmax groups");
    static_assert(RPG >= 4 && RPG <= 16, "rows per softmax group");
    static_assert(CPS == 1 || NSG == 1, "two CTAs per SM with one softmax group");
    static_assert(T_END <= TCOLS, "tensor memory budget");
    static_assert(NPB >= NOB && NPB >= NVB && NPB >= NWB, "completion barriers");
};

struct SmallSmem {
    size_t ring, wbuf, qlimb, xch, xm, lp, xl, crow, lim, pgbad, mbar, misc, total;
};

// NS = ring stages (chunks of 8 pages)
template <int D, int ROWS, int NSG>
__host__ __device__ inline SmallSmem small_layout(int NS) {
    using T = Sm<D, ROWS, NSG>;
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
    s.xch = off;                                  // [4][ROWS][4 warps] chunk row maxima
    off += (size_t)4 * ROWS * 4 * 4;
    s.xm = off;                                   // [NML][XS][ROWS] merge factors (a, b): the chunk's, then its leaf's
    off += (size_t)T::NML * T::XS * ROWS * 8;
    s.lp = off;                                   // [4][4 warps][ROWS] chunk sums of p (fixed point)
    off += (size_t)4 * 4 * ROWS * 4;
    s.xl = off;                                   // [2][ROWS] the CTA's row maxima and l
    off += (size_t)2 * ROWS * 4;
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

template <int D, int ROWS, int NSG>
__global__ void __launch_bounds__(Sm<D, ROWS, NSG>::THREADS, Sm<D, ROWS, NSG>::CPS)
    decode_small_kernel(const DecodeParams p) {
    using T = Sm<D, ROWS, NSG>;
    extern __shared__ __align__(1024) uint8_t smem[];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int NS = p.stages;
    const SmallSmem S = small_layout<D, ROWS, NSG>(NS);
    const unsigned FULL = 0xffffffffu;
    int* misc = reinterpret_cast<int*>(smem + S.misc);   // 0 qoff, 1 abort, 3 TMEM base, 5-9 flat plan

    // ---- this CTA's unit (sequence, kv-head, row block) and split ----
    int b, hk, rb, sp, cpc;
    bool flat = false;
    if constexpr (T::KMAX > 0) flat = p.cta_budget > 0;   // only the fixed-tree classes run flat grids
    if (flat) {
        // a flat grid: warp 0 finds the launch's leaves per CTA and this CTA's unit
        if (warp == 0) {
            SeqShape first;
            const int lpc = flat_lpc(p, ROWS, first);
            int fb = -1, fh = 0, fr = 0, fs = 0;
            if (!flat_locate(p, ROWS, lpc, first, blockIdx.x, fb, fh, fr, fs)) fb = -1;
            if (lane == 0) {
                misc[5] = fb;
                misc[6] = fh;
                misc[7] = fr;
                misc[8] = fs;
                misc[9] = lpc;
            }
            if (blockIdx.x == 0)   // sequences with bad bounds take no CTA: flagged here
                for (int bb = lane; bb < p.n_seqs; bb += 32) {
                    const int Lb = seq_len_of(p, bb), nb = seq_nq_of(p, bb);
                    if (nb < 1 || nb > p.max_q || nb > Lb ||
                        (long long)Lb + (long long)p.bt_col * kPageTokens > (long long)p.max_blocks_per_seq * kPageTokens)
                        atomicOr(p.err, kErrBadSeq);
                }
        }
        __syncthreads();
        if (misc[5] < 0) return;   // past the launch's work
        b = misc[5];
        hk = misc[6];
        rb = misc[7];
        sp = misc[8];
        cpc = misc[9] * p.node_chunks;
    } else {
        b = blockIdx.z;
        hk = blockIdx.y / p.n_rb;
        rb = blockIdx.y % p.n_rb;
        sp = blockIdx.x;
        cpc = p.cpc;
    }

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
    const int c0 = sp * cpc;
    if (c0 >= n_chunks) return;
    const int n_ck = min(c0 + cpc, n_chunks) - c0;
    // The merge tree's leaves are runs of node_chunks chunks, folded in order; the CTA's
    // range is whole leaves, and its partial is the tree node over them (see tree_step).
    // The unit's only CTA writes out and lse; otherwise merge_kernel combines the partials.
    const int node_ch = p.node_chunks;
    const int l0 = c0 / node_ch, l1 = (c0 + n_ck + node_ch - 1) / node_ch;   // this CTA's leaves
    const bool direct = (n_chunks + cpc - 1) / cpc == 1;                    // the unit's only CTA
    const size_t pidx = ((size_t)(b * p.n_kv_heads + hk) * p.n_rb + rb);
    auto leaf_end = [&](int c) { return c % node_ch == node_ch - 1 || c == n_chunks - 1; };

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
    volatile int* abort_flag = misc + 1;
    float* crow_s = reinterpret_cast<float*>(smem + S.crow);
    int* lim_s = reinterpret_cast<int*>(smem + S.lim);
    int* pgbad = reinterpret_cast<int*>(smem + S.pgbad);
    float* xch = reinterpret_cast<float*>(smem + S.xch);
    float2* xm = reinterpret_cast<float2*>(smem + S.xm);
    uint32_t* lpart = reinterpret_cast<uint32_t*>(smem + S.lp);
    float* xlf = reinterpret_cast<float*>(smem + S.xl);   // [ROWS] maxima, then [ROWS] l
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
            mbar_init(empty_b(s), 5 + 4 * T::NSG);   // QK commit + 4 value warps + the softmax warps
        }
        for (int j = 0; j < T::NSB; j++) {
            mbar_init(sfull_b + 8 * j, 1);
            mbar_init(sfree_b + 8 * j, 4 * T::NSG);
        }
        for (int j = 0; j < T::NWB; j++) mbar_init(wfull_b + 8 * j, 4 * T::NSG);
        for (int j = 0; j < T::NVB; j++) mbar_init(vfull_b + 8 * j, 4);
        for (int j = 0; j < T::NPB; j++) mbar_init(pvdone_b + 8 * j, 1);
        for (int j = 0; j < T::NOB; j++) mbar_init(ofree_b + 8 * j, 4);
        for (int j = 0; j < T::NML; j++) mbar_init(mready_b + 8 * j, 1);
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
        q_to_limbs<D, ROWS, T::NQ>(p, smem + S.qlimb, crow_s, lim_s, threadIdx.x - 224, 128 * T::NSG, row0, rows_here,
                                   qoff, L, nq, hk);
        fence_proxy_async_smem();
    }
    // the TMA producer starts at once; the other warps wait for the limbs and TMEM
    if (warp != 0) named_bar_sync(1, T::THREADS - 32);
    tc_fence_after();
    const uint32_t tmem = (uint32_t)misc[3];
    const uint32_t ring = smem_u32(smem + S.ring);

    // the CTA's running output, held by the value warps (lane = channel of each half); the
    // pending left children of its tree node wait in tensor memory
    float Or[T::H][ROWS];
    uint32_t occ_v = 0u;
#pragma unroll
    for (int r = 0; r < ROWS; r++)
#pragma unroll
        for (int h = 0; h < T::H; h++) Or[h][r] = 0.0f;

    if (warp == 0) {
        // ================= TMA producer =================
        // The kernel is a programmatic dependent launch: a preceding kernel that allows it
        // (the append of this step) may still be writing pages.  Wait for it to complete
        // before the first page is read; everything before this point reads only the
        // launch's inputs, which no such kernel writes.  Meanwhile the pages of the first
        // ring-full of chunks are brought into L2 (a prefetch moves no data to the SM and
        // has no effect on what a later read returns: a page the append rewrites is read
        // from L2 after the wait like any other).
        {
            // lane = page (lane % 8) of chunk lane / 8: up to four chunks in one round of loads
            const int i = lane / kChunkPages, lp = (c0 + i) * kChunkPages + lane % kChunkPages;
            if (i < NS && i < n_ck && lp < n_pages) {
                const int blk = __ldg(p.block_table + (long long)b * p.max_blocks_per_seq + p.bt_col + lp);
                if (blk >= 0 && (long long)blk < p.n_blocks)
                    bulk_prefetch_l2(p.pool + ((long long)blk * p.n_kv_heads + hk) * T::PB, T::PB);
            }
        }
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
        // The row state, lane r = row r of the block, kept here once the chunk's value MMAs
        // are issued (off the softmax warps' path): the current leaf's running maximum M
        // and l = sum_t 2^(z_t - M), and the (M, l) of the pending left children of the
        // CTA's merge subtrees.  Per chunk it forms the log-sum-exp factors (a, b) for the
        // value warps' merges: the chunk's into the leaf, then the leaf's into the subtrees.
        float Mrow = -INFINITY, lrow = 0.0f;
        float Ms[T::KMAX > 0 ? T::KMAX : 1], ls[T::KMAX > 0 ? T::KMAX : 1];
        uint32_t occ = 0u;
        auto row_step = [&](int j) {
            const int c = c0 + j, xbuf = j & 3;
            // the chunk's row maximum (the four softmax warps' maxima) and l: their sums of
            // bits(1 + p_t), less 128 x bits(1.0), are sum_t round(p_t * 2^23) < 2^31
            const float4 v = *reinterpret_cast<const float4*>(xch + (xbuf * ROWS + lane) * 4);
            const float cm = fmaxf(fmaxf(v.x, v.y), fmaxf(v.z, v.w));
            uint32_t u = 0u - 128u * 0x3F800000u;
#pragma unroll
            for (int k = 0; k < 4; k++) u += lpart[(xbuf * 4 + k) * ROWS + lane];
            const float lc = __fmul_rn((float)u, 0x1p-23f);
            const float mn = fmaxf(Mrow, cm);
            const float a = Mrow == mn ? 1.0f : ex2(__fsub_rn(Mrow, mn));
            const float bb = cm == mn ? 1.0f : ex2(__fsub_rn(cm, mn));
            Mrow = mn;
            lrow = __fadd_rn(__fmul_rn(lrow, a), __fmul_rn(lc, bb));
            float2* xf = xm + (size_t)(j % T::NML) * T::XS * ROWS + lane;
            xf[0] = make_float2(a, bb);
            if (!leaf_end(c)) return;
            // the leaf's merges into the CTA's tree node
            const int li = c / node_ch;
            const bool last = li == l1 - 1;
            const TreeStep st = tree_step(li, l0, last, occ, T::KMAX);
            int k = 1;
#pragma unroll
            for (int t = 0; t < T::KMAX; t++)
                if ((st.merge_mask >> t) & 1u) {
                    float m, l, fa, fb;
                    merge_coef(Ms[t], ls[t], Mrow, lrow, m, l, fa, fb);
                    xf[k * ROWS] = make_float2(fa, fb);
                    Mrow = m;
                    lrow = l;
                    k++;
                }
            if (st.push) {
#pragma unroll
                for (int t = 0; t < T::KMAX; t++)
                    if (t == st.level) {
                        Ms[t] = Mrow;
                        ls[t] = lrow;
                    }
                occ = (occ & ~st.merge_mask) | (1u << st.level);
                Mrow = -INFINITY;   // the next leaf starts afresh
                lrow = 0.0f;
            } else if (!direct) {
                float* gml = p.part_ml + (pidx * p.split_stride + sp) * (size_t)(2 * ROWS);
                __stcg(gml + lane, Mrow);
                __stcg(gml + ROWS + lane, lrow);
            } else {
                xlf[lane] = Mrow;   // the unit's root, for the epilogue
                xlf[ROWS + lane] = lrow;
            }
        };
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
            // the chunk's maxima and sums of p are complete (the softmax warps wrote them
            // before their arrival on wfull)
            if (lane < ROWS) row_step(j);
            __syncwarp();
            if (lane == 0) mbar_arrive(mready_b + 8 * (j % T::NML));
        }
        if (lane == 0 && *abort_flag != 0 && last_bar != 0) mbar_wait_bounded(last_bar, last_par);
        __syncwarp();
    } else if (warp < 7) {
        // ============ value codes -> V^T in tensor memory; merge of the chunk results ============
        const int q = warp & 3;
        // Chunk j's value accumulator, merged into the running output with the chunk's
        // log-sum-exp factors (a, b) per row, which the softmax computed once per row
        // (merge_val: the merge kernel's arithmetic); at a leaf's end, the leaf's merges
        // into the CTA's subtrees with the factors that follow.
        auto merge_chunk = [&](int j) -> bool {
            if (!wait_warp(pv_bar(j), pv_par(j))) return false;
            const int slot = j % T::NML;
            if (!wait_warp(mready_b + 8 * slot, (uint32_t)(j / T::NML) & 1u)) return false;
            // Row groups of up to 16: each reads its factors and its accumulator columns, and
            // merges them.  (The factor slot stays valid after the accumulator's release: it
            // is rewritten for chunk j + NML, whose value MMAs wait for the release of chunk
            // j + NWB's accumulator, i.e. for this warp to be past chunk j.)
            constexpr int RG = ROWS < 16 ? ROWS : 16;
            tc_fence_after();
#pragma unroll
            for (int g0 = 0; g0 < ROWS; g0 += RG) {
                float2 f[RG];
#pragma unroll
                for (int r = 0; r < RG; r++) f[r] = xm[slot * T::XS * ROWS + g0 + r];
                float o[T::H][RG];
#pragma unroll
                for (int h = 0; h < T::H; h++) {
                    const uint32_t col = T::T_O + (j % T::NOB) * T::H * T::NO + h * T::NO + q * ROWS + g0;
                    uint32_t v[RG];
                    if constexpr (RG == 4) tmem_ld4(tmem_at(tmem, 32 * q, col), v);
                    else if constexpr (RG == 8) tmem_ld8(tmem_at(tmem, 32 * q, col), v);
                    else tmem_ld16(tmem_at(tmem, 32 * q, col), v);
                    tmem_wait_ld();
#pragma unroll
                    for (int r = 0; r < RG; r++) o[h][r] = __uint_as_float(v[r]);
                }
                if (g0 + RG == ROWS) {
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(ofree_b + 8 * (j % T::NOB));
                }
#pragma unroll
                for (int r = 0; r < RG; r++)
#pragma unroll
                    for (int h = 0; h < T::H; h++) Or[h][g0 + r] = merge_val(Or[h][g0 + r], o[h][r], f[r].x, f[r].y);
            }
            const int c = c0 + j;
            if (leaf_end(c)) {
                const int li = c / node_ch;
                const bool last = li == l1 - 1;
                const TreeStep st = tree_step(li, l0, last, occ_v, T::KMAX);
                const float2* xf = xm + (size_t)slot * T::XS * ROWS;
                constexpr int HR = T::H * ROWS;
                if constexpr (T::KMAX > 0) {
                    int k = 1;
#pragma unroll 1
                    for (int t = 0; t < T::KMAX; t++) {
                        if (!((st.merge_mask >> t) & 1u)) continue;
                        uint32_t sv[HR];
                        if constexpr (HR == 4) tmem_ld4(tmem_at(tmem, 32 * q, T::T_STK + t * HR), sv);
                        else tmem_ld8(tmem_at(tmem, 32 * q, T::T_STK + t * HR), sv);
                        tmem_wait_ld();
#pragma unroll
                        for (int r = 0; r < ROWS; r++) {
                            const float2 fk = xf[k * ROWS + r];
#pragma unroll
                            for (int h = 0; h < T::H; h++)
                                Or[h][r] = merge_val(__uint_as_float(sv[h * ROWS + r]), Or[h][r], fk.x, fk.y);
                        }
                        k++;
                    }
                }
                if (st.push) {
                    if constexpr (T::KMAX > 0) {
                        uint32_t sv[HR];
#pragma unroll
                        for (int h = 0; h < T::H; h++)
#pragma unroll
                            for (int r = 0; r < ROWS; r++) sv[h * ROWS + r] = __float_as_uint(Or[h][r]);
                        if constexpr (HR == 4) tmem_st4(tmem_at(tmem, 32 * q, T::T_STK + st.level * HR), sv);
                        else tmem_st8(tmem_at(tmem, 32 * q, T::T_STK + st.level * HR), sv);
                        tmem_wait_st();
                    }
#pragma unroll
                    for (int r = 0; r < ROWS; r++)
#pragma unroll
                        for (int h = 0; h < T::H; h++) Or[h][r] = 0.0f;
                    occ_v = (occ_v & ~st.merge_mask) | (1u << st.level);
                } else if (!direct) {
                    // the CTA's node: its partial (lane = channel)
                    float* go = p.part_o + (pidx * p.split_stride + sp) * (size_t)(ROWS * D);
#pragma unroll
                    for (int r = 0; r < ROWS; r++)
#pragma unroll
                        for (int h = 0; h < T::H; h++) __stcg(go + r * D + 128 * h + 32 * q + lane, Or[h][r]);
                }
            }
            return true;
        };
        bool ok = true;
        int s = 0;
        uint32_t ph = 0;   // ring stage of chunk i and the parity of its fill
        for (int i = 0; i < n_ck && ok; i++) {
            const int vb = i % T::NVB;
            // the V^T buffer of chunk i - NVB is free: its value MMAs were waited for when
            // that chunk was merged (in iteration i - 1, or just below with one buffer)
            if constexpr (T::NVB == 1) {
                if (i > 0 && !(ok = merge_chunk(i - 1))) break;
            }
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
                            r[8 * p4 + 4 * tg + 1] = code_pair_hi(w);
                            r[8 * p4 + 4 * tg + 2] = code_pair(w >> 8);
                            r[8 * p4 + 4 * tg + 3] = code_pair_hi(w >> 8);
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
            if constexpr (T::NVB > 1) {
                if (i > 0) ok = merge_chunk(i - 1);
            }
        }
        if (ok) ok = merge_chunk(n_ck - 1);
        tc_fence_before();
    } else {
        // ================= softmax and weights (one TMEM lane = one token) =================
        // group sg takes rows r0g .. r0g + RPG - 1; its warp k reads TMEM lane quadrant q
        constexpr int RPG = T::RPG;
        const int sg = (warp - 7) >> 2, sw = (warp - 7) & 3, q = warp & 3, t = 32 * q + lane;
        const int r0g = sg * RPG;
        const int tp = t / 16, ttg = (t / 8) & 1, tt = t & 7;
        const uint32_t wb0 = smem_u32(smem + S.wbuf);
        // row factors and limits: registers for up to 8 rows, shared memory beyond
        constexpr bool RREG = RPG <= 8;
        float crow[RREG ? RPG : 1];
        int lim[RREG ? RPG : 1];
        if constexpr (RREG) {
#pragma unroll
            for (int r = 0; r < RPG; r++) {
                crow[r] = crow_s[r0g + r];
                lim[r] = lim_s[r0g + r];
            }
        }
        auto crow_of = [&](int r) { if constexpr (RREG) return crow[r]; else return crow_s[r0g + r]; };
        auto lim_of = [&](int r) { if constexpr (RREG) return lim[r]; else return lim_s[r0g + r]; };
        const int lim_min = p.causal ? L - nq + row0 / p.group + 1 : L;   // smallest limit of the real rows
        // A warp whose wait gave up keeps iterating without work, so that the four warps
        // always meet at their named barrier the same number of times.
        bool ok = true;
        int s = 0;
        uint32_t ph = 0;   // ring stage of chunk i and the parity of its fill
        for (int i = 0; i < n_ck; i++) {
            const int sb = i % T::NSB, wb = i % T::NWB, slot = i % T::NML;
            const int c = c0 + i;
            float sk = 0.0f;
            uint32_t sv2[T::G];   // the token's value scales as fp16 pairs (s_v[g], s_v[g])
            bool any_bad = false, my_bad = false;
            float z[RPG];
            if (ok && wait_warp(full_b(s), ph)) {
                const uint32_t rec = ring + (uint32_t)((s * kChunkPages + tp) * T::PB + ttg * T::REC);
                sk = h_bits_to_f32(ldsa16(rec + rec_ks_off(D) + 2 * tt));
                if constexpr (T::G == 4) {
                    const uint2 v = ldsa64(rec + rec_vs_off(D) + 8 * tt);
                    sv2[0] = __byte_perm(v.x, 0u, 0x1010);
                    sv2[1] = __byte_perm(v.x, 0u, 0x3232);
                    sv2[2] = __byte_perm(v.y, 0u, 0x1010);
                    sv2[3] = __byte_perm(v.y, 0u, 0x3232);
                } else {
                    const uint4 v = ldsa128(rec + rec_vs_off(D) + 16 * tt);
                    const uint32_t u[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
                    for (int k = 0; k < 4; k++) {
                        sv2[2 * k] = __byte_perm(u[k], 0u, 0x1010);
                        sv2[2 * k + 1] = __byte_perm(u[k], 0u, 0x3232);
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
            float* xb = xch + (i & 3) * ROWS * 4 + r0g * 4;
            if (ok) {
                tc_fence_after();
                // ---- scores: the three limb accumulations of each row -> fp32 ----
                uint32_t a[3 * RPG];
                const uint32_t col = T::T_S + sb * T::NQ;
                if constexpr (RPG == 16 || T::NSG > 1) {
                    // limb l of row r sits in column l * ROWS + r: the group's rows of each limb
                    uint32_t v0[RPG], v1[RPG], v2[RPG];
                    if constexpr (RPG == 16) {
                        tmem_ld16(tmem_at(tmem, 32 * q, col + r0g), v0);
                        tmem_ld16(tmem_at(tmem, 32 * q, col + ROWS + r0g), v1);
                        tmem_ld16(tmem_at(tmem, 32 * q, col + 2 * ROWS + r0g), v2);
                    } else if constexpr (RPG == 8) {
                        tmem_ld8(tmem_at(tmem, 32 * q, col + r0g), v0);
                        tmem_ld8(tmem_at(tmem, 32 * q, col + ROWS + r0g), v1);
                        tmem_ld8(tmem_at(tmem, 32 * q, col + 2 * ROWS + r0g), v2);
                    } else {
                        tmem_ld4(tmem_at(tmem, 32 * q, col + r0g), v0);
                        tmem_ld4(tmem_at(tmem, 32 * q, col + ROWS + r0g), v1);
                        tmem_ld4(tmem_at(tmem, 32 * q, col + 2 * ROWS + r0g), v2);
                    }
                    tmem_wait_ld();
#pragma unroll
                    for (int k = 0; k < RPG; k++) {
                        a[k] = v0[k];
                        a[RPG + k] = v1[k];
                        a[2 * RPG + k] = v2[k];
                    }
                } else if constexpr (ROWS == 4) {
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
                for (int r = 0; r < RPG; r++) {
                    // every limb sum is below 2^22 in magnitude: exact as fp32 through the
                    // 1.5 x 2^23 bias (integer add, float subtract)
                    const float f0 = __fsub_rn(__int_as_float((int)a[r] + 0x4B400000), 12582912.0f);
                    const float f1 = __fsub_rn(__int_as_float((int)a[RPG + r] + 0x4B400000), 12582912.0f);
                    const float f2 = __fsub_rn(__int_as_float((int)a[2 * RPG + r] + 0x4B400000), 12582912.0f);
                    const float sc = __fmaf_rn(f0, 65536.0f, __fmaf_rn(f1, 256.0f, f2));
                    z[r] = r0g + r < rows_here ? __fmul_rn(__fmul_rn(sc, crow_of(r)), sk) : -INFINITY;
                }
                // ---- visibility: sequence end, causal drafts, unusable pages ----
                if (!clean) {
                    const int tok = c * kChunkTokens + t;
#pragma unroll
                    for (int r = 0; r < RPG; r++)
                        if (my_bad || tok >= lim_of(r)) z[r] = -INFINITY;
                }
                // ---- chunk row maxima over the 128 tokens ----
                // (the reductions are issued back to back: their latencies overlap)
                float mx[RPG];
#pragma unroll
                for (int r = 0; r < RPG; r++) mx[r] = warp_redux_max(z[r]);
                if (lane == 0) {
#pragma unroll
                    for (int r = 0; r < RPG; r++) xb[r * 4 + sw] = mx[r];
                }
            }
            named_bar_sync(2 + sg, 128);
            if (ok && i >= T::NWB && !wait_warp(pv_bar(i - T::NWB), pv_par(i - T::NWB))) ok = false;
            if (ok) {
                // ---- p = 2^(z - chunk max) <= 1, the warp's sums of p, weights W_g = p * s_v[g] ----
                float pw[RPG];
                uint32_t* lp = lpart + ((i & 3) * 4 + sw) * ROWS + r0g;
#pragma unroll
                for (int r = 0; r < RPG; r++) {
                    const float4 v = *reinterpret_cast<const float4*>(xb + r * 4);
                    const float cm = fmaxf(fmaxf(v.x, v.y), fmaxf(v.z, v.w));
                    pw[r] = z[r] == -INFINITY ? 0.0f : ex2(__fsub_rn(z[r], cm));
                }
                // 1 + p in [1, 2]: its bits are bits(1.0) + round(p * 2^23)
                uint32_t psum[RPG];
#pragma unroll
                for (int r = 0; r < RPG; r++) psum[r] = warp_redux_add(__float_as_uint(__fadd_rn(pw[r], 1.0f)));
                if (lane == 0) {
#pragma unroll
                    for (int r = 0; r < RPG; r++) lp[r] = psum[r];
                }
                const uint32_t wrow = wb0 + (uint32_t)(wb * T::WBYTES + (t / 8) * T::LBO_W + (t % 8) * 16);
                // W_g = fp16(p) * s_v[g], two rows per fp16 pair multiply.  A token that no row
                // sees (past the sequence end, or on an unusable page) may carry unwritten,
                // non-finite scales: its scales are taken as 0 (its p is 0 in every row).
                if (!clean && (my_bad || c * kChunkTokens + t >= L)) {
#pragma unroll
                    for (int g = 0; g < T::G; g++) sv2[g] = 0u;
                }
                uint32_t ph[(RPG + 1) / 2];
#pragma unroll
                for (int k = 0; k < RPG / 2; k++) ph[k] = pack_h2(pw[2 * k], pw[2 * k + 1]);
                auto wpair = [&](int k, int g) { return h2_as_u32(__hmul2(u32_as_h2(ph[k]), u32_as_h2(sv2[g]))); };
                if constexpr (ROWS > 8) {
                    // column g * ROWS + r0g + 8k + (0..7) of the weights: one 8-column group each
#pragma unroll
                    for (int g = 0; g < T::G; g++)
#pragma unroll
                        for (int k = 0; k < RPG / 8; k++)
                            stsa128(wrow + 128u * (uint32_t)((g * ROWS + r0g) / 8 + k), wpair(4 * k, g),
                                    wpair(4 * k + 1, g), wpair(4 * k + 2, g), wpair(4 * k + 3, g));
                } else if constexpr (T::NSG > 1) {
                    // 8 rows in two groups of 4: this group's half of each 8-column group
#pragma unroll
                    for (int g = 0; g < T::G; g++) stsa64(wrow + 128u * g + 2u * r0g, wpair(0, g), wpair(1, g));
                } else if constexpr (ROWS == 4) {
                    // column group cg holds groups 2cg and 2cg + 1, rows 0-3 each
#pragma unroll
                    for (int cg = 0; cg < T::G / 2; cg++)
                        stsa128(wrow + 128u * cg, wpair(0, 2 * cg), wpair(1, 2 * cg), wpair(0, 2 * cg + 1),
                                wpair(1, 2 * cg + 1));
                } else {
#pragma unroll
                    for (int g = 0; g < T::G; g++)
                        stsa128(wrow + 128u * g, wpair(0, g), wpair(1, g), wpair(2, g), wpair(3, g));
                }
                fence_proxy_async_smem();
                __syncwarp();
                if (lane == 0) mbar_arrive(wfull_b + 8 * wb);

            }
            if (++s == NS) {
                s = 0;
                ph ^= 1u;
            }
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
    const float* Mr = xlf;
    const float* lr = xlf + ROWS;
    if (!direct) return;   // the leaves are published; the merge kernel writes the output
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
}

// every (head_dim, rows, softmax groups) built: head_dim 128 with 4, 8, 16 or 32 rows and
// head_dim 256 with 4, 8 or 16; one group of four softmax warps, or two for blocks of 8 and
// more rows (two for 32)
#define MQ_SMALL_CLASSES(X)                                                                         \
    X(128, 4, 1) X(128, 8, 1) X(128, 8, 2) X(128, 16, 1) X(128, 16, 2) X(128, 32, 2) X(256, 4, 1) \
    X(256, 8, 1) X(256, 8, 2) X(256, 16, 1) X(256, 16, 2)

size_t small_smem_bytes(int head_dim, int rows, int groups, int stages) {
#define MQ_SMEM(DD, RR, GG) \
    if (head_dim == DD && rows == RR && groups == GG) return small_layout<DD, RR, GG>(stages).total;
    MQ_SMALL_CLASSES(MQ_SMEM)
#undef MQ_SMEM
    return 0;
}

int small_ctas_per_sm(int head_dim, int rows) { return (head_dim == 128 && rows == 4) ? 2 : 1; }

int small_leaf_kmax(int head_dim, int rows) { return tree_levels(head_dim, rows); }

template <int D, int ROWS, int NSG>
static cudaError_t small_set_smem(size_t smem) {
    cudaError_t e = cudaFuncSetAttribute(decode_small_kernel<D, ROWS, NSG>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    // all of the unified L1 / shared-memory array as shared memory, so that two CTAs fit
    return cudaFuncSetAttribute(decode_small_kernel<D, ROWS, NSG>, cudaFuncAttributePreferredSharedMemoryCarveout,
                                100);
}

cudaError_t small_prepare(int head_dim, int rows, int groups, size_t smem) {
#define MQ_PREP(DD, RR, GG) \
    if (head_dim == DD && rows == RR && groups == GG) return small_set_smem<DD, RR, GG>(smem);
    MQ_SMALL_CLASSES(MQ_PREP)
#undef MQ_PREP
    return cudaErrorInvalidValue;
}

template <int D, int ROWS, int NSG>
static cudaError_t small_launch_t(const DecodeParams& p, dim3 grid, size_t smem, cudaStream_t st) {
    cudaLaunchAttribute pdl[1];
    pdl[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    pdl[0].val.programmaticStreamSerializationAllowed = 1;
    cudaLaunchConfig_t dc{};
    dc.gridDim = grid;
    dc.blockDim = dim3((unsigned)Sm<D, ROWS, NSG>::THREADS);
    dc.dynamicSmemBytes = smem;
    dc.stream = st;
    dc.attrs = pdl;
    dc.numAttrs = 1;
    return cudaLaunchKernelEx(&dc, decode_small_kernel<D, ROWS, NSG>, p);
}

// The decode kernel of the row class, as a programmatic dependent launch.
cudaError_t small_launch(const DecodeParams& p, int head_dim, int rows, int groups, dim3 grid, size_t smem,
                         cudaStream_t st) {
#define MQ_LAUNCH(DD, RR, GG) \
    if (head_dim == DD && rows == RR && groups == GG) return small_launch_t<DD, RR, GG>(p, grid, smem, st);
    MQ_SMALL_CLASSES(MQ_LAUNCH)
#undef MQ_LAUNCH
    return cudaErrorInvalidValue;
}

}  // namespace mq
