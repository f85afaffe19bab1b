// Split-K flash-decode over the K8/V4 paged cache, with draft verification, on the
// sm_100a tensor cores (tcgen05 + tensor memory).
//
// What it computes (the deep dive on magnitudedev/magnitude at blog.123qwe.co.kr,
// section 5: the decode attention unit attention_decode_k8v4 over the 8-bit-key /
// 4-bit-value cache, and the guarantee that verifying several draft tokens is
// one launch against the cache): for query token j of sequence b (n_b query
// tokens, L_b cached tokens including the drafts) and q-head h,
//     z_t = scale * <q, s_k[t] * kcode_t>,  t = 0 .. L_b - n_b + j
//     out = sum_t softmax(z)_t * (s_v[t, group] * vcode_t),  lse = log sum_t exp z_t
//
// How.  One CTA (11 warps, 15 for the 32-row class; two CTAs per SM for the 8-row D=128
// class, one per SM otherwise) takes a contiguous range of 128-token chunks of one
// (sequence, kv-head, row block) and runs a warp-specialised pipeline per chunk:
//  * warp 0 streams the chunk's 8 pages into a shared-memory ring with one 1-D bulk
//    TMA copy per page (block-table lookup, L2 evict-first).  The page format makes
//    the int8 key codes of a chunk one K-major tensor-core operand as they land.
//  * warps 1 and 2 issue the MMAs, one thread each (scores, values).  Scores: S = K q^T with kind::i8, M = 128
//    tokens, the query rows as the N side, q held as a 23-bit fixed-point value per row
//    (q = Q * 2^(E-22)) split into three signed 8-bit limbs stacked along N, so the
//    int32 products are exact; S lands in tensor memory.  Values: O += V^T W with
//    kind::f16, A = V^T from tensor memory (M = 128 channels, K = tokens), B = the
//    weights W_g = p * s_v[token, group] for every group g of 32 channels stacked
//    along N; each channel keeps only its own group's columns.  A second MMA with a
//    constant all-ones A gives, in every lane, the column sums of W: the per-group
//    sums that undo the value-code offset, and l = sum_t p from the p columns.
//  * warps 3-6 turn the int4 value codes into tensor memory as exact fp16 values
//    u * 2^-24 (u = code + 8 in 0..15, a subnormal) with one mask, shift and flip per
//    two tokens, a channel per TMEM lane; out = 2^24 * O - 8 * sum_t W_g.
//  * warps 7-10 (one TMEM lane per token; 7-14 in two row groups for the 32-row class)
//    read S, form z in fp32, take the chunk's row maxima (redux + a named barrier),
//    keep a lazy running max M per row (moved only
//    when a chunk max exceeds it by more than kLazy, after rescaling O and the sums in
//    tensor memory), and write p = 2^(z - M) and the weights W_g (fp16) to shared memory.
// The CTA partials of a (sequence, kv-head, row block) are combined by one fixed binary
// tree over the split index in merge_kernel, launched right after this kernel as a
// programmatic dependent launch; it writes out and lse.  A unit that is not split writes
// them here.  The chunk ranges depend only on the shape, the SM count and the configured
// splits per SM, so the result is bit-identical for every ring depth.
#include "mq_decode_common.cuh"

namespace mq {

// lazy-max threshold of the online softmax, in log2 units (weights stay <= 2^4)
constexpr float kLazy = 4.0f;

template <int D, int ROWS>
struct Tc {
    static constexpr int PB = page_bytes(D);
    static constexpr int REC = rec_bytes(D);
    static constexpr int G = D / 32;                              // value groups
    static constexpr int H = D / 128;                             // 128-channel halves (PV M tiles)
    static constexpr int NQ = (3 * ROWS + 15) / 16 * 16;          // score MMA N: 3 limbs x rows
    static constexpr int NO = 4 * ROWS;                           // value MMA N per half
    static constexpr int NB = G * ROWS;                           // weight columns: W_0 .. W_{G-1}
    // One CTA per SM owns all of tensor memory.  Every hand-off between the roles is
    // buffered as deeply as tensor and shared memory allow, so that several chunks are
    // in flight in each stage and the latency of an MMA (issue to commit) is hidden.
    // The 8-row D=128 class (grouped-query decode, the common case) runs two CTAs per SM
    // instead, each with half of tensor memory: two independent pipelines per SM hide
    // each other's latencies better than deeper buffers in one.
    static constexpr int CPS = (D == 128 && ROWS == 8) ? 2 : 1;
    static constexpr int TCOLS = CPS == 2 ? 256 : 512;                           // TMEM columns allocated
    // Two score buffers let the score MMAs of chunk i + 1 run while the softmax still
    // reads chunk i; two V^T buffers let the conversion of chunk i + 1 overlap the value
    // MMAs of chunk i.
    static constexpr int NSB = CPS == 2 ? 2 : ((D == 128 && ROWS <= 16) ? 4 : 2);   // score buffers (TMEM)
    static constexpr int NVB = 2;                                                // V^T buffers (TMEM)
    static constexpr int NWB = CPS == 2 ? 2 : 3;                                 // weight buffers (smem)
    static constexpr int NPB = NWB > NVB ? NWB : NVB;                            // value-MMA completion barriers
    // Softmax warp groups: the 32-row class splits its rows over two groups of four warps
    // (one warp per TMEM lane quadrant each); rows interact only through the chunk maximum
    // of each row, which a group exchanges on its own named barrier.
    static constexpr int NSG = ROWS == 32 ? 2 : 1;
    static constexpr int RPG = ROWS / NSG;                                       // rows per group
    // warp 0 TMA, 1 QK MMA, 2 PV MMA, 3-6 values, 7.. softmax
    static constexpr int THREADS = 224 + 128 * NSG;
    // tensor-memory columns
    static constexpr int T_S = 0;
    static constexpr int T_O = NSB * NQ;
    static constexpr int T_VT = (T_O + H * NO + 31) / 32 * 32;
    static constexpr int T_END = T_VT + NVB * H * 64;
    static constexpr int WBYTES = kChunkTokens * NB * 2;          // one weight buffer
    static constexpr int LBO_W = NB / 8 * 128;                    // its 8-token group stride
    static constexpr int PART = ROWS * D + 2 * ROWS;              // floats of one partial
    static_assert(T_END <= TCOLS, "tensor memory budget");
    static_assert(NQ <= 256 && NO <= 256, "MMA N range");
};

struct Smem {
    size_t ring, wbuf, qlimb, part, xch, xsv, crow, lim, pgbad, mbar, misc, total;
};

// NS = ring stages (chunks of 8 pages)
template <int D, int ROWS>
__host__ __device__ inline Smem smem_layout(int NS) {
    using T = Tc<D, ROWS>;
    Smem s{};
    auto al = [](size_t x, size_t a) { return (x + a - 1) / a * a; };
    size_t off = 0;
    s.ring = off;
    off += (size_t)NS * kChunkPages * T::PB;
    off = al(off, 128);
    s.wbuf = off;
    off += (size_t)T::NWB * T::WBYTES;
    // the CTA partial is written after the last chunk's value MMAs are complete: every
    // page copy has landed and every role is done with the ring, so it reuses the ring
    s.part = s.ring;
    if ((size_t)T::PART * 4 > (size_t)NS * kChunkPages * T::PB) return Smem{};   // does not fit: total = 0
    off = al(off, 128);
    s.qlimb = off;
    off += (size_t)T::NQ * D;
    off = al(off, 16);
    s.xch = off;                            // [3][ROWS][4 warps] chunk row maxima (2), row sums of p
    off += (size_t)3 * ROWS * 4 * 4;
    s.xsv = off;                            // [2][groups][4 warps] chunk V-scale maxima
    off += (size_t)2 * 2 * 4 * 4;
    s.crow = off;
    off += (size_t)ROWS * 4;
    s.lim = off;
    off += (size_t)ROWS * 4;
    s.pgbad = off;
    off += (size_t)NS * kChunkPages * 4;
    off = al(off, 8);
    s.mbar = off;
    off += (size_t)(2 * NS + 2 * T::NSB + T::NWB + T::NVB + T::NPB) * 8;
    s.misc = off;
    off += 64;
    s.total = al(off, 128);
    return s;
}

template <int ROWS>
struct AlphaRows {
    float a[ROWS];
    __device__ static AlphaRows make(const float (&x)[ROWS]) {
        AlphaRows r;
#pragma unroll
        for (int i = 0; i < ROWS; i++) r.a[i] = x[i];
        return r;
    }
};

// Multiplies this warp's 32 TMEM lanes of the value accumulators (NO columns from t_o)
// by the factor of each column's row (column j holds row j % ROWS), for the RPG rows
// from row rlo (a softmax warp group's rows; al holds their factors).  Out of line: it
// runs only when a running max moves.
template <int ROWS, int RPG, int NO>
__device__ __noinline__ void rescale_acc(uint32_t lane_base, int t_o, int rlo, AlphaRows<RPG> al) {
#pragma unroll 1
    for (int cb = 0; cb < NO / 8; cb++) {
        const int col = t_o + 8 * cb;
        const int r0 = (8 * cb) % ROWS - rlo;   // NO, ROWS and rlo are multiples of 8
        if (r0 < 0 || r0 >= RPG) continue;      // another group's rows
        uint32_t v[8];
        tmem_ld8(lane_base + (uint32_t)col, v);
        tmem_wait_ld();
#pragma unroll
        for (int e = 0; e < 8; e++) v[e] = __float_as_uint(__fmul_rn(__uint_as_float(v[e]), al.a[r0 + e]));
        tmem_st8(lane_base + (uint32_t)col, v);
    }
}

template <int D, int ROWS>
__global__ void __launch_bounds__(Tc<D, ROWS>::THREADS, Tc<D, ROWS>::CPS) decode_kernel(const DecodeParams p) {
    using T = Tc<D, ROWS>;
    extern __shared__ __align__(1024) uint8_t smem[];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int NS = p.stages;
    const Smem S = smem_layout<D, ROWS>(NS);
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
    float* part = reinterpret_cast<float*>(smem + S.part);
    float* crow_s = reinterpret_cast<float*>(smem + S.crow);
    int* lim_s = reinterpret_cast<int*>(smem + S.lim);
    int* pgbad = reinterpret_cast<int*>(smem + S.pgbad);
    const uint32_t bar0 = smem_u32(smem + S.mbar);
    auto full_b = [&](int s) { return bar0 + 8u * (uint32_t)s; };
    auto empty_b = [&](int s) { return bar0 + 8u * (uint32_t)(NS + s); };
    const uint32_t sfull_b = bar0 + 8u * (uint32_t)(2 * NS);   // [NSB] score buffer written
    const uint32_t sfree_b = sfull_b + 8 * T::NSB;             // [NSB] score buffer read
    const uint32_t wfull_b = sfree_b + 8 * T::NSB;             // [NWB] weights written
    const uint32_t vfull_b = wfull_b + 8 * T::NWB;             // [NVB] V^T written
    const uint32_t pvdone_b = vfull_b + 8 * T::NVB;            // [NPB] value MMAs of a chunk done
    // completion barrier of chunk j's value MMAs and the parity of that completion
    auto pv_bar = [&](int j) { return pvdone_b + 8u * (uint32_t)(j % T::NPB); };
    auto pv_par = [&](int j) { return (uint32_t)(j / T::NPB) & 1u; };

    // A bounded wait that the whole warp agrees on; a timeout raises the CTA's abort
    // flag (every role then stops taking new work) and the device error word.  The
    // softmax warps and the two MMA-issuing warps (the critical path) spin; the other
    // roles sleep in hardware while they wait, leaving the issue slots to the warps that
    // compute.  The fast path (already complete) is one test and a vote; the rest is
    // out of line, keeping the role loops small in the instruction cache.
    const bool spin_waits = warp >= 7 || warp == 1 || warp == 2;
    auto wait_warp = [&](uint32_t bar, uint32_t parity) -> bool {
        const bool done = mbar_test_wait(bar, parity);
        if (__all_sync(FULL, done)) return true;
        return wait_slow_warp(bar, parity, spin_waits, done, abort_flag, p.err);
    };
    // ---- set-up: barriers, query-row offset, TMEM, constant operands ----
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

    // ---- q -> three signed 8-bit limbs per row (the score MMA's B operand) ----
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

    if (warp == 0) {
        // ================= TMA producer =================
        // The kernel is a programmatic dependent launch: a preceding kernel that allows it
        // (the append of this step) may still be writing pages.  Wait for it to complete
        // before the first page is read; everything before this point reads only the
        // launch's inputs, which no such kernel writes.
        asm volatile("griddepcontrol.wait;" ::: "memory");
        const uint64_t policy = l2_evict_first_policy();
        // block-table entries of chunk i (lanes < 8), loaded one chunk ahead
        auto bt_load = [&](int i) -> int {
            const int lp = (c0 + i) * kChunkPages + lane;
            return (i < n_ck && lane < kChunkPages && lp < n_pages)
                       ? __ldg(p.block_table + (long long)b * p.max_blocks_per_seq + p.bt_col + lp)
                       : 0;
        };
        int blk_next = blk_first;
        int issued = 0;
        for (int i = 0; i < n_ck; i++) {
            const int s = i % NS;
            if (i >= NS && !wait_warp(empty_b(s), (uint32_t)((i - NS) / NS) & 1u)) break;
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
        }
        // after an abort: let copies still in flight land before the CTA leaves
        if (*abort_flag != 0 && lane == 0)
            for (int k = max(0, issued - NS); k < issued; k++) mbar_wait_bounded(full_b(k % NS), (uint32_t)(k / NS) & 1u);
    } else if (warp == 1) {
        // ================= score MMAs (whole warp; one elected lane issues) =================
        // The loop runs in step on all 32 lanes and every operand is computed the same way
        // on each, so that the MMAs issue back to back (a single-lane loop waits about two
        // hundred cycles per MMA).
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
            const int wb = j % T::NWB, vb = j % T::NVB;
            if (!wait_warp(wfull_b + 8 * wb, (uint32_t)(j / T::NWB) & 1u)) break;
            if (!wait_warp(vfull_b + 8 * vb, (uint32_t)(j / T::NVB) & 1u)) break;
            tc_fence_after();
            // descriptors of the chunk's weight buffer; each k-step adds a constant offset
            // (the 14-bit address field never carries: shared addresses stay below 2^18)
            const uint64_t dw = smem_desc(wb0 + (uint32_t)(wb * T::WBYTES), T::LBO_W, 128);
            const uint32_t vt = tmem + T::T_VT + vb * T::H * 64;
            const uint32_t acc0 = j > 0 ? 1u : 0u;
#pragma unroll
            for (int ks = 0; ks < kChunkTokens / 16; ks++) {
                const uint32_t acc = ks > 0 ? 1u : acc0;
                const uint64_t dk = dw + (uint64_t)((ks * 2 * T::LBO_W) >> 4);
#pragma unroll
                for (int h = 0; h < T::H; h++)
                    mma_f16_ts_w(tmem + T::T_O + h * T::NO, vt + h * 64 + 8 * ks,
                                 dk + (uint64_t)((h * 64 * ROWS) >> 4), IDO, acc);
            }
            tc_commit_w(pv_bar(j));
            last_bar = pv_bar(j);
            last_par = pv_par(j);
        }
        if (lane == 0 && *abort_flag != 0 && last_bar != 0) mbar_wait_bounded(last_bar, last_par);
        __syncwarp();
    } else if (warp < 7) {
        // ================= value codes -> V^T in tensor memory =================
        const int q = warp & 3;
        for (int i = 0; i < n_ck; i++) {
            const int s = i % NS, vb = i % T::NVB;
            if (!wait_warp(full_b(s), (uint32_t)(i / NS) & 1u)) break;
            if (i >= T::NVB && !wait_warp(pv_bar(i - T::NVB), pv_par(i - T::NVB)))
                break;
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
                            // tokens (2k, 2k+1) of the group: bits 4k..4k+3 and 16+4k..; flipping
                            // bit 3 turns the two's-complement code into u = code + 8, and the
                            // exponent bits 0x6400 make the fp16 value 1024 + u; subtracting
                            // 1032 leaves the code itself, exactly
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
        }
    } else {
        // ================= softmax and weights (one TMEM lane = one token) =================
        // warp 7 + 4 * sg + k: lane quadrant (warp & 3), rows r0g .. r0g + RPG - 1
        constexpr int RPG = T::RPG;
        // (with one group the group index is the constant 0, so the row offsets fold away)
        const int sw = warp - 7, sw4 = T::NSG == 1 ? sw : (sw & 3), sg = T::NSG == 1 ? 0 : (sw >> 2);
        const int q = warp & 3, t = 32 * q + lane;
        const int r0g = sg * RPG;
        const int tp = t / 16, ttg = (t / 8) & 1, tt = t & 7;
        const uint32_t wb0 = smem_u32(smem + S.wbuf);
        float* xch = reinterpret_cast<float*>(smem + S.xch);
        float* xsv = reinterpret_cast<float*>(smem + S.xsv);
        // Row factors and visibility limits: registers for the 8-row class, shared memory
        // (broadcast reads) for the larger ones, which would otherwise run out of registers.
        // Below, rows are indexed within the group (0 .. RPG - 1).
        constexpr bool kRowRegs = ROWS <= 8;
        float crow_r[kRowRegs ? RPG : 1], M[RPG];
        int lim_r[kRowRegs ? RPG : 1];
#pragma unroll
        for (int r = 0; r < RPG; r++) {
            if constexpr (kRowRegs) {
                crow_r[r] = crow_s[r0g + r];
                lim_r[r] = lim_s[r0g + r];
            }
            M[r] = -INFINITY;
        }
        auto crow = [&](int r) -> float {
            if constexpr (kRowRegs) return crow_r[r];
            else return crow_s[r0g + r];
        };
        auto lim = [&](int r) -> int {
            if constexpr (kRowRegs) return lim_r[r];
            else return lim_s[r0g + r];
        };
        float Mlane = -INFINITY;   // M of the group's row `lane` (lanes < RPG)
        const int lim_min = p.causal ? L - nq + row0 / p.group + 1 : L;   // smallest limit of the real rows
        const int rh = max(0, min(RPG, rows_here - r0g));                 // the group's real rows
        const int nrg4 = (rh + 3) / 4;                                    // 4-row groups holding real rows
        // A warp whose wait gave up keeps iterating without work, so that the four warps
        // of a group always meet at their named barrier the same number of times.
        bool ok = true;
        float lsum[RPG];   // this token's share of l = sum_t p_t, per row
#pragma unroll
        for (int r = 0; r < RPG; r++) lsum[r] = 0.0f;
        for (int i = 0; i < n_ck; i++) {
            const int s = i % NS, sb = i % T::NSB, wb = i % T::NWB;
            const int c = c0 + i;
            // this token's scales and page flags; then the stage is released
            float sk = 0.0f, sv[T::G];
            bool any_bad = false, my_bad = false;
            float z[RPG];
            if (ok && wait_warp(full_b(s), (uint32_t)(i / NS) & 1u)) {
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
            float* xs = xsv + (i & 1) * 8 + 4 * sg;
            if (ok) {
                tc_fence_after();
                // ---- scores of the real rows: the three limb accumulations -> fp32 ----
#pragma unroll
                for (int rg = 0; rg < RPG / 4; rg++) {
                    if (rg < nrg4) {
                        uint32_t a2[4], a1[4], a0[4];
                        const uint32_t col = T::T_S + sb * T::NQ + r0g + 4 * rg;
                        tmem_ld4(tmem_at(tmem, 32 * q, col), a2);
                        tmem_ld4(tmem_at(tmem, 32 * q, col + ROWS), a1);
                        tmem_ld4(tmem_at(tmem, 32 * q, col + 2 * ROWS), a0);
                        tmem_wait_ld();
#pragma unroll
                        for (int e = 0; e < 4; e++) {
                            const int x = (int)a2[e] * 256 + (int)a1[e];   // exact: |x| < 2^30
                            const float sc = __fmaf_rn((float)x, 256.0f, (float)(int)a0[e]);
                            z[4 * rg + e] = __fmul_rn(__fmul_rn(sc, crow(4 * rg + e)), sk);
                        }
                    } else {
#pragma unroll
                        for (int e = 0; e < 4; e++) z[4 * rg + e] = -INFINITY;
                    }
                }
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(sfree_b + 8 * sb);
                // ---- visibility: sequence end, causal drafts, unusable pages ----
                if (!clean) {
                    const int tok = c * kChunkTokens + t;
#pragma unroll
                    for (int r = 0; r < RPG; r++)
                        if (my_bad || tok >= lim(r)) z[r] = -INFINITY;
                }
                // ---- chunk row maxima over the 128 tokens, and the chunk's largest V scale
                // (tokens some row sees; a non-finite scale is outside the codec's domain and
                // is left out) ----
#pragma unroll
                for (int rg = 0; rg < RPG / 4; rg++)
                    if (rg < nrg4) {
#pragma unroll
                        for (int e = 0; e < 4; e++) {
                            const float m = warp_redux_max(z[4 * rg + e]);
                            if (lane == 0) xb[(r0g + 4 * rg + e) * 4 + sw4] = m;
                        }
                    }
                float svm = 0.0f;
                if (!my_bad && c * kChunkTokens + t < L) {
#pragma unroll
                    for (int g = 0; g < T::G; g++) svm = fmaxf(svm, sv[g]);
                }
                if (!(svm <= 65504.0f)) svm = 0.0f;
                svm = warp_redux_max(svm);
                if (lane == 0) xs[sw4] = svm;
            }
            named_bar_sync(2 + sg, 128);
            if (ok) {
                // ---- running max, moved lazily: only when a chunk max exceeds it by kLazy
                // (p <= 2^kLazy), or when a weight p * s_v could pass 2^15 (the fp16 weights
                // hold up to 65504): then it is raised to cm + log2(smax) - 15 ----
                bool need = false;
                float Mn = Mlane;
                if (lane < rh) {
                    const float4 v = *reinterpret_cast<const float4*>(xb + (r0g + lane) * 4);
                    const float4 w4 = *reinterpret_cast<const float4*>(xs);
                    const float cm = fmaxf(fmaxf(v.x, v.y), fmaxf(v.z, v.w));
                    const float smax = fmaxf(fmaxf(w4.x, w4.y), fmaxf(w4.z, w4.w));
                    // weights of the chunk are at most 2^(cm - M) * smax = 2^(cm - M + B + 15)
                    const float B = smax > 2048.0f ? __fsub_rn(log2f(smax), 15.0f) : -INFINITY;
                    need = cm > __fadd_rn(Mlane, kLazy) || Mlane < __fadd_rn(cm, B);
                    if (need) Mn = __fadd_rn(cm, fmaxf(B, 0.0f));
                }
                if (__any_sync(FULL, need)) {
                    const float al = (Mn == Mlane) ? 1.0f : ex2(__fsub_rn(Mlane, Mn));
                    Mlane = Mn;
                    float alpha[RPG];
#pragma unroll
                    for (int r = 0; r < RPG; r++) {
                        M[r] = __shfl_sync(FULL, Mn, r);
                        alpha[r] = __shfl_sync(FULL, al, r);
                        lsum[r] = __fmul_rn(lsum[r], alpha[r]);
                    }
                    // rescale O (this warp's 32 lanes, this group's rows) once the previous
                    // chunk's value MMAs are complete
                    if (i > 0 && wait_warp(pv_bar(i - 1), pv_par(i - 1))) {
                        tc_fence_after();
                        rescale_acc<ROWS, RPG, T::H * T::NO>(tmem_at(tmem, 32 * q, 0), T::T_O, r0g,
                                                             AlphaRows<RPG>::make(alpha));
                        tmem_wait_st();
                    } else if (i > 0) {
                        ok = false;
                    }
                }
            }
            if (ok && i >= T::NWB && !wait_warp(pv_bar(i - T::NWB), pv_par(i - T::NWB))) ok = false;
            if (ok) {
                // ---- weights of the real rows: p = 2^(z - M), W_g = p * s_v[g] (fp16), formed
                // 8 rows at a time next to their stores ----
                const uint32_t wrow = wb0 + (uint32_t)(wb * T::WBYTES + (t / 8) * T::LBO_W + (t % 8) * 16);
                auto store_group = [&](uint32_t a, const float* w, bool two) {
                    // 8 rows of one 8-column group (two = both 4-row halves hold real rows)
                    const uint32_t h0 = pack_h2(w[0], w[1]), h1 = pack_h2(w[2], w[3]);
                    if (two) {
                        stsa128(a, h0, h1, pack_h2(w[4], w[5]), pack_h2(w[6], w[7]));
                    } else {
                        asm volatile("st.shared.v2.u32 [%0], {%1,%2};" ::"r"(a), "r"(h0), "r"(h1) : "memory");
                    }
                };
#pragma unroll
                for (int rg8 = 0; rg8 < RPG / 8; rg8++) {
                    if (2 * rg8 >= nrg4) continue;
                    const bool two = 2 * rg8 + 1 < nrg4;
                    float pw[8];
#pragma unroll
                    for (int e = 0; e < 8; e++) {
                        const int r = 8 * rg8 + e;
                        pw[e] = (r >= rh || z[r] == -INFINITY) ? 0.0f : ex2(__fsub_rn(z[r], M[r]));
                        lsum[r] = __fadd_rn(lsum[r], pw[e]);
                    }
#pragma unroll
                    for (int g = 0; g < T::G; g++) {
                        float w[8];
#pragma unroll
                        for (int e = 0; e < 8; e++) {
                            const float pv = pw[e];
                            const float wv = __fmul_rn(pv, sv[g]);
                            // masked tokens may carry unwritten (non-finite) scales
                            w[e] = (!clean && pv == 0.0f) ? 0.0f : wv;
                        }
                        store_group(wrow + (uint32_t)(((g * ROWS + r0g + 8 * rg8) / 8) * 128), w, two);
                    }
                }
                fence_proxy_async_smem();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(wfull_b + 8 * wb);
            }
        }
        // ================= epilogue: the CTA partial in natural layout =================
        // l per row: the group's 128 tokens' shares, summed in a fixed order (warp
        // butterfly, then the four warps in index order)
        float* xl = xch + 2 * ROWS * 4;
#pragma unroll
        for (int r = 0; r < RPG; r++) {
            float v = lsum[r];
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) v = __fadd_rn(v, __shfl_xor_sync(FULL, v, o));
            if (lane == 0) xl[(r0g + r) * 4 + sw4] = v;
        }
        named_bar_sync(2 + sg, 128);
        if (ok) ok = wait_warp(pv_bar(n_ck - 1), pv_par(n_ck - 1));
        if (ok) {
            tc_fence_after();
#pragma unroll
            for (int h = 0; h < T::H; h++) {
                const int ch = 128 * h + 32 * q + lane;
#pragma unroll
                for (int rg = 0; rg < RPG / 8; rg++) {
                    uint32_t o[8];
                    tmem_ld8(tmem_at(tmem, 32 * q, T::T_O + h * T::NO + q * ROWS + r0g + 8 * rg), o);
                    tmem_wait_ld();
#pragma unroll
                    for (int e = 0; e < 8; e++) part[(r0g + 8 * rg + e) * D + ch] = __uint_as_float(o[e]);
                }
            }
            if (sw4 == 0 && lane < RPG) {
                const float4 v = *reinterpret_cast<const float4*>(xl + (r0g + lane) * 4);
                part[ROWS * D + ROWS + r0g + lane] = __fadd_rn(__fadd_rn(__fadd_rn(v.x, v.y), v.z), v.w);
            }
            if (sw4 == 0 && lane == 0) {
#pragma unroll
                for (int r = 0; r < RPG; r++) part[ROWS * D + r0g + r] = M[r];
            }
        }
        tc_fence_before();
    }

    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, T::TCOLS);
    }
    if (*abort_flag != 0) return;

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
    if (n_splits == 1) {
        finalize(part, part + ROWS * D, part + ROWS * D + ROWS);
        return;
    }
    // ---- publish this CTA's partial; merge_kernel completes the tree ----
    {
        float* go = p.part_o + (pidx * p.split_stride + sp) * (size_t)(ROWS * D);
        float* gml = p.part_ml + (pidx * p.split_stride + sp) * (size_t)(2 * ROWS);
        for (int i = threadIdx.x; i < ROWS * D / 4; i += blockDim.x)
            __stcg(reinterpret_cast<float4*>(go) + i, reinterpret_cast<const float4*>(part)[i]);
        for (int i = threadIdx.x; i < 2 * ROWS; i += blockDim.x) __stcg(gml + i, part[ROWS * D + i]);
    }
}

// Completes the fixed binary tree over the CTA partials of every (sequence, kv-head,
// row block) with more than one split, and writes out and lse.  Launched right after
// decode_kernel as a programmatic dependent launch: its CTAs may start while the decode
// CTAs finish, and wait (griddepcontrol.wait) until all of them have completed and
// their partials are visible.  One CTA covers 128 float4 elements of one unit's
// [ROWS][D] result; its threads are 128 x (leaf groups of 8 splits).  Thread (e, j)
// loads the 8 leaves of group j for element e (O, m, l) at once and evaluates that
// aligned level-3 subtree, coefficients included; the group results meet in shared
// memory, where thread (e, 0) evaluates the levels above.  Every node is
// merge(left, right) with merge_coef / merge_val, a node without a right child passes
// its left child through.
struct MergeOut {
    float4 o;
    float m, l;
};
// One tree node: merge(left, right), or the left child passed through.
__device__ __forceinline__ MergeOut merge_pair(float4 lo, float lm, float ll, float4 ro, float rm, float rl,
                                               bool has_right) {
    if (!has_right) return MergeOut{lo, lm, ll};
    float m, l, a, b;
    merge_coef(lm, ll, rm, rl, m, l, a, b);
    return MergeOut{make_float4(merge_val(lo.x, ro.x, a, b), merge_val(lo.y, ro.y, a, b), merge_val(lo.z, ro.z, a, b),
                                merge_val(lo.w, ro.w, a, b)),
                    m, l};
}

template <int D, int ROWS>
__global__ void __launch_bounds__(1024) merge_kernel(const DecodeParams p) {
    constexpr int E4 = ROWS * D / 4;   // float4 elements of one partial
    __shared__ float4 g_o[8][128];     // group results: O
    __shared__ float2 g_ml[8][128];    // group results: m, l
    // the sequence's bounds: inputs of the launch, readable before the decode grid ends
    const int b = blockIdx.z, hk = blockIdx.y / p.n_rb, rb = blockIdx.y % p.n_rb;
    const int L = seq_len_of(p, b), nq = seq_nq_of(p, b);
    const int e = threadIdx.x & 127, j = threadIdx.x >> 7;
    const int e4 = blockIdx.x * 128 + e;   // < E4: the grid covers E4 exactly
    const int r = (4 * e4) / D;            // the element's row
    const size_t pidx = ((size_t)(b * p.n_kv_heads + hk) * p.n_rb + rb);
    const float* gml0 = p.part_ml + pidx * p.split_stride * (size_t)(2 * ROWS);
    const float* go0 = p.part_o + pidx * p.split_stride * (size_t)(ROWS * D);
    // the next kernel on the stream may be scheduled now: a decode kernel there reads no
    // page and writes no partial before its own griddepcontrol.wait, which returns only
    // once this grid has completed
    if (threadIdx.x == 0) asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    asm volatile("griddepcontrol.wait;" ::: "memory");
    // the 8 leaves of this thread's group, loads in flight before the split count is
    // known (every slot below split_stride exists; unused ones are ignored below)
    float4 v[8];
    float vm[8], vl[8];
#pragma unroll
    for (int u = 0; u < 8; u++) {
        const int sidx = 8 * j + u;
        const bool slot = sidx < p.split_stride;
        v[u] = slot ? __ldcg(reinterpret_cast<const float4*>(go0 + (size_t)sidx * ROWS * D) + e4)
                    : make_float4(0.f, 0.f, 0.f, 0.f);
        vm[u] = slot ? __ldcg(gml0 + (size_t)sidx * 2 * ROWS + r) : -INFINITY;
        vl[u] = slot ? __ldcg(gml0 + (size_t)sidx * 2 * ROWS + ROWS + r) : 0.0f;
    }
    if (nq < 1 || nq > p.max_q || nq > L ||
        (long long)L + (long long)p.bt_col * kPageTokens > (long long)p.max_blocks_per_seq * kPageTokens)
        return;
    const int rows_b = p.group * nq, row0 = rb * ROWS;
    if (row0 >= rows_b) return;
    const int rows_here = min(ROWS, rows_b - row0);
    const int n_chunks = (L + kChunkTokens - 1) / kChunkTokens;
    const int n_splits = (n_chunks + p.cpc - 1) / p.cpc;
    if (n_splits <= 1) return;   // decode_kernel wrote this unit's output itself
    const int n_groups = (n_splits + 7) >> 3;
    int H = 0;
    while ((1 << H) < n_splits) H++;
    if (j < n_groups) {
        // levels 1..3 within the group
#pragma unroll
        for (int lv = 1; lv <= 3; lv++) {
#pragma unroll
            for (int u = 0; u < (8 >> lv); u++) {
                const int idx = ((8 * j) >> lv) + u;   // node (lv, idx)
                const bool has_right = (2 * idx + 1) * (1 << (lv - 1)) < n_splits;
                const MergeOut mo = merge_pair(v[2 * u], vm[2 * u], vl[2 * u], v[2 * u + 1], vm[2 * u + 1],
                                               vl[2 * u + 1], has_right);
                if (lv <= H) {
                    v[u] = mo.o;
                    vm[u] = mo.m;
                    vl[u] = mo.l;
                }
            }
        }
        g_o[j][e] = v[0];
        g_ml[j][e] = make_float2(vm[0], vl[0]);
    }
    __syncthreads();
    if (j != 0) return;
    // levels 4 .. H over the group results
    float4 gv[8];
    float gm[8], gl[8];
#pragma unroll
    for (int u = 0; u < 8; u++) {
        const bool here = u < n_groups;
        gv[u] = here ? g_o[u][e] : make_float4(0.f, 0.f, 0.f, 0.f);
        const float2 ml = here ? g_ml[u][e] : make_float2(-INFINITY, 0.0f);
        gm[u] = ml.x;
        gl[u] = ml.y;
    }
#pragma unroll
    for (int lv = 4; lv <= 6; lv++) {
#pragma unroll
        for (int u = 0; u < (64 >> lv); u++) {
            const bool has_right = (2 * u + 1) * (1 << (lv - 1)) < n_splits;
            const MergeOut mo = merge_pair(gv[2 * u], gm[2 * u], gl[2 * u], gv[2 * u + 1], gm[2 * u + 1], gl[2 * u + 1],
                                           has_right);
            if (lv <= H && u * (1 << lv) < n_splits) {
                gv[u] = mo.o;
                gm[u] = mo.m;
                gl[u] = mo.l;
            }
        }
    }
    // out = O / l and lse for a real row
    const int c4 = e4 % (D / 4);
    if (r >= rows_here) return;
    const int rr = row0 + r, jq = rr / p.group, hq = rr % p.group;
    int qoff = 0;
    for (int i = 0; i < b; i++) qoff += min(max(seq_nq_of(p, i), 0), p.max_q);
    const long long qrow = (long long)qoff + jq;
    if (qrow >= p.total_q) return;
    const float l = gl[0], m = gm[0];
    float4 o = gv[0];
    o.x = __fdiv_rn(o.x, l);
    o.y = __fdiv_rn(o.y, l);
    o.z = __fdiv_rn(o.z, l);
    o.w = __fdiv_rn(o.w, l);
    const size_t orow = (size_t)qrow * p.n_q_heads + (size_t)hk * p.group + hq;
    reinterpret_cast<float4*>(p.out + orow * D)[c4] = o;
    if (c4 == 0 && p.lse != nullptr) p.lse[orow] = __fmul_rn(__fadd_rn(m, log2f(l)), 0.69314718055994531f);
}

size_t decode_smem_bytes(int head_dim, int rows, int stages) {
    return small_smem_bytes(head_dim, rows, stages);
#define MQ_SMEM(DD, RR) \
    if (head_dim == DD && rows == RR) return smem_layout<DD, RR>(stages).total;
    MQ_SMEM(128, 16) MQ_SMEM(128, 32) MQ_SMEM(256, 16)
#undef MQ_SMEM
    return 0;
}

template <int D, int ROWS>
static cudaError_t set_smem(size_t smem) {
    cudaError_t e = cudaFuncSetAttribute(decode_kernel<D, ROWS>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    // all of the unified L1 / shared-memory array as shared memory, so that the classes
    // built for two CTAs per SM get both
    return cudaFuncSetAttribute(decode_kernel<D, ROWS>, cudaFuncAttributePreferredSharedMemoryCarveout, 100);
}

int decode_ctas_per_sm(int head_dim, int rows) {
    return small_ctas_per_sm(head_dim, rows);
}

cudaError_t decode_prepare(int head_dim, int rows, size_t smem) {
    return small_prepare(head_dim, rows, smem);
    if (head_dim == 128 && rows == 16) return set_smem<128, 16>(smem);
    if (head_dim == 128 && rows == 32) return set_smem<128, 32>(smem);
    if (head_dim == 256 && rows == 16) return set_smem<256, 16>(smem);
    return cudaErrorInvalidValue;
}

// merge_kernel as a programmatic dependent launch on the same stream (after a decode
// launch in which some unit has several splits).
template <int D, int ROWS>
static cudaError_t launch_merge(const DecodeParams& p, dim3 grid, int max_splits, cudaStream_t st) {
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = dim3((unsigned)((ROWS * D / 4 + 127) / 128), grid.y, grid.z);
    cfg.blockDim = dim3((unsigned)(128 * ((max_splits + 7) / 8)));
    cfg.dynamicSmemBytes = 0;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, merge_kernel<D, ROWS>, p);
}

// decode_kernel of the 16- and 32-row classes as a programmatic dependent launch
template <int D, int ROWS>
static cudaError_t launch_wide(const DecodeParams& p, dim3 grid, size_t smem, cudaStream_t st) {
    cudaLaunchAttribute pdl[1];
    pdl[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    pdl[0].val.programmaticStreamSerializationAllowed = 1;
    cudaLaunchConfig_t dc{};
    dc.gridDim = grid;
    dc.blockDim = dim3((unsigned)Tc<D, ROWS>::THREADS);
    dc.dynamicSmemBytes = smem;
    dc.stream = st;
    dc.attrs = pdl;
    dc.numAttrs = 1;
    return cudaLaunchKernelEx(&dc, decode_kernel<D, ROWS>, p);
}

// The decode kernel of the row class, then (when any unit has several splits) the merge.
cudaError_t launch_decode(const DecodeParams& p, int head_dim, int rows, int max_splits, size_t smem,
                          cudaStream_t st) {
    const dim3 grid((unsigned)max_splits, (unsigned)(p.n_kv_heads * p.n_rb), (unsigned)p.n_seqs);
    const cudaError_t e = small_launch(p, head_dim, rows, grid, smem, st);
    if (e != cudaSuccess || max_splits <= 1) return e;
#define MQ_MERGE(DD, RR) \
    if (head_dim == DD && rows == RR) return launch_merge<DD, RR>(p, grid, max_splits, st);
    MQ_MERGE(128, 4) MQ_MERGE(128, 8) MQ_MERGE(128, 16) MQ_MERGE(128, 32) MQ_MERGE(256, 4) MQ_MERGE(256, 8)
    MQ_MERGE(256, 16)
#undef MQ_MERGE
    return cudaErrorInvalidValue;
}

}  // namespace mq
