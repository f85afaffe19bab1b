// Prefill (prompt) attention over the K8/V4 paged cache on the sm_100a tensor cores.
//
// What it computes is the decode attention of mq_decode_small.cu for many query tokens at
// once: for query token j of sequence b (n_b queries, L_b cached tokens including the
// prompt's own, already appended) and q-head h,
//     z_t = scale * <q, s_k[t] * kcode_t>,  t = 0 .. L_b - n_b + j
//     out = sum_t softmax(z)_t * (s_v[t, group] * vcode_t),  lse = log sum_t exp z_t
// The blog.123qwe.co.kr deep dive on magnitudedev/magnitude (section 3, the first-load
// tuner) weighs 4k and 64k prompt prefill among the serving terms, and the stork.ai page
// quotes prefill rates; the cache and the codec are those of the decode path.
//
// How.  One CTA per (sequence, kv-head, tile of 128 query rows); a row is (query token,
// q-head of the kv-head's group), so the group's heads share every key/value chunk.
// Per 128-token chunk of the visible cache:
//  * warp 0 streams the chunk's 8 pages into a shared-memory ring (1-D bulk copies);
//  * warps 6-9 turn the int8 key codes into an fp16 operand (exact: 1024 + (code ^ 128)
//    in the fp16 bit pattern, minus 1152) and the int4 value codes into two fp16 value
//    operands hi + lo = code * s_v (hi the product rounded to fp16, lo the fp16 rounding
//    of the rest: about 22 significant bits), all laid out for the tensor cores;
//  * warp 1 issues S = Q K^T (kind::f16, M = 128 rows, N = 128 tokens; q held in fp16
//    scaled by a power of two per row, exact for bf16 and fp16 input) into tensor
//    memory, one chunk ahead, and O += P V_hi + P V_lo (A = P from tensor memory, N = D);
//  * warps 2-5 (thread = query row = TMEM lane) read S twice: the row maximum first,
//    then p = 2^(z - M) in fp16 into tensor memory, with a lazy running maximum M per
//    row (moved only when a chunk maximum exceeds it by more than 8 in log2 units, after
//    the thread rescales its own row of O) and the row sum l of the fp16 weights as the
//    MMAs see them, in fp32 (so that a dominant token's value comes out exactly).
// At the end each row thread writes out = O / l and lse.  Every wait is bounded.
#include "mq_decode_common.cuh"

namespace mq {

namespace {

constexpr int kPD = 128;                     // head_dim of this kernel
constexpr int kPRows = 128;                  // query rows per tile (MMA M)
constexpr int kPThreads = 320;               // 0 TMA, 1 MMA, 2-5 softmax, 6-9 conversion
constexpr int kPNS = 2;                      // ring stages (chunks of 8 pages)
constexpr int kPNK = 2;                      // fp16 key buffers
constexpr int kPNV = 1;                      // value buffers (each an fp16 pair hi + lo)
constexpr int kPNSB = 2;                     // score buffers (TMEM)
constexpr int kPNP = 2;                      // P buffers (TMEM)
constexpr float kPLazy = 8.0f;               // lazy-max threshold (log2 units): p <= 256
constexpr int kPOpBytes = kChunkTokens * kPD * 2;   // one fp16 operand tile (128 x 128)
// tensor memory: S buffers (128 fp32 columns each), O (D columns), P (64 columns)
constexpr int kPTS = 0;
constexpr int kPTO = kPNSB * 128;
constexpr int kPTP = kPTO + kPD;
static_assert(kPTP + kPNP * 64 <= 512, "tensor memory budget");

struct PrefillSmem {
    size_t ring, kbuf, vbuf, qtile, sk, crow, qlim, pgbad, mbar, misc, total;
};

__host__ __device__ inline PrefillSmem prefill_layout() {
    PrefillSmem s{};
    auto al = [](size_t x, size_t a) { return (x + a - 1) / a * a; };
    size_t off = 0;
    s.ring = off;
    off += (size_t)kPNS * kChunkPages * page_bytes(kPD);
    off = al(off, 128);
    s.kbuf = off;
    off += (size_t)kPNK * kPOpBytes;
    s.vbuf = off;                                 // [NV][hi, lo]
    off += (size_t)kPNV * 2 * kPOpBytes;
    s.qtile = off;
    off += (size_t)kPRows * kPD * 2;
    s.sk = off;                                   // [NK][128] fp32 key scales of the chunk
    off += (size_t)kPNK * kChunkTokens * 4;
    s.crow = off;                                 // [128] per-row score factor
    off += (size_t)kPRows * 4;
    s.qlim = off;                                 // [128] per-row last visible position
    off += (size_t)kPRows * 4;
    s.pgbad = off;
    off += (size_t)kPNS * kChunkPages * 4;
    off = al(off, 8);
    s.mbar = off;
    off += (size_t)(2 * kPNS + 2 * kPNK + 2 * kPNV + 2 * kPNSB + 2 * kPNP) * 8;
    s.misc = off;
    off += 64;
    s.total = al(off, 128);
    return s;
}

// Two signed 8-bit codes (bytes b0, b1 of x, selected by `sel`) as an exact fp16 pair:
// the bit pattern 0x6400 | (code ^ 128) is 1024 + code + 128; subtracting 1152 leaves
// the code.
__device__ __forceinline__ uint32_t i8_pair_to_h2(uint32_t xflip, uint32_t sel) {
    uint32_t d;
    asm("prmt.b32 %0, %1, %2, %3;" : "=r"(d) : "r"(xflip), "r"(0x64646464u), "r"(sel));
    return h2_as_u32(__hsub2(u32_as_h2(d), u32_as_h2(0x64806480u)));
}

}  // namespace

__global__ void __launch_bounds__(kPThreads, 1) prefill_kernel(const DecodeParams p) {
    extern __shared__ __align__(1024) uint8_t smem[];
    const PrefillSmem S = prefill_layout();
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int tile = blockIdx.x, hk = blockIdx.y, b = blockIdx.z;
    const int G = p.group, TQ = kPRows / G;   // query tokens per tile
    const unsigned FULL = 0xffffffffu;
    constexpr int PB = page_bytes(kPD), REC = rec_bytes(kPD);

    const int L = seq_len_of(p, b), nq = seq_nq_of(p, b);
    if (nq < 1 || nq > p.max_q || nq > L || (long long)L > (long long)p.max_blocks_per_seq * kPageTokens) {
        if (tile == 0 && hk == 0 && threadIdx.x == 0) atomicOr(p.err, kErrBadSeq);
        return;
    }
    const int j0 = tile * TQ;   // first query token of the tile
    if (j0 >= nq) return;
    const int tq_here = min(TQ, nq - j0);
    const int lim_lo = L - nq + j0;                // last visible position of the tile's first row
    const int lim_hi = L - nq + j0 + tq_here - 1;  // of its last real row
    const int n_ck = lim_hi / kChunkTokens + 1;    // chunks the tile sees
    const int n_pages_all = (L + kPageTokens - 1) / kPageTokens;

    int* misc = reinterpret_cast<int*>(smem + S.misc);   // 0 qoff, 1 abort, 3 TMEM base
    volatile int* abort_flag = misc + 1;
    float* sk_s = reinterpret_cast<float*>(smem + S.sk);
    float* crow_s = reinterpret_cast<float*>(smem + S.crow);
    int* qlim_s = reinterpret_cast<int*>(smem + S.qlim);
    int* pgbad = reinterpret_cast<int*>(smem + S.pgbad);
    const uint32_t bar0 = smem_u32(smem + S.mbar);
    auto full_b = [&](int s) { return bar0 + 8u * (uint32_t)s; };
    auto empty_b = [&](int s) { return bar0 + 8u * (uint32_t)(kPNS + s); };
    const uint32_t kfull_b = bar0 + 8u * (uint32_t)(2 * kPNS);   // [NK] fp16 keys written
    const uint32_t kfree_b = kfull_b + 8 * kPNK;                  // [NK] score MMAs done with them
    const uint32_t vfull_b = kfree_b + 8 * kPNK;                  // [NV] fp16 values written
    const uint32_t vfree_b = vfull_b + 8 * kPNV;                  // [NV] value MMAs done with them
    const uint32_t sfull_b = vfree_b + 8 * kPNV;                  // [NSB] scores written
    const uint32_t sfree_b = sfull_b + 8 * kPNSB;                 // [NSB] scores read
    const uint32_t pfull_b = sfree_b + 8 * kPNSB;                 // [NP] P written (and O rescaled)
    const uint32_t pvdone_b = pfull_b + 8 * kPNP;                 // [NP] value MMAs of a chunk done
    auto ph = [](int i, int n) { return (uint32_t)(i / n) & 1u; };

    auto wait_warp = [&](uint32_t bar, uint32_t parity) -> bool {
        const bool done = mbar_test_wait(bar, parity);
        if (__all_sync(FULL, done)) return true;
        return wait_slow_warp(bar, parity, false, done, abort_flag, p.err);
    };

    // ---- set-up ----
    if (threadIdx.x == 0) {
        for (int s = 0; s < kPNS; s++) {
            mbar_init(full_b(s), 1);
            mbar_init(empty_b(s), 4);   // the four conversion warps
        }
        for (int j = 0; j < kPNK; j++) {
            mbar_init(kfull_b + 8 * j, 4);
            mbar_init(kfree_b + 8 * j, 1);
        }
        for (int j = 0; j < kPNV; j++) {
            mbar_init(vfull_b + 8 * j, 4);
            mbar_init(vfree_b + 8 * j, 1);
        }
        for (int j = 0; j < kPNSB; j++) {
            mbar_init(sfull_b + 8 * j, 1);
            mbar_init(sfree_b + 8 * j, 4);
        }
        for (int j = 0; j < kPNP; j++) {
            mbar_init(pfull_b + 8 * j, 4);
            mbar_init(pvdone_b + 8 * j, 1);
        }
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
        tmem_alloc(smem_u32(misc + 3), 512);
        tmem_relinquish();
        tc_fence_before();
    }
    __syncthreads();
    const int qoff = misc[0];
    // ---- q -> fp16 tile (A operand, K-major: row r, channel c at (r/8)*2048 + (c/8)*128 +
    // (r%8)*16 + (c%8)*2), each row scaled by 2^(14 - E), |q| < 2^E over the row ----
    if (warp >= 2 && warp < 10) {
        const int tid = threadIdx.x - 64;   // 256 threads: two per row
        const int r = tid >> 1, half = tid & 1;
        const int jq = j0 + r / G, hq = r % G;
        const bool real = r < tq_here * G;
        const long long qrow = (long long)qoff + jq;
        const bool qok = real && qrow < p.total_q;
        if (real && !qok && half == 0) atomicOr(p.err, kErrBadRow);
        const size_t base = ((size_t)qrow * p.n_q_heads + (size_t)hk * G + hq) * kPD + (size_t)64 * half;
        float amax = 0.0f;
        for (int c = 0; c < 64; c++) amax = fmaxf(amax, fabsf(qok ? load_q(p, base + c) : 0.0f));
        amax = fmaxf(amax, __shfl_xor_sync(FULL, amax, 1));
        int E = 0;
        if (amax > 0.0f) frexpf(amax, &E);
        const bool zero_row = !(amax >= 0x1p-100f);
        const float up = zero_row ? 0.0f : ldexpf(1.0f, 14 - E);
        if (half == 0) {
            crow_s[r] = zero_row ? 0.0f : ldexpf(p.scale_log2, E - 14);
            qlim_s[r] = real ? L - nq + jq : -1;
        }
        uint8_t* qt = smem + S.qtile;
        for (int c8 = 0; c8 < 8; c8++) {
            const int c = 64 * half + 8 * c8;
            uint32_t w[4];
#pragma unroll
            for (int e = 0; e < 4; e++) {
                const float x0 = qok ? __fmul_rn(load_q(p, base + 8 * c8 + 2 * e), up) : 0.0f;
                const float x1 = qok ? __fmul_rn(load_q(p, base + 8 * c8 + 2 * e + 1), up) : 0.0f;
                w[e] = pack_h2(x0, x1);
            }
            stsa128(smem_u32(qt + (size_t)(r / 8) * 2048 + (c / 8) * 128 + (r % 8) * 16), w[0], w[1], w[2], w[3]);
        }
        fence_proxy_async_smem();
    }
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = (uint32_t)misc[3];
    const uint32_t ring = smem_u32(smem + S.ring);

    if (warp == 0) {
        // ================= TMA producer =================
        asm volatile("griddepcontrol.wait;" ::: "memory");
        const uint64_t policy = l2_evict_first_policy();
        int issued = 0;
        for (int i = 0; i < n_ck; i++) {
            const int s = i % kPNS;
            if (i >= kPNS && !wait_warp(empty_b(s), ph(i - kPNS, kPNS))) break;
            const int npg = min(kChunkPages, n_pages_all - i * kChunkPages);
            int blk = 0;
            bool bad = true;
            if (lane < npg) {
                blk = __ldg(p.block_table + (long long)b * p.max_blocks_per_seq + i * kChunkPages + lane);
                bad = blk < 0 || (long long)blk >= p.n_blocks;
                if (bad) {
                    atomicOr(p.err, kErrBadBlock);
                    blk = 0;
                }
            }
            if (lane < kChunkPages) pgbad[s * kChunkPages + lane] = bad ? 1 : 0;
            __syncwarp();
            if (lane == 0) mbar_arrive_expect_tx(full_b(s), (uint32_t)(npg * PB));
            __syncwarp();
            if (lane < npg)
                tma_load_1d(ring + (uint32_t)((s * kChunkPages + lane) * PB),
                            p.pool + ((long long)blk * p.n_kv_heads + hk) * PB, PB, full_b(s), policy);
            issued = i + 1;
        }
        if (*abort_flag != 0 && lane == 0)
            for (int k = max(0, issued - kPNS); k < issued; k++) mbar_wait_bounded(full_b(k % kPNS), ph(k, kPNS));
    } else if (warp == 1) {
        // ================= MMAs (whole warp; one elected lane issues) =================
        // S(i) = Q K(i)^T one chunk ahead of O += P(i - 1) V(i - 1)
        constexpr uint32_t IDS = instr_desc(1, 0, 0, 0, 0, 128, 128);   // f32 <- f16 x f16, both K-major
        constexpr uint32_t IDO = instr_desc(1, 0, 0, 0, 0, 128, kPD);   // A = P (TMEM), B = V K-major
        const uint64_t dq = smem_desc(smem_u32(smem + S.qtile), 128, 2048);
        const uint32_t kb0 = smem_u32(smem + S.kbuf), vb0 = smem_u32(smem + S.vbuf);
        uint32_t last_bar = 0, last_par = 0;
        bool ok = true;
        auto issue_qk = [&](int i) -> bool {
            const int kb = i % kPNK, sb = i % kPNSB;
            if (!wait_warp(kfull_b + 8 * kb, ph(i, kPNK))) return false;
            if (i >= kPNSB && !wait_warp(sfree_b + 8 * sb, ph(i - kPNSB, kPNSB))) return false;
            tc_fence_after();
            const uint64_t dk = smem_desc(kb0 + (uint32_t)(kb * kPOpBytes), 128, 2048);
            const uint32_t dst = tmem + kPTS + sb * 128;
#pragma unroll
            for (int k = 0; k < kPD / 16; k++) mma_f16_ss_w(dst, dq + 16 * k, dk + 16 * k, IDS, k > 0 ? 1u : 0u);
            tc_commit_w(sfull_b + 8 * sb);
            tc_commit_w(kfree_b + 8 * kb);
            return true;
        };
        auto issue_pv = [&](int i) -> bool {
            const int vb = i % kPNV, pb = i % kPNP;
            if (!wait_warp(pfull_b + 8 * pb, ph(i, kPNP))) return false;
            if (!wait_warp(vfull_b + 8 * vb, ph(i, kPNV))) return false;
            tc_fence_after();
            const uint64_t dv = smem_desc(vb0 + (uint32_t)(vb * 2 * kPOpBytes), 128, 2048);
            const uint64_t dvl = dv + (uint64_t)(kPOpBytes >> 4);   // the lo operand follows the hi one
            const uint32_t pa = tmem + kPTP + pb * 64;
#pragma unroll
            for (int k = 0; k < kChunkTokens / 16; k++)
                mma_f16_ts_w(tmem + kPTO, pa + 8 * k, dv + 16 * k, IDO, (i > 0 || k > 0) ? 1u : 0u);
#pragma unroll
            for (int k = 0; k < kChunkTokens / 16; k++) mma_f16_ts_w(tmem + kPTO, pa + 8 * k, dvl + 16 * k, IDO, 1u);
            tc_commit_w(pvdone_b + 8 * pb);
            tc_commit_w(vfree_b + 8 * vb);
            last_bar = pvdone_b + 8 * pb;
            last_par = ph(i, kPNP);
            return true;
        };
        if (n_ck > 0) ok = issue_qk(0);
        for (int i = 0; i < n_ck && ok; i++) {
            if (i + 1 < n_ck) ok = issue_qk(i + 1);
            if (ok) ok = issue_pv(i);
        }
        if (lane == 0 && *abort_flag != 0 && last_bar != 0) mbar_wait_bounded(last_bar, last_par);
        __syncwarp();
    } else if (warp >= 6) {
        // ================= key and value codes -> fp16 operands =================
        const int tid = threadIdx.x - 192;   // 128 threads
        const uint32_t kb0 = smem_u32(smem + S.kbuf), vb0 = smem_u32(smem + S.vbuf);
        for (int i = 0; i < n_ck; i++) {
            const int s = i % kPNS, kb = i % kPNK, vb = i % kPNV;
            if (!wait_warp(full_b(s), ph(i, kPNS))) break;
            if (i >= kPNK && !wait_warp(kfree_b + 8 * kb, ph(i - kPNK, kPNK))) break;
            const uint32_t st = ring + (uint32_t)(s * kChunkPages * PB);
            // keys: token t (0..127) of the chunk, channels 16u .. 16u + 15 -> B operand
            // (N = tokens, K = channels): (t/8)*2048 + (c/8)*128 + (t%8)*16 + (c%8)*2
            for (int it = tid; it < kChunkTokens * kPD / 16; it += 128) {
                const int t = it / (kPD / 16), u = it % (kPD / 16);
                const uint32_t src = st + (uint32_t)((t / 16) * PB + ((t / 8) & 1) * REC + u * 128 + (t % 8) * 16);
                const uint4 w = ldsa128(src);
                const uint32_t x[4] = {w.x ^ 0x80808080u, w.y ^ 0x80808080u, w.z ^ 0x80808080u, w.w ^ 0x80808080u};
                const uint32_t dst = kb0 + (uint32_t)(kb * kPOpBytes + (t / 8) * 2048 + (2 * u) * 128 + (t % 8) * 16);
                stsa128(dst, i8_pair_to_h2(x[0], 0x5140u), i8_pair_to_h2(x[0], 0x5342u), i8_pair_to_h2(x[1], 0x5140u),
                        i8_pair_to_h2(x[1], 0x5342u));
                stsa128(dst + 128, i8_pair_to_h2(x[2], 0x5140u), i8_pair_to_h2(x[2], 0x5342u),
                        i8_pair_to_h2(x[3], 0x5140u), i8_pair_to_h2(x[3], 0x5342u));
            }
            // key scales (fp32) for the softmax; tokens of unusable pages get -inf
            {
                const int t = tid;
                const uint32_t rec = st + (uint32_t)((t / 16) * PB + ((t / 8) & 1) * REC);
                const bool bad = pgbad[s * kChunkPages + t / 16] != 0;
                sk_s[kb * kChunkTokens + t] = bad ? __int_as_float(0x7fc00000) : h_bits_to_f32(ldsa16(rec + rec_ks_off(kPD) + 2 * (t % 8)));
            }
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) mbar_arrive(kfull_b + 8 * kb);
            // the value buffer is free once the value MMAs of chunk i - NV are complete; waited
            // for only now, after the keys: the score MMAs of chunk i come before those value
            // MMAs in the MMA warp's order
            if (i >= kPNV && !wait_warp(vfree_b + 8 * vb, ph(i - kPNV, kPNV))) break;
            // values: channel c, 8-token record g (tokens 8g .. 8g + 7) -> B operand
            // (K = tokens, N = channels): (c/8)*2048 + (t/8)*128 + (c%8)*16 + (t%8)*2
            for (int it = tid; it < kPD * (kChunkTokens / 8); it += 128) {
                const int c = it % kPD, g8 = it / kPD;   // consecutive threads: consecutive channels
                const uint32_t rec = st + (uint32_t)((g8 / 2) * PB + (g8 & 1) * REC);
                // positions past the sequence and unusable pages hold no values: zeros, so
                // that a NaN or infinite unwritten scale cannot reach O through p = 0
                const int pos0 = i * kChunkTokens + 8 * g8;
                const bool rec_ok = pgbad[s * kChunkPages + g8 / 2] == 0 && pos0 < L;
                const uint32_t w = ldsa32(rec + rec_v_off(kPD) + 4 * c);
                const uint32_t vs = rec + rec_vs_off(kPD) + 2 * (c / 32);
                uint32_t h[4], lo[4];
#pragma unroll
                for (int k = 0; k < 4; k++) {
                    // tokens 2k, 2k + 1 of the record: code * s_v in fp32 (exact: 4 + 11
                    // significant bits), its fp16 rounding hi, and the fp16 rounding of the rest
                    const float2 cf = __half22float2(u32_as_h2(code_pair(w >> (4 * k))));
                    const float s0 = h_bits_to_f32(ldsa16(vs + (uint32_t)(2 * k * (kPD / 32) * 2)));
                    const float s1 = h_bits_to_f32(ldsa16(vs + (uint32_t)((2 * k + 1) * (kPD / 32) * 2)));
                    const float x0 = __fmul_rn(cf.x, s0), x1 = __fmul_rn(cf.y, s1);
                    const __half2 hh = __floats2half2_rn(x0, x1);
                    const float2 hf = __half22float2(hh);
                    const __half2 ll = __floats2half2_rn(__fsub_rn(x0, hf.x), __fsub_rn(x1, hf.y));
                    const uint32_t keep = (rec_ok && pos0 + 2 * k < L ? 0x0000FFFFu : 0u) |
                                          (rec_ok && pos0 + 2 * k + 1 < L ? 0xFFFF0000u : 0u);
                    h[k] = h2_as_u32(hh) & keep;
                    lo[k] = h2_as_u32(ll) & keep;
                }
                const uint32_t vdst = vb0 + (uint32_t)(vb * 2 * kPOpBytes + (c / 8) * 2048 + g8 * 128 + (c % 8) * 16);
                stsa128(vdst, h[0], h[1], h[2], h[3]);
                stsa128(vdst + kPOpBytes, lo[0], lo[1], lo[2], lo[3]);
            }
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) {
                mbar_arrive(vfull_b + 8 * vb);
                mbar_arrive(empty_b(s));
            }
        }
    } else {
        // ================= softmax: thread = query row = TMEM lane =================
        const int q = warp & 3, r = 32 * q + lane;
        const float crow = crow_s[r];
        const int lim = qlim_s[r];   // last visible position (-1: not a real row)
        const uint32_t lrow = tmem_at(tmem, 32 * q, 0);
        float M = -INFINITY, l = 0.0f;
        bool ok = true;
        for (int i = 0; i < n_ck; i++) {
            const int sb = i % kPNSB, kb = i % kPNK, pb = i % kPNP;
            const bool clean = (i + 1) * kChunkTokens - 1 <= lim_lo;   // every row sees the whole chunk
            if (ok && !wait_warp(sfull_b + 8 * sb, ph(i, kPNSB))) ok = false;
            const float* skc = sk_s + kb * kChunkTokens;
            // pass 1: the chunk's row maximum
            float cm = -INFINITY;
            if (ok) {
                tc_fence_after();
#pragma unroll 1
                for (int cb = 0; cb < 4; cb++) {
                    uint32_t v[32];
                    tmem_ld32(lrow + (uint32_t)(kPTS + sb * 128 + 32 * cb), v);
                    tmem_wait_ld();
#pragma unroll
                    for (int e = 0; e < 32; e++) {
                        const int t = 32 * cb + e;
                        float z = __fmul_rn(__fmul_rn(__uint_as_float(v[e]), crow), skc[t]);
                        if ((!clean && i * kChunkTokens + t > lim) || !(z == z)) z = -INFINITY;
                        cm = fmaxf(cm, z);
                    }
                }
            }
            // lazy running maximum; a move rescales this row of O and l once the previous
            // chunk's value MMAs are complete
            // (TMEM loads and stores are warp-collective: every lane of the warp executes
            // them, with factor 1 on the rows whose maximum stays)
            const bool need = ok && cm > __fadd_rn(M, kPLazy);
            if (__any_sync(FULL, need)) {
                if (i > 0 && !wait_warp(pvdone_b + 8 * ((i - 1) % kPNP), ph(i - 1, kPNP))) ok = false;
                if (ok) {
                    tc_fence_after();
                    float al = 1.0f;
                    if (need) {
                        al = ex2(__fsub_rn(M, cm));
                        l = __fmul_rn(l, al);
                        M = cm;
                    }
                    if (i > 0) {
#pragma unroll 1
                        for (int cb = 0; cb < kPD / 32; cb++) {
                            uint32_t v[32];
                            tmem_ld32(lrow + (uint32_t)(kPTO + 32 * cb), v);
                            tmem_wait_ld();
#pragma unroll
                            for (int e = 0; e < 32; e++) v[e] = __float_as_uint(__fmul_rn(__uint_as_float(v[e]), al));
                            tmem_st32(lrow + (uint32_t)(kPTO + 32 * cb), v);
                        }
                        tmem_wait_st();
                    }
                }
            }
            // the P buffer is free once the previous chunk's value MMAs are complete
            if (ok && i >= kPNP && !wait_warp(pvdone_b + 8 * pb, ph(i - kPNP, kPNP))) ok = false;
            // pass 2: p = 2^(z - M) in fp16 -> P (TMEM), and l
            if (ok) {
#pragma unroll 1
                for (int cb = 0; cb < 4; cb++) {
                    uint32_t v[32], ph16[16];
                    tmem_ld32(lrow + (uint32_t)(kPTS + sb * 128 + 32 * cb), v);
                    tmem_wait_ld();
#pragma unroll
                    for (int e = 0; e < 32; e += 2) {
                        float pp[2];
#pragma unroll
                        for (int u = 0; u < 2; u++) {
                            const int t = 32 * cb + e + u;
                            const float z = __fmul_rn(__fmul_rn(__uint_as_float(v[e + u]), crow), skc[t]);
                            const bool vis = (clean || i * kChunkTokens + t <= lim) && z == z;
                            pp[u] = vis ? ex2(__fsub_rn(z, M)) : 0.0f;
                        }
                        const __half2 hp = __floats2half2_rn(pp[0], pp[1]);
                        const float2 pr = __half22float2(hp);   // the weights the MMAs see
                        l = __fadd_rn(__fadd_rn(l, pr.x), pr.y);
                        ph16[e / 2] = h2_as_u32(hp);
                    }
                    tmem_st16(lrow + (uint32_t)(kPTP + pb * 64 + 16 * cb), ph16);
                }
                tmem_wait_st();
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) {
                mbar_arrive(sfree_b + 8 * sb);
                mbar_arrive(pfull_b + 8 * pb);
            }
        }
        // ---- epilogue: out = O / l, lse ----
        if (ok && n_ck > 0) ok = wait_warp(pvdone_b + 8 * ((n_ck - 1) % kPNP), ph(n_ck - 1, kPNP));
        tc_fence_after();
        if (ok && *abort_flag == 0) {   // warp-uniform: the TMEM loads are warp-collective
            const int jq = j0 + r / G, hq = r % G;
            const long long qrow = (long long)qoff + jq;
            const bool write = lim >= 0 && qrow < p.total_q;   // a real row of this tile
            float* orow = p.out + ((size_t)(write ? qrow : 0) * p.n_q_heads + (size_t)hk * G + hq) * kPD;
#pragma unroll 1
            for (int cb = 0; cb < kPD / 32; cb++) {
                uint32_t v[32];
                tmem_ld32(lrow + (uint32_t)(kPTO + 32 * cb), v);
                tmem_wait_ld();
                if (write) {
#pragma unroll
                    for (int e = 0; e < 32; e += 4)
                        *reinterpret_cast<float4*>(orow + 32 * cb + e) =
                            make_float4(__fdiv_rn(__uint_as_float(v[e]), l), __fdiv_rn(__uint_as_float(v[e + 1]), l),
                                        __fdiv_rn(__uint_as_float(v[e + 2]), l), __fdiv_rn(__uint_as_float(v[e + 3]), l));
                }
            }
            if (write && p.lse != nullptr)
                p.lse[(size_t)qrow * p.n_q_heads + (size_t)hk * G + hq] =
                    __fmul_rn(__fadd_rn(M, log2f(l)), 0.69314718055994531f);
        }
        tc_fence_before();
    }
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, 512);
    }
}

size_t prefill_smem_bytes() { return prefill_layout().total; }

cudaError_t launch_prefill(const DecodeParams& p, int max_tiles, cudaStream_t st) {
    static bool attr_set[64] = {};
    int dev = 0;
    cudaGetDevice(&dev);
    const size_t smem = prefill_smem_bytes();
    if (!attr_set[dev & 63]) {
        cudaError_t e = cudaFuncSetAttribute(prefill_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
        attr_set[dev & 63] = true;
    }
    cudaLaunchAttribute pdl[1];
    pdl[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    pdl[0].val.programmaticStreamSerializationAllowed = 1;
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = dim3((unsigned)max_tiles, (unsigned)p.n_kv_heads, (unsigned)p.n_seqs);
    cfg.blockDim = dim3(kPThreads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cfg.attrs = pdl;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, prefill_kernel, p);
}

}  // namespace mq
