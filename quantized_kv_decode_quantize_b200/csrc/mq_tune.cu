// mq_tune: on-device choice of the decode launch configuration.
//
// Follows the first-load tuner of the blog.123qwe.co.kr deep dive on
// magnitudedev/magnitude, section 3 ("core mechanism 1: the 60 s first-load
// tuner"): one wall-clock budget covers everything (probe set-up, every launch,
// every comparison); candidates are measured on the device over serving shapes
// (decode at 4k and 64k history, and a speculative step: one drafter launch, then the
// verification of 8 drafts), and the cost of a configuration c is
//     cost(c) = sum_p weight(p) * median_time(c, p),
//     weight(p) = sum_t term_weight(t) * launches(t, p) / time_at_defaults(t)
// over the terms t = decode_4k, decode_64k, draft_64k (mq_draft_ngram over a 64K-token
// history), verify8_64k, and the 4k and 64k prompt prefill (mq_prefill_attn), each of
// weight 1 (the speculative-step probe holds one launch of each of its two terms).  No
// candidate changes how the drafter or the prefill launch, so their terms are measured
// once at the defaults and enter every candidate's cost at that time; timing passes
// read data sized beyond the
// last-level cache (here: rotating probe caches that together exceed twice the L2
// size), so no launch finds its data warm; structurally different candidates are
// tried before refinements of one; a candidate is started only when the budget
// left covers its estimated cost; a completed search is stored and reused by the
// next load with the same device, driver, toolchain and library identity
// (mq_tune_store.cu).
//
// Admission, by default, follows the paper-digest.app summary ("Core Mechanics":
// only configurations that do not change the output are kept): a candidate's out
// and lse bytes must equal the default's exactly.  On request it follows the
// deep dive's section 4 ("core mechanism 2: the precision system") instead, with
// alpha = 8: at every checked point the candidate may move the default's result by
// at most alpha times what storage-resolution noise moves it, that noise being the
// movement of the default output when every stored element of the probe cache
// takes one step of its format (the larger of two seeded perturbations).
#include <algorithm>
#include <chrono>
#include <cstdio>
#include <cstring>
#include <string>
#include <vector>

#include "mq.h"
#include "mq_device.cuh"
#include "mq_host.h"
#include "mq_kernels.h"

namespace mq {
namespace {

using Clock = std::chrono::steady_clock;

struct Probe {
    const char* name;
    int seq_len, n_q, cls;
    bool with_draft;        // a drafter launch precedes the decode launch
    double t_default = 0;   // median seconds at the default configuration
    double weight = 0;      // sum over its terms of launches / time_at_defaults (1/s)
};

struct Cand {
    mq_decode_config cfg;
    int cls;
    double t[3] = {0, 0, 0};
    double max_ratio = 0;   // largest |candidate - default| / noise over checked points (alpha rule)
    bool identical = true, measured = false, rejected = false, valid = true;
};

// summary of one probe's storage-resolution noise over its out points
struct NoiseStats {
    double min = 0, median = 0, max = 0;
    long long zero_points = 0;
};

void json_double(FILE* f, double v) {
    if (v != v) std::fprintf(f, "NaN");
    else if (v > 1e300) std::fprintf(f, "Infinity");
    else std::fprintf(f, "%.6g", v);
}

double seconds_since(Clock::time_point t0) {
    return std::chrono::duration<double>(Clock::now() - t0).count();
}

struct Buffers {
    void* pool = nullptr;
    int32_t* bt = nullptr;       // [n_copies][blocks_per_copy]
    int32_t* lens = nullptr;     // one per probe
    int32_t* nq = nullptr;
    int32_t* cu = nullptr;
    int32_t* start = nullptr;
    int32_t* tokens = nullptr;   // the drafter's 64K-token history
    void* q_pf = nullptr;        // prefill probes: q of a 64K-token prompt, and its out
    float* out_pf = nullptr;
    int32_t* pf_lens = nullptr;  // [2]: 4096, 65536
    int32_t* drafts = nullptr;
    int32_t* n_drafts = nullptr;
    void* kv = nullptr;          // staging for K and V
    void* q = nullptr;
    float* out_ref[3] = {nullptr, nullptr, nullptr};
    float* lse_ref[3] = {nullptr, nullptr, nullptr};
    float* out = nullptr;
    float* lse = nullptr;
    void* ws = nullptr;
    unsigned* flag = nullptr;    // [0] bytes differ, [1] alpha rule broken, [2] max ratio (float bits)
    void* pert = nullptr;        // one perturbed probe cache copy (alpha rule)
    float* noise_out[3] = {nullptr, nullptr, nullptr};
    float* noise_lse[3] = {nullptr, nullptr, nullptr};
    cudaEvent_t ev[2] = {nullptr, nullptr};
    cudaStream_t st = nullptr;
    ~Buffers() {
        void* ptrs[] = {pool, bt, lens, nq, cu, start, tokens, drafts, n_drafts, q_pf, out_pf, pf_lens, kv, q, out, lse,
                        ws, flag, pert,
                        out_ref[0], out_ref[1], out_ref[2], lse_ref[0], lse_ref[1], lse_ref[2],
                        noise_out[0], noise_out[1], noise_out[2], noise_lse[0], noise_lse[1], noise_lse[2]};
        for (void* p : ptrs)
            if (p) cudaFree(p);
        for (auto e : ev)
            if (e) cudaEventDestroy(e);
        if (st) cudaStreamDestroy(st);
    }
};

}  // namespace
}  // namespace mq

using namespace mq;

extern "C" mq_status mq_tune(mq_cache* cache, const mq_tune_params* prm, mq_tune_result* res) {
    const auto t0 = Clock::now();
    if (cache == nullptr || prm == nullptr || res == nullptr) return MQ_ERR_INVALID_ARG;
    if (!(prm->budget_s >= 0.0) || prm->n_q_heads < 1 || prm->n_q_heads % cache->n_kv_heads != 0)
        return MQ_ERR_INVALID_ARG;
    if (prm->admission != MQ_ADMIT_BIT_IDENTICAL && prm->admission != MQ_ADMIT_ALPHA) return MQ_ERR_INVALID_ARG;
    if (!(prm->alpha <= 0.0 || prm->alpha < 1e30)) return MQ_ERR_INVALID_ARG;   // NaN or absurd alpha
    const bool alpha_rule = prm->admission == MQ_ADMIT_ALPHA;
    const double alpha = prm->alpha > 0.0 ? prm->alpha : 8.0;
    const int Hkv = cache->n_kv_heads, D = cache->head_dim, Hq = prm->n_q_heads, G = Hq / Hkv;
    if (G > 64) return MQ_ERR_UNSUPPORTED;
    *res = mq_tune_result{};
    for (int k = 0; k < 3; k++) res->chosen[k] = cache->cfg[k];
    res->cost = 1.0;

    // ---- the store: a stored choice for this identity is applied without measuring ----
    char identity[512] = {0};
    if (prm->store_path != nullptr) {
        mq_status s = mq_tune_identity(cache, prm, identity, sizeof identity);
        if (s != MQ_OK) return s;
        mq_decode_config got[3];
        int32_t found = 0;
        if ((s = mq_tune_store_get(prm->store_path, identity, got, &found)) != MQ_OK) return s;
        if (found) {
            for (int k = 0; k < 3; k++) cache->cfg[k] = res->chosen[k] = got[k];
            res->from_store = 1;
            res->elapsed_s = seconds_since(t0);
            if (prm->log_path != nullptr) {
                FILE* f = std::fopen(prm->log_path, "w");
                if (f != nullptr) {
                    std::fprintf(f, "{\n  \"from_store\": true, \"identity\": \"%s\", \"elapsed_s\": %.6f,\n", identity,
                                 res->elapsed_s);
                    std::fprintf(f, "  \"chosen\": [");
                    for (int cls = 0; cls < 3; cls++)
                        std::fprintf(f,
                                     "%s{\"rows_class\": %d, \"ring_stages\": %d, \"splits_per_sm\": %d, "
                                     "\"softmax_warps\": %d}",
                                     cls ? ", " : "", cls, got[cls].ring_stages, got[cls].splits_per_sm,
                                     got[cls].softmax_warps);
                    std::fprintf(f, "],\n  \"n_tried\": 0\n}\n");
                    std::fclose(f);
                }
            }
            return MQ_OK;
        }
    }

    if (prm->budget_s < 0.5) {   // not even the probe set-up fits: keep the defaults
        res->elapsed_s = seconds_since(t0);
        return MQ_TUNE_BUDGET_EXHAUSTED;
    }
    DevGuard guard(cache->device);

    std::vector<Probe> probes = {{"decode_4k", 4096, 1, rows_class_for(D, G), false},
                                 {"decode_64k", 65536, 1, rows_class_for(D, G), false}};
    if (G * 8 <= 64) probes.push_back({"draft_verify8_64k", 65544, 8, rows_class_for(D, G * 8), true});
    const int P = (int)probes.size();
    constexpr int kDraftLen = 65536, kDraftN = 4, kDraftK = 8;   // drafter term: history, n-gram, drafts

    // ---- probe caches: enough rotating copies to exceed 2x L2 ----
    int l2 = 0;
    cudaDeviceGetAttribute(&l2, cudaDevAttrL2CacheSize, cache->device);
    const int max_len = 65544;
    const int blocks_per_copy = (max_len + MQ_PAGE_TOKENS - 1) / MQ_PAGE_TOKENS;
    const size_t copy_bytes = (size_t)blocks_per_copy * Hkv * page_bytes(D);
    int n_copies = (int)std::min<size_t>(64, std::max<size_t>(2, (size_t)(2.0 * l2 / copy_bytes) + 1));
    Buffers B;
    auto ck = [](cudaError_t e) { return e == cudaSuccess; };
    if (!ck(cudaStreamCreateWithFlags(&B.st, cudaStreamNonBlocking)) || !ck(cudaEventCreate(&B.ev[0])) ||
        !ck(cudaEventCreate(&B.ev[1])))
        return MQ_ERR_CUDA;
    size_t ws_bytes = 0;
    for (auto& pr : probes) ws_bytes = std::max(ws_bytes, mq_decode_workspace_bytes(cache, 1, Hq, pr.n_q, pr.seq_len));
    const size_t kv_elems = (size_t)max_len * Hkv * D;
    if (!ck(cudaMalloc(&B.pool, copy_bytes * n_copies)) ||
        !ck(cudaMalloc(&B.bt, sizeof(int32_t) * blocks_per_copy * n_copies)) ||
        !ck(cudaMalloc(&B.lens, sizeof(int32_t) * 4)) || !ck(cudaMalloc(&B.nq, sizeof(int32_t) * 4)) ||
        !ck(cudaMalloc(&B.cu, sizeof(int32_t) * 2)) || !ck(cudaMalloc(&B.start, sizeof(int32_t))) ||
        !ck(cudaMalloc(&B.kv, kv_elems * 2 * 2)) || !ck(cudaMalloc(&B.q, (size_t)8 * Hq * D * 2)) ||
        !ck(cudaMalloc(&B.out, (size_t)8 * Hq * D * 4)) || !ck(cudaMalloc(&B.lse, (size_t)8 * Hq * 4)) ||
        !ck(cudaMalloc(&B.ws, ws_bytes)) || !ck(cudaMalloc(&B.flag, 3 * sizeof(unsigned))) ||
        !ck(cudaMalloc(&B.tokens, sizeof(int32_t) * (kDraftLen + 1))) ||
        !ck(cudaMalloc(&B.drafts, sizeof(int32_t) * kDraftK)) || !ck(cudaMalloc(&B.n_drafts, sizeof(int32_t))))
        return MQ_ERR_CUDA;
    for (int p = 0; p < P; p++)
        if (!ck(cudaMalloc(&B.out_ref[p], (size_t)8 * Hq * D * 4)) || !ck(cudaMalloc(&B.lse_ref[p], (size_t)8 * Hq * 4)))
            return MQ_ERR_CUDA;
    if (!ck(cudaMemsetAsync(B.ws, 0, ws_bytes, B.st))) return MQ_ERR_CUDA;
    {
        std::vector<int32_t> bt((size_t)blocks_per_copy * n_copies);
        for (size_t i = 0; i < bt.size(); i++) bt[i] = (int32_t)i;
        int32_t h[6] = {0, max_len, 0, 0, 0, 0};
        if (!ck(cudaMemcpy(B.bt, bt.data(), sizeof(int32_t) * bt.size(), cudaMemcpyHostToDevice)) ||
            !ck(cudaMemcpy(B.cu, h, sizeof(int32_t) * 2, cudaMemcpyHostToDevice)) ||
            !ck(cudaMemcpy(B.start, h + 2, sizeof(int32_t), cudaMemcpyHostToDevice)))
            return MQ_ERR_CUDA;
        int32_t lens[4], nq[4];
        for (int p = 0; p < P; p++) {
            lens[p] = probes[p].seq_len;
            nq[p] = probes[p].n_q;
        }
        if (!ck(cudaMemcpy(B.lens, lens, sizeof(int32_t) * P, cudaMemcpyHostToDevice)) ||
            !ck(cudaMemcpy(B.nq, nq, sizeof(int32_t) * P, cudaMemcpyHostToDevice)))
            return MQ_ERR_CUDA;
        // the drafter's history: a token stream with repeats (a 4093-token cycle with a
        // few edits), and its length at the end of the buffer
        std::vector<int32_t> tok(kDraftLen + 1);
        for (int i = 0; i < kDraftLen; i++) tok[i] = (int32_t)((i % 4093) * 7 % 32000 + (i % 9973 == 0 ? 1 : 0));
        tok[kDraftLen] = kDraftLen;
        if (!ck(cudaMemcpy(B.tokens, tok.data(), sizeof(int32_t) * tok.size(), cudaMemcpyHostToDevice)))
            return MQ_ERR_CUDA;
    }
    // random K/V for one copy, quantized by the append kernel, then replicated
    mq_cache probe_cache = *cache;
    probe_cache.pool = B.pool;
    probe_cache.pool_bytes = copy_bytes * n_copies;
    probe_cache.n_blocks = (int64_t)blocks_per_copy * n_copies;
    {
        void* kbuf = B.kv;
        void* vbuf = static_cast<uint8_t*>(B.kv) + kv_elems * 2;
        if (!ck(launch_fill_random(kbuf, 1, (long long)kv_elems, D, 0x6B65ull, B.st)) ||
            !ck(launch_fill_random(vbuf, 1, (long long)kv_elems, D, 0x7631ull, B.st)) ||
            !ck(launch_fill_random(B.q, 1, (long long)8 * Hq * D, D, 0x7131ull, B.st)))
            return MQ_ERR_CUDA;
        AppendParams ap{};
        ap.pool = static_cast<uint8_t*>(B.pool);
        ap.n_kv_heads = Hkv;
        ap.n_blocks = probe_cache.n_blocks;
        ap.k = kbuf;
        ap.v = vbuf;
        ap.dtype = 1;
        ap.n_seqs = 1;
        ap.n_tokens = max_len;
        ap.cu_new = B.cu;
        ap.start_pos = B.start;
        ap.block_table = B.bt;
        ap.max_blocks_per_seq = blocks_per_copy;
        ap.err = cache->err_word;
        if (!ck(launch_append(ap, D, cache->n_sm, B.st))) return MQ_ERR_CUDA;
        for (int i = 1; i < n_copies; i++)
            if (!ck(cudaMemcpyAsync(static_cast<uint8_t*>(B.pool) + copy_bytes * i, B.pool, copy_bytes,
                                    cudaMemcpyDeviceToDevice, B.st)))
                return MQ_ERR_CUDA;
        if (!ck(cudaStreamSynchronize(B.st))) return MQ_ERR_CUDA;
    }

    int rot = 0;
    // one launch of probe p with configuration cfg on copy `rot`; returns status
    // (with `pool` set: on that single copy instead, e.g. the perturbed one)
    auto launch = [&](int p, const mq_decode_config& cfg, float* out, float* lse, void* pool = nullptr) -> mq_status {
        mq_cache pc = probe_cache;
        pc.cfg[probes[p].cls] = cfg;
        const int32_t* bt = B.bt + (size_t)(rot % n_copies) * blocks_per_copy;
        rot++;
        if (pool != nullptr) {
            pc.pool = pool;
            pc.pool_bytes = copy_bytes;
            pc.n_blocks = blocks_per_copy;
            bt = B.bt;   // the first copy's table: blocks 0 .. blocks_per_copy - 1
        }
        const DecodePlan pl = plan_decode(&pc, 1, Hq, probes[p].n_q, probes[p].seq_len);
        return launch_decode_plan(&pc, pl, B.q, MQ_BF16, 1, Hq, probes[p].n_q, probes[p].n_q, bt, blocks_per_copy,
                                  B.lens + p, B.nq + p, 1.0f / std::sqrt((float)D), out, lse, B.ws, ws_bytes, B.st);
    };
    // one drafter launch over the 64K-token history
    auto launch_draft = [&]() -> mq_status {
        return mq_draft_ngram(B.tokens, kDraftLen, B.tokens + kDraftLen, 1, kDraftN, kDraftK, B.drafts, B.n_drafts,
                              reinterpret_cast<mq_stream>(B.st));
    };
    const int reps = 7;
    // median device time of `reps` launches of probe p (events around the probe's
    // launches: the drafter's, when it has one, then the decode)
    auto time_probe = [&](int p, const mq_decode_config& cfg, double* out_t) -> mq_status {
        std::vector<float> ts;
        for (int r = 0; r < reps; r++) {
            cudaEventRecord(B.ev[0], B.st);
            mq_status s = probes[p].with_draft ? launch_draft() : MQ_OK;
            if (s == MQ_OK) s = launch(p, cfg, B.out, B.lse);
            if (s != MQ_OK) return s;
            cudaEventRecord(B.ev[1], B.st);
            if (!ck(cudaEventSynchronize(B.ev[1]))) return MQ_ERR_CUDA;
            float ms = 0;
            cudaEventElapsedTime(&ms, B.ev[0], B.ev[1]);
            ts.push_back(ms);
        }
        std::sort(ts.begin(), ts.end());
        *out_t = ts[ts.size() / 2] * 1e-3;
        return MQ_OK;
    };

    // ---- defaults: reference outputs and times; each term's time at the defaults ----
    for (int p = 0; p < P; p++) {
        mq_status s = launch(p, cache->cfg[probes[p].cls], B.out_ref[p], B.lse_ref[p]);
        if (s != MQ_OK) return s;
        if ((s = time_probe(p, cache->cfg[probes[p].cls], &probes[p].t_default)) != MQ_OK) return s;
    }
    // the drafter term alone (median of `reps` launches)
    double t_draft_default = 0;
    {
        std::vector<float> ts;
        for (int r = 0; r < reps; r++) {
            cudaEventRecord(B.ev[0], B.st);
            if (launch_draft() != MQ_OK) return MQ_ERR_CUDA;
            cudaEventRecord(B.ev[1], B.st);
            if (!ck(cudaEventSynchronize(B.ev[1]))) return MQ_ERR_CUDA;
            float ms = 0;
            cudaEventElapsedTime(&ms, B.ev[0], B.ev[1]);
            ts.push_back(ms);
        }
        std::sort(ts.begin(), ts.end());
        t_draft_default = ts[ts.size() / 2] * 1e-3;
    }
    // the prompt-prefill terms (4k and 64k prompts over the probe cache; head_dim 128 and
    // a group size dividing 128, else not part of the cost)
    double t_pf[2] = {0, 0};
    const bool with_prefill = D == 128 && G <= 128 && 128 % G == 0;
    if (with_prefill) {
        const size_t pf_q = (size_t)65536 * Hq * D;
        int32_t pl[2] = {4096, 65536};
        if (!ck(cudaMalloc(&B.q_pf, pf_q * 2)) || !ck(cudaMalloc(&B.out_pf, pf_q * 4)) ||
            !ck(cudaMalloc(&B.pf_lens, sizeof pl)) ||
            !ck(cudaMemcpy(B.pf_lens, pl, sizeof pl, cudaMemcpyHostToDevice)) ||
            !ck(launch_fill_random(B.q_pf, 1, (long long)pf_q, D, 0x7066ull, B.st)))
            return MQ_ERR_CUDA;
        for (int k = 0; k < 2; k++) {
            std::vector<float> ts;
            for (int r = 0; r < (k == 0 ? reps : 3); r++) {
                cudaEventRecord(B.ev[0], B.st);
                if (mq_prefill_attn(&probe_cache, B.q_pf, MQ_BF16, 1, Hq, pl[k], pl[k], pl[k], B.bt, blocks_per_copy,
                                    B.pf_lens + k, B.pf_lens + k, 1.0f / std::sqrt((float)D), B.out_pf, nullptr,
                                    reinterpret_cast<mq_stream>(B.st)) != MQ_OK)
                    return MQ_ERR_CUDA;
                cudaEventRecord(B.ev[1], B.st);
                if (!ck(cudaEventSynchronize(B.ev[1]))) return MQ_ERR_CUDA;
                float ms = 0;
                cudaEventElapsedTime(&ms, B.ev[0], B.ev[1]);
                ts.push_back(ms);
            }
            std::sort(ts.begin(), ts.end());
            t_pf[k] = ts[ts.size() / 2] * 1e-3;
        }
    }
    // weight(p) = sum_t launches(t, p) / time_at_defaults(t): a probe with a drafter holds
    // one launch of the drafter term and one of its decode term, whose time at the
    // defaults is the probe's time less the drafter's
    for (int p = 0; p < P; p++) {
        if (probes[p].with_draft) {
            const double t_dec = std::max(probes[p].t_default - t_draft_default, 1e-9);
            probes[p].weight = 1.0 / std::max(t_draft_default, 1e-9) + 1.0 / t_dec;
        } else {
            probes[p].weight = 1.0 / std::max(probes[p].t_default, 1e-9);
        }
    }
    if (!ck(cudaStreamSynchronize(B.st))) return MQ_ERR_CUDA;

    // ---- storage-resolution noise of the default output (alpha rule only) ----
    NoiseStats nstat[3];
    if (alpha_rule) {
        if (!ck(cudaMalloc(&B.pert, copy_bytes))) return MQ_ERR_CUDA;
        for (int p = 0; p < P; p++) {
            const size_t n_out = (size_t)probes[p].n_q * Hq * D, n_lse = (size_t)probes[p].n_q * Hq;
            if (!ck(cudaMalloc(&B.noise_out[p], n_out * 4)) || !ck(cudaMalloc(&B.noise_lse[p], n_lse * 4)) ||
                !ck(cudaMemsetAsync(B.noise_out[p], 0, n_out * 4, B.st)) ||
                !ck(cudaMemsetAsync(B.noise_lse[p], 0, n_lse * 4, B.st)))
                return MQ_ERR_CUDA;
        }
        const long long n_pages = (long long)blocks_per_copy * Hkv;
        for (unsigned long long seed : {0x5354455031ull, 0x5354455032ull}) {
            if (!ck(launch_perturb_pages(B.pool, B.pert, n_pages, D, seed, B.st))) return MQ_ERR_CUDA;
            for (int p = 0; p < P; p++) {
                const long long n_out = (long long)probes[p].n_q * Hq * D, n_lse = (long long)probes[p].n_q * Hq;
                mq_status s = launch(p, cache->cfg[probes[p].cls], B.out, B.lse, B.pert);
                if (s != MQ_OK) return s;
                if (!ck(launch_noise_max(B.out, B.out_ref[p], B.noise_out[p], n_out, B.st)) ||
                    !ck(launch_noise_max(B.lse, B.lse_ref[p], B.noise_lse[p], n_lse, B.st)))
                    return MQ_ERR_CUDA;
            }
        }
        for (int p = 0; p < P; p++) {
            std::vector<float> h((size_t)probes[p].n_q * Hq * D);
            if (!ck(cudaMemcpyAsync(h.data(), B.noise_out[p], h.size() * 4, cudaMemcpyDeviceToHost, B.st)) ||
                !ck(cudaStreamSynchronize(B.st)))
                return MQ_ERR_CUDA;
            for (float v : h) nstat[p].zero_points += v == 0.0f;
            std::sort(h.begin(), h.end());
            nstat[p].min = h.front();
            nstat[p].median = h[h.size() / 2];
            nstat[p].max = h.back();
        }
    }
    if (seconds_since(t0) > prm->budget_s) {
        res->elapsed_s = seconds_since(t0);
        return MQ_TUNE_BUDGET_EXHAUSTED;
    }

    // ---- candidates: structure (splits per SM, softmax warps) first, then ring depth ----
    std::vector<Cand> cands;
    bool class_used[3] = {false, false, false};
    int class_rows[3] = {0, 0, 0};   // the row block the class's probes run
    for (auto& pr : probes) {
        class_used[pr.cls] = true;
        class_rows[pr.cls] = plan_decode(&probe_cache, 1, Hq, pr.n_q, pr.seq_len).rows;
    }
    for (int r : {8, 6, 4, 3, 2})
        for (int sps : {1, 2, 4})
            for (int w : {4, 8})
                for (int cls = 0; cls < 3; cls++) {
                    if (!class_used[cls]) continue;
                    // 32-row blocks always run 8 softmax warps and 4-row blocks 4: the other
                    // value would repeat a candidate
                    if ((class_rows[cls] == 32 && w == 4) || (class_rows[cls] == 4 && w == 8)) continue;
                    Cand cd;
                    cd.cfg = mq_decode_config{r, sps, w};
                    cd.cls = cls;
                    const mq_decode_config& d = cache->cfg[cls];
                    if (cd.cfg.ring_stages == d.ring_stages && cd.cfg.splits_per_sm == d.splits_per_sm &&
                        cd.cfg.softmax_warps == d.softmax_warps)
                        continue;
                    cands.push_back(cd);
                }
    bool exhausted = false;
    for (auto& cd : cands) {
        double est = 0;
        for (int p = 0; p < P; p++)
            if (probes[p].cls == cd.cls) est += probes[p].t_default * (reps + 2) * 2 + 2e-3;
        if (seconds_since(t0) + est > prm->budget_s) {
            exhausted = true;
            res->n_skipped++;
            continue;
        }
        mq_cache pc = probe_cache;
        pc.cfg[cd.cls] = cd.cfg;
        bool ok = true;
        for (int p = 0; p < P && ok; p++) {
            if (probes[p].cls != cd.cls) continue;
            const DecodePlan pl = plan_decode(&pc, 1, Hq, probes[p].n_q, probes[p].seq_len);
            if (pl.smem == 0 || pl.smem > (size_t)cache->max_smem) {
                cd.valid = false;
                ok = false;
                break;
            }
            // admission: the bytes are compared always (evidence), the alpha rule on request
            if (launch(p, cd.cfg, B.out, B.lse) != MQ_OK) return MQ_ERR_CUDA;
            if (!ck(cudaMemsetAsync(B.flag, 0, 3 * sizeof(unsigned), B.st))) return MQ_ERR_CUDA;
            const long long n_out = (long long)probes[p].n_q * Hq * D, n_lse = (long long)probes[p].n_q * Hq;
            if (!ck(launch_compare(reinterpret_cast<const uint32_t*>(B.out), reinterpret_cast<const uint32_t*>(B.out_ref[p]),
                                   n_out, B.flag, B.st)) ||
                !ck(launch_compare(reinterpret_cast<const uint32_t*>(B.lse), reinterpret_cast<const uint32_t*>(B.lse_ref[p]),
                                   n_lse, B.flag, B.st)))
                return MQ_ERR_CUDA;
            if (alpha_rule &&
                (!ck(launch_alpha_check(B.out, B.out_ref[p], B.noise_out[p], n_out, (float)alpha, B.flag + 1, B.st)) ||
                 !ck(launch_alpha_check(B.lse, B.lse_ref[p], B.noise_lse[p], n_lse, (float)alpha, B.flag + 1, B.st))))
                return MQ_ERR_CUDA;
            unsigned fl[3] = {0, 0, 0};
            if (!ck(cudaMemcpyAsync(fl, B.flag, sizeof fl, cudaMemcpyDeviceToHost, B.st)) ||
                !ck(cudaStreamSynchronize(B.st)))
                return MQ_ERR_CUDA;
            float ratio = 0.0f;
            std::memcpy(&ratio, &fl[2], sizeof ratio);
            cd.max_ratio = std::max(cd.max_ratio, (double)ratio);
            if (fl[0]) cd.identical = false;
            if (alpha_rule ? fl[1] != 0 : fl[0] != 0) {
                cd.rejected = true;
                res->n_rejected++;
                ok = false;
                break;
            }
            if (time_probe(p, cd.cfg, &cd.t[p]) != MQ_OK) return MQ_ERR_CUDA;
        }
        if (cd.valid) {
            cd.measured = true;
            res->n_tried++;
        }
    }

    // ---- choose per rows class ----
    double total = 0;
    int n_terms = 0;
    for (int cls = 0; cls < 3; cls++) {
        if (!class_used[cls]) continue;
        // cost(c) = sum_p weight(p) * time(c, p), relative to the defaults' cost
        double base = 0;
        int terms = 0;
        for (int p = 0; p < P; p++)
            if (probes[p].cls == cls) {
                base += probes[p].weight * probes[p].t_default;
                terms++;
            }
        double best = 1.0;
        mq_decode_config pick = cache->cfg[cls];
        for (auto& cd : cands) {
            if (cd.cls != cls || !cd.measured || cd.rejected || !cd.valid) continue;
            double cost = 0;
            for (int p = 0; p < P; p++)
                if (probes[p].cls == cls) cost += probes[p].weight * cd.t[p] / base;
            if (cost < best) {
                best = cost;
                pick = cd.cfg;
            }
        }
        res->chosen[cls] = pick;
        cache->cfg[cls] = pick;
        total += best * terms;
        n_terms += terms;
    }
    // the prefill terms: the same time for every candidate, weight 1 / time each
    if (with_prefill) {
        total += 2.0;
        n_terms += 2;
    }
    res->cost = n_terms ? total / n_terms : 1.0;
    mq_status status = exhausted ? MQ_TUNE_BUDGET_EXHAUSTED : MQ_OK;
    bool stored = false;
    if (prm->store_path != nullptr && status == MQ_OK) {
        if (mq_tune_store_put(prm->store_path, identity, res->chosen, res->cost) != MQ_OK) status = MQ_ERR_IO;
        else stored = true;
    }
    res->elapsed_s = seconds_since(t0);

    if (prm->log_path != nullptr) {
        FILE* f = std::fopen(prm->log_path, "w");
        if (f != nullptr) {
            std::fprintf(f, "{\n  \"budget_s\": %.3f, \"elapsed_s\": %.3f, \"n_copies\": %d, \"l2_bytes\": %d,\n",
                         prm->budget_s, res->elapsed_s, n_copies, l2);
            std::fprintf(f, "  \"from_store\": false, \"stored\": %s, \"identity\": \"%s\",\n", stored ? "true" : "false",
                         identity);
            std::fprintf(f, "  \"admission\": \"%s\", \"alpha\": %.6g,\n", alpha_rule ? "alpha" : "bit_identical", alpha);
            if (alpha_rule) {
                std::fprintf(f, "  \"noise\": [");
                for (int p = 0; p < P; p++)
                    std::fprintf(f, "%s{\"probe\": \"%s\", \"out_min\": %.6g, \"out_median\": %.6g, \"out_max\": %.6g, "
                                 "\"out_zero_points\": %lld}",
                                 p ? ", " : "", probes[p].name, nstat[p].min, nstat[p].median, nstat[p].max,
                                 nstat[p].zero_points);
                std::fprintf(f, "],\n");
            }
            std::fprintf(f, "  \"terms\": [{\"name\": \"decode_4k\", \"default_us\": %.3f}, "
                         "{\"name\": \"decode_64k\", \"default_us\": %.3f}",
                         probes[0].t_default * 1e6, probes[1].t_default * 1e6);
            if (P > 2)
                std::fprintf(f, ", {\"name\": \"draft_64k\", \"default_us\": %.3f, \"ngram\": %d, \"max_draft\": %d}, "
                             "{\"name\": \"verify8_64k\", \"default_us\": %.3f}",
                             t_draft_default * 1e6, kDraftN, kDraftK,
                             std::max(probes[2].t_default - t_draft_default, 0.0) * 1e6);
            if (with_prefill)
                std::fprintf(f, ", {\"name\": \"prefill_4k\", \"default_us\": %.3f, \"prompt_tokens\": 4096}, "
                             "{\"name\": \"prefill_64k\", \"default_us\": %.3f, \"prompt_tokens\": 65536}",
                             t_pf[0] * 1e6, t_pf[1] * 1e6);
            std::fprintf(f, "],\n  \"probes\": [");
            for (int p = 0; p < P; p++)
                std::fprintf(f, "%s{\"name\": \"%s\", \"seq_len\": %d, \"n_q\": %d, \"rows_class\": %d, "
                             "\"launches\": \"%s\", \"default_us\": %.3f, \"weight_per_s\": %.6g}",
                             p ? ", " : "", probes[p].name, probes[p].seq_len, probes[p].n_q, probes[p].cls,
                             probes[p].with_draft ? "draft_64k + verify8_64k" : probes[p].name,
                             probes[p].t_default * 1e6, probes[p].weight);
            std::fprintf(f, "],\n  \"candidates\": [\n");
            for (size_t i = 0; i < cands.size(); i++) {
                const Cand& cd = cands[i];
                std::fprintf(f,
                             "    {\"rows_class\": %d, \"ring_stages\": %d, \"splits_per_sm\": %d, "
                             "\"softmax_warps\": %d, "
                             "\"measured\": %s, \"valid\": %s, \"bit_identical\": %s, \"admitted\": %s, "
                             "\"times_us\": [%.3f, %.3f, %.3f], \"max_ratio\": ",
                             cd.cls, cd.cfg.ring_stages, cd.cfg.splits_per_sm, cd.cfg.softmax_warps,
                             cd.measured ? "true" : "false", cd.valid ? "true" : "false",
                             cd.identical ? "true" : "false", (cd.measured && !cd.rejected) ? "true" : "false",
                             cd.t[0] * 1e6, cd.t[1] * 1e6, cd.t[2] * 1e6);
                json_double(f, cd.max_ratio);
                std::fprintf(f, "}%s\n", i + 1 < cands.size() ? "," : "");
            }
            std::fprintf(f, "  ],\n  \"chosen\": [");
            for (int cls = 0; cls < 3; cls++)
                std::fprintf(f,
                             "%s{\"rows_class\": %d, \"ring_stages\": %d, \"splits_per_sm\": %d, "
                             "\"softmax_warps\": %d}",
                             cls ? ", " : "", cls, res->chosen[cls].ring_stages, res->chosen[cls].splits_per_sm,
                             res->chosen[cls].softmax_warps);
            std::fprintf(f, "],\n  \"cost\": %.4f, \"n_tried\": %d, \"n_rejected\": %d, \"n_skipped\": %d\n}\n", res->cost,
                         res->n_tried, res->n_rejected, res->n_skipped);
            std::fclose(f);
        }
    }
    return status;
}
