// mq_draft_ngram: history-based drafting for speculative decoding.
//
// The blog.123qwe.co.kr deep dive on magnitudedev/magnitude (section 5, the table of
// drafting guarantees) lists history-based drafters among those whose draft step
// costs only the bytes the drafter itself reads; the drafts are then verified by one
// mq_decode_attn launch with n_q_per_seq > 1.  The pages give no algorithm.  This
// library's reading: propose the tokens that followed the most recent earlier
// occurrence of the history's last n tokens,
//   i* = max { i : 0 <= i < L - n, tokens[i + j] == tokens[L - n + j] for j < n }
//   drafts[j] = tokens[i* + n + j],  j < min(k, L - i* - n)
// One CTA per sequence: its threads test the candidate windows in parallel (each
// window's first token against the suffix's first, then the rest), keep the largest
// match, reduce it over the block, and copy the following tokens.  The step reads the
// history once (4 bytes a token), which is the whole cost the guarantee allows.
#include <cstdint>

#include <cuda_runtime.h>

#include "mq.h"
#include "mq_host.h"

namespace mq {
namespace {

constexpr int kDraftThreads = 256;
constexpr int kMaxNgram = 64;

__global__ void __launch_bounds__(kDraftThreads) draft_ngram_kernel(const int32_t* __restrict__ tokens, int max_len,
                                                                    const int32_t* __restrict__ seq_lens, int n,
                                                                    int k, int32_t* __restrict__ drafts,
                                                                    int32_t* __restrict__ n_drafts) {
    __shared__ int32_t suffix[kMaxNgram];
    __shared__ int warp_best[kDraftThreads / 32];
    __shared__ int best_s;
    const int b = blockIdx.x, tid = threadIdx.x;
    const int L = __ldg(seq_lens + b);
    if (L < 0 || L > max_len) {   // uniform over the block
        if (tid == 0) n_drafts[b] = -1;
        return;
    }
    if (L <= n) {
        if (tid == 0) n_drafts[b] = 0;
        return;
    }
    const int32_t* t = tokens + (size_t)b * max_len;
    if (tid < n) suffix[tid] = __ldg(t + L - n + tid);
    __syncthreads();
    // candidate windows start at 0 .. L - n - 1; a thread's candidates rise, so its
    // last match is its largest
    int best = -1;
    const int32_t first = suffix[0];
    for (int i = tid; i < L - n; i += kDraftThreads) {
        if (__ldg(t + i) != first) continue;
        bool same = true;
        for (int j = 1; j < n && same; j++) same = __ldg(t + i + j) == suffix[j];
        if (same) best = i;
    }
    best = __reduce_max_sync(0xffffffffu, best);
    if ((tid & 31) == 0) warp_best[tid >> 5] = best;
    __syncthreads();
    if (tid == 0) {
        int m = -1;
        for (int w = 0; w < kDraftThreads / 32; w++) m = max(m, warp_best[w]);
        best_s = m;
    }
    __syncthreads();
    const int i_star = best_s;
    const int cnt = i_star < 0 ? 0 : min(k, L - i_star - n);
    for (int j = tid; j < cnt; j += kDraftThreads) drafts[(size_t)b * k + j] = __ldg(t + i_star + n + j);
    if (tid == 0) n_drafts[b] = cnt;
}

}  // namespace
}  // namespace mq

using namespace mq;

extern "C" mq_status mq_draft_ngram(const int32_t* tokens, int32_t max_len, const int32_t* seq_lens, int32_t n_seqs,
                                    int32_t ngram, int32_t max_draft, int32_t* drafts, int32_t* n_drafts,
                                    mq_stream stream) {
    if (tokens == nullptr || seq_lens == nullptr || drafts == nullptr || n_drafts == nullptr) return MQ_ERR_INVALID_ARG;
    if (max_len < 1 || n_seqs < 1 || ngram < 1 || ngram > kMaxNgram || max_draft < 1) return MQ_ERR_INVALID_ARG;
    const cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    draft_ngram_kernel<<<(unsigned)n_seqs, kDraftThreads, 0, st>>>(tokens, max_len, seq_lens, ngram, max_draft, drafts,
                                                                  n_drafts);
    return cudaGetLastError() == cudaSuccess ? MQ_OK : MQ_ERR_CUDA;
}
