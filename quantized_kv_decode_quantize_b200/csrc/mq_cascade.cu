// mq_decode_attn_cascade: decode attention for sessions that share a cached prefix,
// reading the prefix pages once for all of them.
//
// The pages report sessions sharing one prefix cache (the blog.123qwe.co.kr deep dive
// on magnitudedev/magnitude, section 5, and the trawling.dev "Launch HN: Magnitude"
// section on per-device kernel tuning: concurrent sessions share the prefix cache).
// A plain decode reads the shared pages once per session.  Attention over the
// concatenation of two token sets is the log-sum-exp combination of the attentions over
// each set, so the step splits in two passes and a merge:
//   1. prefix pass: one launch over the prefix pages whose query rows are the query
//      tokens of every session (G x total_q rows per kv-head), none of them masked:
//      every session's first query already sees the whole prefix;
//   2. suffix pass: the plain decode over each session's own pages past the prefix,
//      causal among its drafts as usual (same arrays: the lengths are offset by the
//      prefix and the block table read from the prefix's last column on);
//   3. out = (o1 e^{lse1} + o2 e^{lse2}) / (e^{lse1} + e^{lse2}), lse = log of the
//      denominator, per (query token, q-head).
#include <cmath>
#include <cstddef>
#include <cstdint>

#include <cuda_runtime.h>

#include "mq.h"
#include "mq_device.cuh"
#include "mq_host.h"
#include "mq_kernels.h"

namespace mq {
namespace {

size_t al256(size_t x) { return (x + 255) / 256 * 256; }

// Merge of the two passes' normalised outputs by their log-sum-exps, in place into o2.
__global__ void merge_two_kernel(const float* __restrict__ o1, const float* __restrict__ l1, float* o2,
                                 const float* __restrict__ l2, float* lse_out, long long n_rows, int D) {
    const int d4 = D / 4;
    for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < n_rows * d4;
         i += (long long)gridDim.x * blockDim.x) {
        const long long row = i / d4;
        const float a = l1[row], b = l2[row];
        const float m = fmaxf(a, b);
        float4 x = reinterpret_cast<const float4*>(o1)[i];
        float4 y = reinterpret_cast<float4*>(o2)[i];
        float lse;
        if (m == -INFINITY) {   // neither pass saw a token (only after flagged bad input)
            lse = m;
        } else {
            const float wa = expf(__fsub_rn(a, m)), wb = expf(__fsub_rn(b, m));
            const float den = __fadd_rn(wa, wb);
            y.x = __fdiv_rn(__fadd_rn(__fmul_rn(x.x, wa), __fmul_rn(y.x, wb)), den);
            y.y = __fdiv_rn(__fadd_rn(__fmul_rn(x.y, wa), __fmul_rn(y.y, wb)), den);
            y.z = __fdiv_rn(__fadd_rn(__fmul_rn(x.z, wa), __fmul_rn(y.z, wb)), den);
            y.w = __fdiv_rn(__fadd_rn(__fmul_rn(x.w, wa), __fmul_rn(y.w, wb)), den);
            reinterpret_cast<float4*>(o2)[i] = y;
            lse = __fadd_rn(m, logf(den));
        }
        if (lse_out != nullptr && i % d4 == 0) lse_out[row] = lse;
    }
}

struct CascadeLayout {
    size_t part, out1, lse1, lse2, total;
};

CascadeLayout cascade_layout(const mq_cache* c, int n_seqs, int n_q_heads, int total_q, int max_q, int max_seq_len,
                             int prefix_len) {
    CascadeLayout w{};
    const size_t wp = mq_decode_workspace_bytes(c, 1, n_q_heads, total_q, prefix_len);
    const size_t ws = mq_decode_workspace_bytes(c, n_seqs, n_q_heads, max_q, max_seq_len - prefix_len);
    if (wp == 0 || ws == 0) return w;
    const size_t rows = (size_t)total_q * n_q_heads;
    w.part = 0;
    w.out1 = al256(wp > ws ? wp : ws);
    w.lse1 = w.out1 + al256(rows * c->head_dim * 4);
    w.lse2 = w.lse1 + al256(rows * 4);
    w.total = w.lse2 + al256(rows * 4);
    return w;
}

bool cascade_shape_ok(const mq_cache* c, int n_seqs, int n_q_heads, int total_q, int max_q, int max_seq_len,
                      int prefix_len) {
    if (c == nullptr || n_seqs < 1 || n_seqs > 65535 || n_q_heads < 1 || n_q_heads % c->n_kv_heads != 0) return false;
    if (total_q < 1 || max_q < 1 || total_q < max_q) return false;
    if (prefix_len < MQ_PAGE_TOKENS || prefix_len % MQ_PAGE_TOKENS != 0) return false;
    if (total_q > prefix_len || max_seq_len - prefix_len < max_q) return false;
    return true;
}

}  // namespace
}  // namespace mq

using namespace mq;

extern "C" size_t mq_decode_cascade_workspace_bytes(const mq_cache* c, int32_t n_seqs, int32_t n_q_heads,
                                                    int32_t total_q, int32_t max_q_per_seq, int32_t max_seq_len,
                                                    int32_t prefix_len) {
    if (!cascade_shape_ok(c, n_seqs, n_q_heads, total_q, max_q_per_seq, max_seq_len, prefix_len)) return 0;
    return cascade_layout(c, n_seqs, n_q_heads, total_q, max_q_per_seq, max_seq_len, prefix_len).total;
}

extern "C" mq_status mq_decode_attn_cascade(const mq_cache* c, const void* q, mq_dtype q_dtype, int32_t n_seqs,
                                            int32_t n_q_heads, int32_t total_q, int32_t max_q_per_seq,
                                            int32_t max_seq_len, const int32_t* block_table,
                                            int32_t max_blocks_per_seq, const int32_t* seq_lens,
                                            const int32_t* n_q_per_seq, int32_t prefix_len, float softmax_scale,
                                            float* out, float* lse, void* workspace, size_t workspace_bytes,
                                            mq_stream stream) {
    if (c == nullptr || q == nullptr || block_table == nullptr || seq_lens == nullptr || n_q_per_seq == nullptr ||
        out == nullptr)
        return MQ_ERR_INVALID_ARG;
    if (!cascade_shape_ok(c, n_seqs, n_q_heads, total_q, max_q_per_seq, max_seq_len, prefix_len) ||
        max_blocks_per_seq < 1 || !std::isfinite(softmax_scale))
        return MQ_ERR_INVALID_ARG;
    if (q_dtype != MQ_F32 && q_dtype != MQ_BF16 && q_dtype != MQ_F16) return MQ_ERR_UNSUPPORTED;
    const int G = n_q_heads / c->n_kv_heads;
    if (G * total_q > 64) return MQ_ERR_UNSUPPORTED;   // the prefix pass's rows per kv-head
    if ((long long)max_seq_len > (long long)max_blocks_per_seq * MQ_PAGE_TOKENS) return MQ_ERR_CAPACITY;
    if (reinterpret_cast<uintptr_t>(out) % 16 != 0) return MQ_ERR_INVALID_ARG;
    const CascadeLayout w = cascade_layout(c, n_seqs, n_q_heads, total_q, max_q_per_seq, max_seq_len, prefix_len);
    if (w.total == 0) return MQ_ERR_UNSUPPORTED;
    if (workspace == nullptr || workspace_bytes < w.total || reinterpret_cast<uintptr_t>(workspace) % 256 != 0)
        return MQ_ERR_WORKSPACE;
    DevGuard guard(c->device);
    const cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    uint8_t* ws = static_cast<uint8_t*>(workspace);
    float* out1 = reinterpret_cast<float*>(ws + w.out1);
    float* lse1 = reinterpret_cast<float*>(ws + w.lse1);
    float* lse2 = lse != nullptr ? lse : reinterpret_cast<float*>(ws + w.lse2);

    // 1. the prefix, once, for every session's query tokens (row 0 of the block table)
    DecodeView pre;
    pre.causal = 0;
    pre.fixed_len = prefix_len;
    pre.fixed_nq = total_q;
    const DecodePlan plp = plan_decode(c, 1, n_q_heads, total_q, prefix_len);
    mq_status s = launch_decode_plan(c, plp, q, q_dtype, 1, n_q_heads, total_q, total_q, block_table,
                                     max_blocks_per_seq, seq_lens, n_q_per_seq, softmax_scale, out1, lse1, ws + w.part,
                                     w.out1, st, pre);
    if (s != MQ_OK) return s;
    // 2. each session's own pages after the prefix
    DecodeView suf;
    suf.len_offset = prefix_len;
    suf.bt_col = prefix_len / MQ_PAGE_TOKENS;
    const DecodePlan pls = plan_decode(c, n_seqs, n_q_heads, max_q_per_seq, max_seq_len - prefix_len);
    s = launch_decode_plan(c, pls, q, q_dtype, n_seqs, n_q_heads, total_q, max_q_per_seq, block_table,
                           max_blocks_per_seq, seq_lens, n_q_per_seq, softmax_scale, out, lse2, ws + w.part, w.out1, st,
                           suf);
    if (s != MQ_OK) return s;
    // 3. the two results by their log-sum-exps
    const long long rows = (long long)total_q * n_q_heads;
    const long long n4 = rows * (c->head_dim / 4);
    const long long blocks = (n4 + 255) / 256 < 4096 ? (n4 + 255) / 256 : 4096;
    merge_two_kernel<<<(unsigned)blocks, 256, 0, st>>>(out1, lse1, out, lse2, lse, rows, c->head_dim);
    return cudaGetLastError() == cudaSuccess ? MQ_OK : MQ_ERR_CUDA;
}
