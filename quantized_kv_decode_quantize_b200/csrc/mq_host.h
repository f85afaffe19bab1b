// Host-side internals shared by the C-ABI layer and the tuner.
#pragma once
#include <cstddef>
#include <cstdint>
#include <cuda_runtime.h>

#include "mq.h"

struct mq_cache {
    int n_kv_heads;
    int head_dim;
    int64_t n_blocks;
    void* pool;
    size_t pool_bytes;
    int device;
    int n_sm;
    int max_smem;
    int smem_per_sm;
    unsigned* err_word;         // device address of this device's error word
    mq_decode_config cfg[3];    // per rows class
};

namespace mq {

// sequences of a call whose CTAs the device plans (a flat grid: every CTA reads every
// sequence's length, in rounds of 32)
constexpr int kFlatMaxSeqs = 64;

struct DecodePlan {
    int cls, rows, groups, n_rb, stages, cpc, max_splits;
    int node_chunks;               // merge-tree leaf (chunks)
    int cta_budget, flat_ctas;     // > 0: a flat grid of flat_ctas CTAs, balanced on the device
    bool merge;                    // some unit has several CTAs (merge_kernel completes the tree)
    size_t smem;
};

// Switches to `dev` for the lifetime of the guard when it is not current.
struct DevGuard {
    int prev = -1;
    bool switched = false;
    explicit DevGuard(int dev);
    ~DevGuard();
};

int rows_class_rows(int head_dim, int cls);
int rows_class_for(int head_dim, int rows_total);
mq_decode_config default_config(int head_dim, int cls);
bool config_valid(const mq_decode_config& c);
DecodePlan plan_decode(const mq_cache* c, int n_seqs, int n_q_heads, int max_q, int max_seq_len);
// Bytes of the CTA partials of one plan (the decode workspace).
size_t partial_bytes(const mq_cache* c, int n_seqs, const DecodePlan& pl);
cudaError_t ensure_decode_smem(int device, int head_dim, int rows, int groups, size_t smem);
// How one decode launch sees its sequences (see DecodeParams): the defaults are a plain
// causal decode over seq_lens and n_q_per_seq.
struct DecodeView {
    int causal = 1;
    int len_offset = 0;
    int bt_col = 0;
    int fixed_len = 0;
    int fixed_nq = 0;
};

mq_status launch_decode_plan(const mq_cache* c, const DecodePlan& pl, const void* q, mq_dtype q_dtype, int n_seqs,
                             int n_q_heads, int total_q, int max_q, const int32_t* block_table, int max_blocks,
                             const int32_t* seq_lens, const int32_t* n_q_per_seq, float softmax_scale, float* out,
                             float* lse, void* workspace, size_t workspace_bytes, cudaStream_t st,
                             const DecodeView& view = DecodeView{});

}  // namespace mq
