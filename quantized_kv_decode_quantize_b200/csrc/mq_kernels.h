// Internal launch interface between the C-ABI layer (mq_api.cu) and the kernels.
#pragma once
#include <cstdint>
#include <cuda_runtime.h>

namespace mq {

struct AppendParams {
    uint8_t* pool;
    int n_kv_heads;
    long long n_blocks;
    const void* k;
    const void* v;
    int dtype;  // 0 f32, 1 bf16, 2 f16
    int n_seqs;
    int n_tokens;
    const int32_t* cu_new;
    const int32_t* start_pos;
    const int32_t* block_table;
    int max_blocks_per_seq;
    unsigned* err;
    int slices;   // warps per 8-position record (1, or 4 for small appends; set by the launch)
};

cudaError_t launch_append(const AppendParams& p, int head_dim, int n_sm, cudaStream_t st);

struct ExportParams {
    const uint8_t* pool;
    int n_kv_heads;
    long long n_blocks;
    int n_seqs;
    int n_tokens;
    const int32_t* cu_tok;
    const int32_t* start_pos;
    const int32_t* block_table;
    int max_blocks_per_seq;
    int8_t* k_codes;
    uint16_t* k_scales;
    uint8_t* v_packed;
    uint16_t* v_scales;
    unsigned* err;
};

cudaError_t launch_export(const ExportParams& p, int head_dim, cudaStream_t st);

struct DecodeParams {
    const uint8_t* pool;
    int n_kv_heads;
    long long n_blocks;
    const void* q;
    int q_dtype;  // 0 f32, 1 bf16, 2 f16
    int n_q_heads;
    int group;    // n_q_heads / n_kv_heads
    int total_q;
    int max_q;
    int n_seqs;
    const int32_t* block_table;
    int max_blocks_per_seq;
    const int32_t* seq_lens;
    const int32_t* n_q_per_seq;
    float scale_log2;  // softmax_scale * log2(e)
    float* out;
    float* lse;
    // workspace
    float* part_ml;      // [n_seqs][n_kv_heads][n_rb][split_stride][2][rows]: m then l per CTA
    float* part_o;       // [n_seqs][n_kv_heads][n_rb][split_stride][rows][D]
    int split_stride;    // partial slots per unit (>= the CTAs of any unit)
    int n_rb;            // row blocks per kv-head
    int cpc;             // chunks per CTA (a multiple of node_chunks); with cta_budget, set per launch on the device
    int node_chunks;     // chunks per merge-tree leaf
    int cta_budget;      // > 0: a flat grid whose units take CTAs by their own length (flat_lpc, flat_locate)
    int stages;          // TMA ring depth in chunks
    unsigned* err;
    // How the launch sees each sequence (the cascade's two passes use these; a plain
    // decode has causal 1 and the rest 0).
    int causal;          // 1: query j of n sees positions <= L - n + j; 0: every query sees all L
    int len_offset;      // L = seq_lens[b] - len_offset
    int bt_col;          // block-table column of the sequence's first page
    int fixed_len;       // > 0: L = fixed_len for every sequence (seq_lens not read)
    int fixed_nq;        // > 0: n = fixed_nq for every sequence (n_q_per_seq not read)
};

// Cached tokens and query tokens of sequence b as a launch sees them.
#ifdef __CUDACC__
__device__ __forceinline__ int seq_len_of(const DecodeParams& p, int b) {
    return p.fixed_len > 0 ? p.fixed_len : __ldg(p.seq_lens + b) - p.len_offset;
}
__device__ __forceinline__ int seq_nq_of(const DecodeParams& p, int b) {
    return p.fixed_nq > 0 ? p.fixed_nq : __ldg(p.n_q_per_seq + b);
}
#endif

// The small row classes (4 and 8 rows, mq_decode_small.cu).
size_t small_smem_bytes(int head_dim, int rows, int groups, int stages);
int small_ctas_per_sm(int head_dim, int rows);
int small_leaf_kmax(int head_dim, int rows);
cudaError_t small_prepare(int head_dim, int rows, int groups, size_t smem);
cudaError_t small_launch(const DecodeParams& p, int head_dim, int rows, int groups, dim3 grid, size_t smem,
                         cudaStream_t st);

// Prefill attention (mq_prefill.cu): head_dim 128, tiles of 128 query rows.
size_t prefill_smem_bytes();
cudaError_t launch_prefill(const DecodeParams& p, int max_tiles, cudaStream_t st);

// rows: 4, 8, 16 or 32 (padded query rows per kv-head handled by one CTA)
size_t decode_smem_bytes(int head_dim, int rows, int groups, int stages);   // 0: not built / does not fit
cudaError_t decode_prepare(int head_dim, int rows, int groups, size_t smem);  // raises the dynamic smem limit
int decode_ctas_per_sm(int head_dim, int rows);                    // CTAs the kernel is built to co-host
cudaError_t launch_decode(const DecodeParams& p, int head_dim, int rows, int groups, int max_splits, int flat_ctas, bool merge, size_t smem,
                          cudaStream_t st);

// Fills n values of dtype with a deterministic pseudo-random pattern (uniform in
// [-2, 2), channels 0..3 of every head_dim vector scaled by 10).  Used by the tuner
// to build probe caches; not part of any computed result.
cudaError_t launch_fill_random(void* dst, int dtype, long long n, int head_dim, unsigned long long seed,
                               cudaStream_t st);
// Writes a buffer (L2 flush between timed launches).
cudaError_t launch_scribble(void* dst, size_t bytes, unsigned v, cudaStream_t st);
// out[0] = 1 if a[i] != b[i] for some i < n32 (32-bit words), else unchanged.
cudaError_t launch_compare(const uint32_t* a, const uint32_t* b, long long n32, unsigned* out, cudaStream_t st);
// one format step of every stored element of n_pages pages (src -> dst, same layout)
cudaError_t launch_perturb_pages(const void* src, void* dst, long long n_pages, int head_dim,
                                 unsigned long long seed, cudaStream_t st);
// noise[i] = max(noise[i], |moved[i] - ref[i]|)
cudaError_t launch_noise_max(const float* moved, const float* ref, float* noise, long long n, cudaStream_t st);
// out[0] |= (some |cand - ref| > alpha * noise); out[1] = max ratio as float bits
cudaError_t launch_alpha_check(const float* cand, const float* ref, const float* noise, long long n, float alpha,
                               unsigned* out, cudaStream_t st);

}  // namespace mq
