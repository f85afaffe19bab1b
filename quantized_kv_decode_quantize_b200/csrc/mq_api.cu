// C ABI of the mq library: argument validation, the cache handle, the choice of
// launch shape, and the device error word.  Every entry point validates its
// arguments on the host before making any CUDA call.
#include <algorithm>
#include <cmath>
#include <cstring>
#include <new>

#include "mq.h"
#include "mq_device.cuh"
#include "mq_kernels.h"
#include "mq_host.h"

namespace mq {

// One error word per device (every device that loads the library holds its own copy).
__device__ unsigned g_err_word;

cudaError_t error_word_address(unsigned** out) {
    return cudaGetSymbolAddress(reinterpret_cast<void**>(out), g_err_word);
}

int rows_class_rows(int head_dim, int cls) {
    if (cls == 0) return 8;
    if (cls == 1) return 16;
    return head_dim == 128 ? 32 : 16;
}

int rows_class_for(int head_dim, int rows_total) {
    if (rows_total <= 8) return 0;
    if (rows_total <= 16) return 1;
    return head_dim == 128 ? 2 : 1;
}

mq_decode_config default_config(int head_dim, int cls) {
    (void)head_dim;
    mq_decode_config c{};
    c.ring_stages = 8;   // the planner shortens it to what fits in shared memory
    c.splits_per_sm = 1;
    c.softmax_warps = cls == 2 ? 8 : 4;
    return c;
}

bool config_valid(const mq_decode_config& c) {
    return c.ring_stages >= 2 && c.ring_stages <= 8 &&
           (c.splits_per_sm == 1 || c.splits_per_sm == 2 || c.splits_per_sm == 4) &&
           (c.softmax_warps == 4 || c.softmax_warps == 8);
}

DevGuard::DevGuard(int dev) {
    if (cudaGetDevice(&prev) != cudaSuccess) prev = -1;
    if (prev != dev) {
        cudaSetDevice(dev);
        switched = true;
    }
}
DevGuard::~DevGuard() {
    if (switched && prev >= 0) cudaSetDevice(prev);
}

// The plan for one row class: rows per CTA, split count, chunks per CTA, merge-tree leaf,
// ring depth.  The chunk ranges depend only on the shape, the SM count and splits_per_sm.
// For the classes whose CTAs build a node of the fixed merge tree (up to 8 rows: one query
// token per sequence at GQA <= 8; small_leaf_kmax > 0), the leaf is a fixed run of chunks
// that depends on the shape alone (at most 2^kmax leaves per unit), every CTA holds an
// aligned power-of-two run of leaves, and the split count follows from that run: whatever
// the configured splits per SM, the CTAs and the merge kernel evaluate the same tree, so
// the output is bit-identical across split counts and ring depths.  The wider classes (draft verification) split into any
// number of equal ranges, one leaf each (a power of two would idle SMs there).
static DecodePlan plan_for_class(const mq_cache* c, int cls, int n_seqs, int rows_total, int max_seq_len) {
    DecodePlan pl{};
    pl.cls = cls;
    // class 0 runs 4-row blocks when every block holds at most 4 real rows (grouped-query
    // decode at GQA <= 4 with one query token)
    pl.rows = (cls == 0 && rows_total <= 4) ? 4 : rows_class_rows(c->head_dim, pl.cls);
    pl.n_rb = (rows_total + pl.rows - 1) / pl.rows;
    const mq_decode_config cfg = c->cfg[pl.cls];
    // softmax warp groups: 32-row blocks need two, 4-row blocks have one
    pl.groups = pl.rows == 32 ? 2 : (pl.rows == 4 ? 1 : cfg.softmax_warps / 4);
    const long long max_chunks = std::max<long long>(1, (max_seq_len + kChunkTokens - 1) / kChunkTokens);
    const long long units = (long long)n_seqs * c->n_kv_heads * pl.n_rb;
    const int cps = decode_ctas_per_sm(c->head_dim, pl.rows);
    long long splits = (long long)cfg.splits_per_sm * cps * c->n_sm / units;
    splits = std::max<long long>(1, std::min<long long>({splits, max_chunks, (long long)kMaxSplits}));
    const int kmax = small_leaf_kmax(c->head_dim, pl.rows);
    if (kmax > 0) {
        // at most 2^kmax leaves per unit, each ceil(max_chunks / 2^kmax) chunks (the unit
        // fills its leaves up to less than one chunk per leaf).  Every CTA takes an aligned
        // power-of-two run of leaves (lpc): the smallest lpc whose CTAs fit the CTA budget
        // below.  With several sequences the grid is flat and the
        // CTAs find lpc and their unit on the device from every sequence's length (each
        // unit takes CTAs in proportion to its own length: flat_lpc / flat_locate); one
        // sequence, or more than kFlatMaxSeqs, takes the run for max_seq_len on a (split,
        // unit) grid.
        const long long slots = 1LL << kmax;
        const long long leaf = (max_chunks + slots - 1) / slots;
        const long long leaves = (max_chunks + leaf - 1) / leaf;
        // the CTA budget: splits_per_sm x (CTAs per SM) x (number of SMs), and on a flat
        // grid at least 4 CTAs per unit on average (with about one CTA slot per unit,
        // the power-of-two run that fits is too coarse for lengths that differ widely: the
        // longest sequence's units would each go to one CTA)
        // Each CTA of a flat grid reads every sequence's length (rounds of 32), so flat
        // grids are kept to batches of up to kFlatMaxSeqs sequences (two rounds); larger
        // batches take the (split, unit) grid.  The floor is capped at 4 CTAs per slot.
        const bool flat = n_seqs > 1 && n_seqs <= kFlatMaxSeqs;
        long long budget = std::min<long long>((long long)cfg.splits_per_sm * cps * c->n_sm, 1LL << 30);
        if (flat) budget = std::max<long long>(budget, std::min<long long>(4 * units, 4LL * cps * c->n_sm));
        pl.node_chunks = (int)leaf;
        if (flat) {
            pl.cpc = 0;
            pl.cta_budget = (int)budget;
            pl.flat_ctas = (int)std::max<long long>(budget, units);
            pl.max_splits = (int)leaves;   // partial slots per unit: at most one CTA per leaf
        } else {
            long long lpc = 1;
            while (lpc < 64 && units * ((leaves + lpc - 1) / lpc) > budget) lpc *= 2;
            pl.cpc = (int)(lpc * leaf);
            pl.max_splits = (int)((leaves + lpc - 1) / lpc);
        }
    } else {
        const long long cpc = (max_chunks + splits - 1) / splits;
        pl.cpc = (int)cpc;
        pl.node_chunks = (int)cpc;
        pl.max_splits = (int)((max_chunks + pl.cpc - 1) / pl.cpc);
    }
    pl.merge = pl.max_splits > 1;
    // the ring is shortened (never below 2 stages) until the CTA fits in its share of
    // the SM's shared memory (1 KB of each CTA's share is reserved by the hardware)
    const size_t smem_cap = cps == 1 ? (size_t)c->max_smem
                                     : std::min((size_t)c->max_smem, (size_t)c->smem_per_sm / cps - 1024);
    pl.stages = cfg.ring_stages;
    pl.smem = decode_smem_bytes(c->head_dim, pl.rows, pl.groups, pl.stages);
    while ((pl.smem == 0 || pl.smem > smem_cap) && pl.stages > 2) {
        pl.stages--;
        pl.smem = decode_smem_bytes(c->head_dim, pl.rows, pl.groups, pl.stages);
    }
    return pl;
}

DecodePlan plan_decode(const mq_cache* c, int n_seqs, int n_q_heads, int max_q, int max_seq_len) {
    const int G = n_q_heads / c->n_kv_heads;
    const int rows_total = G * max_q;
    return plan_for_class(c, rows_class_for(c->head_dim, rows_total), n_seqs, rows_total, max_seq_len);
}

static size_t al256(size_t x) { return (x + 255) / 256 * 256; }

size_t partial_bytes(const mq_cache* c, int n_seqs, const DecodePlan& pl) {
    const size_t slots = (size_t)n_seqs * c->n_kv_heads * pl.n_rb * pl.max_splits;
    return al256(slots * pl.rows * 2 * 4) + slots * pl.rows * c->head_dim * 4;
}

mq_status launch_decode_plan(const mq_cache* c, const DecodePlan& pl, const void* q, mq_dtype q_dtype, int n_seqs,
                             int n_q_heads, int total_q, int max_q, const int32_t* block_table, int max_blocks,
                             const int32_t* seq_lens, const int32_t* n_q_per_seq, float softmax_scale, float* out,
                             float* lse, void* workspace, size_t workspace_bytes, cudaStream_t st,
                             const DecodeView& view) {
    if (pl.smem == 0 || pl.smem > (size_t)c->max_smem) return MQ_ERR_UNSUPPORTED;
    const size_t units = (size_t)n_seqs * c->n_kv_heads * pl.n_rb;
    if (partial_bytes(c, n_seqs, pl) > workspace_bytes) return MQ_ERR_WORKSPACE;
    cudaError_t e = ensure_decode_smem(c->device, c->head_dim, pl.rows, pl.groups, pl.smem);
    if (e != cudaSuccess) return MQ_ERR_CUDA;
    DecodeParams p{};
    p.pool = static_cast<const uint8_t*>(c->pool);
    p.n_kv_heads = c->n_kv_heads;
    p.n_blocks = c->n_blocks;
    p.q = q;
    p.q_dtype = (int)q_dtype;
    p.n_q_heads = n_q_heads;
    p.group = n_q_heads / c->n_kv_heads;
    p.total_q = total_q;
    p.max_q = max_q;
    p.n_seqs = n_seqs;
    p.block_table = block_table;
    p.max_blocks_per_seq = max_blocks;
    p.seq_lens = seq_lens;
    p.n_q_per_seq = n_q_per_seq;
    p.scale_log2 = (float)((double)softmax_scale * 1.4426950408889634);
    p.out = out;
    p.lse = lse;
    // this call's partials: (m, l) then O, with a stride of max_splits per unit
    uint8_t* ws = static_cast<uint8_t*>(workspace);
    size_t off = 0;
    p.part_ml = reinterpret_cast<float*>(ws + off);
    off += al256(units * pl.max_splits * pl.rows * 2 * 4);
    p.part_o = reinterpret_cast<float*>(ws + off);
    p.cta_budget = pl.cta_budget;
    p.split_stride = pl.max_splits;
    p.n_rb = pl.n_rb;
    p.cpc = pl.cpc;
    p.node_chunks = pl.node_chunks;
    p.stages = pl.stages;
    p.err = c->err_word;
    p.causal = view.causal;
    p.len_offset = view.len_offset;
    p.bt_col = view.bt_col;
    p.fixed_len = view.fixed_len;
    p.fixed_nq = view.fixed_nq;
    e = launch_decode(p, c->head_dim, pl.rows, pl.groups, pl.max_splits, pl.flat_ctas, pl.merge, pl.smem, st);
    return e == cudaSuccess ? MQ_OK : MQ_ERR_CUDA;
}

cudaError_t ensure_decode_smem(int device, int head_dim, int rows, int groups, size_t smem) {
    // raised limit per (device, kernel variant); the attribute only grows
    static size_t done[64][2][4][2] = {};
    const int di = device & 63, hi = head_dim == 128 ? 0 : 1;
    const int ri = rows == 4 ? 0 : (rows == 8 ? 1 : (rows == 16 ? 2 : 3));
    const int gi = groups == 2 ? 1 : 0;
    if (done[di][hi][ri][gi] >= smem) return cudaSuccess;
    cudaError_t e = decode_prepare(head_dim, rows, groups, smem);
    if (e == cudaSuccess) done[di][hi][ri][gi] = smem;
    return e;
}

}  // namespace mq

using namespace mq;

extern "C" {

const char* mq_status_string(mq_status s) {
    switch (s) {
        case MQ_OK: return "ok";
        case MQ_ERR_INVALID_ARG: return "invalid argument";
        case MQ_ERR_UNSUPPORTED: return "unsupported configuration";
        case MQ_ERR_CAPACITY: return "capacity exceeded";
        case MQ_ERR_WORKSPACE: return "workspace missing, too small or misaligned";
        case MQ_ERR_CUDA: return "CUDA error";
        case MQ_ERR_DEVICE: return "a kernel flagged bad input or a timed-out wait";
        case MQ_TUNE_BUDGET_EXHAUSTED: return "tuning budget exhausted before every candidate was measured";
        case MQ_ERR_IO: return "the tuning store could not be written";
    }
    return "unknown status";
}

int32_t mq_version(void) { return 1 * 10000 + 0 * 100 + 0; }

size_t mq_page_bytes(int32_t head_dim) {
    return (head_dim == 128 || head_dim == 256) ? (size_t)page_bytes(head_dim) : 0;
}

size_t mq_cache_pool_bytes(int32_t n_kv_heads, int32_t head_dim, int64_t n_blocks) {
    const size_t pb = mq_page_bytes(head_dim);
    if (pb == 0 || n_kv_heads < 1 || n_blocks < 1) return 0;
    return (size_t)n_blocks * (size_t)n_kv_heads * pb;
}

mq_status mq_cache_create(const mq_cache_desc* d, mq_cache** out) {
    if (out == nullptr) return MQ_ERR_INVALID_ARG;
    *out = nullptr;
    if (d == nullptr || d->pool == nullptr || d->n_kv_heads < 1 || d->n_blocks < 1) return MQ_ERR_INVALID_ARG;
    if (reinterpret_cast<uintptr_t>(d->pool) % 256 != 0) return MQ_ERR_INVALID_ARG;
    if (d->head_dim != 128 && d->head_dim != 256) return MQ_ERR_UNSUPPORTED;
    if (d->page_tokens != MQ_PAGE_TOKENS) return MQ_ERR_UNSUPPORTED;
    if (d->pool_bytes < mq_cache_pool_bytes(d->n_kv_heads, d->head_dim, d->n_blocks)) return MQ_ERR_CAPACITY;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return MQ_ERR_CUDA;
    int n_sm = 0, max_smem = 0, smem_per_sm = 0;
    if (cudaDeviceGetAttribute(&n_sm, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return MQ_ERR_CUDA;
    if (cudaDeviceGetAttribute(&max_smem, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev) != cudaSuccess)
        return MQ_ERR_CUDA;
    if (cudaDeviceGetAttribute(&smem_per_sm, cudaDevAttrMaxSharedMemoryPerMultiprocessor, dev) != cudaSuccess)
        return MQ_ERR_CUDA;
    unsigned* err = nullptr;
    if (error_word_address(&err) != cudaSuccess) return MQ_ERR_CUDA;
    mq_cache* c = new (std::nothrow) mq_cache;
    if (c == nullptr) return MQ_ERR_INVALID_ARG;
    c->n_kv_heads = d->n_kv_heads;
    c->head_dim = d->head_dim;
    c->n_blocks = d->n_blocks;
    c->pool = d->pool;
    c->pool_bytes = d->pool_bytes;
    c->device = dev;
    c->n_sm = n_sm;
    c->max_smem = max_smem;
    c->smem_per_sm = smem_per_sm;
    c->err_word = err;
    for (int k = 0; k < 3; k++) c->cfg[k] = default_config(d->head_dim, k);
    *out = c;
    return MQ_OK;
}

mq_status mq_cache_destroy(mq_cache* c) {
    delete c;
    return MQ_OK;
}

mq_status mq_kv_append(mq_cache* c, const void* k, const void* v, mq_dtype dtype, int32_t n_seqs, int32_t n_tokens,
                       const int32_t* cu_new, const int32_t* start_pos, const int32_t* block_table,
                       int32_t max_blocks_per_seq, mq_stream stream) {
    if (c == nullptr || n_seqs < 1 || n_seqs > 65535 || n_tokens < 0 || max_blocks_per_seq < 1)
        return MQ_ERR_INVALID_ARG;
    if (dtype != MQ_F32 && dtype != MQ_BF16 && dtype != MQ_F16) return MQ_ERR_INVALID_ARG;
    if (n_tokens == 0) return MQ_OK;
    if (k == nullptr || v == nullptr || cu_new == nullptr || start_pos == nullptr || block_table == nullptr)
        return MQ_ERR_INVALID_ARG;
    const size_t esz = dtype == MQ_F32 ? 4 : 2;
    const size_t align = esz * c->head_dim / 32;   // one lane's vector load
    if (reinterpret_cast<uintptr_t>(k) % align || reinterpret_cast<uintptr_t>(v) % align) return MQ_ERR_INVALID_ARG;
    DevGuard guard(c->device);
    AppendParams p{};
    p.pool = static_cast<uint8_t*>(c->pool);
    p.n_kv_heads = c->n_kv_heads;
    p.n_blocks = c->n_blocks;
    p.k = k;
    p.v = v;
    p.dtype = (int)dtype;
    p.n_seqs = n_seqs;
    p.n_tokens = n_tokens;
    p.cu_new = cu_new;
    p.start_pos = start_pos;
    p.block_table = block_table;
    p.max_blocks_per_seq = max_blocks_per_seq;
    p.err = c->err_word;
    return launch_append(p, c->head_dim, c->n_sm, reinterpret_cast<cudaStream_t>(stream)) == cudaSuccess ? MQ_OK
                                                                                               : MQ_ERR_CUDA;
}

mq_status mq_kv_export(const mq_cache* c, int32_t n_seqs, int32_t n_tokens, const int32_t* cu_tok,
                       const int32_t* start_pos, const int32_t* block_table, int32_t max_blocks_per_seq,
                       int8_t* k_codes, uint16_t* k_scales, uint8_t* v_packed, uint16_t* v_scales,
                       mq_stream stream) {
    if (c == nullptr || n_seqs < 1 || n_seqs > 65535 || n_tokens < 0 || max_blocks_per_seq < 1)
        return MQ_ERR_INVALID_ARG;
    if (n_tokens == 0) return MQ_OK;
    if (cu_tok == nullptr || start_pos == nullptr || block_table == nullptr || k_codes == nullptr ||
        k_scales == nullptr || v_packed == nullptr || v_scales == nullptr)
        return MQ_ERR_INVALID_ARG;
    DevGuard guard(c->device);
    ExportParams p{};
    p.pool = static_cast<const uint8_t*>(c->pool);
    p.n_kv_heads = c->n_kv_heads;
    p.n_blocks = c->n_blocks;
    p.n_seqs = n_seqs;
    p.n_tokens = n_tokens;
    p.cu_tok = cu_tok;
    p.start_pos = start_pos;
    p.block_table = block_table;
    p.max_blocks_per_seq = max_blocks_per_seq;
    p.k_codes = k_codes;
    p.k_scales = k_scales;
    p.v_packed = v_packed;
    p.v_scales = v_scales;
    p.err = c->err_word;
    return launch_export(p, c->head_dim, reinterpret_cast<cudaStream_t>(stream)) == cudaSuccess ? MQ_OK
                                                                                               : MQ_ERR_CUDA;
}

size_t mq_decode_workspace_bytes(const mq_cache* c, int32_t n_seqs, int32_t n_q_heads, int32_t max_q_per_seq,
                                 int32_t max_seq_len) {
    if (c == nullptr || n_seqs < 1 || n_q_heads < 1 || n_q_heads % c->n_kv_heads != 0 || max_q_per_seq < 1 ||
        max_seq_len < max_q_per_seq)
        return 0;
    const int G = n_q_heads / c->n_kv_heads;
    const int rows_total = G * max_q_per_seq;
    if (rows_total > 64) return 0;
    // The plan depends on the launch configuration (which mq_tune / mq_set_decode_config
    // may change after the workspace is sized): size the partials for the largest plan
    // over every valid configuration, so the answer depends on the shape alone.
    mq_cache probe = *c;
    size_t part = 0;
    for (int r = 2; r <= 8; r++)
        for (int t = 1; t <= 4; t *= 2) {
            for (int k = 0; k < 3; k++) probe.cfg[k] = mq_decode_config{r, t, k == 2 ? 8 : 4};
            const DecodePlan pl = plan_for_class(&probe, rows_class_for(c->head_dim, rows_total), n_seqs, rows_total,
                                                 max_seq_len);
            part = std::max(part, partial_bytes(c, n_seqs, pl));
        }
    return part;
}

int32_t mq_decode_kernel_count(const mq_cache* c, int32_t n_seqs, int32_t n_q_heads, int32_t max_q_per_seq,
                               int32_t max_seq_len) {
    if (c == nullptr || mq_decode_workspace_bytes(c, n_seqs, n_q_heads, max_q_per_seq, max_seq_len) == 0) return 0;
    const DecodePlan pl = plan_decode(c, n_seqs, n_q_heads, max_q_per_seq, max_seq_len);
    return pl.merge ? 2 : 1;
}

mq_status mq_decode_attn(const mq_cache* c, const void* q, mq_dtype q_dtype, int32_t n_seqs, int32_t n_q_heads,
                         int32_t total_q, int32_t max_q_per_seq, int32_t max_seq_len, const int32_t* block_table,
                         int32_t max_blocks_per_seq, const int32_t* seq_lens, const int32_t* n_q_per_seq,
                         float softmax_scale, float* out, float* lse, void* workspace, size_t workspace_bytes,
                         mq_stream stream) {
    if (c == nullptr || q == nullptr || block_table == nullptr || seq_lens == nullptr || n_q_per_seq == nullptr ||
        out == nullptr)
        return MQ_ERR_INVALID_ARG;
    if (n_seqs < 1 || n_seqs > 65535 || n_q_heads < 1 || n_q_heads % c->n_kv_heads != 0) return MQ_ERR_INVALID_ARG;
    if (max_q_per_seq < 1 || max_seq_len < max_q_per_seq || total_q < 1 || max_blocks_per_seq < 1)
        return MQ_ERR_INVALID_ARG;
    if (!(std::isfinite(softmax_scale))) return MQ_ERR_INVALID_ARG;
    if (q_dtype != MQ_F32 && q_dtype != MQ_BF16 && q_dtype != MQ_F16) return MQ_ERR_UNSUPPORTED;
    const int G = n_q_heads / c->n_kv_heads;
    if (G * max_q_per_seq > 64) return MQ_ERR_UNSUPPORTED;
    if ((long long)max_seq_len > (long long)max_blocks_per_seq * MQ_PAGE_TOKENS) return MQ_ERR_CAPACITY;
    if ((long long)c->n_kv_heads * ((G * max_q_per_seq + 7) / 8) > 65535) return MQ_ERR_UNSUPPORTED;
    if (reinterpret_cast<uintptr_t>(out) % 16 != 0) return MQ_ERR_INVALID_ARG;
    const size_t need = mq_decode_workspace_bytes(c, n_seqs, n_q_heads, max_q_per_seq, max_seq_len);
    if (workspace == nullptr || workspace_bytes < need || reinterpret_cast<uintptr_t>(workspace) % 256 != 0)
        return MQ_ERR_WORKSPACE;
    DevGuard guard(c->device);
    const DecodePlan pl = plan_decode(c, n_seqs, n_q_heads, max_q_per_seq, max_seq_len);
    return launch_decode_plan(c, pl, q, q_dtype, n_seqs, n_q_heads, total_q, max_q_per_seq, block_table,
                              max_blocks_per_seq, seq_lens, n_q_per_seq, softmax_scale, out, lse, workspace,
                              workspace_bytes, reinterpret_cast<cudaStream_t>(stream));
}

mq_status mq_prefill_attn(const mq_cache* c, const void* q, mq_dtype q_dtype, int32_t n_seqs, int32_t n_q_heads,
                          int32_t total_q, int32_t max_q_per_seq, int32_t max_seq_len, const int32_t* block_table,
                          int32_t max_blocks_per_seq, const int32_t* seq_lens, const int32_t* n_q_per_seq,
                          float softmax_scale, float* out, float* lse, mq_stream stream) {
    if (c == nullptr || q == nullptr || block_table == nullptr || seq_lens == nullptr || n_q_per_seq == nullptr ||
        out == nullptr)
        return MQ_ERR_INVALID_ARG;
    if (n_seqs < 1 || n_seqs > 65535 || n_q_heads < 1 || n_q_heads % c->n_kv_heads != 0) return MQ_ERR_INVALID_ARG;
    if (max_q_per_seq < 1 || max_seq_len < max_q_per_seq || total_q < 1 || max_blocks_per_seq < 1)
        return MQ_ERR_INVALID_ARG;
    if (!(std::isfinite(softmax_scale))) return MQ_ERR_INVALID_ARG;
    // q enters the tensor cores as fp16, exactly for BF16 and F16 input (F32 would lose bits)
    if (q_dtype != MQ_BF16 && q_dtype != MQ_F16) return MQ_ERR_UNSUPPORTED;
    const int G = n_q_heads / c->n_kv_heads;
    if (c->head_dim != 128 || G > 128 || 128 % G != 0) return MQ_ERR_UNSUPPORTED;
    if ((long long)max_seq_len > (long long)max_blocks_per_seq * MQ_PAGE_TOKENS) return MQ_ERR_CAPACITY;
    if (c->n_kv_heads > 65535) return MQ_ERR_UNSUPPORTED;
    if (prefill_smem_bytes() > (size_t)c->max_smem) return MQ_ERR_UNSUPPORTED;
    DevGuard guard(c->device);
    DecodeParams p{};
    p.pool = static_cast<const uint8_t*>(c->pool);
    p.n_kv_heads = c->n_kv_heads;
    p.n_blocks = c->n_blocks;
    p.q = q;
    p.q_dtype = (int)q_dtype;
    p.n_q_heads = n_q_heads;
    p.group = G;
    p.total_q = total_q;
    p.max_q = max_q_per_seq;
    p.n_seqs = n_seqs;
    p.block_table = block_table;
    p.max_blocks_per_seq = max_blocks_per_seq;
    p.seq_lens = seq_lens;
    p.n_q_per_seq = n_q_per_seq;
    p.scale_log2 = (float)((double)softmax_scale * 1.4426950408889634);
    p.out = out;
    p.lse = lse;
    p.err = c->err_word;
    p.causal = 1;
    const int tq = 128 / G;   // query tokens per tile
    const long long tiles = ((long long)max_q_per_seq + tq - 1) / tq;
    if (tiles > 0x7fffffffLL) return MQ_ERR_UNSUPPORTED;
    return launch_prefill(p, (int)tiles, reinterpret_cast<cudaStream_t>(stream)) == cudaSuccess ? MQ_OK
                                                                                              : MQ_ERR_CUDA;
}

mq_status mq_get_decode_config(const mq_cache* c, int32_t cls, mq_decode_config* cfg) {
    if (c == nullptr || cfg == nullptr || cls < 0 || cls > 2) return MQ_ERR_INVALID_ARG;
    *cfg = c->cfg[cls];
    return MQ_OK;
}

mq_status mq_set_decode_config(mq_cache* c, int32_t cls, const mq_decode_config* cfg) {
    if (c == nullptr || cfg == nullptr || cls < 0 || cls > 2) return MQ_ERR_INVALID_ARG;
    if (!config_valid(*cfg)) return MQ_ERR_INVALID_ARG;
    c->cfg[cls] = *cfg;
    return MQ_OK;
}

mq_status mq_device_status(const mq_cache* c, mq_stream stream) {
    if (c == nullptr) return MQ_ERR_INVALID_ARG;
    DevGuard guard(c->device);
    if (cudaStreamSynchronize(reinterpret_cast<cudaStream_t>(stream)) != cudaSuccess) return MQ_ERR_CUDA;
    unsigned v = 0;
    if (cudaMemcpy(&v, c->err_word, sizeof v, cudaMemcpyDeviceToHost) != cudaSuccess) return MQ_ERR_CUDA;
    if (v != 0) {
        const unsigned zero = 0;
        if (cudaMemcpy(c->err_word, &zero, sizeof zero, cudaMemcpyHostToDevice) != cudaSuccess) return MQ_ERR_CUDA;
        return MQ_ERR_DEVICE;
    }
    return MQ_OK;
}

}  // extern "C"
