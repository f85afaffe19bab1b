// The split-K merge (K4) and the decode launch sequence.
//
// What the merge computes (the deep dive on magnitudedev/magnitude at blog.123qwe.co.kr,
// section 5: the decode attention unit attention_decode_k8v4, whose sequence splits are
// combined by log-sum-exp): the decode kernel (mq_decode_small.cu) publishes one partial
// per CTA, O = sum_t 2^(z_t - m) v_t, m = max_t z_t (log2 units), l = sum_t 2^(z_t - m)
// over the CTA's tokens.  merge_kernel combines a unit's partials over one fixed binary
// tree over the CTA index:
//     node(lv, i) = merge(node(lv-1, 2i), node(lv-1, 2i+1)),  merge = the log-sum-exp
//     combination (m = max, O and l rescaled by 2^(m_side - m) and added),
// a node whose right child starts past the last CTA passes its left child through; the
// root gives out = O / l and lse = (m + log2 l) ln 2.  Where the CTAs hold aligned
// power-of-two runs of leaves (the classes of up to 8 rows), each partial is a node of
// the fixed tree over the unit's leaves and this tree is that tree's upper part.
// Launched right after the decode kernel as a programmatic dependent launch: its CTAs may
// start while the decode CTAs finish, and wait (griddepcontrol.wait) until all of them
// have completed and their partials are visible.
#include "mq_decode_common.cuh"

namespace mq {

// merge_kernel: one CTA covers 128 float4 elements of one unit's [ROWS][D] result; its
// threads are 128 x (leaf groups of 8 CTA partials).  Thread (e, j) loads the 8 partials
// of group j for element e (O, m, l) at once and evaluates that aligned level-3 subtree;
// the group results meet in shared memory, where thread (e, 0) evaluates the levels above.
// Every node is merge(left, right) with merge_coef / merge_val (the decode kernel's own
// merge arithmetic), and a node without a right child passes its left child through.
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

// One leaf group's subtree (levels 1..3 over the 8 partials from slot 8g) for element e4.
template <int D, int ROWS>
__device__ __forceinline__ MergeOut fold_group(const float* go0, const float* gml0, int g, int n_splits, int e4,
                                               int r) {
    float4 v[8];
    float vm[8], vl[8];
#pragma unroll
    for (int u = 0; u < 8; u++) {
        const int sidx = 8 * g + u;
        const bool slot = sidx < n_splits;
        v[u] = slot ? __ldcg(reinterpret_cast<const float4*>(go0 + (size_t)sidx * ROWS * D) + e4)
                    : make_float4(0.f, 0.f, 0.f, 0.f);
        vm[u] = slot ? __ldcg(gml0 + (size_t)sidx * 2 * ROWS + r) : -INFINITY;
        vl[u] = slot ? __ldcg(gml0 + (size_t)sidx * 2 * ROWS + ROWS + r) : 0.0f;
    }
#pragma unroll
    for (int lv = 1; lv <= 3; lv++) {
#pragma unroll
        for (int u = 0; u < (8 >> lv); u++) {
            const int idx = ((8 * g) >> lv) + u;   // node (lv, idx)
            const bool has_right = (2 * idx + 1) * (1 << (lv - 1)) < n_splits;
            const MergeOut mo =
                merge_pair(v[2 * u], vm[2 * u], vl[2 * u], v[2 * u + 1], vm[2 * u + 1], vl[2 * u + 1], has_right);
            v[u] = mo.o;
            vm[u] = mo.m;
            vl[u] = mo.l;
        }
    }
    return MergeOut{v[0], vm[0], vl[0]};
}
__device__ __forceinline__ MergeOut merge_nodes(const MergeOut& a, const MergeOut& c) {
    return merge_pair(a.o, a.m, a.l, c.o, c.m, c.l, true);
}

// merge_flat_kernel: the merge after a flat decode grid, one CTA of 128 threads per 128
// float4 elements of a unit's result.  The unit's split count follows from the launch's
// leaves per CTA, found again here from every sequence's length (flat_lpc) before the
// decode grid ends.  Thread e folds the unit's leaf groups of 8 partials left to right
// and keeps the pending left nodes of the levels above (group levels 0..2): each group
// result is merged with the pending nodes of the low set bits of its index, and at the
// end the pending nodes of n_groups' set bits are merged from the lowest up.  That is
// the same tree merge_kernel evaluates (a node whose right child starts past the last
// partial passes its left child through), with one thread group and no shared memory.
template <int D, int ROWS>
__global__ void __launch_bounds__(128) merge_flat_kernel(const DecodeParams p) {
    __shared__ int s_lpc;
    // the next kernel on the stream may be scheduled now (it reads no page and writes no
    // partial before its own griddepcontrol.wait, which returns once this grid completes)
    if (threadIdx.x == 0) asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    if (threadIdx.x < 32) {
        SeqShape first;
        const int lpc = flat_lpc(p, ROWS, first);
        if (threadIdx.x == 0) s_lpc = lpc;
    }
    __syncthreads();
    const int b = blockIdx.z, hk = blockIdx.y / p.n_rb, rb = blockIdx.y % p.n_rb;
    const int L = seq_len_of(p, b), nq = seq_nq_of(p, b);
    if (nq < 1 || nq > p.max_q || nq > L ||
        (long long)L + (long long)p.bt_col * kPageTokens > (long long)p.max_blocks_per_seq * kPageTokens)
        return;
    const int rows_b = p.group * nq, row0 = rb * ROWS;
    if (row0 >= rows_b) return;
    const int n_chunks = (L + kChunkTokens - 1) / kChunkTokens;
    const int n_splits = min((n_chunks + s_lpc * p.node_chunks - 1) / (s_lpc * p.node_chunks), p.split_stride);
    if (n_splits <= 1) return;   // the decode kernel wrote this unit's output itself
    const int n_groups = min((n_splits + 7) >> 3, 8);
    const int e4 = blockIdx.x * 128 + threadIdx.x;   // < ROWS * D / 4: the grid covers it exactly
    const int r = (4 * e4) / D, c4 = e4 % (D / 4);   // the element's row and float4 column
    const int rr = row0 + r, jq = rr / p.group, hq = rr % p.group;
    int qoff = 0;
    for (int i = 0; i < b; i++) qoff += min(max(seq_nq_of(p, i), 0), p.max_q);
    const size_t pidx = ((size_t)(b * p.n_kv_heads + hk) * p.n_rb + rb);
    const float* gml0 = p.part_ml + pidx * p.split_stride * (size_t)(2 * ROWS);
    const float* go0 = p.part_o + pidx * p.split_stride * (size_t)(ROWS * D);
    asm volatile("griddepcontrol.wait;" ::: "memory");
    MergeOut s0{}, s1{}, s2{}, s3{};
    for (int g = 0; g < n_groups; g++) {
        MergeOut c = fold_group<D, ROWS>(go0, gml0, g, n_splits, e4, r);
        if (g & 1) {
            c = merge_nodes(s0, c);
            if (g & 2) {
                c = merge_nodes(s1, c);
                if (g & 4)
                    s3 = merge_nodes(s2, c);
                else
                    s2 = c;
            } else {
                s1 = c;
            }
        } else {
            s0 = c;
        }
    }
    MergeOut root = s3;   // n_groups == 8: the counter closed the whole tree
    if (n_groups < 8) {
        bool have = false;
        if (n_groups & 1) {
            root = s0;
            have = true;
        }
        if (n_groups & 2) {
            root = have ? merge_nodes(s1, root) : s1;
            have = true;
        }
        if (n_groups & 4) root = have ? merge_nodes(s2, root) : s2;
    }
    // out = O / l and lse for a real row
    if (r >= min(ROWS, rows_b - row0)) return;
    const long long qrow = (long long)qoff + jq;
    if (qrow >= p.total_q) return;
    float4 o = root.o;
    o.x = __fdiv_rn(o.x, root.l);
    o.y = __fdiv_rn(o.y, root.l);
    o.z = __fdiv_rn(o.z, root.l);
    o.w = __fdiv_rn(o.w, root.l);
    const size_t orow = (size_t)qrow * p.n_q_heads + (size_t)hk * p.group + hq;
    reinterpret_cast<float4*>(p.out + orow * D)[c4] = o;
    if (c4 == 0 && p.lse != nullptr) p.lse[orow] = __fmul_rn(__fadd_rn(root.m, log2f(root.l)), 0.69314718055994531f);
}

size_t decode_smem_bytes(int head_dim, int rows, int groups, int stages) {
    return small_smem_bytes(head_dim, rows, groups, stages);
}

int decode_ctas_per_sm(int head_dim, int rows) { return small_ctas_per_sm(head_dim, rows); }

cudaError_t decode_prepare(int head_dim, int rows, int groups, size_t smem) {
    return small_prepare(head_dim, rows, groups, smem);
}

// The merge as a programmatic dependent launch on the same stream (after a decode launch
// in which some unit's tree is not finished by one CTA): merge_kernel after a (split,
// unit) grid, one thread group per leaf group of 8 partials; merge_flat_kernel after a
// flat grid.
template <int D, int ROWS>
static cudaError_t launch_merge(const DecodeParams& p, dim3 grid, int max_splits, bool flat, cudaStream_t st) {
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = dim3((unsigned)((ROWS * D / 4 + 127) / 128), grid.y, grid.z);
    cfg.blockDim = dim3(flat ? 128u : (unsigned)(128 * ((max_splits + 7) / 8)));
    cfg.dynamicSmemBytes = 0;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return flat ? cudaLaunchKernelEx(&cfg, merge_flat_kernel<D, ROWS>, p)
                : cudaLaunchKernelEx(&cfg, merge_kernel<D, ROWS>, p);
}

// The decode kernel of the row class, then (when some unit needs it) the merge.
cudaError_t launch_decode(const DecodeParams& p, int head_dim, int rows, int groups, int max_splits, int flat_ctas,
                          bool merge, size_t smem, cudaStream_t st) {
    if (max_splits < 1 || max_splits > kMaxSplits || p.split_stride < max_splits) return cudaErrorInvalidValue;
    const dim3 grid((unsigned)max_splits, (unsigned)(p.n_kv_heads * p.n_rb), (unsigned)p.n_seqs);
    const cudaError_t e =
        small_launch(p, head_dim, rows, groups, flat_ctas > 0 ? dim3((unsigned)flat_ctas) : grid, smem, st);
    if (e != cudaSuccess || !merge) return e;
#define MQ_MERGE(DD, RR) \
    if (head_dim == DD && rows == RR) return launch_merge<DD, RR>(p, grid, max_splits, flat_ctas > 0, st);
    MQ_MERGE(128, 4) MQ_MERGE(128, 8) MQ_MERGE(128, 16) MQ_MERGE(128, 32) MQ_MERGE(256, 4) MQ_MERGE(256, 8)
    MQ_MERGE(256, 16)
#undef MQ_MERGE
    return cudaErrorInvalidValue;
}

}  // namespace mq
