// mq_kv_export: tokens of the paged cache read back in the codec's canonical form.
//
// The codec (the deep dive on magnitudedev/magnitude at blog.123qwe.co.kr, section 5:
// "Key 8-bit, Value 4-bit, group 32, f16 scale") stores per (token, kv-head) the int8
// K codes with one fp16 scale, and per 32-channel group the int4 V codes with one fp16
// scale, the V codes two per byte.  The page layout (mq_device.cuh) keeps the V codes
// of one channel for the 8 tokens of a record in one 32-bit word, for the decode
// kernel's tensor cores.  This kernel undoes only that arrangement: it copies codes and
// scales unchanged and packs each token's V codes channel by channel, channel 2j in the
// low nibble of byte j and channel 2j + 1 in the high nibble.  No arithmetic on values.
//
// Work split: one warp per (exported token, kv-head); lane l handles channels
// l * D/32 .. l * D/32 + D/32 - 1 (an even count, so each lane owns whole bytes).
#include "mq_device.cuh"
#include "mq_kernels.h"

namespace mq {

template <int D>
__global__ void __launch_bounds__(256) export_kernel(const ExportParams p) {
    constexpr int CPL = D / 32;   // channels per lane
    const long long wid = (long long)blockIdx.x * 8 + (threadIdx.x >> 5);
    const int lane = threadIdx.x & 31;
    if (wid >= (long long)p.n_tokens * p.n_kv_heads) return;
    const int t = (int)(wid / p.n_kv_heads), h = (int)(wid % p.n_kv_heads);
    // the sequence whose cu_tok range holds t (binary search: cu_tok is ascending)
    int lo = 0, hi = p.n_seqs - 1;
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (__ldg(p.cu_tok + mid) <= t) lo = mid;
        else hi = mid - 1;
    }
    const int b = lo;
    const int c0 = __ldg(p.cu_tok + b), c1 = __ldg(p.cu_tok + b + 1);
    int8_t* kc = p.k_codes + ((size_t)t * p.n_kv_heads + h) * D;
    uint8_t* vp = p.v_packed + ((size_t)t * p.n_kv_heads + h) * (D / 2);
    uint16_t* ks = p.k_scales + (size_t)t * p.n_kv_heads + h;
    uint16_t* vs = p.v_scales + ((size_t)t * p.n_kv_heads + h) * (D / 32);
    const long long pos = (long long)__ldg(p.start_pos + b) + (t - c0);
    bool bad = t < c0 || t >= c1 || pos < 0 || pos >= (long long)p.max_blocks_per_seq * kPageTokens;
    long long blk = 0;
    if (!bad) {
        blk = __ldg(p.block_table + (long long)b * p.max_blocks_per_seq + pos / kPageTokens);
        bad = blk < 0 || blk >= p.n_blocks;
    }
    if (bad) {
        // nothing is read; the token's outputs are zero and the error word is set
        if (lane == 0) atomicOr(p.err, kErrBadPosition);
#pragma unroll
        for (int i = 0; i < CPL; i++) kc[lane * CPL + i] = 0;
#pragma unroll
        for (int i = 0; i < CPL / 2; i++) vp[lane * (CPL / 2) + i] = 0;
        if (lane == 0) *ks = 0;
        if (lane < D / 32) vs[lane] = 0;
        return;
    }
    const uint8_t* page = p.pool + ((size_t)blk * p.n_kv_heads + h) * page_bytes(D);
    const int tau = (int)(pos % kPageTokens);
#pragma unroll
    for (int i = 0; i < CPL; i++) kc[lane * CPL + i] = (int8_t)page[k_code_byte(D, tau, lane * CPL + i)];
    const int sh = v_nibble_bit(tau);
#pragma unroll
    for (int i = 0; i < CPL / 2; i++) {
        const int c = lane * CPL + 2 * i;
        const uint32_t w0 = *reinterpret_cast<const uint32_t*>(page + v_word_byte(D, tau, c));
        const uint32_t w1 = *reinterpret_cast<const uint32_t*>(page + v_word_byte(D, tau, c + 1));
        vp[c / 2] = (uint8_t)(((w0 >> sh) & 0xFu) | (((w1 >> sh) & 0xFu) << 4));
    }
    if (lane == 0) *ks = *reinterpret_cast<const uint16_t*>(page + k_scale_byte(D, tau));
    if (lane < D / 32) vs[lane] = *reinterpret_cast<const uint16_t*>(page + v_scale_byte(D, tau, lane));
}

cudaError_t launch_export(const ExportParams& p, int head_dim, cudaStream_t st) {
    const long long warps = (long long)p.n_tokens * p.n_kv_heads;
    const dim3 grid((unsigned)((warps + 7) / 8));
    if (head_dim == 128) export_kernel<128><<<grid, 256, 0, st>>>(p);
    else if (head_dim == 256) export_kernel<256><<<grid, 256, 0, st>>>(p);
    else return cudaErrorInvalidValue;
    return cudaGetLastError();
}

}  // namespace mq
