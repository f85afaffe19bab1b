// mq_decode_attn_static: decode attention whose scratch is a fixed array inside the
// library instead of a caller-provided workspace.
//
// Who needs it: a caller that cannot hand the library a device allocation at decode
// time.  A serving process that reserves nearly all free HBM for its KV pool up front
// has nothing left to allocate from later, and an allocation that succeeds may still
// fragment that reservation; a plain C host program has no caching allocator to draw a
// workspace from; and cudaMalloc / cudaFree may synchronize the device, which a decode
// loop that keeps several steps in flight cannot afford.  This entry point allocates
// nothing: its scratch is a file-scope __device__ array of fixed size, present on every
// device once the library's module is loaded there.
//
// The decode arithmetic, launch planning and argument checks are those of
// mq_decode_attn, which this entry point calls with the array as its workspace.
#include <cstddef>
#include <cstdint>
#include <mutex>

#include <cuda.h>
#include <cuda_runtime.h>

#include "mq.h"
#include "mq_host.h"

namespace {

constexpr size_t kScratchBytes = MQ_DECODE_STATIC_SCRATCH_BYTES;
constexpr int kMaxDevices = 64;

// The scratch itself (one copy per device): the CTA partials of the split reduction,
// each written before it is read, so nothing has to start at zero.
static __device__ __align__(256) unsigned char g_decode_scratch[kScratchBytes];

std::mutex g_scratch_mu;
void* g_scratch_addr[kMaxDevices] = {};
unsigned long long g_scratch_ctx[kMaxDevices] = {};   // context the address was read in

// Identity of the context current on this thread, read through the driver entry points
// that the runtime hands out (the library does not link the driver library itself);
// 0 when it cannot be read.  Called with g_scratch_mu held.
unsigned long long current_context_id() {
    using GetCurrent = CUresult (*)(CUcontext*);
    using GetId = CUresult (*)(CUcontext, unsigned long long*);
    static GetCurrent get_current = nullptr;
    static GetId get_id = nullptr;
    static bool looked_up = false;
    if (!looked_up) {
        looked_up = true;
        void* f = nullptr;
        cudaDriverEntryPointQueryResult q{};
        if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &f, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            get_current = reinterpret_cast<GetCurrent>(f);
        f = nullptr;
        if (cudaGetDriverEntryPoint("cuCtxGetId", &f, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            get_id = reinterpret_cast<GetId>(f);
    }
    if (get_current == nullptr || get_id == nullptr) return 0;
    CUcontext ctx = nullptr;
    unsigned long long id = 0;
    if (get_current(&ctx) != CUDA_SUCCESS || ctx == nullptr || get_id(ctx, &id) != CUDA_SUCCESS) return 0;
    return id;
}

// Device address of this device's scratch, looked up with that device current (the
// caller makes it current) on the first call, and again whenever the device's context
// has changed since (a cudaDeviceReset ends the context the address belonged to; the
// module, and with it the array, is loaded afresh in the new one).
mq_status scratch_address(int dev, void** out) {
    if (dev < 0 || dev >= kMaxDevices) return MQ_ERR_UNSUPPORTED;
    std::lock_guard<std::mutex> lock(g_scratch_mu);
    const unsigned long long ctx = current_context_id();
    if (g_scratch_addr[dev] == nullptr || ctx != g_scratch_ctx[dev]) {
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_decode_scratch) != cudaSuccess || p == nullptr) return MQ_ERR_CUDA;
        g_scratch_addr[dev] = p;
        g_scratch_ctx[dev] = ctx;
    }
    *out = g_scratch_addr[dev];
    return MQ_OK;
}

}  // namespace

extern "C" mq_status mq_decode_attn_static(const mq_cache* c, const void* q, mq_dtype q_dtype, int32_t n_seqs,
                                           int32_t n_q_heads, int32_t total_q, int32_t max_q_per_seq,
                                           int32_t max_seq_len, const int32_t* block_table,
                                           int32_t max_blocks_per_seq, const int32_t* seq_lens,
                                           const int32_t* n_q_per_seq, float softmax_scale, float* out, float* lse,
                                           mq_stream stream) {
    if (c == nullptr) return MQ_ERR_INVALID_ARG;
    // a shape whose scratch would not fit the fixed array is refused before anything runs
    const size_t need = mq_decode_workspace_bytes(c, n_seqs, n_q_heads, max_q_per_seq, max_seq_len);
    if (need > kScratchBytes) return MQ_ERR_WORKSPACE;
    mq::DevGuard guard(c->device);
    void* scratch = nullptr;
    const mq_status st = scratch_address(c->device, &scratch);
    if (st != MQ_OK) return st;
    return mq_decode_attn(c, q, q_dtype, n_seqs, n_q_heads, total_q, max_q_per_seq, max_seq_len, block_table,
                          max_blocks_per_seq, seq_lens, n_q_per_seq, softmax_scale, out, lse, scratch, kScratchBytes,
                          stream);
}
