// attn_decode_noalloc.cu -- the KV-cache decode for callers that cannot
// allocate device memory.
//
// attn_fwd_varlen_kvcache needs a workspace for its split-K partial results,
// which the caller normally allocates.  Some callers have no way to do that:
// code embedded in a host program whose device memory is planned and owned by
// someone else (no allocator handle is exposed to it), or a latency-critical
// decode loop that must not call cudaMalloc, which can synchronise the whole
// device.  For them this file keeps one fixed scratch area in a file-scope
// __device__ array and passes it as the workspace; nothing here calls
// cudaMalloc, cudaFree or any allocating routine.
#include <cuda.h>
#include <cuda_runtime.h>

#include <mutex>

#include "../../include/attn.h"
#include "attn_internal.h"

namespace {

constexpr int kMaxDevices = 64;

// The scratch itself.  Every GPU that loads this library holds these
// ATTN_NOALLOC_SCRATCH_BYTES until the process exits.  Host code must not use
// the name as an address: on the host it is only a stand-in for the symbol.
static __device__ __align__(256) unsigned char g_decode_scratch[ATTN_NOALLOC_SCRATCH_BYTES];

typedef CUresult (*CtxGetCurrentFn)(CUcontext*);
typedef CUresult (*CtxGetIdFn)(CUcontext, unsigned long long*);

std::mutex g_mu;
void* g_scratch_addr[kMaxDevices] = {nullptr};
unsigned long long g_scratch_ctx[kMaxDevices] = {0};  // context the address belongs to
CtxGetCurrentFn g_ctx_current = nullptr;
CtxGetIdFn g_ctx_id = nullptr;
bool g_ctx_fns_tried = false;

// Unique id of the context current on this thread (0 when it cannot be read).
// A device reset destroys the primary context and the next one gets a new id,
// so a cached address of the scratch is only reused under the same id.
unsigned long long current_context_id() {
    if (!g_ctx_fns_tried) {
        g_ctx_fns_tried = true;
        void* f = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &f, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            g_ctx_current = reinterpret_cast<CtxGetCurrentFn>(f);
        f = nullptr;
        if (cudaGetDriverEntryPoint("cuCtxGetId", &f, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            g_ctx_id = reinterpret_cast<CtxGetIdFn>(f);
    }
    if (!g_ctx_current || !g_ctx_id) return 0;
    CUcontext ctx = nullptr;
    unsigned long long id = 0;
    if (g_ctx_current(&ctx) != CUDA_SUCCESS || ctx == nullptr) return 0;
    if (g_ctx_id(ctx, &id) != CUDA_SUCCESS) return 0;
    return id;
}

// Device address of the scratch on the current device, looked up with that
// device current (cudaGetSymbolAddress, which allocates nothing) on the
// first call and again whenever the current context is not the one the
// cached address was taken in (after a device reset the module is loaded
// anew and the array may sit elsewhere).
int scratch_address(void** out) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return ATTN_ERR_CUDA;
    std::lock_guard<std::mutex> lk(g_mu);
    const unsigned long long ctx = current_context_id();
    if (!g_scratch_addr[dev] || ctx == 0 || ctx != g_scratch_ctx[dev]) {
        void* ptr = nullptr;
        if (cudaGetSymbolAddress(&ptr, g_decode_scratch) != cudaSuccess || ptr == nullptr)
            return ATTN_ERR_CUDA;
        g_scratch_addr[dev] = ptr;
        // the lookup makes the device's primary context current if no context was
        g_scratch_ctx[dev] = ctx != 0 ? ctx : current_context_id();
    }
    *out = g_scratch_addr[dev];
    return ATTN_OK;
}

}  // namespace

extern "C" ATTN_API int attn_fwd_varlen_kvcache_noalloc(
    const void* q, const void* k_cache, const void* v_cache, const int* cu_seqlens_k,
    const int* seqlens_k, int max_seqlen_k, int cache_slots, void* o, float* lse, int B, int Hq,
    int Hkv, int Nq, int d, float scale, int causal, int dtype, int split_keys, void* stream) {
    // the same argument checks, in the same order, as the workspace entry
    // point, so both return the same codes for the same bad arguments
    const int arg_st = attn::decode_check_args(q, k_cache, v_cache, cu_seqlens_k, seqlens_k,
                                               max_seqlen_k, cache_slots, o, lse, B, Hq, Hkv,
                                               Nq, d, scale, dtype, split_keys);
    if (arg_st != ATTN_OK) return arg_st;
    const size_t need =
        attn_decode_workspace_bytes(B, Hq, Hkv, Nq, d, max_seqlen_k, split_keys);
    if (need > (size_t)ATTN_NOALLOC_SCRATCH_BYTES) return ATTN_ERR_WORKSPACE;
    void* scratch = nullptr;
    const int st = scratch_address(&scratch);
    if (st != ATTN_OK) return st;
    // Whatever an earlier call left in the scratch does not matter: the parts
    // that must start at zero (the split counters) are cleared on `stream`
    // before the decode kernel, by a memset or by the plan kernel.
    return attn_fwd_varlen_kvcache(q, k_cache, v_cache, cu_seqlens_k, seqlens_k, max_seqlen_k,
                                   cache_slots, o, lse, B, Hq, Hkv, Nq, d, scale, causal, dtype,
                                   scratch, (size_t)ATTN_NOALLOC_SCRATCH_BYTES, split_keys,
                                   stream);
}
