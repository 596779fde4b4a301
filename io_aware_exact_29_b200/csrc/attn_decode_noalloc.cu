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
#include <cuda_runtime.h>

#include <mutex>

#include "../../include/attn.h"

namespace {

constexpr int kMaxDevices = 64;

// The scratch itself.  Every GPU that loads this library holds these
// ATTN_NOALLOC_SCRATCH_BYTES until the process exits.  Host code must not use
// the name as an address: on the host it is only a stand-in for the symbol.
static __device__ __align__(256) unsigned char g_decode_scratch[ATTN_NOALLOC_SCRATCH_BYTES];

std::mutex g_mu;
void* g_scratch_addr[kMaxDevices] = {nullptr};

// Device address of the scratch on the current device, looked up once per
// device (with that device current) and cached.
int scratch_address(void** out) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return ATTN_ERR_CUDA;
    std::lock_guard<std::mutex> lk(g_mu);
    if (!g_scratch_addr[dev]) {
        void* ptr = nullptr;
        if (cudaGetSymbolAddress(&ptr, g_decode_scratch) != cudaSuccess || ptr == nullptr)
            return ATTN_ERR_CUDA;
        g_scratch_addr[dev] = ptr;
    }
    *out = g_scratch_addr[dev];
    return ATTN_OK;
}

}  // namespace

extern "C" ATTN_API int attn_fwd_varlen_kvcache_noalloc(
    const void* q, const void* k_cache, const void* v_cache, const int* cu_seqlens_k,
    const int* seqlens_k, int max_seqlen_k, int cache_slots, void* o, float* lse, int B, int Hq,
    int Hkv, int Nq, int d, float scale, int causal, int dtype, int split_keys, void* stream) {
    const size_t need =
        attn_decode_workspace_bytes(B, Hq, Hkv, Nq, d, max_seqlen_k, split_keys);
    if (need == 0) return ATTN_ERR_INVALID_ARG;
    if (need > (size_t)ATTN_NOALLOC_SCRATCH_BYTES) return ATTN_ERR_WORKSPACE;
    void* scratch = nullptr;
    const int st = scratch_address(&scratch);
    if (st != ATTN_OK) return st;
    // The decode call clears the split counters inside the scratch with an
    // asynchronous memset on `stream` before its kernel, so whatever an
    // earlier call left there does not matter.
    return attn_fwd_varlen_kvcache(q, k_cache, v_cache, cu_seqlens_k, seqlens_k, max_seqlen_k,
                                   cache_slots, o, lse, B, Hq, Hkv, Nq, d, scale, causal, dtype,
                                   scratch, (size_t)ATTN_NOALLOC_SCRATCH_BYTES, split_keys,
                                   stream);
}
