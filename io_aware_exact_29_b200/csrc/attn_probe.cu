// attn_probe.cu -- a read-only device-memory stream, the denominator of the
// decode's roofline.
//
// The decode reads its KV cache once and writes almost nothing (ai6s.net
// article, section "标准注意力的致命伤不在算力，在搬运": attention is bound by
// data movement, and point 3 of "ops-transformer 里的 FlashAttention 做了什么
// 额外的事": only the real length of each sequence is read).  Its bound is the
// rate at which HBM can be READ, which a copy (half reads, half writes) does
// not measure.  This kernel reads a buffer once with 16-byte non-allocating
// loads, several in flight per thread, folds them with XOR so that no load can
// be dropped, and writes one word per CTA.
#include <cuda_runtime.h>

#include <cstdint>

#include "../../include/attn.h"

namespace attn {
namespace {

constexpr int kProbeThreads = 512;
constexpr int kProbeUnroll = 8;

__device__ __forceinline__ uint4 ld_stream(const uint4* p) {
    uint4 r;
    asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
                 : "l"(p));
    return r;
}

// Each CTA reads whole chunks of kProbeThreads * kProbeUnroll 16-byte words,
// CTAs stepping through the chunks with a stride of the grid size; the tail
// below one chunk is read one word per thread by the last CTAs.
__global__ void __launch_bounds__(kProbeThreads)
    attn_hbm_read_kernel(const uint4* __restrict__ src, unsigned long long n16,
                         unsigned* __restrict__ out) {
    constexpr unsigned long long kChunk = (unsigned long long)kProbeThreads * kProbeUnroll;
    const unsigned long long n_chunks = n16 / kChunk;
    uint32_t acc = 0;
    for (unsigned long long c = blockIdx.x; c < n_chunks; c += gridDim.x) {
        const uint4* base = src + c * kChunk + threadIdx.x;
        uint4 r[kProbeUnroll];
#pragma unroll
        for (int u = 0; u < kProbeUnroll; ++u) r[u] = ld_stream(base + u * kProbeThreads);
#pragma unroll
        for (int u = 0; u < kProbeUnroll; ++u) acc ^= r[u].x ^ r[u].y ^ r[u].z ^ r[u].w;
    }
    for (unsigned long long i = n_chunks * kChunk + (unsigned long long)blockIdx.x * kProbeThreads +
                                threadIdx.x;
         i < n16; i += (unsigned long long)gridDim.x * kProbeThreads) {
        const uint4 r = ld_stream(src + i);
        acc ^= r.x ^ r.y ^ r.z ^ r.w;
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) acc ^= __shfl_xor_sync(0xffffffffu, acc, o);
    __shared__ uint32_t warp_acc[kProbeThreads / 32];
    if ((threadIdx.x & 31) == 0) warp_acc[threadIdx.x >> 5] = acc;
    __syncthreads();
    if (threadIdx.x == 0) {
        uint32_t a = 0;
        for (int w = 0; w < kProbeThreads / 32; ++w) a ^= warp_acc[w];
        out[blockIdx.x] = a;
    }
}

}  // namespace
}  // namespace attn

extern "C" ATTN_API int attn_hbm_read_probe(const void* src, size_t bytes, unsigned* out,
                                            int n_ctas, void* stream) {
    if (!src || !out || bytes == 0 || (bytes & 15u) != 0 ||
        (reinterpret_cast<uintptr_t>(src) & 15u) != 0 || (reinterpret_cast<uintptr_t>(out) & 3u))
        return ATTN_ERR_INVALID_ARG;
    if (n_ctas <= 0 || n_ctas > (1 << 20)) return ATTN_ERR_INVALID_ARG;
    attn::attn_hbm_read_kernel<<<n_ctas, attn::kProbeThreads, 0,
                                 static_cast<cudaStream_t>(stream)>>>(
        static_cast<const uint4*>(src), (unsigned long long)(bytes / 16), out);
    return cudaGetLastError() == cudaSuccess ? ATTN_OK : ATTN_ERR_CUDA;
}
