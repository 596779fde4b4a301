// attn_api.cu -- the C ABI declared in include/attn.h: argument validation,
// tile/split selection, TMA tensor-map encoding and kernel launches.  No
// allocation, no synchronisation (except attn_get_device_error, which is
// documented to synchronise).
#include <cuda.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <atomic>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <mutex>

#include "../../include/attn.h"
#include "attn_internal.h"

namespace attn {

// One device error word per device that loads the library; kernels record
// the first bounded wait that ran out here.
static __device__ unsigned g_device_error = 0u;

namespace {

constexpr int kMaxDevices = 64;
constexpr unsigned long long kDefaultLimitNs = 2000000000ull;  // 2 s per wait

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

std::mutex g_mu;
EncodeTiledFn g_encode = nullptr;
int g_dev_state[kMaxDevices] = {0};  // 0 unknown, 1 supported, -1 unsupported
unsigned* g_err_addr[kMaxDevices] = {nullptr};
int g_sm_count[kMaxDevices] = {0};

EncodeTiledFn encode_fn() {
    std::lock_guard<std::mutex> lk(g_mu);
    if (!g_encode) {
        void* fn = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) !=
                cudaSuccess ||
            q != cudaDriverEntryPointSuccess)
            return nullptr;
        g_encode = reinterpret_cast<EncodeTiledFn>(fn);
    }
    return g_encode;
}

// Current device: 1 if it is a compute-capability 10.0 part, -1 if not, 0 on error.
int check_device(int* dev_out) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return 0;
    *dev_out = dev;
    std::lock_guard<std::mutex> lk(g_mu);
    if (g_dev_state[dev] == 0) {
        int major = 0, minor = 0;
        if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
            cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess)
            return 0;
        g_dev_state[dev] = (major == 10 && minor == 0) ? 1 : -1;
        if (g_dev_state[dev] == 1) {
            void* addr = nullptr;
            if (cudaGetSymbolAddress(&addr, g_device_error) != cudaSuccess) {
                g_dev_state[dev] = 0;
                return 0;
            }
            g_err_addr[dev] = static_cast<unsigned*>(addr);
            if (cudaDeviceGetAttribute(&g_sm_count[dev], cudaDevAttrMultiProcessorCount, dev) !=
                    cudaSuccess ||
                g_sm_count[dev] <= 0) {
                g_dev_state[dev] = 0;
                return 0;
            }
        }
    }
    return g_dev_state[dev];
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Tiled map over a row-major tensor whose dims are given innermost first;
// strides in bytes for dims 1..rank-1; 128-byte swizzle; zero fill outside.
bool encode_map(CUtensorMap* m, int dtype, const void* base, int rank, const uint64_t* dims,
                const uint64_t* strides, const uint32_t* box) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return false;
    cuuint64_t gdim[5], gstride[4];
    cuuint32_t bdim[5], estride[5];
    for (int i = 0; i < rank; ++i) {
        gdim[i] = dims[i];
        bdim[i] = box[i];
        estride[i] = 1;
    }
    for (int i = 0; i < rank - 1; ++i) gstride[i] = strides[i];
    const CUtensorMapDataType dt =
        dtype == ATTN_BF16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT16;
    CUresult r = fn(m, dt, (cuuint32_t)rank, const_cast<void*>(base), gdim, gstride, bdim, estride,
                    CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                    CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

// [B, N, H, d] tensor, box of 64 columns x 1 head x 128 rows x 1 batch.
bool map_bnhd(CUtensorMap* m, int dtype, const void* base, int B, int N, int H, int d) {
    const uint64_t dims[4] = {(uint64_t)d, (uint64_t)H, (uint64_t)N, (uint64_t)B};
    const uint64_t strides[3] = {(uint64_t)d * 2, (uint64_t)H * d * 2, (uint64_t)N * H * d * 2};
    const uint32_t box[4] = {64, 1, 128, 1};
    return encode_map(m, dtype, base, 4, dims, strides, box);
}

// V of a KV cache [slots, Hkv, d] for the tensor-core decode, seen as
// {64 columns, slot, 64-column block, head} (the third dimension's stride,
// 128 bytes, is smaller than the second's: the map walks the same memory in
// another order).  One box of `rows` slots lands as [64-column block][row]
// [128 B]: a run of cache rows with all d columns.
bool map_v_runs(CUtensorMap* m, int dtype, const void* base, uint64_t slots, int Hkv, int d,
                int rows) {
    const uint64_t dims[4] = {64, slots, (uint64_t)d / 64, (uint64_t)Hkv};
    const uint64_t strides[3] = {(uint64_t)Hkv * d * 2, 128, (uint64_t)d * 2};
    const uint32_t box[4] = {64, (uint32_t)rows, (uint32_t)d / 64, 1};
    return encode_map(m, dtype, base, 4, dims, strides, box);
}

constexpr BlockMask kNoBlockMask{nullptr, 0, 0, 0};

int fwd_common(const void* q, const void* k, const void* v, void* o, float* lse, int B, int Hq,
               int Hkv, int Nq, int Nk, int d, float scale, int causal, int dtype,
               const int* seqlens_k, void* stream, int inject, unsigned long long limit_ns,
               int window_left, const BlockMask& bmask) {
    if (window_left < -1) return ATTN_ERR_INVALID_ARG;
    if (bmask.m && (bmask.sb < 0 || bmask.sh < 0 || bmask.srow < (Nk + 127) / 128))
        return ATTN_ERR_INVALID_ARG;
    if (dtype != ATTN_BF16 && dtype != ATTN_FP16) return ATTN_ERR_UNSUPPORTED;
    if (d != 64 && d != 128) return ATTN_ERR_UNSUPPORTED;
    if (B <= 0 || Hq <= 0 || Hkv <= 0 || Nq <= 0 || Nk < 0 || Hq % Hkv != 0)
        return ATTN_ERR_INVALID_ARG;
    if (B > 65535 || Hq > 65535) return ATTN_ERR_INVALID_ARG;
    if (!(scale > 0.f) || !std::isfinite(scale)) return ATTN_ERR_INVALID_ARG;
    if (!q || !o || !lse || !aligned16(q) || !aligned16(o) || !aligned16(lse))
        return ATTN_ERR_INVALID_ARG;
    if (Nk > 0 && (!k || !v || !aligned16(k) || !aligned16(v))) return ATTN_ERR_INVALID_ARG;
    if (seqlens_k && (reinterpret_cast<uintptr_t>(seqlens_k) & 3u)) return ATTN_ERR_INVALID_ARG;
    int dev = 0;
    const int st = check_device(&dev);
    if (st == 0) return ATTN_ERR_CUDA;
    if (st < 0) return ATTN_ERR_UNSUPPORTED;

    FwdMaps maps;
    // With no keys at all the K/V maps are never read; point them at Q.
    const void* kb = Nk > 0 ? k : q;
    const void* vb = Nk > 0 ? v : q;
    const int nk_map = Nk > 0 ? Nk : Nq;
    const int hkv_map = Nk > 0 ? Hkv : Hq;
    if (!map_bnhd(&maps.q, dtype, q, B, Nq, Hq, d) ||
        !map_bnhd(&maps.k, dtype, kb, B, nk_map, hkv_map, d) ||
        !map_bnhd(&maps.v, dtype, vb, B, nk_map, hkv_map, d) ||
        !map_bnhd(&maps.o, dtype, o, B, Nq, Hq, d))
        return ATTN_ERR_INVALID_ARG;

    FwdParams p{};
    p.B = B;
    p.Hq = Hq;
    p.Hkv = Hkv;
    p.Nq = Nq;
    p.Nk = Nk;
    p.G = Hq / Hkv;
    p.n_qtiles = (Nq + 127) / 128;
    p.causal = causal ? 1 : 0;
    p.scale_log2 = scale * 1.4426950408889634f;
    p.seqlens_k = Nk > 0 ? seqlens_k : nullptr;
    p.window_left = window_left;
    p.bmask = bmask;
    // causal row tiles differ in cost (tile t sees about t key tiles): launch
    // them in decreasing cost, in bands of heads whose K/V fit in L2 together
    // (a sliding window evens the costs out and keeps the head-major order)
    p.band = 0;
    if (causal && window_left < 0 && Nk > 0) {
        const long long units = (long long)B * Hq * ((Nq + 255) / 256);
        // K and V bytes of one query head, shared by the G heads of its group
        const long long per_head = 4LL * Nk * d / (Hq / Hkv);
        const long long fit = (48LL << 20) / (per_head > 0 ? per_head : 1);
        if (units <= 0x7fffffffLL)
            p.band = (int)std::min<long long>((long long)B * Hq, std::max<long long>(8, fit));
    }
    // work units of 256 query rows.  Short units of equal cost (no causal,
    // window or block mask, at most 4096 keys) go to the persistent kernel:
    // one CTA per SM takes every n_ctas-th unit, overlapping a unit's last
    // tiles and output with the next unit's loads (measured: BERT-large
    // +9%, 1024 keys +4-11%, 4096 keys +-1% over one CTA per unit).  Causal
    // and block-sparse units differ in cost, and a static split leaves SMs
    // idle at the end (-9 to -15% measured for causal); long units gain
    // nothing from the overlap (-4% at 16384 keys).  Those grids keep one
    // CTA per unit and let the hardware hand units to SMs as they free up.
    const long long n_units = (long long)B * Hq * ((Nq + 255) / 256);
    if (n_units > 0x7fffffffLL) return ATTN_ERR_INVALID_ARG;
    const bool persist = !causal && window_left < 0 && bmask.m == nullptr && Nk <= 4096;
    p.n_ctas = persist ? (int)std::min<long long>(n_units, g_sm_count[dev]) : (int)n_units;
    p.o = o;
    p.lse = lse;
    p.limit_ns = limit_ns;
    p.inject = inject;
    p.err = g_err_addr[dev];
    // seqlens_k with Nk == 0 means every length is 0: same as no keys.
    cudaError_t e =
        persist ? launch_fwd_persist(maps, p, d, dtype == ATTN_BF16, static_cast<cudaStream_t>(stream))
                : launch_fwd(maps, p, d, dtype == ATTN_BF16, static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? ATTN_OK : ATTN_ERR_CUDA;
}

}  // namespace

unsigned* device_error_word() {
    int dev = 0;
    if (check_device(&dev) != 1) return nullptr;
    return g_err_addr[dev];
}

int decode_check_args(const void* q, const void* k_cache, const void* v_cache,
                      const int* cu_seqlens_k, const int* seqlens_k, int max_seqlen_k,
                      int cache_slots, const void* o, const float* lse, int B, int Hq, int Hkv,
                      int Nq, int d, float scale, int dtype, int split_keys) {
    if (dtype != ATTN_BF16 && dtype != ATTN_FP16) return ATTN_ERR_UNSUPPORTED;
    if (d != 64 && d != 128) return ATTN_ERR_UNSUPPORTED;
    if (B <= 0 || Hq <= 0 || Hkv <= 0 || Hq % Hkv != 0 || Nq <= 0 || Nq > 16)
        return ATTN_ERR_INVALID_ARG;
    if (B > 65535 || Hkv > 65535 || max_seqlen_k < 0 || cache_slots <= 0)
        return ATTN_ERR_INVALID_ARG;
    if (split_keys < 0 || (split_keys % 64) != 0) return ATTN_ERR_INVALID_ARG;
    if (!(scale > 0.f) || !std::isfinite(scale)) return ATTN_ERR_INVALID_ARG;
    if (!q || !k_cache || !v_cache || !cu_seqlens_k || !seqlens_k || !o || !lse)
        return ATTN_ERR_INVALID_ARG;
    if (!aligned16(q) || !aligned16(k_cache) || !aligned16(v_cache) || !aligned16(o) ||
        !aligned16(lse) || (reinterpret_cast<uintptr_t>(cu_seqlens_k) & 3u) ||
        (reinterpret_cast<uintptr_t>(seqlens_k) & 3u))
        return ATTN_ERR_INVALID_ARG;
    const DecodeLayout lay = decode_layout(B, Hq, Hkv, Nq, d, max_seqlen_k, split_keys);
    if (lay.max_splits * lay.n_mgroups > 2147483647 / 2) return ATTN_ERR_INVALID_ARG;
    return ATTN_OK;
}

}  // namespace attn

using namespace attn;

extern "C" {

int attn_fwd(const void* q, const void* k, const void* v, void* o, float* lse, int B, int Hq,
             int Hkv, int Nq, int Nk, int d, float scale, int causal, int dtype, void* stream) {
    return fwd_common(q, k, v, o, lse, B, Hq, Hkv, Nq, Nk, d, scale, causal, dtype, nullptr,
                      stream, 0, kDefaultLimitNs, -1, kNoBlockMask);
}

int attn_fwd_kpad(const void* q, const void* k, const void* v, void* o, float* lse, int B,
                  int Hq, int Hkv, int Nq, int Nk, int d, float scale, int causal, int dtype,
                  const int* seqlens_k, void* stream) {
    return fwd_common(q, k, v, o, lse, B, Hq, Hkv, Nq, Nk, d, scale, causal, dtype, seqlens_k,
                      stream, 0, kDefaultLimitNs, -1, kNoBlockMask);
}

int attn_fwd_window(const void* q, const void* k, const void* v, void* o, float* lse, int B,
                    int Hq, int Hkv, int Nq, int Nk, int d, float scale, int causal,
                    int window_left, int dtype, const int* seqlens_k, void* stream) {
    return fwd_common(q, k, v, o, lse, B, Hq, Hkv, Nq, Nk, d, scale, causal, dtype, seqlens_k,
                      stream, 0, kDefaultLimitNs, window_left, kNoBlockMask);
}

int attn_fwd_blocksparse(const void* q, const void* k, const void* v, void* o, float* lse, int B,
                         int Hq, int Hkv, int Nq, int Nk, int d, float scale, int causal,
                         int window_left, int dtype, const int* seqlens_k,
                         const unsigned char* block_mask, long long mask_stride_b,
                         long long mask_stride_h, int mask_stride_row, void* stream) {
    if (!block_mask) return ATTN_ERR_INVALID_ARG;
    const BlockMask bm{block_mask, mask_stride_b, mask_stride_h, mask_stride_row};
    return fwd_common(q, k, v, o, lse, B, Hq, Hkv, Nq, Nk, d, scale, causal, dtype, seqlens_k,
                      stream, 0, kDefaultLimitNs, window_left, bm);
}

int attn_schedule_band_unit(unsigned u, int band, int n_pairs, int n_tiles, int* pair,
                            int* rank) {
    if (!pair || !rank || band <= 0 || n_pairs <= 0 || n_tiles <= 0 || band > n_pairs)
        return ATTN_ERR_INVALID_ARG;
    if ((unsigned long long)u >= (unsigned long long)n_pairs * (unsigned long long)n_tiles)
        return ATTN_ERR_INVALID_ARG;
    band_unit(u, band, n_pairs, n_tiles, *pair, *rank);
    return ATTN_OK;
}

int attn_schedule_sparse_steps(const unsigned char* m0, const unsigned char* m1, int nt0,
                               int nt1, int j00, int j01, int max_steps, int* steps) {
    if (!m0 || !m1 || !steps || nt0 < 0 || nt1 < 0 || j00 < 0 || j01 < 0 || max_steps < 0)
        return ATTN_ERR_INVALID_ARG;
    const int cnt0 = nt0 - j00 > 0 ? nt0 - j00 : 0, cnt1 = nt1 - j01 > 0 ? nt1 - j01 : 0;
    auto use = [&](int a, int j) -> bool {
        const bool in = a == 0 ? (cnt0 > 0 && j >= j00 && j < nt0)
                               : (cnt1 > 0 && j >= j01 && j < nt1);
        return in && (a == 0 ? m0[j] : m1[j]) != 0;
    };
    int n0 = 0, n1 = 0;
    for (int j = j00; cnt0 > 0 && j < nt0; ++j) n0 += use(0, j) ? 1 : 0;
    for (int j = j01; cnt1 > 0 && j < nt1; ++j) n1 += use(1, j) ? 1 : 0;
    const int nsteps = n0 > n1 ? n0 : n1;
    if (nsteps > max_steps) return ATTN_ERR_INVALID_ARG;
    int c0 = j00, c1 = j01, si = 0, pos = 0;
    for (int i = 0; i < nsteps; ++i) {
        const PairStep st = sparse_next_step(use, n0, n1, nt0, nt1, c0, c1, si, pos);
        int* r = steps + 7 * i;
        r[0] = st.x0;
        r[1] = st.x1;
        r[2] = st.pos0;
        r[3] = st.pos1;
        r[4] = st.has0;
        r[5] = st.has1;
        r[6] = st.shared;
    }
    return nsteps;
}

int attn_selftest_watchdog(const void* q, const void* k, const void* v, void* o, float* lse,
                           int limit_ms, void* stream) {
    if (limit_ms <= 0 || limit_ms > 10000) return ATTN_ERR_INVALID_ARG;
    return fwd_common(q, k, v, o, lse, 1, 1, 1, 128, 128, 64, 0.125f, 0, ATTN_BF16, nullptr,
                      stream, 1, (unsigned long long)limit_ms * 1000000ull, -1, kNoBlockMask);
}

size_t attn_decode_workspace_bytes(int B, int Hq, int Hkv, int Nq, int d, int max_seqlen_k,
                                   int split_keys) {
    if (B <= 0 || Hq <= 0 || Hkv <= 0 || Hq % Hkv != 0 || Nq <= 0 || Nq > 16) return 0;
    if ((d != 64 && d != 128) || max_seqlen_k < 0) return 0;
    if (split_keys < 0 || (split_keys % 64) != 0) return 0;
    return decode_layout(B, Hq, Hkv, Nq, d, max_seqlen_k, split_keys).total;
}

int attn_fwd_varlen_kvcache(const void* q, const void* k_cache, const void* v_cache,
                            const int* cu_seqlens_k, const int* seqlens_k, int max_seqlen_k,
                            int cache_slots, void* o, float* lse, int B, int Hq, int Hkv, int Nq,
                            int d, float scale, int causal, int dtype, void* workspace,
                            size_t workspace_bytes, int split_keys, void* stream) {
    const int arg_st = attn::decode_check_args(q, k_cache, v_cache, cu_seqlens_k, seqlens_k,
                                               max_seqlen_k, cache_slots, o, lse, B, Hq, Hkv,
                                               Nq, d, scale, dtype, split_keys);
    if (arg_st != ATTN_OK) return arg_st;
    int dev = 0;
    const int st = check_device(&dev);
    if (st == 0) return ATTN_ERR_CUDA;
    if (st < 0) return ATTN_ERR_UNSUPPORTED;

    const DecodeLayout lay = decode_layout(B, Hq, Hkv, Nq, d, max_seqlen_k, split_keys);
    if (!workspace || workspace_bytes < lay.total ||
        (reinterpret_cast<uintptr_t>(workspace) & 255u))
        return ATTN_ERR_WORKSPACE;

    const int G = Hq / Hkv;
    CUtensorMap kmap, vmap, qmap;
    const uint64_t dims[3] = {(uint64_t)d, (uint64_t)Hkv, (uint64_t)cache_slots};
    const uint64_t strides[2] = {(uint64_t)d * 2, (uint64_t)Hkv * d * 2};
    const uint32_t box[3] = {64, 1, lay.tc ? 128u : 64u};
    if (!encode_map(&kmap, dtype, k_cache, 3, dims, strides, box) ||
        !(lay.tc ? map_v_runs(&vmap, dtype, v_cache, (uint64_t)cache_slots, Hkv, d, 128)
                 : encode_map(&vmap, dtype, v_cache, 3, dims, strides, box)))
        return ATTN_ERR_INVALID_ARG;
    if (lay.tc) {
        // Q and O [B, Nq, Hq, d] seen as {d, G, Hkv, Nq, B}: one box gathers
        // the 128 / G tokens x G heads that share kv head g (row t * G + hh)
        const uint64_t qdims[5] = {(uint64_t)d, (uint64_t)G, (uint64_t)Hkv, (uint64_t)Nq,
                                   (uint64_t)B};
        const uint64_t qstrides[4] = {(uint64_t)d * 2, (uint64_t)G * d * 2, (uint64_t)Hq * d * 2,
                                      (uint64_t)Nq * Hq * d * 2};
        const uint32_t qbox[5] = {64, (uint32_t)G, 1, (uint32_t)(128 / G), 1};
        if (!encode_map(&qmap, dtype, q, 5, qdims, qstrides, qbox)) return ATTN_ERR_INVALID_ARG;
    }

    uint8_t* ws = static_cast<uint8_t*>(workspace);
    DecodeParams p{};
    p.q = q;
    p.o = o;
    p.lse = lse;
    p.cu_seqlens_k = cu_seqlens_k;
    p.seqlens_k = seqlens_k;
    p.part_o = reinterpret_cast<float*>(ws + lay.part_o_off);
    p.part_lse = reinterpret_cast<float*>(ws + lay.part_lse_off);
    p.counters = reinterpret_cast<unsigned*>(ws + lay.counters_off);
    p.plan = reinterpret_cast<DecodePlan*>(ws + lay.plan_off);
    p.seq_prefix = reinterpret_cast<long long*>(ws + lay.prefix_off);
    p.range_units = reinterpret_cast<int2*>(ws + lay.ranges_off);
    p.max_seqlen_k = max_seqlen_k;
    p.max_ranges = lay.max_ranges;
    p.B = B;
    p.Hq = Hq;
    p.Hkv = Hkv;
    p.Nq = Nq;
    p.G = G;
    p.rows = Nq * p.G;
    p.n_mgroups = lay.n_mgroups;
    p.split_keys = lay.split_keys;
    p.max_splits = lay.max_splits;
    p.causal = causal ? 1 : 0;
    p.scale_log2 = scale * 1.4426950408889634f;
    p.limit_ns = kDefaultLimitNs;
    p.err = g_err_addr[dev];
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    cudaError_t e;
    if (lay.tc) {
        // the plan kernel clears the counters; one persistent CTA per SM
        const int n_ctas = std::min(g_sm_count[dev], lay.max_ranges);
        e = launch_decode_tc(qmap, kmap, vmap, p, d, dtype == ATTN_BF16, n_ctas, s);
    } else {
        if (cudaMemsetAsync(p.counters, 0, (size_t)B * Hkv * lay.n_mgroups * sizeof(unsigned),
                            s) != cudaSuccess)
            return ATTN_ERR_CUDA;
        e = launch_decode(kmap, vmap, p, d, dtype == ATTN_BF16, s);
    }
    return e == cudaSuccess ? ATTN_OK : ATTN_ERR_CUDA;
}

int attn_fwd_paged_kvcache(const void* q, void* k_cache, void* v_cache, const int* block_table,
                           int max_blocks, int block_size, int num_blocks, const int* seqlens_k,
                           int max_seqlen_k, const void* k_new, const void* v_new, void* o,
                           float* lse, int B, int Hq, int Hkv, int Nq, int d, float scale,
                           int causal, int dtype, void* workspace, size_t workspace_bytes,
                           int split_keys, void* stream) {
    if (dtype != ATTN_BF16 && dtype != ATTN_FP16) return ATTN_ERR_UNSUPPORTED;
    if (d != 64 && d != 128) return ATTN_ERR_UNSUPPORTED;
    if (B <= 0 || Hq <= 0 || Hkv <= 0 || Hq % Hkv != 0 || Nq <= 0 || Nq > 16)
        return ATTN_ERR_INVALID_ARG;
    if (B > 65535 || max_seqlen_k < 0 || max_blocks <= 0 || num_blocks <= 0)
        return ATTN_ERR_INVALID_ARG;
    if (block_size < 16 || block_size > 1024 || (block_size & (block_size - 1)))
        return ATTN_ERR_INVALID_ARG;
    if ((long)max_blocks * block_size < max_seqlen_k) return ATTN_ERR_INVALID_ARG;
    if ((long)num_blocks * block_size > 0x7fffffffL) return ATTN_ERR_INVALID_ARG;
    if (split_keys < 0 || (split_keys % 64) != 0) return ATTN_ERR_INVALID_ARG;
    if (!(scale > 0.f) || !std::isfinite(scale)) return ATTN_ERR_INVALID_ARG;
    if (!q || !k_cache || !v_cache || !block_table || !seqlens_k || !o || !lse)
        return ATTN_ERR_INVALID_ARG;
    if ((k_new == nullptr) != (v_new == nullptr)) return ATTN_ERR_INVALID_ARG;
    if (!aligned16(q) || !aligned16(k_cache) || !aligned16(v_cache) || !aligned16(o) ||
        !aligned16(lse) || (k_new && (!aligned16(k_new) || !aligned16(v_new))) ||
        (reinterpret_cast<uintptr_t>(block_table) & 3u) ||
        (reinterpret_cast<uintptr_t>(seqlens_k) & 3u))
        return ATTN_ERR_INVALID_ARG;
    const int G = Hq / Hkv;
    // the paged path is the tensor-core decode's
    if (!decode_use_tc(G, Nq, split_keys)) return ATTN_ERR_UNSUPPORTED;
    int dev = 0;
    const int st = check_device(&dev);
    if (st == 0) return ATTN_ERR_CUDA;
    if (st < 0) return ATTN_ERR_UNSUPPORTED;

    const DecodeLayout lay = decode_layout(B, Hq, Hkv, Nq, d, max_seqlen_k, split_keys);
    if (!workspace || workspace_bytes < lay.total ||
        (reinterpret_cast<uintptr_t>(workspace) & 255u))
        return ATTN_ERR_WORKSPACE;

    CUtensorMap kmap, vmap, qmap;
    const uint64_t slots = (uint64_t)num_blocks * block_size;
    const uint64_t dims[3] = {(uint64_t)d, (uint64_t)Hkv, slots};
    const uint64_t strides[2] = {(uint64_t)d * 2, (uint64_t)Hkv * d * 2};
    const uint32_t box[3] = {64, 1, (uint32_t)std::min(128, block_size)};
    if (!encode_map(&kmap, dtype, k_cache, 3, dims, strides, box) ||
        !map_v_runs(&vmap, dtype, v_cache, slots, Hkv, d, std::min(128, block_size)))
        return ATTN_ERR_INVALID_ARG;
    const uint64_t qdims[5] = {(uint64_t)d, (uint64_t)G, (uint64_t)Hkv, (uint64_t)Nq, (uint64_t)B};
    const uint64_t qstrides[4] = {(uint64_t)d * 2, (uint64_t)G * d * 2, (uint64_t)Hq * d * 2,
                                  (uint64_t)Nq * Hq * d * 2};
    const uint32_t qbox[5] = {64, (uint32_t)G, 1, (uint32_t)(128 / G), 1};
    if (!encode_map(&qmap, dtype, q, 5, qdims, qstrides, qbox)) return ATTN_ERR_INVALID_ARG;

    uint8_t* ws = static_cast<uint8_t*>(workspace);
    DecodeParams p{};
    p.q = q;
    p.o = o;
    p.lse = lse;
    p.cu_seqlens_k = nullptr;
    p.seqlens_k = seqlens_k;
    p.part_o = reinterpret_cast<float*>(ws + lay.part_o_off);
    p.part_lse = reinterpret_cast<float*>(ws + lay.part_lse_off);
    p.counters = reinterpret_cast<unsigned*>(ws + lay.counters_off);
    p.plan = reinterpret_cast<DecodePlan*>(ws + lay.plan_off);
    p.seq_prefix = reinterpret_cast<long long*>(ws + lay.prefix_off);
    p.range_units = reinterpret_cast<int2*>(ws + lay.ranges_off);
    p.max_seqlen_k = max_seqlen_k;
    p.max_ranges = lay.max_ranges;
    p.block_table = block_table;
    p.max_blocks = max_blocks;
    p.block_shift = __builtin_ctz((unsigned)block_size);
    p.num_blocks = num_blocks;
    p.k_cache = k_cache;
    p.v_cache = v_cache;
    p.k_new = k_new;
    p.v_new = v_new;
    p.B = B;
    p.Hq = Hq;
    p.Hkv = Hkv;
    p.Nq = Nq;
    p.G = G;
    p.rows = Nq * G;
    p.n_mgroups = lay.n_mgroups;
    p.split_keys = lay.split_keys;
    p.max_splits = lay.max_splits;
    p.causal = causal ? 1 : 0;
    p.scale_log2 = scale * 1.4426950408889634f;
    p.limit_ns = kDefaultLimitNs;
    p.err = g_err_addr[dev];
    const int n_ctas = std::min(g_sm_count[dev], lay.max_ranges);
    cudaError_t e = launch_decode_tc(qmap, kmap, vmap, p, d, dtype == ATTN_BF16, n_ctas,
                                     static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? ATTN_OK : ATTN_ERR_CUDA;
}

size_t attn_bwd_workspace_bytes(int B, int Hq, int Nq) {
    if (B <= 0 || Hq <= 0 || Nq <= 0) return 0;
    const size_t one = (((size_t)B * Hq * Nq * 4) + 255) & ~(size_t)255;
    return 2 * one;
}

int attn_bwd(const void* q, const void* k, const void* v, const void* o, const float* lse,
             const void* dout, void* dq, void* dk, void* dv, int B, int Hq, int Hkv, int Nq,
             int Nk, int d, float scale, int causal, int dtype, const int* seqlens_k,
             void* workspace, size_t workspace_bytes, void* stream) {
    return attn_bwd_window(q, k, v, o, lse, dout, dq, dk, dv, B, Hq, Hkv, Nq, Nk, d, scale,
                           causal, -1, dtype, seqlens_k, workspace, workspace_bytes, stream);
}

int attn_bwd_window(const void* q, const void* k, const void* v, const void* o, const float* lse,
                    const void* dout, void* dq, void* dk, void* dv, int B, int Hq, int Hkv,
                    int Nq, int Nk, int d, float scale, int causal, int window_left, int dtype,
                    const int* seqlens_k, void* workspace, size_t workspace_bytes,
                    void* stream) {
    return attn_bwd_blocksparse(q, k, v, o, lse, dout, dq, dk, dv, B, Hq, Hkv, Nq, Nk, d, scale,
                                causal, window_left, dtype, seqlens_k, nullptr, 0, 0, 0,
                                workspace, workspace_bytes, stream);
}

int attn_bwd_blocksparse(const void* q, const void* k, const void* v, const void* o,
                         const float* lse, const void* dout, void* dq, void* dk, void* dv, int B,
                         int Hq, int Hkv, int Nq, int Nk, int d, float scale, int causal,
                         int window_left, int dtype, const int* seqlens_k,
                         const unsigned char* block_mask, long long mask_stride_b,
                         long long mask_stride_h, int mask_stride_row, void* workspace,
                         size_t workspace_bytes, void* stream) {
    if (window_left < -1) return ATTN_ERR_INVALID_ARG;
    if (block_mask && (mask_stride_b < 0 || mask_stride_h < 0 ||
                       mask_stride_row < (Nk + 127) / 128))
        return ATTN_ERR_INVALID_ARG;
    if (dtype != ATTN_BF16 && dtype != ATTN_FP16) return ATTN_ERR_UNSUPPORTED;
    if (d != 64 && d != 128) return ATTN_ERR_UNSUPPORTED;
    if (B <= 0 || Hq <= 0 || Hkv <= 0 || Nq <= 0 || Nk < 0 || Hq % Hkv != 0)
        return ATTN_ERR_INVALID_ARG;
    if (B > 65535 || Hq > 65535) return ATTN_ERR_INVALID_ARG;
    if (!(scale > 0.f) || !std::isfinite(scale)) return ATTN_ERR_INVALID_ARG;
    if (!q || !o || !lse || !dout || !dq || !aligned16(q) || !aligned16(o) || !aligned16(lse) ||
        !aligned16(dout) || !aligned16(dq))
        return ATTN_ERR_INVALID_ARG;
    if (Nk > 0 && (!k || !v || !dk || !dv || !aligned16(k) || !aligned16(v) || !aligned16(dk) ||
                   !aligned16(dv)))
        return ATTN_ERR_INVALID_ARG;
    if (seqlens_k && (reinterpret_cast<uintptr_t>(seqlens_k) & 3u)) return ATTN_ERR_INVALID_ARG;
    const size_t need = attn_bwd_workspace_bytes(B, Hq, Nq);
    if (!workspace || workspace_bytes < need || (reinterpret_cast<uintptr_t>(workspace) & 255u))
        return ATTN_ERR_WORKSPACE;
    int dev = 0;
    const int st = check_device(&dev);
    if (st == 0) return ATTN_ERR_CUDA;
    if (st < 0) return ATTN_ERR_UNSUPPORTED;

    BwdMaps maps;
    // with no keys the K/V maps are never read; point them at Q
    const void* kb = Nk > 0 ? k : q;
    const void* vb = Nk > 0 ? v : q;
    const int nk_map = Nk > 0 ? Nk : Nq;
    const int hkv_map = Nk > 0 ? Hkv : Hq;
    if (!map_bnhd(&maps.q, dtype, q, B, Nq, Hq, d) ||
        !map_bnhd(&maps.k, dtype, kb, B, nk_map, hkv_map, d) ||
        !map_bnhd(&maps.v, dtype, vb, B, nk_map, hkv_map, d) ||
        !map_bnhd(&maps.dout, dtype, dout, B, Nq, Hq, d))
        return ATTN_ERR_INVALID_ARG;

    BwdParams p{};
    p.B = B;
    p.Hq = Hq;
    p.Hkv = Hkv;
    p.Nq = Nq;
    p.Nk = Nk;
    p.G = Hq / Hkv;
    p.causal = causal ? 1 : 0;
    p.scale = scale;
    p.scale_log2 = scale * 1.4426950408889634f;
    p.seqlens_k = Nk > 0 ? seqlens_k : nullptr;
    p.window_left = window_left;
    p.bmask = BlockMask{block_mask, mask_stride_b, mask_stride_h, mask_stride_row};
    // decreasing-cost launch order for causal, as in the forward, in bands
    // whose streamed operands fit in L2 together: a dK/dV block streams Q and
    // dO of the G heads of its kv head, a dQ block K and V of its kv head
    p.band_kv = p.band_q = 0;
    if (causal && window_left < 0 && Nk > 0) {
        const int G = Hq / Hkv;
        const long long nkt = (Nk + 127) / 128, nqt = (Nq + 127) / 128;
        const long long per_kv = 4LL * Nq * d * G;        // Q + dO of a group
        const long long per_q = 4LL * Nk * d / G;         // K + V, shared by G heads
        const long long fit_kv = (48LL << 20) / (per_kv > 0 ? per_kv : 1);
        const long long fit_q = (48LL << 20) / (per_q > 0 ? per_q : 1);
        if ((long long)B * Hkv * nkt <= 0x7fffffffLL)
            p.band_kv = (int)std::min<long long>((long long)B * Hkv, std::max<long long>(8, fit_kv));
        if ((long long)B * Hq * nqt <= 0x7fffffffLL)
            p.band_q = (int)std::min<long long>((long long)B * Hq, std::max<long long>(8, fit_q));
    }
    p.o = o;
    p.dout = dout;
    p.lse = lse;
    p.lse2 = static_cast<float*>(workspace);
    p.dsum = reinterpret_cast<float*>(static_cast<uint8_t*>(workspace) + need / 2);
    p.dq = dq;
    p.dk = dk;
    p.dv = dv;
    p.limit_ns = kDefaultLimitNs;
    p.err = g_err_addr[dev];
    cudaError_t e = launch_bwd(maps, p, d, dtype == ATTN_BF16, static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? ATTN_OK : ATTN_ERR_CUDA;
}

const char* attn_status_string(int status) {
    switch (status) {
        case ATTN_OK: return "ok";
        case ATTN_ERR_INVALID_ARG: return "invalid argument";
        case ATTN_ERR_UNSUPPORTED: return "unsupported device, dtype or head dimension";
        case ATTN_ERR_CUDA: return "CUDA error";
        case ATTN_ERR_WORKSPACE: return "workspace missing, misaligned or too small";
        case ATTN_ERR_TIMEOUT: return "a bounded in-kernel wait ran out";
        default: return "unknown status";
    }
}

int attn_get_device_error(int* code, void* stream) {
    if (!code) return ATTN_ERR_INVALID_ARG;
    int dev = 0;
    const int st = check_device(&dev);
    if (st == 0) return ATTN_ERR_CUDA;
    if (st < 0) return ATTN_ERR_UNSUPPORTED;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (cudaStreamSynchronize(s) != cudaSuccess) return ATTN_ERR_CUDA;
    unsigned v = 0, zero = 0;
    if (cudaMemcpyFromSymbol(&v, g_device_error, sizeof(v)) != cudaSuccess) return ATTN_ERR_CUDA;
    if (cudaMemcpyToSymbol(g_device_error, &zero, sizeof(zero)) != cudaSuccess)
        return ATTN_ERR_CUDA;
    *code = (int)v;
    return ATTN_OK;
}

const char* attn_version(void) { return "attn-b200 0.1 (sm_100a)"; }

}  // extern "C"
