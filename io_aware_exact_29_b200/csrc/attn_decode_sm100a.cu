// attn_decode_sm100a.cu -- attention of a few new query tokens against a
// packed, variable-length KV cache (decode), split along the keys.
//
// The KV cache grows by one row per generated token and is pre-allocated;
// only the rows up to each sequence's real length are read, and the key
// splits are aligned to that length (ai6s.net article on the ops-transformer
// FlashAttention operator, section "ops-transformer 里的 FlashAttention 做了
// 什么额外的事", point 3).  Within a split the keys are processed tile by tile
// with a running max and sum (section "FlashAttention 拆的不是算法，是数据流").
//
// This kernel serves the shapes the tensor-core decode (attn_decode_tc_sm100a.cu)
// does not take: query heads per kv head that do not divide 128, more than
// 128 query rows per kv head, or a split size that is not a multiple of 128.
//
// Work unit = one CTA: (sequence b, kv head g, key split s, group of 16 query
// rows).  The query rows of a kv head are the Nq tokens x G query heads that
// share it (row r = token r / G, head g*G + r % G), so one pass over the cache
// serves all of them.  The path is bound by reading the cache from HBM:
//   warp 4      TMA loader: 64-key K and V tiles (128-byte swizzled) into a
//               STAGES-deep ring; the copy never reaches past the cache end
//   warps 0..3  each takes 16 keys of every tile: S = Q·Kᵀ and O += P·V with
//               mma.sync m16n8k16 (fp32 accumulate; the math is ~10% of the
//               memory time at Nq = 1, so the legacy warp MMA is enough),
//               online softmax in registers
// then the four warps merge their (max, sum, O) through shared memory.  With
// one split the CTA writes O and LSE; otherwise it writes its normalised
// partial O and LSE to the workspace and the last CTA of the (b, g, row
// group) -- found with an atomic counter, no spinning -- merges all splits in
// split order:  LSE = log sum_s exp(LSE_s),  O = sum_s exp(LSE_s - LSE) O_s.
#include <algorithm>

#include "attn_internal.h"
#include "ptx.cuh"

namespace attn {
namespace {

constexpr int kKeysPerTile = 64;
constexpr int kConsumerWarps = 4;
constexpr int kThreads = 32 * (kConsumerWarps + 1);
constexpr float kRescaleThreshold = 8.0f;
constexpr float kLn2 = 0.69314718055994531f;

template <int D, int STAGES>
struct DecSmem {
    static constexpr uint32_t kTileBytes = kKeysPerTile * D * 2;  // one K or V tile
    static constexpr uint32_t kK = 0;
    static constexpr uint32_t kV = kK + STAGES * kTileBytes;
    static constexpr uint32_t kRing = kV + STAGES * kTileBytes;
    // merge area (reuses the ring once every tile is consumed)
    static constexpr uint32_t kMergeO = 0;  // [4][16][D] fp32
    static constexpr uint32_t kMergeM = kMergeO + kConsumerWarps * 16 * D * 4;
    static constexpr uint32_t kMergeL = kMergeM + kConsumerWarps * 16 * 4;
    static constexpr uint32_t kMergeEnd = kMergeL + kConsumerWarps * 16 * 4;
    static constexpr uint32_t kBars = (kRing > kMergeEnd ? kRing : kMergeEnd);
    static constexpr uint32_t kTotal = kBars + 256;
    static constexpr uint32_t kAlloc = kTotal + 1024;
};

template <int STAGES>
struct DecBars {
    uint64_t full[STAGES];
    uint64_t empty[STAGES];
    float row_lse[16];
    int is_last;
    int abort;
};

__device__ __forceinline__ void record_error(unsigned* err, unsigned code, int* abort_flag) {
    atomicCAS(err, 0u, code);
    *reinterpret_cast<volatile int*>(abort_flag) = 1;
}

__device__ __forceinline__ uint32_t sw128_offset(uint32_t row, uint32_t chunk) {
    return row * 128u + ((chunk ^ (row & 7u)) << 4);
}

template <bool BF16>
__device__ __forceinline__ void store_out(void* o, size_t idx, float v) {
    if constexpr (BF16)
        reinterpret_cast<__nv_bfloat16*>(o)[idx] = __float2bfloat16_rn(v);
    else
        reinterpret_cast<__half*>(o)[idx] = __float2half_rn(v);
}

template <int D, bool BF16, int STAGES>
__global__ void __launch_bounds__(kThreads)
    attn_decode_kernel(const __grid_constant__ CUtensorMap tm_k,
                       const __grid_constant__ CUtensorMap tm_v,
                       const __grid_constant__ DecodeParams p) {
    using L = DecSmem<D, STAGES>;
    constexpr uint32_t kTileBytes = L::kTileBytes;
    constexpr int kDBlocks = D / 64;
    constexpr int kKSteps = D / 16;

    const int split = blockIdx.x / p.n_mgroups;
    const int mg = blockIdx.x % p.n_mgroups;
    const int g = blockIdx.y;
    const int b = blockIdx.z;
    const int Lk = p.seqlens_k[b];
    const int slot0 = p.cu_seqlens_k[b];
    const int nsplit = Lk > 0 ? (Lk + p.split_keys - 1) / p.split_keys : 1;
    if (split >= nsplit) return;  // whole CTA leaves before touching anything

    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw_addr = ptx::smem_u32(smem_raw);
    uint8_t* smem = smem_raw + (((raw_addr + 1023u) & ~1023u) - raw_addr);
    DecBars<STAGES>* bars = reinterpret_cast<DecBars<STAGES>*>(smem + L::kBars);
    volatile int* abort_flag = &bars->abort;

    const int tid = threadIdx.x;
    const int warp = tid >> 5;
    const int lane = tid & 31;

    if (nsplit > p.max_splits) {  // max_seqlen_k was smaller than a real length
        if (tid == 0) atomicCAS(p.err, 0u, kErrDecodeBase + 1);
        return;
    }

    const int key_begin = split * p.split_keys;
    const int key_end = min(Lk, key_begin + p.split_keys);
    const int ntiles = (key_end - key_begin + kKeysPerTile - 1) / kKeysPerTile;  // >= 0

    if (tid == 0) {
        for (int s = 0; s < STAGES; ++s) {
            ptx::mbar_init(&bars->full[s], 1);
            ptx::mbar_init(&bars->empty[s], kConsumerWarps);
        }
        bars->abort = 0;
        bars->is_last = 0;
        ptx::fence_barrier_init();
    }
    __syncthreads();

    if (warp == kConsumerWarps) {
        // ================================================= TMA loader
        if (lane == 0 && ntiles > 0) {
            ptx::prefetch_tmap(&tm_k);
            ptx::prefetch_tmap(&tm_v);
            int issued = 0;
            for (int t = 0; t < ntiles; ++t) {
                const int st = t % STAGES;
                const uint32_t ph = (t / STAGES) & 1;
                if (!ptx::mbar_wait(&bars->empty[st], ph ^ 1, p.limit_ns, abort_flag)) {
                    record_error(p.err, kErrDecodeBase + 2, &bars->abort);
                    break;
                }
                const int row = slot0 + key_begin + t * kKeysPerTile;
                ptx::mbar_arrive_expect_tx(&bars->full[st], 2 * kTileBytes);
                for (int c = 0; c < kDBlocks; ++c) {
                    ptx::tma_load_3d(smem + L::kK + st * kTileBytes + c * (kKeysPerTile * 128),
                                     &tm_k, &bars->full[st], c * 64, g, row);
                    ptx::tma_load_3d(smem + L::kV + st * kTileBytes + c * (kKeysPerTile * 128),
                                     &tm_v, &bars->full[st], c * 64, g, row);
                }
                ++issued;
            }
            int zero = 0;
            volatile int* no_abort = &zero;
            for (int t = max(0, issued - STAGES); t < issued; ++t)
                ptx::mbar_wait(&bars->full[t % STAGES], (t / STAGES) & 1, p.limit_ns, no_abort);
        }
        return;  // the loader takes no part in the merge
    }

    // ===================================================== consumer warps
    const int rlo = mg * 16 + (lane >> 2);  // query rows of this thread
    const int rhi = rlo + 8;
    const int tok_lo = rlo / p.G, tok_hi = rhi / p.G;
    const int head_lo = g * p.G + rlo % p.G, head_hi = g * p.G + rhi % p.G;
    const bool val_lo = rlo < p.rows, val_hi = rhi < p.rows;
    // last visible key of each row (inclusive)
    const int lim_lo = p.causal ? min(Lk - 1, tok_lo + Lk - p.Nq) : Lk - 1;
    const int lim_hi = p.causal ? min(Lk - 1, tok_hi + Lk - p.Nq) : Lk - 1;

    // Q fragments (A operand, row-major 16 x 16 per k-step), zero for padding rows
    uint32_t qa[kKSteps][4];
    {
        const uint32_t* qlo = reinterpret_cast<const uint32_t*>(p.q) +
                              (((size_t)b * p.Nq + tok_lo) * p.Hq + head_lo) * (D / 2);
        const uint32_t* qhi = reinterpret_cast<const uint32_t*>(p.q) +
                              (((size_t)b * p.Nq + tok_hi) * p.Hq + head_hi) * (D / 2);
#pragma unroll
        for (int ks = 0; ks < kKSteps; ++ks) {
            const int c = ks * 8 + (lane & 3);  // pair index along d
            qa[ks][0] = val_lo ? __ldg(qlo + c) : 0u;
            qa[ks][1] = val_hi ? __ldg(qhi + c) : 0u;
            qa[ks][2] = val_lo ? __ldg(qlo + c + 4) : 0u;
            qa[ks][3] = val_hi ? __ldg(qhi + c + 4) : 0u;
        }
    }

    float o[D / 8][4];
#pragma unroll
    for (int n = 0; n < D / 8; ++n) o[n][0] = o[n][1] = o[n][2] = o[n][3] = 0.f;
    float m_lo = -INFINITY, m_hi = -INFINITY;  // reference max, scale*log2 units
    float l_lo = 0.f, l_hi = 0.f;              // this thread's share of the row sums
    const float sl2 = p.scale_log2;
    const uint32_t sbase = ptx::smem_u32(smem);
    bool ok = true;

    for (int t = 0; t < ntiles; ++t) {
        const int st = t % STAGES;
        const uint32_t ph = (t / STAGES) & 1;
        const bool w_ok = ptx::mbar_wait(&bars->full[st], ph, p.limit_ns, abort_flag);
        if (!__all_sync(0xffffffffu, w_ok)) {
            record_error(p.err, kErrDecodeBase + 3, &bars->abort);
            ok = false;
            break;
        }
        const int jw = key_begin + t * kKeysPerTile + warp * 16;  // first key of this warp
        const uint32_t k_tile = sbase + L::kK + st * kTileBytes;
        const uint32_t v_tile = sbase + L::kV + st * kTileBytes;
        bool zeroed = false;
        if (jw < key_end) {
            // ---- S = Q Kᵀ for 16 rows x 16 keys (two n-tiles of 8 keys)
            float s[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
            {
                const int mi = lane >> 3, rr = lane & 7;
                const uint32_t key_local = (uint32_t)(warp * 16 + (mi >> 1) * 8 + rr);
#pragma unroll
                for (int ks = 0; ks < kKSteps; ++ks) {
                    const uint32_t chunk = (uint32_t)(ks * 2 + (mi & 1));
                    const uint32_t addr = k_tile + (chunk >> 3) * (kKeysPerTile * 128) +
                                          sw128_offset(key_local, chunk & 7);
                    uint32_t b00, b01, b10, b11;
                    ptx::ldmatrix_x4(addr, b00, b01, b10, b11);
                    ptx::mma_16816<BF16>(s[0], qa[ks], b00, b01);
                    ptx::mma_16816<BF16>(s[1], qa[ks], b10, b11);
                }
            }
            // ---- mask (only tiles that reach a row's last visible key)
            const int kcol = jw + 2 * (lane & 3);
            if (jw + 15 > min(lim_lo, lim_hi) || jw + 15 >= key_end) {
#pragma unroll
                for (int n = 0; n < 2; ++n)
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const int key = kcol + n * 8 + (e & 1);
                        const int lim = (e < 2) ? lim_lo : lim_hi;
                        if (key > lim || key >= key_end) s[n][e] = -INFINITY;
                    }
            }
            // ---- online softmax, rows lo / hi
            float mx_lo = fmaxf(fmaxf(s[0][0], s[0][1]), fmaxf(s[1][0], s[1][1]));
            float mx_hi = fmaxf(fmaxf(s[0][2], s[0][3]), fmaxf(s[1][2], s[1][3]));
            mx_lo = fmaxf(mx_lo, __shfl_xor_sync(0xffffffffu, mx_lo, 1));
            mx_lo = fmaxf(mx_lo, __shfl_xor_sync(0xffffffffu, mx_lo, 2));
            mx_hi = fmaxf(mx_hi, __shfl_xor_sync(0xffffffffu, mx_hi, 1));
            mx_hi = fmaxf(mx_hi, __shfl_xor_sync(0xffffffffu, mx_hi, 2));
            const float mt_lo = mx_lo * sl2, mt_hi = mx_hi * sl2;
            float a_lo = 1.f, a_hi = 1.f;
            bool rs = false;
            if (mt_lo > m_lo + kRescaleThreshold) {
                a_lo = ptx::ex2_approx(m_lo - mt_lo);
                m_lo = mt_lo;
                rs = true;
            }
            if (mt_hi > m_hi + kRescaleThreshold) {
                a_hi = ptx::ex2_approx(m_hi - mt_hi);
                m_hi = mt_hi;
                rs = true;
            }
            if (__any_sync(0xffffffffu, rs)) {
#pragma unroll
                for (int n = 0; n < D / 8; ++n) {
                    o[n][0] *= a_lo;
                    o[n][1] *= a_lo;
                    o[n][2] *= a_hi;
                    o[n][3] *= a_hi;
                }
                l_lo *= a_lo;
                l_hi *= a_hi;
            }
            const float mu_lo = (m_lo == -INFINITY) ? 0.f : m_lo;
            const float mu_hi = (m_hi == -INFINITY) ? 0.f : m_hi;
            float pr[2][4];
#pragma unroll
            for (int n = 0; n < 2; ++n) {
                pr[n][0] = ptx::ex2_approx(fmaf(s[n][0], sl2, -mu_lo));
                pr[n][1] = ptx::ex2_approx(fmaf(s[n][1], sl2, -mu_lo));
                pr[n][2] = ptx::ex2_approx(fmaf(s[n][2], sl2, -mu_hi));
                pr[n][3] = ptx::ex2_approx(fmaf(s[n][3], sl2, -mu_hi));
                l_lo += pr[n][0] + pr[n][1];
                l_hi += pr[n][2] + pr[n][3];
            }
            uint32_t pa[4];
            pa[0] = ptx::pack2<BF16>(pr[0][0], pr[0][1]);
            pa[1] = ptx::pack2<BF16>(pr[0][2], pr[0][3]);
            pa[2] = ptx::pack2<BF16>(pr[1][0], pr[1][1]);
            pa[3] = ptx::pack2<BF16>(pr[1][2], pr[1][3]);

            // ---- keys behind the real length: zero their V rows (0 * NaN guard)
            if (jw + 15 >= key_end) {
                if (lane < 16 && jw + lane >= key_end) {
                    uint8_t* vrow = smem + L::kV + st * kTileBytes + (warp * 16 + lane) * 128;
#pragma unroll
                    for (int c = 0; c < kDBlocks; ++c)
#pragma unroll
                        for (int ch = 0; ch < 8; ++ch)
                            *reinterpret_cast<uint4*>(vrow + c * (kKeysPerTile * 128) + ch * 16) =
                                make_uint4(0, 0, 0, 0);
                }
                zeroed = true;
                __syncwarp();
            }
            // ---- O += P V (V rows are keys: transposed 8x8 loads give the B operand)
            {
                const int mi = lane >> 3, rr = lane & 7;
                const uint32_t key_local = (uint32_t)(warp * 16 + (mi & 1) * 8 + rr);
#pragma unroll
                for (int np = 0; np < D / 16; ++np) {
                    const uint32_t chunk = (uint32_t)(np * 2 + (mi >> 1));
                    const uint32_t addr = v_tile + (chunk >> 3) * (kKeysPerTile * 128) +
                                          sw128_offset(key_local, chunk & 7);
                    uint32_t b0, b1, b2, b3;
                    ptx::ldmatrix_x4_trans(addr, b0, b1, b2, b3);
                    ptx::mma_16816<BF16>(o[2 * np], pa, b0, b1);
                    ptx::mma_16816<BF16>(o[2 * np + 1], pa, b2, b3);
                }
            }
        }
        if (zeroed) ptx::fence_proxy_async_smem();  // generic writes before the next TMA write
        __syncwarp();
        if (lane == 0) ptx::mbar_arrive(&bars->empty[st]);
    }

    // ---- row sums over the four lanes that share a row
    l_lo += __shfl_xor_sync(0xffffffffu, l_lo, 1);
    l_lo += __shfl_xor_sync(0xffffffffu, l_lo, 2);
    l_hi += __shfl_xor_sync(0xffffffffu, l_hi, 1);
    l_hi += __shfl_xor_sync(0xffffffffu, l_hi, 2);

    // ---- merge the four warps through shared memory (the ring is free now)
    ptx::named_barrier_sync(1, 32 * kConsumerWarps);
    float* mo = reinterpret_cast<float*>(smem + L::kMergeO);
    float* mm = reinterpret_cast<float*>(smem + L::kMergeM);
    float* ml = reinterpret_cast<float*>(smem + L::kMergeL);
    {
        const int r0 = lane >> 2;
        if ((lane & 3) == 0) {
            mm[warp * 16 + r0] = ok ? m_lo : -INFINITY;
            mm[warp * 16 + r0 + 8] = ok ? m_hi : -INFINITY;
            ml[warp * 16 + r0] = l_lo;
            ml[warp * 16 + r0 + 8] = l_hi;
        }
#pragma unroll
        for (int n = 0; n < D / 8; ++n) {
            const int c = n * 8 + 2 * (lane & 3);
            *reinterpret_cast<float2*>(mo + (warp * 16 + r0) * D + c) = make_float2(o[n][0], o[n][1]);
            *reinterpret_cast<float2*>(mo + (warp * 16 + r0 + 8) * D + c) =
                make_float2(o[n][2], o[n][3]);
        }
    }
    ptx::named_barrier_sync(1, 32 * kConsumerWarps);

    const size_t unit = ((size_t)b * p.Hkv + g) * p.n_mgroups + mg;
    const int nthr = 32 * kConsumerWarps;
    if (tid < 16) {
        // per-row combined max/sum of the four warps -> LSE of this split
        const int r = tid;
        float M = -INFINITY;
#pragma unroll
        for (int w = 0; w < kConsumerWarps; ++w) M = fmaxf(M, mm[w * 16 + r]);
        float wsum = 0.f;
        if (M != -INFINITY) {
#pragma unroll
            for (int w = 0; w < kConsumerWarps; ++w)
                wsum += ptx::ex2_approx(mm[w * 16 + r] - M) * ml[w * 16 + r];
        }
        bars->row_lse[r] = (wsum > 0.f) ? (M + ptx::lg2_approx(wsum)) : -INFINITY;  // log2 units
    }
    ptx::named_barrier_sync(1, 32 * kConsumerWarps);
    for (int idx = tid; idx < 16 * D; idx += nthr) {
        const int r = idx / D, c = idx % D;
        const int row = mg * 16 + r;
        if (row >= p.rows) continue;
        const float lse2 = bars->row_lse[r];
        float val = 0.f;
        if (lse2 != -INFINITY) {
#pragma unroll
            for (int w = 0; w < kConsumerWarps; ++w) {
                const float mw = mm[w * 16 + r];
                if (mw != -INFINITY) val += ptx::ex2_approx(mw - lse2) * mo[(w * 16 + r) * D + c];
            }
        }
        const float lse_nat = (lse2 == -INFINITY) ? -INFINITY : lse2 * kLn2;
        const int tok = row / p.G, head = g * p.G + row % p.G;
        if (nsplit == 1) {
            store_out<BF16>(p.o, (((size_t)b * p.Nq + tok) * p.Hq + head) * D + c, val);
            if (c == 0) p.lse[((size_t)b * p.Hq + head) * p.Nq + tok] = lse_nat;
        } else {
            const size_t pr = (unit * p.max_splits + split) * 16 + r;
            p.part_o[pr * D + c] = val;
            if (c == 0) p.part_lse[pr] = lse_nat;
        }
    }
    if (nsplit == 1) return;

    // ---- last CTA of this (sequence, kv head, row group) merges the splits
    __threadfence();
    ptx::named_barrier_sync(1, 32 * kConsumerWarps);
    if (tid == 0) {
        const unsigned prev = atomicAdd(p.counters + unit, 1u);
        bars->is_last = (prev == (unsigned)(nsplit - 1)) ? 1 : 0;
    }
    ptx::named_barrier_sync(1, 32 * kConsumerWarps);
    if (!bars->is_last) return;
    __threadfence();
    const float* po = p.part_o + unit * p.max_splits * 16 * D;
    const float* pl = p.part_lse + unit * p.max_splits * 16;
    if (tid < 16) {
        const int r = tid;
        float M = -INFINITY;
        for (int s2 = 0; s2 < nsplit; ++s2) M = fmaxf(M, __ldcg(pl + s2 * 16 + r));
        float tot = -INFINITY;
        if (M != -INFINITY) {
            float acc = 0.f;
            for (int s2 = 0; s2 < nsplit; ++s2) {
                const float ls = __ldcg(pl + s2 * 16 + r);
                if (ls != -INFINITY) acc += __expf(ls - M);
            }
            tot = M + __logf(acc);
        }
        bars->row_lse[r] = tot;  // natural log
    }
    ptx::named_barrier_sync(1, 32 * kConsumerWarps);
    for (int idx = tid; idx < 16 * D; idx += nthr) {
        const int r = idx / D, c = idx % D;
        const int row = mg * 16 + r;
        if (row >= p.rows) continue;
        const float tot = bars->row_lse[r];
        float val = 0.f;
        if (tot != -INFINITY) {
            for (int s2 = 0; s2 < nsplit; ++s2) {
                const float ls = __ldcg(pl + s2 * 16 + r);
                if (ls != -INFINITY) val += __expf(ls - tot) * __ldcg(po + (s2 * 16 + r) * D + c);
            }
        }
        const int tok = row / p.G, head = g * p.G + row % p.G;
        store_out<BF16>(p.o, (((size_t)b * p.Nq + tok) * p.Hq + head) * D + c, val);
        if (c == 0) p.lse[((size_t)b * p.Hq + head) * p.Nq + tok] = tot;
    }
}

template <int D, bool BF16, int STAGES>
cudaError_t launch_decode_t(const CUtensorMap& kmap, const CUtensorMap& vmap,
                            const DecodeParams& p, cudaStream_t stream) {
    using L = DecSmem<D, STAGES>;
    static_assert(L::kAlloc <= 113 * 1024, "two CTAs per SM");
    auto kern = attn_decode_kernel<D, BF16, STAGES>;
    cudaError_t e =
        cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)L::kAlloc);
    if (e != cudaSuccess) return e;
    dim3 grid(p.max_splits * p.n_mgroups, p.Hkv, p.B);
    kern<<<grid, kThreads, L::kAlloc, stream>>>(kmap, vmap, p);
    return cudaGetLastError();
}

}  // namespace

DecodeLayout decode_layout(int B, int Hq, int Hkv, int Nq, int d, int max_seqlen_k,
                           int split_keys) {
    DecodeLayout l{};
    const int G = Hq / Hkv;
    const int rows = Nq * G;
    auto align = [](size_t x) { return (x + 255) & ~(size_t)255; };
    l.tc = decode_use_tc(G, Nq, split_keys) ? 1 : 0;
    if (l.tc) {
        // stream-K ranges: at most kDecodeMaxRangesAuto in automatic mode,
        // else ranges of split_keys / 128 tiles of weight
        const long units = (long)B * Hkv;
        const long w_max = units * ((max_seqlen_k + 127) / 128 + kDecodeSegCost);
        long ranges;
        if (split_keys <= 0)
            ranges = std::min<long>(kDecodeMaxRangesAuto,
                                    (w_max + kDecodeMinRangeWeight - 1) / kDecodeMinRangeWeight);
        else
            ranges = (w_max + split_keys / 128 - 1) / (split_keys / 128);
        l.max_ranges = (int)std::min<long>(ranges, 1L << 24);
        l.split_keys = split_keys;
        l.max_splits = 1;
        l.n_mgroups = 1;
        const size_t slots = 2 * (size_t)l.max_ranges;
        l.part_o_off = 0;
        l.part_lse_off = align(slots * 128 * (size_t)d * 4);
        l.counters_off = l.prefix_off = l.part_lse_off + align(slots * 128 * 4);
        l.ranges_off = l.prefix_off + align(((size_t)B + 1) * 8);
        l.plan_off = l.ranges_off + align((size_t)l.max_ranges * 8);
        l.total = l.plan_off + align(sizeof(DecodePlan));
        return l;
    }
    l.n_mgroups = (rows + 15) / 16;
    int split = split_keys;
    const long units = (long)B * Hkv * l.n_mgroups;
    if (split <= 0) {
        // enough work units to fill the GPU several times over, but splits of
        // at least 256 keys so that each unit amortises its set-up
        split = 1024;
        while (split > 256 && units * ((max_seqlen_k + split - 1) / split) < 148L * 2 * 8) split /= 2;
    }
    l.split_keys = split;
    l.max_splits = max_seqlen_k > 0 ? (max_seqlen_k + split - 1) / split : 1;
    const size_t n_units = (size_t)units;
    l.part_o_off = 0;
    l.part_lse_off = align(n_units * l.max_splits * 16 * (size_t)d * 4);
    l.counters_off = l.part_lse_off + align(n_units * l.max_splits * 16 * 4);
    l.prefix_off = l.ranges_off = l.plan_off = l.counters_off + align(n_units * 4);
    l.total = l.plan_off;
    return l;
}

cudaError_t launch_decode(const CUtensorMap& kmap, const CUtensorMap& vmap,
                          const DecodeParams& p, int d, bool bf16, cudaStream_t stream) {
    if (d == 64) {
        return bf16 ? launch_decode_t<64, true, 4>(kmap, vmap, p, stream)
                    : launch_decode_t<64, false, 4>(kmap, vmap, p, stream);
    }
    return bf16 ? launch_decode_t<128, true, 3>(kmap, vmap, p, stream)
                : launch_decode_t<128, false, 3>(kmap, vmap, p, stream);
}

}  // namespace attn
