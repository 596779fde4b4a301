// attn_decode_tc_sm100a.cu -- KV-cache decode on tcgen05 tensor cores for
// chunks of new tokens (Nq * Hq/Hkv query rows per kv head, 64 .. 128 rows).
//
// With 16 new tokens and 8 query heads per kv head, the 128 query rows that
// read one kv head form a full tcgen05 M = 128 tile, and the key loop is a
// dense contraction (128 FLOP per cache byte), so it runs on the tensor
// cores.  As in the one-token decode, only the filled rows of each sequence's
// cache are read and the key range is split to fill the GPU (ai6s.net
// article on the ops-transformer FlashAttention operator, section
// "ops-transformer 里的 FlashAttention 做了什么额外的事", point 3), and within a
// split the keys are processed tile by tile with a running max and sum
// (section "FlashAttention 拆的不是算法，是数据流").
//
// Scheduling.  A work item is (sequence b, kv head g, key split s).  A
// one-CTA plan kernel lists the items longest first (all full splits, then
// the last, shorter split of each sequence in decreasing length) and clears
// the counters; the decode kernel is persistent -- one CTA per SM -- and
// its loader warp takes items from the list with an atomic counter, so
// short items fill the end of the run and each CTA pays its set-up once.
// The loader moves on to the next item's Q and K/V tiles while the current
// one finishes, so the memory pipe stays busy across item boundaries.
//
// Query row r = t * G + hh is token t, query head g * G + hh; a 5-D TMA box
// gathers the 128 rows (tokens past Nq read as zeros).
// Warp roles (576 threads):
//   warps 0-15  softmax: rows 32*(w%4) .. +31, score columns 32*(w/4) .. +31
//   warp 16     loader: work list, Q, 128-key K / V tiles of the packed cache
//   warp 17     tensor-memory owner and tcgen05.mma issuer (elected lane)
// Tensor memory: S[0] [0,128), S[1] [128,256) double-buffered scores,
// O [256, 256+D), Q [384, 384+D/2).  The softmax warps copy each item's Q
// into tensor memory, so S = Q·Kᵀ reads only K from shared memory; P
// (bf16/fp16) overwrites the first 64 columns of its S buffer and is the A
// operand of P·V.
//
// With one split an item's O and LSE go straight to the output; otherwise
// the item writes its normalised partial O (fp32) and LSE to the workspace
// and the CTA that finishes the last split of a (sequence, kv head) -- found
// with an atomic counter, no spinning -- merges all splits in split order:
// LSE = log sum_s exp(LSE_s), O = sum_s exp(LSE_s - LSE) O_s.
//
// Every wait is a bounded mbarrier wait (named barriers cannot time out, and
// a persistent loop must be able to leave on an error at any point).
#include "attn_internal.h"
#include "ptx.cuh"

namespace attn {
namespace {

constexpr int kBlockM = 128;  // query rows per item
constexpr int kBlockN = 128;  // keys per K/V tile
constexpr int kSoftmaxWarps = 16;
constexpr int kThreads = 32 * (kSoftmaxWarps + 2);
constexpr int kItemRing = 4;
constexpr uint32_t kTmemCols = 512;
constexpr float kRescaleThreshold = 8.0f;
constexpr float kLn2 = 0.69314718055994531f;
constexpr int kPlanThreads = 1024;
constexpr int kPlanBuckets = 256;

template <int D, int KST, int VST>
struct TcSmem {
    static constexpr uint32_t kTileBytes = kBlockM * D * 2;
    static constexpr uint32_t kQ = 0;
    static constexpr uint32_t kK = kQ + kTileBytes;
    static constexpr uint32_t kV = kK + KST * kTileBytes;
    static constexpr uint32_t kRed = kV + VST * kTileBytes;    // [2 slots][4 parts][128] fp32
    static constexpr uint32_t kRowLse = kRed + 2 * 4 * 128 * 4;  // [128] fp32
    static constexpr uint32_t kBars = kRowLse + 128 * 4;
    static constexpr uint32_t kTotal = kBars + 1024;
    static constexpr uint32_t kAlloc = kTotal + 1024;
};

// One pushed work item: b < 0 ends the work.
struct TcItem {
    int b, g, split, nsplit, Lk, slot0, pad0, pad1;
};

template <int KST, int VST>
struct TcBars {
    uint64_t item_full[kItemRing];
    uint64_t item_empty[kItemRing];
    uint64_t q_full, q_empty, q_tmem;
    uint64_t k_full[KST];
    uint64_t k_empty[KST];
    uint64_t v_full[VST];
    uint64_t v_empty[VST];
    uint64_t s_full[2];
    uint64_t p_full[2];
    uint64_t o_done;   // one phase per P.V tile
    uint64_t o_final;  // one phase per item: every MMA of the item is complete
    uint64_t o_free;   // one phase per item: the softmax warps have read O
    uint64_t row_sync[4];
    uint64_t ep_sync;
    uint64_t drain;
    TcItem item[kItemRing];
    uint32_t tmem_base;
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

__device__ __forceinline__ bool warp_wait(uint64_t* bar, uint32_t parity, uint64_t limit_ns,
                                          volatile int* abort_flag) {
    const bool ok = ptx::mbar_wait(bar, parity, limit_ns, abort_flag);
    return __all_sync(0xffffffffu, ok);
}

// A barrier among the warps that arrive on `bar` (one arrival per warp),
// bounded; `uses` counts this warp's earlier passes.
__device__ __forceinline__ bool warp_barrier(uint64_t* bar, int& uses, uint64_t limit_ns,
                                             volatile int* abort_flag) {
    __syncwarp();
    if (ptx::lane_id() == 0) ptx::mbar_arrive(bar);
    const bool ok = warp_wait(bar, (uint32_t)(uses & 1), limit_ns, abort_flag);
    ++uses;
    return ok;
}

// Running maxima of 32 score columns; keys > row_lim are masked.
template <bool kMask>
__device__ __forceinline__ void part_max(const uint32_t (&r)[32], int key_base, int row_lim,
                                         float (&mx8)[8]) {
#pragma unroll
    for (int c = 0; c < 32; c += 16) {
#pragma unroll
        for (int u = 0; u < 8; ++u) {
            float v0 = __uint_as_float(r[c + u]);
            float v1 = __uint_as_float(r[c + 8 + u]);
            if (kMask) {
                if (key_base + c + u > row_lim) v0 = -INFINITY;
                if (key_base + c + 8 + u > row_lim) v1 = -INFINITY;
            }
            mx8[u] = ptx::max3(mx8[u], v0, v1);
        }
    }
}

// p = 2^(s * scale_log2 - m) for 32 score columns, summed and packed.  Every
// fourth pair uses the FMA-pipe 2^x of ptx.cuh.
template <bool kMask, bool BF16>
__device__ __forceinline__ void part_exp(const uint32_t (&r)[32], int key_base, int row_lim,
                                         uint64_t sl2_2, uint64_t nm_2, uint64_t (&acc2)[4],
                                         uint32_t (&pk)[16]) {
#pragma unroll
    for (int c = 0; c < 32; c += 2) {
        float v0 = __uint_as_float(r[c]);
        float v1 = __uint_as_float(r[c + 1]);
        if (kMask) {
            if (key_base + c > row_lim) v0 = -INFINITY;
            if (key_base + c + 1 > row_lim) v1 = -INFINITY;
        }
        const uint64_t t2 = ptx::f2_fma(ptx::f2_pack(v0, v1), sl2_2, nm_2);
        float p0, p1;
        if (((c >> 1) & 3) == 3) {
            ptx::f2_unpack(ptx::exp2_poly2(t2), p0, p1);
        } else {
            float t0, t1;
            ptx::f2_unpack(t2, t0, t1);
            p0 = ptx::ex2_approx(t0);
            p1 = ptx::ex2_approx(t1);
        }
        acc2[(c >> 1) & 3] = ptx::f2_add(acc2[(c >> 1) & 3], ptx::f2_pack(p0, p1));
        pk[c >> 1] = ptx::pack2<BF16>(p0, p1);
    }
}

// kPartD output columns of one row, scaled, as packed 16-bit values.
template <int kPartD, bool BF16>
__device__ __forceinline__ void store_row_part(void* o, size_t elem, const float* v, float sc) {
    uint4* dst = reinterpret_cast<uint4*>(static_cast<uint16_t*>(o) + elem);
#pragma unroll
    for (int e = 0; e < kPartD; e += 8)
        dst[e / 8] = make_uint4(ptx::pack2<BF16>(v[e] * sc, v[e + 1] * sc),
                                ptx::pack2<BF16>(v[e + 2] * sc, v[e + 3] * sc),
                                ptx::pack2<BF16>(v[e + 4] * sc, v[e + 5] * sc),
                                ptx::pack2<BF16>(v[e + 6] * sc, v[e + 7] * sc));
}

// ------------------------------------------------------------------ plan
// One CTA: lists the work items longest first and clears the counters.
// Items of a bucket (same number of key tiles, capped at 255) keep the
// order the atomics give; results do not depend on it, because every
// partial lands in its own (unit, split) slot and the merge sums in split
// order.
__global__ void __launch_bounds__(kPlanThreads)
    attn_decode_plan_kernel(const __grid_constant__ DecodeParams p) {
    __shared__ int hist[kPlanBuckets];
    __shared__ int offs[kPlanBuckets];
    const int tid = threadIdx.x;
    for (int k = tid; k < kPlanBuckets; k += kPlanThreads) hist[k] = 0;
    const int units = p.B * p.Hkv;
    for (int u = tid; u < units; u += kPlanThreads) p.counters[u] = 0u;
    __syncthreads();
    const int full_tiles = (p.split_keys + kBlockN - 1) / kBlockN;
    const int full_bucket = min(full_tiles, kPlanBuckets - 1);
    for (int b = tid; b < p.B; b += kPlanThreads) {
        const int L = p.seqlens_k[b];
        const int ns = L > 0 ? (L + p.split_keys - 1) / p.split_keys : 1;
        if (ns > p.max_splits || L < 0) {
            atomicCAS(p.err, 0u, kErrDecodeBase + 1);  // max_seqlen_k was too small
            continue;
        }
        const int last_tiles = (L - (ns - 1) * p.split_keys + kBlockN - 1) / kBlockN;
        if (ns > 1) atomicAdd(&hist[full_bucket], (ns - 1) * p.Hkv);
        atomicAdd(&hist[min(last_tiles, kPlanBuckets - 1)], p.Hkv);
    }
    __syncthreads();
    if (tid == 0) {
        int off = 0;
        for (int k = kPlanBuckets - 1; k >= 0; --k) {
            offs[k] = off;
            off += hist[k];
        }
        p.work_meta[0] = off;  // number of items
        p.work_meta[1] = 0;    // next item to take
    }
    __syncthreads();
    for (int b = tid; b < p.B; b += kPlanThreads) {
        const int L = p.seqlens_k[b];
        const int ns = L > 0 ? (L + p.split_keys - 1) / p.split_keys : 1;
        if (ns > p.max_splits || L < 0) continue;
        for (int s = 0; s < ns; ++s) {
            const int keys = min(L, (s + 1) * p.split_keys) - s * p.split_keys;
            const int bucket = min((keys + kBlockN - 1) / kBlockN, kPlanBuckets - 1);
            const int pos = atomicAdd(&offs[bucket], p.Hkv);
            for (int g = 0; g < p.Hkv; ++g) p.items[pos + g] = make_int4(b, g, s, ns);
        }
    }
}

// ------------------------------------------------------------------ decode
template <int D, bool BF16, int KST, int VST>
__global__ void __launch_bounds__(kThreads, 1)
    attn_decode_tc_kernel(const __grid_constant__ CUtensorMap tm_q,
                          const __grid_constant__ CUtensorMap tm_k,
                          const __grid_constant__ CUtensorMap tm_v,
                          const __grid_constant__ DecodeParams p) {
    using L = TcSmem<D, KST, VST>;
    constexpr uint32_t kTileBytes = L::kTileBytes;
    constexpr int kDBlocks = D / 64;
    constexpr uint32_t kBlockBytes = kBlockM * 128;
    constexpr uint32_t kIdescS = ptx::idesc_f16(kBlockM, kBlockN, BF16, false);
    constexpr uint32_t kIdescO = ptx::idesc_f16(kBlockM, D, BF16, true);
    constexpr uint32_t kColO = 256;
    constexpr uint32_t kColQ = 384;
    constexpr int kPartD = D / 4;
    constexpr int kLoaderWarp = kSoftmaxWarps, kMmaWarp = kSoftmaxWarps + 1;
    static_assert(sizeof(TcBars<KST, VST>) <= 1024, "barrier block");

    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw_addr = ptx::smem_u32(smem_raw);
    uint8_t* smem = smem_raw + (((raw_addr + 1023u) & ~1023u) - raw_addr);
    const uint32_t sbase = ptx::smem_u32(smem);
    TcBars<KST, VST>* bars = reinterpret_cast<TcBars<KST, VST>*>(smem + L::kBars);
    volatile int* abort_flag = &bars->abort;

    const int tid = threadIdx.x;
    const int warp = tid >> 5;
    const int lane = tid & 31;

    if (tid == 0) {
        for (int s = 0; s < kItemRing; ++s) {
            ptx::mbar_init(&bars->item_full[s], 1);
            ptx::mbar_init(&bars->item_empty[s], kSoftmaxWarps + 1);
        }
        ptx::mbar_init(&bars->q_full, 1);
        ptx::mbar_init(&bars->q_empty, kSoftmaxWarps);
        ptx::mbar_init(&bars->q_tmem, kSoftmaxWarps);
        for (int s = 0; s < KST; ++s) {
            ptx::mbar_init(&bars->k_full[s], 1);
            ptx::mbar_init(&bars->k_empty[s], 1);
        }
        for (int s = 0; s < VST; ++s) {
            ptx::mbar_init(&bars->v_full[s], 1);
            ptx::mbar_init(&bars->v_empty[s], 1);
        }
        for (int s = 0; s < 2; ++s) {
            ptx::mbar_init(&bars->s_full[s], 1);
            ptx::mbar_init(&bars->p_full[s], kSoftmaxWarps);
        }
        ptx::mbar_init(&bars->o_done, 1);
        ptx::mbar_init(&bars->o_final, 1);
        ptx::mbar_init(&bars->o_free, kSoftmaxWarps);
        for (int s = 0; s < 4; ++s) ptx::mbar_init(&bars->row_sync[s], 4);
        ptx::mbar_init(&bars->ep_sync, kSoftmaxWarps);
        ptx::mbar_init(&bars->drain, 1);
        bars->abort = 0;
        bars->is_last = 0;
        ptx::fence_barrier_init();
    }
    if (warp == kLoaderWarp && lane == 0) {
        ptx::prefetch_tmap(&tm_q);
        ptx::prefetch_tmap(&tm_k);
        ptx::prefetch_tmap(&tm_v);
    }
    if (warp == kMmaWarp) {
        ptx::tmem_alloc<kTmemCols>(&bars->tmem_base);
        ptx::tmem_relinquish();
    }
    ptx::tc_fence_before();
    __syncthreads();
    ptx::tc_fence_after();
    const uint32_t tmem = bars->tmem_base;

    auto item_tiles = [&](const TcItem& it, int& key_begin, int& key_end) {
        key_begin = it.split * p.split_keys;
        key_end = min(it.Lk, key_begin + p.split_keys);
        return (key_end - key_begin + kBlockN - 1) / kBlockN;  // 0 only for an empty sequence
    };

    if (warp == kLoaderWarp) {
        // ================================================= loader
        const int n_items = *reinterpret_cast<volatile int*>(p.work_meta);
        int n = 0;       // items pushed
        int it = 0;      // items with keys (Q loads)
        int tg = 0;      // K/V tile pairs issued
        int k_extra = 0;  // a K tile issued without its V tile (error exit)
        int w = 0;
        if (lane == 0) w = atomicAdd(p.work_meta + 1, 1);
        w = __shfl_sync(0xffffffffu, w, 0);
        while (true) {
            TcItem item{-1, 0, 0, 1, 0, 0, 0, 0};
            int w_next = 0;
            if (w < n_items) {
                const int4 e = p.items[w];
                item.b = e.x;
                item.g = e.y;
                item.split = e.z;
                item.nsplit = e.w;
                item.Lk = p.seqlens_k[e.x];
                item.slot0 = p.cu_seqlens_k[e.x];
                if (lane == 0) w_next = atomicAdd(p.work_meta + 1, 1);  // resolves later
            }
            const int slot = n % kItemRing;
            if (!warp_wait(&bars->item_empty[slot], ((n / kItemRing) & 1) ^ 1, p.limit_ns,
                           abort_flag)) {
                record_error(p.err, kErrDecodeBase + 2, &bars->abort);
                break;
            }
            if (lane == 0) {
                bars->item[slot] = item;
                ptx::mbar_arrive(&bars->item_full[slot]);
            }
            __syncwarp();
            ++n;
            if (item.b < 0) break;
            int key_begin, key_end;
            const int nt = item_tiles(item, key_begin, key_end);
            bool ok = true;
            if (nt > 0) {
                if (!warp_wait(&bars->q_empty, (it & 1) ^ 1, p.limit_ns, abort_flag)) {
                    record_error(p.err, kErrDecodeBase + 3, &bars->abort);
                    break;
                }
                if (lane == 0) {
                    ptx::mbar_arrive_expect_tx(&bars->q_full, kTileBytes);
                    for (int c = 0; c < kDBlocks; ++c)
                        ptx::tma_load_5d(smem + L::kQ + c * kBlockBytes, &tm_q, &bars->q_full,
                                         c * 64, 0, item.g, 0, item.b);
                }
                __syncwarp();
                ++it;
                for (int j = 0; j < nt; ++j, ++tg) {
                    const int row0 = item.slot0 + key_begin + j * kBlockN;
                    const int sk = tg % KST;
                    if (!warp_wait(&bars->k_empty[sk], ((tg / KST) & 1) ^ 1, p.limit_ns,
                                   abort_flag)) {
                        record_error(p.err, kErrDecodeBase + 4, &bars->abort);
                        ok = false;
                        break;
                    }
                    if (lane == 0) {
                        ptx::mbar_arrive_expect_tx(&bars->k_full[sk], kTileBytes);
                        for (int c = 0; c < kDBlocks; ++c)
                            ptx::tma_load_3d(smem + L::kK + sk * kTileBytes + c * kBlockBytes,
                                             &tm_k, &bars->k_full[sk], c * 64, item.g, row0);
                    }
                    __syncwarp();
                    const int sv = tg % VST;
                    if (!warp_wait(&bars->v_empty[sv], ((tg / VST) & 1) ^ 1, p.limit_ns,
                                   abort_flag)) {
                        record_error(p.err, kErrDecodeBase + 5, &bars->abort);
                        ok = false;
                        k_extra = 1;  // its K tile is in flight
                        break;
                    }
                    if (lane == 0) {
                        ptx::mbar_arrive_expect_tx(&bars->v_full[sv], kTileBytes);
                        for (int c = 0; c < kDBlocks; ++c)
                            ptx::tma_load_3d(smem + L::kV + sv * kTileBytes + c * kBlockBytes,
                                             &tm_v, &bars->v_full[sv], c * 64, item.g, row0);
                    }
                    __syncwarp();
                }
            }
            if (!ok) break;
            w = __shfl_sync(0xffffffffu, w_next, 0);
        }
        // leave no copy in flight: the last Q and up to KST / VST tiles
        int zero = 0;
        volatile int* no_abort = &zero;
        if (it > 0) ptx::mbar_wait(&bars->q_full, (it - 1) & 1, p.limit_ns, no_abort);
        const int kc = tg + k_extra;
        for (int j = max(0, kc - KST); j < kc; ++j)
            ptx::mbar_wait(&bars->k_full[j % KST], (j / KST) & 1, p.limit_ns, no_abort);
        for (int j = max(0, tg - VST); j < tg; ++j)
            ptx::mbar_wait(&bars->v_full[j % VST], (j / VST) & 1, p.limit_ns, no_abort);
    } else if (warp == kMmaWarp) {
        // ================================================= MMA issuer
        bool ok = true;
        bool issued = false;
        auto wait_or_fail = [&](uint64_t* bar, uint32_t parity, unsigned site) {
            if (!warp_wait(bar, parity, p.limit_ns, abort_flag)) {
                record_error(p.err, kErrDecodeBase + site, &bars->abort);
                ok = false;
            }
            return ok;
        };
        const uint64_t k_desc0 = ptx::sdesc_sw128(sbase + L::kK, 16, 1024);
        const uint64_t v_desc0 = ptx::sdesc_sw128(sbase + L::kV, kBlockBytes, 1024);
        constexpr uint64_t kTileUnits = kTileBytes >> 4;
        auto issue_s = [&](int t) {
            if (!wait_or_fail(&bars->k_full[t % KST], (t / KST) & 1, 6)) return;
            ptx::tc_fence_after();
            const uint64_t kd = k_desc0 + (uint64_t)(t % KST) * kTileUnits;
            const uint32_t d_s = tmem + (uint32_t)((t & 1) * kBlockN);
#pragma unroll
            for (int kk = 0; kk < D / 16; ++kk) {
                const uint64_t off = (uint64_t)(((kk >> 2) * kBlockBytes + (kk & 3) * 32) >> 4);
                ptx::umma_ts_elect(d_s, tmem + kColQ + kk * 8, kd + off, kIdescS, kk > 0);
            }
            ptx::umma_commit_elect(&bars->s_full[t & 1]);
            ptx::umma_commit_elect(&bars->k_empty[t % KST]);
            __syncwarp();
            issued = true;
        };
        int n = 0, it = 0, tg = 0;
        while (ok) {
            const int slot = n % kItemRing;
            if (!wait_or_fail(&bars->item_full[slot], (n / kItemRing) & 1, 7)) break;
            const TcItem item = bars->item[slot];
            __syncwarp();
            if (lane == 0) ptx::mbar_arrive(&bars->item_empty[slot]);
            ++n;
            if (item.b < 0) break;
            int key_begin, key_end;
            const int nt = item_tiles(item, key_begin, key_end);
            if (nt == 0) continue;
            if (!wait_or_fail(&bars->q_tmem, it & 1, 8)) break;
            ptx::tc_fence_after();
            issue_s(tg);
            for (int j = 0; ok && j < nt; ++j) {
                const int t = tg + j;
                if (j + 1 < nt) {
                    issue_s(t + 1);
                    if (!ok) break;
                }
                if (!wait_or_fail(&bars->p_full[t & 1], (t >> 1) & 1, 9)) break;
                if (!wait_or_fail(&bars->v_full[t % VST], (t / VST) & 1, 10)) break;
                if (j == 0 && !wait_or_fail(&bars->o_free, (it & 1) ^ 1, 11)) break;
                ptx::tc_fence_after();
                const uint64_t vd = v_desc0 + (uint64_t)(t % VST) * kTileUnits;
                const uint32_t a_p = tmem + (uint32_t)((t & 1) * kBlockN);
                const uint32_t acc0 = j > 0 ? 1u : 0u;
#pragma unroll
                for (int kk = 0; kk < kBlockN / 16; ++kk)
                    ptx::umma_ts_elect(tmem + kColO, a_p + kk * 8,
                                       vd + (uint64_t)((kk * 16 * 128) >> 4), kIdescO,
                                       kk > 0 ? 1u : acc0);
                ptx::umma_commit_elect(&bars->o_done);
                if (j == nt - 1) ptx::umma_commit_elect(&bars->o_final);
                ptx::umma_commit_elect(&bars->v_empty[t % VST]);
                __syncwarp();
            }
            tg += nt;
            ++it;
        }
        if (!ok && issued) {
            int zero = 0;
            volatile int* no_abort = &zero;
            ptx::umma_commit_elect(&bars->drain);
            __syncwarp();
            ptx::mbar_wait(&bars->drain, 0, p.limit_ns, no_abort);
        }
    } else {
        // ================================================= softmax warps
        const uint32_t quarter = (uint32_t)(warp & 3);
        const int part = warp >> 2;
        const uint32_t row = quarter * 32u + (uint32_t)lane;
        const uint32_t lane_addr = (quarter * 32u) << 16;
        const int tok = (int)row / p.G;  // token of this query row
        const int head_in_group = (int)row % p.G;
        const bool valid_row = (int)row < p.rows;
        const float sl2 = p.scale_log2;
        float* red = reinterpret_cast<float*>(smem + L::kRed);
        float* row_lse = reinterpret_cast<float*>(smem + L::kRowLse);
        const uint32_t t_o = tmem + lane_addr + kColO + (uint32_t)(part * kPartD);
        uint64_t* row_bar = &bars->row_sync[quarter];
        bool ok = true;
        int n = 0, it = 0, tg = 0, rs = 0, es = 0;

        while (ok) {
            const int slot = n % kItemRing;
            if (!warp_wait(&bars->item_full[slot], (n / kItemRing) & 1, p.limit_ns, abort_flag)) {
                record_error(p.err, kErrDecodeBase + 12, &bars->abort);
                break;
            }
            const TcItem item = bars->item[slot];
            __syncwarp();
            if (lane == 0) ptx::mbar_arrive(&bars->item_empty[slot]);
            ++n;
            if (item.b < 0) break;
            const int b = item.b, g = item.g;
            const int head = g * p.G + head_in_group;
            const size_t o_elem = (((size_t)b * p.Nq + tok) * p.Hq + head) * D + part * kPartD;
            const size_t lse_idx = ((size_t)b * p.Hq + head) * p.Nq + tok;
            int key_begin, key_end;
            const int nt = item_tiles(item, key_begin, key_end);
            if (nt == 0) {
                // empty sequence: nothing to attend to
                if (valid_row) {
                    float zeros[kPartD];
#pragma unroll
                    for (int e = 0; e < kPartD; ++e) zeros[e] = 0.f;
                    store_row_part<kPartD, BF16>(p.o, o_elem, zeros, 1.f);
                    if (part == 0) p.lse[lse_idx] = -INFINITY;
                }
                continue;
            }
            int row_lim = key_end - 1;  // last visible key (absolute index)
            if (p.causal) row_lim = min(row_lim, tok + item.Lk - p.Nq);

            // ---- Q -> tensor memory (A operand of S = Q Kᵀ)
            if (!warp_wait(&bars->q_full, it & 1, p.limit_ns, abort_flag)) {
                record_error(p.err, kErrDecodeBase + 13, &bars->abort);
                break;
            }
            if (part * 32 < D) {
                const int c0 = part * 32;
                const uint8_t* qrow = smem + L::kQ + (c0 >> 6) * kBlockBytes;
                uint32_t qv[16];
#pragma unroll
                for (int q4 = 0; q4 < 4; ++q4) {
                    const uint4 v4 = *reinterpret_cast<const uint4*>(
                        qrow + sw128_offset(row, (uint32_t)(((c0 & 63) >> 3) + q4)));
                    qv[4 * q4] = v4.x;
                    qv[4 * q4 + 1] = v4.y;
                    qv[4 * q4 + 2] = v4.z;
                    qv[4 * q4 + 3] = v4.w;
                }
                ptx::tmem_st16(tmem + lane_addr + kColQ + (uint32_t)(c0 >> 1), qv);
                ptx::tmem_wait_st();
            }
            ptx::tc_fence_before();
            __syncwarp();
            if (lane == 0) {
                ptx::mbar_arrive(&bars->q_tmem);
                ptx::mbar_arrive(&bars->q_empty);
            }

            float m_ref = -INFINITY;
            float l_part = 0.f;
            for (int j = 0; j < nt; ++j) {
                const int t = tg + j;
                const int sb = t & 1;
                if (!warp_wait(&bars->s_full[sb], (t >> 1) & 1, p.limit_ns, abort_flag)) {
                    record_error(p.err, kErrDecodeBase + 14, &bars->abort);
                    ok = false;
                    break;
                }
                ptx::tc_fence_after();
                const uint32_t t_s = tmem + lane_addr + (uint32_t)(sb * kBlockN);
                const int key_base = key_begin + j * kBlockN + part * 32;
                const bool masked = key_base + 31 > row_lim;
                uint32_t r[32];
                ptx::tmem_ld32(t_s + part * 32, r);
                float mx8[8];
#pragma unroll
                for (int u = 0; u < 8; ++u) mx8[u] = -INFINITY;
                ptx::tmem_wait_ld_dep(r);
                if (masked)
                    part_max<true>(r, key_base, row_lim, mx8);
                else
                    part_max<false>(r, key_base, row_lim, mx8);
                float* rm = red + (rs & 1) * 4 * 128;
                rm[part * 128 + row] = ptx::max3(ptx::max3(mx8[0], mx8[1], mx8[2]),
                                                 ptx::max3(mx8[3], mx8[4], mx8[5]),
                                                 fmaxf(mx8[6], mx8[7]));
                if (!warp_barrier(row_bar, rs, p.limit_ns, abort_flag)) {
                    record_error(p.err, kErrDecodeBase + 15, &bars->abort);
                    ok = false;
                    break;
                }
                const float mx = fmaxf(ptx::max3(rm[row], rm[128 + row], rm[256 + row]),
                                       rm[384 + row]);
                const float m_tile = mx * sl2;
                float alpha = 1.f;
                bool rescale = false;
                if (m_tile > m_ref + kRescaleThreshold) {
                    alpha = ptx::ex2_approx(m_ref - m_tile);
                    rescale = (j > 0) && (m_ref != -INFINITY);
                    m_ref = m_tile;
                }
                const float m_use = (m_ref == -INFINITY) ? 0.f : m_ref;
                uint64_t acc2[4] = {0, 0, 0, 0};
                uint32_t pk[16];
                if (masked)
                    part_exp<true, BF16>(r, key_base, row_lim, ptx::f2_pack(sl2, sl2),
                                         ptx::f2_pack(-m_use, -m_use), acc2, pk);
                else
                    part_exp<false, BF16>(r, key_base, row_lim, ptx::f2_pack(sl2, sl2),
                                          ptx::f2_pack(-m_use, -m_use), acc2, pk);
                ptx::tmem_st16(t_s + part * 16, pk);
                float s0, s1, s2, s3, s4, s5, s6, s7;
                ptx::f2_unpack(acc2[0], s0, s1);
                ptx::f2_unpack(acc2[1], s2, s3);
                ptx::f2_unpack(acc2[2], s4, s5);
                ptx::f2_unpack(acc2[3], s6, s7);
                l_part = l_part * alpha + (((s0 + s1) + (s2 + s3)) + ((s4 + s5) + (s6 + s7)));
                if (__any_sync(0xffffffffu, rescale)) {
                    // S_t done implies P_{t-2} V_{t-2} is: phase t-1 of o_done
                    // is the current or the previous one, so the parity wait is
                    // exact (P_t V_t needs this warp's arrival below)
                    if (!warp_wait(&bars->o_done, (t - 1) & 1, p.limit_ns, abort_flag)) {
                        record_error(p.err, kErrDecodeBase + 14, &bars->abort);
                        ok = false;
                        ptx::tmem_wait_st();
                        break;
                    }
                    ptx::tc_fence_after();
                    const float sc = rescale ? alpha : 1.f;
                    if constexpr (kPartD == 32) {
                        uint32_t o[32];
                        ptx::tmem_ld32(t_o, o);
                        ptx::tmem_wait_ld_dep(o);
#pragma unroll
                        for (int e = 0; e < 32; ++e)
                            o[e] = __float_as_uint(__uint_as_float(o[e]) * sc);
                        ptx::tmem_st32(t_o, o);
                    } else {
                        uint32_t o[16];
                        ptx::tmem_ld16(t_o, o);
                        ptx::tmem_wait_ld_dep16(o);
#pragma unroll
                        for (int e = 0; e < 16; ++e)
                            o[e] = __float_as_uint(__uint_as_float(o[e]) * sc);
                        ptx::tmem_st16(t_o, o);
                    }
                }
                ptx::tmem_wait_st();
                if (key_begin + j * kBlockN + kBlockN > key_end && part == 0) {
                    // rows past the item's last key: zero their V rows (0 * NaN guard)
                    const int sv = t % VST;
                    if (!warp_wait(&bars->v_full[sv], (t / VST) & 1, p.limit_ns, abort_flag)) {
                        record_error(p.err, kErrDecodeBase + 14, &bars->abort);
                        ok = false;
                        break;
                    }
                    if (key_begin + j * kBlockN + (int)row >= key_end) {
                        uint8_t* vt = smem + L::kV + sv * kTileBytes;
#pragma unroll
                        for (int c = 0; c < kDBlocks; ++c)
#pragma unroll
                            for (int ch = 0; ch < 8; ++ch)
                                *reinterpret_cast<uint4*>(vt + c * kBlockBytes + row * 128 +
                                                          ch * 16) = make_uint4(0, 0, 0, 0);
                    }
                    ptx::fence_proxy_async_smem();
                }
                ptx::tc_fence_before();
                __syncwarp();
                if (lane == 0) ptx::mbar_arrive(&bars->p_full[sb]);
            }
            if (!ok) break;
            tg += nt;

            // ---- this item's O and LSE
            if (!warp_wait(&bars->o_final, it & 1, p.limit_ns, abort_flag)) {
                record_error(p.err, kErrDecodeBase + 14, &bars->abort);
                break;
            }
            ptx::tc_fence_after();
            float* rsum = red + (rs & 1) * 4 * 128;
            rsum[part * 128 + row] = l_part;
            uint32_t o[kPartD];
            if constexpr (kPartD == 32) {
                ptx::tmem_ld32(t_o, o);
                ptx::tmem_wait_ld_dep(o);
            } else {
                ptx::tmem_ld16(t_o, o);
                ptx::tmem_wait_ld_dep16(o);
            }
            ptx::tc_fence_before();
            __syncwarp();
            if (lane == 0) ptx::mbar_arrive(&bars->o_free);
            ++it;
            if (!warp_barrier(row_bar, rs, p.limit_ns, abort_flag)) {
                record_error(p.err, kErrDecodeBase + 15, &bars->abort);
                break;
            }
            const float l_sum = (rsum[row] + rsum[128 + row]) + (rsum[256 + row] + rsum[384 + row]);
            const bool have = l_sum > 0.f;
            const float inv_l = have ? 1.f / l_sum : 0.f;
            const float lse_nat = have ? (m_ref + ptx::lg2_approx(l_sum)) * kLn2 : -INFINITY;
            float of[kPartD];
#pragma unroll
            for (int e = 0; e < kPartD; ++e) of[e] = __uint_as_float(o[e]);
            if (item.nsplit == 1) {
                if (valid_row) {
                    store_row_part<kPartD, BF16>(p.o, o_elem, of, inv_l);
                    if (part == 0) p.lse[lse_idx] = lse_nat;
                }
                continue;
            }
            // normalised partial O (fp32) and LSE of this split
            const size_t unit = (size_t)b * p.Hkv + g;
            const size_t pbase = (unit * p.max_splits + item.split) * kBlockM + row;
            float* po = p.part_o + pbase * D + part * kPartD;
#pragma unroll
            for (int e = 0; e < kPartD; e += 4)
                *reinterpret_cast<float4*>(po + e) = make_float4(
                    of[e] * inv_l, of[e + 1] * inv_l, of[e + 2] * inv_l, of[e + 3] * inv_l);
            if (part == 0) p.part_lse[pbase] = lse_nat;
            // the CTA that completes the last split of this unit merges them
            __threadfence();
            if (!warp_barrier(&bars->ep_sync, es, p.limit_ns, abort_flag)) {
                record_error(p.err, kErrDecodeBase + 15, &bars->abort);
                break;
            }
            if (tid == 0) {
                const unsigned prev = atomicAdd(p.counters + unit, 1u);
                bars->is_last = (prev == (unsigned)(item.nsplit - 1)) ? 1 : 0;
            }
            if (!warp_barrier(&bars->ep_sync, es, p.limit_ns, abort_flag)) {
                record_error(p.err, kErrDecodeBase + 15, &bars->abort);
                break;
            }
            if (!bars->is_last) continue;
            __threadfence();
            const float* pl = p.part_lse + unit * p.max_splits * kBlockM;
            const float* pov = p.part_o + unit * p.max_splits * kBlockM * D;
            if (tid < kBlockM) {
                float M = -INFINITY;
                for (int s2 = 0; s2 < item.nsplit; ++s2)
                    M = fmaxf(M, __ldcg(pl + s2 * kBlockM + tid));
                float tot = -INFINITY;
                if (M != -INFINITY) {
                    float acc = 0.f;
                    for (int s2 = 0; s2 < item.nsplit; ++s2) {
                        const float ls = __ldcg(pl + s2 * kBlockM + tid);
                        if (ls != -INFINITY) acc += __expf(ls - M);
                    }
                    tot = M + __logf(acc);
                }
                row_lse[tid] = tot;
            }
            if (!warp_barrier(&bars->ep_sync, es, p.limit_ns, abort_flag)) {
                record_error(p.err, kErrDecodeBase + 15, &bars->abort);
                break;
            }
            if (valid_row) {
                const float tot = row_lse[row];
                float acc[kPartD];
#pragma unroll
                for (int e = 0; e < kPartD; ++e) acc[e] = 0.f;
                if (tot != -INFINITY) {
                    for (int s2 = 0; s2 < item.nsplit; ++s2) {
                        const float ls = __ldcg(pl + s2 * kBlockM + row);
                        if (ls == -INFINITY) continue;
                        const float wgt = __expf(ls - tot);
                        const float* src = pov + ((size_t)s2 * kBlockM + row) * D + part * kPartD;
#pragma unroll
                        for (int e = 0; e < kPartD; e += 4) {
                            const float4 v4 = __ldcg(reinterpret_cast<const float4*>(src + e));
                            acc[e] += wgt * v4.x;
                            acc[e + 1] += wgt * v4.y;
                            acc[e + 2] += wgt * v4.z;
                            acc[e + 3] += wgt * v4.w;
                        }
                    }
                }
                store_row_part<kPartD, BF16>(p.o, o_elem, acc, 1.f);
                if (part == 0) p.lse[lse_idx] = tot;
            }
        }
    }

    ptx::tc_fence_before();
    __syncthreads();
    if (warp == kMmaWarp) {
        __syncwarp();
        ptx::tc_fence_after();
        ptx::tmem_dealloc<kTmemCols>(tmem);
    }
}

template <int D, bool BF16, int KST, int VST>
cudaError_t launch_t(const CUtensorMap& qmap, const CUtensorMap& kmap, const CUtensorMap& vmap,
                     const DecodeParams& p, int n_ctas, cudaStream_t stream) {
    using L = TcSmem<D, KST, VST>;
    static_assert(L::kAlloc <= 227 * 1024, "shared memory budget");
    auto kern = attn_decode_tc_kernel<D, BF16, KST, VST>;
    cudaError_t e =
        cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)L::kAlloc);
    if (e != cudaSuccess) return e;
    attn_decode_plan_kernel<<<1, kPlanThreads, 0, stream>>>(p);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    kern<<<n_ctas, kThreads, L::kAlloc, stream>>>(qmap, kmap, vmap, p);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_decode_tc(const CUtensorMap& qmap, const CUtensorMap& kmap,
                             const CUtensorMap& vmap, const DecodeParams& p, int d, bool bf16,
                             int n_ctas, cudaStream_t stream) {
    if (d == 64) {
        return bf16 ? launch_t<64, true, 4, 4>(qmap, kmap, vmap, p, n_ctas, stream)
                    : launch_t<64, false, 4, 4>(qmap, kmap, vmap, p, n_ctas, stream);
    }
    return bf16 ? launch_t<128, true, 2, 3>(qmap, kmap, vmap, p, n_ctas, stream)
                : launch_t<128, false, 2, 3>(qmap, kmap, vmap, p, n_ctas, stream);
}

}  // namespace attn
