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
// Scheduling (stream-K style).  Unit (b, g) -- sequence b, kv head g --
// weighs its 128-key tiles plus a fixed set-up weight; the units are laid
// end to end and the total weight is cut into equal ranges, one per CTA of
// a persistent grid (one CTA per SM).  A CTA walks its range unit by unit;
// a unit is split only where a range boundary falls inside it, so every CTA
// gets the same work whatever the length mix, and only the (at most two)
// units at the ends of a range need a merge.  A one-CTA plan kernel computes
// the weight prefix over sequences and each range's first and last unit.
// The loader warp moves on to the next unit's Q and K/V tiles while the
// current one finishes, so the memory pipe stays busy across unit
// boundaries.
//
// Query row r = t * G + hh is token t, query head g * G + hh; a 5-D TMA box
// gathers the 128 rows (tokens past Nq read as zeros).
// Warp roles (576 threads):
//   warps 0-15  softmax: rows 32*(w%4) .. +31, score columns 32*(w/4) .. +31
//   warp 16     loader: work list, Q, 128-key K / V tiles
//   warp 17     tensor-memory owner and tcgen05.mma issuer (elected lane)
// Tensor memory: S[0] [0,128), S[1] [128,256) double-buffered scores,
// O [256, 256+D), Q [384, 384+D/2).  The softmax warps copy each item's Q
// into tensor memory, so S = Q·Kᵀ reads only K from shared memory; P
// (bf16/fp16) overwrites the first 64 columns of its S buffer and is the A
// operand of P·V.
//
// A unit done in one piece writes O and LSE straight to the output; a
// split unit writes each piece's normalised partial O (fp32) and LSE to the
// slot its range owns (range r: slot 2r for a unit continuing from range
// r-1, slot 2r+1 for a unit continuing into range r+1), and a small merge
// kernel that runs after the decode combines the pieces in key order:
// LSE = log sum_s exp(LSE_s), O = sum_s exp(LSE_s - LSE) O_s.  (Merging in
// the decode kernel, by whichever CTA finishes a unit's last piece, put a
// fence, an atomic and dependent cache misses under full memory load at the
// end of the run.)
//
// Every wait is a bounded mbarrier wait (named barriers cannot time out, and
// a persistent loop must be able to leave on an error at any point).
#include <algorithm>

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

template <int D, int KST, int VST>
struct TcSmem {
    static constexpr uint32_t kTileBytes = kBlockM * D * 2;
    static constexpr uint32_t kQ = 0;
    static constexpr uint32_t kK = kQ + kTileBytes;
    static constexpr uint32_t kV = kK + KST * kTileBytes;
    static constexpr uint32_t kRed = kV + VST * kTileBytes;    // [2 slots][4 parts][128] fp32
    static constexpr uint32_t kBars = kRed + 2 * 4 * 128 * 4;
    static constexpr uint32_t kTotal = kBars + 1024;
    static constexpr uint32_t kAlloc = kTotal + 1024;
};

// One pushed piece of work: keys [key_begin, key_end) of unit (b, g), piece
// seg of nseg, inside range `range`; b < 0 ends the work.
struct TcItem {
    int b, g, key_begin, key_end, nseg, seg, range, Lk, slot0, pad0, pad1, pad2;
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
    uint64_t drain;
    TcItem item[kItemRing];
    uint32_t tmem_base;
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
// Key length of sequence b as the schedule sees it; a length outside
// [0, max_seqlen_k] is reported (by the plan) and treated as empty.
__device__ __forceinline__ int checked_len(const DecodeParams& p, int b) {
    const int L = p.seqlens_k[b];
    return (L < 0 || L > p.max_seqlen_k) ? 0 : L;
}

// One CTA: the exclusive prefix of sequence weights Hkv * (tiles_b + set-up),
// the ranges, and each range's first and last unit (binary search over the
// prefix).
__global__ void __launch_bounds__(kPlanThreads)
    attn_decode_plan_kernel(const __grid_constant__ DecodeParams p, int n_ctas) {
    __shared__ long long warp_incl[kPlanThreads / 32];
    __shared__ long long carry;
    const int tid = threadIdx.x;
    const int lane = tid & 31, warp = tid >> 5;
    if (tid == 0) carry = 0;
    __syncthreads();
    for (int base = 0; base < p.B; base += kPlanThreads) {
        const int b = base + tid;
        long long w = 0;
        if (b < p.B) {
            const int L = p.seqlens_k[b];
            if (L < 0 || L > p.max_seqlen_k) atomicCAS(p.err, 0u, kErrDecodeBase + 1);
            w = (long long)p.Hkv * ((checked_len(p, b) + kBlockN - 1) / kBlockN + kDecodeSegCost);
        }
        long long x = w;  // inclusive scan within the warp
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const long long y = __shfl_up_sync(0xffffffffu, x, o);
            if (lane >= o) x += y;
        }
        if (lane == 31) warp_incl[warp] = x;
        __syncthreads();
        if (warp == 0) {
            long long t = warp_incl[lane];
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const long long y = __shfl_up_sync(0xffffffffu, t, o);
                if (lane >= o) t += y;
            }
            warp_incl[lane] = t;
        }
        __syncthreads();
        const long long before = carry + (warp > 0 ? warp_incl[warp - 1] : 0) + (x - w);
        if (b < p.B) p.seq_prefix[b] = before;
        __syncthreads();
        if (tid == kPlanThreads - 1) carry = before + w;
        __syncthreads();
    }
    const long long total = carry;
    long long rw = 0, n_ranges;
    if (p.split_keys > 0) {
        rw = p.split_keys / kBlockN;
        n_ranges = (total + rw - 1) / rw;
    } else {
        // balanced: range r starts at floor(r * total / n_ranges)
        n_ranges = (total + kDecodeMinRangeWeight - 1) / kDecodeMinRangeWeight;
        n_ranges = max(1ll, min(n_ranges, (long long)n_ctas));
    }
    if (n_ranges > p.max_ranges) {  // cannot happen for lengths <= max_seqlen_k
        if (tid == 0) atomicCAS(p.err, 0u, kErrDecodeBase + 2);
        n_ranges = 0;
    }
    if (tid == 0) {
        p.seq_prefix[p.B] = total;
        p.plan->range_weight = rw;
        p.plan->total_weight = total;
        p.plan->n_ranges = (int)n_ranges;
    }
    // the unit holding weight position x: last sequence whose prefix is <= x,
    // then the kv head within it
    auto unit_at = [&](long long x) {
        int lo = 0, hi = p.B - 1;
        while (lo < hi) {
            const int mid = (lo + hi + 1) >> 1;
            if (p.seq_prefix[mid] <= x) lo = mid;
            else hi = mid - 1;
        }
        const long long wu = (checked_len(p, lo) + kBlockN - 1) / kBlockN + kDecodeSegCost;
        return lo * p.Hkv + (int)min((long long)(p.Hkv - 1), (x - p.seq_prefix[lo]) / wu);
    };
    for (long long r = tid; r < n_ranges; r += kPlanThreads) {
        const long long a = plan_range_begin(rw, total, n_ranges, r);
        const long long e = min(total, plan_range_begin(rw, total, n_ranges, r + 1));
        p.range_units[r] = make_int2(unit_at(a), unit_at(e - 1));
    }
}

// Partial slot of piece `seg` of a unit whose piece lies in range r: the
// unit's first piece takes its range's slot 2r + 1 (a unit continuing into
// the next range), every later piece its range's slot 2r (a unit continuing
// from the previous range).  A range holds at most one of each.
__device__ __forceinline__ int piece_slot(int r, int seg) { return seg == 0 ? 2 * r + 1 : 2 * r; }

// ------------------------------------------------------------------ merge
// One CTA per range (looping when there are more ranges than CTAs): if the
// last unit of range r has its first piece in r and continues into later
// ranges, combine its pieces in key order,
//   LSE = log sum_s exp(LSE_s),  O = sum_s exp(LSE_s - LSE) O_s,
// one thread per (row, quarter of the head dimension).
template <int D, bool BF16>
__global__ void __launch_bounds__(4 * kBlockM, 1)
    attn_decode_merge_kernel(const __grid_constant__ DecodeParams p) {
    constexpr int kPartD = D / 4;
    const volatile DecodePlan* plan = p.plan;
    const long long rw = plan->range_weight;
    const long long total = plan->total_weight;
    const int n_ranges = plan->n_ranges;
    const int row = threadIdx.x % kBlockM;
    const int part = threadIdx.x / kBlockM;
    if (row >= p.rows) return;
    const int tok = row / p.G;
    const int head_in_group = row % p.G;
    for (int r = blockIdx.x; r < n_ranges; r += gridDim.x) {
        const int u = p.range_units[r].y;
        const int b = u / p.Hkv, g = u - b * p.Hkv;
        const int tiles = (checked_len(p, b) + kBlockN - 1) / kBlockN;
        if (tiles == 0) continue;
        const long long k0 = p.seq_prefix[b] + (long long)g * (tiles + kDecodeSegCost) +
                             kDecodeSegCost;
        if (plan_range_of(rw, total, n_ranges, k0) != r) continue;
        const int nseg = (int)plan_range_of(rw, total, n_ranges, k0 + tiles - 1) - r + 1;
        if (nseg == 1) continue;
        float M = -INFINITY;
        for (int s = 0; s < nseg; ++s)
            M = fmaxf(M, p.part_lse[(size_t)piece_slot(r + s, s) * kBlockM + row]);
        float tot = -INFINITY;
        float acc[kPartD];
#pragma unroll
        for (int e = 0; e < kPartD; ++e) acc[e] = 0.f;
        if (M != -INFINITY) {
            float sum = 0.f;
            for (int s = 0; s < nseg; ++s) {
                const size_t sb = (size_t)piece_slot(r + s, s) * kBlockM + row;
                const float ls = p.part_lse[sb];
                const float w = ls == -INFINITY ? 0.f : __expf(ls - M);
                sum += w;
                const float4* src = reinterpret_cast<const float4*>(p.part_o + sb * D +
                                                                     part * kPartD);
#pragma unroll
                for (int e = 0; e < kPartD / 4; ++e) {
                    const float4 v4 = src[e];
                    acc[4 * e] += w * v4.x;
                    acc[4 * e + 1] += w * v4.y;
                    acc[4 * e + 2] += w * v4.z;
                    acc[4 * e + 3] += w * v4.w;
                }
            }
            tot = M + __logf(sum);
            const float inv = 1.f / sum;
#pragma unroll
            for (int e = 0; e < kPartD; ++e) acc[e] *= inv;
        }
        const int head = g * p.G + head_in_group;
        store_row_part<kPartD, BF16>(
            p.o, (((size_t)b * p.Nq + tok) * p.Hq + head) * D + part * kPartD, acc, 1.f);
        if (part == 0) p.lse[((size_t)b * p.Hq + head) * p.Nq + tok] = tot;
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
    // A tile's keys arrive in runs of 2^sub_shift rows: a paged cache's block
    // (or a 128-row piece of a larger one), or the whole tile of a packed
    // cache.  K is laid out [64-column block][row][128 B]; V is laid out
    // [run][64-column block][run row][128 B], so that one TMA box brings a
    // run's rows with all their columns (a 16-row block then costs one V
    // box instead of D / 64; the number of boxes, not of bytes, bounds a
    // 16-row paged decode).  For the whole tile the two layouts coincide.
    const int sub_shift = p.block_table ? min(7, p.block_shift) : 7;
    const uint32_t run_bytes = (uint32_t)D * 2u << sub_shift;
    auto v_row = [&](int key) -> uint32_t {  // byte offset of tile row `key`, block 0
        return (uint32_t)(key >> sub_shift) * run_bytes +
               (uint32_t)(key & ((1 << sub_shift) - 1)) * 128u;
    };

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
        ptx::mbar_init(&bars->drain, 1);
        bars->abort = 0;
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
        key_begin = it.key_begin;
        key_end = it.key_end;
        return (key_end - key_begin + kBlockN - 1) / kBlockN;  // 0 only for an empty sequence
    };

    if (warp == kLoaderWarp) {
        // ================================================= loader
        const volatile DecodePlan* plan = p.plan;
        const long long rw = plan->range_weight;
        const long long total = plan->total_weight;
        const int n_ranges = plan->n_ranges;
        // the units of range r, first to last (those outside it give no piece)
        int r = blockIdx.x;
        int2 ru = r < n_ranges ? p.range_units[r] : make_int2(0, -1);
        int step = 0;
        auto next_item = [&](TcItem& item) {
            item = TcItem{-1, 0, 0, 0, 1, 0, 0, 0, 0, 0, 0, 0};
            while (r < n_ranges) {
                const long long a = plan_range_begin(rw, total, n_ranges, r);
                const long long e = min(total, plan_range_begin(rw, total, n_ranges, r + 1));
                while (step <= ru.y - ru.x) {
                    const int u = ru.x + step;
                    ++step;
                    const int b = u / p.Hkv, g = u - b * p.Hkv;
                    const int Lk = checked_len(p, b);
                    const int tiles = (Lk + kBlockN - 1) / kBlockN;
                    const long long pu = p.seq_prefix[b] + (long long)g * (tiles + kDecodeSegCost);
                    const long long k0 = pu + kDecodeSegCost;  // weight position of tile 0
                    int t0 = 0, t1 = 0, nseg = 1, seg = 0;
                    if (tiles == 0) {
                        if (pu < a || pu >= e) continue;  // owned by the range holding pu
                    } else {
                        t0 = (int)min((long long)tiles, max(0ll, a - k0));
                        t1 = (int)min((long long)tiles, max(0ll, e - k0));
                        if (t1 <= t0) continue;
                        const int r_first = (int)plan_range_of(rw, total, n_ranges, k0);
                        nseg = (int)plan_range_of(rw, total, n_ranges, k0 + tiles - 1) - r_first + 1;
                        seg = r - r_first;
                    }
                    item.b = b;
                    item.g = g;
                    item.key_begin = t0 * kBlockN;
                    item.key_end = min(Lk, t1 * kBlockN);
                    item.nseg = nseg;
                    item.seg = seg;
                    item.range = r;
                    item.Lk = Lk;
                    item.slot0 = p.block_table ? 0 : p.cu_seqlens_k[b];  // packed cache only
                    return;
                }
                r += gridDim.x;  // this range is done
                step = 0;
                if (r < n_ranges) ru = p.range_units[r];
            }
        };
        // a paged cache is read in runs of sub_rows rows (one block, or one
        // 128-row tile of a larger block)
        const int sub_rows = 1 << sub_shift;
        const int n_sub = kBlockN / sub_rows;
        int n = 0;        // items pushed
        int it = 0;       // items with keys (Q loads)
        int tg = 0;       // K/V tile pairs issued
        int k_extra = 0;  // a K tile issued without its V tile (error exit)
        TcItem item;
        next_item(item);
        while (true) {
            const int slot = n % kItemRing;
            if (!warp_wait(&bars->item_empty[slot], ((n / kItemRing) & 1) ^ 1, p.limit_ns,
                           abort_flag)) {
                record_error(p.err, kErrDecodeBase + 3, &bars->abort);
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
            TcItem next;
            bool have_next = false;
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
                    // cache rows of the tile's keys: one contiguous run in a
                    // packed cache; in a paged cache, runs of sub_rows keys
                    // found through the block table (lane u: run u)
                    int row0 = item.slot0 + key_begin + j * kBlockN;
                    if (p.block_table) {
                        row0 = 0;
                        if (lane < n_sub) {
                            const int pos = key_begin + j * kBlockN + lane * sub_rows;
                            const int lb = pos >> p.block_shift;
                            int blk = 0;
                            if (pos < item.Lk) {
                                blk = lb < p.max_blocks
                                          ? p.block_table[(size_t)item.b * p.max_blocks + lb]
                                          : -1;
                                if (blk < 0 || blk >= p.num_blocks) {  // a bad table entry
                                    atomicCAS(p.err, 0u, kErrDecodeBase + 8);
                                    blk = 0;
                                }
                            }
                            row0 = (blk << p.block_shift) + (pos & ((1 << p.block_shift) - 1));
                        }
                    }
                    // issue the tile's copies, lane u run u (the lanes' copies
                    // go out together): for K one box per 64-column block, each
                    // at its own place in the tile; for V one box per run
                    auto load_k = [&](uint8_t* dst, uint64_t* bar) {
                        if (lane < n_sub)
                            for (int c = 0; c < kDBlocks; ++c)
                                ptx::tma_load_3d(dst + c * kBlockBytes + lane * sub_rows * 128,
                                                 &tm_k, bar, c * 64, item.g, row0);
                    };
                    auto load_v = [&](uint8_t* dst, uint64_t* bar) {
                        if (lane < n_sub)
                            ptx::tma_load_4d(dst + lane * run_bytes, &tm_v, bar, 0, row0, 0,
                                             item.g);
                    };
                    const int sk = tg % KST;
                    if (!warp_wait(&bars->k_empty[sk], ((tg / KST) & 1) ^ 1, p.limit_ns,
                                   abort_flag)) {
                        record_error(p.err, kErrDecodeBase + 4, &bars->abort);
                        ok = false;
                        break;
                    }
                    if (lane == 0) ptx::mbar_arrive_expect_tx(&bars->k_full[sk], kTileBytes);
                    __syncwarp();
                    load_k(smem + L::kK + sk * kTileBytes, &bars->k_full[sk]);
                    __syncwarp();
                    const int sv = tg % VST;
                    if (!warp_wait(&bars->v_empty[sv], ((tg / VST) & 1) ^ 1, p.limit_ns,
                                   abort_flag)) {
                        record_error(p.err, kErrDecodeBase + 5, &bars->abort);
                        ok = false;
                        k_extra = 1;  // its K tile is in flight
                        break;
                    }
                    if (lane == 0) ptx::mbar_arrive_expect_tx(&bars->v_full[sv], kTileBytes);
                    __syncwarp();
                    load_v(smem + L::kV + sv * kTileBytes, &bars->v_full[sv]);
                    __syncwarp();
                    if (j == 0) {
                        // look the next piece up while this one's tiles stream in
                        next_item(next);
                        have_next = true;
                    }
                }
            }
            if (!ok) break;
            if (!have_next) next_item(next);
            item = next;
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
        // V: 64-column blocks of a run 2^sub_shift rows apart, 8-row groups 1024 B
        const uint64_t v_desc0 = ptx::sdesc_sw128(sbase + L::kV, 128u << sub_shift, 1024);
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
                                       vd + (uint64_t)(v_row(kk * 16) >> 4), kIdescO,
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
        const uint32_t t_o = tmem + lane_addr + kColO + (uint32_t)(part * kPartD);
        uint64_t* row_bar = &bars->row_sync[quarter];
        bool ok = true;
        int n = 0, it = 0, tg = 0, rs = 0;

        // The softmax warps keep an item's ring slot until they start the
        // next item and read its fields from shared memory when needed
        // (fewer live registers across the tile loop).
        while (ok) {
            if (n > 0) {
                __syncwarp();
                if (lane == 0) ptx::mbar_arrive(&bars->item_empty[(n - 1) % kItemRing]);
            }
            const int slot = n % kItemRing;
            if (!warp_wait(&bars->item_full[slot], (n / kItemRing) & 1, p.limit_ns, abort_flag)) {
                record_error(p.err, kErrDecodeBase + 12, &bars->abort);
                break;
            }
            const TcItem* itp = &bars->item[slot];
            ++n;
            if (itp->b < 0) break;
            auto out_index = [&](size_t& o_elem, size_t& lse_idx) {
                const int head = itp->g * p.G + head_in_group;
                o_elem = (((size_t)itp->b * p.Nq + tok) * p.Hq + head) * D + part * kPartD;
                lse_idx = ((size_t)itp->b * p.Hq + head) * p.Nq + tok;
            };
            const int key_begin = itp->key_begin, key_end = itp->key_end;
            const int nt = (key_end - key_begin + kBlockN - 1) / kBlockN;
            if (nt == 0) {
                size_t o_elem, lse_idx;
                out_index(o_elem, lse_idx);
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
            if (p.causal) row_lim = min(row_lim, tok + itp->Lk - p.Nq);

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
                        uint8_t* vt = smem + L::kV + sv * kTileBytes + v_row((int)row);
#pragma unroll
                        for (int c = 0; c < kDBlocks; ++c)
#pragma unroll
                            for (int ch = 0; ch < 8; ++ch)
                                *reinterpret_cast<uint4*>(vt + (c * 128u << sub_shift) +
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
            size_t o_elem, lse_idx;
            out_index(o_elem, lse_idx);
            const int nseg = itp->nseg;
            if (nseg == 1) {
                if (valid_row) {
                    store_row_part<kPartD, BF16>(p.o, o_elem, of, inv_l);
                    if (part == 0) p.lse[lse_idx] = lse_nat;
                }
                continue;
            }
            // normalised partial O (fp32) and LSE of this piece, in the slot
            // of its range; the merge kernel combines the pieces
            const size_t pbase = (size_t)piece_slot(itp->range, itp->seg) * kBlockM + row;
            float* po = p.part_o + pbase * D + part * kPartD;
#pragma unroll
            for (int e = 0; e < kPartD; e += 4)
                *reinterpret_cast<float4*>(po + e) = make_float4(
                    of[e] * inv_l, of[e + 1] * inv_l, of[e + 2] * inv_l, of[e + 3] * inv_l);
            if (part == 0) p.part_lse[pbase] = lse_nat;
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

// ------------------------------------------------------------------ append
// Paged cache: write the new tokens' K and V rows (k_new, v_new [B, Nq, Hkv, d])
// at logical positions seqlens_k[b] - Nq .. seqlens_k[b] - 1, through the
// block table, before the decode reads them.  One warp per (b, t, g) row,
// 16 bytes per lane.
template <int D>
__global__ void __launch_bounds__(256) attn_paged_append_kernel(const __grid_constant__ DecodeParams p) {
    constexpr int kLanes = D / 8;  // 16-byte chunks per row
    const long rows = (long)p.B * p.Nq * p.Hkv;
    const int lane = threadIdx.x & 31;
    for (long r = ((long)blockIdx.x * blockDim.x + threadIdx.x) / 32; r < rows;
         r += (long)gridDim.x * blockDim.x / 32) {
        const int g = (int)(r % p.Hkv);
        const long bt = r / p.Hkv;
        const int t = (int)(bt % p.Nq);
        const int b = (int)(bt / p.Nq);
        const int pos = p.seqlens_k[b] - p.Nq + t;
        if (pos < 0 || lane >= kLanes) continue;
        const int lb = pos >> p.block_shift;
        const int blk = lb < p.max_blocks ? p.block_table[(size_t)b * p.max_blocks + lb] : -1;
        if (blk < 0 || blk >= p.num_blocks) {
            if (lane == 0) atomicCAS(p.err, 0u, kErrDecodeBase + 9);
            continue;
        }
        const size_t row = ((size_t)blk << p.block_shift) + (pos & ((1 << p.block_shift) - 1));
        const size_t dst = (row * p.Hkv + g) * (D / 8) + lane;
        const size_t src = (((size_t)b * p.Nq + t) * p.Hkv + g) * (D / 8) + lane;
        reinterpret_cast<uint4*>(p.k_cache)[dst] = reinterpret_cast<const uint4*>(p.k_new)[src];
        reinterpret_cast<uint4*>(p.v_cache)[dst] = reinterpret_cast<const uint4*>(p.v_new)[src];
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
    if (p.block_table && p.k_new) {
        const long warps = (long)p.B * p.Nq * p.Hkv;
        const int blocks = (int)std::min<long>((warps + 7) / 8, 148L * 8);
        attn_paged_append_kernel<D><<<blocks, 256, 0, stream>>>(p);
        e = cudaGetLastError();
        if (e != cudaSuccess) return e;
    }
    attn_decode_plan_kernel<<<1, kPlanThreads, 0, stream>>>(p, n_ctas);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    kern<<<n_ctas, kThreads, L::kAlloc, stream>>>(qmap, kmap, vmap, p);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    attn_decode_merge_kernel<D, BF16><<<n_ctas, 4 * kBlockM, 0, stream>>>(p);
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
