// attn_fwd_common.cuh -- device helpers shared by the two forward kernels
// (attn_fwd_sm100a.cu: one CTA per work unit, every mask; and
// attn_fwd_persist_sm100a.cu: persistent CTAs for short units of equal cost).
#pragma once

#include "attn_internal.h"
#include "ptx.cuh"

namespace attn {
namespace fwd {

constexpr int kBlockM = 128;  // rows per Q tile
constexpr int kBlockN = 128;  // keys per K/V tile
constexpr uint32_t kTmemCols = 512;
// Lazy rescaling: the reference maximum of a row only moves when a tile's
// maximum exceeds it by more than this (log2 units), so P <= 2^8; numerator
// and denominator share the reference, so the result is the same exact softmax.
constexpr float kRescaleThreshold = 8.0f;
// one exponential pair in FWD_POLY_EVERY(D) is evaluated on the FMA pipe (the
// one-CTA-per-unit kernel; the persistent kernel sets its own share)
#ifndef FWD_POLY_EVERY
#define FWD_POLY_EVERY(D) 4
#endif

__device__ __forceinline__ void record_error(unsigned* err, unsigned code, int* abort_flag) {
    atomicCAS(err, 0u, code);
    *reinterpret_cast<volatile int*>(abort_flag) = 1;
}

// Byte offset of 16-byte chunk `chunk` (0..7) of row `row` inside a
// 128-byte-swizzled block of 128-byte rows (the layout TMA writes with
// CU_TENSOR_MAP_SWIZZLE_128B and tcgen05 reads with swizzle mode 128B).
__device__ __forceinline__ uint32_t sw128_offset(uint32_t row, uint32_t chunk) {
    return row * 128u + ((chunk ^ (row & 7u)) << 4);
}

// A bounded wait whose outcome is the same for every lane of the warp, so
// that the warp-collective tcgen05 loads and stores that follow it are
// reached by all lanes or by none.
__device__ __forceinline__ bool warp_wait(uint64_t* bar, uint32_t parity, uint64_t limit_ns,
                                          volatile int* abort_flag) {
    const bool ok = ptx::mbar_wait(bar, parity, limit_ns, abort_flag);
    return __all_sync(0xffffffffu, ok);
}

// Number of key tiles that rows [q_first, q_first + 128) need.
__device__ __forceinline__ int tiles_for(int q_first, int Nq, int Lk, int causal) {
    if (q_first >= Nq) return 0;
    int nt = (Lk + kBlockN - 1) / kBlockN;
    if (causal) {
        const int i_last = min(q_first + kBlockM - 1, Nq - 1);
        const int lim = i_last + Lk - Nq;  // last key visible to the last row
        nt = lim < 0 ? 0 : min(nt, lim / kBlockN + 1);
    }
    return nt;
}

// Running maxima of 64 score columns (two 32-column TMEM loads) into eight
// independent chains of three-input maxima.  kMask: the tile reaches past
// the row's visible keys [row_first, row_lim] (others are masked).
template <bool kMask, bool kLow>
__device__ __forceinline__ void half_max(const uint32_t (&r)[2][32], int key_base, int row_first,
                                         int row_lim, float (&mx8)[8]) {
#pragma unroll
    for (int c = 0; c < 64; c += 16) {
#pragma unroll
        for (int u = 0; u < 8; ++u) {
            const int c0 = c + u, c1 = c + 8 + u;
            float v0 = __uint_as_float(r[c0 >> 5][c0 & 31]);
            float v1 = __uint_as_float(r[c1 >> 5][c1 & 31]);
            if (kMask) {
                if (key_base + c0 > row_lim || (kLow && key_base + c0 < row_first)) v0 = -INFINITY;
                if (key_base + c1 > row_lim || (kLow && key_base + c1 < row_first)) v1 = -INFINITY;
            }
            mx8[u] = ptx::max3(mx8[u], v0, v1);
        }
    }
}

// p = 2^(s * scale_log2 - m) for 64 score columns, accumulated into four
// pair sums and packed two per 32-bit word (bf16 or fp16).  One pair in
// kPolyEvery goes to the FMA pipe.
template <bool kMask, bool kLow, bool BF16, int kPolyEvery>
__device__ __forceinline__ void half_exp(const uint32_t (&r)[2][32], int key_base,
                                         int row_first, int row_lim,
                                         uint64_t sl2_2, uint64_t nm_2, uint64_t (&acc2)[4],
                                         uint32_t (&pk)[32]) {
#pragma unroll
    for (int c = 0; c < 64; c += 2) {
        float v0 = __uint_as_float(r[c >> 5][c & 31]);
        float v1 = __uint_as_float(r[c >> 5][(c & 31) + 1]);
        if (kMask) {
            if (key_base + c > row_lim || (kLow && key_base + c < row_first)) v0 = -INFINITY;
            if (key_base + c + 1 > row_lim || (kLow && key_base + c + 1 < row_first))
                v1 = -INFINITY;
        }
        const uint64_t t2 = ptx::f2_fma(ptx::f2_pack(v0, v1), sl2_2, nm_2);
        float p0, p1;
        if (((c >> 1) % kPolyEvery) == kPolyEvery - 1) {
            // a share of the pairs on the FMA pipe, taking load off the exp2
            // unit (each kernel sets its share: it trades exp2-unit cycles
            // for FMA-pipe and issue cycles of the same warps)
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

// Masked tiles, 32 columns at a time: for a chunk of keys
// [key_base, key_base + 32) the warp takes one of three paths, the same for
// all its lanes -- every key visible for every row (kVisible: the unmasked
// arithmetic), every key masked for every row (kHidden: nothing to compute,
// P = 0), or a mix (kMixed: the per-element mask).  On a causal diagonal tile
// most warps have chunks of the first two kinds.  The results are those of
// the per-element mask, bit for bit: a visible key's value is untouched by
// it, and a hidden key's exponential is exactly 0.
enum ChunkMode : int { kVisible = 0, kMixed = 1, kHidden = 2 };

template <bool kLow>
__device__ __forceinline__ int chunk_mode(int key_base, int row_first, int row_lim) {
    const bool vis = key_base + 31 <= row_lim && (!kLow || key_base >= row_first);
    const bool hid = key_base > row_lim || (kLow && key_base + 31 < row_first);
    if (__all_sync(0xffffffffu, vis)) return kVisible;
    if (__all_sync(0xffffffffu, hid)) return kHidden;
    return kMixed;
}

// half_max over a masked tile's 64 columns, chunk by chunk.
template <bool kLow>
__device__ __forceinline__ void half_max_chunks(const uint32_t (&r)[2][32], int key_base,
                                                int row_first, int row_lim, float (&mx8)[8]) {
#pragma unroll
    for (int ch = 0; ch < 2; ++ch) {
        const int mode = chunk_mode<kLow>(key_base + 32 * ch, row_first, row_lim);
        if (mode == kHidden) continue;
        const bool mask = mode == kMixed;
#pragma unroll
        for (int c = 32 * ch; c < 32 * ch + 32; c += 16) {
#pragma unroll
            for (int u = 0; u < 8; ++u) {
                const int c0 = c + u, c1 = c + 8 + u;
                float v0 = __uint_as_float(r[c0 >> 5][c0 & 31]);
                float v1 = __uint_as_float(r[c1 >> 5][c1 & 31]);
                if (mask) {
                    if (key_base + c0 > row_lim || (kLow && key_base + c0 < row_first))
                        v0 = -INFINITY;
                    if (key_base + c1 > row_lim || (kLow && key_base + c1 < row_first))
                        v1 = -INFINITY;
                }
                mx8[u] = ptx::max3(mx8[u], v0, v1);
            }
        }
    }
}

// half_exp over a masked tile's 64 columns, chunk by chunk (hidden chunks
// give P = 0 and add nothing to the row sum).
template <bool kLow, bool BF16, int kPolyEvery>
__device__ __forceinline__ void half_exp_chunks(const uint32_t (&r)[2][32], int key_base,
                                                int row_first, int row_lim, uint64_t sl2_2,
                                                uint64_t nm_2, uint64_t (&acc2)[4],
                                                uint32_t (&pk)[32]) {
#pragma unroll
    for (int ch = 0; ch < 2; ++ch) {
        const int mode = chunk_mode<kLow>(key_base + 32 * ch, row_first, row_lim);
        if (mode == kHidden) {
#pragma unroll
            for (int c = 32 * ch; c < 32 * ch + 32; c += 2) pk[c >> 1] = 0u;
            continue;
        }
        const bool mask = mode == kMixed;
#pragma unroll
        for (int c = 32 * ch; c < 32 * ch + 32; c += 2) {
            float v0 = __uint_as_float(r[c >> 5][c & 31]);
            float v1 = __uint_as_float(r[c >> 5][(c & 31) + 1]);
            if (mask) {
                if (key_base + c > row_lim || (kLow && key_base + c < row_first)) v0 = -INFINITY;
                if (key_base + c + 1 > row_lim || (kLow && key_base + c + 1 < row_first))
                    v1 = -INFINITY;
            }
            const uint64_t t2 = ptx::f2_fma(ptx::f2_pack(v0, v1), sl2_2, nm_2);
            float p0, p1;
            if (((c >> 1) % kPolyEvery) == kPolyEvery - 1) {
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
}

}  // namespace fwd
}  // namespace attn
