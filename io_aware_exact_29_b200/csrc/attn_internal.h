// attn_internal.h -- parameter blocks shared by the C-ABI layer and the
// kernel translation units (host and device).
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace attn {

// Device error word codes: kernel id * 16 + wait site.
enum : unsigned {
    kErrFwdBase = 1 * 16,
    kErrDecodeBase = 2 * 16,
    kErrBwdBase = 3 * 16,
};

// Block mask of block-sparse attention, one entry per (128-query tile,
// 128-key tile): the entry of batch b, query head h, query tile qt and key
// tile kt is m[b * sb + h * sh + qt * srow + kt]; 0 masks every key of the
// tile for those queries.  m == nullptr: no block mask.
struct BlockMask {
    const unsigned char* m;
    long long sb, sh;
    int srow;
};

// Launch order of a grid over (b, head) pairs x tiles whose tiles differ in
// cost (causal): a 1-D grid in bands of `band` pairs; inside a band the
// costliest tile rank of every pair comes first, then the next rank.  Block
// u -> (pair, tile rank 0 = costliest).  Bands bound the K/V (or Q/dO) set
// in flight, so that it stays in L2.
__host__ __device__ __forceinline__ void band_unit(unsigned u, int band, int n_pairs, int n_tiles,
                                                   int& pair, int& rank) {
    const unsigned per_band = (unsigned)band * (unsigned)n_tiles;
    const int bi = (int)(u / per_band);
    const int r = (int)(u - (unsigned)bi * per_band);
    const int hb = min(band, n_pairs - bi * band);  // pairs in this band
    rank = r / hb;
    pair = bi * band + (r - rank * hb);
}

// Block-sparse forward: the two 128-row Q tiles of a CTA walk their own
// lists of key tiles in lockstep.  Step si pairs the si-th key tile of Q0
// (x0, when si < n0) with the si-th of Q1 (x1, when si < n1); the K/V stream
// loads x0, then x1 when it is a different tile, so a step holds one or two
// stream positions (pos0, pos1; pos1 == pos0 when the tile is shared).  The
// loader, the MMA issuer and the softmax warps all call this walk, each with
// its own state (c0, c1: next candidate tile of each Q tile; si: step;
// pos: next stream position), so they agree on every step.  use(a, j): key
// tile j takes part for Q tile a; nt0, nt1: one past each Q tile's last
// candidate tile.
struct PairStep {
    int x0, x1;      // key tiles of Q0 and Q1 (when has0 / has1)
    int pos0, pos1;  // their positions in the K/V stream
    bool has0, has1, shared;
};

template <class Use>
__host__ __device__ __forceinline__ PairStep sparse_next_step(const Use& use, int n0, int n1,
                                                              int nt0, int nt1, int& c0, int& c1,
                                                              int& si, int& pos) {
    PairStep st;
    st.has0 = si < n0;
    st.has1 = si < n1;
    st.x0 = st.x1 = st.pos0 = st.pos1 = -1;
    if (st.has0) {
        while (c0 < nt0 - 1 && !use(0, c0)) ++c0;
        st.x0 = c0++;
    }
    if (st.has1) {
        while (c1 < nt1 - 1 && !use(1, c1)) ++c1;
        st.x1 = c1++;
    }
    st.shared = st.has0 && st.has1 && st.x0 == st.x1;
    if (st.has0) st.pos0 = pos++;
    if (st.has1) st.pos1 = st.shared ? st.pos0 : pos++;
    ++si;
    return st;
}

struct FwdParams {
    int B, Hq, Hkv, Nq, Nk;
    int n_ctas;       // persistent forward: CTAs launched, each taking every n_ctas-th unit
    int G;            // Hq / Hkv
    int n_qtiles;     // ceil(Nq / 128)
    int causal;
    float scale_log2; // scale * log2(e)
    const int* seqlens_k;  // [B] or nullptr
    int window_left;       // -1, or keys before i + (Lk - Nq) - window_left are masked
    BlockMask bmask;       // block-sparse mask, or m == nullptr
    int band;              // >0: 1-D grid, bands of `band` (b, h) pairs, costliest tiles first
    void* o;               // [B, Nq, Hq, d] (persistent forward: rows stored from registers)
    float* lse;            // [B, Hq, Nq]
    unsigned long long limit_ns;
    int inject;       // self-test: the loader skips everything
    unsigned* err;    // device error word
};

struct FwdMaps {
    CUtensorMap q, k, v, o;
};

// Launch the forward kernel for head dim d (64/128) and element type: one
// CTA per work unit of 256 query rows, every mask (attn_fwd_sm100a.cu).
cudaError_t launch_fwd(const FwdMaps& maps, const FwdParams& p, int d, bool bf16,
                       cudaStream_t stream);

// The persistent forward (attn_fwd_persist_sm100a.cu): p.n_ctas CTAs, each
// taking every n_ctas-th work unit; for units of equal cost only (no causal,
// window or block mask).
cudaError_t launch_fwd_persist(const FwdMaps& maps, const FwdParams& p, int d, bool bf16,
                               cudaStream_t stream);

struct BwdParams {
    int B, Hq, Hkv, Nq, Nk;
    int G;                 // Hq / Hkv
    int causal;
    float scale;
    float scale_log2;      // scale * log2(e)
    const int* seqlens_k;  // [B] or nullptr
    int window_left;       // -1, or keys before i + (Lk - Nq) - window_left are masked
    BlockMask bmask;       // block-sparse mask, or m == nullptr
    int band_kv;           // >0: dK/dV grid in bands of (b, kv head) pairs, costliest first
    int band_q;            // >0: dQ grid in bands of (b, q head) pairs, costliest first
    const void* o;         // [B, Nq, Hq, d] forward output
    const void* dout;      // [B, Nq, Hq, d]
    const float* lse;      // [B, Hq, Nq] forward log-sum-exp (natural log)
    float* lse2;           // workspace [B, Hq, Nq]: LSE * log2(e), +inf for empty rows
    float* dsum;           // workspace [B, Hq, Nq]: sum_t dO * O
    void* dq;              // [B, Nq, Hq, d]
    void* dk;              // [B, Nk, Hkv, d]
    void* dv;              // [B, Nk, Hkv, d]
    unsigned long long limit_ns;
    unsigned* err;
};

struct BwdMaps {
    CUtensorMap q, k, v, dout;  // [B, N, H, d], box 64 columns x 1 head x 128 rows
};

// D and LSE * log2 e, then the dK/dV and dQ kernels, on `stream`.
cudaError_t launch_bwd(const BwdMaps& maps, const BwdParams& p, int d, bool bf16,
                       cudaStream_t stream);

struct DecodeParams {
    const void* q;         // [B, Nq, Hq, d]
    void* o;               // [B, Nq, Hq, d] (persistent forward: rows stored from registers)
    float* lse;            // [B, Hq, Nq]
    const int* cu_seqlens_k;
    const int* seqlens_k;
    float* part_o;         // [B, Hkv, n_mgroups, max_splits, R, d] fp32 (R = 16, or 128 for tc)
    float* part_lse;       // [B, Hkv, n_mgroups, max_splits, R]
    unsigned* counters;    // [B, Hkv, n_mgroups]
    // tensor-core decode schedule (written by its plan kernel)
    struct DecodePlan* plan;
    long long* seq_prefix;  // [B + 1] weight before sequence b
    int2* range_units;      // [max_ranges] first and last unit of range r
    int max_seqlen_k;
    int max_ranges;
    // paged cache (tensor-core decode): block_table == nullptr for a packed cache
    const int* block_table;  // [B, max_blocks] physical block of each logical block
    int max_blocks;
    int block_shift;         // block_size = 1 << block_shift
    int num_blocks;
    void* k_cache;           // [num_blocks * block_size, Hkv, d], for the append
    void* v_cache;
    const void* k_new;       // [B, Nq, Hkv, d] rows to append, or nullptr
    const void* v_new;
    int B, Hq, Hkv, Nq, G;
    int rows;              // Nq * G query rows per (sequence, kv head)
    int n_mgroups;         // ceil(rows / 16)
    int split_keys;        // multiple of 64
    int max_splits;
    int causal;
    float scale_log2;
    unsigned long long limit_ns;
    unsigned* err;
};

// Tensor-core decode schedule.  The work of unit (b, g) -- sequence b, kv
// head g -- weighs its key tiles plus kDecodeSegCost tiles of per-segment
// overhead; units are laid end to end in (b, g) order and the total weight
// is cut into n_ranges equal ranges, one CTA each (stream-K style), so that
// a unit is split only where a range boundary falls inside it.
constexpr int kDecodeSegCost = 2;        // weight of a segment's set-up, in tiles
constexpr int kDecodeMinRangeWeight = 8; // smallest range weight in automatic mode
constexpr int kDecodeMaxRangesAuto = 192;

struct DecodePlan {
    long long range_weight;  // > 0: ranges of this weight; 0: n_ranges balanced ranges
    long long total_weight;
    int n_ranges;
    int pad;
};

// First weight position of range r, and the range that holds position x.
__host__ __device__ inline long long plan_range_begin(long long rw, long long total, long long n,
                                                      long long r) {
    return rw > 0 ? r * rw : (r * total) / n;
}
__host__ __device__ inline long long plan_range_of(long long rw, long long total, long long n,
                                                   long long x) {
    return rw > 0 ? x / rw : ((x + 1) * n - 1) / total;
}

struct DecodeLayout {
    int tc;  // 1: tensor-core kernel (one 128-row tile per unit), 0: mma.sync kernel
    int split_keys, max_splits, n_mgroups;
    int max_ranges;  // tc: bound on the number of ranges (two partial slots each)
    size_t part_o_off, part_lse_off, counters_off, prefix_off, ranges_off, plan_off, total;
};

// The tensor-core decode takes the shapes whose Nq * G query rows per kv
// head fit one 128-row tile with whole tokens (G divides 128), with ranges
// of whole 128-key tiles.  Even one token (8 of 128 rows) runs faster there
// than on the mma.sync kernel: the loop is bound by HBM, and the idle MMA
// rows cost nothing that the memory pipe waits for.
inline bool decode_use_tc(int G, int Nq, int split_keys) {
    const int rows = Nq * G;
    return G <= 128 && 128 % G == 0 && rows <= 128 && split_keys % 128 == 0;
}

DecodeLayout decode_layout(int B, int Hq, int Hkv, int Nq, int d, int max_seqlen_k,
                           int split_keys);

cudaError_t launch_decode(const CUtensorMap& kmap, const CUtensorMap& vmap,
                          const DecodeParams& p, int d, bool bf16, cudaStream_t stream);

// Tensor-core decode (a plan kernel, then a persistent kernel of n_ctas
// CTAs): qmap is the 5-D map {d, G, Hkv, Nq, B} of Q with box
// {64, G, 1, 128 / G, 1}; kmap/vmap the packed-cache maps with 128-row boxes.
cudaError_t launch_decode_tc(const CUtensorMap& qmap, const CUtensorMap& kmap,
                             const CUtensorMap& vmap, const DecodeParams& p, int d, bool bf16,
                             int n_ctas, cudaStream_t stream);

// Address of the device error word on the current device.
unsigned* device_error_word();

// The argument checks of attn_fwd_varlen_kvcache that need no device and no
// workspace (dtype and d first: ATTN_ERR_UNSUPPORTED; then sizes, scale,
// pointers and alignment: ATTN_ERR_INVALID_ARG); ATTN_OK when they pass.
int decode_check_args(const void* q, const void* k_cache, const void* v_cache,
                      const int* cu_seqlens_k, const int* seqlens_k, int max_seqlen_k,
                      int cache_slots, const void* o, const float* lse, int B, int Hq, int Hkv,
                      int Nq, int d, float scale, int dtype, int split_keys);

}  // namespace attn
