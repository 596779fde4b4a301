/*
 * attn.h -- C ABI of libattn.so: exact scaled dot-product attention on B200
 * (sm_100a), computed tile by tile with an online softmax so that the N x N
 * score matrix never reaches device memory.
 *
 *   O = softmax(scale * Q K^T + mask) V          LSE = log(sum_j exp(...))
 *
 * The operation is the one stated on the ai6s.net article about the CANN
 * ops-transformer FlashAttention operator: section "标准注意力的致命伤不在算力，
 * 在搬运" gives the four steps (Q·Kᵀ, scale, softmax, ·V); section
 * "FlashAttention 拆的不是算法，是数据流" the tiling and the running max / sum
 * that keep it exact; section "ops-transformer 里的 FlashAttention 做了什么额外
 * 的事" the fused causal mask (point 2) and the variable-length KV cache whose
 * tiles stop at each sequence's real length (point 3).  The effectstory.com
 * article "FlashAttention：IO 感知的精確注意力演算法如何加速 Transformer 訓練
 * 與推論" (section "什麼是 FlashAttention？核心概念與 IO 感知機制") states the
 * single-pass schedule: Q, K and V are read once and O is written once.
 *
 * Conventions shared by every entry point
 *  - Pointers are DEVICE memory owned by the caller.  The library never
 *    allocates, never synchronises and keeps no pointer after returning.
 *    Work is queued on `stream` (a cudaStream_t; NULL = legacy default).
 *  - Layouts are row-major with the head dimension d contiguous:
 *      q, o     [B, Nq, Hq, d]         k, v [B, Nk, Hkv, d]
 *      lse      [B, Hq, Nq] float32, natural logarithm
 *    Query head h reads key/value head h / (Hq / Hkv) (grouped-query heads).
 *  - Element type: bf16 or fp16 (`dtype`), fp32 accumulation.
 *  - Masks are additive 0 / -inf.  Causal is bottom-right aligned: query i
 *    sees key j iff j <= i + (Lk - Nq), where Lk is the number of real keys;
 *    for Nq == Lk this is the usual lower-triangular mask.  A query row with
 *    no visible key gets O = 0 and LSE = -inf.
 *  - Requirements: d in {64, 128}; B, Hq, Hkv, Nq > 0; Nk >= 0;
 *    Hq % Hkv == 0; every pointer 16-byte aligned; a device of compute
 *    capability 10.0 (B200).  Violations return an error code before any
 *    work is queued.  Faults during execution surface at the caller's next
 *    synchronisation.  Every wait inside a kernel is bounded; a wait that
 *    runs out records an error word, read with attn_get_device_error().
 *  - Thread safety: calls are independent (tensor maps are built per call
 *    and passed by value to the kernel).
 *  - One exception to both of the last two points:
 *    attn_fwd_varlen_kvcache_noalloc uses a scratch array that the library
 *    itself holds in device memory (one per device, shared by every call), so
 *    calls of it that overlap on the GPU must be serialised by the caller.
 */
#ifndef ATTN_B200_H
#define ATTN_B200_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define ATTN_API __attribute__((visibility("default")))
#else
#define ATTN_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum { ATTN_BF16 = 0, ATTN_FP16 = 1 } attn_dtype;

enum {
    ATTN_OK = 0,
    ATTN_ERR_INVALID_ARG = -1, /* bad size, pointer, alignment or length */
    ATTN_ERR_UNSUPPORTED = -2, /* not a B200 / sm_100 device, unknown dtype or d */
    ATTN_ERR_CUDA = -3,        /* a CUDA call or the kernel launch failed */
    ATTN_ERR_WORKSPACE = -4,   /* decode workspace missing or too small */
    ATTN_ERR_TIMEOUT = -5      /* a bounded in-kernel wait ran out (device error word) */
};

/*
 * Forward attention (prefill / training forward), dense keys.
 *   q [B, Nq, Hq, d], k/v [B, Nk, Hkv, d], o [B, Nq, Hq, d] (same dtype),
 *   lse [B, Hq, Nq] float32.  scale is usually 1/sqrt(d).  causal: 0 or 1.
 * The tcgen05 kernel stages Q, K and V tiles of 128 rows in shared memory by
 * TMA, keeps S and the O accumulator in tensor memory and writes only O and
 * LSE (ai6s.net article, section "FlashAttention 拆的不是算法，是数据流").
 */
ATTN_API int attn_fwd(const void* q, const void* k, const void* v, void* o, float* lse, int B, int Hq,
             int Hkv, int Nq, int Nk, int d, float scale, int causal, int dtype, void* stream);

/*
 * Forward attention with per-sequence key lengths: as attn_fwd, plus
 * seqlens_k (device, int32 [B], each in [0, Nk]).  Keys j >= seqlens_k[b]
 * are masked (the variable-length KV point 3 of the ai6s.net article); the
 * K/V rows behind the length may hold anything, NaN included.  Every query
 * row is computed.  NULL seqlens_k behaves as attn_fwd.
 */
ATTN_API int attn_fwd_kpad(const void* q, const void* k, const void* v, void* o, float* lse, int B,
                  int Hq, int Hkv, int Nq, int Nk, int d, float scale, int causal, int dtype,
                  const int* seqlens_k, void* stream);

/*
 * Forward attention with a sliding window: as attn_fwd_kpad (seqlens_k may be
 * NULL), plus window_left: -1 for none, else query i also masks every key
 * j < i + (Lk - Nq) - window_left, i.e. it sees at most window_left keys
 * before its own position (with causal: the window_left + 1 most recent
 * keys).  The pages list mask extensions as a direction without a form
 * (machinelearning.ru page, "directions"); key tiles wholly outside the
 * window are skipped like those above the causal diagonal.
 */
ATTN_API int attn_fwd_window(const void* q, const void* k, const void* v, void* o, float* lse,
                             int B, int Hq, int Hkv, int Nq, int Nk, int d, float scale,
                             int causal, int window_left, int dtype, const int* seqlens_k,
                             void* stream);

/* Rows and keys per entry of a block mask (the kernels' tile sizes). */
#define ATTN_MASK_BLOCK 128

/*
 * Block-sparse forward attention: as attn_fwd_window (window_left -1 = none,
 * seqlens_k may be NULL), plus a block mask that removes whole 128 x 128
 * blocks of (query, key) pairs.  The pages name mask extensions as a
 * direction without a form (machinelearning.ru page, "directions"); this is
 * the block-granular one, which the tile loop can skip without touching the
 * skipped keys.
 *   block_mask: device bytes, owned by the caller; the entry for batch b,
 *     query head h, query block qb = i / ATTN_MASK_BLOCK and key block
 *     kb = j / ATTN_MASK_BLOCK is block_mask[b * mask_stride_b +
 *     h * mask_stride_h + qb * mask_stride_row + kb].  Nonzero: the block
 *     takes part (subject to the causal, length and window rules); 0: every
 *     key of the block is masked for those queries and its K/V rows are not
 *     read for them.  Strides count bytes; 0 shares one mask across batches
 *     or heads.  mask_stride_row >= ceil(Nk / 128); ceil(Nq / 128) rows.
 * A row whose visible keys are all masked gives O = 0, LSE = -inf.
 * Returns the status codes of attn_fwd (ATTN_ERR_INVALID_ARG for a NULL
 * mask, a negative stride or a row stride below the key-block count).
 */
ATTN_API int attn_fwd_blocksparse(const void* q, const void* k, const void* v, void* o,
                                  float* lse, int B, int Hq, int Hkv, int Nq, int Nk, int d,
                                  float scale, int causal, int window_left, int dtype,
                                  const int* seqlens_k, const unsigned char* block_mask,
                                  long long mask_stride_b, long long mask_stride_h,
                                  int mask_stride_row, void* stream);

/*
 * Bytes of device workspace that attn_fwd_varlen_kvcache needs for these
 * sizes.  split_keys: keys per split-K work unit, a multiple of 64, or 0 to
 * let the library choose (the same rule the decode call applies).  Returns 0
 * for invalid sizes.
 */
ATTN_API size_t attn_decode_workspace_bytes(int B, int Hq, int Hkv, int Nq, int d, int max_seqlen_k,
                                   int split_keys);

/*
 * Attention of Nq new query tokens per sequence (1 <= Nq <= 16) against a
 * packed, variable-length KV cache (decode).
 *   q            [B, Nq, Hq, d]
 *   k_cache, v_cache [slots, Hkv, d]; sequence b owns slots
 *                cu_seqlens_k[b] .. cu_seqlens_k[b+1]-1 (device int32 [B+1],
 *                non-decreasing, cu_seqlens_k[0] >= 0)
 *   seqlens_k    device int32 [B]: filled length of each sequence,
 *                0 <= seqlens_k[b] <= cu_seqlens_k[b+1] - cu_seqlens_k[b]
 *                (the cache is pre-allocated and grows by one row per
 *                token; only the filled rows are read: ai6s.net article,
 *                adaptation point 3).  Unfilled slots may hold anything.
 *   max_seqlen_k host int, >= every seqlens_k[b] (sizes the grid)
 *   cache_slots  host int, rows of k_cache / v_cache; no copy reads past it
 *   o [B, Nq, Hq, d], lse [B, Hq, Nq] float32
 *   causal       bottom-right within the chunk: token i sees keys
 *                j <= i + seqlens_k[b] - Nq
 *   workspace    device buffer of at least attn_decode_workspace_bytes(...)
 *                bytes (256-byte aligned), owned by the caller; holds the
 *                work schedule, split-K partial results and counters.  Calls
 *                that share one workspace must not overlap on the GPU.
 *   split_keys   0 for automatic, else a multiple of 64: keys per split (or,
 *                on the tensor-core path, per schedule range).
 * The Nq tokens x Hq/Hkv query heads that share a kv head are scored together
 * in one pass over its filled cache rows, with a running max and sum.  When
 * Hq/Hkv divides 128, Nq * Hq/Hkv <= 128 and split_keys is 0 or a multiple of
 * 128, the rows form one tcgen05 tile and the work of all sequences is cut
 * into equal ranges, one per SM (a plan kernel, the decode kernel and a merge
 * kernel); otherwise one CTA per (sequence, kv head, split, 16 rows) on
 * mma.sync.  Pieces of a split sequence are merged in key order:
 * LSE = log sum_i exp(LSE_i), O = sum_i exp(LSE_i - LSE) O_i.
 */
ATTN_API int attn_fwd_varlen_kvcache(const void* q, const void* k_cache, const void* v_cache,
                            const int* cu_seqlens_k, const int* seqlens_k, int max_seqlen_k,
                            int cache_slots, void* o, float* lse, int B, int Hq, int Hkv, int Nq, int d,
                            float scale, int causal, int dtype, void* workspace,
                            size_t workspace_bytes, int split_keys, void* stream);

/*
 * The decode of attn_fwd_varlen_kvcache against a PAGED KV cache: the cache
 * is cut into blocks of block_size rows and sequence b's logical key j lives
 * in physical block block_table[b * max_blocks + j / block_size], row
 * j % block_size (the pre-allocated, one-row-per-token cache of the ai6s.net
 * article, adaptation point 3, with its rows found through a table).
 *   k_cache, v_cache  [num_blocks, block_size, Hkv, d] (dtype)
 *   block_table       device int32 [B, max_blocks]; entries past a sequence's
 *                     last filled block are never read
 *   block_size        a power of two, 16 .. 1024
 *   seqlens_k         device int32 [B]: lengths INCLUDING the Nq new tokens
 *   k_new, v_new      NULL, or device [B, Nq, Hkv, d]: the new tokens' K and V,
 *                     written into the cache at logical positions
 *                     seqlens_k[b] - Nq .. seqlens_k[b] - 1 before the
 *                     attention reads them (so the cache is modified)
 *   everything else as attn_fwd_varlen_kvcache, workspace of
 *   attn_decode_workspace_bytes(B, Hq, Hkv, Nq, d, max_seqlen_k, split_keys).
 * Only the tensor-core decode reads a paged cache: Hq/Hkv must divide 128,
 * Nq * Hq/Hkv <= 128 and split_keys must be 0 or a multiple of 128, else
 * ATTN_ERR_UNSUPPORTED.  A table entry outside [0, num_blocks) for a filled
 * block is reported in the device error word (the rows read are block 0's).
 */
ATTN_API int attn_fwd_paged_kvcache(const void* q, void* k_cache, void* v_cache,
                                    const int* block_table, int max_blocks, int block_size,
                                    int num_blocks, const int* seqlens_k, int max_seqlen_k,
                                    const void* k_new, const void* v_new, void* o, float* lse,
                                    int B, int Hq, int Hkv, int Nq, int d, float scale,
                                    int causal, int dtype, void* workspace,
                                    size_t workspace_bytes, int split_keys, void* stream);

/*
 * Bytes of device workspace that attn_bwd needs for these sizes: two float32
 * arrays of B * Hq * Nq (per query row, the dot product of dO and O, and the
 * forward's LSE in base 2), each 256-byte aligned.  Returns 0 for invalid
 * sizes.
 */
ATTN_API size_t attn_bwd_workspace_bytes(int B, int Hq, int Nq);

/*
 * Gradients of attention (the training backward pass) for
 * L = sum(dout * O), O = attn_fwd[_kpad](q, k, v) with the same scale, causal
 * flag and key lengths.  The pages report the method's training speed-ups
 * (effectstory.com article, "訓練性能量化提升" table) without its backward
 * algorithm; this recomputes every score tile on chip from q, k and the
 * forward's lse, as the forward does, and never writes an N x N matrix.
 *   q, o, dout, dq  [B, Nq, Hq, d]      k, v, dk, dv  [B, Nk, Hkv, d]
 *   (all in dtype; o and lse are the forward's outputs, lse [B, Hq, Nq]
 *   float32, -inf for a row with no visible key)
 *   dk, dv are summed over the Hq/Hkv query heads that share a kv head; rows
 *   of keys at or beyond seqlens_k[b] (NULL = Nk) are written as zero and
 *   the K/V rows there may hold anything, NaN included.
 *   workspace: at least attn_bwd_workspace_bytes(B, Hq, Nq) bytes, 256-byte
 *   aligned, owned by the caller; calls sharing it must not overlap.
 * Kernels, in order on `stream`: the per-row dot products, one CTA per
 * 128-key tile of a kv head accumulating dK and dV in tensor memory over all
 * query tiles of its group, one CTA per 128-row query tile accumulating dQ.
 * No atomics: the result does not depend on scheduling.
 * Returns the status codes of attn_fwd, or ATTN_ERR_WORKSPACE.
 */
ATTN_API int attn_bwd(const void* q, const void* k, const void* v, const void* o,
                      const float* lse, const void* dout, void* dq, void* dk, void* dv, int B,
                      int Hq, int Hkv, int Nq, int Nk, int d, float scale, int causal, int dtype,
                      const int* seqlens_k, void* workspace, size_t workspace_bytes,
                      void* stream);

/*
 * attn_bwd for the sliding-window forward (attn_fwd_window): the same
 * arguments plus window_left (-1 = none), which must match the forward's.
 */
ATTN_API int attn_bwd_window(const void* q, const void* k, const void* v, const void* o,
                             const float* lse, const void* dout, void* dq, void* dk, void* dv,
                             int B, int Hq, int Hkv, int Nq, int Nk, int d, float scale,
                             int causal, int window_left, int dtype, const int* seqlens_k,
                             void* workspace, size_t workspace_bytes, void* stream);

/*
 * attn_bwd for the block-sparse forward (attn_fwd_blocksparse): the same
 * arguments as attn_bwd_window plus the forward's block mask and strides
 * (NULL block_mask = attn_bwd_window).  Masked blocks are skipped in both
 * gradient kernels: a key tile's dK/dV visits only the (head, query tile)
 * pairs whose entry is set, a query tile's dQ only its set key tiles.
 */
ATTN_API int attn_bwd_blocksparse(const void* q, const void* k, const void* v, const void* o,
                                  const float* lse, const void* dout, void* dq, void* dk,
                                  void* dv, int B, int Hq, int Hkv, int Nq, int Nk, int d,
                                  float scale, int causal, int window_left, int dtype,
                                  const int* seqlens_k, const unsigned char* block_mask,
                                  long long mask_stride_b, long long mask_stride_h,
                                  int mask_stride_row, void* workspace, size_t workspace_bytes,
                                  void* stream);

/* Size in bytes of the scratch area built into the library for
 * attn_fwd_varlen_kvcache_noalloc (32 MiB). */
#define ATTN_NOALLOC_SCRATCH_BYTES (32u << 20)

/*
 * attn_fwd_varlen_kvcache for callers that cannot allocate device memory.
 * (An addition of this library: the pages have no counterpart.)
 *
 * The decode needs a workspace for its split-K partial results.  Some callers
 * cannot provide one: code embedded in a host program that plans and owns all
 * device memory without giving it an allocator, or a decode loop that must
 * not call cudaMalloc because that call can synchronise the whole device.
 * This entry point takes the same arguments as attn_fwd_varlen_kvcache minus
 * the workspace and uses a scratch area of ATTN_NOALLOC_SCRATCH_BYTES that the
 * library keeps in a static device array; it calls no cudaMalloc, cudaFree or
 * other allocating routine.  The caller still passes every input and output.
 *  - Limit: if the sizes need more scratch than ATTN_NOALLOC_SCRATCH_BYTES
 *    (see attn_decode_workspace_bytes; a larger split_keys needs less), the
 *    call returns ATTN_ERR_WORKSPACE before queuing any work.
 *  - Set-up: the first call on a device looks up the array's device address
 *    (cudaGetSymbolAddress, with that device current) and caches it; make
 *    that first call before any stream capture on the device.  The address
 *    is looked up again when the current context is not the one it was taken
 *    in (a device reset destroys the context and may move the array); make
 *    the first call after a reset before any stream capture too.
 *  - Sharing: every GPU that loads the library holds the array until the
 *    process exits, and all calls on a device share it.  It keeps whatever the
 *    last call left; each call clears the parts that must start at zero (the
 *    split counters) on `stream` before its kernel.  Calls that overlap on the
 *    GPU (other streams, other host threads) race on it: serialise them.
 * Returns the same status codes as attn_fwd_varlen_kvcache for the same
 * arguments (its argument checks run first, in the same order), plus
 * ATTN_ERR_WORKSPACE for sizes beyond the scratch.
 */
ATTN_API int attn_fwd_varlen_kvcache_noalloc(const void* q, const void* k_cache,
                                             const void* v_cache, const int* cu_seqlens_k,
                                             const int* seqlens_k, int max_seqlen_k,
                                             int cache_slots, void* o, float* lse, int B, int Hq,
                                             int Hkv, int Nq, int d, float scale, int causal,
                                             int dtype, int split_keys, void* stream);

/* Human-readable text of a status code (static storage). */
ATTN_API const char* attn_status_string(int status);

/*
 * Read and clear the device error word of the current device after
 * synchronising `stream`.  *code receives 0 when every bounded wait since the
 * last call completed, otherwise a non-zero code naming the wait that ran out
 * (kernel id * 16 + wait site).  Returns ATTN_OK, or ATTN_ERR_CUDA.
 */
ATTN_API int attn_get_device_error(int* code, void* stream);

/*
 * Self-test of the bounded waits: launches the forward kernel on a tiny
 * problem with its loader told to skip the first arrival, with wait limit
 * `limit_ms`.  No copy is issued, so nothing is in flight when the waits give
 * up; the kernel frees its tensor memory and returns.  The status of the
 * launch is returned; the timeout shows up in attn_get_device_error().
 * q/k/v/o/lse as for attn_fwd with B = Hq = Hkv = 1, Nq = Nk = 128, d = 64.
 */
ATTN_API int attn_selftest_watchdog(const void* q, const void* k, const void* v, void* o, float* lse,
                           int limit_ms, void* stream);

/*
 * Schedule introspection (host only, no device work): the mappings the
 * kernels use, evaluated by the same code on the host so that a model of the
 * schedule can be checked against them.
 *
 * attn_schedule_band_unit: the launch order of causal grids.  Causal row
 * tiles differ in cost (ai6s.net article, section "ops-transformer 里的
 * FlashAttention 做了什么额外的事", point 2: the causal mask is fused into
 * the blockwise computation and tiles above the diagonal are skipped), so
 * the 1-D grid runs in bands of `band` (batch, head) pairs and, inside a
 * band, the costliest tile rank of every pair first.  Block u of a grid of
 * n_pairs x n_tiles blocks runs *pair, tile rank *rank (0 = costliest).
 * Requires 0 < band <= n_pairs, n_tiles > 0, u < n_pairs * n_tiles;
 * returns ATTN_OK or ATTN_ERR_INVALID_ARG.
 *
 * attn_schedule_sparse_steps: the lockstep walk of a block-sparse forward
 * CTA's two 128-row query tiles over their key tiles.  m0, m1: host arrays of
 * one byte per key tile (nonzero = the tile takes part); Q tile a considers
 * key tiles [j0a, nta).  Writes 7 ints per step to steps[7 * i ...]:
 * x0, x1 (key tiles, -1 when absent), pos0, pos1 (their K/V stream
 * positions), has0, has1, shared (the step's two tiles are one load).
 * Returns the number of steps (max of the two tile counts), or
 * ATTN_ERR_INVALID_ARG when it exceeds max_steps or an argument is invalid.
 */
ATTN_API int attn_schedule_band_unit(unsigned u, int band, int n_pairs, int n_tiles, int* pair,
                                     int* rank);
ATTN_API int attn_schedule_sparse_steps(const unsigned char* m0, const unsigned char* m1, int nt0,
                                        int nt1, int j00, int j01, int max_steps, int* steps);

/* Library version string. */
ATTN_API const char* attn_version(void);

/*
 * Measurement helper, not part of the attention path: reads `bytes` of device
 * memory at `src` once (16-byte loads that do not allocate in L1) on
 * `stream` and writes one XOR-folded word per CTA to out[0 .. n_ctas-1].
 * Timing it gives the read-only device-memory bandwidth, the roofline
 * denominator of the decode, which reads its KV cache once and writes next to
 * nothing (ai6s.net article, section "标准注意力的致命伤不在算力，在搬运":
 * attention is bound by data movement).  src and bytes multiples of 16;
 * out holds n_ctas words (1 <= n_ctas <= 2^20).  Returns ATTN_OK,
 * ATTN_ERR_INVALID_ARG or ATTN_ERR_CUDA (launch failure).
 */
ATTN_API int attn_hbm_read_probe(const void* src, size_t bytes, unsigned* out, int n_ctas,
                                 void* stream);

#ifdef __cplusplus
}
#endif

#endif /* ATTN_B200_H */
