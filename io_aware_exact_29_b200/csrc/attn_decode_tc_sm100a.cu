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
// Work unit = one CTA: (sequence b, kv head g, key split s).  Query row
// r = t * G + hh is token t, query head g * G + hh; a 5-D TMA box gathers the
// 128 rows (tokens past Nq are zero-filled) and the same box stores O.
// Warp roles (576 threads):
//   warps 0-15  softmax: rows 32*(w%4) .. +31, score columns 32*(w/4) .. +31
//   warp 16     TMA loader: Q once, then 128-key K / V tiles of the packed
//               cache (the copy is clipped at the cache end)
//   warp 17     tensor-memory owner and tcgen05.mma issuer (elected lane)
// Tensor memory: S[0] [0,128), S[1] [128,256) double-buffered scores,
// O [256, 256+D), Q [384, 384+D/2).  The softmax copies Q into tensor memory
// once, so S = Q·Kᵀ reads only K from shared memory; P (bf16/fp16) overwrites
// the first 64 columns of its S buffer and is the A operand of P·V.
//
// With one split the CTA stores O and LSE; otherwise it writes its
// normalised partial O (fp32) and LSE to the workspace and the last CTA of
// the (sequence, kv head) -- found with an atomic counter, no spinning --
// merges all splits in split order: LSE = log sum_s exp(LSE_s),
// O = sum_s exp(LSE_s - LSE) O_s.
#include "attn_internal.h"
#include "ptx.cuh"

namespace attn {
namespace {

constexpr int kBlockM = 128;  // query rows per CTA
constexpr int kBlockN = 128;  // keys per K/V tile
constexpr int kSoftmaxWarps = 16;
constexpr int kThreads = 32 * (kSoftmaxWarps + 2);
constexpr uint32_t kTmemCols = 512;
constexpr float kRescaleThreshold = 8.0f;
constexpr float kLn2 = 0.69314718055994531f;

template <int D, int KST, int VST>
struct TcSmem {
    static constexpr uint32_t kTileBytes = kBlockM * D * 2;
    static constexpr uint32_t kQ = 0;
    static constexpr uint32_t kK = kQ + kTileBytes;
    static constexpr uint32_t kV = kK + KST * kTileBytes;
    static constexpr uint32_t kRedMax = kV + VST * kTileBytes;  // [2 slots][4 parts][128] fp32
    static constexpr uint32_t kRedSum = kRedMax + 2 * 4 * 128 * 4;  // [4 parts][128] fp32
    static constexpr uint32_t kRowLse = kRedSum + 4 * 128 * 4;      // [128] fp32
    static constexpr uint32_t kBars = kRowLse + 128 * 4;
    static constexpr uint32_t kTotal = kBars + 512;
    static constexpr uint32_t kAlloc = kTotal + 1024;
};

template <int KST, int VST>
struct TcBars {
    uint64_t q_full;
    uint64_t k_full[KST];
    uint64_t k_empty[KST];
    uint64_t v_full[VST];
    uint64_t v_empty[VST];
    uint64_t s_full[2];
    uint64_t p_full[2];
    uint64_t o_done;   // one phase per P.V tile
    uint64_t o_final;  // single phase: every P.V of the split is complete
    uint64_t q_tmem;
    uint64_t drain;
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

template <int D, bool BF16, int KST, int VST>
__global__ void __launch_bounds__(kThreads, 1)
    attn_decode_tc_kernel(const __grid_constant__ CUtensorMap tm_q,
                          const __grid_constant__ CUtensorMap tm_k,
                          const __grid_constant__ CUtensorMap tm_v,
                          const __grid_constant__ CUtensorMap tm_o,
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

    const int split = blockIdx.x;
    const int g = blockIdx.y;
    const int b = blockIdx.z;
    const int Lk = p.seqlens_k[b];
    const int slot0 = p.cu_seqlens_k[b];
    const int nsplit = Lk > 0 ? (Lk + p.split_keys - 1) / p.split_keys : 1;
    if (split >= nsplit) return;  // whole CTA leaves before touching anything

    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw_addr = ptx::smem_u32(smem_raw);
    uint8_t* smem = smem_raw + (((raw_addr + 1023u) & ~1023u) - raw_addr);
    const uint32_t sbase = ptx::smem_u32(smem);
    TcBars<KST, VST>* bars = reinterpret_cast<TcBars<KST, VST>*>(smem + L::kBars);
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
    const int nt = (key_end - key_begin + kBlockN - 1) / kBlockN;  // >= 0

    if (tid == 0) {
        ptx::mbar_init(&bars->q_full, 1);
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
            ptx::mbar_init(&bars->p_full[s], kSoftmaxWarps);  // one arrival per warp
        }
        ptx::mbar_init(&bars->o_done, 1);
        ptx::mbar_init(&bars->o_final, 1);
        ptx::mbar_init(&bars->q_tmem, kSoftmaxWarps);
        ptx::mbar_init(&bars->drain, 1);
        bars->abort = 0;
        bars->is_last = 0;
        ptx::fence_barrier_init();
    }
    if (warp == kLoaderWarp && lane == 0) {
        ptx::prefetch_tmap(&tm_q);
        ptx::prefetch_tmap(&tm_k);
        ptx::prefetch_tmap(&tm_v);
        ptx::prefetch_tmap(&tm_o);
    }
    if (warp == kMmaWarp) {
        ptx::tmem_alloc<kTmemCols>(&bars->tmem_base);
        ptx::tmem_relinquish();
    }
    ptx::tc_fence_before();
    __syncthreads();
    ptx::tc_fence_after();
    const uint32_t tmem = bars->tmem_base;

    if (warp == kLoaderWarp) {
        // ================================================= TMA loader
        if (nt > 0) {
            int issued_k = 0, issued_v = 0;
            if (lane == 0) {
                ptx::mbar_arrive_expect_tx(&bars->q_full, kTileBytes);
                for (int c = 0; c < kDBlocks; ++c)
                    ptx::tma_load_5d(smem + L::kQ + c * kBlockBytes, &tm_q, &bars->q_full, c * 64,
                                     0, g, 0, b);
            }
            __syncwarp();
            for (int j = 0; j < nt; ++j) {
                const int row0 = slot0 + key_begin + j * kBlockN;
                const int sk = j % KST;
                if (!warp_wait(&bars->k_empty[sk], ((j / KST) & 1) ^ 1, p.limit_ns, abort_flag)) {
                    record_error(p.err, kErrDecodeBase + 4, &bars->abort);
                    break;
                }
                if (lane == 0) {
                    ptx::mbar_arrive_expect_tx(&bars->k_full[sk], kTileBytes);
                    for (int c = 0; c < kDBlocks; ++c)
                        ptx::tma_load_3d(smem + L::kK + sk * kTileBytes + c * kBlockBytes, &tm_k,
                                         &bars->k_full[sk], c * 64, g, row0);
                }
                __syncwarp();
                ++issued_k;
                const int sv = j % VST;
                if (!warp_wait(&bars->v_empty[sv], ((j / VST) & 1) ^ 1, p.limit_ns, abort_flag)) {
                    record_error(p.err, kErrDecodeBase + 5, &bars->abort);
                    break;
                }
                if (lane == 0) {
                    ptx::mbar_arrive_expect_tx(&bars->v_full[sv], kTileBytes);
                    for (int c = 0; c < kDBlocks; ++c)
                        ptx::tma_load_3d(smem + L::kV + sv * kTileBytes + c * kBlockBytes, &tm_v,
                                         &bars->v_full[sv], c * 64, g, row0);
                }
                __syncwarp();
                ++issued_v;
            }
            int zero = 0;
            volatile int* no_abort = &zero;
            ptx::mbar_wait(&bars->q_full, 0, p.limit_ns, no_abort);
            for (int j = max(0, issued_k - KST); j < issued_k; ++j)
                ptx::mbar_wait(&bars->k_full[j % KST], (j / KST) & 1, p.limit_ns, no_abort);
            for (int j = max(0, issued_v - VST); j < issued_v; ++j)
                ptx::mbar_wait(&bars->v_full[j % VST], (j / VST) & 1, p.limit_ns, no_abort);
        }
    } else if (warp == kMmaWarp) {
        // ================================================= MMA issuer
        if (nt > 0) {
            bool ok = true;
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
            auto issue_s = [&](int j) {
                if (!wait_or_fail(&bars->k_full[j % KST], (j / KST) & 1, 6)) return;
                ptx::tc_fence_after();
                const uint64_t kd = k_desc0 + (uint64_t)(j % KST) * kTileUnits;
                const uint32_t d_s = tmem + (uint32_t)((j & 1) * kBlockN);
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk) {
                    const uint64_t off = (uint64_t)(((kk >> 2) * kBlockBytes + (kk & 3) * 32) >> 4);
                    ptx::umma_ts_elect(d_s, tmem + kColQ + kk * 8, kd + off, kIdescS, kk > 0);
                }
                ptx::umma_commit_elect(&bars->s_full[j & 1]);
                ptx::umma_commit_elect(&bars->k_empty[j % KST]);
                __syncwarp();
            };
            if (wait_or_fail(&bars->q_tmem, 0, 7)) {
                ptx::tc_fence_after();
                issue_s(0);
            }
            for (int j = 0; ok && j < nt; ++j) {
                if (j + 1 < nt) {
                    issue_s(j + 1);
                    if (!ok) break;
                }
                if (!wait_or_fail(&bars->p_full[j & 1], (j >> 1) & 1, 8)) break;
                if (!wait_or_fail(&bars->v_full[j % VST], (j / VST) & 1, 9)) break;
                ptx::tc_fence_after();
                const uint64_t vd = v_desc0 + (uint64_t)(j % VST) * kTileUnits;
                const uint32_t a_p = tmem + (uint32_t)((j & 1) * kBlockN);
                const uint32_t acc0 = j > 0 ? 1u : 0u;
#pragma unroll
                for (int kk = 0; kk < kBlockN / 16; ++kk)
                    ptx::umma_ts_elect(tmem + kColO, a_p + kk * 8,
                                       vd + (uint64_t)((kk * 16 * 128) >> 4), kIdescO,
                                       kk > 0 ? 1u : acc0);
                ptx::umma_commit_elect(&bars->o_done);
                if (j == nt - 1) ptx::umma_commit_elect(&bars->o_final);
                ptx::umma_commit_elect(&bars->v_empty[j % VST]);
                __syncwarp();
            }
            if (!ok) {
                int zero = 0;
                volatile int* no_abort = &zero;
                ptx::umma_commit_elect(&bars->drain);
                __syncwarp();
                ptx::mbar_wait(&bars->drain, 0, p.limit_ns, no_abort);
            }
        }
    } else {
        // ================================================= softmax warps
        const uint32_t quarter = (uint32_t)(warp & 3);
        const int part = warp >> 2;
        const uint32_t row = quarter * 32u + (uint32_t)lane;
        const uint32_t lane_addr = (quarter * 32u) << 16;
        const int tok = (int)row / p.G;  // token of this query row
        int row_lim = key_end - 1;       // last visible key (absolute index)
        if (p.causal) row_lim = min(row_lim, tok + Lk - p.Nq);
        const float sl2 = p.scale_log2;
        float m_ref = -INFINITY;
        float l_part = 0.f;
        bool ok = true;
        float* red_max = reinterpret_cast<float*>(smem + L::kRedMax);
        float* red_sum = reinterpret_cast<float*>(smem + L::kRedSum);
        const uint32_t row_bar = 1 + quarter;
        const uint32_t t_o = tmem + lane_addr + kColO + (uint32_t)(part * kPartD);

        // ---- Q -> tensor memory (A operand of S = Q Kᵀ)
        if (nt > 0) {
            if (!warp_wait(&bars->q_full, 0, p.limit_ns, abort_flag)) {
                record_error(p.err, kErrDecodeBase + 10, &bars->abort);
                ok = false;
            } else if (part * 32 < D) {
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
            if (ok && lane == 0) ptx::mbar_arrive(&bars->q_tmem);
        }

        // Every warp walks all nt iterations and reaches every row barrier.
        for (int j = 0; j < nt; ++j) {
            const int sb = j & 1;
            if (ok && !warp_wait(&bars->s_full[sb], (j >> 1) & 1, p.limit_ns, abort_flag)) {
                record_error(p.err, kErrDecodeBase + 11, &bars->abort);
                ok = false;
            }
            const uint32_t t_s = tmem + lane_addr + (uint32_t)(sb * kBlockN);
            const int key_base = key_begin + j * kBlockN + part * 32;
            const bool masked = key_base + 31 > row_lim;
            uint32_t r[32];
            float pmax = -INFINITY;
            if (ok) {
                ptx::tc_fence_after();
                ptx::tmem_ld32(t_s + part * 32, r);
                float mx8[8];
#pragma unroll
                for (int u = 0; u < 8; ++u) mx8[u] = -INFINITY;
                ptx::tmem_wait_ld_dep(r);
                if (masked)
                    part_max<true>(r, key_base, row_lim, mx8);
                else
                    part_max<false>(r, key_base, row_lim, mx8);
                pmax = ptx::max3(ptx::max3(mx8[0], mx8[1], mx8[2]),
                                 ptx::max3(mx8[3], mx8[4], mx8[5]), fmaxf(mx8[6], mx8[7]));
            }
            red_max[((j & 1) * 4 + part) * 128 + row] = pmax;
            ptx::named_barrier_sync(row_bar, 128);
            if (!ok) continue;
            const float* rm = red_max + (j & 1) * 4 * 128 + row;
            const float mx = fmaxf(ptx::max3(rm[0], rm[128], rm[256]), rm[384]);
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
                // S_j done implies P_{j-2} V_{j-2} is: phase j-1 of o_done is
                // the current or the previous one, so the parity wait is exact
                if (!warp_wait(&bars->o_done, (j - 1) & 1, p.limit_ns, abort_flag)) {
                    record_error(p.err, kErrDecodeBase + 12, &bars->abort);
                    ok = false;
                    ptx::tmem_wait_st();
                    continue;
                }
                ptx::tc_fence_after();
                const float sc = rescale ? alpha : 1.f;
                if constexpr (kPartD == 32) {
                    uint32_t o[32];
                    ptx::tmem_ld32(t_o, o);
                    ptx::tmem_wait_ld_dep(o);
#pragma unroll
                    for (int e = 0; e < 32; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * sc);
                    ptx::tmem_st32(t_o, o);
                } else {
                    uint32_t o[16];
                    ptx::tmem_ld16(t_o, o);
                    ptx::tmem_wait_ld_dep16(o);
#pragma unroll
                    for (int e = 0; e < 16; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * sc);
                    ptx::tmem_st16(t_o, o);
                }
            }
            ptx::tmem_wait_st();
            if (key_begin + j * kBlockN + kBlockN > key_end && part == 0) {
                // rows past the split's last key: zero their V rows (0 * NaN guard)
                const int sv = j % VST;
                if (!warp_wait(&bars->v_full[sv], (j / VST) & 1, p.limit_ns, abort_flag)) {
                    record_error(p.err, kErrDecodeBase + 13, &bars->abort);
                    ok = false;
                    continue;
                }
                if (key_begin + j * kBlockN + (int)row >= key_end) {
                    uint8_t* vt = smem + L::kV + sv * kTileBytes;
#pragma unroll
                    for (int c = 0; c < kDBlocks; ++c)
#pragma unroll
                        for (int ch = 0; ch < 8; ++ch)
                            *reinterpret_cast<uint4*>(vt + c * kBlockBytes + row * 128 + ch * 16) =
                                make_uint4(0, 0, 0, 0);
                }
                ptx::fence_proxy_async_smem();
            }
            ptx::tc_fence_before();
            __syncwarp();
            if (lane == 0) ptx::mbar_arrive(&bars->p_full[sb]);
        }

        // ---- this split's O and LSE
        if (ok && nt > 0) {
            if (!warp_wait(&bars->o_final, 0, p.limit_ns, abort_flag)) {
                record_error(p.err, kErrDecodeBase + 14, &bars->abort);
                ok = false;
            }
            ptx::tc_fence_after();
        }
        red_sum[part * 128 + row] = l_part;
        ptx::named_barrier_sync(row_bar, 128);
        const float l_sum =
            (red_sum[row] + red_sum[128 + row]) + (red_sum[256 + row] + red_sum[384 + row]);
        const bool have = ok && nt > 0 && l_sum > 0.f;
        const float inv_l = have ? 1.f / l_sum : 0.f;
        const float lse_nat = have ? (m_ref + ptx::lg2_approx(l_sum)) * kLn2 : -INFINITY;
        uint32_t o[kPartD];
        if (ok && nt > 0) {
            if constexpr (kPartD == 32) {
                ptx::tmem_ld32(t_o, o);
                ptx::tmem_wait_ld_dep(o);
            } else {
                ptx::tmem_ld16(t_o, o);
                ptx::tmem_wait_ld_dep16(o);
            }
        } else {
#pragma unroll
            for (int e = 0; e < kPartD; ++e) o[e] = 0u;
        }
        const size_t unit = (size_t)b * p.Hkv + g;
        const bool valid_row = (int)row < p.rows;
        const int head = g * p.G + (int)row % p.G;
        if (nsplit == 1) {
            // final output: swizzled staging in the Q buffer -> TMA store
            uint8_t* stage = smem + L::kQ;
            uint32_t o2[kPartD / 2];
#pragma unroll
            for (int e = 0; e < kPartD / 2; ++e)
                o2[e] = ptx::pack2<BF16>(__uint_as_float(o[2 * e]) * inv_l,
                                         __uint_as_float(o[2 * e + 1]) * inv_l);
            const int col = part * kPartD;
#pragma unroll
            for (int q4 = 0; q4 < kPartD / 8; ++q4) {
                const uint32_t ch = (uint32_t)(((col & 63) >> 3) + q4);
                *reinterpret_cast<uint4*>(stage + (col >> 6) * kBlockBytes + sw128_offset(row, ch)) =
                    make_uint4(o2[q4 * 4], o2[q4 * 4 + 1], o2[q4 * 4 + 2], o2[q4 * 4 + 3]);
            }
            ptx::fence_proxy_async_smem();
            ptx::named_barrier_sync(5, 32 * kSoftmaxWarps);
            if (warp == 0 && lane == 0) {
                for (int c = 0; c < kDBlocks; ++c)
                    ptx::tma_store_5d(&tm_o, stage + c * kBlockBytes, c * 64, 0, g, 0, b);
                ptx::bulk_commit_group();
                ptx::bulk_wait_group_read0();
            }
            if (part == 0 && valid_row)
                p.lse[((size_t)b * p.Hq + head) * p.Nq + tok] = lse_nat;
        } else {
            // normalised partial O (fp32) and LSE of this split
            float* po = p.part_o + ((unit * p.max_splits + split) * kBlockM + row) * D + part * kPartD;
#pragma unroll
            for (int e = 0; e < kPartD; e += 4)
                *reinterpret_cast<float4*>(po + e) =
                    make_float4(__uint_as_float(o[e]) * inv_l, __uint_as_float(o[e + 1]) * inv_l,
                                __uint_as_float(o[e + 2]) * inv_l, __uint_as_float(o[e + 3]) * inv_l);
            if (part == 0) p.part_lse[(unit * p.max_splits + split) * kBlockM + row] = lse_nat;
            // the last CTA of this (sequence, kv head) merges the splits
            __threadfence();
            ptx::named_barrier_sync(5, 32 * kSoftmaxWarps);
            if (tid == 0) {
                const unsigned prev = atomicAdd(p.counters + unit, 1u);
                bars->is_last = (prev == (unsigned)(nsplit - 1)) ? 1 : 0;
            }
            ptx::named_barrier_sync(5, 32 * kSoftmaxWarps);
            if (bars->is_last) {
                __threadfence();
                float* row_lse = reinterpret_cast<float*>(smem + L::kRowLse);
                const float* pl = p.part_lse + unit * p.max_splits * kBlockM;
                const float* pov = p.part_o + unit * p.max_splits * kBlockM * D;
                if (tid < kBlockM) {
                    float M = -INFINITY;
                    for (int s2 = 0; s2 < nsplit; ++s2) M = fmaxf(M, __ldcg(pl + s2 * kBlockM + tid));
                    float tot = -INFINITY;
                    if (M != -INFINITY) {
                        float acc = 0.f;
                        for (int s2 = 0; s2 < nsplit; ++s2) {
                            const float ls = __ldcg(pl + s2 * kBlockM + tid);
                            if (ls != -INFINITY) acc += __expf(ls - M);
                        }
                        tot = M + __logf(acc);
                    }
                    row_lse[tid] = tot;
                }
                ptx::named_barrier_sync(5, 32 * kSoftmaxWarps);
                // this thread: row `row`, columns part * D/4 .. +D/4
                if (valid_row) {
                    const float tot = row_lse[row];
                    float acc[kPartD];
#pragma unroll
                    for (int e = 0; e < kPartD; ++e) acc[e] = 0.f;
                    if (tot != -INFINITY) {
                        for (int s2 = 0; s2 < nsplit; ++s2) {
                            const float ls = __ldcg(pl + s2 * kBlockM + row);
                            if (ls == -INFINITY) continue;
                            const float w = __expf(ls - tot);
                            const float* src = pov + ((size_t)s2 * kBlockM + row) * D + part * kPartD;
#pragma unroll
                            for (int e = 0; e < kPartD; e += 4) {
                                const float4 v4 = __ldcg(reinterpret_cast<const float4*>(src + e));
                                acc[e] += w * v4.x;
                                acc[e + 1] += w * v4.y;
                                acc[e + 2] += w * v4.z;
                                acc[e + 3] += w * v4.w;
                            }
                        }
                    }
                    const size_t obase = (((size_t)b * p.Nq + tok) * p.Hq + head) * D + part * kPartD;
                    uint4* dst = reinterpret_cast<uint4*>(static_cast<uint16_t*>(p.o) + obase);
#pragma unroll
                    for (int e = 0; e < kPartD; e += 8)
                        dst[e / 8] = make_uint4(ptx::pack2<BF16>(acc[e], acc[e + 1]),
                                                ptx::pack2<BF16>(acc[e + 2], acc[e + 3]),
                                                ptx::pack2<BF16>(acc[e + 4], acc[e + 5]),
                                                ptx::pack2<BF16>(acc[e + 6], acc[e + 7]));
                    if (part == 0) p.lse[((size_t)b * p.Hq + head) * p.Nq + tok] = tot;
                }
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
                     const CUtensorMap& omap, const DecodeParams& p, cudaStream_t stream) {
    using L = TcSmem<D, KST, VST>;
    static_assert(L::kAlloc <= 227 * 1024, "shared memory budget");
    auto kern = attn_decode_tc_kernel<D, BF16, KST, VST>;
    cudaError_t e =
        cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)L::kAlloc);
    if (e != cudaSuccess) return e;
    dim3 grid(p.max_splits, p.Hkv, p.B);
    kern<<<grid, kThreads, L::kAlloc, stream>>>(qmap, kmap, vmap, omap, p);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_decode_tc(const CUtensorMap& qmap, const CUtensorMap& kmap,
                             const CUtensorMap& vmap, const CUtensorMap& omap,
                             const DecodeParams& p, int d, bool bf16, cudaStream_t stream) {
    if (d == 64) {
        return bf16 ? launch_t<64, true, 4, 4>(qmap, kmap, vmap, omap, p, stream)
                    : launch_t<64, false, 4, 4>(qmap, kmap, vmap, omap, p, stream);
    }
    return bf16 ? launch_t<128, true, 2, 3>(qmap, kmap, vmap, omap, p, stream)
                : launch_t<128, false, 2, 3>(qmap, kmap, vmap, omap, p, stream);
}

}  // namespace attn
