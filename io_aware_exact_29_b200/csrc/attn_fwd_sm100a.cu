// attn_fwd_sm100a.cu -- exact attention forward on tcgen05 tensor cores.
//
// One CTA owns one 128-row tile of queries of one (batch, head) and streams
// the key/value tiles of its head through shared memory (ai6s.net article on
// the ops-transformer FlashAttention operator, section "FlashAttention 拆的不是
// 算法，是数据流": split Q, K, V along the sequence into on-chip tiles, run
// Q_tile·K_tileᵀ -> softmax -> ·V_tile on chip, write back only O; the
// effectstory.com article "FlashAttention：IO 感知的精確注意力演算法..." states
// the same single pass: Q, K, V loaded once, O written once).
//
// Warp roles (576 threads):
//   warps 0-15  softmax: warp w owns query rows 32*(w%4) .. +31 (its TMEM lane
//               quarter) and score columns 32*(w/4) .. +31 of every tile:
//               four warps share each row, four softmax warps per SM
//               sub-partition hide each other's latencies
//   warp 16     TMA loader: Q once, then K_j / V_j into rings
//   warp 17     tensor-memory owner and tcgen05.mma issuer (one lane)
// Tensor memory (512 columns): score buffers S[0] = [0,128) and S[1] =
// [128,256) (double-buffered: S_{j+1} is computed while the softmax of tile j
// runs), O accumulator [256, 256+D), Q [384, 384+D/2) (two 16-bit values per
// column).  The softmax warps copy Q from shared memory into tensor memory
// once, so S = Q·Kᵀ reads only K from shared memory.  Each softmax thread
// reads its 32 scores of S[j%2], agrees on the row maximum with the three
// other warps of its rows through shared memory, keeps the running max m and
// its share of the running sum l (the online softmax of the section above),
// and writes P (bf16/fp16) back over the first 64 columns of S[j%2]; the P·V
// MMA reads P from tensor memory as its A operand and V from shared memory.
//
// MMA issue order: S_0, then per tile j: S_{j+1}, P_j·V_j.  MMAs from one
// thread execute in issue order, so S_{j+1} (into the buffer of P_{j-1}) never
// overtakes P_{j-1}·V_{j-1}.
//
// Fused masks: the causal rule (adaptation point 2 of the ai6s.net article)
// and the per-sequence key length (point 3) are index arithmetic on the score
// row; tiles wholly outside them are never loaded, and V rows behind the real
// length are zeroed in shared memory so that 0 * NaN cannot reach O.
//
// Lazy rescaling: the reference maximum of a row only moves when a tile's
// maximum exceeds it by more than 8 (log2 units), so P <= 2^8; numerator and
// denominator share the reference, so the result is the same exact softmax.
#include "attn_internal.h"
#include "ptx.cuh"

namespace attn {
namespace {

constexpr int kBlockM = 128;  // rows per Q tile
constexpr int kBlockN = 128;  // keys per K/V tile
constexpr int kThreads = 576;
constexpr int kSoftmaxWarps = 16;
constexpr uint32_t kTmemCols = 512;
constexpr float kRescaleThreshold = 8.0f;

template <int D, int KST, int VST>
struct FwdSmem {
    static constexpr uint32_t kTileBytes = kBlockM * D * 2;  // one 128 x D tile
    static constexpr uint32_t kQ = 0;
    static constexpr uint32_t kK = kQ + kTileBytes;
    static constexpr uint32_t kV = kK + KST * kTileBytes;
    static constexpr uint32_t kRedMax = kV + VST * kTileBytes;  // [2 slots][4 parts][128] fp32
    static constexpr uint32_t kRedSum = kRedMax + 2 * 4 * 128 * 4;  // [4 parts][128] fp32
    static constexpr uint32_t kBars = kRedSum + 4 * 128 * 4;
    static constexpr uint32_t kTotal = kBars + 512;
    static constexpr uint32_t kAlloc = kTotal + 1024;  // manual 1024-B alignment
};

template <int KST, int VST>
struct FwdBars {
    uint64_t q_full;
    uint64_t k_full[KST];
    uint64_t k_empty[KST];
    uint64_t v_full[VST];
    uint64_t v_empty[VST];
    uint64_t s_full[2];
    uint64_t p_full[2];
    uint64_t o_done;
    uint64_t q_tmem;  // Q copied into tensor memory
    uint64_t drain;
    uint32_t tmem_base;
    int abort;
};

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

// Running maxima of 32 score columns (one 32-column TMEM load) into eight
// independent chains.  kMask: the tile reaches past the row's last visible
// key (key_base + c > row_lim is masked).
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

// p = 2^(s * scale_log2 - m) for 32 score columns, accumulated into four
// pair sums and packed two per 32-bit word (bf16 or fp16).
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
            // every fourth pair on the FMA pipe: the exp2 unit and the tensor
            // pipe carry equal work at d = 128, this takes a quarter off the former
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
    attn_fwd_kernel(const __grid_constant__ CUtensorMap tm_q,
                    const __grid_constant__ CUtensorMap tm_k,
                    const __grid_constant__ CUtensorMap tm_v,
                    const __grid_constant__ CUtensorMap tm_o, const __grid_constant__ FwdParams p) {
    using L = FwdSmem<D, KST, VST>;
    constexpr uint32_t kTileBytes = L::kTileBytes;
    constexpr int kDBlocks = D / 64;  // 64-column (128-byte) blocks per row
    constexpr uint32_t kBlockBytes = kBlockM * 128;
    constexpr uint32_t kIdescS = ptx::idesc_f16(kBlockM, kBlockN, BF16, false);
    constexpr uint32_t kIdescO = ptx::idesc_f16(kBlockM, D, BF16, true);
    constexpr uint32_t kColO = 256;
    constexpr uint32_t kColQ = 384;
    constexpr int kPartD = D / 4;  // O columns per softmax warp
    constexpr int kLoaderWarp = kSoftmaxWarps, kMmaWarp = kSoftmaxWarps + 1;

    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw_addr = ptx::smem_u32(smem_raw);
    uint8_t* smem = smem_raw + (((raw_addr + 1023u) & ~1023u) - raw_addr);
    const uint32_t sbase = ptx::smem_u32(smem);
    FwdBars<KST, VST>* bars = reinterpret_cast<FwdBars<KST, VST>*>(smem + L::kBars);
    volatile int* abort_flag = &bars->abort;

    const int tid = threadIdx.x;
    const int warp = tid >> 5;
    const int lane = tid & 31;

    // ---- work unit: rows [q0, q0 + 128) of head h of batch b
    const int qt = p.causal ? (p.n_qtiles - 1 - (int)blockIdx.x) : (int)blockIdx.x;
    const int h = blockIdx.y;
    const int b = blockIdx.z;
    const int g = h / p.G;
    const int Lk = p.seqlens_k ? p.seqlens_k[b] : p.Nk;
    const int q0 = qt * kBlockM;
    const int nt = tiles_for(q0, p.Nq, Lk, p.causal);

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
        ptx::mbar_init(&bars->q_tmem, kSoftmaxWarps);
        ptx::mbar_init(&bars->drain, 1);
        bars->abort = 0;
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

    // The loader and MMA loops run on all 32 lanes of their warp; one lane
    // issues the copies and MMAs, and every wait's outcome is warp-uniform.
    if (warp == kLoaderWarp) {
        // ================================================= TMA loader
        if (nt > 0 && !p.inject) {
            int issued_k = 0, issued_v = 0;
            if (lane == 0) {
                ptx::mbar_arrive_expect_tx(&bars->q_full, kTileBytes);
                for (int c = 0; c < kDBlocks; ++c)
                    ptx::tma_load_4d(smem + L::kQ + c * kBlockBytes, &tm_q, &bars->q_full, c * 64,
                                     h, q0, b);
            }
            __syncwarp();
            for (int j = 0; j < nt; ++j) {
                const int sk = j % KST;
                if (!warp_wait(&bars->k_empty[sk], ((j / KST) & 1) ^ 1, p.limit_ns, abort_flag)) {
                    record_error(p.err, kErrFwdBase + 1, &bars->abort);
                    break;
                }
                if (lane == 0) {
                    ptx::mbar_arrive_expect_tx(&bars->k_full[sk], kTileBytes);
                    for (int c = 0; c < kDBlocks; ++c)
                        ptx::tma_load_4d(smem + L::kK + sk * kTileBytes + c * kBlockBytes, &tm_k,
                                         &bars->k_full[sk], c * 64, g, j * kBlockN, b);
                }
                __syncwarp();
                ++issued_k;
                const int sv = j % VST;
                if (!warp_wait(&bars->v_empty[sv], ((j / VST) & 1) ^ 1, p.limit_ns, abort_flag)) {
                    record_error(p.err, kErrFwdBase + 2, &bars->abort);
                    break;
                }
                if (lane == 0) {
                    ptx::mbar_arrive_expect_tx(&bars->v_full[sv], kTileBytes);
                    for (int c = 0; c < kDBlocks; ++c)
                        ptx::tma_load_4d(smem + L::kV + sv * kTileBytes + c * kBlockBytes, &tm_v,
                                         &bars->v_full[sv], c * 64, g, j * kBlockN, b);
                }
                __syncwarp();
                ++issued_v;
            }
            // Never leave the CTA with a copy in flight: wait (bounded, and
            // regardless of the abort flag) for the last phase of each
            // barrier that received a copy.
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
                    record_error(p.err, kErrFwdBase + site, &bars->abort);
                    ok = false;
                }
                return ok;
            };
            // Descriptors are built once; each MMA adds a compile-time offset
            // (in 16-byte units) to a base descriptor.
            const uint64_t k_desc0 = ptx::sdesc_sw128(sbase + L::kK, 16, 1024);
            const uint64_t v_desc0 = ptx::sdesc_sw128(sbase + L::kV, kBlockBytes, 1024);
            constexpr uint64_t kTileUnits = kTileBytes >> 4;
            auto issue_s = [&](int j) {
                if (!wait_or_fail(&bars->k_full[j % KST], (j / KST) & 1, 4)) return;
                ptx::tc_fence_after();
                const uint64_t kd = k_desc0 + (uint64_t)(j % KST) * kTileUnits;
                const uint32_t d_s = tmem + (uint32_t)((j & 1) * kBlockN);
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk) {
                    // A = Q from tensor memory (8 columns per 16 values);
                    // B = K, K-major: +32 B per 16 values, +16 KB per block
                    const uint64_t off = (uint64_t)(((kk >> 2) * kBlockBytes + (kk & 3) * 32) >> 4);
                    ptx::umma_ts_elect(d_s, tmem + kColQ + kk * 8, kd + off, kIdescS, kk > 0);
                }
                ptx::umma_commit_elect(&bars->s_full[j & 1]);
                ptx::umma_commit_elect(&bars->k_empty[j % KST]);
                __syncwarp();
            };
            if (wait_or_fail(&bars->q_tmem, 0, 3)) {
                ptx::tc_fence_after();
                issue_s(0);
            }
            for (int j = 0; ok && j < nt; ++j) {
                if (j + 1 < nt) {
                    issue_s(j + 1);
                    if (!ok) break;
                }
                if (!wait_or_fail(&bars->p_full[j & 1], (j >> 1) & 1, 5)) break;
                if (!wait_or_fail(&bars->v_full[j % VST], (j / VST) & 1, 6)) break;
                ptx::tc_fence_after();
                {
                    const uint64_t vd = v_desc0 + (uint64_t)(j % VST) * kTileUnits;
                    const uint32_t a_p = tmem + (uint32_t)((j & 1) * kBlockN);
                    const uint32_t acc0 = j > 0 ? 1u : 0u;
#pragma unroll
                    for (int kk = 0; kk < kBlockN / 16; ++kk) {
                        // MN-major V: +16 keys = +2 KB per step
                        ptx::umma_ts_elect(tmem + kColO, a_p + kk * 8,
                                           vd + (uint64_t)((kk * 16 * 128) >> 4), kIdescO,
                                           kk > 0 ? 1u : acc0);
                    }
                    ptx::umma_commit_elect(&bars->o_done);
                    ptx::umma_commit_elect(&bars->v_empty[j % VST]);
                }
                __syncwarp();
            }
            if (!ok) {
                // make sure no MMA is still running before TMEM is freed
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
        const int part = warp >> 2;  // which 32 score columns / D/4 output columns
        const uint32_t row = quarter * 32u + (uint32_t)lane;
        const uint32_t lane_addr = (quarter * 32u) << 16;
        const int i = q0 + (int)row;
        int row_lim = Lk - 1;  // last visible key of this row
        if (p.causal) row_lim = min(row_lim, i + Lk - p.Nq);
        const float sl2 = p.scale_log2;
        float m_ref = -INFINITY;  // running reference max, scale*log2 units
        float l_part = 0.f;       // this warp's share of the running sum
        bool ok = true;
        float* red_max = reinterpret_cast<float*>(smem + L::kRedMax);
        float* red_sum = reinterpret_cast<float*>(smem + L::kRedSum);
        const uint32_t row_bar = 1 + quarter;  // the four warps of these rows
        const uint32_t t_o = tmem + lane_addr + kColO + (uint32_t)(part * kPartD);

        // ---- Q -> tensor memory (A operand of S = Q Kᵀ): this warp copies
        // d values [32 part, 32 part + 32) of its rows, two per column
        if (nt > 0) {
            if (!warp_wait(&bars->q_full, 0, p.limit_ns, abort_flag)) {
                record_error(p.err, kErrFwdBase + 11, &bars->abort);
                ok = false;
            } else if (part * 32 < D) {
                const int c0 = part * 32;  // first d value
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

        // Every warp walks all nt iterations and reaches every row barrier,
        // also after a failed wait (then it only skips its work), so that its
        // partners can never be left waiting at a barrier.
        for (int j = 0; j < nt; ++j) {
            const int sb = j & 1;
            if (ok && !warp_wait(&bars->s_full[sb], (j >> 1) & 1, p.limit_ns, abort_flag)) {
                record_error(p.err, kErrFwdBase + 7, &bars->abort);
                ok = false;
            }
            const uint32_t t_s = tmem + lane_addr + (uint32_t)(sb * kBlockN);
            const int key_base = j * kBlockN + part * 32;
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
            // the row maximum over the four parts, through shared memory
            red_max[((j & 1) * 4 + part) * 128 + row] = pmax;
            ptx::named_barrier_sync(row_bar, 128);
            if (!ok) continue;
            const float* rm = red_max + (j & 1) * 4 * 128 + row;
            const float mx = fmaxf(ptx::max3(rm[0], rm[128], rm[256]), rm[384]);
            const float m_tile = mx * sl2;  // -inf stays -inf (sl2 > 0)
            float alpha = 1.f;
            bool rescale = false;
            if (m_tile > m_ref + kRescaleThreshold) {
                alpha = ptx::ex2_approx(m_ref - m_tile);  // 0 when m_ref = -inf
                rescale = (j > 0) && (m_ref != -INFINITY);
                m_ref = m_tile;
            }
            const float m_use = (m_ref == -INFINITY) ? 0.f : m_ref;
            uint64_t acc2[4] = {0, 0, 0, 0};  // four pair accumulators of the row sum
            uint32_t pk[16];
            if (masked)
                part_exp<true, BF16>(r, key_base, row_lim, ptx::f2_pack(sl2, sl2),
                                     ptx::f2_pack(-m_use, -m_use), acc2, pk);
            else
                part_exp<false, BF16>(r, key_base, row_lim, ptx::f2_pack(sl2, sl2),
                                      ptx::f2_pack(-m_use, -m_use), acc2, pk);
            // P of these 32 keys over columns [16 part, 16 part + 16) of S[sb]
            ptx::tmem_st16(t_s + part * 16, pk);
            float s0, s1, s2, s3, s4, s5, s6, s7;
            ptx::f2_unpack(acc2[0], s0, s1);
            ptx::f2_unpack(acc2[1], s2, s3);
            ptx::f2_unpack(acc2[2], s4, s5);
            ptx::f2_unpack(acc2[3], s6, s7);
            l_part = l_part * alpha + (((s0 + s1) + (s2 + s3)) + ((s4 + s5) + (s6 + s7)));
            if (__any_sync(0xffffffffu, rescale)) {
                // O must hold P_{j-1} V_{j-1} before it is rescaled (all four
                // warps of a row take the same decision).  S_j being done
                // implies P_{j-2} V_{j-2} is, so phase j-1 is the current or
                // the previous phase of o_done and a parity wait is exact.
                if (!warp_wait(&bars->o_done, (j - 1) & 1, p.limit_ns, abort_flag)) {
                    record_error(p.err, kErrFwdBase + 10, &bars->abort);
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
            const bool zero_v = p.seqlens_k != nullptr && j * kBlockN + kBlockN > Lk && part == 0;
            if (zero_v) {
                // keys behind the real length: zero their V rows so that a
                // non-finite value stored there cannot reach O through 0 * NaN
                const int sv = j % VST;
                if (!warp_wait(&bars->v_full[sv], (j / VST) & 1, p.limit_ns, abort_flag)) {
                    record_error(p.err, kErrFwdBase + 8, &bars->abort);
                    ok = false;
                    continue;
                }
                if (j * kBlockN + (int)row >= Lk) {
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
            // each thread's P stores are complete (wait::st above); one
            // arrival per warp after the warp has converged
            ptx::tc_fence_before();
            __syncwarp();
            if (lane == 0) ptx::mbar_arrive(&bars->p_full[sb]);
        }

        // ---- epilogue: O / l -> bf16/fp16 -> swizzled staging (the Q
        // buffer, free once Q is in tensor memory and the last MMA is done)
        // -> TMA store.  o_done completes once per P·V.  When the last tile's
        // softmax ends, P_{nt-2}·V may still be pending (S_{nt-1} was issued
        // before it), and a parity wait only tells the current phase from the
        // one before it: wait for phase nt-2, then for phase nt-1.
        if (ok && nt > 0) {
            if ((nt >= 2 && !warp_wait(&bars->o_done, (nt - 2) & 1, p.limit_ns, abort_flag)) ||
                !warp_wait(&bars->o_done, (nt - 1) & 1, p.limit_ns, abort_flag)) {
                record_error(p.err, kErrFwdBase + 9, &bars->abort);
                ok = false;
            }
            ptx::tc_fence_after();
        }
        // the four parts' sums of the row
        red_sum[part * 128 + row] = l_part;
        ptx::named_barrier_sync(row_bar, 128);
        const float l_sum = (red_sum[row] + red_sum[128 + row]) + (red_sum[256 + row] + red_sum[384 + row]);
        const bool have = ok && nt > 0 && l_sum > 0.f;
        const float inv_l = have ? 1.f / l_sum : 0.f;
        uint8_t* stage = smem + L::kQ;
        if (q0 < p.Nq) {
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
            uint32_t o2[kPartD / 2];
#pragma unroll
            for (int e = 0; e < kPartD / 2; ++e)
                o2[e] = ptx::pack2<BF16>(__uint_as_float(o[2 * e]) * inv_l,
                                         __uint_as_float(o[2 * e + 1]) * inv_l);
            // output columns part * D/4 .. +D/4: 128-byte block col / 64,
            // 16-byte chunks (col % 64) / 8 ..
            const int col = part * kPartD;
#pragma unroll
            for (int q4 = 0; q4 < kPartD / 8; ++q4) {
                const uint32_t ch = (uint32_t)(((col & 63) >> 3) + q4);
                *reinterpret_cast<uint4*>(stage + (col >> 6) * kBlockBytes +
                                          sw128_offset(row, ch)) =
                    make_uint4(o2[q4 * 4], o2[q4 * 4 + 1], o2[q4 * 4 + 2], o2[q4 * 4 + 3]);
            }
            ptx::fence_proxy_async_smem();
        }
        ptx::named_barrier_sync(5, 32 * kSoftmaxWarps);
        if (warp == 0 && lane == 0 && q0 < p.Nq) {
            for (int c = 0; c < kDBlocks; ++c)
                ptx::tma_store_4d(&tm_o, stage + c * kBlockBytes, c * 64, h, q0, b);
            ptx::bulk_commit_group();
            ptx::bulk_wait_group_read0();
        }
        if (part == 0 && i < p.Nq) {
            const float lse = have ? (m_ref + ptx::lg2_approx(l_sum)) * 0.69314718055994531f
                                   : -INFINITY;
            p.lse[((size_t)b * p.Hq + h) * p.Nq + i] = lse;
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
cudaError_t launch_fwd_t(const FwdMaps& maps, const FwdParams& p, cudaStream_t stream) {
    using L = FwdSmem<D, KST, VST>;
    static_assert(L::kAlloc <= 227 * 1024, "shared memory budget");
    auto kern = attn_fwd_kernel<D, BF16, KST, VST>;
    cudaError_t e =
        cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)L::kAlloc);
    if (e != cudaSuccess) return e;
    dim3 grid(p.n_qtiles, p.Hq, p.B);
    kern<<<grid, kThreads, L::kAlloc, stream>>>(maps.q, maps.k, maps.v, maps.o, p);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_fwd(const FwdMaps& maps, const FwdParams& p, int d, bool bf16,
                       cudaStream_t stream) {
    if (d == 64) {
        return bf16 ? launch_fwd_t<64, true, 4, 4>(maps, p, stream)
                    : launch_fwd_t<64, false, 4, 4>(maps, p, stream);
    }
    return bf16 ? launch_fwd_t<128, true, 2, 3>(maps, p, stream)
                : launch_fwd_t<128, false, 2, 3>(maps, p, stream);
}

}  // namespace attn
