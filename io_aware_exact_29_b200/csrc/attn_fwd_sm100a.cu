// attn_fwd_sm100a.cu -- exact attention forward on tcgen05 tensor cores.
//
// One CTA owns one 128-row tile of queries of one (batch, head) and streams
// the key/value tiles of its head through shared memory (ai6s.net article on
// the ops-transformer FlashAttention operator, section "FlashAttention 拆的不是
// 算法，是数据流": split Q, K, V along the sequence into on-chip tiles, run
// Q_tile·K_tileᵀ -> softmax -> ·V_tile on chip, write back only O).
//
// Warp roles (192 threads):
//   warp 0      TMA loader: Q once, then K_j and V_j into a STAGES-deep ring
//   warp 1      tensor-memory owner and single-thread tcgen05.mma issuer:
//               S_j = Q·K_jᵀ into one of two TMEM score buffers, then
//               O += P_{j-1}·V_{j-1} into the TMEM output accumulator
//   warps 2..5  softmax: thread t owns query row t (TMEM lane t); per tile it
//               reads its score row from TMEM, applies the fused mask, keeps
//               the running max m and running sum l (the online softmax of
//               the same section), rescales its O row in TMEM when the max
//               grows, and writes P (bf16/fp16) into swizzled shared memory
//               as the A operand of the next MMA; at the end it normalises O,
//               stores it by TMA and writes LSE.
//
// The causal mask (adaptation point 2 of the same article) is index
// arithmetic on the score row; tiles wholly above the diagonal are never
// loaded.  With per-sequence key lengths (adaptation point 3) the tile loop
// stops at the real length and the rows behind it are masked and their V rows
// zeroed in shared memory.
//
// Lazy rescaling: the reference maximum only moves when a tile's maximum
// exceeds it by more than 8 (log2 units), so P <= 2^8 and the result is the
// same exact softmax (numerator and denominator use one reference).
#include "attn_internal.h"
#include "ptx.cuh"

namespace attn {
namespace {

constexpr int kBlockM = 128;
constexpr int kBlockN = 128;
constexpr int kThreads = 192;
constexpr uint32_t kTmemCols = 512;
constexpr float kRescaleThreshold = 8.0f;

template <int D, int STAGES>
struct FwdSmem {
    static constexpr uint32_t kTileBytes = kBlockM * D * 2;  // one 128 x D tile
    static constexpr uint32_t kPBytes = kBlockM * kBlockN * 2;
    static constexpr uint32_t kQ = 0;
    static constexpr uint32_t kK = kQ + kTileBytes;
    static constexpr uint32_t kV = kK + STAGES * kTileBytes;
    static constexpr uint32_t kP = kV + STAGES * kTileBytes;
    static constexpr uint32_t kBars = kP + kPBytes;
    static constexpr uint32_t kTotal = kBars + 256;
    static constexpr uint32_t kAlloc = kTotal + 1024;  // manual 1024-B alignment
};

template <int STAGES>
struct FwdBars {
    uint64_t q_full;
    uint64_t k_full[STAGES];
    uint64_t k_empty[STAGES];
    uint64_t v_full[STAGES];
    uint64_t v_empty[STAGES];
    uint64_t s_full[2];
    uint64_t p_full;
    uint64_t o_done;
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

template <int D, bool BF16, int STAGES>
__global__ void __launch_bounds__(kThreads, 1)
    attn_fwd_kernel(const __grid_constant__ CUtensorMap tm_q,
                    const __grid_constant__ CUtensorMap tm_k,
                    const __grid_constant__ CUtensorMap tm_v,
                    const __grid_constant__ CUtensorMap tm_o, const __grid_constant__ FwdParams p) {
    using L = FwdSmem<D, STAGES>;
    constexpr uint32_t kTileBytes = L::kTileBytes;
    constexpr int kDBlocks = D / 64;  // 64-column (128-byte) blocks per row
    constexpr uint32_t kIdescS = ptx::idesc_f16(kBlockM, kBlockN, BF16, false);
    constexpr uint32_t kIdescO = ptx::idesc_f16(kBlockM, D, BF16, true);
    constexpr uint32_t kOCol = 256;  // TMEM columns: S0 [0,128), S1 [128,256), O [256, 256+D)

    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw_addr = ptx::smem_u32(smem_raw);
    uint8_t* smem = smem_raw + (((raw_addr + 1023u) & ~1023u) - raw_addr);
    const uint32_t sbase = ptx::smem_u32(smem);
    FwdBars<STAGES>* bars = reinterpret_cast<FwdBars<STAGES>*>(smem + L::kBars);
    volatile int* abort_flag = &bars->abort;

    const int tid = threadIdx.x;
    const int warp = tid >> 5;
    const int lane = tid & 31;

    // ---- work unit
    const int qt = p.causal ? (p.n_qtiles - 1 - (int)blockIdx.x) : (int)blockIdx.x;
    const int h = blockIdx.y;
    const int b = blockIdx.z;
    const int g = h / p.G;
    const int Lk = p.seqlens_k ? p.seqlens_k[b] : p.Nk;
    const int q0 = qt * kBlockM;
    const int i_last = min(q0 + kBlockM - 1, p.Nq - 1);
    int nt = (Lk + kBlockN - 1) / kBlockN;
    if (p.causal) {
        const int lim = i_last + Lk - p.Nq;
        nt = lim < 0 ? 0 : min(nt, lim / kBlockN + 1);
    }

    if (tid == 0) {
        ptx::mbar_init(&bars->q_full, 1);
        for (int s = 0; s < STAGES; ++s) {
            ptx::mbar_init(&bars->k_full[s], 1);
            ptx::mbar_init(&bars->k_empty[s], 1);
            ptx::mbar_init(&bars->v_full[s], 1);
            ptx::mbar_init(&bars->v_empty[s], 1);
        }
        ptx::mbar_init(&bars->s_full[0], 1);
        ptx::mbar_init(&bars->s_full[1], 1);
        ptx::mbar_init(&bars->p_full, 128);
        ptx::mbar_init(&bars->o_done, 1);
        ptx::mbar_init(&bars->drain, 1);
        bars->abort = 0;
        ptx::fence_barrier_init();
    }
    if (warp == 0 && lane == 0) {
        ptx::prefetch_tmap(&tm_q);
        ptx::prefetch_tmap(&tm_k);
        ptx::prefetch_tmap(&tm_v);
        ptx::prefetch_tmap(&tm_o);
    }
    if (warp == 1) {
        ptx::tmem_alloc<kTmemCols>(&bars->tmem_base);
        ptx::tmem_relinquish();
    }
    ptx::tc_fence_before();
    __syncthreads();
    ptx::tc_fence_after();
    const uint32_t tmem = bars->tmem_base;

    if (warp == 0) {
        // ================================================= TMA loader
        if (lane == 0 && nt > 0 && !p.inject) {
            int issued_k = 0, issued_v = 0;
            ptx::mbar_arrive_expect_tx(&bars->q_full, kTileBytes);
            for (int c = 0; c < kDBlocks; ++c)
                ptx::tma_load_4d(smem + L::kQ + c * (kBlockM * 128), &tm_q, &bars->q_full, c * 64,
                                 h, q0, b);
            for (int j = 0; j < nt; ++j) {
                const int st = j % STAGES;
                const uint32_t ph = (j / STAGES) & 1;
                if (!ptx::mbar_wait(&bars->k_empty[st], ph ^ 1, p.limit_ns, abort_flag)) {
                    record_error(p.err, kErrFwdBase + 1, &bars->abort);
                    break;
                }
                ptx::mbar_arrive_expect_tx(&bars->k_full[st], kTileBytes);
                for (int c = 0; c < kDBlocks; ++c)
                    ptx::tma_load_4d(smem + L::kK + st * kTileBytes + c * (kBlockN * 128), &tm_k,
                                     &bars->k_full[st], c * 64, g, j * kBlockN, b);
                ++issued_k;
                if (!ptx::mbar_wait(&bars->v_empty[st], ph ^ 1, p.limit_ns, abort_flag)) {
                    record_error(p.err, kErrFwdBase + 2, &bars->abort);
                    break;
                }
                ptx::mbar_arrive_expect_tx(&bars->v_full[st], kTileBytes);
                for (int c = 0; c < kDBlocks; ++c)
                    ptx::tma_load_4d(smem + L::kV + st * kTileBytes + c * (kBlockN * 128), &tm_v,
                                     &bars->v_full[st], c * 64, g, j * kBlockN, b);
                ++issued_v;
            }
            // Never leave the CTA with a copy in flight: wait (bounded, and
            // regardless of the abort flag) for the last phase of each
            // barrier that received a copy.
            int zero = 0;
            volatile int* no_abort = &zero;
            ptx::mbar_wait(&bars->q_full, 0, p.limit_ns, no_abort);
            for (int j = max(0, issued_k - STAGES); j < issued_k; ++j)
                ptx::mbar_wait(&bars->k_full[j % STAGES], (j / STAGES) & 1, p.limit_ns, no_abort);
            for (int j = max(0, issued_v - STAGES); j < issued_v; ++j)
                ptx::mbar_wait(&bars->v_full[j % STAGES], (j / STAGES) & 1, p.limit_ns, no_abort);
        }
    } else if (warp == 1) {
        // ================================================= MMA issuer
        if (lane == 0 && nt > 0) {
            bool ok = ptx::mbar_wait(&bars->q_full, 0, p.limit_ns, abort_flag);
            if (!ok) record_error(p.err, kErrFwdBase + 3, &bars->abort);
            ptx::tc_fence_after();
            const uint32_t q_addr = sbase + L::kQ;
            const uint32_t p_addr = sbase + L::kP;
            for (int j = 0; ok && j <= nt; ++j) {
                if (j < nt) {
                    const int st = j % STAGES;
                    const uint32_t ph = (j / STAGES) & 1;
                    if (!ptx::mbar_wait(&bars->k_full[st], ph, p.limit_ns, abort_flag)) {
                        record_error(p.err, kErrFwdBase + 4, &bars->abort);
                        ok = false;
                        break;
                    }
                    ptx::tc_fence_after();
                    const uint32_t k_addr = sbase + L::kK + st * kTileBytes;
                    const uint32_t d_s = tmem + (uint32_t)((j & 1) * kBlockN);
#pragma unroll
                    for (int kk = 0; kk < D / 16; ++kk) {
                        const uint32_t off = (kk >> 2) * (kBlockM * 128) + (kk & 3) * 32;
                        ptx::umma_ss(d_s, ptx::sdesc_sw128(q_addr + off, 16, 1024),
                                     ptx::sdesc_sw128(k_addr + off, 16, 1024), kIdescS, kk > 0);
                    }
                    ptx::umma_commit(&bars->s_full[j & 1]);
                    ptx::umma_commit(&bars->k_empty[st]);
                }
                if (j >= 1) {
                    const int jj = j - 1;
                    const int st = jj % STAGES;
                    const uint32_t ph = (jj / STAGES) & 1;
                    if (!ptx::mbar_wait(&bars->p_full, jj & 1, p.limit_ns, abort_flag) ||
                        !ptx::mbar_wait(&bars->v_full[st], ph, p.limit_ns, abort_flag)) {
                        record_error(p.err, kErrFwdBase + 5, &bars->abort);
                        ok = false;
                        break;
                    }
                    ptx::tc_fence_after();
                    const uint32_t v_addr = sbase + L::kV + st * kTileBytes;
#pragma unroll
                    for (int kk = 0; kk < kBlockN / 16; ++kk) {
                        const uint32_t a_off = (kk >> 2) * (kBlockM * 128) + (kk & 3) * 32;
                        ptx::umma_ss(tmem + kOCol, ptx::sdesc_sw128(p_addr + a_off, 16, 1024),
                                     ptx::sdesc_sw128(v_addr + kk * 16 * 128, kBlockN * 128, 1024),
                                     kIdescO, (jj > 0 || kk > 0) ? 1u : 0u);
                    }
                    ptx::umma_commit(&bars->o_done);
                    ptx::umma_commit(&bars->v_empty[st]);
                }
            }
            if (!ok) {
                // make sure no MMA is still running before TMEM is freed
                int zero = 0;
                volatile int* no_abort = &zero;
                ptx::umma_commit(&bars->drain);
                ptx::mbar_wait(&bars->drain, 0, p.limit_ns, no_abort);
            }
        }
    } else {
        // ================================================= softmax warpgroup
        const uint32_t quarter = (uint32_t)(warp & 3);
        const uint32_t row = quarter * 32u + (uint32_t)lane;
        const uint32_t lane_addr = (quarter * 32u) << 16;
        const int i = q0 + (int)row;
        int row_lim = Lk - 1;  // last visible key of this row
        if (p.causal) row_lim = min(row_lim, i + Lk - p.Nq);
        const float sl2 = p.scale_log2;
        float m_ref = -INFINITY;  // running reference max, scale*log2 units
        float l_sum = 0.f;        // running sum of exp2(s*sl2 - m_ref)
        bool ok = true;
        uint8_t* p_tile = smem + L::kP;

        for (int j = 0; j < nt; ++j) {
            if (!warp_wait(&bars->s_full[j & 1], (j >> 1) & 1, p.limit_ns, abort_flag)) {
                record_error(p.err, kErrFwdBase + 6, &bars->abort);
                ok = false;
                break;
            }
            ptx::tc_fence_after();
            float x[kBlockN];
            {
                uint32_t r[kBlockN / 32][32];
#pragma unroll
                for (int c = 0; c < kBlockN / 32; ++c)
                    ptx::tmem_ld32(tmem + lane_addr + (uint32_t)((j & 1) * kBlockN + c * 32), r[c]);
#pragma unroll
                for (int c = 0; c < kBlockN / 32; ++c) {
                    ptx::tmem_wait_ld_dep(r[c]);
#pragma unroll
                    for (int e = 0; e < 32; ++e) x[c * 32 + e] = __uint_as_float(r[c][e]);
                }
            }
            const int key0 = j * kBlockN;
            if (key0 + kBlockN - 1 > row_lim) {
#pragma unroll
                for (int c = 0; c < kBlockN; ++c)
                    if (key0 + c > row_lim) x[c] = -INFINITY;
            }
            float mx = x[0];
#pragma unroll
            for (int c = 1; c < kBlockN; ++c) mx = fmaxf(mx, x[c]);
            const float m_tile = mx * sl2;  // -inf stays -inf (sl2 > 0)
            float alpha = 1.f;
            bool rescale = false;
            if (m_tile > m_ref + kRescaleThreshold) {
                alpha = ptx::ex2_approx(m_ref - m_tile);  // 0 when m_ref = -inf
                rescale = (j > 0) && (m_ref != -INFINITY);
                m_ref = m_tile;
            }
            const float m_use = (m_ref == -INFINITY) ? 0.f : m_ref;
            float rowsum = 0.f;
            uint32_t pk[kBlockN / 2];
#pragma unroll
            for (int c = 0; c < kBlockN; c += 2) {
                const float p0 = ptx::ex2_approx(fmaf(x[c], sl2, -m_use));
                const float p1 = ptx::ex2_approx(fmaf(x[c + 1], sl2, -m_use));
                rowsum += p0 + p1;
                pk[c / 2] = ptx::pack2<BF16>(p0, p1);
            }
            l_sum = l_sum * alpha + rowsum;

            if (j > 0) {
                // PV_{j-1} must be complete before O is touched and before the
                // P buffer is overwritten
                if (!warp_wait(&bars->o_done, (j - 1) & 1, p.limit_ns, abort_flag)) {
                    record_error(p.err, kErrFwdBase + 7, &bars->abort);
                    ok = false;
                    break;
                }
                ptx::tc_fence_after();
                if (__any_sync(0xffffffffu, rescale)) {
                    const float a = rescale ? alpha : 1.f;
#pragma unroll
                    for (int c = 0; c < D / 32; ++c) {
                        uint32_t r[32];
                        const uint32_t ta = tmem + lane_addr + kOCol + (uint32_t)(c * 32);
                        ptx::tmem_ld32(ta, r);
                        ptx::tmem_wait_ld_dep(r);
#pragma unroll
                        for (int e = 0; e < 32; ++e)
                            r[e] = __float_as_uint(__uint_as_float(r[e]) * a);
                        ptx::tmem_st32(ta, r);
                    }
                    ptx::tmem_wait_st();
                }
            }
            // P row -> shared memory, K-major, 128-byte swizzle, two 64-key blocks
#pragma unroll
            for (int blk = 0; blk < 2; ++blk) {
#pragma unroll
                for (int ch = 0; ch < 8; ++ch) {
                    const int e = blk * 32 + ch * 4;
                    uint4 v4 = make_uint4(pk[e], pk[e + 1], pk[e + 2], pk[e + 3]);
                    *reinterpret_cast<uint4*>(p_tile + blk * (kBlockM * 128) +
                                              sw128_offset(row, ch)) = v4;
                }
            }
            if (p.seqlens_k != nullptr && key0 + kBlockN > Lk) {
                // keys behind the real length: zero their V rows so that a
                // non-finite value stored there cannot reach O through 0 * NaN
                const int st = j % STAGES;
                if (!warp_wait(&bars->v_full[st], (j / STAGES) & 1, p.limit_ns, abort_flag)) {
                    record_error(p.err, kErrFwdBase + 8, &bars->abort);
                    ok = false;
                    break;
                }
                if (key0 + (int)row >= Lk) {
                    uint8_t* vt = smem + L::kV + st * kTileBytes;
#pragma unroll
                    for (int c = 0; c < kDBlocks; ++c)
#pragma unroll
                        for (int ch = 0; ch < 8; ++ch)
                            *reinterpret_cast<uint4*>(vt + c * (kBlockN * 128) + row * 128 +
                                                      ch * 16) = make_uint4(0, 0, 0, 0);
                }
            }
            ptx::fence_proxy_async_smem();
            ptx::tc_fence_before();
            ptx::mbar_arrive(&bars->p_full);
        }

        // ---- epilogue: O / l -> bf16/fp16 -> swizzled staging -> TMA store
        if (ok && nt > 0) {
            if (!warp_wait(&bars->o_done, (nt - 1) & 1, p.limit_ns, abort_flag)) {
                record_error(p.err, kErrFwdBase + 9, &bars->abort);
                ok = false;
            }
            ptx::tc_fence_after();
        }
        const bool have = ok && nt > 0 && l_sum > 0.f;
        const float inv_l = have ? 1.f / l_sum : 0.f;
        uint8_t* stage = smem + L::kP;  // P buffer is free once the last PV is done
#pragma unroll
        for (int c = 0; c < D / 32; ++c) {
            uint32_t r[32];
            if (ok && nt > 0) {
                ptx::tmem_ld32(tmem + lane_addr + kOCol + (uint32_t)(c * 32), r);
                ptx::tmem_wait_ld_dep(r);
            } else {
#pragma unroll
                for (int e = 0; e < 32; ++e) r[e] = 0u;
            }
            uint32_t o2[16];
#pragma unroll
            for (int e = 0; e < 16; ++e)
                o2[e] = ptx::pack2<BF16>(__uint_as_float(r[2 * e]) * inv_l,
                                         __uint_as_float(r[2 * e + 1]) * inv_l);
            // 32 columns = 4 chunks of 16 bytes in block c/2, chunks (c%2)*4..+3
#pragma unroll
            for (int q4 = 0; q4 < 4; ++q4) {
                const uint32_t ch = (uint32_t)((c & 1) * 4 + q4);
                *reinterpret_cast<uint4*>(stage + (c >> 1) * (kBlockM * 128) +
                                          sw128_offset(row, ch)) =
                    make_uint4(o2[q4 * 4], o2[q4 * 4 + 1], o2[q4 * 4 + 2], o2[q4 * 4 + 3]);
            }
        }
        ptx::fence_proxy_async_smem();
        ptx::named_barrier_sync(1, 128);
        if (warp == 2 && lane == 0) {
            for (int c = 0; c < kDBlocks; ++c)
                ptx::tma_store_4d(&tm_o, stage + c * (kBlockM * 128), c * 64, h, q0, b);
            ptx::bulk_commit_group();
            ptx::bulk_wait_group_read0();
        }
        if (i < p.Nq) {
            const float lse = have ? (m_ref + ptx::lg2_approx(l_sum)) * 0.69314718055994531f
                                   : -INFINITY;
            p.lse[((size_t)b * p.Hq + h) * p.Nq + i] = lse;
        }
    }

    ptx::tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        __syncwarp();
        ptx::tc_fence_after();
        ptx::tmem_dealloc<kTmemCols>(tmem);
    }
}

template <int D, bool BF16, int STAGES>
cudaError_t launch_fwd_t(const FwdMaps& maps, const FwdParams& p, cudaStream_t stream) {
    using L = FwdSmem<D, STAGES>;
    static_assert(L::kAlloc <= 227 * 1024, "shared memory budget");
    auto kern = attn_fwd_kernel<D, BF16, STAGES>;
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
        return bf16 ? launch_fwd_t<64, true, 3>(maps, p, stream)
                    : launch_fwd_t<64, false, 3>(maps, p, stream);
    }
    return bf16 ? launch_fwd_t<128, true, 2>(maps, p, stream)
                : launch_fwd_t<128, false, 2>(maps, p, stream);
}

}  // namespace attn
