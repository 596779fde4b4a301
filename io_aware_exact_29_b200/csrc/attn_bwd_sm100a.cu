// attn_bwd_sm100a.cu -- gradients of exact attention (dQ, dK, dV) on tcgen05
// tensor cores.
//
// The pages report the training speed-ups of the method (effectstory.com
// article, "訓練性能量化提升" table) but print no backward algorithm; the
// plainest reading keeps the forward's rule of never writing the N×N score
// matrix to HBM: every score tile is recomputed on chip from Q, K and the
// forward's log-sum-exp (ai6s.net article, section "FlashAttention 拆的不是
// 算法，是数据流": tiles of Q, K, V on chip, only small per-row statistics kept).
// For one (b, h) and the row softmax P of the forward:
//
//   D_i   = sum_t dO[i][t] * O[i][t]                    (= sum_j P_ij dP_ij)
//   P_ij  = 2^(S_ij * scale * log2 e - LSE_i * log2 e)   (masked entries: 0)
//   dP_ij = dO_i . V_j
//   dS_ij = P_ij * (dP_ij - D_i)
//   dV_j  = sum_i P_ij dO_i      dK_j = scale * sum_i dS_ij Q_i
//   dQ_i  = scale * sum_j dS_ij K_j
//
// Three kernels, all in one stream:
//   attn_bwd_pre_kernel   D and LSE * log2 e per query row (HBM-bound)
//   attn_bwd_dkdv_kernel  one CTA per 128-key tile of a kv head; loops over
//                         the query tiles of every query head of its group,
//                         keeping dK and dV in tensor memory (no atomics)
//   attn_bwd_dq_kernel    one CTA per 128-row query tile; loops over the key
//                         tiles, keeping dQ in tensor memory
// The score tile is recomputed in both gradient kernels (S and dP twice):
// seven tile products instead of five, in exchange for no cross-CTA
// reduction and a deterministic result.
//
// dK/dV kernel, per query tile (M = 128 keys = TMEM lanes):
//   Sᵀ = K Qᵀ -> TMEM [0,128)        dPᵀ = V dOᵀ -> TMEM [128,256)
//   compute warps: Pᵀ, dSᵀ in bf16/fp16 over the first 64 columns of each
//   dV += Pᵀ dO  (A = Pᵀ from TMEM, B = dO, MN-major)  -> TMEM [256, 256+D)
//   dK += dSᵀ Q  (A = dSᵀ from TMEM, B = Q, MN-major)  -> TMEM [256+D, 256+2D)
// dQ kernel, per key tile (M = 128 query rows):
//   S = Q Kᵀ -> [0,128)   dP = dO Vᵀ -> [128,256)   dS over S's first 64 columns
//   dQ += dS K  (A = dS from TMEM, B = K, MN-major)  -> [256, 256+D)
// MMAs from one thread run in issue order, so the next tile's S/dP products
// overwrite P and dS only after the products that read them.
#include <algorithm>

#include "attn_internal.h"
#include "ptx.cuh"

namespace attn {
namespace {

constexpr int kBlock = 128;  // rows of a Q tile and of a K/V tile
// warps 0-15 compute: rows 32*(w%4) .. +31 (their TMEM lanes), columns
// 32*(w/4) .. +31 of the 128-column score tile; warp 16 loader, warp 17 MMA
constexpr int kComputeWarps = 16;
constexpr int kThreads = 32 * (kComputeWarps + 2);
constexpr int kLoaderWarp = kComputeWarps, kMmaWarp = kComputeWarps + 1;
constexpr uint32_t kTmemCols = 512;
constexpr float kLog2e = 1.4426950408889634f;

__device__ __forceinline__ void record_error(unsigned* err, unsigned code, int* abort_flag) {
    atomicCAS(err, 0u, code);
    *reinterpret_cast<volatile int*>(abort_flag) = 1;
}

__device__ __forceinline__ bool warp_wait(uint64_t* bar, uint32_t parity, uint64_t limit_ns,
                                          volatile int* abort_flag) {
    const bool ok = ptx::mbar_wait(bar, parity, limit_ns, abort_flag);
    return __all_sync(0xffffffffu, ok);
}

// kPart output columns of one row as packed 16-bit values (16-byte stores).
template <int kPart, bool BF16>
__device__ __forceinline__ void store_row(void* out, size_t elem, const uint32_t* v, float sc) {
    uint4* dst = reinterpret_cast<uint4*>(static_cast<uint16_t*>(out) + elem);
#pragma unroll
    for (int e = 0; e < kPart; e += 8)
        dst[e / 8] = make_uint4(
            ptx::pack2<BF16>(__uint_as_float(v[e]) * sc, __uint_as_float(v[e + 1]) * sc),
            ptx::pack2<BF16>(__uint_as_float(v[e + 2]) * sc, __uint_as_float(v[e + 3]) * sc),
            ptx::pack2<BF16>(__uint_as_float(v[e + 4]) * sc, __uint_as_float(v[e + 5]) * sc),
            ptx::pack2<BF16>(__uint_as_float(v[e + 6]) * sc, __uint_as_float(v[e + 7]) * sc));
}

// kPart columns of a row of tensor memory to the output, scaled.  `zero`
// (the same for the whole warp) writes zeros without touching tensor memory;
// `store` is this lane's own predicate.  The tensor-memory loads are
// warp-collective, so every lane runs them and only the stores are
// predicated.
template <int kPart, bool BF16>
__device__ __forceinline__ void tmem_row_out(uint32_t taddr, void* out, size_t elem, float sc,
                                             bool zero, bool store) {
    uint32_t r[kPart];
    if (!zero) {
        if constexpr (kPart == 32) {
            ptx::tmem_ld32(taddr, r);
            ptx::tmem_wait_ld_dep(r);
        } else {
            ptx::tmem_ld16(taddr, r);
            ptx::tmem_wait_ld_dep16(r);
        }
    } else {
#pragma unroll
        for (int e = 0; e < kPart; ++e) r[e] = 0u;
    }
    if (store) store_row<kPart, BF16>(out, elem, r, sc);
}

// ------------------------------------------------------------------ D, LSE
// D[b,h,i] = sum_t dO[b,i,h,t] * O[b,i,h,t]; lse2 = LSE * log2 e (+inf for
// a row with no visible key, so that its P is exactly 0).  d / 8 threads per
// row, 16-byte loads; rows [B, Nq, Hq] are contiguous in O and dO.
template <int D, bool BF16>
__global__ void __launch_bounds__(256) attn_bwd_pre_kernel(const __grid_constant__ BwdParams p) {
    constexpr int kTpr = D / 8;            // threads per row
    constexpr int kRowsPerWarp = 32 / kTpr;
    const long rows = (long)p.B * p.Nq * p.Hq;
    const int lane = threadIdx.x & 31;
    const int sub = lane % kTpr;
    const long warp0 = ((long)blockIdx.x * blockDim.x + threadIdx.x) / 32;
    const long n_warps = (long)gridDim.x * blockDim.x / 32;
    // every lane of a warp runs the same iterations (the shuffles need all 32)
    for (long base = warp0 * kRowsPerWarp; base < rows; base += n_warps * kRowsPerWarp) {
        const long r = base + lane / kTpr;
        const bool valid = r < rows;
        float acc = 0.f;
        if (valid) {
            const uint4 a = reinterpret_cast<const uint4*>(p.o)[r * kTpr + sub];
            const uint4 c = reinterpret_cast<const uint4*>(p.dout)[r * kTpr + sub];
            const uint32_t av[4] = {a.x, a.y, a.z, a.w};
            const uint32_t cv[4] = {c.x, c.y, c.z, c.w};
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                const float2 x = ptx::unpack2<BF16>(av[u]);
                const float2 y = ptx::unpack2<BF16>(cv[u]);
                acc = fmaf(x.x, y.x, acc);
                acc = fmaf(x.y, y.y, acc);
            }
        }
#pragma unroll
        for (int o = kTpr / 2; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
        if (valid && sub == 0) {
            const int h = (int)(r % p.Hq);
            const long bi = r / p.Hq;
            const int i = (int)(bi % p.Nq);
            const int b = (int)(bi / p.Nq);
            const size_t idx = ((size_t)b * p.Hq + h) * p.Nq + i;
            const float l = p.lse[idx];
            p.dsum[idx] = acc;
            p.lse2[idx] = l == -INFINITY ? INFINITY : l * kLog2e;
        }
    }
}

// ------------------------------------------------------------------ dK, dV
template <int D, int QST>
struct DkdvSmem {
    static constexpr uint32_t kTile = kBlock * D * 2;
    static constexpr uint32_t kK = 0;
    static constexpr uint32_t kV = kK + kTile;
    static constexpr uint32_t kQ = kV + kTile;             // QST stages
    static constexpr uint32_t kDO = kQ + QST * kTile;      // QST stages
    static constexpr uint32_t kLse = kDO + QST * kTile;    // QST x 128 fp32: -LSE * log2 e
    static constexpr uint32_t kDs = kLse + QST * 128 * 4;  // QST x 128 fp32: -D
    static constexpr uint32_t kBars = kDs + QST * 128 * 4;
    static constexpr uint32_t kAlloc = kBars + 256 + 1024;
};

template <int QST>
struct DkdvBars {
    uint64_t kv_full;
    uint64_t q_full[QST];
    uint64_t q_empty[QST];
    uint64_t s_full[2];  // per query half
    uint64_t p_full[2];
    uint64_t o_done;
    uint64_t drain;
    uint32_t tmem_base;
    int abort;
};

template <int D, bool BF16, int QST, bool kSparse>
__global__ void __launch_bounds__(kThreads, 1)
    attn_bwd_dkdv_kernel(const __grid_constant__ CUtensorMap tm_q,
                         const __grid_constant__ CUtensorMap tm_k,
                         const __grid_constant__ CUtensorMap tm_v,
                         const __grid_constant__ CUtensorMap tm_do,
                         const __grid_constant__ BwdParams p) {
    using L = DkdvSmem<D, QST>;
    constexpr uint32_t kTile = L::kTile;
    constexpr int kDBlocks = D / 64;
    constexpr uint32_t kBlockBytes = kBlock * 128;
    constexpr uint32_t kIdescS = ptx::idesc_f16(kBlock, 64, BF16, false);  // half tiles
    constexpr uint32_t kIdescO = ptx::idesc_f16(kBlock, D, BF16, true);
    constexpr uint32_t kColDP = 128, kColDV = 256, kColDK = 256 + D;
    static_assert(sizeof(DkdvBars<QST>) <= 256, "barrier block");

    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw_addr = ptx::smem_u32(smem_raw);
    uint8_t* smem = smem_raw + (((raw_addr + 1023u) & ~1023u) - raw_addr);
    const uint32_t sbase = ptx::smem_u32(smem);
    DkdvBars<QST>* bars = reinterpret_cast<DkdvBars<QST>*>(smem + L::kBars);
    volatile int* abort_flag = &bars->abort;

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    // causal: a 1-D grid in bands of (b, kv head) pairs, the first key tiles
    // (seen by the most query tiles) first; otherwise (key tiles, Hkv, B)
    int kt, g, b;
    if (p.band_kv > 0) {
        int pair, rank;
        band_unit(blockIdx.x, p.band_kv, p.B * p.Hkv, (p.Nk + kBlock - 1) / kBlock, pair, rank);
        kt = rank;
        g = pair % p.Hkv;
        b = pair / p.Hkv;
    } else {
        kt = blockIdx.x;
        g = blockIdx.y;
        b = blockIdx.z;
    }
    const int k0 = kt * kBlock;
    const int Lk = p.seqlens_k ? p.seqlens_k[b] : p.Nk;
    const int off = Lk - p.Nq;  // key j visible to query i iff j <= i + off (causal)
    // query tiles that see at least one key of this tile
    int qt_first = 0;
    if (p.causal) qt_first = max(0, k0 - off) / kBlock;
    const int n_qt = (p.Nq + kBlock - 1) / kBlock;
    int qt_end = n_qt;
    if (p.window_left >= 0) {
        // the last query that sees a key of this tile: i <= key - off + window_left
        const int i_max = min(Lk - 1, k0 + kBlock - 1) - off + p.window_left;
        qt_end = i_max < 0 ? 0 : min(n_qt, i_max / kBlock + 1);
    }
    const int nqs = (k0 < Lk) ? max(0, qt_end - qt_first) : 0;
    const int nsteps_all = p.G * nqs;
    // step sa = (query head g*G + sa / nqs, query tile qt_first + sa % nqs);
    // with a block mask only the steps whose entry for this key tile is set
    // take part, and stages and phases count those
    auto step_on = [&](int sa) -> bool {
        if constexpr (kSparse) {
            const long long hq = g * p.G + sa / nqs;
            const long long qt = qt_first + sa % nqs;
            return __ldg(p.bmask.m + (long long)b * p.bmask.sb + hq * p.bmask.sh +
                         qt * p.bmask.srow + kt) != 0;
        }
        return true;
    };
    // the step after sa that takes part (sa = -1: the first)
    auto next_step = [&](int sa) -> int {
        if constexpr (kSparse) {
            do {
                ++sa;
            } while (sa < nsteps_all - 1 && !step_on(sa));
            return sa;
        } else {
            return sa + 1;
        }
    };
    int nsteps = nsteps_all;
    if constexpr (kSparse) {
        int c = 0;
        for (int base = 0; base < nsteps_all; base += 32) {
            const int sa = base + lane;
            c += __popc(__ballot_sync(0xffffffffu, sa < nsteps_all && step_on(sa)));
        }
        nsteps = c;
    }

    if (tid == 0) {
        ptx::mbar_init(&bars->kv_full, 1);
        for (int s = 0; s < QST; ++s) {
            ptx::mbar_init(&bars->q_full[s], 1);
            ptx::mbar_init(&bars->q_empty[s], 1);
        }
        for (int hh = 0; hh < 2; ++hh) {
            ptx::mbar_init(&bars->s_full[hh], 1);
            ptx::mbar_init(&bars->p_full[hh], kComputeWarps / 2);
        }
        ptx::mbar_init(&bars->o_done, 1);
        ptx::mbar_init(&bars->drain, 1);
        bars->abort = 0;
        ptx::fence_barrier_init();
    }
    if (warp == kLoaderWarp && lane == 0) {
        ptx::prefetch_tmap(&tm_q);
        ptx::prefetch_tmap(&tm_k);
        ptx::prefetch_tmap(&tm_v);
        ptx::prefetch_tmap(&tm_do);
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
        // ================================================= loader
        if (nsteps > 0) {
            if (lane == 0) {
                ptx::mbar_arrive_expect_tx(&bars->kv_full, 2 * kTile);
                for (int c = 0; c < kDBlocks; ++c) {
                    ptx::tma_load_4d(smem + L::kK + c * kBlockBytes, &tm_k, &bars->kv_full,
                                     c * 64, g, k0, b);
                    ptx::tma_load_4d(smem + L::kV + c * kBlockBytes, &tm_v, &bars->kv_full,
                                     c * 64, g, k0, b);
                }
            }
            __syncwarp();
            int issued = 0;
            int sa = -1;
            for (int s = 0; s < nsteps; ++s) {
                sa = next_step(sa);
                const int st = s % QST;
                const int h = g * p.G + sa / nqs;
                const int i0 = (qt_first + sa % nqs) * kBlock;
                if (!warp_wait(&bars->q_empty[st], ((s / QST) & 1) ^ 1, p.limit_ns, abort_flag)) {
                    record_error(p.err, kErrBwdBase + 1, &bars->abort);
                    break;
                }
                // per-row statistics of this query tile
                float* lse_s = reinterpret_cast<float*>(smem + L::kLse) + st * 128;
                float* ds_s = reinterpret_cast<float*>(smem + L::kDs) + st * 128;
                const size_t base = ((size_t)b * p.Hq + h) * p.Nq;
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                    const int i = i0 + lane * 4 + u;
                    // negated, so that the compute warps add them with f32x2 FMAs
                    lse_s[lane * 4 + u] = i < p.Nq ? -p.lse2[base + i] : -INFINITY;
                    ds_s[lane * 4 + u] = i < p.Nq ? -p.dsum[base + i] : 0.f;
                }
                __syncwarp();
                if (lane == 0) {
                    ptx::mbar_arrive_expect_tx(&bars->q_full[st], 2 * kTile);
                    for (int c = 0; c < kDBlocks; ++c) {
                        ptx::tma_load_4d(smem + L::kQ + st * kTile + c * kBlockBytes, &tm_q,
                                         &bars->q_full[st], c * 64, h, i0, b);
                        ptx::tma_load_4d(smem + L::kDO + st * kTile + c * kBlockBytes, &tm_do,
                                         &bars->q_full[st], c * 64, h, i0, b);
                    }
                }
                __syncwarp();
                ++issued;
            }
            int zero = 0;
            volatile int* no_abort = &zero;
            ptx::mbar_wait(&bars->kv_full, 0, p.limit_ns, no_abort);
            for (int s = max(0, issued - QST); s < issued; ++s)
                ptx::mbar_wait(&bars->q_full[s % QST], (s / QST) & 1, p.limit_ns, no_abort);
        }
    } else if (warp == kMmaWarp) {
        // ================================================= MMA issuer
        if (nsteps > 0) {
            bool ok = true;
            bool issued = false;
            auto wait_or_fail = [&](uint64_t* bar, uint32_t parity, unsigned site) {
                if (!warp_wait(bar, parity, p.limit_ns, abort_flag)) {
                    record_error(p.err, kErrBwdBase + site, &bars->abort);
                    ok = false;
                }
                return ok;
            };
            const uint64_t k_desc = ptx::sdesc_sw128(sbase + L::kK, 16, 1024);
            const uint64_t v_desc = ptx::sdesc_sw128(sbase + L::kV, 16, 1024);
            constexpr uint64_t kTileUnits = kTile >> 4;
            constexpr uint64_t kHalfUnits = (64 * 128) >> 4;  // 64 rows into a 128-row tile
            // S^T and dP^T of query half h (queries 64h .. 64h+63) of step s
            auto issue_sdp = [&](int s, int h) {
                const int st = s % QST;
                const uint64_t q_k = ptx::sdesc_sw128(sbase + L::kQ, 16, 1024) + st * kTileUnits +
                                     h * kHalfUnits;
                const uint64_t do_k = ptx::sdesc_sw128(sbase + L::kDO, 16, 1024) +
                                      st * kTileUnits + h * kHalfUnits;
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk) {
                    const uint64_t o16 = (uint64_t)(((kk >> 2) * kBlockBytes + (kk & 3) * 32) >> 4);
                    ptx::umma_ss_elect(tmem + 64 * h, k_desc + o16, q_k + o16, kIdescS, kk > 0);
                }
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk) {
                    const uint64_t o16 = (uint64_t)(((kk >> 2) * kBlockBytes + (kk & 3) * 32) >> 4);
                    ptx::umma_ss_elect(tmem + kColDP + 64 * h, v_desc + o16, do_k + o16, kIdescS,
                                       kk > 0);
                }
                ptx::umma_commit_elect(&bars->s_full[h]);
            };
            // dV += P_h^T dO_h and dK += dS_h^T Q_h (K = the 64 queries of half h)
            auto issue_dvk = [&](int s, int h) {
                const int st = s % QST;
                const uint64_t q_mn = ptx::sdesc_sw128(sbase + L::kQ + st * kTile, kBlockBytes, 1024);
                const uint64_t do_mn =
                    ptx::sdesc_sw128(sbase + L::kDO + st * kTile, kBlockBytes, 1024);
#pragma unroll
                for (int kk = 4 * h; kk < 4 * h + 4; ++kk) {
                    const uint64_t r16 = (uint64_t)((kk * 16 * 128) >> 4);
                    const uint32_t acc = (s > 0 || kk > 0) ? 1u : 0u;
                    // queries 16kk..16kk+15 of P and dS: part kk/2 keeps its
                    // 32 columns packed in the first 16 of its own 32
                    const uint32_t a_col = (uint32_t)(32 * (kk >> 1) + 8 * (kk & 1));
                    ptx::umma_ts_elect(tmem + kColDV, tmem + a_col, do_mn + r16, kIdescO, acc);
                    ptx::umma_ts_elect(tmem + kColDK, tmem + kColDP + a_col, q_mn + r16, kIdescO,
                                       acc);
                }
            };
            // Order per step s: dVK_0(s), SdP_0(s+1), dVK_1(s), SdP_1(s+1): the
            // products of one half run while the other half's warps compute.
            if (wait_or_fail(&bars->kv_full, 0, 2) && wait_or_fail(&bars->q_full[0], 0, 3)) {
                ptx::tc_fence_after();
                issue_sdp(0, 0);
                issue_sdp(0, 1);
                __syncwarp();
                issued = true;
                for (int s = 0; s < nsteps; ++s) {
                    if (!wait_or_fail(&bars->p_full[0], s & 1, 4)) break;
                    ptx::tc_fence_after();
                    issue_dvk(s, 0);
                    if (s + 1 < nsteps) {
                        const int s1 = s + 1;
                        if (!wait_or_fail(&bars->q_full[s1 % QST], (s1 / QST) & 1, 3)) break;
                        ptx::tc_fence_after();
                        issue_sdp(s1, 0);
                    }
                    __syncwarp();
                    if (!wait_or_fail(&bars->p_full[1], s & 1, 4)) break;
                    ptx::tc_fence_after();
                    issue_dvk(s, 1);
                    ptx::umma_commit_elect(&bars->q_empty[s % QST]);
                    if (s + 1 < nsteps) issue_sdp(s + 1, 1);
                    if (s == nsteps - 1) ptx::umma_commit_elect(&bars->o_done);
                    __syncwarp();
                }
            }
            if (!ok && issued) {
                int zero = 0;
                volatile int* no_abort = &zero;
                ptx::umma_commit_elect(&bars->drain);
                __syncwarp();
                ptx::mbar_wait(&bars->drain, 0, p.limit_ns, no_abort);
            }
        }
    } else {
        // ================================================= compute warps
        constexpr int kPartD = D / 4;
        const uint32_t quarter = (uint32_t)(warp & 3);
        const int part = warp >> 2;                   // query columns 32*part .. +31
        const int half = part >> 1;                   // query half of those columns
        const uint32_t row = quarter * 32u + (uint32_t)lane;  // key row of the tile
        const int kr = k0 + (int)row;
        const uint32_t lane_addr = (quarter * 32u) << 16;
        const uint32_t t_s = tmem + lane_addr + (uint32_t)(32 * part);
        const uint32_t t_dp = tmem + lane_addr + kColDP + (uint32_t)(32 * part);
        const float sl2 = p.scale_log2;
        const bool key_ok = kr < Lk;
        bool ok = true;
        int sa = -1;
        for (int s = 0; s < nsteps; ++s) {
            sa = next_step(sa);
            const int st = s % QST;
            const int i0 = (qt_first + sa % nqs) * kBlock;
            if (!warp_wait(&bars->s_full[half], s & 1, p.limit_ns, abort_flag)) {
                record_error(p.err, kErrBwdBase + 5, &bars->abort);
                ok = false;
                break;
            }
            ptx::tc_fence_after();
            const int qc0 = 32 * part;
            const float* lse_s = reinterpret_cast<const float*>(smem + L::kLse) + st * 128 + qc0;
            const float* ds_s = reinterpret_cast<const float*>(smem + L::kDs) + st * 128 + qc0;
            uint32_t sv[32], dv[32];
            ptx::tmem_ld32(t_s, sv);
            ptx::tmem_ld32(t_dp, dv);
            // every (key, query) pair of this thread's 32 columns visible?
            const bool full = key_ok && i0 + qc0 + 32 <= p.Nq && (!p.causal || kr <= i0 + qc0 + off) &&
                              (p.window_left < 0 || kr >= i0 + qc0 + 31 + off - p.window_left);
            const bool masked = __any_sync(0xffffffffu, !full);
            ptx::tmem_wait_ld_dep(sv);
            ptx::tmem_wait_ld_dep(dv);
            uint32_t pk_p[16], pk_ds[16];
            const uint64_t sl2_2 = ptx::f2_pack(sl2, sl2);
#pragma unroll
            for (int e4 = 0; e4 < 32; e4 += 4) {
                // 16-byte loads of four queries' -LSE*log2e and -D
                const float4 nl = *reinterpret_cast<const float4*>(lse_s + e4);
                const float4 nd = *reinterpret_cast<const float4*>(ds_s + e4);
#pragma unroll
                for (int e2 = 0; e2 < 4; e2 += 2) {
                    const int e = e4 + e2;
                    const uint64_t nl2 = e2 == 0 ? ptx::f2_pack(nl.x, nl.y) : ptx::f2_pack(nl.z, nl.w);
                    const uint64_t nd2 = e2 == 0 ? ptx::f2_pack(nd.x, nd.y) : ptx::f2_pack(nd.z, nd.w);
                    float t0, t1;
                    ptx::f2_unpack(ptx::f2_fma(ptx::f2_pack(__uint_as_float(sv[e]),
                                                            __uint_as_float(sv[e + 1])),
                                               sl2_2, nl2), t0, t1);
                    float p0 = ptx::ex2_approx(t0), p1 = ptx::ex2_approx(t1);
                    const uint64_t d2 = ptx::f2_add(
                        ptx::f2_pack(__uint_as_float(dv[e]), __uint_as_float(dv[e + 1])), nd2);
                    float ds0, ds1;
                    ptx::f2_unpack(ptx::f2_mul(ptx::f2_pack(p0, p1), d2), ds0, ds1);
                    if (masked) {
                        const int qi = i0 + qc0 + e;
                        const bool w0 = p.window_left < 0 || kr >= qi + off - p.window_left;
                        const bool w1 = p.window_left < 0 || kr >= qi + 1 + off - p.window_left;
                        const bool v0 = key_ok && qi < p.Nq && (!p.causal || kr <= qi + off) && w0;
                        const bool v1 =
                            key_ok && qi + 1 < p.Nq && (!p.causal || kr <= qi + 1 + off) && w1;
                        p0 = v0 ? p0 : 0.f;
                        ds0 = v0 ? ds0 : 0.f;
                        p1 = v1 ? p1 : 0.f;
                        ds1 = v1 ? ds1 : 0.f;
                    }
                    pk_p[e / 2] = ptx::pack2<BF16>(p0, p1);
                    pk_ds[e / 2] = ptx::pack2<BF16>(ds0, ds1);
                }
            }
            // P and dS of these 32 queries go to the first 16 of this warp's
            // own 32 columns (no other warp reads them as scores)
            ptx::tmem_st16(t_s, pk_p);
            ptx::tmem_st16(t_dp, pk_ds);
            ptx::tmem_wait_st();
            ptx::tc_fence_before();
            __syncwarp();
            if (lane == 0) ptx::mbar_arrive(&bars->p_full[half]);
        }
        if (ok && nsteps > 0) {
            if (!warp_wait(&bars->o_done, 0, p.limit_ns, abort_flag)) {
                record_error(p.err, kErrBwdBase + 6, &bars->abort);
                ok = false;
            }
            ptx::tc_fence_after();
        }
        // dV, dK of this key row, columns part * D/4 .. +D/4 (zero behind the
        // real length or on an error)
        {
            const bool store = kr < p.Nk;
            const size_t elem =
                (((size_t)b * p.Nk + (store ? kr : 0)) * p.Hkv + g) * D + part * kPartD;
            const bool zero = !(__all_sync(0xffffffffu, ok) && nsteps > 0);
            const uint32_t col = (uint32_t)(part * kPartD);
            tmem_row_out<kPartD, BF16>(tmem + lane_addr + kColDV + col, p.dv, elem, 1.f, zero,
                                       store);
            tmem_row_out<kPartD, BF16>(tmem + lane_addr + kColDK + col, p.dk, elem, p.scale, zero,
                                       store);
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

// ------------------------------------------------------------------ dQ
template <int D, int KST>
struct DqSmem {
    static constexpr uint32_t kTile = kBlock * D * 2;
    static constexpr uint32_t kQ = 0;
    static constexpr uint32_t kDO = kQ + kTile;
    static constexpr uint32_t kK = kDO + kTile;      // KST stages
    static constexpr uint32_t kV = kK + KST * kTile;  // KST stages
    static constexpr uint32_t kBars = kV + KST * kTile;
    static constexpr uint32_t kAlloc = kBars + 256 + 1024;
};

template <int KST>
struct DqBars {
    uint64_t q_full;
    uint64_t k_full[KST];
    uint64_t k_empty[KST];
    uint64_t v_full[KST];
    uint64_t v_empty[KST];
    uint64_t s_full[2];  // per key half
    uint64_t p_full[2];
    uint64_t o_done;
    uint64_t drain;
    uint32_t tmem_base;
    int abort;
};

__device__ __forceinline__ int dq_tiles(int q_first, int Nq, int Lk, int causal) {
    if (q_first >= Nq || Lk <= 0) return 0;
    int nt = (Lk + kBlock - 1) / kBlock;
    if (causal) {
        const int i_last = min(q_first + kBlock - 1, Nq - 1);
        const int lim = i_last + Lk - Nq;  // last key visible to the tile's last row
        nt = lim < 0 ? 0 : min(nt, lim / kBlock + 1);
    }
    return nt;
}

template <int D, bool BF16, int KST, bool kSparse>
__global__ void __launch_bounds__(kThreads, 1)
    attn_bwd_dq_kernel(const __grid_constant__ CUtensorMap tm_q,
                       const __grid_constant__ CUtensorMap tm_k,
                       const __grid_constant__ CUtensorMap tm_v,
                       const __grid_constant__ CUtensorMap tm_do,
                       const __grid_constant__ BwdParams p) {
    using L = DqSmem<D, KST>;
    constexpr uint32_t kTile = L::kTile;
    constexpr int kDBlocks = D / 64;
    constexpr uint32_t kBlockBytes = kBlock * 128;
    constexpr uint32_t kIdescS = ptx::idesc_f16(kBlock, 64, BF16, false);  // half tiles
    constexpr uint32_t kIdescO = ptx::idesc_f16(kBlock, D, BF16, true);
    constexpr uint32_t kColDP = 128, kColDQ = 256;
    static_assert(sizeof(DqBars<KST>) <= 256, "barrier block");

    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw_addr = ptx::smem_u32(smem_raw);
    uint8_t* smem = smem_raw + (((raw_addr + 1023u) & ~1023u) - raw_addr);
    const uint32_t sbase = ptx::smem_u32(smem);
    DqBars<KST>* bars = reinterpret_cast<DqBars<KST>*>(smem + L::kBars);
    volatile int* abort_flag = &bars->abort;

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    // causal: a 1-D grid in bands of (b, q head) pairs, the last query tiles
    // (which see the most keys) first; otherwise (query tiles, Hq, B)
    const int n_qt = (p.Nq + kBlock - 1) / kBlock;
    int qt, h, b;
    if (p.band_q > 0) {
        int pair, rank;
        band_unit(blockIdx.x, p.band_q, p.B * p.Hq, n_qt, pair, rank);
        qt = n_qt - 1 - rank;
        h = pair % p.Hq;
        b = pair / p.Hq;
    } else {
        qt = blockIdx.x;
        h = blockIdx.y;
        b = blockIdx.z;
    }
    const int i0 = qt * kBlock;
    const int g = h / p.G;
    const int Lk = p.seqlens_k ? p.seqlens_k[b] : p.Nk;
    const int off = Lk - p.Nq;
    // key tiles j0 .. j0 + nt - 1 (the sliding window's first tile is j0);
    // stages and phases count from 0
    const int j0 = p.window_left >= 0 ? max(0, i0 + off - p.window_left) / kBlock : 0;
    const int nt_all = max(0, dq_tiles(i0, p.Nq, Lk, p.causal) - j0);
    // with a block mask only the key tiles whose entry for this query tile
    // is set take part, and stages and phases count those
    const unsigned char* mrow = nullptr;
    if constexpr (kSparse)
        mrow = p.bmask.m + (long long)b * p.bmask.sb + (long long)h * p.bmask.sh +
               (long long)qt * p.bmask.srow;
    // the absolute key tile after jj that takes part (jj = j0 - 1: the first)
    auto next_tile = [&](int jj) -> int {
        if constexpr (kSparse) {
            do {
                ++jj;
            } while (jj < j0 + nt_all - 1 && __ldg(mrow + jj) == 0);
            return jj;
        } else {
            return jj + 1;
        }
    };
    int nt = nt_all;
    if constexpr (kSparse) {
        int c = 0;
        for (int base = 0; base < nt_all; base += 32) {
            const int jj = j0 + base + lane;
            c += __popc(__ballot_sync(0xffffffffu, base + lane < nt_all && __ldg(mrow + jj) != 0));
        }
        nt = c;
    }

    if (tid == 0) {
        ptx::mbar_init(&bars->q_full, 1);
        for (int s = 0; s < KST; ++s) {
            ptx::mbar_init(&bars->k_full[s], 1);
            ptx::mbar_init(&bars->k_empty[s], 1);
            ptx::mbar_init(&bars->v_full[s], 1);
            ptx::mbar_init(&bars->v_empty[s], 1);
        }
        for (int hh = 0; hh < 2; ++hh) {
            ptx::mbar_init(&bars->s_full[hh], 1);
            ptx::mbar_init(&bars->p_full[hh], kComputeWarps / 2);
        }
        ptx::mbar_init(&bars->o_done, 1);
        ptx::mbar_init(&bars->drain, 1);
        bars->abort = 0;
        ptx::fence_barrier_init();
    }
    if (warp == kLoaderWarp && lane == 0) {
        ptx::prefetch_tmap(&tm_q);
        ptx::prefetch_tmap(&tm_k);
        ptx::prefetch_tmap(&tm_v);
        ptx::prefetch_tmap(&tm_do);
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
        // ================================================= loader
        if (nt > 0) {
            if (lane == 0) {
                ptx::mbar_arrive_expect_tx(&bars->q_full, 2 * kTile);
                for (int c = 0; c < kDBlocks; ++c) {
                    ptx::tma_load_4d(smem + L::kQ + c * kBlockBytes, &tm_q, &bars->q_full,
                                     c * 64, h, i0, b);
                    ptx::tma_load_4d(smem + L::kDO + c * kBlockBytes, &tm_do, &bars->q_full,
                                     c * 64, h, i0, b);
                }
            }
            __syncwarp();
            int issued_k = 0, issued_v = 0;
            int jj = j0 - 1;  // absolute key tile
            for (int j = 0; j < nt; ++j) {
                jj = next_tile(jj);
                const int st = j % KST;
                if (!warp_wait(&bars->k_empty[st], ((j / KST) & 1) ^ 1, p.limit_ns, abort_flag)) {
                    record_error(p.err, kErrBwdBase + 7, &bars->abort);
                    break;
                }
                if (lane == 0) {
                    ptx::mbar_arrive_expect_tx(&bars->k_full[st], kTile);
                    for (int c = 0; c < kDBlocks; ++c)
                        ptx::tma_load_4d(smem + L::kK + st * kTile + c * kBlockBytes, &tm_k,
                                         &bars->k_full[st], c * 64, g, jj * kBlock, b);
                }
                __syncwarp();
                ++issued_k;
                if (!warp_wait(&bars->v_empty[st], ((j / KST) & 1) ^ 1, p.limit_ns, abort_flag)) {
                    record_error(p.err, kErrBwdBase + 8, &bars->abort);
                    break;
                }
                if (lane == 0) {
                    ptx::mbar_arrive_expect_tx(&bars->v_full[st], kTile);
                    for (int c = 0; c < kDBlocks; ++c)
                        ptx::tma_load_4d(smem + L::kV + st * kTile + c * kBlockBytes, &tm_v,
                                         &bars->v_full[st], c * 64, g, jj * kBlock, b);
                }
                __syncwarp();
                ++issued_v;
            }
            int zero = 0;
            volatile int* no_abort = &zero;
            ptx::mbar_wait(&bars->q_full, 0, p.limit_ns, no_abort);
            for (int j = max(0, issued_k - KST); j < issued_k; ++j)
                ptx::mbar_wait(&bars->k_full[j % KST], (j / KST) & 1, p.limit_ns, no_abort);
            for (int j = max(0, issued_v - KST); j < issued_v; ++j)
                ptx::mbar_wait(&bars->v_full[j % KST], (j / KST) & 1, p.limit_ns, no_abort);
        }
    } else if (warp == kMmaWarp) {
        // ================================================= MMA issuer
        if (nt > 0) {
            bool ok = true;
            bool issued = false;
            auto wait_or_fail = [&](uint64_t* bar, uint32_t parity, unsigned site) {
                if (!warp_wait(bar, parity, p.limit_ns, abort_flag)) {
                    record_error(p.err, kErrBwdBase + site, &bars->abort);
                    ok = false;
                }
                return ok;
            };
            const uint64_t q_desc = ptx::sdesc_sw128(sbase + L::kQ, 16, 1024);
            const uint64_t do_desc = ptx::sdesc_sw128(sbase + L::kDO, 16, 1024);
            constexpr uint64_t kTileUnits = kTile >> 4;
            constexpr uint64_t kHalfUnits = (64 * 128) >> 4;  // 64 rows into a 128-row tile
            // S and dP of key half h (keys 64h .. 64h+63) of key tile j
            auto issue_sdp = [&](int j, int h) {
                const int st = j % KST;
                const uint64_t k_k = ptx::sdesc_sw128(sbase + L::kK, 16, 1024) + st * kTileUnits +
                                     h * kHalfUnits;
                const uint64_t v_k = ptx::sdesc_sw128(sbase + L::kV, 16, 1024) + st * kTileUnits +
                                     h * kHalfUnits;
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk) {
                    const uint64_t o16 = (uint64_t)(((kk >> 2) * kBlockBytes + (kk & 3) * 32) >> 4);
                    ptx::umma_ss_elect(tmem + 64 * h, q_desc + o16, k_k + o16, kIdescS, kk > 0);
                }
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk) {
                    const uint64_t o16 = (uint64_t)(((kk >> 2) * kBlockBytes + (kk & 3) * 32) >> 4);
                    ptx::umma_ss_elect(tmem + kColDP + 64 * h, do_desc + o16, v_k + o16, kIdescS,
                                       kk > 0);
                }
                ptx::umma_commit_elect(&bars->s_full[h]);
            };
            // dQ += dS_h K_h (K = the 64 keys of half h)
            auto issue_dq = [&](int j, int h) {
                const int st = j % KST;
                const uint64_t k_mn = ptx::sdesc_sw128(sbase + L::kK + st * kTile, kBlockBytes, 1024);
#pragma unroll
                for (int kk = 4 * h; kk < 4 * h + 4; ++kk)
                    ptx::umma_ts_elect(tmem + kColDQ,
                                       tmem + (uint32_t)(32 * (kk >> 1) + 8 * (kk & 1)),
                                       k_mn + (uint64_t)((kk * 16 * 128) >> 4), kIdescO,
                                       (j > 0 || kk > 0) ? 1u : 0u);
            };
            auto wait_kv = [&](int j) {
                const int st = j % KST;
                return wait_or_fail(&bars->k_full[st], (j / KST) & 1, 10) &&
                       wait_or_fail(&bars->v_full[st], (j / KST) & 1, 10);
            };
            // Order per key tile j: dQ_0(j), SdP_0(j+1), dQ_1(j), SdP_1(j+1).
            if (wait_or_fail(&bars->q_full, 0, 9) && wait_kv(0)) {
                ptx::tc_fence_after();
                issue_sdp(0, 0);
                issue_sdp(0, 1);
                ptx::umma_commit_elect(&bars->v_empty[0]);
                __syncwarp();
                issued = true;
                for (int j = 0; j < nt; ++j) {
                    if (!wait_or_fail(&bars->p_full[0], j & 1, 11)) break;
                    ptx::tc_fence_after();
                    issue_dq(j, 0);
                    if (j + 1 < nt) {
                        if (!wait_kv(j + 1)) break;
                        ptx::tc_fence_after();
                        issue_sdp(j + 1, 0);
                    }
                    __syncwarp();
                    if (!wait_or_fail(&bars->p_full[1], j & 1, 11)) break;
                    ptx::tc_fence_after();
                    issue_dq(j, 1);
                    ptx::umma_commit_elect(&bars->k_empty[j % KST]);
                    if (j + 1 < nt) {
                        issue_sdp(j + 1, 1);
                        ptx::umma_commit_elect(&bars->v_empty[(j + 1) % KST]);
                    }
                    if (j == nt - 1) ptx::umma_commit_elect(&bars->o_done);
                    __syncwarp();
                }
            }
            if (!ok && issued) {
                int zero = 0;
                volatile int* no_abort = &zero;
                ptx::umma_commit_elect(&bars->drain);
                __syncwarp();
                ptx::mbar_wait(&bars->drain, 0, p.limit_ns, no_abort);
            }
        }
    } else {
        // ================================================= compute warps
        constexpr int kPartD = D / 4;
        const uint32_t quarter = (uint32_t)(warp & 3);
        const int part = warp >> 2;                   // key columns 32*part .. +31
        const int half = part >> 1;                   // key half of those columns
        const uint32_t row = quarter * 32u + (uint32_t)lane;  // query row of the tile
        const int qi = i0 + (int)row;
        const uint32_t lane_addr = (quarter * 32u) << 16;
        const uint32_t t_s = tmem + lane_addr + (uint32_t)(32 * part);
        const uint32_t t_dp = tmem + lane_addr + kColDP + (uint32_t)(32 * part);
        const float sl2 = p.scale_log2;
        const bool row_ok = qi < p.Nq;
        const size_t sidx = ((size_t)b * p.Hq + h) * p.Nq + (row_ok ? qi : 0);
        const float lse2 = row_ok ? p.lse2[sidx] : INFINITY;
        const float dsum = row_ok ? p.dsum[sidx] : 0.f;
        bool ok = true;
        int jj = j0 - 1;  // absolute key tile
        for (int j = 0; j < nt; ++j) {
            jj = next_tile(jj);
            const int st = j % KST;
            const int kc0 = jj * kBlock + 32 * part;  // first key of this warp's columns
            if (!warp_wait(&bars->s_full[half], j & 1, p.limit_ns, abort_flag)) {
                record_error(p.err, kErrBwdBase + 12, &bars->abort);
                ok = false;
                break;
            }
            ptx::tc_fence_after();
            uint32_t sv[32], dv[32];
            ptx::tmem_ld32(t_s, sv);
            ptx::tmem_ld32(t_dp, dv);
            const bool full = row_ok && kc0 + 32 <= Lk && (!p.causal || kc0 + 31 <= qi + off) &&
                              (p.window_left < 0 || kc0 >= qi + off - p.window_left);
            const bool masked = __any_sync(0xffffffffu, !full);
            ptx::tmem_wait_ld_dep(sv);
            ptx::tmem_wait_ld_dep(dv);
            uint32_t pk[16];
            const uint64_t sl2_2 = ptx::f2_pack(sl2, sl2);
            const uint64_t nl2 = ptx::f2_pack(-lse2, -lse2);
            const uint64_t nd2 = ptx::f2_pack(-dsum, -dsum);
#pragma unroll
            for (int e = 0; e < 32; e += 2) {
                float t0, t1;
                ptx::f2_unpack(ptx::f2_fma(ptx::f2_pack(__uint_as_float(sv[e]),
                                                        __uint_as_float(sv[e + 1])),
                                           sl2_2, nl2), t0, t1);
                const float p0 = ptx::ex2_approx(t0), p1 = ptx::ex2_approx(t1);
                const uint64_t d2 = ptx::f2_add(
                    ptx::f2_pack(__uint_as_float(dv[e]), __uint_as_float(dv[e + 1])), nd2);
                float ds0, ds1;
                ptx::f2_unpack(ptx::f2_mul(ptx::f2_pack(p0, p1), d2), ds0, ds1);
                if (masked) {
                    const int kj = kc0 + e;
                    const bool w0 = p.window_left < 0 || kj >= qi + off - p.window_left;
                    const bool w1 = p.window_left < 0 || kj + 1 >= qi + off - p.window_left;
                    const bool v0 = row_ok && kj < Lk && (!p.causal || kj <= qi + off) && w0;
                    const bool v1 = row_ok && kj + 1 < Lk && (!p.causal || kj + 1 <= qi + off) && w1;
                    ds0 = v0 ? ds0 : 0.f;
                    ds1 = v1 ? ds1 : 0.f;
                }
                pk[e / 2] = ptx::pack2<BF16>(ds0, ds1);
            }
            ptx::tmem_st16(t_s, pk);
            // key rows of this half behind the real length: zero them in K (the
            // B operand of dS K), so that 0 * NaN cannot reach dQ; the quarter-0
            // warps of the half take its 64 rows (its S product is complete)
            const int krow = 64 * half + 32 * (part & 1) + lane;
            if (quarter == 0 && jj * kBlock + kBlock > Lk && jj * kBlock + krow >= Lk) {
                uint8_t* kt = smem + L::kK + st * kTile;
#pragma unroll
                for (int c = 0; c < kDBlocks; ++c)
#pragma unroll
                    for (int ch = 0; ch < 8; ++ch)
                        *reinterpret_cast<uint4*>(kt + c * kBlockBytes + krow * 128 + ch * 16) =
                            make_uint4(0, 0, 0, 0);
            }
            ptx::fence_proxy_async_smem();
            ptx::tmem_wait_st();
            ptx::tc_fence_before();
            __syncwarp();
            if (lane == 0) ptx::mbar_arrive(&bars->p_full[half]);
        }
        if (ok && nt > 0) {
            if (!warp_wait(&bars->o_done, 0, p.limit_ns, abort_flag)) {
                record_error(p.err, kErrBwdBase + 13, &bars->abort);
                ok = false;
            }
            ptx::tc_fence_after();
        }
        {
            const size_t elem =
                (((size_t)b * p.Nq + (row_ok ? qi : 0)) * p.Hq + h) * D + part * kPartD;
            const bool zero = !(__all_sync(0xffffffffu, ok) && nt > 0);
            tmem_row_out<kPartD, BF16>(tmem + lane_addr + kColDQ + (uint32_t)(part * kPartD),
                                       p.dq, elem, p.scale, zero, row_ok);
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

template <int D, bool BF16, int QST, int KST, bool kSparse>
cudaError_t launch_bwd_s(const BwdMaps& m, const BwdParams& p, cudaStream_t stream) {
    using L1 = DkdvSmem<D, QST>;
    using L2 = DqSmem<D, KST>;
    static_assert(L1::kAlloc <= 227 * 1024 && L2::kAlloc <= 227 * 1024, "shared memory");
    auto k1 = attn_bwd_dkdv_kernel<D, BF16, QST, kSparse>;
    auto k2 = attn_bwd_dq_kernel<D, BF16, KST, kSparse>;
    cudaError_t e =
        cudaFuncSetAttribute(k1, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)L1::kAlloc);
    if (e != cudaSuccess) return e;
    e = cudaFuncSetAttribute(k2, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)L2::kAlloc);
    if (e != cudaSuccess) return e;
    const long rows = (long)p.B * p.Nq * p.Hq;
    const long pre_blocks = std::min<long>((rows * (D / 8) + 255) / 256, 148L * 16);
    attn_bwd_pre_kernel<D, BF16><<<(int)pre_blocks, 256, 0, stream>>>(p);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    if (p.Nk > 0) {
        const unsigned nkt = (unsigned)((p.Nk + kBlock - 1) / kBlock);
        const dim3 g1 = p.band_kv > 0 ? dim3((unsigned)p.B * p.Hkv * nkt, 1, 1)
                                      : dim3(nkt, p.Hkv, p.B);
        k1<<<g1, kThreads, L1::kAlloc, stream>>>(m.q, m.k, m.v, m.dout, p);
        e = cudaGetLastError();
        if (e != cudaSuccess) return e;
    }
    const unsigned nqt = (unsigned)((p.Nq + kBlock - 1) / kBlock);
    const dim3 g2 = p.band_q > 0 ? dim3((unsigned)p.B * p.Hq * nqt, 1, 1) : dim3(nqt, p.Hq, p.B);
    k2<<<g2, kThreads, L2::kAlloc, stream>>>(m.q, m.k, m.v, m.dout, p);
    return cudaGetLastError();
}

// the block-mask reads are compiled only into the instances a block-sparse
// call launches
template <int D, bool BF16, int QST, int KST>
cudaError_t launch_bwd_t(const BwdMaps& m, const BwdParams& p, cudaStream_t stream) {
    return p.bmask.m != nullptr ? launch_bwd_s<D, BF16, QST, KST, true>(m, p, stream)
                                : launch_bwd_s<D, BF16, QST, KST, false>(m, p, stream);
}

}  // namespace

cudaError_t launch_bwd(const BwdMaps& maps, const BwdParams& p, int d, bool bf16,
                       cudaStream_t stream) {
    if (d == 64) {
        return bf16 ? launch_bwd_t<64, true, 3, 3>(maps, p, stream)
                    : launch_bwd_t<64, false, 3, 3>(maps, p, stream);
    }
    return bf16 ? launch_bwd_t<128, true, 2, 2>(maps, p, stream)
                : launch_bwd_t<128, false, 2, 2>(maps, p, stream);
}

}  // namespace attn
