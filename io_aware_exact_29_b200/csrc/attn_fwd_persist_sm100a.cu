// attn_fwd_persist_sm100a.cu -- the exact attention forward for short work
// units of equal cost (no causal, window or block mask; at most 4096 keys):
// persistent CTAs, one per SM.
//
// The computation is the one of attn_fwd_sm100a.cu (ai6s.net article on the
// ops-transformer FlashAttention operator, section "FlashAttention 拆的不是
// 算法，是数据流": Q, K, V tiles on chip, S = Q·Kᵀ, a running max and sum per
// row, O corrected tile by tile, only O written back); what changes is how
// the work is spread and how the softmax keeps its scores:
//
// Persistent work units: a unit is two 128-row Q tiles of one (batch, head);
// each CTA takes every gridDim.x-th unit and keeps its barriers, tensor memory
// and K/V ring across units, so that the next unit's Q and K/V loads overlap
// the current unit's last tiles.  Before the CTA's last unit each thread
// stores its own output row straight from registers, which leaves the Q
// buffers free for the next unit's Q as soon as the last S that reads them is
// complete; the last unit stages O in its Q buffer and writes it with TMA
// stores.
//
// Warp roles (384 threads):
//   warps 0-3   softmax of Q0 (thread t owns query row t = TMEM lane t)
//   warps 4-7   softmax of Q1
//   warp 8      TMA loader: Q0, Q1 of each work unit, K_j / V_j into rings
//   warp 9      tensor-memory owner and single-thread tcgen05.mma issuer
//   warps 10-11 idle; with warps 8-9 they give registers to the softmax
//               warpgroups (setmaxnreg), which keep a whole score row in
//               registers between the two passes (one tensor-memory read of
//               S per tile)
// Tensor memory (512 columns): S0 [0,128), S1 [128,256), O0 [256,256+D),
// O1 [256+D, 256+2D); at d = 128 P_a overwrites the first 64 columns of S_a,
// at d = 64 it has its own columns, P0 [384, 448) and P1 [448, 512).
//
// MMA issue order per key tile j, d = 128:  S0_j, PV1_{j-1}, S1_j, PV0_j.
// MMAs from one thread execute in issue order, so when S_a_j is complete the
// previous P_a·V has finished reading P_a and updating O_a.  d = 64: S0_j and
// S1_j as soon as the softmax of each has loaded its previous S into
// registers (s_free), then PV0_{j-1}, PV1_{j-1}; the softmax waits for the
// previous P_a·V (pv_done) before it rescales O_a or writes P_a.  Each P_a·V
// is issued in two halves of 64 keys, the first as soon as the softmax has
// written the first half of P_a.
//
// Masks: the per-sequence key length (adaptation point 3 of the ai6s.net
// article) is index arithmetic on the score row, tiles behind it are never
// loaded, and V rows behind it are zeroed in shared memory so that 0 * NaN
// cannot reach O.
#include "attn_fwd_common.cuh"

namespace attn {
namespace {

using namespace fwd;
// warps 0-7 softmax (two warpgroups), warp 8 loader, warp 9 MMA issuer,
// warps 10-11 idle: the producer warpgroup (warps 8-11) gives registers to
// the softmax warpgroups (setmaxnreg), so that a softmax thread keeps its whole
// 128-score row in registers between the two passes
constexpr int kThreads = 384;
constexpr uint32_t kLaunchRegs = 168;  // 65536 / 384, rounded down to a multiple of 8
constexpr uint32_t kProducerRegs = 88;
// the softmax warpgroups' share of the launch's registers: 256 threads x 208
// + 128 x 88 = 64512 = 384 x 168; per SM sub-partition 2 x 208 + 88 = 504
// registers of a thread slot (<= 512)
constexpr uint32_t kSoftmaxRegs = 208;
static_assert(256 * kSoftmaxRegs + 128 * kProducerRegs <= kThreads * kLaunchRegs,
              "register split exceeds the launch allocation");
static_assert(2 * kSoftmaxRegs + kProducerRegs <= 512, "register split exceeds a sub-partition");

template <int D, int KST, int VST>
struct FwdSmem {
    static constexpr uint32_t kTileBytes = kBlockM * D * 2;  // one 128 x D tile
    static constexpr uint32_t kQ = 0;                          // Q0, Q1
    static constexpr uint32_t kK = kQ + 2 * kTileBytes;
    static constexpr uint32_t kV = kK + KST * kTileBytes;
    static constexpr uint32_t kBars = kV + VST * kTileBytes;
    static constexpr uint32_t kTotal = kBars + 512;
    static constexpr uint32_t kAlloc = kTotal + 1024;  // manual 1024-B alignment
};

// One work unit of the forward: rows [qbase, qbase + 256) of head h of batch
// b, with the key-tile ranges of its two 128-row Q tiles.
struct FwdUnit {
    int b, h, g, Lk, qbase;
    int nt0, nt1;      // key tiles of Q0, Q1
    int nt;            // the unit's K/V stream covers tiles [0, nt)
    int last0, last1;  // last key tile used by Q0, Q1 (-1: none)
};

template <int KST, int VST>
struct FwdBars {
    uint64_t q_full[2];
    uint64_t q_empty[2];  // the last S of a unit that read Q_a is complete
    uint64_t k_full[KST];
    uint64_t k_empty[KST];
    uint64_t v_full[VST];
    uint64_t v_empty[VST];
    uint64_t s_full[2];
    uint64_t p_full[2];
    uint64_t p_half[2];  // first half of P (keys 0..63) is in tensor memory
    uint64_t o_done[2];
    uint64_t s_free[2];   // separate-P instance: the softmax has read S_a
    uint64_t pv_done[2];  // separate-P instance: P_a V is complete, P_a may be rewritten
    uint64_t stage_full[2];  // the last unit's output rows are staged for the TMA store
    uint64_t drain;
    uint32_t tmem_base;
    int abort;
};

template <int D, bool BF16, int KST, int VST>
__global__ void __launch_bounds__(kThreads, 1)
    attn_fwd_persist_kernel(const __grid_constant__ CUtensorMap tm_q,
                    const __grid_constant__ CUtensorMap tm_k,
                    const __grid_constant__ CUtensorMap tm_v,
                    const __grid_constant__ CUtensorMap tm_o, const __grid_constant__ FwdParams p) {
    using L = FwdSmem<D, KST, VST>;
    constexpr uint32_t kTileBytes = L::kTileBytes;
    constexpr int kDBlocks = D / 64;  // 64-column (128-byte) blocks per row
    constexpr uint32_t kBlockBytes = kBlockM * 128;
    constexpr uint32_t kIdescS = ptx::idesc_f16(kBlockM, kBlockN, BF16, false);
    constexpr uint32_t kIdescO = ptx::idesc_f16(kBlockM, D, BF16, true);
    // one exponential pair in kPolyEvery on the FMA pipe: fewer than in the
    // one-CTA-per-unit kernel, whose long causal grids prefer a quarter
    // (measured on this kernel: 1/6 at d = 128 +1.4% at 4096 keys against
    // 1/4, 1/12 at d = 64 +4%; more or fewer lost)
    constexpr int kPolyEvery = D == 64 ? 12 : 6;
    // d = 64 leaves 128 tensor-memory columns free: P_a gets its own 64
    // columns (P0 [384, 448), P1 [448, 512)), so S_a of the next tile can be
    // computed as soon as the softmax has loaded S_a, while it still forms P_a
    constexpr bool kSepP = D == 64;

    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw_addr = ptx::smem_u32(smem_raw);
    uint8_t* smem = smem_raw + (((raw_addr + 1023u) & ~1023u) - raw_addr);
    const uint32_t sbase = ptx::smem_u32(smem);
    FwdBars<KST, VST>* bars = reinterpret_cast<FwdBars<KST, VST>*>(smem + L::kBars);
    volatile int* abort_flag = &bars->abort;

    const int tid = threadIdx.x;
    const int warp = tid >> 5;
    const int lane = tid & 31;

    // ---- work units: rows [qbase, qbase + 256) of head h of batch b, row
    // tile fastest, then head, then batch, so that consecutive units share a
    // head's K/V in L2.  CTA c takes units c, c + gridDim.x, c + 2 gridDim.x,
    // ...; launched with one CTA per SM it keeps its barriers, tensor memory
    // and pipeline across units, so that a unit's last tiles and output
    // overlap the next unit's loads.  (The launcher sends only units of equal
    // cost here: no causal, window or block mask.)
    const int n_ctiles = (p.Nq + 2 * kBlockM - 1) / (2 * kBlockM);
    const int n_units = n_ctiles * p.Hq * p.B;

    // key tile j is used by Q tile a when j < nta; the unit's K/V stream is
    // tiles [0, nt) of its kv head
    auto use = [&](const FwdUnit& U, int a, int j) -> bool {
        return j < (a == 0 ? U.nt0 : U.nt1);
    };
    auto make_unit = [&](int u) -> FwdUnit {
        FwdUnit U;
        const int ct = u % n_ctiles;
        U.h = (u / n_ctiles) % p.Hq;
        U.b = u / (n_ctiles * p.Hq);
        U.g = U.h / p.G;
        U.Lk = p.seqlens_k ? p.seqlens_k[U.b] : p.Nk;
        U.qbase = ct * 2 * kBlockM;
        U.nt0 = tiles_for(U.qbase, p.Nq, U.Lk, p.causal);
        U.nt1 = tiles_for(U.qbase + kBlockM, p.Nq, U.Lk, p.causal);
        U.nt = max(U.nt0, U.nt1);
        // the last key tile each Q tile uses (-1: none, the tile's rows get O = 0)
        U.last0 = U.nt0 - 1;
        U.last1 = U.nt1 - 1;
        return U;
    };

    if (tid == 0) {
        for (int a = 0; a < 2; ++a) {
            ptx::mbar_init(&bars->q_full[a], 1);
            ptx::mbar_init(&bars->q_empty[a], 1);
            ptx::mbar_init(&bars->s_full[a], 1);
            ptx::mbar_init(&bars->p_full[a], 128);
            ptx::mbar_init(&bars->p_half[a], 128);
            ptx::mbar_init(&bars->o_done[a], 1);
            ptx::mbar_init(&bars->stage_full[a], 128);
            ptx::mbar_init(&bars->s_free[a], 128);
            ptx::mbar_init(&bars->pv_done[a], 1);
        }
        for (int s = 0; s < KST; ++s) {
            ptx::mbar_init(&bars->k_full[s], 1);
            ptx::mbar_init(&bars->k_empty[s], 1);
        }
        for (int s = 0; s < VST; ++s) {
            ptx::mbar_init(&bars->v_full[s], 1);
            ptx::mbar_init(&bars->v_empty[s], 1);
        }
        ptx::mbar_init(&bars->drain, 1);
        bars->abort = 0;
        ptx::fence_barrier_init();
    }
    if (warp == 8 && lane == 0) {
        ptx::prefetch_tmap(&tm_q);
        ptx::prefetch_tmap(&tm_k);
        ptx::prefetch_tmap(&tm_v);
        ptx::prefetch_tmap(&tm_o);
    }
    if (warp == 9) {
        ptx::tmem_alloc<kTmemCols>(&bars->tmem_base);
        ptx::tmem_relinquish();
    }
    ptx::tc_fence_before();
    __syncthreads();
    ptx::tc_fence_after();
    const uint32_t tmem = bars->tmem_base;

    if (warp >= 8) {
      // the producer warpgroup hands registers to the softmax warpgroups
      ptx::setmaxnreg_dec<kProducerRegs>();
      if (warp == 8) {
        // ================================================= TMA loader
        if (lane == 0 && !p.inject) {
            int issued_k = 0, issued_v = 0;  // over all units
            int nq[2] = {0, 0};              // Q_a loads so far
            int t = -1;                      // stream position, over all units
            bool fail = false;
            for (int u = blockIdx.x; !fail && u < n_units; u += gridDim.x) {
                const FwdUnit U = make_unit(u);
                if (U.nt <= 0) continue;
                for (int a = 0; a < 2; ++a) {
                    // only a Q tile that takes part is loaded; a buffer is
                    // reused once the last S of the previous unit that read
                    // it is complete
                    if ((a == 0 ? U.last0 : U.last1) < 0) continue;
                    if (nq[a] > 0 && !ptx::mbar_wait(&bars->q_empty[a], (nq[a] - 1) & 1,
                                                     p.limit_ns, abort_flag)) {
                        record_error(p.err, kErrFwdBase + 12, &bars->abort);
                        fail = true;
                        break;
                    }
                    ptx::mbar_arrive_expect_tx(&bars->q_full[a], kTileBytes);
                    for (int c = 0; c < kDBlocks; ++c)
                        ptx::tma_load_4d(smem + L::kQ + a * kTileBytes + c * kBlockBytes, &tm_q,
                                         &bars->q_full[a], c * 64, U.h, U.qbase + a * kBlockM,
                                         U.b);
                    ++nq[a];
                }
                if (fail) break;
                for (int j = 0; j < U.nt; ++j) {
                    ++t;
                    const int sk = t % KST;
                    if (!ptx::mbar_wait(&bars->k_empty[sk], ((t / KST) & 1) ^ 1, p.limit_ns,
                                        abort_flag)) {
                        record_error(p.err, kErrFwdBase + 1, &bars->abort);
                        fail = true;
                        break;
                    }
                    ptx::mbar_arrive_expect_tx(&bars->k_full[sk], kTileBytes);
                    for (int c = 0; c < kDBlocks; ++c)
                        ptx::tma_load_4d(smem + L::kK + sk * kTileBytes + c * kBlockBytes, &tm_k,
                                         &bars->k_full[sk], c * 64, U.g, j * kBlockN, U.b);
                    ++issued_k;
                    const int sv = t % VST;
                    if (!ptx::mbar_wait(&bars->v_empty[sv], ((t / VST) & 1) ^ 1, p.limit_ns,
                                        abort_flag)) {
                        record_error(p.err, kErrFwdBase + 2, &bars->abort);
                        fail = true;
                        break;
                    }
                    ptx::mbar_arrive_expect_tx(&bars->v_full[sv], kTileBytes);
                    for (int c = 0; c < kDBlocks; ++c)
                        ptx::tma_load_4d(smem + L::kV + sv * kTileBytes + c * kBlockBytes, &tm_v,
                                         &bars->v_full[sv], c * 64, U.g, j * kBlockN, U.b);
                    ++issued_v;
                }
            }
            // Never leave the CTA with a copy in flight: wait (bounded, and
            // regardless of the abort flag) for the last phase of each
            // barrier that received a copy.
            int zero = 0;
            volatile int* no_abort = &zero;
            for (int a = 0; a < 2; ++a)
                if (nq[a] > 0)
                    ptx::mbar_wait(&bars->q_full[a], (nq[a] - 1) & 1, p.limit_ns, no_abort);
            for (int j = max(0, issued_k - KST); j < issued_k; ++j)
                ptx::mbar_wait(&bars->k_full[j % KST], (j / KST) & 1, p.limit_ns, no_abort);
            for (int j = max(0, issued_v - VST); j < issued_v; ++j)
                ptx::mbar_wait(&bars->v_full[j % VST], (j / VST) & 1, p.limit_ns, no_abort);
        }
    } else if (warp == 9) {
        // ================================================= MMA issuer
        if (lane == 0) {
            bool ok = true;
            int t_base = 0;                       // stream position of the unit's first tile
            int nq[2] = {0, 0};                   // Q_a loads consumed
            int npv[2] = {0, 0};                  // P_a V products issued
            const uint32_t col_s[2] = {0u, 128u};
            const uint32_t col_o[2] = {256u, 256u + D};
            const uint32_t col_p[2] = {kSepP ? 384u : 0u, kSepP ? 448u : 128u};
            int ns[2] = {0, 0};  // S_a products issued
            const uint32_t q_addr[2] = {sbase + L::kQ, sbase + L::kQ + kTileBytes};
            auto wait_or_fail = [&](uint64_t* bar, uint32_t parity, unsigned site) {
                if (!ptx::mbar_wait(bar, parity, p.limit_ns, abort_flag)) {
                    record_error(p.err, kErrFwdBase + site, &bars->abort);
                    ok = false;
                }
                return ok;
            };
            for (int u = blockIdx.x; ok && u < n_units; u += gridDim.x) {
                const FwdUnit U = make_unit(u);
                if (U.nt <= 0) continue;
                bool q_ready[2] = {false, false};
                // S_a of the tile at stream position t; last: the unit's last
                // S_a, after which its Q buffer may be reloaded
                auto issue_s = [&](int a, int t, bool last) {
                    if (kSepP && ns[a] > 0) {
                        // the softmax has loaded the previous S_a
                        if (!wait_or_fail(&bars->s_free[a], (ns[a] - 1) & 1, 11)) return;
                        ptx::tc_fence_after();
                    }
                    ++ns[a];
                    if (!q_ready[a]) {
                        if (!wait_or_fail(&bars->q_full[a], nq[a] & 1, 3)) return;
                        ++nq[a];
                        ptx::tc_fence_after();
                        q_ready[a] = true;
                    }
                    const uint32_t k_addr = sbase + L::kK + (t % KST) * kTileBytes;
#pragma unroll
                    for (int kk = 0; kk < D / 16; ++kk) {
                        const uint32_t off = (kk >> 2) * kBlockBytes + (kk & 3) * 32;
                        ptx::umma_ss(tmem + col_s[a],
                                     ptx::sdesc_sw128(q_addr[a] + off, 16, 1024),
                                     ptx::sdesc_sw128(k_addr + off, 16, 1024), kIdescS, kk > 0);
                    }
                    ptx::umma_commit(&bars->s_full[a]);
                    if (last) ptx::umma_commit(&bars->q_empty[a]);
                };
                // P_a·V of the tile at stream position t, the Q tile's ia-th
                // tile of the unit; last: the Q tile's O is complete after it
                auto issue_pv = [&](int a, int t, int ia, bool last) {
                    if (!wait_or_fail(&bars->p_half[a], npv[a] & 1, 5)) return;
                    if (!wait_or_fail(&bars->v_full[t % VST], (t / VST) & 1, 6)) return;
                    ptx::tc_fence_after();
                    const uint32_t v_addr = sbase + L::kV + (t % VST) * kTileBytes;
#pragma unroll
                    for (int kk = 0; kk < kBlockN / 16; ++kk) {
                        if (kk == kBlockN / 32) {
                            if (!wait_or_fail(&bars->p_full[a], npv[a] & 1, 5)) return;
                            ptx::tc_fence_after();
                        }
                        ptx::umma_ts(tmem + col_o[a], tmem + col_p[a] + kk * 8,
                                     ptx::sdesc_sw128(v_addr + kk * 16 * 128, kBlockBytes, 1024),
                                     kIdescO, (ia > 0 || kk > 0) ? 1u : 0u);
                    }
                    ++npv[a];
                    if (kSepP) ptx::umma_commit(&bars->pv_done[a]);
                    if (last) ptx::umma_commit(&bars->o_done[a]);
                };
                {
                    // a stage is released after its last user's product
                    int t = t_base, i0 = 0, i1 = 0;           // stream position, per-tile counts
                    int prev_t = 0, prev_i1 = 0, prev_j = -1;  // the previous tile of the stream
                    bool prev_u1 = false;
                    if constexpr (kSepP) {
                        // separate P columns: per tile S0_j, S1_j (each as soon
                        // as its softmax has loaded the previous S), then
                        // P0_{j-1} V, P1_{j-1} V
                        int prev_i0 = 0;
                        bool prev_u0 = false;
                        for (int j = 0; ok && j <= U.nt; ++j) {
                            bool u0 = false, u1 = false;
                            if (j < U.nt) {
                                u0 = use(U, 0, j);
                                u1 = use(U, 1, j);
                                if (!wait_or_fail(&bars->k_full[t % KST], (t / KST) & 1, 4)) break;
                                ptx::tc_fence_after();
                                if (u0) issue_s(0, t, j == U.last0);
                                if (!ok) break;
                                if (u1) issue_s(1, t, j == U.last1);
                                if (!ok) break;
                                ptx::umma_commit(&bars->k_empty[t % KST]);
                            }
                            if (prev_u0) {
                                issue_pv(0, prev_t, prev_i0, prev_j == U.last0);
                                if (!ok) break;
                                if (!prev_u1) ptx::umma_commit(&bars->v_empty[prev_t % VST]);
                            }
                            if (prev_u1) {
                                issue_pv(1, prev_t, prev_i1, prev_j == U.last1);
                                if (!ok) break;
                                ptx::umma_commit(&bars->v_empty[prev_t % VST]);
                            }
                            prev_u0 = u0;
                            prev_u1 = u1;
                            prev_t = t;
                            prev_i0 = i0;
                            prev_i1 = i1;
                            prev_j = j;
                            i0 += u0 ? 1 : 0;
                            i1 += u1 ? 1 : 0;
                            ++t;
                        }
                    } else {
                    for (int j = 0; ok && j <= U.nt; ++j) {
                        bool u0 = false, u1 = false;
                        if (j < U.nt) {
                            u0 = use(U, 0, j);
                            u1 = use(U, 1, j);
                            if (!wait_or_fail(&bars->k_full[t % KST], (t / KST) & 1, 4)) break;
                            ptx::tc_fence_after();
                            if (u0) issue_s(0, t, j == U.last0);
                            if (!ok) break;
                        }
                        if (prev_u1) {
                            issue_pv(1, prev_t, prev_i1, prev_j == U.last1);
                            if (!ok) break;
                            ptx::umma_commit(&bars->v_empty[prev_t % VST]);
                        }
                        if (j < U.nt) {
                            if (u1) issue_s(1, t, j == U.last1);
                            if (!ok) break;
                            ptx::umma_commit(&bars->k_empty[t % KST]);
                            if (u0) {
                                issue_pv(0, t, i0, j == U.last0);
                                if (!ok) break;
                            }
                            if (!u1) ptx::umma_commit(&bars->v_empty[t % VST]);
                        }
                        prev_u1 = u1;
                        prev_t = t;
                        prev_i1 = i1;
                        prev_j = j;
                        i0 += u0 ? 1 : 0;
                        i1 += u1 ? 1 : 0;
                        ++t;
                    }
                    }  // the in-place P order
                }
                t_base += U.nt;
            }
            if (!ok) {
                // make sure no MMA is still running before TMEM is freed
                int zero = 0;
                volatile int* no_abort = &zero;
                ptx::umma_commit(&bars->drain);
                ptx::mbar_wait(&bars->drain, 0, p.limit_ns, no_abort);
            }
        }
      }
    } else {
        ptx::setmaxnreg_inc<kSoftmaxRegs>();
        // ================================================= softmax warpgroups
        const int a = warp >> 2;  // which Q tile
        const uint32_t quarter = (uint32_t)(warp & 3);
        const uint32_t row = quarter * 32u + (uint32_t)lane;
        const uint32_t lane_addr = (quarter * 32u) << 16;
        const float sl2 = p.scale_log2;
        const uint64_t sl2_2 = ptx::f2_pack(sl2, sl2);
        const uint32_t t_s = tmem + lane_addr + (a == 0 ? 0u : 128u);
        // P_a: over the first 64 columns of S_a, or its own columns (kSepP)
        const uint32_t t_p = kSepP ? tmem + lane_addr + (a == 0 ? 384u : 448u) : t_s;
        const uint32_t t_o = tmem + lane_addr + (a == 0 ? 256u : 256u + D);
        bool ok = true;
        int t_base = 0;      // stream position of the unit's first tile
        int tiles_done = 0;  // S_a products consumed (parity of s_full)
        int units_done = 0;  // units in which this Q tile had work (parity of o_done)
        for (int u = blockIdx.x; ok && u < n_units; u += gridDim.x) {
            const FwdUnit U = make_unit(u);
            const int nta = a == 0 ? U.nt0 : U.nt1;
            const int qa = U.qbase + a * kBlockM;
            const int i = qa + (int)row;
            int row_lim = U.Lk - 1;  // last visible key of this row
            if (p.causal) row_lim = min(row_lim, i + U.Lk - p.Nq);
            // first visible key of this row (the sliding window's lower edge)
            const int row_first = 0;  // no window: every key from 0 on
            float m_ref = -INFINITY;  // running reference max, scale*log2 units
            float l_sum = 0.f;        // running sum of exp2(s*sl2 - m_ref)

            int ia = 0;  // key tiles of this Q tile done so far in the unit
            const int n_iter = nta;
            for (int it = 0; it < n_iter; ++it) {
                int j, t;         // key tile, its stream position
                bool first_user;  // this Q tile's P·V is the first to read V_j
                {
                    j = it;
                    t = t_base + j;
                    first_user = a == 0 || !use(U, 0, j);
                }
                if (!warp_wait(&bars->s_full[a], tiles_done & 1, p.limit_ns, abort_flag)) {
                    record_error(p.err, kErrFwdBase + 7, &bars->abort);
                    ok = false;
                    break;
                }
                ++tiles_done;
                ptx::tc_fence_after();
                const int key0 = j * kBlockN;
                const bool masked = key0 + kBlockN - 1 > row_lim;
                // d = 64: masked tiles are taken 32 columns at a time, by the
                // whole warp (the chunk votes are warp-collective; a row
                // without masked keys finds its chunks visible, with the same
                // results).  At d = 128 the chunk code cost the unmasked tiles
                // 1.3% (measured), so that instance keeps the per-element mask.
                constexpr bool kChunkMask = D == 64;
                const bool masked_w = kChunkMask && __any_sync(0xffffffffu, masked);
                // pass 1: row maximum, two halves of 64 columns, eight independent
                // chains of three-input maxima
                float mx8[8];
#pragma unroll
                for (int uu = 0; uu < 8; ++uu) mx8[uu] = -INFINITY;
                // the whole row stays in registers for pass 2 (one load of S per tile)
                uint32_t rs[2][2][32];
                {
                    auto& r = rs;
#pragma unroll
                    for (int hf = 0; hf < 2; ++hf) {
                        ptx::tmem_ld32(t_s + hf * 64, r[hf][0]);
                        ptx::tmem_ld32(t_s + hf * 64 + 32, r[hf][1]);
                    }
#pragma unroll
                    for (int hf = 0; hf < 2; ++hf) {
                        ptx::tmem_wait_ld_dep(r[hf][0]);
                        ptx::tmem_wait_ld_dep(r[hf][1]);
                        if (masked_w)
                            half_max_chunks<false>(r[hf], key0 + hf * 64, row_first, row_lim, mx8);
                        else if (!kChunkMask && masked)
                            half_max<true, false>(r[hf], key0 + hf * 64, row_first, row_lim, mx8);
                        else
                            half_max<false, false>(r[hf], key0 + hf * 64, row_first, row_lim,
                                                     mx8);
                    }
                }
                if constexpr (kSepP) {
                    // S_a is in registers: the next tile's S_a may be computed
                    ptx::tc_fence_before();
                    ptx::mbar_arrive(&bars->s_free[a]);
                }
                const float mx = ptx::max3(ptx::max3(mx8[0], mx8[1], mx8[2]),
                                           ptx::max3(mx8[3], mx8[4], mx8[5]), fmaxf(mx8[6], mx8[7]));
                const float m_tile = mx * sl2;  // -inf stays -inf (sl2 > 0)
                float alpha = 1.f;
                bool rescale = false;
                if (m_tile > m_ref + kRescaleThreshold) {
                    alpha = ptx::ex2_approx(m_ref - m_tile);  // 0 when m_ref = -inf
                    rescale = (ia > 0) && (m_ref != -INFINITY);
                    m_ref = m_tile;
                }
                const float m_use = (m_ref == -INFINITY) ? 0.f : m_ref;
                const uint64_t nm_2 = ptx::f2_pack(-m_use, -m_use);
                if (kSepP && tiles_done >= 2) {
                    // the previous P_a V has completed: O_a may be rescaled and
                    // P_a rewritten
                    if (!warp_wait(&bars->pv_done[a], (tiles_done - 2) & 1, p.limit_ns, abort_flag)) {
                        record_error(p.err, kErrFwdBase + 10, &bars->abort);
                        ok = false;
                        break;
                    }
                    ptx::tc_fence_after();
                }
                if (__any_sync(0xffffffffu, rescale)) {
                    // the previous P_a V has completed (it precedes S_a_j); done
                    // before the exponentials, since the first half of P_a V may
                    // start while the second half of P_a is still being formed
                    const float sc = rescale ? alpha : 1.f;
#pragma unroll 1
                    for (int c = 0; c < D / 32; ++c) {
                        uint32_t r[32];
                        ptx::tmem_ld32(t_o + c * 32, r);
                        ptx::tmem_wait_ld_dep(r);
#pragma unroll
                        for (int e = 0; e < 32; ++e)
                            r[e] = __float_as_uint(__uint_as_float(r[e]) * sc);
                        ptx::tmem_st32(t_o + c * 32, r);
                    }
                    ptx::tmem_wait_st();
                }
                ptx::tmem_wait_st();
                // the Q tile whose P·V reads V_j first zeroes its rows behind the
                // real length (Q0 if it uses the tile, else Q1)
                const bool zero_v = p.seqlens_k != nullptr && key0 + kBlockN > U.Lk && first_user;
                if (zero_v) {
                    // keys behind the real length: zero their V rows so that a
                    // non-finite value stored there cannot reach O through 0 * NaN
                    const int sv = t % VST;
                    if (!warp_wait(&bars->v_full[sv], (t / VST) & 1, p.limit_ns, abort_flag)) {
                        record_error(p.err, kErrFwdBase + 8, &bars->abort);
                        ok = false;
                        break;
                    }
                    if (key0 + (int)row >= U.Lk) {
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
                uint64_t acc2[4] = {0, 0, 0, 0};  // four pair accumulators of the row sum
                // pass 2: exponentials per half; P of half hf goes to columns
                // [32 hf, 32 hf + 32) of S_a, which pass 2 has already consumed,
                // and is published on its own barrier (p_half, then p_full) so
                // that the MMA of keys 0..63 overlaps the exponentials of 64..127
#pragma unroll
                for (int hf = 0; hf < 2; ++hf) {
                    auto& r = rs[hf];
                    uint32_t pk[32];
                    if (masked_w)
                        half_exp_chunks<false, BF16, kPolyEvery>(r, key0 + hf * 64, row_first,
                                                                  row_lim, sl2_2, nm_2, acc2, pk);
                    else if (!kChunkMask && masked)
                        half_exp<true, false, BF16, kPolyEvery>(r, key0 + hf * 64, row_first,
                                                                  row_lim, sl2_2, nm_2, acc2, pk);
                    else
                        half_exp<false, false, BF16, kPolyEvery>(r, key0 + hf * 64, row_first,
                                                                   row_lim, sl2_2, nm_2, acc2, pk);
                    ptx::tmem_st32(t_p + hf * 32, pk);
                    ptx::tmem_wait_st();
                    ptx::tc_fence_before();
                    ptx::mbar_arrive(hf == 0 ? &bars->p_half[a] : &bars->p_full[a]);
                }
                float s0, s1, s2, s3, s4, s5, s6, s7;
                ptx::f2_unpack(acc2[0], s0, s1);
                ptx::f2_unpack(acc2[1], s2, s3);
                ptx::f2_unpack(acc2[2], s4, s5);
                ptx::f2_unpack(acc2[3], s6, s7);
                const float rowsum = ((s0 + s1) + (s2 + s3)) + ((s4 + s5) + (s6 + s7));
                l_sum = l_sum * alpha + rowsum;
                ++ia;
            }
            if (!ok) break;

            // ---- epilogue of the unit: O / l -> bf16/fp16 and LSE.  The CTA's
            // last unit stages O in its Q buffer (free: no Q follows) and
            // writes it with TMA stores; earlier units store each thread's
            // row straight from registers, since their Q buffer already holds
            // the next unit's Q.
            const bool last_unit = u + (int)gridDim.x >= n_units;
            if (ia > 0) {
                if (!warp_wait(&bars->o_done[a], units_done & 1, p.limit_ns, abort_flag)) {
                    record_error(p.err, kErrFwdBase + 9, &bars->abort);
                    ok = false;
                    break;
                }
                ++units_done;
                ptx::tc_fence_after();
            }
            const bool have = ia > 0 && l_sum > 0.f;
            const float inv_l = have ? 1.f / l_sum : 0.f;
            if (qa < p.Nq) {
                uint8_t* orow = static_cast<uint8_t*>(p.o) +
                                (((size_t)U.b * p.Nq + (size_t)i) * p.Hq + U.h) * (size_t)(D * 2);
                uint8_t* stage = smem + L::kQ + a * kTileBytes;
#pragma unroll
                for (int c = 0; c < D / 32; ++c) {
                    uint32_t r[32];
                    if (ia > 0) {
                        ptx::tmem_ld32(t_o + c * 32, r);
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
#pragma unroll
                    for (int q4 = 0; q4 < 4; ++q4) {
                        const uint4 w = make_uint4(o2[q4 * 4], o2[q4 * 4 + 1], o2[q4 * 4 + 2],
                                                   o2[q4 * 4 + 3]);
                        if (last_unit) {
                            // 32 columns = 4 chunks of 16 bytes in block c/2, chunks
                            // (c%2)*4 .. +3 of the 128-byte swizzled row
                            const uint32_t ch = (uint32_t)((c & 1) * 4 + q4);
                            *reinterpret_cast<uint4*>(stage + (c >> 1) * kBlockBytes + row * 128u +
                                                      ((ch ^ (row & 7u)) << 4)) = w;
                        } else if (i < p.Nq) {
                            *reinterpret_cast<uint4*>(orow + c * 64 + q4 * 16) = w;
                        }
                    }
                }
                if (last_unit) {
                    // the staged tile goes out by TMA once all 128 rows are in;
                    // a bounded wait, so that a warp that left on an error
                    // cannot hold the others
                    ptx::fence_proxy_async_smem();
                    ptx::mbar_arrive(&bars->stage_full[a]);
                    if (quarter == 0 && lane == 0) {
                        if (ptx::mbar_wait(&bars->stage_full[a], 0, p.limit_ns, abort_flag)) {
                            for (int c = 0; c < kDBlocks; ++c)
                                ptx::tma_store_4d(&tm_o, stage + c * kBlockBytes, c * 64, U.h,
                                                  qa, U.b);
                            ptx::bulk_commit_group();
                            ptx::bulk_wait_group_read0();
                        } else {
                            record_error(p.err, kErrFwdBase + 13, &bars->abort);
                        }
                    }
                }
            }
            if (i < p.Nq) {
                const float lse = have ? (m_ref + ptx::lg2_approx(l_sum)) * 0.69314718055994531f
                                       : -INFINITY;
                p.lse[((size_t)U.b * p.Hq + U.h) * p.Nq + i] = lse;
            }
            // the tensor-memory reads of O complete before this warpgroup
            // publishes the next unit's first P, after which the first P·V
            // of that unit overwrites O
            ptx::tc_fence_before();
            t_base += U.nt;
        }
    }

    ptx::tc_fence_before();
    __syncthreads();
    if (warp == 9) {
        __syncwarp();
        ptx::tc_fence_after();
        ptx::tmem_dealloc<kTmemCols>(tmem);
    }
}

template <int D, bool BF16, int KST, int VST>
cudaError_t launch_fwd_persist_t(const FwdMaps& maps, const FwdParams& p, cudaStream_t stream) {
    using L = FwdSmem<D, KST, VST>;
    static_assert(L::kAlloc <= 227 * 1024, "shared memory budget");
    auto kern = attn_fwd_persist_kernel<D, BF16, KST, VST>;
    cudaError_t e =
        cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)L::kAlloc);
    if (e != cudaSuccess) return e;
    kern<<<dim3((unsigned)p.n_ctas), kThreads, L::kAlloc, stream>>>(maps.q, maps.k, maps.v, maps.o,
                                                                    p);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_fwd_persist(const FwdMaps& maps, const FwdParams& p, int d, bool bf16,
                               cudaStream_t stream) {
    if (d == 64) {
        return bf16 ? launch_fwd_persist_t<64, true, 3, 4>(maps, p, stream)
                    : launch_fwd_persist_t<64, false, 3, 4>(maps, p, stream);
    }
    return bf16 ? launch_fwd_persist_t<128, true, 2, 3>(maps, p, stream)
                : launch_fwd_persist_t<128, false, 2, 3>(maps, p, stream);
}

}  // namespace attn
