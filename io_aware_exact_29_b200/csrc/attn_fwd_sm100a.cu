// attn_fwd_sm100a.cu -- exact attention forward on tcgen05 tensor cores.
//
// One CTA owns two 128-row tiles of queries (Q0, Q1) of one (batch, head) and
// streams the key/value tiles of its head through shared memory once for both
// (ai6s.net article on the ops-transformer FlashAttention operator, section
// "FlashAttention 拆的不是算法，是数据流": split Q, K, V along the sequence into
// on-chip tiles, run Q_tile·K_tileᵀ -> softmax -> ·V_tile on chip, write back
// only O; the effectstory.com article "FlashAttention：IO 感知的精確注意力演算
// 法..." states the same single pass: Q, K, V loaded once, O written once).
//
// Warp roles (320 threads):
//   warps 0-3   softmax of Q0 (thread t owns query row t = TMEM lane t)
//   warps 4-7   softmax of Q1
//   warp 8      TMA loader: Q0, Q1 once, then K_j / V_j into rings
//   warp 9      tensor-memory owner and single-thread tcgen05.mma issuer
// Tensor memory (512 columns): S0 [0,128), S1 [128,256), O0 [256,256+D),
// O1 [256+D, 256+2D).  Each softmax thread reads its score row from S_a,
// keeps the running max m and sum l (the online softmax of the section above),
// and writes P (bf16/fp16) back over the first 64 columns of S_a; the P·V MMA
// reads P straight from tensor memory as its A operand, V from shared memory.
//
// MMA issue order per key tile j:  S0_j, PV1_{j-1}, S1_j, PV0_j.  While the
// softmax of Q0 works on S0_j the tensor core runs PV1_{j-1} and S1_j, and
// while the softmax of Q1 works on S1_j it runs PV0_j and S0_{j+1}.  MMAs from
// one thread execute in issue order, so when S_a_j is complete the previous
// P_a·V has finished reading P_a and updating O_a: the softmax may rescale
// O_a and overwrite P_a without another wait.  Each P_a·V is issued in two
// halves of 64 keys, the first as soon as the softmax has written the first
// half of P_a, so that it overlaps the exponentials of the second half.
//
// Fused masks: the causal rule (adaptation point 2 of the ai6s.net article)
// and the per-sequence key length (point 3) are index arithmetic on the score
// row; tiles wholly outside them are never loaded, and V rows behind the real
// length are zeroed in shared memory so that 0 * NaN cannot reach O.  Two
// more instances add the mask extensions: a sliding window (a lower edge on
// each row, tiles before a Q tile's window skipped) and a block mask over
// 128 x 128 tiles, where the two Q tiles walk their own tile lists in
// lockstep.
//
// Short units of equal cost (no causal, window or block mask, at most 4096
// keys) run on the persistent variant in attn_fwd_persist_sm100a.cu instead.
//
// Launch order: causal row tiles differ in cost, so the causal grid is 1-D,
// in bands of (batch, head) pairs whose K/V fit in L2 together, the costliest
// row tile of every pair of a band first.
//
// Lazy rescaling: the reference maximum of a row only moves when a tile's
// maximum exceeds it by more than 8 (log2 units), so P <= 2^8; numerator and
// denominator share the reference, so the result is the same exact softmax.
#include "attn_fwd_common.cuh"

namespace attn {
namespace {

using namespace fwd;
constexpr int kThreads = 320;
// a window wider than any key range (i + Lk - Nq - kNoWindow stays negative)
constexpr int kNoWindow = 1 << 30;

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

template <int KST, int VST>
struct FwdBars {
    uint64_t q_full[2];
    uint64_t k_full[KST];
    uint64_t k_empty[KST];
    uint64_t v_full[VST];
    uint64_t v_empty[VST];
    uint64_t s_full[2];
    uint64_t p_full[2];
    uint64_t p_half[2];  // first half of P (keys 0..63) is in tensor memory
    uint64_t o_done[2];
    uint64_t drain;
    uint32_t tmem_base;
    int abort;
};

template <int D, bool BF16, int KST, int VST, bool kWindow, bool kSparse>
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
    constexpr int kPolyEvery = FWD_POLY_EVERY(D);

    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw_addr = ptx::smem_u32(smem_raw);
    uint8_t* smem = smem_raw + (((raw_addr + 1023u) & ~1023u) - raw_addr);
    const uint32_t sbase = ptx::smem_u32(smem);
    FwdBars<KST, VST>* bars = reinterpret_cast<FwdBars<KST, VST>*>(smem + L::kBars);
    volatile int* abort_flag = &bars->abort;

    const int tid = threadIdx.x;
    const int warp = tid >> 5;
    const int lane = tid & 31;

    // ---- work unit: rows [qbase, qbase + 256) of head h of batch b
    // causal: a 1-D grid in bands of (b, h) pairs, the costliest (last) row
    // tile of every pair of a band first, so that blocks launch in
    // decreasing cost; otherwise (row tiles, Hq, B), consecutive blocks
    // sharing a head's K/V in L2
    const int n_ctiles = (p.Nq + 2 * kBlockM - 1) / (2 * kBlockM);
    int ct, h, b;
    if (p.band > 0) {
        int pair, rank;
        band_unit(blockIdx.x, p.band, p.B * p.Hq, n_ctiles, pair, rank);
        ct = n_ctiles - 1 - rank;
        h = pair % p.Hq;
        b = pair / p.Hq;
    } else {
        ct = blockIdx.x;
        h = blockIdx.y;
        b = blockIdx.z;
    }
    const int g = h / p.G;
    const int Lk = p.seqlens_k ? p.seqlens_k[b] : p.Nk;
    const int qbase = ct * 2 * kBlockM;
    const int nt0 = tiles_for(qbase, p.Nq, Lk, p.causal);
    const int nt1 = tiles_for(qbase + kBlockM, p.Nq, Lk, p.causal);
    // sliding window: the first key tile each Q tile needs (tiles before it
    // are never loaded); stages and phases count from the CTA's first tile
    // jstart and from each Q tile's own first tile
    const int qoff = Lk - p.Nq;  // query i's own key position is i + qoff
    int j00 = 0, j01 = 0;
    if constexpr (kWindow) {  // kWindow: the instance launched for window_left >= 0
        j00 = max(0, qbase + qoff - p.window_left) / kBlockN;
        j01 = max(0, qbase + kBlockM + qoff - p.window_left) / kBlockN;
    }
    const int cnt0 = max(0, nt0 - j00), cnt1 = max(0, nt1 - j01);
    const int jstart = cnt0 > 0 ? j00 : j01;
    const int nt = max(cnt0 > 0 ? nt0 : 0, cnt1 > 0 ? nt1 : 0);
    // block-sparse instance: the mask rows of the two Q tiles
    const unsigned char* mrow = nullptr;
    if constexpr (kSparse)
        mrow = p.bmask.m + (long long)b * p.bmask.sb + (long long)h * p.bmask.sh +
               (long long)(qbase / kBlockM) * p.bmask.srow;
    // key tile j is used by Q0 when j in [j00, nt0), by Q1 when j in
    // [j01, nt1), and (block-sparse) when the mask entry of the pair is set;
    // without a block mask the K/V stream is the union of the two, in
    // increasing j
    auto use = [&](int a, int j) -> bool {
        bool u = a == 0 ? (cnt0 > 0 && j >= j00 && j < nt0) : (cnt1 > 0 && j >= j01 && j < nt1);
        if constexpr (kSparse) {
            if (u) u = __ldg(mrow + (a == 0 ? 0 : p.bmask.srow) + j) != 0;
        }
        return u;
    };
    // the last key tile each Q tile uses (-1: none, the tile's rows get O = 0)
    int last0 = -1, last1 = -1;
    for (int j = nt0 - 1; cnt0 > 0 && j >= j00; --j)
        if (use(0, j)) {
            last0 = j;
            break;
        }
    for (int j = nt1 - 1; cnt1 > 0 && j >= j01; --j)
        if (use(1, j)) {
            last1 = j;
            break;
        }
    // Block-sparse schedule: the two Q tiles walk their own tile lists in
    // lockstep.  Step i pairs the i-th key tile of Q0 with the i-th of Q1, and
    // the K/V stream loads Q0's tile, then Q1's when it is a different one, so
    // that masks that differ between the two cost max(n0, n1) steps, not the
    // size of the union.
    int n0 = 0, n1 = 0;  // key tiles of each Q tile
    if constexpr (kSparse) {
        for (int j = j00; cnt0 > 0 && j < nt0; ++j) n0 += use(0, j) ? 1 : 0;
        for (int j = j01; cnt1 > 0 && j < nt1; ++j) n1 += use(1, j) ? 1 : 0;
    }
    const int nsteps = max(n0, n1);
    // c0, c1: next candidate tile of each Q tile; si: step; pos: next position
    auto next_pair = [&](int& c0, int& c1, int& si, int& pos) -> PairStep {
        return sparse_next_step(use, n0, n1, nt0, nt1, c0, c1, si, pos);
    };

    if (tid == 0) {
        for (int a = 0; a < 2; ++a) {
            ptx::mbar_init(&bars->q_full[a], 1);
            ptx::mbar_init(&bars->s_full[a], 1);
            ptx::mbar_init(&bars->p_full[a], 128);
            ptx::mbar_init(&bars->p_half[a], 128);
            ptx::mbar_init(&bars->o_done[a], 1);
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

    if (warp == 8) {
        // ================================================= TMA loader
        if (lane == 0 && nt > 0 && !p.inject) {
            int issued_k = 0, issued_v = 0;
            bool issued_q[2] = {false, false};
            for (int a = 0; a < 2; ++a) {
                // only a Q tile that takes part: the epilogue of the others
                // stages O in the Q buffer without waiting for anything
                if ((a == 0 ? last0 : last1) < 0) continue;
                ptx::mbar_arrive_expect_tx(&bars->q_full[a], kTileBytes);
                for (int c = 0; c < kDBlocks; ++c)
                    ptx::tma_load_4d(smem + L::kQ + a * kTileBytes + c * kBlockBytes, &tm_q,
                                     &bars->q_full[a], c * 64, h, qbase + a * kBlockM, b);
                issued_q[a] = true;
            }
            int t = -1;  // position of tile j in the stream
            int c0 = j00, c1 = j01, si = 0, spos = 0;  // block-sparse schedule
            PairStep st{};
            int e = 1;   // block-sparse: which tile of step st comes next
            const int n_iter = kSparse ? 2 * nsteps : nt - jstart;
            for (int it = 0; it < n_iter; ++it) {
                int j;
                if constexpr (kSparse) {
                    if (e == 1) {
                        st = next_pair(c0, c1, si, spos);
                        e = 0;
                    } else {
                        e = 1;
                    }
                    const bool has = e == 0 ? st.has0 : (st.has1 && !st.shared);
                    if (!has) continue;
                    j = e == 0 ? st.x0 : st.x1;
                } else {
                    j = jstart + it;
                }
                ++t;
                const int sk = t % KST;
                if (!ptx::mbar_wait(&bars->k_empty[sk], ((t / KST) & 1) ^ 1, p.limit_ns,
                                    abort_flag)) {
                    record_error(p.err, kErrFwdBase + 1, &bars->abort);
                    break;
                }
                ptx::mbar_arrive_expect_tx(&bars->k_full[sk], kTileBytes);
                for (int c = 0; c < kDBlocks; ++c)
                    ptx::tma_load_4d(smem + L::kK + sk * kTileBytes + c * kBlockBytes, &tm_k,
                                     &bars->k_full[sk], c * 64, g, j * kBlockN, b);
                ++issued_k;
                const int sv = t % VST;
                if (!ptx::mbar_wait(&bars->v_empty[sv], ((t / VST) & 1) ^ 1, p.limit_ns,
                                    abort_flag)) {
                    record_error(p.err, kErrFwdBase + 2, &bars->abort);
                    break;
                }
                ptx::mbar_arrive_expect_tx(&bars->v_full[sv], kTileBytes);
                for (int c = 0; c < kDBlocks; ++c)
                    ptx::tma_load_4d(smem + L::kV + sv * kTileBytes + c * kBlockBytes, &tm_v,
                                     &bars->v_full[sv], c * 64, g, j * kBlockN, b);
                ++issued_v;
            }
            // Never leave the CTA with a copy in flight: wait (bounded, and
            // regardless of the abort flag) for the last phase of each
            // barrier that received a copy.
            int zero = 0;
            volatile int* no_abort = &zero;
            for (int a = 0; a < 2; ++a)
                if (issued_q[a]) ptx::mbar_wait(&bars->q_full[a], 0, p.limit_ns, no_abort);
            for (int j = max(0, issued_k - KST); j < issued_k; ++j)
                ptx::mbar_wait(&bars->k_full[j % KST], (j / KST) & 1, p.limit_ns, no_abort);
            for (int j = max(0, issued_v - VST); j < issued_v; ++j)
                ptx::mbar_wait(&bars->v_full[j % VST], (j / VST) & 1, p.limit_ns, no_abort);
        }
    } else if (warp == 9) {
        // ================================================= MMA issuer
        if (lane == 0 && nt > 0) {
            bool ok = true;
            bool q_ready[2] = {false, false};
            const uint32_t col_s[2] = {0u, 128u};
            const uint32_t col_o[2] = {256u, 256u + D};
            const uint32_t q_addr[2] = {sbase + L::kQ, sbase + L::kQ + kTileBytes};
            auto wait_or_fail = [&](uint64_t* bar, uint32_t parity, unsigned site) {
                if (!ptx::mbar_wait(bar, parity, p.limit_ns, abort_flag)) {
                    record_error(p.err, kErrFwdBase + site, &bars->abort);
                    ok = false;
                }
                return ok;
            };
            // S_a of the tile at stream position t
            auto issue_s = [&](int a, int t) {
                if (!q_ready[a]) {
                    if (!wait_or_fail(&bars->q_full[a], 0, 3)) return;
                    ptx::tc_fence_after();
                    q_ready[a] = true;
                }
                const uint32_t k_addr = sbase + L::kK + (t % KST) * kTileBytes;
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk) {
                    const uint32_t off = (kk >> 2) * kBlockBytes + (kk & 3) * 32;
                    ptx::umma_ss(tmem + col_s[a], ptx::sdesc_sw128(q_addr[a] + off, 16, 1024),
                                 ptx::sdesc_sw128(k_addr + off, 16, 1024), kIdescS, kk > 0);
                }
                ptx::umma_commit(&bars->s_full[a]);
            };
            // P_a·V of the tile at stream position t, the Q tile's ia-th tile;
            // last: the Q tile's O is complete after it
            auto issue_pv = [&](int a, int t, int ia, bool last) {
                if (!wait_or_fail(&bars->p_half[a], ia & 1, 5)) return;
                if (!wait_or_fail(&bars->v_full[t % VST], (t / VST) & 1, 6)) return;
                ptx::tc_fence_after();
                const uint32_t v_addr = sbase + L::kV + (t % VST) * kTileBytes;
#pragma unroll
                for (int kk = 0; kk < kBlockN / 16; ++kk) {
                    if (kk == kBlockN / 32) {
                        if (!wait_or_fail(&bars->p_full[a], ia & 1, 5)) return;
                        ptx::tc_fence_after();
                    }
                    ptx::umma_ts(tmem + col_o[a], tmem + col_s[a] + kk * 8,
                                 ptx::sdesc_sw128(v_addr + kk * 16 * 128, kBlockBytes, 1024),
                                 kIdescO, (ia > 0 || kk > 0) ? 1u : 0u);
                }
                if (last) ptx::umma_commit(&bars->o_done[a]);
            };
            if constexpr (kSparse) {
                // lockstep steps: S0_i, PV1_{i-1}, S1_i, PV0_i, a stage is
                // released after its last user's product
                int c0 = j00, c1 = j01, si = 0, spos = 0;
                PairStep prev{};
                bool have_prev = false;
                for (int i = 0; ok && i <= nsteps; ++i) {
                    PairStep st{};
                    if (i < nsteps) {
                        st = next_pair(c0, c1, si, spos);
                        if (st.has0) {
                            if (!wait_or_fail(&bars->k_full[st.pos0 % KST], (st.pos0 / KST) & 1,
                                              4))
                                break;
                            ptx::tc_fence_after();
                            issue_s(0, st.pos0);
                            if (!ok) break;
                            if (!st.shared) ptx::umma_commit(&bars->k_empty[st.pos0 % KST]);
                        }
                    }
                    if (have_prev && prev.has1) {
                        issue_pv(1, prev.pos1, i - 1, i - 1 == n1 - 1);
                        if (!ok) break;
                        ptx::umma_commit(&bars->v_empty[prev.pos1 % VST]);
                    }
                    if (i < nsteps) {
                        if (st.has1) {
                            if (!st.shared) {
                                if (!wait_or_fail(&bars->k_full[st.pos1 % KST],
                                                  (st.pos1 / KST) & 1, 4))
                                    break;
                                ptx::tc_fence_after();
                            }
                            issue_s(1, st.pos1);
                            if (!ok) break;
                            ptx::umma_commit(&bars->k_empty[st.pos1 % KST]);
                        }
                        if (st.has0) {
                            issue_pv(0, st.pos0, i, i == n0 - 1);
                            if (!ok) break;
                            if (!st.shared) ptx::umma_commit(&bars->v_empty[st.pos0 % VST]);
                        }
                    }
                    prev = st;
                    have_prev = i < nsteps;
                }
            } else {
            // a stage is released after its last user's product
            int t = 0, i0 = 0, i1 = 0;                      // stream position, per-tile counts
            int prev_t = 0, prev_i1 = 0, prev_j = -1;       // the previous tile of the stream
            bool prev_u1 = false;
            for (int j = jstart; ok && j <= nt; ++j) {
                bool u0 = false, u1 = false;
                if (j < nt) {
                    u0 = use(0, j);
                    u1 = use(1, j);
                    if (!wait_or_fail(&bars->k_full[t % KST], (t / KST) & 1, 4)) break;
                    ptx::tc_fence_after();
                    if (u0) issue_s(0, t);
                    if (!ok) break;
                }
                if (prev_u1) {
                    issue_pv(1, prev_t, prev_i1, prev_j == last1);
                    if (!ok) break;
                    ptx::umma_commit(&bars->v_empty[prev_t % VST]);
                }
                if (j < nt) {
                    if (u1) issue_s(1, t);
                    if (!ok) break;
                    ptx::umma_commit(&bars->k_empty[t % KST]);
                    if (u0) {
                        issue_pv(0, t, i0, j == last0);
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
            }  // dense / window stream
            if (!ok) {
                // make sure no MMA is still running before TMEM is freed
                int zero = 0;
                volatile int* no_abort = &zero;
                ptx::umma_commit(&bars->drain);
                ptx::mbar_wait(&bars->drain, 0, p.limit_ns, no_abort);
            }
        }
    } else {
        // ================================================= softmax warpgroups
        const int a = warp >> 2;  // which Q tile
        const int nta = a == 0 ? (cnt0 > 0 ? nt0 : 0) : (cnt1 > 0 ? nt1 : 0);
        const int ja = a == 0 ? j00 : j01;  // its first key tile
        const uint32_t quarter = (uint32_t)(warp & 3);
        const uint32_t row = quarter * 32u + (uint32_t)lane;
        const uint32_t lane_addr = (quarter * 32u) << 16;
        const int qa = qbase + a * kBlockM;
        const int i = qa + (int)row;
        int row_lim = Lk - 1;  // last visible key of this row
        if (p.causal) row_lim = min(row_lim, i + Lk - p.Nq);
        // first visible key of this row (the sliding window's lower edge)
        const int row_first = kWindow ? i + qoff - p.window_left : 0;
        const float sl2 = p.scale_log2;
        float m_ref = -INFINITY;  // running reference max, scale*log2 units
        float l_sum = 0.f;        // running sum of exp2(s*sl2 - m_ref)
        bool ok = true;
        const uint32_t t_s = tmem + lane_addr + (a == 0 ? 0u : 128u);
        const uint32_t t_o = tmem + lane_addr + (a == 0 ? 256u : 256u + D);

        int ia = 0;  // key tiles of this Q tile done so far
        int c0 = j00, c1 = j01, si = 0, spos = 0;  // block-sparse schedule
        const int n_iter = kSparse ? (a == 0 ? n0 : n1) : max(0, nta - ja);
        for (int it = 0; it < n_iter; ++it) {
            int j, t;         // key tile, its stream position
            bool first_user;  // this Q tile's P·V is the first to read V_j
            if constexpr (kSparse) {
                const PairStep st = next_pair(c0, c1, si, spos);
                j = a == 0 ? st.x0 : st.x1;
                t = a == 0 ? st.pos0 : st.pos1;
                first_user = a == 0 || !st.shared;
            } else {
                j = ja + it;
                t = j - jstart;
                first_user = a == 0 || !use(0, j);
            }
            if (!warp_wait(&bars->s_full[a], ia & 1, p.limit_ns, abort_flag)) {
                record_error(p.err, kErrFwdBase + 7, &bars->abort);
                ok = false;
                break;
            }
            ptx::tc_fence_after();
            const int key0 = j * kBlockN;
            const bool masked = key0 + kBlockN - 1 > row_lim || (kWindow && key0 < row_first);
            // the chunk-wise path holds warp-collective votes: taken by the
            // whole warp when any of its rows needs the mask (a row that does
            // not finds all its chunks visible, with the same results)
            const bool masked_w = __any_sync(0xffffffffu, masked);
            // pass 1: row maximum, two halves of 64 columns, eight independent
            // chains of three-input maxima
            float mx8[8];
#pragma unroll
            for (int u = 0; u < 8; ++u) mx8[u] = -INFINITY;
            // d = 128 keeps the first half of the row in registers for pass 2
            // (one tensor-memory round trip less per tile; at d = 64 the
            // extra registers cost more than the load)
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
                    if (masked && kWindow)
                        half_max<true, kWindow>(r[hf], key0 + hf * 64, row_first, row_lim, mx8);
                    else if (!kWindow && masked_w)
                        half_max_chunks<false>(r[hf], key0 + hf * 64, row_first, row_lim, mx8);
                    else
                        half_max<false, kWindow>(r[hf], key0 + hf * 64, row_first, row_lim, mx8);
                }
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
            const uint64_t sl2_2 = ptx::f2_pack(sl2, sl2);
            const uint64_t nm_2 = ptx::f2_pack(-m_use, -m_use);
            if (__any_sync(0xffffffffu, rescale)) {
                // the previous P_a V has completed (it precedes S_a_j); done
                // before the exponentials, since the first half of P_a V may
                // start while the second half of P_a is still being formed
                const float s = rescale ? alpha : 1.f;
#pragma unroll 1
                for (int c = 0; c < D / 32; ++c) {
                    uint32_t r[32];
                    ptx::tmem_ld32(t_o + c * 32, r);
                    ptx::tmem_wait_ld_dep(r);
#pragma unroll
                    for (int e = 0; e < 32; ++e) r[e] = __float_as_uint(__uint_as_float(r[e]) * s);
                    ptx::tmem_st32(t_o + c * 32, r);
                }
                ptx::tmem_wait_st();
            }
            ptx::tmem_wait_st();
            // the Q tile whose P·V reads V_j first zeroes its rows behind the
            // real length (Q0 if it uses the tile, else Q1)
            const bool zero_v = p.seqlens_k != nullptr && key0 + kBlockN > Lk && first_user;
            if (zero_v) {
                // keys behind the real length: zero their V rows so that a
                // non-finite value stored there cannot reach O through 0 * NaN
                const int sv = t % VST;
                if (!warp_wait(&bars->v_full[sv], (t / VST) & 1, p.limit_ns, abort_flag)) {
                    record_error(p.err, kErrFwdBase + 8, &bars->abort);
                    ok = false;
                    break;
                }
                if (key0 + (int)row >= Lk) {
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
                constexpr int kKept = D == 128 ? 1 : 0;  // halves kept from pass 1
                uint32_t rl[2][32];
                if (hf >= kKept) {
                    ptx::tmem_ld32(t_s + hf * 64, rl[0]);
                    ptx::tmem_ld32(t_s + hf * 64 + 32, rl[1]);
                    ptx::tmem_wait_ld_dep(rl[0]);
                    ptx::tmem_wait_ld_dep(rl[1]);
                }
                auto& r = hf >= kKept ? rl : rs[hf];
                uint32_t pk[32];
                if (masked && kWindow)
                    half_exp<true, kWindow, BF16, kPolyEvery>(r, key0 + hf * 64, row_first,
                                                              row_lim, sl2_2, nm_2, acc2, pk);
                else if (!kWindow && masked_w)
                    half_exp_chunks<false, BF16, kPolyEvery>(r, key0 + hf * 64, row_first,
                                                             row_lim, sl2_2, nm_2, acc2, pk);
                else
                    half_exp<false, kWindow, BF16, kPolyEvery>(r, key0 + hf * 64, row_first,
                                                               row_lim, sl2_2,
                                                      nm_2, acc2, pk);
                ptx::tmem_st32(t_s + hf * 32, pk);
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

        // ---- epilogue: O / l -> bf16/fp16 -> swizzled staging (the Q_a
        // buffer, free once the last S_a MMA is done) -> TMA store
        if (ok && ia > 0) {
            if (!warp_wait(&bars->o_done[a], 0, p.limit_ns, abort_flag)) {
                record_error(p.err, kErrFwdBase + 9, &bars->abort);
                ok = false;
            }
            ptx::tc_fence_after();
        }
        const bool have = ok && ia > 0 && l_sum > 0.f;
        const float inv_l = have ? 1.f / l_sum : 0.f;
        uint8_t* stage = smem + L::kQ + a * kTileBytes;
        if (qa < p.Nq) {
#pragma unroll
            for (int c = 0; c < D / 32; ++c) {
                uint32_t r[32];
                if (ok && ia > 0) {
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
                // 32 columns = 4 chunks of 16 bytes in block c/2, chunks (c%2)*4..+3
#pragma unroll
                for (int q4 = 0; q4 < 4; ++q4) {
                    const uint32_t ch = (uint32_t)((c & 1) * 4 + q4);
                    *reinterpret_cast<uint4*>(stage + (c >> 1) * kBlockBytes +
                                              sw128_offset(row, ch)) =
                        make_uint4(o2[q4 * 4], o2[q4 * 4 + 1], o2[q4 * 4 + 2], o2[q4 * 4 + 3]);
                }
            }
            ptx::fence_proxy_async_smem();
        }
        ptx::named_barrier_sync(1 + a, 128);
        if (quarter == 0 && lane == 0 && qa < p.Nq) {
            for (int c = 0; c < kDBlocks; ++c)
                ptx::tma_store_4d(&tm_o, stage + c * kBlockBytes, c * 64, h, qa, b);
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
    if (warp == 9) {
        __syncwarp();
        ptx::tc_fence_after();
        ptx::tmem_dealloc<kTmemCols>(tmem);
    }
}

template <int D, bool BF16, int KST, int VST, bool kWindow, bool kSparse>
cudaError_t launch_fwd_w(const FwdMaps& maps, const FwdParams& p, cudaStream_t stream) {
    using L = FwdSmem<D, KST, VST>;
    static_assert(L::kAlloc <= 227 * 1024, "shared memory budget");
    auto kern = attn_fwd_kernel<D, BF16, KST, VST, kWindow, kSparse>;
    cudaError_t e =
        cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)L::kAlloc);
    if (e != cudaSuccess) return e;
    const unsigned n_ctiles = (unsigned)((p.Nq + 2 * kBlockM - 1) / (2 * kBlockM));
    const dim3 grid = p.band > 0 ? dim3((unsigned)p.B * p.Hq * n_ctiles, 1, 1)
                                 : dim3(n_ctiles, p.Hq, p.B);
    kern<<<grid, kThreads, L::kAlloc, stream>>>(maps.q, maps.k, maps.v, maps.o, p);
    return cudaGetLastError();
}

// the sliding-window masks and tile ranges are compiled only into the
// instances that window and block-sparse calls launch; the block-sparse
// instance takes a window that reaches past every key when it has none
template <int D, bool BF16, int KST, int VST>
cudaError_t launch_fwd_t(const FwdMaps& maps, const FwdParams& p, cudaStream_t stream) {
    if (p.bmask.m != nullptr) {
        FwdParams q = p;
        if (q.window_left < 0) q.window_left = kNoWindow;
        return launch_fwd_w<D, BF16, KST, VST, true, true>(maps, q, stream);
    }
    return p.window_left >= 0 ? launch_fwd_w<D, BF16, KST, VST, true, false>(maps, p, stream)
                              : launch_fwd_w<D, BF16, KST, VST, false, false>(maps, p, stream);
}

}  // namespace

cudaError_t launch_fwd(const FwdMaps& maps, const FwdParams& p, int d, bool bf16,
                       cudaStream_t stream) {
    if (d == 64) {
        return bf16 ? launch_fwd_t<64, true, 3, 4>(maps, p, stream)
                    : launch_fwd_t<64, false, 3, 4>(maps, p, stream);
    }
    return bf16 ? launch_fwd_t<128, true, 2, 3>(maps, p, stream)
                : launch_fwd_t<128, false, 2, 3>(maps, p, stream);
}

}  // namespace attn
