// Persistent forward kernel (head dimension 64): O = sigma(alpha Q K^T + b) V
// with key padding masked and padded query rows zeroed (gist.science summary,
// section 2.A; paper.rainbus.top summary, method steps (1)-(3)).
//
// The grid has one CTA per SM, and each CTA works through a
// list of work items.  An item is a pair of 128-row query tiles of one
// (sample, head) that hold at least one valid query row; it streams the key
// and value tiles j < ceil(n_k / 128) through shared memory.  Tiles lying
// wholly in padding never become items: their output rows are zero-filled by
// an otherwise idle warp, without any load (the pages' block-sparse skip,
// paperlayer.ai summary, section 4).
//
// Work order.  Up to 64 samples are ranked by key length (longest first)
// and their items listed in that order (for each sample: its two-tile items
// head by head, then its lone last tiles); CTA c takes the items of the
// list in snake order: c, then 2G-1-c, then 2G+c, ... (G CTAs).  The long
// items are thus spread over all SMs first and the short ones even out the
// rest.  Above 64 samples the items are taken in sample-index order, CTA c
// visiting items c, c+G, ... of the full (sample, tile pair, head) grid and
// skipping those without work.
//
// Warp roles (640 threads):
//   warp 0       TMA producer: Q tiles of each item, then K_j into the key ring
//   warp 2       TMA producer: V_j into the value ring
//   warp 1       owns TMEM and issues every tcgen05.mma, the whole warp running
//                converged (elect.sync picks the issuing lane; issuing from one
//                lane of a diverged warp made the kernel 11-15% slower)
//   warp 3       zero-fills the output rows no item covers
//   warps 4-19   four sigma warpgroups (thread = query row = TMEM lane):
//                warpgroup g serves query tile t = g / 2 of every item, key
//                columns [64 c, 64 c + 64) of each key tile with c = g % 2,
//                then writes columns [c D/2, c D/2 + D/2) of tile t's output.
// Each SM sub-partition thus runs four sigma warps, two per query tile, so
// one tile's sigma work keeps the MUFU busy while the other tile's warps wait
// for their next scores (the MUFU reaches its full rate only with two or more
// warps issuing on a sub-partition).
//
// Units.  The CTA's work is a sequence of units u = (item, key tile j, query
// tile t), t fastest.  Unit u's scores S_u = Q_t K_j^T go to TMEM score buffer
// u mod NB; the sigma warpgroups of tile t turn them into P_u (bf16, two per
// column, over the buffer's columns [0,32) for keys 0-63 and [64,96) for keys
// 64-127), and O_t += P_u V_j reads P_u from TMEM (the TS form), so P never
// touches shared memory.  The MMA thread issues S_{u+NB} right after
// O += P_u V (same buffer; MMAs from one thread run in issue order), so the
// scores of the next NB units are always ready or on their way: the MMA
// runs ahead across key tiles and into the next item while the sigma warps
// work.  TMEM (512 columns): NB score buffers of 128 columns, then O0, O1.
// Each buffer has one "scores ready" barrier per query tile: the two tiles'
// warpgroups each wait only for their own units, and with one barrier per
// buffer a tile that sits out some one-tile items would wait on phases the
// other tile advanced, where a parity wait cannot tell two phases apart.
#pragma once

#include "fwd_sm100.cuh"
#include "sm100.cuh"
#include "sigmoid.cuh"

namespace sigattn {

constexpr int kFwdMaxRanked = 64;   // samples ranked by length (above: index order)

// Key ring slots, value ring slots, TMEM score buffers and query-tile pairs
// held in shared memory (a second pair lets the next item's queries load
// during the current item).  Head dimension 64 only: at 128 the tile kernel
// (fwd_sm100.cuh) runs long sequences faster, and the persistent form's gain
// is on short, ragged batches, which the pages' workloads have at 64.
template <int D> struct FwdCfg {
    static_assert(D == 64, "the persistent forward is built for head dimension 64");
    static constexpr int KS = 4, VS = 4, NB = 3, NQ = 2;
};

// One ranked sample: its index, clamped lengths and the position of its
// first item in the CTA-independent item list.
struct FwdSample {
    int z, nq, nk, start;
};

template <int D>
struct FwdPersistLayout {
    using C = FwdCfg<D>;
    static constexpr int BM = 128;                 // query rows per tile
    static constexpr int BN = 128;                 // keys per tile
    static constexpr int NSUB = D / 64;            // 64-column swizzle atoms per row
    static constexpr int SUB_BYTES = 128 * 64 * 2; // one [128][64] bf16 atom column
    static constexpr int TILE_BYTES = NSUB * SUB_BYTES;
    static constexpr int OFF_Q = 0;
    static constexpr int OFF_K = OFF_Q + C::NQ * 2 * TILE_BYTES;
    static constexpr int OFF_V = OFF_K + C::KS * TILE_BYTES;
    static constexpr int OFF_BAR = OFF_V + C::VS * TILE_BYTES;
    // q_full[NQ], q_empty[NQ], k_full[KS], k_empty[KS], v_full[VS], v_empty[VS],
    // s_full[NB][2], p_full[NB], o_full[2], drain
    static constexpr int NBAR = 2 * C::NQ + 2 * C::KS + 2 * C::VS + 3 * C::NB + 3;
    static constexpr int OFF_TMEM = OFF_BAR + NBAR * 8;
    static constexpr int OFF_ABORT = OFF_TMEM + 8;
    static constexpr int OFF_META = OFF_ABORT + 8;       // item count
    static constexpr int OFF_TABLE = OFF_META + 16;      // FwdSample[kFwdMaxRanked]
    static constexpr int BYTES = OFF_TABLE + kFwdMaxRanked * 16;
    static constexpr int SMEM_ALLOC = BYTES + 1024;  // slack to align the base to 1 KiB
    static constexpr uint32_t TMEM_COLS = 512;
    static constexpr uint32_t COL_O0 = 128 * C::NB, COL_O1 = COL_O0 + D;
    static_assert(COL_O1 + D <= TMEM_COLS, "TMEM budget");
    static_assert(SMEM_ALLOC <= 232448, "shared memory budget");
};

// One work item: query tiles qtile0 and (when ntiles == 2) qtile0 + 1 of
// (z, h), against key tiles 0..nkv-1.
struct FwdItem {
    int z, h, qtile0, ntiles, nkv, nq, nk;
};

// The CTA's walk over its items, in the order described at the top.  Every
// role runs its own copy; all copies see the same sequence.
struct FwdWalk {
    const FwdParams *p;
    const FwdSample *table;   // ranked samples (shared memory)
    int total;                // ranked: items in the list; index order: grid size
    bool ranked;
    int step;

    __device__ __forceinline__ bool next(FwdItem &it) {
        const int G = static_cast<int>(gridDim.x), c = static_cast<int>(blockIdx.x);
        if (ranked) {
            const int m = step * G + ((step & 1) ? G - 1 - c : c);
            ++step;
            if (m >= total) return false;
            // the last ranked sample whose first item is at or before m
            // (samples without items share the next one's start)
            int lo = 0, hi = p->Z - 1;
            while (lo < hi) {
                const int mid = (lo + hi + 1) >> 1;
                if (table[mid].start <= m) lo = mid; else hi = mid - 1;
            }
            const FwdSample s = table[lo];
            const int local = m - s.start;
            it.z = s.z;
            it.nq = s.nq;
            it.nk = s.nk;
            // the sample's two-tile items first, head major (CTAs that run at
            // the same time then share the key and value tiles of few heads in
            // L2), then its lone last tiles, one per head
            const int nfull = (s.nq + 127) / 256;        // pairs whose both tiles hold a valid row
            if (local < p->H * nfull) {
                it.h = local / nfull;
                it.qtile0 = 2 * (local - it.h * nfull);
            } else {
                it.h = local - p->H * nfull;
                it.qtile0 = 2 * nfull;
            }
        } else {
            const int per = p->H * ((p->Lq + 255) / 256);   // items per sample
            for (;;) {
                const int k = c + step * G;
                ++step;
                if (k >= total) return false;
                const int z = k / per, rem = k - z * per;
                int nq = p->seqlens_q[z], nk = p->seqlens_k[z];
                if (nq < 0 || nq > p->Lq || nk < 0 || nk > p->Lk) {
                    if ((threadIdx.x & 31) == 0) record_status(p->status, kStatusSeqlenRange);
                    nq = min(max(nq, 0), p->Lq);
                    nk = min(max(nk, 0), p->Lk);
                }
                const int qt = 2 * (rem / p->H);
                if (qt * 128 >= nq || nk == 0) continue;   // no work in this item
                it.z = z;
                it.nq = nq;
                it.nk = nk;
                it.h = rem % p->H;
                it.qtile0 = qt;
                break;
            }
        }
        it.ntiles = ((it.qtile0 + 1) * 128 < it.nq) ? 2 : 1;
        it.nkv = (it.nk + 127) / 128;
        return true;
    }
};

// Unit cursor: (item, key tile j, query tile t), t fastest.  Besides the
// position it keeps, updated step by step, the ring slot and phase bit of
// everything the unit touches: its score buffer (u mod NB), K_j and V_j
// (their (item, j) index mod KS and mod VS) and the item's query tiles
// (item index mod NQ), so the issuing thread does no division per unit.
template <int NB, int NQ, int KS, int VS>
struct FwdUnits {
    FwdWalk walk;
    FwdItem it;
    bool live;
    int j, t;
    int buf, bph;   // score buffer and the phase parity of its barriers
    int ks, kph;    // key ring slot and phase
    int vs, vph;    // value ring slot and phase
    int qs, qph;    // query-tile pair slot and phase

    __device__ __forceinline__ void start() {
        j = t = buf = bph = ks = kph = vs = vph = qs = qph = 0;
        live = walk.next(it);
    }
    __device__ __forceinline__ void advance() {
        if (++buf == NB) {
            buf = 0;
            bph ^= 1;
        }
        if (++t < it.ntiles) return;
        t = 0;
        if (++ks == KS) {
            ks = 0;
            kph ^= 1;
        }
        if (++vs == VS) {
            vs = 0;
            vph ^= 1;
        }
        if (++j < it.nkv) return;
        j = 0;
        if (++qs == NQ) {
            qs = 0;
            qph ^= 1;
        }
        live = walk.next(it);
    }
};

template <int D, int MODE>
__global__ void __launch_bounds__(kFwdThreads, 1)
    fwd_persistent_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
               const __grid_constant__ CUtensorMap tmV, const __grid_constant__ FwdParams p) {
    using Lay = FwdPersistLayout<D>;
    using Cfg = FwdCfg<D>;
    constexpr int NB = Cfg::NB, NQ = Cfg::NQ, KS = Cfg::KS, VS = Cfg::VS;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = align_1k(smem_raw);
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + Lay::OFF_BAR);
    uint64_t *q_full = bars;
    uint64_t *q_empty = q_full + NQ;
    uint64_t *k_full = q_empty + NQ;
    uint64_t *k_empty = k_full + KS;
    uint64_t *v_full = k_empty + KS;
    uint64_t *v_empty = v_full + VS;
    uint64_t *s_full = v_empty + VS;   // [buffer][tile]: the tile's scores are in the buffer
    uint64_t *p_full = s_full + 2 * NB;
    uint64_t *o_full = p_full + NB;
    uint64_t *drain = o_full + 2;
    static_assert(2 * NQ + 2 * KS + 2 * VS + 3 * NB + 3 == Lay::NBAR, "barrier count");
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + Lay::OFF_TMEM);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + Lay::OFF_ABORT);
    int *meta = reinterpret_cast<int *>(smem + Lay::OFF_META);
    FwdSample *table = reinterpret_cast<FwdSample *>(smem + Lay::OFF_TABLE);

    const int warp = warp_id(), lane = lane_id();
    cta_log(0, globaltimer_ns());
    const bool ranked = p.Z <= kFwdMaxRanked;
    if (warp == 0) {
        // ranks samples by decreasing key length (0 when the sample has no
        // query), ties by index; lane l holds samples l and l + 32
        if (ranked) {
            int nq[2], nk[2], w[2], rank[2] = {0, 0};
#pragma unroll
            for (int c = 0; c < 2; ++c) {
                const int i = lane + 32 * c;
                nq[c] = i < p.Z ? p.seqlens_q[i] : 0;
                nk[c] = i < p.Z ? p.seqlens_k[i] : 0;
                if (i < p.Z && (nq[c] < 0 || nq[c] > p.Lq || nk[c] < 0 || nk[c] > p.Lk)) {
                    record_status(p.status, kStatusSeqlenRange);
                    nq[c] = min(max(nq[c], 0), p.Lq);
                    nk[c] = min(max(nk[c], 0), p.Lk);
                }
                w[c] = nq[c] > 0 ? nk[c] : 0;
            }
            for (int j = 0; j < p.Z; ++j) {
                const int wj = __shfl_sync(0xffffffffu, j < 32 ? w[0] : w[1], j & 31);
#pragma unroll
                for (int c = 0; c < 2; ++c) rank[c] += ranks_before(wj, j, w[c], lane + 32 * c);
            }
#pragma unroll
            for (int c = 0; c < 2; ++c)
                if (lane + 32 * c < p.Z) table[rank[c]] = FwdSample{lane + 32 * c, nq[c], nk[c], 0};
            __syncwarp();
            if (lane == 0) {
                // items per sample: one per (query-tile pair with a valid row, head)
                int start = 0;
                for (int r = 0; r < p.Z; ++r) {
                    table[r].start = start;
                    if (table[r].nq > 0 && table[r].nk > 0)
                        start += p.H * ((table[r].nq + 255) / 256);
                }
                meta[0] = start;
            }
        } else if (lane == 0) {
            meta[0] = p.Z * p.H * ((p.Lq + 255) / 256);
        }
    }
    if (threadIdx.x == 0) {
        for (int s = 0; s < NQ; ++s) {
            mbar_init(&q_full[s], 1);
            mbar_init(&q_empty[s], 1);
        }
        for (int s = 0; s < KS; ++s) {
            mbar_init(&k_full[s], 1);
            mbar_init(&k_empty[s], 1);
        }
        for (int s = 0; s < VS; ++s) {
            mbar_init(&v_full[s], 1);
            mbar_init(&v_empty[s], 1);
        }
        for (int b = 0; b < NB; ++b) {
            mbar_init(&s_full[2 * b], 1);
            mbar_init(&s_full[2 * b + 1], 1);
            mbar_init(&p_full[b], 256);  // the two sigma warpgroups of the unit's tile
        }
        mbar_init(&o_full[0], 1);
        mbar_init(&o_full[1], 1);
        mbar_init(drain, 1);
        *abort_flag = 0;
        fence_barrier_init();
    }
    if (warp == 0 && lane == 0) {
        prefetch_tensormap(&tmQ);
        prefetch_tensormap(&tmK);
        prefetch_tensormap(&tmV);
    }
    if (warp == 1) {
        tmem_alloc(tmem_slot, Lay::TMEM_COLS);
        tmem_relinquish();
        tc_fence_before();
    }
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    const WaitCtx wctx{abort_flag, p.status, p.timeout_ns};
    const FwdWalk walk0{&p, table, meta[0], ranked, 0};
    const size_t row_stride = static_cast<size_t>(p.H) * D;

    if (warp == 0) {
        // ------------------------------------------------------------ Q and K producer
        if (lane == 0) {
            uint8_t *sQ = smem + Lay::OFF_Q;
            uint8_t *sK = smem + Lay::OFF_K;
            FwdWalk walk = walk0;
            FwdItem it;
            int n = 0, jk = 0;
            bool ok = true;
            while (ok && walk.next(it)) {
                const int qs = n % NQ;
                if (n >= NQ && !(ok = mbar_wait(&q_empty[qs], ((n / NQ) - 1) & 1, wctx))) break;
                mbar_arrive_expect_tx(&q_full[qs], it.ntiles * Lay::TILE_BYTES);
                for (int t = 0; t < it.ntiles; ++t)
                    for (int s = 0; s < Lay::NSUB; ++s)
                        tma_load_4d(&tmQ, &q_full[qs],
                                    sQ + (qs * 2 + t) * Lay::TILE_BYTES + s * Lay::SUB_BYTES, 64 * s,
                                    it.h, (it.qtile0 + t) * Lay::BM, it.z);
                ++n;
                for (int j = 0; j < it.nkv; ++j, ++jk) {
                    const int sk = jk % KS;
                    if (jk >= KS && !(ok = mbar_wait(&k_empty[sk], ((jk / KS) - 1) & 1, wctx))) break;
                    mbar_arrive_expect_tx(&k_full[sk], Lay::TILE_BYTES);
                    for (int s = 0; s < Lay::NSUB; ++s)
                        tma_load_4d(&tmK, &k_full[sk], sK + sk * Lay::TILE_BYTES + s * Lay::SUB_BYTES,
                                    64 * s, it.h, j * Lay::BN, it.z);
                    trace(0, jk, 0);
                    cta_log_any(2, (static_cast<unsigned long long>(n) << 32) | static_cast<uint32_t>(jk + 1));
                }
            }
            // Every issued load must land before the CTA's shared memory is released.
            for (int i = (n > NQ ? n - NQ : 0); i < n; ++i)
                mbar_wait_drain(&q_full[i % NQ], (i / NQ) & 1, p.timeout_ns);
            for (int i = (jk > KS ? jk - KS : 0); i < jk; ++i)
                mbar_wait_drain(&k_full[i % KS], (i / KS) & 1, p.timeout_ns);
        }
    } else if (warp == 2) {
        // ------------------------------------------------------------ V producer
        // V_j is released later than K_j, so its ring is fed by its own thread
        // and never waits behind a key slot.
        if (lane == 0) {
            uint8_t *sV = smem + Lay::OFF_V;
            FwdWalk walk = walk0;
            FwdItem it;
            int jv = 0;
            bool ok = true;
            while (ok && walk.next(it)) {
                for (int j = 0; j < it.nkv; ++j, ++jv) {
                    const int sv = jv % VS;
                    if (jv >= VS && !(ok = mbar_wait(&v_empty[sv], ((jv / VS) - 1) & 1, wctx))) break;
                    mbar_arrive_expect_tx(&v_full[sv], Lay::TILE_BYTES);
                    for (int s = 0; s < Lay::NSUB; ++s)
                        tma_load_4d(&tmV, &v_full[sv], sV + sv * Lay::TILE_BYTES + s * Lay::SUB_BYTES,
                                    64 * s, it.h, j * Lay::BN, it.z);
                    trace(0, jv, 1);
                    cta_log_any(3, static_cast<uint32_t>(jv + 1));
                }
            }
            for (int i = (jv > VS ? jv - VS : 0); i < jv; ++i)
                mbar_wait_drain(&v_full[i % VS], (i / VS) & 1, p.timeout_ns);
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer
        {
            // the whole warp runs converged; elect.sync picks the issuing lane
            auto wt = [&](uint64_t *bar, uint32_t parity) {
                return __all_sync(0xffffffffu, mbar_wait(bar, parity, wctx));
            };
            using Units = FwdUnits<NB, NQ, KS, VS>;
            const uint32_t idesc_s = idesc_bf16_f32(128, Lay::BN, false, false);
            const uint32_t idesc_o = idesc_bf16_f32(128, D, false, true);
            constexpr uint32_t hi = desc_hi(1024);
            // low descriptor words of slot 0 of each operand region; a slot
            // further on adds its byte offset >> 4
            const uint32_t q_lo = desc_lo(smem_u32(smem + Lay::OFF_Q), 16);
            const uint32_t k_lo = desc_lo(smem_u32(smem + Lay::OFF_K), 16);
            const uint32_t v_lo = desc_lo(smem_u32(smem + Lay::OFF_V), Lay::SUB_BYTES);
            constexpr uint32_t kTile = Lay::TILE_BYTES >> 4;
            bool ok = true;
            // S of unit `sc` into its score buffer: waits for the item's
            // queries at its first unit and for K_j at the first tile of j;
            // releases K_j after the last tile of j and the queries after the
            // item's last unit.
            auto issue_s = [&](const Units &sc) -> bool {
                if (sc.j == 0 && sc.t == 0 && !wt(&q_full[sc.qs], sc.qph)) return false;
                if (sc.t == 0 && !wt(&k_full[sc.ks], sc.kph)) return false;
                tc_fence_after();
                const uint32_t a_lo = q_lo + (sc.qs * 2 + sc.t) * kTile;
                const uint32_t b_lo = k_lo + sc.ks * kTile;
                const uint32_t d_tmem = tmem + 128 * sc.buf;
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk) {
                    const uint32_t koff = ((kk >> 2) * Lay::SUB_BYTES + (kk & 3) * 32) >> 4;
                    mma_ss_lhw(d_tmem, a_lo + koff, b_lo + koff, hi, idesc_s, kk > 0 ? 1u : 0u);
                }
                mma_commit_w(&s_full[2 * sc.buf + sc.t]);
                if (sc.t == sc.it.ntiles - 1) {
                    mma_commit_w(&k_empty[sc.ks]);
                    if (sc.j == sc.it.nkv - 1) mma_commit_w(&q_empty[sc.qs]);
                }
                return true;
            };
            Units sc{walk0}, pc{walk0};
            sc.start();
            pc.start();
            for (int b = 0; ok && b < NB && sc.live; ++b) {
                ok = issue_s(sc);
                sc.advance();
            }
            int kvt = 0;   // (item, key tile) pairs passed, for the timeline trace
            while (ok && pc.live) {
                if (pc.t == 0 && !(ok = wt(&v_full[pc.vs], pc.vph))) break;
                if (pc.t == 0) trace(1, kvt, 0);
                if (!(ok = wt(&p_full[pc.buf], pc.bph))) break;
                trace(1, kvt, 1 + 3 * pc.t);
                tc_fence_after();
                // O_t += P_u V_j, P_u read from TMEM (16 keys = 8 packed columns per
                // step; keys 64-127 sit 32 columns further on)
                const uint32_t d_tmem = tmem + (pc.t ? Lay::COL_O1 : Lay::COL_O0);
                const uint32_t a_tmem = tmem + 128 * pc.buf;
                const uint32_t b_lo = v_lo + pc.vs * kTile;
#pragma unroll
                for (int kk = 0; kk < Lay::BN / 16; ++kk)
                    mma_ts_lhw(d_tmem, a_tmem + kk * 8 + (kk >= 4 ? 32 : 0), b_lo + kk * 128, hi,
                              idesc_o, (pc.j > 0 || kk > 0) ? 1u : 0u);
                trace(1, kvt, 2 + 3 * pc.t);
                if (pc.t == pc.it.ntiles - 1) mma_commit_w(&v_empty[pc.vs]);
                if (pc.j == pc.it.nkv - 1) mma_commit_w(&o_full[pc.t]);   // O_t of this item done
                // the scores NB units ahead go into the buffer P_u was just read from
                if (sc.live) {
                    if (!(ok = issue_s(sc))) break;
                    sc.advance();
                }
                trace(1, kvt, 3 + 3 * pc.t);
                if (pc.t == pc.it.ntiles - 1) ++kvt;
                pc.advance();
            }
            // No MMA may still be running when TMEM is released.
            mma_commit_w(drain);
            mbar_wait_drain(drain, 0, p.timeout_ns);
            __syncwarp();
        }
    } else if (warp == 3) {
        // ------------------------------------------------------------ zero fill
        // Output rows that no item covers: rows at or beyond ceil(n_q / 128) * 128
        // of every (sample, head), or all rows when the sample has no query or
        // no key.  Blocks of 128 rows are spread over the CTAs; whole rows of
        // zeros, 16 bytes per lane.
        const int nblk = (p.Lq + 127) / 128;
        const int64_t total = static_cast<int64_t>(p.Z) * p.H * nblk;
        constexpr int V4 = D / 8;   // 16-byte chunks per row
        for (int64_t b = blockIdx.x; b < total; b += gridDim.x) {
            const int z = static_cast<int>(b / (static_cast<int64_t>(p.H) * nblk));
            const int rem = static_cast<int>(b - static_cast<int64_t>(z) * p.H * nblk);
            const int h = rem / nblk, blk = rem - h * nblk;
            const int nq = min(max(p.seqlens_q[z], 0), p.Lq), nk = min(max(p.seqlens_k[z], 0), p.Lk);
            const int covered = (nq > 0 && nk > 0) ? ((nq + 127) / 128) * 128 : 0;
            if (blk * 128 < covered) continue;
            const int r0 = blk * 128, rows = min(128, p.Lq - r0);
            for (int e = lane; e < rows * V4; e += 32) {
                const int r = r0 + e / V4, c = e % V4;
                uint4 *dst = reinterpret_cast<uint4 *>(
                    p.o + (static_cast<size_t>(z) * p.Lq + r) * row_stride + static_cast<size_t>(h) * D);
                dst[c] = make_uint4(0u, 0u, 0u, 0u);
            }
        }
    } else {
        // ------------------------------------------------------------ sigma warpgroups
        // Warpgroup g works on query tile t = g / 2 of every item, on key
        // columns [64 c, 64 c + 64) of the tile's scores (c = g % 2).  The
        // warpgroups of the two tiles run side by side on every SM
        // sub-partition: while one tile's warps wait for their next scores,
        // the other tile's warps keep the MUFU busy.
        const int g = (warp - 4) >> 2;
        const int t = g >> 1, c = g & 1;
        const int quarter = warp & 3;  // TMEM lane quarter this warp may access
        const uint32_t lane_bits = static_cast<uint32_t>(quarter * 32) << 16;
        constexpr int HALF = D / 2;
        FwdWalk walk = walk0;
        FwdItem it;
        int u = 0, no = 0;   // units passed; items in which this tile took part
        int kvg = 0;         // (item, key tile) pairs passed
        // this tile's units so far in each score buffer: the phase of that
        // buffer's score barrier for this tile (each tile has its own barrier
        // per buffer, so a tile that sits out some items never falls behind a
        // barrier that the other tile keeps advancing)
        int used[NB];
#pragma unroll
        for (int b = 0; b < NB; ++b) used[b] = 0;
        bool ok = true;
        while (ok && walk.next(it)) {
            const SigmoidCoef cf = make_coef<MODE>(p.alpha, bias_of(p.bias_z, p.bias, it.z));
            const bool mine = t < it.ntiles;
            for (int j = 0; j < it.nkv; ++j) {
                if (mine) {
                    const int uu = u + t, buf = uu % NB;
                    int phase = 0;
#pragma unroll
                    for (int b = 0; b < NB; ++b)
                        if (b == buf) phase = used[b]++;
                    if (quarter == 0) trace(2 + c, kvg, 2 * t);
                    ok = __all_sync(0xffffffffu, mbar_wait(&s_full[2 * buf + t], phase & 1, wctx));
                    if (!ok) break;
                    trace(4 + quarter, kvg, 4 + 2 * t + c);
                    tc_fence_after();
                    const uint32_t tS = tmem + lane_bits + 128 * buf + 64 * c;
                    const int kvalid = it.nk - j * Lay::BN - 64 * c;  // keys of this half below n_k
                    // two chunks of 32 scores per thread; P of chunk v lies over S
                    // columns [16 v, 16 v + 16) of this half, already read
#pragma unroll
                    for (int v = 0; v < 2; ++v) {
                        uint32_t r[32];
                        tmem_ld32(tS + 32 * v, r);
                        uint32_t pk[16];
#pragma unroll
                        for (int i = 0; i < 16; ++i) {
                            const float2 pr = sigma2<MODE>(
                                scale2(__uint_as_float(r[2 * i]), __uint_as_float(r[2 * i + 1]), cf));
                            pk[i] = pack_bf16x2(pr.x, pr.y);
                        }
                        if (kvalid < 64) {
                            // last key tile: keys at or beyond n_k weigh exactly zero
#pragma unroll
                            for (int i = 0; i < 16; ++i) {
                                const int col = 32 * v + 2 * i;
                                const uint32_t lo = col < kvalid ? 0x0000FFFFu : 0u;
                                const uint32_t hi = col + 1 < kvalid ? 0xFFFF0000u : 0u;
                                pk[i] &= (lo | hi);
                            }
                        }
                        tmem_st16(tS + 16 * v, pk);
                    }
                    tmem_wait_st();
                    tc_fence_before();
                    mbar_arrive(&p_full[buf]);
                    if (quarter == 0) trace(2 + c, kvg, 4 + t);
                    trace(4 + quarter, kvg, 2 * t + c);
                    if (quarter == 0 && c == 0 && lane == 0) cta_log_any(6 + t, static_cast<uint32_t>(uu + 1));
                }
                u += it.ntiles;
                ++kvg;
            }
            if (!ok || !mine) continue;
            // epilogue: columns [c D/2, c D/2 + D/2) of query tile t, once every
            // P.V of the tile in this item has finished
            ok = __all_sync(0xffffffffu, mbar_wait(&o_full[t], no & 1, wctx));
            ++no;
            if (!ok) break;
            tc_fence_after();
            const int row = (it.qtile0 + t) * Lay::BM + quarter * 32 + lane;
            __nv_bfloat16 *orow = p.o + (static_cast<size_t>(it.z) * p.Lq + row) * row_stride +
                                  static_cast<size_t>(it.h) * D + c * HALF;
            const uint32_t tO = tmem + lane_bits + (t ? Lay::COL_O1 : Lay::COL_O0) + c * HALF;
            const bool valid = row < it.nq;
#pragma unroll
            for (int cc = 0; cc < HALF / 32; ++cc) {
                uint32_t r[32];
                tmem_ld32(tO + 32 * cc, r);
                if (row < p.Lq) {
                    uint4 *dst = reinterpret_cast<uint4 *>(orow + 32 * cc);
#pragma unroll
                    for (int v4 = 0; v4 < 4; ++v4) {
                        uint4 w;
                        w.x = valid ? pack_bf16x2(__uint_as_float(r[8 * v4 + 0]), __uint_as_float(r[8 * v4 + 1])) : 0u;
                        w.y = valid ? pack_bf16x2(__uint_as_float(r[8 * v4 + 2]), __uint_as_float(r[8 * v4 + 3])) : 0u;
                        w.z = valid ? pack_bf16x2(__uint_as_float(r[8 * v4 + 4]), __uint_as_float(r[8 * v4 + 5])) : 0u;
                        w.w = valid ? pack_bf16x2(__uint_as_float(r[8 * v4 + 6]), __uint_as_float(r[8 * v4 + 7])) : 0u;
                        dst[v4] = w;
                    }
                }
            }
            // The next item's O_t += P V waits for this warpgroup's next P, which
            // comes after these loads: the accumulator is never overwritten early.
            tc_fence_before();
        }
    }

    // every warp converges before the block-wide barrier (the producer and MMA
    // roles ran on one lane)
    __syncwarp();
    __syncthreads();
    cta_log(1, globaltimer_ns());
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, Lay::TMEM_COLS);
    }
}

}  // namespace sigattn
