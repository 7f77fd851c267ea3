// Persistent backward kernels (head dimension 64): the dQ and dK/dV passes of
// bwd_sm100.cuh (paper.rainbus.top summary, method steps (4)-(5); paperlayer.ai
// summary, section 4: one kernel per output, no atomics), run by one CTA per
// SM over a list of work items instead of one CTA per tile.
//
// An item is one 128-row tile of this kernel's rows (dQ: query tiles, dK/dV:
// key tiles) of one (sample, head) that has work: at least one valid row and a
// non-empty other side.  It streams the other side's tiles j < ceil(n / 128)
// (dQ: K_j and V_j; dK/dV: Q_j and dO_j) exactly as the tile kernels do, with
// the same sigma warpgroups and the same TMEM plan.  Tiles without work never
// become items: their output rows are zero-filled by warp 3, which the tile
// kernels leave idle, so the CTA launches, barrier set-up and tensor-memory
// allocation that empty tiles cost the tile kernels are gone (the pages'
// block-sparse skip of padded tiles, paperlayer.ai summary, section 4).
//
// Work order.  Up to 64 samples are ranked by the cost of their items (the
// other side's length; 0 when either side is empty), longest first, and their
// items listed in that order, head by head (CTAs that run at the same time
// then stream the tiles of few heads, which stay in L2); CTA c takes the
// list's items in snake order c, 2G-1-c, 2G+c, ... (G CTAs).  Above 64
// samples the CTAs visit the full (sample, head, tile) grid in index order
// (c, c+G, ...) and skip the tiles without work.
//
// Units.  The CTA's work is one stream of units u = (item, j): ring slots and
// hand-off barrier phases run on from one item into the next, so the MMA
// thread issues the first scores of item k+1 while the warpgroups finish item
// k.  The resident tiles of consecutive items (dQ: Q and dO; dK/dV: K and V)
// alternate between two shared-memory slots: res_full[k % 2] tells the MMA
// thread that item k's tiles are in, and res_empty[k % 2], committed after
// the item's last MMA, lets the producer load item k+2's.  After an item's
// last unit the MMA thread commits acc_full; the warpgroups then read the
// item's accumulators and store them.  The next item's first accumulating
// MMA (which overwrites them) is issued only after every warpgroup's next
// readiness arrival, which comes after those reads.  The protocol (phases,
// slots, hand-offs) is model-checked on the host in test_barrier_protocols.py.
#pragma once

#include "bwd_sm100.cuh"
#include "sm100.cuh"
#include "sigmoid.cuh"

namespace sigattn {

constexpr int kBwdMaxRanked = 64;   // samples ranked by cost (above: index order)

// Shared memory: two slots of the two resident tiles, the X ring (dQ: K_j;
// dK/dV: Q_j) and the Y ring (dQ: V_j; dK/dV: dO_j), barriers, the sample
// table.
template <int D>
struct BwdPersistLayout {
    static_assert(D == 64, "the persistent backward is built for head dimension 64");
    static constexpr int SX = 4, SY = 4, NR = 2;
    static constexpr int NSUB = D / 64;
    static constexpr int SUB_BYTES = 128 * 64 * 2;
    static constexpr int TILE_BYTES = NSUB * SUB_BYTES;
    static constexpr int OFF_R = 0;                                   // [NR][2] resident tiles
    static constexpr int OFF_X = OFF_R + NR * 2 * TILE_BYTES;
    static constexpr int OFF_Y = OFF_X + SX * TILE_BYTES;
    static constexpr int OFF_BAR = OFF_Y + SY * TILE_BYTES;
    // x_full[SX], x_empty[SX], y_full[SY], y_empty[SY], res_full[NR],
    // res_empty[NR], then up to MAX_HANDOFF hand-off barriers
    static constexpr int MAX_HANDOFF = 8;
    static constexpr int NBAR = 2 * SX + 2 * SY + 2 * NR + MAX_HANDOFF;
    static constexpr int OFF_TMEM = OFF_BAR + NBAR * 8;
    static constexpr int OFF_ABORT = OFF_TMEM + 8;
    static constexpr int OFF_RED = OFF_ABORT + 8;          // 16 floats: per-warp db partials
    static constexpr int OFF_META = OFF_RED + 64;          // item count
    static constexpr int OFF_TABLE = OFF_META + 16;        // BwdSample[kBwdMaxRanked]
    static constexpr int SMEM_ALLOC = OFF_TABLE + kBwdMaxRanked * 16 + 1024;
    static constexpr uint32_t TMEM_COLS = 512;
    static_assert(SMEM_ALLOC <= 232448, "shared memory budget");
};

// One ranked sample: its index, clamped lengths on this kernel's side (self)
// and the other side, and the position of its first item in the list.
struct BwdSample {
    int z, nself, nother, start;
};

// One work item: tile `tile` of (z, h) on this kernel's side, against the
// other side's tiles 0..nsteps-1.
struct BwdItem {
    int z, h, tile, nself, nother, nsteps;
};

// Lengths of sample z on this kernel's side and the other, clamped to the
// padded lengths (an out-of-range length is recorded in the status word).
__device__ __forceinline__ void bwd_lengths(const BwdParams &p, bool rows_are_queries, int z, int &nself,
                                            int &nother) {
    int nq = p.seqlens_q[z], nk = p.seqlens_k[z];
    if (nq < 0 || nq > p.Lq || nk < 0 || nk > p.Lk) {
        record_status(p.status, kStatusSeqlenRange);
        nq = min(max(nq, 0), p.Lq);
        nk = min(max(nk, 0), p.Lk);
    }
    nself = rows_are_queries ? nq : nk;
    nother = rows_are_queries ? nk : nq;
}

// Warp 0 of the CTA: ranks up to kBwdMaxRanked samples by item cost into
// `table` and writes the item count to meta[0] (above kBwdMaxRanked samples:
// the size of the full grid).  Lane l holds samples l and l + 32.
__device__ __forceinline__ void bwd_build_table(const BwdParams &p, bool rows_are_queries, BwdSample *table,
                                                int *meta) {
    const int lane = lane_id();
    const int Lself = rows_are_queries ? p.Lq : p.Lk;
    if (p.Z > kBwdMaxRanked) {
        if (lane == 0) meta[0] = p.Z * p.H * ((Lself + 127) / 128);
        return;
    }
    int ns[2], no[2], w[2], rank[2] = {0, 0};
#pragma unroll
    for (int c = 0; c < 2; ++c) {
        const int i = lane + 32 * c;
        ns[c] = no[c] = 0;
        if (i < p.Z) bwd_lengths(p, rows_are_queries, i, ns[c], no[c]);
        w[c] = ns[c] > 0 ? no[c] : 0;
    }
    for (int j = 0; j < p.Z; ++j) {
        const int wj = __shfl_sync(0xffffffffu, j < 32 ? w[0] : w[1], j & 31);
#pragma unroll
        for (int c = 0; c < 2; ++c) rank[c] += ranks_before(wj, j, w[c], lane + 32 * c);
    }
#pragma unroll
    for (int c = 0; c < 2; ++c)
        if (lane + 32 * c < p.Z) table[rank[c]] = BwdSample{lane + 32 * c, ns[c], no[c], 0};
    __syncwarp();
    if (lane == 0) {
        // items per sample: one per (tile with a valid row, head)
        int start = 0;
        for (int r = 0; r < p.Z; ++r) {
            table[r].start = start;
            if (table[r].nself > 0 && table[r].nother > 0) start += p.H * ((table[r].nself + 127) / 128);
        }
        meta[0] = start;
    }
    __syncwarp();
}

// The CTA's walk over its items, in the order described at the top.  Every
// role runs its own copy; all copies see the same sequence.
struct BwdWalk {
    const BwdParams *p;
    const BwdSample *table;   // ranked samples (shared memory)
    int total;                // ranked: items in the list; index order: grid size
    bool ranked, rows_are_queries;
    int step;

    __device__ __forceinline__ bool next(BwdItem &it) {
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
            const BwdSample s = table[lo];
            const int ntl = (s.nself + 127) / 128;
            const int local = m - s.start;
            it.z = s.z;
            it.nself = s.nself;
            it.nother = s.nother;
            it.h = local / ntl;
            it.tile = local - it.h * ntl;
        } else {
            const int ntl = ((rows_are_queries ? p->Lq : p->Lk) + 127) / 128;
            const int per = p->H * ntl;   // tiles per sample
            for (;;) {
                const int k = c + step * G;
                ++step;
                if (k >= total) return false;
                const int z = k / per, rem = k - z * per;
                int ns, no;
                bwd_lengths(*p, rows_are_queries, z, ns, no);
                const int h = rem / ntl, tile = rem - h * ntl;
                if (tile * 128 >= ns || no == 0) continue;   // no work in this tile
                it.z = z;
                it.h = h;
                it.tile = tile;
                it.nself = ns;
                it.nother = no;
                break;
            }
        }
        it.nsteps = (it.nother + 127) / 128;
        return true;
    }
};

// Unit cursor: (item k, step j) with the unit count u and the ring slot and
// phase of unit u's X and Y tiles, updated step by step.
template <int SX, int SY>
struct BwdUnits {
    BwdWalk walk;
    BwdItem it;
    bool live;
    int k, j, u;
    int xs, xph, ys, yph;

    __device__ __forceinline__ void start() {
        k = j = u = xs = xph = ys = yph = 0;
        live = walk.next(it);
    }
    __device__ __forceinline__ bool last() const { return j == it.nsteps - 1; }
    __device__ __forceinline__ void advance() {
        ++u;
        if (++xs == SX) {
            xs = 0;
            xph ^= 1;
        }
        if (++ys == SY) {
            ys = 0;
            yph ^= 1;
        }
        if (++j < it.nsteps) return;
        j = 0;
        ++k;
        live = walk.next(it);
    }
};

// Streams one ring (S slots) over every item of the walk, after the resident
// tiles of each item when `res` is set.  The whole warp runs it converged: all
// lanes wait, lane 0 arms the barrier and issues the copies (0.5-1% faster
// than one lane of a diverged warp).  `issued` receives the ring loads
// issued and `res_n` the resident loads issued (both stop early when a wait
// gives up), for the drain before the CTA exits.
template <int S, int NSUB>
__device__ __forceinline__ void bwd_persistent_producer(const CUtensorMap *map, uint64_t *full, uint64_t *empty,
                                                        uint8_t *ring, int tile_bytes, BwdWalk walk,
                                                        const CUtensorMap *res_a, const CUtensorMap *res_b,
                                                        uint64_t *res_full, uint64_t *res_empty, uint8_t *res,
                                                        const WaitCtx &wctx, int &issued, int &res_n) {
    constexpr int SUB = 128 * 64 * 2;
    const bool leader = lane_id() == 0;
    BwdItem it;
    int q = 0, k = 0;
    bool ok = true;
    while (ok && walk.next(it)) {
        if (res != nullptr) {
            const int rs = k & 1;
            if (k >= 2 && !(ok = __all_sync(0xffffffffu, mbar_wait(&res_empty[rs], ((k >> 1) - 1) & 1, wctx))))
                break;
            if (leader) {
                mbar_arrive_expect_tx(&res_full[rs], 2 * tile_bytes);
                for (int s = 0; s < NSUB; ++s) {
                    tma_load_4d(res_a, &res_full[rs], res + (2 * rs) * tile_bytes + s * SUB, 64 * s, it.h,
                                it.tile * 128, it.z);
                    tma_load_4d(res_b, &res_full[rs], res + (2 * rs + 1) * tile_bytes + s * SUB, 64 * s, it.h,
                                it.tile * 128, it.z);
                }
            }
            __syncwarp();
            ++k;
        }
        for (int j = 0; j < it.nsteps; ++j) {
            const int st = q % S;
            if (q >= S && !(ok = __all_sync(0xffffffffu, mbar_wait(&empty[st], ((q / S) - 1) & 1, wctx)))) break;
            if (leader) {
                mbar_arrive_expect_tx(&full[st], tile_bytes);
                for (int s = 0; s < NSUB; ++s)
                    tma_load_4d(map, &full[st], ring + st * tile_bytes + s * SUB, 64 * s, it.h, j * 128, it.z);
            }
            __syncwarp();
            ++q;
        }
    }
    issued = q;
    res_n = k;
}

// Waits (time-bounded, ignoring the abort flag) until the loads a producer
// issued have landed, so no TMA write is in flight when the CTA exits.
template <int S>
__device__ __forceinline__ void bwd_persistent_drain(uint64_t *full, int issued, uint64_t *res_full, int res_n,
                                                     uint64_t limit_ns) {
    for (int i = (res_n > 2 ? res_n - 2 : 0); i < res_n; ++i)
        mbar_wait_drain(&res_full[i & 1], (i >> 1) & 1, limit_ns);
    for (int q = (issued > S ? issued - S : 0); q < issued; ++q)
        mbar_wait_drain(&full[q % S], (q / S) & 1, limit_ns);
}

// Warp 3: zero-fills the output rows of every tile without work (all rows of
// the tile, with no valid row or an empty other side), spread over the CTAs,
// 16 bytes per lane; with `db`, also the tile's bias-gradient partial.
template <int D>
__device__ __forceinline__ void bwd_zero_fill(const BwdParams &p, bool rows_are_queries, __nv_bfloat16 *out0,
                                              __nv_bfloat16 *out1, float *db) {
    const int lane = lane_id();
    const int Lself = rows_are_queries ? p.Lq : p.Lk;
    const int ntl = (Lself + 127) / 128;
    const int64_t total = static_cast<int64_t>(p.Z) * p.H * ntl;
    constexpr int V4 = D / 8;   // 16-byte chunks per row
    const size_t row_stride = static_cast<size_t>(p.H) * D;
    for (int64_t b = blockIdx.x; b < total; b += gridDim.x) {
        const int z = static_cast<int>(b / (static_cast<int64_t>(p.H) * ntl));
        const int rem = static_cast<int>(b - static_cast<int64_t>(z) * p.H * ntl);
        const int h = rem / ntl, tile = rem - h * ntl;
        int ns, no;
        bwd_lengths(p, rows_are_queries, z, ns, no);
        if (tile * 128 < ns && no > 0) continue;   // an item covers this tile
        const int r0 = tile * 128, rows = min(128, Lself - r0);
        for (int e = lane; e < rows * V4; e += 32) {
            const size_t off = (static_cast<size_t>(z) * Lself + r0 + e / V4) * row_stride +
                               static_cast<size_t>(h) * D;
            const uint4 zero = make_uint4(0u, 0u, 0u, 0u);
            reinterpret_cast<uint4 *>(out0 + off)[e % V4] = zero;
            if (out1 != nullptr) reinterpret_cast<uint4 *>(out1 + off)[e % V4] = zero;
        }
        if (db != nullptr && lane == 0) db[(static_cast<size_t>(z) * p.H + h) * ntl + tile] = 0.0f;
    }
}

// ============================================================================
// Persistent dQ kernel.  TMEM as in the dQ tile kernel: [0,128) S, [128,256)
// and [256,384) dP of even / odd units (each overwritten by its dS),
// [384,384+D) dQ.
// ============================================================================
template <int D, int MODE, bool DB>
__global__ void __launch_bounds__(BwdSigma<D>::kThreads, 1)
    bwd_dq_persistent_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                             const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmDO,
                             const BwdParams p) {
    using Lay = BwdPersistLayout<D>;
    using SG = BwdSigma<D>;
    constexpr int SX = Lay::SX, SY = Lay::SY;
    constexpr uint32_t kColS = 0, kColDP0 = 128, kColDP1 = 256, kColDQ = 384;
    static_assert(kColDQ + D <= Lay::TMEM_COLS, "TMEM budget");
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = align_1k(smem_raw);
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + Lay::OFF_BAR);
    uint64_t *x_full = bars;                  // K_j ring
    uint64_t *x_empty = x_full + SX;
    uint64_t *y_full = x_empty + SX;          // V_j ring
    uint64_t *y_empty = y_full + SY;
    uint64_t *res_full = y_empty + SY;        // [2] Q, dO of item k in slot k % 2
    uint64_t *res_empty = res_full + 2;       // [2] MMA -> producer: item k's MMAs done
    uint64_t *s_full = res_empty + 2;         // MMA -> WGs: S_u in TMEM
    uint64_t *dp_full = s_full + 1;           // [2] MMA -> WGs: dP_u in buffer u % 2
    uint64_t *s_free = dp_full + 2;           // WGs -> MMA: S_u read
    uint64_t *ds_ready = s_free + 1;          // [2] WGs -> MMA: dS_u in buffer u % 2
    uint64_t *acc_full = ds_ready + 2;        // MMA -> WGs: the item's dQ finished
    uint64_t *drain = acc_full + 1;
    static_assert(8 <= Lay::MAX_HANDOFF, "barrier count");
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + Lay::OFF_TMEM);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + Lay::OFF_ABORT);
    int *meta = reinterpret_cast<int *>(smem + Lay::OFF_META);
    BwdSample *table = reinterpret_cast<BwdSample *>(smem + Lay::OFF_TABLE);

    const int warp = warp_id(), lane = lane_id();
    if (warp == 0) bwd_build_table(p, true, table, meta);
    if (threadIdx.x == 0) {
        for (int s = 0; s < SX; ++s) {
            mbar_init(&x_full[s], 1);
            mbar_init(&x_empty[s], 1);
        }
        for (int s = 0; s < SY; ++s) {
            mbar_init(&y_full[s], 1);
            mbar_init(&y_empty[s], 1);
        }
        for (int r = 0; r < 2; ++r) {
            mbar_init(&res_full[r], 1);
            mbar_init(&res_empty[r], 1);
            mbar_init(&dp_full[r], 1);
            mbar_init(&ds_ready[r], SG::kArrivals);
        }
        mbar_init(s_full, 1);
        mbar_init(s_free, SG::kArrivals);
        mbar_init(acc_full, 1);
        mbar_init(drain, 1);
        *abort_flag = 0;
        fence_barrier_init();
    }
    if (warp == 0 && lane == 0) {
        prefetch_tensormap(&tmQ);
        prefetch_tensormap(&tmK);
        prefetch_tensormap(&tmV);
        prefetch_tensormap(&tmDO);
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
    const BwdWalk walk0{&p, table, meta[0], p.Z <= kBwdMaxRanked, true, 0};

    if (warp == 0) {
        {
            int issued, res_n;
            bwd_persistent_producer<SX, Lay::NSUB>(&tmK, x_full, x_empty, smem + Lay::OFF_X, Lay::TILE_BYTES,
                                                   walk0, &tmQ, &tmDO, res_full, res_empty, smem + Lay::OFF_R,
                                                   wctx, issued, res_n);
            bwd_persistent_drain<SX>(x_full, issued, res_full, res_n, p.timeout_ns);
        }
    } else if (warp == 2) {
        // V_j ring, fed by its own thread so it never waits behind a key slot
        {
            int issued, res_n;
            bwd_persistent_producer<SY, Lay::NSUB>(&tmV, y_full, y_empty, smem + Lay::OFF_Y, Lay::TILE_BYTES,
                                                   walk0, nullptr, nullptr, nullptr, nullptr, nullptr, wctx,
                                                   issued, res_n);
            bwd_persistent_drain<SY>(y_full, issued, nullptr, 0, p.timeout_ns);
        }
    } else if (warp == 1) {
        // the whole warp runs converged; elect.sync picks the issuing lane
        auto wait = [&](uint64_t *bar, uint32_t parity) {
            return __all_sync(0xffffffffu, mbar_wait(bar, parity, wctx));
        };
        const uint32_t idesc_s = idesc_bf16_f32(128, 128, false, false);
        const uint32_t idesc_q = idesc_bf16_f32(128, D, false, true);
        // descriptors as low words: slot 0 of each region plus the slot's byte
        // offset >> 4, so the issuing loop does no descriptor arithmetic
        constexpr uint32_t hi = desc_hi(1024);
        constexpr uint32_t kTile = Lay::TILE_BYTES >> 4;
        const uint32_t r_lo = desc_lo(smem_u32(smem + Lay::OFF_R), 16);
        const uint32_t x_lo = desc_lo(smem_u32(smem + Lay::OFF_X), 16);
        const uint32_t y_lo = desc_lo(smem_u32(smem + Lay::OFF_Y), 16);
        const uint32_t xmn_lo = desc_lo(smem_u32(smem + Lay::OFF_X), Lay::SUB_BYTES);   // K as MN-major B
        auto q_of = [&](int k) { return r_lo + (2 * (k & 1)) * kTile; };
        auto do_of = [&](int k) { return r_lo + (2 * (k & 1) + 1) * kTile; };
        // X (128 rows of Q or dO) times Y^T (128 rows of K or V) into TMEM column `col`
        auto issue_xyT = [&](uint32_t col, uint32_t a_lo, uint32_t b_lo) {
#pragma unroll
            for (int kk = 0; kk < D / 16; ++kk) {
                const uint32_t koff = ((kk >> 2) * Lay::SUB_BYTES + (kk & 3) * 32) >> 4;
                mma_ss_lhw(tmem + col, a_lo + koff, b_lo + koff, hi, idesc_s, kk > 0 ? 1u : 0u);
            }
        };
        using Units = BwdUnits<SX, SY>;
        Units cur{walk0};
        cur.start();
        bool ok = true;
        if (cur.live) {
            ok = wait(&res_full[0], 0) && wait(&x_full[0], 0) && wait(&y_full[0], 0);
            if (ok) {
                tc_fence_after();
                issue_xyT(kColS, q_of(0), x_lo);
                mma_commit_w(s_full);
                issue_xyT(kColDP0, do_of(0), y_lo);
                mma_commit_w(&dp_full[0]);
                mma_commit_w(&y_empty[0]);
            }
        }
        Units nx = cur;
        if (nx.live) nx.advance();
        while (ok && cur.live) {
            const int u = cur.u;
            if (nx.live) {
                // S_{u+1} as soon as the warpgroups have read S_u, then dP_{u+1}
                // into the other dP buffer: it still holds dS_{u-1}, read by an
                // earlier MMA of this thread (MMAs run in issue order)
                if (nx.j == 0 && !(ok = wait(&res_full[nx.k & 1], (nx.k >> 1) & 1))) break;
                if (!(ok = wait(&x_full[nx.xs], nx.xph))) break;
                if (!(ok = wait(s_free, u & 1))) break;
                tc_fence_after();
                issue_xyT(kColS, q_of(nx.k), x_lo + nx.xs * kTile);
                mma_commit_w(s_full);
                if (!(ok = wait(&y_full[nx.ys], nx.yph))) break;
                tc_fence_after();
                issue_xyT(nx.u & 1 ? kColDP1 : kColDP0, do_of(nx.k), y_lo + nx.ys * kTile);
                mma_commit_w(&dp_full[nx.u & 1]);
                mma_commit_w(&y_empty[nx.ys]);   // V: its only MMA
            }
            if (!(ok = wait(&ds_ready[u & 1], (u >> 1) & 1))) break;
            tc_fence_after();
            const uint32_t dcol = u & 1 ? kColDP1 : kColDP0;
            const uint32_t k_lo = xmn_lo + cur.xs * kTile;
#pragma unroll
            for (int kk = 0; kk < 8; ++kk)
                mma_ts_lhw(tmem + kColDQ, tmem + dcol + SG::packed_col(kk), k_lo + kk * ((16 * 128) >> 4), hi,
                           idesc_q, (cur.j > 0 || kk > 0) ? 1u : 0u);
            mma_commit_w(&x_empty[cur.xs]);   // K: S and dQ done
            if (cur.last()) {
                mma_commit_w(&res_empty[cur.k & 1]);   // Q, dO of this item no longer read
                mma_commit_w(acc_full);
            }
            cur = nx;
            if (nx.live) nx.advance();
        }
        mma_commit_w(drain);
        mbar_wait_drain(drain, 0, p.timeout_ns);
        __syncwarp();
    } else if (warp == 3) {
        bwd_zero_fill<D>(p, true, p.dq, nullptr, DB ? p.db_part : nullptr);
    } else {
        const int w = (warp - 4) >> 2;      // warpgroup: tile columns [kCols w, kCols (w + 1))
        const int quarter = warp & 3;
        const uint32_t lane_bits = static_cast<uint32_t>(quarter * 32) << 16;
        const int ntl = (p.Lq + 127) / 128;
        // dQ's D columns split over the warpgroups, at least 32 each (with four
        // warpgroups at D = 64 the last two have none)
        constexpr int kEpi = D / SG::NG >= 32 ? D / SG::NG : 32;
        BwdWalk walk = walk0;
        BwdItem it;
        int u = 0, k = 0;
        bool ok = true;
        while (ok && walk.next(it)) {
            const SigmoidCoef cf = make_coef<MODE>(p.alpha, bias_of(p.bias_z, p.bias, it.z));
            float dbacc = 0.0f;   // bias gradient: sum of this row's dS (valid keys)
            for (int j = 0; j < it.nsteps; ++j, ++u) {
                ok = dq_sigma_tile<D, MODE, DB>(tmem + lane_bits, w, kColS, u & 1 ? kColDP1 : kColDP0, s_full,
                                                u & 1, s_free, &dp_full[u & 1], (u >> 1) & 1, &ds_ready[u & 1],
                                                cf, it.nother - j * 128, dbacc, wctx, u);
                if (!ok) break;
            }
            if (!ok) break;
            // the item's dQ += dS K have finished
            ok = __all_sync(0xffffffffu, mbar_wait(acc_full, k & 1, wctx));
            ++k;
            if (!ok) break;
            tc_fence_after();
            const int row = it.tile * 128 + quarter * 32 + lane;
            if (w * kEpi < D) {
                __nv_bfloat16 *drow = p.dq + (static_cast<size_t>(it.z) * p.Lq + row) * (static_cast<size_t>(p.H) * D) +
                                      static_cast<size_t>(it.h) * D;
                store_row_from_tmem<D>(tmem + lane_bits + kColDQ, drow, row < p.Lq, row < it.nself, p.alpha,
                                       w * kEpi, kEpi);
            }
            if constexpr (DB) {
                // one partial per tile (rows at or beyond n_q add nothing).  Warp 4
                // reads the shared partials before its next arrival on s_free, and
                // no warp reaches the next item's sum without that arrival.
                sigma_block_sum<D>(row < it.nself ? dbacc : 0.0f, reinterpret_cast<float *>(smem + Lay::OFF_RED),
                                   &p.db_part[(static_cast<size_t>(it.z) * p.H + it.h) * ntl + it.tile]);
            }
            // The next item's first dQ MMA overwrites the accumulator only after
            // this warpgroup's next ds_ready arrival, which follows these loads.
            tc_fence_before();
        }
    }

    // every warp converges before the block-wide barrier (the producer roles
    // ran on one lane)
    __syncwarp();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, Lay::TMEM_COLS);
    }
}

// ============================================================================
// Persistent dK/dV kernel.  TMEM as in the dK/dV tile kernel: [0,128) S^T,
// [128,256) dP^T with P^T and dS^T over it, [256,256+D) dV, [256+D,256+2D) dK.
// MMA order per unit: S^T_{u+1} (as soon as S^T_u is read), dV_u, dK_u, then
// dP^T_{u+1} over P^T_u and dS^T_u (read by dV_u and dK_u just before; MMAs
// from one thread run in issue order).
// ============================================================================
template <int D, int MODE>
__global__ void __launch_bounds__(BwdSigma<D>::kThreads, 1)
    bwd_dkdv_persistent_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                               const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmDO,
                               const BwdParams p) {
    using Lay = BwdPersistLayout<D>;
    using SG = BwdSigma<D>;
    constexpr int SX = Lay::SX, SY = Lay::SY;
    constexpr uint32_t kColS = 0, kColDP = 128, kColAcc0 = 256, kColAcc1 = 256 + D;
    static_assert(kColAcc1 + D <= Lay::TMEM_COLS, "TMEM budget");
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = align_1k(smem_raw);
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + Lay::OFF_BAR);
    uint64_t *x_full = bars;                  // Q_j ring
    uint64_t *x_empty = x_full + SX;
    uint64_t *y_full = x_empty + SX;          // dO_j ring
    uint64_t *y_empty = y_full + SY;
    uint64_t *res_full = y_empty + SY;        // [2] K, V of item k in slot k % 2
    uint64_t *res_empty = res_full + 2;       // [2] MMA -> producer: item k's MMAs done
    uint64_t *s_full = res_empty + 2;         // MMA -> WGs: S^T_u in TMEM
    uint64_t *dp_full = s_full + 1;           // MMA -> WGs: dP^T_u in TMEM
    uint64_t *s_free = dp_full + 1;           // WGs -> MMA: S^T_u read
    uint64_t *p_ready = s_free + 1;           // WGs -> MMA: P^T_u in TMEM
    uint64_t *ds_ready = p_ready + 1;         // WGs -> MMA: dS^T_u in TMEM
    uint64_t *acc_full = ds_ready + 1;        // MMA -> WGs: the item's dK, dV finished
    uint64_t *drain = acc_full + 1;
    static_assert(7 <= Lay::MAX_HANDOFF, "barrier count");
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + Lay::OFF_TMEM);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + Lay::OFF_ABORT);
    int *meta = reinterpret_cast<int *>(smem + Lay::OFF_META);
    BwdSample *table = reinterpret_cast<BwdSample *>(smem + Lay::OFF_TABLE);

    const int warp = warp_id(), lane = lane_id();
    if (warp == 0) bwd_build_table(p, false, table, meta);
    if (threadIdx.x == 0) {
        for (int s = 0; s < SX; ++s) {
            mbar_init(&x_full[s], 1);
            mbar_init(&x_empty[s], 1);
        }
        for (int s = 0; s < SY; ++s) {
            mbar_init(&y_full[s], 1);
            mbar_init(&y_empty[s], 1);
        }
        for (int r = 0; r < 2; ++r) {
            mbar_init(&res_full[r], 1);
            mbar_init(&res_empty[r], 1);
        }
        mbar_init(s_full, 1);
        mbar_init(dp_full, 1);
        mbar_init(s_free, SG::kArrivals);
        mbar_init(p_ready, SG::kArrivals);
        mbar_init(ds_ready, SG::kArrivals);
        mbar_init(acc_full, 1);
        mbar_init(drain, 1);
        *abort_flag = 0;
        fence_barrier_init();
    }
    if (warp == 0 && lane == 0) {
        prefetch_tensormap(&tmQ);
        prefetch_tensormap(&tmK);
        prefetch_tensormap(&tmV);
        prefetch_tensormap(&tmDO);
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
    const BwdWalk walk0{&p, table, meta[0], p.Z <= kBwdMaxRanked, false, 0};

    if (warp == 0) {
        {
            int issued, res_n;
            bwd_persistent_producer<SX, Lay::NSUB>(&tmQ, x_full, x_empty, smem + Lay::OFF_X, Lay::TILE_BYTES,
                                                   walk0, &tmK, &tmV, res_full, res_empty, smem + Lay::OFF_R,
                                                   wctx, issued, res_n);
            bwd_persistent_drain<SX>(x_full, issued, res_full, res_n, p.timeout_ns);
        }
    } else if (warp == 2) {
        {
            int issued, res_n;
            bwd_persistent_producer<SY, Lay::NSUB>(&tmDO, y_full, y_empty, smem + Lay::OFF_Y, Lay::TILE_BYTES,
                                                   walk0, nullptr, nullptr, nullptr, nullptr, nullptr, wctx,
                                                   issued, res_n);
            bwd_persistent_drain<SY>(y_full, issued, nullptr, 0, p.timeout_ns);
        }
    } else if (warp == 1) {
        auto wait = [&](uint64_t *bar, uint32_t parity) {
            return __all_sync(0xffffffffu, mbar_wait(bar, parity, wctx));
        };
        const uint32_t idesc_s = idesc_bf16_f32(128, 128, false, false);
        const uint32_t idesc_kv = idesc_bf16_f32(128, D, false, true);
        constexpr uint32_t hi = desc_hi(1024);
        constexpr uint32_t kTile = Lay::TILE_BYTES >> 4;
        const uint32_t r_lo = desc_lo(smem_u32(smem + Lay::OFF_R), 16);
        const uint32_t x_lo = desc_lo(smem_u32(smem + Lay::OFF_X), 16);
        const uint32_t y_lo = desc_lo(smem_u32(smem + Lay::OFF_Y), 16);
        const uint32_t xmn_lo = desc_lo(smem_u32(smem + Lay::OFF_X), Lay::SUB_BYTES);   // Q as MN-major B
        const uint32_t ymn_lo = desc_lo(smem_u32(smem + Lay::OFF_Y), Lay::SUB_BYTES);   // dO as MN-major B
        auto k_of = [&](int k) { return r_lo + (2 * (k & 1)) * kTile; };
        auto v_of = [&](int k) { return r_lo + (2 * (k & 1) + 1) * kTile; };
        auto issue_xyT = [&](uint32_t col, uint32_t a_lo, uint32_t b_lo) {
#pragma unroll
            for (int kk = 0; kk < D / 16; ++kk) {
                const uint32_t koff = ((kk >> 2) * Lay::SUB_BYTES + (kk & 3) * 32) >> 4;
                mma_ss_lhw(tmem + col, a_lo + koff, b_lo + koff, hi, idesc_s, kk > 0 ? 1u : 0u);
            }
        };
        // acc += A(TMEM, packed over `acol`) * B (128 rows, MN-major, low word b_lo)
        auto issue_acc = [&](uint32_t acc, uint32_t acol, uint32_t b_lo, bool first) {
#pragma unroll
            for (int kk = 0; kk < 8; ++kk)
                mma_ts_lhw(tmem + acc, tmem + acol + SG::packed_col(kk), b_lo + kk * ((16 * 128) >> 4), hi,
                           idesc_kv, (!first || kk > 0) ? 1u : 0u);
        };
        using Units = BwdUnits<SX, SY>;
        Units cur{walk0};
        cur.start();
        bool ok = true;
        if (cur.live) {
            ok = wait(&res_full[0], 0) && wait(&x_full[0], 0) && wait(&y_full[0], 0);
            if (ok) {
                tc_fence_after();
                issue_xyT(kColS, k_of(0), x_lo);
                mma_commit_w(s_full);
                issue_xyT(kColDP, v_of(0), y_lo);
                mma_commit_w(dp_full);
            }
        }
        Units nx = cur;
        if (nx.live) nx.advance();
        while (ok && cur.live) {
            const int u = cur.u;
            if (nx.live) {
                // S^T_{u+1} into the S^T buffer as soon as the warpgroups have read S^T_u
                if (nx.j == 0 && !(ok = wait(&res_full[nx.k & 1], (nx.k >> 1) & 1))) break;
                if (!(ok = wait(&x_full[nx.xs], nx.xph))) break;
                if (!(ok = wait(s_free, u & 1))) break;
                tc_fence_after();
                issue_xyT(kColS, k_of(nx.k), x_lo + nx.xs * kTile);
                mma_commit_w(s_full);
            }
            if (!(ok = wait(p_ready, u & 1))) break;
            tc_fence_after();
            issue_acc(kColAcc0, kColDP, ymn_lo + cur.ys * kTile, cur.j == 0);             // dV += P^T dO
            mma_commit_w(&y_empty[cur.ys]);                                                         // dO: dP^T, dV done
            if (!(ok = wait(ds_ready, u & 1))) break;
            tc_fence_after();
            issue_acc(kColAcc1, kColDP + SG::kPacked, xmn_lo + cur.xs * kTile, cur.j == 0);  // dK += dS^T Q
            mma_commit_w(&x_empty[cur.xs]);                                                         // Q: S^T, dK done
            if (cur.last()) {
                mma_commit_w(&res_empty[cur.k & 1]);   // K, V of this item no longer read
                mma_commit_w(acc_full);
            }
            if (nx.live) {
                // dP^T_{u+1} overwrites P^T_u and dS^T_u, read by the two MMAs just
                // issued (MMAs run in issue order); its V is resident since the
                // S^T_{u+1} step above
                if (!(ok = wait(&y_full[nx.ys], nx.yph))) break;
                tc_fence_after();
                issue_xyT(kColDP, v_of(nx.k), y_lo + nx.ys * kTile);
                mma_commit_w(dp_full);
            }
            cur = nx;
            if (nx.live) nx.advance();
        }
        mma_commit_w(drain);
        mbar_wait_drain(drain, 0, p.timeout_ns);
        __syncwarp();
    } else if (warp == 3) {
        bwd_zero_fill<D>(p, false, p.dk, p.dv, nullptr);
    } else {
        const int w = (warp - 4) >> 2;      // warpgroup: query columns [kCols w, kCols (w + 1))
        const int quarter = warp & 3;
        const uint32_t lane_bits = static_cast<uint32_t>(quarter * 32) << 16;
        // epilogue: the first half of the warpgroups writes dV, the second dK,
        // D / kOut columns each
        constexpr int kOut = SG::NG / 2;
        const bool is_dv = w < kOut;
        const uint32_t tS = tmem + lane_bits + kColS + SG::kCols * w;
        const uint32_t tD = tmem + lane_bits + kColDP + SG::kCols * w;
        BwdWalk walk = walk0;
        BwdItem it;
        int u = 0, k = 0;
        bool ok = true;
        while (ok && walk.next(it)) {
            const SigmoidCoef cf = make_coef<MODE>(p.alpha, bias_of(p.bias_z, p.bias, it.z));
            for (int i = 0; i < it.nsteps; ++i, ++u) {
                ok = dkdv_sigma_tile<D, MODE>(tS, tD, w, s_full, s_free, dp_full, p_ready, ds_ready, u & 1, cf,
                                              it.nother - i * 128, wctx, u);
                if (!ok) break;
            }
            if (!ok) break;
            // the item's dV += P^T dO and dK += dS^T Q have finished
            ok = __all_sync(0xffffffffu, mbar_wait(acc_full, k & 1, wctx));
            ++k;
            if (!ok) break;
            tc_fence_after();
            const int row = it.tile * 128 + quarter * 32 + lane;   // key row
            const size_t roff = (static_cast<size_t>(it.z) * p.Lk + row) * (static_cast<size_t>(p.H) * D) +
                                static_cast<size_t>(it.h) * D;
            store_row_from_tmem<D>(tmem + lane_bits + (is_dv ? kColAcc0 : kColAcc1), (is_dv ? p.dv : p.dk) + roff,
                                   row < p.Lk, row < it.nself, is_dv ? 1.0f : p.alpha, (w % kOut) * (D / kOut),
                                   D / kOut);
            // The next item's first dV and dK MMAs overwrite the accumulators only
            // after this warpgroup's next p_ready / ds_ready arrivals, which follow
            // these loads.
            tc_fence_before();
        }
    }

    __syncwarp();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, Lay::TMEM_COLS);
    }
}

}  // namespace sigattn
