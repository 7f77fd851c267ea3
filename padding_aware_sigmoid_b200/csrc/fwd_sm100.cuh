// Forward kernel, one CTA per pair of query tiles (used for head dimension
// 128): O = sigma(alpha Q K^T + b) V with key padding masked and padded query
// rows zeroed (gist.science summary, section 2.A; paper.rainbus.top summary,
// method steps (1)-(3)).  The persistent kernel for head dimension 64 is in
// fwd_persist_sm100.cuh.
//
// One CTA owns two 128-row query tiles of one (z, h) and streams the key/value
// tiles j < ceil(n_k / 128) through shared memory; key tiles wholly in padding
// are never loaded.  A CTA whose tiles hold no valid (query, key) pair writes
// its output rows as zeros and exits before it sets up barriers or tensor
// memory (the pages' block-sparse skip, paperlayer.ai summary, section 4).
//
// Warp roles (640 threads):
//   warp 0       TMA producer: Q tiles once, then K_j into the key ring
//   warp 2       TMA producer: V_j into the value ring
//   warp 1       owns TMEM and issues every tcgen05.mma, the whole warp running
//                converged (elect.sync picks the issuing lane)
//   warp 3       idle
//   warps 4-19   four sigma warpgroups (thread = query row = TMEM lane):
//                warpgroup g serves query tile t = g / 2, key columns
//                [64 c, 64 c + 64) of each key tile with c = g % 2, then
//                writes columns [c D/2, c D/2 + D/2) of tile t's output.
// Each SM sub-partition thus runs four sigma warps, two per query tile, so
// one tile's sigma work keeps the MUFU busy while the other tile's warps wait
// for their next scores (the MUFU reaches its full rate only with two or more
// warps issuing on a sub-partition).
// Tensor memory (512 columns, fp32):
//   [0,128) S0   [128,256) S1   [256,256+D) O0   [256+D,256+2D) O1
// P_t (bf16, two per column) overwrites S_t columns [0,32) (keys 0-63) and
// [64,96) (keys 64-127), each written by the warpgroup that read those scores,
// and is the TMEM-resident A operand of O_t += P_t V_j, so P never touches
// shared memory.
//
// Per key tile j the MMA thread issues S0 = Q0 K_j^T, S1 = Q1 K_j^T, then
// O0 += P0 V_j, O1 += P1 V_j as the warpgroups publish P.  S_t of tile j+1 is
// issued right after O_t += P_t V_j (P_t aliases S_t; MMAs from one thread run
// in issue order); the other query tile's work fills the tensor pipe meanwhile.
#pragma once

#include "sm100.cuh"
#include "sigmoid.cuh"

namespace sigattn {

struct FwdParams {
    __nv_bfloat16 *o;
    const int *seqlens_q;
    const int *seqlens_k;
    int Z, Lq, Lk, H;       // batch; padded lengths of Q (and O) and of K, V; heads
    float alpha, bias;
    int *status;
    uint64_t timeout_ns;
    const float *bias_z;   // device float[Z], one bias per sample; null: the scalar `bias`
};

// Shared memory: the two query tiles, a ring of KS key tiles and a ring of VS
// value tiles (V_j's last use, O += P V_j, comes later than K_j's, so its ring
// is the deeper one).
template <int D, int KS, int VS>
struct FwdLayout {
    static constexpr int BM = 128;                 // query rows per tile
    static constexpr int BN = 128;                 // keys per tile
    static constexpr int NSUB = D / 64;            // 64-column swizzle atoms per row
    static constexpr int SUB_BYTES = 128 * 64 * 2; // one [128][64] bf16 atom column
    static constexpr int TILE_BYTES = NSUB * SUB_BYTES;
    static constexpr int OFF_Q = 0;
    static constexpr int OFF_K = OFF_Q + 2 * TILE_BYTES;
    static constexpr int OFF_V = OFF_K + KS * TILE_BYTES;
    static constexpr int OFF_BAR = OFF_V + VS * TILE_BYTES;
    // q_full, k_full[KS], k_empty[KS], v_full[VS], v_empty[VS], s_full[2], p_full[2],
    // drain
    static constexpr int NBAR = 1 + 2 * KS + 2 * VS + 5;
    static constexpr int OFF_TMEM = OFF_BAR + NBAR * 8;
    static constexpr int OFF_ABORT = OFF_TMEM + 8;
    static constexpr int OFF_SAMPLE = OFF_ABORT + 8;   // this block's sample and lengths
    static constexpr int BYTES = OFF_SAMPLE + 16;
    static constexpr int SMEM_ALLOC = BYTES + 1024;  // slack to align the base to 1 KiB
    static constexpr uint32_t TMEM_COLS = 512;
    static constexpr uint32_t COL_S0 = 0, COL_S1 = 128, COL_O0 = 256, COL_O1 = 256 + D;
    static_assert(COL_O1 + D <= TMEM_COLS, "TMEM budget");
    static_assert(SMEM_ALLOC <= 232448, "shared memory budget");
};

constexpr int kFwdThreads = 640;
// ring depths per head dimension: key slots K and value slots V
template <int D> struct FwdStages { static constexpr int K = D == 128 ? 2 : 4, V = D == 128 ? 3 : 4; };

template <int D, int MODE, int KS, int VS>
__global__ void __launch_bounds__(kFwdThreads, 1)
    fwd_tiles_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
               const __grid_constant__ CUtensorMap tmV, const FwdParams p) {
    using Lay = FwdLayout<D, KS, VS>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = align_1k(smem_raw);
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + Lay::OFF_BAR);
    uint64_t *q_full = bars;
    uint64_t *k_full = bars + 1;
    uint64_t *k_empty = k_full + KS;
    uint64_t *v_full = k_empty + KS;
    uint64_t *v_empty = v_full + VS;
    uint64_t *s_full = v_empty + VS;
    uint64_t *p_full = s_full + 2;
    uint64_t *drain = p_full + 2;
    static_assert(1 + 2 * KS + 2 * VS + 5 == Lay::NBAR, "barrier count");
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + Lay::OFF_TMEM);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + Lay::OFF_ABORT);

    const int warp = warp_id(), lane = lane_id();
    // samples start by decreasing key length: warp 0 picks this block's sample
    BlockSample *sample_slot = reinterpret_cast<BlockSample *>(smem + Lay::OFF_SAMPLE);
    if (warp == 0) publish_block_sample(p.seqlens_q, p.seqlens_k, true, sample_slot);
    __syncthreads();
    const BlockSample bs = *sample_slot;
    const int z = bs.z, h = blockIdx.y;
    const int qtile0 = blockIdx.x * 2;
    const int L = p.Lq;     // query rows of this problem (O has the same layout)
    int nq = bs.nq, nk = bs.nk;
    if (nq < 0 || nq > L || nk < 0 || nk > p.Lk) {
        if (threadIdx.x == 0) record_status(p.status, kStatusSeqlenRange);
        nq = min(max(nq, 0), L);
        nk = min(max(nk, 0), p.Lk);
    }
    const int ntiles = (qtile0 * Lay::BM < nq ? 1 : 0) + ((qtile0 + 1) * Lay::BM < nq ? 1 : 0);
    const int nkv = (nk + Lay::BN - 1) / Lay::BN;
    const size_t row_stride = static_cast<size_t>(p.H) * D;
    if (ntiles == 0 || nkv == 0) {
        // No valid (query, key) pair in this block's tiles: its output rows are
        // zeros, written by every thread, and the block ends here.
        const int r0 = qtile0 * Lay::BM, rows = min(2 * Lay::BM, L - r0);
        constexpr int V4 = D / 8;   // 16-byte chunks per row
        for (int e = threadIdx.x; e < rows * V4; e += kFwdThreads) {
            uint4 *dst = reinterpret_cast<uint4 *>(p.o + (static_cast<size_t>(z) * L + r0 + e / V4) *
                                                             row_stride + static_cast<size_t>(h) * D);
            dst[e % V4] = make_uint4(0u, 0u, 0u, 0u);
        }
        return;
    }
    if (threadIdx.x == 0) {
        mbar_init(q_full, 1);
        for (int s = 0; s < KS; ++s) {
            mbar_init(&k_full[s], 1);
            mbar_init(&k_empty[s], 1);
        }
        for (int s = 0; s < VS; ++s) {
            mbar_init(&v_full[s], 1);
            mbar_init(&v_empty[s], 1);
        }
        for (int t = 0; t < 2; ++t) {
            mbar_init(&s_full[t], 1);
            mbar_init(&p_full[t], 256);  // the two sigma warpgroups of tile t
        }
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


    if (warp == 0) {
        // ------------------------------------------------------------ producer
        if (lane == 0) {
            uint8_t *sQ = smem + Lay::OFF_Q;
            uint8_t *sK = smem + Lay::OFF_K;
            uint8_t *sV = smem + Lay::OFF_V;
            mbar_arrive_expect_tx(q_full, ntiles * Lay::TILE_BYTES);
            for (int t = 0; t < ntiles; ++t)
                for (int s = 0; s < Lay::NSUB; ++s)
                    tma_load_4d(&tmQ, q_full, sQ + t * Lay::TILE_BYTES + s * Lay::SUB_BYTES,
                                64 * s, h, (qtile0 + t) * Lay::BM, z);
            int issued_k = 0;
            for (int j = 0; j < nkv; ++j) {
                const int sk = j % KS;
                if (j >= KS && !mbar_wait(&k_empty[sk], ((j / KS) - 1) & 1, wctx)) break;
                mbar_arrive_expect_tx(&k_full[sk], Lay::TILE_BYTES);
                for (int s = 0; s < Lay::NSUB; ++s)
                    tma_load_4d(&tmK, &k_full[sk], sK + sk * Lay::TILE_BYTES + s * Lay::SUB_BYTES,
                                64 * s, h, j * Lay::BN, z);
                issued_k = j + 1;
                trace(0, j, 0);
            }
            // Every issued load must land before the CTA's shared memory is released.
            mbar_wait_drain(q_full, 0, p.timeout_ns);
            for (int j = (issued_k > KS ? issued_k - KS : 0); j < issued_k; ++j)
                mbar_wait_drain(&k_full[j % KS], (j / KS) & 1, p.timeout_ns);
        }
    } else if (warp == 2) {
        // ------------------------------------------------------------ value producer
        // V_j is released later than K_j, so its ring is fed by its own thread
        // and never waits behind a key slot.
        if (lane == 0) {
            uint8_t *sV = smem + Lay::OFF_V;
            int issued_v = 0;
            for (int j = 0; j < nkv; ++j) {
                const int sv = j % VS;
                if (j >= VS && !mbar_wait(&v_empty[sv], ((j / VS) - 1) & 1, wctx)) break;
                mbar_arrive_expect_tx(&v_full[sv], Lay::TILE_BYTES);
                for (int s = 0; s < Lay::NSUB; ++s)
                    tma_load_4d(&tmV, &v_full[sv], sV + sv * Lay::TILE_BYTES + s * Lay::SUB_BYTES,
                                64 * s, h, j * Lay::BN, z);
                issued_v = j + 1;
                trace(0, j, 1);
            }
            for (int j = (issued_v > VS ? issued_v - VS : 0); j < issued_v; ++j)
                mbar_wait_drain(&v_full[j % VS], (j / VS) & 1, p.timeout_ns);
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer
        {
            // the whole warp runs converged; elect.sync picks the issuing lane
            auto wt = [&](uint64_t *bar, uint32_t parity) {
                return __all_sync(0xffffffffu, mbar_wait(bar, parity, wctx));
            };
            const uint32_t idesc_s = idesc_bf16_f32(128, Lay::BN, false, false);
            const uint32_t idesc_o = idesc_bf16_f32(128, D, false, true);
            const uint32_t sQ = smem_u32(smem + Lay::OFF_Q);
            const uint32_t sK = smem_u32(smem + Lay::OFF_K);
            const uint32_t sV = smem_u32(smem + Lay::OFF_V);
            // S_t = Q_t K_j^T into TMEM columns of tile t
            auto issue_s = [&](int t, uint32_t kbase) {
                const uint32_t qbase = sQ + t * Lay::TILE_BYTES;
                const uint32_t d_tmem = tmem + (t ? Lay::COL_S1 : Lay::COL_S0);
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk) {
                    const uint32_t koff = (kk >> 2) * Lay::SUB_BYTES + (kk & 3) * 32;
                    mma_ss_w(d_tmem, smem_desc_sw128(qbase + koff, 16, 1024),
                           smem_desc_sw128(kbase + koff, 16, 1024), idesc_s, kk > 0 ? 1u : 0u);
                }
                mma_commit_w(&s_full[t]);
            };
            // O_t += P_t V_j, P_t read from TMEM (16 keys = 8 packed columns per step;
            // keys 64-127 sit 32 columns further on, see the sigma warpgroups)
            auto issue_pv = [&](int t, uint32_t vbase, bool first) {
                const uint32_t d_tmem = tmem + (t ? Lay::COL_O1 : Lay::COL_O0);
                const uint32_t a_tmem = tmem + (t ? Lay::COL_S1 : Lay::COL_S0);
#pragma unroll
                for (int kk = 0; kk < Lay::BN / 16; ++kk)
                    mma_ts_w(d_tmem, a_tmem + kk * 8 + (kk >= 4 ? 32 : 0),
                           smem_desc_sw128(vbase + kk * 16 * 128, Lay::SUB_BYTES, 1024), idesc_o,
                           (!first || kk > 0) ? 1u : 0u);
            };
            // Order per key tile j: PV0_j, S0_{j+1}, PV1_j, S1_{j+1}.  Tile 0's next
            // scores never wait for tile 1's P, so the sigma warps can evaluate
            // one tile while the tensor pipe works on the other.  S_t of
            // j+1 overwrites P_t of j right after O_t += P_t V_j is issued: MMAs
            // issued by one thread execute in issue order, so the P.V MMA has read
            // P_t before the next scores are written over it.
            bool ok = wt(q_full, 0) && wt(&k_full[0], 0);
            if (ok) {
                tc_fence_after();
                for (int t = 0; t < ntiles; ++t) issue_s(t, sK);
                mma_commit_w(&k_empty[0]);
            }
            for (int j = 0; ok && j < nkv; ++j) {
                const int stv = j % VS;
                const int stk = (j + 1) % KS;
                const bool more = j + 1 < nkv;
                const uint32_t vbase = sV + stv * Lay::TILE_BYTES;
                const uint32_t knext = sK + stk * Lay::TILE_BYTES;
                if (!(ok = wt(&v_full[stv], (j / VS) & 1))) break;
                trace(1, j, 0);
                for (int t = 0; t < ntiles; ++t) {
                    if (!(ok = wt(&p_full[t], j & 1))) break;
                    trace(1, j, 1 + 3 * t);
                    tc_fence_after();
                    issue_pv(t, vbase, j == 0);
                    trace(1, j, 2 + 3 * t);
                    if (t == ntiles - 1) mma_commit_w(&v_empty[stv]);
                    if (more) {
                        if (t == 0 && !(ok = wt(&k_full[stk], ((j + 1) / KS) & 1))) break;
                        tc_fence_after();
                        issue_s(t, knext);
                        trace(1, j, 3 + 3 * t);
                        if (t == ntiles - 1) mma_commit_w(&k_empty[stk]);
                    }
                }
            }
            // No MMA may still be running when TMEM is released.
            mma_commit_w(drain);
            mbar_wait_drain(drain, 0, p.timeout_ns);
            __syncwarp();
        }
    } else if (warp >= 4) {
        // ------------------------------------------------------------ sigma warpgroups
        // Warpgroup g works on query tile t = g / 2 only, on key columns
        // [64 c, 64 c + 64) of S_t (c = g % 2).  The warpgroups of the two tiles
        // run side by side on every SM sub-partition: while one tile's warps
        // wait for their next scores (P.V and the next Q K^T of that tile on
        // the tensor pipe), the other tile's warps keep the MUFU busy.
        const int g = (warp - 4) >> 2;
        const int t = g >> 1, c = g & 1;
        const int quarter = warp & 3;  // TMEM lane quarter this warp may access
        const uint32_t lane_bits = static_cast<uint32_t>(quarter * 32) << 16;
        bool ok = true;
        const bool mine = t < ntiles;
        if (mine) {
            const SigmoidCoef cf = make_coef<MODE>(p.alpha, bias_of(p.bias_z, p.bias, z));
            const uint32_t tS = tmem + lane_bits + (t ? Lay::COL_S1 : Lay::COL_S0) + 64 * c;
            for (int j = 0; j < nkv; ++j) {
                if (quarter == 0) trace(2 + c, j, 2 * t);
                ok = __all_sync(0xffffffffu, mbar_wait(&s_full[t], j & 1, wctx));
                if (!ok) break;
                if (quarter == 0) trace(2 + c, j, 2 * t + 1);
                tc_fence_after();
                const int kvalid = nk - j * Lay::BN - 64 * c;  // keys of this half below n_k
                // two chunks of 32 scores per thread; P of chunk u lies over S
                // columns [16 u, 16 u + 16) of this half, already read
#pragma unroll
                for (int u = 0; u < 2; ++u) {
                    uint32_t r[32];
                    tmem_ld32(tS + 32 * u, r);
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
                            const int col = 32 * u + 2 * i;
                            const uint32_t lo = col < kvalid ? 0x0000FFFFu : 0u;
                            const uint32_t hi = col + 1 < kvalid ? 0xFFFF0000u : 0u;
                            pk[i] &= (lo | hi);
                        }
                    }
                    tmem_st16(tS + 16 * u, pk);
                }
                tmem_wait_st();
                tc_fence_before();
                mbar_arrive(&p_full[t]);
                if (quarter == 0) trace(2 + c, j, 4 + t);
            }
            // every MMA of this CTA has finished once the MMA thread's final commit lands
            if (ok) ok = __all_sync(0xffffffffu, mbar_wait(drain, 0, wctx));
        }
        // epilogue: warpgroup g writes columns [c D/2, c D/2 + D/2) of query tile t
        constexpr int HALF = D / 2;
        const int row = (qtile0 + t) * Lay::BM + quarter * 32 + lane;
        __nv_bfloat16 *orow = p.o + (static_cast<size_t>(z) * L + row) * row_stride +
                              static_cast<size_t>(h) * D + c * HALF;
        if (mine) {
            if (ok) {
                tc_fence_after();
                const uint32_t tO = tmem + lane_bits + (t ? Lay::COL_O1 : Lay::COL_O0) + c * HALF;
                const bool valid = row < nq;
#pragma unroll
                for (int cc = 0; cc < HALF / 32; ++cc) {
                    uint32_t r[32];
                    tmem_ld32(tO + 32 * cc, r);
                    if (row < L) {
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
            }
        } else if (row < L) {
            // the block's second query tile lies wholly in padding: exact zeros, no loads
            uint4 *dst = reinterpret_cast<uint4 *>(orow);
#pragma unroll
            for (int v4 = 0; v4 < HALF / 8; ++v4) dst[v4] = make_uint4(0u, 0u, 0u, 0u);
        }
    }

    // every warp converges before the block-wide barrier (the producer and MMA
    // roles ran on one lane)
    __syncwarp();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, Lay::TMEM_COLS);
    }
}

}  // namespace sigattn
