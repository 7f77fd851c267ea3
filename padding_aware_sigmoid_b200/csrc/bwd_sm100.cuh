// Backward kernels (paper.rainbus.top summary, method steps (4)-(5);
// paperlayer.ai summary, section 4: a dQ kernel and a dK/dV kernel, so that
// each output has one owner and no atomics are needed; P is recomputed).
//
//   dP = dO V^T,  dS = sigma'(S) dP  (sigma' = P (1 - P)),
//   dQ = alpha dS K,   dK = alpha dS^T Q,   dV = P^T dO.
//
// Both kernels share the forward's structure: warp 0 issues TMA loads, one
// thread of warp 1 issues tcgen05.mma, and two warpgroups (warps 4-7 and
// 8-11) turn the fp32 score tiles in TMEM into bf16 operands, each owning 64
// of the 128 columns (thread = TMEM lane = tile row).  The bf16 results are
// written back into TMEM over the columns their own warpgroup has already
// read, and become the TMEM-resident A operand of the next MMA:
//   warpgroup 0 writes packed columns [base, base+32)     for tile columns 0..63
//   warpgroup 1 writes packed columns [base+64, base+96)  for tile columns 64..127
// so the MMA step kk (16 tile columns) reads TMEM column
//   base + (kk < 4 ? 8 kk : 64 + 8 (kk - 4)).
#pragma once

#include "fwd_sm100.cuh"
#include "sm100.cuh"
#include "sigmoid.cuh"

namespace sigattn {

struct BwdParams {
    __nv_bfloat16 *dq;
    __nv_bfloat16 *dk;
    __nv_bfloat16 *dv;
    const int *seqlens_q;
    const int *seqlens_k;
    int L, H;
    float alpha, bias;
    int *status;
    uint64_t timeout_ns;
};

template <int D, int STAGES>
struct BwdLayout {
    static constexpr int NSUB = D / 64;
    static constexpr int SUB_BYTES = 128 * 64 * 2;
    static constexpr int TILE_BYTES = NSUB * SUB_BYTES;
    // two resident tiles (dq: Q, dO; dkdv: K, V) and a ring of streamed pairs
    static constexpr int OFF_A = 0;
    static constexpr int OFF_B = TILE_BYTES;
    static constexpr int OFF_RING = 2 * TILE_BYTES;   // stage s: [X_s][Y_s]
    static constexpr int STAGE_BYTES = 2 * TILE_BYTES;
    static constexpr int OFF_BAR = OFF_RING + STAGES * STAGE_BYTES;
    // res_full, ring_full[S], ring_empty[S], sdp_full, ds_full, mm_done, drain
    static constexpr int NBAR = 1 + 2 * STAGES + 4;
    static constexpr int OFF_TMEM = OFF_BAR + NBAR * 8;
    static constexpr int OFF_ABORT = OFF_TMEM + 8;
    static constexpr int SMEM_ALLOC = OFF_ABORT + 8 + 1024;
    static constexpr uint32_t TMEM_COLS = 512;
    static constexpr uint32_t COL_S = 0, COL_DP = 128, COL_ACC0 = 256, COL_ACC1 = 256 + D;
    static_assert(COL_ACC1 + D <= TMEM_COLS, "TMEM budget");
};

__device__ __forceinline__ uint32_t packed_col(int kk) { return kk < 4 ? 8 * kk : 64 + 8 * (kk - 4); }

// Stores one row of D fp32 accumulator columns from TMEM as bf16, scaled by
// `scale`, or zeros when !valid.  All 32 lanes of the warp must call it.
template <int D>
__device__ __forceinline__ void store_row_from_tmem(uint32_t taddr, __nv_bfloat16 *dst, bool in_range,
                                                    bool valid, float scale, int col0, int ncols) {
    for (int c = col0; c < col0 + ncols; c += 32) {
        uint32_t r[32];
        tmem_ld32(taddr + c, r);
        if (in_range) {
            uint4 *o = reinterpret_cast<uint4 *>(dst + c);
#pragma unroll
            for (int v4 = 0; v4 < 4; ++v4) {
                uint4 w;
                w.x = valid ? pack_bf16x2(scale * __uint_as_float(r[8 * v4 + 0]), scale * __uint_as_float(r[8 * v4 + 1])) : 0u;
                w.y = valid ? pack_bf16x2(scale * __uint_as_float(r[8 * v4 + 2]), scale * __uint_as_float(r[8 * v4 + 3])) : 0u;
                w.z = valid ? pack_bf16x2(scale * __uint_as_float(r[8 * v4 + 4]), scale * __uint_as_float(r[8 * v4 + 5])) : 0u;
                w.w = valid ? pack_bf16x2(scale * __uint_as_float(r[8 * v4 + 6]), scale * __uint_as_float(r[8 * v4 + 7])) : 0u;
                o[v4] = w;
            }
        }
    }
}

template <int D>
__device__ __forceinline__ void zero_row(__nv_bfloat16 *dst, int col0, int ncols) {
    uint4 *o = reinterpret_cast<uint4 *>(dst + col0);
    for (int v4 = 0; v4 < ncols / 8; ++v4) o[v4] = make_uint4(0u, 0u, 0u, 0u);
}

// ============================================================================
// dQ kernel: one CTA per 128-row query tile; streams K_j, V_j for j < ceil(n_k/128).
// TMEM: [0,128) S -> dS (bf16, packed), [128,256) dP, [256,256+D) dQ.
// ============================================================================
template <int D, int MODE, int STAGES>
__global__ void __launch_bounds__(384, 1)
    bwd_dq_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                  const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmDO,
                  const BwdParams p) {
    using Lay = BwdLayout<D, STAGES>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = align_1k(smem_raw);
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + Lay::OFF_BAR);
    uint64_t *res_full = bars;
    uint64_t *ring_full = bars + 1;
    uint64_t *ring_empty = ring_full + STAGES;
    uint64_t *sdp_full = ring_empty + STAGES;
    uint64_t *ds_full = sdp_full + 1;
    uint64_t *mm_done = ds_full + 1;
    uint64_t *drain = mm_done + 1;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + Lay::OFF_TMEM);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + Lay::OFF_ABORT);

    const int warp = warp_id(), lane = lane_id();
    const int z = blockIdx.z, h = blockIdx.y, qtile = blockIdx.x;
    const int L = p.L;
    int nq = p.seqlens_q[z], nk = p.seqlens_k[z];
    if (nq < 0 || nq > L || nk < 0 || nk > L) {
        if (threadIdx.x == 0) record_status(p.status, kStatusSeqlenRange);
        nq = min(max(nq, 0), L);
        nk = min(max(nk, 0), L);
    }
    const int nkv = (nk + 127) / 128;
    const bool work = qtile * 128 < nq && nkv > 0;

    if (threadIdx.x == 0) {
        mbar_init(res_full, 1);
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(&ring_full[s], 1);
            mbar_init(&ring_empty[s], 1);
        }
        mbar_init(sdp_full, 1);
        mbar_init(ds_full, 256);
        mbar_init(mm_done, 1);
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

    if (warp == 0) {
        if (work && lane == 0) {
            uint8_t *sQ = smem + Lay::OFF_A, *sDO = smem + Lay::OFF_B, *ring = smem + Lay::OFF_RING;
            mbar_arrive_expect_tx(res_full, 2 * Lay::TILE_BYTES);
            for (int s = 0; s < Lay::NSUB; ++s) {
                tma_load_4d(&tmQ, res_full, sQ + s * Lay::SUB_BYTES, 64 * s, h, qtile * 128, z);
                tma_load_4d(&tmDO, res_full, sDO + s * Lay::SUB_BYTES, 64 * s, h, qtile * 128, z);
            }
            int issued = 0;
            for (int j = 0; j < nkv; ++j) {
                const int st = j % STAGES, round = j / STAGES;
                if (j >= STAGES && !mbar_wait(&ring_empty[st], (round - 1) & 1, wctx)) break;
                uint8_t *sK = ring + st * Lay::STAGE_BYTES, *sV = sK + Lay::TILE_BYTES;
                mbar_arrive_expect_tx(&ring_full[st], 2 * Lay::TILE_BYTES);
                for (int s = 0; s < Lay::NSUB; ++s) {
                    tma_load_4d(&tmK, &ring_full[st], sK + s * Lay::SUB_BYTES, 64 * s, h, j * 128, z);
                    tma_load_4d(&tmV, &ring_full[st], sV + s * Lay::SUB_BYTES, 64 * s, h, j * 128, z);
                }
                issued = j + 1;
            }
            mbar_wait_drain(res_full, 0, p.timeout_ns);
            for (int j = (issued > STAGES ? issued - STAGES : 0); j < issued; ++j)
                mbar_wait_drain(&ring_full[j % STAGES], (j / STAGES) & 1, p.timeout_ns);
        }
    } else if (warp == 1) {
        if (work && lane == 0) {
            const uint32_t idesc_s = idesc_bf16_f32(128, 128, false, false);
            const uint32_t idesc_q = idesc_bf16_f32(128, D, false, true);
            const uint32_t sQ = smem_u32(smem + Lay::OFF_A), sDO = smem_u32(smem + Lay::OFF_B);
            const uint32_t ring = smem_u32(smem + Lay::OFF_RING);
            bool ok = mbar_wait(res_full, 0, wctx);
            for (int j = 0; ok && j < nkv; ++j) {
                const int st = j % STAGES, round = j / STAGES;
                if (!(ok = mbar_wait(&ring_full[st], round & 1, wctx))) break;
                if (j > 0 && !(ok = mbar_wait(mm_done, (j - 1) & 1, wctx))) break;
                tc_fence_after();
                const uint32_t sK = ring + st * Lay::STAGE_BYTES, sV = sK + Lay::TILE_BYTES;
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk) {
                    const uint32_t koff = (kk >> 2) * Lay::SUB_BYTES + (kk & 3) * 32;
                    mma_ss(tmem + Lay::COL_S, smem_desc_sw128(sQ + koff, 16, 1024),
                           smem_desc_sw128(sK + koff, 16, 1024), idesc_s, kk > 0 ? 1u : 0u);
                }
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk) {
                    const uint32_t koff = (kk >> 2) * Lay::SUB_BYTES + (kk & 3) * 32;
                    mma_ss(tmem + Lay::COL_DP, smem_desc_sw128(sDO + koff, 16, 1024),
                           smem_desc_sw128(sV + koff, 16, 1024), idesc_s, kk > 0 ? 1u : 0u);
                }
                mma_commit(sdp_full);
                if (!(ok = mbar_wait(ds_full, j & 1, wctx))) break;
                tc_fence_after();
#pragma unroll
                for (int kk = 0; kk < 8; ++kk) {
                    mma_ts(tmem + Lay::COL_ACC0, tmem + Lay::COL_S + packed_col(kk),
                           smem_desc_sw128(sK + kk * 16 * 128, Lay::SUB_BYTES, 1024), idesc_q,
                           (j > 0 || kk > 0) ? 1u : 0u);
                }
                mma_commit(mm_done);
                mma_commit(&ring_empty[st]);
            }
            mma_commit(drain);
            mbar_wait_drain(drain, 0, p.timeout_ns);
        }
    } else if (warp >= 4) {
        const int w = (warp - 4) >> 2;      // warpgroup: tile columns [64w, 64w+64)
        const int quarter = warp & 3;
        const int row = qtile * 128 + quarter * 32 + lane;
        const uint32_t lane_bits = static_cast<uint32_t>(quarter * 32) << 16;
        __nv_bfloat16 *drow = p.dq + (static_cast<size_t>(z) * L + row) * (static_cast<size_t>(p.H) * D) +
                              static_cast<size_t>(h) * D;
        bool ok = true;
        if (work) {
            const SigmoidCoef cf = make_coef<MODE>(p.alpha, p.bias);
            for (int j = 0; j < nkv; ++j) {
                ok = __all_sync(0xffffffffu, mbar_wait(sdp_full, j & 1, wctx));
                if (!ok) break;
                tc_fence_after();
                const int kbase = j * 128;
                const bool partial = kbase + 128 > nk;
#pragma unroll
                for (int c = 0; c < 2; ++c) {
                    const int col = 64 * w + 32 * c;
                    uint32_t rs[32], rd[32];
                    tmem_ld32x2(tmem + lane_bits + Lay::COL_S + col, rs,
                                tmem + lane_bits + Lay::COL_DP + col, rd);
                                        uint32_t pk[16];
#pragma unroll
                    for (int i = 0; i < 16; ++i) {
                        float2 pr, gr;
                        sigma_grad2<MODE>(scale2(__uint_as_float(rs[2 * i]), __uint_as_float(rs[2 * i + 1]), cf),
                                          pr, gr);
                        const float2 ds = mul2(gr, f2(__uint_as_float(rd[2 * i]), __uint_as_float(rd[2 * i + 1])));
                        float ds0 = ds.x, ds1 = ds.y;
                        if (partial) {
                            const int key = kbase + col + 2 * i;
                            if (key >= nk) ds0 = 0.0f;
                            if (key + 1 >= nk) ds1 = 0.0f;
                        }
                        pk[i] = pack_bf16x2(ds0, ds1);
                    }
                    tmem_st16(tmem + lane_bits + Lay::COL_S + 64 * w + 16 * c, pk);
                }
                tmem_wait_st();
                tc_fence_before();
                mbar_arrive(ds_full);
            }
            if (ok) ok = __all_sync(0xffffffffu, mbar_wait(mm_done, (nkv - 1) & 1, wctx));
            if (ok) {
                tc_fence_after();
                store_row_from_tmem<D>(tmem + lane_bits + Lay::COL_ACC0, drow, row < L, row < nq,
                                       p.alpha, w * (D / 2), D / 2);
            }
        } else if (row < L) {
            zero_row<D>(drow, w * (D / 2), D / 2);
        }
    }

    __syncthreads();
    if (warp == 1) {
        __syncwarp();
        tc_fence_after();
        tmem_dealloc(tmem, Lay::TMEM_COLS);
    }
}

// ============================================================================
// dK/dV kernel: one CTA per 128-key tile; streams Q_i, dO_i for i < ceil(n_q/128).
// Works on the transposed scores (rows = keys):
//   S^T = K Q_i^T, dP^T = V dO_i^T, P^T -> TMEM over S^T, dS^T -> TMEM over dP^T,
//   dV += P^T dO_i, dK += dS^T Q_i.
// TMEM: [0,128) S^T / P^T, [128,256) dP^T / dS^T, [256,256+D) dV, [256+D,256+2D) dK.
// ============================================================================
template <int D, int MODE, int STAGES>
__global__ void __launch_bounds__(384, 1)
    bwd_dkdv_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                    const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmDO,
                    const BwdParams p) {
    using Lay = BwdLayout<D, STAGES>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = align_1k(smem_raw);
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + Lay::OFF_BAR);
    uint64_t *res_full = bars;
    uint64_t *ring_full = bars + 1;
    uint64_t *ring_empty = ring_full + STAGES;
    uint64_t *sdp_full = ring_empty + STAGES;
    uint64_t *pds_full = sdp_full + 1;
    uint64_t *mm_done = pds_full + 1;
    uint64_t *drain = mm_done + 1;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + Lay::OFF_TMEM);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + Lay::OFF_ABORT);

    const int warp = warp_id(), lane = lane_id();
    const int z = blockIdx.z, h = blockIdx.y, ktile = blockIdx.x;
    const int L = p.L;
    int nq = p.seqlens_q[z], nk = p.seqlens_k[z];
    if (nq < 0 || nq > L || nk < 0 || nk > L) {
        if (threadIdx.x == 0) record_status(p.status, kStatusSeqlenRange);
        nq = min(max(nq, 0), L);
        nk = min(max(nk, 0), L);
    }
    const int nqt = (nq + 127) / 128;
    const bool work = ktile * 128 < nk && nqt > 0;

    if (threadIdx.x == 0) {
        mbar_init(res_full, 1);
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(&ring_full[s], 1);
            mbar_init(&ring_empty[s], 1);
        }
        mbar_init(sdp_full, 1);
        mbar_init(pds_full, 256);
        mbar_init(mm_done, 1);
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

    if (warp == 0) {
        if (work && lane == 0) {
            uint8_t *sK = smem + Lay::OFF_A, *sV = smem + Lay::OFF_B, *ring = smem + Lay::OFF_RING;
            mbar_arrive_expect_tx(res_full, 2 * Lay::TILE_BYTES);
            for (int s = 0; s < Lay::NSUB; ++s) {
                tma_load_4d(&tmK, res_full, sK + s * Lay::SUB_BYTES, 64 * s, h, ktile * 128, z);
                tma_load_4d(&tmV, res_full, sV + s * Lay::SUB_BYTES, 64 * s, h, ktile * 128, z);
            }
            int issued = 0;
            for (int i = 0; i < nqt; ++i) {
                const int st = i % STAGES, round = i / STAGES;
                if (i >= STAGES && !mbar_wait(&ring_empty[st], (round - 1) & 1, wctx)) break;
                uint8_t *sQ = ring + st * Lay::STAGE_BYTES, *sDO = sQ + Lay::TILE_BYTES;
                mbar_arrive_expect_tx(&ring_full[st], 2 * Lay::TILE_BYTES);
                for (int s = 0; s < Lay::NSUB; ++s) {
                    tma_load_4d(&tmQ, &ring_full[st], sQ + s * Lay::SUB_BYTES, 64 * s, h, i * 128, z);
                    tma_load_4d(&tmDO, &ring_full[st], sDO + s * Lay::SUB_BYTES, 64 * s, h, i * 128, z);
                }
                issued = i + 1;
            }
            mbar_wait_drain(res_full, 0, p.timeout_ns);
            for (int i = (issued > STAGES ? issued - STAGES : 0); i < issued; ++i)
                mbar_wait_drain(&ring_full[i % STAGES], (i / STAGES) & 1, p.timeout_ns);
        }
    } else if (warp == 1) {
        if (work && lane == 0) {
            const uint32_t idesc_s = idesc_bf16_f32(128, 128, false, false);
            const uint32_t idesc_kv = idesc_bf16_f32(128, D, false, true);
            const uint32_t sK = smem_u32(smem + Lay::OFF_A), sV = smem_u32(smem + Lay::OFF_B);
            const uint32_t ring = smem_u32(smem + Lay::OFF_RING);
            bool ok = mbar_wait(res_full, 0, wctx);
            for (int i = 0; ok && i < nqt; ++i) {
                const int st = i % STAGES, round = i / STAGES;
                if (!(ok = mbar_wait(&ring_full[st], round & 1, wctx))) break;
                if (i > 0 && !(ok = mbar_wait(mm_done, (i - 1) & 1, wctx))) break;
                tc_fence_after();
                const uint32_t sQ = ring + st * Lay::STAGE_BYTES, sDO = sQ + Lay::TILE_BYTES;
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk) {
                    const uint32_t koff = (kk >> 2) * Lay::SUB_BYTES + (kk & 3) * 32;
                    mma_ss(tmem + Lay::COL_S, smem_desc_sw128(sK + koff, 16, 1024),
                           smem_desc_sw128(sQ + koff, 16, 1024), idesc_s, kk > 0 ? 1u : 0u);
                }
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk) {
                    const uint32_t koff = (kk >> 2) * Lay::SUB_BYTES + (kk & 3) * 32;
                    mma_ss(tmem + Lay::COL_DP, smem_desc_sw128(sV + koff, 16, 1024),
                           smem_desc_sw128(sDO + koff, 16, 1024), idesc_s, kk > 0 ? 1u : 0u);
                }
                mma_commit(sdp_full);
                if (!(ok = mbar_wait(pds_full, i & 1, wctx))) break;
                tc_fence_after();
#pragma unroll
                for (int kk = 0; kk < 8; ++kk) {
                    mma_ts(tmem + Lay::COL_ACC0, tmem + Lay::COL_S + packed_col(kk),
                           smem_desc_sw128(sDO + kk * 16 * 128, Lay::SUB_BYTES, 1024), idesc_kv,
                           (i > 0 || kk > 0) ? 1u : 0u);
                }
#pragma unroll
                for (int kk = 0; kk < 8; ++kk) {
                    mma_ts(tmem + Lay::COL_ACC1, tmem + Lay::COL_DP + packed_col(kk),
                           smem_desc_sw128(sQ + kk * 16 * 128, Lay::SUB_BYTES, 1024), idesc_kv,
                           (i > 0 || kk > 0) ? 1u : 0u);
                }
                mma_commit(mm_done);
                mma_commit(&ring_empty[st]);
            }
            mma_commit(drain);
            mbar_wait_drain(drain, 0, p.timeout_ns);
        }
    } else if (warp >= 4) {
        const int w = (warp - 4) >> 2;      // warpgroup: query columns [64w, 64w+64)
        const int quarter = warp & 3;
        const int row = ktile * 128 + quarter * 32 + lane;   // key row
        const uint32_t lane_bits = static_cast<uint32_t>(quarter * 32) << 16;
        const size_t roff = (static_cast<size_t>(z) * L + row) * (static_cast<size_t>(p.H) * D) +
                            static_cast<size_t>(h) * D;
        __nv_bfloat16 *dst = (w == 0 ? p.dv : p.dk) + roff;
        bool ok = true;
        if (work) {
            const SigmoidCoef cf = make_coef<MODE>(p.alpha, p.bias);
            for (int i = 0; i < nqt; ++i) {
                ok = __all_sync(0xffffffffu, mbar_wait(sdp_full, i & 1, wctx));
                if (!ok) break;
                tc_fence_after();
                const int qbase = i * 128;
                const bool partial = qbase + 128 > nq;
#pragma unroll
                for (int c = 0; c < 2; ++c) {
                    const int col = 64 * w + 32 * c;
                    uint32_t rs[32], rd[32];
                    tmem_ld32x2(tmem + lane_bits + Lay::COL_S + col, rs,
                                tmem + lane_bits + Lay::COL_DP + col, rd);
                                        uint32_t pkp[16], pks[16];
#pragma unroll
                    for (int ii = 0; ii < 16; ++ii) {
                        float2 pr, gr;
                        sigma_grad2<MODE>(scale2(__uint_as_float(rs[2 * ii]), __uint_as_float(rs[2 * ii + 1]), cf),
                                          pr, gr);
                        const float2 ds = mul2(gr, f2(__uint_as_float(rd[2 * ii]), __uint_as_float(rd[2 * ii + 1])));
                        float p0 = pr.x, p1 = pr.y, ds0 = ds.x, ds1 = ds.y;
                        if (partial) {
                            const int q = qbase + col + 2 * ii;
                            if (q >= nq) { p0 = 0.0f; ds0 = 0.0f; }
                            if (q + 1 >= nq) { p1 = 0.0f; ds1 = 0.0f; }
                        }
                        pkp[ii] = pack_bf16x2(p0, p1);
                        pks[ii] = pack_bf16x2(ds0, ds1);
                    }
                    tmem_st16(tmem + lane_bits + Lay::COL_S + 64 * w + 16 * c, pkp);
                    tmem_st16(tmem + lane_bits + Lay::COL_DP + 64 * w + 16 * c, pks);
                }
                tmem_wait_st();
                tc_fence_before();
                mbar_arrive(pds_full);
            }
            if (ok) ok = __all_sync(0xffffffffu, mbar_wait(mm_done, (nqt - 1) & 1, wctx));
            if (ok) {
                tc_fence_after();
                store_row_from_tmem<D>(tmem + lane_bits + (w == 0 ? Lay::COL_ACC0 : Lay::COL_ACC1), dst,
                                       row < L, row < nk, w == 0 ? 1.0f : p.alpha, 0, D);
            }
        } else if (row < L) {
            zero_row<D>(dst, 0, D);
        }
    }

    __syncthreads();
    if (warp == 1) {
        __syncwarp();
        tc_fence_after();
        tmem_dealloc(tmem, Lay::TMEM_COLS);
    }
}

}  // namespace sigattn
