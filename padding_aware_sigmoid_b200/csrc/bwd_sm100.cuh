// Backward kernels (paper.rainbus.top summary, method steps (4)-(5);
// paperlayer.ai summary, section 4: a dQ kernel and a dK/dV kernel, so that
// each output has one owner and no atomics are needed; P is recomputed).
//
//   dP = dO V^T,  dS = sigma'(S) dP  (sigma' = P (1 - P)),
//   dQ = alpha dS K,   dK = alpha dS^T Q,   dV = P^T dO.
//
// Both kernels share the forward's structure: warps 0 and 2 issue TMA loads
// (one ring each), warp 1 issues tcgen05.mma (running converged, one elected
// lane issuing), and NG sigma warpgroups (warps 4 and up; NG = 2 at D = 128,
// 4 at D = 64, see BwdSigma) turn the fp32 score tiles in TMEM into bf16
// operands, warpgroup w owning the kCols = 128 / NG tile columns
// [kCols w, kCols (w + 1)) (thread = TMEM lane = tile row).  The bf16 results
// are written back into TMEM over columns their own warpgroup has already
// read, and become the TMEM-resident A operand of the next MMA: warpgroup w
// writes its kCols tile columns packed two per TMEM column at
// [base + kCols w, base + kCols w + kCols / 2), so the MMA step kk (16 tile
// columns) reads the TMEM column BwdSigma<D>::packed_col(kk) past base.
// The warpgroups release each score buffer as soon as they have read it, so
// that the next scores' MMA runs while they still work on the current tile.
#pragma once

#include "sm100.cuh"
#include "sigmoid.cuh"

namespace sigattn {

struct BwdParams {
    __nv_bfloat16 *dq;
    __nv_bfloat16 *dk;
    __nv_bfloat16 *dv;
    const int *seqlens_q;
    const int *seqlens_k;
    int Lq, Lk, H;          // padded lengths of Q, dO, dQ and of K, V, dK, dV; heads
    float alpha, bias;
    int *status;
    uint64_t timeout_ns;
    const float *bias_z;   // device float[Z], one bias per sample; null: the scalar `bias`
    float *db_part;        // dQ kernel: one partial of db_z = sum dS per query tile, or null
    int Z;                 // samples
};

// Shared memory: two resident tiles (dq: Q, dO; dkdv: K, V) and two rings of
// streamed tiles, X (dq: K_j; dkdv: Q_i) with SX slots and Y (dq: V_j; dkdv:
// dO_i) with SY slots.  The rings are separate so that each tile's slot is
// released as soon as its own last MMA has finished; X holds the tile whose
// last use comes later in the step, so it gets the deeper ring.
template <int D, int SX, int SY>
struct BwdLayout {
    static constexpr int NSUB = D / 64;
    static constexpr int SUB_BYTES = 128 * 64 * 2;
    static constexpr int TILE_BYTES = NSUB * SUB_BYTES;
    static constexpr int OFF_A = 0;
    static constexpr int OFF_B = TILE_BYTES;
    static constexpr int OFF_X = 2 * TILE_BYTES;
    static constexpr int OFF_Y = OFF_X + SX * TILE_BYTES;
    static constexpr int OFF_BAR = OFF_Y + SY * TILE_BYTES;
    // res_full, x_full[SX], x_empty[SX], y_full[SY], y_empty[SY], then up to
    // MAX_HANDOFF per-kernel hand-off barriers
    static constexpr int MAX_HANDOFF = 10;
    static constexpr int NBAR = 1 + 2 * SX + 2 * SY + MAX_HANDOFF;
    static constexpr int OFF_TMEM = OFF_BAR + NBAR * 8;
    static constexpr int OFF_ABORT = OFF_TMEM + 8;
    static constexpr int OFF_RED = OFF_ABORT + 8;      // 16 floats: per-warp db partials
    static constexpr int OFF_SAMPLE = OFF_RED + 64;    // this block's sample and lengths
    static constexpr int SMEM_ALLOC = OFF_SAMPLE + 16 + 1024;
    static constexpr uint32_t TMEM_COLS = 512;
    static constexpr uint32_t COL_S = 0, COL_DP = 128, COL_ACC0 = 256, COL_ACC1 = 256 + D;
    static_assert(COL_ACC1 + D <= TMEM_COLS, "TMEM budget");
    static_assert(SMEM_ALLOC <= 232448, "shared memory budget");
};

// ring depths per head dimension: X (dq: K, dkdv: Q) and Y (dq: V, dkdv: dO) slots
template <int D> struct BwdStages { static constexpr int X = D == 128 ? 3 : 4, Y = D == 128 ? 2 : 4; };

// Streams tiles j = 0..n-1 of one tensor map into a ring of S slots; returns
// false when a wait gave up.  `issued` counts the loads issued so far.
template <int S, int NSUB>
__device__ __forceinline__ bool ring_load(const CUtensorMap *map, uint64_t *full, uint64_t *empty,
                                          uint8_t *base, int tile_bytes, int j, int h, int z,
                                          const WaitCtx &w) {
    const int st = j % S;
    if (j >= S && !mbar_wait(&empty[st], ((j / S) - 1) & 1, w)) return false;
    mbar_arrive_expect_tx(&full[st], tile_bytes);
    for (int s = 0; s < NSUB; ++s)
        tma_load_4d(map, &full[st], base + st * tile_bytes + s * (128 * 64 * 2), 64 * s, h, j * 128, z);
    return true;
}

// Waits (time-bounded, ignoring the abort flag) until the last min(issued, S)
// loads of a ring have landed, so no TMA write is in flight at exit.
template <int S>
__device__ __forceinline__ void ring_drain(uint64_t *full, int issued, uint64_t limit_ns) {
    for (int j = (issued > S ? issued - S : 0); j < issued; ++j)
        mbar_wait_drain(&full[j % S], (j / S) & 1, limit_ns);
}

// Sigma warpgroups per backward block.  At D = 64 a tile's sigma' work is
// twice its MMA work and four warpgroups (32 tile columns each) keep up with
// the tensor core; at D = 128 the two are equal and two warpgroups (64 columns
// each, with more registers per thread) measured faster.
template <int D>
struct BwdSigma {
    static constexpr int NG = D == 64 ? 4 : 2;
    static constexpr int kThreads = 128 + 128 * NG;
    static constexpr int kCols = 128 / NG;       // tile columns per warpgroup
    static constexpr int kPacked = kCols / 2;    // TMEM columns of their bf16 pairs
    static constexpr int kArrivals = 128 * NG;   // one per sigma thread
    // TMEM column (relative to the buffer) of the packed bf16 values of K step
    // kk (tile columns 16 kk .. 16 kk + 15), which warpgroup 16 kk / kCols wrote
    // over the first kPacked of its own columns.
    static __device__ __forceinline__ uint32_t packed_col(int kk) {
        return kCols * ((16 * kk) / kCols) + ((16 * kk) % kCols) / 2;
    }
};

template <int N>
__device__ __forceinline__ void tmem_ld_cols(uint32_t taddr, uint32_t (&r)[N]) {
    static_assert(N == 16 || N == 32 || N == 64, "column count");
    if constexpr (N == 16) tmem_ld16(taddr, r);
    else if constexpr (N == 32) tmem_ld32(taddr, r);
    else tmem_ld64(taddr, r);
}

template <int N>
__device__ __forceinline__ void tmem_st_cols(uint32_t taddr, const uint32_t (&r)[N]) {
    static_assert(N == 16 || N == 32, "column count");
    if constexpr (N == 16) tmem_st16(taddr, r);
    else tmem_st32(taddr, r);
}

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

// Zeroes rows [r0, r0 + rows) of head h of sample z in a [Z][L][H][D] bf16
// tensor, 16 bytes per thread and step, with every thread of the block.
template <int D>
__device__ __forceinline__ void zero_rows(__nv_bfloat16 *base, int z, int h, int r0, int rows, int L,
                                          int H) {
    constexpr int V4 = D / 8;   // 16-byte chunks per row
    const size_t row_stride = static_cast<size_t>(H) * D;
    for (int e = threadIdx.x; e < rows * V4; e += blockDim.x) {
        uint4 *dst = reinterpret_cast<uint4 *>(base + (static_cast<size_t>(z) * L + r0 + e / V4) * row_stride +
                                               static_cast<size_t>(h) * D);
        dst[e % V4] = make_uint4(0u, 0u, 0u, 0u);
    }
}

// Zeroes the packed bf16 pairs at tile columns >= valid (pk holds columns
// [col0, col0 + 2 N) of the tile; valid = count of in-range columns).
template <int N>
__device__ __forceinline__ void mask_packed(uint32_t (&pk)[N], int col0, int valid) {
#pragma unroll
    for (int i = 0; i < N; ++i) {
        const int c = col0 + 2 * i;
        const uint32_t lo = c < valid ? 0x0000FFFFu : 0u;
        const uint32_t hi = c + 1 < valid ? 0xFFFF0000u : 0u;
        pk[i] &= (lo | hi);
    }
}

// One key tile of a dQ sigma warpgroup (w: the warpgroup, which owns tile
// columns [kCols w, kCols (w + 1))); `trow` is the TMEM address of this
// thread's lane.  Reads its columns of S (buffer column col_s) once s_full has
// completed the phase of parity s_par and releases them (s_free); waits for
// dP (buffer column dcol, barrier dp_full, parity dp_par); writes
// dS = sigma'(S) dP, packed bf16, over the first kPacked of its dP columns;
// then arrives on ds_ready.  kvalid: keys of the tile below n_k (the others
// give dS = 0); with DB, dbacc adds this row's dS over them.  Returns false
// when a wait gave up.
template <int D, int MODE, bool DB>
__device__ __forceinline__ bool dq_sigma_tile(uint32_t trow, int w, uint32_t col_s, uint32_t dcol,
                                              uint64_t *s_full, uint32_t s_par, uint64_t *s_free,
                                              uint64_t *dp_full, uint32_t dp_par, uint64_t *ds_ready,
                                              const SigmoidCoef &cf, int kvalid, float &dbacc,
                                              const WaitCtx &wctx, int tstep) {
    using SG = BwdSigma<D>;
    const int quarter = warp_id() & 3;
    if (quarter == 0) trace(2 + (w & 1), tstep, 0);
    if (!__all_sync(0xffffffffu, mbar_wait(s_full, s_par, wctx))) return false;
    if (quarter == 0) trace(2 + (w & 1), tstep, 1);
    tc_fence_after();
    uint32_t r[SG::kCols];
    tmem_ld_cols(trow + col_s + SG::kCols * w, r);
    if (quarter == 0) trace(2 + (w & 1), tstep, 2);
    tc_fence_before();
    mbar_arrive(s_free);
    // sigma'(S) and dS = sigma' dP are formed 32 columns at a time, so that
    // the MUFU work of one chunk overlaps the multiplies and bf16 packing of
    // the other.  The first chunk's sigma' (all of it with one chunk of 32
    // columns, at D = 64) is taken before dP is waited for, covering the time
    // dP may still need.
    constexpr int kChunks = SG::kCols / 32;
    constexpr int kPre = 1;   // chunks of sigma' before the dP wait
    float2 gpre[16 * kPre + 1];
#pragma unroll
    for (int i = 0; i < 16 * kPre; ++i) {
        float2 pr;
        sigma_grad2<MODE>(scale2(__uint_as_float(r[2 * i]), __uint_as_float(r[2 * i + 1]), cf), pr, gpre[i]);
    }
    const uint32_t dc = dcol + SG::kCols * w;
    if (quarter == 0) trace(2 + (w & 1), tstep, 3);
    if (!__all_sync(0xffffffffu, mbar_wait(dp_full, dp_par, wctx))) return false;
    if (quarter == 0) trace(2 + (w & 1), tstep, 4);
    tc_fence_after();
    float2 dsum = f2(0.0f, 0.0f);   // this row's fp32 dS over keys below n_k
#pragma unroll
    for (int ch = 0; ch < kChunks; ++ch) {
        uint32_t d[32];
        tmem_ld32(trow + dc + 32 * ch, d);
        uint32_t pk[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) {
            float2 g;
            if (ch < kPre) {
                g = gpre[16 * ch + i];
            } else {
                float2 pr;
                sigma_grad2<MODE>(scale2(__uint_as_float(r[32 * ch + 2 * i]),
                                         __uint_as_float(r[32 * ch + 2 * i + 1]), cf),
                                  pr, g);
            }
            const float2 ds = mul2(g, f2(__uint_as_float(d[2 * i]), __uint_as_float(d[2 * i + 1])));
            pk[i] = pack_bf16x2(ds.x, ds.y);
            if constexpr (DB) {
                const int c = SG::kCols * w + 32 * ch + 2 * i;
                dsum.x += c < kvalid ? ds.x : 0.0f;
                dsum.y += c + 1 < kvalid ? ds.y : 0.0f;
            }
        }
        if (kvalid < 128) mask_packed(pk, SG::kCols * w + 32 * ch, kvalid);
        // dS over the first kPacked of this warpgroup's dP columns: chunk ch's
        // 16 packed columns sit over dP columns this warpgroup has read
        tmem_st16(trow + dc + 16 * ch, pk);
    }
    if (quarter == 0) trace(2 + (w & 1), tstep, 5);
    if constexpr (DB) dbacc += dsum.x + dsum.y;
    tmem_wait_st();
    tc_fence_before();
    mbar_arrive(ds_ready);
    if (quarter == 0) trace(2 + (w & 1), tstep, 6);
    return true;
}

// One query tile of a dK/dV sigma warpgroup (w: the warpgroup, which owns
// tile columns [kCols w, kCols (w + 1))); tS and tD are the TMEM addresses of
// its columns of S^T and dP^T in this thread's lane.  S^T, dP^T, P^T and dS^T
// complete one phase per tile, all of parity `par`.  Reads S^T and releases it
// (s_free); forms P^T = sigma(S^T) and sigma'; once dP^T is in (dp_full) writes
// P^T over the first half of its dP^T columns (p_ready), then dS^T =
// sigma' dP^T over the second half (ds_ready).  qvalid: queries of the tile
// below n_q (the others give P^T = dS^T = 0).  Returns false when a wait gave up.
template <int D, int MODE>
__device__ __forceinline__ bool dkdv_sigma_tile(uint32_t tS, uint32_t tD, int w, uint64_t *s_full,
                                                uint64_t *s_free, uint64_t *dp_full, uint64_t *p_ready,
                                                uint64_t *ds_ready, uint32_t par, const SigmoidCoef &cf,
                                                int qvalid, const WaitCtx &wctx, int tstep) {
    using SG = BwdSigma<D>;
    const int quarter = warp_id() & 3;
    float2 g[SG::kPacked];
    uint32_t pk[SG::kPacked];
    if (quarter == 0) trace(2 + (w & 1), tstep, 0);
    if (!__all_sync(0xffffffffu, mbar_wait(s_full, par, wctx))) return false;
    if (quarter == 0) trace(2 + (w & 1), tstep, 1);
    tc_fence_after();
    {
        uint32_t r[SG::kCols];
        tmem_ld_cols(tS, r);
        // S^T is in registers: the MMA warp may compute the next S^T now
        tc_fence_before();
        mbar_arrive(s_free);
#pragma unroll
        for (int ii = 0; ii < SG::kPacked; ++ii) {
            float2 pr;
            sigma_grad2<MODE>(scale2(__uint_as_float(r[2 * ii]), __uint_as_float(r[2 * ii + 1]), cf), pr, g[ii]);
            pk[ii] = pack_bf16x2(pr.x, pr.y);
        }
    }
    if (qvalid < 128) mask_packed(pk, SG::kCols * w, qvalid);
    if (quarter == 0) trace(2 + (w & 1), tstep, 2);
    if (!__all_sync(0xffffffffu, mbar_wait(dp_full, par, wctx))) return false;
    if (quarter == 0) trace(2 + (w & 1), tstep, 3);
    tc_fence_after();
    uint32_t ds[SG::kPacked];
    {
        // the first kPacked of this warpgroup's dP^T columns, then P^T over them
        uint32_t d[SG::kPacked];
        tmem_ld_cols(tD, d);
        tmem_st_cols(tD, pk);
#pragma unroll
        for (int ii = 0; ii < SG::kPacked / 2; ++ii) {
            const float2 v = mul2(g[ii], f2(__uint_as_float(d[2 * ii]), __uint_as_float(d[2 * ii + 1])));
            ds[ii] = pack_bf16x2(v.x, v.y);
        }
        tmem_wait_st();
        tc_fence_before();
        mbar_arrive(p_ready);
    }
    {
        // the other kPacked dP^T columns, then dS^T over them
        uint32_t d[SG::kPacked];
        tmem_ld_cols(tD + SG::kPacked, d);
#pragma unroll
        for (int ii = 0; ii < SG::kPacked / 2; ++ii) {
            const float2 v = mul2(g[SG::kPacked / 2 + ii],
                                  f2(__uint_as_float(d[2 * ii]), __uint_as_float(d[2 * ii + 1])));
            ds[SG::kPacked / 2 + ii] = pack_bf16x2(v.x, v.y);
        }
    }
    if (qvalid < 128) mask_packed(ds, SG::kCols * w, qvalid);
    tmem_st_cols(tD + SG::kPacked, ds);
    tmem_wait_st();
    tc_fence_before();
    mbar_arrive(ds_ready);
    if (quarter == 0) trace(2 + (w & 1), tstep, 4);
    return true;
}

// Sum of `v` over the 4 NG sigma warps of the block, in a fixed order (each
// warp's lanes by a butterfly, then the warps in warp order), written to *dst
// by warp 4.  Every sigma thread must call it; `red` holds 4 NG floats of
// shared memory.
template <int D>
__device__ __forceinline__ void sigma_block_sum(float v, float *red, float *dst) {
    using SG = BwdSigma<D>;
    const int warp = warp_id(), lane = lane_id();
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    if (lane == 0) red[warp - 4] = v;
    sigma_warps_sync(SG::kArrivals);
    if (warp == 4 && lane == 0) {
        float t = 0.0f;
        for (int u = 0; u < 4 * SG::NG; ++u) t += red[u];
        *dst = t;
    }
}

// ============================================================================
// dQ kernel: one CTA per 128-row query tile; streams K_j, V_j for j < ceil(n_k/128).
// TMEM: [0,128) S, [128,256) and [256,384) dP of even / odd key tiles (each
// overwritten by its dS, bf16 packed), [384,384+D) dQ.
//
// Per key tile j the warpgroups read S_j into registers and release it, then
// read dP_j 32 columns at a time and write dS_j = sigma'(S_j) dP_j over it,
// forming sigma' and dS in one pass so that the MUFU work of one chunk
// overlaps the multiplies and bf16 packing of the other (done one after the
// other, the two phases took ~1000 and ~490 clk per tile at D = 128).  The
// MMA thread issues S_{j+1} as soon as S_j is released and dP_{j+1} right
// after it into the other dP buffer (its dS_{j-1} is read by an earlier MMA of
// the same thread, and MMAs run in issue order), so both are ready when the
// warpgroups reach tile j+1; dQ += dS_j K_j follows when dS_j is ready.  The
// NG warpgroups (each with kCols tile columns) work on a tile at the same
// time, so that NG warps share each SM sub-partition's MUFU (one warp alone
// leaves it idle between issues).
// ============================================================================
// DB: also accumulate the bias gradient (p.db_part must then be set)
template <int D, int MODE, int SX, int SY, bool DB>
__global__ void __launch_bounds__(BwdSigma<D>::kThreads, 1)
    bwd_dq_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                  const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmDO,
                  const BwdParams p) {
    using Lay = BwdLayout<D, SX, SY>;
    using SG = BwdSigma<D>;
    constexpr uint32_t kColS = 0, kColDP0 = 128, kColDP1 = 256, kColDQ = 384;
    static_assert(kColDQ + D <= Lay::TMEM_COLS, "TMEM budget");
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = align_1k(smem_raw);
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + Lay::OFF_BAR);
    uint64_t *res_full = bars;
    uint64_t *x_full = bars + 1;              // K_j ring
    uint64_t *x_empty = x_full + SX;
    uint64_t *y_full = x_empty + SX;          // V_j ring
    uint64_t *y_empty = y_full + SY;
    uint64_t *s_full = y_empty + SY;          // MMA -> WGs: S_j in TMEM
    uint64_t *dp_full = s_full + 1;           // [2] MMA -> WGs: dP_j in buffer j % 2
    uint64_t *s_free = dp_full + 2;           // WGs -> MMA: S_j read
    uint64_t *ds_ready = s_free + 1;          // [2] WGs -> MMA: dS_j in buffer j % 2
    uint64_t *dq_done = ds_ready + 2;         // MMA -> all: dQ += dS_j K_j finished
    uint64_t *drain = dq_done + 1;
    static_assert(8 <= Lay::MAX_HANDOFF, "barrier count");
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + Lay::OFF_TMEM);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + Lay::OFF_ABORT);

    const int warp = warp_id(), lane = lane_id();

    // samples start by decreasing key length: warp 0 picks this block's sample
    BlockSample *sample_slot = reinterpret_cast<BlockSample *>(smem + Lay::OFF_SAMPLE);
    if (warp == 0) publish_block_sample(p.seqlens_q, p.seqlens_k, true, sample_slot);
    __syncthreads();
    const BlockSample bs = *sample_slot;
    const int z = bs.z, h = blockIdx.y, qtile = blockIdx.x;
    const int L = p.Lq;     // rows of this kernel's tiles and outputs: queries
    int nq = bs.nq, nk = bs.nk;
    if (nq < 0 || nq > L || nk < 0 || nk > p.Lk) {
        if (threadIdx.x == 0) record_status(p.status, kStatusSeqlenRange);
        nq = min(max(nq, 0), L);
        nk = min(max(nk, 0), p.Lk);
    }
    const int nkv = (nk + 127) / 128;
    if (qtile * 128 >= nq || nkv == 0) {
        // No valid (query, key) pair in this query tile: its dQ rows are zeros
        // (and so is its share of db), written by every thread; the block ends
        // here, before it sets up barriers or tensor memory.
        zero_rows<D>(p.dq, z, h, qtile * 128, min(128, L - qtile * 128), L, p.H);
        if constexpr (DB) {
            if (threadIdx.x == 0) p.db_part[(static_cast<size_t>(z) * p.H + h) * gridDim.x + qtile] = 0.0f;
        }
        return;
    }
    if (threadIdx.x == 0) {
        mbar_init(res_full, 1);
        for (int s = 0; s < SX; ++s) {
            mbar_init(&x_full[s], 1);
            mbar_init(&x_empty[s], 1);
        }
        for (int s = 0; s < SY; ++s) {
            mbar_init(&y_full[s], 1);
            mbar_init(&y_empty[s], 1);
        }
        mbar_init(s_full, 1);
        mbar_init(&dp_full[0], 1);
        mbar_init(&dp_full[1], 1);
        mbar_init(s_free, BwdSigma<D>::kArrivals);
        mbar_init(&ds_ready[0], BwdSigma<D>::kArrivals);
        mbar_init(&ds_ready[1], BwdSigma<D>::kArrivals);
        mbar_init(dq_done, 1);
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
        if (lane == 0) {
            uint8_t *sQ = smem + Lay::OFF_A, *sDO = smem + Lay::OFF_B;
            mbar_arrive_expect_tx(res_full, 2 * Lay::TILE_BYTES);
            for (int s = 0; s < Lay::NSUB; ++s) {
                tma_load_4d(&tmQ, res_full, sQ + s * Lay::SUB_BYTES, 64 * s, h, qtile * 128, z);
                tma_load_4d(&tmDO, res_full, sDO + s * Lay::SUB_BYTES, 64 * s, h, qtile * 128, z);
            }
            int ix = 0;
            for (int j = 0; j < nkv; ++j) {
                if (!ring_load<SX, Lay::NSUB>(&tmK, x_full, x_empty, smem + Lay::OFF_X, Lay::TILE_BYTES,
                                             j, h, z, wctx))
                    break;
                ix = j + 1;
            }
            mbar_wait_drain(res_full, 0, p.timeout_ns);
            ring_drain<SX>(x_full, ix, p.timeout_ns);
        }
    } else if (warp == 2) {
        // V_j ring, fed by its own thread so it never waits behind a key slot
        if (lane == 0) {
            int iy = 0;
            for (int j = 0; j < nkv; ++j) {
                if (!ring_load<SY, Lay::NSUB>(&tmV, y_full, y_empty, smem + Lay::OFF_Y, Lay::TILE_BYTES,
                                             j, h, z, wctx))
                    break;
                iy = j + 1;
            }
            ring_drain<SY>(y_full, iy, p.timeout_ns);
        }
    } else if (warp == 1) {
        // the whole warp runs converged; elect.sync picks the issuing lane
        {
            auto wait = [&](uint64_t *bar, uint32_t parity) {
                return __all_sync(0xffffffffu, mbar_wait(bar, parity, wctx));
            };
            const uint32_t idesc_s = idesc_bf16_f32(128, 128, false, false);
            const uint32_t idesc_q = idesc_bf16_f32(128, D, false, true);
            const uint32_t sQ = smem_u32(smem + Lay::OFF_A), sDO = smem_u32(smem + Lay::OFF_B);
            const uint32_t xring = smem_u32(smem + Lay::OFF_X), yring = smem_u32(smem + Lay::OFF_Y);
            auto kslot = [&](int j) { return xring + (j % SX) * Lay::TILE_BYTES; };
            auto vslot = [&](int j) { return yring + (j % SY) * Lay::TILE_BYTES; };
            // X (128 rows of Q or dO) times Y^T (128 rows of K or V) into TMEM column `col`
            auto issue_xyT = [&](uint32_t col, uint32_t xbase, uint32_t ybase) {
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk) {
                    const uint32_t koff = (kk >> 2) * Lay::SUB_BYTES + (kk & 3) * 32;
                    mma_ss_w(tmem + col, smem_desc_sw128(xbase + koff, 16, 1024),
                             smem_desc_sw128(ybase + koff, 16, 1024), idesc_s, kk > 0 ? 1u : 0u);
                }
            };
            bool ok = wait(res_full, 0) && wait(&x_full[0], 0) && wait(&y_full[0], 0);
            if (ok) {
                tc_fence_after();
                issue_xyT(kColS, sQ, kslot(0));
                mma_commit_w(s_full);
                issue_xyT(kColDP0, sDO, vslot(0));
                mma_commit_w(&dp_full[0]);
                mma_commit_w(&y_empty[0]);
            }
            for (int j = 0; ok && j < nkv; ++j) {
                const bool more = j + 1 < nkv;
                if (more) {
                    if (!(ok = wait(&x_full[(j + 1) % SX], ((j + 1) / SX) & 1))) break;
                    if (!(ok = wait(s_free, j & 1))) break;
                    if (lane == 0) trace(1, j, 0);
                    tc_fence_after();
                    issue_xyT(kColS, sQ, kslot(j + 1));
                    mma_commit_w(s_full);
                    if (!(ok = wait(&y_full[(j + 1) % SY], ((j + 1) / SY) & 1))) break;
                    // buffer (j+1) % 2 still holds dS_{j-1}: dQ += dS_{j-1} K_{j-1} was
                    // issued earlier by this thread and MMAs run in issue order
                    if (lane == 0) trace(1, j, 1);
                    tc_fence_after();
                    issue_xyT((j + 1) & 1 ? kColDP1 : kColDP0, sDO, vslot(j + 1));
                    mma_commit_w(&dp_full[(j + 1) & 1]);
                    mma_commit_w(&y_empty[(j + 1) % SY]);  // V_{j+1}: its only MMA
                }
                if (!(ok = wait(&ds_ready[j & 1], (j >> 1) & 1))) break;
                if (lane == 0) trace(1, j, 2);
                tc_fence_after();
                const uint32_t dcol = j & 1 ? kColDP1 : kColDP0;
                const uint32_t sK = kslot(j);
#pragma unroll
                for (int kk = 0; kk < 8; ++kk)
                    mma_ts_w(tmem + kColDQ, tmem + dcol + BwdSigma<D>::packed_col(kk),
                             smem_desc_sw128(sK + kk * 16 * 128, Lay::SUB_BYTES, 1024), idesc_q,
                             (j > 0 || kk > 0) ? 1u : 0u);
                mma_commit_w(&x_empty[j % SX]);           // K_j: S_j and dQ_j done
            }
            mma_commit_w(drain);
            mbar_wait_drain(drain, 0, p.timeout_ns);
            __syncwarp();
        }
    } else if (warp >= 4) {
        const int w = (warp - 4) >> 2;      // warpgroup: tile columns [kCols w, kCols (w + 1))
        const int quarter = warp & 3;
        const int row = qtile * 128 + quarter * 32 + lane;
        const uint32_t lane_bits = static_cast<uint32_t>(quarter * 32) << 16;
        __nv_bfloat16 *drow = p.dq + (static_cast<size_t>(z) * L + row) * (static_cast<size_t>(p.H) * D) +
                              static_cast<size_t>(h) * D;
        bool ok = true;
        float dbacc = 0.0f;   // bias gradient: sum of this row's dS (valid rows and keys)
        {
            const SigmoidCoef cf = make_coef<MODE>(p.alpha, bias_of(p.bias_z, p.bias, z));
            for (int j = 0; j < nkv; ++j) {
                ok = dq_sigma_tile<D, MODE, DB>(tmem + lane_bits, w, kColS, j & 1 ? kColDP1 : kColDP0, s_full,
                                                j & 1, s_free, &dp_full[j & 1], (j >> 1) & 1, &ds_ready[j & 1],
                                                cf, nk - j * 128, dbacc, wctx, j);
                if (!ok) break;
            }
            // every MMA of this CTA has finished once the MMA thread's final commit lands
            if (ok) ok = __all_sync(0xffffffffu, mbar_wait(drain, 0, wctx));
            // dQ's D columns split over the warpgroups, at least 32 each (with
            // four warpgroups at D = 64 the last two have none)
            constexpr int kEpi = D / SG::NG >= 32 ? D / SG::NG : 32;
            if (ok && w * kEpi < D) {
                tc_fence_after();
                store_row_from_tmem<D>(tmem + lane_bits + kColDQ, drow, row < L, row < nq,
                                       p.alpha, w * kEpi, kEpi);
            }
        }
        if constexpr (DB) {
            // one partial per CTA (rows at or beyond n_q add nothing)
            sigma_block_sum<D>(row < nq ? dbacc : 0.0f, reinterpret_cast<float *>(smem + Lay::OFF_RED),
                               &p.db_part[(static_cast<size_t>(z) * p.H + h) * gridDim.x + qtile]);
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
// dK/dV kernel: one CTA per 128-key tile; streams Q_i, dO_i for i < ceil(n_q/128).
// Works on the transposed scores (rows = keys):
//   S^T = K Q_i^T, dP^T = V dO_i^T, P^T and dS^T -> TMEM over dP^T,
//   dV += P^T dO_i, dK += dS^T Q_i.
// TMEM: [0,128) S^T, [128,256) dP^T, then P^T and dS^T over it,
// [256,256+D) dV, [256+D,256+2D) dK.
//
// A warpgroup reads its kCols columns of S^T into registers and releases the
// S^T buffer at once, so S^T_{i+1} is computed while it evaluates sigma and
// sigma' for tile i.  It keeps P^T in registers until it has read the first
// half of its dP^T columns, then writes P^T over them (its kCols tile columns
// packed two per TMEM column) and dS^T over the other half.  MMA order per query
// tile: S^T_{i+1} (as soon as S^T_i is read), dV_i, dK_i, dP^T_{i+1} (over P^T_i
// and dS^T_i, read by dV_i and dK_i just before: MMAs from one thread run in
// issue order).
// ============================================================================
template <int D, int MODE, int SX, int SY>
__global__ void __launch_bounds__(BwdSigma<D>::kThreads, 1)
    bwd_dkdv_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                    const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmDO,
                    const BwdParams p) {
    using Lay = BwdLayout<D, SX, SY>;
    using SG = BwdSigma<D>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = align_1k(smem_raw);
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + Lay::OFF_BAR);
    uint64_t *res_full = bars;
    uint64_t *x_full = bars + 1;              // Q_i ring
    uint64_t *x_empty = x_full + SX;
    uint64_t *y_full = x_empty + SX;          // dO_i ring
    uint64_t *y_empty = y_full + SY;
    uint64_t *s_full = y_empty + SY;          // MMA -> WGs: S^T_i in TMEM
    uint64_t *dp_full = s_full + 1;           // MMA -> WGs: dP^T_i in TMEM
    uint64_t *s_free = dp_full + 1;           // WGs -> MMA: S^T_i read
    uint64_t *p_ready = s_free + 1;           // WGs -> MMA: P^T_i in TMEM
    uint64_t *ds_ready = p_ready + 1;         // WGs -> MMA: dS^T_i in TMEM
    uint64_t *drain = ds_ready + 1;
    static_assert(6 <= Lay::MAX_HANDOFF, "barrier count");
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + Lay::OFF_TMEM);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + Lay::OFF_ABORT);

    const int warp = warp_id(), lane = lane_id();

    // samples start by decreasing query length: warp 0 picks this block's sample
    BlockSample *sample_slot = reinterpret_cast<BlockSample *>(smem + Lay::OFF_SAMPLE);
    if (warp == 0) publish_block_sample(p.seqlens_q, p.seqlens_k, false, sample_slot);
    __syncthreads();
    const BlockSample bs = *sample_slot;
    const int z = bs.z, h = blockIdx.y, ktile = blockIdx.x;
    const int L = p.Lk;     // rows of this kernel's tiles and outputs: keys
    int nq = bs.nq, nk = bs.nk;
    if (nq < 0 || nq > p.Lq || nk < 0 || nk > L) {
        if (threadIdx.x == 0) record_status(p.status, kStatusSeqlenRange);
        nq = min(max(nq, 0), p.Lq);
        nk = min(max(nk, 0), L);
    }
    const int nqt = (nq + 127) / 128;
    if (ktile * 128 >= nk || nqt == 0) {
        // No valid (query, key) pair for this key tile: its dK and dV rows are
        // zeros, written by every thread; the block ends here.
        const int rows = min(128, L - ktile * 128);
        zero_rows<D>(p.dk, z, h, ktile * 128, rows, L, p.H);
        zero_rows<D>(p.dv, z, h, ktile * 128, rows, L, p.H);
        return;
    }
    if (threadIdx.x == 0) {
        mbar_init(res_full, 1);
        for (int s = 0; s < SX; ++s) {
            mbar_init(&x_full[s], 1);
            mbar_init(&x_empty[s], 1);
        }
        for (int s = 0; s < SY; ++s) {
            mbar_init(&y_full[s], 1);
            mbar_init(&y_empty[s], 1);
        }
        mbar_init(s_full, 1);
        mbar_init(dp_full, 1);
        mbar_init(s_free, BwdSigma<D>::kArrivals);
        mbar_init(p_ready, BwdSigma<D>::kArrivals);
        mbar_init(ds_ready, BwdSigma<D>::kArrivals);
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
        if (lane == 0) {
            uint8_t *sK = smem + Lay::OFF_A, *sV = smem + Lay::OFF_B;
            mbar_arrive_expect_tx(res_full, 2 * Lay::TILE_BYTES);
            for (int s = 0; s < Lay::NSUB; ++s) {
                tma_load_4d(&tmK, res_full, sK + s * Lay::SUB_BYTES, 64 * s, h, ktile * 128, z);
                tma_load_4d(&tmV, res_full, sV + s * Lay::SUB_BYTES, 64 * s, h, ktile * 128, z);
            }
            int ix = 0;
            for (int i = 0; i < nqt; ++i) {
                if (!ring_load<SX, Lay::NSUB>(&tmQ, x_full, x_empty, smem + Lay::OFF_X, Lay::TILE_BYTES,
                                             i, h, z, wctx))
                    break;
                ix = i + 1;
                trace(0, i, 0);
            }
            mbar_wait_drain(res_full, 0, p.timeout_ns);
            ring_drain<SX>(x_full, ix, p.timeout_ns);
        }
    } else if (warp == 2) {
        // dO_i ring, fed by its own thread so it never waits behind a query slot
        if (lane == 0) {
            int iy = 0;
            for (int i = 0; i < nqt; ++i) {
                if (!ring_load<SY, Lay::NSUB>(&tmDO, y_full, y_empty, smem + Lay::OFF_Y, Lay::TILE_BYTES,
                                             i, h, z, wctx))
                    break;
                iy = i + 1;
                trace(0, i, 1);
            }
            ring_drain<SY>(y_full, iy, p.timeout_ns);
        }
    } else if (warp == 1) {
        // the whole warp runs converged; elect.sync picks the issuing lane
        {
            auto wait = [&](uint64_t *bar, uint32_t parity) {
                return __all_sync(0xffffffffu, mbar_wait(bar, parity, wctx));
            };
            const uint32_t idesc_s = idesc_bf16_f32(128, 128, false, false);
            const uint32_t idesc_kv = idesc_bf16_f32(128, D, false, true);
            const uint32_t sK = smem_u32(smem + Lay::OFF_A), sV = smem_u32(smem + Lay::OFF_B);
            const uint32_t xring = smem_u32(smem + Lay::OFF_X), yring = smem_u32(smem + Lay::OFF_Y);
            auto qslot = [&](int i) { return xring + (i % SX) * Lay::TILE_BYTES; };
            auto doslot = [&](int i) { return yring + (i % SY) * Lay::TILE_BYTES; };
            // descriptors as low words (start and LBO) plus the K step's offset >> 4
            constexpr uint32_t kDescHi = desc_hi(1024);
            auto issue_xyT = [&](uint32_t col, uint32_t xbase, uint32_t ybase) {
                const uint32_t x_lo = desc_lo(xbase, 16), y_lo = desc_lo(ybase, 16);
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk) {
                    const uint32_t koff = ((kk >> 2) * Lay::SUB_BYTES + (kk & 3) * 32) >> 4;
                    mma_ss_lhw(tmem + col, x_lo + koff, y_lo + koff, kDescHi, idesc_s, kk > 0 ? 1u : 0u);
                }
            };
            // acc += A(TMEM, packed over `acol`) * B (128 query rows, MN-major)
            auto issue_acc = [&](uint32_t acc, uint32_t acol, uint32_t bbase, bool first) {
                const uint32_t b_lo = desc_lo(bbase, Lay::SUB_BYTES);
#pragma unroll
                for (int kk = 0; kk < 8; ++kk)
                    mma_ts_lhw(tmem + acc, tmem + acol + BwdSigma<D>::packed_col(kk), b_lo + kk * ((16 * 128) >> 4),
                               kDescHi, idesc_kv, (!first || kk > 0) ? 1u : 0u);
            };
            bool ok = wait(res_full, 0) && wait(&x_full[0], 0) && wait(&y_full[0], 0);
            if (ok) {
                tc_fence_after();
                issue_xyT(Lay::COL_S, sK, qslot(0));
                mma_commit_w(s_full);
                issue_xyT(Lay::COL_DP, sV, doslot(0));
                mma_commit_w(dp_full);
            }
            for (int i = 0; ok && i < nqt; ++i) {
                const bool more = i + 1 < nqt;
                if (more) {
                    // S^T_{i+1} into the S^T buffer as soon as the warpgroups have read S^T_i
                    if (!(ok = wait(&x_full[(i + 1) % SX], ((i + 1) / SX) & 1))) break;
                    if (!(ok = wait(s_free, i & 1))) break;
                    if (lane == 0) trace(1, i, 0);
                    tc_fence_after();
                    issue_xyT(Lay::COL_S, sK, qslot(i + 1));
                    mma_commit_w(s_full);
                }
                if (!(ok = wait(p_ready, i & 1))) break;
                if (lane == 0) trace(1, i, 1);
                tc_fence_after();
                issue_acc(Lay::COL_ACC0, Lay::COL_DP, doslot(i), i == 0);       // dV += P^T dO_i
                mma_commit_w(&y_empty[i % SY]);                                 // dO_i: dP^T_i, dV_i done
                if (!(ok = wait(ds_ready, i & 1))) break;
                if (lane == 0) trace(1, i, 2);
                tc_fence_after();
                issue_acc(Lay::COL_ACC1, Lay::COL_DP + SG::kPacked, qslot(i), i == 0);  // dK += dS^T Q_i
                mma_commit_w(&x_empty[i % SX]);                                 // Q_i: S^T_i, dK_i done
                if (more) {
                    // dP^T_{i+1} overwrites P^T_i and dS^T_i, read by the two MMAs just
                    // issued (MMAs run in issue order)
                    if (!(ok = wait(&y_full[(i + 1) % SY], ((i + 1) / SY) & 1))) break;
                    if (lane == 0) trace(1, i, 3);
                    tc_fence_after();
                    issue_xyT(Lay::COL_DP, sV, doslot(i + 1));
                    mma_commit_w(dp_full);
                }
            }
            mma_commit_w(drain);
            mbar_wait_drain(drain, 0, p.timeout_ns);
            __syncwarp();
        }
    } else if (warp >= 4) {
        const int w = (warp - 4) >> 2;      // warpgroup: query columns [kCols w, kCols (w + 1))
        const int quarter = warp & 3;
        const int row = ktile * 128 + quarter * 32 + lane;   // key row
        const uint32_t lane_bits = static_cast<uint32_t>(quarter * 32) << 16;
        const size_t roff = (static_cast<size_t>(z) * L + row) * (static_cast<size_t>(p.H) * D) +
                            static_cast<size_t>(h) * D;
        // epilogue: the first half of the warpgroups writes dV, the second dK,
        // D / kOut columns each
        constexpr int kOut = SG::NG / 2;
        const bool is_dv = w < kOut;
        __nv_bfloat16 *dst = (is_dv ? p.dv : p.dk) + roff;
        bool ok = true;
        {
            const SigmoidCoef cf = make_coef<MODE>(p.alpha, bias_of(p.bias_z, p.bias, z));
            const uint32_t tS = tmem + lane_bits + Lay::COL_S + SG::kCols * w;
            const uint32_t tD = tmem + lane_bits + Lay::COL_DP + SG::kCols * w;
            for (int i = 0; i < nqt; ++i) {
                ok = dkdv_sigma_tile<D, MODE>(tS, tD, w, s_full, s_free, dp_full, p_ready, ds_ready, i & 1, cf,
                                              nq - i * 128, wctx, i);
                if (!ok) break;
            }
            // every MMA of this CTA has finished once the MMA thread's final commit lands
            if (ok) ok = __all_sync(0xffffffffu, mbar_wait(drain, 0, wctx));
            if (ok) {
                tc_fence_after();
                store_row_from_tmem<D>(tmem + lane_bits + (is_dv ? Lay::COL_ACC0 : Lay::COL_ACC1), dst,
                                       row < L, row < nk, is_dv ? 1.0f : p.alpha, (w % kOut) * (D / kOut),
                                       D / kOut);
            }
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

// db_z = sum of the per-CTA (or per-row) partials of sample z, in double and in
// a fixed order: thread t adds partials t, t + 256, ...; then a fixed tree.
__global__ void __launch_bounds__(256) dbias_reduce_kernel(const float *part, int64_t per_z,
                                                           float *dbias) {
    __shared__ double red[256];
    const int z = blockIdx.x;
    double acc = 0.0;
    for (int64_t t = threadIdx.x; t < per_z; t += 256) acc += part[z * per_z + t];
    red[threadIdx.x] = acc;
    __syncthreads();
    for (int s = 128; s > 0; s >>= 1) {
        if (static_cast<int>(threadIdx.x) < s) red[threadIdx.x] += red[threadIdx.x + s];
        __syncthreads();
    }
    if (threadIdx.x == 0) dbias[z] = static_cast<float>(red[0]);
}

}  // namespace sigattn
