// fp32 accuracy path: the same operation on CUDA cores, one warp per output
// row, fp32 arithmetic throughout and sigma through the library expf:
//   u = e^-|x|,  r = 1 / (1 + u),  sigma = r (x >= 0) or u r (x < 0),
//   sigma' = sigma(x) sigma(-x) = u r^2   (no cancellation in either tail).
// Meant for accuracy checks at small sizes, not for speed.
#pragma once

#include <stdint.h>

#include "sm100.cuh"
#include "sigmoid.cuh"

namespace sigattn {

__device__ __forceinline__ void exact_sigma(float x, float &p, float &g) {
    float u = expf(-fabsf(x));
    float r = 1.0f / (1.0f + u);
    float ur = u * r;
    p = x >= 0.0f ? r : ur;
    g = ur * r;
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

struct F32Params {
    const float *q, *k, *v, *dout;
    float *o, *dq, *dk, *dv;
    const int *seqlens_q, *seqlens_k;
    int Z, Lq, Lk, H;       // batch, padded lengths of Q / dO / O / dQ and of K / V / dK / dV
    float alpha, bias;
    int *status;
    const float *bias_z;   // device float[Z], one bias per sample; null: the scalar `bias`
    float *db_part;        // dQ kernel: sum of dS per row ([Z][L][H] order), or null
};

__device__ __forceinline__ void clamp_lengths(const F32Params &p, int z, int &nq, int &nk) {
    nq = p.seqlens_q[z];
    nk = p.seqlens_k[z];
    if (nq < 0 || nq > p.Lq || nk < 0 || nk > p.Lk) {
        if ((threadIdx.x & 31) == 0) record_status(p.status, kStatusSeqlenRange);
        nq = min(max(nq, 0), p.Lq);
        nk = min(max(nk, 0), p.Lk);
    }
}

// rows are enumerated in [Z][L][H] order (L = Lq for query rows, Lk for key
// rows), so row r starts at r * D
template <int D>
__global__ void __launch_bounds__(256) f32_fwd_kernel(const F32Params p) {
    constexpr int E = D / 32;
    const int64_t r = static_cast<int64_t>(blockIdx.x) * 8 + (threadIdx.x >> 5);
    const int lane = threadIdx.x & 31;
    const int64_t rows = static_cast<int64_t>(p.Z) * p.Lq * p.H;
    if (r >= rows) return;
    const int h = static_cast<int>(r % p.H);
    const int i = static_cast<int>((r / p.H) % p.Lq);
    const int z = static_cast<int>(r / (static_cast<int64_t>(p.H) * p.Lq));
    int nq, nk;
    clamp_lengths(p, z, nq, nk);
    const float bias = bias_of(p.bias_z, p.bias, z);
    float acc[E];
#pragma unroll
    for (int e = 0; e < E; ++e) acc[e] = 0.0f;
    if (i < nq) {
        float qv[E];
#pragma unroll
        for (int e = 0; e < E; ++e) qv[e] = p.q[r * D + lane + 32 * e];
        for (int j = 0; j < nk; ++j) {
            const int64_t kr = (static_cast<int64_t>(z) * p.Lk + j) * p.H + h;
            float s = 0.0f;
#pragma unroll
            for (int e = 0; e < E; ++e) s = fmaf(qv[e], p.k[kr * D + lane + 32 * e], s);
            s = warp_sum(s);
            float pr, g;
            exact_sigma(fmaf(p.alpha, s, bias), pr, g);
#pragma unroll
            for (int e = 0; e < E; ++e) acc[e] = fmaf(pr, p.v[kr * D + lane + 32 * e], acc[e]);
        }
    }
#pragma unroll
    for (int e = 0; e < E; ++e) p.o[r * D + lane + 32 * e] = acc[e];
}

template <int D>
__global__ void __launch_bounds__(256) f32_dq_kernel(const F32Params p) {
    constexpr int E = D / 32;
    const int64_t r = static_cast<int64_t>(blockIdx.x) * 8 + (threadIdx.x >> 5);
    const int lane = threadIdx.x & 31;
    const int64_t rows = static_cast<int64_t>(p.Z) * p.Lq * p.H;
    if (r >= rows) return;
    const int h = static_cast<int>(r % p.H);
    const int i = static_cast<int>((r / p.H) % p.Lq);
    const int z = static_cast<int>(r / (static_cast<int64_t>(p.H) * p.Lq));
    int nq, nk;
    clamp_lengths(p, z, nq, nk);
    const float bias = bias_of(p.bias_z, p.bias, z);
    float acc[E];
#pragma unroll
    for (int e = 0; e < E; ++e) acc[e] = 0.0f;
    float dbacc = 0.0f;   // sum of this row's dS over keys below n_k
    if (i < nq) {
        float qv[E], gv[E];
#pragma unroll
        for (int e = 0; e < E; ++e) {
            qv[e] = p.q[r * D + lane + 32 * e];
            gv[e] = p.dout[r * D + lane + 32 * e];
        }
        for (int j = 0; j < nk; ++j) {
            const int64_t kr = (static_cast<int64_t>(z) * p.Lk + j) * p.H + h;
            float s = 0.0f, dp = 0.0f;
#pragma unroll
            for (int e = 0; e < E; ++e) {
                s = fmaf(qv[e], p.k[kr * D + lane + 32 * e], s);
                dp = fmaf(gv[e], p.v[kr * D + lane + 32 * e], dp);
            }
            s = warp_sum(s);
            dp = warp_sum(dp);
            float pr, g;
            exact_sigma(fmaf(p.alpha, s, bias), pr, g);
            const float ds = g * dp;
            dbacc += ds;
#pragma unroll
            for (int e = 0; e < E; ++e) acc[e] = fmaf(ds, p.k[kr * D + lane + 32 * e], acc[e]);
        }
    }
#pragma unroll
    for (int e = 0; e < E; ++e) p.dq[r * D + lane + 32 * e] = p.alpha * acc[e];
    if (p.db_part != nullptr && lane == 0) p.db_part[r] = dbacc;
}

template <int D>
__global__ void __launch_bounds__(256) f32_dkdv_kernel(const F32Params p) {
    constexpr int E = D / 32;
    const int64_t r = static_cast<int64_t>(blockIdx.x) * 8 + (threadIdx.x >> 5);
    const int lane = threadIdx.x & 31;
    const int64_t rows = static_cast<int64_t>(p.Z) * p.Lk * p.H;
    if (r >= rows) return;
    const int h = static_cast<int>(r % p.H);
    const int j = static_cast<int>((r / p.H) % p.Lk);
    const int z = static_cast<int>(r / (static_cast<int64_t>(p.H) * p.Lk));
    int nq, nk;
    clamp_lengths(p, z, nq, nk);
    const float bias = bias_of(p.bias_z, p.bias, z);
    float ak[E], av[E];
#pragma unroll
    for (int e = 0; e < E; ++e) ak[e] = av[e] = 0.0f;
    if (j < nk) {
        float kv[E], vv[E];
#pragma unroll
        for (int e = 0; e < E; ++e) {
            kv[e] = p.k[r * D + lane + 32 * e];
            vv[e] = p.v[r * D + lane + 32 * e];
        }
        for (int i = 0; i < nq; ++i) {
            const int64_t qr = (static_cast<int64_t>(z) * p.Lq + i) * p.H + h;
            float s = 0.0f, dp = 0.0f;
#pragma unroll
            for (int e = 0; e < E; ++e) {
                s = fmaf(p.q[qr * D + lane + 32 * e], kv[e], s);
                dp = fmaf(p.dout[qr * D + lane + 32 * e], vv[e], dp);
            }
            s = warp_sum(s);
            dp = warp_sum(dp);
            float pr, g;
            exact_sigma(fmaf(p.alpha, s, bias), pr, g);
            const float ds = g * dp;
#pragma unroll
            for (int e = 0; e < E; ++e) {
                av[e] = fmaf(pr, p.dout[qr * D + lane + 32 * e], av[e]);
                ak[e] = fmaf(ds, p.q[qr * D + lane + 32 * e], ak[e]);
            }
        }
    }
#pragma unroll
    for (int e = 0; e < E; ++e) {
        p.dv[r * D + lane + 32 * e] = av[e];
        p.dk[r * D + lane + 32 * e] = p.alpha * ak[e];
    }
}

// The bf16 kernels' sigma routine on an array (alpha = 1, b = 0).
template <int MODE>
__global__ void sigmoid_eval_kernel(const float *x, float *y, float *dy, int64_t n) {
    const int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
    if (i >= n) return;
    const SigmoidCoef cf = make_coef<MODE>(1.0f, 0.0f);
    const float2 a = scale2(x[i], x[i], cf);
    float2 pr, g;
    sigma_grad2<MODE>(a, pr, g);
    y[i] = sigma2<MODE>(a).x;
    if (dy != nullptr) dy[i] = g.x;
}

// Waits on a barrier that nothing signals; the bounded wait must give up,
// record the timeout and let the kernel exit normally.
__global__ void wait_timeout_selftest_kernel(int *status, uint64_t timeout_ns) {
    __shared__ uint64_t bar;
    __shared__ int abort_flag;
    if (threadIdx.x == 0) {
        mbar_init(&bar, 1);
        abort_flag = 0;
        fence_barrier_init();
    }
    __syncthreads();
    const WaitCtx w{&abort_flag, status, timeout_ns};
    (void)mbar_wait(&bar, 0, w);
    __syncthreads();
}

}  // namespace sigattn
