/*
 * Plain fp64 CPU oracle for padding-aware bidirectional sigmoid attention.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path may include, link or
 * call this file: only the test suite, the smoke check and the benchmark's CPU
 * baseline use it.  It shares no code, header or constant with the CUDA path.
 *
 * What it computes (all arithmetic in double, on the exact input values):
 *
 *   gist.science summary, section 2.A (sigmoid attention mechanism):
 *       O = sigma(Q K^T / sqrt(d) + b) V,  sigma(x) = 1 / (1 + e^-x),
 *       applied element-wise with no row normalisation; alpha generalises
 *       1/sqrt(d) as in the paper.rainbus.top summary, method step (2)
 *       ("S = Q K^T alpha + b").
 *   paper.rainbus.top summary, method steps (1)-(2): inputs are Z x L x H x D
 *       with per-sample true lengths n_q, n_k; key positions at or beyond n_k
 *       get -inf added, i.e. weight sigma = 0; query rows at or beyond n_q are
 *       written as zero.
 *   paper.rainbus.top summary, method step (4): dS = P (1 - P) (dO V^T);
 *       dQ = alpha dS K; dK/dV by the transposed view: dK = alpha dS^T Q,
 *       dV = P^T dO.  Padded query rows are constants (written as zero), so no
 *       gradient flows from them: their dO is ignored.
 *   paperlayer.ai summary, section 3 (background on sigmoid attention) and
 *       gist.science summary, section 2.A (bias term): the bias is set to
 *       b = -log(n); here b may differ per sample (bias_z[z], e.g. -ln n_z),
 *       and since x_ij = alpha q_i.k_j + b_z, the gradient of a per-sample
 *       bias is db_z = sum over heads and valid (i, j) of dS_ij.
 *
 * Readings where the pages are silent are listed in the design notes; here:
 *   - the -inf mask is applied by selection (P = 0), never by adding -inf;
 *   - sigma is the exact logistic function, not the tanh approximation the
 *     kernel pages describe (the approximation is what the oracle judges).
 *
 * Layout of every tensor: [Z][L][H][D], contiguous; element (z,l,h,d) sits at
 * ((z*L + l)*H + h)*D + d, with L = Lq for Q, dO and the query-side outputs
 * (O, dQ) and L = Lk for K, V, dK, dV (Lq = Lk for self-attention; a shorter
 * query slice against all keys is the context-parallel case).
 * dtype 0 = bf16 (raw uint16 bits), 1 = fp32.
 * Row lists are int64 triples (z, h, row).  Outputs are double, D per row.
 * bias_z holds one bias per sample (double[Z]).
 *
 * Parallelism: OpenMP over independent rows only; each row is summed in
 * ascending index order, exactly as the definition reads.
 */
#include <math.h>
#include <stdint.h>
#include <string.h>

/* Exact widening of one stored element to double. */
static double load_elem(const void *base, int dtype, int64_t idx) {
    if (dtype == 0) {
        uint16_t b = ((const uint16_t *)base)[idx];
        uint32_t bits = ((uint32_t)b) << 16;
        float f;
        memcpy(&f, &bits, sizeof f);
        return (double)f;
    }
    return (double)((const float *)base)[idx];
}

static int64_t offset_of(int64_t z, int64_t l, int64_t h, int L, int H, int D) {
    return ((z * L + l) * H + h) * (int64_t)D;
}

/* logistic function, gist.science summary section 2.A; both branches are the
 * same closed form, written so that exp never overflows. */
double oracle_sigmoid(double x) {
    if (x >= 0.0) return 1.0 / (1.0 + exp(-x));
    double e = exp(x);
    return e / (1.0 + e);
}

/* its derivative as the pages state it: sigma'(x) = sigma(x) (1 - sigma(x)) */
double oracle_sigmoid_grad(double x) {
    double p = oracle_sigmoid(x);
    return p * (1.0 - p);
}

/* score x_ij = alpha * sum_d Q[i,d] K[j,d] + b for one (z, h); Q and dO rows are
 * laid out with the query length Lq, K and V rows with the key length Lk */
static double score(const void *q, const void *k, int dtype, int64_t z, int64_t h,
                    int64_t i, int64_t j, int Lq, int Lk, int H, int D, double alpha,
                    double bias) {
    int64_t qo = offset_of(z, i, h, Lq, H, D), ko = offset_of(z, j, h, Lk, H, D);
    double s = 0.0;
    for (int d = 0; d < D; ++d) s += load_elem(q, dtype, qo + d) * load_elem(k, dtype, ko + d);
    return alpha * s + bias;
}

/* sum_d A[i,d] B[j,d] with A in the query layout (Lq) and B in the key layout (Lk) */
static double dot_rows(const void *a, const void *b, int dtype, int64_t z, int64_t h,
                       int64_t i, int64_t j, int Lq, int Lk, int H, int D) {
    int64_t ao = offset_of(z, i, h, Lq, H, D), bo = offset_of(z, j, h, Lk, H, D);
    double s = 0.0;
    for (int d = 0; d < D; ++d) s += load_elem(a, dtype, ao + d) * load_elem(b, dtype, bo + d);
    return s;
}

static int clamp_len(int n, int L) { return n < 0 ? 0 : (n > L ? L : n); }

/* Forward rows: O[z, i, h, :] = [i < n_q] sum_{j < n_k} sigma(x_ij) V[z, j, h, :]. */
void oracle_fwd_rows(const void *q, const void *k, const void *v, int dtype,
                     int Z, int Lq, int Lk, int H, int D, const int32_t *nq, const int32_t *nk,
                     double alpha, const double *bias_z, const int64_t *items, int64_t nitems,
                     double *out) {
    (void)Z;
#pragma omp parallel for schedule(dynamic, 4)
    for (int64_t t = 0; t < nitems; ++t) {
        int64_t z = items[3 * t], h = items[3 * t + 1], i = items[3 * t + 2];
        double *o = out + t * D;
        for (int d = 0; d < D; ++d) o[d] = 0.0;
        int n_q = clamp_len(nq[z], Lq), n_k = clamp_len(nk[z], Lk);
        const double bias = bias_z[z];
        if (i >= n_q) continue;
        for (int64_t j = 0; j < n_k; ++j) {
            double p = oracle_sigmoid(score(q, k, dtype, z, h, i, j, Lq, Lk, H, D, alpha, bias));
            int64_t vo = offset_of(z, j, h, Lk, H, D);
            for (int d = 0; d < D; ++d) o[d] += p * load_elem(v, dtype, vo + d);
        }
    }
}

/* dQ rows: dQ[z, i, h, :] = [i < n_q] alpha sum_{j < n_k} dS_ij K[z, j, h, :],
 * dS_ij = P_ij (1 - P_ij) (dO_i . V_j). */
void oracle_dq_rows(const void *q, const void *k, const void *v, const void *dout, int dtype,
                    int Z, int Lq, int Lk, int H, int D, const int32_t *nq, const int32_t *nk,
                    double alpha, const double *bias_z, const int64_t *items, int64_t nitems,
                    double *out) {
    (void)Z;
#pragma omp parallel for schedule(dynamic, 4)
    for (int64_t t = 0; t < nitems; ++t) {
        int64_t z = items[3 * t], h = items[3 * t + 1], i = items[3 * t + 2];
        double *g = out + t * D;
        for (int d = 0; d < D; ++d) g[d] = 0.0;
        int n_q = clamp_len(nq[z], Lq), n_k = clamp_len(nk[z], Lk);
        const double bias = bias_z[z];
        if (i >= n_q) continue;
        for (int64_t j = 0; j < n_k; ++j) {
            double p = oracle_sigmoid(score(q, k, dtype, z, h, i, j, Lq, Lk, H, D, alpha, bias));
            double dp = dot_rows(dout, v, dtype, z, h, i, j, Lq, Lk, H, D);
            double ds = p * (1.0 - p) * dp;
            int64_t ko = offset_of(z, j, h, Lk, H, D);
            for (int d = 0; d < D; ++d) g[d] += ds * load_elem(k, dtype, ko + d);
        }
        for (int d = 0; d < D; ++d) g[d] *= alpha;
    }
}

/* dK and dV rows for key j:
 *   dV[z, j, h, :] = [j < n_k] sum_{i < n_q} P_ij dO[z, i, h, :]
 *   dK[z, j, h, :] = [j < n_k] alpha sum_{i < n_q} dS_ij Q[z, i, h, :] */
void oracle_dkdv_rows(const void *q, const void *k, const void *v, const void *dout, int dtype,
                      int Z, int Lq, int Lk, int H, int D, const int32_t *nq, const int32_t *nk,
                      double alpha, const double *bias_z, const int64_t *items, int64_t nitems,
                      double *dk_out, double *dv_out) {
    (void)Z;
#pragma omp parallel for schedule(dynamic, 4)
    for (int64_t t = 0; t < nitems; ++t) {
        int64_t z = items[3 * t], h = items[3 * t + 1], j = items[3 * t + 2];
        double *gk = dk_out + t * D, *gv = dv_out + t * D;
        for (int d = 0; d < D; ++d) { gk[d] = 0.0; gv[d] = 0.0; }
        int n_q = clamp_len(nq[z], Lq), n_k = clamp_len(nk[z], Lk);
        const double bias = bias_z[z];
        if (j >= n_k) continue;
        for (int64_t i = 0; i < n_q; ++i) {
            double p = oracle_sigmoid(score(q, k, dtype, z, h, i, j, Lq, Lk, H, D, alpha, bias));
            double dp = dot_rows(dout, v, dtype, z, h, i, j, Lq, Lk, H, D);
            double ds = p * (1.0 - p) * dp;
            int64_t qo = offset_of(z, i, h, Lq, H, D);
            for (int d = 0; d < D; ++d) {
                gv[d] += p * load_elem(dout, dtype, qo + d);
                gk[d] += ds * load_elem(q, dtype, qo + d);
            }
        }
        for (int d = 0; d < D; ++d) gk[d] *= alpha;
    }
}

/* Bias gradient per sample: db_z = sum_h sum_{i < n_q} sum_{j < n_k} dS_ij with
 * dS_ij = P_ij (1 - P_ij) (dO_i . V_j).  One partial per (z, h, i) row, each summed
 * in ascending j; the partials are then added in ascending (h, i) order per
 * sample, so the result does not depend on the thread count. */
void oracle_dbias(const void *q, const void *k, const void *v, const void *dout, int dtype,
                  int Z, int Lq, int Lk, int H, int D, const int32_t *nq, const int32_t *nk,
                  double alpha, const double *bias_z, double *rowsum, double *dbias) {
    const int64_t nrows = (int64_t)Z * H * Lq;
#pragma omp parallel for schedule(dynamic, 4)
    for (int64_t t = 0; t < nrows; ++t) {
        int64_t z = t / ((int64_t)H * Lq), h = (t / Lq) % H, i = t % Lq;
        double acc = 0.0;
        int n_q = clamp_len(nq[z], Lq), n_k = clamp_len(nk[z], Lk);
        const double bias = bias_z[z];
        if (i < n_q) {
            for (int64_t j = 0; j < n_k; ++j) {
                double p = oracle_sigmoid(score(q, k, dtype, z, h, i, j, Lq, Lk, H, D, alpha, bias));
                double dp = dot_rows(dout, v, dtype, z, h, i, j, Lq, Lk, H, D);
                acc += p * (1.0 - p) * dp;
            }
        }
        rowsum[t] = acc;
    }
    for (int64_t z = 0; z < Z; ++z) {
        double s = 0.0;
        for (int64_t r = 0; r < (int64_t)H * Lq; ++r) s += rowsum[z * H * Lq + r];
        dbias[z] = s;
    }
}

/* Number of OpenMP threads the oracle runs with (for reporting). */
int oracle_num_threads(void) {
#ifdef _OPENMP
    extern int omp_get_max_threads(void);
    return omp_get_max_threads();
#else
    return 1;
#endif
}
