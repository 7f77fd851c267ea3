/*
 * sigattn — padding-aware bidirectional sigmoid self-attention on NVIDIA B200
 * (sm_100a).  C ABI of libsigattn.so.
 *
 * The operation (gist.science summary of "Better Models, Faster Training:
 * Sigmoid Attention for single-cell Foundation Models", section 2.A, and the
 * paper.rainbus.top summary of the same paper, method steps (1)-(5)):
 *
 *   S  = alpha * Q K^T + b                        per sample z and head h
 *   P  = sigma(S) with P[i, j] = 0 for keys j >= n_k(z)   (the "-inf" mask)
 *   O  = P V, and O[i, :] = 0 for query rows i >= n_q(z)
 *   dS = P (1 - P) (dO V^T)          (padded query rows carry no gradient)
 *   dQ = alpha dS K,  dK = alpha dS^T Q,  dV = P^T dO
 *
 * sigma is the logistic function 1 / (1 + e^-x); there is no row
 * normalisation.  The backward recomputes P (method step (5)); it needs
 * neither O nor any saved statistic.
 *
 * Layout of every tensor argument: [Z][L][H][D], contiguous, row-major:
 * element (z, l, h, d) at ((z * L + l) * H + h) * D + d.  Z = batch, L =
 * padded length, H = heads, D = head dimension.  Base pointers must be
 * 16-byte aligned (every pointer PyTorch allocates is).
 *
 * Sequence lengths are int32[Z] arrays in DEVICE memory (n_q and n_k may
 * differ).  They are read by the kernels, not by the host.  Values outside
 * [0, L] are clamped on the device and flag SIGATTN_ERR_SEQLEN_RANGE in the
 * device status word (see sigattn_last_device_status).
 *
 * Ownership: the caller owns and allocates every buffer; calls allocate
 * no device memory per call.  The library lazily allocates, once per device,
 * a small device status buffer that lives until process exit.  In host
 * memory it caches the TMA tensor maps it encodes, keyed by (base address,
 * Z, L, H, D), which is all a map depends on (at most 1024, then the cache is
 * emptied).
 *
 * CUDA graphs: the compute calls (not sigattn_fwd_bwd_host) can be captured
 * after a first call on the device; a replay reads the lengths and tensors
 * from the captured addresses again.
 *
 * Asynchrony: every compute call enqueues its kernels on `stream` (a
 * cudaStream_t passed as void*; NULL = the legacy default stream) and
 * returns without synchronising.  The return code covers argument
 * validation and launch errors only; errors detected on the device (bounded
 * waits that ran out, clamped lengths) accumulate in the device status word.
 *
 * Precision: SIGATTN_BF16 inputs/outputs run on the tcgen05 tensor cores
 * with fp32 accumulation in tensor memory (P and dS are rounded to bf16
 * before their second matmul).  SIGATTN_FP32 runs an fp32 CUDA-core path
 * meant for accuracy checks, not speed.
 */
#ifndef SIGATTN_H
#define SIGATTN_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    SIGATTN_OK = 0,
    SIGATTN_ERR_INVALID_ARG = 1,          /* null pointer, non-positive size, ... */
    SIGATTN_ERR_UNSUPPORTED_HEADDIM = 2,  /* D not in {64, 128} */
    SIGATTN_ERR_UNSUPPORTED_DTYPE = 3,
    SIGATTN_ERR_UNSUPPORTED_DEVICE = 4,   /* bf16 path needs compute capability 10.0 */
    SIGATTN_ERR_MISALIGNED = 5,           /* a base pointer is not 16-byte aligned */
    SIGATTN_ERR_CUDA = 6,                 /* a CUDA runtime/driver call failed */
    SIGATTN_ERR_TIMEOUT = 7,              /* device: a bounded wait ran out */
    SIGATTN_ERR_SEQLEN_RANGE = 8,         /* device: a length was outside [0, L] */
    SIGATTN_ERR_TOO_LARGE = 9             /* a size exceeds a fixed limit (sigattn_fwd_noalloc) */
} sigattn_status;

typedef enum {
    SIGATTN_BF16 = 0,
    SIGATTN_FP32 = 1
} sigattn_dtype;

/* How the bf16 kernels evaluate sigma in registers.
 * SIGATTN_SIGMOID_TANH: sigma(x) = 0.5 tanh(x / 2) + 0.5 with the hardware
 *   tanh.approx.f32 (paper.rainbus.top summary, method step (3)); one MUFU
 *   operation per score.
 * SIGATTN_SIGMOID_EXP: u = e^-|x| with one hardware ex2.approx, then
 *   g = 1/(1+u) by a degree-4 minimax polynomial on the FMA pipe (relative
 *   error < 3.4e-4) and sigma = g (x >= 0) or u g (x < 0); one MUFU
 *   operation per score and relative accuracy in both tails.
 * The fp32 path always uses the exact library expf. */
typedef enum {
    SIGATTN_SIGMOID_TANH = 0,
    SIGATTN_SIGMOID_EXP = 1
} sigattn_sigmoid_mode;

/* Forward: O = [i < n_q] * sum_{j < n_k} sigma(alpha q_i . k_j + b) v_j.
 * q, k, v: [Z][L][H][D] inputs (device, read only).  o: [Z][L][H][D] output
 * (device); every element is written, padded query rows as exact zeros.
 * D in {64, 128}; any L >= 1 (partial tiles are masked); Z, H >= 1.
 * Errors: SIGATTN_ERR_INVALID_ARG, _UNSUPPORTED_HEADDIM, _UNSUPPORTED_DTYPE,
 * _UNSUPPORTED_DEVICE, _MISALIGNED, _CUDA.  On error nothing is launched. */
sigattn_status sigattn_fwd(const void *q, const void *k, const void *v, void *o,
                           const int32_t *seqlens_q, const int32_t *seqlens_k,
                           int Z, int L, int H, int D, float alpha, float bias,
                           sigattn_dtype dtype, void *stream);

/* Backward: given dout = dL/dO, writes dq, dk, dv (each [Z][L][H][D],
 * device, fully written; rows at or beyond n_q (dq) or n_k (dk, dv) are exact
 * zeros).  dout rows at or beyond n_q are ignored.  Launches a dQ kernel and
 * a dK/dV kernel on `stream`; neither uses atomics.  Same errors as
 * sigattn_fwd. */
sigattn_status sigattn_bwd(const void *q, const void *k, const void *v, const void *dout,
                           void *dq, void *dk, void *dv,
                           const int32_t *seqlens_q, const int32_t *seqlens_k,
                           int Z, int L, int H, int D, float alpha, float bias,
                           sigattn_dtype dtype, void *stream);

/* The two halves of sigattn_bwd, for callers that want to run them on
 * separate streams (they only read q, k, v, dout and write disjoint
 * outputs) or time them apart.  sigattn_bwd_dq writes dq; sigattn_bwd_dkdv
 * writes dk and dv.  Arguments, layout and errors as sigattn_bwd. */
sigattn_status sigattn_bwd_dq(const void *q, const void *k, const void *v, const void *dout,
                              void *dq, const int32_t *seqlens_q, const int32_t *seqlens_k,
                              int Z, int L, int H, int D, float alpha, float bias,
                              sigattn_dtype dtype, void *stream);
sigattn_status sigattn_bwd_dkdv(const void *q, const void *k, const void *v, const void *dout,
                                void *dk, void *dv, const int32_t *seqlens_q,
                                const int32_t *seqlens_k, int Z, int L, int H, int D,
                                float alpha, float bias, sigattn_dtype dtype, void *stream);

/* Queries and keys of different padded lengths: q, dout, o, dq are
 * [Z][Lq][H][D]; k, v, dk, dv are [Z][Lk][H][D]; n_q <= Lq and n_k <= Lk.
 * This is the shape of one rank's work when a sequence is split across GPUs
 * (context parallelism): its slice of queries against every key, and dK, dV
 * contributions of its queries to every key, which the ranks then add up.
 * Since sigma needs no row normalisation, those contributions are plain sums
 * (the operation as in sigattn_fwd / sigattn_bwd, gist.science summary,
 * section 2.A).  Lq = Lk gives exactly sigattn_fwd / sigattn_bwd.
 * Errors as sigattn_fwd / sigattn_bwd, plus SIGATTN_ERR_INVALID_ARG when
 * exactly one of Lq, Lk is zero (both zero, or Z or H zero: nothing to do). */
sigattn_status sigattn_fwd_rect(const void *q, const void *k, const void *v, void *o,
                                const int32_t *seqlens_q, const int32_t *seqlens_k, int Z, int Lq,
                                int Lk, int H, int D, float alpha, float bias, sigattn_dtype dtype,
                                void *stream);
sigattn_status sigattn_bwd_rect(const void *q, const void *k, const void *v, const void *dout,
                                void *dq, void *dk, void *dv, const int32_t *seqlens_q,
                                const int32_t *seqlens_k, int Z, int Lq, int Lk, int H, int D,
                                float alpha, float bias, sigattn_dtype dtype, void *stream);

/* Forward and backward of a batch held in HOST memory, with the transfers
 * overlapped.  The batch is cut into units of one sample and a group of heads
 * (about 16 units in all, so that the first copy in and the last copy out,
 * which nothing overlaps, are short, but never less than 8 MB per tensor of a
 * unit, so that whole samples stay whole when they are small; the first and
 * the last group are then halved, as nothing overlaps their copies).
 * Per unit, its rows of q, k, v, dout (host, [Z][L][H][D]) are copied into a
 * compact device slot on a library-owned copy stream while earlier units
 * compute; the forward and the backward of the unit run on one of two
 * library-owned compute streams (consecutive units alternate, so one unit's
 * last wave overlaps the next unit's first); its o, dq, dk, dv rows go back to
 * the host tensors on a second copy stream while later units compute.  The
 * results equal sigattn_fwd + sigattn_bwd on the same data bit for bit (every
 * (sample, head) pair is computed on its own by the same kernels).
 * host_seqlens_q / host_seqlens_k: int32[Z] in host memory, checked and read
 * on the host during the call (values outside [0, L] are
 * SIGATTN_ERR_INVALID_ARG); they may be reused as soon as it returns.
 * workspace: caller-owned device memory of at least
 * sigattn_fwd_bwd_host_workspace_bytes(Z, L, H, D, dtype) bytes, 256-byte
 * aligned (three unit slots of the eight tensors plus their lengths).
 * The transfers overlap the compute only when the host buffers are pinned
 * (page-locked); pageable buffers work but serialise the copies.  Returns when
 * all work is enqueued; it is complete once `stream` has passed it (the
 * pipeline's streams start after the work already on `stream`).  The streams
 * are created on the first call on each device and kept; calls on one device
 * must not overlap each other (they share those streams).
 * Errors as sigattn_bwd, plus SIGATTN_ERR_INVALID_ARG for a missing or small
 * workspace and SIGATTN_ERR_MISALIGNED for a misaligned one. */
sigattn_status sigattn_fwd_bwd_host(const void *q, const void *k, const void *v, const void *dout,
                                    void *o, void *dq, void *dk, void *dv,
                                    const int32_t *host_seqlens_q, const int32_t *host_seqlens_k,
                                    int Z, int L, int H, int D, float alpha, float bias,
                                    sigattn_dtype dtype, void *workspace, size_t workspace_bytes,
                                    void *stream);
size_t sigattn_fwd_bwd_host_workspace_bytes(int Z, int L, int H, int D, sigattn_dtype dtype);

/* Per-sample bias and its gradient.
 *
 * The pages set the bias to b = -log(n) (paperlayer.ai summary, section 3,
 * background on sigmoid attention; gist.science summary, section 2.A, bias
 * term) and note that this choice was never swept (paper.rainbus.top summary,
 * limitations).  These calls take one bias per sample, so b_z = -ln n_z or a
 * learned value can be used, and return the bias gradient
 *     db_z = sum over heads h and valid (i < n_q, j < n_k) of dS_zhij,
 * since x = alpha q.k + b_z.  For one bias shared by all samples, sum db over z.
 *
 * sigattn_fwd_bias: as sigattn_fwd, with `bias` a device float[Z] (not NULL
 * when Z > 0) in place of the scalar.
 *
 * sigattn_bwd_bias: as sigattn_bwd, with `bias` a device float[Z].  `dbias`,
 * if not NULL, is a device float[Z] that receives db; it is computed from the
 * fp32 dS values of the dQ pass, summed per dQ work unit and then per sample
 * in a fixed order (the result does not depend on scheduling).  That needs a
 * caller-owned device `workspace` of at least
 * sigattn_dbias_workspace_bytes(Z, L, H, dtype) bytes, 4-byte aligned, which
 * the call overwrites (its contents on entry do not matter).  With dbias NULL
 * the workspace is not used and may be NULL.
 * Errors: SIGATTN_ERR_INVALID_ARG when bias is NULL, or dbias is set and the
 * workspace is missing, too small or misaligned; otherwise as sigattn_bwd. */
sigattn_status sigattn_fwd_bias(const void *q, const void *k, const void *v, void *o,
                                const int32_t *seqlens_q, const int32_t *seqlens_k, int Z, int L,
                                int H, int D, float alpha, const float *bias, sigattn_dtype dtype,
                                void *stream);
sigattn_status sigattn_bwd_bias(const void *q, const void *k, const void *v, const void *dout,
                                void *dq, void *dk, void *dv, const int32_t *seqlens_q,
                                const int32_t *seqlens_k, int Z, int L, int H, int D, float alpha,
                                const float *bias, float *dbias, void *workspace,
                                size_t workspace_bytes, sigattn_dtype dtype, void *stream);
/* The pages' per-sample bias b_z = -ln n_z (paperlayer.ai summary, section 3;
 * gist.science summary, section 2.A), for sigattn_fwd_bias / sigattn_bwd_bias:
 * seqlens is a device int32[Z] (typically seqlens_k), bias a device float[Z]
 * that receives -logf(n_z), or 0 where n_z <= 1.  Asynchronous on `stream`.
 * Errors: SIGATTN_ERR_INVALID_ARG for Z < 0 or a NULL pointer with Z > 0,
 * SIGATTN_ERR_CUDA for a launch failure. */
sigattn_status sigattn_log_length_bias(const int32_t *seqlens, int Z, float *bias, void *stream);

/* Bytes of device workspace sigattn_bwd_bias needs to return dbias (0 for an
 * empty problem): one float per dQ work unit (bf16: per 128-row query tile
 * and head; fp32: per query row and head) of every sample. */
size_t sigattn_dbias_workspace_bytes(int Z, int L, int H, sigattn_dtype dtype);

/* Selects how later bf16 calls in this process evaluate sigma (process-wide,
 * default SIGATTN_SIGMOID_TANH, the pages' form; see sigattn_sigmoid_mode).  Returns
 * SIGATTN_ERR_INVALID_ARG for an unknown mode.
 *
 * Accuracy against the fp64 definition grows worse with L in TANH mode: with
 * b = -ln L most scores sit in sigma's left tail, where 0.5 + 0.5 tanh(x/2)
 * cancels (relative error of sigma up to 1.4% for x in [-12, -8]).  Measured
 * L1 relative error of the outputs on B200 (sampled rows, tanh mode): <= 3.4e-3
 * at L = 16384, 4.6e-3 to 4.8e-3 at L = 65536, against a bf16 bar of 5e-3;
 * EXP mode stays near 2.3e-3 at every L.  Use EXP for sequences longer than
 * about 32K, or wherever the left tail must be accurate. */
sigattn_status sigattn_set_sigmoid_mode(sigattn_sigmoid_mode mode);
sigattn_sigmoid_mode sigattn_get_sigmoid_mode(void);

/* Evaluates the kernels' own device sigma routine for `mode` on n fp32
 * values: y[i] = sigma(x[i]) and, if dy != NULL, dy[i] = sigma'(x[i]) as
 * the backward kernels form it.  x, y, dy are device arrays of n floats.
 * Used to measure the error of the in-register sigma against fp64. */
sigattn_status sigattn_sigmoid_eval(const float *x, float *y, float *dy, int64_t n,
                                    sigattn_sigmoid_mode mode, void *stream);

/* Reads and clears the current device's status word: synchronises `stream`
 * and returns SIGATTN_OK or the first device-side error recorded since the
 * last call (SIGATTN_ERR_TIMEOUT or SIGATTN_ERR_SEQLEN_RANGE). */
sigattn_status sigattn_last_device_status(void *stream);

/* Bound, in nanoseconds, on every wait inside the bf16 kernels (default
 * 4e9, at least 1e6, else SIGATTN_ERR_INVALID_ARG).  A wait that runs out
 * records SIGATTN_ERR_TIMEOUT, the kernel abandons its work, waits (with the
 * same bound) for the tile loads and MMAs it has in flight, frees its tensor
 * memory and exits. */
sigattn_status sigattn_set_wait_timeout_ns(uint64_t ns);

/* Launches a one-CTA kernel whose only job is to wait on a barrier that
 * nothing signals, bounded by timeout_ns; it must return with
 * SIGATTN_ERR_TIMEOUT recorded in the status word and leave the context
 * usable.  Exercises the failure path of the bounded waits. */
sigattn_status sigattn_selftest_wait_timeout(uint64_t timeout_ns, void *stream);

/* Forward for callers that must not allocate device memory.
 *
 * No counterpart in the paper; this is a deployment convenience.  Some
 * callers cannot call cudaMalloc at the time they run attention: code running
 * inside a framework whose caching allocator owns all device memory (a
 * cudaMalloc behind its back can fail or fragment the pool it manages), or a
 * service that reserves its memory at start-up and forbids allocation on the
 * request path (an allocation there can stall or fail under load).  Such
 * callers often also have the per-sample lengths only on the host.  This entry point
 * computes exactly what sigattn_fwd computes, with the same kernel, but takes
 * seqlens_q / seqlens_k as HOST int32[Z] arrays and never allocates: the
 * lengths and the kernel's device status word live in a fixed array in the
 * library's own device memory (a file-scope __device__ array, loaded with
 * the module, present on every GPU that loads the library until exit).
 *
 * Limits and behaviour:
 *  - Z <= SIGATTN_NOALLOC_MAX_Z (8192), else SIGATTN_ERR_TOO_LARGE and
 *    nothing is launched.  Lengths are checked on the host: any value
 *    outside [0, L] returns SIGATTN_ERR_SEQLEN_RANGE before any launch.
 *  - The host arrays are read during the call: their values reach the
 *    device as kernel arguments (up to 480 samples per small launch), so
 *    they may be reused or freed as soon as the call returns, pageable or
 *    pinned alike.
 *  - The first call on a device looks up the array's device address
 *    (cudaGetSymbolAddress); make that first call before any stream capture.
 *  - Every call shares the one array, and it keeps the last call's contents
 *    (the status word is cleared at the start of each call): calls whose
 *    work overlaps on the GPU (different streams, or devices driven from
 *    several threads at once) race on it and must be serialised by the
 *    caller.  A wait that runs out inside the kernel is recorded in that
 *    array's status word only; sigattn_last_device_status does not see it.
 * Other arguments, layout and errors as sigattn_fwd. */
#define SIGATTN_NOALLOC_MAX_Z 8192
sigattn_status sigattn_fwd_noalloc(const void *q, const void *k, const void *v, void *o,
                                   const int32_t *host_seqlens_q, const int32_t *host_seqlens_k,
                                   int Z, int L, int H, int D, float alpha, float bias,
                                   sigattn_dtype dtype, void *stream);

/* Text of the CUDA error behind the most recent SIGATTN_ERR_CUDA returned
 * by any call in this process (static string; "no error" if none). */
const char *sigattn_last_cuda_error(void);

/* Human-readable name of a status code (static string). */
const char *sigattn_status_string(sigattn_status s);

/* Order in which the bf16 kernels start the samples of a batch: blocks are
 * dispatched in grid order, and the block of grid position z works on the
 * sample of rank z by decreasing work, ties by increasing index, so the
 * samples with the most tiles start first and the short ones fill in behind
 * them.  A sample's work is its key length n_k (forward, dQ kernel) or its
 * query length n_q (dK/dV kernel), and 0 when its other length is 0.  For
 * Z > 64 the kernels keep the index order.
 *
 * This host function applies the same rule: work is host int32[Z], order
 * (host int32[Z], written) receives the sample index for each rank.  It runs
 * no device code.  Returns SIGATTN_ERR_INVALID_ARG for a NULL pointer or
 * Z < 0. */
sigattn_status sigattn_launch_order(const int32_t *work, int Z, int32_t *order);

/* Library version, major * 10000 + minor * 100 + patch. */
int sigattn_version(void);

#ifdef __cplusplus
}
#endif

#endif /* SIGATTN_H */
