// C ABI of libsigattn.so (declared in include/sigattn.h): argument checks,
// TMA tensor-map encoding and kernel launches on the caller's stream.
#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <algorithm>
#include <atomic>
#include <cstdio>
#include <mutex>
#include <unordered_map>
#include <unordered_set>

#include "../../include/sigattn.h"
#include "bwd_persist_sm100.cuh"
#include "bwd_sm100.cuh"
#include "fp32_simt.cuh"
#include "fwd_persist_sm100.cuh"
#include "fwd_sm100.cuh"

namespace {

using namespace sigattn;

constexpr int kMaxDevices = 64;

std::mutex g_mu;
int *g_status[kMaxDevices] = {};          // device status word per device (lazy, never freed)
int g_cc_major[kMaxDevices] = {};         // 0 = not queried yet
int g_sm_count[kMaxDevices] = {};         // multiprocessors per device (persistent grids)
std::atomic<int> g_sigmoid_mode{kSigmoidTanh};
std::atomic<uint64_t> g_timeout_ns{4000000000ull};
constexpr uint64_t kMinWaitTimeoutNs = 1000000ull;   // 1 ms
PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;
std::atomic<int> g_last_cuda_error{0};

// Records the failing call's error (and clears the runtime's last error).
sigattn_status cuda_fail(cudaError_t e = cudaSuccess) {
    cudaError_t last = cudaGetLastError();
    g_last_cuda_error.store(static_cast<int>(e != cudaSuccess ? e : last));
    return SIGATTN_ERR_CUDA;
}

// b_z = -ln n_z for each sample; 0 for n_z <= 1 (a sample with no key has
// nothing to weigh, and one key gives ln 1 = 0).
__global__ void log_length_bias_kernel(const int32_t *n, int Z, float *bias) {
    const int z = blockIdx.x * blockDim.x + threadIdx.x;
    if (z < Z) bias[z] = n[z] > 1 ? -logf(static_cast<float>(n[z])) : 0.0f;
}

// Writes one sample's two lengths into device memory; the values travel as
// kernel arguments, so nothing is read from host memory after the call returns.
__global__ void store_lengths_kernel(int32_t *dst, int32_t nq, int32_t nk) {
    dst[0] = nq;
    dst[1] = nk;
}

// Streams and events of the host-buffer pipeline, created once per device on
// first use and kept until process exit (no per-call allocation): one stream
// for host-to-device copies, one for device-to-host copies, and two compute
// streams so that consecutive units' kernels overlap where one unit's last
// wave leaves SMs idle.
constexpr int kPipeSlots = 3;
struct HostPipe {
    cudaStream_t in = nullptr, out = nullptr, comp[2] = {};
    cudaEvent_t start = nullptr, in_done[kPipeSlots] = {}, comp_done[kPipeSlots] = {},
                freed[kPipeSlots] = {};
};

// The pipeline's unit of work: a group of heads of one sample (the last group
// of a sample may be smaller).  A batch of few samples is split by heads into
// about kPipeUnitsTarget units, so that the first copy in and the last copy
// out, which nothing overlaps, are short; but one tensor of a unit keeps at
// least kPipeMinUnitBytes, below which the kernels' launches are too small to
// fill the GPU.  The groups are made as even as the head count allows.
constexpr int kPipeUnitsTarget = 16;
constexpr size_t kPipeMinUnitBytes = size_t(8) << 20;
int pipe_heads_per_unit(int Z, int L, int H, int D, size_t elem_bytes) {
    int chunks = std::min(H, (kPipeUnitsTarget + Z - 1) / Z);
    int hpu = (H + chunks - 1) / chunks;
    const size_t per_head = static_cast<size_t>(L) * D * elem_bytes;
    const size_t min_heads = (kPipeMinUnitBytes + per_head - 1) / per_head;
    hpu = std::max(hpu, static_cast<int>(std::min<size_t>(H, min_heads)));
    chunks = (H + hpu - 1) / hpu;
    return (H + chunks - 1) / chunks;
}
HostPipe g_pipe[kMaxDevices];

sigattn_status device_state(int *dev, int *cc_major, int **status);

sigattn_status host_pipe(int dev, HostPipe **hp) {
    std::lock_guard<std::mutex> lk(g_mu);
    HostPipe &p = g_pipe[dev];
    if (p.in == nullptr) {
        const unsigned ef = cudaEventDisableTiming;
        if (cudaStreamCreateWithFlags(&p.in, cudaStreamNonBlocking) != cudaSuccess ||
            cudaStreamCreateWithFlags(&p.out, cudaStreamNonBlocking) != cudaSuccess ||
            cudaStreamCreateWithFlags(&p.comp[0], cudaStreamNonBlocking) != cudaSuccess ||
            cudaStreamCreateWithFlags(&p.comp[1], cudaStreamNonBlocking) != cudaSuccess ||
            cudaEventCreateWithFlags(&p.start, ef) != cudaSuccess)
            return cuda_fail();
        for (int i = 0; i < kPipeSlots; ++i)
            if (cudaEventCreateWithFlags(&p.in_done[i], ef) != cudaSuccess ||
                cudaEventCreateWithFlags(&p.comp_done[i], ef) != cudaSuccess ||
                cudaEventCreateWithFlags(&p.freed[i], ef) != cudaSuccess)
                return cuda_fail();
    }
    *hp = &p;
    return SIGATTN_OK;
}

sigattn_status device_state(int *dev, int *cc_major, int **status) {
    cudaError_t e = cudaGetDevice(dev);
    if (e != cudaSuccess) return cuda_fail(e);
    if (*dev < 0 || *dev >= kMaxDevices) return SIGATTN_ERR_UNSUPPORTED_DEVICE;
    // Makes the device's primary context current in the calling thread: the
    // tensor-map encoder is a driver call and needs one (a fresh thread, such
    // as PyTorch's autograd worker, may not have one yet).
    e = cudaSetDevice(*dev);
    if (e != cudaSuccess) return cuda_fail(e);
    std::lock_guard<std::mutex> lk(g_mu);
    if (g_cc_major[*dev] == 0) {
        int major = 0, minor = 0;
        if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, *dev) != cudaSuccess ||
            cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, *dev) != cudaSuccess)
            return cuda_fail();
        int sms = 0;
        if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, *dev) != cudaSuccess)
            return cuda_fail();
        g_sm_count[*dev] = sms;
        g_cc_major[*dev] = major * 10 + minor;
    }
    if (g_status[*dev] == nullptr) {
        int *s = nullptr;
        if (cudaMalloc(&s, 64) != cudaSuccess) return cuda_fail();
        if (cudaMemset(s, 0, 64) != cudaSuccess) return cuda_fail();
        g_status[*dev] = s;
    }
    *cc_major = g_cc_major[*dev];
    *status = g_status[*dev];
    return SIGATTN_OK;
}

sigattn_status get_encoder() {
    std::lock_guard<std::mutex> lk(g_mu);
    if (g_encode != nullptr) return SIGATTN_OK;
    void *fn = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess || fn == nullptr)
        return cuda_fail();
    g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
    return SIGATTN_OK;
}

// [Z][L][H][D] bf16 viewed as a 4-D tensor (D, H, L, Z), boxes of 64 x 1 x 128 x 1
// elements with 128-byte swizzle: one box is one [128 rows][64 cols] operand atom.
sigattn_status encode_bf16_map_uncached(CUtensorMap *m, const void *base, int Z, int L, int H,
                                        int D) {
    cuuint64_t dims[4] = {static_cast<cuuint64_t>(D), static_cast<cuuint64_t>(H),
                          static_cast<cuuint64_t>(L), static_cast<cuuint64_t>(Z)};
    cuuint64_t strides[3] = {static_cast<cuuint64_t>(D) * 2, static_cast<cuuint64_t>(H) * D * 2,
                             static_cast<cuuint64_t>(L) * H * D * 2};
    cuuint32_t box[4] = {64, 1, 128, 1};
    cuuint32_t estr[4] = {1, 1, 1, 1};
    CUresult r = g_encode(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void *>(base), dims,
                          strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                          CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                          CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) {
        g_last_cuda_error.store(10000 + static_cast<int>(r));
        return SIGATTN_ERR_CUDA;
    }
    return SIGATTN_OK;
}

// Encoded maps, keyed by everything that goes into one: a bf16 map is a pure
// function of (base address, Z, L, H, D), so a hit returns exactly what a new
// encoding would, and repeated calls on the same buffers skip the driver call.
// Bounded: the cache is emptied when it reaches kMaxCachedMaps entries.
struct MapKey {
    const void *base;
    int Z, L, H, D;
    bool operator==(const MapKey &o) const {
        return base == o.base && Z == o.Z && L == o.L && H == o.H && D == o.D;
    }
};
struct MapKeyHash {
    size_t operator()(const MapKey &k) const {
        size_t h = std::hash<const void *>()(k.base);
        for (int v : {k.Z, k.L, k.H, k.D}) h = h * 1000003u ^ static_cast<size_t>(v);
        return h;
    }
};
constexpr size_t kMaxCachedMaps = 1024;
std::mutex g_map_mu;
std::unordered_map<MapKey, CUtensorMap, MapKeyHash> g_maps;

sigattn_status encode_bf16_map(CUtensorMap *m, const void *base, int Z, int L, int H, int D) {
    const MapKey key{base, Z, L, H, D};
    {
        std::lock_guard<std::mutex> lk(g_map_mu);
        auto it = g_maps.find(key);
        if (it != g_maps.end()) {
            *m = it->second;
            return SIGATTN_OK;
        }
    }
    sigattn_status s = encode_bf16_map_uncached(m, base, Z, L, H, D);
    if (s != SIGATTN_OK) return s;
    std::lock_guard<std::mutex> lk(g_map_mu);
    if (g_maps.size() >= kMaxCachedMaps) g_maps.clear();
    g_maps.emplace(key, *m);
    return SIGATTN_OK;
}

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

sigattn_status check_shape(int Z, int L, int H, int D, sigattn_dtype dtype, bool *empty) {
    if (Z < 0 || L < 0 || H < 0) return SIGATTN_ERR_INVALID_ARG;
    if (D != 64 && D != 128) return SIGATTN_ERR_UNSUPPORTED_HEADDIM;
    if (dtype != SIGATTN_BF16 && dtype != SIGATTN_FP32) return SIGATTN_ERR_UNSUPPORTED_DTYPE;
    if (H > 65535 || Z > 65535) return SIGATTN_ERR_INVALID_ARG;
    *empty = (Z == 0 || L == 0 || H == 0);
    return SIGATTN_OK;
}

// check_shape for queries and keys of padded lengths Lq and Lk: both zero is an
// empty problem, exactly one zero is an error (the other side's outputs would
// have rows but no keys or queries to read).
sigattn_status check_lengths(int Z, int Lq, int Lk, int H, int D, sigattn_dtype dtype,
                             bool *empty) {
    bool eq = false, ek = false;
    sigattn_status s = check_shape(Z, Lq, H, D, dtype, &eq);
    if (s != SIGATTN_OK) return s;
    if ((s = check_shape(Z, Lk, H, D, dtype, &ek)) != SIGATTN_OK) return s;
    if (Z == 0 || H == 0 || (Lq == 0 && Lk == 0)) {
        *empty = true;
        return SIGATTN_OK;
    }
    *empty = false;
    return (Lq == 0 || Lk == 0) ? SIGATTN_ERR_INVALID_ARG : SIGATTN_OK;
}

// (kernel, device) pairs whose dynamic shared-memory limit has been raised; a
// kernel always asks for the same amount, so once per device is enough.
struct FuncDev {
    const void *f;
    int dev;
    bool operator==(const FuncDev &o) const { return f == o.f && dev == o.dev; }
};
struct FuncDevHash {
    size_t operator()(const FuncDev &k) const {
        return std::hash<const void *>()(k.f) * 31u ^ static_cast<size_t>(k.dev);
    }
};
std::mutex g_attr_mu;
std::unordered_set<FuncDev, FuncDevHash> g_attr_set;

template <typename... KArgs, typename... Args>
sigattn_status launch(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem,
                      cudaStream_t stream, Args... args) {
    if (smem > 48 * 1024) {
        int dev = 0;
        cudaError_t e = cudaGetDevice(&dev);
        if (e != cudaSuccess) return cuda_fail(e);
        const FuncDev key{reinterpret_cast<const void *>(kernel), dev};
        std::lock_guard<std::mutex> lk(g_attr_mu);
        if (g_attr_set.count(key) == 0) {
            e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                     static_cast<int>(smem));
            if (e != cudaSuccess) return cuda_fail(e);
            g_attr_set.insert(key);
        }
    }
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaError_t e = cudaLaunchKernelEx(&cfg, kernel, args...);
    if (e != cudaSuccess) return cuda_fail(e);
    return SIGATTN_OK;
}

// Head dimension 128: one CTA per pair of query tiles (fwd_sm100.cuh).  Head
// dimension 64: one CTA per SM, or per work item when there are fewer, each
// walking its share of the items (fwd_persist_sm100.cuh).  At 64 the sigma
// work dominates the short, ragged batches of the pages' workloads, where
// block start-up, blocks over padded tiles and the last wave cost more than
// the persistent loop's bookkeeping; at 128 the long sequences run faster
// as independent blocks.
template <int D, int MODE>
sigattn_status fwd_bf16(const CUtensorMap &mq, const CUtensorMap &mk, const CUtensorMap &mv,
                        const FwdParams &p, int sms, cudaStream_t st) {
    if constexpr (D == 64) {
        const int64_t items = static_cast<int64_t>(p.Z) * p.H * ((p.Lq + 255) / 256);
        dim3 grid(static_cast<unsigned>(std::max<int64_t>(1, std::min<int64_t>(sms, items))));
        return launch(fwd_persistent_kernel<D, MODE>, grid, dim3(kFwdThreads),
                      FwdPersistLayout<D>::SMEM_ALLOC, st, mq, mk, mv, p);
    } else {
        constexpr int KS = FwdStages<D>::K, VS = FwdStages<D>::V;
        dim3 grid((p.Lq + 255) / 256, p.H, p.Z);
        return launch(fwd_tiles_kernel<D, MODE, KS, VS>, grid, dim3(kFwdThreads),
                      FwdLayout<D, KS, VS>::SMEM_ALLOC, st, mq, mk, mv, p);
    }
}

enum BwdParts : int { kPartDq = 1, kPartDkdv = 2 };

// Head dimension 128: one CTA per tile (bwd_sm100.cuh).  Head dimension 64:
// one CTA per SM, or per tile when there are fewer, each walking its share of
// the tiles with work while an idle warp zero-fills the rest
// (bwd_persist_sm100.cuh): the pages' short, ragged batches at 64 leave most
// tiles in padding, and a CTA launched per padded tile held its SM for longer
// than the zeros take to write.
template <int D, int MODE>
sigattn_status bwd_bf16(const CUtensorMap &mq, const CUtensorMap &mk, const CUtensorMap &mv,
                        const CUtensorMap &mdo, const BwdParams &p, int Z, int Lq, int Lk,
                        int H, int parts, int sms, cudaStream_t st) {
    if constexpr (D == 64) {
        using Lay = BwdPersistLayout<D>;
        auto grid_of = [&](int L) {
            const int64_t tiles = static_cast<int64_t>(Z) * H * ((L + 127) / 128);
            return dim3(static_cast<unsigned>(std::max<int64_t>(1, std::min<int64_t>(sms, tiles))));
        };
        if (parts & kPartDq) {
            sigattn_status s =
                p.db_part != nullptr
                    ? launch(bwd_dq_persistent_kernel<D, MODE, true>, grid_of(Lq), dim3(BwdSigma<D>::kThreads),
                             Lay::SMEM_ALLOC, st, mq, mk, mv, mdo, p)
                    : launch(bwd_dq_persistent_kernel<D, MODE, false>, grid_of(Lq), dim3(BwdSigma<D>::kThreads),
                             Lay::SMEM_ALLOC, st, mq, mk, mv, mdo, p);
            if (s != SIGATTN_OK) return s;
        }
        if (parts & kPartDkdv)
            return launch(bwd_dkdv_persistent_kernel<D, MODE>, grid_of(Lk), dim3(BwdSigma<D>::kThreads),
                          Lay::SMEM_ALLOC, st, mq, mk, mv, mdo, p);
        return SIGATTN_OK;
    } else {
        dim3 grid((Lq + 127) / 128, H, Z);      // dQ: one CTA per query tile
        dim3 grid_kv((Lk + 127) / 128, H, Z);   // dK/dV: one CTA per key tile
        constexpr int SX = BwdStages<D>::X, SY = BwdStages<D>::Y;
        constexpr size_t smem = BwdLayout<D, SX, SY>::SMEM_ALLOC;
        if (parts & kPartDq) {
            sigattn_status s =
                p.db_part != nullptr
                    ? launch(bwd_dq_kernel<D, MODE, SX, SY, true>, grid, dim3(BwdSigma<D>::kThreads), smem, st,
                             mq, mk, mv, mdo, p)
                    : launch(bwd_dq_kernel<D, MODE, SX, SY, false>, grid, dim3(BwdSigma<D>::kThreads), smem, st,
                             mq, mk, mv, mdo, p);
            if (s != SIGATTN_OK) return s;
        }
        if (parts & kPartDkdv)
            return launch(bwd_dkdv_kernel<D, MODE, SX, SY>, grid_kv, dim3(BwdSigma<D>::kThreads), smem, st, mq,
                          mk, mv, mdo, p);
        return SIGATTN_OK;
    }
}

// Partials of db per sample: one per dQ CTA (bf16) or per query row (fp32).
int64_t dbias_partials_per_sample(int L, int H, sigattn_dtype dtype) {
    return dtype == SIGATTN_FP32 ? static_cast<int64_t>(L) * H
                                 : static_cast<int64_t>((L + 127) / 128) * H;
}

// Shared body of sigattn_bwd, sigattn_bwd_dq, sigattn_bwd_dkdv and sigattn_bwd_bias.
// bias_z (device float[Z]) replaces the scalar bias when not null; dbias (device
// float[Z]) receives the bias gradient when not null, through `work`.
sigattn_status bwd_impl(const void *q, const void *k, const void *v, const void *dout, void *dq,
                        void *dk, void *dv, const int32_t *seqlens_q, const int32_t *seqlens_k,
                        int Z, int Lq, int Lk, int H, int D, float alpha, float bias,
                        sigattn_dtype dtype, void *stream, int parts, const float *bias_z = nullptr,
                        float *dbias = nullptr, float *work = nullptr) {
    bool empty = false;
    sigattn_status s = check_lengths(Z, Lq, Lk, H, D, dtype, &empty);
    if (s != SIGATTN_OK) return s;
    if (empty) return SIGATTN_OK;
    if (!q || !k || !v || !dout || !seqlens_q || !seqlens_k) return SIGATTN_ERR_INVALID_ARG;
    if (((parts & kPartDq) && !dq) || ((parts & kPartDkdv) && (!dk || !dv)))
        return SIGATTN_ERR_INVALID_ARG;
    if (dbias && (!work || !(parts & kPartDq))) return SIGATTN_ERR_INVALID_ARG;
    float *db_part = dbias ? work : nullptr;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(dout) ||
        ((parts & kPartDq) && !aligned16(dq)) ||
        ((parts & kPartDkdv) && (!aligned16(dk) || !aligned16(dv))))
        return SIGATTN_ERR_MISALIGNED;
    int dev, cc;
    int *status;
    if ((s = device_state(&dev, &cc, &status)) != SIGATTN_OK) return s;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (dtype == SIGATTN_FP32) {
        F32Params p{static_cast<const float *>(q),    static_cast<const float *>(k),
                    static_cast<const float *>(v),    static_cast<const float *>(dout),
                    nullptr,                          static_cast<float *>(dq),
                    static_cast<float *>(dk),         static_cast<float *>(dv),
                    seqlens_q,                        seqlens_k,
                    Z, Lq, Lk, H, alpha, bias, status, bias_z, db_part};
        const int64_t rows = static_cast<int64_t>(Z) * Lq * H;
        const int64_t rows_kv = static_cast<int64_t>(Z) * Lk * H;
        dim3 grid(static_cast<unsigned>((rows + 7) / 8));
        dim3 grid_kv(static_cast<unsigned>((rows_kv + 7) / 8));
        if (parts & kPartDq) {
            s = D == 64 ? launch(f32_dq_kernel<64>, grid, dim3(256), 0, st, p)
                        : launch(f32_dq_kernel<128>, grid, dim3(256), 0, st, p);
            if (s != SIGATTN_OK) return s;
        }
        if (parts & kPartDkdv) {
            s = D == 64 ? launch(f32_dkdv_kernel<64>, grid_kv, dim3(256), 0, st, p)
                        : launch(f32_dkdv_kernel<128>, grid_kv, dim3(256), 0, st, p);
            if (s != SIGATTN_OK) return s;
        }
        if (dbias)
            return launch(dbias_reduce_kernel, dim3(Z), dim3(256), 0, st, static_cast<const float *>(db_part),
                          dbias_partials_per_sample(Lq, H, dtype), dbias);
        return SIGATTN_OK;
    }
    if (cc != 100) return SIGATTN_ERR_UNSUPPORTED_DEVICE;
    if ((s = get_encoder()) != SIGATTN_OK) return s;
    CUtensorMap mq, mk, mv, mdo;
    if ((s = encode_bf16_map(&mq, q, Z, Lq, H, D)) != SIGATTN_OK) return s;
    if ((s = encode_bf16_map(&mk, k, Z, Lk, H, D)) != SIGATTN_OK) return s;
    if ((s = encode_bf16_map(&mv, v, Z, Lk, H, D)) != SIGATTN_OK) return s;
    if ((s = encode_bf16_map(&mdo, dout, Z, Lq, H, D)) != SIGATTN_OK) return s;
    BwdParams p{static_cast<__nv_bfloat16 *>(dq), static_cast<__nv_bfloat16 *>(dk),
                static_cast<__nv_bfloat16 *>(dv), seqlens_q, seqlens_k, Lq, Lk, H, alpha, bias, status,
                g_timeout_ns.load(), bias_z, db_part, Z};
    const int mode = g_sigmoid_mode.load(), sms = g_sm_count[dev];
    if (D == 128)
        s = mode == kSigmoidTanh ? bwd_bf16<128, kSigmoidTanh>(mq, mk, mv, mdo, p, Z, Lq, Lk, H, parts, sms, st)
                                 : bwd_bf16<128, kSigmoidExp>(mq, mk, mv, mdo, p, Z, Lq, Lk, H, parts, sms, st);
    else
        s = mode == kSigmoidTanh ? bwd_bf16<64, kSigmoidTanh>(mq, mk, mv, mdo, p, Z, Lq, Lk, H, parts, sms, st)
                                 : bwd_bf16<64, kSigmoidExp>(mq, mk, mv, mdo, p, Z, Lq, Lk, H, parts, sms, st);
    if (s != SIGATTN_OK || !dbias) return s;
    return launch(dbias_reduce_kernel, dim3(Z), dim3(256), 0, st, static_cast<const float *>(db_part),
                  dbias_partials_per_sample(Lq, H, dtype), dbias);
}

// Shared body of sigattn_fwd and sigattn_fwd_bias.
sigattn_status fwd_impl(const void *q, const void *k, const void *v, void *o,
                        const int32_t *seqlens_q, const int32_t *seqlens_k, int Z, int Lq,
                        int Lk, int H, int D, float alpha, float bias, const float *bias_z,
                        sigattn_dtype dtype, void *stream) {
    bool empty = false;
    sigattn_status s = check_lengths(Z, Lq, Lk, H, D, dtype, &empty);
    if (s != SIGATTN_OK) return s;
    if (empty) return SIGATTN_OK;
    if (!q || !k || !v || !o || !seqlens_q || !seqlens_k) return SIGATTN_ERR_INVALID_ARG;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o))
        return SIGATTN_ERR_MISALIGNED;
    int dev, cc;
    int *status;
    if ((s = device_state(&dev, &cc, &status)) != SIGATTN_OK) return s;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (dtype == SIGATTN_FP32) {
        F32Params p{static_cast<const float *>(q), static_cast<const float *>(k),
                    static_cast<const float *>(v), nullptr, static_cast<float *>(o), nullptr,
                    nullptr, nullptr, seqlens_q, seqlens_k, Z, Lq, Lk, H, alpha, bias, status,
                    bias_z, nullptr};
        const int64_t rows = static_cast<int64_t>(Z) * Lq * H;
        dim3 grid(static_cast<unsigned>((rows + 7) / 8));
        return D == 64 ? launch(f32_fwd_kernel<64>, grid, dim3(256), 0, st, p)
                       : launch(f32_fwd_kernel<128>, grid, dim3(256), 0, st, p);
    }
    if (cc != 100) return SIGATTN_ERR_UNSUPPORTED_DEVICE;
    if ((s = get_encoder()) != SIGATTN_OK) return s;
    CUtensorMap mq, mk, mv;
    if ((s = encode_bf16_map(&mq, q, Z, Lq, H, D)) != SIGATTN_OK) return s;
    if ((s = encode_bf16_map(&mk, k, Z, Lk, H, D)) != SIGATTN_OK) return s;
    if ((s = encode_bf16_map(&mv, v, Z, Lk, H, D)) != SIGATTN_OK) return s;
    FwdParams p{static_cast<__nv_bfloat16 *>(o), seqlens_q, seqlens_k, Z, Lq, Lk, H, alpha, bias,
                status, g_timeout_ns.load(), bias_z};
    const int mode = g_sigmoid_mode.load(), sms = g_sm_count[dev];
    if (D == 128)
        return mode == kSigmoidTanh ? fwd_bf16<128, kSigmoidTanh>(mq, mk, mv, p, sms, st)
                                    : fwd_bf16<128, kSigmoidExp>(mq, mk, mv, p, sms, st);
    return mode == kSigmoidTanh ? fwd_bf16<64, kSigmoidTanh>(mq, mk, mv, p, sms, st)
                                : fwd_bf16<64, kSigmoidExp>(mq, mk, mv, p, sms, st);
}

}  // namespace

extern "C" {

sigattn_status sigattn_fwd(const void *q, const void *k, const void *v, void *o,
                           const int32_t *seqlens_q, const int32_t *seqlens_k, int Z, int L, int H,
                           int D, float alpha, float bias, sigattn_dtype dtype, void *stream) {
    return fwd_impl(q, k, v, o, seqlens_q, seqlens_k, Z, L, L, H, D, alpha, bias, nullptr, dtype,
                    stream);
}

sigattn_status sigattn_fwd_bias(const void *q, const void *k, const void *v, void *o,
                                const int32_t *seqlens_q, const int32_t *seqlens_k, int Z, int L,
                                int H, int D, float alpha, const float *bias, sigattn_dtype dtype,
                                void *stream) {
    if (!bias && Z > 0) return SIGATTN_ERR_INVALID_ARG;
    return fwd_impl(q, k, v, o, seqlens_q, seqlens_k, Z, L, L, H, D, alpha, 0.0f, bias, dtype,
                    stream);
}

size_t sigattn_dbias_workspace_bytes(int Z, int L, int H, sigattn_dtype dtype) {
    if (Z <= 0 || L <= 0 || H <= 0) return 0;
    return static_cast<size_t>(Z) * static_cast<size_t>(dbias_partials_per_sample(L, H, dtype)) *
           sizeof(float);
}

sigattn_status sigattn_bwd_bias(const void *q, const void *k, const void *v, const void *dout,
                                void *dq, void *dk, void *dv, const int32_t *seqlens_q,
                                const int32_t *seqlens_k, int Z, int L, int H, int D, float alpha,
                                const float *bias, float *dbias, void *workspace,
                                size_t workspace_bytes, sigattn_dtype dtype, void *stream) {
    if (!bias && Z > 0) return SIGATTN_ERR_INVALID_ARG;
    if (dbias && Z > 0 && L > 0 && H > 0) {
        if (!workspace || workspace_bytes < sigattn_dbias_workspace_bytes(Z, L, H, dtype) ||
            (reinterpret_cast<uintptr_t>(workspace) & 3u) != 0)
            return SIGATTN_ERR_INVALID_ARG;
    }
    return bwd_impl(q, k, v, dout, dq, dk, dv, seqlens_q, seqlens_k, Z, L, L, H, D, alpha, 0.0f, dtype,
                    stream, kPartDq | kPartDkdv, bias, dbias, static_cast<float *>(workspace));
}

sigattn_status sigattn_bwd(const void *q, const void *k, const void *v, const void *dout, void *dq,
                           void *dk, void *dv, const int32_t *seqlens_q, const int32_t *seqlens_k,
                           int Z, int L, int H, int D, float alpha, float bias,
                           sigattn_dtype dtype, void *stream) {
    return bwd_impl(q, k, v, dout, dq, dk, dv, seqlens_q, seqlens_k, Z, L, L, H, D, alpha, bias, dtype,
                    stream, kPartDq | kPartDkdv);
}

sigattn_status sigattn_bwd_dq(const void *q, const void *k, const void *v, const void *dout,
                              void *dq, const int32_t *seqlens_q, const int32_t *seqlens_k, int Z,
                              int L, int H, int D, float alpha, float bias, sigattn_dtype dtype,
                              void *stream) {
    return bwd_impl(q, k, v, dout, dq, nullptr, nullptr, seqlens_q, seqlens_k, Z, L, L, H, D, alpha,
                    bias, dtype, stream, kPartDq);
}

sigattn_status sigattn_bwd_dkdv(const void *q, const void *k, const void *v, const void *dout,
                                void *dk, void *dv, const int32_t *seqlens_q,
                                const int32_t *seqlens_k, int Z, int L, int H, int D, float alpha,
                                float bias, sigattn_dtype dtype, void *stream) {
    return bwd_impl(q, k, v, dout, nullptr, dk, dv, seqlens_q, seqlens_k, Z, L, L, H, D, alpha, bias,
                    dtype, stream, kPartDkdv);
}

sigattn_status sigattn_fwd_rect(const void *q, const void *k, const void *v, void *o,
                                const int32_t *seqlens_q, const int32_t *seqlens_k, int Z, int Lq,
                                int Lk, int H, int D, float alpha, float bias, sigattn_dtype dtype,
                                void *stream) {
    return fwd_impl(q, k, v, o, seqlens_q, seqlens_k, Z, Lq, Lk, H, D, alpha, bias, nullptr, dtype,
                    stream);
}

sigattn_status sigattn_bwd_rect(const void *q, const void *k, const void *v, const void *dout,
                                void *dq, void *dk, void *dv, const int32_t *seqlens_q,
                                const int32_t *seqlens_k, int Z, int Lq, int Lk, int H, int D,
                                float alpha, float bias, sigattn_dtype dtype, void *stream) {
    return bwd_impl(q, k, v, dout, dq, dk, dv, seqlens_q, seqlens_k, Z, Lq, Lk, H, D, alpha, bias,
                    dtype, stream, kPartDq | kPartDkdv);
}

size_t sigattn_fwd_bwd_host_workspace_bytes(int Z, int L, int H, int D, sigattn_dtype dtype) {
    if (Z <= 0 || L <= 0 || H <= 0 || (D != 64 && D != 128)) return 0;
    if (dtype != SIGATTN_BF16 && dtype != SIGATTN_FP32) return 0;
    const size_t es = dtype == SIGATTN_BF16 ? 2 : 4;
    const size_t per = static_cast<size_t>(L) * pipe_heads_per_unit(Z, L, H, D, es) * D * es;
    // kPipeSlots unit slots of eight tensors, then one 256-byte length record per slot
    return kPipeSlots * 8 * per + kPipeSlots * 256;
}

sigattn_status sigattn_fwd_bwd_host(const void *q, const void *k, const void *v, const void *dout,
                                    void *o, void *dq, void *dk, void *dv,
                                    const int32_t *host_seqlens_q, const int32_t *host_seqlens_k,
                                    int Z, int L, int H, int D, float alpha, float bias,
                                    sigattn_dtype dtype, void *workspace, size_t workspace_bytes,
                                    void *stream) {
    bool empty = false;
    sigattn_status s = check_shape(Z, L, H, D, dtype, &empty);
    if (s != SIGATTN_OK) return s;
    if (empty) return SIGATTN_OK;
    if (!q || !k || !v || !dout || !o || !dq || !dk || !dv || !host_seqlens_q || !host_seqlens_k)
        return SIGATTN_ERR_INVALID_ARG;
    if (!workspace || workspace_bytes < sigattn_fwd_bwd_host_workspace_bytes(Z, L, H, D, dtype))
        return SIGATTN_ERR_INVALID_ARG;
    if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) return SIGATTN_ERR_MISALIGNED;
    for (int z = 0; z < Z; ++z)
        if (host_seqlens_q[z] < 0 || host_seqlens_q[z] > L || host_seqlens_k[z] < 0 ||
            host_seqlens_k[z] > L)
            return SIGATTN_ERR_INVALID_ARG;
    int dev, cc;
    int *status;
    if ((s = device_state(&dev, &cc, &status)) != SIGATTN_OK) return s;
    HostPipe *hp;
    if ((s = host_pipe(dev, &hp)) != SIGATTN_OK) return s;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    const size_t es = dtype == SIGATTN_BF16 ? 2 : 4;
    const int hpu = pipe_heads_per_unit(Z, L, H, D, es);
    const int chunks = (H + hpu - 1) / hpu;
    const size_t slot_tensor = static_cast<size_t>(L) * hpu * D * es;   // one tensor of a slot
    const size_t host_row = static_cast<size_t>(H) * D * es;             // one row of a host tensor
    uint8_t *ws = static_cast<uint8_t *>(workspace);
    const uint8_t *hin[4] = {static_cast<const uint8_t *>(q), static_cast<const uint8_t *>(k),
                             static_cast<const uint8_t *>(v), static_cast<const uint8_t *>(dout)};
    uint8_t *hout[4] = {static_cast<uint8_t *>(o), static_cast<uint8_t *>(dq),
                        static_cast<uint8_t *>(dk), static_cast<uint8_t *>(dv)};
    // every pipeline stream starts after the caller's earlier work on `stream`
    if (cudaEventRecord(hp->start, st) != cudaSuccess) return cuda_fail();
    for (cudaStream_t x : {hp->in, hp->out, hp->comp[0], hp->comp[1]})
        if (cudaStreamWaitEvent(x, hp->start, 0) != cudaSuccess) return cuda_fail();
    // Units in order: sample-major, head groups of up to hpu heads.  Nothing
    // overlaps the first unit's copy in or the last unit's copy out, so those
    // two groups are halved (when they hold two heads or more).
    struct Unit {
        int z, h0, hc;
    };
    auto unit_at = [&](int i) -> Unit {
        // i-th unit of the plain list (before halving)
        const int z = i / chunks, h0 = (i % chunks) * hpu;
        return Unit{z, h0, std::min(hpu, H - h0)};
    };
    const int plain = Z * chunks;
    const bool split_first = plain >= 2 && unit_at(0).hc >= 2;
    const bool split_last = plain >= 2 && unit_at(plain - 1).hc >= 2;
    const int units = plain + (split_first ? 1 : 0) + (split_last ? 1 : 0);
    auto unit = [&](int u) -> Unit {
        if (split_first) {
            if (u == 0) {
                const Unit a = unit_at(0);
                return Unit{a.z, a.h0, a.hc / 2};
            }
            if (u == 1) {
                const Unit a = unit_at(0);
                return Unit{a.z, a.h0 + a.hc / 2, a.hc - a.hc / 2};
            }
            --u;
        }
        if (split_last && u >= plain - 1) {
            const Unit b = unit_at(plain - 1);
            return u == plain - 1 ? Unit{b.z, b.h0, b.hc / 2}
                                  : Unit{b.z, b.h0 + b.hc / 2, b.hc - b.hc / 2};
        }
        return unit_at(u);
    };
    for (int u = 0; u < units; ++u) {
        const Unit un = unit(u);
        const int z = un.z, h0 = un.h0, hc = un.hc;
        const int slot = u % kPipeSlots;
        cudaStream_t cs = hp->comp[u & 1];
        uint8_t *base = ws + static_cast<size_t>(slot) * 8 * slot_tensor;
        int32_t *lens = reinterpret_cast<int32_t *>(ws + kPipeSlots * 8 * slot_tensor + slot * 256);
        // rows of this unit: L rows of hc heads, host rows H heads apart
        const size_t width = static_cast<size_t>(hc) * D * es;
        const size_t host_off = (static_cast<size_t>(z) * L * H + h0) * D * es;
        // inputs: the slot is free once unit u - kPipeSlots has been read back
        if (u >= kPipeSlots && cudaStreamWaitEvent(hp->in, hp->freed[slot], 0) != cudaSuccess)
            return cuda_fail();
        if ((s = launch(store_lengths_kernel, dim3(1), dim3(1), 0, hp->in, lens,
                        static_cast<int32_t>(host_seqlens_q[z]),
                        static_cast<int32_t>(host_seqlens_k[z]))) != SIGATTN_OK)
            return s;
        for (int t = 0; t < 4; ++t)
            if (cudaMemcpy2DAsync(base + t * slot_tensor, width, hin[t] + host_off, host_row, width,
                                  static_cast<size_t>(L), cudaMemcpyHostToDevice,
                                  hp->in) != cudaSuccess)
                return cuda_fail();
        if (cudaEventRecord(hp->in_done[slot], hp->in) != cudaSuccess ||
            cudaStreamWaitEvent(cs, hp->in_done[slot], 0) != cudaSuccess)
            return cuda_fail();
        // forward and backward of the unit, as one sample of hc heads
        s = fwd_impl(base, base + slot_tensor, base + 2 * slot_tensor, base + 4 * slot_tensor, lens,
                     lens + 1, 1, L, L, hc, D, alpha, bias, nullptr, dtype, cs);
        if (s != SIGATTN_OK) return s;
        s = bwd_impl(base, base + slot_tensor, base + 2 * slot_tensor, base + 3 * slot_tensor,
                     base + 5 * slot_tensor, base + 6 * slot_tensor, base + 7 * slot_tensor, lens,
                     lens + 1, 1, L, L, hc, D, alpha, bias, dtype, cs, kPartDq | kPartDkdv);
        if (s != SIGATTN_OK) return s;
        if (cudaEventRecord(hp->comp_done[slot], cs) != cudaSuccess ||
            cudaStreamWaitEvent(hp->out, hp->comp_done[slot], 0) != cudaSuccess)
            return cuda_fail();
        // outputs back to their rows of the host tensors while later units compute
        for (int t = 0; t < 4; ++t)
            if (cudaMemcpy2DAsync(hout[t] + host_off, host_row, base + (4 + t) * slot_tensor, width,
                                  width, static_cast<size_t>(L), cudaMemcpyDeviceToHost,
                                  hp->out) != cudaSuccess)
                return cuda_fail();
        if (cudaEventRecord(hp->freed[slot], hp->out) != cudaSuccess) return cuda_fail();
    }
    // the call completes on `stream` once every output has reached the host (the
    // copy-out stream runs in unit order, so its last event covers all units)
    if (cudaStreamWaitEvent(st, hp->freed[(units - 1) % kPipeSlots], 0) != cudaSuccess)
        return cuda_fail();
    return SIGATTN_OK;
}

sigattn_status sigattn_log_length_bias(const int32_t *seqlens, int Z, float *bias, void *stream) {
    if (Z < 0 || (Z > 0 && (!seqlens || !bias))) return SIGATTN_ERR_INVALID_ARG;
    if (Z == 0) return SIGATTN_OK;
    return launch(log_length_bias_kernel, dim3((Z + 255) / 256), dim3(256), 0,
                  static_cast<cudaStream_t>(stream), seqlens, Z, bias);
}

sigattn_status sigattn_set_sigmoid_mode(sigattn_sigmoid_mode mode) {
    if (mode != SIGATTN_SIGMOID_TANH && mode != SIGATTN_SIGMOID_EXP) return SIGATTN_ERR_INVALID_ARG;
    g_sigmoid_mode.store(mode == SIGATTN_SIGMOID_TANH ? kSigmoidTanh : kSigmoidExp);
    return SIGATTN_OK;
}

sigattn_sigmoid_mode sigattn_get_sigmoid_mode(void) {
    return g_sigmoid_mode.load() == kSigmoidTanh ? SIGATTN_SIGMOID_TANH : SIGATTN_SIGMOID_EXP;
}

sigattn_status sigattn_sigmoid_eval(const float *x, float *y, float *dy, int64_t n,
                                    sigattn_sigmoid_mode mode, void *stream) {
    if (n < 0 || (n > 0 && (!x || !y))) return SIGATTN_ERR_INVALID_ARG;
    if (mode != SIGATTN_SIGMOID_TANH && mode != SIGATTN_SIGMOID_EXP) return SIGATTN_ERR_INVALID_ARG;
    if (n == 0) return SIGATTN_OK;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    dim3 grid(static_cast<unsigned>((n + 255) / 256));
    return mode == SIGATTN_SIGMOID_TANH
               ? launch(sigmoid_eval_kernel<kSigmoidTanh>, grid, dim3(256), 0, st, x, y, dy, n)
               : launch(sigmoid_eval_kernel<kSigmoidExp>, grid, dim3(256), 0, st, x, y, dy, n);
}

sigattn_status sigattn_last_device_status(void *stream) {
    int dev, cc;
    int *status;
    sigattn_status s = device_state(&dev, &cc, &status);
    if (s != SIGATTN_OK) return s;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    int host = 0;
    if (cudaMemcpyAsync(&host, status, sizeof(int), cudaMemcpyDeviceToHost, st) != cudaSuccess)
        return cuda_fail();
    if (cudaStreamSynchronize(st) != cudaSuccess) return cuda_fail();
    if (cudaMemsetAsync(status, 0, sizeof(int), st) != cudaSuccess) return cuda_fail();
    if (cudaStreamSynchronize(st) != cudaSuccess) return cuda_fail();
    return static_cast<sigattn_status>(host);
}

sigattn_status sigattn_set_wait_timeout_ns(uint64_t ns) {
    // the same bound limits the waits with which a block, after a wait ran
    // out, lets its in-flight tile loads and MMAs land before it releases its
    // shared and tensor memory: those take microseconds, so 1 ms is the floor
    if (ns < kMinWaitTimeoutNs) return SIGATTN_ERR_INVALID_ARG;
    g_timeout_ns.store(ns);
    return SIGATTN_OK;
}

sigattn_status sigattn_selftest_wait_timeout(uint64_t timeout_ns, void *stream) {
    if (timeout_ns == 0 || timeout_ns > 10000000000ull) return SIGATTN_ERR_INVALID_ARG;
    int dev, cc;
    int *status;
    sigattn_status s = device_state(&dev, &cc, &status);
    if (s != SIGATTN_OK) return s;
    return launch(wait_timeout_selftest_kernel, dim3(1), dim3(32), 0,
                  static_cast<cudaStream_t>(stream), status, timeout_ns);
}

const char *sigattn_status_string(sigattn_status s) {
    switch (s) {
        case SIGATTN_OK: return "SIGATTN_OK";
        case SIGATTN_ERR_INVALID_ARG: return "SIGATTN_ERR_INVALID_ARG";
        case SIGATTN_ERR_UNSUPPORTED_HEADDIM: return "SIGATTN_ERR_UNSUPPORTED_HEADDIM";
        case SIGATTN_ERR_UNSUPPORTED_DTYPE: return "SIGATTN_ERR_UNSUPPORTED_DTYPE";
        case SIGATTN_ERR_UNSUPPORTED_DEVICE: return "SIGATTN_ERR_UNSUPPORTED_DEVICE";
        case SIGATTN_ERR_MISALIGNED: return "SIGATTN_ERR_MISALIGNED";
        case SIGATTN_ERR_CUDA: return "SIGATTN_ERR_CUDA";
        case SIGATTN_ERR_TIMEOUT: return "SIGATTN_ERR_TIMEOUT";
        case SIGATTN_ERR_SEQLEN_RANGE: return "SIGATTN_ERR_SEQLEN_RANGE";
        case SIGATTN_ERR_TOO_LARGE: return "SIGATTN_ERR_TOO_LARGE";
    }
    return "SIGATTN_UNKNOWN_STATUS";
}

const char *sigattn_last_cuda_error(void) {
    const int e = g_last_cuda_error.load();
    if (e == 0) return "no error";
    if (e >= 10000) {
        static thread_local char buf[64];
        snprintf(buf, sizeof buf, "cuTensorMapEncodeTiled failed (CUresult %d)", e - 10000);
        return buf;
    }
    return cudaGetErrorString(static_cast<cudaError_t>(e));
}

sigattn_status sigattn_launch_order(const int32_t *work, int Z, int32_t *order) {
    if (Z < 0 || (Z > 0 && (!work || !order))) return SIGATTN_ERR_INVALID_ARG;
    for (int i = 0; i < Z; ++i) order[rank_by_work(i, work, Z)] = i;
    return SIGATTN_OK;
}

int sigattn_version(void) { return 101; }

}  // extern "C"

// ---------------------------------------------------------------------------
// Scratch-free forward (sigattn_fwd_noalloc): the lengths and the status word
// of its kernel live in this fixed device array instead of caller or library
// allocations.  Layout (int32): [0] status word, [64, 64 + Z) n_q,
// [64 + MAX_Z, 64 + MAX_Z + Z) n_k.
namespace {
constexpr int kNoallocHeader = 64;   // 256 bytes: status word and padding
static __device__ __align__(256) int32_t g_noalloc_scratch[kNoallocHeader + 2 * SIGATTN_NOALLOC_MAX_Z];

std::mutex g_noalloc_mu;
int32_t *g_noalloc_ptr[kMaxDevices] = {};   // device address of the array, per device

// Looks up (once per device, with that device current) where the array lives
// on the device; the host-side name is only a stand-in for it.
sigattn_status noalloc_scratch(int dev, int32_t **ptr) {
    std::lock_guard<std::mutex> lk(g_noalloc_mu);
    if (g_noalloc_ptr[dev] == nullptr) {
        void *p = nullptr;
        cudaError_t e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
        if (e != cudaSuccess || p == nullptr) return cuda_fail(e);
        g_noalloc_ptr[dev] = static_cast<int32_t *>(p);
    }
    *ptr = g_noalloc_ptr[dev];
    return SIGATTN_OK;
}

// The lengths reach the array as kernel arguments, in chunks that keep one
// launch's parameters under 4 KB, so nothing is read from host memory after the
// call returns, whatever kind of host memory holds them.  The chunk at z0 = 0
// also clears the status word left by the previous call.
constexpr int kLenChunk = 480;
struct LenChunk {
    int32_t nq[kLenChunk], nk[kLenChunk];
    int z0, count;
};
static_assert(sizeof(LenChunk) <= 4000, "kernel parameter size");
__global__ void store_length_chunk_kernel(int32_t *status, int32_t *nq, int32_t *nk,
                                          const LenChunk c) {
    for (int i = threadIdx.x; i < c.count; i += blockDim.x) {
        nq[c.z0 + i] = c.nq[i];
        nk[c.z0 + i] = c.nk[i];
    }
    if (c.z0 == 0 && threadIdx.x == 0) *status = 0;
}
}  // namespace

extern "C" {

sigattn_status sigattn_fwd_noalloc(const void *q, const void *k, const void *v, void *o,
                                   const int32_t *host_seqlens_q, const int32_t *host_seqlens_k,
                                   int Z, int L, int H, int D, float alpha, float bias,
                                   sigattn_dtype dtype, void *stream) {
    bool empty = false;
    sigattn_status s = check_shape(Z, L, H, D, dtype, &empty);
    if (s != SIGATTN_OK) return s;
    if (Z > SIGATTN_NOALLOC_MAX_Z) return SIGATTN_ERR_TOO_LARGE;
    if (empty) return SIGATTN_OK;
    if (!q || !k || !v || !o || !host_seqlens_q || !host_seqlens_k) return SIGATTN_ERR_INVALID_ARG;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o))
        return SIGATTN_ERR_MISALIGNED;
    for (int z = 0; z < Z; ++z)
        if (host_seqlens_q[z] < 0 || host_seqlens_q[z] > L || host_seqlens_k[z] < 0 ||
            host_seqlens_k[z] > L)
            return SIGATTN_ERR_SEQLEN_RANGE;
    // device and capability without the status-buffer allocation of device_state()
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return cuda_fail(e);
    if (dev < 0 || dev >= kMaxDevices) return SIGATTN_ERR_UNSUPPORTED_DEVICE;
    if ((e = cudaSetDevice(dev)) != cudaSuccess) return cuda_fail(e);
    int major = 0, minor = 0, sms = 0;
    if ((e = cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev)) != cudaSuccess ||
        (e = cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev)) != cudaSuccess ||
        (e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess)
        return cuda_fail(e);
    if (dtype == SIGATTN_BF16 && major * 10 + minor != 100) return SIGATTN_ERR_UNSUPPORTED_DEVICE;
    int32_t *scratch = nullptr;
    if ((s = noalloc_scratch(dev, &scratch)) != SIGATTN_OK) return s;
    int32_t *status = scratch;
    int32_t *nq = scratch + kNoallocHeader;
    int32_t *nk = scratch + kNoallocHeader + SIGATTN_NOALLOC_MAX_Z;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    // the array keeps the previous call's contents: the first chunk clears the
    // status word, and every length of this call is written before the forward
    for (int z0 = 0; z0 < Z; z0 += kLenChunk) {
        LenChunk c;
        c.z0 = z0;
        c.count = std::min(kLenChunk, Z - z0);
        for (int i = 0; i < c.count; ++i) {
            c.nq[i] = host_seqlens_q[z0 + i];
            c.nk[i] = host_seqlens_k[z0 + i];
        }
        if ((s = launch(store_length_chunk_kernel, dim3(1), dim3(128), 0, st, status, nq, nk, c)) !=
            SIGATTN_OK)
            return s;
    }
    if (dtype == SIGATTN_FP32) {
        F32Params p{static_cast<const float *>(q), static_cast<const float *>(k),
                    static_cast<const float *>(v), nullptr, static_cast<float *>(o), nullptr,
                    nullptr, nullptr, nq, nk, Z, L, L, H, alpha, bias, status};
        const int64_t rows = static_cast<int64_t>(Z) * L * H;
        dim3 grid(static_cast<unsigned>((rows + 7) / 8));
        return D == 64 ? launch(f32_fwd_kernel<64>, grid, dim3(256), 0, st, p)
                       : launch(f32_fwd_kernel<128>, grid, dim3(256), 0, st, p);
    }
    if ((s = get_encoder()) != SIGATTN_OK) return s;
    CUtensorMap mq, mk, mv;
    if ((s = encode_bf16_map(&mq, q, Z, L, H, D)) != SIGATTN_OK) return s;
    if ((s = encode_bf16_map(&mk, k, Z, L, H, D)) != SIGATTN_OK) return s;
    if ((s = encode_bf16_map(&mv, v, Z, L, H, D)) != SIGATTN_OK) return s;
    FwdParams p{static_cast<__nv_bfloat16 *>(o), nq, nk, Z, L, L, H, alpha, bias, status,
                g_timeout_ns.load(), nullptr};
    const int mode = g_sigmoid_mode.load();
    if (D == 128)
        return mode == kSigmoidTanh ? fwd_bf16<128, kSigmoidTanh>(mq, mk, mv, p, sms, st)
                                    : fwd_bf16<128, kSigmoidExp>(mq, mk, mv, p, sms, st);
    return mode == kSigmoidTanh ? fwd_bf16<64, kSigmoidTanh>(mq, mk, mv, p, sms, st)
                                : fwd_bf16<64, kSigmoidExp>(mq, mk, mv, p, sms, st);
}

#ifdef SIGATTN_TRACE
// Diagnostic build only: copies the timeline trace (see sm100.cuh) to host
// memory `dst` of `n` uint64 entries and clears it on the device.
int sigattn_trace_dump(unsigned long long *dst, int n) {
    const int total = kTraceRoles * kTraceSteps * kTraceEvents;
    if (dst == nullptr || n < total) return -1;
    if (cudaDeviceSynchronize() != cudaSuccess) return -2;
    if (cudaMemcpyFromSymbol(dst, g_sigattn_trace, sizeof(unsigned long long) * total) != cudaSuccess)
        return -3;
    static unsigned long long zeros[kTraceRoles * kTraceSteps * kTraceEvents];
    if (cudaMemcpyToSymbol(g_sigattn_trace, zeros, sizeof zeros) != cudaSuccess) return -4;
    return total;
}

// Diagnostic build only: copies the per-CTA log of the last launch (start ns,
// end ns, smid << 32 | work, unused per CTA) to host memory and clears it.
int sigattn_cta_log_dump(unsigned long long *dst, int n) {
    const int total = kCtaLogMax * 8;
    if (dst == nullptr || n < total) return -1;
    if (cudaDeviceSynchronize() != cudaSuccess) return -2;
    if (cudaMemcpyFromSymbol(dst, g_sigattn_cta_log, sizeof(unsigned long long) * total) != cudaSuccess)
        return -3;
    static unsigned long long zeros[kCtaLogMax * 8];
    if (cudaMemcpyToSymbol(g_sigattn_cta_log, zeros, sizeof zeros) != cudaSuccess) return -4;
    return total;
}
#endif

}  // extern "C"
