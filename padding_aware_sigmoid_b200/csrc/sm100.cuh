// Thin inline-PTX layer for the sm_100a kernels: mbarriers with bounded
// waits, TMA tile loads, and the tcgen05 family (TMEM allocation, MMA issue,
// commit, TMEM <-> register copies).  Only forms that run on one CTA and one
// GPU are used: no cluster multicast anywhere.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <stdint.h>

namespace sigattn {

// Bits of the device status word (also the values of sigattn_status).
constexpr int kStatusTimeout = 7;
constexpr int kStatusSeqlenRange = 8;

__device__ __forceinline__ uint32_t smem_u32(const void *p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ uint64_t globaltimer_ns() {
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

// Records the first device error; later errors do not overwrite it.
__device__ __forceinline__ void record_status(int *status, int code) {
    if (status != nullptr) atomicCAS(status, 0, code);
}

// ------------------------------------------------------------------ mbarrier

__device__ __forceinline__ void mbar_init(uint64_t *bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count)
                 : "memory");
}

// Makes barrier initialisation visible to the async proxy (TMA, tcgen05).
__device__ __forceinline__ void fence_barrier_init() {
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t *bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t *bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)),
                 "r"(bytes)
                 : "memory");
}

// One poll of the barrier; a thread whose phase has not completed may be
// suspended by the hardware for up to `kSuspendHintNs` (it wakes as soon as the
// phase completes), so waiting roles do not take issue slots from the warps
// that share their scheduler.
#ifndef SIGATTN_SUSPEND_HINT_NS
#define SIGATTN_SUSPEND_HINT_NS 20000
#endif
constexpr uint32_t kSuspendHintNs = SIGATTN_SUSPEND_HINT_NS;

__device__ __forceinline__ bool mbar_try_wait(uint64_t *bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity), "r"(kSuspendHintNs)
        : "memory");
    return ok != 0;
}

// Per-CTA failure state shared by every role of a kernel: when any wait runs
// out, `abort` is set in shared memory so that every other wait gives up at
// its next check, and the first cause is recorded in the global status word.
struct WaitCtx {
    volatile int *abort;   // shared memory flag
    int *status;           // device status word
    uint64_t timeout_ns;
};

// Waits until the phase with parity `parity` of `bar` has completed.  Returns
// false (and leaves the CTA in the aborted state) when the wait ran out or
// another role already aborted.
__device__ __forceinline__ bool mbar_wait(uint64_t *bar, uint32_t parity, const WaitCtx &w) {
    if (mbar_try_wait(bar, parity)) return true;
    uint64_t t0 = globaltimer_ns();
    for (uint32_t it = 1;; ++it) {
        if (mbar_try_wait(bar, parity)) return true;
        if ((it & 15u) == 0u) {
            if (*w.abort) return false;
            if (globaltimer_ns() - t0 > w.timeout_ns) {
                *w.abort = 1;
                record_status(w.status, kStatusTimeout);
                return false;
            }
        }
    }
}

// Waits that never consult the abort flag: used to drain in-flight async work
// before the CTA releases its shared and tensor memory.
__device__ __forceinline__ void mbar_wait_drain(uint64_t *bar, uint32_t parity, uint64_t limit_ns) {
    if (mbar_try_wait(bar, parity)) return;
    uint64_t t0 = globaltimer_ns();
    while (!mbar_try_wait(bar, parity)) {
        if (globaltimer_ns() - t0 > limit_ns) return;
    }
}

// ------------------------------------------------------------------ TMA

__device__ __forceinline__ void prefetch_tensormap(const CUtensorMap *map) {
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(map)) : "memory");
}

// 4-D tiled bulk-tensor load into this CTA's shared memory; completion is
// signalled on `bar` as transaction bytes.  Coordinates are innermost first.
__device__ __forceinline__ void tma_load_4d(const CUtensorMap *map, uint64_t *bar, void *dst,
                                            int c0, int c1, int c2, int c3) {
    asm volatile(
        "cp.async.bulk.tensor.4d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%3, %4, %5, %6}], [%2];" ::"r"(smem_u32(dst)),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_u32(bar)), "r"(c0), "r"(c1), "r"(c2),
        "r"(c3)
        : "memory");
}

// ------------------------------------------------------------------ tcgen05

// Allocates `ncols` TMEM columns (power of two >= 32); one full warp calls it.
// The TMEM base address is written to `dst` in shared memory.
__device__ __forceinline__ void tmem_alloc(uint32_t *dst, uint32_t ncols) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_u32(dst)),
                 "r"(ncols)
                 : "memory");
}
__device__ __forceinline__ void tmem_relinquish() {
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols)
                 : "memory");
}

__device__ __forceinline__ void tc_fence_before() {
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

// Shared-memory matrix descriptor for the tcgen05 MMA (SWIZZLE_128B).
//   start: shared address of the first 16-byte chunk the MMA reads;
//   lbo/sbo: leading / stride byte offsets (multiples of 16).
// Bits: [0,14) start>>4, [16,30) lbo>>4, [32,46) sbo>>4, [46,48) version 1,
// [49,52) base offset 0, [61,64) layout 2 = 128-byte swizzle.
__device__ __forceinline__ uint64_t smem_desc_sw128(uint32_t start, uint32_t lbo, uint32_t sbo) {
    uint64_t d = 0;
    d |= static_cast<uint64_t>((start >> 4) & 0x3FFFu);
    d |= static_cast<uint64_t>((lbo >> 4) & 0x3FFFu) << 16;
    d |= static_cast<uint64_t>((sbo >> 4) & 0x3FFFu) << 32;
    d |= static_cast<uint64_t>(1u) << 46;
    d |= static_cast<uint64_t>(2u) << 61;
    return d;
}

// Instruction descriptor for kind::f16 with bf16 A/B and fp32 accumulation.
//   [4,6) D format (1 = f32), [7,10) A format (1 = bf16), [10,13) B format,
//   bit 15 A major (0 = K), bit 16 B major (1 = MN), [17,23) N>>3, [24,29) M>>4.
__host__ __device__ constexpr uint32_t idesc_bf16_f32(int M, int N, bool a_mn_major,
                                                      bool b_mn_major) {
    return (1u << 4) | (1u << 7) | (1u << 10) | ((a_mn_major ? 1u : 0u) << 15) |
           ((b_mn_major ? 1u : 0u) << 16) | ((static_cast<uint32_t>(N) >> 3) << 17) |
           ((static_cast<uint32_t>(M) >> 4) << 24);
}

// D[tmem] (+)= A[smem] * B[smem]
__device__ __forceinline__ void mma_ss(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                       uint32_t idesc, uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
        "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
        : "memory");
}

// D[tmem] (+)= A[tmem] * B[smem]
__device__ __forceinline__ void mma_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc,
                                       uint32_t idesc, uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
        "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate)
        : "memory");
}

// The same two MMA forms with each 64-bit shared-memory descriptor given as
// its low and high 32-bit halves (see smem_desc_sw128): issuing loops keep one
// base low word per operand and add a constant per K step, instead of
// rebuilding the descriptor for every instruction.
__device__ __forceinline__ void mma_ss_lh(uint32_t d_tmem, uint32_t a_lo, uint32_t b_lo, uint32_t hi,
                                          uint32_t idesc, uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t.reg .b64 da, db;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "mov.b64 da, {%1, %3};\n\t"
        "mov.b64 db, {%2, %3};\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], da, db, %5, p;\n\t}" ::"r"(d_tmem),
        "r"(a_lo), "r"(b_lo), "r"(hi), "r"(accumulate), "r"(idesc)
        : "memory");
}
__device__ __forceinline__ void mma_ts_lh(uint32_t d_tmem, uint32_t a_tmem, uint32_t b_lo, uint32_t hi,
                                          uint32_t idesc, uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t.reg .b64 db;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "mov.b64 db, {%2, %3};\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], db, %5, p;\n\t}" ::"r"(d_tmem),
        "r"(a_tmem), "r"(b_lo), "r"(hi), "r"(accumulate), "r"(idesc)
        : "memory");
}
// Halves of smem_desc_sw128(start, lbo, sbo): the low word holds start >> 4 in
// bits [0,14) (shared addresses stay below 2^18, so adding the >> 4 offset of
// a later K step never carries out of the field) and lbo >> 4 in [16,30).
__device__ __forceinline__ uint32_t desc_lo(uint32_t start, uint32_t lbo) {
    return ((start >> 4) & 0x3FFFu) | (((lbo >> 4) & 0x3FFFu) << 16);
}
__host__ __device__ constexpr uint32_t desc_hi(uint32_t sbo) {
    return ((sbo >> 4) & 0x3FFFu) | (1u << 14) | (2u << 29);
}

// Warp-converged forms: the whole warp executes them and elect.sync picks the
// one lane that issues, so the issuing warp never runs a divergent branch.
__device__ __forceinline__ void mma_ss_w(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                         uint32_t idesc, uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p, e;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "elect.sync _|e, 0xffffffff;\n\t"
        "@e tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
        "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
        : "memory");
}
__device__ __forceinline__ void mma_ts_w(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc,
                                         uint32_t idesc, uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p, e;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "elect.sync _|e, 0xffffffff;\n\t"
        "@e tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
        "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate)
        : "memory");
}
// mma_ss_lh / mma_ts_lh in the warp-converged form.
__device__ __forceinline__ void mma_ss_lhw(uint32_t d_tmem, uint32_t a_lo, uint32_t b_lo, uint32_t hi,
                                           uint32_t idesc, uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p, e;\n\t.reg .b64 da, db;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "mov.b64 da, {%1, %3};\n\t"
        "mov.b64 db, {%2, %3};\n\t"
        "elect.sync _|e, 0xffffffff;\n\t"
        "@e tcgen05.mma.cta_group::1.kind::f16 [%0], da, db, %5, p;\n\t}" ::"r"(d_tmem),
        "r"(a_lo), "r"(b_lo), "r"(hi), "r"(accumulate), "r"(idesc)
        : "memory");
}
__device__ __forceinline__ void mma_ts_lhw(uint32_t d_tmem, uint32_t a_tmem, uint32_t b_lo, uint32_t hi,
                                           uint32_t idesc, uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p, e;\n\t.reg .b64 db;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "mov.b64 db, {%2, %3};\n\t"
        "elect.sync _|e, 0xffffffff;\n\t"
        "@e tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], db, %5, p;\n\t}" ::"r"(d_tmem),
        "r"(a_tmem), "r"(b_lo), "r"(hi), "r"(accumulate), "r"(idesc)
        : "memory");
}
__device__ __forceinline__ void mma_commit_w(uint64_t *bar) {
    asm volatile(
        "{\n\t.reg .pred e;\n\t"
        "elect.sync _|e, 0xffffffff;\n\t"
        "@e tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];\n\t}" ::"r"(
            smem_u32(bar))
        : "memory");
}

// Arrives once on `bar` when every MMA this thread issued so far has completed.
__device__ __forceinline__ void mma_commit(uint64_t *bar) {
    asm volatile(
        "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
            smem_u32(bar))
        : "memory");
}

// 32 lanes x 32 consecutive 32-bit columns: thread t of the warp receives
// columns [col, col+32) of lane (lane_base + t).  The wait is inside the same
// asm statement, so no use of the registers can be scheduled before the data
// has arrived.
#define SIGATTN_R32(a) "=r"(a[0]), "=r"(a[1]), "=r"(a[2]), "=r"(a[3]), "=r"(a[4]), "=r"(a[5]), \
    "=r"(a[6]), "=r"(a[7]), "=r"(a[8]), "=r"(a[9]), "=r"(a[10]), "=r"(a[11]), "=r"(a[12]),      \
    "=r"(a[13]), "=r"(a[14]), "=r"(a[15]), "=r"(a[16]), "=r"(a[17]), "=r"(a[18]), "=r"(a[19]),  \
    "=r"(a[20]), "=r"(a[21]), "=r"(a[22]), "=r"(a[23]), "=r"(a[24]), "=r"(a[25]), "=r"(a[26]),  \
    "=r"(a[27]), "=r"(a[28]), "=r"(a[29]), "=r"(a[30]), "=r"(a[31])

__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&r)[32]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];\n\t"
        "tcgen05.wait::ld.sync.aligned;"
        : SIGATTN_R32(r)
        : "r"(taddr)
        : "memory");
}

// 32 lanes x 16 consecutive 32-bit columns, with the wait.
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, uint32_t (&r)[16]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];\n\t"
        "tcgen05.wait::ld.sync.aligned;"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
          "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
          "=r"(r[14]), "=r"(r[15])
        : "r"(taddr)
        : "memory");
}

// Two such loads (e.g. S and dP of the same rows) and one wait.
__device__ __forceinline__ void tmem_ld32x2(uint32_t ta, uint32_t (&a)[32], uint32_t tb,
                                            uint32_t (&b)[32]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%64];\n\t"
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%32,%33,%34,%35,%36,%37,%38,%39,%40,%41,%42,%43,%44,%45,%46,%47,%48,%49,%50,%51,%52,%53,%54,%55,%56,%57,%58,%59,%60,%61,%62,%63}, [%65];\n\t"
        "tcgen05.wait::ld.sync.aligned;"
        : SIGATTN_R32(a), SIGATTN_R32(b)
        : "r"(ta), "r"(tb)
        : "memory");
}

// 32 lanes x 64 consecutive columns in two x32 loads and one wait.
__device__ __forceinline__ void tmem_ld64(uint32_t taddr, uint32_t (&r)[64]) {
    uint32_t(&a)[32] = *reinterpret_cast<uint32_t(*)[32]>(&r[0]);
    uint32_t(&b)[32] = *reinterpret_cast<uint32_t(*)[32]>(&r[32]);
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%64];\n\t"
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%32,%33,%34,%35,%36,%37,%38,%39,%40,%41,%42,%43,%44,%45,%46,%47,%48,%49,%50,%51,%52,%53,%54,%55,%56,%57,%58,%59,%60,%61,%62,%63}, [%65];\n\t"
        "tcgen05.wait::ld.sync.aligned;"
        : SIGATTN_R32(a), SIGATTN_R32(b)
        : "r"(taddr), "r"(taddr + 32)
        : "memory");
}

// 32 lanes x 128 consecutive columns in four x32 loads and one wait.
__device__ __forceinline__ void tmem_ld128(uint32_t taddr, uint32_t (&r)[128]) {
    uint32_t(&a)[32] = *reinterpret_cast<uint32_t(*)[32]>(&r[0]);
    uint32_t(&b)[32] = *reinterpret_cast<uint32_t(*)[32]>(&r[32]);
    uint32_t(&c)[32] = *reinterpret_cast<uint32_t(*)[32]>(&r[64]);
    uint32_t(&d)[32] = *reinterpret_cast<uint32_t(*)[32]>(&r[96]);
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%128];\n\t"
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%32,%33,%34,%35,%36,%37,%38,%39,%40,%41,%42,%43,%44,%45,%46,%47,%48,%49,%50,%51,%52,%53,%54,%55,%56,%57,%58,%59,%60,%61,%62,%63}, [%129];\n\t"
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%64,%65,%66,%67,%68,%69,%70,%71,%72,%73,%74,%75,%76,%77,%78,%79,%80,%81,%82,%83,%84,%85,%86,%87,%88,%89,%90,%91,%92,%93,%94,%95}, [%130];\n\t"
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%96,%97,%98,%99,%100,%101,%102,%103,%104,%105,%106,%107,%108,%109,%110,%111,%112,%113,%114,%115,%116,%117,%118,%119,%120,%121,%122,%123,%124,%125,%126,%127}, [%131];\n\t"
        "tcgen05.wait::ld.sync.aligned;"
        : SIGATTN_R32(a), SIGATTN_R32(b), SIGATTN_R32(c), SIGATTN_R32(d)
        : "r"(taddr), "r"(taddr + 32), "r"(taddr + 64), "r"(taddr + 96)
        : "memory");
}

// Two 64-column loads from different bases (e.g. S and dP) and one wait.
__device__ __forceinline__ void tmem_ld64x2(uint32_t ta, uint32_t (&ra)[64], uint32_t tb,
                                            uint32_t (&rb)[64]) {
    uint32_t(&a0)[32] = *reinterpret_cast<uint32_t(*)[32]>(&ra[0]);
    uint32_t(&a1)[32] = *reinterpret_cast<uint32_t(*)[32]>(&ra[32]);
    uint32_t(&b0)[32] = *reinterpret_cast<uint32_t(*)[32]>(&rb[0]);
    uint32_t(&b1)[32] = *reinterpret_cast<uint32_t(*)[32]>(&rb[32]);
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%128];\n\t"
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%32,%33,%34,%35,%36,%37,%38,%39,%40,%41,%42,%43,%44,%45,%46,%47,%48,%49,%50,%51,%52,%53,%54,%55,%56,%57,%58,%59,%60,%61,%62,%63}, [%129];\n\t"
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%64,%65,%66,%67,%68,%69,%70,%71,%72,%73,%74,%75,%76,%77,%78,%79,%80,%81,%82,%83,%84,%85,%86,%87,%88,%89,%90,%91,%92,%93,%94,%95}, [%130];\n\t"
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%96,%97,%98,%99,%100,%101,%102,%103,%104,%105,%106,%107,%108,%109,%110,%111,%112,%113,%114,%115,%116,%117,%118,%119,%120,%121,%122,%123,%124,%125,%126,%127}, [%131];\n\t"
        "tcgen05.wait::ld.sync.aligned;"
        : SIGATTN_R32(a0), SIGATTN_R32(a1), SIGATTN_R32(b0), SIGATTN_R32(b1)
        : "r"(ta), "r"(ta + 32), "r"(tb), "r"(tb + 32)
        : "memory");
}

// 32 lanes x 16 consecutive 32-bit columns, registers -> TMEM.
__device__ __forceinline__ void tmem_st16(uint32_t taddr, const uint32_t (&r)[16]) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], "
        "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};" ::"r"(taddr),
        "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]),
        "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]),
        "r"(r[15])
        : "memory");
}

// 32 lanes x 32 consecutive 32-bit columns, registers -> TMEM.
__device__ __forceinline__ void tmem_st32(uint32_t taddr, const uint32_t *r) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], "
        "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,"
        "%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};" ::"r"(taddr),
        "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]),
        "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]),
        "r"(r[15]), "r"(r[16]), "r"(r[17]), "r"(r[18]), "r"(r[19]), "r"(r[20]), "r"(r[21]),
        "r"(r[22]), "r"(r[23]), "r"(r[24]), "r"(r[25]), "r"(r[26]), "r"(r[27]), "r"(r[28]),
        "r"(r[29]), "r"(r[30]), "r"(r[31])
        : "memory");
}

__device__ __forceinline__ void tmem_wait_st() {
    asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
    __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t *>(&v);
}

// Bias of sample z: one value per sample when the caller passes an array
// (e.g. b_z = -ln n_z), otherwise the scalar.
__device__ __forceinline__ float bias_of(const float *bias_z, float bias, int z) {
    return bias_z != nullptr ? bias_z[z] : bias;
}

// Named barrier 1 over the `count` threads of the sigma warpgroups.
__device__ __forceinline__ void sigma_warps_sync(int count) {
    asm volatile("bar.sync 1, %0;" ::"r"(count) : "memory");
}

// ------------------------------------------------------------------ launch order

// Sample j (work wj) comes before sample i (work wi) when samples are ordered by
// decreasing work, ties by increasing index: a stable descending sort.
__host__ __device__ inline bool ranks_before(int wj, int j, int wi, int i) {
    return wj > wi || (wj == wi && j < i);
}

// Position of sample i in that order; over Z samples the positions are a
// permutation of 0..Z-1.
__host__ __device__ inline int rank_by_work(int i, const int *work, int Z) {
    int r = 0;
    for (int j = 0; j < Z; ++j) r += ranks_before(work[j], j, work[i], i);
    return r;
}

// Blocks are dispatched in increasing linear index (x fastest, z slowest), so a
// grid whose z coordinate runs over the samples starts them in index order, and
// the blocks of a long sample that comes last run on alone at the end.  Here the
// block at z = r works on the sample of rank r by decreasing work: the key
// length n_k (keys_are_work) or the query length n_q, and 0 when the sample's
// other length is 0.  The longest samples start first and the short ones fill
// in behind them.
//
// One warp finds the sample with shuffles (lane l holds samples l and l + 32)
// and writes it to `slot` in shared memory; the other warps read it there after
// the block barrier that ends their setup, so the lookup overlaps the setup and
// adds no barrier.  All 32 lanes of that warp call it.  The slot holds the
// sample and its two lengths as stored (range checks stay with the reader).
// Above kMaxRankedSamples samples the index order is kept.
struct BlockSample {
    int z, nq, nk, unused;
};
constexpr int kMaxRankedSamples = 64;
__device__ __forceinline__ void publish_block_sample(const int32_t *seqlens_q,
                                                     const int32_t *seqlens_k, bool keys_are_work,
                                                     BlockSample *slot) {
    const int Z = static_cast<int>(gridDim.z), r = static_cast<int>(blockIdx.z);
    const int lane = static_cast<int>(threadIdx.x & 31);
    if (Z > kMaxRankedSamples) {
        if (lane == 0) *slot = BlockSample{r, seqlens_q[r], seqlens_k[r], 0};
        return;
    }
    int nq[2], nk[2], w[2], rank[2] = {0, 0};
#pragma unroll
    for (int c = 0; c < 2; ++c) {
        const int i = lane + 32 * c;
        nq[c] = i < Z ? seqlens_q[i] : 0;
        nk[c] = i < Z ? seqlens_k[i] : 0;
        w[c] = keys_are_work ? (nq[c] > 0 ? nk[c] : 0) : (nk[c] > 0 ? nq[c] : 0);
    }
    // only the Z live samples are compared (a short loop for small batches)
    for (int j = 0; j < Z; ++j) {
        const int wj = __shfl_sync(0xffffffffu, j < 32 ? w[0] : w[1], j & 31);
#pragma unroll
        for (int c = 0; c < 2; ++c) rank[c] += ranks_before(wj, j, w[c], lane + 32 * c);
    }
#pragma unroll
    for (int c = 0; c < 2; ++c)
        if (lane + 32 * c < Z && rank[c] == r) *slot = BlockSample{lane + 32 * c, nq[c], nk[c], 0};
}

__device__ __forceinline__ int lane_id() { return threadIdx.x & 31; }

// Start of the dynamic shared memory rounded up to 1 KiB (the alignment of
// the 128-byte-swizzled operand tiles); every layout reserves 1 KiB of slack.
__device__ __forceinline__ uint8_t *align_1k(uint8_t *p) {
    uint32_t a = smem_u32(p);
    return p + ((1024u - (a & 1023u)) & 1023u);
}
__device__ __forceinline__ int warp_id() { return threadIdx.x >> 5; }

}  // namespace sigattn

// ---------------------------------------------------------------- timeline trace
// Built only with -DSIGATTN_TRACE (libsigattn_trace.so, a diagnostic build): one
// CTA per launch (the one at blockIdx (gridDim.x / 2, 0, 0)) records clock64()
// at each role's waits and hand-offs into g_sigattn_trace[role][step][event],
// read back with sigattn_trace_dump().  The default build compiles it away.
namespace sigattn {
constexpr int kTraceRoles = 8, kTraceSteps = 256, kTraceEvents = 8;
#ifdef SIGATTN_TRACE
__device__ unsigned long long g_sigattn_trace[kTraceRoles * kTraceSteps * kTraceEvents];
__device__ __forceinline__ bool trace_cta() {
    return blockIdx.x == gridDim.x / 2 && blockIdx.y == 0 && blockIdx.z == 0;
}
__device__ __forceinline__ void trace(int role, int step, int ev) {
    if (trace_cta() && (threadIdx.x & 31) == 0 && step < kTraceSteps)
        g_sigattn_trace[(role * kTraceSteps + step) * kTraceEvents + ev] = clock64();
}
// per-CTA record of one launch: start and end (%globaltimer), SM id, work
constexpr int kCtaLogMax = 1 << 16;
__device__ unsigned long long g_sigattn_cta_log[kCtaLogMax * 8];
__device__ __forceinline__ uint32_t smid() {
    uint32_t r;
    asm volatile("mov.u32 %0, %%smid;" : "=r"(r));
    return r;
}
__device__ __forceinline__ void cta_log(int slot, unsigned long long v) {
    const unsigned long long id = blockIdx.x + static_cast<unsigned long long>(gridDim.x) *
                                  (blockIdx.y + static_cast<unsigned long long>(gridDim.y) * blockIdx.z);
    if (threadIdx.x == 0 && id < kCtaLogMax) g_sigattn_cta_log[id * 8 + slot] = v;
}
__device__ __forceinline__ void cta_log_any(int slot, unsigned long long v) {
    const unsigned long long id = blockIdx.x + static_cast<unsigned long long>(gridDim.x) *
                                  (blockIdx.y + static_cast<unsigned long long>(gridDim.y) * blockIdx.z);
    if (id < kCtaLogMax) g_sigattn_cta_log[id * 8 + slot] = v;
}
#else
__device__ __forceinline__ void trace(int, int, int) {}
__device__ __forceinline__ void cta_log(int, unsigned long long) {}
__device__ __forceinline__ void cta_log_any(int, unsigned long long) {}
__device__ __forceinline__ uint32_t smid() { return 0; }
#endif
}  // namespace sigattn
