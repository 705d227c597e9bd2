// common.cuh -- shared device helpers of the lbq library (sm_100a only).
//
// Inline-PTX wrappers for mbarriers, TMA bulk tensor copies and the 5th
// generation tensor core (tcgen05: TMEM allocation, MMA, TMEM loads/stores),
// plus the device status word that bounded waits report into.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/lbq.h"

#if defined(__CUDA_ARCH__) && (__CUDA_ARCH__ != 1000)
#error "lbq is written for sm_100a (B200) only"
#endif

namespace lbq {

// ---------------------------------------------------------------------------
// Device status word.  Kernels OR flags in here instead of trapping; the host
// reads and clears it with lbq_device_status().
// ---------------------------------------------------------------------------
enum : uint32_t {
    kStatusTimeout = 1u << 0,   // a bounded wait gave up
    kStatusBadTable = 1u << 1,  // a codebook failed its device-side check
};

__device__ uint32_t g_status;

__device__ __forceinline__ void record_status(uint32_t flag) { atomicOr(&g_status, flag); }

// Optional pipeline trace (built only with -DLBQ_TRACE): SM clock stamps of
// the pipeline events of CTA (0, 0, 0), read back with lbq_trace_read().
#ifdef LBQ_TRACE
constexpr int kTraceKinds = 8, kTraceLen = 256;
__device__ long long g_trace[kTraceKinds][kTraceLen];
#define LBQ_TRACE_EVENT(kind, idx)                                                                   \
    do {                                                                                             \
        if (blockIdx.x == 0 && blockIdx.y == 0 && blockIdx.z == 0 && (idx) < kTraceLen && (idx) >= 0) \
            g_trace[(kind)][(idx)] = clock64();                                                      \
    } while (0)
#else
#define LBQ_TRACE_EVENT(kind, idx) \
    do {                           \
    } while (0)
#endif

// Upper bound for every spin-wait: about two seconds of device time.
constexpr uint64_t kWaitLimitNs = 2000000000ull;
constexpr uint32_t kWaitLimitIters = 1u << 30;

__device__ __forceinline__ uint64_t globaltimer_ns() {
    uint64_t t;
    asm volatile("mov.u64 %0, %globaltimer;" : "=l"(t));
    return t;
}

// ---------------------------------------------------------------------------
// Shared-memory addresses and mbarriers
// ---------------------------------------------------------------------------
__device__ __forceinline__ uint32_t smem_u32(const void* p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}

__device__ __forceinline__ void fence_mbar_init() {
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes)
                 : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity)
        : "memory");
    return ok != 0;
}

// Wait until the barrier's phase with the given parity has completed.  Gives
// up after kWaitLimitNs (or kWaitLimitIters polls), records kStatusTimeout,
// sets *abort so the other roles of the CTA stop too, and returns false.
// try_wait that may suspend the thread until the phase completes or about
// 20 us pass, so that a waiting warp does not spin on the issue slots that the
// working warps of its SM need.
__device__ __forceinline__ bool mbar_try_wait_sleep(uint64_t* bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity), "r"(20000u)
        : "memory");
    return ok != 0;
}

__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity, volatile int* abort,
                                          uint64_t limit_ns = kWaitLimitNs) {
    if (mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = globaltimer_ns();
    for (uint32_t it = 0; it < kWaitLimitIters; ++it) {
        if (mbar_try_wait_sleep(bar, parity)) return true;
        if (*abort) return false;
        if ((it & 63u) == 63u && globaltimer_ns() - t0 > limit_ns) break;
    }
    *abort = 1;
    record_status(kStatusTimeout);
    return false;
}

// Bounded wait that ignores the abort flag: used to let this CTA's own
// asynchronous copies and MMAs finish before it frees memory and exits.
__device__ __forceinline__ bool mbar_wait_drain(uint64_t* bar, uint32_t parity, uint64_t limit_ns = kWaitLimitNs) {
    if (mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = globaltimer_ns();
    for (uint32_t it = 0; it < kWaitLimitIters; ++it) {
        if (mbar_try_wait_sleep(bar, parity)) return true;
        if ((it & 63u) == 63u && globaltimer_ns() - t0 > limit_ns) break;
    }
    record_status(kStatusTimeout);
    return false;
}

// A producer's bounded wait for "nothing could be issued": call with
// progress = whether anything was issued this round; returns false (and sets
// *abort and the timeout status) once no progress was made for kWaitLimitNs
// or another warp gave up.
struct ProgressGuard {
    uint64_t t0 = 0;
    __device__ __forceinline__ bool step(bool progress, volatile int* abort) {
        if (progress) {
            t0 = 0;
            return true;
        }
        if (*abort) return false;
        const uint64_t now = globaltimer_ns();
        if (t0 == 0) {
            t0 = now;
        } else if (now - t0 > kWaitLimitNs) {
            *abort = 1;
            record_status(kStatusTimeout);
            return false;
        }
        return true;
    }
};

// Split-tile flags: a contributor publishes its partial sums (stored by all
// threads of the CTA before the barrier that precedes this call) and counts
// itself; the finishing CTA waits for the count with acquire semantics.
__device__ __forceinline__ void flag_publish(uint32_t* f) {
    asm volatile("fence.acq_rel.gpu;\n\tred.relaxed.gpu.global.add.u32 [%0], 1;" ::"l"(f) : "memory");
}

__device__ __forceinline__ uint32_t flag_load_acquire(const uint32_t* f) {
    uint32_t v;
    asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(f) : "memory");
    return v;
}

// Bounded wait for *f >= want; records kStatusTimeout and returns false when
// it gives up.
__device__ __forceinline__ bool flag_wait_geq(const uint32_t* f, uint32_t want, uint64_t limit_ns = kWaitLimitNs) {
    if (flag_load_acquire(f) >= want) return true;
    const uint64_t t0 = globaltimer_ns();
    for (uint32_t it = 0; it < kWaitLimitIters; ++it) {
        __nanosleep(64);
        if (flag_load_acquire(f) >= want) return true;
        if ((it & 63u) == 63u && globaltimer_ns() - t0 > limit_ns) break;
    }
    record_status(kStatusTimeout);
    return false;
}

// ---------------------------------------------------------------------------
// Programmatic dependent launch: a kernel launched with programmatic stream
// serialisation may start while the previous kernel on the stream is still
// running; griddep_wait() returns once that kernel has completed and its
// memory is visible.  Without the launch attribute both are no-ops.
// ---------------------------------------------------------------------------
__device__ __forceinline__ void griddep_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void griddep_launch_dependents() {
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

// ---------------------------------------------------------------------------
// TMA (bulk tensor copies global -> shared, no multicast)
// ---------------------------------------------------------------------------
__device__ __forceinline__ void tma_prefetch_desc(const CUtensorMap* map) {
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(map)) : "memory");
}

__device__ __forceinline__ void tma_load_2d(void* dst, const CUtensorMap* map, uint64_t* bar, int c0, int c1) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%3, %4}], [%2];"
        ::"r"(smem_u32(dst)), "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_u32(bar)), "r"(c0), "r"(c1)
        : "memory");
}

__device__ __forceinline__ void tma_load_3d(void* dst, const CUtensorMap* map, uint64_t* bar, int c0, int c1,
                                            int c2) {
    asm volatile(
        "cp.async.bulk.tensor.3d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%3, %4, %5}], [%2];"
        ::"r"(smem_u32(dst)), "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_u32(bar)), "r"(c0), "r"(c1), "r"(c2)
        : "memory");
}

// ---------------------------------------------------------------------------
// tcgen05: tensor memory and the 5th-generation MMA
// ---------------------------------------------------------------------------
__device__ __forceinline__ void tmem_alloc(uint32_t* dst_smem, uint32_t ncols) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;"
                 ::"r"(smem_u32(dst_smem)), "r"(ncols) : "memory");
}

__device__ __forceinline__ void tmem_relinquish() {
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}

__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}

__device__ __forceinline__ void tc_fence_before() {
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}

__device__ __forceinline__ void tc_fence_after() {
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

// D[tmem] (+)= A[tmem] * B[smem]^T, kind::f16 (bf16 inputs, fp32 accumulate).
__device__ __forceinline__ void mma_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc, uint32_t idesc,
                                       uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}"
        ::"r"(d_tmem), "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate)
        : "memory");
}

// Arrive on an mbarrier once all tcgen05 operations issued so far by this
// thread have completed.
__device__ __forceinline__ void mma_commit(uint64_t* bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];"
                 ::"r"(smem_u32(bar)) : "memory");
}

// 32 lanes x 32 bits, 32 consecutive columns per thread (one register each).
__device__ __forceinline__ void tmem_st_32x32b_x32(uint32_t taddr, const uint32_t (&r)[32]) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], "
        "{%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, %16, "
        "%17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31, %32};"
        ::"r"(taddr),
        "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]),
        "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15]),
        "r"(r[16]), "r"(r[17]), "r"(r[18]), "r"(r[19]), "r"(r[20]), "r"(r[21]), "r"(r[22]), "r"(r[23]),
        "r"(r[24]), "r"(r[25]), "r"(r[26]), "r"(r[27]), "r"(r[28]), "r"(r[29]), "r"(r[30]), "r"(r[31])
        : "memory");
}

__device__ __forceinline__ void tmem_st_wait() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

// 32 lanes x 32 bits, 16 consecutive columns per thread.
__device__ __forceinline__ void tmem_ld_32x32b_x16(uint32_t taddr, uint32_t (&r)[16]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
        "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15}, [%16];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
        : "r"(taddr)
        : "memory");
}

__device__ __forceinline__ void tmem_ld_wait() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }

// Shared-memory matrix descriptor of a K-major operand tile written by TMA
// with 128-byte swizzling: rows of 128 bytes, 8-row groups 1024 bytes apart.
// Bits: [0,14) start address >> 4, [16,30) leading byte offset >> 4 (unused
// for swizzled K-major, set to 1), [32,46) stride byte offset >> 4,
// [46,48) descriptor version (1 on sm_100), [61,64) layout (2 = 128B swizzle).
__device__ __forceinline__ uint64_t smem_desc_k_sw128(uint32_t smem_addr) {
    uint64_t d = 0;
    d |= static_cast<uint64_t>((smem_addr >> 4) & 0x3FFFu);
    d |= static_cast<uint64_t>(1u) << 16;
    d |= static_cast<uint64_t>(1024u >> 4) << 32;
    d |= static_cast<uint64_t>(1u) << 46;
    d |= static_cast<uint64_t>(2u) << 61;
    return d;
}

// Instruction descriptor for kind::f16 with bf16 A and B, fp32 accumulator,
// both operands K-major, shape M x N.
__host__ __device__ constexpr uint32_t idesc_bf16_f32(int M, int N) {
    return (1u << 4)                                 // D format: f32
           | (1u << 7)                               // A format: bf16
           | (1u << 10)                              // B format: bf16
           | (static_cast<uint32_t>(N >> 3) << 17)   // N / 8
           | (static_cast<uint32_t>(M >> 4) << 24);  // M / 16
}

// ---------------------------------------------------------------------------
// Number formats
// ---------------------------------------------------------------------------
__device__ __forceinline__ float bf16_bits_to_f32(uint32_t b) { return __uint_as_float(b << 16); }

__device__ __forceinline__ float f16_bits_to_f32(uint16_t h) {
    return __half2float(__ushort_as_half(h));
}

__device__ __forceinline__ uint16_t f32_to_f16_bits(float x) {
    return __half_as_ushort(__float2half_rn(x));
}

__device__ __forceinline__ uint32_t pack_bf16x2_rn(float lo, float hi) {
    __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t*>(&v);
}

// (a & MASK) | c in one logic op.
template <uint32_t MASK>
__device__ __forceinline__ uint32_t and_or(uint32_t a, uint32_t c) {
    uint32_t d;
    asm("lop3.b32 %0, %1, %2, %3, 0xEA;" : "=r"(d) : "r"(a), "n"(MASK), "r"(c));
    return d;
}

// Code pairs of one 32-bit word of 4-bit codes (bytes b0..b3 = codes 0..7):
// P0 = (1, 5), P1 = (0, 4), P2 = (3, 7), P3 = (2, 6), each half the bf16
// number 128 + code (mg = 0x43004300 is passed in a register).
__device__ __forceinline__ void int4_pairs(uint32_t w, uint32_t mg, uint32_t* o) {
    o[0] = and_or<0x000F000Fu>(w, mg);
    o[1] = and_or<0x000F000Fu>(w >> 4, mg);
    o[2] = and_or<0x000F000Fu>(w >> 8, mg);
    o[3] = and_or<0x000F000Fu>(w >> 12, mg);
}

// Code pairs of one 32-bit word of 2-bit codes (bytes b0..b3 = codes 0..15,
// first code in the top bits): pair t = (t, t + 8), t = 0..7.
__device__ __forceinline__ void int2_pairs(uint32_t w, uint32_t mg, uint32_t* o) {
    o[0] = and_or<0x00030003u>(w >> 6, mg);
    o[1] = and_or<0x00030003u>(w >> 4, mg);
    o[2] = and_or<0x00030003u>(w >> 2, mg);
    o[3] = and_or<0x00030003u>(w, mg);
    o[4] = and_or<0x00030003u>(w >> 14, mg);
    o[5] = and_or<0x00030003u>(w >> 12, mg);
    o[6] = and_or<0x00030003u>(w >> 10, mg);
    o[7] = and_or<0x00030003u>(w >> 8, mg);
}

}  // namespace lbq
