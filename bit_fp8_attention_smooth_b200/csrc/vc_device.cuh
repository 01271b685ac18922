// vc_device.cuh -- sm_100a device helpers: mbarriers with bounded waits, TMA
// and bulk copies, tcgen05 (TMEM allocation, MMA, loads/stores), the E4M3
// encoder and the ExpCast byte map.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <stdint.h>

#include "vc_attention.h"

namespace vc {

// ---------------------------------------------------------------- status
// Word 0 of the workspace.  The first failing wait records its code; later
// ones leave it.
struct DevCtl {
    int* status;       // device status word
    int64_t limit_ns;  // bound on one wait
};

__device__ __forceinline__ uint64_t globaltimer() {
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

__device__ __forceinline__ void record_error(const DevCtl& ctl, int code) {
    atomicCAS(ctl.status, 0, code);
}

// True, for every thread of the CTA, when an earlier kernel on the same
// workspace recorded a device error: its outputs are undefined, so a kernel
// that would index memory with them does nothing instead.  Call at the top of
// the kernel, by all threads.
__device__ __forceinline__ bool ctl_failed(const int* status) {
    return __syncthreads_or(threadIdx.x == 0 && *reinterpret_cast<const volatile int*>(status) != 0) != 0;
}

// ---------------------------------------------------------------- smem
__device__ __forceinline__ uint32_t smem_u32(const void* p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// ---------------------------------------------------------------- mbarrier
__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}

__device__ __forceinline__ void fence_mbar_init() {
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}

__device__ __forceinline__ void mbar_expect_tx_arrive(uint32_t bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes) : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(bar), "r"(parity)
        : "memory");
    return ok != 0;
}

// Non-blocking test of the phase of parity `parity`.
__device__ __forceinline__ bool mbar_test_wait(uint32_t bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(bar), "r"(parity)
        : "memory");
    return ok != 0;
}

// Bound on draining a CTA's own in-flight copies and MMAs after an abort; it
// does not depend on the (possibly tiny) wait limit.
constexpr int64_t kDrainNs = 2000000000LL;

// Wait limits below this leave no time to wait at all: only a phase already
// complete at the first (non-blocking) poll passes.  A blocking try_wait can
// hold a thread for longer than such a limit, and the global timer ticks more
// coarsely, so a shorter limit could not be told apart from none.
constexpr int64_t kMinWaitNs = 1000;

// Waits for the phase of parity `parity` to complete.  Gives up when the CTA
// abort flag is raised by another warp, or after ctl.limit_ns, in which case
// it raises the flag and records VC_ERR_DEVICE_TIMEOUT.  Returns false when it
// gave up.
__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity, const DevCtl& ctl,
                                          volatile int* abort_flag) {
    if (mbar_test_wait(bar, parity)) return true;
    if (ctl.limit_ns < kMinWaitNs) {
        *abort_flag = 1;
        record_error(ctl, VC_ERR_DEVICE_TIMEOUT);
        return false;
    }
    const uint64_t t0 = globaltimer();
    while (true) {
        if (mbar_try_wait(bar, parity)) return true;
        if (*abort_flag) return false;
        if ((int64_t)(globaltimer() - t0) > ctl.limit_ns) {
            *abort_flag = 1;
            record_error(ctl, VC_ERR_DEVICE_TIMEOUT);
            return false;
        }
    }
}

__device__ __forceinline__ float exp2_neg_int(int k) {
    // 2^-k for an integer k >= 0, exactly (0 below the normal range).
    return k < 127 ? __uint_as_float((uint32_t)(127 - k) << 23) : 0.0f;
}

// Wait with a warp-uniform verdict: the warp continues only if every lane saw
// the phase complete.
__device__ __forceinline__ bool warp_wait(uint32_t bar, uint32_t parity, const DevCtl& ctl, volatile int* abort_flag) {
    const bool ok = mbar_wait(bar, parity, ctl, abort_flag);
    return __all_sync(0xffffffffu, ok);
}

// mbar_wait for warps off the critical path: between polls the thread sleeps
// about `sleep_ns`, so a long wait takes almost no issue slots from the warps
// of its sub-partition that have work.  Same limits and verdicts as mbar_wait.
__device__ __forceinline__ bool mbar_wait_idle(uint32_t bar, uint32_t parity, const DevCtl& ctl,
                                               volatile int* abort_flag, uint32_t sleep_ns) {
    if (mbar_test_wait(bar, parity)) return true;
    if (ctl.limit_ns < kMinWaitNs) {
        *abort_flag = 1;
        record_error(ctl, VC_ERR_DEVICE_TIMEOUT);
        return false;
    }
    const uint64_t t0 = globaltimer();
    while (true) {
        __nanosleep(sleep_ns);
        if (mbar_test_wait(bar, parity)) return true;
        if (*abort_flag) return false;
        if ((int64_t)(globaltimer() - t0) > ctl.limit_ns) {
            *abort_flag = 1;
            record_error(ctl, VC_ERR_DEVICE_TIMEOUT);
            return false;
        }
    }
}

__device__ __forceinline__ bool warp_wait_idle(uint32_t bar, uint32_t parity, const DevCtl& ctl,
                                               volatile int* abort_flag, uint32_t sleep_ns) {
    const bool ok = mbar_wait_idle(bar, parity, ctl, abort_flag, sleep_ns);
    return __all_sync(0xffffffffu, ok);
}

// Bounded wait that ignores the abort flag (used to drain in-flight copies and
// MMAs before the CTA exits).
__device__ __forceinline__ void drain_wait(uint32_t bar, uint32_t parity, const DevCtl& ctl) {
    const uint64_t t0 = globaltimer();
    while (!mbar_try_wait(bar, parity)) {
        if ((int64_t)(globaltimer() - t0) > kDrainNs) {
            record_error(ctl, VC_ERR_DEVICE_TIMEOUT);
            return;
        }
    }
}

// ---------------------------------------------------------------- TMA / bulk copy
__device__ __forceinline__ void tma_load_3d(uint32_t dst, const CUtensorMap* map, uint32_t bar, int x, int y,
                                            int z) {
    asm volatile(
        "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%2, %3, %4}], [%5];" ::"r"(dst),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(z), "r"(bar)
        : "memory");
}

__device__ __forceinline__ void bulk_load(uint32_t dst, const void* src, uint32_t bytes, uint32_t bar) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(dst),
        "l"(src), "r"(bytes), "r"(bar)
        : "memory");
}

__device__ __forceinline__ void prefetch_tmap(const CUtensorMap* map) {
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(map)) : "memory");
}

// Barrier `id` (1..15) over `count` threads (a multiple of 32).
__device__ __forceinline__ void named_barrier_sync(int id, int count) {
    asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(count) : "memory");
}

__device__ __forceinline__ void named_barrier_arrive(int id, int count) {
    asm volatile("bar.arrive %0, %1;" ::"r"(id), "r"(count) : "memory");
}

// Generic-proxy shared-memory writes -> visible to the async proxy (tensor core).
__device__ __forceinline__ void fence_proxy_async_smem() {
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// ---------------------------------------------------------------- tcgen05
__device__ __forceinline__ void tmem_alloc(uint32_t dst_smem, uint32_t ncols) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(dst_smem), "r"(ncols)
                 : "memory");
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
// D[tmem] (+)= A[smem] * B[smem]^T, E4M3 x E4M3 -> fp32.
__device__ __forceinline__ void mma_f8(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                       uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f8f6f4 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
        "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
        : "memory");
}
// D[tmem] (+)= A[tmem] * B[smem]^T, E4M3 x E4M3 -> fp32; A is K-major in TMEM
// (lane = row, four E4M3 values per 32-bit column).
__device__ __forceinline__ void mma_f8_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc, uint32_t idesc,
                                          uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f8f6f4 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
        "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate)
        : "memory");
}
// Warp-wide forms: every lane of a converged warp executes them with the same
// (warp-uniform) operands, and elect.sync picks the one lane that issues.
__device__ __forceinline__ void mma_f8_ts_warp(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc, uint32_t idesc,
                                               uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred pe, pa;\n\t"
        "elect.sync _|pe, 0xffffffff;\n\t"
        "setp.ne.b32 pa, %4, 0;\n\t"
        "@pe tcgen05.mma.cta_group::1.kind::f8f6f4 [%0], [%1], %2, %3, pa;\n\t}" ::"r"(d_tmem),
        "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate)
        : "memory");
}
__device__ __forceinline__ void mma_commit_warp(uint32_t bar) {
    asm volatile(
        "{\n\t.reg .pred pe;\n\t"
        "elect.sync _|pe, 0xffffffff;\n\t"
        "@pe tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];\n\t}" ::"r"(bar)
        : "memory");
}
// Arrive on `bar` once all previously issued tcgen05 async operations of this
// thread have completed.
__device__ __forceinline__ void mma_commit(uint32_t bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar)
                 : "memory");
}
__device__ __forceinline__ void tmem_wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }
__device__ __forceinline__ void tmem_wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

// 32 consecutive fp32 columns of this thread's TMEM lane.
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, float* v) {
    uint32_t* r = reinterpret_cast<uint32_t*>(v);
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
        "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, "
        "%16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
          "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]),
          "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
        : "r"(taddr));
}
__device__ __forceinline__ void tmem_st32(uint32_t taddr, const float* v) {
    const uint32_t* r = reinterpret_cast<const uint32_t*>(v);
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], "
        "{%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, %16, "
        "%17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31, %32};" ::"r"(taddr),
        "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]),
        "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15]), "r"(r[16]), "r"(r[17]),
        "r"(r[18]), "r"(r[19]), "r"(r[20]), "r"(r[21]), "r"(r[22]), "r"(r[23]), "r"(r[24]), "r"(r[25]), "r"(r[26]),
        "r"(r[27]), "r"(r[28]), "r"(r[29]), "r"(r[30]), "r"(r[31])
        : "memory");
}
__device__ __forceinline__ void tmem_st16(uint32_t taddr, const uint32_t* r) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], "
        "{%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, %16};" ::"r"(taddr),
        "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]),
        "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15])
        : "memory");
}
__device__ __forceinline__ void tmem_st8(uint32_t taddr, const uint32_t* r) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x8.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8};" ::"r"(taddr), "r"(r[0]),
        "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7])
        : "memory");
}
__device__ __forceinline__ void tmem_st1(uint32_t taddr, float v) {
    asm volatile("tcgen05.st.sync.aligned.32x32b.x1.b32 [%0], {%1};" ::"r"(taddr), "r"(__float_as_uint(v)) : "memory");
}
__device__ __forceinline__ float tmem_ld1(uint32_t taddr) {
    uint32_t r;
    asm volatile("tcgen05.ld.sync.aligned.32x32b.x1.b32 {%0}, [%1];" : "=r"(r) : "r"(taddr));
    return __uint_as_float(r);
}

// D[tmem] (+)= A[smem] * B[smem]^T, bf16 x bf16 -> fp32.
__device__ __forceinline__ void mma_bf16(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                         uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
        "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
        : "memory");
}

// 8 consecutive fp32 columns of this thread's TMEM lane.
__device__ __forceinline__ void tmem_ld8(uint32_t taddr, float* v) {
    uint32_t* r = reinterpret_cast<uint32_t*>(v);
    asm volatile("tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0, %1, %2, %3, %4, %5, %6, %7}, [%8];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7])
                 : "r"(taddr));
}
// 16 consecutive fp32 columns of this thread's TMEM lane.
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, float* v) {
    uint32_t* r = reinterpret_cast<uint32_t*>(v);
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
        "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15}, [%16];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
        : "r"(taddr));
}

// Instruction descriptor of kind::f16: D fp32, A and B bf16, both K-major,
// M = 128, N = n (multiple of 16, 16..256).
__host__ __device__ constexpr uint32_t idesc_bf16_f32(int n) {
    return (1u << 4)                          // D format: fp32
           | (1u << 7) | (1u << 10)           // A, B format: bf16
           | (uint32_t(n >> 3) << 17)         // N / 8
           | (uint32_t(128 >> 4) << 24);      // M / 16
}

// Instruction descriptor of kind::f8f6f4: D fp32, A and B E4M3, both K-major,
// M = 128, N = n (multiple of 16, 16..256).
__host__ __device__ constexpr uint32_t idesc_e4m3_f32(int n) {
    return (1u << 4)                          // D format: fp32
           | (0u << 7) | (0u << 10)           // A, B format: E4M3
           | (uint32_t(n >> 3) << 17)         // N / 8
           | (uint32_t(128 >> 4) << 24);      // M / 16
}

// Instruction descriptor of kind::mxf4nvf4 with block16 scaling: D fp32, A and
// B E2M1 (two codes a byte), both K-major, UE4M3 scale factors, M = 128,
// N = n, K = 64 an instruction; the scale-factor byte offsets (sf ids) are 0.
__host__ __device__ constexpr uint32_t idesc_nvf4_f32(int n) {
    return (1u << 7) | (1u << 10)           // A, B format: E2M1
           | (uint32_t(n >> 3) << 17)       // N / 8
           | (0u << 23)                     // scale format: UE4M3
           | (uint32_t(128 >> 4) << 24);    // M / 16
}

// D[tmem] (+)= (sfa . A[smem]) (sfb . B[smem])^T, kind::mxf4nvf4, one elected
// lane of the warp.  Scale factors live in tensor memory: for row r of A (B)
// and 16-element block j of this instruction's K = 64, the byte j of column
// sf + r/32, in lane r%32 of every 32-lane quadrant.
__device__ __forceinline__ void mma_nvf4_ss_warp(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                                 uint32_t sfa_tmem, uint32_t sfb_tmem, uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred pe, pa;\n\t"
        "elect.sync _|pe, 0xffffffff;\n\t"
        "setp.ne.b32 pa, %4, 0;\n\t"
        "@pe tcgen05.mma.cta_group::1.kind::mxf4nvf4.block_scale.block16 [%0], %1, %2, %3, [%5], [%6], pa;\n\t}"
        ::"r"(d_tmem), "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate), "r"(sfa_tmem), "r"(sfb_tmem)
        : "memory");
}

// Shared-memory matrix descriptor for a K-major operand stored as rows of
// `row_bytes` (64 or 128) with the matching swizzle, 8-row groups packed
// (stride 8 * row_bytes).  The tile base must be 1024-byte aligned.
__device__ __forceinline__ uint64_t smem_desc(uint32_t addr, int row_bytes) {
    const uint64_t start = (addr >> 4) & 0x3FFFu;
    const uint64_t lbo = 1;                                  // unused for swizzled K-major
    const uint64_t sbo = (uint64_t)((8 * row_bytes) >> 4);   // between 8-row groups
    const uint64_t layout = row_bytes == 128 ? 2 : 4;        // SWIZZLE_128B : SWIZZLE_64B
    return start | (lbo << 16) | (sbo << 32) | (1ull << 46) | (layout << 61);
}

// Byte offset of 16-byte chunk `chunk` of row `row` in a swizzled K-major tile
// with rows of `row_bytes` (the layout TMA writes with the same swizzle).
__device__ __forceinline__ uint32_t swz_offset(int row, int chunk, int row_bytes) {
    if (row_bytes == 128) return row * 128 + ((chunk ^ (row & 7)) << 4);
    return row * 64 + ((chunk ^ ((row >> 1) & 3)) << 4);
}

// ---------------------------------------------------------------- E4M3
// Two fp32 values -> two E4M3 bytes (round to nearest even, saturate to
// +-448); lo ends up in the low byte.
// A non-negative E4M3 byte -> its fp32 value, exactly: a 20-bit shift puts
// the byte's exponent and mantissa fields on fp32's (a subnormal byte on a
// subnormal float), and the bias difference (127 - 7) is a factor 2^120.
__device__ __forceinline__ float e4m3_to_f32(uint32_t code) {
    return __fmul_rn(__uint_as_float(code << 20), 0x1p120f);
}

// Eight fp32 values -> E2M1 codes (nearest, ties to even, saturating at 6),
// four bits each, x[0] in the lowest nibble.
__device__ __forceinline__ uint32_t e2m1x8(const float* x) {
    uint32_t out;
    asm("{\n\t.reg .b8 b0, b1, b2, b3;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b0, %2, %1;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b1, %4, %3;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b2, %6, %5;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b3, %8, %7;\n\t"
        "mov.b32 %0, {b0, b1, b2, b3};\n\t}"
        : "=r"(out)
        : "f"(x[0]), "f"(x[1]), "f"(x[2]), "f"(x[3]), "f"(x[4]), "f"(x[5]), "f"(x[6]), "f"(x[7]));
    return out;
}

__device__ __forceinline__ uint16_t e4m3x2(float lo, float hi) {
    uint16_t r;
    asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(hi), "f"(lo));
    return r;
}

// ---------------------------------------------------------------- ExpCast-FP8
// 1.5 * 2^23: adding it places an integer in the low mantissa bits of an fp32
// in [2^23, 2^24), where one unit is one ulp, so the FMA's own rounding
// (to nearest, ties to even) is the rounding to an integer.
constexpr float kMagic = 12582912.0f;

// Packed fp32 pair FMA (two IEEE fma.rn lanes in one instruction).
__device__ __forceinline__ float2 ffma2(float2 a, float2 b, float2 c) {
    float2 d;
    asm("{\n\t.reg .b64 ra, rb, rc, rd;\n\t"
        "mov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\tmov.b64 rc, {%6, %7};\n\t"
        "fma.rn.f32x2 rd, ra, rb, rc;\n\tmov.b64 {%0, %1}, rd;\n\t}"
        : "=f"(d.x), "=f"(d.y)
        : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y), "f"(c.x), "f"(c.y));
    return d;
}

__device__ __forceinline__ float fmax3(float a, float b, float c) {
    float r;
    asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
    return r;
}

// Four ExpCast bytes in one word (byte j from s_j), exactly
// clamp(round_half_even(A*s + cb), 0, 255) for an integer cb, |cb| < 2^22:
//  1. t = A*s + cbm, cbm = cb + 1.5*2^23: the packed FMA rounds A*s + cb, once,
//     to the integer n held in t's low mantissa bits (the one FMA per score).
//  2. w = t * 2^-149 - 1.5*2^-126 = n * 2^-149, exactly: a subnormal whose bit
//     pattern, read as int32, is n (n < 0, -inf included, gives a negative int).
//  3. cvt.pack.sat.u8.s32 clamps two such ints to [0, 255] and packs them.
// Six instructions for four scores, all exact.
__device__ __forceinline__ uint32_t pack2_sat_u8(int32_t hi, int32_t lo, uint32_t upper) {
    // [sat(lo), sat(hi), upper.b0, upper.b1] from byte 0 up
    uint32_t d;
    asm("cvt.pack.sat.u8.s32.b32 %0, %1, %2, %3;" : "=r"(d) : "r"(hi), "r"(lo), "r"(upper));
    return d;
}
__device__ __forceinline__ uint32_t expcast4(float A, float s0, float s1, float s2, float s3, float cbm) {
    const float2 t01 = ffma2(make_float2(A, A), make_float2(s0, s1), make_float2(cbm, cbm));
    const float2 t23 = ffma2(make_float2(A, A), make_float2(s2, s3), make_float2(cbm, cbm));
    const float k = __uint_as_float(1u);             // 2^-149
    const float mk = __uint_as_float(0x80C00000u);   // -1.5 * 2^-126 = -(1.5*2^23) * 2^-149
    const float2 w01 = ffma2(t01, make_float2(k, k), make_float2(mk, mk));
    const float2 w23 = ffma2(t23, make_float2(k, k), make_float2(mk, mk));
    const uint32_t hi = pack2_sat_u8(__float_as_int(w23.y), __float_as_int(w23.x), 0u);
    return pack2_sat_u8(__float_as_int(w01.y), __float_as_int(w01.x), hi);
}

// Mask of the bytes of a word of four codes that belong to keys inside the
// sequence: `left` keys remain from the word's first key on (<= 0: none, >= 4:
// all four, else the low `left` bytes).
__device__ __forceinline__ uint32_t tail_keep_mask(int left) {
    return left >= 4 ? 0xFFFFFFFFu : (left <= 0 ? 0u : (1u << (8 * left)) - 1u);
}

}  // namespace vc
