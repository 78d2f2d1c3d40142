// Shared device helpers for the sm_100a kernels: inline-PTX wrappers for
// mbarriers, TMA bulk-tensor copies, tcgen05 (TMEM allocation, MMA, loads),
// bounded waits and the sticky device status word.
//
// Every wait in these kernels is bounded: after IC_WAIT_TIMEOUT_NS of
// wall-clock time (the %globaltimer register) the waiting thread sets the
// CTA's abort flag and the device status to IC_ERR_TIMEOUT and returns
// false. Callers then run the rest of their loop without waiting (all later
// waits return at once) and without issuing new copies, MMAs or barrier
// arms, so every thread reaches the same named barriers; at teardown the
// copy and MMA issuers wait (bounded again) for what they issued before the
// abort to land, then the kernel frees its tensor memory and exits. Results
// are garbage and the host learns of it through ic_get_device_status().
//
// Every shared- and global-memory index in the hot loops is bounded by
// construction (list counts never pass their capacity, select outputs never
// pass k, compacted index rows hold only keys in [0, n_k)); the one count
// read back from global memory (the split lists' lengths in the merge) is
// checked, and a failed check records IC_ERR_INTERNAL. The IC_DEBUG build
// checks the by-construction indices too (IC_DCHECK).
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/indexcache.h"

#ifndef IC_WAIT_TIMEOUT_NS
#define IC_WAIT_TIMEOUT_NS 2000000000ull  // 2 s
#endif

namespace ic {

// Sticky status word of this device (IC_OK, or the first error recorded).
__device__ int g_device_status;

__device__ __forceinline__ void record_status(ic_status code) {
    atomicCAS(&g_device_status, 0, static_cast<int>(code));
}

// Consistency check on a value read back from memory: false (and
// IC_ERR_INTERNAL recorded) when it fails; the caller skips the access.
__device__ __forceinline__ bool in_bounds(bool ok) {
    if (__builtin_expect(!ok, 0)) record_status(IC_ERR_INTERNAL);
    return ok;
}

// Checks of indices that are in bounds by construction (list appends,
// select outputs, compacted index rows, gathered rows). The release build
// compiles them away; a build with -DIC_DEBUG (build.py --debug) evaluates
// them like in_bounds: a failure records IC_ERR_INTERNAL and skips the
// access, with no trap.
#ifdef IC_DEBUG
#define IC_DCHECK(cond) ::ic::in_bounds(cond)
#else
#define IC_DCHECK(cond) true
#endif

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ uint64_t globaltimer_ns() {
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

__device__ __forceinline__ uint32_t lane_id() { return threadIdx.x & 31; }

__device__ __forceinline__ uint32_t lanemask_lt() {
    uint32_t m;
    asm("mov.u32 %0, %%lanemask_lt;" : "=r"(m));
    return m;
}

// ---------------------------------------------------------------------------
// mbarrier
// ---------------------------------------------------------------------------
__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}

__device__ __forceinline__ void fence_mbar_init() {
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint32_t bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes)
                 : "memory");
}

// First 1024-byte aligned byte of dynamic shared memory. The offset is
// taken from the shared-window address and applied to the shared pointer
// itself, so accesses through the result stay shared-memory instructions
// (a round trip through an integer would make them generic).
__device__ __forceinline__ uint8_t* align_smem_1024(uint8_t* smem_raw) {
    const uint32_t a = smem_u32(smem_raw);
    return smem_raw + (((a + 1023u) & ~1023u) - a);
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

// Non-blocking test of the phase with the given parity (a poll: unlike
// try_wait, test_wait never suspends the thread).
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

// Like mbar_try_wait, but a thread whose phase is not complete may be
// suspended until it completes or for at most IC_WAIT_SUSPEND_NS: the waiting
// loops below poll far less often (fewer issue slots taken from the warps
// that share the scheduler).
#ifndef IC_WAIT_SUSPEND_NS
#define IC_WAIT_SUSPEND_NS 1000000u  // 1 ms
#endif
__device__ __forceinline__ bool mbar_try_wait_suspend(uint32_t bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(bar), "r"(parity), "r"(static_cast<uint32_t>(IC_WAIT_SUSPEND_NS))
        : "memory");
    return ok != 0;
}

// Bounded wait for the phase with the given parity to complete. Returns
// false (without waiting) once the CTA is in abort mode, or after the
// timeout, which also puts the CTA in abort mode.
__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity, volatile int* abort_flag,
                                          uint64_t timeout_ns = IC_WAIT_TIMEOUT_NS) {
    if (mbar_try_wait(bar, parity)) return true;
    if (*abort_flag) return false;
    const uint64_t t0 = globaltimer_ns();
    uint32_t spins = 0;
    while (true) {
        if (mbar_try_wait_suspend(bar, parity)) return true;
        if ((++spins & 15u) == 0) {
            if (*abort_flag) return false;
            if (globaltimer_ns() - t0 > timeout_ns) {
                *abort_flag = 1;
                record_status(IC_ERR_TIMEOUT);
                return false;
            }
        }
    }
}

// Teardown wait of an aborted CTA for a phase its own copies or MMAs will
// complete (they always land): ignores the abort flag, bounded all the same.
__device__ __forceinline__ void mbar_drain(uint32_t bar, uint32_t parity,
                                           uint64_t timeout_ns = IC_WAIT_TIMEOUT_NS) {
    if (mbar_try_wait(bar, parity)) return;
    const uint64_t t0 = globaltimer_ns();
    while (!mbar_try_wait_suspend(bar, parity)) {
        if (globaltimer_ns() - t0 > timeout_ns) {
            record_status(IC_ERR_TIMEOUT);
            return;
        }
    }
}

// ---------------------------------------------------------------------------
// Programmatic dependent launch. A kernel of the layer loop may be launched
// while its predecessor (another kernel of this library) is still finishing.
// Before a thread reads anything an earlier kernel of the loop wrote, or
// writes any global memory, it waits for the predecessor grid to complete
// (griddep_wait; a no-op for a kernel launched without the dependency). Only
// then does the CTA allow its own dependents to launch, so a dependent can
// never start while a kernel two launches back is still running.
// ---------------------------------------------------------------------------
__device__ __forceinline__ void griddep_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void griddep_launch_dependents() {
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}
__device__ __forceinline__ void griddep_sync() {
    griddep_wait();
    griddep_launch_dependents();
}

// ---------------------------------------------------------------------------
// Named barriers (a warpgroup synchronising among itself)
// ---------------------------------------------------------------------------
__device__ __forceinline__ void named_bar_sync(int id, int nthreads) {
    asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(nthreads) : "memory");
}

// Warp-specialised register reallocation (all warps of a warpgroup execute it).
template <int N>
__device__ __forceinline__ void regs_inc() {
    asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(N));
}
template <int N>
__device__ __forceinline__ void regs_dec() {
    asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(N));
}

// Barrier that also returns the OR of a predicate over the participating threads.
__device__ __forceinline__ bool named_bar_or(int id, int nthreads, bool pred) {
    uint32_t r;
    asm volatile(
        "{\n\t.reg .pred p, q;\n\t"
        "setp.ne.u32 p, %1, 0;\n\t"
        "bar.red.or.pred q, %2, %3, p;\n\t"
        "selp.u32 %0, 1, 0, q;\n\t}"
        : "=r"(r)
        : "r"(static_cast<uint32_t>(pred)), "r"(id), "r"(nthreads)
        : "memory");
    return r != 0;
}

// Count the entries of an index row that fall in [0, n_k), one warp.
__device__ __forceinline__ int warp_count_valid(const int32_t* row, int topk, int n_k, int lane) {
    int n = 0;
    for (int e = lane; e < topk; e += 32) {
        const int v = row[e];
        n += (v >= 0 && v < n_k) ? 1 : 0;
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) n += __shfl_xor_sync(0xffffffffu, n, o);
    return n;
}

// ---------------------------------------------------------------------------
// TMA (bulk tensor copies global -> shared, no multicast)
// ---------------------------------------------------------------------------
__device__ __forceinline__ void tma_load_2d(uint32_t dst, const CUtensorMap* tmap, uint32_t bar,
                                            int x, int y) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%3, %4}], [%2];" ::"r"(dst),
        "l"(reinterpret_cast<uint64_t>(tmap)), "r"(bar), "r"(x), "r"(y)
        : "memory");
}

// Row gather: 4 rows (row0..row3) x one box of columns starting at column x,
// written as 4 consecutive box rows at dst. The tensor map's box is one row
// high. No multicast.
__device__ __forceinline__ void tma_gather4(uint32_t dst, const CUtensorMap* tmap, uint32_t bar, int x,
                                            int row0, int row1, int row2, int row3) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.tile::gather4.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%3, %4, %5, %6, %7}], [%2];" ::"r"(dst),
        "l"(reinterpret_cast<uint64_t>(tmap)), "r"(bar), "r"(x), "r"(row0), "r"(row1), "r"(row2),
        "r"(row3)
        : "memory");
}

// Ask L2 to fetch `bytes` (a multiple of 16) at a 16-byte aligned global
// address; no data reaches the SM and nothing waits for it.
__device__ __forceinline__ void prefetch_l2_bulk(const void* src, uint32_t bytes) {
    asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(reinterpret_cast<uint64_t>(src)), "r"(bytes)
                 : "memory");
}

__device__ __forceinline__ void prefetch_tmap(const CUtensorMap* tmap) {
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(tmap)) : "memory");
}

// Order this thread's generic-proxy shared-memory writes before later
// async-proxy reads (tensor-core operand fetches).
__device__ __forceinline__ void fence_proxy_async_smem() {
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// ---------------------------------------------------------------------------
// cp.async (16-byte LDGSTS) for row gathers
// ---------------------------------------------------------------------------
__device__ __forceinline__ void cp_async_16(uint32_t dst, const void* src) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dst), "l"(src) : "memory");
}
__device__ __forceinline__ float ex2_approx(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

// 16-byte cp.async with source size `src_bytes` (0 writes 16 zero bytes).
__device__ __forceinline__ void cp_async_16_zfill(uint32_t dst, const void* src, uint32_t src_bytes) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(src_bytes)
                 : "memory");
}

__device__ __forceinline__ void cp_async_mbar_arrive_noinc(uint32_t bar) {
    asm volatile("cp.async.mbarrier.arrive.noinc.shared::cta.b64 [%0];" ::"r"(bar) : "memory");
}

__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() {
    asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}
__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_all;" ::: "memory"); }

// ---------------------------------------------------------------------------
// tcgen05: tensor memory and the 5th-generation tensor-core MMA
// ---------------------------------------------------------------------------
__device__ __forceinline__ void tmem_alloc(uint32_t dst_smem, uint32_t ncols) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(dst_smem),
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

// D(tmem) (+)= A(smem desc) * B(smem desc)^T, BF16/FP16 inputs, fp32 accumulate.
__device__ __forceinline__ void mma_f16(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                        uint32_t idesc, uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
        "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
        : "memory");
}

// Same with FP8/FP6/FP4 inputs (used for E4M3 x E4M3).
__device__ __forceinline__ void mma_f8(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                       uint32_t idesc, uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f8f6f4 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
        "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
        : "memory");
}

// Arrive on an mbarrier once all previously issued tcgen05 async operations
// of this thread have completed.
__device__ __forceinline__ void mma_commit(uint32_t bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                     bar)
                 : "memory");
}

__device__ __forceinline__ void tmem_wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }
__device__ __forceinline__ void tmem_wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

// Instruction descriptor (tcgen05 "instruction descriptor", 32 bits):
// D format fp32 (bits 4-5 = 1), A/B format (bits 7-9 / 10-12), both
// operands K-major unless mn_major bits are set (15 / 16), N >> 3 at bits
// 17-22, M >> 4 at bits 24-28.
__host__ __device__ constexpr uint32_t make_idesc(int M, int N, uint32_t a_fmt, uint32_t b_fmt,
                                                  uint32_t a_mn_major = 0, uint32_t b_mn_major = 0) {
    return (1u << 4) | (a_fmt << 7) | (b_fmt << 10) | (a_mn_major << 15) | (b_mn_major << 16) |
           ((static_cast<uint32_t>(N) >> 3) << 17) | ((static_cast<uint32_t>(M) >> 4) << 24);
}
constexpr uint32_t FMT_BF16 = 1;   // kind::f16
constexpr uint32_t FMT_E4M3 = 0;   // kind::f8f6f4

// Shared-memory matrix descriptor for a 128-byte-swizzled operand
// (bits 0-13 start address >> 4, 16-29 leading byte offset >> 4, 32-45
// stride byte offset >> 4, 46-47 version 1, 61-63 layout 2 = SWIZZLE_128B).
// K-major tiles: rows of 128 B, 8-row groups 1024 B apart (SBO), the leading
// offset is unused. MN-major tiles: `lbo` is the distance between 64-element
// (128 B) column blocks along M/N, SBO the distance between 8-row groups
// along K.
__device__ __forceinline__ uint64_t make_sw128_desc(uint32_t smem_addr, uint32_t lbo_bytes = 16,
                                                    uint32_t sbo_bytes = 1024) {
    uint64_t d = 0;
    d |= static_cast<uint64_t>((smem_addr & 0x3FFFFu) >> 4);
    d |= static_cast<uint64_t>((lbo_bytes >> 4) & 0x3FFFu) << 16;
    d |= static_cast<uint64_t>((sbo_bytes >> 4) & 0x3FFFu) << 32;
    d |= 1ull << 46;
    d |= 2ull << 61;
    return d;
}

// 32 lanes x 32 bit, N columns: thread i of the warp receives TMEM lane
// (warp's lane quarter + i), columns [col, col + N).
template <int N>
struct TmemLd;

template <>
struct TmemLd<4> {
    __device__ __forceinline__ static void ld(uint32_t taddr, uint32_t* r) {
        asm volatile("tcgen05.ld.sync.aligned.32x32b.x4.b32 {%0, %1, %2, %3}, [%4];"
                     : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
                     : "r"(taddr));
    }
};
template <>
struct TmemLd<8> {
    __device__ __forceinline__ static void ld(uint32_t taddr, uint32_t* r) {
        asm volatile("tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0, %1, %2, %3, %4, %5, %6, %7}, [%8];"
                     : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]),
                       "=r"(r[6]), "=r"(r[7])
                     : "r"(taddr));
    }
};
template <>
struct TmemLd<16> {
    __device__ __forceinline__ static void ld(uint32_t taddr, uint32_t* r) {
        asm volatile(
            "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, "
            "%11, %12, %13, %14, %15}, [%16];"
            : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
              "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]),
              "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
            : "r"(taddr));
    }
};
template <>
struct TmemLd<32> {
    __device__ __forceinline__ static void ld(uint32_t taddr, uint32_t* r) {
        asm volatile(
            "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, "
            "%11, %12, %13, %14, %15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, "
            "%28, %29, %30, %31}, [%32];"
            : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
              "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]),
              "=r"(r[13]), "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]),
              "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]),
              "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]),
              "=r"(r[31])
            : "r"(taddr));
    }
};
template <>
struct TmemLd<64> {
    __device__ __forceinline__ static void ld(uint32_t taddr, uint32_t* r) {
        TmemLd<32>::ld(taddr, r);
        TmemLd<32>::ld(taddr + 32, r + 32);
    }
};

template <int W>
__device__ __forceinline__ void tmem_ld(uint32_t taddr, uint32_t* r) {
    TmemLd<W>::ld(taddr, r);
}

// 16 lanes x 64 bit shape, 32 repetitions (64 columns of a 16-lane block):
// thread t receives TMEM lane (lane base + 8*(t&1) + (t>>2)), columns
// 2*r + ((t>>1)&1) for r = 0..31 - each lane's 64 columns are split between
// two threads (even / odd columns).
__device__ __forceinline__ void tmem_ld_16x64b_x32(uint32_t taddr, uint32_t* r) {
    asm volatile(
        "tcgen05.ld.sync.aligned.16x64b.x32.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, "
        "%11, %12, %13, %14, %15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, "
        "%28, %29, %30, %31}, [%32];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
          "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]),
          "=r"(r[13]), "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]),
          "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]),
          "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]),
          "=r"(r[31])
        : "r"(taddr));
}

// 16 lanes x 64 bit shape, repeated 16 times along the columns (32 columns):
// the first half of tmem_ld_16x64b_x32's registers.
__device__ __forceinline__ void tmem_ld_16x64b_x16(uint32_t taddr, uint32_t* r) {
    asm volatile(
        "tcgen05.ld.sync.aligned.16x64b.x16.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, "
        "%11, %12, %13, %14, %15}, [%16];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
          "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]),
          "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
        : "r"(taddr));
}

// 16 lanes x 256 bit shape, repeated 8 times along the columns (64 columns).
// Thread t receives, for repetition i (columns 8i .. 8i+7 of the window):
//   r[4i+0], r[4i+1]: lane t/4,     columns 8i + 2(t%4), 8i + 2(t%4) + 1
//   r[4i+2], r[4i+3]: lane t/4 + 8, the same two columns
// (lanes relative to the address's lane field).
__device__ __forceinline__ void tmem_ld_16x256b_x8(uint32_t taddr, uint32_t* r) {
    asm volatile(
        "tcgen05.ld.sync.aligned.16x256b.x8.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, "
        "%11, %12, %13, %14, %15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, "
        "%28, %29, %30, %31}, [%32];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
          "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]),
          "=r"(r[13]), "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]),
          "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]),
          "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]),
          "=r"(r[31])
        : "r"(taddr));
}

// 32 lanes x 32 bit store of 32 columns (the mirror of TmemLd<32>).
__device__ __forceinline__ void tmem_st32(uint32_t taddr, const uint32_t* r) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, "
        "%11, %12, %13, %14, %15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, "
        "%28, %29, %30, %31, %32};" ::"r"(taddr),
        "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]),
        "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]),
        "r"(r[15]), "r"(r[16]), "r"(r[17]), "r"(r[18]), "r"(r[19]), "r"(r[20]), "r"(r[21]),
        "r"(r[22]), "r"(r[23]), "r"(r[24]), "r"(r[25]), "r"(r[26]), "r"(r[27]), "r"(r[28]),
        "r"(r[29]), "r"(r[30]), "r"(r[31])
        : "memory");
}

// Order-preserving map of an fp32 value to an unsigned key (larger float ->
// larger key); -0.0 is first mapped to +0.0 so the two compare equal.
__device__ __forceinline__ uint32_t float_to_ordered(float f) {
    f = (f == 0.0f) ? 0.0f : f;
    const uint32_t u = __float_as_uint(f);
    return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

__host__ __device__ constexpr int ceil_div(int a, int b) { return (a + b - 1) / b; }

}  // namespace ic
