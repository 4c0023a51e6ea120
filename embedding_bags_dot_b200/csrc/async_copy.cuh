// Row gathers into shared memory with bulk copies (cp.async.bulk, no
// multicast) completing on an mbarrier, plus the ldmatrix load and bit-set
// helpers the warp-per-sample interaction kernels share.
#pragma once

#include "common.cuh"

namespace dlrm {
namespace ac {

constexpr int WAIT_TRIES = 1 << 20;  // bound on the mbarrier polls for one sample's rows (~1 s at 1 us each)

__device__ __forceinline__ void ldmatrix_x4(uint32_t addr, uint32_t (&r)[4]) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
                 : "r"(addr));
}

__device__ __forceinline__ void bar_init(uint32_t bar) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" ::"r"(bar) : "memory");
}
// The phase's single arrival, announcing the bytes its copies will deliver.
__device__ __forceinline__ void bar_expect(uint32_t bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes) : "memory");
}
// One contiguous global -> shared copy (addresses 16-byte aligned, bytes a multiple of 16).
__device__ __forceinline__ void bulk_row(uint32_t dst, const void* src, uint32_t bytes, uint32_t bar) {
    asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(dst),
                 "l"(src), "r"(bytes), "r"(bar)
                 : "memory");
}
// Orders this thread's earlier generic shared-memory accesses before later bulk-copy writes.
__device__ __forceinline__ void fence_proxy_async() { asm volatile("fence.proxy.async.shared::cta;" ::: "memory"); }
// Polls of the first wait for a sample's rows on this device (WAIT_TRIES unless a test lowered it with
// dlrm_set_wait_polls to make that wait run out). Each translation unit that includes this header has its
// own copy, set through its own set_rows_wait_tries_* function.
static __device__ int g_rows_wait_tries = WAIT_TRIES;

// Bounded wait for the phase of the given parity; false if it never completed within `tries` polls. Each
// poll suspends for at most about 1 us (the hint, in ns), so the bound is time-like, not a count of
// instructions.
__device__ __forceinline__ bool bar_wait_n(uint32_t bar, uint32_t parity, int tries) {
    for (int i = 0; i < tries; ++i) {
        uint32_t ok;
        asm volatile(
            "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n selp.u32 %0, 1, 0, p;\n}\n"
            : "=r"(ok)
            : "r"(bar), "r"(parity), "r"(1000u)
            : "memory");
        if (ok) return true;
    }
    return false;
}
__device__ __forceinline__ bool bar_wait(uint32_t bar, uint32_t parity) { return bar_wait_n(bar, parity, WAIT_TRIES); }

// The warp's wait for the rows of one phase (call with the whole warp converged), first with `tries` polls
// (a kernel reads g_rows_wait_tries once at its start). If any lane gives up, every lane waits again with
// the full bound, so that no copy is still landing in the region when the caller stops using it, and
// false is returned on every lane.
__device__ __forceinline__ bool rows_ready(uint32_t bar, uint32_t parity, int tries) {
    const bool ok = bar_wait_n(bar, parity, tries);
    if (__all_sync(0xffffffffu, ok)) return true;
    bar_wait_n(bar, parity, WAIT_TRIES);
    return false;
}

// Host side: sets this translation unit's first-wait bound on the current device (tries < 0: the default).
static inline cudaError_t set_rows_wait_tries_here(int tries) {
    const int v = tries < 0 ? WAIT_TRIES : tries;
    return cudaMemcpyToSymbol(g_rows_wait_tries, &v, sizeof(v));
}

// Position of the n-th (0-based) set bit of m, or -1.
__device__ __forceinline__ int nth_bit(unsigned long long m, int n) {
    for (int t = 0; t < n; ++t) m &= m - 1;
    return m ? __ffsll((long long)m) - 1 : -1;
}
__device__ __forceinline__ unsigned long long drop_bits(unsigned long long m, int n) {
    for (int t = 0; t < n; ++t) m &= m - 1;
    return m;
}

}  // namespace ac
}  // namespace dlrm
