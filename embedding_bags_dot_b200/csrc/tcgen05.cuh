// tcgen05 / TMA / mbarrier building blocks shared by the tensor-core GEMM kernels
// (inline PTX for sm_100a). Included by gemm_tc.cu and gemm_tf32.cu.
#pragma once

#include <cuda.h>

#include "common.cuh"

namespace dlrm {
namespace tc {

constexpr int BM = 128, BN = 256, BK = 64, STAGES = 4;
constexpr int A_BYTES = BM * BK * 2;
constexpr int B_BYTES = BN * BK * 2;
constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
constexpr int TMEM_COLS = 2 * BN;
constexpr int EPI_WARPS = 8;                       // two per TMEM lane quadrant, each half of the columns
constexpr int THREADS = 64 + 32 * EPI_WARPS;
constexpr int STAGE_OUT_BYTES = 32 * 128;          // per epilogue warp: 32 rows x 128 bytes, 128-byte swizzle
constexpr int OUT_BYTES = EPI_WARPS * STAGE_OUT_BYTES;
constexpr int SMEM_BYTES = STAGES * STAGE_BYTES + OUT_BYTES + 1024 + 256;
constexpr long long WAIT_LIMIT = 1ll << 26;

struct Bars {
    unsigned long long full[STAGES];
    unsigned long long empty[STAGES];
    unsigned long long tfull[2];
    unsigned long long tempty[2];
    unsigned long long drain;
    unsigned int tmem_base;
    int abort;
};

__device__ __forceinline__ uint32_t su32(const void* p) { return (uint32_t)__cvta_generic_to_shared(p); }

__device__ __forceinline__ void mbar_init(unsigned long long* b, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(su32(b)), "r"(count));
}
__device__ __forceinline__ void mbar_expect_tx(unsigned long long* b, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(su32(b)), "r"(bytes) : "memory");
}
__device__ __forceinline__ void mbar_arrive(unsigned long long* b) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(su32(b)) : "memory");
}
__device__ __forceinline__ bool mbar_try(unsigned long long* b, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n selp.u32 %0, 1, 0, p;\n}\n"
        : "=r"(ok)
        : "r"(su32(b)), "r"(parity)
        : "memory");
    return ok != 0;
}
// Bounded wait (at most `limit` polls) for the phase with the given parity to
// complete. Gives up early when another role has already aborted (unless
// ignore_abort).
__device__ __forceinline__ bool mbar_wait_n(unsigned long long* b, uint32_t parity, volatile int* abort,
                                            long long limit, bool ignore_abort = false) {
    for (long long i = 0; i < limit; ++i) {
        if (mbar_try(b, parity)) return true;
        if (!ignore_abort && (i & 255) == 255 && *abort) return false;
    }
    return false;
}
__device__ __forceinline__ bool mbar_wait(unsigned long long* b, uint32_t parity, volatile int* abort,
                                          bool ignore_abort = false) {
    return mbar_wait_n(b, parity, abort, WAIT_LIMIT, ignore_abort);
}

__device__ __forceinline__ void tma_load_2d(uint32_t dst, const CUtensorMap* map, unsigned long long* bar, int x,
                                            int y) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%3, %4}], [%2];" ::"r"(dst),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(su32(bar)), "r"(x), "r"(y)
        : "memory");
}

__device__ __forceinline__ void fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

// K-major operand tile with 128-byte swizzle: 8-row groups of 1024 bytes.
__device__ __forceinline__ uint64_t sdesc(uint32_t addr) {
    uint64_t d = (uint64_t)((addr & 0x3FFFFu) >> 4);
    d |= (uint64_t)1 << 16;            // leading byte offset (unused for swizzled K-major)
    d |= (uint64_t)(1024 >> 4) << 32;  // stride byte offset: next 8-row group
    d |= (uint64_t)1 << 46;            // descriptor version
    d |= (uint64_t)2 << 61;            // 128-byte swizzle
    return d;
}

// kind::f16 instruction descriptor: fp32 accumulate, A/B bf16 (1) or fp16 (0), both K-major, M = 128, N = n.
__host__ __device__ constexpr uint32_t idesc(int ab_fmt, int n = BN) {
    return (1u << 4) | ((uint32_t)ab_fmt << 7) | ((uint32_t)ab_fmt << 10) | ((uint32_t)(n >> 3) << 17) |
           ((uint32_t)(BM >> 4) << 24);
}

__device__ __forceinline__ void umma(uint32_t d_tmem, uint64_t a, uint64_t b, uint32_t id, uint32_t accum) {
    asm volatile(
        "{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n}\n" ::"r"(
            d_tmem),
        "l"(a), "l"(b), "r"(id), "r"(accum));
}
__device__ __forceinline__ void umma_commit(unsigned long long* bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(su32(bar))
                 : "memory");
}

__device__ __forceinline__ void tmem_ld32_issue(uint32_t taddr, uint32_t (&r)[32]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,%17,%18,%"
        "19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]), "=r"(r[8]),
          "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]), "=r"(r[16]),
          "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]),
          "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
        : "r"(taddr));
}
__device__ __forceinline__ void tmem_ld_wait() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }

template <int ACT>
__device__ __forceinline__ float act_fn(float v) {
    if constexpr (ACT == DLRM_ACT_RELU) return v > 0.f ? v : 0.f;
    if constexpr (ACT == DLRM_ACT_SIGMOID) return 1.f / (1.f + expf(-v));
    return v;
}

// Output tile rows of one epilogue warp, written through shared memory by TMA: for
// each 128-byte wide column chunk, the 32 lanes (one row each) convert their
// TMEM values, store them 128-byte swizzled into the warp's staging buffer,
// and lane 0 issues a bulk tensor store of the 32 x chunk box (rows and
// columns beyond the tensor are clipped by the TMA unit).
__device__ __forceinline__ void tma_store_2d(const CUtensorMap* map, uint32_t src, int x, int y) {
    asm volatile("cp.async.bulk.tensor.2d.global.shared::cta.bulk_group [%0, {%1, %2}], [%3];" ::"l"(
                     reinterpret_cast<uint64_t>(map)),
                 "r"(x), "r"(y), "r"(src)
                 : "memory");
    asm volatile("cp.async.bulk.commit_group;" ::: "memory");
}
__device__ __forceinline__ void bulk_wait_read0() { asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory"); }
__device__ __forceinline__ void bulk_wait_all0() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }

template <typename TC, int ACT, int NCOLS>
__device__ __forceinline__ void epilogue_tma(uint32_t taddr, int m0, int n_base, int N, const float* __restrict__ bias,
                                             const CUtensorMap* mapC, unsigned char* stage, uint32_t stage_s) {
    constexpr int CW = 128 / (int)sizeof(TC);   // columns per chunk: 64 (16-bit) or 32 (fp32)
    constexpr int NL = CW / 32;                 // 32-column TMEM loads per chunk
    const int lane = threadIdx.x & 31;
#pragma unroll 1
    for (int c = 0; c < NCOLS / CW; ++c) {
        const int n0 = n_base + c * CW;
        if (n0 >= N) break;   // uniform across the warp
        uint32_t r[NL][32];
#pragma unroll
        for (int h = 0; h < NL; ++h) tmem_ld32_issue(taddr + c * CW + 32 * h, r[h]);
        tmem_ld_wait();
        float v[CW];
#pragma unroll
        for (int h = 0; h < NL; ++h) {
            const int nh = n0 + 32 * h;
            if (nh + 32 <= N) {
                const float4* b4 = reinterpret_cast<const float4*>(bias + nh);
#pragma unroll
                for (int q = 0; q < 8; ++q) {
                    const float4 bq = __ldg(b4 + q);
                    v[32 * h + 4 * q + 0] = act_fn<ACT>(__uint_as_float(r[h][4 * q + 0]) + bq.x);
                    v[32 * h + 4 * q + 1] = act_fn<ACT>(__uint_as_float(r[h][4 * q + 1]) + bq.y);
                    v[32 * h + 4 * q + 2] = act_fn<ACT>(__uint_as_float(r[h][4 * q + 2]) + bq.z);
                    v[32 * h + 4 * q + 3] = act_fn<ACT>(__uint_as_float(r[h][4 * q + 3]) + bq.w);
                }
            } else {
#pragma unroll
                for (int j = 0; j < 32; ++j)
                    v[32 * h + j] = act_fn<ACT>(__uint_as_float(r[h][j]) + ((nh + j < N) ? __ldg(bias + nh + j) : 0.f));
            }
        }
        if (lane == 0) bulk_wait_read0();   // the previous chunk's store has read the staging buffer
        __syncwarp();
        unsigned char* row = stage + lane * 128;
#pragma unroll
        for (int q = 0; q < 8; ++q) {
            uint4 w;
            if constexpr (sizeof(TC) == 2) {
                TC t[8];
#pragma unroll
                for (int e = 0; e < 8; ++e) t[e] = Cvt<TC>::from_f(v[8 * q + e]);
                w = *reinterpret_cast<const uint4*>(t);
            } else {
                w = make_uint4(__float_as_uint(v[4 * q]), __float_as_uint(v[4 * q + 1]), __float_as_uint(v[4 * q + 2]),
                               __float_as_uint(v[4 * q + 3]));
            }
            *reinterpret_cast<uint4*>(row + 16 * (q ^ (lane & 7))) = w;
        }
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
        __syncwarp();
        if (lane == 0) tma_store_2d(mapC, stage_s, n0, m0);
    }
}


// ------------------------------------------------------------------ SM-pair building blocks
constexpr int BN2 = 256, STAGES2 = 6;
constexpr int A2_BYTES = 128 * BK * 2;
constexpr int B2_BYTES = (BN2 / 2) * BK * 2;
constexpr int STAGE2_BYTES = A2_BYTES + B2_BYTES;
constexpr int SMEM2_BYTES = STAGES2 * STAGE2_BYTES + OUT_BYTES + 1024 + 256;

struct Bars2 {
    unsigned long long full[STAGES2];
    unsigned long long empty[STAGES2];
    unsigned long long tfull[2];
    unsigned long long tempty[2];
    unsigned long long drain;
    unsigned int tmem_base;
    int abort;
};

__device__ __forceinline__ uint32_t cluster_rank() {
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
    return r;
}
// shared::cluster address of the same shared variable in CTA `rank` of the cluster
__device__ __forceinline__ uint32_t map_rank(uint32_t shared_addr, uint32_t rank) {
    uint32_t r;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(shared_addr), "r"(rank));
    return r;
}
__device__ __forceinline__ void mbar_arrive_cluster(uint32_t cluster_addr) {
    asm volatile("mbarrier.arrive.shared::cluster.b64 _, [%0];" ::"r"(cluster_addr) : "memory");
}
__device__ __forceinline__ void cluster_sync_all() {
    asm volatile("barrier.cluster.arrive.release.aligned;\nbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}
__device__ __forceinline__ void tma_load_2d_pair(uint32_t dst, const CUtensorMap* map, uint32_t leader_bar, int x,
                                                 int y) {
    asm volatile(
        "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%3, "
        "%4}], [%2];" ::"r"(dst),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(leader_bar), "r"(x), "r"(y)
        : "memory");
}
__device__ __forceinline__ void umma2(uint32_t d_tmem, uint64_t a, uint64_t b, uint32_t id, uint32_t accum) {
    asm volatile(
        "{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %3, p;\n}\n" ::"r"(
            d_tmem),
        "l"(a), "l"(b), "r"(id), "r"(accum));
}
// arrive on the barrier at this offset in both CTAs of the pair once all prior MMAs complete
__device__ __forceinline__ void umma2_commit_both(unsigned long long* bar) {
    const uint16_t mask = 0x3;
    asm volatile(
        "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64 [%0], %1;" ::"r"(
            su32(bar)),
        "h"(mask)
        : "memory");
}

__host__ __device__ constexpr uint32_t idesc2(int ab_fmt) {
    return (1u << 4) | ((uint32_t)ab_fmt << 7) | ((uint32_t)ab_fmt << 10) | ((uint32_t)(BN2 >> 3) << 17) |
           ((uint32_t)(256 >> 4) << 24);
}


typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);
// cuTensorMapEncodeTiled through the runtime's driver entry point (no link-time libcuda dependency).
EncodeTiledFn encode_fn();

}  // namespace tc
}  // namespace dlrm
