// Tensor-core fully connected layer for 16-bit activations and weights:
//   C[M][N] = act(A[M][K] W[N][K]^T + bias)      (fp32 accumulation in TMEM)
// the bottom/top MLP layers of DLRM ("Deep Learning Recommendation Model
// (DLRM)", nadeemcite summary, Key Method Details: FC layers with ReLU).
//
// sm_100a design: a persistent kernel, one 320-thread CTA per SM.
//   warp 0      TMA producer: 128x64 tiles of A and BNTx64 tiles of W (both
//               K-major, 128-byte swizzle) into a shared-memory ring;
//   warp 1      allocates 2 BNT TMEM columns (two 128 x BNT fp32
//               accumulators) and one thread issues tcgen05.mma (M=128,
//               N=BNT, K=16);
//   warps 2..9  epilogue: tcgen05.ld of the finished accumulator (each warp
//               owns the 32 TMEM lanes of its quadrant and a share of the
//               columns), bias, activation, conversion into a 128-byte
//               swizzled shared-memory stage written out by TMA bulk tensor
//               stores, while the MMA warp already fills the other accumulator.
// Two tile widths: BNT = 256 (4-stage ring), and BNT = 64 (8-stage ring) for
// small batches, where a layer has few 128-row tiles: four times the CTAs, each
// streaming a quarter of the weights, with twice the loads in flight. Below 128
// rows the A box holds only the batch's rows (rounded up to 8); the MMA still
// reads 128 rows, and the rows past the box only reach accumulator rows that
// are never stored.
// Shared-memory stages are released by tcgen05.commit onto an mbarrier. All
// waits are bounded: on timeout the kernel records DLRM_ERR_TIMEOUT in the
// error record, drains its own copies and MMAs (again bounded), frees TMEM
// and returns. No cluster multicast is used. Launched as a programmatic
// dependent: barriers and TMEM are set up before pdl_wait().
#include <cuda.h>

#include "common.cuh"
#include "kernels.cuh"
#include "tcgen05.cuh"

namespace dlrm {
namespace tc {

// Polls of the ordinary waits of linear_tc_kernel on this device (WAIT_LIMIT unless a test lowered it
// with dlrm_set_wait_polls to make them run out). The drains after a timeout always use WAIT_LIMIT.
static __device__ long long g_tc1_wait_polls = WAIT_LIMIT;

// Shared-memory plan of the single-CTA kernel for tile width BNT.
template <int BNT>
struct Tile1 {
    static constexpr int NS = BNT == BN ? STAGES : 8;     // ring stages
    static constexpr int W_BYTES = BNT * BK * 2;
    static constexpr int STAGE = A_BYTES + W_BYTES;
    static constexpr int TMEM = 2 * BNT;
    static constexpr int SMEM = NS * STAGE + OUT_BYTES + 1024 + 256;
    // epilogue columns per warp: half the tile per warp of a quadrant, or the whole tile for the first
    // warp when half of it is narrower than one 128-byte chunk of 16-bit output
    static constexpr int WC = BNT >= 128 ? BNT / 2 : BNT;
};

template <int NS>
struct BarsN {
    unsigned long long full[NS];
    unsigned long long empty[NS];
    unsigned long long tfull[2];
    unsigned long long tempty[2];
    unsigned long long drain;
    unsigned int tmem_base;
    int abort;
};

template <typename TC, int ACT, int BNT>
__global__ void __launch_bounds__(THREADS, 1)
    linear_tc_kernel(const __grid_constant__ CUtensorMap mapA, const __grid_constant__ CUtensorMap mapW,
                     const __grid_constant__ CUtensorMap mapC, int M, int N, int K, const float* __restrict__ bias,
                     uint32_t id, uint32_t a_tx, ErrRecord* err) {
    using T = Tile1<BNT>;
    constexpr int NS = T::NS;
    extern __shared__ __align__(1024) unsigned char smem_raw[];
    const uint32_t raw = su32(smem_raw);
    const uint32_t base = (raw + 1023u) & ~1023u;
    unsigned char* gbase = smem_raw + (base - raw);
    BarsN<NS>* bars = reinterpret_cast<BarsN<NS>*>(gbase + NS * T::STAGE + OUT_BYTES);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int nbn = (N + BNT - 1) / BNT;
    const int ntiles = ((M + BM - 1) / BM) * nbn;
    const int nk = (K + BK - 1) / BK;

    if (threadIdx.x == 0) {
        for (int s = 0; s < NS; ++s) {
            mbar_init(&bars->full[s], 1);
            mbar_init(&bars->empty[s], 1);
        }
        for (int a = 0; a < 2; ++a) {
            mbar_init(&bars->tfull[a], 1);
            mbar_init(&bars->tempty[a], EPI_WARPS);
        }
        mbar_init(&bars->drain, 1);
        bars->abort = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    if (warp == 1) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(su32(&bars->tmem_base)),
                     "r"(T::TMEM));
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
    }
    if (warp == 0 && lane == 0) {
        asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&mapA)) : "memory");
        asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&mapW)) : "memory");
    }
    fence_before();
    __syncthreads();
    fence_after();
    pdl_wait();      // the previous kernel's outputs (A) are complete and visible from here on
    const uint32_t tmem = bars->tmem_base;
    volatile int* abort = &bars->abort;
    bool timed_out = false;
    const long long lim = g_tc1_wait_polls;

    if (warp == 0) {
        if (lane == 0) {
            int s = 0;
            uint32_t ph = 0;
            for (int t = blockIdx.x; t < ntiles && !timed_out; t += gridDim.x) {
                const int mb = t / nbn, nb = t - mb * nbn;
                for (int kb = 0; kb < nk; ++kb) {
                    if (!mbar_wait_n(&bars->empty[s], ph ^ 1u, abort, lim)) {
                        timed_out = true;
                        break;
                    }
                    const uint32_t sa = base + s * T::STAGE;
                    mbar_expect_tx(&bars->full[s], a_tx + T::W_BYTES);
                    tma_load_2d(sa, &mapA, &bars->full[s], kb * BK, mb * BM);
                    tma_load_2d(sa + A_BYTES, &mapW, &bars->full[s], kb * BK, nb * BNT);
                    if (++s == NS) {
                        s = 0;
                        ph ^= 1u;
                    }
                }
            }
            if (timed_out) *abort = 1;
            // drain, also when another role gave up: every stage whose load may still be in flight
            // completes its full phase before the CTA may exit (a stage never loaded, or already
            // consumed, passes at once)
            for (int q = 0; q < NS; ++q) {
                if (--s < 0) {
                    s = NS - 1;
                    ph ^= 1u;
                }
                mbar_wait(&bars->full[s], ph, abort, true);
            }
        }
    } else if (warp == 1) {
        if (lane == 0) {
            const uint32_t id_ = id;
            int s = 0;
            uint32_t ph = 0;
            int i = 0;
            for (int t = blockIdx.x; t < ntiles && !timed_out; t += gridDim.x, ++i) {
                const int acc = i & 1;
                const uint32_t use = (uint32_t)(i >> 1);
                if (!mbar_wait_n(&bars->tempty[acc], (use & 1u) ^ 1u, abort, lim)) {
                    timed_out = true;
                    break;
                }
                fence_after();
                const uint32_t d = tmem + (uint32_t)(acc * BNT);
                for (int kb = 0; kb < nk; ++kb) {
                    if (!mbar_wait_n(&bars->full[s], ph, abort, lim)) {
                        timed_out = true;
                        break;
                    }
                    fence_after();
                    const uint32_t sa = base + s * T::STAGE;
#pragma unroll
                    for (int k = 0; k < BK / 16; ++k)
                        umma(d, sdesc(sa + k * 32), sdesc(sa + A_BYTES + k * 32), id_, (kb | k) != 0);
                    umma_commit(&bars->empty[s]);
                    if (++s == NS) {
                        s = 0;
                        ph ^= 1u;
                    }
                }
                if (timed_out) break;
                umma_commit(&bars->tfull[acc]);
            }
            if (timed_out) *abort = 1;
            // all MMAs issued by this thread have completed once this fires
            umma_commit(&bars->drain);
            mbar_wait(&bars->drain, 0, abort, true);
        }
    } else {
        const int ew = warp - 2;   // epilogue warp 0..7
        const int q = warp & 3;    // TMEM lane quadrant this warp may access
        const int h = ew >> 2;     // which share of the tile's columns
        const bool active = h * T::WC < BNT;
        unsigned char* stage = gbase + NS * T::STAGE + ew * STAGE_OUT_BYTES;
        const uint32_t stage_s = base + NS * T::STAGE + ew * STAGE_OUT_BYTES;
        int i = 0;
        for (int t = blockIdx.x; t < ntiles && !timed_out; t += gridDim.x, ++i) {
            const int acc = i & 1;
            const uint32_t use = (uint32_t)(i >> 1);
            if (!mbar_wait_n(&bars->tfull[acc], use & 1u, abort, lim)) {
                timed_out = true;
                break;
            }
            fence_after();
            if (active) {
                const int mb = t / nbn, nb = t - mb * nbn;
                const uint32_t taddr = tmem + ((uint32_t)(q * 32) << 16) + (uint32_t)(acc * BNT + h * T::WC);
                epilogue_tma<TC, ACT, T::WC>(taddr, mb * BM + q * 32, nb * BNT + h * T::WC, N, bias, &mapC, stage,
                                             stage_s);
            }
            fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&bars->tempty[acc]);
        }
        if (timed_out) *abort = 1;
        if (lane == 0) bulk_wait_all0();
    }

    if (timed_out && lane == 0) atomicOr(&err->flags, (unsigned)ERR_TIMEOUT);
    fence_before();
    __syncthreads();
    fence_after();
    if (warp == 1) {
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(T::TMEM));
    }
}


// ------------------------------------------------------------------ 2-SM variant
//
// A cluster of two CTAs (one per SM of a pair) computes a 256x256 tile with
// tcgen05.mma.cta_group::2 (M = 256, N = 256, K = 16): CTA r loads rows
// [128 r, 128 r + 128) of the A tile and of the W tile (its halves of M and
// N), so each SM streams 32 KB per 64-deep k-block instead of 48 KB. The
// leader (rank 0) issues the MMAs; both CTAs' TMA loads complete on the
// leader's full barrier; the MMA commits are multicast to both CTAs' empty and
// accumulator-full barriers; both CTAs' epilogues release the accumulator on
// the leader's barrier. Each CTA's TMEM holds the 128 rows of its M half.
// ACT_RELU_LOGIT: the layer's ReLU output h (N <= 256, one tile wide) is not
// stored; the epilogue forms the next, one-column layer instead:
// y[m] = sigmoid(sum_j h[m][j] w[j] + b). Both epilogue warps of a TMEM lane
// quadrant take 128 columns of the quadrant's 32 rows (one thread per row,
// columns in order, bias and w read from shared memory); the two partial sums
// of a row meet in a shared slot by atomic exchange, and the thread that finds
// its partner's sum there finishes the row. No warp waits on the other.
constexpr int ACT_RELU_LOGIT = 16;
constexpr uint32_t LOGIT_EMPTY = 0x7FC0DEADu;   // slot holding no partial sum (a NaN no arithmetic produces)
template <typename TW>
struct LogitArgs {
    const TW* w;       // [N] weights of the one-column layer
    const float* b;    // its bias (one float)
    float* y;          // [M] output
};

template <typename TC, int ACT>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(THREADS, 1)
    linear_tc2_kernel(const __grid_constant__ CUtensorMap mapA, const __grid_constant__ CUtensorMap mapW,
                      const __grid_constant__ CUtensorMap mapC, int M, int N, int K, const float* __restrict__ bias,
                      uint32_t id, ErrRecord* err, LogitArgs<TC> la) {
    extern __shared__ __align__(1024) unsigned char smem_raw[];
    const uint32_t raw = su32(smem_raw);
    const uint32_t base = (raw + 1023u) & ~1023u;
    unsigned char* gbase = smem_raw + (base - raw);
    Bars2* bars = reinterpret_cast<Bars2*>(gbase + STAGES2 * STAGE2_BYTES + OUT_BYTES);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t rank = cluster_rank();
    const bool leader = rank == 0;
    const int npair = gridDim.x >> 1, pair = blockIdx.x >> 1;
    const int nbn = (N + BN2 - 1) / BN2;
    const int ntiles = ((M + 255) / 256) * nbn;
    const int nk = (K + BK - 1) / BK;

    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES2; ++s) {
            mbar_init(&bars->full[s], 1);
            mbar_init(&bars->empty[s], 1);
        }
        for (int a = 0; a < 2; ++a) {
            mbar_init(&bars->tfull[a], 1);
            mbar_init(&bars->tempty[a], 2 * EPI_WARPS);   // lane 0 of every epilogue warp of both CTAs
        }
        mbar_init(&bars->drain, 1);
        bars->abort = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    if (warp == 1) {
        asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(su32(&bars->tmem_base)),
                     "r"(TMEM_COLS));
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;");
    }
    pdl_wait();      // the previous kernel's outputs (A) are complete and visible from here on
    if constexpr (ACT == ACT_RELU_LOGIT) {
        // each epilogue warp's (unused) output stage: [0, 128) bias and [128, 256) w of its 128 columns;
        // the quadrant's first warp also holds the exchange slots [256, 320): two tile parities x 32 rows
        if (warp >= 2) {
            const int ew = warp - 2, h = ew >> 2;
            float* bw = reinterpret_cast<float*>(gbase + STAGES2 * STAGE2_BYTES + ew * STAGE_OUT_BYTES);
            for (int j = lane; j < BN2 / 2; j += 32) {
                const int col = h * (BN2 / 2) + j;
                bw[j] = col < N ? __ldg(bias + col) : 0.f;
                bw[BN2 / 2 + j] = col < N ? Cvt<TC>::to_f(la.w[col]) : 0.f;
            }
            if (h == 0)
                for (int j = lane; j < 64; j += 32) bw[BN2 + j] = __uint_as_float(LOGIT_EMPTY);
        }
    }
    fence_before();
    cluster_sync_all();   // both CTAs' barriers initialised and TMEM allocated before any cross-CTA signal
    fence_after();
    const uint32_t tmem = bars->tmem_base;
    volatile int* abort = &bars->abort;
    bool timed_out = false;

    if (warp == 0) {
        if (lane == 0) {
            asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&mapA)) : "memory");
            asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&mapW)) : "memory");
            int s = 0;
            uint32_t ph = 0;
            for (int t = pair; t < ntiles && !timed_out; t += npair) {
                const int mb = t / nbn, nb = t - mb * nbn;
                for (int kb = 0; kb < nk; ++kb) {
                    if (!mbar_wait(&bars->empty[s], ph ^ 1u, abort)) {
                        timed_out = true;
                        break;
                    }
                    const uint32_t sa = base + s * STAGE2_BYTES;
                    const uint32_t lead_full = map_rank(su32(&bars->full[s]), 0);
                    if (leader) mbar_expect_tx(&bars->full[s], 2 * STAGE2_BYTES);
                    tma_load_2d_pair(sa, &mapA, lead_full, kb * BK, mb * 256 + (int)rank * 128);
                    tma_load_2d_pair(sa + A2_BYTES, &mapW, lead_full, kb * BK, nb * BN2 + (int)rank * (BN2 / 2));
                    if (++s == STAGES2) {
                        s = 0;
                        ph ^= 1u;
                    }
                }
            }
            if (timed_out) *abort = 1;
            // every load this CTA issued completes before it may exit: wait (bounded) for the
            // empty barriers, which the leader's MMA commits after consuming each stage
            for (int q = 0; q < STAGES2; ++q) {
                mbar_wait(&bars->empty[s], ph ^ 1u, abort, true);
                if (++s == STAGES2) {
                    s = 0;
                    ph ^= 1u;
                }
            }
        }
    } else if (warp == 1) {
        if (lane == 0 && leader) {
            int s = 0;
            uint32_t ph = 0;
            int i = 0;
            for (int t = pair; t < ntiles && !timed_out; t += npair, ++i) {
                const int acc = i & 1;
                const uint32_t use = (uint32_t)(i >> 1);
                if (!mbar_wait(&bars->tempty[acc], (use & 1u) ^ 1u, abort)) {
                    timed_out = true;
                    break;
                }
                fence_after();
                const uint32_t d = tmem + (uint32_t)(acc * BN2);
                for (int kb = 0; kb < nk; ++kb) {
                    if (!mbar_wait(&bars->full[s], ph, abort)) {
                        timed_out = true;
                        break;
                    }
                    fence_after();
                    const uint32_t sa = base + s * STAGE2_BYTES;
#pragma unroll
                    for (int k = 0; k < BK / 16; ++k)
                        umma2(d, sdesc(sa + k * 32), sdesc(sa + A2_BYTES + k * 32), id, (kb | k) != 0);
                    umma2_commit_both(&bars->empty[s]);
                    if (++s == STAGES2) {
                        s = 0;
                        ph ^= 1u;
                    }
                }
                if (timed_out) break;
                umma2_commit_both(&bars->tfull[acc]);
            }
            if (timed_out) *abort = 1;
            umma2_commit_both(&bars->drain);
            mbar_wait(&bars->drain, 0, abort, true);
        } else if (lane == 0) {
            // the peer's MMA-issue thread has nothing to issue; it waits for the leader's drain
            mbar_wait(&bars->drain, 0, abort, true);
        }
    } else {
        const int ew = warp - 2;
        const int q = warp & 3;
        const int h = ew >> 2;
        unsigned char* stage = gbase + STAGES2 * STAGE2_BYTES + ew * STAGE_OUT_BYTES;
        const uint32_t stage_s = base + STAGES2 * STAGE2_BYTES + ew * STAGE_OUT_BYTES;
        const uint32_t lead_tempty0 = map_rank(su32(&bars->tempty[0]), 0);
        const uint32_t lead_tempty1 = map_rank(su32(&bars->tempty[1]), 0);
        int i = 0;
        for (int t = pair; t < ntiles && !timed_out; t += npair, ++i) {
            const int acc = i & 1;
            const uint32_t use = (uint32_t)(i >> 1);
            if (!mbar_wait(&bars->tfull[acc], use & 1u, abort)) {
                timed_out = true;
                break;
            }
            fence_after();
            const int mb = t / nbn, nb = t - mb * nbn;
            const uint32_t taddr = tmem + ((uint32_t)(q * 32) << 16) + (uint32_t)(acc * BN2 + h * (BN2 / 2));
            if constexpr (ACT == ACT_RELU_LOGIT) {
                const float* bw = reinterpret_cast<const float*>(stage);
                float part = 0.f;
#pragma unroll 1
                for (int c = 0; c < BN2 / 64; ++c) {
                    uint32_t r[32];
                    tmem_ld32_issue(taddr + 32 * c, r);
                    tmem_ld_wait();
#pragma unroll
                    for (int e = 0; e < 32; e += 4) {
                        const float4 bb = *reinterpret_cast<const float4*>(bw + 32 * c + e);
                        const float4 ww = *reinterpret_cast<const float4*>(bw + BN2 / 2 + 32 * c + e);
                        part = fmaf(fmaxf(__uint_as_float(r[e]) + bb.x, 0.f), ww.x, part);
                        part = fmaf(fmaxf(__uint_as_float(r[e + 1]) + bb.y, 0.f), ww.y, part);
                        part = fmaf(fmaxf(__uint_as_float(r[e + 2]) + bb.z, 0.f), ww.z, part);
                        part = fmaf(fmaxf(__uint_as_float(r[e + 3]) + bb.w, 0.f), ww.w, part);
                    }
                }
                // the row's two halves meet in the quadrant's slot for this accumulator; the slot is next used two
                // tiles later, after both warps have released this accumulator
                float* slot = reinterpret_cast<float*>(gbase + STAGES2 * STAGE2_BYTES + ((q + 2) & 3) * STAGE_OUT_BYTES) +
                              BN2 + 32 * acc + lane;
                const float other = atomicExch(slot, part);
                if (__float_as_uint(other) != LOGIT_EMPTY) {
                    *slot = __uint_as_float(LOGIT_EMPTY);
                    const long long row = (long long)mb * 256 + (int)rank * 128 + q * 32 + lane;
                    if (row < M) la.y[row] = 1.f / (1.f + expf(-((part + other) + __ldg(la.b))));
                }
            } else {
                epilogue_tma<TC, ACT, BN2 / 2>(taddr, mb * 256 + (int)rank * 128 + q * 32, nb * BN2 + h * (BN2 / 2),
                                               N, bias, &mapC, stage, stage_s);
            }
            fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive_cluster(acc ? lead_tempty1 : lead_tempty0);
        }
        if (timed_out) *abort = 1;
        if (lane == 0) bulk_wait_all0();
    }

    if (timed_out && lane == 0) atomicOr(&err->flags, (unsigned)ERR_TIMEOUT);
    fence_before();
    cluster_sync_all();   // no CTA frees TMEM or exits while its pair still signals it
    fence_after();
    if (warp == 1) {
        asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(TMEM_COLS));
    }
}

// ------------------------------------------------------------------ host side

EncodeTiledFn encode_fn() {
    static EncodeTiledFn fn = nullptr;
    if (!fn) {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(p);
    }
    return fn;
}

static bool make_map(CUtensorMap* map, const void* ptr, dlrm_dtype dt, int inner, int outer, int ld, int box_outer,
                     int box_inner = BK) {
    EncodeTiledFn enc = encode_fn();
    if (!enc) return false;
    const cuuint64_t dims[2] = {(cuuint64_t)inner, (cuuint64_t)outer};
    const size_t es = dt == DLRM_F32 ? 4 : 2;
    const cuuint64_t strides[1] = {(cuuint64_t)ld * es};
    const cuuint32_t box[2] = {(cuuint32_t)box_inner, (cuuint32_t)box_outer};
    const cuuint32_t estr[2] = {1, 1};
    const CUtensorMapDataType t = dt == DLRM_BF16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16
                                  : dt == DLRM_F16 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16
                                                   : CU_TENSOR_MAP_DATA_TYPE_FLOAT32;
    return enc(map, t, 2, const_cast<void*>(ptr), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
               CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

static int sm_count() {
    static int n[64] = {0};
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev < 0 || dev >= 64) return 148;
    if (!n[dev]) {
        int v = 0;
        cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev);
        n[dev] = v > 0 ? v : 148;
    }
    return n[dev];
}

template <typename TC, int ACT, int BNT>
static dlrm_status launch_t(const CUtensorMap& ma, const CUtensorMap& mw, const CUtensorMap& mc, int M, int N, int K,
                            const float* bias, uint32_t id, uint32_t a_tx, ErrRecord* err, cudaStream_t st) {
    auto kern = linear_tc_kernel<TC, ACT, BNT>;
    cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, Tile1<BNT>::SMEM);
    const int ntiles = ((M + BM - 1) / BM) * ((N + BNT - 1) / BNT);
    const int grid = ntiles < sm_count() ? ntiles : sm_count();
    DLRM_PDL_CHECK(launch_pdl(kern, dim3(grid), dim3(THREADS), (size_t)Tile1<BNT>::SMEM, st, ma, mw, mc, M, N, K, bias,
                              id, a_tx, err));
    return DLRM_OK;
}

template <typename TC, int ACT>
static dlrm_status launch_t2(const CUtensorMap& ma, const CUtensorMap& mw, const CUtensorMap& mc, int M, int N, int K,
                             const float* bias, uint32_t id, ErrRecord* err, cudaStream_t st,
                             LogitArgs<TC> la = LogitArgs<TC>{nullptr, nullptr, nullptr}) {
    auto kern = linear_tc2_kernel<TC, ACT>;
    cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM2_BYTES);
    const int ntiles = ((M + 255) / 256) * ((N + BN2 - 1) / BN2);
    const int pairs = sm_count() / 2;
    const int grid = 2 * (ntiles < pairs ? ntiles : pairs);
    DLRM_PDL_CHECK(launch_pdl(kern, dim3(grid), dim3(THREADS), (size_t)SMEM2_BYTES, st, ma, mw, mc, M, N, K, bias, id,
                              err, la));
    return DLRM_OK;
}

}  // namespace tc

cudaError_t set_wait_polls_gemm_tc(long long polls) {
    const long long v = polls < 0 ? tc::WAIT_LIMIT : polls;
    return cudaMemcpyToSymbol(tc::g_tc1_wait_polls, &v, sizeof(v));
}

bool linear_tc_logit_supported(int M, int N, int K, const void* A, dlrm_dtype a_dt, int lda, const void* W,
                               dlrm_dtype w_dt, int ldw, const float* bias) {
    // the SM-pair kernel (M >= 4096) with the whole layer output in one 256-wide tile
    if (M < 256 * 16 || N > tc::BN2) return false;
    if (a_dt != w_dt || a_dt == DLRM_F32 || N < 2 || K < 1 || (lda % 8) || (ldw % 8)) return false;
    if (((uintptr_t)A & 15) || ((uintptr_t)W & 15) || ((uintptr_t)bias & 15)) return false;
    return tc::encode_fn() != nullptr;
}

dlrm_status launch_linear_tc_logit(int M, int N, int K, const void* A, dlrm_dtype a_dt, int lda, const void* W,
                                   int ldw, const float* bias, const void* w_next, const float* b_next, float* y,
                                   ErrRecord* err, cudaStream_t st) {
    CUtensorMap ma, mw;
    if (!tc::make_map(&ma, A, a_dt, K, M, lda, tc::BM) || !tc::make_map(&mw, W, a_dt, K, N, ldw, tc::BN2 / 2))
        return DLRM_ERR_CUDA;
    const int fmt = a_dt == DLRM_BF16 ? 1 : 0;
    if (a_dt == DLRM_BF16)
        return tc::launch_t2<__nv_bfloat16, tc::ACT_RELU_LOGIT>(
            ma, mw, mw, M, N, K, bias, tc::idesc2(fmt), err, st,
            tc::LogitArgs<__nv_bfloat16>{static_cast<const __nv_bfloat16*>(w_next), b_next, y});
    return tc::launch_t2<__half, tc::ACT_RELU_LOGIT>(ma, mw, mw, M, N, K, bias, tc::idesc2(fmt), err, st,
                                                     tc::LogitArgs<__half>{static_cast<const __half*>(w_next), b_next, y});
}

bool linear_tc_supported(int M, int N, int K, const void* A, dlrm_dtype a_dt, int lda, const void* W, dlrm_dtype w_dt,
                         int ldw, const float* bias, void* C, dlrm_dtype c_dt, int ldc) {
    if (a_dt != w_dt || a_dt == DLRM_F32) return false;
    if (M < 1 || N < 2 || K < 1) return false;
    if ((lda % 8) || (ldw % 8)) return false;
    if (((uintptr_t)A & 15) || ((uintptr_t)W & 15) || ((uintptr_t)C & 15) || ((uintptr_t)bias & 15)) return false;
    if (c_dt != DLRM_F32 && c_dt != a_dt) return false;
    if (ldc % (c_dt == DLRM_F32 ? 4 : 8)) return false;
    return tc::encode_fn() != nullptr;
}

dlrm_status launch_linear_tc(int M, int N, int K, const void* A, dlrm_dtype a_dt, int lda, const void* W, int ldw,
                             const float* bias, void* C, dlrm_dtype c_dt, int ldc, int act, ErrRecord* err,
                             cudaStream_t st) {
    // 256-row tiles on SM pairs when there are enough of them to fill the GPU; otherwise 128-row tiles,
    // 64 columns wide when 256-wide tiles would leave most SMs idle
    const bool pair = M >= 256 * 16;
    const bool narrow = !pair && (long long)((M + tc::BM - 1) / tc::BM) * ((N + tc::BN - 1) / tc::BN) * 2 <= tc::sm_count();
    const int bnt = pair ? tc::BN2 / 2 : narrow ? 64 : tc::BN;
    // A box: the batch's rows (rounded up to 8) when they fit one tile, else a whole tile
    const int a_rows = M < tc::BM ? (M + 7) & ~7 : tc::BM;
    CUtensorMap ma, mw, mc;
    if (!tc::make_map(&ma, A, a_dt, K, M, lda, pair ? tc::BM : a_rows) || !tc::make_map(&mw, W, a_dt, K, N, ldw, bnt) ||
        !tc::make_map(&mc, C, c_dt, N, M, ldc, 32, c_dt == DLRM_F32 ? 32 : 64))
        return DLRM_ERR_CUDA;
    const int fmt = a_dt == DLRM_BF16 ? 1 : 0;
    const uint32_t a_tx = (uint32_t)a_rows * tc::BK * 2;
#define DLRM_TC_ACT(TC, ACT)                                                                                    \
    return pair     ? tc::launch_t2<TC, ACT>(ma, mw, mc, M, N, K, bias, tc::idesc2(fmt), err, st)               \
           : narrow ? tc::launch_t<TC, ACT, 64>(ma, mw, mc, M, N, K, bias, tc::idesc(fmt, 64), a_tx, err, st)   \
                    : tc::launch_t<TC, ACT, tc::BN>(ma, mw, mc, M, N, K, bias, tc::idesc(fmt), a_tx, err, st);
#define DLRM_TC(TC)                                       \
    switch (act) {                                        \
        case DLRM_ACT_RELU: DLRM_TC_ACT(TC, DLRM_ACT_RELU)       \
        case DLRM_ACT_SIGMOID: DLRM_TC_ACT(TC, DLRM_ACT_SIGMOID) \
        default: DLRM_TC_ACT(TC, DLRM_ACT_NONE)                  \
    }
    if (c_dt == DLRM_F32) {
        DLRM_TC(float)
    } else if (c_dt == DLRM_BF16) {
        DLRM_TC(__nv_bfloat16)
    } else {
        DLRM_TC(__half)
    }
#undef DLRM_TC
#undef DLRM_TC_ACT
}

}  // namespace dlrm
