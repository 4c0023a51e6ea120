// fp32 GEMMs of the training step on the tensor cores, 3xTF32:
//   C(i, j) = sum_r A(i, r) B(j, r)
// every fp32 operand x is held as a pair (hi, lo): hi = x rounded to the
// nearest TF32 number, lo = x - hi (exact in fp32, at most 12 significant
// bits, taken to TF32 by the tensor core). Each product is formed as
//   A_lo B_hi + A_hi B_lo + A_hi B_hi
// (the dropped A_lo B_lo term and the TF32 rounding of lo are ~2^-23 of
// |A||B|), on a tensor pipe that runs TF32 at half the bf16 rate.
//
// The tensor core's fp32 accumulation truncates at every MMA, which biases
// long sums (measured: ~1e-5 of sum |terms| after 1024 same-sign terms). So no
// accumulator lives longer than one 32-deep k-block: each block's partial
// product is taken out of TMEM by the epilogue warps and added into fp32
// registers with round-to-nearest, while the next block accumulates in the
// other TMEM buffer.
//
// The three GEMMs of a fully connected layer ("Deep Learning Recommendation
// Model (DLRM)", Key Method Details: FC layers; their gradients by the chain
// rule) differ only in which operand is stored K-major (r contiguous) and
// which MN-major (i or j contiguous); tcgen05 reads TF32 operands in either
// major order, so no transpose is ever materialised:
//   forward  y[b][n]  = relu(sum_k x[b][k] W[n][k] + bias[n])   A = x  (K),  B = W  (K)
//   dgrad    dx[b][k] = mask(b,k) sum_n dy[b][n] W[n][k]        A = dy (K),  B = W  (MN)
//   wgrad    dW[n][k] = sum_b dy[b][n] x[b][k]                  A = dy (MN), B = x  (MN)
// The weight gradient reduces over the batch: it is cut into S fixed
// r-ranges (S depends only on the shape) whose partial tiles are added in a
// fixed order, so results are bit-reproducible run to run.
//
// Kernel: a cluster of two CTAs (an SM pair) computes 256x256 tiles with
// tcgen05.mma.cta_group::2.kind::tf32 (M = 256, N = 256, K = 8); each CTA
// stages its 128 rows of A and its 128 rows of B, hi and lo (64 KB per
// 32-deep k-block, three stages), by TMA with 128-byte swizzle (32-byte
// atoms for MN-major operands); the leader issues 12 MMAs per k-block into
// one of two TMEM buffers; 8 epilogue warps per CTA add each finished block
// into registers (128 fp32 per thread: 32 rows x 128 columns per warp), then
// apply bias/ReLU or the ReLU mask, split the result into its (hi, lo) pair
// and write it by TMA bulk tensor stores.
// Every wait is bounded (timeout -> DLRM_ERR_TIMEOUT in the error record,
// copies and MMAs drained, TMEM freed). No cluster-multicast load is used.
#include <cuda.h>

#include "common.cuh"
#include "kernels.cuh"
#include "tcgen05.cuh"

namespace dlrm {
namespace tc {

constexpr int BR3 = 32;                       // reduction depth of one stage: one 128-byte fp32 row
constexpr int STAGES3 = 3;
constexpr int PART3 = 128 * BR3 * 4;          // one operand part (hi or lo) of one CTA: 16 KB
constexpr int STAGE3_BYTES = 4 * PART3;       // A_hi, A_lo, B_hi, B_lo
constexpr int SMEM3_BYTES = STAGES3 * STAGE3_BYTES + OUT_BYTES + 1024 + 256;
static_assert(SMEM3_BYTES <= 227 * 1024, "shared memory");
constexpr int PAIRS_REF = 74;                 // SM pairs assumed when choosing the split count (shape-only)
// 12 warps: warpgroup 0 = TMA producer (warp 0), MMA issuer and TMEM owner
// (warp 1), two idle warps; warpgroups 1 and 2 = 8 epilogue warps. The block
// launches with 168 registers per thread (64,512 in all); warpgroup 0 gives
// back to 40 and the epilogue warpgroups take 232 each:
// 128 * 40 + 256 * 232 = 64,512.
constexpr int THREADS3 = 384;
constexpr int REGS_LOW = 40, REGS_HIGH = 232;
static_assert(128 * REGS_LOW + 256 * REGS_HIGH <= 168 * THREADS3, "register split exceeds the launch allocation");

enum Epi3 { E3_RELU_PAIR = 0, E3_MASK_PAIR = 1, E3_PLAIN = 2 };

// Epilogue operands (unused ones null).
struct Epi3Args {
    const float* bias;          // E3_RELU_PAIR: bias[J]
    const float* mhi;           // E3_MASK_PAIR without bits: the saved post-ReLU activation pair [I][ldm]
    const float* mlo;
    long long ldm;
    uint32_t* bits_out;         // E3_RELU_PAIR: ReLU bitmask of the output, bit j % 32 of word [i][j / 32]
    const uint32_t* bits_in;    // E3_MASK_PAIR: the saved activation's ReLU bitmask (instead of mhi/mlo)
    long long ldbits;           // words per row of either bitmask
    float* csum;                // E3_MASK_PAIR: column sums of each 32-row group of the output, [I / 32][J]
};

struct Bars3 {
    unsigned long long full[STAGES3];
    unsigned long long empty[STAGES3];
    unsigned long long tfull[2];
    unsigned long long tempty[2];
    unsigned long long drain;
    unsigned int tmem_base;
    int abort;
};

struct Maps3 {
    CUtensorMap a_hi, a_lo, b_hi, b_lo;   // operands
    CUtensorMap c0, c1;                   // output: (hi, lo) pair, or plain in c0; 3D {J, I, S}
};

// MN-major TF32 operand. For 32-bit MN-major operands tcgen05 takes only the
// "128-byte swizzle, 32-byte atom" layout: each k-row is 128 bytes (32
// consecutive M/N elements) whose four 32-byte chunks are permuted by XOR with
// (k-row mod 4); TMA writes it with CU_TENSOR_MAP_SWIZZLE_128B_ATOM_32B.
// Here 4-row groups are 512 bytes apart and 32-wide M/N blocks 4 KB apart.
__device__ __forceinline__ uint64_t sdesc_mn(uint32_t addr) {
    uint64_t d = (uint64_t)((addr & 0x3FFFFu) >> 4);
    d |= (uint64_t)((BR3 * 128) >> 4) << 16;   // leading byte offset: next 32-wide M/N block
    d |= (uint64_t)(512 >> 4) << 32;           // stride byte offset: next 4 k-rows
    d |= (uint64_t)1 << 46;
    d |= (uint64_t)1 << 61;                    // layout: 128-byte swizzle with 32-byte atoms
    return d;
}

// kind::tf32 instruction descriptor, M = 256 (SM pair), N = 256, fp32 accumulate.
__host__ __device__ constexpr uint32_t idesc_tf32(bool a_mn, bool b_mn) {
    return (1u << 4) | (2u << 7) | (2u << 10) | ((uint32_t)a_mn << 15) | ((uint32_t)b_mn << 16) |
           ((uint32_t)(256 >> 3) << 17) | ((uint32_t)(256 >> 4) << 24);
}

__device__ __forceinline__ void umma2_tf32(uint32_t d_tmem, uint64_t a, uint64_t b, uint32_t id, uint32_t accum) {
    asm volatile(
        "{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n tcgen05.mma.cta_group::2.kind::tf32 [%0], %1, %2, %3, p;\n}\n" ::"r"(
            d_tmem),
        "l"(a), "l"(b), "r"(id), "r"(accum));
}

__device__ __forceinline__ void tma_store_3d(const CUtensorMap* map, uint32_t src, int x, int y, int z) {
    asm volatile("cp.async.bulk.tensor.3d.global.shared::cta.bulk_group [%0, {%1, %2, %3}], [%4];" ::"l"(
                     reinterpret_cast<uint64_t>(map)),
                 "r"(x), "r"(y), "r"(z), "r"(src)
                 : "memory");
    asm volatile("cp.async.bulk.commit_group;" ::: "memory");
}

// One operand's hi and lo parts for rows [base, base + 128) and reduction
// columns [r0, r0 + 32): one 128x32 box each when K-major, four 32x32 boxes
// (one per 32-wide block of rows) each when MN-major.
template <bool MN>
__device__ __forceinline__ void load_operand(uint32_t dst, const CUtensorMap* hi, const CUtensorMap* lo,
                                             uint32_t bar, int r0, int base) {
    if constexpr (!MN) {
        tma_load_2d_pair(dst, hi, bar, r0, base);
        tma_load_2d_pair(dst + PART3, lo, bar, r0, base);
    } else {
#pragma unroll
        for (int b = 0; b < 4; ++b) {
            tma_load_2d_pair(dst + b * (BR3 * 128), hi, bar, base + 32 * b, r0);
            tma_load_2d_pair(dst + PART3 + b * (BR3 * 128), lo, bar, base + 32 * b, r0);
        }
    }
}

// hi part of a 3xTF32 pair: v rounded to the nearest TF32 value (ties away
// from zero), so that lo = v - hi is exact and has at most 12 significant bits;
// magnitudes that would round up to infinity are truncated instead.
__device__ __forceinline__ float tf32_hi(float v) {
    const uint32_t u = __float_as_uint(v);
    uint32_t r = u + 0x1000u;
    if ((r & 0x7F800000u) == 0x7F800000u) r = u;
    return __uint_as_float(r & 0xFFFFE000u);
}

// Stage one 32-row x 32-column fp32 chunk (128-byte swizzle) and store it.
__device__ __forceinline__ void stage_store(const float (&v)[32], unsigned char* stage, uint32_t stage_s,
                                           const CUtensorMap* map, int x, int y, int z) {
    const int lane = threadIdx.x & 31;
    if (lane == 0) bulk_wait_read0();   // the previous store has read the staging buffer
    __syncwarp();
    unsigned char* row = stage + lane * 128;
#pragma unroll
    for (int q = 0; q < 8; ++q)
        *reinterpret_cast<uint4*>(row + 16 * (q ^ (lane & 7))) =
            make_uint4(__float_as_uint(v[4 * q]), __float_as_uint(v[4 * q + 1]), __float_as_uint(v[4 * q + 2]),
                       __float_as_uint(v[4 * q + 3]));
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    __syncwarp();
    if (lane == 0) tma_store_3d(map, stage_s, x, y, z);
}

// Lane l ends with the sum over lanes of part[l] (part is consumed): the
// column sums of a warp's 32 rows, a fixed summation tree.
__device__ __forceinline__ float reduce_scatter32(float (&part)[32], int lane) {
#pragma unroll
    for (int w = 16; w >= 1; w >>= 1) {
        const bool upper = (lane & w) != 0;
#pragma unroll
        for (int k = 0; k < w; ++k) {
            const float send = upper ? part[k] : part[k + w];
            const float keep = upper ? part[k + w] : part[k];
            part[k] = keep + __shfl_xor_sync(0xffffffffu, send, w);
        }
    }
    return part[0];
}

// Final epilogue of one warp from its fp32 register accumulator: rows i0 ..
// i0 + 31 (one per lane), columns jb .. jb + 127 (acc[c][e] = column jb + 32c + e).
template <int EPI>
__device__ __forceinline__ void epilogue3(float (&acc)[4][32], int i0, int jb, int I, int J, int z,
                                          const Epi3Args& ea, const CUtensorMap* c0, const CUtensorMap* c1,
                                          unsigned char* stage, uint32_t stage_s) {
    const int lane = threadIdx.x & 31;
    const int i = i0 + lane;
    const float* __restrict__ bias = ea.bias;
    const float* __restrict__ mhi = ea.mhi;
    const float* __restrict__ mlo = ea.mlo;
    const long long ldm = ea.ldm;
    // the saved activation's ReLU bits for this lane's row, one word per 32-column chunk, loaded up front
    uint32_t mbits[4] = {0u, 0u, 0u, 0u};
    if constexpr (EPI == E3_MASK_PAIR) {
        if (ea.bits_in && i < I) {
#pragma unroll
            for (int c = 0; c < 4; ++c)
                if (jb + 32 * c < J) mbits[c] = __ldg(ea.bits_in + (long long)i * ea.ldbits + (jb + 32 * c) / 32);
        }
    }
#pragma unroll
    for (int c = 0; c < 4; ++c) {
        const int j0 = jb + 32 * c;
        if (j0 >= J) break;   // uniform across the warp
        float (&v)[32] = acc[c];
        if constexpr (EPI == E3_RELU_PAIR) {
            if (j0 + 32 <= J) {
                const float4* b4 = reinterpret_cast<const float4*>(bias + j0);
#pragma unroll
                for (int q = 0; q < 8; ++q) {
                    const float4 bq = __ldg(b4 + q);
                    v[4 * q + 0] = fmaxf(v[4 * q + 0] + bq.x, 0.f);
                    v[4 * q + 1] = fmaxf(v[4 * q + 1] + bq.y, 0.f);
                    v[4 * q + 2] = fmaxf(v[4 * q + 2] + bq.z, 0.f);
                    v[4 * q + 3] = fmaxf(v[4 * q + 3] + bq.w, 0.f);
                }
            } else {
#pragma unroll
                for (int e = 0; e < 32; ++e) {
                    const float s = v[e] + ((j0 + e < J) ? __ldg(bias + j0 + e) : 0.f);
                    v[e] = s > 0.f ? s : 0.f;
                }
            }
        }
        if constexpr (EPI == E3_RELU_PAIR) {
            if (ea.bits_out && i < I) {
                uint32_t b = 0u;
#pragma unroll
                for (int e = 0; e < 32; ++e) b |= (v[e] > 0.f ? 1u : 0u) << e;
                ea.bits_out[(long long)i * ea.ldbits + j0 / 32] = b;
            }
        }
        if constexpr (EPI == E3_MASK_PAIR) {
            // ReLU'(pre-activation): 1 where the saved post-ReLU value m = hi + lo is > 0
            if (ea.bits_in) {
#pragma unroll
                for (int e = 0; e < 32; ++e)
                    if (!((mbits[c] >> e) & 1u)) v[e] = 0.f;
            } else if (i < I) {
                const float* h = mhi + (long long)i * ldm + j0;
                const float* l = mlo + (long long)i * ldm + j0;
                if (j0 + 32 <= J) {
#pragma unroll
                    for (int q = 0; q < 8; ++q) {
                        const float4 x = __ldg(reinterpret_cast<const float4*>(h) + q);
                        const float4 y = __ldg(reinterpret_cast<const float4*>(l) + q);
                        if (!(x.x + y.x > 0.f)) v[4 * q + 0] = 0.f;
                        if (!(x.y + y.y > 0.f)) v[4 * q + 1] = 0.f;
                        if (!(x.z + y.z > 0.f)) v[4 * q + 2] = 0.f;
                        if (!(x.w + y.w > 0.f)) v[4 * q + 3] = 0.f;
                    }
                } else {
#pragma unroll
                    for (int e = 0; e < 32; ++e)
                        if (j0 + e < J && !(__ldg(h + e) + __ldg(l + e) > 0.f)) v[e] = 0.f;
                }
            }
        }
        if constexpr (EPI == E3_PLAIN) {
            stage_store(v, stage, stage_s, c0, j0, i0, z);
        } else {
            float w[32];
#pragma unroll
            for (int e = 0; e < 32; ++e) w[e] = tf32_hi(v[e]);
            stage_store(w, stage, stage_s, c0, j0, i0, 0);
#pragma unroll
            for (int e = 0; e < 32; ++e) w[e] = v[e] - w[e];
            stage_store(w, stage, stage_s, c1, j0, i0, 0);
            if constexpr (EPI == E3_MASK_PAIR) {
                if (ea.csum && i0 < I) {   // uniform across the warp; groups wholly beyond I have no slot
                    // rows beyond I hold zeros (their A rows are zero-filled), so they add nothing
                    const float cs = reduce_scatter32(v, lane);
                    if (j0 + lane < J) ea.csum[(long long)(i0 / 32) * J + j0 + lane] = cs;
                }
            }
        }
    }
}

// acc[c] += the 32 TMEM columns at taddr + 32c, c = 0..3
__device__ __forceinline__ void promote(float (&acc)[4][32], uint32_t taddr) {
#pragma unroll
    for (int c = 0; c < 4; ++c) {
        uint32_t r[32];
        tmem_ld32_issue(taddr + 32 * c, r);
        tmem_ld_wait();
#pragma unroll
        for (int e = 0; e < 32; ++e) acc[c][e] += __uint_as_float(r[e]);
    }
}

template <bool AMN, bool BMN, int EPI>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(THREADS3, 1)
    gemm3x_kernel(const __grid_constant__ Maps3 maps, int I, int J, int R, int r_chunk, int S, const Epi3Args ea,
                  ErrRecord* err) {
    pdl_wait();
    extern __shared__ __align__(1024) unsigned char smem_raw[];
    const uint32_t raw = su32(smem_raw);
    const uint32_t base = (raw + 1023u) & ~1023u;
    unsigned char* gbase = smem_raw + (base - raw);
    Bars3* bars = reinterpret_cast<Bars3*>(gbase + STAGES3 * STAGE3_BYTES + OUT_BYTES);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t rank = cluster_rank();
    const bool leader = rank == 0;
    const int npair = gridDim.x >> 1, pair = blockIdx.x >> 1;
    const int nbi = (I + 255) / 256, nbj = (J + 255) / 256;
    const int per_split = nbi * nbj;
    const int ntiles = per_split * S;
    constexpr uint32_t ID = idesc_tf32(AMN, BMN);
    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES3; ++s) {
            mbar_init(&bars->full[s], 1);
            mbar_init(&bars->empty[s], 1);
        }
        for (int a = 0; a < 2; ++a) {
            mbar_init(&bars->tfull[a], 1);
            mbar_init(&bars->tempty[a], 2 * EPI_WARPS);
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
    fence_before();
    cluster_sync_all();
    fence_after();
    const uint32_t tmem = bars->tmem_base;
    volatile int* abort = &bars->abort;
    bool timed_out = false;
    auto tile_of = [&](int t, int& z, int& mb, int& nb, int& rb, int& nk) {
        z = t / per_split;
        const int rem = t - z * per_split;
        mb = rem / nbj;
        nb = rem - mb * nbj;
        rb = z * r_chunk;
        const int re = rb + r_chunk < R ? rb + r_chunk : R;
        nk = (re - rb + BR3 - 1) / BR3;
    };
    if (warp < 4) {
        asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(REGS_LOW));
    if (warp == 0) {
        if (lane == 0) {
            asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&maps.a_hi)) : "memory");
            asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&maps.b_hi)) : "memory");
            int s = 0;
            uint32_t ph = 0;
            for (int t = pair; t < ntiles && !timed_out; t += npair) {
                int z, mb, nb, rb, nk;
                tile_of(t, z, mb, nb, rb, nk);
                for (int kb = 0; kb < nk; ++kb) {
                    if (!mbar_wait(&bars->empty[s], ph ^ 1u, abort)) {
                        timed_out = true;
                        break;
                    }
                    const uint32_t sa = base + s * STAGE3_BYTES;
                    const uint32_t lead_full = map_rank(su32(&bars->full[s]), 0);
                    if (leader) mbar_expect_tx(&bars->full[s], 2 * STAGE3_BYTES);
                    const int r0 = rb + kb * BR3;
                    load_operand<AMN>(sa, &maps.a_hi, &maps.a_lo, lead_full, r0, mb * 256 + (int)rank * 128);
                    load_operand<BMN>(sa + 2 * PART3, &maps.b_hi, &maps.b_lo, lead_full, r0,
                                      nb * 256 + (int)rank * 128);
                    if (++s == STAGES3) {
                        s = 0;
                        ph ^= 1u;
                    }
                }
            }
            if (timed_out) *abort = 1;
            for (int q = 0; q < STAGES3; ++q) {
                mbar_wait(&bars->empty[s], ph ^ 1u, abort, true);
                if (++s == STAGES3) {
                    s = 0;
                    ph ^= 1u;
                }
            }
        }
    } else if (warp == 1) {
        if (lane == 0 && leader) {
            int s = 0;
            uint32_t ph = 0;
            uint32_t blk = 0;   // k-blocks issued so far: block n accumulates in TMEM buffer n & 1
            for (int t = pair; t < ntiles && !timed_out; t += npair) {
                int z, mb, nb, rb, nk;
                tile_of(t, z, mb, nb, rb, nk);
                for (int kb = 0; kb < nk; ++kb, ++blk) {
                    const int acc = (int)(blk & 1u);
                    if (!mbar_wait(&bars->tempty[acc], ((blk >> 1) & 1u) ^ 1u, abort) ||
                        !mbar_wait(&bars->full[s], ph, abort)) {
                        timed_out = true;
                        break;
                    }
                    fence_after();
                    const uint32_t d = tmem + (uint32_t)(acc * 256);
                    const uint32_t sa = base + s * STAGE3_BYTES;
                    const uint32_t sb = sa + 2 * PART3;
#pragma unroll
                    for (int k = 0; k < BR3 / 8; ++k) {
                        const uint32_t ao = AMN ? (uint32_t)(k * 1024) : (uint32_t)(k * 32);
                        const uint32_t bo = BMN ? (uint32_t)(k * 1024) : (uint32_t)(k * 32);
                        const uint64_t a_hi = AMN ? sdesc_mn(sa + ao) : sdesc(sa + ao);
                        const uint64_t a_lo = AMN ? sdesc_mn(sa + PART3 + ao) : sdesc(sa + PART3 + ao);
                        const uint64_t b_hi = BMN ? sdesc_mn(sb + bo) : sdesc(sb + bo);
                        const uint64_t b_lo = BMN ? sdesc_mn(sb + PART3 + bo) : sdesc(sb + PART3 + bo);
                        umma2_tf32(d, a_lo, b_hi, ID, k != 0);
                        umma2_tf32(d, a_hi, b_lo, ID, 1u);
                        umma2_tf32(d, a_hi, b_hi, ID, 1u);
                    }
                    umma2_commit_both(&bars->empty[s]);
                    umma2_commit_both(&bars->tfull[acc]);
                    if (++s == STAGES3) {
                        s = 0;
                        ph ^= 1u;
                    }
                }
            }
            if (timed_out) *abort = 1;
            umma2_commit_both(&bars->drain);
            mbar_wait(&bars->drain, 0, abort, true);
        } else if (lane == 0) {
            mbar_wait(&bars->drain, 0, abort, true);
        }
    }
    } else {
        asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(REGS_HIGH));
        // epilogue warps: every k-block's partial product is added into fp32
        // registers (round to nearest) as soon as its accumulator is complete,
        // so that the tensor core accumulates at most one 32-deep block at a time
        const int ew = warp - 4;
        const int q = warp & 3;
        const int h = ew >> 2;
        unsigned char* stage = gbase + STAGES3 * STAGE3_BYTES + ew * STAGE_OUT_BYTES;
        const uint32_t stage_s = base + STAGES3 * STAGE3_BYTES + ew * STAGE_OUT_BYTES;
        const uint32_t lead_tempty0 = map_rank(su32(&bars->tempty[0]), 0);
        const uint32_t lead_tempty1 = map_rank(su32(&bars->tempty[1]), 0);
        uint32_t blk = 0;
        for (int t = pair; t < ntiles && !timed_out; t += npair) {
            int z, mb, nb, rb, nk;
            tile_of(t, z, mb, nb, rb, nk);
            float acc[4][32];
#pragma unroll
            for (int c = 0; c < 4; ++c)
#pragma unroll
                for (int e = 0; e < 32; ++e) acc[c][e] = 0.f;
            for (int kb = 0; kb < nk; ++kb, ++blk) {
                const int a = (int)(blk & 1u);
                if (!mbar_wait(&bars->tfull[a], (blk >> 1) & 1u, abort)) {
                    timed_out = true;
                    break;
                }
                fence_after();
                promote(acc, tmem + ((uint32_t)(q * 32) << 16) + (uint32_t)(a * 256 + h * 128));
                fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive_cluster(a ? lead_tempty1 : lead_tempty0);
            }
            if (timed_out) break;
            epilogue3<EPI>(acc, mb * 256 + (int)rank * 128 + q * 32, nb * 256 + h * 128, I, J, z, ea, &maps.c0,
                           &maps.c1, stage, stage_s);
        }
        if (timed_out) *abort = 1;
        if (lane == 0) bulk_wait_all0();
    }
    if (timed_out && lane == 0) atomicOr(&err->flags, (unsigned)ERR_TIMEOUT);
    fence_before();
    cluster_sync_all();
    fence_after();
    if (warp == 1) {
        asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(TMEM_COLS));
    }
}

// ------------------------------------------------------------------ host side
namespace {

int sm_count3() {
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

// fp32 operand X stored row-major with leading dimension ld; K-major: X[i][r]
// (inner extent R), MN-major: X[r][i] (inner extent I); swizzle as the operand order requires.
bool operand_map(CUtensorMap* m, const float* p, bool mn, int I, int R, int ld) {
    EncodeTiledFn enc = encode_fn();
    if (!enc) return false;
    const cuuint64_t dims[2] = {(cuuint64_t)(mn ? I : R), (cuuint64_t)(mn ? R : I)};
    const cuuint64_t strides[1] = {(cuuint64_t)ld * 4};
    const cuuint32_t box[2] = {32, (cuuint32_t)(mn ? BR3 : 128)};
    const cuuint32_t estr[2] = {1, 1};
    return enc(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, const_cast<float*>(p), dims, strides, box, estr,
               CU_TENSOR_MAP_INTERLEAVE_NONE, mn ? CU_TENSOR_MAP_SWIZZLE_128B_ATOM_32B : CU_TENSOR_MAP_SWIZZLE_128B,
               CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Output C[z][i][j] (z < S), row stride ld floats, split stride I * ld floats; 32x32 boxes.
bool output_map(CUtensorMap* m, float* p, int I, int J, int ld, int S) {
    EncodeTiledFn enc = encode_fn();
    if (!enc) return false;
    const cuuint64_t dims[3] = {(cuuint64_t)J, (cuuint64_t)I, (cuuint64_t)S};
    const cuuint64_t strides[2] = {(cuuint64_t)ld * 4, (cuuint64_t)ld * 4 * (cuuint64_t)I};
    const cuuint32_t box[3] = {32, 32, 1};
    const cuuint32_t estr[3] = {1, 1, 1};
    return enc(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3, p, dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
               CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_NONE,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <bool AMN, bool BMN, int EPI>
dlrm_status launch3(const Maps3& maps, int I, int J, int R, int r_chunk, int S, const Epi3Args& ea, ErrRecord* err,
                    cudaStream_t st) {
    auto kern = gemm3x_kernel<AMN, BMN, EPI>;
    cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM3_BYTES);
    const long long ntiles = (long long)((I + 255) / 256) * ((J + 255) / 256) * S;
    const int pairs = sm_count3() / 2;
    const int grid = 2 * (int)(ntiles < pairs ? ntiles : pairs);
    (void)launch_pdl(kern, dim3(grid), dim3(THREADS3), (size_t)(SMEM3_BYTES), st, maps, I, J, R, r_chunk, S, ea, err);
    DLRM_LAUNCH_CHECK();
    return DLRM_OK;
}

inline bool al16(const void* p) { return ((uintptr_t)p & 15u) == 0; }

bool pair_ok(F32Pair x) { return x.hi && x.lo && al16(x.hi) && al16(x.lo) && x.ld % 4 == 0 && x.ld > 0; }

}  // namespace
}  // namespace tc

bool tf32x3_supported(int M, int N, int K, F32Pair a, F32Pair b) {
    // the output width must fill a good part of a 256-wide tile
    return M >= 1 && N >= 16 && K >= 1 && tc::pair_ok(a) && tc::pair_ok(b) && tc::encode_fn() != nullptr;
}

dlrm_status tf32x3_fwd(int M, int N, int K, F32Pair x, F32Pair W, const float* bias, float* y_hi, float* y_lo,
                       int ldy, uint32_t* relu_bits, int ldbits, ErrRecord* err, cudaStream_t st) {
    using namespace tc;
    if (!tc::al16(bias) || !tc::al16(y_hi) || !tc::al16(y_lo) || ldy % 4) return DLRM_ERR_UNSUPPORTED;
    Maps3 m;
    if (!operand_map(&m.a_hi, x.hi, false, M, K, x.ld) || !operand_map(&m.a_lo, x.lo, false, M, K, x.ld) ||
        !operand_map(&m.b_hi, W.hi, false, N, K, W.ld) || !operand_map(&m.b_lo, W.lo, false, N, K, W.ld) ||
        !output_map(&m.c0, y_hi, M, N, ldy, 1) || !output_map(&m.c1, y_lo, M, N, ldy, 1))
        return DLRM_ERR_CUDA;
    Epi3Args ea{};
    ea.bias = bias;
    ea.bits_out = relu_bits;
    ea.ldbits = ldbits;
    return launch3<false, false, E3_RELU_PAIR>(m, M, N, K, K, 1, ea, err, st);
}

dlrm_status tf32x3_dgrad(int M, int N, int K, F32Pair dy, F32Pair W, F32Pair mask, const uint32_t* mask_bits,
                         int ldbits, float* dx_hi, float* dx_lo, int lddx, float* csum, ErrRecord* err,
                         cudaStream_t st) {
    // dx[m][k] = sum_n dy[m][n] W[n][k]; masked by (mask.hi + mask.lo > 0) when mask.hi is given
    // (a masked gradient is written as a (hi, lo) pair, an unmasked one plain)
    using namespace tc;
    if (!tc::al16(dx_hi) || lddx % 4 || (dx_lo && !tc::al16(dx_lo))) return DLRM_ERR_UNSUPPORTED;
    if (mask.hi ? (!dx_lo || !tc::pair_ok(mask)) : dx_lo != nullptr) return DLRM_ERR_UNSUPPORTED;
    Maps3 m;
    if (!operand_map(&m.a_hi, dy.hi, false, M, N, dy.ld) || !operand_map(&m.a_lo, dy.lo, false, M, N, dy.ld) ||
        !operand_map(&m.b_hi, W.hi, true, K, N, W.ld) || !operand_map(&m.b_lo, W.lo, true, K, N, W.ld) ||
        !output_map(&m.c0, dx_hi, M, K, lddx, 1) || (dx_lo && !output_map(&m.c1, dx_lo, M, K, lddx, 1)))
        return DLRM_ERR_CUDA;
    if (!dx_lo) m.c1 = m.c0;
    if (mask.hi) {
        Epi3Args ea{};
        ea.mhi = mask.hi;
        ea.mlo = mask.lo;
        ea.ldm = mask.ld;
        ea.bits_in = mask_bits;
        ea.ldbits = ldbits;
        ea.csum = csum;
        return launch3<false, true, E3_MASK_PAIR>(m, M, K, N, N, 1, ea, err, st);
    }
    return launch3<false, true, E3_PLAIN>(m, M, K, N, N, 1, Epi3Args{}, err, st);
}

int tf32x3_wgrad_splits(int N, int K, int M) {
    // the fewest splits that come within reach of the best fill of PAIRS_REF SM pairs; shape-only
    const long long tiles = (long long)((N + 255) / 256) * ((K + 255) / 256);
    const int max_s = M / 512 > 1 ? (M / 512 < 16 ? M / 512 : 16) : 1;
    int best = 1;
    double best_cost = 1e30;
    for (int s = 1; s <= max_s; ++s) {
        const long long waves = (tiles * s + tc::PAIRS_REF - 1) / tc::PAIRS_REF;
        const double cost = (double)waves / s;
        if (cost < best_cost * 0.97) {
            best_cost = cost;
            best = s;
        }
    }
    return best;
}

size_t tf32x3_wgrad_scratch_floats(int N, int K, int M) {
    const int s = tf32x3_wgrad_splits(N, K, M);
    return s > 1 ? (size_t)s * (size_t)N * (size_t)dlrm_ld(K, DLRM_F32) : 0;
}

dlrm_status tf32x3_gemm(int I, int J, int R, F32Pair A, bool a_mn, F32Pair Bm, bool b_mn, float* C, int ldc,
                        float* scratch, ErrRecord* err, cudaStream_t st) {
    // C[i][j] = sum_r A(i, r) B(j, r), fixed-order split over r
    using namespace tc;
    if (!tc::al16(C) || ldc % 4 || !tc::pair_ok(A) || !tc::pair_ok(Bm)) return DLRM_ERR_UNSUPPORTED;
    if (I < 1 || J < 1 || R < 1) return DLRM_ERR_INVALID_ARG;
    int S = tf32x3_wgrad_splits(I, J, R);
    long long chunk = ((long long)R + S - 1) / S;
    chunk = (chunk + BR3 - 1) / BR3 * BR3;
    S = (int)((R + chunk - 1) / chunk);
    const int ldp = dlrm_ld(J, DLRM_F32);
    float* out = S > 1 ? scratch : C;
    const int ldo = S > 1 ? ldp : ldc;
    if (S > 1 && (!scratch || !tc::al16(scratch))) return DLRM_ERR_WORKSPACE;
    Maps3 m;
    if (!operand_map(&m.a_hi, A.hi, a_mn, I, R, A.ld) || !operand_map(&m.a_lo, A.lo, a_mn, I, R, A.ld) ||
        !operand_map(&m.b_hi, Bm.hi, b_mn, J, R, Bm.ld) || !operand_map(&m.b_lo, Bm.lo, b_mn, J, R, Bm.ld) ||
        !output_map(&m.c0, out, I, J, ldo, S))
        return DLRM_ERR_CUDA;
    m.c1 = m.c0;
    dlrm_status r;
    if (a_mn && b_mn)
        r = launch3<true, true, E3_PLAIN>(m, I, J, R, (int)chunk, S, Epi3Args{}, err, st);
    else if (a_mn)
        r = launch3<true, false, E3_PLAIN>(m, I, J, R, (int)chunk, S, Epi3Args{}, err, st);
    else if (b_mn)
        r = launch3<false, true, E3_PLAIN>(m, I, J, R, (int)chunk, S, Epi3Args{}, err, st);
    else
        r = launch3<false, false, E3_PLAIN>(m, I, J, R, (int)chunk, S, Epi3Args{}, err, st);
    if (r || S == 1) return r;
    return launch_split_sum(S, I, J, scratch, ldp, C, ldc, st);
}

dlrm_status tf32x3_wgrad(int M, int N, int K, F32Pair dy, F32Pair x, float* dW, int ldw, float* scratch,
                         ErrRecord* err, cudaStream_t st) {
    // dW[n][k] = sum_m dy[m][n] x[m][k]: both operands MN-major
    return tf32x3_gemm(N, K, M, dy, true, x, true, dW, ldw, scratch, err, st);
}

}  // namespace dlrm
