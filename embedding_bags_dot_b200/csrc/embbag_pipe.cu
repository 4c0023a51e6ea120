// Fused gather + interaction for bf16 tables into a bf16 concat, pipelined per warp (the forward pass of
// bf16 models: the large configuration).
//
// The operation is the fused kernels' (per sample b: pool the K bags into e_1..e_K, "DLRM", briansu.co,
// section 3; write [x_dense, Z_10, Z_20, Z_21, ...] with Z_ij = <X_i, X_j>, j < i, over
// X = [x_dense; e_1..e_K], "DLRM", briansu.co, section 4, equations "Interaction" and "Output").
//
// Persistent: every warp walks its own sequence of samples (b, b + all warps, ...), with no block-wide
// synchronisation after the first one. Per sample the warp keeps one tile in shared memory, rows
//   0 = bf16(x_dense) (hi), 1 = bf16(x_dense - hi) (lo), 2 .. K+1 = e_1 .. e_K,
// padded by one 16-byte chunk (the 8 rows an ldmatrix reads fall in distinct bank groups), and one staged
// concat row (bf16, in rows past K+1 that only reach Gram entries nothing reads). For sample b:
//  1. the bag codes of sample b+1 (lane k: its CSR range and, for a one-row bag, the table row) are
//     loaded, to be used once b's Gram is done;
//  2. empty bags of b become zero rows, bags of several rows are summed in fp32 by lane groups, x_dense is
//     split into its hi and lo rows, while b's one-row bags (issued one step earlier) land in the tile by
//     bulk copy (cp.async.bulk, completing on the warp's mbarrier; the wait is bounded);
//  3. the lower-triangle Gram of the 16 MT padded rows on mma.sync.m16n8k16 (bf16 in, fp32 accumulate);
//  4. the tile is free: the one-row bags of b+1 are issued into it (one bulk copy of the whole row per
//     bag), so that their latency overlaps the rest of b;
//  5. every Z value goes from the accumulators into its concat column d + i(i-1)/2 + j of the staged row;
//     Z_i0 = G[i+1][0] + G[i+1][1] (hi and lo of x_dense, held by the same thread) keeps x_dense's fp32
//     precision; one bulk store (shared -> global) writes the row.
// One-row bf16 bags are exact in the tile, so the one-hot path is accurate to ~2^-16 of the terms.
#include <algorithm>

#include "async_copy.cuh"
#include "common.cuh"
#include "kernels.cuh"

namespace dlrm {

namespace {

using namespace ac;

constexpr int PW = 8;                 // warps per block
constexpr unsigned PFULL = 0xffffffffu;
constexpr uint32_t P_EMPTY = 0xFFFFFFFFu;
constexpr uint32_t P_MULTI = 0xFFFFFFFEu;

__device__ __forceinline__ uint32_t pack2(float lo, float hi) {
    __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t*>(&h);
}

__device__ __forceinline__ void mma16816(float (&c)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%0,%1,%2,%3};"
        : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

__device__ __forceinline__ void store_row_async(void* dst, uint32_t src, uint32_t bytes) {
    asm volatile("cp.async.bulk.global.shared::cta.bulk_group [%0], [%1], %2;" ::"l"(dst), "r"(src), "r"(bytes)
                 : "memory");
    asm volatile("cp.async.bulk.commit_group;" ::: "memory");
}
__device__ __forceinline__ void stores_read_done() { asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory"); }
__device__ __forceinline__ void stores_done() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }

// Bytes of a warp's region: the tile (enough padded rows for the m-tiles and, after row K+1, the staged
// concat row), 16-byte aligned.
__host__ __device__ inline int pipe_rows(int K, int d, int ld, int MT) {
    const int RS = 2 * d + 16;
    const int stage_rows = (2 * ld + RS - 1) / RS;
    return std::max(16 * MT, K + 2 + stage_rows);
}

// The code of bag (k, b): the global row of a one-row bag with a valid index, P_MULTI for several rows,
// P_EMPTY for no row, an out-of-range index or bad offsets (counted).
__device__ __forceinline__ uint32_t bag_code(int k, long long b, int B, const int32_t* __restrict__ offsets,
                                             const int32_t* __restrict__ indices, long long nnz, const TableMeta& tm,
                                             unsigned& oob, unsigned& bad) {
    const long long o = (long long)k * B + b;
    const long long st = offsets[o], en = offsets[o + 1];
    if (st < 0 || en < st || en > nnz) {
        ++bad;
        return P_EMPTY;
    }
    if (en - st == 1) {
        const int idx = __ldg(indices + st);
        if (idx >= 0 && (long long)idx < tm.rows[k]) return (uint32_t)(tm.base[k] + idx);
        ++oob;
        return P_EMPTY;
    }
    return en - st > 1 ? P_MULTI : P_EMPTY;
}

}  // namespace

// MT: m-tiles of 16 rows (16 MT >= K + 2); GL: lanes per row (d = 8 GL); TWO: K > 32 (two bags per lane).
template <int MT, int GL, bool TWO>
__global__ void __launch_bounds__(PW * 32, MT >= 3 ? 2 : 3) embbag_interact_pipe_kernel(
    const __nv_bfloat16* __restrict__ tables, const __grid_constant__ TableMeta tm, int K, int B,
    const int32_t* __restrict__ offsets, const int32_t* __restrict__ indices, long long nnz,
    const float* __restrict__ x_dense, __nv_bfloat16* __restrict__ out, int ld, int warp_bytes, ErrRecord* err) {
    constexpr int d = 8 * GL;
    constexpr int RS = 2 * d + 16;
    constexpr int NTILE = MT * (MT + 1);
    constexpr int NG = 32 / GL;
    extern __shared__ __align__(128) unsigned char smem[];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int P = K * (K + 1) / 2;
    unsigned char* xw = smem + (size_t)warp * warp_bytes;
    const uint32_t xw_s = (uint32_t)__cvta_generic_to_shared(xw);
    __nv_bfloat16* orow = reinterpret_cast<__nv_bfloat16*>(xw + (K + 2) * RS);
    const uint32_t orow_s = xw_s + (uint32_t)((K + 2) * RS);
    const uint32_t bar = (uint32_t)__cvta_generic_to_shared(smem + (size_t)PW * warp_bytes) + 8u * (uint32_t)warp;
    const int gi = lane / GL, g = lane % GL;
    const int gr = lane >> 2, tc = (lane & 3) * 2;
    unsigned oob = 0, bad = 0;
    bool timed_out = false;
    const int first_tries = g_rows_wait_tries;

    if (lane == 0) {
        bar_init(bar);
        fence_proxy_async();
    }
    // zero padding after the last Z: written once, the staged row is reused by every sample
    for (int c = d + P + lane; c < ld; c += 32) orow[c] = __float2bfloat16_rn(0.f);
    __syncwarp();

    const long long nwarps = (long long)gridDim.x * PW;
    long long b = (long long)blockIdx.x * PW + warp;
    if (b >= B) return;
    uint32_t parity = 0;

    // issue the one-row bags of sample bb (codes c0, c1 of this lane's bags) into the tile
    auto issue = [&](uint32_t c0, uint32_t c1) {
        const unsigned long long one = (unsigned long long)__ballot_sync(PFULL, c0 < P_MULTI) |
                                       (TWO ? (unsigned long long)__ballot_sync(PFULL, c1 < P_MULTI) << 32 : 0ull);
        fence_proxy_async();     // this warp's earlier reads of the tile before the copies' writes
        __syncwarp();
        if (lane == 0) bar_expect(bar, (uint32_t)__popcll(one) * (uint32_t)(2 * d));
        __syncwarp();
        if (c0 < P_MULTI) bulk_row(xw_s + (uint32_t)((lane + 2) * RS), tables + (long long)c0 * d, 2 * d, bar);
        if (TWO && c1 < P_MULTI) bulk_row(xw_s + (uint32_t)((lane + 34) * RS), tables + (long long)c1 * d, 2 * d, bar);
    };

    uint32_t c0 = lane < K ? bag_code(lane, b, B, offsets, indices, nnz, tm, oob, bad) : P_EMPTY;
    uint32_t c1 = (TWO && lane + 32 < K) ? bag_code(lane + 32, b, B, offsets, indices, nnz, tm, oob, bad) : P_EMPTY;
    issue(c0, c1);

    for (;;) {
        const long long bn = b + nwarps;
        // 1. next sample's codes, in flight while this sample is finished
        uint32_t n0 = P_EMPTY, n1 = P_EMPTY;
        if (bn < B) {
            if (lane < K) n0 = bag_code(lane, bn, B, offsets, indices, nnz, tm, oob, bad);
            if (TWO && lane + 32 < K) n1 = bag_code(lane + 32, bn, B, offsets, indices, nnz, tm, oob, bad);
        }
        float4 xv[(d + 127) / 128];
#pragma unroll
        for (int q = 0; q < (d + 127) / 128; ++q) {
            const int c = 4 * lane + 128 * q;
            xv[q] = c < d ? *reinterpret_cast<const float4*>(x_dense + b * d + c) : make_float4(0.f, 0.f, 0.f, 0.f);
        }
        // 2. empty bags -> zero rows; several rows -> fp32 sums rounded to bf16 (NG bags at a time)
        const unsigned long long multi = (unsigned long long)__ballot_sync(PFULL, c0 == P_MULTI) |
                                         (TWO ? (unsigned long long)__ballot_sync(PFULL, c1 == P_MULTI) << 32 : 0ull);
        const unsigned long long empty = (unsigned long long)__ballot_sync(PFULL, lane < K && c0 == P_EMPTY) |
                                         (TWO ? (unsigned long long)__ballot_sync(PFULL, lane + 32 < K && c1 == P_EMPTY) << 32
                                              : 0ull);
        for (unsigned long long rest = empty | multi; rest; rest = drop_bits(rest, NG)) {
            const int k = nth_bit(rest, gi);
            if (k < 0) continue;
            uint4 w = make_uint4(0, 0, 0, 0);
            if ((multi >> k) & 1ull) {
                const long long o = (long long)k * B + b;
                const int st = offsets[o], en = offsets[o + 1];
                float a[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
                for (int p = st; p < en; ++p) {
                    const int idx = __ldg(indices + p);
                    if (idx >= 0 && (long long)idx < tm.rows[k])
                        Chunk16<__nv_bfloat16>::add(ldg16_stream(tables + (tm.base[k] + idx) * (long long)d + 8 * g), a);
                    else if (g == 0)
                        ++oob;
                }
                w = make_uint4(pack2(a[0], a[1]), pack2(a[2], a[3]), pack2(a[4], a[5]), pack2(a[6], a[7]));
            }
            *reinterpret_cast<uint4*>(xw + (k + 2) * RS + 16 * g) = w;
        }
        // x_dense -> rows 0 (hi) and 1 (lo)
#pragma unroll
        for (int q = 0; q < (d + 127) / 128; ++q) {
            const int c = 4 * lane + 128 * q;
            if (c < d) {
                const float4 x = xv[q];
                const __nv_bfloat162 h01 = __floats2bfloat162_rn(x.x, x.y), h23 = __floats2bfloat162_rn(x.z, x.w);
                const float2 f01 = __bfloat1622float2(h01), f23 = __bfloat1622float2(h23);
                *reinterpret_cast<uint2*>(xw + 2 * c) =
                    make_uint2(*reinterpret_cast<const uint32_t*>(&h01), *reinterpret_cast<const uint32_t*>(&h23));
                *reinterpret_cast<uint2*>(xw + RS + 2 * c) =
                    make_uint2(pack2(x.x - f01.x, x.y - f01.y), pack2(x.z - f23.x, x.w - f23.y));
            }
        }
        if (!rows_ready(bar, parity, first_tries)) {   // rows landed (drained): stop this warp's samples
            timed_out = true;
            break;
        }
        parity ^= 1u;
        __syncwarp();

        // 3. lower-triangle Gram tiles
        float acc[NTILE][4];
#pragma unroll
        for (int t = 0; t < NTILE; ++t) acc[t][0] = acc[t][1] = acc[t][2] = acc[t][3] = 0.f;
#pragma unroll
        for (int ks = 0; ks < d / 16; ++ks) {
            uint32_t a[MT][4];
#pragma unroll
            for (int mt = 0; mt < MT; ++mt)
                ldmatrix_x4(xw_s + (uint32_t)((16 * mt + (lane & 15)) * RS + 16 * (2 * ks + (lane >> 4))), a[mt]);
            int t = 0;
#pragma unroll
            for (int mt = 0; mt < MT; ++mt) {
#pragma unroll
                for (int nt = 0; nt <= 2 * mt + 1; ++nt, ++t)
                    mma16816(acc[t], a[mt], a[nt >> 1][(nt & 1) ? 1 : 0], a[nt >> 1][(nt & 1) ? 3 : 2]);
            }
        }
        __syncwarp();   // every lane's ldmatrix of the tile is done

        // 4. the next sample's one-row bags into the tile (the staged row is past row K+1, untouched)
        if (bn < B) issue(n0, n1);

        // 5. staged concat row: x_dense, then every Z from the accumulators; one bulk store
        if (lane == 0) stores_read_done();   // the previous sample's row has left the staging area
        __syncwarp();
#pragma unroll
        for (int q = 0; q < (d + 127) / 128; ++q) {
            const int c = 4 * lane + 128 * q;
            if (c < d) {
                const float4 x = xv[q];
                *reinterpret_cast<uint2*>(orow + c) = make_uint2(pack2(x.x, x.y), pack2(x.z, x.w));
            }
        }
        {
            int t = 0;
#pragma unroll
            for (int mt = 0; mt < MT; ++mt) {
#pragma unroll
                for (int nt = 0; nt <= 2 * mt + 1; ++nt, ++t) {
#pragma unroll
                    for (int h = 0; h < 2; ++h) {
                        const int r = 16 * mt + gr + 8 * h;          // tile row: e_{r-1}
                        if (r < 2 || r > K + 1) continue;
                        const int i = r - 1;
                        const int base = d + i * (i - 1) / 2;        // concat column of Z_i0
                        const int c = 8 * nt + tc;                   // tile columns c, c + 1
                        if (c == 0) {
                            orow[base] = __float2bfloat16_rn(acc[t][2 * h] + acc[t][2 * h + 1]);
                        } else {
                            if (c < r) orow[base + c - 1] = __float2bfloat16_rn(acc[t][2 * h]);
                            if (c + 1 < r) orow[base + c] = __float2bfloat16_rn(acc[t][2 * h + 1]);
                        }
                    }
                }
            }
        }
        fence_proxy_async();   // the staged row's generic writes before the bulk store reads it
        __syncwarp();
        if (lane == 0) store_row_async(out + b * ld, orow_s, (uint32_t)(2 * ld));
        if (bn >= B) break;
        b = bn;
        c0 = n0;
        c1 = n1;
    }
    if (lane == 0) stores_done();
    if (timed_out && lane == 0) atomicOr(&err->flags, ERR_TIMEOUT);
    report_warp(err, oob, bad);
}

// ------------------------------------------------------------------ host side

static int pipe_warp_bytes(int K, int d, int ld) {
    const int MT = (K + 2 + 15) / 16;
    return (pipe_rows(K, d, ld, MT) * (2 * d + 16) + 15) & ~15;
}

static size_t pipe_smem(int K, int d, int ld) { return (size_t)PW * pipe_warp_bytes(K, d, ld) + 8 * PW; }

bool embbag_interact_pipe_supported(dlrm_dtype dt, int K, int d, int ld, const void* out, dlrm_dtype out_dt,
                                    long long total_rows) {
    if (dt != DLRM_BF16 || out_dt != DLRM_BF16) return false;
    if (!(d == 32 || d == 64 || d == 128 || d == 256)) return false;
    if (K < 1 || K + 2 > 64) return false;
    if (total_rows >= (long long)P_MULTI) return false;
    if (ld % 8 || ((uintptr_t)out & 15) || ld < d + K * (K + 1) / 2) return false;
    return pipe_smem(K, d, ld) <= 227 * 1024;
}

template <int MT, int GL, bool TWO>
static void launch_pipe_t(const TableMeta& tm, const void* tables, int K, int B, const int32_t* offsets,
                          const int32_t* indices, long long nnz, const float* x_dense, void* out, int ld, int wb,
                          size_t smem, ErrRecord* err, cudaStream_t st) {
    auto kern = embbag_interact_pipe_kernel<MT, GL, TWO>;
    cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    int per_sm = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, PW * 32, smem) != cudaSuccess || per_sm < 1)
        per_sm = 1;
    int sms = 148;
    int dev = 0;
    if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const long long need = ((long long)B + PW - 1) / PW;
    const int grid = (int)std::min<long long>(need, (long long)sms * per_sm);
    kern<<<grid, PW * 32, smem, st>>>(static_cast<const __nv_bfloat16*>(tables), tm, K, B, offsets, indices, nnz,
                                      x_dense, static_cast<__nv_bfloat16*>(out), ld, wb, err);
}

dlrm_status launch_embbag_interact_pipe(const TableMeta& tm, const void* tables, int K, int d, int B,
                                        const int32_t* offsets, const int32_t* indices, long long nnz,
                                        const float* x_dense, void* out, int ld, ErrRecord* err, cudaStream_t st) {
    if (B == 0) return DLRM_OK;
    const int MT = (K + 2 + 15) / 16;
    const int wb = pipe_warp_bytes(K, d, ld);
    const size_t smem = pipe_smem(K, d, ld);
    const bool two = K > 32;
#define DLRM_PIPE(MTV, TWOV)                                                                                     \
    switch (d) {                                                                                                 \
        case 32: launch_pipe_t<MTV, 4, TWOV>(tm, tables, K, B, offsets, indices, nnz, x_dense, out, ld, wb, smem, err, st); break;  \
        case 64: launch_pipe_t<MTV, 8, TWOV>(tm, tables, K, B, offsets, indices, nnz, x_dense, out, ld, wb, smem, err, st); break;  \
        case 128: launch_pipe_t<MTV, 16, TWOV>(tm, tables, K, B, offsets, indices, nnz, x_dense, out, ld, wb, smem, err, st); break; \
        default: launch_pipe_t<MTV, 32, TWOV>(tm, tables, K, B, offsets, indices, nnz, x_dense, out, ld, wb, smem, err, st); break;  \
    }
    switch (MT) {
        case 1: DLRM_PIPE(1, false) break;
        case 2: DLRM_PIPE(2, false) break;
        case 3: if (two) { DLRM_PIPE(3, true) } else { DLRM_PIPE(3, false) } break;
        default: DLRM_PIPE(4, true) break;
    }
#undef DLRM_PIPE
    DLRM_LAUNCH_CHECK();
    return DLRM_OK;
}

cudaError_t set_wait_polls_embbag_pipe(long long polls) {
    return ac::set_rows_wait_tries_here(polls < 0 ? -1 : (int)(polls < ac::WAIT_TRIES ? polls : ac::WAIT_TRIES));
}

}  // namespace dlrm
