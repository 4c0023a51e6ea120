// Three fully connected layers in one tensor-core kernel, for the bottom MLP of
// DLRM ("Deep Learning Recommendation Model (DLRM)", nadeemcite summary, Key
// Method Details: the dense features go through FC layers with ReLU):
//   h1 = relu(x W1^T + b1), h2 = relu(h1 W2^T + b2), y = relu(h2 W3^T + b3)
// with x fp32 [M][n0 <= 16] (rounded to bf16, as the layer-by-layer path does),
// bf16 weights, h1 and h2 rounded to bf16, fp32 accumulation and fp32 output.
//
// The layer-by-layer path writes h1 (n1 wide) and h2 to HBM and reads them
// back; at M = 65536 that is 200 MB of traffic for 22 GFLOP. Here a 128-row
// tile never leaves the SM:
//   warp 0      TMA producer: W1 once (n1 x 16, 32-byte swizzle, resident),
//               then per tile the 64-deep k-blocks of W2 and of W3 through a
//               4-stage ring (128-byte swizzle);
//   warp 1      allocates the 512 TMEM columns and one thread issues the MMAs;
//   warps 2..9  epilogue (two warps per TMEM lane quadrant, half the columns
//               each): x -> bf16 tile, and every accumulator -> bias, ReLU ->
//               the next layer's operand in shared memory or the fp32 output.
// Layer 1 runs in 64-column chunks: chunk j of h1 is exactly k-block j of
// layer 2's A operand. The MMA thread keeps layer 1 LAG chunks ahead of layer
// 2 (M=128, N=64, K=16 into one of four TMEM slots), so the epilogue's work on
// a chunk overlaps the layer-2 MMAs of the chunks before it. The four 16 KB
// slots of the operand ring hold the h1 chunks, then, once layer 2 is done,
// the k-blocks of h2 for layer 3.
// TMEM: layer-2 accumulator [0, 256), whose first n3 columns then hold the
// layer-3 accumulator; layer-1 slots [256, 512). Biases sit in shared memory.
// All waits are bounded: on timeout the kernel records DLRM_ERR_TIMEOUT,
// drains its own copies and MMAs, frees TMEM and returns.
#include <cuda.h>

#include "common.cuh"
#include "kernels.cuh"
#include "tcgen05.cuh"

namespace dlrm {
namespace tc {
namespace {

constexpr int M3_THREADS = 64 + 32 * EPI_WARPS;
constexpr int SLOTS = 4;                               // layer-1 TMEM slots and operand-ring tiles
constexpr int LAG = 3;                                 // layer-1 chunks issued ahead of layer 2
constexpr int W_STAGES = 4;
constexpr int W_STAGE_BYTES = 256 * BK * 2;            // one k-block of up to 256 weight rows
constexpr int TILE_BYTES = BM * BK * 2;                // one 128 x 64 bf16 operand tile
constexpr int OFF_W1 = 0;                              // n1 / 64 chunks of 64 rows x 32 bytes
constexpr int OFF_X0 = 16 * 1024;                      // 128 x 32-byte tile
constexpr int OFF_BIAS = 20 * 1024;                    // b1 | b2 | b3, up to 896 floats
constexpr int OFF_ACT = 24 * 1024;                     // SLOTS operand tiles (h1 chunks, then h2)
constexpr int OFF_WR = OFF_ACT + SLOTS * TILE_BYTES;   // weight ring
constexpr int OFF_BARS = OFF_WR + W_STAGES * W_STAGE_BYTES;
constexpr int M3_SMEM = OFF_BARS + 512 + 1024;
constexpr uint32_t COL_ACC = 0, COL_A1 = 256;
static_assert(M3_SMEM <= 227 * 1024, "shared memory of the fused MLP");

struct Bars3 {
    unsigned long long wfull[W_STAGES], wempty[W_STAGES];
    unsigned long long w1full, x0full, x0empty;
    unsigned long long a1full[SLOTS], a1empty[SLOTS];   // layer-1 TMEM slots
    unsigned long long s1full[SLOTS], s1empty[SLOTS];   // h1 chunk tiles in the operand ring
    unsigned long long acc2full, s2full, s2empty, acc3full, acc3empty;
    unsigned long long drain;
    unsigned int tmem_base;
    int abort;
};
static_assert(sizeof(Bars3) <= 512, "barrier block");

static __device__ long long g_mlp3_wait_polls = WAIT_LIMIT;

// K-major operand with 32-byte swizzle (rows of 16 bf16): 8-row groups of 256 bytes.
__device__ __forceinline__ uint64_t sdesc32(uint32_t addr) {
    uint64_t d = (uint64_t)((addr & 0x3FFFFu) >> 4);
    d |= (uint64_t)1 << 16;
    d |= (uint64_t)(256 >> 4) << 32;
    d |= (uint64_t)1 << 46;
    d |= (uint64_t)6 << 61;
    return d;
}

__host__ __device__ constexpr uint32_t idesc_mn(int m, int n) {
    return (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(n >> 3) << 17) | ((uint32_t)(m >> 4) << 24);
}

__device__ __forceinline__ uint32_t pack2(float a, float b) {
    __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
    return *reinterpret_cast<uint32_t*>(&h);
}

// 32 accumulator columns of one row + bias (shared memory), ReLU, rounded to bf16 and stored as four 16-byte
// chunks of a 128-byte swizzled K-major row (chunk index kc0 .. kc0 + 3 of the row's 8).
__device__ __forceinline__ void store_bf16_chunks(const uint32_t (&r)[32], const float* bias, unsigned char* row,
                                                  int kc0, int rsw) {
#pragma unroll
    for (int p = 0; p < 4; ++p) {
        const float4 b0 = reinterpret_cast<const float4*>(bias)[2 * p];
        const float4 b1 = reinterpret_cast<const float4*>(bias)[2 * p + 1];
        const float* v = reinterpret_cast<const float*>(r) + 8 * p;
        uint4 w;
        w.x = pack2(fmaxf(v[0] + b0.x, 0.f), fmaxf(v[1] + b0.y, 0.f));
        w.y = pack2(fmaxf(v[2] + b0.z, 0.f), fmaxf(v[3] + b0.w, 0.f));
        w.z = pack2(fmaxf(v[4] + b1.x, 0.f), fmaxf(v[5] + b1.y, 0.f));
        w.w = pack2(fmaxf(v[6] + b1.z, 0.f), fmaxf(v[7] + b1.w, 0.f));
        *reinterpret_cast<uint4*>(row + 16 * ((kc0 + p) ^ rsw)) = w;
    }
}

// Uses of slot s per tile (chunks j < nc1 with j % SLOTS == s) and the global use count of chunk j of tile i.
__device__ __forceinline__ uint32_t slot_use(int i, int j, int nc1) {
    const int s = j % SLOTS;
    const int per = (nc1 - s + SLOTS - 1) / SLOTS;
    return (uint32_t)(i * per + j / SLOTS);
}

__global__ void __launch_bounds__(M3_THREADS, 1)
    mlp3_tc_kernel(const __grid_constant__ CUtensorMap mapW1, const __grid_constant__ CUtensorMap mapW2,
                   const __grid_constant__ CUtensorMap mapW3, const float* __restrict__ x, int ldx, int n0, int M,
                   int n1, int n2, int n3, const float* __restrict__ b1, const float* __restrict__ b2,
                   const float* __restrict__ b3, float* __restrict__ out, int ldo, ErrRecord* err) {
    extern __shared__ __align__(1024) unsigned char smem_raw[];
    const uint32_t raw = su32(smem_raw);
    const uint32_t base = (raw + 1023u) & ~1023u;
    unsigned char* g = smem_raw + (base - raw);
    Bars3* bars = reinterpret_cast<Bars3*>(g + OFF_BARS);
    float* bias_s = reinterpret_cast<float*>(g + OFF_BIAS);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int ntiles = (M + BM - 1) / BM;
    const int nc1 = n1 / 64, nk3 = n2 / 64;

    if (threadIdx.x == 0) {
        for (int s = 0; s < W_STAGES; ++s) {
            mbar_init(&bars->wfull[s], 1);
            mbar_init(&bars->wempty[s], 1);
        }
        mbar_init(&bars->w1full, 1);
        mbar_init(&bars->x0full, 4);
        mbar_init(&bars->x0empty, 1);
        for (int a = 0; a < SLOTS; ++a) {
            mbar_init(&bars->a1full[a], 1);
            mbar_init(&bars->a1empty[a], EPI_WARPS);
            mbar_init(&bars->s1full[a], EPI_WARPS);
            mbar_init(&bars->s1empty[a], 1);
        }
        mbar_init(&bars->acc2full, 1);
        mbar_init(&bars->s2full, EPI_WARPS);
        mbar_init(&bars->s2empty, 1);
        mbar_init(&bars->acc3full, 1);
        mbar_init(&bars->acc3empty, EPI_WARPS);
        mbar_init(&bars->drain, 1);
        bars->abort = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    for (int c = threadIdx.x; c < n1 + n2 + n3; c += blockDim.x)
        bias_s[c] = c < n1 ? __ldg(b1 + c) : c < n1 + n2 ? __ldg(b2 + c - n1) : __ldg(b3 + c - n1 - n2);
    if (warp == 1) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(su32(&bars->tmem_base)),
                     "r"(512));
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
    }
    fence_before();
    __syncthreads();
    fence_after();
    const uint32_t tmem = bars->tmem_base;
    volatile int* abort = &bars->abort;
    bool timed_out = false;
    const long long lim = g_mlp3_wait_polls;

    if (warp == 0) {
        if (lane == 0) {
            asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&mapW2)) : "memory");
            asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&mapW3)) : "memory");
            const bool any = (int)blockIdx.x < ntiles;
            if (any) {
                mbar_expect_tx(&bars->w1full, (uint32_t)(nc1 * 64 * 32));
                for (int j = 0; j < nc1; ++j) tma_load_2d(base + OFF_W1 + j * 2048, &mapW1, &bars->w1full, 0, 64 * j);
            }
            int s = 0;
            uint32_t ph = 0;
            for (int t = blockIdx.x; t < ntiles && !timed_out; t += gridDim.x) {
                for (int kb = 0; kb < nc1 + nk3; ++kb) {
                    if (!mbar_wait_n(&bars->wempty[s], ph ^ 1u, abort, lim)) {
                        timed_out = true;
                        break;
                    }
                    const bool l2 = kb < nc1;
                    mbar_expect_tx(&bars->wfull[s], (uint32_t)((l2 ? n2 : n3) * BK * 2));
                    tma_load_2d(base + OFF_WR + s * W_STAGE_BYTES, l2 ? &mapW2 : &mapW3, &bars->wfull[s],
                                (l2 ? kb : kb - nc1) * BK, 0);
                    if (++s == W_STAGES) {
                        s = 0;
                        ph ^= 1u;
                    }
                }
            }
            if (timed_out) *abort = 1;
            // drain: every copy this thread issued lands before the CTA may exit (a stage never
            // filled passes at once)
            if (any) mbar_wait(&bars->w1full, 0, abort, true);
            for (int q = 0; q < W_STAGES; ++q) {
                if (--s < 0) {
                    s = W_STAGES - 1;
                    ph ^= 1u;
                }
                mbar_wait(&bars->wfull[s], ph, abort, true);
            }
        }
    } else if (warp == 1) {
        if (lane == 0) {
            const uint32_t id1 = idesc_mn(BM, 64), id2 = idesc_mn(BM, n2), id3 = idesc_mn(BM, n3);
            int ws = 0;
            uint32_t wph = 0;
            if ((int)blockIdx.x < ntiles && !mbar_wait_n(&bars->w1full, 0, abort, lim)) timed_out = true;
            int i = 0;
            for (int t = blockIdx.x; t < ntiles && !timed_out; t += gridDim.x, ++i) {
                const uint32_t ip = (uint32_t)i & 1u;
                if (!mbar_wait_n(&bars->x0full, ip, abort, lim)) {
                    timed_out = true;
                    break;
                }
                for (int jj = 0; jj < nc1 + LAG && !timed_out; ++jj) {
                    if (jj < nc1) {   // layer 1, chunk jj -> TMEM slot jj % SLOTS
                        const int sl = jj % SLOTS;
                        const uint32_t u = slot_use(i, jj, nc1);
                        if (!mbar_wait_n(&bars->a1empty[sl], (u & 1u) ^ 1u, abort, lim)) {
                            timed_out = true;
                            break;
                        }
                        fence_after();
                        umma(tmem + COL_A1 + 64 * sl, sdesc32(base + OFF_X0), sdesc32(base + OFF_W1 + jj * 2048), id1, 0);
                        umma_commit(&bars->a1full[sl]);
                        if (jj == nc1 - 1) umma_commit(&bars->x0empty);
                    }
                    if (jj >= LAG) {   // layer 2, k-block j = h1 chunk j (operand slot j % SLOTS)
                        const int j = jj - LAG, sl = j % SLOTS;
                        const uint32_t u = slot_use(i, j, nc1);
                        if (j == 0 && !mbar_wait_n(&bars->acc3empty, ip ^ 1u, abort, lim)) {
                            timed_out = true;
                            break;
                        }
                        if (!mbar_wait_n(&bars->s1full[sl], u & 1u, abort, lim) ||
                            !mbar_wait_n(&bars->wfull[ws], wph, abort, lim)) {
                            timed_out = true;
                            break;
                        }
                        fence_after();
                        const uint32_t a = base + OFF_ACT + sl * TILE_BYTES, w = base + OFF_WR + ws * W_STAGE_BYTES;
#pragma unroll
                        for (int k = 0; k < BK / 16; ++k)
                            umma(tmem + COL_ACC, sdesc(a + k * 32), sdesc(w + k * 32), id2, (j | k) != 0);
                        umma_commit(&bars->wempty[ws]);
                        umma_commit(&bars->s1empty[sl]);
                        if (++ws == W_STAGES) {
                            ws = 0;
                            wph ^= 1u;
                        }
                    }
                }
                if (timed_out) break;
                umma_commit(&bars->acc2full);
                // layer 3 on h2 (operand slots 0 .. n2/64 - 1), accumulator in the first n3 columns
                if (!mbar_wait_n(&bars->s2full, ip, abort, lim)) {
                    timed_out = true;
                    break;
                }
                fence_after();
                for (int kb = 0; kb < nk3; ++kb) {
                    if (!mbar_wait_n(&bars->wfull[ws], wph, abort, lim)) {
                        timed_out = true;
                        break;
                    }
                    fence_after();
                    const uint32_t a = base + OFF_ACT + kb * TILE_BYTES, w = base + OFF_WR + ws * W_STAGE_BYTES;
#pragma unroll
                    for (int k = 0; k < BK / 16; ++k)
                        umma(tmem + COL_ACC, sdesc(a + k * 32), sdesc(w + k * 32), id3, (kb | k) != 0);
                    umma_commit(&bars->wempty[ws]);
                    if (++ws == W_STAGES) {
                        ws = 0;
                        wph ^= 1u;
                    }
                }
                if (timed_out) break;
                umma_commit(&bars->acc3full);
                umma_commit(&bars->s2empty);
            }
            if (timed_out) *abort = 1;
            umma_commit(&bars->drain);
            mbar_wait(&bars->drain, 0, abort, true);
        }
    } else {
        const int ew = warp - 2;
        const int q = warp & 3;                  // TMEM lane quadrant
        const int h = ew >> 2;                   // half of the columns
        const int r = q * 32 + lane;             // row of the tile
        const int rsw = r & 7;                   // 128-byte swizzle phase of the row
        const uint32_t lanes = (uint32_t)(q * 32) << 16;
        const float* bs1 = bias_s;
        const float* bs2 = bias_s + n1;
        const float* bs3 = bias_s + n1 + n2;
        // x rows of a tile, loaded one tile ahead by the first warp of each quadrant
        float xr[16];
        auto load_x = [&](int t) {
            const long long row = (long long)t * BM + r;
#pragma unroll
            for (int k = 0; k < 16; ++k) xr[k] = (row < M && k < n0) ? __ldg(x + row * ldx + k) : 0.f;
        };
        // x (registers) -> bf16, row r of the 32-byte swizzled tile
        auto store_x = [&]() {
            unsigned char* dst = g + OFF_X0 + r * 32;
            const int sw = (r >> 2) & 1;
            *reinterpret_cast<uint4*>(dst + 16 * (0 ^ sw)) =
                make_uint4(pack2(xr[0], xr[1]), pack2(xr[2], xr[3]), pack2(xr[4], xr[5]), pack2(xr[6], xr[7]));
            *reinterpret_cast<uint4*>(dst + 16 * (1 ^ sw)) =
                make_uint4(pack2(xr[8], xr[9]), pack2(xr[10], xr[11]), pack2(xr[12], xr[13]), pack2(xr[14], xr[15]));
            asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
            __syncwarp();
            if (lane == 0) mbar_arrive(&bars->x0full);
        };
        if (h == 0 && (int)blockIdx.x < ntiles) {
            load_x(blockIdx.x);
            store_x();
            if ((int)(blockIdx.x + gridDim.x) < ntiles) load_x(blockIdx.x + gridDim.x);
        }
        int i = 0;
        for (int t = blockIdx.x; t < ntiles && !timed_out; t += gridDim.x, ++i) {
            const uint32_t ip = (uint32_t)i & 1u;
            // layer-1 chunks -> h1 tiles in the operand ring
            for (int j = 0; j < nc1; ++j) {
                const int sl = j % SLOTS;
                const uint32_t u = slot_use(i, j, nc1);
                if (!mbar_wait_n(&bars->a1full[sl], u & 1u, abort, lim)) {
                    timed_out = true;
                    break;
                }
                fence_after();
                uint32_t acc[32];
                tmem_ld32_issue(tmem + lanes + COL_A1 + 64 * sl + 32 * h, acc);
                tmem_ld_wait();
                fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&bars->a1empty[sl]);
                // the slot's previous reader: layer 2 on chunk j - SLOTS of this tile, else the last tile's layer 3
                const bool ok = j >= SLOTS ? mbar_wait_n(&bars->s1empty[sl], (u & 1u) ^ 1u, abort, lim)
                                           : mbar_wait_n(&bars->s2empty, ip ^ 1u, abort, lim);
                if (!ok) {
                    timed_out = true;
                    break;
                }
                store_bf16_chunks(acc, bs1 + 64 * j + 32 * h, g + OFF_ACT + sl * TILE_BYTES + r * 128, 4 * h, rsw);
                asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
                __syncwarp();
                if (lane == 0) mbar_arrive(&bars->s1full[sl]);
            }
            if (timed_out) break;
            // the next tile's x, once this tile's layer 1 has read the x tile
            if (h == 0 && t + (int)gridDim.x < ntiles) {
                if (!mbar_wait_n(&bars->x0empty, ip, abort, lim)) {
                    timed_out = true;
                    break;
                }
                store_x();
                if (t + 2 * (int)gridDim.x < ntiles) load_x(t + 2 * gridDim.x);
            }
            // layer-2 accumulator -> h2 tiles (layer 2 has finished reading the ring)
            if (!mbar_wait_n(&bars->acc2full, ip, abort, lim)) {
                timed_out = true;
                break;
            }
            fence_after();
            for (int cb = 0; cb < n2 / 64; ++cb) {
                const int col = h * (n2 / 2) + 32 * cb;
                uint32_t acc[32];
                tmem_ld32_issue(tmem + lanes + COL_ACC + col, acc);
                tmem_ld_wait();
                store_bf16_chunks(acc, bs2 + col, g + OFF_ACT + (col / 64) * TILE_BYTES + r * 128, (col % 64) / 8,
                                  rsw);
            }
            fence_before();
            asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
            __syncwarp();
            if (lane == 0) mbar_arrive(&bars->s2full);
            // layer-3 accumulator -> fp32 output rows
            if (!mbar_wait_n(&bars->acc3full, ip, abort, lim)) {
                timed_out = true;
                break;
            }
            fence_after();
            const long long row = (long long)t * BM + r;
            for (int cb = 0; cb < n3 / 64; ++cb) {
                const int col = h * (n3 / 2) + 32 * cb;
                uint32_t acc[32];
                tmem_ld32_issue(tmem + lanes + COL_ACC + col, acc);
                tmem_ld_wait();
                if (row < M) {
                    float4* o = reinterpret_cast<float4*>(out + row * ldo + col);
                    const float4* bb4 = reinterpret_cast<const float4*>(bs3 + col);
#pragma unroll
                    for (int p = 0; p < 8; ++p) {
                        const float4 bb = bb4[p];
                        o[p] = make_float4(fmaxf(__uint_as_float(acc[4 * p]) + bb.x, 0.f),
                                           fmaxf(__uint_as_float(acc[4 * p + 1]) + bb.y, 0.f),
                                           fmaxf(__uint_as_float(acc[4 * p + 2]) + bb.z, 0.f),
                                           fmaxf(__uint_as_float(acc[4 * p + 3]) + bb.w, 0.f));
                    }
                }
            }
            fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&bars->acc3empty);
        }
        if (timed_out) *abort = 1;
    }

    if (timed_out && lane == 0) atomicOr(&err->flags, (unsigned)ERR_TIMEOUT);
    fence_before();
    __syncthreads();
    fence_after();
    if (warp == 1) asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(512));
}

bool make_map_sw(CUtensorMap* map, const void* ptr, int inner, int outer, int ld, int box_inner, int box_outer,
                 CUtensorMapSwizzle sw) {
    EncodeTiledFn enc = encode_fn();
    if (!enc) return false;
    const cuuint64_t dims[2] = {(cuuint64_t)inner, (cuuint64_t)outer};
    const cuuint64_t strides[1] = {(cuuint64_t)ld * 2};
    const cuuint32_t box[2] = {(cuuint32_t)box_inner, (cuuint32_t)box_outer};
    const cuuint32_t estr[2] = {1, 1};
    return enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(ptr), dims, strides, box, estr,
               CU_TENSOR_MAP_INTERLEAVE_NONE, sw, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

int sm_count_here() {
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

}  // namespace
}  // namespace tc

cudaError_t set_wait_polls_mlp3(long long polls) {
    const long long v = polls < 0 ? tc::WAIT_LIMIT : polls;
    return cudaMemcpyToSymbol(tc::g_mlp3_wait_polls, &v, sizeof(v));
}

bool mlp3_tc_supported(const dlrm_mlp* m, int B, dlrm_dtype in_dt, int ld_in, const void* out, int ld_out,
                       int final_act) {
    if (!m || m->n_layers != 3 || m->dt != DLRM_BF16 || in_dt != DLRM_F32 || final_act != DLRM_ACT_RELU) return false;
    const int n0 = m->dims[0], n1 = m->dims[1], n2 = m->dims[2], n3 = m->dims[3];
    if (B < 1 || n0 < 1 || n0 > 16 || ld_in < n0) return false;
    if (n1 % 64 || n1 > 512 || n2 % 64 || n2 > 256 || n3 % 64 || n3 > 128) return false;
    if (ld_out < n3 || (ld_out % 4) || ((uintptr_t)out & 15)) return false;
    for (int l = 0; l < 3; ++l)
        if (((uintptr_t)m->W[l] & 15) || ((uintptr_t)m->b[l] & 15)) return false;
    return tc::encode_fn() != nullptr;
}

dlrm_status launch_mlp3_tc(const dlrm_mlp* m, int B, const float* in, int ld_in, float* out, int ld_out, ErrRecord* err,
                           cudaStream_t st) {
    const int n0 = m->dims[0], n1 = m->dims[1], n2 = m->dims[2], n3 = m->dims[3];
    CUtensorMap m1, m2, m3;
    if (!tc::make_map_sw(&m1, m->W[0], n0, n1, dlrm_ld(n0, DLRM_BF16), 16, 64, CU_TENSOR_MAP_SWIZZLE_32B) ||
        !tc::make_map_sw(&m2, m->W[1], n1, n2, dlrm_ld(n1, DLRM_BF16), tc::BK, n2, CU_TENSOR_MAP_SWIZZLE_128B) ||
        !tc::make_map_sw(&m3, m->W[2], n2, n3, dlrm_ld(n2, DLRM_BF16), tc::BK, n3, CU_TENSOR_MAP_SWIZZLE_128B))
        return DLRM_ERR_CUDA;
    cudaFuncSetAttribute(tc::mlp3_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, tc::M3_SMEM);
    const int ntiles = (B + tc::BM - 1) / tc::BM;
    const int grid = ntiles < tc::sm_count_here() ? ntiles : tc::sm_count_here();
    tc::mlp3_tc_kernel<<<grid, tc::M3_THREADS, tc::M3_SMEM, st>>>(m1, m2, m3, in, ld_in, n0, B, n1, n2, n3, m->b[0],
                                                                  m->b[1], m->b[2], out, ld_out, err);
    DLRM_LAUNCH_CHECK();
    return DLRM_OK;
}

}  // namespace dlrm
