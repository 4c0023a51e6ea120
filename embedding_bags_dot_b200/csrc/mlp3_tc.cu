// Three fully connected layers in one kernel, for the bottom MLP of DLRM
// ("Deep Learning Recommendation Model (DLRM)", nadeemcite summary, Key Method
// Details: the dense features go through FC layers with ReLU):
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
//   warp 1      allocates 512 TMEM columns; one thread issues the tcgen05 MMAs
//               of layers 2 and 3;
//   warps 2..9  two per TMEM lane quadrant (32 rows), half the columns each.
// Layer 1 (K = 16) is too thin for the tcgen05 pipe: the epilogue warps
// compute it themselves, 64 columns at a time, with mma.sync (x fragments
// straight from global memory, W1 fragments by ldmatrix, accumulators started
// at the bias), and write the ReLU'd bf16 chunk with stmatrix into one of four
// 16 KB operand tiles; the two warp groups take alternate chunks. Chunk j of h1 is exactly k-block j of layer 2's A
// operand, so the epilogue runs up to four chunks ahead of the layer-2 MMAs.
// Once layer 2 is done the four tiles take h2 (bias, ReLU, bf16 from TMEM)
// for layer 3, whose accumulator alternates between two TMEM buffers so that
// its epilogue overlaps the next tile.
// TMEM: layer-2 accumulator [0, 256), layer-3 accumulators [256, 384) and
// [384, 512). Biases sit in shared memory. All waits are bounded: on timeout
// the kernel records DLRM_ERR_TIMEOUT, drains its own copies and MMAs, frees
// TMEM and returns. Launched as a programmatic dependent: barriers and TMEM are
// set up before pdl_wait().
#include <cuda.h>

#include "common.cuh"
#include "kernels.cuh"
#include "tcgen05.cuh"

namespace dlrm {
namespace tc {
namespace {

constexpr int M3_THREADS = 64 + 32 * EPI_WARPS;
constexpr int SLOTS = 4;                               // operand-ring tiles (h1 chunks, then h2)
constexpr int W_STAGES = 4;
constexpr int W_STAGE_BYTES = 256 * BK * 2;            // one k-block of up to 256 weight rows
constexpr int TILE_BYTES = BM * BK * 2;                // one 128 x 64 bf16 operand tile
constexpr int OFF_W1 = 0;                              // n1 / 64 chunks of 64 rows x 32 bytes
constexpr int OFF_BIAS = 16 * 1024;                    // b1 | b2 | b3, up to 896 floats
constexpr int OFF_ACT = 20 * 1024;                     // SLOTS operand tiles
constexpr int OFF_WR = OFF_ACT + SLOTS * TILE_BYTES;   // weight ring
constexpr int OFF_BARS = OFF_WR + W_STAGES * W_STAGE_BYTES;
constexpr int M3_SMEM = OFF_BARS + 512 + 1024;
constexpr uint32_t COL_ACC2 = 0, COL_ACC3 = 256;
static_assert(M3_SMEM <= 227 * 1024, "shared memory of the fused MLP");
static_assert(OFF_ACT % 1024 == 0 && OFF_WR % 1024 == 0, "swizzled tiles are 1024-byte aligned");

struct Bars3 {
    unsigned long long wfull[W_STAGES], wempty[W_STAGES];
    unsigned long long w1full;
    unsigned long long s1full[SLOTS], s1empty[SLOTS];   // h1 chunk tiles in the operand ring
    unsigned long long acc2full, acc2empty, s2full, s2empty;
    unsigned long long acc3full[2], acc3empty[2];
    unsigned long long drain;
    unsigned int tmem_base;
    int abort;
};
static_assert(sizeof(Bars3) <= 512, "barrier block");

static __device__ long long g_mlp3_wait_polls = WAIT_LIMIT;

__host__ __device__ constexpr uint32_t idesc_mn(int m, int n) {
    return (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(n >> 3) << 17) | ((uint32_t)(m >> 4) << 24);
}

__device__ __forceinline__ uint32_t pack2(float a, float b) {
    __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
    return *reinterpret_cast<uint32_t*>(&h);
}

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t (&r)[4]) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
                 : "r"(addr));
}
__device__ __forceinline__ void stsm_x4(uint32_t addr, uint32_t r0, uint32_t r1, uint32_t r2, uint32_t r3) {
    asm volatile("stmatrix.sync.aligned.m8n8.x4.shared.b16 [%0], {%1,%2,%3,%4};" ::"r"(addr), "r"(r0), "r"(r1),
                 "r"(r2), "r"(r3)
                 : "memory");
}
__device__ __forceinline__ void mma16816(float (&c)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%0,%1,%2,%3};"
        : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
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

// Global use count of operand slot j % SLOTS by chunk j of tile i (uses per tile: chunks with that slot).
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
        for (int a = 0; a < SLOTS; ++a) {
            mbar_init(&bars->s1full[a], EPI_WARPS / 2);   // one warp group writes a chunk
            mbar_init(&bars->s1empty[a], 1);
        }
        mbar_init(&bars->acc2full, 1);
        mbar_init(&bars->acc2empty, EPI_WARPS);
        mbar_init(&bars->s2full, EPI_WARPS);
        mbar_init(&bars->s2empty, 1);
        for (int a = 0; a < 2; ++a) {
            mbar_init(&bars->acc3full[a], 1);
            mbar_init(&bars->acc3empty[a], EPI_WARPS);
        }
        mbar_init(&bars->drain, 1);
        bars->abort = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    if (warp == 1) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(su32(&bars->tmem_base)),
                     "r"(512));
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
    }
    pdl_wait();      // the previous kernel on the stream has completed; global memory from here on
    for (int c = threadIdx.x; c < n1 + n2 + n3; c += blockDim.x)
        bias_s[c] = c < n1 ? __ldg(b1 + c) : c < n1 + n2 ? __ldg(b2 + c - n1) : __ldg(b3 + c - n1 - n2);
    fence_before();
    __syncthreads();
    fence_after();
    const uint32_t tmem = bars->tmem_base;
    volatile int* abort = &bars->abort;
    bool timed_out = false;
    const long long lim = g_mlp3_wait_polls;
    const bool any = (int)blockIdx.x < ntiles;

    if (warp == 0) {
        if (lane == 0) {
            asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&mapW2)) : "memory");
            asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&mapW3)) : "memory");
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
            const uint32_t id2 = idesc_mn(BM, n2), id3 = idesc_mn(BM, n3);
            int ws = 0;
            uint32_t wph = 0;
            int i = 0;
            for (int t = blockIdx.x; t < ntiles && !timed_out; t += gridDim.x, ++i) {
                const uint32_t ip = (uint32_t)i & 1u;
                // layer 2: k-block j is h1 chunk j (operand slot j % SLOTS)
                for (int j = 0; j < nc1; ++j) {
                    const int sl = j % SLOTS;
                    const uint32_t u = slot_use(i, j, nc1);
                    if ((j == 0 && !mbar_wait_n(&bars->acc2empty, ip ^ 1u, abort, lim)) ||
                        !mbar_wait_n(&bars->s1full[sl], u & 1u, abort, lim) ||
                        !mbar_wait_n(&bars->wfull[ws], wph, abort, lim)) {
                        timed_out = true;
                        break;
                    }
                    fence_after();
                    const uint32_t a = base + OFF_ACT + sl * TILE_BYTES, w = base + OFF_WR + ws * W_STAGE_BYTES;
#pragma unroll
                    for (int k = 0; k < BK / 16; ++k)
                        umma(tmem + COL_ACC2, sdesc(a + k * 32), sdesc(w + k * 32), id2, (j | k) != 0);
                    umma_commit(&bars->wempty[ws]);
                    umma_commit(&bars->s1empty[sl]);
                    if (++ws == W_STAGES) {
                        ws = 0;
                        wph ^= 1u;
                    }
                }
                if (timed_out) break;
                umma_commit(&bars->acc2full);
                // layer 3 on h2 (operand slots 0 .. n2/64 - 1) into accumulator i & 1
                const uint32_t d3 = tmem + COL_ACC3 + 128 * ip;
                if (!mbar_wait_n(&bars->s2full, ip, abort, lim) ||
                    !mbar_wait_n(&bars->acc3empty[ip], (((uint32_t)i >> 1) & 1u) ^ 1u, abort, lim)) {
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
                    for (int k = 0; k < BK / 16; ++k) umma(d3, sdesc(a + k * 32), sdesc(w + k * 32), id3, (kb | k) != 0);
                    umma_commit(&bars->wempty[ws]);
                    if (++ws == W_STAGES) {
                        ws = 0;
                        wph ^= 1u;
                    }
                }
                if (timed_out) break;
                umma_commit(&bars->acc3full[ip]);
                umma_commit(&bars->s2empty);
            }
            if (timed_out) *abort = 1;
            umma_commit(&bars->drain);
            mbar_wait(&bars->drain, 0, abort, true);
        }
    } else {
        const int ew = warp - 2;
        const int q = warp & 3;                  // TMEM lane quadrant: rows 32 q .. 32 q + 31
        const int h = ew >> 2;                   // half of the columns
        const int r = q * 32 + lane;             // this thread's row for the TMEM epilogues
        const int rsw = r & 7;                   // 128-byte swizzle phase of that row
        const uint32_t lanes = (uint32_t)(q * 32) << 16;
        const int gr = lane >> 2, tc = 2 * (lane & 3);
        const float* bs1 = bias_s;
        const float* bs2 = bias_s + n1;
        const float* bs3 = bias_s + n1 + n2;
        // x fragments (mma.sync A layout) of rows 32 q + 16 mt + {gr, gr + 8}, columns {tc, tc+1, tc+8, tc+9}
        float xf[2][8];
        auto load_x = [&](int t) {
#pragma unroll
            for (int mt = 0; mt < 2; ++mt)
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    const long long row = (long long)t * BM + q * 32 + 16 * mt + gr + 8 * ((e >> 1) & 1);
                    const int k = tc + (e & 1) + 8 * (e >> 2);
                    xf[mt][e] = (row < M && k < n0) ? __ldg(x + row * ldx + k) : 0.f;
                }
        };
        // layer-3 accumulator of tile tt (local index ii) -> fp32 output rows
        auto out_tile = [&](int tt, int ii) -> bool {
            const uint32_t b = (uint32_t)ii & 1u;
            if (!mbar_wait_n(&bars->acc3full[b], ((uint32_t)ii >> 1) & 1u, abort, lim)) return false;
            fence_after();
            const long long row = (long long)tt * BM + r;
            for (int cb = 0; cb < n3 / 64; ++cb) {
                const int col = h * (n3 / 2) + 32 * cb;
                uint32_t acc[32];
                tmem_ld32_issue(tmem + lanes + COL_ACC3 + 128 * b + col, acc);
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
            if (lane == 0) mbar_arrive(&bars->acc3empty[b]);
            return true;
        };
        if (any) {
            load_x(blockIdx.x);
            if (!mbar_wait_n(&bars->w1full, 0, abort, lim)) timed_out = true;
        }
        int i = 0;
        for (int t = blockIdx.x; t < ntiles && !timed_out; t += gridDim.x, ++i) {
            const uint32_t ip = (uint32_t)i & 1u;
            uint32_t af[2][4];
#pragma unroll
            for (int mt = 0; mt < 2; ++mt)
#pragma unroll
                for (int p = 0; p < 4; ++p) af[mt][p] = pack2(xf[mt][2 * p], xf[mt][2 * p + 1]);
            if (t + (int)gridDim.x < ntiles) load_x(t + gridDim.x);   // the next tile's x, a tile ahead
            // layer 1, chunk j on mma.sync -> h1 tile j % SLOTS: the two warp groups (h = 0, 1) take alternate
            // chunks, each warp 32 rows x 64 columns, so two chunks are in progress at a time
            for (int j = h; j < nc1; j += 2) {
                const int sl = j % SLOTS;
                const uint32_t u = slot_use(i, j, nc1);
                const uint32_t slot = base + OFF_ACT + sl * TILE_BYTES;
#pragma unroll
                for (int cc = 0; cc < 2; ++cc) {   // columns 32 cc .. 32 cc + 31 of the chunk
                    uint32_t bf[2][4];
#pragma unroll
                    for (int hh = 0; hh < 2; ++hh) {
                        const int n = 32 * cc + 16 * hh + (lane & 15);         // W1 row within chunk j
                        ldsm_x4(base + OFF_W1 + j * 2048 + n * 32 + 16 * ((lane >> 4) ^ ((n >> 2) & 1)), bf[hh]);
                    }
                    float acc[2][4][4];
#pragma unroll
                    for (int nt = 0; nt < 4; ++nt) {
                        const float2 bb = *reinterpret_cast<const float2*>(bs1 + 64 * j + 32 * cc + 8 * nt + tc);
#pragma unroll
                        for (int mt = 0; mt < 2; ++mt) {
                            acc[mt][nt][0] = bb.x;
                            acc[mt][nt][1] = bb.y;
                            acc[mt][nt][2] = bb.x;
                            acc[mt][nt][3] = bb.y;
                            mma16816(acc[mt][nt], af[mt], bf[nt >> 1][(nt & 1) ? 1 : 0], bf[nt >> 1][(nt & 1) ? 3 : 2]);
                        }
                    }
                    // the slot's previous reader: layer 2 on chunk j - SLOTS of this tile, else the last tile's layer 3
                    if (cc == 0) {
                        const bool ok = j >= SLOTS ? mbar_wait_n(&bars->s1empty[sl], (u & 1u) ^ 1u, abort, lim)
                                                   : mbar_wait_n(&bars->s2empty, ip ^ 1u, abort, lim);
                        if (!ok) {
                            timed_out = true;
                            break;
                        }
                    }
#pragma unroll
                    for (int mt = 0; mt < 2; ++mt)
#pragma unroll
                        for (int np = 0; np < 2; ++np) {
                            uint32_t v[4];
#pragma unroll
                            for (int m = 0; m < 4; ++m) {   // matrix m: n-tile 2 np + (m >> 1), rows gr (+8 if m odd)
                                const float* c = acc[mt][2 * np + (m >> 1)];
                                v[m] = (m & 1) ? pack2(fmaxf(c[2], 0.f), fmaxf(c[3], 0.f))
                                               : pack2(fmaxf(c[0], 0.f), fmaxf(c[1], 0.f));
                            }
                            const int m = lane >> 3;
                            const int row = q * 32 + 16 * mt + 8 * (m & 1) + (lane & 7);
                            const int kc = 4 * cc + 2 * np + (m >> 1);
                            stsm_x4(slot + row * 128 + 16 * (kc ^ (row & 7)), v[0], v[1], v[2], v[3]);
                        }
                }
                if (timed_out) break;
                asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
                __syncwarp();
                if (lane == 0) mbar_arrive(&bars->s1full[sl]);
            }
            if (timed_out) break;
            // layer-2 accumulator -> h2 tiles (layer 2 has finished reading the ring)
            if (!mbar_wait_n(&bars->acc2full, ip, abort, lim)) {
                timed_out = true;
                break;
            }
            fence_after();
            for (int cb = 0; cb < n2 / 64; ++cb) {
                const int col = h * (n2 / 2) + 32 * cb;
                uint32_t acc[32];
                tmem_ld32_issue(tmem + lanes + COL_ACC2 + col, acc);
                tmem_ld_wait();
                store_bf16_chunks(acc, bs2 + col, g + OFF_ACT + (col / 64) * TILE_BYTES + r * 128, (col % 64) / 8,
                                  rsw);
            }
            fence_before();
            asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
            __syncwarp();
            if (lane == 0) {
                mbar_arrive(&bars->acc2empty);
                mbar_arrive(&bars->s2full);
            }
            // the previous tile's output while this tile's layer 3 runs
            if (i > 0 && !out_tile(t - (int)gridDim.x, i - 1)) {
                timed_out = true;
                break;
            }
        }
        if (!timed_out && i > 0 && !out_tile(blockIdx.x + (i - 1) * (int)gridDim.x, i - 1)) timed_out = true;
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
    DLRM_PDL_CHECK(launch_pdl(tc::mlp3_tc_kernel, dim3(grid), dim3(tc::M3_THREADS), (size_t)tc::M3_SMEM, st, m1, m2, m3,
                              in, ld_in, n0, B, n1, n2, n3, m->b[0], m->b[1], m->b[2], out, ld_out, err));
    return DLRM_OK;
}

}  // namespace dlrm
