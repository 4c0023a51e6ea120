// The bottom MLP of DLRM ("Deep Learning Recommendation Model (DLRM)",
// nadeemcite summary, Key Method Details: FC layers with ReLU, mapping the
// dense features to the embedding width d) as one tensor-core kernel, for the
// shape of the pages' configurations: K0 <= 64 dense features -> 512 -> 256 ->
// N3 (ReLU after every layer), 16-bit weights and hidden activations, fp32
// input and output.
//
// One CTA (128 threads, one per TMEM lane) takes a 128-row tile through all
// three layers; only x_dense leaves the SM:
//   A0   the tile's dense features, read as fp32, converted to 16 bits and
//        written by the threads in the 128-byte-swizzled K-major layout the
//        MMA reads (64 columns, zero beyond K0);
//   L1   D[128][512] = A0 W1^T in TMEM (two N = 256 MMAs per k-step);
//        epilogue: bias, ReLU, 16-bit, written back as A1 (8 swizzled
//        64-column blocks, 128 KB);
//   L2   D[128][256] = A1 W2^T, 8 k-blocks; epilogue -> A2 (4 blocks) in
//        A1's space (its MMAs have completed);
//   L3   D[128][N3] = A2 W3^T, 4 k-blocks; epilogue: bias, ReLU, fp32 rows
//        of x_dense to global memory.
// Weights stream through a two-slot 32 KB TMA ring (they stay in L2), one
// thread issues the loads and the MMAs, every wait is bounded (timeout ->
// DLRM_ERR_TIMEOUT, TMEM freed). The numbers are those of the layer-by-layer
// path: fp32 accumulation, hidden activations rounded to 16 bits.
#include <cuda.h>

#include "common.cuh"
#include "kernels.cuh"
#include "tcgen05.cuh"

namespace dlrm {
namespace tc {

constexpr int FB_ROWS = 128;
constexpr int FB_N1 = 512, FB_N2 = 256;
constexpr int FB_KB = 64;                          // 16-bit elements per 128-byte row
constexpr int FB_BLK = FB_ROWS * FB_KB * 2;        // one 64-column block of a 128-row operand: 16 KB
constexpr int FB_A0 = FB_BLK;
constexpr int FB_A1 = FB_BLK * (FB_N1 / FB_KB);    // 128 KB; A2 (4 blocks) reuses it
constexpr int FB_SLOT = 256 * FB_KB * 2;           // weight chunk: up to 256 rows x 64 columns
constexpr int FB_SMEM = FB_A0 + FB_A1 + 2 * FB_SLOT + 1024 + 256;
static_assert(FB_SMEM <= 227 * 1024, "shared memory");

struct FBars {
    unsigned long long wfull[2];
    unsigned long long wempty[2];
    unsigned long long done;
    unsigned int tmem_base;
    int abort;
};

// byte offset of 16-byte chunk c of row r in a 128-byte-swizzled 64-column block
__device__ __forceinline__ uint32_t swz(int r, int c) { return (uint32_t)((r >> 3) * 1024 + (r & 7) * 128 + 16 * (c ^ (r & 7))); }

__host__ __device__ constexpr uint32_t idesc_n(int ab_fmt, int n) {
    return (1u << 4) | ((uint32_t)ab_fmt << 7) | ((uint32_t)ab_fmt << 10) | ((uint32_t)(n >> 3) << 17) |
           ((uint32_t)(FB_ROWS >> 4) << 24);
}

// One weight chunk: TMA map, coordinates, bytes, the A block it multiplies, where it accumulates.
struct FChunk {
    const CUtensorMap* map;
    int x, y;
    uint32_t bytes;
    uint32_t a;        // shared address of the A block
    uint32_t dcol;     // TMEM column offset of the accumulator
    uint32_t id;
    bool accum;        // add to the accumulator (false: the first k-block overwrites it)
};

template <typename T>
__global__ void __launch_bounds__(FB_ROWS, 1)
    bottom_mlp_fused_kernel(const __grid_constant__ CUtensorMap mW1, const __grid_constant__ CUtensorMap mW2,
                            const __grid_constant__ CUtensorMap mW3, const float* __restrict__ dense, int ldd, int B,
                            int K0, int N3, const float* __restrict__ b1, const float* __restrict__ b2,
                            const float* __restrict__ b3, float* __restrict__ out, int ldo, int relu_last, int fmt,
                            ErrRecord* err) {
    extern __shared__ __align__(1024) unsigned char smem_raw[];
    const uint32_t raw = su32(smem_raw);
    const uint32_t base = (raw + 1023u) & ~1023u;
    unsigned char* g = smem_raw + (base - raw);
    const uint32_t sA0 = base, sA1 = base + FB_A0, sW = base + FB_A0 + FB_A1;
    unsigned char* A0 = g;
    unsigned char* A1 = g + FB_A0;
    FBars* bars = reinterpret_cast<FBars*>(g + FB_A0 + FB_A1 + 2 * FB_SLOT);
    const int tid = threadIdx.x, warp = tid >> 5;
    if (tid == 0) {
        for (int s = 0; s < 2; ++s) {
            mbar_init(&bars->wfull[s], 1);
            mbar_init(&bars->wempty[s], 1);
        }
        mbar_init(&bars->done, 1);
        bars->abort = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    if (warp == 0) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(su32(&bars->tmem_base)),
                     "r"(512));
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
    }
    fence_before();
    __syncthreads();
    fence_after();
    const uint32_t tmem = bars->tmem_base;
    volatile int* abort = &bars->abort;
    const uint32_t lane_base = tmem + ((uint32_t)(warp * 32) << 16);   // this warp's 32 TMEM lanes = its rows
    const uint32_t id256 = idesc_n(fmt, 256), idN3 = idesc_n(fmt, N3);
    uint32_t chunk = 0;        // weight chunks issued so far (thread 0): slot chunk & 1
    uint32_t done_par = 0;     // completions of `done` seen so far
    bool timed_out = false;

    // thread 0: stream the chunks of one layer through the ring and issue its MMAs
    auto run_layer = [&](const FChunk* q, int n) {
        auto load = [&](const FChunk& c, uint32_t k) {
            const int s = (int)(k & 1u);
            if (!mbar_wait(&bars->wempty[s], ((k >> 1) & 1u) ^ 1u, abort)) return false;
            mbar_expect_tx(&bars->wfull[s], c.bytes);
            tma_load_2d(sW + s * FB_SLOT, c.map, &bars->wfull[s], c.x, c.y);
            return true;
        };
        if (!load(q[0], chunk)) return false;
        for (int i = 0; i < n; ++i) {
            const uint32_t k = chunk + (uint32_t)i;
            if (i + 1 < n && !load(q[i + 1], k + 1)) return false;
            const int s = (int)(k & 1u);
            if (!mbar_wait(&bars->wfull[s], (k >> 1) & 1u, abort)) return false;
            fence_after();
#pragma unroll
            for (int kk = 0; kk < FB_KB / 16; ++kk)
                umma(tmem + q[i].dcol, sdesc(q[i].a + kk * 32), sdesc(sW + s * FB_SLOT + kk * 32), q[i].id,
                     (q[i].accum || kk > 0) ? 1u : 0u);
            umma_commit(&bars->wempty[s]);
        }
        chunk += (uint32_t)n;
        umma_commit(&bars->done);
        return true;
    };
    auto wait_done = [&]() {
        const bool ok = mbar_wait(&bars->done, done_par & 1u, abort);
        ++done_par;
        fence_after();
        return ok;
    };
    // rows of this thread: D row `tid` = TMEM lane tid; 32 columns at a time -> 16-bit swizzled A blocks
    auto epilogue_to_smem = [&](int ncols, const float* __restrict__ bias, unsigned char* dst) {
#pragma unroll 1
        for (int c = 0; c < ncols / 32; ++c) {
            uint32_t r[32];
            tmem_ld32_issue(lane_base + 32 * c, r);
            tmem_ld_wait();
            unsigned char* blk = dst + (c >> 1) * FB_BLK;
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                T t[8];
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    const float v = __uint_as_float(r[8 * q + e]) + __ldg(bias + 32 * c + 8 * q + e);
                    t[e] = Cvt<T>::from_f(v > 0.f ? v : 0.f);
                }
                *reinterpret_cast<uint4*>(blk + swz(tid, (c & 1) * 4 + q)) = *reinterpret_cast<const uint4*>(t);
            }
        }
        fence_before();
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
        __syncthreads();
        fence_after();
    };

    const int ntiles = (B + FB_ROWS - 1) / FB_ROWS;
    for (int t = blockIdx.x; t < ntiles && !timed_out; t += gridDim.x) {
        const long long row = (long long)t * FB_ROWS + tid;
        // ---- A0: dense features of this thread's row, 16-bit, zero beyond K0 and beyond B
        {
            float x[FB_KB];
#pragma unroll
            for (int k = 0; k < FB_KB; ++k) x[k] = (row < B && k < K0) ? __ldg(dense + row * ldd + k) : 0.f;
#pragma unroll
            for (int c = 0; c < 8; ++c) {
                T v[8];
#pragma unroll
                for (int e = 0; e < 8; ++e) v[e] = Cvt<T>::from_f(x[8 * c + e]);
                *reinterpret_cast<uint4*>(A0 + swz(tid, c)) = *reinterpret_cast<const uint4*>(v);
            }
            asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
            __syncthreads();
        }
        // ---- layer 1: D[:, 0:256] and D[:, 256:512] from the two halves of W1
        if (tid == 0) {
            const FChunk q[2] = {{&mW1, 0, 0, (uint32_t)FB_SLOT, sA0, 0u, id256, false},
                                 {&mW1, 0, 256, (uint32_t)FB_SLOT, sA0, 256u, id256, false}};
            if (!run_layer(q, 2)) *abort = 1;
        }
        if (!wait_done()) { timed_out = true; break; }
        epilogue_to_smem(FB_N1, b1, A1);
        // ---- layer 2: 8 k-blocks of W2 against the 8 blocks of A1
        if (tid == 0) {
            FChunk q[FB_N1 / FB_KB];
            for (int i = 0; i < FB_N1 / FB_KB; ++i)
                q[i] = {&mW2, FB_KB * i, 0, (uint32_t)FB_SLOT, sA1 + (uint32_t)(i * FB_BLK), 0u, id256, i > 0};
            if (!run_layer(q, FB_N1 / FB_KB)) *abort = 1;
        }
        if (!wait_done()) { timed_out = true; break; }
        epilogue_to_smem(FB_N2, b2, A1);   // A2 overwrites A1: layer 2's MMAs have completed
        // ---- layer 3: 4 k-blocks of W3 (N3 rows) against A2
        if (tid == 0) {
            FChunk q[FB_N2 / FB_KB];
            for (int i = 0; i < FB_N2 / FB_KB; ++i)
                q[i] = {&mW3, FB_KB * i, 0, (uint32_t)(N3 * FB_KB * 2), sA1 + (uint32_t)(i * FB_BLK), 0u, idN3, i > 0};
            if (!run_layer(q, FB_N2 / FB_KB)) *abort = 1;
        }
        if (!wait_done()) { timed_out = true; break; }
        // ---- x_dense rows: bias, ReLU, fp32
#pragma unroll 1
        for (int c = 0; c < N3 / 32; ++c) {
            uint32_t r[32];
            tmem_ld32_issue(lane_base + 32 * c, r);
            tmem_ld_wait();
            if (row < B) {
                float4* o = reinterpret_cast<float4*>(out + row * ldo + 32 * c);
#pragma unroll
                for (int q = 0; q < 8; ++q) {
                    float v[4];
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        v[e] = __uint_as_float(r[4 * q + e]) + __ldg(b3 + 32 * c + 4 * q + e);
                        if (relu_last) v[e] = v[e] > 0.f ? v[e] : 0.f;
                    }
                    o[q] = make_float4(v[0], v[1], v[2], v[3]);
                }
            }
        }
        fence_before();
        __syncthreads();   // TMEM and A0 are reused by the next tile
        fence_after();
    }
    if (timed_out) {
        if (tid == 0) atomicOr(&err->flags, (unsigned)ERR_TIMEOUT);
        *abort = 1;
    }
    // every MMA this CTA issued has completed (or the wait for it ran out) before TMEM is freed
    if (tid == 0) {
        umma_commit(&bars->done);
        mbar_wait(&bars->done, done_par & 1u, abort, true);
    }
    fence_before();
    __syncthreads();
    fence_after();
    if (warp == 0) asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(512));
}

namespace {

bool weight_map(CUtensorMap* m, const void* W, dlrm_dtype dt, int K, int N, int ldw, int box_rows) {
    EncodeTiledFn enc = encode_fn();
    if (!enc) return false;
    const cuuint64_t dims[2] = {(cuuint64_t)K, (cuuint64_t)N};
    const cuuint64_t strides[1] = {(cuuint64_t)ldw * 2};
    const cuuint32_t box[2] = {(cuuint32_t)FB_KB, (cuuint32_t)box_rows};
    const cuuint32_t estr[2] = {1, 1};
    return enc(m, dt == DLRM_BF16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2,
               const_cast<void*>(W), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
               CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

int sm_count_fb() {
    int dev = 0, v = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev);
    return v > 0 ? v : 148;
}

inline bool al16(const void* p) { return ((uintptr_t)p & 15u) == 0; }

}  // namespace
}  // namespace tc

bool bottom_mlp_fused_supported(const dlrm_mlp* m, dlrm_dtype in_dt, const void* out, int ld_out, int final_act) {
    if (m->n_layers != 3 || in_dt != DLRM_F32 || (m->dt != DLRM_BF16 && m->dt != DLRM_F16)) return false;
    if (m->dims[0] < 1 || m->dims[0] > tc::FB_KB || m->dims[1] != tc::FB_N1 || m->dims[2] != tc::FB_N2) return false;
    const int n3 = m->dims[3];
    if (n3 < 32 || n3 > 256 || n3 % 32) return false;
    if (final_act != DLRM_ACT_RELU && final_act != DLRM_ACT_NONE) return false;
    if (!tc::al16(out) || ld_out % 4) return false;
    for (int l = 0; l < 3; ++l)
        if (!tc::al16(m->W[l]) || !tc::al16(m->b[l])) return false;
    return tc::encode_fn() != nullptr;
}

dlrm_status launch_bottom_mlp_fused(const dlrm_mlp* m, int B, const float* dense, int ldd, float* out, int ld_out,
                                    int final_act, ErrRecord* err, cudaStream_t st) {
    using namespace tc;
    if (B == 0) return DLRM_OK;
    CUtensorMap m1, m2, m3;
    if (!weight_map(&m1, m->W[0], m->dt, m->dims[0], FB_N1, dlrm_ld(m->dims[0], m->dt), 256) ||
        !weight_map(&m2, m->W[1], m->dt, FB_N1, FB_N2, dlrm_ld(FB_N1, m->dt), 256) ||
        !weight_map(&m3, m->W[2], m->dt, FB_N2, m->dims[3], dlrm_ld(FB_N2, m->dt), m->dims[3]))
        return DLRM_ERR_CUDA;
    const int ntiles = (B + FB_ROWS - 1) / FB_ROWS;
    const int sms = sm_count_fb();
    const int grid = ntiles < sms ? ntiles : sms;
    const int fmt = m->dt == DLRM_BF16 ? 1 : 0;
    if (m->dt == DLRM_BF16) {
        auto kern = bottom_mlp_fused_kernel<__nv_bfloat16>;
        cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, FB_SMEM);
        kern<<<grid, FB_ROWS, FB_SMEM, st>>>(m1, m2, m3, dense, ldd, B, m->dims[0], m->dims[3], m->b[0], m->b[1],
                                             m->b[2], out, ld_out, final_act == DLRM_ACT_RELU, fmt, err);
    } else {
        auto kern = bottom_mlp_fused_kernel<__half>;
        cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, FB_SMEM);
        kern<<<grid, FB_ROWS, FB_SMEM, st>>>(m1, m2, m3, dense, ldd, B, m->dims[0], m->dims[3], m->b[0], m->b[1],
                                             m->b[2], out, ld_out, final_act == DLRM_ACT_RELU, fmt, err);
    }
    DLRM_LAUNCH_CHECK();
    return DLRM_OK;
}

}  // namespace dlrm
