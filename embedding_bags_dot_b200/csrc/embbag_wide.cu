// Fused gather + interaction for many tables (K + 1 > 64 vectors) of bf16 rows, on the tensor cores.
//
// The operation is the fused kernels' (per sample b: pool the K bags into e_1..e_K, "DLRM", briansu.co,
// section 3; write [x_dense, Z_10, Z_20, Z_21, ...] with Z_ij = <X_i, X_j>, j < i, over
// X = [x_dense; e_1..e_K], "DLRM", briansu.co, section 4, equations "Interaction" and "Output"). With
// K + 1 = 101 vectors the Gram is a real contraction (5,050 terms of d products per sample), so it runs on
// mma.sync; the bags hold dozens of rows each, so the gather is built for rows in flight, not for one row
// per bag.
//
// A block owns S samples (S = 4 for d = 64):
//  1. gather: work items (sample, table) are taken from a shared counter by lane groups of d/8 lanes
//     (16 bytes of a row per lane); a group walks its bag's CSR range U rows at a time (U row loads in
//     flight per lane), sums in fp32 and stores the pooled row as bf16 into row k of the sample's tile
//     (rows padded by 16 bytes: the 8 rows an ldmatrix reads fall in distinct bank groups). Empty bags and
//     bags with bad offsets give a zero row; out-of-range indices are skipped. x_dense (fp32) goes in as
//     two bf16 rows of a small tile, hi = bf16(x) and lo = bf16(x - hi), and as bf16(x) into the first d
//     columns of the sample's output row, which is assembled in shared memory.
//  2. Gram: the warps of a sample take its 16-row m-tiles; for m-tile mt the lower-triangle n8 tiles
//     (columns < 16 mt + 16) of G = E E^T come from mma.sync.m16n8k16 (bf16 in, fp32 accumulate), and one
//     more n8 tile against the x tile gives <e_i, x_hi> and <e_i, x_lo> side by side in the same thread,
//     whose sum is Z_i0 at fp32 precision of x_dense. Each value goes straight from the accumulators to its
//     concat column d + i(i-1)/2 + j in the staged row. Rows of the tile past the sample's K are never
//     written: they only reach Gram entries nothing reads.
//  3. one bulk copy (cp.async.bulk, shared -> global) per sample writes the whole concat row.
// Nothing waits on another block or on a flag: the only waits are the bulk stores' own completion.
#include <algorithm>

#include "async_copy.cuh"
#include "common.cuh"
#include "kernels.cuh"

namespace dlrm {

namespace {

using namespace ac;

constexpr int WW = 8;                 // warps per block
constexpr int NC = 2;                 // 16-column blocks of the Gram accumulated at a time per m-tile
constexpr unsigned FULLW = 0xffffffffu;

__device__ __forceinline__ uint32_t pack_bf16w(float lo, float hi) {
    __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t*>(&h);
}

__device__ __forceinline__ void mma_bf16w(float (&c)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%0,%1,%2,%3};"
        : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

__device__ __forceinline__ void ldmatrix_x2(uint32_t addr, uint32_t& r0, uint32_t& r1) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x2.shared.b16 {%0,%1}, [%2];" : "=r"(r0), "=r"(r1) : "r"(addr));
}

__device__ __forceinline__ void bulk_store_row(void* dst, uint32_t src, uint32_t bytes) {
    asm volatile("cp.async.bulk.global.shared::cta.bulk_group [%0], [%1], %2;" ::"l"(dst), "r"(src), "r"(bytes)
                 : "memory");
    asm volatile("cp.async.bulk.commit_group;" ::: "memory");
}
__device__ __forceinline__ void bulk_store_read_done() {
    asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory");
}

// Shared-memory layout of one sample: e tile [KP][RS], x tile [8][RS], output row [ld] bf16.
struct WideLayout {
    int RS, KP, tile, xtile, orow, per_sample;
};

__host__ __device__ inline WideLayout wide_layout(int d, int MT, int ld) {
    WideLayout L;
    L.RS = 2 * d + 16;
    L.KP = 16 * MT;
    L.tile = L.KP * L.RS;
    L.xtile = 8 * L.RS;
    L.orow = (2 * ld + 15) / 16 * 16;
    L.per_sample = L.tile + L.xtile + L.orow;
    return L;
}

}  // namespace

// GL: lanes per row (d = 8 GL); MT: 16-row m-tiles of the e tile (16 MT >= K); U: rows in flight per lane.
template <int GL, int MT, int U>
__global__ void __launch_bounds__(WW * 32, 3) embbag_interact_wide_kernel(
    const __nv_bfloat16* __restrict__ tables, const __grid_constant__ TableMeta tm, int K, int B, int S,
    const int32_t* __restrict__ offsets, const int32_t* __restrict__ indices, long long nnz,
    const float* __restrict__ x_dense, __nv_bfloat16* __restrict__ out, int ld, ErrRecord* err) {
    pdl_wait();   // programmatic dependent: the previous kernel's outputs are visible from here on
    constexpr int d = 8 * GL;
    constexpr int NG = 32 / GL;                   // lane groups per warp
    const WideLayout L = wide_layout(d, MT, ld);
    extern __shared__ __align__(128) unsigned char smem[];
    int* next_item = reinterpret_cast<int*>(smem + (size_t)S * L.per_sample);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int g = lane % GL, grp = lane / GL;
    const int b0 = blockIdx.x * S;
    const int nb = min(S, B - b0);
    const int P = K * (K + 1) / 2;
    unsigned oob = 0, bad = 0;

    auto tile_of = [&](int s) { return smem + (size_t)s * L.per_sample; };
    auto xtile_of = [&](int s) { return smem + (size_t)s * L.per_sample + L.tile; };
    auto orow_of = [&](int s) { return reinterpret_cast<__nv_bfloat16*>(smem + (size_t)s * L.per_sample + L.tile + L.xtile); };

    if (threadIdx.x == 0) *next_item = 0;
    // x_dense: hi / lo rows of the x tile and the first d output columns; zero padding after the last Z
    for (int q = threadIdx.x; q < nb * d; q += blockDim.x) {
        const int s = q / d, t = q - s * d;
        const float x = x_dense[(long long)(b0 + s) * d + t];
        const __nv_bfloat16 hi = __float2bfloat16_rn(x);
        const __nv_bfloat16 lo = __float2bfloat16_rn(x - __bfloat162float(hi));
        __nv_bfloat16* xr = reinterpret_cast<__nv_bfloat16*>(xtile_of(s));
        xr[t] = hi;
        xr[L.RS / 2 + t] = lo;
        orow_of(s)[t] = hi;
    }
    for (int q = threadIdx.x; q < nb * (ld - d - P); q += blockDim.x) {
        const int s = q / (ld - d - P), t = q - s * (ld - d - P);
        orow_of(s)[d + P + t] = __float2bfloat16_rn(0.f);
    }
    __syncthreads();

    // ---- 1. gather: items (table k, sample s), k-major; a warp takes NG consecutive items from the shared
    // counter at a time (warp-uniform loop), one per lane group
    const int n_items = K * nb;
    for (;;) {
        int it0 = 0;
        if (lane == 0) it0 = atomicAdd(next_item, NG);
        it0 = __shfl_sync(FULLW, it0, 0);
        if (it0 >= n_items) break;
        const int it = it0 + grp;
        if (it >= n_items) continue;
        const int k = it / nb, s = it - k * nb;
        const long long o = (long long)k * B + b0 + s;
        const long long st = offsets[o], en = offsets[o + 1];
        float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
        if (st < 0 || en < st || en > nnz) {
            if (g == 0) ++bad;
        } else {
            const __nv_bfloat16* tab = tables + tm.base[k] * (long long)d + 8 * g;
            const long long m = tm.rows[k];
            // the next U indices are loaded while this step's rows are in flight
            int idx[U];
#pragma unroll
            for (int u = 0; u < U; ++u) idx[u] = st + u < en ? __ldg(indices + st + u) : -1;
            for (long long p = st; p < en; p += U) {
                int nxt[U];
                if (p + 2 * U <= en) {
#pragma unroll
                    for (int u = 0; u < U; ++u) nxt[u] = __ldg(indices + p + U + u);
                } else {
#pragma unroll
                    for (int u = 0; u < U; ++u) nxt[u] = p + U + u < en ? __ldg(indices + p + U + u) : -1;
                }
                uint4 v[U];
                unsigned okm = 0;
#pragma unroll
                for (int u = 0; u < U; ++u) {
                    const bool ok = (unsigned long long)(unsigned)idx[u] < (unsigned long long)m;   // -1: past the bag
                    okm |= (unsigned)ok << u;
                    v[u] = ok ? ldg16_stream(tab + (long long)idx[u] * d) : make_uint4(0, 0, 0, 0);
                }
                if (g == 0) {   // indices of the bag that are out of range (not the slots past its end)
                    const int n = en - p < U ? (int)(en - p) : U;
                    oob += __popc(~okm & ((1u << n) - 1u));
                }
#pragma unroll
                for (int u = 0; u < U; ++u) Chunk16<__nv_bfloat16>::add(v[u], acc);
#pragma unroll
                for (int u = 0; u < U; ++u) idx[u] = nxt[u];
            }
        }
        *reinterpret_cast<uint4*>(tile_of(s) + k * L.RS + 16 * g) =
            make_uint4(pack_bf16w(acc[0], acc[1]), pack_bf16w(acc[2], acc[3]), pack_bf16w(acc[4], acc[5]),
                       pack_bf16w(acc[6], acc[7]));
    }
    __syncthreads();

    // ---- 2. Gram per sample: the WPS warps of sample s take its m-tiles round robin
    const int WPS = WW / S;
    const int s = warp / WPS, wsub = warp - s * WPS;
    if (s < nb) {
        const uint32_t tile_s = (uint32_t)__cvta_generic_to_shared(tile_of(s));
        const uint32_t xt_s = (uint32_t)__cvta_generic_to_shared(xtile_of(s));
        __nv_bfloat16* orow = orow_of(s);
        const int gr = lane >> 2, tc = (lane & 3) * 2;
#pragma unroll
        for (int mt = 0; mt < MT; ++mt) {
            if (mt % WPS != wsub || 16 * mt >= K) continue;
            // the lower-triangle n8 tiles of this m-tile in chunks of NC 16-column blocks (few accumulators
            // live at a time), the x tile with the first chunk
#pragma unroll
            for (int c0 = 0; c0 <= mt; c0 += NC) {
                float acc[2 * NC][4];
                float ax[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
                for (int t = 0; t < 2 * NC; ++t) acc[t][0] = acc[t][1] = acc[t][2] = acc[t][3] = 0.f;
#pragma unroll
                for (int ks = 0; ks < d / 16; ++ks) {
                    uint32_t a[4];
                    ldmatrix_x4(tile_s + (uint32_t)((16 * mt + (lane & 15)) * L.RS + 16 * (2 * ks + (lane >> 4))), a);
#pragma unroll
                    for (int j = 0; j < NC; ++j) {
                        const int n2 = c0 + j;
                        if (n2 > mt) break;
                        uint32_t b[4];
                        if (n2 == mt) {
                            b[0] = a[0]; b[1] = a[1]; b[2] = a[2]; b[3] = a[3];
                        } else {
                            ldmatrix_x4(tile_s + (uint32_t)((16 * n2 + (lane & 15)) * L.RS + 16 * (2 * ks + (lane >> 4))), b);
                        }
                        mma_bf16w(acc[2 * j], a, b[0], b[2]);
                        mma_bf16w(acc[2 * j + 1], a, b[1], b[3]);
                    }
                    if (c0 == 0) {
                        uint32_t x0, x1;
                        ldmatrix_x2(xt_s + (uint32_t)((lane & 7) * L.RS + 16 * (2 * ks + ((lane >> 3) & 1))), x0, x1);
                        mma_bf16w(ax, a, x0, x1);
                    }
                }
                // rows r = 16 mt + gr (+ 8) hold e_{r+1}: Z_{r+1, c+1} for c < r, and (first chunk) Z_{r+1, 0}
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    const int r = 16 * mt + gr + 8 * h;
                    if (r >= K) continue;
                    const int base = d + (r + 1) * r / 2;          // concat column of Z_{r+1, 0}
                    if (c0 == 0 && tc == 0) orow[base] = __float2bfloat16_rn(ax[2 * h] + ax[2 * h + 1]);
#pragma unroll
                    for (int t = 0; t < 2 * NC; ++t) {
                        const int c = 16 * c0 + 8 * t + tc;
                        if (c < r) orow[base + 1 + c] = __float2bfloat16_rn(acc[t][2 * h]);
                        if (c + 1 < r) orow[base + 2 + c] = __float2bfloat16_rn(acc[t][2 * h + 1]);
                    }
                }
            }
        }
    }
    // ---- 3. one bulk store per sample of its staged row (generic writes made visible to the copy first)
    fence_proxy_async();
    __syncthreads();
    if (threadIdx.x < nb) {
        const int q = threadIdx.x;
        bulk_store_row(out + (size_t)(b0 + q) * ld, (uint32_t)__cvta_generic_to_shared(orow_of(q)),
                       (uint32_t)(2 * ld));
        bulk_store_read_done();
    }
    report_warp(err, oob, bad);
}

// ------------------------------------------------------------------ host side

static size_t wide_smem(int d, int MT, int ld, int S) {
    return (size_t)S * wide_layout(d, MT, ld).per_sample + 16;
}

// Samples per block: the most that still lets three blocks share an SM (the register budget allows three),
// else the most that let two, else 1
// (0: does not fit).
static int wide_samples(int d, int MT, int ld) {
    for (int blocks : {3, 2})
        for (int S : {4, 2, 1})
            if ((size_t)blocks * (wide_smem(d, MT, ld, S) + 1024) <= 228 * 1024) return S;
    return wide_smem(d, MT, ld, 1) <= 227 * 1024 ? 1 : 0;
}

bool embbag_interact_wide_supported(dlrm_dtype dt, int K, int d, int ld, const void* out, dlrm_dtype out_dt) {
    if (dt != DLRM_BF16 || out_dt != DLRM_BF16) return false;
    if (!(d == 64 || d == 128)) return false;
    if (K < 1 || K > 128) return false;
    if (ld % 8 || ((uintptr_t)out & 15)) return false;
    if (ld < d + K * (K + 1) / 2) return false;
    return wide_samples(d, (K + 15) / 16, ld) > 0;
}

template <int GL, int MT>
static void launch_wide_t(const TableMeta& tm, const void* tables, int K, int B, const int32_t* offsets,
                          const int32_t* indices, long long nnz, const float* x_dense, void* out, int ld,
                          ErrRecord* err, cudaStream_t st) {
    constexpr int d = 8 * GL;
    const int S = wide_samples(d, MT, ld);
    const size_t smem = wide_smem(d, MT, ld, S);
    auto kern = embbag_interact_wide_kernel<GL, MT, 8>;
    cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    (void)launch_pdl(kern, dim3((B + S - 1) / S), dim3(WW * 32), smem, st, static_cast<const __nv_bfloat16*>(tables), tm,
                     K, B, S, offsets, indices, nnz, x_dense, static_cast<__nv_bfloat16*>(out), ld, err);
}

dlrm_status launch_embbag_interact_wide(const TableMeta& tm, const void* tables, int K, int d, int B,
                                        const int32_t* offsets, const int32_t* indices, long long nnz,
                                        const float* x_dense, void* out, int ld, ErrRecord* err, cudaStream_t st) {
    const int MT = (K + 15) / 16;
#define DLRM_WIDE(GLV)                                                                                          \
    switch (MT) {                                                                                               \
        case 1: launch_wide_t<GLV, 1>(tm, tables, K, B, offsets, indices, nnz, x_dense, out, ld, err, st); break; \
        case 2: launch_wide_t<GLV, 2>(tm, tables, K, B, offsets, indices, nnz, x_dense, out, ld, err, st); break; \
        case 3: launch_wide_t<GLV, 3>(tm, tables, K, B, offsets, indices, nnz, x_dense, out, ld, err, st); break; \
        case 4: launch_wide_t<GLV, 4>(tm, tables, K, B, offsets, indices, nnz, x_dense, out, ld, err, st); break; \
        case 5: launch_wide_t<GLV, 5>(tm, tables, K, B, offsets, indices, nnz, x_dense, out, ld, err, st); break; \
        case 6: launch_wide_t<GLV, 6>(tm, tables, K, B, offsets, indices, nnz, x_dense, out, ld, err, st); break; \
        case 7: launch_wide_t<GLV, 7>(tm, tables, K, B, offsets, indices, nnz, x_dense, out, ld, err, st); break; \
        default: launch_wide_t<GLV, 8>(tm, tables, K, B, offsets, indices, nnz, x_dense, out, ld, err, st); break; \
    }
    if (d == 64) {
        DLRM_WIDE(8)
    } else {
        DLRM_WIDE(16)
    }
#undef DLRM_WIDE
    DLRM_LAUNCH_CHECK();
    return DLRM_OK;
}

}  // namespace dlrm
