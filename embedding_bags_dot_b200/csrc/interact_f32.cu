// fp32 pairwise dot interaction of the training step, forward and backward,
// on 3xTF32 (hi, lo) pairs ("DLRM", briansu.co, section 4, equation
// "Interaction": Z = tril(X X^T) over X = [x_dense; e_1; ...; e_K], self-
// interactions left out; the backward is its derivative:
// dX_i = sum_{j != i} dZ_ij X_j with dZ symmetric).
//
// One warp per sample. Lane l holds columns [V l, V l + V) of all N1 = K + 1
// vectors in registers (d = 32 V), so every product is formed once:
//   forward:  for 32 pairs at a time each lane sums its V products per pair,
//             then a five-step reduce-scatter across the warp leaves lane l
//             with the whole dot product of pair l of the group, written
//             straight into the concat row (pairs in row-major strict-lower
//             order (1,0), (2,0), (2,1), ...);
//   backward: the sample's dZ (K(K+1)/2 values) is expanded into a
//             symmetric N1 x N1 matrix with zero diagonal in the warp's
//             shared memory; lane l forms dX_i for its columns from
//             broadcast 16-byte reads of row i.
// The vectors come in as x_dense (a pair: the bottom MLP's output) and the
// pooled embeddings E [B][K][d] (plain fp32); concat, dx_dense are written as
// pairs, dE plain. N1 and V are template parameters so that every register
// index is static.
#include "common.cuh"
#include "kernels.cuh"

namespace dlrm {
namespace {

__device__ __forceinline__ float tf32_hi_i(float v) {
    const uint32_t u = __float_as_uint(v);
    uint32_t r = u + 0x1000u;
    if ((r & 0x7F800000u) == 0x7F800000u) r = u;
    return __uint_as_float(r & 0xFFFFE000u);
}

template <int V>
struct VecF;
template <>
struct VecF<2> {
    float v[2];
    __device__ __forceinline__ void load(const float* p) {
        const float2 t = __ldg(reinterpret_cast<const float2*>(p));
        v[0] = t.x;
        v[1] = t.y;
    }
    __device__ __forceinline__ void load_cs(const float* p) {
        const float2 t = __ldcs(reinterpret_cast<const float2*>(p));
        v[0] = t.x;
        v[1] = t.y;
    }
    __device__ __forceinline__ void store(float* p) const { *reinterpret_cast<float2*>(p) = make_float2(v[0], v[1]); }
};
template <>
struct VecF<4> {
    float v[4];
    __device__ __forceinline__ void load(const float* p) {
        const float4 t = __ldg(reinterpret_cast<const float4*>(p));
        v[0] = t.x;
        v[1] = t.y;
        v[2] = t.z;
        v[3] = t.w;
    }
    __device__ __forceinline__ void load_cs(const float* p) {
        const float4 t = __ldcs(reinterpret_cast<const float4*>(p));
        v[0] = t.x;
        v[1] = t.y;
        v[2] = t.z;
        v[3] = t.w;
    }
    __device__ __forceinline__ void store(float* p) const {
        *reinterpret_cast<float4*>(p) = make_float4(v[0], v[1], v[2], v[3]);
    }
};

// Sample b's vectors into registers: x[0] from the x_dense pair, x[1..K] from E.
template <int N1, int V>
__device__ __forceinline__ void load_sample(float (&x)[N1][V], long long b, const float* __restrict__ xh,
                                            const float* __restrict__ xl, int ldx, const float* __restrict__ E,
                                            int lane) {
    constexpr int d = 32 * V;
    VecF<V> h, l;
    h.load(xh + b * ldx + V * lane);
    l.load(xl + b * ldx + V * lane);
#pragma unroll
    for (int e = 0; e < V; ++e) x[0][e] = h.v[e] + l.v[e];
#pragma unroll
    for (int k = 1; k < N1; ++k) {
        VecF<V> t;
        t.load_cs(E + (b * (N1 - 1) + (k - 1)) * (long long)d + V * lane);
#pragma unroll
        for (int e = 0; e < V; ++e) x[k][e] = t.v[e];
    }
}

// Lane l ends with the sum over lanes of part[l] (part is consumed).
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

// Pair (I, J), J < I, of the strict lower triangle; p = I(I-1)/2 + J is its
// concat position. Every 32 pairs (and at the last one) the group is reduced
// across the warp and stored. Compile-time recursion over the pairs of row I
// keeps every register index static.
template <int I, int J, int N1, int V>
__device__ __forceinline__ void pair_step(const float (&x)[N1][V], float (&part)[32], int lane, float* rh,
                                          float* rl) {
    constexpr int P = N1 * (N1 - 1) / 2;
    constexpr int p = I * (I - 1) / 2 + J;
    float s = x[I][0] * x[J][0];
#pragma unroll
    for (int e = 1; e < V; ++e) s = fmaf(x[I][e], x[J][e], s);
    part[p & 31] = s;
    if constexpr (((p + 1) & 31) == 0 || p + 1 == P) {
        constexpr int n = (p & 31) + 1;   // pairs in this group
#pragma unroll
        for (int q = n; q < 32; ++q) part[q] = 0.f;
        const float z = reduce_scatter32(part, lane);
        if (lane < n) {
            const int col = 32 * V + (p & ~31) + lane;
            const float zh = tf32_hi_i(z);
            rh[col] = zh;
            rl[col] = z - zh;
        }
    }
    if constexpr (J + 1 < I) pair_step<I, J + 1, N1, V>(x, part, lane, rh, rl);
}

// rows I .. N1-1 of the triangle (two recursion levels keep the template depth below 2 N1)
template <int I, int N1, int V>
__device__ __forceinline__ void pair_rows(const float (&x)[N1][V], float (&part)[32], int lane, float* rh, float* rl) {
    pair_step<I, 0, N1, V>(x, part, lane, rh, rl);
    if constexpr (I + 1 < N1) pair_rows<I + 1, N1, V>(x, part, lane, rh, rl);
}

template <int N1, int V>
__global__ void __launch_bounds__(128, 3)
    interact_fwd_pair_kernel(int B, const float* __restrict__ xh, const float* __restrict__ xl, int ldx,
                             const float* __restrict__ E, float* __restrict__ ch, float* __restrict__ cl, int ldc) {
    const int lane = threadIdx.x & 31;
    const long long warps = (long long)gridDim.x * (blockDim.x >> 5);
    for (long long b = (long long)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); b < B; b += warps) {
        float x[N1][V];
        load_sample<N1, V>(x, b, xh, xl, ldx, E, lane);
        float* rh = ch + b * ldc;
        float* rl = cl + b * ldc;
        {   // concat columns [0, d): x_dense, already a pair
            VecF<V> h, l;
            h.load(xh + b * ldx + V * lane);
            l.load(xl + b * ldx + V * lane);
            h.store(rh + V * lane);
            l.store(rl + V * lane);
        }
        float part[32];
        pair_rows<1, N1, V>(x, part, lane, rh, rl);
    }
}

template <int N1, int V>
__global__ void __launch_bounds__(128, 3)
    interact_bwd_pair_kernel(int B, const float* __restrict__ xh, const float* __restrict__ xl, int ldx,
                             const float* __restrict__ E, const float* __restrict__ dcat, int ldc,
                             float* __restrict__ dxh, float* __restrict__ dxl, int lddx, float* __restrict__ dE) {
    constexpr int d = 32 * V;
    constexpr int SR = (N1 + 3) / 4 * 4;   // row stride of the symmetric dZ matrix
    constexpr int P = N1 * (N1 - 1) / 2;
    __shared__ __align__(16) float Sm[4][N1 * SR];
    const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
    float* S = Sm[w];
    // the diagonal and the padding columns stay zero; every other entry is rewritten per sample
    for (int q = lane; q < N1 * SR; q += 32) S[q] = 0.f;
    const long long warps = (long long)gridDim.x * (blockDim.x >> 5);
    for (long long b = (long long)blockIdx.x * (blockDim.x >> 5) + w; b < B; b += warps) {
        float x[N1][V];
        load_sample<N1, V>(x, b, xh, xl, ldx, E, lane);
        __syncwarp();
        // S[i][j] = S[j][i] = dZ(i, j) for j < i
        const float* dz = dcat + b * ldc + d;
        for (int q = lane; q < P; q += 32) {
            int i = (int)((1.0f + sqrtf(8.0f * (float)q + 1.0f)) * 0.5f);
            while (i * (i - 1) / 2 > q) --i;
            while ((i + 1) * i / 2 <= q) ++i;
            const int j = q - i * (i - 1) / 2;
            const float g = __ldcs(dz + q);
            S[i * SR + j] = g;
            S[j * SR + i] = g;
        }
        __syncwarp();
#pragma unroll
        for (int i = 0; i < N1; ++i) {
            float acc[V];
#pragma unroll
            for (int e = 0; e < V; ++e) acc[e] = 0.f;
#pragma unroll
            for (int j4 = 0; j4 < SR; j4 += 4) {
                const float4 s4 = *reinterpret_cast<const float4*>(S + i * SR + j4);
                const float sv[4] = {s4.x, s4.y, s4.z, s4.w};
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                    if (j4 + u < N1 && j4 + u != i) {
#pragma unroll
                        for (int e = 0; e < V; ++e) acc[e] = fmaf(sv[u], x[j4 + u][e], acc[e]);
                    }
                }
            }
            if (i == 0) {
                // x_dense is a ReLU output: its pre-activation gradient is masked
                VecF<V> dc, oh, ol;
                dc.load(dcat + b * ldc + V * lane);
#pragma unroll
                for (int e = 0; e < V; ++e) {
                    const float g = x[0][e] > 0.f ? acc[e] + dc.v[e] : 0.f;
                    oh.v[e] = tf32_hi_i(g);
                    ol.v[e] = g - oh.v[e];
                }
                oh.store(dxh + b * lddx + V * lane);
                ol.store(dxl + b * lddx + V * lane);
            } else {
                VecF<V> o;
#pragma unroll
                for (int e = 0; e < V; ++e) o.v[e] = acc[e];
                o.store(dE + (b * (N1 - 1) + (i - 1)) * (long long)d + V * lane);
            }
        }
        __syncwarp();
    }
}

int grid_for_warps(long long B) {
    const long long blocks = (B + 3) / 4;
    return (int)(blocks < 148 * 12 ? blocks : 148 * 12);
}

}  // namespace

bool interact_pair_supported(int K, int d) { return K == 26 && (d == 64 || d == 128); }

dlrm_status launch_interact_fwd_pair(int B, int K, int d, F32Pair x_dense, const float* E, float* concat_hi,
                                     float* concat_lo, int ldc, cudaStream_t st) {
    if (!interact_pair_supported(K, d)) return DLRM_ERR_UNSUPPORTED;
    if (B == 0) return DLRM_OK;
    if (d == 128)
        interact_fwd_pair_kernel<27, 4><<<grid_for_warps(B), 128, 0, st>>>(B, x_dense.hi, x_dense.lo, x_dense.ld, E,
                                                                           concat_hi, concat_lo, ldc);
    else
        interact_fwd_pair_kernel<27, 2><<<grid_for_warps(B), 128, 0, st>>>(B, x_dense.hi, x_dense.lo, x_dense.ld, E,
                                                                           concat_hi, concat_lo, ldc);
    DLRM_LAUNCH_CHECK();
    return DLRM_OK;
}

dlrm_status launch_interact_bwd_pair(int B, int K, int d, F32Pair x_dense, const float* E, const float* dconcat,
                                     int ldc, float* dx_hi, float* dx_lo, int lddx, float* dE, cudaStream_t st) {
    if (!interact_pair_supported(K, d)) return DLRM_ERR_UNSUPPORTED;
    if (B == 0) return DLRM_OK;
    if (d == 128)
        interact_bwd_pair_kernel<27, 4><<<grid_for_warps(B), 128, 0, st>>>(
            B, x_dense.hi, x_dense.lo, x_dense.ld, E, dconcat, ldc, dx_hi, dx_lo, lddx, dE);
    else
        interact_bwd_pair_kernel<27, 2><<<grid_for_warps(B), 128, 0, st>>>(
            B, x_dense.hi, x_dense.lo, x_dense.ld, E, dconcat, ldc, dx_hi, dx_lo, lddx, dE);
    DLRM_LAUNCH_CHECK();
    return DLRM_OK;
}

}  // namespace dlrm
