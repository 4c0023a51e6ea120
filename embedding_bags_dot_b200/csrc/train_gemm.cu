// fp32 GEMMs of the training step (forward with saved activations, data
// gradient, weight gradient). The training workload keeps every tensor in
// fp32, so these run on the CUDA cores with fp32 accumulation.
//
// One kernel covers the three operand layouts:
//   C(i, j) = sum_r A(i, r) B(j, r)
//   A(i, r) = A[i*lda + r]  (AT = false)   or  A[r*lda + i]  (AT = true)
//   B(j, r) = B[j*ldb + r]  (BT = false)   or  B[r*ldb + j]  (BT = true)
// forward:  y = x W^T + b             A = x,   B = W     (AT = 0, BT = 0)
// dgrad:    dx = dy W  (* ReLU mask)  A = dy,  B = W     (AT = 0, BT = 1)
// wgrad:    dW = dy^T x, db = dy^T 1  A = dy,  B = x     (AT = 1, BT = 1), split over r
// The weight gradient reduces over the batch; it is split into fixed r-ranges
// whose partial sums are added in a fixed order, so results are
// bit-reproducible run to run.
#include "common.cuh"
#include "kernels.cuh"

namespace dlrm {

namespace {

constexpr int TM = 64, TN = 64, TK = 16;

enum Epi { EPI_BIAS = 0, EPI_BIAS_RELU = 1, EPI_MASK = 2, EPI_PLAIN = 3, EPI_PARTIAL = 4 };

template <bool T>
__device__ __forceinline__ void load_tile(float (&S)[TK][TN + 4], const float* __restrict__ X, long long ld, long long i0,
                                          long long r0, long long ni, long long nr, bool ones_col) {
    // S[r][i] = X(i0 + i, r0 + r), zero outside, 1 for the synthesized column i == ni when ones_col
    if constexpr (!T) {
        const int i = threadIdx.x >> 2, r = (threadIdx.x & 3) * 4;
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            const long long gi = i0 + i, gr = r0 + r + e;
            float v = 0.f;
            if (gr < nr) {
                if (gi < ni) v = X[gi * ld + gr];
                else if (ones_col && gi == ni) v = 1.f;
            }
            S[r + e][i] = v;
        }
    } else {
        const int r = threadIdx.x >> 4, i = (threadIdx.x & 15) * 4;
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            const long long gi = i0 + i + e, gr = r0 + r;
            float v = 0.f;
            if (gr < nr) {
                if (gi < ni) v = X[gr * ld + gi];
                else if (ones_col && gi == ni) v = 1.f;
            }
            S[r][i + e] = v;
        }
    }
}

// Output tile (i0.., j0..) of C(i, j), reduction over r in [r_begin, r_end).
// B_ONES: B has a synthesized extra column j == NB of ones (weight-gradient bias term).
template <bool AT, bool BT, int EPI, bool B_ONES>
__global__ void __launch_bounds__(256) gemm_f32_kernel(long long NI, long long NJ, long long NR, const float* __restrict__ A,
                                                       long long lda, const float* __restrict__ Bm, long long ldb,
                                                       const float* __restrict__ bias, const float* __restrict__ mask,
                                                       long long ldm, float* __restrict__ C, long long ldc,
                                                       long long r_chunk, long long part_stride) {
    __shared__ float As[TK][TN + 4];
    __shared__ float Bs[TK][TN + 4];
    const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
    const long long i0 = (long long)blockIdx.y * TM, j0 = (long long)blockIdx.x * TN;
    const long long rb = (long long)blockIdx.z * r_chunk;
    const long long re = rb + r_chunk < NR ? rb + r_chunk : NR;
    const long long NJe = B_ONES ? NJ + 1 : NJ;
    float acc[4][4];
#pragma unroll
    for (int a = 0; a < 4; ++a)
#pragma unroll
        for (int b = 0; b < 4; ++b) acc[a][b] = 0.f;
    for (long long r0 = rb; r0 < re; r0 += TK) {
        load_tile<AT>(As, A, lda, i0, r0, NI, re, false);
        load_tile<BT>(Bs, Bm, ldb, j0, r0, NJ, re, B_ONES);
        __syncthreads();
#pragma unroll
        for (int kk = 0; kk < TK; ++kk) {
            const float4 a = *reinterpret_cast<const float4*>(&As[kk][ty * 4]);
            const float4 b = *reinterpret_cast<const float4*>(&Bs[kk][tx * 4]);
            const float av[4] = {a.x, a.y, a.z, a.w}, bv[4] = {b.x, b.y, b.z, b.w};
#pragma unroll
            for (int x = 0; x < 4; ++x)
#pragma unroll
                for (int y = 0; y < 4; ++y) acc[x][y] = fmaf(av[x], bv[y], acc[x][y]);
        }
        __syncthreads();
    }
#pragma unroll
    for (int x = 0; x < 4; ++x) {
        const long long i = i0 + ty * 4 + x;
        if (i >= NI) continue;
#pragma unroll
        for (int y = 0; y < 4; ++y) {
            const long long j = j0 + tx * 4 + y;
            if (j >= NJe) continue;
            float v = acc[x][y];
            if constexpr (EPI == EPI_BIAS || EPI == EPI_BIAS_RELU) v += bias[j];
            if constexpr (EPI == EPI_BIAS_RELU) v = v > 0.f ? v : 0.f;
            if constexpr (EPI == EPI_MASK) v = (mask[i * ldm + j] > 0.f) ? v : 0.f;
            if constexpr (EPI == EPI_PARTIAL)
                C[(long long)blockIdx.z * part_stride + i * (NJ + 1) + j] = v;
            else
                C[i * ldc + j] = v;
        }
    }
}

// dW[i][j] = sum over splits (in order) of part[s][i][j]; db[i] from column NJ.
__global__ void wgrad_reduce_kernel(int splits, long long NI, long long NJ, const float* __restrict__ part,
                                    long long part_stride, float* __restrict__ dW, long long ldw, float* __restrict__ db) {
    const long long n = NI * (NJ + 1);
    for (long long q = (long long)blockIdx.x * blockDim.x + threadIdx.x; q < n; q += (long long)gridDim.x * blockDim.x) {
        float s = 0.f;
        for (int z = 0; z < splits; ++z) s += part[z * part_stride + q];
        const long long i = q / (NJ + 1), j = q - i * (NJ + 1);
        if (j < NJ) dW[i * ldw + j] = s;
        else db[i] = s;
    }
}

dim3 grid_for(long long NI, long long NJ, int z) {
    return dim3((unsigned)((NJ + TN - 1) / TN), (unsigned)((NI + TM - 1) / TM), (unsigned)z);
}

}  // namespace

dlrm_status train_linear_fwd(int M, int N, int K, const float* x, int ldx, const float* W, int ldw, const float* b,
                             float* y, int ldy, bool relu, cudaStream_t st) {
    if (M == 0) return DLRM_OK;
    if (relu)
        gemm_f32_kernel<false, false, EPI_BIAS_RELU, false><<<grid_for(M, N, 1), 256, 0, st>>>(
            M, N, K, x, ldx, W, ldw, b, nullptr, 0, y, ldy, K, 0);
    else
        gemm_f32_kernel<false, false, EPI_BIAS, false><<<grid_for(M, N, 1), 256, 0, st>>>(
            M, N, K, x, ldx, W, ldw, b, nullptr, 0, y, ldy, K, 0);
    DLRM_LAUNCH_CHECK();
    return DLRM_OK;
}

dlrm_status train_linear_dgrad(int M, int N, int K, const float* dy, int lddy, const float* W, int ldw,
                               const float* relu_of, int ldr, float* dx, int lddx, cudaStream_t st) {
    // dx[m][k] = sum_n dy[m][n] W[n][k], zeroed where relu_of[m][k] <= 0 (if given)
    if (M == 0) return DLRM_OK;
    if (relu_of)
        gemm_f32_kernel<false, true, EPI_MASK, false><<<grid_for(M, K, 1), 256, 0, st>>>(
            M, K, N, dy, lddy, W, ldw, nullptr, relu_of, ldr, dx, lddx, N, 0);
    else
        gemm_f32_kernel<false, true, EPI_PLAIN, false><<<grid_for(M, K, 1), 256, 0, st>>>(
            M, K, N, dy, lddy, W, ldw, nullptr, nullptr, 0, dx, lddx, N, 0);
    DLRM_LAUNCH_CHECK();
    return DLRM_OK;
}

size_t train_wgrad_scratch_floats(int N, int K, int M) {
    const int splits = train_wgrad_splits(N, K, M);
    return (size_t)splits * (size_t)N * (size_t)(K + 1);
}

int train_wgrad_splits(int N, int K, int M) {
    // enough blocks to fill the GPU; fixed per shape so results do not depend on the device
    const long long tiles = ((N + TM - 1) / TM) * (long long)((K + 1 + TN - 1) / TN);
    long long s = (1184 + tiles - 1) / tiles;
    const long long max_s = (M + 255) / 256;
    if (s > max_s) s = max_s;
    if (s < 1) s = 1;
    if (s > 64) s = 64;
    return (int)s;
}

dlrm_status train_linear_wgrad(int M, int N, int K, const float* dy, int lddy, const float* x, int ldx, float* dW,
                               int ldw, float* db, float* scratch, cudaStream_t st) {
    // dW[n][k] = sum_m dy[m][n] x[m][k]; db[n] = sum_m dy[m][n]
    const int splits = train_wgrad_splits(N, K, M);
    long long chunk = ((long long)M + splits - 1) / splits;
    chunk = (chunk + TK - 1) / TK * TK;
    const long long pstride = (long long)N * (K + 1);
    gemm_f32_kernel<true, true, EPI_PARTIAL, true><<<grid_for(N, K + 1, splits), 256, 0, st>>>(
        N, K, M, dy, lddy, x, ldx, nullptr, nullptr, 0, scratch, 0, chunk, pstride);
    DLRM_LAUNCH_CHECK();
    const long long n = pstride;
    const int blocks = (int)((n + 255) / 256 < 4096 ? (n + 255) / 256 : 4096);
    wgrad_reduce_kernel<<<blocks, 256, 0, st>>>(splits, N, K, scratch, pstride, dW, ldw, db);
    DLRM_LAUNCH_CHECK();
    return DLRM_OK;
}

}  // namespace dlrm
