// fp32 GEMMs of the training step (forward with saved activations, data
// gradient, weight gradient): dispatch between the tensor-core 3xTF32 kernel
// (gemm_tf32.cu) and a CUDA-core fp32 kernel for the shapes it does not take
// (the 13-wide first bottom layer, the one-column logit layer), plus the
// pair-split, split-sum and bias-gradient helpers.
//
// Operands are F32Pair: plain fp32, or a 3xTF32 (hi, lo) pair whose value is
// hi + lo exactly; the CUDA-core kernel reads either and writes either.
//
// Shapes the tensor cores do not take get kernels of their own: the 13-wide
// first bottom layer (narrow_fwd_kernel; its weight gradient is a weighted
// column sum of dy, one pass), the one-column logit layer (gemv_rows_kernel,
// outer_mask_kernel, weighted column sums), and every bias gradient is a
// fixed-order column sum (colsum_w_kernel).
//
// The general CUDA-core kernel covers the three operand layouts:
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
__device__ __forceinline__ void load_tile(float (&S)[TK][TN + 4], const float* __restrict__ X,
                                          const float* __restrict__ Xlo, long long ld, long long i0, long long r0,
                                          long long ni, long long nr, bool ones_col) {
    // S[r][i] = X(i0 + i, r0 + r) (+ its lo part), zero outside, 1 for the synthesized column i == ni when ones_col
    if constexpr (!T) {
        const int i = threadIdx.x >> 2, r = (threadIdx.x & 3) * 4;
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            const long long gi = i0 + i, gr = r0 + r + e;
            float v = 0.f;
            if (gr < nr) {
                if (gi < ni) v = Xlo ? X[gi * ld + gr] + Xlo[gi * ld + gr] : X[gi * ld + gr];
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
                if (gi < ni) v = Xlo ? X[gr * ld + gi] + Xlo[gr * ld + gi] : X[gr * ld + gi];
                else if (ones_col && gi == ni) v = 1.f;
            }
            S[r][i + e] = v;
        }
    }
}

// hi part of a 3xTF32 pair: v rounded to the nearest TF32 value (ties away from
// zero; magnitudes that would round up to infinity are truncated), lo = v - hi exactly.
__device__ __forceinline__ float tf32_hi_part(float v) {
    const uint32_t u = __float_as_uint(v);
    uint32_t r = u + 0x1000u;
    if ((r & 0x7F800000u) == 0x7F800000u) r = u;
    return __uint_as_float(r & 0xFFFFE000u);
}

// Output tile (i0.., j0..) of C(i, j), reduction over r in [r_begin, r_end).
// B_ONES: B has a synthesized extra column j == NB of ones (weight-gradient bias term).
// C_lo non-null: the output is written as a (hi, lo) pair.
template <bool AT, bool BT, int EPI, bool B_ONES>
__global__ void __launch_bounds__(256) gemm_f32_kernel(long long NI, long long NJ, long long NR, const float* __restrict__ A,
                                                       const float* __restrict__ A_lo, long long lda,
                                                       const float* __restrict__ Bm, const float* __restrict__ B_lo,
                                                       long long ldb, const float* __restrict__ bias,
                                                       const float* __restrict__ mask, const float* __restrict__ mask_lo,
                                                       long long ldm, float* __restrict__ C, float* __restrict__ C_lo,
                                                       long long ldc, long long r_chunk, long long part_stride) {
    pdl_wait();
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
        load_tile<AT>(As, A, A_lo, lda, i0, r0, NI, re, false);
        load_tile<BT>(Bs, Bm, B_lo, ldb, j0, r0, NJ, re, B_ONES);
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
            if constexpr (EPI == EPI_MASK) {
                const float m = mask_lo ? mask[i * ldm + j] + mask_lo[i * ldm + j] : mask[i * ldm + j];
                v = (m > 0.f) ? v : 0.f;
            }
            if constexpr (EPI == EPI_PARTIAL) {
                C[(long long)blockIdx.z * part_stride + i * (NJ + 1) + j] = v;
            } else if (C_lo) {
                const float h = tf32_hi_part(v);
                C[i * ldc + j] = h;
                C_lo[i * ldc + j] = v - h;
            } else {
                C[i * ldc + j] = v;
            }
        }
    }
}

// dW[i][j] = sum over splits (in order) of part[s][i][j]; db[i] from column NJ.
__global__ void wgrad_reduce_kernel(int splits, long long NI, long long NJ, const float* __restrict__ part,
                                    long long part_stride, float* __restrict__ dW, long long ldw, float* __restrict__ db) {
    pdl_wait();
    const long long n = NI * (NJ + 1);
    for (long long q = (long long)blockIdx.x * blockDim.x + threadIdx.x; q < n; q += (long long)gridDim.x * blockDim.x) {
        float s = 0.f;
        for (int z = 0; z < splits; ++z) s += part[z * part_stride + q];
        const long long i = q / (NJ + 1), j = q - i * (NJ + 1);
        if (j < NJ) dW[i * ldw + j] = s;
        else db[i] = s;
    }
}

__global__ void split_pair_kernel(long long rows, int cols, const float* __restrict__ src, long long lds,
                                  float* __restrict__ hi, float* __restrict__ lo, long long ldd) {
    pdl_wait();
    const long long n = rows * cols;
    for (long long q = (long long)blockIdx.x * blockDim.x + threadIdx.x; q < n; q += (long long)gridDim.x * blockDim.x) {
        const long long r = q / cols, c = q - r * cols;
        const float v = src[r * lds + c];
        const float h = tf32_hi_part(v);
        hi[r * ldd + c] = h;
        lo[r * ldd + c] = v - h;
    }
}

__global__ void split_pair_vec_kernel(long long rows, int cols4, const float4* __restrict__ src, long long lds4,
                                      float4* __restrict__ hi, float4* __restrict__ lo, long long ldd4) {
    pdl_wait();
    const long long n = rows * cols4;
    for (long long q = (long long)blockIdx.x * blockDim.x + threadIdx.x; q < n; q += (long long)gridDim.x * blockDim.x) {
        const long long r = q / cols4, c = q - r * cols4;
        const float4 v = src[r * lds4 + c];
        const float4 h = make_float4(tf32_hi_part(v.x), tf32_hi_part(v.y), tf32_hi_part(v.z), tf32_hi_part(v.w));
        hi[r * ldd4 + c] = h;
        lo[r * ldd4 + c] = make_float4(v.x - h.x, v.y - h.y, v.z - h.z, v.w - h.w);
    }
}

__global__ void merge_pair_kernel(long long rows, int cols, const float* __restrict__ hi,
                                  const float* __restrict__ lo, long long lds, float* __restrict__ out, long long ldo) {
    pdl_wait();
    const long long n = rows * cols;
    for (long long q = (long long)blockIdx.x * blockDim.x + threadIdx.x; q < n; q += (long long)gridDim.x * blockDim.x) {
        const long long r = q / cols, c = q - r * cols;
        out[r * ldo + c] = hi[r * lds + c] + lo[r * lds + c];
    }
}

__global__ void split_sum_kernel(int S, long long N, int K, const float* __restrict__ part, long long ldp,
                                 float* __restrict__ out, long long ldo) {
    pdl_wait();
    const long long n = N * K;
    const long long zs = N * ldp;
    for (long long q = (long long)blockIdx.x * blockDim.x + threadIdx.x; q < n; q += (long long)gridDim.x * blockDim.x) {
        const long long i = q / K, j = q - i * K;
        float s = 0.f;
        for (int z = 0; z < S; ++z) s += part[z * zs + i * ldp + j];
        out[i * ldo + j] = s;
    }
}

// Weighted column sums over fixed row chunks:
//   part[p][c][w] = sum_{b in chunk p} A(b, c) * Wt(b, w),  w < NW
// A is [M][N] plain or a pair (value hi + lo); Wt(b, w) = X[b][w] for w < kx
// and 1 for w == kx when `ones`, 0 beyond. Each thread owns four columns, the
// warps of a block (CS_WARPS(NW)) take rows in turn, and their partials are
// combined in warp order: a fixed summation order for every result.
__host__ __device__ constexpr int CS_WARPS(int nw) { return nw > 4 ? 4 : 8; }

template <int NW>
__global__ void __launch_bounds__(256) colsum_w_kernel(long long M, int N, const float* __restrict__ ah,
                                                       const float* __restrict__ al, long long lda,
                                                       const float* __restrict__ X, long long ldx, int kx, bool ones,
                                                       long long rows_per, float* __restrict__ part) {
    pdl_wait();
    constexpr int WARPS = CS_WARPS(NW);
    __shared__ float red[WARPS][128 * NW + 1];
    const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
    const int c0 = blockIdx.x * 128 + 4 * lane;
    const long long rb = (long long)blockIdx.y * rows_per;
    const long long re = rb + rows_per < M ? rb + rows_per : M;
    const bool vec = (lda & 3) == 0 && c0 + 4 <= N;
    float acc[4][NW];
#pragma unroll
    for (int e = 0; e < 4; ++e)
#pragma unroll
        for (int q = 0; q < NW; ++q) acc[e][q] = 0.f;
    for (long long r = rb + w; r < re; r += WARPS) {
        float v[4];
        if (vec) {
            const float4 h = __ldg(reinterpret_cast<const float4*>(ah + r * lda + c0));
            v[0] = h.x, v[1] = h.y, v[2] = h.z, v[3] = h.w;
            if (al) {
                const float4 l = __ldg(reinterpret_cast<const float4*>(al + r * lda + c0));
                v[0] += l.x, v[1] += l.y, v[2] += l.z, v[3] += l.w;
            }
        } else {
#pragma unroll
            for (int e = 0; e < 4; ++e)
                v[e] = (c0 + e < N) ? (al ? ah[r * lda + c0 + e] + al[r * lda + c0 + e] : ah[r * lda + c0 + e]) : 0.f;
        }
        float wt[NW];
#pragma unroll
        for (int q = 0; q < NW; ++q) wt[q] = q < kx ? __ldg(X + r * ldx + q) : ((ones && q == kx) ? 1.f : 0.f);
#pragma unroll
        for (int e = 0; e < 4; ++e)
#pragma unroll
            for (int q = 0; q < NW; ++q) acc[e][q] = fmaf(v[e], wt[q], acc[e][q]);
    }
#pragma unroll
    for (int e = 0; e < 4; ++e)
#pragma unroll
        for (int q = 0; q < NW; ++q) red[w][(4 * lane + e) * NW + q] = acc[e][q];
    __syncthreads();
    for (int i = threadIdx.x; i < 128 * NW; i += blockDim.x) {
        const int c = blockIdx.x * 128 + i / NW;
        if (c >= N) continue;
        float t = 0.f;
#pragma unroll
        for (int y = 0; y < WARPS; ++y) t += red[y][i];
        part[((long long)blockIdx.y * N + c) * NW + (i % NW)] = t;
    }
}

// out(c, w) = sum over p of part[p][c][w], one warp per output: lane l adds p = l, l + 32, ... in order,
// then a fixed butterfly across lanes; w < kx -> dW[c * ldw + w], w == kx -> db[c]
__global__ void colsum_w_final_kernel(int P, int N, int NW, int kx, bool ones, const float* __restrict__ part,
                                      float* __restrict__ dW, long long ldw, float* __restrict__ db) {
    pdl_wait();
    const long long n = (long long)N * NW;
    const int lane = threadIdx.x & 31;
    const long long warps = (long long)gridDim.x * (blockDim.x >> 5);
    for (long long i = (long long)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); i < n; i += warps) {
        const int c = (int)(i / NW), q = (int)(i % NW);
        if (q > kx || (q == kx && !ones)) continue;   // uniform across the warp
        float s = 0.f;
        for (int p = lane; p < P; p += 32) s += part[(long long)p * n + i];
#pragma unroll
        for (int o = 16; o >= 1; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
        if (lane == 0) {
            if (q < kx) dW[c * ldw + q] = s;
            else db[c] = s;
        }
    }
}

// bits[m][j / 32] bit j % 32 = (y(m, j) > 0), y plain or a pair: one warp per (row, 32 columns)
__global__ void relu_bits_kernel(long long M, int N, const float* __restrict__ yh, const float* __restrict__ yl,
                                 long long ldy, uint32_t* __restrict__ bits, long long ldbits) {
    pdl_wait();
    const int lane = threadIdx.x & 31;
    const long long words = M * ldbits;
    const long long warps = (long long)gridDim.x * (blockDim.x >> 5);
    for (long long q = (long long)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); q < words; q += warps) {
        const long long m = q / ldbits;
        const int j = (int)(q - m * ldbits) * 32 + lane;
        bool pos = false;
        if (j < N) pos = (yl ? yh[m * ldy + j] + yl[m * ldy + j] : yh[m * ldy + j]) > 0.f;
        const uint32_t w = __ballot_sync(0xffffffffu, pos);
        if (lane == 0) bits[q] = w;
    }
}

// db[j] = sum over 32-row groups g of csum[g][j] in increasing g (one warp per column: lane l adds
// g = l, l + 32, ... in order, then a fixed butterfly)
__global__ void csum_final_kernel(int G, int J, const float* __restrict__ csum, float* __restrict__ db) {
    pdl_wait();
    const int lane = threadIdx.x & 31;
    const int warps = gridDim.x * (blockDim.x >> 5);
    for (int j = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); j < J; j += warps) {
        float s = 0.f;
        for (int g = lane; g < G; g += 32) s += csum[(long long)g * J + j];
#pragma unroll
        for (int o = 16; o >= 1; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
        if (lane == 0) db[j] = s;
    }
}

// y[b][n] = act(sum_{k < K} x(b, k) W[n][k] + bias[n]) for K <= 16 (the 13 dense features): one thread
// per output column with its weight row in registers; the block's rows of x are staged in shared memory
// (read there as broadcasts), four rows per step; y written as a pair or plain.
constexpr int NARROW_ROWS = 256;
__global__ void __launch_bounds__(128) narrow_fwd_kernel(long long M, int N, int K, const float* __restrict__ xh,
                                                         const float* __restrict__ xl, long long ldx,
                                                         const float* __restrict__ W, const float* __restrict__ Wl,
                                                         long long ldw, const float* __restrict__ bias, bool relu,
                                                         float* __restrict__ yh, float* __restrict__ yl, long long ldy,
                                                         uint32_t* __restrict__ bits, long long ldbits) {
    pdl_wait();
    __shared__ float xs[NARROW_ROWS][17];
    const long long rb = (long long)blockIdx.y * NARROW_ROWS;
    const int nr = (int)(M - rb < NARROW_ROWS ? M - rb : NARROW_ROWS);
    for (int q = threadIdx.x; q < nr * K; q += blockDim.x) {
        const int r = q / K, k = q - r * K;
        const long long g = (rb + r) * ldx + k;
        xs[r][k] = xl ? xh[g] + xl[g] : xh[g];
    }
    __syncthreads();
    const int n = blockIdx.x * 128 + threadIdx.x;
    const bool active = n < N;   // inactive lanes stay for the bitmask ballots
    float wr[16];
#pragma unroll
    for (int k = 0; k < 16; ++k)
        wr[k] = (active && k < K) ? (Wl ? W[n * ldw + k] + Wl[n * ldw + k] : W[n * ldw + k]) : 0.f;
    const float bn = active ? bias[n] : 0.f;
    for (int r0 = 0; r0 < nr; r0 += 4) {
        float s[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int k = 0; k < 16; ++k)
            if (k < K)
#pragma unroll
                for (int u = 0; u < 4; ++u) s[u] = fmaf(xs[r0 + u < nr ? r0 + u : r0][k], wr[k], s[u]);
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            if (r0 + u >= nr) break;   // uniform across the block
            float v = s[u] + bn;
            if (relu) v = v > 0.f ? v : 0.f;
            const long long o = (rb + r0 + u) * ldy + n;
            if (active) {
                if (yl) {
                    const float h = tf32_hi_part(v);
                    yh[o] = h;
                    yl[o] = v - h;
                } else {
                    yh[o] = v;
                }
            }
            if (bits) {
                const uint32_t w = __ballot_sync(0xffffffffu, active && v > 0.f);
                if ((threadIdx.x & 31) == 0 && n < N) bits[(rb + r0 + u) * ldbits + n / 32] = w;
            }
        }
    }
}

// z[b] = sum_k x(b, k) w[k] + bias[0] (a one-column layer): one warp per row
__global__ void __launch_bounds__(256) gemv_rows_kernel(long long M, int K, const float* __restrict__ xh,
                                                        const float* __restrict__ xl, long long ldx,
                                                        const float* __restrict__ w, const float* __restrict__ wl,
                                                        const float* __restrict__ bias, float* __restrict__ z) {
    pdl_wait();
    const int lane = threadIdx.x & 31;
    const long long warps = (long long)gridDim.x * (blockDim.x >> 5);
    for (long long b = (long long)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); b < M; b += warps) {
        float s = 0.f;
        for (int k = lane; k < K; k += 32) {
            const float v = xl ? xh[b * ldx + k] + xl[b * ldx + k] : xh[b * ldx + k];
            s = fmaf(v, wl ? __ldg(w + k) + __ldg(wl + k) : __ldg(w + k), s);
        }
#pragma unroll
        for (int o = 16; o >= 1; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
        if (lane == 0) z[b] = s + bias[0];
    }
}

// dx[b][k] = dz[b] * w[k] where relu_of(b, k) > 0, else 0 (data gradient of a one-column layer), as a pair
__global__ void outer_mask_kernel(long long M, int K, const float* __restrict__ dz, const float* __restrict__ w,
                                  const float* __restrict__ wl, const float* __restrict__ mh, const float* __restrict__ ml, long long ldm,
                                  float* __restrict__ dh, float* __restrict__ dl, long long ldd) {
    pdl_wait();
    const long long n = M * K;
    for (long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += (long long)gridDim.x * blockDim.x) {
        const long long b = i / K;
        const int k = (int)(i - b * K);
        const float m = ml ? mh[b * ldm + k] + ml[b * ldm + k] : mh[b * ldm + k];
        const float v = m > 0.f ? dz[b] * (wl ? __ldg(w + k) + __ldg(wl + k) : __ldg(w + k)) : 0.f;
        const float h = tf32_hi_part(v);
        dh[b * ldd + k] = h;
        dl[b * ldd + k] = v - h;
    }
}

int colsum_chunks(int M) {
    const int p = (M + 511) / 512;
    return p < 1 ? 1 : (p > 128 ? 128 : p);
}

dim3 grid_for(long long NI, long long NJ, int z) {
    return dim3((unsigned)((NJ + TN - 1) / TN), (unsigned)((NI + TM - 1) / TM), (unsigned)z);
}

int grid_stride_blocks(long long n) { return (int)((n + 255) / 256 < 8192 ? (n + 255) / 256 : 8192); }

int simt_wgrad_splits(int N, int K, int M) {
    // enough blocks to fill the GPU; fixed per shape so results do not depend on the device
    const long long tiles = ((N + TM - 1) / TM) * (long long)((K + 1 + TN - 1) / TN);
    long long s = (1184 + tiles - 1) / tiles;
    const long long max_s = (M + 255) / 256;
    if (s > max_s) s = max_s;
    if (s < 1) s = 1;
    if (s > 64) s = 64;
    return (int)s;
}

bool is_pair(F32Pair p) { return p.lo != nullptr; }

}  // namespace

dlrm_status launch_split_pair(int rows, int cols, const float* src, int lds, float* hi, float* lo, int ldd,
                              cudaStream_t st) {
    if (rows <= 0 || cols <= 0) return DLRM_OK;
    const bool vec = cols % 4 == 0 && lds % 4 == 0 && ldd % 4 == 0 && ((uintptr_t)src & 15) == 0 &&
                     ((uintptr_t)hi & 15) == 0 && ((uintptr_t)lo & 15) == 0;
    if (vec) {
        const long long n = (long long)rows * (cols / 4);
        (void)launch_pdl(split_pair_vec_kernel, dim3(grid_stride_blocks(n)), dim3(256), (size_t)(0), st, 
            rows, cols / 4, reinterpret_cast<const float4*>(src), lds / 4, reinterpret_cast<float4*>(hi),
            reinterpret_cast<float4*>(lo), ldd / 4);
    } else {
        (void)launch_pdl(split_pair_kernel, dim3(grid_stride_blocks((long long)rows * cols)), dim3(256), (size_t)(0), st, rows, cols, src, lds, hi, lo,
                                                                                       ldd);
    }
    DLRM_LAUNCH_CHECK();
    return DLRM_OK;
}

dlrm_status launch_merge_pair(int rows, int cols, const float* hi, const float* lo, int lds, float* out, int ldo,
                              cudaStream_t st) {
    const long long n = (long long)rows * cols;
    if (n <= 0) return DLRM_OK;
    (void)launch_pdl(merge_pair_kernel, dim3(grid_stride_blocks(n)), dim3(256), (size_t)(0), st, rows, cols, hi, lo, lds, out, ldo);
    DLRM_LAUNCH_CHECK();
    return DLRM_OK;
}

dlrm_status launch_split_sum(int S, int N, int K, const float* part, int ldp, float* out, int ldo, cudaStream_t st) {
    const long long n = (long long)N * K;
    if (n == 0) return DLRM_OK;
    (void)launch_pdl(split_sum_kernel, dim3(grid_stride_blocks(n)), dim3(256), (size_t)(0), st, S, N, K, part, ldp, out, ldo);
    DLRM_LAUNCH_CHECK();
    return DLRM_OK;
}

// Columns of a weighted column sum (launch_colsum_w) per chunk; chunks of 512 rows, at most 128.
constexpr int CS_NW = 16;

dlrm_status launch_colsum_w(int M, int N, F32Pair A, const float* X, int ldx, int kx, bool ones, float* dW, int ldw,
                            float* db, float* scratch, cudaStream_t st) {
    const int P = colsum_chunks(M);
    const long long rows_per = ((long long)M + P - 1) / P;
    const dim3 grid((unsigned)((N + 127) / 128), (unsigned)P);
    const int nw = kx + (ones ? 1 : 0);
    int NW;
    if (nw <= 1) {
        (void)launch_pdl(colsum_w_kernel<1>, dim3(grid), dim3(32 * CS_WARPS(1)), (size_t)(0), st, M, N, A.hi, A.lo, A.ld, X, ldx, kx, ones, rows_per,
                                                              scratch);
        NW = 1;
    } else {
        (void)launch_pdl(colsum_w_kernel<CS_NW>, dim3(grid), dim3(32 * CS_WARPS(CS_NW)), (size_t)(0), st, M, N, A.hi, A.lo, A.ld, X, ldx, kx, ones,
                                                                      rows_per, scratch);
        NW = CS_NW;
    }
    DLRM_LAUNCH_CHECK();
    const long long outs = (long long)N * NW;
    (void)launch_pdl(colsum_w_final_kernel, dim3((int)((outs + 7) / 8 < 148 * 16 ? (outs + 7) / 8 : 148 * 16)), dim3(256), (size_t)(0), st, 
        P, N, NW, kx, ones, scratch, dW, ldw, db);
    DLRM_LAUNCH_CHECK();
    return DLRM_OK;
}

dlrm_status train_linear_fwd(int M, int N, int K, F32Pair x, F32Pair W, const float* b, float* y, float* y_lo,
                             int ldy, bool relu, uint32_t* relu_bits, ErrRecord* err, cudaStream_t st) {
    if (M == 0) return DLRM_OK;
    if (!relu) relu_bits = nullptr;
    if (relu && y_lo && tf32x3_supported(M, N, K, x, W))
        return tf32x3_fwd(M, N, K, x, W, b, y, y_lo, ldy, relu_bits, relu_bits_ld(N), err, st);
    if (K <= 16) {
        const dim3 grid((unsigned)((N + 127) / 128), (unsigned)((M + NARROW_ROWS - 1) / NARROW_ROWS));
        (void)launch_pdl(narrow_fwd_kernel, dim3(grid), dim3(128), (size_t)(0), st, M, N, K, x.hi, x.lo, x.ld, W.hi, W.lo, W.ld, b, relu, y, y_lo, ldy,
                                                relu_bits, relu_bits_ld(N));
        DLRM_LAUNCH_CHECK();
        return DLRM_OK;
    }
    if (N == 1 && !relu && !y_lo) {
        const long long blocks = (M + 7) / 8;
        (void)launch_pdl(gemv_rows_kernel, dim3((int)(blocks < 148 * 16 ? blocks : 148 * 16)), dim3(256), (size_t)(0), st, M, K, x.hi, x.lo, x.ld, W.hi,
                                                                                     W.lo, b, y);
        DLRM_LAUNCH_CHECK();
        return DLRM_OK;
    }
    if (relu)
        (void)launch_pdl(gemm_f32_kernel<false, false, EPI_BIAS_RELU, false>, dim3(grid_for(M, N, 1)), dim3(256), (size_t)(0), st, 
            M, N, K, x.hi, x.lo, x.ld, W.hi, W.lo, W.ld, b, nullptr, nullptr, 0, y, y_lo, ldy, K, 0);
    else
        (void)launch_pdl(gemm_f32_kernel<false, false, EPI_BIAS, false>, dim3(grid_for(M, N, 1)), dim3(256), (size_t)(0), st, 
            M, N, K, x.hi, x.lo, x.ld, W.hi, W.lo, W.ld, b, nullptr, nullptr, 0, y, y_lo, ldy, K, 0);
    DLRM_LAUNCH_CHECK();
    if (relu_bits) {
        const long long words = (long long)M * relu_bits_ld(N);
        (void)launch_pdl(relu_bits_kernel, dim3(grid_stride_blocks(words * 32)), dim3(256), (size_t)(0), st, M, N, y, y_lo, ldy, relu_bits,
                                                                         relu_bits_ld(N));
        DLRM_LAUNCH_CHECK();
    }
    return DLRM_OK;
}

dlrm_status train_linear_dgrad(int M, int N, int K, F32Pair dy, F32Pair W, F32Pair relu_of,
                               const uint32_t* relu_bits, float* dx, float* dx_lo, int lddx, float* csum,
                               bool* csum_done, ErrRecord* err, cudaStream_t st) {
    if (csum_done) *csum_done = false;
    if (M == 0) return DLRM_OK;
    const bool shape_ok = relu_of.hi ? (dx_lo && is_pair(relu_of)) : !dx_lo;
    if (shape_ok && tf32x3_supported(M, K, N, dy, W)) {
        float* cs = relu_of.hi ? csum : nullptr;
        dlrm_status r = tf32x3_dgrad(M, N, K, dy, W, relu_of, relu_of.hi ? relu_bits : nullptr, relu_bits_ld(K), dx,
                                     dx_lo, lddx, cs, err, st);
        if (!r && cs && csum_done) *csum_done = true;
        return r;
    }
    if (N == 1 && relu_of.hi && dx_lo && !dy.lo) {
        (void)launch_pdl(outer_mask_kernel, dim3(grid_stride_blocks((long long)M * K)), dim3(256), (size_t)(0), st, M, K, dy.hi, W.hi, W.lo, relu_of.hi,
                                                                               relu_of.lo, relu_of.ld, dx, dx_lo, lddx);
        DLRM_LAUNCH_CHECK();
        return DLRM_OK;
    }
    if (relu_of.hi)
        (void)launch_pdl(gemm_f32_kernel<false, true, EPI_MASK, false>, dim3(grid_for(M, K, 1)), dim3(256), (size_t)(0), st, 
            M, K, N, dy.hi, dy.lo, dy.ld, W.hi, W.lo, W.ld, nullptr, relu_of.hi, relu_of.lo, relu_of.ld, dx, dx_lo,
            lddx, N, 0);
    else
        (void)launch_pdl(gemm_f32_kernel<false, true, EPI_PLAIN, false>, dim3(grid_for(M, K, 1)), dim3(256), (size_t)(0), st, 
            M, K, N, dy.hi, dy.lo, dy.ld, W.hi, W.lo, W.ld, nullptr, nullptr, nullptr, 0, dx, dx_lo, lddx, N, 0);
    DLRM_LAUNCH_CHECK();
    return DLRM_OK;
}

size_t train_wgrad_scratch_floats(int N, int K, int M) {
    const size_t simt = (size_t)simt_wgrad_splits(N, K, M) * (size_t)N * (size_t)(K + 1);
    const size_t tc = tf32x3_wgrad_scratch_floats(N, K, M);
    const size_t cs = (size_t)colsum_chunks(M) * (size_t)(N > K ? N : K) * CS_NW;
    return simt > tc ? (simt > cs ? simt : cs) : (tc > cs ? tc : cs);
}

dlrm_status train_linear_wgrad(int M, int N, int K, F32Pair dy, F32Pair x, float* dW, int ldw, float* db,
                               const float* csum, float* scratch, ErrRecord* err, cudaStream_t st) {
    // dW[n][k] = sum_m dy[m][n] x[m][k]; db[n] = sum_m dy[m][n]
    if (N >= 16 && tf32x3_supported(N, K, M, dy, x)) {
        dlrm_status r = tf32x3_wgrad(M, N, K, dy, x, dW, ldw, scratch, err, st);
        if (r) return r;
        if (csum) {
            // bias gradient from the column sums per 32-row group that the data-gradient epilogue left
            const int G = (M + 31) / 32;
            (void)launch_pdl(csum_final_kernel, dim3((N + 7) / 8 < 148 * 8 ? (N + 7) / 8 : 148 * 8), dim3(256), (size_t)(0), st, G, N, csum, db);
            DLRM_LAUNCH_CHECK();
            return DLRM_OK;
        }
        // bias gradient: fixed-order column sums of dy (the split partials above are consumed by now)
        return launch_colsum_w(M, N, dy, nullptr, 0, 0, true, nullptr, 0, db, scratch, st);
    }
    if (K < CS_NW && !x.lo) {
        // narrow input (the 13 dense features): dW[n][k] and db[n] from one pass over dy
        return launch_colsum_w(M, N, dy, x.hi, x.ld, K, true, dW, ldw, db, scratch, st);
    }
    if (N == 1 && !dy.lo) {
        // one-column layer: dW[0][k] = sum_m x[m][k] dz[m], db[0] = sum_m dz[m]
        dlrm_status r = launch_colsum_w(M, K, x, dy.hi, dy.ld, 1, false, dW, 1, nullptr, scratch, st);
        if (r) return r;
        return launch_colsum_w(M, 1, dy, nullptr, 0, 0, true, nullptr, 0, db, scratch, st);
    }
    const int splits = simt_wgrad_splits(N, K, M);
    long long chunk = ((long long)M + splits - 1) / splits;
    chunk = (chunk + TK - 1) / TK * TK;
    const long long pstride = (long long)N * (K + 1);
    (void)launch_pdl(gemm_f32_kernel<true, true, EPI_PARTIAL, true>, dim3(grid_for(N, K + 1, splits)), dim3(256), (size_t)(0), st, 
        N, K, M, dy.hi, dy.lo, dy.ld, x.hi, x.lo, x.ld, nullptr, nullptr, nullptr, 0, scratch, nullptr, 0, chunk,
        pstride);
    DLRM_LAUNCH_CHECK();
    const long long n = pstride;
    (void)launch_pdl(wgrad_reduce_kernel, dim3(grid_stride_blocks(n)), dim3(256), (size_t)(0), st, splits, N, K, scratch, pstride, dW, ldw, db);
    DLRM_LAUNCH_CHECK();
    return DLRM_OK;
}

}  // namespace dlrm
