// Fully connected layers y = act(x W^T + b) of the bottom and top MLPs
// ("Deep Learning Recommendation Model (DLRM)", nadeemcite summary, Key Method
// Details: FC layers with ReLU; "DLRM", briansu.co, section 4, equation
// "Output": a sigmoid on the top MLP's output).
//
// This file holds the CUDA-core paths: a tiled FFMA GEMM used for fp32
// layers and for layers the tensor-core path does not take, and a
// warp-per-row GEMV for the single-logit last layer with its activation.
// Every kernel here is launched as a programmatic dependent and waits
// (pdl_wait) before its first access to global memory.
#include "common.cuh"
#include "kernels.cuh"

namespace dlrm {

template <int ACT>
__device__ __forceinline__ float activate(float v) {
    if constexpr (ACT == DLRM_ACT_RELU) return v > 0.f ? v : 0.f;
    if constexpr (ACT == DLRM_ACT_SIGMOID) return 1.f / (1.f + expf(-v));
    return v;
}

// 64 x 64 output tile per 256-thread block, 16-deep k slices through shared
// memory, 4 x 4 outputs per thread. Software-pipelined: the next slice's
// global loads are issued into registers before the current slice's
// multiply-adds, and the slices alternate between two shared buffers, so each
// slice costs one barrier and its load latency hides behind the arithmetic.
template <typename TA, typename TW, typename TC, int ACT>
__global__ void __launch_bounds__(256) linear_ffma_kernel(int M, int N, int K, const TA* __restrict__ A, int lda,
                                                          const TW* __restrict__ W, int ldw,
                                                          const float* __restrict__ bias, TC* __restrict__ C,
                                                          int ldc) {
    pdl_wait();
    constexpr int RM = 64, TM = 4;   // tile rows, output rows per thread
    __shared__ __align__(16) float As[2][16][RM + 4];
    __shared__ __align__(16) float Ws[2][16][64 + 4];
    const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
    const long long m0 = (long long)blockIdx.y * RM;
    const int n0 = blockIdx.x * 64;
    float acc[TM][4];
#pragma unroll
    for (int i = 0; i < TM; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = 0.f;
    // this thread's loads: row lr of the A and W tiles, k = k0 + lk .. k0 + lk + 3
    const int lr = threadIdx.x >> 2, lk = (threadIdx.x & 3) * 4;
    const long long gm = m0 + lr;
    const int gn = n0 + lr;
    float ra[4], rw[4];
    auto load = [&](int k0) {
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            const int gk = k0 + lk + e;
            ra[e] = (gm < M && gk < K) ? Cvt<TA>::to_f(A[gm * lda + gk]) : 0.f;
            rw[e] = (gn < N && gk < K) ? Cvt<TW>::to_f(W[(long long)gn * ldw + gk]) : 0.f;
        }
    };
    auto stage = [&](int b) {
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            As[b][lk + e][lr] = ra[e];
            Ws[b][lk + e][lr] = rw[e];
        }
    };
    load(0);
    stage(0);
    __syncthreads();
    int b = 0;
    for (int k0 = 0; k0 < K; k0 += 16, b ^= 1) {
        const bool more = k0 + 16 < K;
        if (more) load(k0 + 16);   // in flight during this slice's multiply-adds
#pragma unroll
        for (int kk = 0; kk < 16; ++kk) {
            const float4 a = *reinterpret_cast<const float4*>(&As[b][kk][ty * 4]);
            const float av[TM] = {a.x, a.y, a.z, a.w};
            const float4 w = *reinterpret_cast<const float4*>(&Ws[b][kk][tx * 4]);
            const float wv[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
            for (int i = 0; i < TM; ++i)
#pragma unroll
                for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(av[i], wv[j], acc[i][j]);
        }
        if (more) stage(b ^ 1);    // the other buffer: its last readers finished before the previous barrier
        __syncthreads();
    }
#pragma unroll
    for (int i = 0; i < TM; ++i) {
        const long long m = m0 + ty * TM + i;
        if (m >= M) continue;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const int n = n0 + tx * 4 + j;
            if (n < N) C[m * ldc + n] = Cvt<TC>::from_f(activate<ACT>(acc[i][j] + bias[n]));
        }
    }
}

// fp32 A and W (rows 16-byte aligned): RM x 64 output tile per 256-thread block (RM = 64, or 32 when the
// 64-row grid would leave more than half of the SMs idle), 32-deep k slices in a
// 3-stage shared-memory ring filled by cp.async (16-byte copies straight from global memory, zero-filled past
// M, N and K), so that two slices are always in flight while the block multiplies the third. Thread (ty, tx)
// owns rows ty + 16 i (i < RM / 16) and columns tx + 16 j (j < 4): its A and W reads are 16-byte vectors along k, the
// 16 W rows a warp reads fall in distinct bank groups (row stride 36 floats), and every output row is written
// by 16 consecutive threads.
namespace f32p {
constexpr int BK = 32, LDS = BK + 4, STAGES = 3;
constexpr int TILE_FLOATS = 64 * LDS;   // one 64-row tile; an RM-row A tile uses the first RM rows of it
constexpr int SMEM = STAGES * 2 * TILE_FLOATS * 4;
}  // namespace f32p

__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src, uint32_t src_bytes) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(src_bytes) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory"); }

template <typename TC, int ACT, int RM>
__global__ void __launch_bounds__(256) linear_f32_pipe_kernel(int M, int N, int K, const float* __restrict__ A,
                                                              int lda, const float* __restrict__ W, int ldw,
                                                              const float* __restrict__ bias, TC* __restrict__ C,
                                                              int ldc) {
    pdl_wait();
    using namespace f32p;
    constexpr int TM = RM / 16;   // output rows per thread
    extern __shared__ __align__(16) float fsm[];
    const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
    const long long m0 = (long long)blockIdx.y * RM;
    const int n0 = blockIdx.x * 64;
    const int nk = (K + BK - 1) / BK;
    const uint32_t sbase = (uint32_t)__cvta_generic_to_shared(fsm);
    // this thread's copies: rows lr and lr + 32 of both tiles, 16-byte column chunk lc of the slice
    const int lr = threadIdx.x >> 3, lc = (threadIdx.x & 7) * 4;
    auto issue = [&](int kt) {
        const int st = kt % STAGES;
        const int k = kt * BK + lc;
        const uint32_t bytes = k < K ? (uint32_t)(min(4, K - k) * 4) : 0u;
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            const int r = lr + 32 * h;
            const long long gm = m0 + r;
            const int gn = n0 + r;
            if (r < RM) {
                const uint32_t da = sbase + (uint32_t)(((st * 2) * TILE_FLOATS + r * LDS + lc) * 4);
                cp_async16(da, gm < M && bytes ? A + gm * lda + k : A, gm < M ? bytes : 0u);
            }
            const uint32_t dw = sbase + (uint32_t)(((st * 2 + 1) * TILE_FLOATS + r * LDS + lc) * 4);
            cp_async16(dw, gn < N && bytes ? W + (long long)gn * ldw + k : W, gn < N ? bytes : 0u);
        }
    };
    float acc[TM][4];
#pragma unroll
    for (int i = 0; i < TM; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = 0.f;
#pragma unroll
    for (int kt = 0; kt < STAGES - 1; ++kt) {
        if (kt < nk) issue(kt);
        cp_async_commit();
    }
    for (int kt = 0; kt < nk; ++kt) {
        cp_async_wait<STAGES - 2>();   // slice kt has landed (this thread's copies)
        __syncthreads();               // ... and every thread's; the slot refilled below was last read before this
        if (kt + STAGES - 1 < nk) issue(kt + STAGES - 1);
        cp_async_commit();
        const float* As = fsm + (kt % STAGES) * 2 * TILE_FLOATS;
        const float* Ws = As + TILE_FLOATS;
#pragma unroll
        for (int kk = 0; kk < BK; kk += 4) {
            float4 a[TM], w[4];
#pragma unroll
            for (int i = 0; i < TM; ++i) a[i] = *reinterpret_cast<const float4*>(As + (ty + 16 * i) * LDS + kk);
#pragma unroll
            for (int j = 0; j < 4; ++j) w[j] = *reinterpret_cast<const float4*>(Ws + (tx + 16 * j) * LDS + kk);
#pragma unroll
            for (int i = 0; i < TM; ++i)
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    float t = acc[i][j];
                    t = fmaf(a[i].x, w[j].x, t);
                    t = fmaf(a[i].y, w[j].y, t);
                    t = fmaf(a[i].z, w[j].z, t);
                    t = fmaf(a[i].w, w[j].w, t);
                    acc[i][j] = t;
                }
        }
    }
    cp_async_wait<0>();
#pragma unroll
    for (int i = 0; i < TM; ++i) {
        const long long m = m0 + ty + 16 * i;
        if (m >= M) continue;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const int n = n0 + tx + 16 * j;
            if (n < N) C[m * ldc + n] = Cvt<TC>::from_f(activate<ACT>(acc[i][j] + bias[n]));
        }
    }
}

template <typename TC, int ACT>
static void run_f32_pipe(int M, int N, int K, const float* A, int lda, const float* W, int ldw, const float* bias,
                         void* C, int ldc, cudaStream_t st) {
    int sms = 148, dev = 0;
    if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    if (2LL * ((N + 63) / 64) * ((M + 63) / 64) < sms) {
        auto kern = linear_f32_pipe_kernel<TC, ACT, 32>;
        cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, f32p::SMEM);
        const dim3 grid((N + 63) / 64, (M + 31) / 32);
        (void)launch_pdl(kern, grid, dim3(256), (size_t)f32p::SMEM, st, M, N, K, A, lda, W, ldw, bias,
                         static_cast<TC*>(C), ldc);
    } else {
        auto kern = linear_f32_pipe_kernel<TC, ACT, 64>;
        cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, f32p::SMEM);
        const dim3 grid((N + 63) / 64, (M + 63) / 64);
        (void)launch_pdl(kern, grid, dim3(256), (size_t)f32p::SMEM, st, M, N, K, A, lda, W, ldw, bias,
                         static_cast<TC*>(C), ldc);
    }
}

template <typename TC>
static void dispatch_f32_pipe(int M, int N, int K, const float* A, int lda, const float* W, int ldw,
                              const float* bias, void* C, int ldc, int act, cudaStream_t st) {
    if (act == DLRM_ACT_RELU) run_f32_pipe<TC, DLRM_ACT_RELU>(M, N, K, A, lda, W, ldw, bias, C, ldc, st);
    else if (act == DLRM_ACT_SIGMOID) run_f32_pipe<TC, DLRM_ACT_SIGMOID>(M, N, K, A, lda, W, ldw, bias, C, ldc, st);
    else run_f32_pipe<TC, DLRM_ACT_NONE>(M, N, K, A, lda, W, ldw, bias, C, ldc, st);
}

// N == 1: one warp per row.
template <typename TA, typename TW, int ACT>
__global__ void __launch_bounds__(256) gemv_kernel(int M, int K, const TA* __restrict__ A, int lda,
                                                   const TW* __restrict__ w, const float* __restrict__ bias,
                                                   float* __restrict__ y, int ldy) {
    pdl_wait();
    const long long row = (long long)blockIdx.x * 8 + (threadIdx.x >> 5);
    const int lane = threadIdx.x & 31;
    if (row >= M) return;
    const TA* a = A + row * lda;
    float s = 0.f;
    for (int k = lane; k < K; k += 32) s = fmaf(Cvt<TA>::to_f(a[k]), Cvt<TW>::to_f(w[k]), s);
    for (int o = 16; o; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
    if (lane == 0) y[row * ldy] = activate<ACT>(s + bias[0]);
}

template <typename TA, typename TW, typename TC, int ACT>
static void run_ffma(int M, int N, int K, const void* A, int lda, const void* W, int ldw, const float* bias, void* C,
                     int ldc, cudaStream_t st) {
    const dim3 grid((N + 63) / 64, (M + 63) / 64);
    (void)launch_pdl(linear_ffma_kernel<TA, TW, TC, ACT>, grid, dim3(256), 0, st, M, N, K, static_cast<const TA*>(A),
                     lda, static_cast<const TW*>(W), ldw, bias, static_cast<TC*>(C), ldc);
}

template <typename TA, typename TW, int ACT>
static void run_gemv(int M, int K, const void* A, int lda, const void* W, const float* bias, void* C, int ldc,
                     cudaStream_t st) {
    (void)launch_pdl(gemv_kernel<TA, TW, ACT>, dim3((M + 7) / 8), dim3(256), 0, st, M, K, static_cast<const TA*>(A),
                     lda, static_cast<const TW*>(W), bias, static_cast<float*>(C), ldc);
}

template <typename TA, typename TW, typename TC>
static void dispatch_act(int M, int N, int K, const void* A, int lda, const void* W, int ldw, const float* bias,
                         void* C, int ldc, int act, cudaStream_t st) {
    if (act == DLRM_ACT_RELU) run_ffma<TA, TW, TC, DLRM_ACT_RELU>(M, N, K, A, lda, W, ldw, bias, C, ldc, st);
    else if (act == DLRM_ACT_SIGMOID) run_ffma<TA, TW, TC, DLRM_ACT_SIGMOID>(M, N, K, A, lda, W, ldw, bias, C, ldc, st);
    else run_ffma<TA, TW, TC, DLRM_ACT_NONE>(M, N, K, A, lda, W, ldw, bias, C, ldc, st);
}

template <typename TA, typename TW>
static dlrm_status dispatch_out(int M, int N, int K, const void* A, int lda, const void* W, int ldw,
                                const float* bias, void* C, dlrm_dtype c_dt, int ldc, int act, cudaStream_t st) {
    if (N == 1 && c_dt == DLRM_F32) {
        if (act == DLRM_ACT_RELU) run_gemv<TA, TW, DLRM_ACT_RELU>(M, K, A, lda, W, bias, C, ldc, st);
        else if (act == DLRM_ACT_SIGMOID) run_gemv<TA, TW, DLRM_ACT_SIGMOID>(M, K, A, lda, W, bias, C, ldc, st);
        else run_gemv<TA, TW, DLRM_ACT_NONE>(M, K, A, lda, W, bias, C, ldc, st);
        return DLRM_OK;
    }
    switch (c_dt) {
        case DLRM_F32: dispatch_act<TA, TW, float>(M, N, K, A, lda, W, ldw, bias, C, ldc, act, st); break;
        case DLRM_BF16: dispatch_act<TA, TW, __nv_bfloat16>(M, N, K, A, lda, W, ldw, bias, C, ldc, act, st); break;
        case DLRM_F16: dispatch_act<TA, TW, __half>(M, N, K, A, lda, W, ldw, bias, C, ldc, act, st); break;
    }
    return DLRM_OK;
}

template <typename TA>
static dlrm_status dispatch_w(int M, int N, int K, const void* A, int lda, const void* W, dlrm_dtype w_dt, int ldw,
                              const float* bias, void* C, dlrm_dtype c_dt, int ldc, int act, cudaStream_t st) {
    switch (w_dt) {
        case DLRM_F32: return dispatch_out<TA, float>(M, N, K, A, lda, W, ldw, bias, C, c_dt, ldc, act, st);
        case DLRM_BF16: return dispatch_out<TA, __nv_bfloat16>(M, N, K, A, lda, W, ldw, bias, C, c_dt, ldc, act, st);
        case DLRM_F16: return dispatch_out<TA, __half>(M, N, K, A, lda, W, ldw, bias, C, c_dt, ldc, act, st);
    }
    return DLRM_ERR_UNSUPPORTED;
}

dlrm_status launch_linear_ffma(int M, int N, int K, const void* A, dlrm_dtype a_dt, int lda, const void* W,
                               dlrm_dtype w_dt, int ldw, const float* bias, void* C, dlrm_dtype c_dt, int ldc,
                               int act, cudaStream_t st) {
    // fp32 operands whose rows are 16-byte aligned: the cp.async pipeline
    if (a_dt == DLRM_F32 && w_dt == DLRM_F32 && N > 1 && lda % 4 == 0 && ldw % 4 == 0 &&
        !((uintptr_t)A & 15) && !((uintptr_t)W & 15)) {
        const float* a = static_cast<const float*>(A);
        const float* w = static_cast<const float*>(W);
        switch (c_dt) {
            case DLRM_F32: dispatch_f32_pipe<float>(M, N, K, a, lda, w, ldw, bias, C, ldc, act, st); break;
            case DLRM_BF16: dispatch_f32_pipe<__nv_bfloat16>(M, N, K, a, lda, w, ldw, bias, C, ldc, act, st); break;
            case DLRM_F16: dispatch_f32_pipe<__half>(M, N, K, a, lda, w, ldw, bias, C, ldc, act, st); break;
        }
        DLRM_LAUNCH_CHECK();
        return DLRM_OK;
    }
    dlrm_status r = DLRM_ERR_UNSUPPORTED;
    switch (a_dt) {
        case DLRM_F32: r = dispatch_w<float>(M, N, K, A, lda, W, w_dt, ldw, bias, C, c_dt, ldc, act, st); break;
        case DLRM_BF16: r = dispatch_w<__nv_bfloat16>(M, N, K, A, lda, W, w_dt, ldw, bias, C, c_dt, ldc, act, st); break;
        case DLRM_F16: r = dispatch_w<__half>(M, N, K, A, lda, W, w_dt, ldw, bias, C, c_dt, ldc, act, st); break;
    }
    if (r != DLRM_OK) return r;
    DLRM_LAUNCH_CHECK();
    return DLRM_OK;
}

// out[b][c] = in[b][c] converted to out_dt for c < K, 0 for K <= c < ldo.
template <typename TI, typename TO>
__global__ void convert_kernel(int B, int K, const TI* __restrict__ in, int ldi, TO* __restrict__ out, int ldo) {
    pdl_wait();
    const long long n = (long long)B * ldo;
    for (long long q = (long long)blockIdx.x * blockDim.x + threadIdx.x; q < n; q += (long long)gridDim.x * blockDim.x) {
        const long long b = q / ldo;
        const int c = (int)(q - b * ldo);
        out[q] = Cvt<TO>::from_f(c < K ? Cvt<TI>::to_f(in[b * ldi + c]) : 0.f);
    }
}

// One thread per row, 16-bit output rows written as 16-byte chunks (ldo % 8 == 0, 16-byte aligned rows):
// no per-element index division.
template <typename TI, typename TO>
__global__ void convert_rows_kernel(int B, int K, const TI* __restrict__ in, int ldi, TO* __restrict__ out, int ldo) {
    pdl_wait();
    for (int b = blockIdx.x * blockDim.x + threadIdx.x; b < B; b += gridDim.x * blockDim.x) {
        const TI* src = in + (long long)b * ldi;
        TO* dst = out + (long long)b * ldo;
        for (int c0 = 0; c0 < ldo; c0 += 8) {
            TO t[8];
#pragma unroll
            for (int e = 0; e < 8; ++e) t[e] = Cvt<TO>::from_f(c0 + e < K ? Cvt<TI>::to_f(src[c0 + e]) : 0.f);
            *reinterpret_cast<uint4*>(dst + c0) = *reinterpret_cast<const uint4*>(t);
        }
    }
}

template <typename TI>
static void convert_to(int B, int K, const void* in, int ldi, void* out, dlrm_dtype out_dt, int ldo, cudaStream_t st) {
    if (out_dt != DLRM_F32 && ldo % 8 == 0 && ((uintptr_t)out & 15) == 0) {
        const int blocks = (B + 255) / 256 < 148 * 8 ? (B + 255) / 256 : 148 * 8;
        const TI* i = static_cast<const TI*>(in);
        if (out_dt == DLRM_BF16)
            (void)launch_pdl(convert_rows_kernel<TI, __nv_bfloat16>, dim3(blocks), dim3(256), 0, st, B, K, i, ldi,
                             static_cast<__nv_bfloat16*>(out), ldo);
        else
            (void)launch_pdl(convert_rows_kernel<TI, __half>, dim3(blocks), dim3(256), 0, st, B, K, i, ldi,
                             static_cast<__half*>(out), ldo);
        return;
    }
    long long blocks = ((long long)B * ldo + 255) / 256;
    if (blocks > 148 * 16) blocks = 148 * 16;
    if (blocks < 1) blocks = 1;
    const TI* i = static_cast<const TI*>(in);
    if (out_dt == DLRM_BF16)
        (void)launch_pdl(convert_kernel<TI, __nv_bfloat16>, dim3((int)blocks), dim3(256), 0, st, B, K, i, ldi,
                         static_cast<__nv_bfloat16*>(out), ldo);
    else if (out_dt == DLRM_F16)
        (void)launch_pdl(convert_kernel<TI, __half>, dim3((int)blocks), dim3(256), 0, st, B, K, i, ldi,
                         static_cast<__half*>(out), ldo);
    else
        (void)launch_pdl(convert_kernel<TI, float>, dim3((int)blocks), dim3(256), 0, st, B, K, i, ldi,
                         static_cast<float*>(out), ldo);
}

dlrm_status launch_convert(int B, int K, const void* in, dlrm_dtype in_dt, int ldi, void* out, dlrm_dtype out_dt,
                           int ldo, cudaStream_t st) {
    if (B == 0) return DLRM_OK;
    if (in_dt == DLRM_F32) convert_to<float>(B, K, in, ldi, out, out_dt, ldo, st);
    else if (in_dt == DLRM_BF16) convert_to<__nv_bfloat16>(B, K, in, ldi, out, out_dt, ldo, st);
    else convert_to<__half>(B, K, in, ldi, out, out_dt, ldo, st);
    DLRM_LAUNCH_CHECK();
    return DLRM_OK;
}

dlrm_status launch_linear(int M, int N, int K, const void* A, dlrm_dtype a_dt, int lda, const void* W,
                          dlrm_dtype w_dt, int ldw, const float* bias, void* C, dlrm_dtype c_dt, int ldc, int act,
                          ErrRecord* err, cudaStream_t st) {
    if (M == 0) return DLRM_OK;
    if (N > 1 && linear_tc_supported(M, N, K, A, a_dt, lda, W, w_dt, ldw, bias, C, c_dt, ldc))
        return launch_linear_tc(M, N, K, A, a_dt, lda, W, ldw, bias, C, c_dt, ldc, act, err, st);
    return launch_linear_ffma(M, N, K, A, a_dt, lda, W, w_dt, ldw, bias, C, c_dt, ldc, act, st);
}

}  // namespace dlrm
