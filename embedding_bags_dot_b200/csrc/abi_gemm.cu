// extern "C" fp32 GEMM on the tensor cores (3xTF32): splits both operands into
// TF32 (hi, lo) pairs in the caller's workspace, then runs the SM-pair
// tcgen05 kernel of gemm_tf32.cu.
#include "common.cuh"
#include "kernels.cuh"

using namespace dlrm;

namespace {

struct GemmWs {
    size_t a[2], b[2], scratch, total;
    int lda4, ldb4;
};

bool args_ok(int I, int J, int R) { return I >= 1 && J >= 1 && R >= 1; }

GemmWs gemm_ws(int I, int J, int R, int a_mn, int b_mn) {
    GemmWs W;
    size_t off = DLRM_ERR_RECORD_BYTES;
    auto take = [&](size_t bytes) {
        const size_t o = off;
        off = align_up(off + bytes, 256);
        return o;
    };
    const int a_rows = a_mn ? R : I, a_cols = a_mn ? I : R;
    const int b_rows = b_mn ? R : J, b_cols = b_mn ? J : R;
    W.lda4 = dlrm_ld(a_cols, DLRM_F32);
    W.ldb4 = dlrm_ld(b_cols, DLRM_F32);
    for (int h = 0; h < 2; ++h) W.a[h] = take(sizeof(float) * (size_t)a_rows * W.lda4);
    for (int h = 0; h < 2; ++h) W.b[h] = take(sizeof(float) * (size_t)b_rows * W.ldb4);
    W.scratch = take(sizeof(float) * tf32x3_wgrad_scratch_floats(I, J, R));
    W.total = off;
    return W;
}

}  // namespace

extern "C" {

size_t dlrm_gemm_f32_workspace_size(int I, int J, int R, int a_mn, int b_mn) {
    if (!args_ok(I, J, R)) return 0;
    return gemm_ws(I, J, R, a_mn, b_mn).total;
}

dlrm_status dlrm_gemm_f32(int I, int J, int R, const float* A, int lda, int a_mn, const float* B, int ldb, int b_mn,
                          float* C, int ldc, void* ws, size_t ws_bytes, dlrm_stream stream) {
    if (!args_ok(I, J, R) || !A || !B || !C) return DLRM_ERR_INVALID_ARG;
    const int a_cols = a_mn ? I : R, b_cols = b_mn ? J : R;
    if (lda < a_cols || ldb < b_cols || ldc < J || ldc % 4 || ((uintptr_t)C & 15)) return DLRM_ERR_INVALID_ARG;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    const GemmWs W = gemm_ws(I, J, R, a_mn, b_mn);
    if (!ws || ((uintptr_t)ws & 15) || ws_bytes < W.total) return DLRM_ERR_WORKSPACE;
    char* w = static_cast<char*>(ws);
    auto F = [&](size_t o) { return reinterpret_cast<float*>(w + o); };
    ErrRecord* err = reinterpret_cast<ErrRecord*>(w);
    dlrm_status r;
    if ((r = launch_split_pair(a_mn ? R : I, a_cols, A, lda, F(W.a[0]), F(W.a[1]), W.lda4, st)) ||
        (r = launch_split_pair(b_mn ? R : J, b_cols, B, ldb, F(W.b[0]), F(W.b[1]), W.ldb4, st)))
        return r;
    const F32Pair a{F(W.a[0]), F(W.a[1]), W.lda4}, b{F(W.b[0]), F(W.b[1]), W.ldb4};
    r = tf32x3_gemm(I, J, R, a, a_mn != 0, b, b_mn != 0, C, ldc, F(W.scratch), err, st);
    return r;
}

dlrm_status dlrm_tf32_split(int rows, int cols, const float* src, int lds, float* hi, float* lo, int ldd,
                            dlrm_stream stream) {
    if (rows < 0 || cols < 0 || lds < cols || ldd < cols) return DLRM_ERR_INVALID_ARG;
    if ((long long)rows * cols > 0 && (!src || !hi || !lo)) return DLRM_ERR_INVALID_ARG;
    return launch_split_pair(rows, cols, src, lds, hi, lo, ldd, reinterpret_cast<cudaStream_t>(stream));
}

size_t dlrm_gemm_tf32x3_workspace_size(int I, int J, int R) {
    if (!args_ok(I, J, R)) return 0;
    return align_up(DLRM_ERR_RECORD_BYTES, 256) + sizeof(float) * tf32x3_wgrad_scratch_floats(I, J, R);
}

dlrm_status dlrm_gemm_tf32x3(int I, int J, int R, const float* A_hi, const float* A_lo, int lda, int a_mn,
                             const float* B_hi, const float* B_lo, int ldb, int b_mn, float* C, int ldc, void* ws,
                             size_t ws_bytes, dlrm_stream stream) {
    if (!args_ok(I, J, R) || !A_hi || !A_lo || !B_hi || !B_lo || !C) return DLRM_ERR_INVALID_ARG;
    const int a_cols = a_mn ? I : R, b_cols = b_mn ? J : R;
    if (lda < a_cols || ldb < b_cols || ldc < J || lda % 4 || ldb % 4 || ldc % 4) return DLRM_ERR_INVALID_ARG;
    const uintptr_t al = (uintptr_t)A_hi | (uintptr_t)A_lo | (uintptr_t)B_hi | (uintptr_t)B_lo | (uintptr_t)C;
    if (al & 15) return DLRM_ERR_INVALID_ARG;
    if (!ws || ((uintptr_t)ws & 15) || ws_bytes < dlrm_gemm_tf32x3_workspace_size(I, J, R)) return DLRM_ERR_WORKSPACE;
    char* w = static_cast<char*>(ws);
    return tf32x3_gemm(I, J, R, F32Pair{A_hi, A_lo, lda}, a_mn != 0, F32Pair{B_hi, B_lo, ldb}, b_mn != 0, C, ldc,
                       reinterpret_cast<float*>(w + align_up(DLRM_ERR_RECORD_BYTES, 256)),
                       reinterpret_cast<ErrRecord*>(w), reinterpret_cast<cudaStream_t>(stream));
}

}  // extern "C"
