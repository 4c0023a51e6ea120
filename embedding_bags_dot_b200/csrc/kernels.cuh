// Launchers shared between the kernel files and the C ABI layer.
#pragma once

#include "common.cuh"

namespace dlrm {

bool gather_supported(int d, dlrm_dtype dt);
size_t interact_smem_per_sample(int K, int d);

dlrm_status launch_embbag(const TableMeta& tm, const void* tables, dlrm_dtype dt, int K, int d, int B,
                          const int32_t* offsets, const int32_t* indices, long long nnz, float* pooled,
                          int32_t* bag_len, ErrRecord* err, cudaStream_t st);

dlrm_status launch_interact(int B, int K, int d, const float* x_dense, const float* pooled, void* out, int ld,
                            dlrm_dtype out_dt, cudaStream_t st);

dlrm_status launch_embbag_interact(const TableMeta& tm, const void* tables, dlrm_dtype dt, int K, int d, int B,
                                   const int32_t* offsets, const int32_t* indices, long long nnz,
                                   const float* x_dense, void* out, int ld, dlrm_dtype out_dt, ErrRecord* err,
                                   cudaStream_t st);

// Tensor-core (mma.sync) variant of launch_embbag_interact for bf16 tables with
// d in {32, 64, 128, 256} and K + 2 <= 64; launch_embbag_interact picks it when supported.
bool embbag_interact_mma_supported(dlrm_dtype dt, int K, int d, int ld, const void* out, dlrm_dtype out_dt,
                                   long long total_rows);
dlrm_status launch_embbag_interact_mma(const TableMeta& tm, const void* tables, int K, int d, int B,
                                       const int32_t* offsets, const int32_t* indices, long long nnz,
                                       const float* x_dense, void* out, int ld, dlrm_dtype out_dt, ErrRecord* err,
                                       cudaStream_t st);

// One fully connected layer: C[M][N] = act(A[M][K] W[N][K]^T + bias), fp32 accumulation.
// A has dtype a_dt (ld lda), W has dtype w_dt (ld ldw), C has dtype c_dt (ld ldc).
// Takes the tcgen05 path when linear_tc_supported(), else CUDA-core FFMA (or the N = 1 GEMV).
// err receives DLRM_ERR_TIMEOUT if a bounded wait of the tensor-core kernel gives up.
dlrm_status launch_linear(int M, int N, int K, const void* A, dlrm_dtype a_dt, int lda, const void* W,
                          dlrm_dtype w_dt, int ldw, const float* bias, void* C, dlrm_dtype c_dt, int ldc, int act,
                          ErrRecord* err, cudaStream_t st);

bool linear_tc_supported(int M, int N, int K, const void* A, dlrm_dtype a_dt, int lda, const void* W, dlrm_dtype w_dt,
                         int ldw, void* C, dlrm_dtype c_dt, int ldc);
dlrm_status launch_linear_tc(int M, int N, int K, const void* A, dlrm_dtype a_dt, int lda, const void* W, int ldw,
                             const float* bias, void* C, dlrm_dtype c_dt, int ldc, int act, ErrRecord* err,
                             cudaStream_t st);

}  // namespace dlrm
