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
// Concat-only interaction for tables stored in the concat's dtype (embbag_cat_bulk.cu): each sample's row is
// assembled in shared memory from bulk-copied table rows and written with one bulk store.
bool embbag_cat_bulk_supported(dlrm_dtype dt, dlrm_dtype out_dt, int K, int d, int ld, const void* out,
                               long long total_rows);
dlrm_status launch_embbag_cat_bulk(const TableMeta& tm, const void* tables, dlrm_dtype dt, int K, int d, int B,
                                   const int32_t* offsets, const int32_t* indices, long long nnz,
                                   const float* x_dense, void* out, int ld, ErrRecord* err, cudaStream_t st);
bool embbag_interact_mma_supported(dlrm_dtype dt, int K, int d, int ld, const void* out, dlrm_dtype out_dt,
                                   long long total_rows);
dlrm_status launch_embbag_interact_mma(const TableMeta& tm, const void* tables, dlrm_dtype dt, int K, int d, int B,
                                       const int32_t* offsets, const int32_t* indices, long long nnz,
                                       const float* x_dense, void* out, int ld, dlrm_dtype out_dt, ErrRecord* err,
                                       cudaStream_t st);
// Many tables (K up to 128, bf16 tables and concat, d = 64 or 128): U-deep row gather and mma.sync Gram.
bool embbag_interact_wide_supported(dlrm_dtype dt, int K, int d, int ld, const void* out, dlrm_dtype out_dt);
dlrm_status launch_embbag_interact_wide(const TableMeta& tm, const void* tables, int K, int d, int B,
                                        const int32_t* offsets, const int32_t* indices, long long nnz,
                                        const float* x_dense, void* out, int ld, ErrRecord* err, cudaStream_t st);

// One fully connected layer: C[M][N] = act(A[M][K] W[N][K]^T + bias), fp32 accumulation.
// A has dtype a_dt (ld lda), W has dtype w_dt (ld ldw), C has dtype c_dt (ld ldc).
// Takes the tcgen05 path when linear_tc_supported(), else CUDA-core FFMA (or the N = 1 GEMV).
// err receives DLRM_ERR_TIMEOUT if a bounded wait of the tensor-core kernel gives up.
dlrm_status launch_linear(int M, int N, int K, const void* A, dlrm_dtype a_dt, int lda, const void* W,
                          dlrm_dtype w_dt, int ldw, const float* bias, void* C, dlrm_dtype c_dt, int ldc, int act,
                          ErrRecord* err, cudaStream_t st);

// Three bf16 layers in one tensor-core kernel (mlp3_tc.cu): fp32 input [B][ld_in] with dims[0] <= 16,
// h1 and h2 kept on chip, fp32 ReLU output [B][ld_out]; dims[1] <= 512, dims[2] <= 256, dims[3] <= 128, each a
// multiple of 64.
bool mlp3_tc_supported(const dlrm_mlp* m, int B, dlrm_dtype in_dt, int ld_in, const void* out, int ld_out,
                       int final_act);
dlrm_status launch_mlp3_tc(const dlrm_mlp* m, int B, const float* in, int ld_in, float* out, int ld_out, ErrRecord* err,
                           cudaStream_t st);
cudaError_t set_wait_polls_mlp3(long long polls);

// out[b][c] = in[b][c] (converted) for c < K, zero up to ldo.
// offsets[i] = sum of lengths[0..i) for i <= n, uint8 lengths (lengths.cu); scratch: lengths_scratch_ints(n) ints.
size_t lengths_scratch_ints(long long n);
dlrm_status launch_offsets_from_lengths(const uint8_t* lengths, long long n, int32_t* offsets, int* scratch,
                                        cudaStream_t st);
dlrm_status launch_convert(int B, int K, const void* in, dlrm_dtype in_dt, int ldi, void* out, dlrm_dtype out_dt,
                           int ldo, cudaStream_t st);

bool linear_tc_supported(int M, int N, int K, const void* A, dlrm_dtype a_dt, int lda, const void* W, dlrm_dtype w_dt,
                         int ldw, const float* bias, void* C, dlrm_dtype c_dt, int ldc);
dlrm_status launch_linear_tc(int M, int N, int K, const void* A, dlrm_dtype a_dt, int lda, const void* W, int ldw,
                             const float* bias, void* C, dlrm_dtype c_dt, int ldc, int act, ErrRecord* err,
                             cudaStream_t st);

// Concat-only interaction: out row b = [x_dense_b, e_1 .. e_K, zeros up to ld] (embbag.cu)
dlrm_status launch_embbag_cat(const TableMeta& tm, const void* tables, dlrm_dtype dt, int K, int d, int B,
                              const int32_t* offsets, const int32_t* indices, long long nnz, const float* x_dense,
                              void* out, int ld, dlrm_dtype out_dt, ErrRecord* err, cudaStream_t st);

// DLRM_U8ROW record bytes of a row of width d (quant.cu)
size_t u8row_bytes(int d);

// A hidden ReLU layer (N <= 256, M >= 4096, 16-bit) whose output feeds a one-column layer with a
// sigmoid: y[m] = sigmoid(relu(A W^T + bias)[m] . w_next + b_next), the hidden output never stored.
bool linear_tc_logit_supported(int M, int N, int K, const void* A, dlrm_dtype a_dt, int lda, const void* W,
                               dlrm_dtype w_dt, int ldw, const float* bias);
dlrm_status launch_linear_tc_logit(int M, int N, int K, const void* A, dlrm_dtype a_dt, int lda, const void* W,
                                   int ldw, const float* bias, const void* w_next, const float* b_next, float* y,
                                   ErrRecord* err, cudaStream_t st);

// ---- training (fp32)
// An fp32 matrix row-major with leading dimension ld, held either plain
// (lo == nullptr, value = hi) or as a 3xTF32 pair: hi = value with its 13 low
// mantissa bits cleared, lo = value - hi (value = hi + lo exactly).
struct F32Pair {
    const float* hi;
    const float* lo;
    int ld;
};

// Tensor-core 3xTF32 GEMMs (gemm_tf32.cu); operands must be pairs.
bool tf32x3_supported(int M, int N, int K, F32Pair a, F32Pair b);
// relu_bits (optional): the output's ReLU bitmask, bit j % 32 of word [m][j / 32], ldbits words per row.
dlrm_status tf32x3_fwd(int M, int N, int K, F32Pair x, F32Pair W, const float* bias, float* y_hi, float* y_lo,
                       int ldy, uint32_t* relu_bits, int ldbits, ErrRecord* err, cudaStream_t st);
// mask_bits (optional): the saved activation's ReLU bitmask, read instead of the pair; csum (optional):
// column sums of each 32-row group of the masked output, [ceil(M / 32)][K].
dlrm_status tf32x3_dgrad(int M, int N, int K, F32Pair dy, F32Pair W, F32Pair mask, const uint32_t* mask_bits,
                         int ldbits, float* dx_hi, float* dx_lo, int lddx, float* csum, ErrRecord* err,
                         cudaStream_t st);
int tf32x3_wgrad_splits(int N, int K, int M);
size_t tf32x3_wgrad_scratch_floats(int N, int K, int M);
dlrm_status tf32x3_wgrad(int M, int N, int K, F32Pair dy, F32Pair x, float* dW, int ldw, float* scratch,
                         ErrRecord* err, cudaStream_t st);
// C[i][j] = sum_r A(i, r) B(j, r); A(i, r) = A[i][r] (K-major) or A[r][i] (a_mn), likewise B
dlrm_status tf32x3_gemm(int I, int J, int R, F32Pair A, bool a_mn, F32Pair B, bool b_mn, float* C, int ldc,
                        float* scratch, ErrRecord* err, cudaStream_t st);

// CUDA-core fp32 GEMMs and helpers (train_gemm.cu). Inputs may be plain or
// pairs; y_lo / dx_lo non-null selects a pair output.
// ReLU bitmasks of saved activations: ceil(n / 32) words per row (bit j % 32 of word j / 32).
inline int relu_bits_ld(int n) { return (n + 31) / 32; }

// relu_bits (optional, with relu): the output's ReLU bitmask is written too.
dlrm_status train_linear_fwd(int M, int N, int K, F32Pair x, F32Pair W, const float* b, float* y, float* y_lo,
                             int ldy, bool relu, uint32_t* relu_bits, ErrRecord* err, cudaStream_t st);
// dx[m][k] = sum_n dy[m][n] W[n][k], zeroed where relu_of (post-ReLU value) <= 0 when relu_of.hi is given;
// relu_bits (optional) is relu_of's bitmask. If csum is given and *csum_done comes back true, csum holds
// the column sums of dx per 32-row group ([ceil(M / 32)][K]) for the next layer's bias gradient.
dlrm_status train_linear_dgrad(int M, int N, int K, F32Pair dy, F32Pair W, F32Pair relu_of,
                               const uint32_t* relu_bits, float* dx, float* dx_lo, int lddx, float* csum,
                               bool* csum_done, ErrRecord* err, cudaStream_t st);
size_t train_wgrad_scratch_floats(int N, int K, int M);
// dW[n][k] = sum_m dy[m][n] x[m][k]; db[n] = sum_m dy[m][n] (from csum, the column sums of dy per
// 32-row group, when given)
dlrm_status train_linear_wgrad(int M, int N, int K, F32Pair dy, F32Pair x, float* dW, int ldw, float* db,
                               const float* csum, float* scratch, ErrRecord* err, cudaStream_t st);
// hi/lo pair of a plain [rows][cols] matrix
dlrm_status launch_split_pair(int rows, int cols, const float* src, int lds, float* hi, float* lo, int ldd,
                              cudaStream_t st);
// plain[r][c] = hi[r][c] + lo[r][c]
dlrm_status launch_merge_pair(int rows, int cols, const float* hi, const float* lo, int lds, float* out, int ldo,
                              cudaStream_t st);
// out[n][k] = sum_{z < S} part[z][n][k] in increasing z (part split stride N * ldp)
dlrm_status launch_split_sum(int S, int N, int K, const float* part, int ldp, float* out, int ldo, cudaStream_t st);

// Warp-per-sample fp32 interaction of the training step with the gather fused in (interact_tc.cu):
// fp32 tables, K = 26, d in {64, 128}. The forward reads the bags itself (counting skipped indices and
// bad bags in err), forms the Gram as 3xTF32 on the tensor cores and writes the concat as a TF32 pair;
// the backward gathers the same rows again and writes dx_dense (pair, ReLU-masked) and dE [B][K][d]
// from the CUDA cores.
bool interact_tc_supported(int K, int d, long long total_rows, int ldc);
dlrm_status launch_interact_fwd_tc(const TableMeta& tm, const float* tables, int K, int d, int B,
                                   const int32_t* offsets, const int32_t* indices, long long nnz, F32Pair x_dense,
                                   float* concat_hi, float* concat_lo, int ldc, ErrRecord* err, cudaStream_t st);
dlrm_status launch_interact_bwd_tc(const TableMeta& tm, const float* tables, int K, int d, int B,
                                   const int32_t* offsets, const int32_t* indices, long long nnz, F32Pair x_dense,
                                   const float* dconcat, int ldc, float* dx_hi, float* dx_lo, int lddx, float* dE,
                                   ErrRecord* err, cudaStream_t st);

dlrm_status launch_bce(int B, const float* z, const float* y, float* dz, float* y_hat, float* partial, float* loss,
                       cudaStream_t st);
size_t interact_bwd_smem(int K, int d);
// dx_dense receives the gradient w.r.t. the pre-activation of the bottom MLP's last (ReLU) layer.
dlrm_status launch_interact_bwd(int B, int K, int d, const float* x_dense, const float* E, const float* dconcat,
                                int ldc, float* dx_dense, float* dE, cudaStream_t st);

constexpr int SPARSE_PIECE = 64;   // occurrences summed per warp before the per-row combine

// Byte offsets of the sparse-update arrays inside the gradient buffer.
struct SparseLayout {
    long long cap;
    size_t counts, bag_len, occ_off, keys[2], vals[2], hist, hist_off, head, seg_id, seg_start, seg_row, seg_pieces,
        piece_base, piece_seg, partial, scan_sums, total;
};
SparseLayout sparse_layout(long long KB, long long nnz, int d);
int radix_passes(long long total_rows);
dlrm_status launch_sparse_prepare(int K, int B, const TableMeta& tm, long long total_rows, const int32_t* offsets,
                                  const int32_t* indices, long long nnz, char* base, const SparseLayout& L,
                                  ErrRecord* err, int* sorted_buf, cudaStream_t st);
dlrm_status launch_sparse_apply(int d, const char* base, const SparseLayout& L, int sorted_buf, const float* dE,
                                float lr, float* table, float* grad_out, uint32_t* rows_out, int32_t* n_rows_out,
                                cudaStream_t st);
dlrm_status launch_sgd(long long n, float lr, float* w, const float* g, cudaStream_t st);
size_t train_workspace_size(const dlrm_tables* T, const dlrm_mlp* bot, const dlrm_mlp* top, int B);
// Test hook behind dlrm_set_wait_polls: the first-wait bound of each file's kernels on the current device.
cudaError_t set_wait_polls_gemm_tc(long long polls);
cudaError_t set_wait_polls_embbag_mma(long long polls);
cudaError_t set_wait_polls_embbag_cat(long long polls);
cudaError_t set_wait_polls_interact_tc(long long polls);
// Every host-side check of dlrm_forward (cat = false) or dlrm_forward_cat (cat = true), ws_bytes included.
dlrm_status forward_check(const dlrm_tables* T, const dlrm_mlp* bot, const dlrm_mlp* top, int B, const float* dense,
                          const int32_t* offsets, const int32_t* indices, int64_t nnz, const float* y_hat,
                          const void* ws, size_t ws_bytes, bool cat);

}  // namespace dlrm
