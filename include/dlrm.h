/*
 * dlrm.h -- C ABI of the B200 (sm_100a) DLRM hot-path library, libdlrm.so.
 *
 * The operations follow the DLRM architecture as two pages state it:
 *   [N] "Deep Learning Recommendation Model (DLRM)" (nadeemcite summary):
 *       Core Idea; Key Method Details.
 *   [S] "DLRM" (briansu.co/recsys/dlrm): section 3 "How it works";
 *       section 4 "Key equations" (equations "Interaction" and "Output");
 *       section 6 "Limitations & trade-offs".
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 *  - Pointers are DEVICE pointers unless marked "host". The caller owns every
 *    buffer (tables, weights, inputs, outputs, workspace); the library never
 *    allocates device memory and keeps no pointer after a call returns.
 *  - Every call is asynchronous on `stream` (NULL = legacy default stream).
 *    Its kernels are launched as programmatic dependents (each may start its
 *    setup while the previous kernel on the stream finishes, and waits for
 *    that kernel's completion before touching global memory), so the calls
 *    keep plain stream order with any other work on the stream and can be
 *    captured in CUDA graphs.
 *    Host-detectable argument errors return a status before anything is
 *    launched. Errors found on the device (an index outside its table, bag
 *    offsets that decrease or leave [0, nnz]) never trap: the offending
 *    index contributes nothing, the offending bag pools to zero, and the
 *    event is recorded in the error record at the start of the workspace;
 *    dlrm_check_error() reads and clears it.
 *  - Every caller-provided scratch buffer (workspace `ws`, gradient buffer
 *    `grads`) comes with its size in bytes (`ws_bytes`, `grads_bytes`). A
 *    buffer smaller than the call needs (the matching *_size query) or not
 *    16-byte aligned is refused with DLRM_ERR_WORKSPACE before anything is
 *    launched; the library never writes past the size it is given.
 *  - Bags are CSR, table-major: bag (k, b) of table k and sample b holds
 *    indices[offsets[k*B + b] .. offsets[k*B + b + 1]), each a row id local to
 *    table k. offsets has K*B + 1 int32 entries; nnz < 2^31.
 *  - All K tables live in one contiguous row-major buffer; table k starts at
 *    row base_k = rows[0] + ... + rows[k-1]. Rows are d elements wide (all
 *    features share d: [N] Key Method Details, [S] section 6).
 *  - A matrix with a leading dimension `ld` stores row i at element i*ld;
 *    ld must make every row start on a 16-byte boundary (dlrm_ld()). Padding
 *    columns are never read by the library; outputs zero their padding.
 *  - Limits: 1 <= K <= DLRM_MAX_TABLES; 1 <= d, and d*sizeof(elem) <= 2048
 *    when d*sizeof(elem) is a multiple of 16, else d <= 256.
 */
#ifndef DLRM_H
#define DLRM_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define DLRM_MAX_TABLES 256
#define DLRM_MAX_LAYERS 16
#define DLRM_ERR_RECORD_BYTES 256

typedef struct CUstream_st* dlrm_stream; /* a cudaStream_t */

typedef enum {
    DLRM_OK = 0,
    DLRM_ERR_INVALID_ARG = 1,   /* null pointer, bad size, misaligned pointer or leading dimension */
    DLRM_ERR_UNSUPPORTED = 2,   /* a valid request this build does not implement (dtype, d, K) */
    DLRM_ERR_INDEX_OOB = 3,     /* device: some index was outside [0, m_k); it was skipped */
    DLRM_ERR_BAD_OFFSETS = 4,   /* device: some bag had decreasing offsets or left [0, nnz]; it pooled to 0 */
    DLRM_ERR_TIMEOUT = 5,       /* device: a bounded wait gave up */
    DLRM_ERR_CUDA = 6,          /* a CUDA runtime call failed (launch, copy) */
    DLRM_ERR_WORKSPACE = 7      /* workspace too small or misaligned */
} dlrm_status;

/* DLRM_U8ROW (tables only): row-wise 8-bit quantised rows. Each row is one
 * record of dlrm_row_bytes(d, DLRM_U8ROW) = d + 8 bytes rounded up to a
 * multiple of 16: d uint8 codes q[c], then fp32 scale s, fp32 offset m, then
 * zero padding; the value of column c is s * q[c] + m. The pages call the
 * lookup memory-bound ("DLRM", briansu.co, section 6) and the tables the bulk
 * of the parameters ([N] Key Method Details); storing rows at ~1.1 bytes per
 * value instead of 2 cuts the gathered bytes. Supported by the fused gather +
 * interaction path (dlrm_embbag_interact_fwd, dlrm_forward) for d = 64 or 128;
 * other entry points return DLRM_ERR_UNSUPPORTED for it. */
typedef enum { DLRM_F32 = 0, DLRM_F16 = 1, DLRM_BF16 = 2, DLRM_U8ROW = 3 } dlrm_dtype;

typedef enum { DLRM_ACT_NONE = 0, DLRM_ACT_RELU = 1, DLRM_ACT_SIGMOID = 2 } dlrm_act;

/* K embedding tables of m_k x d ([N] Key Method Details). */
typedef struct {
    void* data;             /* device, all tables, row-major, 16-byte aligned */
    const int64_t* rows;    /* host, K row counts m_k >= 1 */
    int K;
    int d;
    dlrm_dtype dt;          /* storage dtype of the table values; pooling accumulates in fp32 */
} dlrm_tables;

/* A stack of fully connected layers y = act(x W^T + b) ([N] Key Method Details). */
typedef struct {
    int n_layers;           /* 1 .. DLRM_MAX_LAYERS */
    const int* dims;        /* host, n_layers + 1 widths */
    void* const* W;         /* host array of device pointers: W[l] is [dims[l+1]][dlrm_ld(dims[l], dt)] */
    float* const* b;        /* host array of device pointers: b[l] is fp32 [dims[l+1]] */
    dlrm_dtype dt;          /* dtype of weights and of hidden activations */
} dlrm_mlp;

/* Smallest leading dimension >= n whose rows are 16-byte multiples for dtype dt. */
int dlrm_ld(int n, dlrm_dtype dt);

/* Bytes of one table row of width d stored as dt (DLRM_U8ROW: the record). */
size_t dlrm_row_bytes(int d, dlrm_dtype dt);

/* Row-wise 8-bit quantisation of `rows` rows of width d (src: device,
 * row-major [rows][d], DLRM_F32 or DLRM_BF16) into DLRM_U8ROW records at dst
 * (device, 16-byte aligned, rows * dlrm_row_bytes(d, DLRM_U8ROW) bytes). Per
 * row, in IEEE fp32 with round-to-nearest: lo = min_c v, hi = max_c v,
 * s = (hi - lo) / 255, q[c] = rint((v[c] - lo) / s) clamped to [0, 255]
 * (q = 0 when s = 0), m = lo. No counterpart in the pages, which describe no
 * storage format; this is the standard min/max affine form. */
dlrm_status dlrm_quantize_rows_u8(const void* src, dlrm_dtype src_dt, int64_t rows, int d, void* dst,
                                  dlrm_stream stream);

/* Number of kernels this library has launched in the calling process so far
 * (all devices, all streams). Used to count launches inside a timed region. */
uint64_t dlrm_launch_count(void);

/* Test hook, no counterpart in the pages: sets, on the current device, how
 * many times the first bounded wait of the row-gathering kernels (the bulk
 * copies of a sample's rows), the ordinary waits of the single-CTA
 * tensor-core layer (batches below 4,096 rows) and those of the one-kernel
 * three-layer MLP (the bf16 bottom MLP) poll before giving up;
 * polls < 0 restores the defaults (about a second). A test sets 0 to make
 * those waits run out at once and checks that the call returns, that
 * dlrm_check_error reports DLRM_ERR_TIMEOUT, and that the next call (after
 * restoring) is correct. After giving up, a kernel still waits with the full
 * bound for the copies it has in flight, frees its tensor memory and returns;
 * outputs of the samples or tiles it did not finish are undefined. Not for
 * production use; synchronise the device before and after calling it. */
dlrm_status dlrm_set_wait_polls(int64_t polls);

/* Human-readable name of a status code (static string). */
const char* dlrm_status_str(dlrm_status s);

/* Bytes of device workspace dlrm_forward (training = 0) or dlrm_backward
 * (training = 1) needs for batch B. Also enough for every single-step entry
 * point on the same model and batch. The first DLRM_ERR_RECORD_BYTES bytes
 * hold the error record: zero the whole workspace once after allocating it. */
size_t dlrm_workspace_size(const dlrm_tables* T, const dlrm_mlp* bot, const dlrm_mlp* top, int B, int training);

/* Reads the error record of `ws` (synchronising `stream`), clears it, and
 * returns DLRM_ERR_BAD_OFFSETS if any bag had bad offsets, else
 * DLRM_ERR_INDEX_OOB if any index was out of range, else DLRM_ERR_TIMEOUT if
 * a bounded wait gave up, else DLRM_OK. If `info` (host, 3 entries) is not
 * NULL it receives {flags, skipped indices, bad bags}. */
dlrm_status dlrm_check_error(void* ws, size_t ws_bytes, dlrm_stream stream, int64_t* info);

/* Sum-pooled embedding bags ([S] section 3: each sparse feature looks up a
 * row of its own table; a bag of several ids sums their rows, an empty bag
 * gives zeros).
 *   pooled   out, fp32 [B][K][d]
 *   bag_len  out, optional (may be NULL): int32 [K*B], end - start of each bag
 *            (0 for a bag with bad offsets)
 *   ws       workspace holding the error record (ws_bytes >= DLRM_ERR_RECORD_BYTES) */
dlrm_status dlrm_embbag_fwd(const dlrm_tables* T, int B, const int32_t* offsets, const int32_t* indices,
                            int64_t nnz, float* pooled, int32_t* bag_len, void* ws, size_t ws_bytes,
                            dlrm_stream stream);

/* Pairwise dot-product interaction and concat ([S] section 4, equations
 * "Interaction" and "Output"; [N] Core Idea: self-interactions excluded).
 * With X = [x_dense; e_1; ...; e_K] ((K+1) x d), writes per sample the row
 *   [x_dense (d values), Z_10, Z_20, Z_21, Z_30, ..., Z_K(K-1)],  Z_ij = <X_i, X_j>,
 * i.e. d + K(K+1)/2 values, then zeros up to ld.
 *   x_dense  fp32 [B][d];  pooled fp32 [B][K][d]
 *   concat   out, [B][ld] of out_dt, ld >= d + K(K+1)/2 */
dlrm_status dlrm_interact_fwd(int B, int K, int d, const float* x_dense, const float* pooled,
                              void* concat, int ld, dlrm_dtype out_dt, dlrm_stream stream);

/* dlrm_embbag_fwd fused with dlrm_interact_fwd: the pooled vectors stay on
 * chip and only the concat rows are written. Same arguments and errors. */
dlrm_status dlrm_embbag_interact_fwd(const dlrm_tables* T, int B, const int32_t* offsets, const int32_t* indices,
                                     int64_t nnz, const float* x_dense, void* concat, int ld, dlrm_dtype out_dt,
                                     void* ws, size_t ws_bytes, dlrm_stream stream);

/* MLP forward ([N] Key Method Details: FC layers with ReLU). ReLU after every
 * hidden layer; after the last layer `final_act` (none, ReLU or sigmoid).
 *   in    [B][ld_in] of in_dt, dims[0] logical columns
 *   out   out, fp32 [B][ld_out], dims[n_layers] logical columns
 *   ws    16-byte aligned, ws_bytes >= dlrm_mlp_workspace_size(mlp, B, in_dt)
 *         (dlrm_workspace_size of a model with this MLP as top or bottom is
 *         enough); the hidden activations live there. A smaller ws_bytes is
 *         refused with DLRM_ERR_WORKSPACE before any launch.
 * Three bf16 layers on fp32 input with final_act ReLU (the bottom MLP), with
 * dims[0] <= 16 and dims[1..3] multiples of 64 up to 512 / 256 / 128, run as
 * one kernel whose hidden activations stay on chip (same roundings: input and
 * hidden outputs to bf16, fp32 accumulation). Padding columns of a weight row
 * (between dims[l] and its leading dimension) are never read there. */
dlrm_status dlrm_mlp_fwd(const dlrm_mlp* mlp, int B, const void* in, dlrm_dtype in_dt, int ld_in,
                         float* out, int ld_out, int final_act, void* ws, size_t ws_bytes, dlrm_stream stream);

/* Bytes of workspace dlrm_mlp_fwd needs for this MLP, batch and input dtype:
 * the error record, one or two buffers of the widest hidden-layer output and,
 * when in_dt differs from a 16-bit MLP dtype, the converted input.
 * 0 for an invalid MLP, B < 0 or an invalid in_dt. */
size_t dlrm_mlp_workspace_size(const dlrm_mlp* mlp, int B, dlrm_dtype in_dt);

/* Whole forward pass ([S] sections 3-4):
 *   y_hat = sigmoid(top([x_dense, vec(Z)])),  x_dense = bottom(dense) with ReLU after every bottom layer,
 * hidden top layers with ReLU, last top layer linear (dims must end in 1).
 *   dense  fp32 [B][bot->dims[0]];  y_hat out, fp32 [B]
 *   ws     ws_bytes >= dlrm_workspace_size(T, bot, top, B, 0) */
dlrm_status dlrm_forward(const dlrm_tables* T, const dlrm_mlp* bot, const dlrm_mlp* top, int B, const float* dense,
                         const int32_t* offsets, const int32_t* indices, int64_t nnz, float* y_hat,
                         void* ws, size_t ws_bytes, dlrm_stream stream);

/* dlrm_forward with the bags given by their lengths instead of CSR offsets
 * (the pages fix no input format; this is a compact form of the same bags):
 *   lengths  uint8 [K * B], bag (k, b) at k * B + b (the order of the
 *            offsets), each bag's index count (at most 255); the bags'
 *            indices follow one another in `indices` in that order.
 * The offsets are derived on the device into the workspace (prefix sums), so
 * a caller copying inputs from host memory moves 1 byte per bag instead of 4.
 * The result is identical to dlrm_forward on offsets[i] = sum of
 * lengths[0..i). Lengths that do not add up to nnz are caught like bad offsets.
 * Workspace: dlrm_workspace_size(T, bot, top, B, 0). */
dlrm_status dlrm_forward_lengths(const dlrm_tables* T, const dlrm_mlp* bot, const dlrm_mlp* top, int B,
                                 const float* dense, const uint8_t* lengths, const int32_t* indices, int64_t nnz,
                                 float* y_hat, void* ws, size_t ws_bytes, dlrm_stream stream);

/* offsets[i] = sum_{j < i} lengths[j] for 0 <= i <= n (int32 out, device
 * pointers, the scan dlrm_forward_lengths runs). ws: 16-byte aligned,
 * dlrm_offsets_from_lengths_workspace_size(n) bytes (error record, then the
 * scan's chunk sums). The total must stay below 2^31. */
size_t dlrm_offsets_from_lengths_workspace_size(int64_t n);
dlrm_status dlrm_offsets_from_lengths(const uint8_t* lengths, int64_t n, int32_t* offsets, void* ws,
                                      size_t ws_bytes, dlrm_stream stream);

/* ------------------------------------------------------------ training step
 * fp32 tables and MLPs only (DLRM_ERR_UNSUPPORTED otherwise); d % 4 == 0.
 * The pages state the loss ([N] Key Method Details: binary cross-entropy);
 * the gradients are the calculus of the forward definition and the update is
 * plain SGD, w <- w - lr * grad, applied to the MLP parameters and to the
 * embedding rows the batch touched (no other row is written). */

/* Bytes of the gradient buffer for batch B with nnz indices. No zeroing needed. */
size_t dlrm_grads_size(const dlrm_tables* T, const dlrm_mlp* bot, const dlrm_mlp* top, int B, int64_t nnz);

/* Byte offsets inside the gradient buffer (host arrays of n_layers entries; any may be NULL):
 * dW[l] is fp32 [dims[l+1]][dlrm_ld(dims[l], DLRM_F32)], db[l] fp32 [dims[l+1]],
 * dE fp32 [B][K][d] (gradient of each pooled bag), loss one fp32. */
dlrm_status dlrm_grads_offsets(const dlrm_tables* T, const dlrm_mlp* bot, const dlrm_mlp* top, int B, int64_t nnz,
                               size_t* bot_dW, size_t* bot_db, size_t* top_dW, size_t* top_db, size_t* dE,
                               size_t* loss);

/* Forward (as dlrm_forward, keeping every activation in `ws`, which must
 * come from dlrm_workspace_size(..., training = 1)), then the mean BCE loss
 * against labels (fp32 [B] of 0/1), then the backward pass: batch-summed
 * gradients of the mean loss for every MLP weight and bias, the gradient of
 * every pooled bag, and the occurrences of the batch sorted by table row
 * (stable, so equal rows keep occurrence order). loss (device, 1 float) and
 * y_hat (device, fp32 [B]) are optional outputs. Bit-reproducible.
 * Skipped (out-of-range) indices and bags with bad offsets are handled as in
 * dlrm_forward and counted once per call in the error record at the start of
 * `ws` (read with dlrm_check_error). grads_bytes must be at least
 * dlrm_grads_size(T, bot, top, B, nnz) and ws_bytes at least
 * dlrm_workspace_size(T, bot, top, B, 1). */
dlrm_status dlrm_backward(const dlrm_tables* T, const dlrm_mlp* bot, const dlrm_mlp* top, int B, const float* dense,
                          const int32_t* offsets, const int32_t* indices, int64_t nnz, const float* labels,
                          float* loss, float* y_hat, void* grads, size_t grads_bytes, void* ws, size_t ws_bytes,
                          dlrm_stream stream);

/* SGD step from a gradient buffer filled by dlrm_backward on the same batch
 * shape: every table row the batch touched gets T[r] -= lr * g_r, where g_r
 * sums the gradients of the bags that use row r (once per occurrence) in
 * occurrence order; untouched rows are not written. Then W -= lr * dW and
 * b -= lr * db for every MLP layer. n_touched (device int32, optional)
 * receives the number of distinct rows updated. grads_bytes: as dlrm_backward. */
dlrm_status dlrm_sparse_sgd(const dlrm_tables* T, const dlrm_mlp* bot, const dlrm_mlp* top, int B, int64_t nnz,
                            float lr, void* grads, size_t grads_bytes, int32_t* n_touched, dlrm_stream stream);

/* The per-row embedding gradients dlrm_sparse_sgd would apply, without
 * applying them: rows (device uint32 [nnz]) gets the touched rows as global
 * row ids (base_k + r) in increasing order, row_grads (device fp32 [nnz][d])
 * their summed gradients, n_rows (device int32) their count. grads_bytes:
 * as dlrm_backward. */
dlrm_status dlrm_embedding_row_grads(const dlrm_tables* T, const dlrm_mlp* bot, const dlrm_mlp* top, int B,
                                     int64_t nnz, const void* grads, size_t grads_bytes, uint32_t* rows,
                                     float* row_grads, int32_t* n_rows, dlrm_stream stream);

/* Concat-only interaction, the alternative the pages set DLRM against
 * ("Deep Learning Recommendation Model (DLRM)", Key Method Details: Wide &
 * Deep concatenates embeddings without explicit interactions; "DLRM",
 * briansu.co, section 3: variants swap the interaction layer and keep the
 * sparse/dense skeleton). Row b of concat ([B][ld], out_dt, ld >= d (K + 1))
 * becomes [x_dense_b, e_1, ..., e_K, zeros up to ld] with e_k the sum-pooled
 * bag (k, b); x_dense fp32 [B][d]. Bags, errors and dtypes as
 * dlrm_embbag_interact_fwd (DLRM_U8ROW tables: DLRM_ERR_UNSUPPORTED). */
dlrm_status dlrm_embbag_cat_fwd(const dlrm_tables* T, int B, const int32_t* offsets, const int32_t* indices,
                                int64_t nnz, const float* x_dense, void* concat, int ld, dlrm_dtype out_dt, void* ws,
                                size_t ws_bytes, dlrm_stream stream);

/* dlrm_forward with the concat-only interaction: top->dims[0] must be
 * d (K + 1). Workspace: dlrm_workspace_size(T, bot, top, B, 0). */
dlrm_status dlrm_forward_cat(const dlrm_tables* T, const dlrm_mlp* bot, const dlrm_mlp* top, int B, const float* dense,
                             const int32_t* offsets, const int32_t* indices, int64_t nnz, float* y_hat, void* ws,
                             size_t ws_bytes, dlrm_stream stream);

/* fp32 GEMM of the training step, on the tensor cores at fp32 accuracy
 * (the matrix products of the fully connected layers, "Deep Learning
 * Recommendation Model (DLRM)", Key Method Details: bottom and top MLPs, and
 * their gradients by the chain rule):
 *   C[i][j] = sum_{r < R} A(i, r) B(j, r)        i < I, j < J
 * A(i, r) = A[i*lda + r] (a_mn = 0) or A[r*lda + i] (a_mn = 1); B likewise
 * with b_mn. All pointers are device fp32, 16-byte aligned; lda, ldb, ldc
 * are multiples of 4 (ldc >= J). Each operand is split in `ws` into a TF32
 * pair (hi = value with its 13 low mantissa bits cleared, lo = value - hi)
 * and the product is summed as A_lo B_hi + A_hi B_lo + A_hi B_hi in fp32
 * (error about 2^-20 of sum_r |A(i,r) B(j,r)|). Long reductions are cut into
 * shape-determined r-ranges added in a fixed order: bit-reproducible.
 * ws: 16-byte aligned, ws_bytes >= dlrm_gemm_f32_workspace_size(...), caller-owned.
 * Returns DLRM_ERR_INVALID_ARG (sizes < 1, null, misaligned, ld),
 * DLRM_ERR_WORKSPACE (ws null, misaligned or short), DLRM_ERR_UNSUPPORTED (no
 * tensor-map support in the driver); device timeouts land in the error
 * record read by dlrm_check_error. */
size_t dlrm_gemm_f32_workspace_size(int I, int J, int R, int a_mn, int b_mn);
dlrm_status dlrm_gemm_f32(int I, int J, int R, const float* A, int lda, int a_mn, const float* B, int ldb, int b_mn,
                          float* C, int ldc, void* ws, size_t ws_bytes, dlrm_stream stream);

/* The two halves of dlrm_gemm_f32, for callers that keep operands in pair
 * form (as the training step does for every activation and gradient).
 * dlrm_tf32_split: hi[r][c] = src[r][c] rounded to the nearest TF32 value,
 * lo[r][c] = src[r][c] - hi[r][c] (exact), for r < rows, c < cols; device
 * fp32 pointers, leading dimensions in elements (lds >= cols, ldd >= cols).
 * dlrm_gemm_tf32x3: the product of dlrm_gemm_f32 from pairs (A_hi, A_lo)
 * and (B_hi, B_lo) that share the layout and leading dimension given; all
 * pointers 16-byte aligned, lda/ldb/ldc multiples of 4. ws: 16-byte aligned,
 * dlrm_gemm_tf32x3_workspace_size(I, J, R) bytes (error record and the
 * partial sums of long reductions). Errors as dlrm_gemm_f32. */
dlrm_status dlrm_tf32_split(int rows, int cols, const float* src, int lds, float* hi, float* lo, int ldd,
                            dlrm_stream stream);
size_t dlrm_gemm_tf32x3_workspace_size(int I, int J, int R);
dlrm_status dlrm_gemm_tf32x3(int I, int J, int R, const float* A_hi, const float* A_lo, int lda, int a_mn,
                             const float* B_hi, const float* B_lo, int ldb, int b_mn, float* C, int ldc, void* ws,
                             size_t ws_bytes, dlrm_stream stream);

/* ------------------------------------------------- table-wise model parallelism
 * The pages' system keeps the embedding tables model-parallel and the fully
 * connected layers data-parallel, with an all-to-all of the lookup results
 * between the two (arXiv 1906.00091 index page, Abstract; the
 * science.uptrusthq.com citation snippet on all-to-all communication of the
 * embedding lookups; "DLRM", briansu.co, section 5). Each rank owns a
 * contiguous range of tables, pools its own tables' bags for the whole
 * batch (dlrm_embbag_fwd), and the caller's collective (NCCL all-to-all)
 * sends each rank the rows of its batch shard. These calls place the
 * received blocks and apply the owner's sparse update.
 *
 * dlrm_pooled_assemble: parts[p] (device, fp32 [B][n_tables[p]][d]) holds
 * tables first_table[p] .. first_table[p] + n_tables[p] - 1; the parts must
 * tile 0 .. K-1 in order (first_table[0] = 0, each next part starting where
 * the previous ends). out (device, fp32 [B][K][d]) receives every part in
 * its columns. first_table, n_tables and parts are host arrays of n_parts
 * entries. Strided device-to-device copies on `stream`, no kernel.
 * dlrm_pooled_split: the inverse (in [B][K][d] -> parts), for the gradients
 * of the pooled vectors on their way back to the owners.
 * DLRM_ERR_INVALID_ARG for parts that do not tile 0 .. K-1 or null pointers. */
dlrm_status dlrm_pooled_assemble(int B, int K, int d, int n_parts, const int* first_table, const int* n_tables,
                                 const float* const* parts, float* out, dlrm_stream stream);
dlrm_status dlrm_pooled_split(int B, int K, int d, int n_parts, const int* first_table, const int* n_tables,
                              const float* in, float* const* parts, dlrm_stream stream);

/* The data-parallel half of a sharded training step, for one rank's batch
 * shard: dlrm_backward with the pooled vectors given instead of tables and
 * bags. pooled: device fp32 [B][K][d], 16-byte aligned (the vectors the
 * all-to-all brought, placed by dlrm_pooled_assemble). The forward (bottom
 * MLP, interaction, top MLP, sigmoid), the mean BCE loss over these B samples
 * and the backward run as in dlrm_backward; grads receives every MLP
 * gradient and, at the dE offset, the gradient of every pooled vector
 * [B][K][d] (to be split per owner with dlrm_pooled_split and sent back). No
 * row of any table is read or written. Offsets inside grads:
 * dlrm_grads_pooled_offsets (dense_end: the MLP gradients occupy bytes
 * [0, dense_end), one contiguous range for the data-parallel all-reduce).
 * Sizes: grads_bytes >= dlrm_grads_pooled_size(...), ws_bytes >=
 * dlrm_backward_pooled_workspace_size(...). fp32 MLPs, d % 4 == 0. */
size_t dlrm_backward_pooled_workspace_size(int K, int d, const dlrm_mlp* bot, const dlrm_mlp* top, int B);
size_t dlrm_grads_pooled_size(int K, int d, const dlrm_mlp* bot, const dlrm_mlp* top, int B);
dlrm_status dlrm_grads_pooled_offsets(int K, int d, const dlrm_mlp* bot, const dlrm_mlp* top, int B, size_t* bot_dW,
                                      size_t* bot_db, size_t* top_dW, size_t* top_db, size_t* dE, size_t* loss,
                                      size_t* dense_end);
dlrm_status dlrm_backward_pooled(int K, int d, const dlrm_mlp* bot, const dlrm_mlp* top, int B, const float* dense,
                                 const float* pooled, const float* labels, float* loss, float* y_hat, void* grads,
                                 size_t grads_bytes, void* ws, size_t ws_bytes, dlrm_stream stream);
/* W -= lr * dW and b -= lr * db for every layer of both MLPs, from a
 * gradient buffer laid out by dlrm_grads_pooled_offsets (grads_bytes >=
 * dense_end). */
dlrm_status dlrm_mlp_sgd(int K, int d, const dlrm_mlp* bot, const dlrm_mlp* top, int B, float lr, const void* grads,
                         size_t grads_bytes, dlrm_stream stream);

/* The owner's half of the sparse SGD step (the update dlrm_sparse_sgd applies
 * to the embedding rows), from the gradient of every pooled bag of its own
 * tables: T[r] -= lr * g_r for every row r a valid index of the batch
 * touches, with g_r = sum of dE[b][k] over the occurrences of r in bag (k, b),
 * added in occurrence order (bit-reproducible); untouched rows are not
 * written. fp32 tables only (d % 4 == 0); bags as dlrm_embbag_fwd (skipped
 * indices and bad bags contribute nothing). dE: device fp32 [B][K][d], 16-byte
 * aligned. scratch: 16-byte aligned, scratch_bytes >=
 * dlrm_embbag_sgd_scratch_size(T, B, nnz) (error record, then the sort and
 * segment arrays). n_touched (device int32, optional): rows updated. */
size_t dlrm_embbag_sgd_scratch_size(const dlrm_tables* T, int B, int64_t nnz);
dlrm_status dlrm_embbag_sgd(const dlrm_tables* T, int B, const int32_t* offsets, const int32_t* indices, int64_t nnz,
                            const float* dE, float lr, void* scratch, size_t scratch_bytes, int32_t* n_touched,
                            dlrm_stream stream);

/* Size of the device scratch array that dlrm_forward_noalloc uses (32 MiB). */
#define DLRM_NOALLOC_SCRATCH_BYTES (32u << 20)

/* dlrm_forward for callers that cannot allocate device memory. The pages
 * describe no counterpart: this is a deployment convenience, not part of the
 * method.
 *
 * Some callers are not allowed to call cudaMalloc: a plugin inside a host
 * application or serving runtime that owns all device memory and hands the
 * plugin only its input and output buffers; a latency-bound request path on
 * which an allocation, and the device-wide synchronisation that
 * cudaMalloc/cudaFree may cause, is not acceptable; a plain C caller with no
 * device allocator. This entry point takes the same inputs and outputs as
 * dlrm_forward but no workspace: its scratch is one fixed array of
 * DLRM_NOALLOC_SCRATCH_BYTES compiled into the library, which every GPU that
 * loads the library holds until the process exits. It calls no cudaMalloc,
 * cudaFree or other allocating routine.
 *
 *  - Limit: dlrm_workspace_size(T, bot, top, B, 0) must not exceed
 *    DLRM_NOALLOC_SCRATCH_BYTES; larger requests return DLRM_ERR_WORKSPACE
 *    before anything is launched (split the batch, or use dlrm_forward).
 *  - Set-up: the first call on each device looks up the array's device
 *    address (with that device current). Make that first call before any
 *    stream capture.
 *  - Sharing: every call on a device uses the same array, which keeps the
 *    previous call's contents. Calls whose work overlaps on the GPU (other
 *    streams, other host threads) race on it; order them on one stream or
 *    serialise them.
 *  - Errors: every argument check of dlrm_forward runs first, and a refused
 *    call returns the status dlrm_forward would return, having queued
 *    nothing and written neither the array nor err_flags. Device-detected
 *    input errors are handled as in dlrm_forward (skipped index, empty bag).
 *    The error record is cleared at the start of each accepted call; if
 *    err_flags (device, optional) is not NULL it receives this call's flags
 *    once the call's work completes: bit 0 = an index was out of range,
 *    bit 1 = a bag had bad offsets. On any status other than DLRM_OK,
 *    err_flags is left as it was. */
dlrm_status dlrm_forward_noalloc(const dlrm_tables* T, const dlrm_mlp* bot, const dlrm_mlp* top, int B,
                                 const float* dense, const int32_t* offsets, const int32_t* indices, int64_t nnz,
                                 float* y_hat, uint32_t* err_flags, dlrm_stream stream);

#ifdef __cplusplus
}
#endif

#endif /* DLRM_H */
