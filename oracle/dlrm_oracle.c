/*
 * dlrm_oracle.c -- plain fp64 CPU oracle for the DLRM hot path.
 *
 * TEST INFRASTRUCTURE. Only the tests, the package's smoke check and the
 * benchmark's CPU-baseline leg may load this code. The CUDA library shares no
 * code with it and never calls it.
 *
 * What it computes, and where the pages define it:
 *   - embedding bags: each categorical feature owns an m_k x d table, all
 *     tables share d ("Deep Learning Recommendation Model (DLRM)",
 *     nadeemcite summary, Key Method Details; "DLRM", briansu.co, section 6).
 *     A sparse feature looks up a row of its own table ("DLRM", briansu.co,
 *     section 3); a bag of several ids sums their rows, an empty bag gives 0.
 *   - bottom MLP: FC layers with ReLU mapping the dense features to d
 *     (nadeemcite summary, Key Method Details). ReLU follows every layer.
 *   - interaction: Z = tril(X X^T) over X = [x_dense; e_1; ...; e_K]
 *     ("DLRM", briansu.co, section 4, equation "Interaction") with
 *     self-interactions left out (nadeemcite summary, Core Idea and Key Method
 *     Details: n(n-1)/2 values for n vectors). Order: (1,0),(2,0),(2,1),(3,0)...
 *   - concat [x_dense, vec(Z)] and top MLP then sigmoid ("DLRM", briansu.co,
 *     section 4, equation "Output"); hidden top layers use ReLU, the last one is
 *     linear so that the sigmoid sees the raw logit.
 *   - BCE loss, mean over the batch (nadeemcite summary, Key Method Details),
 *     written as softplus(z) - y z.
 *   - backward and SGD: the pages state none; the gradients below are the
 *     calculus of the forward definition, and SGD is w <- w - lr * grad.
 *
 *   - row-wise 8-bit tables (the storage the fused gather path also reads):
 *     the pages fix no format; the reading used is the min/max affine form
 *     per row, computed in fp32 exactly as the library's quantiser specifies
 *     (so both sides take the same integer decisions), and dequantised here
 *     in fp64 as s q + m.
 *
 * Arithmetic is fp64 throughout (except the quantiser's fp32 codes). Inputs arrive already widened to fp64
 * (exactly) by the caller. Weights are [out][in] row-major with no padding.
 * Invalid indices (outside [0, m_k)) are skipped and counted; a bag whose
 * offsets are decreasing or outside [0, nnz] pools to zero and is counted.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

int oracle_threads(void) {
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

void oracle_set_threads(int n) {
#ifdef _OPENMP
    if (n > 0) omp_set_num_threads(n);
#else
    (void)n;
#endif
}

/* ------------------------------------------------------------------ bags */

/* Sum one bag of table k into out[d]. Returns (number of skipped indices) and
 * sets *bad = 1 when the bag's offsets are unusable. *len gets end - start. */
static long pool_one_bag(int k, int B, int b, int d, long nnz, const int64_t* rows, const int64_t* base,
                         const double* tables, const int32_t* offsets, const int32_t* indices,
                         double* out, int32_t* len, int* bad) {
    long oob = 0;
    int64_t start = offsets[(int64_t)k * B + b];
    int64_t end = offsets[(int64_t)k * B + b + 1];
    for (int t = 0; t < d; ++t) out[t] = 0.0;
    *bad = 0;
    *len = (int32_t)(end - start);
    if (start < 0 || end < start || end > nnz) {
        *bad = 1;
        *len = 0;
        return 0;
    }
    for (int64_t p = start; p < end; ++p) {
        int64_t r = indices[p];
        if (r < 0 || r >= rows[k]) { ++oob; continue; }
        const double* row = tables + (base[k] + r) * d;
        for (int t = 0; t < d; ++t) out[t] += row[t];
    }
    return oob;
}

static void table_bases(int K, const int64_t* rows, int64_t* base) {
    int64_t acc = 0;
    for (int k = 0; k < K; ++k) { base[k] = acc; acc += rows[k]; }
}

/* pooled: [B][K][d]; bag_len: [K*B] (table-major like offsets); counts[0] =
 * skipped indices, counts[1] = bags with bad offsets. */
void oracle_embbag(int K, int B, int d, long nnz, const int64_t* rows, const double* tables,
                   const int32_t* offsets, const int32_t* indices,
                   double* pooled, int32_t* bag_len, long* counts) {
    int64_t* base = (int64_t*)malloc(sizeof(int64_t) * (K > 0 ? K : 1));
    table_bases(K, rows, base);
    long oob = 0, badn = 0;
    for (int b = 0; b < B; ++b) {
        for (int k = 0; k < K; ++k) {
            int bad;
            oob += pool_one_bag(k, B, b, d, nnz, rows, base, tables, offsets, indices,
                                pooled + ((int64_t)b * K + k) * d, bag_len + (int64_t)k * B + b, &bad);
            badn += bad;
        }
    }
    counts[0] = oob;
    counts[1] = badn;
    free(base);
}

/* ----------------------------------------------------------- interaction */

/* One sample: X rows are x_dense then e_1..e_K. Writes d + K(K+1)/2 values:
 * x_dense, then Z_ij = <X_i, X_j> for i = 1..K, j = 0..i-1. */
static void interact_one(int K, int d, const double* x_dense, const double* e, double* out) {
    for (int t = 0; t < d; ++t) out[t] = x_dense[t];
    int p = d;
    for (int i = 1; i <= K; ++i) {
        const double* xi = e + (int64_t)(i - 1) * d;
        for (int j = 0; j < i; ++j) {
            const double* xj = (j == 0) ? x_dense : e + (int64_t)(j - 1) * d;
            double s = 0.0;
            for (int t = 0; t < d; ++t) s += xi[t] * xj[t];
            out[p++] = s;
        }
    }
}

/* x_dense [B][d], pooled [B][K][d] -> concat [B][d + K(K+1)/2]. */
void oracle_interact(int B, int K, int d, const double* x_dense, const double* pooled, double* concat) {
    int width = d + K * (K + 1) / 2;
    for (int b = 0; b < B; ++b)
        interact_one(K, d, x_dense + (int64_t)b * d, pooled + (int64_t)b * K * d, concat + (int64_t)b * width);
}

/* -------------------------------------------------------------------- MLP */

/* y[out] = act(W x + b) for one sample; W [n_out][n_in]. */
static void linear_one(int n_in, int n_out, const double* W, const double* bias, const double* x, double* y, int relu) {
    for (int o = 0; o < n_out; ++o) {
        double s = bias[o];
        const double* w = W + (int64_t)o * n_in;
        for (int i = 0; i < n_in; ++i) s += w[i] * x[i];
        y[o] = (relu && s < 0.0) ? 0.0 : s;
    }
}

/* Whole MLP on a batch. dims[0..n_layers]; W[l] is [dims[l+1]][dims[l]].
 * relu_last selects ReLU after the final layer. out: [B][dims[n_layers]]. */
void oracle_mlp(int n_layers, const int* dims, const double* const* W, const double* const* bias,
                int B, const double* in, double* out, int relu_last) {
    int maxw = 0;
    for (int l = 0; l <= n_layers; ++l) if (dims[l] > maxw) maxw = dims[l];
#pragma omp parallel
    {
        double* a = (double*)malloc(sizeof(double) * maxw);
        double* c = (double*)malloc(sizeof(double) * maxw);
#pragma omp for schedule(static)
        for (int b = 0; b < B; ++b) {
            memcpy(a, in + (int64_t)b * dims[0], sizeof(double) * dims[0]);
            for (int l = 0; l < n_layers; ++l) {
                int relu = (l < n_layers - 1) || relu_last;
                linear_one(dims[l], dims[l + 1], W[l], bias[l], a, c, relu);
                double* t = a; a = c; c = t;
            }
            memcpy(out + (int64_t)b * dims[n_layers], a, sizeof(double) * dims[n_layers]);
        }
        free(a);
        free(c);
    }
}

static double sigmoid(double z) { return 1.0 / (1.0 + exp(-z)); }

/* ---------------------------------------------------------------- forward */

typedef struct {
    int K, d, n_bot, n_top;       /* tables, width, bottom layers, top layers */
    const int* bot_dims;          /* n_bot + 1 widths, bot_dims[0] = dense features, last = d */
    const int* top_dims;          /* n_top + 1 widths, top_dims[0] = d + K(K+1)/2, last = 1 */
    const double* const* bot_W; const double* const* bot_b;
    const double* const* top_W; const double* const* top_b;
    const int64_t* rows;          /* K row counts */
    const double* tables;         /* all tables, row-major, concatenated */
} oracle_model;

/* y_hat[b] = sigmoid(top([x_dense, vec(Z)])); logits optional [B]; counts as oracle_embbag. */
void oracle_forward(const oracle_model* M, int B, long nnz, const double* dense,
                    const int32_t* offsets, const int32_t* indices,
                    double* y_hat, double* logits, long* counts) {
    int K = M->K, d = M->d;
    int width = d + K * (K + 1) / 2;
    int maxw = width;
    for (int l = 0; l <= M->n_bot; ++l) if (M->bot_dims[l] > maxw) maxw = M->bot_dims[l];
    for (int l = 0; l <= M->n_top; ++l) if (M->top_dims[l] > maxw) maxw = M->top_dims[l];
    int64_t* base = (int64_t*)malloc(sizeof(int64_t) * (K > 0 ? K : 1));
    table_bases(K, M->rows, base);
    long oob = 0, badn = 0;
#pragma omp parallel reduction(+ : oob, badn)
    {
        double* a = (double*)malloc(sizeof(double) * maxw);
        double* c = (double*)malloc(sizeof(double) * maxw);
        double* xd = (double*)malloc(sizeof(double) * d);
        double* e = (double*)malloc(sizeof(double) * (size_t)(K > 0 ? K : 1) * d);
#pragma omp for schedule(dynamic, 16)
        for (int b = 0; b < B; ++b) {
            /* bottom MLP, ReLU after every layer */
            memcpy(a, dense + (int64_t)b * M->bot_dims[0], sizeof(double) * M->bot_dims[0]);
            for (int l = 0; l < M->n_bot; ++l) {
                linear_one(M->bot_dims[l], M->bot_dims[l + 1], M->bot_W[l], M->bot_b[l], a, c, 1);
                double* t = a; a = c; c = t;
            }
            memcpy(xd, a, sizeof(double) * d);
            /* pooled bags */
            for (int k = 0; k < K; ++k) {
                int bad; int32_t len;
                oob += pool_one_bag(k, B, b, d, nnz, M->rows, base, M->tables, offsets, indices, e + (int64_t)k * d, &len, &bad);
                badn += bad;
            }
            /* interaction + concat */
            interact_one(K, d, xd, e, a);
            /* top MLP: ReLU on hidden layers, last layer linear */
            for (int l = 0; l < M->n_top; ++l) {
                linear_one(M->top_dims[l], M->top_dims[l + 1], M->top_W[l], M->top_b[l], a, c, l < M->n_top - 1);
                double* t = a; a = c; c = t;
            }
            if (logits) logits[b] = a[0];
            y_hat[b] = sigmoid(a[0]);
        }
        free(a); free(c); free(xd); free(e);
    }
    counts[0] = oob;
    counts[1] = badn;
    free(base);
}

/* --------------------------------------------------------------- training */

/* Mean BCE over the batch in logit form: L = (1/B) sum softplus(z) - y z. */
double oracle_bce(int B, const double* z, const double* y) {
    double s = 0.0;
    for (int b = 0; b < B; ++b) {
        double sp = (z[b] > 0.0) ? z[b] + log1p(exp(-z[b])) : log1p(exp(z[b]));
        s += sp - y[b] * z[b];
    }
    return s / B;
}

/* Backward of one linear layer for the batch.
 *   A   [B][n_in]   layer input
 *   Y   [B][n_out]  layer output after its activation (used for the ReLU mask)
 *   dY  [B][n_out]  gradient w.r.t. the output (after activation); overwritten
 *                   with the gradient w.r.t. the pre-activation when relu != 0
 *   dW  [n_out][n_in], db [n_out]: summed over the batch
 *   dA  [B][n_in]   gradient w.r.t. the input (may be NULL)
 * ReLU'(0) is taken as 0. */
static void linear_backward(int B, int n_in, int n_out, const double* W, const double* A, const double* Y,
                            double* dY, double* dW, double* db, double* dA, int relu) {
    if (relu) {
        for (int64_t q = 0; q < (int64_t)B * n_out; ++q)
            if (!(Y[q] > 0.0)) dY[q] = 0.0;
    }
#pragma omp parallel for schedule(static)
    for (int o = 0; o < n_out; ++o) {
        double sb = 0.0;
        for (int b = 0; b < B; ++b) sb += dY[(int64_t)b * n_out + o];
        db[o] = sb;
        for (int i = 0; i < n_in; ++i) {
            double s = 0.0;
            for (int b = 0; b < B; ++b) s += dY[(int64_t)b * n_out + o] * A[(int64_t)b * n_in + i];
            dW[(int64_t)o * n_in + i] = s;
        }
    }
    if (dA) {
#pragma omp parallel for schedule(static)
        for (int b = 0; b < B; ++b) {
            for (int i = 0; i < n_in; ++i) {
                double s = 0.0;
                for (int o = 0; o < n_out; ++o) s += dY[(int64_t)b * n_out + o] * W[(int64_t)o * n_in + i];
                dA[(int64_t)b * n_in + i] = s;
            }
        }
    }
}

/* Forward + backward of the whole model on one batch.
 * Outputs:
 *   loss                      mean BCE
 *   y_hat [B]
 *   bot_dW[l] [out][in], bot_db[l] [out], top_dW[l], top_db[l]: batch-summed gradients of the mean loss
 *   table_grad [sum rows][d]  gradient of every table row (zero for rows no valid index touches)
 *   row_count  [sum rows]     number of valid occurrences of each row in the batch
 *   counts[0..1]              as oracle_embbag */
void oracle_train_grads(const oracle_model* M, int B, long nnz, const double* dense,
                        const int32_t* offsets, const int32_t* indices, const double* labels,
                        double* loss, double* y_hat,
                        double* const* bot_dW, double* const* bot_db, double* const* top_dW, double* const* top_db,
                        double* table_grad, int64_t* row_count, long* counts) {
    int K = M->K, d = M->d;
    int width = d + K * (K + 1) / 2;
    int64_t* base = (int64_t*)malloc(sizeof(int64_t) * (K > 0 ? K : 1));
    table_bases(K, M->rows, base);
    int64_t total_rows = 0;
    for (int k = 0; k < K; ++k) total_rows += M->rows[k];

    /* activations: bot_act[0] = dense, bot_act[l+1] = output of bottom layer l; same for top */
    double** bot_act = (double**)malloc(sizeof(double*) * (M->n_bot + 1));
    double** top_act = (double**)malloc(sizeof(double*) * (M->n_top + 1));
    for (int l = 0; l <= M->n_bot; ++l) bot_act[l] = (double*)malloc(sizeof(double) * (size_t)B * M->bot_dims[l]);
    for (int l = 0; l <= M->n_top; ++l) top_act[l] = (double*)malloc(sizeof(double) * (size_t)B * M->top_dims[l]);
    double* E = (double*)malloc(sizeof(double) * (size_t)B * (K > 0 ? K : 1) * d);
    int32_t* lens = (int32_t*)malloc(sizeof(int32_t) * ((size_t)K * B + 1));
    memcpy(bot_act[0], dense, sizeof(double) * (size_t)B * M->bot_dims[0]);

    /* forward, keeping every activation */
    for (int l = 0; l < M->n_bot; ++l)
#pragma omp parallel for schedule(static)
        for (int b = 0; b < B; ++b)
            linear_one(M->bot_dims[l], M->bot_dims[l + 1], M->bot_W[l], M->bot_b[l],
                       bot_act[l] + (int64_t)b * M->bot_dims[l], bot_act[l + 1] + (int64_t)b * M->bot_dims[l + 1], 1);
    const double* xd = bot_act[M->n_bot];
    long oob = 0, badn = 0;
    for (int b = 0; b < B; ++b)
        for (int k = 0; k < K; ++k) {
            int bad;
            oob += pool_one_bag(k, B, b, d, nnz, M->rows, base, M->tables, offsets, indices,
                                E + ((int64_t)b * K + k) * d, lens + (int64_t)k * B + b, &bad);
            badn += bad;
        }
    counts[0] = oob;
    counts[1] = badn;
#pragma omp parallel for schedule(static)
    for (int b = 0; b < B; ++b)
        interact_one(K, d, xd + (int64_t)b * d, E + (int64_t)b * K * d, top_act[0] + (int64_t)b * width);
    for (int l = 0; l < M->n_top; ++l)
#pragma omp parallel for schedule(static)
        for (int b = 0; b < B; ++b)
            linear_one(M->top_dims[l], M->top_dims[l + 1], M->top_W[l], M->top_b[l],
                       top_act[l] + (int64_t)b * M->top_dims[l], top_act[l + 1] + (int64_t)b * M->top_dims[l + 1],
                       l < M->n_top - 1);
    const double* z = top_act[M->n_top];
    *loss = oracle_bce(B, z, labels);
    for (int b = 0; b < B; ++b) y_hat[b] = sigmoid(z[b]);

    /* dL/dz = (sigmoid(z) - y) / B */
    double* dY = (double*)malloc(sizeof(double) * (size_t)B);
    for (int b = 0; b < B; ++b) dY[b] = (sigmoid(z[b]) - labels[b]) / B;

    /* top MLP backward */
    for (int l = M->n_top - 1; l >= 0; --l) {
        double* dA = (double*)malloc(sizeof(double) * (size_t)B * M->top_dims[l]);
        linear_backward(B, M->top_dims[l], M->top_dims[l + 1], M->top_W[l], top_act[l], top_act[l + 1],
                        dY, top_dW[l], top_db[l], dA, l < M->n_top - 1);
        free(dY);
        dY = dA;
    }
    /* dY is now d(concat) [B][width]. Interaction backward:
     * Z_ij = <X_i, X_j>  =>  dX_i += dZ_ij X_j and dX_j += dZ_ij X_i. */
    double* dX = (double*)calloc((size_t)B * (K + 1) * d, sizeof(double));
#pragma omp parallel for schedule(static)
    for (int b = 0; b < B; ++b) {
        const double* dc = dY + (int64_t)b * width;
        double* g = dX + (int64_t)b * (K + 1) * d;
        for (int t = 0; t < d; ++t) g[t] += dc[t];          /* direct x_dense part of the concat */
        int p = d;
        for (int i = 1; i <= K; ++i) {
            const double* xi = E + ((int64_t)b * K + (i - 1)) * d;
            for (int j = 0; j < i; ++j) {
                const double* xj = (j == 0) ? xd + (int64_t)b * d : E + ((int64_t)b * K + (j - 1)) * d;
                double dz = dc[p++];
                for (int t = 0; t < d; ++t) {
                    g[(int64_t)i * d + t] += dz * xj[t];
                    g[(int64_t)j * d + t] += dz * xi[t];
                }
            }
        }
    }
    /* bottom MLP backward, starting from dX row 0 */
    double* dB = (double*)malloc(sizeof(double) * (size_t)B * d);
    for (int b = 0; b < B; ++b) memcpy(dB + (int64_t)b * d, dX + (int64_t)b * (K + 1) * d, sizeof(double) * d);
    for (int l = M->n_bot - 1; l >= 0; --l) {
        double* dA = (l > 0) ? (double*)malloc(sizeof(double) * (size_t)B * M->bot_dims[l]) : NULL;
        linear_backward(B, M->bot_dims[l], M->bot_dims[l + 1], M->bot_W[l], bot_act[l], bot_act[l + 1],
                        dB, bot_dW[l], bot_db[l], dA, 1);
        free(dB);
        dB = dA;
    }
    /* embedding rows: every valid occurrence of row r in bag (k, b) adds dE_k[b] */
    memset(table_grad, 0, sizeof(double) * (size_t)total_rows * d);
    memset(row_count, 0, sizeof(int64_t) * (size_t)total_rows);
    for (int k = 0; k < K; ++k) {
        for (int b = 0; b < B; ++b) {
            int64_t start = offsets[(int64_t)k * B + b], end = offsets[(int64_t)k * B + b + 1];
            if (start < 0 || end < start || end > nnz) continue;
            const double* g = dX + ((int64_t)b * (K + 1) + (k + 1)) * d;
            for (int64_t p = start; p < end; ++p) {
                int64_t r = indices[p];
                if (r < 0 || r >= M->rows[k]) continue;
                double* tg = table_grad + (base[k] + r) * d;
                for (int t = 0; t < d; ++t) tg[t] += g[t];
                row_count[base[k] + r] += 1;
            }
        }
    }
    free(dX); free(dY);

    for (int l = 0; l <= M->n_bot; ++l) free(bot_act[l]);
    for (int l = 0; l <= M->n_top; ++l) free(top_act[l]);
    free(bot_act); free(top_act); free(E); free(lens); free(base);
}

/* Plain SGD: w <- w - lr * g, elementwise. */
void oracle_sgd(int64_t n, double lr, double* w, const double* g) {
    for (int64_t q = 0; q < n; ++q) w[q] -= lr * g[q];
}

/* Row-wise 8-bit quantisation of fp32 rows (the DLRM_U8ROW storage). Per row,
 * in fp32 with round-to-nearest: lo = min, hi = max, s = (hi - lo) / 255,
 * q = rint((v - lo) / s) clamped to [0, 255] (q = 0 when s = 0), m = lo. */
void oracle_quantize_rows_u8(int64_t rows, int d, const float* src, unsigned char* codes, float* scale,
                             float* offset) {
    for (int64_t r = 0; r < rows; ++r) {
        const float* v = src + r * d;
        float lo = INFINITY, hi = -INFINITY;
        for (int c = 0; c < d; ++c) {
            lo = fminf(lo, v[c]);
            hi = fmaxf(hi, v[c]);
        }
        const float s = (hi - lo) / 255.0f;
        for (int c = 0; c < d; ++c) {
            float q = 0.0f;
            if (s > 0.0f) q = rintf((v[c] - lo) / s);
            if (q < 0.0f) q = 0.0f;
            if (q > 255.0f) q = 255.0f;
            codes[r * d + c] = (unsigned char)q;
        }
        scale[r] = s;
        offset[r] = lo;
    }
}

/* Value of every entry of row-wise 8-bit rows: s * q + m, in fp64 (exact for fp32 s, m and 8-bit q). */
void oracle_dequantize_rows_u8(int64_t rows, int d, const unsigned char* codes, const float* scale,
                               const float* offset, double* out) {
    for (int64_t r = 0; r < rows; ++r)
        for (int c = 0; c < d; ++c) out[r * d + c] = (double)scale[r] * (double)codes[r * d + c] + (double)offset[r];
}

/* Concat-only interaction (the Wide & Deep alternative the pages contrast
 * DLRM with, "Deep Learning Recommendation Model (DLRM)", Key Method Details):
 * out[b] = [x_dense[b], e_1, ..., e_K], width d (K + 1). */
void oracle_concat(int B, int K, int d, const double* x_dense, const double* pooled, double* out) {
    const int64_t w = (int64_t)d * (K + 1);
    for (int b = 0; b < B; ++b) {
        double* o = out + (int64_t)b * w;
        for (int t = 0; t < d; ++t) o[t] = x_dense[(int64_t)b * d + t];
        for (int k = 0; k < K; ++k)
            for (int t = 0; t < d; ++t) o[(int64_t)(k + 1) * d + t] = pooled[((int64_t)b * K + k) * d + t];
    }
}
