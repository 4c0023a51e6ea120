// extern "C" entry points of the training step: forward with saved
// activations, BCE loss, backward through the top MLP, the interaction and the
// bottom MLP, the row-sorted embedding gradient, and the SGD updates.
// The training path is fp32 throughout (tables, weights, activations).
#include <string.h>

#include <algorithm>

#include "common.cuh"
#include "kernels.cuh"

using namespace dlrm;

namespace {

inline bool aligned16(const void* p) { return ((uintptr_t)p & 15u) == 0; }
inline cudaStream_t cs(dlrm_stream s) { return reinterpret_cast<cudaStream_t>(s); }

struct TrainWs {
    size_t bact[DLRM_MAX_LAYERS], E, concat, tact[DLRM_MAX_LAYERS], g0, g1, wscratch, lpart, total;
    int ldb[DLRM_MAX_LAYERS], ldt[DLRM_MAX_LAYERS], ldc, gmax;
};

struct Grads {
    size_t bdW[DLRM_MAX_LAYERS], bdb[DLRM_MAX_LAYERS], tdW[DLRM_MAX_LAYERS], tdb[DLRM_MAX_LAYERS], dE, loss, sparse,
        total;
    SparseLayout sp;
};

int ldf(int n) { return dlrm_ld(n, DLRM_F32); }

TrainWs train_ws(const dlrm_tables* T, const dlrm_mlp* bot, const dlrm_mlp* top, int B) {
    TrainWs W;
    size_t off = DLRM_ERR_RECORD_BYTES;
    auto take = [&](size_t bytes) {
        const size_t o = off;
        off = align_up(off + bytes, 256);
        return o;
    };
    const int K = T->K, d = T->d;
    int gmax = 0;
    for (int l = 0; l < bot->n_layers; ++l) {
        W.ldb[l] = ldf(bot->dims[l + 1]);
        W.bact[l] = take(sizeof(float) * (size_t)B * W.ldb[l]);
        gmax = std::max(gmax, W.ldb[l]);
    }
    W.E = take(sizeof(float) * (size_t)B * K * d);
    W.ldc = ldf(d + K * (K + 1) / 2);
    W.concat = take(sizeof(float) * (size_t)B * W.ldc);
    gmax = std::max(gmax, W.ldc);
    for (int l = 0; l < top->n_layers; ++l) {
        // the logit (last layer, one column) is stored densely: BCE reads z[B]
        W.ldt[l] = (l == top->n_layers - 1 && top->dims[l + 1] == 1) ? 1 : ldf(top->dims[l + 1]);
        W.tact[l] = take(sizeof(float) * (size_t)B * W.ldt[l]);
        gmax = std::max(gmax, W.ldt[l]);
    }
    W.gmax = gmax;
    W.g0 = take(sizeof(float) * (size_t)B * gmax);
    W.g1 = take(sizeof(float) * (size_t)B * gmax);
    size_t ws = 0;
    for (int l = 0; l < bot->n_layers; ++l)
        ws = std::max(ws, train_wgrad_scratch_floats(bot->dims[l + 1], bot->dims[l], B));
    for (int l = 0; l < top->n_layers; ++l)
        ws = std::max(ws, train_wgrad_scratch_floats(top->dims[l + 1], top->dims[l], B));
    W.wscratch = take(sizeof(float) * ws);
    W.lpart = take(sizeof(float) * ((size_t)(B + 255) / 256 + 1));
    W.total = off;
    return W;
}

Grads grads_layout(const dlrm_tables* T, const dlrm_mlp* bot, const dlrm_mlp* top, int B, long long nnz) {
    Grads G;
    size_t off = 0;
    auto take = [&](size_t bytes) {
        const size_t o = off;
        off = align_up(off + bytes, 256);
        return o;
    };
    for (int l = 0; l < bot->n_layers; ++l) {
        G.bdW[l] = take(sizeof(float) * (size_t)bot->dims[l + 1] * ldf(bot->dims[l]));
        G.bdb[l] = take(sizeof(float) * (size_t)bot->dims[l + 1]);
    }
    for (int l = 0; l < top->n_layers; ++l) {
        G.tdW[l] = take(sizeof(float) * (size_t)top->dims[l + 1] * ldf(top->dims[l]));
        G.tdb[l] = take(sizeof(float) * (size_t)top->dims[l + 1]);
    }
    G.dE = take(sizeof(float) * (size_t)B * T->K * T->d);
    G.loss = take(sizeof(float));
    G.sp = sparse_layout((long long)T->K * B, nnz, T->d);
    G.sparse = take(G.sp.total);
    G.total = off;
    return G;
}

dlrm_status check_train(const dlrm_tables* T, const dlrm_mlp* bot, const dlrm_mlp* top, int B, TableMeta& tm) {
    if (!T || !T->rows || !T->data || !bot || !top || !bot->dims || !top->dims || !bot->W || !bot->b || !top->W ||
        !top->b)
        return DLRM_ERR_INVALID_ARG;
    if (T->K < 1 || T->d < 1 || B < 0) return DLRM_ERR_INVALID_ARG;
    if (T->K > DLRM_MAX_TABLES || bot->n_layers < 1 || top->n_layers < 1 || bot->n_layers > DLRM_MAX_LAYERS ||
        top->n_layers > DLRM_MAX_LAYERS)
        return DLRM_ERR_UNSUPPORTED;
    if (T->dt != DLRM_F32 || bot->dt != DLRM_F32 || top->dt != DLRM_F32) return DLRM_ERR_UNSUPPORTED;
    if (!aligned16(T->data)) return DLRM_ERR_INVALID_ARG;
    long long acc = 0;
    for (int k = 0; k < T->K; ++k) {
        if (T->rows[k] < 1) return DLRM_ERR_INVALID_ARG;
        tm.base[k] = acc;
        tm.rows[k] = T->rows[k];
        acc += T->rows[k];
    }
    if (acc >= 0xFFFFFFFFll) return DLRM_ERR_UNSUPPORTED;   // row ids are sorted as 32-bit keys
    for (int l = 0; l <= bot->n_layers; ++l)
        if (bot->dims[l] < 1) return DLRM_ERR_INVALID_ARG;
    for (int l = 0; l <= top->n_layers; ++l)
        if (top->dims[l] < 1) return DLRM_ERR_INVALID_ARG;
    for (int l = 0; l < bot->n_layers; ++l)
        if (!bot->W[l] || !bot->b[l]) return DLRM_ERR_INVALID_ARG;
    for (int l = 0; l < top->n_layers; ++l)
        if (!top->W[l] || !top->b[l]) return DLRM_ERR_INVALID_ARG;
    const int K = T->K, d = T->d;
    if (bot->dims[bot->n_layers] != d || top->dims[0] != d + K * (K + 1) / 2 || top->dims[top->n_layers] != 1)
        return DLRM_ERR_INVALID_ARG;
    if (d % 4 || !gather_supported(d, DLRM_F32) || interact_bwd_smem(K, d) > 227 * 1024 ||
        interact_smem_per_sample(K, d) > 227 * 1024)
        return DLRM_ERR_UNSUPPORTED;
    return DLRM_OK;
}

long long total_rows_of(const TableMeta& tm, int K) { return tm.base[K - 1] + tm.rows[K - 1]; }

}  // namespace

namespace dlrm {
size_t train_workspace_size(const dlrm_tables* T, const dlrm_mlp* bot, const dlrm_mlp* top, int B) {
    TableMeta tm;
    if (check_train(T, bot, top, B, tm) != DLRM_OK) return 0;
    return train_ws(T, bot, top, B).total;
}
}  // namespace dlrm

extern "C" {

size_t dlrm_grads_size(const dlrm_tables* T, const dlrm_mlp* bot, const dlrm_mlp* top, int B, int64_t nnz) {
    TableMeta tm;
    if (check_train(T, bot, top, B, tm) != DLRM_OK || nnz < 0) return 0;
    return grads_layout(T, bot, top, B, nnz).total;
}

dlrm_status dlrm_grads_offsets(const dlrm_tables* T, const dlrm_mlp* bot, const dlrm_mlp* top, int B, int64_t nnz,
                               size_t* bot_dW, size_t* bot_db, size_t* top_dW, size_t* top_db, size_t* dE,
                               size_t* loss) {
    TableMeta tm;
    dlrm_status r = check_train(T, bot, top, B, tm);
    if (r) return r;
    const Grads G = grads_layout(T, bot, top, B, nnz);
    for (int l = 0; l < bot->n_layers; ++l) {
        if (bot_dW) bot_dW[l] = G.bdW[l];
        if (bot_db) bot_db[l] = G.bdb[l];
    }
    for (int l = 0; l < top->n_layers; ++l) {
        if (top_dW) top_dW[l] = G.tdW[l];
        if (top_db) top_db[l] = G.tdb[l];
    }
    if (dE) *dE = G.dE;
    if (loss) *loss = G.loss;
    return DLRM_OK;
}

dlrm_status dlrm_backward(const dlrm_tables* T, const dlrm_mlp* bot, const dlrm_mlp* top, int B, const float* dense,
                          const int32_t* offsets, const int32_t* indices, int64_t nnz, const float* labels,
                          float* loss, float* y_hat, void* grads, void* ws, dlrm_stream stream) {
    TableMeta tm;
    dlrm_status r = check_train(T, bot, top, B, tm);
    if (r) return r;
    if (nnz < 0 || nnz >= (int64_t(1) << 31)) return DLRM_ERR_INVALID_ARG;
    if (!ws || !aligned16(ws) || !grads || !aligned16(grads)) return DLRM_ERR_WORKSPACE;
    if (B == 0) return DLRM_OK;
    if (!dense || !offsets || (nnz > 0 && !indices) || !labels) return DLRM_ERR_INVALID_ARG;
    const int K = T->K, d = T->d;
    const TrainWs W = train_ws(T, bot, top, B);
    const Grads G = grads_layout(T, bot, top, B, nnz);
    char* w = static_cast<char*>(ws);
    char* g = static_cast<char*>(grads);
    ErrRecord* err = reinterpret_cast<ErrRecord*>(w);
    cudaStream_t st = cs(stream);
    auto F = [&](size_t o) { return reinterpret_cast<float*>(w + o); };
    auto GF = [&](size_t o) { return reinterpret_cast<float*>(g + o); };
    const int nb = bot->n_layers, nt = top->n_layers;

    // dW padding columns stay zero so that SGD leaves the weights' padding untouched
    if (cudaMemsetAsync(g, 0, G.dE, st) != cudaSuccess) return DLRM_ERR_CUDA;

    // ---- forward, keeping every activation
    for (int l = 0; l < nb; ++l) {
        const float* in = l == 0 ? dense : F(W.bact[l - 1]);
        const int ldin = l == 0 ? bot->dims[0] : W.ldb[l - 1];
        if ((r = train_linear_fwd(B, bot->dims[l + 1], bot->dims[l], in, ldin, static_cast<const float*>(bot->W[l]),
                                  ldf(bot->dims[l]), bot->b[l], F(W.bact[l]), W.ldb[l], true, st)))
            return r;
    }
    const float* x_dense = F(W.bact[nb - 1]);   // ld = ldf(d) = d (d % 4 == 0 on this path)
    if ((r = launch_embbag(tm, T->data, DLRM_F32, K, d, B, offsets, indices, nnz, F(W.E), nullptr, err, st))) return r;
    if ((r = launch_interact(B, K, d, x_dense, F(W.E), F(W.concat), W.ldc, DLRM_F32, st))) return r;
    for (int l = 0; l < nt; ++l) {
        const float* in = l == 0 ? F(W.concat) : F(W.tact[l - 1]);
        const int ldin = l == 0 ? W.ldc : W.ldt[l - 1];
        if ((r = train_linear_fwd(B, top->dims[l + 1], top->dims[l], in, ldin, static_cast<const float*>(top->W[l]),
                                  ldf(top->dims[l]), top->b[l], F(W.tact[l]), W.ldt[l], l < nt - 1, st)))
            return r;
    }

    // ---- loss and dL/dz
    float* dz = F(W.g0);
    const float* z = F(W.tact[nt - 1]);
    if ((r = launch_bce(B, z, labels, dz, y_hat, F(W.lpart), GF(G.loss), st))) return r;
    if (loss && cudaMemcpyAsync(loss, GF(G.loss), sizeof(float), cudaMemcpyDeviceToDevice, st) != cudaSuccess)
        return DLRM_ERR_CUDA;

    // ---- top MLP backward: cur = dL/d(pre-activation of layer l), ld curld
    float* cur = dz;
    int curld = 1;
    float* other = F(W.g1);
    for (int l = nt - 1; l >= 0; --l) {
        const float* in = l == 0 ? F(W.concat) : F(W.tact[l - 1]);
        const int ldin = l == 0 ? W.ldc : W.ldt[l - 1];
        const int N = top->dims[l + 1], Kin = top->dims[l];
        if ((r = train_linear_wgrad(B, N, Kin, cur, curld, in, ldin, GF(G.tdW[l]), ldf(Kin), GF(G.tdb[l]),
                                    F(W.wscratch), st)))
            return r;
        const int ldo = l == 0 ? W.ldc : W.ldt[l - 1];
        if ((r = train_linear_dgrad(B, N, Kin, cur, curld, static_cast<const float*>(top->W[l]), ldf(Kin),
                                    l == 0 ? nullptr : F(W.tact[l - 1]), ldo, other, ldo, st)))
            return r;
        float* t = cur;
        cur = other;
        other = t;
        curld = ldo;
    }
    // cur = d(concat) [B][ldc]
    float* dxd = other;   // gradient of the last bottom layer's pre-activation [B][d]
    if ((r = launch_interact_bwd(B, K, d, x_dense, F(W.E), cur, W.ldc, dxd, GF(G.dE), st))) return r;
    cur = dxd;
    curld = d;
    other = (cur == F(W.g0)) ? F(W.g1) : F(W.g0);
    for (int l = nb - 1; l >= 0; --l) {
        const float* in = l == 0 ? dense : F(W.bact[l - 1]);
        const int ldin = l == 0 ? bot->dims[0] : W.ldb[l - 1];
        const int N = bot->dims[l + 1], Kin = bot->dims[l];
        if ((r = train_linear_wgrad(B, N, Kin, cur, curld, in, ldin, GF(G.bdW[l]), ldf(Kin), GF(G.bdb[l]),
                                    F(W.wscratch), st)))
            return r;
        if (l > 0) {
            if ((r = train_linear_dgrad(B, N, Kin, cur, curld, static_cast<const float*>(bot->W[l]), ldf(Kin),
                                        F(W.bact[l - 1]), W.ldb[l - 1], other, W.ldb[l - 1], st)))
                return r;
            float* t = cur;
            cur = other;
            other = t;
            curld = W.ldb[l - 1];
        }
    }

    // ---- embedding rows: sort occurrences by row, cut segments and pieces
    int sorted_buf = 0;
    if ((r = launch_sparse_prepare(K, B, tm, total_rows_of(tm, K), offsets, indices, nnz, g + G.sparse, G.sp, err,
                                   &sorted_buf, st)))
        return r;
    return DLRM_OK;
}

dlrm_status dlrm_sparse_sgd(const dlrm_tables* T, const dlrm_mlp* bot, const dlrm_mlp* top, int B, int64_t nnz,
                            float lr, void* grads, int32_t* n_touched, dlrm_stream stream) {
    TableMeta tm;
    dlrm_status r = check_train(T, bot, top, B, tm);
    if (r) return r;
    if (nnz < 0 || nnz >= (int64_t(1) << 31)) return DLRM_ERR_INVALID_ARG;
    if (!grads || !aligned16(grads)) return DLRM_ERR_WORKSPACE;
    if (B == 0) return DLRM_OK;
    const Grads G = grads_layout(T, bot, top, B, nnz);
    const char* g = static_cast<const char*>(grads);
    cudaStream_t st = cs(stream);
    const int sorted = radix_passes(total_rows_of(tm, T->K)) & 1;
    if ((r = launch_sparse_apply(T->d, g + G.sparse, G.sp, sorted, reinterpret_cast<const float*>(g + G.dE), lr,
                                 static_cast<float*>(T->data), nullptr, nullptr, n_touched, st)))
        return r;
    for (int l = 0; l < bot->n_layers; ++l) {
        const long long n = (long long)bot->dims[l + 1] * ldf(bot->dims[l]);
        if ((r = launch_sgd(n, lr, static_cast<float*>(bot->W[l]), reinterpret_cast<const float*>(g + G.bdW[l]), st)) ||
            (r = launch_sgd(bot->dims[l + 1], lr, bot->b[l], reinterpret_cast<const float*>(g + G.bdb[l]), st)))
            return r;
    }
    for (int l = 0; l < top->n_layers; ++l) {
        const long long n = (long long)top->dims[l + 1] * ldf(top->dims[l]);
        if ((r = launch_sgd(n, lr, static_cast<float*>(top->W[l]), reinterpret_cast<const float*>(g + G.tdW[l]), st)) ||
            (r = launch_sgd(top->dims[l + 1], lr, top->b[l], reinterpret_cast<const float*>(g + G.tdb[l]), st)))
            return r;
    }
    return DLRM_OK;
}

dlrm_status dlrm_embedding_row_grads(const dlrm_tables* T, const dlrm_mlp* bot, const dlrm_mlp* top, int B,
                                     int64_t nnz, void* grads, uint32_t* rows, float* row_grads,
                                     int32_t* n_rows, dlrm_stream stream) {
    TableMeta tm;
    dlrm_status r = check_train(T, bot, top, B, tm);
    if (r) return r;
    if (nnz < 0 || nnz >= (int64_t(1) << 31)) return DLRM_ERR_INVALID_ARG;
    if (!grads || !aligned16(grads)) return DLRM_ERR_WORKSPACE;
    if (!rows || !row_grads || !n_rows) return DLRM_ERR_INVALID_ARG;
    if (B == 0) return DLRM_OK;
    const Grads G = grads_layout(T, bot, top, B, nnz);
    const char* g = static_cast<const char*>(grads);
    const int sorted = radix_passes(total_rows_of(tm, T->K)) & 1;
    return launch_sparse_apply(T->d, g + G.sparse, G.sp, sorted, reinterpret_cast<const float*>(g + G.dE), 0.f,
                               nullptr, row_grads, rows, n_rows, cs(stream));
}

}  // extern "C"
