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

// Workspace of the training step. Every tensor that a GEMM reads is kept as a
// 3xTF32 (hi, lo) pair (F32Pair); x_dense, the concat vector, the logit and the
// gradients that feed the interaction backward are also (or only) plain fp32.
struct TrainWs {
    size_t bW[DLRM_MAX_LAYERS][2], tW[DLRM_MAX_LAYERS][2];   // weight pairs, ld ldf(in)
    size_t bact[DLRM_MAX_LAYERS][2];                         // bottom outputs (pairs), ld ldb
    size_t xd;                                               // x_dense plain [B][d] (fallback path only)
    size_t E;                                                // pooled [B][K][d] (fallback path only)
    size_t concat, concat_p[2];                              // [B][ldc] plain (fallback only) and pair
    size_t tact[DLRM_MAX_LAYERS][2];                         // top hidden outputs (pairs), ld ldt
    size_t z, dz;                                            // logit and dL/dz [B]
    size_t g[2][2];                                          // gradient ping-pong pairs [B][gmax]
    size_t dcat, dxd;                                        // plain d(concat) [B][ldc], d(x_dense pre-act) [B][d]
    size_t bbits[DLRM_MAX_LAYERS], tbits[DLRM_MAX_LAYERS];   // ReLU bitmasks of the saved activations
    size_t csum;                                             // column sums per 32-row group of a gradient
    size_t wscratch, lpart, total;
    int ldb[DLRM_MAX_LAYERS], ldt[DLRM_MAX_LAYERS], ldc, gmax;
    bool tc;                                                 // fused tensor-core interaction (no E, xd, concat, dxd)
};

struct Grads {
    size_t bdW[DLRM_MAX_LAYERS], bdb[DLRM_MAX_LAYERS], tdW[DLRM_MAX_LAYERS], tdb[DLRM_MAX_LAYERS], dE, loss, sparse,
        total;
    SparseLayout sp;
};

int ldf(int n) { return dlrm_ld(n, DLRM_F32); }

// Layout for K tables of width d holding total_rows rows; allow_tc = false forces the path that reads pooled
// vectors (the caller's, or the ones the step pools itself).
TrainWs train_ws(int K, int d, long long total_rows, bool allow_tc, const dlrm_mlp* bot, const dlrm_mlp* top, int B) {
    TrainWs W;
    size_t off = DLRM_ERR_RECORD_BYTES;
    auto take = [&](size_t bytes) {
        const size_t o = off;
        off = align_up(off + bytes, 256);
        return o;
    };
    const int nb = bot->n_layers, nt = top->n_layers;
    for (int l = 0; l < nb; ++l)
        for (int h = 0; h < 2; ++h) W.bW[l][h] = take(sizeof(float) * (size_t)bot->dims[l + 1] * ldf(bot->dims[l]));
    for (int l = 0; l < nt; ++l)
        for (int h = 0; h < 2; ++h) W.tW[l][h] = take(sizeof(float) * (size_t)top->dims[l + 1] * ldf(top->dims[l]));
    int gmax = 0;
    for (int l = 0; l < nb; ++l) {
        W.ldb[l] = ldf(bot->dims[l + 1]);
        for (int h = 0; h < 2; ++h) W.bact[l][h] = take(sizeof(float) * (size_t)B * W.ldb[l]);
        gmax = std::max(gmax, W.ldb[l]);
    }
    W.ldc = ldf(d + K * (K + 1) / 2);
    // the fused tensor-core interaction gathers the bags itself: no pooled vectors, no plain-fp32 copies
    W.tc = allow_tc && interact_tc_supported(K, d, total_rows, W.ldc);
    W.xd = W.tc ? 0 : take(sizeof(float) * (size_t)B * d);
    W.E = W.tc ? 0 : take(sizeof(float) * (size_t)B * K * d);
    W.concat = W.tc ? 0 : take(sizeof(float) * (size_t)B * W.ldc);
    for (int h = 0; h < 2; ++h) W.concat_p[h] = take(sizeof(float) * (size_t)B * W.ldc);
    for (int l = 0; l < nt - 1; ++l) {
        W.ldt[l] = ldf(top->dims[l + 1]);
        for (int h = 0; h < 2; ++h) W.tact[l][h] = take(sizeof(float) * (size_t)B * W.ldt[l]);
        gmax = std::max(gmax, W.ldt[l]);
    }
    W.ldt[nt - 1] = 1;   // the logit is stored densely: BCE reads z[B]
    W.z = take(sizeof(float) * (size_t)B);
    W.dz = take(sizeof(float) * (size_t)B);
    W.gmax = gmax;
    for (int p = 0; p < 2; ++p)
        for (int h = 0; h < 2; ++h) W.g[p][h] = take(sizeof(float) * (size_t)B * gmax);
    W.dcat = take(sizeof(float) * (size_t)B * W.ldc);
    W.dxd = W.tc ? 0 : take(sizeof(float) * (size_t)B * d);
    for (int l = 0; l < nb; ++l) W.bbits[l] = take(sizeof(uint32_t) * (size_t)B * relu_bits_ld(bot->dims[l + 1]));
    for (int l = 0; l < nt - 1; ++l) W.tbits[l] = take(sizeof(uint32_t) * (size_t)B * relu_bits_ld(top->dims[l + 1]));
    W.csum = take(sizeof(float) * (size_t)((B + 31) / 32) * gmax);
    size_t ws = 0;
    for (int l = 0; l < nb; ++l)
        ws = std::max(ws, train_wgrad_scratch_floats(bot->dims[l + 1], bot->dims[l], B));
    for (int l = 0; l < nt; ++l)
        ws = std::max(ws, train_wgrad_scratch_floats(top->dims[l + 1], top->dims[l], B));
    W.wscratch = take(sizeof(float) * ws);
    W.lpart = take(sizeof(float) * ((size_t)(B + 255) / 256 + 1));
    W.total = off;
    return W;
}

Grads grads_layout(int K, int d, const dlrm_mlp* bot, const dlrm_mlp* top, int B, long long nnz) {
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
    G.dE = take(sizeof(float) * (size_t)B * K * d);
    G.loss = take(sizeof(float));
    G.sp = sparse_layout((long long)K * B, nnz, d);
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
    return train_ws(T->K, T->d, total_rows_of(tm, T->K), true, bot, top, B).total;
}
}  // namespace dlrm

extern "C" {

size_t dlrm_grads_size(const dlrm_tables* T, const dlrm_mlp* bot, const dlrm_mlp* top, int B, int64_t nnz) {
    TableMeta tm;
    if (check_train(T, bot, top, B, tm) != DLRM_OK || nnz < 0) return 0;
    return grads_layout(T->K, T->d, bot, top, B, nnz).total;
}

dlrm_status dlrm_grads_offsets(const dlrm_tables* T, const dlrm_mlp* bot, const dlrm_mlp* top, int B, int64_t nnz,
                               size_t* bot_dW, size_t* bot_db, size_t* top_dW, size_t* top_db, size_t* dE,
                               size_t* loss) {
    TableMeta tm;
    dlrm_status r = check_train(T, bot, top, B, tm);
    if (r) return r;
    const Grads G = grads_layout(T->K, T->d, bot, top, B, nnz);
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

}  // extern "C"

namespace {

// The training step's forward and backward on one batch. With pooled == nullptr it gathers the bags of the
// tables itself (tm, tables, offsets, indices) and finishes with the row-sorted preparation of the sparse
// update; with pooled ([B][K][d] fp32) the given vectors stand in for the pooled bags and no row is touched.
dlrm_status backward_impl(int K, int d, const TableMeta& tm, const float* tables, const dlrm_mlp* bot,
                          const dlrm_mlp* top, int B, const float* dense, const int32_t* offsets,
                          const int32_t* indices, int64_t nnz, const float* pooled, const float* labels, float* loss,
                          float* y_hat, void* grads, void* ws, const TrainWs& W, const Grads& G, cudaStream_t st) {
    dlrm_status r;
    char* w = static_cast<char*>(ws);
    char* g = static_cast<char*>(grads);
    ErrRecord* err = reinterpret_cast<ErrRecord*>(w);
    auto F = [&](size_t o) { return reinterpret_cast<float*>(w + o); };
    auto U = [&](size_t o) { return reinterpret_cast<uint32_t*>(w + o); };
    auto GF = [&](size_t o) { return reinterpret_cast<float*>(g + o); };
    const int nb = bot->n_layers, nt = top->n_layers;

    // dW padding columns stay zero so that SGD leaves the weights' padding untouched
    if (cudaMemsetAsync(g, 0, G.dE, st) != cudaSuccess) return DLRM_ERR_CUDA;
    auto P = [&](const size_t (&o)[2], int ld) { return F32Pair{F(o[0]), F(o[1]), ld}; };

    // ---- weights as (hi, lo) pairs (they change with every SGD step)
    for (int l = 0; l < nb; ++l)
        if ((r = launch_split_pair(bot->dims[l + 1], bot->dims[l], static_cast<const float*>(bot->W[l]),
                                   ldf(bot->dims[l]), F(W.bW[l][0]), F(W.bW[l][1]), ldf(bot->dims[l]), st)))
            return r;
    for (int l = 0; l < nt; ++l)
        if ((r = launch_split_pair(top->dims[l + 1], top->dims[l], static_cast<const float*>(top->W[l]),
                                   ldf(top->dims[l]), F(W.tW[l][0]), F(W.tW[l][1]), ldf(top->dims[l]), st)))
            return r;

    // ---- forward, keeping every activation
    const F32Pair dense_in{dense, nullptr, bot->dims[0]};
    for (int l = 0; l < nb; ++l) {
        const F32Pair in = l == 0 ? dense_in : P(W.bact[l - 1], W.ldb[l - 1]);
        if ((r = train_linear_fwd(B, bot->dims[l + 1], bot->dims[l], in, P(W.bW[l], ldf(bot->dims[l])), bot->b[l],
                                  F(W.bact[l][0]), F(W.bact[l][1]), W.ldb[l], true, U(W.bbits[l]), err, st)))
            return r;
    }
    const F32Pair xd_pair = P(W.bact[nb - 1], W.ldb[nb - 1]);   // ld = d (d % 4 == 0 on this path)
    const float* x_dense = W.tc ? nullptr : F(W.xd);
    const float* E = pooled ? pooled : (W.tc ? nullptr : F(W.E));
    // the fused tensor-core interaction gathers the bags and reads/writes pairs; other shapes pool the bags
    // first and go through plain fp32 copies
    if (W.tc) {
        if ((r = launch_interact_fwd_tc(tm, tables, K, d, B, offsets, indices, nnz, xd_pair, F(W.concat_p[0]),
                                        F(W.concat_p[1]), W.ldc, err, st)))
            return r;
    } else {
        if (!pooled && (r = launch_embbag(tm, tables, DLRM_F32, K, d, B, offsets, indices, nnz, F(W.E), nullptr, err,
                                          st)))
            return r;
        if ((r = launch_merge_pair(B, d, xd_pair.hi, xd_pair.lo, xd_pair.ld, F(W.xd), d, st))) return r;
        if ((r = launch_interact(B, K, d, x_dense, E, F(W.concat), W.ldc, DLRM_F32, st))) return r;
        if ((r = launch_split_pair(B, top->dims[0], F(W.concat), W.ldc, F(W.concat_p[0]), F(W.concat_p[1]), W.ldc,
                                   st)))
            return r;
    }
    const F32Pair concat_p = P(W.concat_p, W.ldc);
    for (int l = 0; l < nt; ++l) {
        const F32Pair in = l == 0 ? concat_p : P(W.tact[l - 1], W.ldt[l - 1]);
        const bool last = l == nt - 1;
        if ((r = train_linear_fwd(B, top->dims[l + 1], top->dims[l], in, P(W.tW[l], ldf(top->dims[l])), top->b[l],
                                  last ? F(W.z) : F(W.tact[l][0]), last ? nullptr : F(W.tact[l][1]), W.ldt[l], !last,
                                  last ? nullptr : U(W.tbits[l]), err, st)))
            return r;
    }

    // ---- loss and dL/dz
    float* dz = F(W.dz);
    if ((r = launch_bce(B, F(W.z), labels, dz, y_hat, F(W.lpart), GF(G.loss), st))) return r;
    if (loss && cudaMemcpyAsync(loss, GF(G.loss), sizeof(float), cudaMemcpyDeviceToDevice, st) != cudaSuccess)
        return DLRM_ERR_CUDA;

    // ---- top MLP backward: cur = dL/d(pre-activation of layer l)
    F32Pair cur{dz, nullptr, 1};
    int pp = 0;           // next gradient pair buffer
    bool csum_ok = false;  // W.csum holds the column sums of cur per 32-row group
    for (int l = nt - 1; l >= 0; --l) {
        const F32Pair in = l == 0 ? concat_p : P(W.tact[l - 1], W.ldt[l - 1]);
        const int N = top->dims[l + 1], Kin = top->dims[l];
        const F32Pair Wp = P(W.tW[l], ldf(Kin));
        if ((r = train_linear_wgrad(B, N, Kin, cur, in, GF(G.tdW[l]), ldf(Kin), GF(G.tdb[l]),
                                    csum_ok ? F(W.csum) : nullptr, F(W.wscratch), err, st)))
            return r;
        csum_ok = false;
        if (l > 0) {
            const int ldo = W.gmax;
            if ((r = train_linear_dgrad(B, N, Kin, cur, Wp, in, U(W.tbits[l - 1]), F(W.g[pp][0]), F(W.g[pp][1]), ldo,
                                        F(W.csum), &csum_ok, err, st)))
                return r;
            cur = F32Pair{F(W.g[pp][0]), F(W.g[pp][1]), ldo};
            pp ^= 1;
        } else {
            if ((r = train_linear_dgrad(B, N, Kin, cur, Wp, F32Pair{nullptr, nullptr, 0}, nullptr, F(W.dcat), nullptr,
                                        W.ldc, nullptr, nullptr, err, st)))
                return r;
        }
    }
    // d(concat) -> gradient of the last bottom layer's pre-activation (ReLU mask applied) and dE
    if (W.tc) {
        if ((r = launch_interact_bwd_tc(tm, tables, K, d, B, offsets, indices, nnz, xd_pair, F(W.dcat), W.ldc,
                                        F(W.g[pp][0]), F(W.g[pp][1]), d, GF(G.dE), err, st)))
            return r;
    } else {
        if ((r = launch_interact_bwd(B, K, d, x_dense, E, F(W.dcat), W.ldc, F(W.dxd), GF(G.dE), st))) return r;
        if ((r = launch_split_pair(B, d, F(W.dxd), d, F(W.g[pp][0]), F(W.g[pp][1]), d, st))) return r;
    }
    cur = F32Pair{F(W.g[pp][0]), F(W.g[pp][1]), d};
    pp ^= 1;
    csum_ok = false;
    for (int l = nb - 1; l >= 0; --l) {
        const F32Pair in = l == 0 ? dense_in : P(W.bact[l - 1], W.ldb[l - 1]);
        const int N = bot->dims[l + 1], Kin = bot->dims[l];
        if ((r = train_linear_wgrad(B, N, Kin, cur, in, GF(G.bdW[l]), ldf(Kin), GF(G.bdb[l]),
                                    csum_ok ? F(W.csum) : nullptr, F(W.wscratch), err, st)))
            return r;
        csum_ok = false;
        if (l > 0) {
            const int ldo = W.gmax;
            // the first layer's bias gradient comes with its weight gradient (one pass over dy): no column sums
            if ((r = train_linear_dgrad(B, N, Kin, cur, P(W.bW[l], ldf(Kin)), in, U(W.bbits[l - 1]), F(W.g[pp][0]),
                                        F(W.g[pp][1]), ldo, l - 1 > 0 ? F(W.csum) : nullptr, &csum_ok, err, st)))
                return r;
            cur = F32Pair{F(W.g[pp][0]), F(W.g[pp][1]), ldo};
            pp ^= 1;
        }
    }

    // ---- embedding rows: sort occurrences by row, cut segments and pieces
    if (pooled) return DLRM_OK;
    int sorted_buf = 0;
    if ((r = launch_sparse_prepare(K, B, tm, total_rows_of(tm, K), offsets, indices, nnz, g + G.sparse, G.sp, err,
                                   &sorted_buf, st)))
        return r;
    return DLRM_OK;
}

// Shapes of the pooled-input step: the same MLP and width rules as check_train, for K vectors of width d.
dlrm_status check_pooled(int K, int d, const dlrm_mlp* bot, const dlrm_mlp* top, int B) {
    if (K < 1 || d < 1 || B < 0 || !bot || !top || !bot->dims || !top->dims || !bot->W || !bot->b || !top->W ||
        !top->b)
        return DLRM_ERR_INVALID_ARG;
    if (K > DLRM_MAX_TABLES || bot->n_layers < 1 || top->n_layers < 1 || bot->n_layers > DLRM_MAX_LAYERS ||
        top->n_layers > DLRM_MAX_LAYERS)
        return DLRM_ERR_UNSUPPORTED;
    if (bot->dt != DLRM_F32 || top->dt != DLRM_F32) return DLRM_ERR_UNSUPPORTED;
    for (int l = 0; l <= bot->n_layers; ++l)
        if (bot->dims[l] < 1) return DLRM_ERR_INVALID_ARG;
    for (int l = 0; l <= top->n_layers; ++l)
        if (top->dims[l] < 1) return DLRM_ERR_INVALID_ARG;
    for (int l = 0; l < bot->n_layers; ++l)
        if (!bot->W[l] || !bot->b[l]) return DLRM_ERR_INVALID_ARG;
    for (int l = 0; l < top->n_layers; ++l)
        if (!top->W[l] || !top->b[l]) return DLRM_ERR_INVALID_ARG;
    if (bot->dims[bot->n_layers] != d || top->dims[0] != d + K * (K + 1) / 2 || top->dims[top->n_layers] != 1)
        return DLRM_ERR_INVALID_ARG;
    if (d % 4 || interact_bwd_smem(K, d) > 227 * 1024 || interact_smem_per_sample(K, d) > 227 * 1024)
        return DLRM_ERR_UNSUPPORTED;
    return DLRM_OK;
}

}  // namespace

extern "C" {

dlrm_status dlrm_backward(const dlrm_tables* T, const dlrm_mlp* bot, const dlrm_mlp* top, int B, const float* dense,
                          const int32_t* offsets, const int32_t* indices, int64_t nnz, const float* labels,
                          float* loss, float* y_hat, void* grads, size_t grads_bytes, void* ws, size_t ws_bytes,
                          dlrm_stream stream) {
    TableMeta tm;
    dlrm_status r = check_train(T, bot, top, B, tm);
    if (r) return r;
    if (nnz < 0 || nnz >= (int64_t(1) << 31)) return DLRM_ERR_INVALID_ARG;
    if (!ws || !aligned16(ws) || !grads || !aligned16(grads)) return DLRM_ERR_WORKSPACE;
    if (ws_bytes < dlrm_workspace_size(T, bot, top, B, 1) || grads_bytes < grads_layout(T->K, T->d, bot, top, B, nnz).total)
        return DLRM_ERR_WORKSPACE;
    if (B == 0) return DLRM_OK;
    if (!dense || !offsets || (nnz > 0 && !indices) || !labels) return DLRM_ERR_INVALID_ARG;
    const int K = T->K, d = T->d;
    const TrainWs W = train_ws(K, d, total_rows_of(tm, K), true, bot, top, B);
    const Grads G = grads_layout(K, d, bot, top, B, nnz);
    return backward_impl(K, d, tm, static_cast<const float*>(T->data), bot, top, B, dense, offsets, indices, nnz,
                         nullptr, labels, loss, y_hat, grads, ws, W, G, cs(stream));
}

size_t dlrm_backward_pooled_workspace_size(int K, int d, const dlrm_mlp* bot, const dlrm_mlp* top, int B) {
    if (check_pooled(K, d, bot, top, B) != DLRM_OK) return 0;
    return train_ws(K, d, 0, false, bot, top, B).total;
}

size_t dlrm_grads_pooled_size(int K, int d, const dlrm_mlp* bot, const dlrm_mlp* top, int B) {
    if (check_pooled(K, d, bot, top, B) != DLRM_OK) return 0;
    return grads_layout(K, d, bot, top, B, 0).total;
}

dlrm_status dlrm_grads_pooled_offsets(int K, int d, const dlrm_mlp* bot, const dlrm_mlp* top, int B, size_t* bot_dW,
                                      size_t* bot_db, size_t* top_dW, size_t* top_db, size_t* dE, size_t* loss,
                                      size_t* dense_end) {
    dlrm_status r = check_pooled(K, d, bot, top, B);
    if (r) return r;
    const Grads G = grads_layout(K, d, bot, top, B, 0);
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
    if (dense_end) *dense_end = G.dE;
    return DLRM_OK;
}

dlrm_status dlrm_backward_pooled(int K, int d, const dlrm_mlp* bot, const dlrm_mlp* top, int B, const float* dense,
                                 const float* pooled, const float* labels, float* loss, float* y_hat, void* grads,
                                 size_t grads_bytes, void* ws, size_t ws_bytes, dlrm_stream stream) {
    dlrm_status r = check_pooled(K, d, bot, top, B);
    if (r) return r;
    if (!ws || !aligned16(ws) || !grads || !aligned16(grads)) return DLRM_ERR_WORKSPACE;
    const TrainWs W = train_ws(K, d, 0, false, bot, top, B);
    const Grads G = grads_layout(K, d, bot, top, B, 0);
    if (ws_bytes < W.total || grads_bytes < G.total) return DLRM_ERR_WORKSPACE;
    if (B == 0) return DLRM_OK;
    if (!dense || !pooled || !labels || !aligned16(pooled)) return DLRM_ERR_INVALID_ARG;
    TableMeta tm;
    return backward_impl(K, d, tm, nullptr, bot, top, B, dense, nullptr, nullptr, 0, pooled, labels, loss, y_hat,
                         grads, ws, W, G, cs(stream));
}

dlrm_status dlrm_mlp_sgd(int K, int d, const dlrm_mlp* bot, const dlrm_mlp* top, int B, float lr, const void* grads,
                         size_t grads_bytes, dlrm_stream stream) {
    dlrm_status r = check_pooled(K, d, bot, top, B);
    if (r) return r;
    const Grads G = grads_layout(K, d, bot, top, B, 0);
    if (!grads || !aligned16(grads) || grads_bytes < G.dE) return DLRM_ERR_WORKSPACE;
    const char* g = static_cast<const char*>(grads);
    cudaStream_t st = cs(stream);
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


dlrm_status dlrm_sparse_sgd(const dlrm_tables* T, const dlrm_mlp* bot, const dlrm_mlp* top, int B, int64_t nnz,
                            float lr, void* grads, size_t grads_bytes, int32_t* n_touched, dlrm_stream stream) {
    TableMeta tm;
    dlrm_status r = check_train(T, bot, top, B, tm);
    if (r) return r;
    if (nnz < 0 || nnz >= (int64_t(1) << 31)) return DLRM_ERR_INVALID_ARG;
    if (!grads || !aligned16(grads) || grads_bytes < grads_layout(T->K, T->d, bot, top, B, nnz).total)
        return DLRM_ERR_WORKSPACE;
    if (B == 0) return DLRM_OK;
    const Grads G = grads_layout(T->K, T->d, bot, top, B, nnz);
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
                                     int64_t nnz, const void* grads, size_t grads_bytes, uint32_t* rows,
                                     float* row_grads, int32_t* n_rows, dlrm_stream stream) {
    TableMeta tm;
    dlrm_status r = check_train(T, bot, top, B, tm);
    if (r) return r;
    if (nnz < 0 || nnz >= (int64_t(1) << 31)) return DLRM_ERR_INVALID_ARG;
    if (!grads || !aligned16(grads) || grads_bytes < grads_layout(T->K, T->d, bot, top, B, nnz).total)
        return DLRM_ERR_WORKSPACE;
    if (!rows || !row_grads || !n_rows) return DLRM_ERR_INVALID_ARG;
    if (B == 0) return DLRM_OK;
    const Grads G = grads_layout(T->K, T->d, bot, top, B, nnz);
    const char* g = static_cast<const char*>(grads);
    const int sorted = radix_passes(total_rows_of(tm, T->K)) & 1;
    return launch_sparse_apply(T->d, g + G.sparse, G.sp, sorted, reinterpret_cast<const float*>(g + G.dE), 0.f,
                               nullptr, row_grads, rows, n_rows, cs(stream));
}

}  // extern "C"
