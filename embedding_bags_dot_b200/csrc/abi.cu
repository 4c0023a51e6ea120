// extern "C" entry points of libdlrm: argument checks, workspace carving and
// launch order. Every operation runs in the kernels of this library; nothing
// here computes on the host beyond sizes and table bases.
#include <stdio.h>
#include <string.h>

#include <atomic>

#include <algorithm>

#include "common.cuh"
#include "kernels.cuh"

using namespace dlrm;

namespace dlrm {
static std::atomic<unsigned long long> g_launches{0};
void count_launch() { g_launches.fetch_add(1, std::memory_order_relaxed); }
}  // namespace dlrm

namespace {

inline bool aligned16(const void* p) { return ((uintptr_t)p & 15u) == 0; }
inline bool valid_dt(int dt) { return dt == DLRM_F32 || dt == DLRM_F16 || dt == DLRM_BF16; }
inline bool valid_table_dt(int dt) { return valid_dt(dt) || dt == DLRM_U8ROW; }
inline cudaStream_t cs(dlrm_stream s) { return reinterpret_cast<cudaStream_t>(s); }

dlrm_status check_tables(const dlrm_tables* T, TableMeta& tm) {
    if (!T || !T->rows || !T->data) return DLRM_ERR_INVALID_ARG;
    if (T->K < 1 || T->d < 1 || !valid_table_dt(T->dt)) return DLRM_ERR_INVALID_ARG;
    if (T->K > DLRM_MAX_TABLES) return DLRM_ERR_UNSUPPORTED;
    if (!aligned16(T->data)) return DLRM_ERR_INVALID_ARG;
    long long acc = 0;
    for (int k = 0; k < T->K; ++k) {
        if (T->rows[k] < 1) return DLRM_ERR_INVALID_ARG;
        tm.base[k] = acc;
        tm.rows[k] = T->rows[k];
        acc += T->rows[k];
    }
    // uint8 records are read by the fused tensor-core kernel only (d = 64, 128)
    if (T->dt == DLRM_U8ROW ? !(T->d == 64 || T->d == 128) : !gather_supported(T->d, T->dt)) return DLRM_ERR_UNSUPPORTED;
    return DLRM_OK;
}

dlrm_status check_bags(int B, const int32_t* offsets, const int32_t* indices, int64_t nnz) {
    if (B < 0 || nnz < 0 || nnz >= (int64_t(1) << 31)) return DLRM_ERR_INVALID_ARG;
    if (B > 0 && !offsets) return DLRM_ERR_INVALID_ARG;
    if (nnz > 0 && !indices) return DLRM_ERR_INVALID_ARG;
    return DLRM_OK;
}

dlrm_status check_mlp(const dlrm_mlp* m) {
    if (!m || !m->dims || !m->W || !m->b) return DLRM_ERR_INVALID_ARG;
    if (m->n_layers < 1 || m->n_layers > DLRM_MAX_LAYERS || !valid_dt(m->dt)) return DLRM_ERR_INVALID_ARG;
    for (int l = 0; l <= m->n_layers; ++l)
        if (m->dims[l] < 1) return DLRM_ERR_INVALID_ARG;
    for (int l = 0; l < m->n_layers; ++l)
        if (!m->W[l] || !m->b[l] || !aligned16(m->W[l])) return DLRM_ERR_INVALID_ARG;
    return DLRM_OK;
}

// Bytes of one activation buffer: the widest layer input of m (the first layer's input
// is converted into such a buffer when it does not come in the MLP's dtype).
size_t hidden_bytes(const dlrm_mlp* m, int B) {
    size_t w = 0;
    for (int l = 0; l < m->n_layers; ++l) {
        const size_t b = (size_t)dlrm_ld(m->dims[l], m->dt) * esize(m->dt);
        if (b > w) w = b;
    }
    return w * (size_t)B;
}

// dlrm_mlp_fwd's workspace after the error record: `nact` activation buffers of `act` bytes (the
// widest hidden layer output; none for one layer, one for two), then the input converted to the MLP's
// dtype when it comes in another one.
struct MlpWs {
    size_t act, cvt, f32tc, total;
    int nact;
};

// fp32 MLPs run their layers on the tensor cores as 3xTF32 GEMMs, whose operands are (hi, lo) pairs: the
// split weights of every layer, the split input, two pair buffers for the hidden outputs and the last
// layer's pair output. Byte offsets relative to the start of this region.
struct F32TcWs {
    size_t w[DLRM_MAX_LAYERS][2], in[2], act[2][2], total;
    int ld_in, ld_act;
};

F32TcWs f32tc_ws(const dlrm_mlp* m, int B) {
    F32TcWs W{};
    size_t off = 0;
    auto take = [&](size_t bytes) {
        const size_t o = off;
        off = align_up(off + bytes, 256);
        return o;
    };
    int widest = 1, widest_in = 1;
    for (int l = 0; l < m->n_layers; ++l) {
        for (int h = 0; h < 2; ++h) W.w[l][h] = take(sizeof(float) * (size_t)m->dims[l + 1] * dlrm_ld(m->dims[l], DLRM_F32));
        widest = std::max(widest, m->dims[l + 1]);
        widest_in = std::max(widest_in, m->dims[l]);
    }
    W.ld_in = dlrm_ld(std::max(widest_in, widest), DLRM_F32);   // plain buffers: any layer's input or output
    W.ld_act = W.ld_in;                                            // pair buffers: likewise
    for (int h = 0; h < 2; ++h) W.in[h] = take(sizeof(float) * (size_t)B * W.ld_in);
    for (int p = 0; p < 2; ++p)
        for (int h = 0; h < 2; ++h) W.act[p][h] = take(sizeof(float) * (size_t)B * W.ld_act);
    W.total = off;
    return W;
}

MlpWs mlp_ws(const dlrm_mlp* m, int B, dlrm_dtype in_dt) {
    MlpWs w{};
    size_t row = 0;
    for (int l = 1; l < m->n_layers; ++l) row = std::max(row, (size_t)dlrm_ld(m->dims[l], m->dt) * esize(m->dt));
    w.act = align_up(row * (size_t)B, 256);
    w.nact = m->n_layers >= 3 ? 2 : m->n_layers - 1;
    const bool conv = in_dt != m->dt && m->dt != DLRM_F32;
    w.cvt = conv ? align_up((size_t)dlrm_ld(m->dims[0], m->dt) * esize(m->dt) * (size_t)B, 256) : 0;
    w.f32tc = m->dt == DLRM_F32 ? f32tc_ws(m, B).total : 0;
    w.total = DLRM_ERR_RECORD_BYTES + (size_t)w.nact * w.act + w.cvt + w.f32tc;
    return w;
}

struct FwdLayout {
    size_t x_dense, concat, act0, act1, cvt, offs, lscratch, f32tc, total;
};

FwdLayout fwd_layout(const dlrm_tables* T, const dlrm_mlp* bot, const dlrm_mlp* top, int B) {
    FwdLayout L;
    size_t off = DLRM_ERR_RECORD_BYTES;
    const int d = T->d;
    const int ldc = dlrm_ld(top->dims[0], top->dt);   // the concat: d + K(K+1)/2 (dot) or d(K+1) (concat-only)
    L.x_dense = off;
    off = align_up(off + sizeof(float) * (size_t)B * d, 256);
    L.concat = off;
    off = align_up(off + (size_t)B * ldc * esize(top->dt), 256);
    size_t h = hidden_bytes(bot, B);
    const size_t ht = hidden_bytes(top, B);
    if (ht > h) h = ht;
    L.act0 = off;
    off = align_up(off + h, 256);
    L.act1 = off;
    off = align_up(off + h, 256);
    L.cvt = off;
    off = align_up(off + h, 256);
    // offsets derived from bag lengths (dlrm_forward_lengths) and the scan's chunk sums
    const long long nbags = (long long)T->K * B;
    L.offs = off;
    off = align_up(off + sizeof(int32_t) * (size_t)(nbags + 1), 256);
    L.lscratch = off;
    off = align_up(off + sizeof(int) * lengths_scratch_ints(nbags), 256);
    // fp32 MLPs: the 3xTF32 pair buffers of the larger of the two (one MLP runs at a time)
    const size_t f32 = std::max(bot->dt == DLRM_F32 ? f32tc_ws(bot, B).total : 0,
                                top->dt == DLRM_F32 ? f32tc_ws(top, B).total : 0);
    L.f32tc = off;
    off = align_up(off + f32, 256);
    L.total = off;
    return L;
}

// The MLP chain: ReLU after hidden layers, final_act after the last layer. An fp32 input
// to a 16-bit MLP is first converted (into cvt) so that every layer can take the
// tensor-core path.
// A layer of an fp32 MLP goes to the 3xTF32 tensor-core GEMM (256x256 tiles on SM pairs) when the batch
// gives it enough tiles to be worth the pair conversions: at 2,048 rows (the medium configuration) the
// CUDA-core layers measured faster in total. The 13-wide first bottom layer stays on the CUDA cores.
bool f32_layer_on_tc(int M, int N, int K) { return M >= 4096 && N >= 64 && K > 16; }

// fp32 MLP with tensor-core layers: buffers in `tc` (F32TcWs layout): two (hi, lo) pair buffers for the
// tensor-core layers' inputs and outputs, two plain buffers for the CUDA-core layers'. A tensor-core layer
// takes a pair (a plain input is split first), a CUDA-core layer a plain input (a pair is merged first);
// the last layer writes `out` plain.
dlrm_status run_mlp_f32(const dlrm_mlp* m, int B, const float* in, int ld_in, float* out, int ld_out, int final_act,
                        char* tc, ErrRecord* err, cudaStream_t st) {
    const F32TcWs W = f32tc_ws(m, B);
    auto F = [&](size_t o) { return reinterpret_cast<float*>(tc + o); };
    float* pairs[2][2] = {{F(W.act[0][0]), F(W.act[0][1])}, {F(W.act[1][0]), F(W.act[1][1])}};
    float* plain[2] = {F(W.in[0]), F(W.in[1])};
    dlrm_status r;
    // cur: the layer input; where = 0/1 for pair buffer 0/1, 2/3 for plain buffer 0/1, -1 for the caller's input
    F32Pair cur{in, nullptr, ld_in};
    int where = -1;
    for (int l = 0; l < m->n_layers; ++l) {
        const int K = m->dims[l], N = m->dims[l + 1], ldw = dlrm_ld(K, DLRM_F32);
        const bool last = l == m->n_layers - 1;
        if (!(f32_layer_on_tc(B, N, K) && (!last || final_act == DLRM_ACT_RELU))) {
            if (cur.lo) {                       // merge the pair into a plain buffer
                if ((r = launch_merge_pair(B, K, cur.hi, cur.lo, cur.ld, plain[0], W.ld_in, st))) return r;
                cur = F32Pair{plain[0], nullptr, W.ld_in};
                where = 2;
            }
            if (last)
                return launch_linear(B, N, K, cur.hi, DLRM_F32, cur.ld, m->W[l], DLRM_F32, ldw, m->b[l], out, DLRM_F32,
                                     ld_out, final_act, err, st);
            const int dst = where == 2 ? 1 : 0;
            if ((r = launch_linear(B, N, K, cur.hi, DLRM_F32, cur.ld, m->W[l], DLRM_F32, ldw, m->b[l], plain[dst],
                                   DLRM_F32, W.ld_in, DLRM_ACT_RELU, err, st)))
                return r;
            cur = F32Pair{plain[dst], nullptr, W.ld_in};
            where = 2 + dst;
            continue;
        }
        if (!cur.lo) {                          // split the plain input into a pair buffer
            if ((r = launch_split_pair(B, K, cur.hi, cur.ld, pairs[0][0], pairs[0][1], W.ld_act, st))) return r;
            cur = F32Pair{pairs[0][0], pairs[0][1], W.ld_act};
            where = 0;
        }
        if ((r = launch_split_pair(N, K, static_cast<const float*>(m->W[l]), ldw, F(W.w[l][0]), F(W.w[l][1]), ldw, st)))
            return r;
        const int dst = where == 0 ? 1 : 0;
        if ((r = train_linear_fwd(B, N, K, cur, F32Pair{F(W.w[l][0]), F(W.w[l][1]), ldw}, m->b[l], pairs[dst][0],
                                  pairs[dst][1], W.ld_act, true, nullptr, err, st)))
            return r;
        cur = F32Pair{pairs[dst][0], pairs[dst][1], W.ld_act};
        where = dst;
        if (last) return launch_merge_pair(B, N, cur.hi, cur.lo, cur.ld, out, ld_out, st);
    }
    return DLRM_OK;
}

dlrm_status run_mlp(const dlrm_mlp* m, int B, const void* in, dlrm_dtype in_dt, int ld_in, float* out, int ld_out,
                    int final_act, void* act0, void* act1, void* cvt, ErrRecord* err, cudaStream_t st,
                    char* f32tc = nullptr) {
    if (m->dt == DLRM_F32 && in_dt == DLRM_F32 && f32tc) {
        bool any = false;
        for (int l = 0; l < m->n_layers; ++l) any |= f32_layer_on_tc(B, m->dims[l + 1], m->dims[l]);
        if (any)
            return run_mlp_f32(m, B, static_cast<const float*>(in), ld_in, out, ld_out, final_act, f32tc, err, st);
    }
    // three bf16 layers from fp32 input (the bottom MLP): one kernel, the hidden activations never in HBM
    if (mlp3_tc_supported(m, B, in_dt, ld_in, out, ld_out, final_act))
        return launch_mlp3_tc(m, B, static_cast<const float*>(in), ld_in, out, ld_out, err, st);
    const void* cur = in;
    dlrm_dtype cur_dt = in_dt;
    int cur_ld = ld_in;
    if (in_dt != m->dt && m->dt != DLRM_F32 && cvt) {
        const int ldk = dlrm_ld(m->dims[0], m->dt);
        dlrm_status r = launch_convert(B, m->dims[0], in, in_dt, ld_in, cvt, m->dt, ldk, st);
        if (r != DLRM_OK) return r;
        cur = cvt;
        cur_dt = m->dt;
        cur_ld = ldk;
    }
    for (int l = 0; l < m->n_layers; ++l) {
        const int K = m->dims[l], N = m->dims[l + 1];
        const int ldw = dlrm_ld(K, m->dt);
        dlrm_status r;
        // last hidden layer followed by the one-column sigmoid output: one kernel, the hidden output unstored
        if (l == m->n_layers - 2 && m->dims[l + 2] == 1 && final_act == DLRM_ACT_SIGMOID && ld_out == 1 &&
            linear_tc_logit_supported(B, N, K, cur, cur_dt, cur_ld, m->W[l], m->dt, ldw, m->b[l]))
            return launch_linear_tc_logit(B, N, K, cur, cur_dt, cur_ld, m->W[l], ldw, m->b[l], m->W[l + 1],
                                          m->b[l + 1], out, err, st);
        if (l == m->n_layers - 1) {
            r = launch_linear(B, N, K, cur, cur_dt, cur_ld, m->W[l], m->dt, ldw, m->b[l], out, DLRM_F32, ld_out,
                              final_act, err, st);
        } else {
            void* dst = (l & 1) ? act1 : act0;
            const int ldd = dlrm_ld(N, m->dt);
            r = launch_linear(B, N, K, cur, cur_dt, cur_ld, m->W[l], m->dt, ldw, m->b[l], dst, m->dt, ldd,
                              DLRM_ACT_RELU, err, st);
            cur = dst;
            cur_dt = m->dt;
            cur_ld = ldd;
        }
        if (r != DLRM_OK) return r;
    }
    return DLRM_OK;
}

}  // namespace

extern "C" {

uint64_t dlrm_launch_count(void) { return g_launches.load(std::memory_order_relaxed); }

dlrm_status dlrm_set_wait_polls(int64_t polls) {
    if (set_wait_polls_gemm_tc(polls) != cudaSuccess || set_wait_polls_embbag_mma(polls) != cudaSuccess ||
        set_wait_polls_mlp3(polls) != cudaSuccess ||
        set_wait_polls_embbag_cat(polls) != cudaSuccess || set_wait_polls_interact_tc(polls) != cudaSuccess)
        return DLRM_ERR_CUDA;
    return DLRM_OK;
}

int dlrm_ld(int n, dlrm_dtype dt) {
    const int per = 16 / (int)esize(dt);
    return (n + per - 1) / per * per;
}

const char* dlrm_status_str(dlrm_status s) {
    switch (s) {
        case DLRM_OK: return "ok";
        case DLRM_ERR_INVALID_ARG: return "invalid argument";
        case DLRM_ERR_UNSUPPORTED: return "unsupported";
        case DLRM_ERR_INDEX_OOB: return "index out of range (skipped)";
        case DLRM_ERR_BAD_OFFSETS: return "bad bag offsets (bag pooled to zero)";
        case DLRM_ERR_TIMEOUT: return "bounded wait timed out";
        case DLRM_ERR_CUDA: return "CUDA error";
        case DLRM_ERR_WORKSPACE: return "workspace too small or misaligned";
    }
    return "unknown status";
}

size_t dlrm_workspace_size(const dlrm_tables* T, const dlrm_mlp* bot, const dlrm_mlp* top, int B, int training) {
    TableMeta tm;
    if (check_tables(T, tm) != DLRM_OK || check_mlp(bot) != DLRM_OK || check_mlp(top) != DLRM_OK || B < 0) return 0;
    const size_t f = fwd_layout(T, bot, top, B).total;
    if (!training) return f;
    const size_t t = train_workspace_size(T, bot, top, B);
    if (t == 0) return 0;
    return t > f ? t : f;
}

dlrm_status dlrm_check_error(void* ws, size_t ws_bytes, dlrm_stream stream, int64_t* info) {
    if (!ws) return DLRM_ERR_INVALID_ARG;
    if (ws_bytes < DLRM_ERR_RECORD_BYTES) return DLRM_ERR_WORKSPACE;
    ErrRecord h;
    if (cudaMemcpyAsync(&h, ws, sizeof(h), cudaMemcpyDeviceToHost, cs(stream)) != cudaSuccess) return DLRM_ERR_CUDA;
    if (cudaStreamSynchronize(cs(stream)) != cudaSuccess) return DLRM_ERR_CUDA;
    if (cudaMemsetAsync(ws, 0, sizeof(h), cs(stream)) != cudaSuccess) return DLRM_ERR_CUDA;
    if (info) {
        info[0] = h.flags;
        info[1] = (int64_t)h.n_oob;
        info[2] = (int64_t)h.n_bad;
    }
    if (h.flags & ERR_BAD_OFFSETS) return DLRM_ERR_BAD_OFFSETS;
    if (h.flags & ERR_OOB) return DLRM_ERR_INDEX_OOB;
    if (h.flags & ERR_TIMEOUT) return DLRM_ERR_TIMEOUT;
    return DLRM_OK;
}

dlrm_status dlrm_embbag_fwd(const dlrm_tables* T, int B, const int32_t* offsets, const int32_t* indices,
                            int64_t nnz, float* pooled, int32_t* bag_len, void* ws, size_t ws_bytes,
                            dlrm_stream stream) {
    TableMeta tm;
    dlrm_status r = check_tables(T, tm);
    if (r != DLRM_OK) return r;
    if ((r = check_bags(B, offsets, indices, nnz)) != DLRM_OK) return r;
    if (!ws || !aligned16(ws) || ws_bytes < DLRM_ERR_RECORD_BYTES) return DLRM_ERR_WORKSPACE;
    if (B > 0 && (!pooled || !aligned16(pooled))) return DLRM_ERR_INVALID_ARG;
    if (B == 0) return DLRM_OK;
    return launch_embbag(tm, T->data, T->dt, T->K, T->d, B, offsets, indices, nnz, pooled, bag_len,
                         static_cast<ErrRecord*>(ws), cs(stream));
}

dlrm_status dlrm_interact_fwd(int B, int K, int d, const float* x_dense, const float* pooled, void* concat, int ld,
                              dlrm_dtype out_dt, dlrm_stream stream) {
    if (B < 0 || K < 1 || d < 1 || !valid_dt(out_dt)) return DLRM_ERR_INVALID_ARG;
    if (K > DLRM_MAX_TABLES) return DLRM_ERR_UNSUPPORTED;
    if (ld < d + K * (K + 1) / 2) return DLRM_ERR_INVALID_ARG;
    if (B == 0) return DLRM_OK;
    if (!x_dense || !pooled || !concat || !aligned16(x_dense) || !aligned16(pooled) || !aligned16(concat))
        return DLRM_ERR_INVALID_ARG;
    return launch_interact(B, K, d, x_dense, pooled, concat, ld, out_dt, cs(stream));
}

dlrm_status dlrm_embbag_interact_fwd(const dlrm_tables* T, int B, const int32_t* offsets, const int32_t* indices,
                                     int64_t nnz, const float* x_dense, void* concat, int ld, dlrm_dtype out_dt,
                                     void* ws, size_t ws_bytes, dlrm_stream stream) {
    TableMeta tm;
    dlrm_status r = check_tables(T, tm);
    if (r != DLRM_OK) return r;
    if ((r = check_bags(B, offsets, indices, nnz)) != DLRM_OK) return r;
    if (!valid_dt(out_dt) || ld < T->d + T->K * (T->K + 1) / 2) return DLRM_ERR_INVALID_ARG;
    if (!ws || !aligned16(ws) || ws_bytes < DLRM_ERR_RECORD_BYTES) return DLRM_ERR_WORKSPACE;
    if (B == 0) return DLRM_OK;
    if (!x_dense || !concat || !aligned16(x_dense) || !aligned16(concat)) return DLRM_ERR_INVALID_ARG;
    return launch_embbag_interact(tm, T->data, T->dt, T->K, T->d, B, offsets, indices, nnz, x_dense, concat, ld,
                                  out_dt, static_cast<ErrRecord*>(ws), cs(stream));
}

dlrm_status dlrm_mlp_fwd(const dlrm_mlp* mlp, int B, const void* in, dlrm_dtype in_dt, int ld_in, float* out,
                         int ld_out, int final_act, void* ws, size_t ws_bytes, dlrm_stream stream) {
    dlrm_status r = check_mlp(mlp);
    if (r != DLRM_OK) return r;
    if (B < 0 || !valid_dt(in_dt) || ld_in < mlp->dims[0] || ld_out < mlp->dims[mlp->n_layers]) return DLRM_ERR_INVALID_ARG;
    if (final_act < DLRM_ACT_NONE || final_act > DLRM_ACT_SIGMOID) return DLRM_ERR_INVALID_ARG;
    if (B == 0) return DLRM_OK;
    if (!in || !out) return DLRM_ERR_INVALID_ARG;
    const MlpWs L = mlp_ws(mlp, B, in_dt);
    if (!ws || !aligned16(ws) || ws_bytes < L.total) return DLRM_ERR_WORKSPACE;
    char* w = static_cast<char*>(ws) + DLRM_ERR_RECORD_BYTES;
    return run_mlp(mlp, B, in, in_dt, ld_in, out, ld_out, final_act, w, w + L.act, w + (size_t)L.nact * L.act,
                   static_cast<ErrRecord*>(ws), cs(stream), L.f32tc ? w + (size_t)L.nact * L.act + L.cvt : nullptr);
}

size_t dlrm_mlp_workspace_size(const dlrm_mlp* mlp, int B, dlrm_dtype in_dt) {
    if (check_mlp(mlp) != DLRM_OK || B < 0 || !valid_dt(in_dt)) return 0;
    return mlp_ws(mlp, B, in_dt).total;
}

}  // extern "C"

namespace dlrm {

// Every host-side check of the forward pass (dot interaction, or concat-only when cat), in the order the
// entry points apply them, before anything is launched. ws_bytes is the workspace's size.
dlrm_status forward_check(const dlrm_tables* T, const dlrm_mlp* bot, const dlrm_mlp* top, int B, const float* dense,
                          const int32_t* offsets, const int32_t* indices, int64_t nnz, const float* y_hat,
                          const void* ws, size_t ws_bytes, bool cat) {
    TableMeta tm;
    dlrm_status r = check_tables(T, tm);
    if (r != DLRM_OK) return r;
    if ((r = check_bags(B, offsets, indices, nnz)) != DLRM_OK) return r;
    if ((r = check_mlp(bot)) != DLRM_OK || (r = check_mlp(top)) != DLRM_OK) return r;
    const int K = T->K, d = T->d;
    const int width = cat ? d * (K + 1) : d + K * (K + 1) / 2;
    if (bot->dims[bot->n_layers] != d || top->dims[0] != width || top->dims[top->n_layers] != 1)
        return DLRM_ERR_INVALID_ARG;
    if (!ws || !aligned16(ws) || ws_bytes < fwd_layout(T, bot, top, B).total) return DLRM_ERR_WORKSPACE;
    if (B > 0 && (!dense || !y_hat)) return DLRM_ERR_INVALID_ARG;
    return DLRM_OK;
}

}  // namespace dlrm

extern "C" {

namespace {

// The forward pass with the dot interaction (cat = false) or the concat-only one (cat = true).
dlrm_status forward_impl(const dlrm_tables* T, const dlrm_mlp* bot, const dlrm_mlp* top, int B, const float* dense,
                         const int32_t* offsets, const int32_t* indices, int64_t nnz, float* y_hat, void* ws,
                         size_t ws_bytes, dlrm_stream stream, bool cat) {
    dlrm_status r = forward_check(T, bot, top, B, dense, offsets, indices, nnz, y_hat, ws, ws_bytes, cat);
    if (r != DLRM_OK || B == 0) return r;
    TableMeta tm;
    check_tables(T, tm);
    const int K = T->K, d = T->d;
    const int width = cat ? d * (K + 1) : d + K * (K + 1) / 2;
    const FwdLayout L = fwd_layout(T, bot, top, B);
    char* w = static_cast<char*>(ws);
    cudaStream_t st = cs(stream);
    float* x_dense = reinterpret_cast<float*>(w + L.x_dense);
    void* concat = w + L.concat;
    const int ldc = dlrm_ld(width, top->dt);
    ErrRecord* err = reinterpret_cast<ErrRecord*>(w);
    if ((r = run_mlp(bot, B, dense, DLRM_F32, bot->dims[0], x_dense, d, DLRM_ACT_RELU, w + L.act0, w + L.act1,
                     w + L.cvt, err, st, w + L.f32tc)))
        return r;
    r = cat ? launch_embbag_cat(tm, T->data, T->dt, K, d, B, offsets, indices, nnz, x_dense, concat, ldc, top->dt, err,
                                st)
            : launch_embbag_interact(tm, T->data, T->dt, K, d, B, offsets, indices, nnz, x_dense, concat, ldc, top->dt,
                                     err, st);
    if (r) return r;
    return run_mlp(top, B, concat, top->dt, ldc, y_hat, 1, DLRM_ACT_SIGMOID, w + L.act0, w + L.act1, w + L.cvt, err,
                   st, w + L.f32tc);
}

}  // namespace

dlrm_status dlrm_forward(const dlrm_tables* T, const dlrm_mlp* bot, const dlrm_mlp* top, int B, const float* dense,
                         const int32_t* offsets, const int32_t* indices, int64_t nnz, float* y_hat, void* ws,
                         size_t ws_bytes, dlrm_stream stream) {
    return forward_impl(T, bot, top, B, dense, offsets, indices, nnz, y_hat, ws, ws_bytes, stream, false);
}

dlrm_status dlrm_forward_lengths(const dlrm_tables* T, const dlrm_mlp* bot, const dlrm_mlp* top, int B,
                                 const float* dense, const uint8_t* lengths, const int32_t* indices, int64_t nnz,
                                 float* y_hat, void* ws, size_t ws_bytes, dlrm_stream stream) {
    TableMeta tm;
    dlrm_status r = check_tables(T, tm);
    if (r != DLRM_OK) return r;
    if (B < 0 || nnz < 0 || nnz >= (int64_t(1) << 31)) return DLRM_ERR_INVALID_ARG;
    if (B > 0 && !lengths) return DLRM_ERR_INVALID_ARG;
    if ((r = check_mlp(bot)) != DLRM_OK || (r = check_mlp(top)) != DLRM_OK) return r;
    if (!ws || !aligned16(ws)) return DLRM_ERR_WORKSPACE;
    if (B == 0) return DLRM_OK;
    const FwdLayout L = fwd_layout(T, bot, top, B);
    char* w = static_cast<char*>(ws);
    int32_t* offsets = reinterpret_cast<int32_t*>(w + L.offs);
    // every check of the forward pass before the scan is launched (the scan's output stands in for the offsets)
    if ((r = forward_check(T, bot, top, B, dense, offsets, indices, nnz, y_hat, ws, ws_bytes, false)) != DLRM_OK)
        return r;
    if ((r = launch_offsets_from_lengths(lengths, (long long)T->K * B, offsets, reinterpret_cast<int*>(w + L.lscratch),
                                         cs(stream))) != DLRM_OK)
        return r;
    return forward_impl(T, bot, top, B, dense, offsets, indices, nnz, y_hat, ws, ws_bytes, stream, false);
}

size_t dlrm_offsets_from_lengths_workspace_size(int64_t n) {
    if (n < 0) return 0;
    return DLRM_ERR_RECORD_BYTES + sizeof(int) * lengths_scratch_ints(n);
}

dlrm_status dlrm_offsets_from_lengths(const uint8_t* lengths, int64_t n, int32_t* offsets, void* ws,
                                      size_t ws_bytes, dlrm_stream stream) {
    if (n < 0 || (n > 0 && !lengths) || !offsets) return DLRM_ERR_INVALID_ARG;
    if (!ws || !aligned16(ws) || ws_bytes < dlrm_offsets_from_lengths_workspace_size(n)) return DLRM_ERR_WORKSPACE;
    return launch_offsets_from_lengths(lengths, n, offsets,
                                       reinterpret_cast<int*>(static_cast<char*>(ws) + DLRM_ERR_RECORD_BYTES), cs(stream));
}

dlrm_status dlrm_forward_cat(const dlrm_tables* T, const dlrm_mlp* bot, const dlrm_mlp* top, int B, const float* dense,
                             const int32_t* offsets, const int32_t* indices, int64_t nnz, float* y_hat, void* ws,
                             size_t ws_bytes, dlrm_stream stream) {
    return forward_impl(T, bot, top, B, dense, offsets, indices, nnz, y_hat, ws, ws_bytes, stream, true);
}

dlrm_status dlrm_embbag_cat_fwd(const dlrm_tables* T, int B, const int32_t* offsets, const int32_t* indices,
                                int64_t nnz, const float* x_dense, void* concat, int ld, dlrm_dtype out_dt, void* ws,
                                size_t ws_bytes, dlrm_stream stream) {
    TableMeta tm;
    dlrm_status r = check_tables(T, tm);
    if (r != DLRM_OK) return r;
    if ((r = check_bags(B, offsets, indices, nnz)) != DLRM_OK) return r;
    if (!valid_dt(out_dt) || ld < T->d * (T->K + 1)) return DLRM_ERR_INVALID_ARG;
    if (!ws || !aligned16(ws) || ws_bytes < DLRM_ERR_RECORD_BYTES) return DLRM_ERR_WORKSPACE;
    if (B == 0) return DLRM_OK;
    if (!x_dense || !concat) return DLRM_ERR_INVALID_ARG;
    return launch_embbag_cat(tm, T->data, T->dt, T->K, T->d, B, offsets, indices, nnz, x_dense, concat, ld, out_dt,
                             static_cast<ErrRecord*>(ws), cs(stream));
}

}  // extern "C"
