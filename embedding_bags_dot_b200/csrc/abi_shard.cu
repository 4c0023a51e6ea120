// extern "C" entry points for table-wise model parallelism: the embedding tables are split into
// contiguous ranges, one per rank, and the pooled vectors cross between ranks by an all-to-all (the
// hybrid scheme of the arXiv 1906.00091 index page, Abstract: model-parallel embedding tables,
// data-parallel fully connected layers; the science.uptrusthq.com citation snippet: all-to-all
// communication of the embedding lookup results; "DLRM", briansu.co, section 5).
//
// The exchange itself is the caller's collective (NCCL all-to-all over NVLink through
// torch.distributed). These calls place the received blocks (strided device copies) and run the owner's
// half of the sparse update from the gradients the exchange brings back.
#include "common.cuh"
#include "kernels.cuh"

using namespace dlrm;

namespace {

inline cudaStream_t cs_(dlrm_stream s) { return reinterpret_cast<cudaStream_t>(s); }

// The parts must tile tables 0 .. K-1 in order.
bool parts_ok(int K, int n_parts, const int* first_table, const int* n_tables) {
    if (n_parts < 1 || !first_table || !n_tables) return false;
    int next = 0;
    for (int p = 0; p < n_parts; ++p) {
        if (first_table[p] != next || n_tables[p] < 0) return false;
        next += n_tables[p];
    }
    return next == K;
}

dlrm_status check_sgd_tables(const dlrm_tables* T, TableMeta& tm) {
    if (!T || !T->rows || !T->data || T->K < 1 || T->d < 1) return DLRM_ERR_INVALID_ARG;
    if (T->K > DLRM_MAX_TABLES) return DLRM_ERR_UNSUPPORTED;
    if (T->dt != DLRM_F32 || T->d % 4) return DLRM_ERR_UNSUPPORTED;
    if (((uintptr_t)T->data & 15) != 0) return DLRM_ERR_INVALID_ARG;
    long long acc = 0;
    for (int k = 0; k < T->K; ++k) {
        if (T->rows[k] < 1) return DLRM_ERR_INVALID_ARG;
        tm.base[k] = acc;
        tm.rows[k] = T->rows[k];
        acc += T->rows[k];
    }
    if (acc >= 0xFFFFFFFFll) return DLRM_ERR_UNSUPPORTED;   // row ids are sorted as 32-bit keys
    return DLRM_OK;
}

}  // namespace

extern "C" {

dlrm_status dlrm_pooled_assemble(int B, int K, int d, int n_parts, const int* first_table, const int* n_tables,
                                 const float* const* parts, float* out, dlrm_stream stream) {
    if (B < 0 || K < 1 || d < 1 || !parts_ok(K, n_parts, first_table, n_tables) || !parts) return DLRM_ERR_INVALID_ARG;
    if (B == 0) return DLRM_OK;
    if (!out) return DLRM_ERR_INVALID_ARG;
    const size_t row = sizeof(float) * (size_t)d;
    for (int p = 0; p < n_parts; ++p) {
        if (n_tables[p] == 0) continue;
        if (!parts[p]) return DLRM_ERR_INVALID_ARG;
        // rows b of part p ([B][n_p][d]) -> out[b][first_p .. first_p + n_p)
        if (cudaMemcpy2DAsync(out + (size_t)first_table[p] * d, row * K, parts[p], row * n_tables[p],
                              row * n_tables[p], (size_t)B, cudaMemcpyDeviceToDevice, cs_(stream)) != cudaSuccess)
            return DLRM_ERR_CUDA;
    }
    return DLRM_OK;
}

dlrm_status dlrm_pooled_split(int B, int K, int d, int n_parts, const int* first_table, const int* n_tables,
                              const float* in, float* const* parts, dlrm_stream stream) {
    if (B < 0 || K < 1 || d < 1 || !parts_ok(K, n_parts, first_table, n_tables) || !parts) return DLRM_ERR_INVALID_ARG;
    if (B == 0) return DLRM_OK;
    if (!in) return DLRM_ERR_INVALID_ARG;
    const size_t row = sizeof(float) * (size_t)d;
    for (int p = 0; p < n_parts; ++p) {
        if (n_tables[p] == 0) continue;
        if (!parts[p]) return DLRM_ERR_INVALID_ARG;
        if (cudaMemcpy2DAsync(parts[p], row * n_tables[p], in + (size_t)first_table[p] * d, row * K,
                              row * n_tables[p], (size_t)B, cudaMemcpyDeviceToDevice, cs_(stream)) != cudaSuccess)
            return DLRM_ERR_CUDA;
    }
    return DLRM_OK;
}

size_t dlrm_embbag_sgd_scratch_size(const dlrm_tables* T, int B, int64_t nnz) {
    TableMeta tm;
    if (check_sgd_tables(T, tm) != DLRM_OK || B < 0 || nnz < 0) return 0;
    return align_up(DLRM_ERR_RECORD_BYTES, 256) + sparse_layout((long long)T->K * B, nnz, T->d).total;
}

dlrm_status dlrm_embbag_sgd(const dlrm_tables* T, int B, const int32_t* offsets, const int32_t* indices, int64_t nnz,
                            const float* dE, float lr, void* scratch, size_t scratch_bytes, int32_t* n_touched,
                            dlrm_stream stream) {
    TableMeta tm;
    dlrm_status r = check_sgd_tables(T, tm);
    if (r != DLRM_OK) return r;
    if (B < 0 || nnz < 0 || nnz >= (int64_t(1) << 31)) return DLRM_ERR_INVALID_ARG;
    if (B > 0 && (!offsets || !dE || ((uintptr_t)dE & 15))) return DLRM_ERR_INVALID_ARG;
    if (nnz > 0 && !indices) return DLRM_ERR_INVALID_ARG;
    if (!scratch || ((uintptr_t)scratch & 15) || scratch_bytes < dlrm_embbag_sgd_scratch_size(T, B, nnz))
        return DLRM_ERR_WORKSPACE;
    if (B == 0) return DLRM_OK;
    const int K = T->K;
    const SparseLayout L = sparse_layout((long long)K * B, nnz, T->d);
    char* base = static_cast<char*>(scratch) + align_up(DLRM_ERR_RECORD_BYTES, 256);
    ErrRecord* err = static_cast<ErrRecord*>(scratch);
    const long long total_rows = tm.base[K - 1] + tm.rows[K - 1];
    cudaStream_t st = cs_(stream);
    int sorted = 0;
    if ((r = launch_sparse_prepare(K, B, tm, total_rows, offsets, indices, nnz, base, L, err, &sorted, st)))
        return r;
    return launch_sparse_apply(T->d, base, L, sorted, dE, lr, static_cast<float*>(T->data), nullptr, nullptr,
                               n_touched, st);
}

}  // extern "C"
