// Concat-only interaction with bulk copies: row b of out is
// [x_dense_b, e_1, ..., e_K, 0 padding up to ld], each e_k the sum-pooled bag
// (k, b) (the Wide & Deep alternative "DLRM", briansu.co, section 4 sets
// against the dot interaction; "Deep Learning Recommendation Model (DLRM)",
// nadeemcite summary, Key Method Details). Fast path for tables stored in the
// concat's dtype: a one-row bag's row is already its e_k.
//
// Block prologue as in the fused dot kernel (warp per table, lane per
// sample: each bag resolved to a row, "empty" or "several rows"). Then one
// warp assembles one sample's whole concat row in its shared-memory buffer:
// one bulk copy per one-row bag straight into the bag's slot (completing on
// the warp's mbarrier), x_dense converted into slot 0, several-row bags summed
// in fp32 by lane groups, the padding zeroed; then one bulk store writes the
// row (ld elements) to global memory. Before the buffer is refilled the
// previous store must have finished reading it.
#include "async_copy.cuh"
#include "common.cuh"
#include "kernels.cuh"

namespace dlrm {
namespace {

using namespace ac;

constexpr int CW = 8;                // warps per block
constexpr int CSPW = 4;              // samples per warp per block
constexpr int CS = CW * CSPW;        // samples per block: one lane each in the prologue
static_assert(CS == 32, "the prologue maps the block's samples to the lanes of a warp");
constexpr uint32_t CODE_EMPTY = 0xFFFFFFFFu;
constexpr uint32_t CODE_MULTI = 0xFFFFFFFEu;
constexpr unsigned FULL = 0xffffffffu;

__device__ __forceinline__ void bulk_store(void* dst, uint32_t src, uint32_t bytes) {
    asm volatile("cp.async.bulk.global.shared::cta.bulk_group [%0], [%1], %2;" ::"l"(dst), "r"(src), "r"(bytes)
                 : "memory");
    asm volatile("cp.async.bulk.commit_group;" ::: "memory");
}
// The issuing thread's earlier bulk stores have finished reading shared memory.
__device__ __forceinline__ void bulk_store_read_done() {
    asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory");
}
// ... and have completed.
__device__ __forceinline__ void bulk_store_done() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }

template <typename T>
__global__ void __launch_bounds__(CW * 32) embbag_cat_bulk_kernel(const T* __restrict__ tables,
                                                                  const __grid_constant__ TableMeta tm, int K, int d,
                                                                  int B, const int32_t* __restrict__ offsets,
                                                                  const int32_t* __restrict__ indices, long long nnz,
                                                                  const float* __restrict__ x_dense, T* __restrict__ out,
                                                                  int ld, int warp_bytes, ErrRecord* err) {
    pdl_wait();   // programmatic dependent: the previous kernel's outputs are visible from here on
    extern __shared__ __align__(16) unsigned char smem[];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    T* row = reinterpret_cast<T*>(smem + (size_t)warp * warp_bytes);
    const uint32_t row_s = (uint32_t)__cvta_generic_to_shared(row);
    unsigned char* tail = smem + (size_t)CW * warp_bytes;
    const int KS = K | 1;
    uint32_t* code_s = reinterpret_cast<uint32_t*>(tail);                       // [CS][KS]
    const uint32_t bar = (uint32_t)__cvta_generic_to_shared(code_s + CS * KS) + 8u * (uint32_t)warp;
    const uint32_t rowb = (uint32_t)(d * sizeof(T));
    const int b0 = blockIdx.x * CS;
    const int nb = min(CS, B - b0);
    unsigned oob = 0, bad = 0;

    for (int k = warp; k < K; k += CW) {
        if (lane < nb) {
            const long long o = (long long)k * B + b0 + lane;
            const long long st = offsets[o], en = offsets[o + 1];
            uint32_t code = CODE_EMPTY;
            if (st < 0 || en < st || en > nnz) {
                ++bad;
            } else if (en - st == 1) {
                const int idx = __ldg(indices + st);
                if (idx >= 0 && (long long)idx < tm.rows[k])
                    code = (uint32_t)(tm.base[k] + idx);
                else
                    ++oob;
            } else if (en - st > 1) {
                code = CODE_MULTI;
            }
            code_s[lane * KS + k] = code;
        }
    }
    if (lane == 0) {
        bar_init(bar);
        fence_proxy_async();
    }
    __syncthreads();

    uint32_t parity = 0;
    bool timed_out = false;
    const int first_tries = g_rows_wait_tries;
    constexpr int E16 = 16 / (int)sizeof(T);       // elements per 16-byte chunk
    const int nch = d / E16;                       // chunks per bag slot
    for (int r = 0; r < CSPW; ++r) {
        const int s = warp * CSPW + r;
        if (s >= nb) break;
        const long long b = b0 + s;
        // the buffer is free once the previous row's store has read it
        if (lane == 0) bulk_store_read_done();
        fence_proxy_async();
        __syncwarp();
        const uint32_t* cs = code_s + s * KS;
        unsigned long long one = 0, multi = 0, empty = 0;
        uint32_t c0 = CODE_EMPTY, c1 = CODE_EMPTY;
        c0 = lane < K ? cs[lane] : CODE_EMPTY;
        c1 = lane + 32 < K ? cs[lane + 32] : CODE_EMPTY;
        one = __ballot_sync(FULL, c0 < CODE_MULTI) | ((unsigned long long)__ballot_sync(FULL, c1 < CODE_MULTI) << 32);
        multi = __ballot_sync(FULL, c0 == CODE_MULTI) | ((unsigned long long)__ballot_sync(FULL, c1 == CODE_MULTI) << 32);
        empty = __ballot_sync(FULL, lane < K && c0 == CODE_EMPTY) |
                ((unsigned long long)__ballot_sync(FULL, lane + 32 < K && c1 == CODE_EMPTY) << 32);
        if (lane == 0) bar_expect(bar, (uint32_t)__popcll(one) * rowb);
        __syncwarp();
        if (c0 < CODE_MULTI) bulk_row(row_s + (uint32_t)(lane + 1) * rowb, tables + (long long)c0 * d, rowb, bar);
        if (c1 < CODE_MULTI) bulk_row(row_s + (uint32_t)(lane + 33) * rowb, tables + (long long)c1 * d, rowb, bar);
        // x_dense -> slot 0, zero padding behind the last slot
        for (int c = lane; c < d; c += 32) row[c] = Cvt<T>::from_f(x_dense[b * d + c]);
        for (int c = d * (K + 1) + lane; c < ld; c += 32) row[c] = Cvt<T>::from_f(0.f);
        // bags of several rows (fp32 sums) and empty bags: one bag per round, lanes over its chunks
        for (unsigned long long rest = multi | empty; rest; rest &= rest - 1) {
            const int k = __ffsll((long long)rest) - 1;
            T* slot = row + (size_t)(k + 1) * d;
            const bool many = (multi >> k) & 1ull;
            const int st = many ? offsets[(long long)k * B + b] : 0, en = many ? offsets[(long long)k * B + b + 1] : 0;
            for (int ch = lane; ch < nch; ch += 32) {
                float a[E16];
#pragma unroll
                for (int e = 0; e < E16; ++e) a[e] = 0.f;
                for (int p = st; p < en; ++p) {
                    const int idx = __ldg(indices + p);
                    if (idx >= 0 && (long long)idx < tm.rows[k]) {
                        Chunk16<T>::add(ldg16_stream(tables + (tm.base[k] + idx) * (long long)d + ch * E16), a);
                    } else if (ch == 0) {
                        ++oob;
                    }
                }
                T t[E16];
#pragma unroll
                for (int e = 0; e < E16; ++e) t[e] = Cvt<T>::from_f(a[e]);
                reinterpret_cast<uint4*>(slot)[ch] = *reinterpret_cast<const uint4*>(t);
            }
        }
        if (!rows_ready(bar, parity, first_tries)) {   // rows landed (drained): stop this warp's samples
            timed_out = true;
            break;
        }
        parity ^= 1u;
        // ordinary stores into the buffer become visible to the bulk store
        fence_proxy_async();
        __syncwarp();
        if (lane == 0) bulk_store(out + b * ld, row_s, (uint32_t)(ld * sizeof(T)));
    }
    if (lane == 0) bulk_store_done();
    if (timed_out && lane == 0) atomicOr(&err->flags, ERR_TIMEOUT);
    report_warp(err, oob, bad);
}

int cat_warp_bytes(int ld, size_t esize) { return (int)(((size_t)ld * esize + 15) & ~(size_t)15); }
size_t cat_smem(int K, int ld, size_t esize, int& wb) {
    wb = cat_warp_bytes(ld, esize);
    return (size_t)CW * wb + (((size_t)CS * (K | 1) * 4 + 7) & ~(size_t)7) + 8 * CW;
}

}  // namespace

bool embbag_cat_bulk_supported(dlrm_dtype dt, dlrm_dtype out_dt, int K, int d, int ld, const void* out,
                               long long total_rows) {
    if (dt != out_dt || (dt != DLRM_BF16 && dt != DLRM_F16 && dt != DLRM_F32)) return false;
    const size_t es = esize(dt);
    if (K < 1 || K > 64 || (d * es) % 16 || (ld * es) % 16 || ((uintptr_t)out & 15)) return false;
    if (ld < d * (K + 1) || total_rows >= (long long)CODE_MULTI) return false;
    int wb;
    return cat_smem(K, ld, es, wb) <= 227 * 1024;
}

dlrm_status launch_embbag_cat_bulk(const TableMeta& tm, const void* tables, dlrm_dtype dt, int K, int d, int B,
                                   const int32_t* offsets, const int32_t* indices, long long nnz,
                                   const float* x_dense, void* out, int ld, ErrRecord* err, cudaStream_t st) {
    int wb;
    const size_t smem = cat_smem(K, ld, esize(dt), wb);
    const int grid = (B + CS - 1) / CS;
#define DLRM_CAT_BULK(TT)                                                                                        \
    {                                                                                                           \
        auto kern = embbag_cat_bulk_kernel<TT>;                                                                 \
        cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);                     \
        (void)launch_pdl(kern, dim3(grid), dim3(CW * 32), smem, st, static_cast<const TT*>(tables), tm, K, d, B, \
                         offsets, indices, nnz, x_dense, static_cast<TT*>(out), ld, wb, err);                   \
    }
    if (dt == DLRM_BF16) DLRM_CAT_BULK(__nv_bfloat16) else if (dt == DLRM_F16) DLRM_CAT_BULK(__half) else DLRM_CAT_BULK(float)
#undef DLRM_CAT_BULK
    DLRM_LAUNCH_CHECK();
    return DLRM_OK;
}

cudaError_t set_wait_polls_embbag_cat(long long polls) {
    return ac::set_rows_wait_tries_here(polls < 0 ? -1 : (int)(polls < ac::WAIT_TRIES ? polls : ac::WAIT_TRIES));
}

}  // namespace dlrm
