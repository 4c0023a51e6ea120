// Embedding-bag gather, pairwise dot-product interaction, and the two fused.
//
// Pooling ("DLRM", briansu.co, section 3): bag (k, b) sums the rows of table
// k named by its indices; an empty bag gives zeros.
// Interaction ("DLRM", briansu.co, section 4, equations "Interaction" and
// "Output"; "Deep Learning Recommendation Model (DLRM)", nadeemcite summary,
// Key Method Details): X = [x_dense; e_1..e_K], Z_ij = <X_i, X_j> for
// 0 <= j < i <= K, written after x_dense in row-major strict-lower order.
//
// Gather geometry. A row of d elements is cut into n_ch chunks: 16-byte
// vectors when d * sizeof(T) is a multiple of 16, else single elements. A
// "group" of GL lanes (a power of two, GL <= 32) owns one row at a time; lane
// g of the group holds chunks g, g + GL, ... (NCH of them). A warp therefore
// works on 32 / GL bags at once. Each group walks the CSR positions of a run
// of consecutive bags of one table (they are contiguous in table-major CSR)
// U positions at a time, so U independent row loads per lane are in flight
// even when every bag holds one row.
#include "common.cuh"
#include "kernels.cuh"

#include <mutex>
#include <type_traits>

namespace dlrm {

template <typename T, bool VEC>
struct RowIO {
    static constexpr int E = VEC ? Chunk16<T>::E : 1;
};

// A loaded chunk: 16 raw bytes on the vector path, one widened element otherwise.
template <typename T, bool VEC>
using LdT = typename std::conditional<VEC, uint4, float>::type;

template <typename T, bool VEC>
__device__ __forceinline__ void chunk_add(const LdT<T, VEC>& v, float* a) {
    if constexpr (VEC) {
        Chunk16<T>::add(v, a);
    } else {
        a[0] += v;
    }
}

template <typename T, bool VEC>
__device__ __forceinline__ LdT<T, VEC> chunk_load(const T* row, int c) {
    if constexpr (VEC) {
        return ldg16_stream(row + c * Chunk16<T>::E);
    } else {
        return Cvt<T>::to_f(row[c]);
    }
}

template <typename T, bool VEC>
__device__ __forceinline__ LdT<T, VEC> chunk_zero() {
    if constexpr (VEC) {
        return make_uint4(0, 0, 0, 0);
    } else {
        return 0.f;
    }
}

// Walk the bags s = 0 .. nb-1 whose CSR ranges are off[s] .. off[s+1]
// (non-decreasing, inside [0, nnz]); call sink(s, acc) once per bag in order.
template <typename T, bool VEC, int NCH, int U, typename Sink>
__device__ __forceinline__ void walk_bags(const T* __restrict__ table, long long m, int d, int n_ch,
                                          const int32_t* __restrict__ indices, const int* off, int nb,
                                          int g, int GL, unsigned& oob, Sink& sink) {
    constexpr int E = RowIO<T, VEC>::E;
    float acc[NCH][E];
#pragma unroll
    for (int c = 0; c < NCH; ++c)
#pragma unroll
        for (int e = 0; e < E; ++e) acc[c][e] = 0.f;
    int s = 0;
    int p = off[0];
    const int pend = off[nb];
    int bag_end = off[1];
    int idx[U];
#pragma unroll
    for (int u = 0; u < U; ++u) idx[u] = (p + u < pend) ? __ldg(indices + p + u) : -1;
    while (p < pend) {
        const int n = min(U, pend - p);
        // the next step's indices are loaded while this step's rows are in flight
        int nxt[U];
#pragma unroll
        for (int u = 0; u < U; ++u) nxt[u] = (p + n + u < pend) ? __ldg(indices + p + n + u) : -1;
        LdT<T, VEC> v[U][NCH];
#pragma unroll
        for (int u = 0; u < U; ++u) {
            const bool ok = (u < n) && idx[u] >= 0 && (long long)idx[u] < m;
            if (g == 0 && u < n && !ok) ++oob;
            const T* row = table + (long long)(ok ? idx[u] : 0) * d;
#pragma unroll
            for (int c = 0; c < NCH; ++c) {
                const int cg = g + GL * c;
                v[u][c] = (ok && cg < n_ch) ? chunk_load<T, VEC>(row, cg) : chunk_zero<T, VEC>();
            }
        }
#pragma unroll
        for (int u = 0; u < U; ++u) {
            if (u < n) {
                while (p + u >= bag_end) {
                    sink(s, acc);
#pragma unroll
                    for (int c = 0; c < NCH; ++c)
#pragma unroll
                        for (int e = 0; e < E; ++e) acc[c][e] = 0.f;
                    ++s;
                    bag_end = off[s + 1];
                }
#pragma unroll
                for (int c = 0; c < NCH; ++c) chunk_add<T, VEC>(v[u][c], acc[c]);
            }
        }
        p += n;
#pragma unroll
        for (int u = 0; u < U; ++u) idx[u] = nxt[u];
    }
    while (s < nb) {
        sink(s, acc);
#pragma unroll
        for (int c = 0; c < NCH; ++c)
#pragma unroll
            for (int e = 0; e < E; ++e) acc[c][e] = 0.f;
        ++s;
    }
}

// Stores a pooled bag as fp32 at dst (row of d floats, any alignment for
// scalar chunks, 16-byte aligned when VEC and the element count per chunk is 4 or 8).
template <typename T, bool VEC, int NCH>
struct RowSink {
    float* base;       // row for bag s is base + s * stride
    long long stride;
    int g, GL, n_ch;
    template <typename Acc>
    __device__ __forceinline__ void operator()(int s, Acc& acc) {
        constexpr int E = RowIO<T, VEC>::E;
        float* dst = base + s * stride;
#pragma unroll
        for (int c = 0; c < NCH; ++c) {
            const int cg = g + GL * c;
            if (cg < n_ch) {
                if constexpr (E == 8) {
                    reinterpret_cast<float4*>(dst + cg * 8)[0] = make_float4(acc[c][0], acc[c][1], acc[c][2], acc[c][3]);
                    reinterpret_cast<float4*>(dst + cg * 8)[1] = make_float4(acc[c][4], acc[c][5], acc[c][6], acc[c][7]);
                } else if constexpr (E == 4) {
                    reinterpret_cast<float4*>(dst + cg * 4)[0] = make_float4(acc[c][0], acc[c][1], acc[c][2], acc[c][3]);
                } else {
                    dst[cg] = acc[c][0];
                }
            }
        }
    }
};

// Loads the tile's offsets into smem (off_s[k*(S+1) + s], s <= nb) and marks
// bags whose offsets are unusable; those bags are given an empty range.
// Returns through `bad` the number of bad bags this thread found.
__device__ __forceinline__ void load_tile_offsets(const int32_t* __restrict__ offsets, int B, int K, int b0, int nb,
                                                  int S, long long nnz, int* off_s, unsigned char* bad_s,
                                                  int32_t* bag_len, unsigned& bad) {
    for (int q = threadIdx.x; q < K * (nb + 1); q += blockDim.x) {
        const int k = q / (nb + 1), s = q - k * (nb + 1);
        off_s[k * (S + 1) + s] = offsets[(long long)k * B + b0 + s];
    }
    __syncthreads();
    for (int q = threadIdx.x; q < K * nb; q += blockDim.x) {
        const int k = q / nb, s = q - k * nb;
        const long long st = off_s[k * (S + 1) + s], en = off_s[k * (S + 1) + s + 1];
        const bool isbad = st < 0 || en < st || en > nnz;
        bad_s[k * S + s] = isbad;
        if (isbad) ++bad;
        if (bag_len) bag_len[(long long)k * B + b0 + s] = isbad ? 0 : (int32_t)(en - st);
    }
    __syncthreads();
}

// Pool every bag of the tile: work items are (table k, run of up to 8 samples).
template <typename T, bool VEC, int NCH, int U, typename MakeSink>
__device__ __forceinline__ void pool_tile(const T* __restrict__ tables, const TableMeta& tm, int K, int d, int n_ch,
                                          int GL, const int32_t* __restrict__ indices, const int* off_s,
                                          const unsigned char* bad_s, int S, int nb, unsigned& oob,
                                          MakeSink make_sink) {
    const int lane = threadIdx.x & 31;
    const int g = lane & (GL - 1);
    const int group = threadIdx.x / GL;
    const int n_groups = blockDim.x / GL;
    constexpr int RUN = 8;
    const int runs = (nb + RUN - 1) / RUN;
    for (int it = group; it < K * runs; it += n_groups) {
        const int k = it / runs, r = it - k * runs;
        const int s0 = r * RUN, ns = min(RUN, nb - s0);
        const T* table = tables + tm.base[k] * (long long)d;
        const int* off = off_s + k * (S + 1) + s0;
        bool anybad = false;
        for (int s = 0; s < ns; ++s) anybad |= bad_s[k * S + s0 + s];
        auto sink = make_sink(k, s0, g);
        if (!anybad) {
            walk_bags<T, VEC, NCH, U>(table, tm.rows[k], d, n_ch, indices, off, ns, g, GL, oob, sink);
        } else {
            // rare path: bags one by one, bad ones empty
            for (int s = 0; s < ns; ++s) {
                int one[2];
                one[0] = bad_s[k * S + s0 + s] ? 0 : off[s];
                one[1] = bad_s[k * S + s0 + s] ? 0 : off[s + 1];
                auto sub = make_sink(k, s0 + s, g);
                walk_bags<T, VEC, NCH, U>(table, tm.rows[k], d, n_ch, indices, one, 1, g, GL, oob, sub);
            }
        }
    }
}

// Pool every bag of the tile, one bag per work item: items (table k, sample s) are taken from a shared
// counter by lane groups, so that long and short bags even out across the groups, with U rows in flight
// per lane. The counter (shared, zeroed before the block's first __syncthreads) is consumed.
template <typename T, bool VEC, int NCH, int U, typename MakeSink>
__device__ __forceinline__ void pool_items(const T* __restrict__ tables, const TableMeta& tm, int K, int d, int n_ch,
                                           int GL, const int32_t* __restrict__ indices, const int* off_s,
                                           const unsigned char* bad_s, int S, int nb, unsigned& oob,
                                           MakeSink make_sink, int* counter) {
    const int lane = threadIdx.x & 31;
    const int g = lane & (GL - 1);
    const int leader = lane & ~(GL - 1);
    const unsigned gmask = GL == 32 ? 0xffffffffu : ((1u << GL) - 1u) << leader;
    const int n_items = K * nb;
    for (;;) {
        int it = 0;
        if (g == 0) it = atomicAdd(counter, 1);
        it = __shfl_sync(gmask, it, leader);
        if (it >= n_items) break;
        const int k = it / nb, s = it - k * nb;
        const T* table = tables + tm.base[k] * (long long)d;
        auto sink = make_sink(k, s, g);
        const bool isbad = bad_s[k * S + s];
        int one[2];
        one[0] = isbad ? 0 : off_s[k * (S + 1) + s];
        one[1] = isbad ? 0 : off_s[k * (S + 1) + s + 1];
        walk_bags<T, VEC, NCH, U>(table, tm.rows[k], d, n_ch, indices, one, 1, g, GL, oob, sink);
    }
}

// ------------------------------------------------------------------ K1: pooling only

template <typename T, bool VEC, int NCH>
__global__ void __launch_bounds__(256) embbag_kernel(const T* __restrict__ tables, const __grid_constant__ TableMeta tm,
                                                     int K, int d, int n_ch, int GL, int B, int S,
                                                     const int32_t* __restrict__ offsets,
                                                     const int32_t* __restrict__ indices, long long nnz,
                                                     float* __restrict__ pooled, int32_t* __restrict__ bag_len,
                                                     ErrRecord* err) {
    pdl_wait();
    extern __shared__ __align__(16) unsigned char smem[];
    int* off_s = reinterpret_cast<int*>(smem);
    unsigned char* bad_s = smem + sizeof(int) * K * (S + 1);
    const int b0 = blockIdx.x * S;
    const int nb = min(S, B - b0);
    unsigned oob = 0, bad = 0;
    load_tile_offsets(offsets, B, K, b0, nb, S, nnz, off_s, bad_s, bag_len, bad);
    auto make_sink = [&](int k, int s0, int g) {
        return RowSink<T, VEC, NCH>{pooled + ((long long)(b0 + s0) * K + k) * d, (long long)K * d, g, GL, n_ch};
    };
    pool_tile<T, VEC, NCH, 4>(tables, tm, K, d, n_ch, GL, indices, off_s, bad_s, S, nb, oob, make_sink);
    report_warp(err, oob, bad);
}

// ------------------------------------------------------------------ concat-only interaction

// Writes a pooled bag into its d-wide slot of a concat row, converted to OT
// (16-byte stores where the slot is aligned, element stores otherwise).
template <typename T, bool VEC, int NCH, typename OT>
struct CatSink {
    OT* base;          // slot of bag s is base + s * stride
    long long stride;
    int g, GL, n_ch;
    bool vec_ok;
    template <typename Acc>
    __device__ __forceinline__ void operator()(int s, Acc& acc) {
        constexpr int E = RowIO<T, VEC>::E;
        OT* dst = base + s * stride;
#pragma unroll
        for (int c = 0; c < NCH; ++c) {
            const int cg = g + GL * c;
            if (cg < n_ch) {
                OT* p = dst + cg * E;
                if constexpr (E * sizeof(OT) % 16 == 0) {
                    if (vec_ok) {
#pragma unroll
                        for (int h = 0; h < (int)(E * sizeof(OT) / 16); ++h) {
                            OT t[16 / sizeof(OT)];
#pragma unroll
                            for (int e = 0; e < (int)(16 / sizeof(OT)); ++e)
                                t[e] = Cvt<OT>::from_f(acc[c][h * (16 / sizeof(OT)) + e]);
                            reinterpret_cast<uint4*>(p)[h] = *reinterpret_cast<const uint4*>(t);
                        }
                        continue;
                    }
                }
#pragma unroll
                for (int e = 0; e < E; ++e) p[e] = Cvt<OT>::from_f(acc[c][e]);
            }
        }
    }
};

// Concat-only interaction (the Wide & Deep alternative the pages contrast
// DLRM with: embeddings concatenated with the dense vector, no dot products):
// row b of out is [x_dense_b, e_1, ..., e_K, 0 padding up to ld], each e_k the
// sum-pooled bag (k, b). The gather is K1's; only the destination differs.
template <typename T, bool VEC, int NCH, typename OT>
__global__ void __launch_bounds__(256) embbag_cat_kernel(const T* __restrict__ tables, const __grid_constant__ TableMeta tm,
                                                         int K, int d, int n_ch, int GL, int B, int S,
                                                         const int32_t* __restrict__ offsets,
                                                         const int32_t* __restrict__ indices, long long nnz,
                                                         const float* __restrict__ x_dense, OT* __restrict__ out, int ld,
                                                         bool vec_ok, ErrRecord* err) {
    pdl_wait();
    extern __shared__ __align__(16) unsigned char smem[];
    int* off_s = reinterpret_cast<int*>(smem);
    unsigned char* bad_s = smem + sizeof(int) * K * (S + 1);
    const int b0 = blockIdx.x * S;
    const int nb = min(S, B - b0);
    unsigned oob = 0, bad = 0;
    load_tile_offsets(offsets, B, K, b0, nb, S, nnz, off_s, bad_s, nullptr, bad);
    auto make_sink = [&](int k, int s0, int g) {
        return CatSink<T, VEC, NCH, OT>{out + (long long)(b0 + s0) * ld + (long long)(k + 1) * d, (long long)ld, g, GL,
                                        n_ch, vec_ok};
    };
    pool_tile<T, VEC, NCH, 4>(tables, tm, K, d, n_ch, GL, indices, off_s, bad_s, S, nb, oob, make_sink);
    // x_dense in front, zero padding behind
    const int tail = ld - d * (K + 1);
    for (int q = threadIdx.x; q < nb * (d + tail); q += blockDim.x) {
        const int s = q / (d + tail), c = q - s * (d + tail);
        const long long b = b0 + s;
        if (c < d) out[b * ld + c] = Cvt<OT>::from_f(x_dense[b * d + c]);
        else out[b * ld + d * (K + 1) + (c - d)] = Cvt<OT>::from_f(0.f);
    }
    report_warp(err, oob, bad);
}

// ------------------------------------------------------------------ interaction on a smem tile

__device__ __forceinline__ int pair_row(int p) {
    int i = (int)((1.0f + sqrtf(8.0f * (float)p + 1.0f)) * 0.5f);
    while (i * (i - 1) / 2 > p) --i;
    while ((i + 1) * i / 2 <= p) ++i;
    return i;
}

// X: nb samples, each (K+1) rows of stride xs floats. Writes rows b0.. of out.
__device__ __forceinline__ void interact_tile(const float* X, int xs, int K, int d, int nb, int b0, void* out,
                                              int ld, int out_dt) {
    const int P = K * (K + 1) / 2;
    const int n1 = K + 1;
    for (int q = threadIdx.x; q < nb * ld; q += blockDim.x) {
        const int s = q / ld, c = q - s * ld;
        if (c >= d && c < d + P) continue;
        const float v = (c < d) ? X[(long long)s * n1 * xs + c] : 0.f;
        store_as(out, (size_t)(b0 + s) * ld + c, v, out_dt);
    }
    const bool v4 = (d & 3) == 0;
    for (int q = threadIdx.x; q < nb * P; q += blockDim.x) {
        const int s = q / P, p = q - s * P;
        const int i = pair_row(p), j = p - i * (i - 1) / 2;
        const float* xi = X + ((long long)s * n1 + i) * xs;
        const float* xj = X + ((long long)s * n1 + j) * xs;
        float a0 = 0.f, a1 = 0.f, a2 = 0.f, a3 = 0.f;
        if (v4) {
            for (int t = 0; t < d; t += 4) {
                const float4 u = *reinterpret_cast<const float4*>(xi + t);
                const float4 w = *reinterpret_cast<const float4*>(xj + t);
                a0 = fmaf(u.x, w.x, a0); a1 = fmaf(u.y, w.y, a1);
                a2 = fmaf(u.z, w.z, a2); a3 = fmaf(u.w, w.w, a3);
            }
        } else {
            for (int t = 0; t < d; ++t) a0 = fmaf(xi[t], xj[t], a0);
        }
        store_as(out, (size_t)(b0 + s) * ld + d + p, (a0 + a1) + (a2 + a3), out_dt);
    }
}

// Copies x_dense rows (fp32 [B][d]) for the tile into row 0 of each sample block.
__device__ __forceinline__ void load_dense_rows(const float* __restrict__ x_dense, int d, int b0, int nb, float* X,
                                                int xs, int n1) {
    for (int q = threadIdx.x; q < nb * d; q += blockDim.x) {
        const int s = q / d, t = q - s * d;
        X[(long long)s * n1 * xs + t] = x_dense[(long long)(b0 + s) * d + t];
    }
}

__global__ void __launch_bounds__(256) interact_kernel(int B, int K, int d, int S, int xs,
                                                       const float* __restrict__ x_dense,
                                                       const float* __restrict__ pooled, void* out, int ld,
                                                       int out_dt) {
    pdl_wait();
    extern __shared__ __align__(16) unsigned char smem[];
    float* X = reinterpret_cast<float*>(smem);
    const int b0 = blockIdx.x * S;
    const int nb = min(S, B - b0);
    const int n1 = K + 1;
    load_dense_rows(x_dense, d, b0, nb, X, xs, n1);
    for (int q = threadIdx.x; q < nb * K * d; q += blockDim.x) {
        const int s = q / (K * d), r = q - s * K * d;
        const int k = r / d, t = r - k * d;
        X[((long long)s * n1 + 1 + k) * xs + t] = pooled[(long long)(b0 + s) * K * d + r];
    }
    __syncthreads();
    interact_tile(X, xs, K, d, nb, b0, out, ld, out_dt);
}

// ------------------------------------------------------------------ K2: fused gather + interaction

template <typename T, bool VEC, int NCH>
__global__ void __launch_bounds__(256) embbag_interact_kernel(
    const T* __restrict__ tables, const __grid_constant__ TableMeta tm, int K, int d, int n_ch, int GL, int B, int S,
    int xs, const int32_t* __restrict__ offsets, const int32_t* __restrict__ indices, long long nnz,
    const float* __restrict__ x_dense, void* out, int ld, int out_dt, ErrRecord* err) {
    pdl_wait();
    extern __shared__ __align__(16) unsigned char smem[];
    const int n1 = K + 1;
    float* X = reinterpret_cast<float*>(smem);
    int* off_s = reinterpret_cast<int*>(smem + sizeof(float) * (size_t)S * n1 * xs);
    unsigned char* bad_s = reinterpret_cast<unsigned char*>(off_s + K * (S + 1));
    int* counter = reinterpret_cast<int*>(bad_s + (((size_t)K * S + 3) & ~(size_t)3));
    const int b0 = blockIdx.x * S;
    const int nb = min(S, B - b0);
    unsigned oob = 0, bad = 0;
    if (threadIdx.x == 0) *counter = 0;
    load_dense_rows(x_dense, d, b0, nb, X, xs, n1);
    load_tile_offsets(offsets, B, K, b0, nb, S, nnz, off_s, bad_s, nullptr, bad);
    auto make_sink = [&](int k, int s0, int g) {
        return RowSink<T, VEC, NCH>{X + ((long long)s0 * n1 + 1 + k) * xs, (long long)n1 * xs, g, GL, n_ch};
    };
    constexpr int U = NCH >= 4 ? 2 : (NCH == 2 ? 4 : 8);
    pool_items<T, VEC, NCH, U>(tables, tm, K, d, n_ch, GL, indices, off_s, bad_s, S, nb, oob, make_sink, counter);
    __syncthreads();
    interact_tile(X, xs, K, d, nb, b0, out, ld, out_dt);
    report_warp(err, oob, bad);
}

// ------------------------------------------------------------------ K2 for fp32 tables of d = 4 GL

// fp32 tables with 16-byte rows of d = 16, 32, 64 or 128 floats (the medium and tiny configurations): the
// generic kernel's interaction on the block's fp32 tile, with a leaner gather. Work items (table k, sample s)
// are taken NG at a time per warp from a shared counter, one bag per lane group of GL = d/4 lanes (16 bytes
// of a row per lane); the group walks the bag U rows at a time with the next U indices loaded while the
// rows are in flight, one range test per row against the table's row count (an index past the bag reads
// as -1, i.e. out of range), out-of-range indices counted from one bit mask per step, fp32 sums with packed
// adds, and the pooled row stored as one 16-byte vector per lane into row 1 + k of the sample's tile.
template <int GL, int U>
__global__ void __launch_bounds__(256) embbag_interact_f32_kernel(
    const float* __restrict__ tables, const __grid_constant__ TableMeta tm, int K, int B, int S, int xs,
    const int32_t* __restrict__ offsets, const int32_t* __restrict__ indices, long long nnz,
    const float* __restrict__ x_dense, void* out, int ld, int out_dt, ErrRecord* err) {
    pdl_wait();   // programmatic dependent: the previous kernel's outputs are visible from here on
    constexpr int d = 4 * GL;
    constexpr int NG = 32 / GL;
    extern __shared__ __align__(16) unsigned char smem[];
    const int n1 = K + 1;
    float* X = reinterpret_cast<float*>(smem);
    int* counter = reinterpret_cast<int*>(smem + sizeof(float) * (size_t)S * n1 * xs);
    const int lane = threadIdx.x & 31;
    const int g = lane % GL, grp = lane / GL;
    const int b0 = blockIdx.x * S;
    const int nb = min(S, B - b0);
    unsigned oob = 0, bad = 0;
    if (threadIdx.x == 0) *counter = 0;
    load_dense_rows(x_dense, d, b0, nb, X, xs, n1);
    __syncthreads();
    const int n_items = K * nb;
    for (;;) {
        int it0 = 0;
        if (lane == 0) it0 = atomicAdd(counter, NG);
        it0 = __shfl_sync(0xffffffffu, it0, 0);
        if (it0 >= n_items) break;
        const int it = it0 + grp;
        if (it >= n_items) continue;
        const int k = it / nb, s = it - k * nb;
        const long long o = (long long)k * B + b0 + s;
        const long long st = offsets[o], en = offsets[o + 1];
        float acc[4] = {0.f, 0.f, 0.f, 0.f};
        if (st < 0 || en < st || en > nnz) {
            if (g == 0) ++bad;
        } else {
            const float* tab = tables + tm.base[k] * (long long)d + 4 * g;
            const unsigned long long m = (unsigned long long)tm.rows[k];
            int idx[U];
#pragma unroll
            for (int u = 0; u < U; ++u) idx[u] = st + u < en ? __ldg(indices + st + u) : -1;
            for (long long p = st; p < en; p += U) {
                int nxt[U];
                if (p + 2 * U <= en) {
#pragma unroll
                    for (int u = 0; u < U; ++u) nxt[u] = __ldg(indices + p + U + u);
                } else {
#pragma unroll
                    for (int u = 0; u < U; ++u) nxt[u] = p + U + u < en ? __ldg(indices + p + U + u) : -1;
                }
                uint4 v[U];
                unsigned okm = 0;
#pragma unroll
                for (int u = 0; u < U; ++u) {
                    const bool ok = (unsigned long long)(unsigned)idx[u] < m;   // -1: past the bag
                    okm |= (unsigned)ok << u;
                    v[u] = ok ? ldg16_stream(tab + (long long)idx[u] * d) : make_uint4(0, 0, 0, 0);
                }
                if (g == 0) {   // out-of-range indices of the bag (not the slots past its end)
                    const int n = en - p < U ? (int)(en - p) : U;
                    oob += __popc(~okm & ((1u << n) - 1u));
                }
#pragma unroll
                for (int u = 0; u < U; ++u) Chunk16<float>::add(v[u], acc);
#pragma unroll
                for (int u = 0; u < U; ++u) idx[u] = nxt[u];
            }
        }
        *reinterpret_cast<float4*>(X + ((long long)s * n1 + 1 + k) * xs + 4 * g) =
            make_float4(acc[0], acc[1], acc[2], acc[3]);
    }
    __syncthreads();
    interact_tile(X, xs, K, d, nb, b0, out, ld, out_dt);
    report_warp(err, oob, bad);
}

// ------------------------------------------------------------------ host launchers

struct Geometry {
    bool vec;
    int n_ch, GL, NCH;
};

static bool gather_geometry(int d, dlrm_dtype dt, Geometry& g) {
    const size_t rb = (size_t)d * esize(dt);
    if (rb % 16 == 0 && rb <= 2048) {
        g.vec = true;
        g.n_ch = (int)(rb / 16);
    } else if (d <= 256) {
        g.vec = false;
        g.n_ch = d;
    } else {
        return false;
    }
    if (g.n_ch <= 32) {
        g.NCH = 1;
        g.GL = 1;
        while (g.GL < g.n_ch) g.GL <<= 1;
    } else {
        g.GL = 32;
        g.NCH = (g.n_ch + 31) / 32;
        g.NCH = g.NCH <= 2 ? 2 : (g.NCH <= 4 ? 4 : 8);
    }
    return !(g.vec && g.NCH > 4);
}

bool gather_supported(int d, dlrm_dtype dt) {
    if (dt == DLRM_U8ROW) return false;   // only the fused tensor-core kernel reads uint8 records
    Geometry g;
    return gather_geometry(d, dt, g);
}

static int xstride(int d) {
    const int r = (d + 3) / 4 * 4;
    return r + 4;
}

size_t interact_smem_per_sample(int K, int d) { return sizeof(float) * (size_t)(K + 1) * xstride(d); }

static const size_t kSmemBudget = 72 * 1024;
static const size_t kSmemMax = 227 * 1024;

template <typename T>
static dlrm_status launch_embbag_t(const TableMeta& tm, const void* tables, int K, int d, int B,
                                   const int32_t* offsets, const int32_t* indices, long long nnz, float* pooled,
                                   int32_t* bag_len, ErrRecord* err, cudaStream_t st, const Geometry& g) {
    const int S = 32;
    const size_t smem = sizeof(int) * (size_t)K * (S + 1) + (size_t)K * S;
    const dim3 grid((B + S - 1) / S);
    const T* tb = static_cast<const T*>(tables);
#define DLRM_K1(VEC, NCH)                                                                                  \
    {                                                                                                      \
        auto kern = embbag_kernel<T, VEC, NCH>;                                                            \
        if (smem > 48 * 1024) cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem); \
        (void)launch_pdl(kern, dim3(grid), dim3(256), (size_t)(smem), st, tb, tm, K, d, g.n_ch, g.GL, B, S, offsets, indices, nnz, pooled, bag_len, err); \
    }
    if (g.vec) {
        if (g.NCH == 1) DLRM_K1(true, 1) else if (g.NCH == 2) DLRM_K1(true, 2) else DLRM_K1(true, 4)
    } else {
        if (g.NCH == 1) DLRM_K1(false, 1) else if (g.NCH == 2) DLRM_K1(false, 2)
        else if (g.NCH == 4) DLRM_K1(false, 4) else DLRM_K1(false, 8)
    }
#undef DLRM_K1
    DLRM_LAUNCH_CHECK();
    return DLRM_OK;
}

dlrm_status launch_embbag(const TableMeta& tm, const void* tables, dlrm_dtype dt, int K, int d, int B,
                          const int32_t* offsets, const int32_t* indices, long long nnz, float* pooled,
                          int32_t* bag_len, ErrRecord* err, cudaStream_t st) {
    Geometry g;
    if (dt == DLRM_U8ROW || !gather_geometry(d, dt, g)) return DLRM_ERR_UNSUPPORTED;
    if ((size_t)sizeof(int) * K * 33 + (size_t)K * 32 > kSmemMax) return DLRM_ERR_UNSUPPORTED;
    switch (dt) {
        case DLRM_F32: return launch_embbag_t<float>(tm, tables, K, d, B, offsets, indices, nnz, pooled, bag_len, err, st, g);
        case DLRM_BF16: return launch_embbag_t<__nv_bfloat16>(tm, tables, K, d, B, offsets, indices, nnz, pooled, bag_len, err, st, g);
        case DLRM_F16: return launch_embbag_t<__half>(tm, tables, K, d, B, offsets, indices, nnz, pooled, bag_len, err, st, g);
    }
    return DLRM_ERR_UNSUPPORTED;
}

dlrm_status launch_interact(int B, int K, int d, const float* x_dense, const float* pooled, void* out, int ld,
                            dlrm_dtype out_dt, cudaStream_t st) {
    const size_t per = interact_smem_per_sample(K, d);
    if (per > kSmemMax) return DLRM_ERR_UNSUPPORTED;
    int S = (int)(kSmemBudget / per);
    S = S < 1 ? 1 : (S > 8 ? 8 : S);
    const size_t smem = per * S;
    if (smem > 48 * 1024) cudaFuncSetAttribute(interact_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    (void)launch_pdl(interact_kernel, dim3((B + S - 1) / S), dim3(256), (size_t)(smem), st, B, K, d, S, xstride(d), x_dense, pooled, out, ld, (int)out_dt);
    DLRM_LAUNCH_CHECK();
    return DLRM_OK;
}

template <typename T>
static dlrm_status launch_fused_t(const TableMeta& tm, const void* tables, int K, int d, int B,
                                  const int32_t* offsets, const int32_t* indices, long long nnz,
                                  const float* x_dense, void* out, int ld, dlrm_dtype out_dt, ErrRecord* err,
                                  cudaStream_t st, const Geometry& g) {
    const size_t per = interact_smem_per_sample(K, d);
    const auto extra = [&](int S) { return sizeof(int) * (size_t)K * (S + 1) + (((size_t)K * S + 3) & ~(size_t)3) + 16; };
    int S = (int)(kSmemBudget / per);
    S = S < 1 ? 1 : (S > 8 ? 8 : S);
    // enough blocks for about four per SM, so that small batches still spread over the GPU
    const int s_fill = B / (148 * 4);
    if (s_fill < S) S = s_fill < 1 ? 1 : s_fill;
    while (S > 1 && per * S + extra(S) > kSmemMax) --S;
    const size_t smem = per * S + extra(S);
    if (smem > kSmemMax) return DLRM_ERR_UNSUPPORTED;
    const T* tb = static_cast<const T*>(tables);
    const dim3 grid((B + S - 1) / S);
#define DLRM_K2(VEC, NCH)                                                                                  \
    {                                                                                                      \
        auto kern = embbag_interact_kernel<T, VEC, NCH>;                                                   \
        if (smem > 48 * 1024) cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem); \
        (void)launch_pdl(kern, dim3(grid), dim3(256), (size_t)(smem), st, tb, tm, K, d, g.n_ch, g.GL, B, S, xstride(d), offsets, indices, nnz, x_dense, \
                                      out, ld, (int)out_dt, err);                                         \
    }
    if (g.vec) {
        if (g.NCH == 1) DLRM_K2(true, 1) else if (g.NCH == 2) DLRM_K2(true, 2) else DLRM_K2(true, 4)
    } else {
        if (g.NCH == 1) DLRM_K2(false, 1) else if (g.NCH == 2) DLRM_K2(false, 2)
        else if (g.NCH == 4) DLRM_K2(false, 4) else DLRM_K2(false, 8)
    }
#undef DLRM_K2
    DLRM_LAUNCH_CHECK();
    return DLRM_OK;
}

// Resident blocks per SM of embbag_interact_f32_kernel<GL> with `smem` bytes of dynamic shared memory: asked
// of the runtime once per (GL, smem) and kept (a property of the code and the GPU model; one model per process).
template <typename Query>
static int f32_occupancy(int gl, size_t smem, Query query) {
    struct Entry {
        int gl;
        size_t smem;
        int occ;
    };
    static Entry cache[32];
    static int used = 0;
    static std::mutex mu;
    std::lock_guard<std::mutex> lock(mu);
    for (int i = 0; i < used; ++i)
        if (cache[i].gl == gl && cache[i].smem == smem) return cache[i].occ;
    int occ = 1;
    query(occ);
    cache[used < 32 ? used++ : (int)(smem % 32)] = Entry{gl, smem, occ};
    return occ;
}

static dlrm_status launch_fused_f32(const TableMeta& tm, const void* tables, int K, int d, int B,
                                    const int32_t* offsets, const int32_t* indices, long long nnz,
                                    const float* x_dense, void* out, int ld, dlrm_dtype out_dt, ErrRecord* err,
                                    cudaStream_t st) {
    const size_t per = interact_smem_per_sample(K, d);
    const float* tb = static_cast<const float*>(tables);
    int sms = 148, dev = 0;
    if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    // S samples per block: as few as keep the whole grid resident at once (one wave: a partial second wave
    // would leave most SMs idle while it runs), at most 8 and within the shared-memory budget
#define DLRM_KF(GLV)                                                                                           \
    {                                                                                                          \
        auto kern = embbag_interact_f32_kernel<GLV, 8>;                                                        \
        int S = 1;                                                                                             \
        for (;; ++S) {                                                                                         \
            const size_t sm = per * S + 16;                                                                    \
            if (S > 1 && (S > 8 || sm > kSmemMax)) { --S; break; }                                            \
            int occ = f32_occupancy(GLV, sm, [&](int& o) {                                                   \
                if (sm > 48 * 1024) cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm); \
                if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&o, kern, 256, sm) != cudaSuccess || o < 1) o = 1; \
            });                                                                                                \
            if ((long long)(B + S - 1) / S <= (long long)occ * sms) break;                                    \
        }                                                                                                      \
        const size_t smem = per * S + 16;                                                                      \
        if (smem > kSmemMax) return DLRM_ERR_UNSUPPORTED;                                                      \
        if (smem > 48 * 1024) cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem); \
        const dim3 grid((B + S - 1) / S);                                                                      \
        (void)launch_pdl(kern, grid, dim3(256), smem, st, tb, tm, K, B, S, xstride(d), offsets, indices, nnz,   \
                         x_dense, out, ld, (int)out_dt, err);                                                  \
    }
    switch (d) {
        case 16: DLRM_KF(4) break;
        case 32: DLRM_KF(8) break;
        case 64: DLRM_KF(16) break;
        default: DLRM_KF(32) break;
    }
#undef DLRM_KF
    DLRM_LAUNCH_CHECK();
    return DLRM_OK;
}

dlrm_status launch_embbag_interact(const TableMeta& tm, const void* tables, dlrm_dtype dt, int K, int d, int B,
                                   const int32_t* offsets, const int32_t* indices, long long nnz,
                                   const float* x_dense, void* out, int ld, dlrm_dtype out_dt, ErrRecord* err,
                                   cudaStream_t st) {
    if (embbag_interact_mma_supported(dt, K, d, ld, out, out_dt, tm.base[K - 1] + tm.rows[K - 1]))
        return launch_embbag_interact_mma(tm, tables, dt, K, d, B, offsets, indices, nnz, x_dense, out, ld, out_dt,
                                          err, st);
    if (embbag_interact_wide_supported(dt, K, d, ld, out, out_dt))
        return launch_embbag_interact_wide(tm, tables, K, d, B, offsets, indices, nnz, x_dense, out, ld, err, st);
    if (dt == DLRM_F32 && (d == 16 || d == 32 || d == 64 || d == 128) && K >= 1)
        return launch_fused_f32(tm, tables, K, d, B, offsets, indices, nnz, x_dense, out, ld, out_dt, err, st);
    Geometry g;
    if (dt == DLRM_U8ROW || !gather_geometry(d, dt, g)) return DLRM_ERR_UNSUPPORTED;
    switch (dt) {
        case DLRM_F32: return launch_fused_t<float>(tm, tables, K, d, B, offsets, indices, nnz, x_dense, out, ld, out_dt, err, st, g);
        case DLRM_BF16: return launch_fused_t<__nv_bfloat16>(tm, tables, K, d, B, offsets, indices, nnz, x_dense, out, ld, out_dt, err, st, g);
        case DLRM_F16: return launch_fused_t<__half>(tm, tables, K, d, B, offsets, indices, nnz, x_dense, out, ld, out_dt, err, st, g);
    }
    return DLRM_ERR_UNSUPPORTED;
}

template <typename T, typename OT>
static dlrm_status launch_cat_t(const TableMeta& tm, const void* tables, int K, int d, int B, const int32_t* offsets,
                                const int32_t* indices, long long nnz, const float* x_dense, void* out, int ld,
                                ErrRecord* err, cudaStream_t st, const Geometry& g) {
    const int S = 32;
    const size_t smem = sizeof(int) * (size_t)K * (S + 1) + (size_t)K * S;
    const dim3 grid((B + S - 1) / S);
    const T* tb = static_cast<const T*>(tables);
    OT* o = static_cast<OT*>(out);
    const bool vec_ok = ((uintptr_t)out & 15) == 0 && ((size_t)d * sizeof(OT)) % 16 == 0 && ((size_t)ld * sizeof(OT)) % 16 == 0;
#define DLRM_CAT(VEC, NCH)                                                                                       \
    {                                                                                                            \
        auto kern = embbag_cat_kernel<T, VEC, NCH, OT>;                                                          \
        if (smem > 48 * 1024) cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem); \
        (void)launch_pdl(kern, dim3(grid), dim3(256), (size_t)(smem), st, tb, tm, K, d, g.n_ch, g.GL, B, S, offsets, indices, nnz, x_dense, o, ld,   \
                                      vec_ok, err);                                                              \
    }
    if (g.vec) {
        if (g.NCH == 1) DLRM_CAT(true, 1) else if (g.NCH == 2) DLRM_CAT(true, 2) else DLRM_CAT(true, 4)
    } else {
        if (g.NCH == 1) DLRM_CAT(false, 1) else if (g.NCH == 2) DLRM_CAT(false, 2)
        else if (g.NCH == 4) DLRM_CAT(false, 4) else DLRM_CAT(false, 8)
    }
#undef DLRM_CAT
    DLRM_LAUNCH_CHECK();
    return DLRM_OK;
}

template <typename T>
static dlrm_status launch_cat_out(const TableMeta& tm, const void* tables, int K, int d, int B, const int32_t* offsets,
                                  const int32_t* indices, long long nnz, const float* x_dense, void* out, int ld,
                                  dlrm_dtype out_dt, ErrRecord* err, cudaStream_t st, const Geometry& g) {
    switch (out_dt) {
        case DLRM_F32: return launch_cat_t<T, float>(tm, tables, K, d, B, offsets, indices, nnz, x_dense, out, ld, err, st, g);
        case DLRM_BF16: return launch_cat_t<T, __nv_bfloat16>(tm, tables, K, d, B, offsets, indices, nnz, x_dense, out, ld, err, st, g);
        case DLRM_F16: return launch_cat_t<T, __half>(tm, tables, K, d, B, offsets, indices, nnz, x_dense, out, ld, err, st, g);
        default: return DLRM_ERR_UNSUPPORTED;
    }
}

dlrm_status launch_embbag_cat(const TableMeta& tm, const void* tables, dlrm_dtype dt, int K, int d, int B,
                              const int32_t* offsets, const int32_t* indices, long long nnz, const float* x_dense,
                              void* out, int ld, dlrm_dtype out_dt, ErrRecord* err, cudaStream_t st) {
    if (embbag_cat_bulk_supported(dt, out_dt, K, d, ld, out, tm.base[K - 1] + tm.rows[K - 1]))
        return launch_embbag_cat_bulk(tm, tables, dt, K, d, B, offsets, indices, nnz, x_dense, out, ld, err, st);
    Geometry g;
    if (dt == DLRM_U8ROW || !gather_geometry(d, dt, g)) return DLRM_ERR_UNSUPPORTED;
    if ((size_t)sizeof(int) * K * 33 + (size_t)K * 32 > kSmemMax) return DLRM_ERR_UNSUPPORTED;
    switch (dt) {
        case DLRM_F32: return launch_cat_out<float>(tm, tables, K, d, B, offsets, indices, nnz, x_dense, out, ld, out_dt, err, st, g);
        case DLRM_BF16: return launch_cat_out<__nv_bfloat16>(tm, tables, K, d, B, offsets, indices, nnz, x_dense, out, ld, out_dt, err, st, g);
        case DLRM_F16: return launch_cat_out<__half>(tm, tables, K, d, B, offsets, indices, nnz, x_dense, out, ld, out_dt, err, st, g);
        default: return DLRM_ERR_UNSUPPORTED;
    }
}

}  // namespace dlrm
