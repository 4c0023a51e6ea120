// Training-step kernels other than the GEMMs.
//
//  - BCE loss in logit form, mean over the batch ("Deep Learning
//    Recommendation Model (DLRM)", nadeemcite summary, Key Method Details:
//    BCE loss), and dL/dz = (sigmoid(z) - y) / B.
//  - interaction backward: from Z_ij = <X_i, X_j> ("DLRM", briansu.co,
//    section 4), dX_i = sum_{j != i} dZ_ij X_j; the concat's direct copy of
//    x_dense adds its gradient to dX_0.
//  - sparse embedding update: every valid occurrence (bag, row) becomes a key
//    (global row id) and a value (bag id); a stable LSD radix sort groups equal
//    rows in occurrence order, each row's bag gradients are summed in that
//    order (in fixed-size pieces whose partial sums are added in order), and
//    only touched rows are updated: T[row] -= lr * g. Everything is
//    deterministic: integer counting, fixed-order scans and sums.
//  - dense SGD: w -= lr * dw.
#include <algorithm>

#include "common.cuh"
#include "kernels.cuh"

namespace dlrm {

namespace {

constexpr int RADIX_BITS = 8;
constexpr int RADIX = 1 << RADIX_BITS;
constexpr int SORT_THREADS = 256;
constexpr int SORT_ITEMS = 16;                      // keys per thread per tile
constexpr int SORT_TILE = SORT_THREADS * SORT_ITEMS;  // 4096

// ------------------------------------------------------------------ BCE

__global__ void bce_kernel(int B, const float* __restrict__ z, const float* __restrict__ y, float* __restrict__ dz,
                           float* __restrict__ y_hat, float* __restrict__ partial) {
    pdl_wait();
    __shared__ float red[256];
    const int i = blockIdx.x * blockDim.x + threadIdx.x;
    float l = 0.f;
    if (i < B) {
        const float zi = z[i], yi = y[i];
        const float sp = fmaxf(zi, 0.f) + log1pf(expf(-fabsf(zi)));
        l = sp - yi * zi;
        const float s = 1.f / (1.f + expf(-zi));
        dz[i] = (s - yi) / (float)B;
        if (y_hat) y_hat[i] = s;
    }
    red[threadIdx.x] = l;
    __syncthreads();
    for (int o = blockDim.x / 2; o; o >>= 1) {
        if (threadIdx.x < o) red[threadIdx.x] += red[threadIdx.x + o];
        __syncthreads();
    }
    if (threadIdx.x == 0) partial[blockIdx.x] = red[0];
}

// Fixed-order sum of n partials (one block), divided by B.
__global__ void mean_reduce_kernel(int n, const float* __restrict__ partial, int B, float* __restrict__ out) {
    pdl_wait();
    __shared__ float red[1024];
    float s = 0.f;
    for (int i = threadIdx.x; i < n; i += blockDim.x) s += partial[i];
    red[threadIdx.x] = s;
    __syncthreads();
    for (int o = blockDim.x / 2; o; o >>= 1) {
        if (threadIdx.x < o) red[threadIdx.x] += red[threadIdx.x + o];
        __syncthreads();
    }
    if (threadIdx.x == 0) *out = red[0] / (float)B;
}

// ------------------------------------------------------------------ interaction backward

// One block handles samples b = blockIdx.x, += gridDim.x. smem: X [(K+1)][d], S [(K+1)][(K+1)].
__global__ void interact_bwd_kernel(int B, int K, int d, const float* __restrict__ x_dense,
                                    const float* __restrict__ E, const float* __restrict__ dconcat, int ldc,
                                    float* __restrict__ dx_dense, float* __restrict__ dE) {
    pdl_wait();
    extern __shared__ float sm[];
    const int n1 = K + 1;
    float* X = sm;
    float* S = sm + (size_t)n1 * d;
    for (long long b = blockIdx.x; b < B; b += gridDim.x) {
        for (int q = threadIdx.x; q < n1 * d; q += blockDim.x) {
            const int i = q / d, t = q - i * d;
            X[q] = (i == 0) ? x_dense[b * d + t] : E[(b * K + (i - 1)) * (long long)d + t];
        }
        for (int q = threadIdx.x; q < n1 * n1; q += blockDim.x) {
            const int i = q / n1, j = q - i * n1;
            float v = 0.f;
            if (i > j) v = dconcat[b * ldc + d + i * (i - 1) / 2 + j];
            else if (j > i) v = dconcat[b * ldc + d + j * (j - 1) / 2 + i];
            S[q] = v;
        }
        __syncthreads();
        for (int q = threadIdx.x; q < n1 * d; q += blockDim.x) {
            const int i = q / d, t = q - i * d;
            float s = 0.f;
            for (int j = 0; j < n1; ++j) s = fmaf(S[i * n1 + j], X[j * d + t], s);
            if (i == 0)  // x_dense is a ReLU output: its pre-activation gradient is masked
                dx_dense[b * d + t] = (X[t] > 0.f) ? s + dconcat[b * ldc + t] : 0.f;
            else
                dE[(b * K + (i - 1)) * (long long)d + t] = s;
        }
        __syncthreads();
    }
}

// ------------------------------------------------------------------ device-wide exclusive scan (int)

// Block-level inclusive scan of v across the block (blockDim.x <= 1024), returns inclusive value.
__device__ __forceinline__ long long block_scan_incl(long long v, long long* tmp) {
    const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
    for (int o = 1; o < 32; o <<= 1) {
        const long long n = __shfl_up_sync(0xffffffffu, v, o);
        if (lane >= o) v += n;
    }
    if (lane == 31) tmp[w] = v;
    __syncthreads();
    if (w == 0) {
        long long t = lane < (int)(blockDim.x >> 5) ? tmp[lane] : 0;
        for (int o = 1; o < 32; o <<= 1) {
            const long long n = __shfl_up_sync(0xffffffffu, t, o);
            if (lane >= o) t += n;
        }
        tmp[lane] = t;
    }
    __syncthreads();
    if (w > 0) v += tmp[w - 1];
    __syncthreads();
    return v;
}

// Per-block sums of in[0..n) (n read from n_dev if not null).
__global__ void scan_reduce_kernel(const int* __restrict__ in, long long n_host, const long long* n_dev,
                                   long long per_block, long long* __restrict__ block_sums) {
    pdl_wait();
    __shared__ long long tmp[32];
    const long long n = n_dev ? *n_dev : n_host;
    const long long b0 = (long long)blockIdx.x * per_block;
    long long s = 0;
    for (long long i = b0 + threadIdx.x; i < b0 + per_block && i < n; i += blockDim.x) s += in[i];
    s = block_scan_incl(s, tmp);
    if (threadIdx.x == blockDim.x - 1) block_sums[blockIdx.x] = s;
}

// Exclusive scan of the block sums (one block, sequential chunks in order). total -> *total.
__global__ void scan_blocks_kernel(long long* __restrict__ sums, int nblocks, long long* __restrict__ total) {
    pdl_wait();
    __shared__ long long tmp[32];
    long long carry = 0;
    for (int base = 0; base < nblocks; base += blockDim.x) {
        const int i = base + threadIdx.x;
        const long long v = i < nblocks ? sums[i] : 0;
        const long long incl = block_scan_incl(v, tmp);
        if (i < nblocks) sums[i] = carry + incl - v;
        __shared__ long long last;
        if (threadIdx.x == blockDim.x - 1) last = incl;
        __syncthreads();
        carry += last;
        __syncthreads();
    }
    if (threadIdx.x == 0 && total) *total = carry;
}

// out[i] = exclusive prefix of in[] (as long long) for i < n; out[n] = total.
__global__ void scan_down_kernel(const int* __restrict__ in, long long n_host, const long long* n_dev,
                                 long long per_block, const long long* __restrict__ block_off,
                                 long long* __restrict__ out) {
    pdl_wait();
    __shared__ long long tmp[32];
    const long long n = n_dev ? *n_dev : n_host;
    const long long b0 = (long long)blockIdx.x * per_block;
    long long carry = block_off[blockIdx.x];
    for (long long base = b0; base < b0 + per_block; base += blockDim.x) {
        const long long i = base + threadIdx.x;
        const long long v = (i < n && i < b0 + per_block) ? in[i] : 0;
        const long long incl = block_scan_incl(v, tmp);
        if (i < n && i < b0 + per_block) out[i] = carry + incl - v;
        __shared__ long long last;
        if (threadIdx.x == blockDim.x - 1) last = incl;
        __syncthreads();
        carry += last;
        __syncthreads();
        if (base + blockDim.x >= n) break;
    }
    if (blockIdx.x == gridDim.x - 1 && threadIdx.x == 0) out[n] = carry;
}

// ------------------------------------------------------------------ occurrences -> (key, value)

// Valid length of bag kb (0 for bad offsets).
__global__ void bag_len_kernel(long long KB, const int32_t* __restrict__ offsets, long long nnz, int* __restrict__ len,
                               ErrRecord* err) {
    pdl_wait();
    for (long long q = (long long)blockIdx.x * blockDim.x + threadIdx.x; q < KB; q += (long long)gridDim.x * blockDim.x) {
        const long long st = offsets[q], en = offsets[q + 1];
        const bool isbad = st < 0 || en < st || en > nnz;
        len[q] = isbad ? 0 : (int)(en - st);
    }
    (void)err;   // bad bags were counted by the step's forward, which read the same offsets
}

// Writes occurrence o = occ_off[kb] + (p - start) of bag (k, b): key = global row (or `invalid`), value = b*K + k.
__global__ void occ_keys_kernel(int K, int B, const __grid_constant__ TableMeta tm, const int32_t* __restrict__ offsets,
                                const int32_t* __restrict__ indices, const int* __restrict__ len,
                                const long long* __restrict__ occ_off, long long cap, uint32_t invalid,
                                uint32_t* __restrict__ keys, uint32_t* __restrict__ vals, ErrRecord* err) {
    pdl_wait();
    unsigned over = 0;
    const long long KB = (long long)K * B;
    for (long long q = (long long)blockIdx.x * blockDim.x + threadIdx.x; q < KB; q += (long long)gridDim.x * blockDim.x) {
        const int n = len[q];
        if (!n) continue;
        const int k = (int)(q / B), b = (int)(q - (long long)k * B);
        const long long st = offsets[q];
        const long long o0 = occ_off[q];
        for (int e = 0; e < n; ++e) {
            const long long o = o0 + e;
            if (o >= cap) {
                ++over;
                break;
            }
            const int idx = indices[st + e];
            const bool ok = idx >= 0 && (long long)idx < tm.rows[k];
            keys[o] = ok ? (uint32_t)(tm.base[k] + idx) : invalid;
            vals[o] = (uint32_t)b * (uint32_t)K + (uint32_t)k;
        }
    }
    // skipped indices were counted by the step's forward, which read the same bags; occurrences past the
    // gradient buffer's capacity are reported here
    report_warp(err, 0, over);
}

// ------------------------------------------------------------------ stable LSD radix sort of (key, value)

// counts[digit * nblocks + block]
__global__ void __launch_bounds__(SORT_THREADS) radix_hist_kernel(const uint32_t* __restrict__ keys,
                                                                  const long long* __restrict__ n_dev, int shift,
                                                                  int* __restrict__ counts, int nblocks) {
    pdl_wait();
    __shared__ int h[RADIX];
    for (int i = threadIdx.x; i < RADIX; i += blockDim.x) h[i] = 0;
    __syncthreads();
    const long long n = *n_dev;
    const long long t0 = (long long)blockIdx.x * SORT_TILE;
    for (int e = 0; e < SORT_ITEMS; ++e) {
        const long long i = t0 + (long long)e * SORT_THREADS + threadIdx.x;
        if (i < n) atomicAdd(&h[(keys[i] >> shift) & (RADIX - 1)], 1);
    }
    __syncthreads();
    for (int dg = threadIdx.x; dg < RADIX; dg += blockDim.x) counts[dg * nblocks + blockIdx.x] = h[dg];
}

// Stable scatter: tile order is (warp, step, lane); each warp ranks its keys per step with match_any.
__global__ void __launch_bounds__(SORT_THREADS) radix_scatter_kernel(const uint32_t* __restrict__ kin,
                                                                     const uint32_t* __restrict__ vin,
                                                                     const long long* __restrict__ n_dev, int shift,
                                                                     const long long* __restrict__ goff, int nblocks,
                                                                     uint32_t* __restrict__ kout,
                                                                     uint32_t* __restrict__ vout) {
    pdl_wait();
    constexpr int W = SORT_THREADS / 32;
    __shared__ int wcount[W][RADIX];
    __shared__ long long base[W][RADIX];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    for (int i = lane; i < RADIX; i += 32) wcount[warp][i] = 0;
    __syncwarp();
    const long long n = *n_dev;
    const long long w0 = (long long)blockIdx.x * SORT_TILE + (long long)warp * (SORT_ITEMS * 32);
    uint32_t key[SORT_ITEMS], val[SORT_ITEMS];
    int rank[SORT_ITEMS];
    const unsigned lt = (1u << lane) - 1u;
#pragma unroll
    for (int e = 0; e < SORT_ITEMS; ++e) {
        const long long i = w0 + e * 32 + lane;
        const bool valid = i < n;
        key[e] = valid ? kin[i] : 0xFFFFFFFFu;
        val[e] = valid ? vin[i] : 0u;
        const int dg = valid ? (int)((key[e] >> shift) & (RADIX - 1)) : RADIX;  // RADIX: no digit
        const unsigned peers = __match_any_sync(0xffffffffu, dg);
        const int before = __popc(peers & lt);
        int cnt = 0;
        if (valid) cnt = wcount[warp][dg];
        rank[e] = valid ? cnt + before : -1;
        __syncwarp();
        if (valid && before == 0) wcount[warp][dg] = cnt + __popc(peers);
        __syncwarp();
    }
    __syncthreads();
    // base[w][dg] = global offset of (dg, block) + keys of digit dg in warps before w
    for (int dg = threadIdx.x; dg < RADIX; dg += blockDim.x) {
        long long run = goff[(long long)dg * nblocks + blockIdx.x];
        for (int w = 0; w < W; ++w) {
            base[w][dg] = run;
            run += wcount[w][dg];
        }
    }
    __syncthreads();
#pragma unroll
    for (int e = 0; e < SORT_ITEMS; ++e) {
        if (rank[e] >= 0) {
            const int dg = (int)((key[e] >> shift) & (RADIX - 1));
            const long long pos = base[warp][dg] + rank[e];
            kout[pos] = key[e];
            vout[pos] = val[e];
        }
    }
}

// ------------------------------------------------------------------ segments of equal rows

// head[i] = 1 if sorted key i starts a new row (valid keys only: key < invalid).
__global__ void seg_head_kernel(const uint32_t* __restrict__ keys, const long long* __restrict__ n_dev,
                                uint32_t invalid, int* __restrict__ head) {
    pdl_wait();
    const long long n = *n_dev;
    for (long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += (long long)gridDim.x * blockDim.x)
        head[i] = (keys[i] < invalid && (i == 0 || keys[i] != keys[i - 1])) ? 1 : 0;
}

// For each head at i: seg_start[s] = i, seg_row[s] = key; n_valid -> seg_start[n_seg].
__global__ void seg_fill_kernel(const uint32_t* __restrict__ keys, const long long* __restrict__ n_dev,
                                uint32_t invalid, const int* __restrict__ head, const long long* __restrict__ seg_id,
                                long long* __restrict__ seg_start, uint32_t* __restrict__ seg_row,
                                int* __restrict__ seg_pieces, int piece) {
    pdl_wait();
    const long long n = *n_dev;
    for (long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += (long long)gridDim.x * blockDim.x) {
        if (head[i]) {
            const long long s = seg_id[i];
            seg_start[s] = i;
            seg_row[s] = keys[i];
        }
        // the last valid key closes the last segment
        if (keys[i] < invalid && (i + 1 == n || keys[i + 1] >= invalid)) seg_start[seg_id[n]] = i + 1;
    }
    (void)seg_pieces;
    (void)piece;
}

// pieces of segment s = ceil(len / piece)
__global__ void seg_pieces_kernel(const long long* __restrict__ n_seg_dev, const long long* __restrict__ seg_start,
                                  int piece, int* __restrict__ seg_pieces) {
    pdl_wait();
    const long long ns = *n_seg_dev;
    for (long long s = (long long)blockIdx.x * blockDim.x + threadIdx.x; s < ns; s += (long long)gridDim.x * blockDim.x)
        seg_pieces[s] = (int)((seg_start[s + 1] - seg_start[s] + piece - 1) / piece);
}

// piece_seg[p] = segment of piece p
__global__ void piece_owner_kernel(const long long* __restrict__ n_seg_dev, const long long* __restrict__ piece_base,
                                   int* __restrict__ piece_seg) {
    pdl_wait();
    const long long ns = *n_seg_dev;
    for (long long s = (long long)blockIdx.x * blockDim.x + threadIdx.x; s < ns; s += (long long)gridDim.x * blockDim.x)
        for (long long p = piece_base[s]; p < piece_base[s + 1]; ++p) piece_seg[p] = (int)s;
}

// One warp per piece: partial[p][d] = sum over its sorted occurrences (in order) of dE[value].
__global__ void piece_sum_kernel(int d, const long long* __restrict__ n_piece_dev, const int* __restrict__ piece_seg,
                                 const long long* __restrict__ piece_base, const long long* __restrict__ seg_start,
                                 const uint32_t* __restrict__ vals, const float* __restrict__ dE, int piece,
                                 float* __restrict__ partial) {
    pdl_wait();
    const long long np = *n_piece_dev;
    const int lane = threadIdx.x & 31;
    const long long wstride = (long long)gridDim.x * (blockDim.x >> 5);
    for (long long p = (long long)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); p < np; p += wstride) {
        const int s = piece_seg[p];
        const long long j = p - piece_base[s];
        const long long beg = seg_start[s] + j * piece;
        const long long end = beg + piece < seg_start[s + 1] ? beg + piece : seg_start[s + 1];
        for (int t = lane; t < d; t += 32) {
            float acc = 0.f;
            for (long long o = beg; o < end; ++o) acc += dE[(long long)vals[o] * d + t];
            partial[p * d + t] = acc;
        }
    }
}

// Rows of 32 V floats, V per lane (d = 32, 64, 128): one 4/8/16-byte access per lane and row.
template <int V>
struct LaneVec {
    float v[V];
    __device__ __forceinline__ void load(const float* p) {
        if constexpr (V == 4) {
            const float4 t = __ldg(reinterpret_cast<const float4*>(p));
            v[0] = t.x, v[1] = t.y, v[2] = t.z, v[3] = t.w;
        } else if constexpr (V == 2) {
            const float2 t = __ldg(reinterpret_cast<const float2*>(p));
            v[0] = t.x, v[1] = t.y;
        } else {
            v[0] = __ldg(p);
        }
    }
    __device__ __forceinline__ void load_rw(const float* p) {
        if constexpr (V == 4) {
            const float4 t = *reinterpret_cast<const float4*>(p);
            v[0] = t.x, v[1] = t.y, v[2] = t.z, v[3] = t.w;
        } else if constexpr (V == 2) {
            const float2 t = *reinterpret_cast<const float2*>(p);
            v[0] = t.x, v[1] = t.y;
        } else {
            v[0] = *p;
        }
    }
    __device__ __forceinline__ void store(float* p) const {
        if constexpr (V == 4) *reinterpret_cast<float4*>(p) = make_float4(v[0], v[1], v[2], v[3]);
        else if constexpr (V == 2) *reinterpret_cast<float2*>(p) = make_float2(v[0], v[1]);
        else *p = v[0];
    }
};

// piece_sum_kernel for d = 32 V: the same sums in the same order, each occurrence's row read once by the
// warp (16 bytes per lane at d = 128) with four rows in flight.
template <int V>
__global__ void piece_sum_vec_kernel(const long long* __restrict__ n_piece_dev, const int* __restrict__ piece_seg,
                                     const long long* __restrict__ piece_base, const long long* __restrict__ seg_start,
                                     const uint32_t* __restrict__ vals, const float* __restrict__ dE, int piece,
                                     float* __restrict__ partial) {
    pdl_wait();
    constexpr int d = 32 * V;
    const long long np = *n_piece_dev;
    const int lane = threadIdx.x & 31;
    const long long wstride = (long long)gridDim.x * (blockDim.x >> 5);
    for (long long p = (long long)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); p < np; p += wstride) {
        const int s = piece_seg[p];
        const long long j = p - piece_base[s];
        const long long beg = seg_start[s] + j * piece;
        const long long end = beg + piece < seg_start[s + 1] ? beg + piece : seg_start[s + 1];
        float acc[V];
#pragma unroll
        for (int e = 0; e < V; ++e) acc[e] = 0.f;
        long long o = beg;
        for (; o + 4 <= end; o += 4) {
            LaneVec<V> r[4];
#pragma unroll
            for (int u = 0; u < 4; ++u) r[u].load(dE + (long long)vals[o + u] * d + V * lane);
#pragma unroll
            for (int u = 0; u < 4; ++u)
#pragma unroll
                for (int e = 0; e < V; ++e) acc[e] += r[u].v[e];
        }
        for (; o < end; ++o) {
            LaneVec<V> r;
            r.load(dE + (long long)vals[o] * d + V * lane);
#pragma unroll
            for (int e = 0; e < V; ++e) acc[e] += r.v[e];
        }
        LaneVec<V> out;
#pragma unroll
        for (int e = 0; e < V; ++e) out.v[e] = acc[e];
        out.store(partial + p * d + V * lane);
    }
}

// seg_apply_kernel for d = 32 V (same sums, same order)
template <int V>
__global__ void seg_apply_vec_kernel(const long long* __restrict__ n_seg_dev, const long long* __restrict__ piece_base,
                                     const uint32_t* __restrict__ seg_row, const float* __restrict__ partial, float lr,
                                     float* __restrict__ table, float* __restrict__ grad_out) {
    pdl_wait();
    constexpr int d = 32 * V;
    const long long ns = *n_seg_dev;
    const int lane = threadIdx.x & 31;
    const long long wstride = (long long)gridDim.x * (blockDim.x >> 5);
    for (long long s = (long long)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); s < ns; s += wstride) {
        float g[V];
#pragma unroll
        for (int e = 0; e < V; ++e) g[e] = 0.f;
        for (long long p = piece_base[s]; p < piece_base[s + 1]; ++p) {
            LaneVec<V> r;
            r.load(partial + p * d + V * lane);
#pragma unroll
            for (int e = 0; e < V; ++e) g[e] += r.v[e];
        }
        if (table) {
            float* w = table + (long long)seg_row[s] * d + V * lane;
            LaneVec<V> t;
            t.load_rw(w);
#pragma unroll
            for (int e = 0; e < V; ++e) t.v[e] -= lr * g[e];
            t.store(w);
        }
        if (grad_out) {
            LaneVec<V> o;
#pragma unroll
            for (int e = 0; e < V; ++e) o.v[e] = g[e];
            o.store(grad_out + s * d + V * lane);
        }
    }
}

// One warp per segment: g = sum of its piece partials in order; T[row] -= lr * g if table is given,
// and g is written to grad_out[s] if given.
__global__ void seg_apply_kernel(int d, const long long* __restrict__ n_seg_dev, const long long* __restrict__ piece_base,
                                 const uint32_t* __restrict__ seg_row, const float* __restrict__ partial, float lr,
                                 float* __restrict__ table, float* __restrict__ grad_out) {
    pdl_wait();
    const long long ns = *n_seg_dev;
    const int lane = threadIdx.x & 31;
    const long long wstride = (long long)gridDim.x * (blockDim.x >> 5);
    for (long long s = (long long)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); s < ns; s += wstride) {
        for (int t = lane; t < d; t += 32) {
            float g = 0.f;
            for (long long p = piece_base[s]; p < piece_base[s + 1]; ++p) g += partial[p * d + t];
            if (table) {
                float* w = table + (long long)seg_row[s] * d + t;
                *w -= lr * g;
            }
            if (grad_out) grad_out[s * d + t] = g;
        }
    }
}

__global__ void sgd_kernel(long long n, float lr, float* __restrict__ w, const float* __restrict__ g) {
    pdl_wait();
    for (long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += (long long)gridDim.x * blockDim.x)
        w[i] -= lr * g[i];
}

__global__ void copy_count_kernel(const long long* __restrict__ src, int32_t* __restrict__ dst) {
    pdl_wait(); *dst = (int32_t)*src; }

__global__ void clamp_count_kernel(long long* v, long long cap) {
    pdl_wait();
    if (*v > cap) *v = cap;
}

int grid_cap(long long n, int threads, int cap = 148 * 16) {
    long long b = (n + threads - 1) / threads;
    if (b < 1) b = 1;
    return (int)(b < cap ? b : cap);
}

}  // namespace

// ------------------------------------------------------------------ host launchers

dlrm_status launch_bce(int B, const float* z, const float* y, float* dz, float* y_hat, float* partial, float* loss,
                       cudaStream_t st) {
    const int nb = (B + 255) / 256;
    (void)launch_pdl(bce_kernel, dim3(nb), dim3(256), (size_t)(0), st, B, z, y, dz, y_hat, partial);
    DLRM_LAUNCH_CHECK();
    (void)launch_pdl(mean_reduce_kernel, dim3(1), dim3(1024), (size_t)(0), st, nb, partial, B, loss);
    DLRM_LAUNCH_CHECK();
    return DLRM_OK;
}

size_t interact_bwd_smem(int K, int d) { return sizeof(float) * ((size_t)(K + 1) * d + (size_t)(K + 1) * (K + 1)); }

dlrm_status launch_interact_bwd(int B, int K, int d, const float* x_dense, const float* E, const float* dconcat,
                                int ldc, float* dx_dense, float* dE, cudaStream_t st) {
    const size_t smem = interact_bwd_smem(K, d);
    if (smem > 227 * 1024) return DLRM_ERR_UNSUPPORTED;
    if (smem > 48 * 1024) cudaFuncSetAttribute(interact_bwd_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    const int grid = B < 148 * 8 ? B : 148 * 8;
    (void)launch_pdl(interact_bwd_kernel, dim3(grid), dim3(256), (size_t)(smem), st, B, K, d, x_dense, E, dconcat, ldc, dx_dense, dE);
    DLRM_LAUNCH_CHECK();
    return DLRM_OK;
}

// Exclusive scan of int in[0..n) into long long out[0..n], out[n] = total (n from n_dev if given).
static dlrm_status scan_ints(const int* in, long long n_upper, const long long* n_dev, long long* out,
                             long long* block_sums, long long* total, cudaStream_t st) {
    const long long per_block = 8192;
    const int nblocks = (int)((n_upper + per_block - 1) / per_block) + 1;
    (void)launch_pdl(scan_reduce_kernel, dim3(nblocks), dim3(1024), (size_t)(0), st, in, n_upper, n_dev, per_block, block_sums);
    DLRM_LAUNCH_CHECK();
    (void)launch_pdl(scan_blocks_kernel, dim3(1), dim3(1024), (size_t)(0), st, block_sums, nblocks, total);
    DLRM_LAUNCH_CHECK();
    (void)launch_pdl(scan_down_kernel, dim3(nblocks), dim3(1024), (size_t)(0), st, in, n_upper, n_dev, per_block, block_sums, out);
    DLRM_LAUNCH_CHECK();
    return DLRM_OK;
}

size_t scan_block_sums_len(long long n_upper) { return (size_t)((n_upper + 8191) / 8192 + 1); }

size_t sort_blocks(long long n) { return (size_t)((n + SORT_TILE - 1) / SORT_TILE); }

static int key_bits(long long total_rows) {
    int bits = 1;
    while (((long long)1 << bits) <= total_rows) ++bits;
    return bits;
}

int radix_passes(long long total_rows) { return (key_bits(total_rows) + RADIX_BITS - 1) / RADIX_BITS; }

SparseLayout sparse_layout(long long KB, long long nnz, int d) {
    SparseLayout L;
    size_t off = 0;
    auto take = [&](size_t bytes) {
        const size_t o = off;
        off = align_up(off + bytes, 256);
        return o;
    };
    const long long cap = nnz > 0 ? nnz : 1;
    const size_t nsb = sort_blocks(cap);
    L.cap = cap;
    L.counts = take(sizeof(long long) * 8);
    L.bag_len = take(sizeof(int) * (size_t)KB);
    L.occ_off = take(sizeof(long long) * ((size_t)KB + 1));
    L.keys[0] = take(sizeof(uint32_t) * cap);
    L.keys[1] = take(sizeof(uint32_t) * cap);
    L.vals[0] = take(sizeof(uint32_t) * cap);
    L.vals[1] = take(sizeof(uint32_t) * cap);
    L.hist = take(sizeof(int) * (size_t)RADIX * nsb);
    L.hist_off = take(sizeof(long long) * ((size_t)RADIX * nsb + 1));
    L.head = take(sizeof(int) * cap);
    L.seg_id = take(sizeof(long long) * (cap + 1));
    L.seg_start = take(sizeof(long long) * (cap + 1));
    L.seg_row = take(sizeof(uint32_t) * cap);
    L.seg_pieces = take(sizeof(int) * cap);
    L.piece_base = take(sizeof(long long) * (cap + 1));
    const long long max_pieces = cap / SPARSE_PIECE + cap;
    L.piece_seg = take(sizeof(int) * max_pieces);
    L.partial = take(sizeof(float) * (size_t)max_pieces * d);
    const long long nscan = std::max<long long>(std::max<long long>(KB, cap), (long long)RADIX * nsb);
    L.scan_sums = take(sizeof(long long) * scan_block_sums_len(nscan));
    L.total = off;
    return L;
}

// Sort the batch's occurrences by row and cut them into segments and pieces.
// counts: [0] n_occ, [1] n_valid (unused), [2] n_seg, [3] n_pieces.
dlrm_status launch_sparse_prepare(int K, int B, const TableMeta& tm, long long total_rows, const int32_t* offsets,
                                  const int32_t* indices, long long nnz, char* base, const SparseLayout& L,
                                  ErrRecord* err, int* sorted_buf, cudaStream_t st) {
    const long long KB = (long long)K * B;
    long long* counts = reinterpret_cast<long long*>(base + L.counts);
    int* bag_len = reinterpret_cast<int*>(base + L.bag_len);
    long long* occ_off = reinterpret_cast<long long*>(base + L.occ_off);
    long long* sums = reinterpret_cast<long long*>(base + L.scan_sums);
    const uint32_t invalid = (uint32_t)total_rows;
    const int bits = key_bits(total_rows);

    (void)launch_pdl(bag_len_kernel, dim3(grid_cap(KB, 256)), dim3(256), (size_t)(0), st, KB, offsets, nnz, bag_len, err);
    DLRM_LAUNCH_CHECK();
    dlrm_status r = scan_ints(bag_len, KB, nullptr, occ_off, sums, &counts[0], st);
    if (r) return r;
    // n_occ = min(total occurrences, capacity)
    uint32_t* keys[2] = {reinterpret_cast<uint32_t*>(base + L.keys[0]), reinterpret_cast<uint32_t*>(base + L.keys[1])};
    uint32_t* vals[2] = {reinterpret_cast<uint32_t*>(base + L.vals[0]), reinterpret_cast<uint32_t*>(base + L.vals[1])};
    (void)launch_pdl(occ_keys_kernel, dim3(grid_cap(KB, 256)), dim3(256), (size_t)(0), st, K, B, tm, offsets, indices, bag_len, occ_off, L.cap, invalid,
                                                        keys[0], vals[0], err);
    DLRM_LAUNCH_CHECK();
    (void)launch_pdl(clamp_count_kernel, dim3(1), dim3(1), (size_t)(0), st, &counts[0], L.cap);
    DLRM_LAUNCH_CHECK();

    const int nsb = (int)sort_blocks(L.cap);
    int* hist = reinterpret_cast<int*>(base + L.hist);
    long long* hist_off = reinterpret_cast<long long*>(base + L.hist_off);
    int cur = 0;
    for (int shift = 0; shift < bits; shift += RADIX_BITS) {
        (void)launch_pdl(radix_hist_kernel, dim3(nsb), dim3(SORT_THREADS), (size_t)(0), st, keys[cur], &counts[0], shift, hist, nsb);
        DLRM_LAUNCH_CHECK();
        if ((r = scan_ints(hist, (long long)RADIX * nsb, nullptr, hist_off, sums, nullptr, st))) return r;
        (void)launch_pdl(radix_scatter_kernel, dim3(nsb), dim3(SORT_THREADS), (size_t)(0), st, keys[cur], vals[cur], &counts[0], shift, hist_off, nsb,
                                                            keys[cur ^ 1], vals[cur ^ 1]);
        DLRM_LAUNCH_CHECK();
        cur ^= 1;
    }
    *sorted_buf = cur;
    int* head = reinterpret_cast<int*>(base + L.head);
    long long* seg_id = reinterpret_cast<long long*>(base + L.seg_id);
    long long* seg_start = reinterpret_cast<long long*>(base + L.seg_start);
    uint32_t* seg_row = reinterpret_cast<uint32_t*>(base + L.seg_row);
    int* seg_pieces = reinterpret_cast<int*>(base + L.seg_pieces);
    long long* piece_base = reinterpret_cast<long long*>(base + L.piece_base);
    int* piece_seg = reinterpret_cast<int*>(base + L.piece_seg);
    (void)launch_pdl(seg_head_kernel, dim3(grid_cap(L.cap, 256)), dim3(256), (size_t)(0), st, keys[cur], &counts[0], invalid, head);
    DLRM_LAUNCH_CHECK();
    if ((r = scan_ints(head, L.cap, &counts[0], seg_id, sums, &counts[2], st))) return r;
    (void)launch_pdl(seg_fill_kernel, dim3(grid_cap(L.cap, 256)), dim3(256), (size_t)(0), st, keys[cur], &counts[0], invalid, head, seg_id, seg_start, seg_row,
                                                          seg_pieces, SPARSE_PIECE);
    DLRM_LAUNCH_CHECK();
    (void)launch_pdl(seg_pieces_kernel, dim3(grid_cap(L.cap, 256)), dim3(256), (size_t)(0), st, &counts[2], seg_start, SPARSE_PIECE, seg_pieces);
    DLRM_LAUNCH_CHECK();
    if ((r = scan_ints(seg_pieces, L.cap, &counts[2], piece_base, sums, &counts[3], st))) return r;
    (void)launch_pdl(piece_owner_kernel, dim3(grid_cap(L.cap, 256)), dim3(256), (size_t)(0), st, &counts[2], piece_base, piece_seg);
    DLRM_LAUNCH_CHECK();
    return DLRM_OK;
}

dlrm_status launch_sparse_apply(int d, const char* base, const SparseLayout& L, int sorted_buf, const float* dE,
                                float lr, float* table, float* grad_out, uint32_t* rows_out, int32_t* n_rows_out,
                                cudaStream_t st) {
    const long long* counts = reinterpret_cast<const long long*>(base + L.counts);
    const uint32_t* vals = reinterpret_cast<const uint32_t*>(base + L.vals[sorted_buf]);
    const long long* seg_start = reinterpret_cast<const long long*>(base + L.seg_start);
    const uint32_t* seg_row = reinterpret_cast<const uint32_t*>(base + L.seg_row);
    const long long* piece_base = reinterpret_cast<const long long*>(base + L.piece_base);
    const int* piece_seg = reinterpret_cast<const int*>(base + L.piece_seg);
    float* partial = const_cast<float*>(reinterpret_cast<const float*>(base + L.partial));
    const int blocks = 148 * 8;
    // the vector kernels need d = 32, 64 or 128 and 16-byte aligned rows everywhere (dE, partials and the
    // table are aligned by construction; a caller's grad_out may not be)
    const bool vec = (d == 32 || d == 64 || d == 128) && (((uintptr_t)grad_out & 15) == 0);
#define DLRM_SPARSE_VEC(V)                                                                                        \
    (void)launch_pdl(piece_sum_vec_kernel<V>, dim3(blocks), dim3(256), (size_t)(0), st, &counts[3], piece_seg, piece_base, seg_start, vals, dE,        \
                                                    SPARSE_PIECE, partial);                                         \
    DLRM_LAUNCH_CHECK();                                                                                          \
    (void)launch_pdl(seg_apply_vec_kernel<V>, dim3(blocks), dim3(256), (size_t)(0), st, &counts[2], piece_base, seg_row, partial, lr, table, grad_out); \
    DLRM_LAUNCH_CHECK();
    if (vec && d == 128) {
        DLRM_SPARSE_VEC(4)
    } else if (vec && d == 64) {
        DLRM_SPARSE_VEC(2)
    } else if (vec && d == 32) {
        DLRM_SPARSE_VEC(1)
    } else {
        (void)launch_pdl(piece_sum_kernel, dim3(blocks), dim3(256), (size_t)(0), st, d, &counts[3], piece_seg, piece_base, seg_start, vals, dE,
                                                 SPARSE_PIECE, partial);
        DLRM_LAUNCH_CHECK();
        (void)launch_pdl(seg_apply_kernel, dim3(blocks), dim3(256), (size_t)(0), st, d, &counts[2], piece_base, seg_row, partial, lr, table, grad_out);
        DLRM_LAUNCH_CHECK();
    }
#undef DLRM_SPARSE_VEC
    if (rows_out) {
        cudaMemcpyAsync(rows_out, seg_row, sizeof(uint32_t) * L.cap, cudaMemcpyDeviceToDevice, st);
    }
    if (n_rows_out) {
        (void)launch_pdl(copy_count_kernel, dim3(1), dim3(1), (size_t)(0), st, &counts[2], n_rows_out);
        DLRM_LAUNCH_CHECK();
    }
    return DLRM_OK;
}

dlrm_status launch_sgd(long long n, float lr, float* w, const float* g, cudaStream_t st) {
    if (n <= 0) return DLRM_OK;
    (void)launch_pdl(sgd_kernel, dim3(grid_cap(n, 256)), dim3(256), (size_t)(0), st, n, lr, w, g);
    DLRM_LAUNCH_CHECK();
    return DLRM_OK;
}

}  // namespace dlrm
