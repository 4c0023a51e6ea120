// fp32 pairwise dot interaction of the training step on the tensor cores,
// with the EmbeddingBag gather fused in ("DLRM", briansu.co, section 3 for the
// sum pooling and section 4, equation "Interaction": Z = tril(X X^T) over
// X = [x_dense; e_1; ...; e_K], self-interactions left out; the backward is its
// derivative: dX_i = sum_{j != i} dZ_ij X_j with dZ symmetric).
//
// One warp per sample, fp32 tables, K = 26 bags of d in {64, 128}.
// Both directions gather the sample's rows themselves (one bulk copy of the
// whole row per one-row bag, completing on the warp's mbarrier; fp32 sums for
// bags of several rows; zeros for empty bags), so the pooled vectors are never
// written to memory. The forward's products are 3xTF32 on mma.sync.m16n8k8:
// x = hi + lo with hi the TF32 rounding of x, and a b = a_hi b_hi + a_hi b_lo +
// a_lo b_hi; the three products of each 8-deep step are summed on their own
// and then added to fp32 accumulators in registers, so no long sum is carried
// by the tensor core's accumulation.
//  forward:  X in shared memory (row 0 = x_dense, rows 1..K the bags); the
//            Gram's lower-triangle 16x8 tiles; G staged over X, each concat
//            column written as a TF32 pair (hi, lo) for the top MLP's 3xTF32
//            GEMM. The forward also counts skipped indices and bad bags.
//  backward: on the CUDA cores (at this size 3xTF32 with padding to 32 costs
//            about four times the FP32 multiply-adds, more than the legacy
//            tensor pipe gains): lane l holds columns [V l, V l + V) of all
//            K + 1 vectors in registers, the sample's dZ is expanded into a
//            symmetric matrix S in shared memory (zero diagonal), and lane l
//            forms dX_i for its columns from broadcast reads of row i; the
//            next sample's rows are gathered by bulk copies while this one
//            computes. x_dense's gradient is masked by its ReLU and written as
//            a pair, dE plain [B][K][d].
#include "async_copy.cuh"
#include "common.cuh"
#include "kernels.cuh"

namespace dlrm {
namespace {

using namespace ac;

constexpr int KP = 32;                  // padded vector count
constexpr int FW = 7;                   // forward: warps per block (2 blocks per SM)
constexpr int BW = 4;                   // backward: warps per block (3 blocks per SM)
constexpr uint32_t CODE_EMPTY = 0xFFFFFFFFu;
constexpr uint32_t CODE_MULTI = 0xFFFFFFFEu;
constexpr unsigned FULL = 0xffffffffu;

// x rounded to the nearest TF32 value (10 stored mantissa bits), left in fp32.
__device__ __forceinline__ float tf32_hi(float v) {
    const uint32_t u = __float_as_uint(v);
    uint32_t r = u + 0x1000u;
    if ((r & 0x7F800000u) == 0x7F800000u) r = u;   // keep inf/NaN and do not round up into them
    return __uint_as_float(r & 0xFFFFE000u);
}
__device__ __forceinline__ void split(uint32_t x, uint32_t& hi, uint32_t& lo) {
    const float h = tf32_hi(__uint_as_float(x));
    hi = __float_as_uint(h);
    lo = __float_as_uint(__uint_as_float(x) - h);
}

__device__ __forceinline__ void mma_tf32(float (&c)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k8.row.col.f32.tf32.tf32.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%0,%1,%2,%3};"
        : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// One 8-deep 3xTF32 step of a 16x8 tile, added to acc.
__device__ __forceinline__ void mma3(float (&acc)[4], const uint32_t (&ah)[4], const uint32_t (&al)[4], uint32_t bh0,
                                     uint32_t bh1, uint32_t bl0, uint32_t bl1) {
    float t[4] = {0.f, 0.f, 0.f, 0.f};
    mma_tf32(t, al, bh0, bh1);
    mma_tf32(t, ah, bl0, bl1);
    mma_tf32(t, ah, bh0, bh1);
#pragma unroll
    for (int e = 0; e < 4; ++e) acc[e] += t[e];
}

// Strict-lower-triangle pair of position p: (i, j), j < i, p = i(i-1)/2 + j.
__device__ __forceinline__ void tri_pair(int p, int& i, int& j) {
    i = (int)((1.0f + sqrtf(8.0f * (float)p + 1.0f)) * 0.5f);
    while (i * (i - 1) / 2 > p) --i;
    while ((i + 1) * i / 2 <= p) ++i;
    j = p - i * (i - 1) / 2;
}

// Rows 1..K of the sample's tile X (row stride RS floats): one bulk copy per one-row bag, issued on
// `bar` with the phase's byte count; fp32 sums for bags of several rows and zeros for empty bags,
// written with ordinary stores. With `count`, skipped indices and bad bags are counted.
template <int D, int RS>
__device__ __forceinline__ void gather_rows(float* X, uint32_t X_s, const float* __restrict__ tables,
                                            const TableMeta& tm, int K, int B, long long b,
                                            const int32_t* __restrict__ offsets, const int32_t* __restrict__ indices,
                                            long long nnz, uint32_t bar, bool count, unsigned& oob, unsigned& bad,
                                            int lane) {
    uint32_t code = CODE_EMPTY;
    if (lane < K) {
        const long long o = (long long)lane * B + b;
        const long long st = offsets[o], en = offsets[o + 1];
        if (st < 0 || en < st || en > nnz) {
            if (count) ++bad;
        } else if (en - st == 1) {
            const int idx = __ldg(indices + st);
            if (idx >= 0 && (long long)idx < tm.rows[lane])
                code = (uint32_t)(tm.base[lane] + idx);
            else if (count)
                ++oob;
        } else if (en - st > 1) {
            code = CODE_MULTI;
        }
    }
    const unsigned one = __ballot_sync(FULL, code < CODE_MULTI);
    const unsigned multi = __ballot_sync(FULL, code == CODE_MULTI);
    const unsigned empty = __ballot_sync(FULL, lane < K && code == CODE_EMPTY);
    // the previous sample's accesses to the tile come before the copies that overwrite it
    fence_proxy_async();
    __syncwarp();
    if (lane == 0) bar_expect(bar, (uint32_t)__popc(one) * D * 4);
    __syncwarp();
    if (code < CODE_MULTI) bulk_row(X_s + (uint32_t)((lane + 1) * RS * 4), tables + (long long)code * D, D * 4, bar);
    // bags of several rows and empty bags: D/4 lanes per row, 32/(D/4) rows at a time
    constexpr int GL = D / 4, NG = 32 / GL;
    const int gi = lane / GL, g = lane % GL;
    for (unsigned long long rest = empty | multi; rest; rest = drop_bits(rest, NG)) {
        const int k = nth_bit(rest, gi);
        if (k < 0) continue;
        float4 a = make_float4(0.f, 0.f, 0.f, 0.f);
        if ((multi >> k) & 1u) {
            const int st = offsets[(long long)k * B + b], en = offsets[(long long)k * B + b + 1];
            for (int p = st; p < en; ++p) {
                const int idx = __ldg(indices + p);
                if (idx >= 0 && (long long)idx < tm.rows[k]) {
                    const float4 v = __ldg(reinterpret_cast<const float4*>(tables + (tm.base[k] + idx) * (long long)D) + g);
                    a.x += v.x;
                    a.y += v.y;
                    a.z += v.z;
                    a.w += v.w;
                } else if (count && g == 0) {
                    ++oob;
                }
            }
        }
        *reinterpret_cast<float4*>(X + (k + 1) * RS + 4 * g) = a;
    }
}

template <int D>
__global__ void __launch_bounds__(FW * 32, 2) interact_fwd_tc_kernel(
    const float* __restrict__ tables, const __grid_constant__ TableMeta tm, int K, int B,
    const int32_t* __restrict__ offsets, const int32_t* __restrict__ indices, long long nnz,
    const float* __restrict__ xh, const float* __restrict__ xl, int ldx, float* __restrict__ ch,
    float* __restrict__ cl, int ldc, int warp_bytes, ErrRecord* err) {
    pdl_wait();
    constexpr int RS = D + 4;        // X row stride in floats: rows 16 bytes apart modulo 128 (conflict-free ldmatrix)
    constexpr int GS = KP + 8;       // G row stride in floats
    constexpr uint32_t ZERO_SLOT = KP * GS;
    constexpr int NX = (D + 127) / 128;
    extern __shared__ __align__(16) unsigned char smem[];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    unsigned char* xw = smem + (size_t)warp * warp_bytes;
    float* X = reinterpret_cast<float*>(xw);
    float* G = X;                    // staged over the tile once the MMAs have read it
    const uint32_t X_s = (uint32_t)__cvta_generic_to_shared(xw);
    unsigned char* tail = smem + (size_t)FW * warp_bytes;
    uint16_t* src_s = reinterpret_cast<uint16_t*>(tail);   // G slot of concat column D + c
    const int nsrc = ldc - D;
    const uint32_t bar = (uint32_t)__cvta_generic_to_shared(tail + ((nsrc * 2 + 7) & ~7)) + 8u * (uint32_t)warp;
    const int P = K * (K + 1) / 2;
    for (int c = threadIdx.x; c < nsrc; c += blockDim.x) {
        uint32_t src = ZERO_SLOT;
        if (c < P) {
            int i, j;
            tri_pair(c, i, j);
            src = (uint32_t)(i * GS + j);
        }
        src_s[c] = (uint16_t)src;
    }
    if (lane == 0) {
        bar_init(bar);
        fence_proxy_async();
    }
    __syncthreads();

    unsigned oob = 0, bad = 0;
    bool timed_out = false;
    uint32_t parity = 0;
    const int first_tries = g_rows_wait_tries;
    const long long nw = (long long)gridDim.x * FW;
    for (long long b = (long long)blockIdx.x * FW + warp; b < B; b += nw) {
        float4 h[NX], l[NX];
#pragma unroll
        for (int q = 0; q < NX; ++q) {
            const int c = 4 * lane + 128 * q;
            if (c < D) {
                h[q] = __ldg(reinterpret_cast<const float4*>(xh + b * ldx + c));
                l[q] = __ldg(reinterpret_cast<const float4*>(xl + b * ldx + c));
            }
        }
        gather_rows<D, RS>(X, X_s, tables, tm, K, B, b, offsets, indices, nnz, bar, true, oob, bad, lane);
#pragma unroll
        for (int q = 0; q < NX; ++q) {
            const int c = 4 * lane + 128 * q;
            if (c < D)
                *reinterpret_cast<float4*>(X + c) =
                    make_float4(h[q].x + l[q].x, h[q].y + l[q].y, h[q].z + l[q].z, h[q].w + l[q].w);
        }
        if (!rows_ready(bar, parity, first_tries)) {   // rows landed (drained): stop this warp's samples
            timed_out = true;
            break;
        }
        parity ^= 1u;
        __syncwarp();

        // lower-triangle tiles of the Gram: (mt, nt) for nt <= 2 mt + 1
        float acc[6][4];
#pragma unroll
        for (int t = 0; t < 6; ++t) acc[t][0] = acc[t][1] = acc[t][2] = acc[t][3] = 0.f;
#pragma unroll 2
        for (int ks = 0; ks < D / 8; ++ks) {
            uint32_t ah[2][4], al[2][4];
#pragma unroll
            for (int mt = 0; mt < 2; ++mt) {
                uint32_t a[4];
                ldmatrix_x4(X_s + (uint32_t)(((16 * mt + (lane & 15)) * RS + 8 * ks + 4 * (lane >> 4)) * 4), a);
#pragma unroll
                for (int e = 0; e < 4; ++e) split(a[e], ah[mt][e], al[mt][e]);
            }
            int t = 0;
#pragma unroll
            for (int mt = 0; mt < 2; ++mt) {
#pragma unroll
                for (int nt = 0; nt <= 2 * mt + 1; ++nt, ++t) {
                    const int r0 = (nt & 1) ? 1 : 0, r1 = (nt & 1) ? 3 : 2;
                    mma3(acc[t], ah[mt], al[mt], ah[nt >> 1][r0], ah[nt >> 1][r1], al[nt >> 1][r0], al[nt >> 1][r1]);
                }
            }
        }
        __syncwarp();  // every lane's ldmatrix of X is done before G overwrites it
        {
            const int gr = lane >> 2, tc = (lane & 3) * 2;
            int t = 0;
#pragma unroll
            for (int mt = 0; mt < 2; ++mt) {
#pragma unroll
                for (int nt = 0; nt <= 2 * mt + 1; ++nt, ++t) {
                    float* p0 = G + (16 * mt + gr) * GS + 8 * nt + tc;
                    *reinterpret_cast<float2*>(p0) = make_float2(acc[t][0], acc[t][1]);
                    *reinterpret_cast<float2*>(p0 + 8 * GS) = make_float2(acc[t][2], acc[t][3]);
                }
            }
            if (lane == 0) G[ZERO_SLOT] = 0.f;
        }
        __syncwarp();

        // concat row as a pair: x_dense (already a pair), then Z
        float* rh = ch + b * ldc;
        float* rl = cl + b * ldc;
#pragma unroll
        for (int q = 0; q < NX; ++q) {
            const int c = 4 * lane + 128 * q;
            if (c < D) {
                *reinterpret_cast<float4*>(rh + c) = h[q];
                *reinterpret_cast<float4*>(rl + c) = l[q];
            }
        }
        for (int c = lane; c < nsrc; c += 32) {
            const float z = G[src_s[c]];
            const float zh = tf32_hi(z);
            rh[D + c] = zh;
            rl[D + c] = z - zh;
        }
        __syncwarp();  // the tile is reused by the next sample
    }
    if (timed_out && lane == 0) atomicOr(&err->flags, ERR_TIMEOUT);
    report_warp(err, oob, bad);
}

// Backward on the CUDA cores: lane l holds columns [V l, V l + V) of all N1 = K + 1 vectors in registers
// and forms dX_i = sum_j S_ij X_j from broadcast 16-byte reads of row i of S. The next sample's rows are
// gathered into the warp's shared-memory buffer (bulk copies) while this sample computes.
template <int N1, int V>
__global__ void __launch_bounds__(BW * 32, 3) interact_bwd_fma_kernel(
    const float* __restrict__ tables, const __grid_constant__ TableMeta tm, int B,
    const int32_t* __restrict__ offsets, const int32_t* __restrict__ indices, long long nnz,
    const float* __restrict__ xh, const float* __restrict__ xl, int ldx, const float* __restrict__ dcat, int ldc,
    float* __restrict__ dxh, float* __restrict__ dxl, int lddx, float* __restrict__ dE, int warp_bytes,
    ErrRecord* err) {
    pdl_wait();
    constexpr int K = N1 - 1;
    constexpr int D = 32 * V;
    constexpr int SR = (N1 + 3) / 4 * 4;   // row stride of the symmetric dZ matrix
    constexpr int P = N1 * (N1 - 1) / 2;
    extern __shared__ __align__(16) unsigned char smem[];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    unsigned char* xw = smem + (size_t)warp * warp_bytes;
    float* R = reinterpret_cast<float*>(xw);        // rows 1..K (row k at k * D); row 0 unused
    float* S = R + N1 * D;
    const uint32_t R_s = (uint32_t)__cvta_generic_to_shared(xw);
    unsigned char* tail = smem + (size_t)BW * warp_bytes;
    uint16_t* ij_s = reinterpret_cast<uint16_t*>(tail);     // (i << 8) | j of dZ position p
    const uint32_t bar = (uint32_t)__cvta_generic_to_shared(tail + ((P * 2 + 7) & ~7)) + 8u * (uint32_t)warp;
    for (int p = threadIdx.x; p < P; p += blockDim.x) {
        int i, j;
        tri_pair(p, i, j);
        ij_s[p] = (uint16_t)((i << 8) | j);
    }
    // the diagonal and the padding columns of S stay zero; every other entry is rewritten per sample
    for (int q = lane; q < N1 * SR; q += 32) S[q] = 0.f;
    if (lane == 0) {
        bar_init(bar);
        fence_proxy_async();
    }
    __syncthreads();

    unsigned oob = 0, bad = 0;
    bool timed_out = false;
    uint32_t parity = 0;
    const int first_tries = g_rows_wait_tries;
    const long long nw = (long long)gridDim.x * BW;
    long long b = (long long)blockIdx.x * BW + warp;
    if (b < B) gather_rows<D, D>(R, R_s, tables, tm, K, B, b, offsets, indices, nnz, bar, false, oob, bad, lane);
    for (; b < B; b += nw) {
        float x[N1][V];
        {
            float h[V], l[V];
            if constexpr (V == 4) {
                const float4 th = __ldg(reinterpret_cast<const float4*>(xh + b * ldx) + lane);
                const float4 tl = __ldg(reinterpret_cast<const float4*>(xl + b * ldx) + lane);
                h[0] = th.x; h[1] = th.y; h[2] = th.z; h[3] = th.w;
                l[0] = tl.x; l[1] = tl.y; l[2] = tl.z; l[3] = tl.w;
            } else {
                const float2 th = __ldg(reinterpret_cast<const float2*>(xh + b * ldx) + lane);
                const float2 tl = __ldg(reinterpret_cast<const float2*>(xl + b * ldx) + lane);
                h[0] = th.x; h[1] = th.y;
                l[0] = tl.x; l[1] = tl.y;
            }
#pragma unroll
            for (int e = 0; e < V; ++e) x[0][e] = h[e] + l[e];
        }
        if (!rows_ready(bar, parity, first_tries)) {   // rows landed (drained): stop this warp's samples
            timed_out = true;
            break;
        }
        parity ^= 1u;
        __syncwarp();
#pragma unroll
        for (int k = 1; k < N1; ++k) {
            if constexpr (V == 4) {
                const float4 t = reinterpret_cast<const float4*>(R + k * D)[lane];
                x[k][0] = t.x; x[k][1] = t.y; x[k][2] = t.z; x[k][3] = t.w;
            } else {
                const float2 t = reinterpret_cast<const float2*>(R + k * D)[lane];
                x[k][0] = t.x; x[k][1] = t.y;
            }
        }
        // the next sample's rows come in while this one computes (gather_rows orders the reads above first)
        if (b + nw < B)
            gather_rows<D, D>(R, R_s, tables, tm, K, B, b + nw, offsets, indices, nnz, bar, false, oob, bad, lane);
        // S[i][j] = S[j][i] = dZ(i, j) for j < i
        const float* dz = dcat + b * ldc + D;
        for (int p = lane; p < P; p += 32) {
            const float g = __ldcs(dz + p);
            const uint32_t ij = ij_s[p];
            const int i = (int)(ij >> 8), j = (int)(ij & 255u);
            S[i * SR + j] = g;
            S[j * SR + i] = g;
        }
        __syncwarp();
#pragma unroll
        for (int i = 0; i < N1; ++i) {
            float acc[V];
#pragma unroll
            for (int e = 0; e < V; ++e) acc[e] = 0.f;
#pragma unroll
            for (int j4 = 0; j4 < SR; j4 += 4) {
                const float4 s4 = *reinterpret_cast<const float4*>(S + i * SR + j4);
                const float sv[4] = {s4.x, s4.y, s4.z, s4.w};
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                    if (j4 + u < N1 && j4 + u != i) {
#pragma unroll
                        for (int e = 0; e < V; ++e) acc[e] = fmaf(sv[u], x[j4 + u][e], acc[e]);
                    }
                }
            }
            if (i == 0) {
                // x_dense is a ReLU output: its pre-activation gradient is masked
                float gd[V], oh[V], ol[V];
                if constexpr (V == 4) {
                    const float4 dc = __ldg(reinterpret_cast<const float4*>(dcat + b * ldc) + lane);
                    gd[0] = dc.x; gd[1] = dc.y; gd[2] = dc.z; gd[3] = dc.w;
                } else {
                    const float2 dc = __ldg(reinterpret_cast<const float2*>(dcat + b * ldc) + lane);
                    gd[0] = dc.x; gd[1] = dc.y;
                }
#pragma unroll
                for (int e = 0; e < V; ++e) {
                    const float g = x[0][e] > 0.f ? acc[e] + gd[e] : 0.f;
                    oh[e] = tf32_hi(g);
                    ol[e] = g - oh[e];
                }
                if constexpr (V == 4) {
                    reinterpret_cast<float4*>(dxh + b * lddx)[lane] = make_float4(oh[0], oh[1], oh[2], oh[3]);
                    reinterpret_cast<float4*>(dxl + b * lddx)[lane] = make_float4(ol[0], ol[1], ol[2], ol[3]);
                } else {
                    reinterpret_cast<float2*>(dxh + b * lddx)[lane] = make_float2(oh[0], oh[1]);
                    reinterpret_cast<float2*>(dxl + b * lddx)[lane] = make_float2(ol[0], ol[1]);
                }
            } else {
                float* o = dE + (b * K + (i - 1)) * (long long)D;
                if constexpr (V == 4)
                    reinterpret_cast<float4*>(o)[lane] = make_float4(acc[0], acc[1], acc[2], acc[3]);
                else
                    reinterpret_cast<float2*>(o)[lane] = make_float2(acc[0], acc[1]);
            }
        }
        __syncwarp();  // S is rewritten by the next sample
    }
    if (timed_out && lane == 0) atomicOr(&err->flags, ERR_TIMEOUT);
}

// Bytes of one warp's region and of the whole block.
int fwd_warp_bytes(int K, int d) {
    const int x = (K + 1) * (d + 4) * 4;
    const int gb = (KP * (KP + 8) + 1) * 4;
    return ((x > gb ? x : gb) + 15) & ~15;
}
size_t fwd_smem(int K, int d, int ldc, int& wb) {
    wb = fwd_warp_bytes(K, d);
    const size_t tail = (((size_t)(ldc - d) * 2 + 7) & ~(size_t)7) + 8 * FW;
    // ldmatrix reads rows up to KP-1 of the last warp's tile: keep those reads inside the allocation
    const size_t reach = (size_t)KP * (d + 4) * 4;
    const size_t slack = reach > (size_t)wb + tail ? reach - wb - tail : 0;
    return (size_t)FW * wb + tail + ((slack + 15) & ~(size_t)15);
}
int bwd_warp_bytes(int K, int d) { return ((K + 1) * d + (K + 1) * ((K + 4) / 4 * 4)) * 4; }
size_t bwd_smem(int K, int d, int& wb) {
    wb = bwd_warp_bytes(K, d);
    const int P = K * (K + 1) / 2;
    return (size_t)BW * wb + (((size_t)P * 2 + 7) & ~(size_t)7) + 8 * BW;
}

int persistent_grid(long long B, int warps) {
    const long long blocks = (B + warps - 1) / warps;
    return (int)(blocks < 148 * 2 ? blocks : 148 * 2);
}

}  // namespace

bool interact_tc_supported(int K, int d, long long total_rows, int ldc) {
    // the backward keeps the K + 1 vectors in registers: compiled for K = 26 and d = 64, 128
    if (K != 26 || !(d == 64 || d == 128)) return false;
    if (total_rows >= (long long)CODE_MULTI) return false;
    if (ldc < d + K * (K + 1) / 2 || ldc % 4) return false;
    int wb;
    return fwd_smem(K, d, ldc, wb) <= 227 * 1024 && bwd_smem(K, d, wb) <= 227 * 1024;
}

dlrm_status launch_interact_fwd_tc(const TableMeta& tm, const float* tables, int K, int d, int B,
                                   const int32_t* offsets, const int32_t* indices, long long nnz, F32Pair x_dense,
                                   float* concat_hi, float* concat_lo, int ldc, ErrRecord* err, cudaStream_t st) {
    if (!interact_tc_supported(K, d, tm.base[K - 1] + tm.rows[K - 1], ldc)) return DLRM_ERR_UNSUPPORTED;
    if (B == 0) return DLRM_OK;
    int wb;
    const size_t smem = fwd_smem(K, d, ldc, wb);
    const int grid = persistent_grid(B, FW);
#define DLRM_FWD_TC(DV)                                                                                     \
    {                                                                                                      \
        auto kern = interact_fwd_tc_kernel<DV>;                                                            \
        cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);                \
        (void)launch_pdl(kern, dim3(grid), dim3(FW * 32), (size_t)(smem), st, tables, tm, K, B, offsets, indices, nnz, x_dense.hi, x_dense.lo, \
                                          x_dense.ld, concat_hi, concat_lo, ldc, wb, err);                 \
    }
    if (d == 128) DLRM_FWD_TC(128) else DLRM_FWD_TC(64)
#undef DLRM_FWD_TC
    DLRM_LAUNCH_CHECK();
    return DLRM_OK;
}

dlrm_status launch_interact_bwd_tc(const TableMeta& tm, const float* tables, int K, int d, int B,
                                   const int32_t* offsets, const int32_t* indices, long long nnz, F32Pair x_dense,
                                   const float* dconcat, int ldc, float* dx_hi, float* dx_lo, int lddx, float* dE,
                                   ErrRecord* err, cudaStream_t st) {
    if (!interact_tc_supported(K, d, tm.base[K - 1] + tm.rows[K - 1], ldc)) return DLRM_ERR_UNSUPPORTED;
    if (B == 0) return DLRM_OK;
    int wb;
    const size_t smem = bwd_smem(K, d, wb);
    const long long blocks = (B + BW - 1) / BW;
    const int grid = (int)(blocks < 148 * 3 ? blocks : 148 * 3);
#define DLRM_BWD(VV)                                                                                         \
    {                                                                                                        \
        auto kern = interact_bwd_fma_kernel<27, VV>;                                                         \
        cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);                  \
        (void)launch_pdl(kern, dim3(grid), dim3(BW * 32), (size_t)(smem), st, tables, tm, B, offsets, indices, nnz, x_dense.hi, x_dense.lo,      \
                                          x_dense.ld, dconcat, ldc, dx_hi, dx_lo, lddx, dE, wb, err);        \
    }
    if (d == 128) DLRM_BWD(4) else DLRM_BWD(2)
#undef DLRM_BWD
    DLRM_LAUNCH_CHECK();
    return DLRM_OK;
}

cudaError_t set_wait_polls_interact_tc(long long polls) {
    return ac::set_rows_wait_tries_here(polls < 0 ? -1 : (int)(polls < ac::WAIT_TRIES ? polls : ac::WAIT_TRIES));
}

}  // namespace dlrm
