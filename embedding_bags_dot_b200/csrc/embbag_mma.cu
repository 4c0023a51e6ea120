// Fused gather + interaction for bf16 or row-wise uint8 tables on the tensor cores.
//
// Same operation as embbag.cu's fused kernel: per sample b, pool the K bags
// into e_1..e_K ("DLRM", briansu.co, section 3), form X = [x_dense; e_1..e_K]
// and write [x_dense, Z_10, Z_20, Z_21, ...] with Z_ij = <X_i, X_j>, j < i
// ("DLRM", briansu.co, section 4, equations "Interaction" and "Output").
//
// Block prologue: one warp per table, one lane per sample of the 32-sample
// tile; each lane reads its bag's two CSR offsets and resolves the bag to a
// code: the global row of a one-row bag, "empty" (no rows, bad offsets or an
// out-of-range index) or "several rows". Then one warp owns one sample at a
// time:
//  1. gather: lane k issues ONE bulk copy (cp.async.bulk, completing on the
//     warp's mbarrier) for the whole row of a one-row bag k, straight into row
//     1+k of the sample's tile. Tile rows are unswizzled and padded by one
//     16-byte chunk, so the 8 rows an ldmatrix reads land in 8 distinct bank
//     groups. Empty bags are zeroed and bags of several rows are summed in
//     fp32 by lane groups while the copies are in flight.
//  2. bf16 tables: x_dense (fp32) is split into hi = bf16(x) and
//     lo = bf16(x - hi); hi is row 0 and lo row K+1, so that
//     Z_i0 = G[i][0] + G[K+1][i] keeps the dense vector's fp32 precision.
//  3. Gram G = X X^T over the 16*MT padded rows with mma.sync.m16n8k16 (bf16
//     in, fp32 accumulate), lower-triangle tiles only. The same ldmatrix
//     fragments serve as A and as B (B = X^T), so X is read from shared memory
//     once per sample. Rows past the sample's last one are never written: they
//     only reach Gram entries that nothing reads.
//  4. G is staged in shared memory, the x_dense low-half terms are folded into
//     column 0, and each lane writes fixed 8-column chunks of the concat row
//     whose sources in G are computed once per block.
//  5. Row-wise uint8 tables, samples whose bags hold at most one row (and
//     whose x_dense is finite): the codes are never converted. Each record
//     (d codes, fp32 scale s, fp32 offset m) is copied whole into row 1+k of
//     an 8-bit tile whose row stride is the record size; row 0 is all ones;
//     x_dense is quantised per sample to 24 bits, x ~ sx qx + mn with
//     qx = 65536 h + 256 u + l, and its three byte planes are rows K+1..K+3.
//     One u8 x u8 -> s32 Gram (mma.sync m16n8k32) then holds, exactly, every
//     <q_i, q_j>, the code sums S_i = <q_i, 1> and the plane products. With
//     e_i = s_i q_i + m_i,
//       Z_ij = s_i s_j <q_i, q_j> + s_i S_i m_j + s_j S_j m_i + d m_i m_j,
//     and the same with (sx, mn, <q_i, qx>, sum qx) for the x_dense column;
//     the affine terms are applied in fp32 while the concat row is written.
//     Other uint8 samples take steps 1-4 with each one-row record copied into
//     its bf16 row slot and dequantised there (s q + m, rounded to bf16).
#include <algorithm>

#include "async_copy.cuh"
#include "common.cuh"
#include "kernels.cuh"

namespace dlrm {

namespace {

using namespace ac;

constexpr int WARPS = 8;
constexpr int SPW = 4;               // samples per warp per block
constexpr int S = WARPS * SPW;       // samples per block: one lane each in the prologue
static_assert(S == 32, "the prologue maps the block's samples to the lanes of a warp");
constexpr uint32_t CODE_EMPTY = 0xFFFFFFFFu;
constexpr uint32_t CODE_MULTI = 0xFFFFFFFEu;
constexpr int SRC_CACHE = 1;         // concat chunks per lane whose sources stay in registers
constexpr unsigned FULL = 0xffffffffu;

__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
    __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t*>(&h);
}

__device__ __forceinline__ void mma_bf16(float (&c)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%0,%1,%2,%3};"
        : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

__device__ __forceinline__ void mma_u8(int (&c)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k32.row.col.s32.u8.u8.s32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%0,%1,%2,%3};"
        : "+r"(c[0]), "+r"(c[1]), "+r"(c[2]), "+r"(c[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// Source of concat column c (c >= d) in the staged Gram G (row stride GS):
// i*GS + j for Z_ij, or `zero` (a slot holding 0) for a padding column.
__device__ __forceinline__ uint32_t column_source(int c, int d, int P, int GS, uint32_t zero) {
    const int p = c - d;
    if (p < 0 || p >= P) return zero;
    int i = (int)((1.0f + sqrtf(8.0f * (float)p + 1.0f)) * 0.5f);
    while (i * (i - 1) / 2 > p) --i;
    while ((i + 1) * i / 2 <= p) ++i;
    return (uint32_t)(i * GS + (p - i * (i - 1) / 2));
}

// Dequantise 8 codes of a DLRM_U8ROW record: v = s q + m.
__device__ __forceinline__ void dequant8(uint2 codes, float sc, float of, float (&v)[8]) {
#pragma unroll
    for (int e = 0; e < 4; ++e) {
        v[e] = fmaf(sc, (float)((codes.x >> (8 * e)) & 0xFFu), of);
        v[4 + e] = fmaf(sc, (float)((codes.y >> (8 * e)) & 0xFFu), of);
    }
}

// Byte offset of the integer route's (s, m, u, 0) slots: after the 8-bit tile and the staged Gram.
__host__ __device__ constexpr int u8_meta_offset(int K, int KP, int qrb) {
    return (std::max((K + 4) * qrb, (KP * (KP + 8) + 1) * 4) + 15) / 16 * 16;
}

// The bag masks of one sample: bit k set for bag k.
struct BagMasks {
    unsigned long long one, multi, empty;
};

// One sample on the integer route (every bag holds at most one row, x_dense finite with minimum mn and
// range max - mn). The records' bulk copies into rows 1..K (stride QRB) are already issued on `bar`.
// Writes the whole concat row.
template <int MT, int GL>
__device__ __forceinline__ void u8_sample(unsigned char* xw, uint32_t xw_s, int K, const BagMasks& bm,
                                          uint32_t bar, uint32_t parity, int tries, bool& timed_out, const float4* xv,
                                          float mn, float range, const uint32_t (&srcr)[SRC_CACHE][4],
                                          const uint16_t* src_s, int nzc, const float* __restrict__ xrow,
                                          void* out, size_t row0, int ld, int out_dt, int lane) {
    constexpr int d = 8 * GL;
    constexpr int KP = 16 * MT;
    constexpr int GS = KP + 8;
    constexpr int QRB = (d + 8 + 15) / 16 * 16;   // record bytes = 8-bit tile row stride
    constexpr int CHQ = QRB / 16;                 // 16-byte chunks of a record
    constexpr int NGQ = 32 / CHQ;                 // records zeroed per round
    constexpr int NTILE = MT * (MT + 1);
    constexpr uint32_t ZERO_SLOT = KP * GS;
    float* G = reinterpret_cast<float*>(xw);
    float4* meta = reinterpret_cast<float4*>(xw + u8_meta_offset(K, KP, QRB));
    const int P0 = K + 1;                         // x_dense byte planes: P0 (weight 1), P0+1 (256), P0+2 (65536)

    // empty bags: codes and (s, m) all zero
    {
        const int gq = lane / CHQ, cq = lane % CHQ;
        for (unsigned long long rest = bm.empty; rest; rest = drop_bits(rest, NGQ)) {
            const int k = gq < NGQ ? nth_bit(rest, gq) : -1;
            if (k >= 0) *reinterpret_cast<uint4*>(xw + (k + 1) * QRB + 16 * cq) = make_uint4(0, 0, 0, 0);
        }
    }
    // row 0: ones
    if (lane < d / 16)
        *reinterpret_cast<uint4*>(xw + 16 * lane) = make_uint4(0x01010101u, 0x01010101u, 0x01010101u, 0x01010101u);
    // x_dense -> 24-bit codes qx = rint((x - mn) / sx), sx = range / (2^24 - 1), as three byte planes
    constexpr float QMAX = 16777215.f;
    const float inv = range > 0.f ? QMAX / range : 0.f;
    const float sx = range / QMAX;
#pragma unroll
    for (int q = 0; q < (d + 127) / 128; ++q) {
        const int c = 4 * lane + 128 * q;
        if (c < d) {
            const float4 x = xv[q];
            uint32_t qv[4];
            qv[0] = (uint32_t)fminf(rintf((x.x - mn) * inv), QMAX);
            qv[1] = (uint32_t)fminf(rintf((x.y - mn) * inv), QMAX);
            qv[2] = (uint32_t)fminf(rintf((x.z - mn) * inv), QMAX);
            qv[3] = (uint32_t)fminf(rintf((x.w - mn) * inv), QMAX);
            const uint32_t lo01 = __byte_perm(qv[0], qv[1], 0x0040), lo23 = __byte_perm(qv[2], qv[3], 0x0040);
            const uint32_t mi01 = __byte_perm(qv[0], qv[1], 0x0051), mi23 = __byte_perm(qv[2], qv[3], 0x0051);
            const uint32_t hi01 = __byte_perm(qv[0], qv[1], 0x0062), hi23 = __byte_perm(qv[2], qv[3], 0x0062);
            *reinterpret_cast<uint32_t*>(xw + P0 * QRB + c) = __byte_perm(lo01, lo23, 0x5410);
            *reinterpret_cast<uint32_t*>(xw + (P0 + 1) * QRB + c) = __byte_perm(mi01, mi23, 0x5410);
            *reinterpret_cast<uint32_t*>(xw + (P0 + 2) * QRB + c) = __byte_perm(hi01, hi23, 0x5410);
        }
    }
    if (!rows_ready(bar, parity, tries)) {   // rows landed (drained); the caller stops after this sample
        timed_out = true;
        return;
    }
    __syncwarp();

    // exact integer Gram of the lower-triangle tiles
    int acc[NTILE][4];
#pragma unroll
    for (int t = 0; t < NTILE; ++t) acc[t][0] = acc[t][1] = acc[t][2] = acc[t][3] = 0;
#pragma unroll
    for (int ks = 0; ks < d / 32; ++ks) {
        uint32_t a[MT][4];
#pragma unroll
        for (int mt = 0; mt < MT; ++mt)
            ldmatrix_x4(xw_s + (uint32_t)((16 * mt + (lane & 15)) * QRB + 16 * (2 * ks + (lane >> 4))), a[mt]);
        int t = 0;
#pragma unroll
        for (int mt = 0; mt < MT; ++mt) {
#pragma unroll
            for (int nt = 0; nt <= 2 * mt + 1; ++nt, ++t)
                mma_u8(acc[t], a[mt], a[nt >> 1][(nt & 1) ? 1 : 0], a[nt >> 1][(nt & 1) ? 3 : 2]);
        }
    }
    // each bag's (s, m) from its record, before G overwrites the tile
    float2 sm[(KP + 31) / 32];
#pragma unroll
    for (int w = 0; w < (KP + 31) / 32; ++w) {
        const int k = lane + 32 * w;
        sm[w] = k < K ? *reinterpret_cast<const float2*>(xw + (k + 1) * QRB + d) : make_float2(0.f, 0.f);
    }
    __syncwarp();  // every lane's reads of the tile are done before G overwrites it

    // stage G in fp32 (every entry is below 2^24, so exact)
    {
        const int gr = lane >> 2, tc = (lane & 3) * 2;
        int t = 0;
#pragma unroll
        for (int mt = 0; mt < MT; ++mt) {
#pragma unroll
            for (int nt = 0; nt <= 2 * mt + 1; ++nt, ++t) {
                float* p0 = G + (16 * mt + gr) * GS + 8 * nt + tc;
                *reinterpret_cast<float2*>(p0) = make_float2((float)acc[t][0], (float)acc[t][1]);
                *reinterpret_cast<float2*>(p0 + 8 * GS) = make_float2((float)acc[t][2], (float)acc[t][3]);
            }
        }
        if (lane == 0) G[ZERO_SLOT] = 0.f;
    }
    __syncwarp();
    // per bag: slot (s, m, u = s S + (d/2) m); column 0 of its Gram row becomes <q_i, qx>
    const float* Gx0 = G + P0 * GS;
#pragma unroll
    for (int w = 0; w < (KP + 31) / 32; ++w) {
        const int i = lane + 32 * w + 1;
        if (i <= K) {
            const float S_i = G[i * GS];
            G[i * GS] = fmaf(65536.f, Gx0[2 * GS + i], fmaf(256.f, Gx0[GS + i], Gx0[i]));
            meta[i] = make_float4(sm[w].x, sm[w].y, fmaf(0.5f * (float)d, sm[w].y, sm[w].x * S_i), 0.f);
        }
    }
    if (lane == 0) {
        const float Sx = fmaf(65536.f, Gx0[2 * GS], fmaf(256.f, Gx0[GS], Gx0[0]));
        meta[0] = make_float4(sx, mn, fmaf(0.5f * (float)d, mn, sx * Sx), 0.f);
    }
    if (lane == 1) meta[KP] = make_float4(0.f, 0.f, 0.f, 0.f);
    __syncwarp();

    // Z for the Gram entry at `src`: s_i s_j g + t_i m_j + t_j m_i + d m_i m_j (t = s S), written as
    // s_i s_j g + u_i m_j + u_j m_i with u = t + (d/2) m
    auto zval = [&](uint32_t src) {
        const int i = (int)(src / GS), j = (int)(src - (uint32_t)i * GS);
        const float4 a = meta[i], c = meta[j];
        return fmaf(a.x * c.x, G[src], fmaf(a.z, c.y, c.z * a.y));
    };
    if (out_dt == DLRM_BF16) {
        __nv_bfloat16* orow = static_cast<__nv_bfloat16*>(out) + row0;
        uint4* zrow = reinterpret_cast<uint4*>(orow) + d / 8;
#pragma unroll
        for (int q = 0; q < (d + 127) / 128; ++q) {
            const int c = 4 * lane + 128 * q;
            if (c < d) {
                const float4 x = xv[q];
                reinterpret_cast<uint2*>(orow)[c / 4] = make_uint2(pack_bf16(x.x, x.y), pack_bf16(x.z, x.w));
            }
        }
#pragma unroll
        for (int j = 0; j < SRC_CACHE; ++j) {
            const int c8 = lane + 32 * j;
            if (c8 < nzc) {
                float f[8];
#pragma unroll
                for (int e = 0; e < 8; ++e) f[e] = zval((srcr[j][e >> 1] >> (16 * (e & 1))) & 0xFFFFu);
                zrow[c8] = make_uint4(pack_bf16(f[0], f[1]), pack_bf16(f[2], f[3]), pack_bf16(f[4], f[5]),
                                      pack_bf16(f[6], f[7]));
            }
        }
        for (int c8 = lane + 32 * SRC_CACHE; c8 < nzc; c8 += 32) {
            float f[8];
#pragma unroll
            for (int e = 0; e < 8; ++e) f[e] = zval(src_s[8 * c8 + e]);
            zrow[c8] = make_uint4(pack_bf16(f[0], f[1]), pack_bf16(f[2], f[3]), pack_bf16(f[4], f[5]),
                                  pack_bf16(f[6], f[7]));
        }
    } else {
        for (int c = lane; c < ld; c += 32) store_as(out, row0 + c, c < d ? xrow[c] : zval(src_s[c - d]), out_dt);
    }
}

}  // namespace

// MT: m-tiles of 16 rows (16 MT >= K + 2; K + 4 with Q). GL: lanes per row (d = 8 GL).
// Q: row-wise uint8 tables.
template <int MT, int GL, bool Q>
__global__ void __launch_bounds__(WARPS * 32, MT >= 3 ? 2 : 3) embbag_interact_mma_kernel(
    const void* __restrict__ tables_v, const __grid_constant__ TableMeta tm, int K, int B,
    const int32_t* __restrict__ offsets, const int32_t* __restrict__ indices, long long nnz,
    const float* __restrict__ x_dense, void* out, int ld, int out_dt, int warp_bytes, ErrRecord* err) {
    pdl_wait();   // programmatic dependent: the previous kernel's outputs are visible from here on
    constexpr int d = 8 * GL;
    constexpr int KP = 16 * MT;
    constexpr int RS = 2 * d + 16;   // bf16 tile row: 2d bytes plus one pad chunk (conflict-free ldmatrix)
    constexpr int GS = KP + 8;       // G row stride in floats (float2 staging without bank conflicts)
    constexpr int NG = 32 / GL;      // row groups per warp
    constexpr int NTILE = MT * (MT + 1);
    constexpr int QRB = (d + 8 + 15) / 16 * 16;   // uint8 record bytes
    constexpr int ROWB = Q ? QRB : 2 * d;         // bytes of one table row in global memory
    constexpr bool TWO = KP > 32;                 // K may exceed 32: two bags per lane
    const __nv_bfloat16* __restrict__ tables = static_cast<const __nv_bfloat16*>(tables_v);
    const unsigned char* __restrict__ qtab = static_cast<const unsigned char*>(tables_v);
    extern __shared__ __align__(16) unsigned char smem[];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int P = K * (K + 1) / 2;
    const int L = K + 1;             // row holding the low half of x_dense
    const int KS = K | 1;            // code_s row stride (odd: the prologue's writes are conflict-free)
    unsigned char* xw = smem + (size_t)warp * warp_bytes;
    unsigned char* tail = smem + (size_t)WARPS * warp_bytes;
    uint32_t* code_s = reinterpret_cast<uint32_t*>(tail);                       // [S][KS]
    uint16_t* src_s = reinterpret_cast<uint16_t*>(code_s + S * KS);             // sources of columns d .. ld-1
    const int bar_off = (S * KS * 4 + (ld - d + 8) * 2 + 7) & ~7;
    const uint32_t bar = (uint32_t)__cvta_generic_to_shared(tail + bar_off) + 8u * (uint32_t)warp;
    const int nzc = (ld - d) / 8;                                               // 8-column chunks after x_dense
    constexpr uint32_t ZERO_SLOT = KP * GS;
    const bool bf16_out = out_dt == DLRM_BF16;

    const int b0 = blockIdx.x * S;
    const int nb = min(S, B - b0);
    unsigned oob = 0, bad = 0;

    // ---- block prologue: bag codes (warp per table, lane per sample), concat column sources, barriers
    for (int k = warp; k < K; k += WARPS) {
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
    for (int c = d + threadIdx.x; c < ld; c += blockDim.x) src_s[c - d] = (uint16_t)column_source(c, d, P, GS, ZERO_SLOT);
    if (lane == 0) {
        bar_init(bar);
        fence_proxy_async();
    }
    __syncthreads();

    // per-lane sources of its Z chunks (two 16-bit sources per register), fixed for the whole block
    uint32_t srcr[SRC_CACHE][4];
#pragma unroll
    for (int j = 0; j < SRC_CACHE; ++j)
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            const int c = 8 * (lane + 32 * j) + 2 * e;
            const uint32_t lo = c < ld - d ? src_s[c] : ZERO_SLOT, hi = c + 1 < ld - d ? src_s[c + 1] : ZERO_SLOT;
            srcr[j][e] = lo | (hi << 16);
        }

    const uint32_t xw_s = (uint32_t)__cvta_generic_to_shared(xw);
    float* G = reinterpret_cast<float*>(xw + RS);
    const int gi = lane / GL, g = lane % GL;
    uint32_t parity = 0;
    bool timed_out = false;
    const int first_tries = g_rows_wait_tries;

    for (int r = 0; r < SPW; ++r) {
        const int s = warp * SPW + r;
        if (s >= nb) break;
        const long long b = b0 + s;

        // x_dense in flight alongside the rows
        float4 xv[(d + 127) / 128];
#pragma unroll
        for (int q = 0; q < (d + 127) / 128; ++q) {
            const int c = 4 * lane + 128 * q;
            xv[q] = c < d ? *reinterpret_cast<const float4*>(x_dense + b * d + c) : make_float4(0.f, 0.f, 0.f, 0.f);
        }

        // this sample's bags: lane k holds bag k (and k + 32)
        const uint32_t* cs = code_s + s * KS;
        const uint32_t c0 = lane < K ? cs[lane] : CODE_EMPTY;
        const uint32_t c1 = TWO && lane + 32 < K ? cs[lane + 32] : CODE_EMPTY;
        BagMasks bm;
        bm.one = __ballot_sync(FULL, c0 < CODE_MULTI);
        bm.multi = __ballot_sync(FULL, c0 == CODE_MULTI);
        bm.empty = __ballot_sync(FULL, lane < K && c0 == CODE_EMPTY);
        if (TWO) {
            bm.one |= (unsigned long long)__ballot_sync(FULL, c1 < CODE_MULTI) << 32;
            bm.multi |= (unsigned long long)__ballot_sync(FULL, c1 == CODE_MULTI) << 32;
            bm.empty |= (unsigned long long)__ballot_sync(FULL, lane + 32 < K && c1 == CODE_EMPTY) << 32;
        }

        // uint8 tables: the integer route unless a bag holds several rows or x_dense is not finite
        bool int_route = false;
        float mn = 0.f, range = 0.f;
        if constexpr (Q) {
            float mx = -INFINITY;
            mn = INFINITY;
            bool nonfinite = false;
#pragma unroll
            for (int q = 0; q < (d + 127) / 128; ++q) {
                if (4 * lane + 128 * q < d) {
                    const float4 x = xv[q];
                    mn = fminf(fminf(mn, x.x), fminf(x.y, fminf(x.z, x.w)));
                    mx = fmaxf(fmaxf(mx, x.x), fmaxf(x.y, fmaxf(x.z, x.w)));
                    nonfinite |= !(isfinite(x.x) && isfinite(x.y) && isfinite(x.z) && isfinite(x.w));
                }
            }
            // warp-wide min and max (a non-finite x_dense sends the sample to the dequantising route
            // whatever these return)
            asm volatile("redux.sync.min.f32 %0, %0, 0xffffffff;" : "+f"(mn));
            asm volatile("redux.sync.max.f32 %0, %0, 0xffffffff;" : "+f"(mx));
            range = mx - mn;
            int_route = bm.multi == 0 && !__any_sync(FULL, nonfinite) && isfinite(range);
        }

        // ---- 1. one bulk copy per one-row bag (after the previous sample's accesses to the region)
        fence_proxy_async();
        __syncwarp();
        if (lane == 0) bar_expect(bar, (uint32_t)__popcll(bm.one) * ROWB);
        __syncwarp();
        {
            const int stride = Q && int_route ? QRB : RS;
            if (c0 < CODE_MULTI)
                bulk_row(xw_s + (uint32_t)((lane + 1) * stride),
                         Q ? (const void*)(qtab + (long long)c0 * QRB) : (const void*)(tables + (long long)c0 * d),
                         ROWB, bar);
            if (TWO && c1 < CODE_MULTI)
                bulk_row(xw_s + (uint32_t)((lane + 33) * stride),
                         Q ? (const void*)(qtab + (long long)c1 * QRB) : (const void*)(tables + (long long)c1 * d),
                         ROWB, bar);
        }
        if constexpr (Q) {
            if (int_route) {
                u8_sample<MT, GL>(xw, xw_s, K, bm, bar, parity, first_tries, timed_out, xv, mn, range, srcr, src_s,
                                  nzc, x_dense + b * d, out, (size_t)b * ld, ld, out_dt, lane);
                parity ^= 1u;
                __syncwarp();  // the region is reused by the next sample
                if (timed_out) break;
                continue;
            }
        }

        // empty bags -> zero rows; bags of several rows -> fp32 sums rounded to bf16 (NG bags at a time)
        for (unsigned long long rest = bm.empty | bm.multi; rest; rest = drop_bits(rest, NG)) {
            const int k = nth_bit(rest, gi);
            if (k < 0) continue;
            uint4 w = make_uint4(0, 0, 0, 0);
            if ((bm.multi >> k) & 1ull) {
                const int st = offsets[(long long)k * B + b], en = offsets[(long long)k * B + b + 1];
                float a[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
                for (int p = st; p < en; ++p) {
                    const int idx = __ldg(indices + p);
                    if (idx >= 0 && (long long)idx < tm.rows[k]) {
                        if constexpr (Q) {
                            const unsigned char* rec = qtab + (tm.base[k] + idx) * (long long)QRB;
                            const uint2 cq = __ldg(reinterpret_cast<const uint2*>(rec + 8 * g));
                            const float2 so = __ldg(reinterpret_cast<const float2*>(rec + d));
                            float v[8];
                            dequant8(cq, so.x, so.y, v);
#pragma unroll
                            for (int e = 0; e < 8; ++e) a[e] += v[e];
                        } else {
                            Chunk16<__nv_bfloat16>::add(ldg16_stream(tables + (tm.base[k] + idx) * (long long)d + 8 * g),
                                                        a);
                        }
                    } else if (g == 0) {
                        ++oob;
                    }
                }
                w = make_uint4(pack_bf16(a[0], a[1]), pack_bf16(a[2], a[3]), pack_bf16(a[4], a[5]), pack_bf16(a[6], a[7]));
            }
            *reinterpret_cast<uint4*>(xw + (k + 1) * RS + 16 * g) = w;
        }

        // ---- 2. x_dense -> rows 0 (hi) and K+1 (lo)
#pragma unroll
        for (int q = 0; q < (d + 127) / 128; ++q) {
            const int c = 4 * lane + 128 * q;
            if (c < d) {
                const float4 x = xv[q];
                const __nv_bfloat162 h01 = __floats2bfloat162_rn(x.x, x.y), h23 = __floats2bfloat162_rn(x.z, x.w);
                const float2 f01 = __bfloat1622float2(h01), f23 = __bfloat1622float2(h23);
                *reinterpret_cast<uint2*>(xw + 2 * c) =
                    make_uint2(*reinterpret_cast<const uint32_t*>(&h01), *reinterpret_cast<const uint32_t*>(&h23));
                *reinterpret_cast<uint2*>(xw + L * RS + 2 * c) =
                    make_uint2(pack_bf16(x.x - f01.x, x.y - f01.y), pack_bf16(x.z - f23.x, x.w - f23.y));
            }
        }
        if (!rows_ready(bar, parity, first_tries)) {   // rows landed (drained): stop this warp's samples
            timed_out = true;
            break;
        }
        parity ^= 1u;
        __syncwarp();
        if constexpr (Q) {
            // one-row bags: records -> dequantised bf16 rows, in place (every lane reads before any writes)
            for (unsigned long long rest = bm.one; rest; rest = drop_bits(rest, NG)) {
                const int k = nth_bit(rest, gi);
                uint4 w = make_uint4(0, 0, 0, 0);
                if (k >= 0) {
                    const unsigned char* rec = xw + (k + 1) * RS;
                    const uint2 cq = *reinterpret_cast<const uint2*>(rec + 8 * g);
                    const float2 so = *reinterpret_cast<const float2*>(rec + d);
                    float v[8];
                    dequant8(cq, so.x, so.y, v);
                    w = make_uint4(pack_bf16(v[0], v[1]), pack_bf16(v[2], v[3]), pack_bf16(v[4], v[5]),
                                   pack_bf16(v[6], v[7]));
                }
                __syncwarp();
                if (k >= 0) *reinterpret_cast<uint4*>(xw + (k + 1) * RS + 16 * g) = w;
            }
            __syncwarp();
        }

        // ---- 3. lower-triangle Gram tiles on the tensor cores
        float acc[NTILE][4];
#pragma unroll
        for (int t = 0; t < NTILE; ++t) acc[t][0] = acc[t][1] = acc[t][2] = acc[t][3] = 0.f;
#pragma unroll
        for (int ks = 0; ks < d / 16; ++ks) {
            uint32_t a[MT][4];
#pragma unroll
            for (int mt = 0; mt < MT; ++mt)
                ldmatrix_x4(xw_s + (uint32_t)((16 * mt + (lane & 15)) * RS + 16 * (2 * ks + (lane >> 4))), a[mt]);
            int t = 0;
#pragma unroll
            for (int mt = 0; mt < MT; ++mt) {
#pragma unroll
                for (int nt = 0; nt <= 2 * mt + 1; ++nt, ++t) {
                    const uint32_t b0r = a[nt >> 1][(nt & 1) ? 1 : 0];
                    const uint32_t b1r = a[nt >> 1][(nt & 1) ? 3 : 2];
                    mma_bf16(acc[t], a[mt], b0r, b1r);
                }
            }
        }
        __syncwarp();  // every lane's ldmatrix of X is done before G overwrites it

        // ---- 4. stage G (row stride GS floats, after X row 0, which keeps bf16(x_dense))
        {
            const int gr = lane >> 2, tc = (lane & 3) * 2;
            int t = 0;
#pragma unroll
            for (int mt = 0; mt < MT; ++mt) {
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
        // Z_i0 = <e_i, x_hi> + <e_i, x_lo>: fold the low half (row L) into column 0
        for (int i = 1 + lane; i <= K; i += 32) G[i * GS] += G[L * GS + i];
        __syncwarp();

        // ---- 5. concat row: x_dense, Z, zero padding
        if (bf16_out) {
            uint4* orow = reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(out) + b * ld);
            for (int c8 = lane; c8 < d / 8; c8 += 32) orow[c8] = *reinterpret_cast<const uint4*>(xw + 16 * c8);
            uint4* zrow = orow + d / 8;
#pragma unroll
            for (int j = 0; j < SRC_CACHE; ++j) {
                const int c8 = lane + 32 * j;
                if (c8 < nzc) {
                    float f[8];
#pragma unroll
                    for (int e = 0; e < 8; ++e) f[e] = G[(srcr[j][e >> 1] >> (16 * (e & 1))) & 0xFFFFu];
                    zrow[c8] = make_uint4(pack_bf16(f[0], f[1]), pack_bf16(f[2], f[3]), pack_bf16(f[4], f[5]),
                                          pack_bf16(f[6], f[7]));
                }
            }
            for (int c8 = lane + 32 * SRC_CACHE; c8 < nzc; c8 += 32) {
                float f[8];
#pragma unroll
                for (int e = 0; e < 8; ++e) f[e] = G[src_s[8 * c8 + e]];
                zrow[c8] = make_uint4(pack_bf16(f[0], f[1]), pack_bf16(f[2], f[3]), pack_bf16(f[4], f[5]),
                                      pack_bf16(f[6], f[7]));
            }
        } else {
            for (int c = lane; c < ld; c += 32) {
                const float val = c < d ? x_dense[b * d + c] : G[src_s[c - d]];
                store_as(out, (size_t)b * ld + c, val, out_dt);
            }
        }
        __syncwarp();  // X / G reused by the next sample
    }
    if (timed_out && lane == 0) atomicOr(&err->flags, ERR_TIMEOUT);
    report_warp(err, oob, bad);
}

// ------------------------------------------------------------------ host side

// Bytes of a warp's region. bf16 tile: rows 0..K+1 of 2d+16 bytes, or row 0 plus the staged Gram; uint8
// tables add the integer route's tile (rows 0..K+3 of one record each) or Gram, then its (s, m, u) slots.
static int mma_warp_bytes(int K, int d, bool q, int& MT) {
    MT = (K + (q ? 4 : 2) + 15) / 16;
    const int KP = 16 * MT;
    const int RS = 2 * d + 16;
    const int gf = (KP * (KP + 8) + 1) * 4;
    int bytes = std::max((K + 2) * RS, RS + gf);
    if (q) {
        const int qrb = (d + 8 + 15) / 16 * 16;
        bytes = std::max(bytes, u8_meta_offset(K, KP, qrb) + (KP + 1) * 16);
    }
    return (bytes + 15) & ~15;
}

// Rows past a sample's last one are read by ldmatrix but never written; the last warp's may reach past
// its region and the tail, so the allocation ends with enough slack to keep those reads inside it.
static size_t mma_smem(int K, int d, bool q, int ld, int& MT, int& warp_bytes) {
    warp_bytes = mma_warp_bytes(K, d, q, MT);
    const int KP = 16 * MT;
    const size_t tail = (((size_t)S * (K | 1) * 4 + (size_t)(ld - d + 8) * 2 + 7) & ~(size_t)7) + 8 * WARPS;
    const size_t reach = (size_t)KP * std::max(2 * d + 16, q ? (d + 8 + 15) / 16 * 16 : 0);
    const size_t slack = reach > (size_t)warp_bytes + tail ? reach - warp_bytes - tail : 0;
    return (size_t)WARPS * warp_bytes + tail + ((slack + 15) & ~(size_t)15);
}

bool embbag_interact_mma_supported(dlrm_dtype dt, int K, int d, int ld, const void* out, dlrm_dtype out_dt,
                                   long long total_rows) {
    if (dt != DLRM_BF16 && dt != DLRM_U8ROW) return false;
    if (!(d == 32 || d == 64 || d == 128 || d == 256)) return false;
    if (dt == DLRM_U8ROW && !(d == 64 || d == 128)) return false;
    if (K + (dt == DLRM_U8ROW ? 4 : 2) > 64) return false;
    if (total_rows >= (long long)CODE_MULTI) return false;
    if (out_dt == DLRM_BF16 && (ld % 8 || ((uintptr_t)out & 15))) return false;
    if (ld - d > 8 * 0x1FFF) return false;
    const int P = K * (K + 1) / 2;
    if (P + d > ld || ld > 0x7FFF) return false;
    int MT, wb;
    return mma_smem(K, d, dt == DLRM_U8ROW, ld, MT, wb) <= 227 * 1024;
}

template <int MT, int GL, bool Q>
static void launch_mma_t(const TableMeta& tm, const void* tables, int K, int B, const int32_t* offsets,
                         const int32_t* indices, long long nnz, const float* x_dense, void* out, int ld, int out_dt,
                         int warp_bytes, size_t smem, ErrRecord* err, cudaStream_t st) {
    auto kern = embbag_interact_mma_kernel<MT, GL, Q>;
    cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    (void)launch_pdl(kern, dim3((B + S - 1) / S), dim3(WARPS * 32), smem, st, tables, tm, K, B, offsets, indices, nnz,
                     x_dense, out, ld, out_dt, warp_bytes, err);
}

dlrm_status launch_embbag_interact_mma(const TableMeta& tm, const void* tables, dlrm_dtype dt, int K, int d, int B,
                                       const int32_t* offsets, const int32_t* indices, long long nnz,
                                       const float* x_dense, void* out, int ld, dlrm_dtype out_dt, ErrRecord* err,
                                       cudaStream_t st) {
    int MT, wb;
    const bool q = dt == DLRM_U8ROW;
    const size_t smem = mma_smem(K, d, q, ld, MT, wb);
#define DLRM_MMA_GL(MTV)                                                                                       \
    switch (d) {                                                                                               \
        case 32: launch_mma_t<MTV, 4, false>(tm, tables, K, B, offsets, indices, nnz, x_dense, out, ld, out_dt, wb, smem, err, st); break;   \
        case 64:                                                                                               \
            if (q) launch_mma_t<MTV, 8, true>(tm, tables, K, B, offsets, indices, nnz, x_dense, out, ld, out_dt, wb, smem, err, st);  \
            else launch_mma_t<MTV, 8, false>(tm, tables, K, B, offsets, indices, nnz, x_dense, out, ld, out_dt, wb, smem, err, st); \
            break;                                                                                             \
        case 128:                                                                                              \
            if (q) launch_mma_t<MTV, 16, true>(tm, tables, K, B, offsets, indices, nnz, x_dense, out, ld, out_dt, wb, smem, err, st); \
            else launch_mma_t<MTV, 16, false>(tm, tables, K, B, offsets, indices, nnz, x_dense, out, ld, out_dt, wb, smem, err, st); \
            break;                                                                                             \
        default: launch_mma_t<MTV, 32, false>(tm, tables, K, B, offsets, indices, nnz, x_dense, out, ld, out_dt, wb, smem, err, st); break;  \
    }
    switch (MT) {
        case 1: DLRM_MMA_GL(1) break;
        case 2: DLRM_MMA_GL(2) break;
        case 3: DLRM_MMA_GL(3) break;
        default: DLRM_MMA_GL(4) break;
    }
#undef DLRM_MMA_GL
    DLRM_LAUNCH_CHECK();
    return DLRM_OK;
}

cudaError_t set_wait_polls_embbag_mma(long long polls) {
    return ac::set_rows_wait_tries_here(polls < 0 ? -1 : (int)(polls < ac::WAIT_TRIES ? polls : ac::WAIT_TRIES));
}

}  // namespace dlrm
