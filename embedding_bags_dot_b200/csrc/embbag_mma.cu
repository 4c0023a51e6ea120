// Fused gather + interaction for bf16 or row-wise uint8 tables on the tensor cores.
//
// Same operation as embbag.cu's fused kernel: per sample b, pool the K bags
// into e_1..e_K ("DLRM", briansu.co, section 3), form X = [x_dense; e_1..e_K]
// and write [x_dense, Z_10, Z_20, Z_21, ...] with Z_ij = <X_i, X_j>, j < i
// ("DLRM", briansu.co, section 4, equations "Interaction" and "Output").
//
// Block prologue (all threads): the tile's CSR offsets are read once,
// coalesced, and every bag is resolved to a code: the global row of a
// one-row bag, "empty" (no rows, bad offsets or an out-of-range index), or
// "several rows". Then one warp owns one sample at a time:
//  1. gather: lanes form groups of GL = d/8 lanes, one 16-byte chunk of a bf16
//     row per lane. A one-row bag is copied global -> shared with cp.async,
//     so every row of the sample is in flight at once without registers;
//     a bag of several rows is summed in fp32 and rounded to bf16.
//     Row-wise uint8 tables (Q), a sample with a bag of several rows (or a
//     non-finite x_dense): a one-row bag's record (d codes, fp32 scale s, fp32
//     offset m) is copied the same way, unswizzled, into the first bytes of
//     its X row slot; once it has landed each lane reads its 8 codes and the
//     scale/offset, the warp synchronises, and the lane writes the dequantised
//     values (s q + m, rounded to bf16) as its swizzled 16-byte chunk.
//     Every other uint8 sample takes the integer route (5. below).
//  2. x_dense (fp32) is split into hi = bf16(x) and lo = bf16(x - hi); hi is
//     row 0 of X and lo row K+1, so that Z_i0 = G[i][0] + G[K+1][i] keeps the
//     dense vector's fp32 precision.
//  3. Gram G = X X^T over the Kp = 16*MT padded rows with
//     mma.sync.m16n8k16 (bf16 in, fp32 accumulate), lower-triangle tiles only.
//     The same ldmatrix fragments serve as A and as B (B = X^T), so X is read
//     from shared memory once per sample.
//  4. G is staged in shared memory, the x_dense low-half terms are folded into
//     column 0, and each lane writes fixed 8-column chunks of the concat row
//     whose sources in G are computed once per block.
//  5. Row-wise uint8 tables, samples whose bags hold at most one row: the
//     codes are never converted. Each bag's d codes go by cp.async straight
//     into row 1+k of an 8-bit tile, its (s, m) into a per-row slot; row 0 is
//     all ones; x_dense is quantised per sample to 24 bits,
//     x ~ sx qx + mn with qx = 65536 h + 256 u + l, and its three byte planes
//     are rows K+1..K+3. One u8 x u8 -> s32 Gram on the tensor cores
//     (mma.sync m16n8k32) then holds, exactly, every <q_i, q_j>, the code sums
//     S_i = <q_i, 1> and the plane products. With e_i = s_i q_i + m_i,
//       Z_ij = s_i s_j <q_i, q_j> + s_i S_i m_j + s_j S_j m_i + d m_i m_j,
//     and the same with (sx, mn, <q_i, qx>, sum qx) for the x_dense column;
//     the affine terms are applied in fp32 while the concat row is written.
#include <algorithm>

#include "common.cuh"
#include "kernels.cuh"

namespace dlrm {

namespace {

constexpr int WARPS = 8;
constexpr int SPW = 4;               // samples per warp per block
constexpr int S = WARPS * SPW;       // samples per block
constexpr uint32_t CODE_EMPTY = 0xFFFFFFFFu;
constexpr uint32_t CODE_MULTI = 0xFFFFFFFEu;
constexpr int SRC_CACHE = 1;         // concat chunks per lane whose sources stay in registers

__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
    __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t*>(&h);
}

__device__ __forceinline__ void ldmatrix_x4(uint32_t addr, uint32_t (&r)[4]) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
                 : "r"(addr));
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

__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dst), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async_wait_all() {
    asm volatile("cp.async.commit_group;\ncp.async.wait_group 0;" ::: "memory");
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

}  // namespace

// Dequantise 8 codes of a DLRM_U8ROW record: v = s q + m.
__device__ __forceinline__ void dequant8(uint2 codes, float sc, float of, float (&v)[8]) {
#pragma unroll
    for (int e = 0; e < 4; ++e) {
        v[e] = fmaf(sc, (float)((codes.x >> (8 * e)) & 0xFFu), of);
        v[4 + e] = fmaf(sc, (float)((codes.y >> (8 * e)) & 0xFFu), of);
    }
}

// Layout of a warp's region on the integer route: KP+1 16-byte row slots
// (s, m, s S, 0) -- slot 0 for x_dense, slots 1..K for the bags, slot KP all
// zero for padding columns -- then the 8-bit tile X8 (KP rows of d bytes),
// which the staged Gram (fp32, row stride KP + 8) overwrites after the MMAs.

// One sample on the integer route: bags of at most one row, finite x_dense
// (minimum mn, range = max - mn). Writes the whole concat row.
template <int MT, int GL>
__device__ __forceinline__ void u8_sample(unsigned char* xw, uint32_t xw_s, const uint32_t* code_k, int K,
                                          const unsigned char* __restrict__ qtab, const float4* xv, float mn,
                                          float range, const uint32_t (&srcr)[SRC_CACHE][4], const uint16_t* src_s,
                                          int nzc, const float* __restrict__ xrow, void* out, size_t row0, int ld,
                                          int out_dt, int lane) {
    constexpr int d = 8 * GL;
    constexpr int KP = 16 * MT;
    constexpr int GS = KP + 8;
    constexpr int CH = d / 16;               // 16-byte chunks of an 8-bit row
    constexpr int NG8 = 32 / CH;             // rows per round of the gather
    constexpr int QRB = (d + 8 + 15) / 16 * 16;
    constexpr int NTILE = MT * (MT + 1);
    constexpr uint32_t ZERO_SLOT = KP * GS;
    constexpr int X8 = (KP + 1) * 16;     // start of the 8-bit tile
    // 128-byte rows: chunk c of row r at c ^ (r & 7); 64-byte rows: c ^ ((r >> 1) & 3). Either way the
    // 8 rows an ldmatrix reads fall in 8 distinct 16-byte bank groups.
    auto xoff8 = [](int r, int c) { return X8 + r * d + 16 * (d == 128 ? (c ^ (r & 7)) : (c ^ ((r >> 1) & 3))); };
    float4* meta = reinterpret_cast<float4*>(xw);
    float* G = reinterpret_cast<float*>(xw + X8);
    const int P0 = K + 1;                    // x_dense byte planes: P0 (weight 1), P0+1 (256), P0+2 (65536)

    // codes of the one-row bags, row 1+k; their (s, m) into slot 1+k; empty bags are all zero
    {
        const int gi = lane / CH, g = lane % CH;
        for (int k = gi; k < K; k += NG8) {
            const uint32_t code = code_k[k * S];
            if (code < CODE_MULTI)
                cp_async16(xw_s + (uint32_t)xoff8(k + 1, g), qtab + (long long)code * QRB + 16 * g);
            else
                *reinterpret_cast<uint4*>(xw + xoff8(k + 1, g)) = make_uint4(0, 0, 0, 0);
        }
        for (int k = lane; k < K; k += 32) {
            const uint32_t code = code_k[k * S];
            if (code < CODE_MULTI)
                cp_async16(xw_s + 16u * (uint32_t)(k + 1), qtab + (long long)code * QRB + d);
            else
                meta[k + 1] = make_float4(0.f, 0.f, 0.f, 0.f);
        }
    }
    // row 0: ones; rows K+4 .. KP-1: zero; slot KP: zero
    if (lane < CH) *reinterpret_cast<uint4*>(xw + xoff8(0, lane)) = make_uint4(0x01010101u, 0x01010101u, 0x01010101u, 0x01010101u);
    for (int q = lane; q < (KP - K - 4) * CH; q += 32)
        reinterpret_cast<uint4*>(xw + X8 + (K + 4) * d)[q] = make_uint4(0, 0, 0, 0);
    if (lane == 0) meta[KP] = make_float4(0.f, 0.f, 0.f, 0.f);
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
            const int ch = c / 16, byte = c % 16;
            *reinterpret_cast<uint32_t*>(xw + xoff8(P0, ch) + byte) = __byte_perm(lo01, lo23, 0x5410);
            *reinterpret_cast<uint32_t*>(xw + xoff8(P0 + 1, ch) + byte) = __byte_perm(mi01, mi23, 0x5410);
            *reinterpret_cast<uint32_t*>(xw + xoff8(P0 + 2, ch) + byte) = __byte_perm(hi01, hi23, 0x5410);
        }
    }
    cp_async_wait_all();
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
            ldmatrix_x4(xw_s + (uint32_t)xoff8(16 * mt + (lane & 15), 2 * ks + (lane >> 4)), a[mt]);
        int t = 0;
#pragma unroll
        for (int mt = 0; mt < MT; ++mt) {
#pragma unroll
            for (int nt = 0; nt <= 2 * mt + 1; ++nt, ++t)
                mma_u8(acc[t], a[mt], a[nt >> 1][(nt & 1) ? 1 : 0], a[nt >> 1][(nt & 1) ? 3 : 2]);
        }
    }
    __syncwarp();  // every lane's ldmatrix of X8 is done before G overwrites it

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
    // per bag: slot (s, m, s S); column 0 of its Gram row becomes <q_i, qx>
    const float* Gx0 = G + P0 * GS;
    for (int i = 1 + lane; i <= K; i += 32) {
        const float S_i = G[i * GS];
        G[i * GS] = fmaf(65536.f, Gx0[2 * GS + i], fmaf(256.f, Gx0[GS + i], Gx0[i]));
        const float4 sm = meta[i];
        meta[i] = make_float4(sm.x, sm.y, sm.x * S_i, 0.f);
    }
    if (lane == 0) {
        const float Sx = fmaf(65536.f, Gx0[2 * GS], fmaf(256.f, Gx0[GS], Gx0[0]));
        meta[0] = make_float4(sx, mn, sx * Sx, 0.f);
    }
    __syncwarp();

    // Z for the Gram entry at `src`: s_i s_j g + t_i m_j + t_j m_i + d m_i m_j
    auto zval = [&](uint32_t src) {
        const int i = (int)(src / GS), j = (int)(src - (uint32_t)i * GS);
        const float4 a = meta[i], c = meta[j];
        return fmaf(a.x * c.x, G[src], fmaf(a.z, c.y, fmaf(c.z, a.y, (float)d * a.y * c.y)));
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
    __syncwarp();  // the region is reused by the next sample
}

// MT: m-tiles of 16 rows (Kp = 16 MT >= K + 2; K + 4 with Q). GL: lanes per row (d = 8 GL).
// Q: row-wise uint8 tables.
template <int MT, int GL, bool Q>
__global__ void __launch_bounds__(WARPS * 32, MT >= 3 ? 2 : 3) embbag_interact_mma_kernel(
    const void* __restrict__ tables_v, const __grid_constant__ TableMeta tm, int K, int B,
    const int32_t* __restrict__ offsets, const int32_t* __restrict__ indices, long long nnz,
    const float* __restrict__ x_dense, void* out, int ld, int out_dt, int warp_bytes, ErrRecord* err) {
    constexpr int d = 8 * GL;
    constexpr int KP = 16 * MT;
    // X rows: d >= 64 uses 2d-byte rows whose 16-byte chunks are XOR-swizzled by (row & 7); d = 32
    // pads rows to an odd number of chunks. Either way ldmatrix reads 8 rows without bank conflicts.
    constexpr bool SWZ = d >= 64;
    constexpr int RS = SWZ ? 2 * d : 2 * d + 16;
    constexpr int GS = KP + 8;       // G row stride in floats (float2 staging without bank conflicts)
    constexpr int NG = 32 / GL;      // row groups per warp
    constexpr int NTILE = MT * (MT + 1);
    constexpr int QRB = (d + 8 + 15) / 16 * 16;   // uint8 record bytes
    const __nv_bfloat16* __restrict__ tables = static_cast<const __nv_bfloat16*>(tables_v);
    const unsigned char* __restrict__ qtab = static_cast<const unsigned char*>(tables_v);
    // byte offset of 16-byte chunk c of X row r
    auto xoff = [](int r, int c) { return r * RS + 16 * (SWZ ? (c ^ (r & 7)) : c); };
    extern __shared__ __align__(16) unsigned char smem[];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int P = K * (K + 1) / 2;
    const int L = K + 1;             // row holding the low half of x_dense
    unsigned char* xw = smem + (size_t)warp * warp_bytes;
    unsigned char* tail = smem + (size_t)WARPS * warp_bytes;
    int* off_s = reinterpret_cast<int*>(smem);   // prologue only: lives in the X regions until samples start
    uint32_t* code_s = reinterpret_cast<uint32_t*>(tail);
    uint16_t* src_s = reinterpret_cast<uint16_t*>(code_s + K * S);   // sources of columns d .. ld-1
    const int nzc = (ld - d) / 8;                                    // 8-column chunks after x_dense
    constexpr uint32_t ZERO_SLOT = KP * GS;
    const bool bf16_out = out_dt == DLRM_BF16;

    const int b0 = blockIdx.x * S;
    const int nb = min(S, B - b0);
    unsigned oob = 0, bad = 0;

    // ---- block prologue: tile offsets, bag codes, concat column sources
    for (int q = threadIdx.x; q < K * (nb + 1); q += blockDim.x) {
        const int k = q / (nb + 1), s = q - k * (nb + 1);
        off_s[k * (S + 1) + s] = offsets[(long long)k * B + b0 + s];
    }
    for (int c = d + threadIdx.x; c < ld; c += blockDim.x) src_s[c - d] = (uint16_t)column_source(c, d, P, GS, ZERO_SLOT);
    __syncthreads();
    for (int q = threadIdx.x; q < K * nb; q += blockDim.x) {
        const int k = q / nb, s = q - k * nb;
        const long long st = off_s[k * (S + 1) + s], en = off_s[k * (S + 1) + s + 1];
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
        code_s[k * S + s] = code;
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

        if constexpr (Q) {
            // ---- 5. integer route, unless a bag holds several rows or x_dense is not finite
            float mn = INFINITY, mx = -INFINITY;
            bool slow = false;
#pragma unroll
            for (int q = 0; q < (d + 127) / 128; ++q) {
                if (4 * lane + 128 * q < d) {
                    const float4 x = xv[q];
                    mn = fminf(fminf(mn, x.x), fminf(x.y, fminf(x.z, x.w)));
                    mx = fmaxf(fmaxf(mx, x.x), fmaxf(x.y, fmaxf(x.z, x.w)));
                    slow |= !(isfinite(x.x) && isfinite(x.y) && isfinite(x.z) && isfinite(x.w));
                }
            }
            for (int k = lane; k < K; k += 32) slow |= code_s[k * S + s] == CODE_MULTI;
#pragma unroll
            for (int o = 16; o >= 1; o >>= 1) {
                mn = fminf(mn, __shfl_xor_sync(0xffffffffu, mn, o));
                mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
            }
            const float range = mx - mn;
            if (!__any_sync(0xffffffffu, slow) && isfinite(range)) {
                u8_sample<MT, GL>(xw, xw_s, code_s + s, K, qtab, xv, mn, range, srcr, src_s, nzc, x_dense + b * d,
                                  out, (size_t)b * ld, ld, out_dt, lane);
                continue;
            }
        }

        // ---- 1. gather: X rows 1..K
        for (int k = gi; k < K; k += NG) {
            const uint32_t code = code_s[k * S + s];
            const uint32_t dst = xw_s + (uint32_t)xoff(k + 1, g);
            if (code < CODE_MULTI) {
                if constexpr (Q) {
                    if (16 * g < QRB)
                        cp_async16(xw_s + (uint32_t)((k + 1) * RS + 16 * g), qtab + (long long)code * QRB + 16 * g);
                } else {
                    cp_async16(dst, tables + (long long)code * d + 8 * g);
                }
            } else if (code == CODE_EMPTY) {
                *reinterpret_cast<uint4*>(xw + xoff(k + 1, g)) = make_uint4(0, 0, 0, 0);
            } else {
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
                *reinterpret_cast<uint4*>(xw + xoff(k + 1, g)) =
                    make_uint4(pack_bf16(a[0], a[1]), pack_bf16(a[2], a[3]), pack_bf16(a[4], a[5]), pack_bf16(a[6], a[7]));
            }
        }
        // zero the padding rows K+2 .. KP-1 (G of the previous sample may have overwritten them)
        for (int q = lane; q < (KP - K - 2) * (RS / 16); q += 32)
            reinterpret_cast<uint4*>(xw + (size_t)(K + 2) * RS)[q] = make_uint4(0, 0, 0, 0);

        // ---- 2. x_dense -> rows 0 (hi) and K+1 (lo)
#pragma unroll
        for (int q = 0; q < (d + 127) / 128; ++q) {
            const int c = 4 * lane + 128 * q;
            if (c < d) {
                const float4 x = xv[q];
                const __nv_bfloat162 h01 = __floats2bfloat162_rn(x.x, x.y), h23 = __floats2bfloat162_rn(x.z, x.w);
                const float2 f01 = __bfloat1622float2(h01), f23 = __bfloat1622float2(h23);
                *reinterpret_cast<uint2*>(xw + xoff(0, c / 8) + 2 * (c % 8)) =
                    make_uint2(*reinterpret_cast<const uint32_t*>(&h01), *reinterpret_cast<const uint32_t*>(&h23));
                *reinterpret_cast<uint2*>(xw + xoff(L, c / 8) + 2 * (c % 8)) =
                    make_uint2(pack_bf16(x.x - f01.x, x.y - f01.y), pack_bf16(x.z - f23.x, x.w - f23.y));
            }
        }
        cp_async_wait_all();
        __syncwarp();
        if constexpr (Q) {
            // one-row bags: staged records -> dequantised bf16 rows, in place (every lane reads before any writes)
            for (int kk = 0; kk < (K + NG - 1) / NG; ++kk) {
                const int k = kk * NG + gi;
                const bool one = k < K && code_s[k * S + s] < CODE_MULTI;
                uint4 w = make_uint4(0, 0, 0, 0);
                if (one) {
                    const unsigned char* rec = xw + (size_t)(k + 1) * RS;
                    const uint2 cq = *reinterpret_cast<const uint2*>(rec + 8 * g);
                    const float2 so = *reinterpret_cast<const float2*>(rec + d);
                    float v[8];
                    dequant8(cq, so.x, so.y, v);
                    w = make_uint4(pack_bf16(v[0], v[1]), pack_bf16(v[2], v[3]), pack_bf16(v[4], v[5]),
                                   pack_bf16(v[6], v[7]));
                }
                __syncwarp();
                if (one) *reinterpret_cast<uint4*>(xw + xoff(k + 1, g)) = w;
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
                ldmatrix_x4(xw_s + (uint32_t)xoff(16 * mt + (lane & 15), 2 * ks + (lane >> 4)), a[mt]);
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
    report_warp(err, oob, bad);
}

// ------------------------------------------------------------------ host side

// Bytes of a warp's region: the bf16 tile or its staged Gram, and for uint8 tables (q) also the integer
// route's row slots plus its 8-bit tile or staged Gram.
static int mma_warp_bytes(int K, int d, bool q, int& MT) {
    MT = (K + (q ? 4 : 2) + 15) / 16;
    const int KP = 16 * MT;
    const int RS = d >= 64 ? 2 * d : 2 * d + 16;
    const int gf = (KP * (KP + 8) + 1) * 4;
    int bytes = std::max(KP * RS, RS + gf);
    if (q) bytes = std::max(bytes, (KP + 1) * 16 + std::max(KP * d, gf));
    return (bytes + 15) & ~15;
}

static size_t mma_smem(int K, int d, bool q, int ld, int& MT, int& warp_bytes) {
    warp_bytes = mma_warp_bytes(K, d, q, MT);
    return (size_t)WARPS * warp_bytes + sizeof(uint32_t) * (size_t)K * S + sizeof(uint16_t) * (size_t)(ld - d + 8);
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
    kern<<<(B + S - 1) / S, WARPS * 32, smem, st>>>(tables, tm, K, B, offsets, indices, nnz, x_dense, out, ld, out_dt,
                                                    warp_bytes, err);
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

}  // namespace dlrm
