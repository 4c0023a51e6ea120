// Row-wise 8-bit table quantisation (DLRM_U8ROW records) and the record
// layout helper. One warp per row: min/max by shuffle, then the codes.
#include "common.cuh"
#include "kernels.cuh"

namespace dlrm {

size_t u8row_bytes(int d) { return align_up((size_t)d + 8, 16); }

namespace {

template <typename T>
__global__ void quantize_rows_kernel(const T* __restrict__ src, long long rows, int d, unsigned char* __restrict__ dst,
                                     long long rb) {
    pdl_wait();
    const int lane = threadIdx.x & 31;
    const long long warps = (long long)gridDim.x * (blockDim.x >> 5);
    for (long long r = (long long)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); r < rows; r += warps) {
        const T* row = src + r * d;
        float lo = INFINITY, hi = -INFINITY;
        for (int c = lane; c < d; c += 32) {
            const float v = Cvt<T>::to_f(row[c]);
            lo = fminf(lo, v);
            hi = fmaxf(hi, v);
        }
#pragma unroll
        for (int o = 16; o >= 1; o >>= 1) {
            lo = fminf(lo, __shfl_xor_sync(0xffffffffu, lo, o));
            hi = fmaxf(hi, __shfl_xor_sync(0xffffffffu, hi, o));
        }
        const float s = __fdiv_rn(__fsub_rn(hi, lo), 255.0f);
        unsigned char* rec = dst + r * rb;
        for (int c = lane; c < d; c += 32) {
            const float v = Cvt<T>::to_f(row[c]);
            float q = 0.f;
            if (s > 0.f) q = rintf(__fdiv_rn(__fsub_rn(v, lo), s));
            q = fminf(fmaxf(q, 0.f), 255.f);
            rec[c] = (unsigned char)q;
        }
        if (lane == 0) {
            reinterpret_cast<float*>(rec + d)[0] = s;
            reinterpret_cast<float*>(rec + d)[1] = lo;
        }
        for (long long c = d + 8 + lane; c < rb; c += 32) rec[c] = 0;
    }
}

}  // namespace
}  // namespace dlrm

using namespace dlrm;

extern "C" {

size_t dlrm_row_bytes(int d, dlrm_dtype dt) {
    if (d < 1) return 0;
    if (dt == DLRM_U8ROW) return u8row_bytes(d);
    return (size_t)d * esize(dt);
}

dlrm_status dlrm_quantize_rows_u8(const void* src, dlrm_dtype src_dt, int64_t rows, int d, void* dst,
                                  dlrm_stream stream) {
    if (rows < 0 || d < 1 || d % 4) return DLRM_ERR_INVALID_ARG;
    if (src_dt != DLRM_F32 && src_dt != DLRM_BF16) return DLRM_ERR_UNSUPPORTED;
    if (rows == 0) return DLRM_OK;
    if (!src || !dst || ((uintptr_t)dst & 15)) return DLRM_ERR_INVALID_ARG;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    const long long blocks = (rows + 7) / 8;
    const int grid = (int)(blocks < 148 * 32 ? blocks : 148 * 32);
    const long long rb = (long long)u8row_bytes(d);
    if (src_dt == DLRM_F32)
        (void)launch_pdl(quantize_rows_kernel<float>, dim3(grid), dim3(256), (size_t)(0), st, static_cast<const float*>(src), rows, d,
                                                          static_cast<unsigned char*>(dst), rb);
    else
        (void)launch_pdl(quantize_rows_kernel<__nv_bfloat16>, dim3(grid), dim3(256), (size_t)(0), st, static_cast<const __nv_bfloat16*>(src), rows, d,
                                                                  static_cast<unsigned char*>(dst), rb);
    DLRM_LAUNCH_CHECK();
    return DLRM_OK;
}

}  // extern "C"
