// Device-side twin of synth/gen.py's table generator, for tables too large to
// build on the host. Input generation only.
//
// Element (table k, row r, column c) is output n = (k << 40) + r*d + c of the
// SplitMix64 stream that starts at `seed` (Steele, Lea & Flood, OOPSLA 2014):
//   z = seed + (n + 1) * 0x9E3779B97F4A7C15
//   z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9
//   z = (z ^ (z >> 27)) * 0x94D049BB133111EB
//   z = z ^ (z >> 31)
// u = z >> 40 (24 bits); value = fp32(fp32((2u - 2^24) * 2^-24) * scale), with
// scale = fp32(1/sqrt(m_k)) supplied by the host; 16-bit tables round that
// fp32 value to nearest-even.
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace {

__device__ __forceinline__ unsigned long long splitmix64_at(unsigned long long seed, unsigned long long n) {
    unsigned long long z = seed + (n + 1ull) * 0x9E3779B97F4A7C15ull;
    z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
    z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
    return z ^ (z >> 31);
}

template <typename T>
__device__ __forceinline__ T cvt(float v);
template <> __device__ __forceinline__ float cvt<float>(float v) { return v; }
template <> __device__ __forceinline__ __nv_bfloat16 cvt<__nv_bfloat16>(float v) { return __float2bfloat16_rn(v); }
template <> __device__ __forceinline__ __half cvt<__half>(float v) { return __float2half_rn(v); }

template <typename T>
__global__ void fill_kernel(T* __restrict__ dst, long long count, unsigned long long first, unsigned long long seed,
                            float scale) {
    const long long stride = (long long)gridDim.x * blockDim.x;
    for (long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x; i < count; i += stride) {
        const unsigned long long z = splitmix64_at(seed, first + (unsigned long long)i);
        const int u = (int)(z >> 40);
        const float t = __int2float_rn(2 * u - (1 << 24));
        dst[i] = cvt<T>(__fmul_rn(__fmul_rn(t, 5.9604644775390625e-08f), scale));
    }
}

}  // namespace

extern "C" {

// Fills rows [0, m) of table `table_id` (width d) at dst. dtype: 0 fp32, 1 fp16, 2 bf16.
// Returns 0 on success, a cudaError_t otherwise.
int synth_fill_table(void* dst, int dtype, long long m, int d, int table_id, unsigned long long seed, float scale,
                     void* stream) {
    const long long count = m * (long long)d;
    if (count == 0) return 0;
    const unsigned long long first = (unsigned long long)table_id << 40;
    const int threads = 256;
    long long blocks = (count + threads - 1) / threads;
    if (blocks > 148LL * 32) blocks = 148LL * 32;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    switch (dtype) {
        case 0: fill_kernel<float><<<(int)blocks, threads, 0, st>>>((float*)dst, count, first, seed, scale); break;
        case 1: fill_kernel<__half><<<(int)blocks, threads, 0, st>>>((__half*)dst, count, first, seed, scale); break;
        case 2: fill_kernel<__nv_bfloat16><<<(int)blocks, threads, 0, st>>>((__nv_bfloat16*)dst, count, first, seed, scale); break;
        default: return (int)cudaErrorInvalidValue;
    }
    return (int)cudaPeekAtLastError();
}
}
