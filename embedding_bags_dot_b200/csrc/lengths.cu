// Bag lengths -> CSR offsets on the device: offsets[i] = sum_{j < i} lengths[j]
// for i <= n, from one uint8 length per bag (table-major, the order of the
// offsets array). A compact form of the same bags for callers that ship
// inputs over the host link: 1 byte per bag instead of 4.
//
// Two launches over chunks of LCH lengths: the first writes each chunk's sum;
// the second gives every block its chunk's offset (the sum of the sums before
// it) and scans the chunk, 32 lengths per thread.
#include "common.cuh"
#include "kernels.cuh"

namespace dlrm {
namespace {

constexpr int LTHREADS = 256;
constexpr int LPER = 32;                      // lengths per thread
constexpr int LCH = LTHREADS * LPER;          // lengths per chunk (8192)

__device__ __forceinline__ int block_sum(int v, int* tmp) {
    const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    if (lane == 0) tmp[w] = v;
    __syncthreads();
    int t = lane < LTHREADS / 32 ? tmp[lane] : 0;
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) t += __shfl_xor_sync(0xffffffffu, t, o);
    __syncthreads();
    return t;
}

// Lengths lengths[32 t .. 32 t + 32) of this thread's slice of the chunk, 0 past n.
__device__ __forceinline__ void load_slice(const uint8_t* __restrict__ lengths, long long n, long long i0,
                                           uint8_t (&v)[LPER]) {
    if (i0 + LPER <= n && (((uintptr_t)(lengths + i0)) & 15) == 0) {
        const uint4 a = *reinterpret_cast<const uint4*>(lengths + i0);
        const uint4 b = *reinterpret_cast<const uint4*>(lengths + i0 + 16);
        const uint32_t w[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
#pragma unroll
        for (int e = 0; e < LPER; ++e) v[e] = (uint8_t)(w[e >> 2] >> (8 * (e & 3)));
    } else {
#pragma unroll
        for (int e = 0; e < LPER; ++e) v[e] = i0 + e < n ? lengths[i0 + e] : (uint8_t)0;
    }
}

__global__ void __launch_bounds__(LTHREADS) chunk_sums_kernel(const uint8_t* __restrict__ lengths, long long n,
                                                              int* __restrict__ sums) {
    pdl_wait();
    __shared__ int tmp[32];
    uint8_t v[LPER];
    load_slice(lengths, n, (long long)blockIdx.x * LCH + (long long)threadIdx.x * LPER, v);
    int s = 0;
#pragma unroll
    for (int e = 0; e < LPER; ++e) s += v[e];
    s = block_sum(s, tmp);
    if (threadIdx.x == 0) sums[blockIdx.x] = s;
}

__global__ void __launch_bounds__(LTHREADS) chunk_scan_kernel(const uint8_t* __restrict__ lengths, long long n,
                                                              const int* __restrict__ sums, int32_t* __restrict__ offsets) {
    pdl_wait();
    __shared__ int tmp[32];
    __shared__ int scan[LTHREADS];
    // this chunk's offset: the sums of the chunks before it
    int before = 0;
    for (int c = threadIdx.x; c < (int)blockIdx.x; c += LTHREADS) before += sums[c];
    before = block_sum(before, tmp);
    // the thread's own 32 lengths, then an exclusive scan of the thread totals across the block
    const long long i0 = (long long)blockIdx.x * LCH + (long long)threadIdx.x * LPER;
    uint8_t v[LPER];
    load_slice(lengths, n, i0, v);
    int own = 0;
#pragma unroll
    for (int e = 0; e < LPER; ++e) own += v[e];
    scan[threadIdx.x] = own;
    __syncthreads();
    // inclusive Hillis-Steele scan over the 256 thread totals
    for (int o = 1; o < LTHREADS; o <<= 1) {
        const int add = threadIdx.x >= o ? scan[threadIdx.x - o] : 0;
        __syncthreads();
        scan[threadIdx.x] += add;
        __syncthreads();
    }
    int run = before + scan[threadIdx.x] - own;
#pragma unroll
    for (int e = 0; e < LPER; ++e) {
        if (i0 + e < n) offsets[i0 + e] = run;
        run += v[e];
    }
    if (i0 < n && i0 + LPER >= n) offsets[n] = run;   // the thread holding the last length writes the total
}

}  // namespace

size_t lengths_scratch_ints(long long n) { return (size_t)((n + LCH - 1) / LCH + 1); }

dlrm_status launch_offsets_from_lengths(const uint8_t* lengths, long long n, int32_t* offsets, int* scratch,
                                        cudaStream_t st) {
    if (n == 0) return cudaMemsetAsync(offsets, 0, sizeof(int32_t), st) == cudaSuccess ? DLRM_OK : DLRM_ERR_CUDA;
    const long long nb = (n + LCH - 1) / LCH;
    if (nb > 0x7FFFFFFF) return DLRM_ERR_UNSUPPORTED;
    (void)launch_pdl(chunk_sums_kernel, dim3((int)nb), dim3(LTHREADS), (size_t)(0), st, lengths, n, scratch);
    DLRM_LAUNCH_CHECK();
    (void)launch_pdl(chunk_scan_kernel, dim3((int)nb), dim3(LTHREADS), (size_t)(0), st, lengths, n, scratch, offsets);
    DLRM_LAUNCH_CHECK();
    return DLRM_OK;
}

}  // namespace dlrm
