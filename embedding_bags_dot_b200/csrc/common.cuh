// Shared device helpers of libdlrm: dtype conversion, 16-byte row loads, the
// device error record and launch checking.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "dlrm.h"

namespace dlrm {

// ----------------------------------------------------------------- error record
// Lives at the start of every workspace. Device code only ever ORs flags and
// adds counts, so concurrent reports are order independent.
struct ErrRecord {
    unsigned int flags;
    unsigned int reserved;
    unsigned long long n_oob;   // skipped indices
    unsigned long long n_bad;   // bags with bad offsets
};
enum : unsigned { ERR_OOB = 1u, ERR_BAD_OFFSETS = 2u, ERR_TIMEOUT = 4u };

__device__ __forceinline__ void report(ErrRecord* e, unsigned long long oob, unsigned long long bad) {
    if (oob) {
        atomicOr(&e->flags, ERR_OOB);
        atomicAdd(&e->n_oob, oob);
    }
    if (bad) {
        atomicOr(&e->flags, ERR_BAD_OFFSETS);
        atomicAdd(&e->n_bad, bad);
    }
}

// Warp-wide sum then one atomic per warp.
__device__ __forceinline__ void report_warp(ErrRecord* e, unsigned oob, unsigned bad) {
    unsigned any = __ballot_sync(0xffffffffu, oob | bad);
    if (!any) return;
    for (int o = 16; o; o >>= 1) {
        oob += __shfl_xor_sync(0xffffffffu, oob, o);
        bad += __shfl_xor_sync(0xffffffffu, bad, o);
    }
    if ((threadIdx.x & 31) == 0) report(e, oob, bad);
}

// ----------------------------------------------------------------- dtypes
template <typename T> struct Cvt;
template <> struct Cvt<float> {
    static __device__ __forceinline__ float to_f(float x) { return x; }
    static __device__ __forceinline__ float from_f(float x) { return x; }
};
template <> struct Cvt<__nv_bfloat16> {
    static __device__ __forceinline__ float to_f(__nv_bfloat16 x) { return __bfloat162float(x); }
    static __device__ __forceinline__ __nv_bfloat16 from_f(float x) { return __float2bfloat16_rn(x); }
};
template <> struct Cvt<__half> {
    static __device__ __forceinline__ float to_f(__half x) { return __half2float(x); }
    static __device__ __forceinline__ __half from_f(float x) { return __float2half_rn(x); }
};

__device__ __forceinline__ void store_as(void* base, size_t i, float v, int dt) {
    if (dt == DLRM_F32) static_cast<float*>(base)[i] = v;
    else if (dt == DLRM_BF16) static_cast<__nv_bfloat16*>(base)[i] = __float2bfloat16_rn(v);
    else static_cast<__half*>(base)[i] = __float2half_rn(v);
}

// 16-byte load that bypasses L1 allocation (rows are gathered once per bag).
__device__ __forceinline__ uint4 ldg16_stream(const void* p) {
    uint4 v;
    asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "l"(p));
    return v;
}

// Unpack a 16-byte chunk of T into fp32 and add it to acc[16 / sizeof(T)].
template <typename T> struct Chunk16;
template <> struct Chunk16<float> {
    static constexpr int E = 4;
    static __device__ __forceinline__ void add(const uint4& v, float* a) {
        const float2 lo = __fadd2_rn(make_float2(a[0], a[1]), make_float2(__uint_as_float(v.x), __uint_as_float(v.y)));
        const float2 hi = __fadd2_rn(make_float2(a[2], a[3]), make_float2(__uint_as_float(v.z), __uint_as_float(v.w)));
        a[0] = lo.x; a[1] = lo.y; a[2] = hi.x; a[3] = hi.y;
    }
};
template <> struct Chunk16<__nv_bfloat16> {
    static constexpr int E = 8;
    static __device__ __forceinline__ void add2(unsigned w, float* a) {
        // both halves widened exactly, then one packed two-lane fp32 add (round to nearest)
        const float2 s = __fadd2_rn(make_float2(a[0], a[1]),
                                    make_float2(__uint_as_float(w << 16), __uint_as_float(w & 0xffff0000u)));
        a[0] = s.x;
        a[1] = s.y;
    }
    static __device__ __forceinline__ void add(const uint4& v, float* a) {
        add2(v.x, a); add2(v.y, a + 2); add2(v.z, a + 4); add2(v.w, a + 6);
    }
};
template <> struct Chunk16<__half> {
    static constexpr int E = 8;
    static __device__ __forceinline__ void add2(unsigned w, float* a) {
        __half2 h = *reinterpret_cast<const __half2*>(&w);
        float2 f = __half22float2(h);
        a[0] += f.x; a[1] += f.y;
    }
    static __device__ __forceinline__ void add(const uint4& v, float* a) {
        add2(v.x, a); add2(v.y, a + 2); add2(v.z, a + 4); add2(v.w, a + 6);
    }
};

// Per-table layout passed by value to the gather kernels.
struct TableMeta {
    long long base[DLRM_MAX_TABLES];   // first row of table k in the shared buffer
    long long rows[DLRM_MAX_TABLES];   // m_k
};

// ----------------------------------------------------------------- programmatic dependent launch
// Every kernel of this library is launched with programmatic stream
// serialisation (launch_pdl): a kernel is scheduled as soon as every block of
// the kernel before it on the stream has exited (the implicit trigger at a
// block's exit, not the kernel's completion), and sets up its shared
// memory, barriers and TMEM while that kernel's completion is still being
// made visible. It calls pdl_wait() before its first access to global memory;
// that returns once the previous kernel has completed and its writes are
// visible, so reads and writes keep plain stream order. No kernel asks for its
// dependent to be scheduled earlier than its own exit: a dependent grid
// scheduled while a kernel of several blocks per SM still runs piles its
// blocks onto the few SMs that happen to be free (measured: the medium
// forward's fp32 layers ran 25 % slower that way). Launched without the
// attribute, pdl_wait() returns at once.
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

template <typename... KArgs, typename... Args>
inline cudaError_t launch_pdl(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st,
                              Args&&... args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute at[1];
    at[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    at[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = at;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kern, static_cast<Args&&>(args)...);
}

inline size_t esize(dlrm_dtype dt) { return dt == DLRM_F32 ? 4 : 2; }

inline size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

// Number of kernels this library has launched in the process (dlrm_launch_count()).
void count_launch();

}  // namespace dlrm

// Status of a launch_pdl call: counts the launch, clears and reports a failure.
#define DLRM_PDL_CHECK(call)                                     \
    do {                                                         \
        dlrm::count_launch();                                    \
        if ((call) != cudaSuccess) {                             \
            (void)cudaGetLastError();                            \
            return DLRM_ERR_CUDA;                                \
        }                                                        \
    } while (0)

#define DLRM_LAUNCH_CHECK()                                      \
    do {                                                         \
        dlrm::count_launch();                                    \
        if (cudaPeekAtLastError() != cudaSuccess) {              \
            (void)cudaGetLastError();                            \
            return DLRM_ERR_CUDA;                                \
        }                                                        \
    } while (0)
