// dlrm_forward_noalloc: the whole forward pass with its scratch memory in a
// fixed device array compiled into this library, for callers that cannot
// allocate device memory themselves.
//
// Who needs it: code that runs inside a host application or serving runtime
// which owns every byte of device memory (a plugin handed only its input and
// output buffers), request paths where an allocation and the device-wide
// synchronisation cudaMalloc/cudaFree can imply are not allowed, and small C
// callers with no device allocator of their own. They pass inputs and
// outputs only; the scratch that dlrm_forward takes as `ws` is this array.
//
// The array holds DLRM_NOALLOC_SCRATCH_BYTES on every GPU that loads the
// library, for the life of the process. In host code its name is only a
// host-side stand-in, so its device address is looked up once per device
// (cudaGetSymbolAddress, with that device current) on the first call made
// on that device.
#include <mutex>

#include "common.cuh"
#include "kernels.cuh"

static __device__ __align__(256) unsigned char g_noalloc_scratch[DLRM_NOALLOC_SCRATCH_BYTES];

namespace {

constexpr int kMaxDevices = 64;
std::mutex g_mu;
void* g_scratch_addr[kMaxDevices] = {};

// Device address of the scratch array on the current device (set up once per device).
cudaError_t scratch_address(void** out) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
    std::lock_guard<std::mutex> lock(g_mu);
    if (!g_scratch_addr[dev]) {
        void* p = nullptr;
        e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
        if (e != cudaSuccess) return e;
        g_scratch_addr[dev] = p;
    }
    *out = g_scratch_addr[dev];
    return cudaSuccess;
}

}  // namespace

extern "C" dlrm_status dlrm_forward_noalloc(const dlrm_tables* T, const dlrm_mlp* bot, const dlrm_mlp* top, int B,
                                            const float* dense, const int32_t* offsets, const int32_t* indices,
                                            int64_t nnz, float* y_hat, uint32_t* err_flags, dlrm_stream stream) {
    void* scratch = nullptr;
    if (scratch_address(&scratch) != cudaSuccess) return DLRM_ERR_CUDA;
    // Every check dlrm_forward makes, with the array as its workspace, before anything is queued: a
    // refused call returns the same status as dlrm_forward and leaves err_flags and the array alone.
    dlrm_status r = dlrm::forward_check(T, bot, top, B, dense, offsets, indices, nnz, y_hat, scratch,
                                        DLRM_NOALLOC_SCRATCH_BYTES, false);
    if (r != DLRM_OK) return r;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    // The array keeps the previous call's contents: the error record must start at zero.
    if (cudaMemsetAsync(scratch, 0, DLRM_ERR_RECORD_BYTES, st) != cudaSuccess) return DLRM_ERR_CUDA;
    r = dlrm_forward(T, bot, top, B, dense, offsets, indices, nnz, y_hat, scratch, DLRM_NOALLOC_SCRATCH_BYTES, stream);
    if (r != DLRM_OK) return r;
    if (err_flags && cudaMemcpyAsync(err_flags, scratch, sizeof(uint32_t), cudaMemcpyDeviceToDevice, st) != cudaSuccess)
        return DLRM_ERR_CUDA;
    return DLRM_OK;
}
