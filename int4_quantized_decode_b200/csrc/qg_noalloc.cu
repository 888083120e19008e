// qg_noalloc.cu -- qg_head_argmax_noalloc: the fused head GEMV + argmax for
// callers that cannot hand the library a device workspace.
//
// Some callers cannot allocate device memory at the point where they decode:
// a plugin or custom operator whose host framework owns and budgets every
// device allocation, or a latency-critical loop in which a device allocation
// (and the synchronization it can imply) is not acceptable.  This entry point
// needs no workspace from them: the reduction scratch of the head kernel lives
// in a file-scope device array that every GPU loading the library holds until
// the process exits.  Nothing here calls cudaMalloc, cudaFree or any
// allocating routine.
#include <mutex>

#include "qg_internal.h"

namespace qg {
namespace {

// The scratch: the head kernel needs 16 bytes (a 64-bit argmax key and a
// 32-bit ticket) whatever the vocabulary size; 256 bytes are reserved.
constexpr size_t kNoAllocScratchBytes = 256;
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

// Device address of g_noalloc_scratch on each device.  In host code the
// symbol's name is only a host-side handle, never a device address.  The
// address is looked up again on every call whose stream is not being captured
// (a reset context reloads the module and may move the array); a captured call
// uses the address of the last uncaptured one, since a lookup during capture
// may not be allowed.
constexpr int kMaxDevices = 64;
std::mutex g_setup_mutex;
void* g_scratch_ptr[kMaxDevices] = {nullptr};

qg_status scratch_for_current_device(cudaStream_t stream, void** out) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return cuda_status(e);
    if (dev < 0 || dev >= kMaxDevices) return QG_ERR_CUDA;
    cudaStreamCaptureStatus cap = cudaStreamCaptureStatusNone;
    e = cudaStreamIsCapturing(stream, &cap);
    if (e != cudaSuccess) return cuda_status(e);
    std::lock_guard<std::mutex> lock(g_setup_mutex);
    if (cap == cudaStreamCaptureStatusNone) {
        void* p = nullptr;
        e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
        if (e != cudaSuccess) return cuda_status(e);
        g_scratch_ptr[dev] = p;
    } else if (g_scratch_ptr[dev] == nullptr) {
        return QG_ERR_CUDA;  // first call on this device made during capture
    }
    *out = g_scratch_ptr[dev];
    return QG_OK;
}

}  // namespace
}  // namespace qg

extern "C" qg_status qg_head_argmax_noalloc(const qg_weight* W, const uint16_t* x, float* logits,
                                           int32_t* idx, cudaStream_t stream) {
    if (!W || !x || !idx) return QG_ERR_NULL;
    if (W->n < 1) return QG_ERR_SHAPE;
    // A request for more scratch than the built-in array holds is refused.
    if (qg_head_argmax_workspace_bytes(W->n) > qg::kNoAllocScratchBytes) return QG_ERR_WORKSPACE;
    void* scratch = nullptr;
    qg_status st = qg::scratch_for_current_device(stream, &scratch);
    if (st != QG_OK) return st;
    // The array keeps whatever the previous call left; the kernel needs its
    // key and ticket at zero, so clear them on this stream first.
    cudaError_t e = cudaMemsetAsync(scratch, 0, qg::kHeadWorkspaceBytes, stream);
    if (e != cudaSuccess) return qg::cuda_status(e);
    return qg_head_argmax(W, x, logits, idx, scratch, qg::kNoAllocScratchBytes, stream);
}
