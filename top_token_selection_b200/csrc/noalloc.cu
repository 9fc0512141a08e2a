// noalloc.cu -- the MTP decode step for callers that cannot allocate.
//
// pivot_decode() takes its scratch space from the caller.  Some callers have
// none to give: a plugin running inside an inference engine whose memory
// planner owns every byte of the device, or a decode loop that may not add an
// allocation in the middle of its per-token step.  pivot_decode_noalloc()
// runs the same decode step with its scratch in a fixed array that lives in
// the library's own device memory, so the call allocates nothing.
//
// The array is a file-scope __device__ variable: every GPU on which the
// library's module is loaded holds its 64 MiB until the process exits.  In
// host code its name is only a host-side stand-in, never a device address,
// so its device address is looked up with cudaGetSymbolAddress, with the
// caller's device current.  The lookup is repeated on every call made
// outside stream capture, so a device reset or another current context
// (which load the module again, at another address) is picked up by the next
// such call; during capture the address last looked up on that device is
// used.
#include <mutex>

#include "common.cuh"
#include "kernels.h"

namespace pivot {
// pivot_decode's argument checks (api.cu)
pivot_status_t decode_check_args(const pivot_decode_t* b, int32_t mode, int32_t C, int32_t topk,
                                 const int32_t* idx);
}  // namespace pivot

namespace {

constexpr size_t kNoallocScratchBytes = size_t(64) << 20;   // 64 MiB per device
constexpr int kMaxDevices = 64;

static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoallocScratchBytes];

std::mutex g_noalloc_mu;
void* g_noalloc_addr[kMaxDevices] = {nullptr};

// Device address of the current device's scratch array.  Outside capture it
// is looked up afresh (and remembered); while `stream` is being captured the
// remembered address is used, since a lookup may have to load the module,
// which capture does not allow.
pivot_status_t noalloc_scratch(cudaStream_t stream, void** out) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices)
        return PIVOT_ERR_CUDA;
    cudaStreamCaptureStatus cap = cudaStreamCaptureStatusNone;
    if (cudaStreamIsCapturing(stream, &cap) != cudaSuccess) return PIVOT_ERR_CUDA;
    std::lock_guard<std::mutex> lk(g_noalloc_mu);
    if (cap == cudaStreamCaptureStatusNone || !g_noalloc_addr[dev]) {
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || !p)
            return PIVOT_ERR_CUDA;
        g_noalloc_addr[dev] = p;
    }
    *out = g_noalloc_addr[dev];
    return PIVOT_OK;
}

}  // namespace

extern "C" {

pivot_status_t pivot_decode_noalloc(const pivot_decode_t* batch, int32_t mode, int32_t C,
                                    int32_t topk, int32_t* idx, int32_t* cand, void* stream) {
    // the checks pivot_decode runs come first, so both report the same status
    pivot_status_t st = pivot::decode_check_args(batch, mode, C, topk, idx);
    if (st != PIVOT_OK) return st;
    const size_t need = pivot_decode_workspace_size(batch, mode, C, topk);
    if (need == 0 || need > kNoallocScratchBytes) return PIVOT_ERR_WORKSPACE;
    void* scratch = nullptr;
    st = noalloc_scratch(static_cast<cudaStream_t>(stream), &scratch);
    if (st != PIVOT_OK) return st;
    // Nothing in the decode scratch has to start at zero: every entry a
    // kernel reads was written earlier in the same call.
    return pivot_decode(batch, mode, C, topk, idx, cand, scratch, kNoallocScratchBytes, stream);
}

}  // extern "C"
