// noalloc.cu - trimul_forward_noalloc: the whole layer without a caller-supplied
// workspace, for callers that cannot allocate device memory.
//
// Some callers of this library have no way to obtain scratch memory: a plugin
// whose host application owns the entire device memory pool and forbids any
// other allocation, or a latency-critical loop that must never risk a
// cudaMalloc failure or the implicit synchronisation an allocation can cause.
// For them this entry point keeps the layer's scratch (the a, b and x
// intermediates and the status word) in one file-scope device array that is
// part of the library image. Every GPU that loads the library holds this array
// until the process exits.
//
// The array is shared by every call: calls whose GPU work overlaps (several
// streams, several host threads) race on it and produce garbage. Only the
// status word must start at zero; trimul_forward clears it on every call. a,
// b and x are fully rewritten before they are read.
//
// The device address of the array is looked up once per device, on the first
// call made with that device current; that first call should therefore come
// before any stream capture. The status word at the start of the array is read
// with trimul_device_status on a params block whose workspace is NULL.
#include <cuda_runtime.h>

#include <mutex>

#include "trimul.h"

namespace {

// Large enough for the bf16 layer at N <= 128 and the fp32 layer at N <= 88.
static __device__ __align__(256) unsigned char g_noalloc_scratch[TRIMUL_NOALLOC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;
std::mutex g_mu;
void *g_scratch_ptr[kMaxDevices];  // device address of g_noalloc_scratch, per device

}  // namespace

namespace trimul {

// Device address of the static scratch for the current device (looked up once
// per device). Used by trimul_forward_noalloc and, for a params block without
// a workspace, by trimul_device_status.
int noalloc_scratch_address(void **out) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return TRIMUL_ERR_CUDA;
    std::lock_guard<std::mutex> lk(g_mu);
    if (!g_scratch_ptr[dev]) {
        // In host code the array's name is only a stand-in; its device address
        // comes from the runtime, with this device current.
        void *p = nullptr;
        if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || !p) {
            cudaGetLastError();
            return TRIMUL_ERR_CUDA;
        }
        g_scratch_ptr[dev] = p;
    }
    *out = g_scratch_ptr[dev];
    return TRIMUL_OK;
}

}  // namespace trimul

extern "C" int trimul_forward_noalloc(const void *z, const void *mask, const trimul_params *p, int direction,
                                      void *out, trimul_stream_t stream) {
    if (!p) return TRIMUL_ERR_INVALID_ARG;
    const size_t need = trimul_workspace_size_dtype(p->N, p->c_z, p->c_h, p->dtype);
    if (need == 0)
        return (p->N < 1 || p->N > 16384 || p->c_z < 1 || p->c_h < 1) ? TRIMUL_ERR_INVALID_ARG
                                                                       : TRIMUL_ERR_UNSUPPORTED;
    if (need > (size_t)TRIMUL_NOALLOC_SCRATCH_BYTES) return TRIMUL_ERR_WORKSPACE;  // beyond the static scratch
    void *scratch = nullptr;
    int rc = trimul::noalloc_scratch_address(&scratch);
    if (rc) return rc;
    trimul_params q = *p;
    q.workspace = scratch;
    q.workspace_bytes = TRIMUL_NOALLOC_SCRATCH_BYTES;
    return trimul_forward(z, mask, &q, direction, out, stream);
}
