// ssd_static_scratch.cu -- the selective scan for callers that cannot allocate.
//
// ssd_scan_forward needs device scratch (the stripe states) that the caller
// allocates and passes in as `workspace`.  Some callers cannot do that: code
// that runs while a memory pool forbids new allocations, plugin or driver
// code handed only input and output buffers by its host framework, or code
// that must not call cudaMalloc (it synchronises the device and may fail under
// memory pressure at an unpredictable moment).  This file gives them one entry
// point, ssd_scan_forward_static_scratch, whose scratch is a fixed array
// compiled into the library itself.  The caller still passes inputs and
// outputs.  Nothing here calls cudaMalloc, cudaFree or any allocating routine.
//
// Costs and limits, stated for the user:
//  - Every GPU that loads libssd.so holds kStaticScratchBytes (80 MiB) of
//    device memory for this array until the process exits.
//  - Shapes whose scratch need (ssd_scan_workspace_size) exceeds that are
//    rejected with SSD_ERR_WORKSPACE before anything is launched.
//  - All calls on a device share the one array and it keeps whatever the last
//    call left there.  Two calls whose kernels overlap on the GPU (different
//    streams, or different host threads) race on it and corrupt each other:
//    serialise them.  No part of the array has to start at zero: each call
//    writes every scratch element before it reads it.
//  - The array's address is looked up (cudaGetSymbolAddress) by the first
//    call made on each device, with that device current.  Make that first
//    call before any stream capture on that device.
#include <atomic>
#include <cstdio>

#include "../../include/ssd.h"
#include "ssd_common.cuh"

namespace ssd {
int set_error(int code, const char *msg);
}

namespace {

constexpr size_t kStaticScratchBytes = size_t(80) << 20;  // 80 MiB

// The scratch itself.  In host code `g_static_scratch` is only a stand-in for
// the device symbol, never a device address: it must be resolved with
// cudaGetSymbolAddress on each device before a kernel may be given it.
static __device__ __align__(256) unsigned char g_static_scratch[kStaticScratchBytes];

constexpr int kMaxDevices = 64;
// One address per device.  Host threads making their first call together may
// both look it up; they store the same value, and the atomics make that well defined.
std::atomic<void *> g_scratch_addr[kMaxDevices];

// Device address of the scratch on the current device (looked up once per device).
int scratch_address(void **out)
{
    int dev = -1;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess || dev < 0 || dev >= kMaxDevices)
        return ssd::set_error(SSD_ERR_LAUNCH, "static scratch: no usable current CUDA device");
    void *addr = g_scratch_addr[dev].load(std::memory_order_acquire);
    if (!addr) {
        void *p = nullptr;
        e = cudaGetSymbolAddress(&p, g_static_scratch);
        if (e != cudaSuccess || !p) {
            char msg[256];
            snprintf(msg, sizeof msg, "static scratch: cudaGetSymbolAddress failed on device %d: %s", dev,
                     cudaGetErrorString(e));
            return ssd::set_error(SSD_ERR_LAUNCH, msg);
        }
        g_scratch_addr[dev].store(p, std::memory_order_release);
        addr = p;
    }
    *out = addr;
    return SSD_OK;
}

}  // namespace

extern "C" SSD_API int ssd_scan_forward_static_scratch(const ssd_scan_args *args, ssd_stream_t stream)
{
    if (!args) return ssd::set_error(SSD_ERR_NULL, "args is NULL");
    const size_t need = ssd_scan_workspace_size(args->b, args->L, args->H, args->P, args->N, args->Q);
    if (need > kStaticScratchBytes) {
        char msg[256];
        snprintf(msg, sizeof msg,
                 "static scratch: this shape needs %zu bytes of scratch, more than the %zu-byte "
                 "array compiled into the library; use ssd_scan_forward with a workspace",
                 need, kStaticScratchBytes);
        return ssd::set_error(SSD_ERR_WORKSPACE, msg);
    }
    void *scratch = nullptr;
    const int rc = scratch_address(&scratch);
    if (rc != SSD_OK) return rc;
    ssd_scan_args a = *args;
    a.workspace = scratch;
    a.workspace_bytes = need > 0 ? kStaticScratchBytes : 0;
    return ssd_scan_forward(&a, stream);
}
