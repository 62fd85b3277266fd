// kda_bwd_noalloc.cu -- kda_chunk_bwd_noalloc: the recompute backward with library-held scratch.
//
// kda_chunk_bwd needs a device workspace (the state entering every chunk plus per-chain
// scratch) that its caller allocates.  Some callers cannot allocate device memory at the
// point where they run the backward: their device memory is owned by another allocator
// (a framework's caching pool that has already reserved what is free, so cudaMalloc fails),
// or they run under a rule of no allocation after start-up, because cudaMalloc and cudaFree
// synchronise the device and can stall work on every other stream.  For them this file holds
// a fixed scratch array in the library's own device image and passes it to the same kernel.
//
// The array is a file-scope __device__ variable: each GPU that loads this library's device
// code holds its KDA_BWD_NOALLOC_SCRATCH_BYTES until the process exits.  In host code its
// name is only a host-side stand-in, so its device address is looked up with
// cudaGetSymbolAddress, once per device, with that device current, on the first call made
// on that device.
#include <cuda_runtime.h>
#include <stdint.h>
#include <stdio.h>

#include <mutex>

#include "../../include/kda.h"
#include "kda_internal.h"

namespace {

static __device__ __align__(256) unsigned char g_bwd_noalloc_scratch[KDA_BWD_NOALLOC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;
void *g_scratch_ptr[kMaxDevices] = {nullptr};
std::mutex g_scratch_mu;

kda_status fail_msg(kda_status s, const char *msg) { return (kda_status)kda::set_last_error((int)s, msg); }

// Device address of this device's scratch array (looked up once per device).
kda_status scratch_ptr(void **out) {
    int dev = -1;
    cudaError_t e = cudaGetDevice(&dev);
    char msg[256];
    if (e != cudaSuccess) {
        snprintf(msg, sizeof(msg), "cudaGetDevice: %s", cudaGetErrorString(e));
        return fail_msg(KDA_ERR_CUDA, msg);
    }
    if (dev < 0 || dev >= kMaxDevices) {
        snprintf(msg, sizeof(msg), "device id %d out of range", dev);
        return fail_msg(KDA_ERR_UNSUPPORTED_DEVICE, msg);
    }
    int major = 0, minor = 0;
    cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev);
    cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev);
    if (major != 10 || minor != 0) {
        snprintf(msg, sizeof(msg), "device %d is sm_%d%d; libkda is built for sm_100a (B200) only", dev, major,
                 minor);
        return fail_msg(KDA_ERR_UNSUPPORTED_DEVICE, msg);
    }
    std::lock_guard<std::mutex> lock(g_scratch_mu);
    if (!g_scratch_ptr[dev]) {
        void *p = nullptr;
        e = cudaGetSymbolAddress(&p, g_bwd_noalloc_scratch);
        if (e != cudaSuccess) {
            snprintf(msg, sizeof(msg), "cudaGetSymbolAddress(backward scratch): %s", cudaGetErrorString(e));
            return fail_msg(KDA_ERR_CUDA, msg);
        }
        g_scratch_ptr[dev] = p;
    }
    *out = g_scratch_ptr[dev];
    return KDA_OK;
}

}  // namespace

extern "C" kda_status kda_chunk_bwd_noalloc(const uint16_t *q, const uint16_t *k, const uint16_t *v,
                                            const float *g, const float *beta, const int32_t *cu_seqlens,
                                            int n_docs, int64_t T, int H, const uint16_t *dout, uint16_t *dq,
                                            uint16_t *dk, uint16_t *dv, float *dg, float *dbeta, void *stream) {
    // Calls that need no workspace (T = 0) or that kda_chunk_bwd rejects on their sizes are
    // passed straight through: it reports them before any device work.
    if (n_docs < 1 || H < 1 || T <= 0 || T > (int64_t)INT32_MAX || !cu_seqlens)
        return kda_chunk_bwd(q, k, v, g, beta, cu_seqlens, n_docs, T, H, dout, dq, dk, dv, dg, dbeta, nullptr, 0,
                             stream);
    const size_t need = kda_chunk_bwd_workspace_size(n_docs, T, H);
    if (need > (size_t)KDA_BWD_NOALLOC_SCRATCH_BYTES) {
        char msg[256];
        snprintf(msg, sizeof(msg),
                 "kda_chunk_bwd_noalloc: n_docs=%d, T=%lld, H=%d needs %zu bytes of scratch, more than the "
                 "%zu bytes this entry point holds; use kda_chunk_bwd with a caller-owned workspace",
                 n_docs, (long long)T, H, need, (size_t)KDA_BWD_NOALLOC_SCRATCH_BYTES);
        return fail_msg(KDA_ERR_INVALID_ARG, msg);
    }
    void *scratch = nullptr;
    kda_status s = scratch_ptr(&scratch);
    if (s != KDA_OK) return s;
    // The kernel initialises every scratch value it reads (the states it starts from are
    // zeroed in the kernel), so the previous call's contents need no clearing.
    return kda_chunk_bwd(q, k, v, g, beta, cu_seqlens, n_docs, T, H, dout, dq, dk, dv, dg, dbeta, scratch,
                         (size_t)KDA_BWD_NOALLOC_SCRATCH_BYTES, stream);
}
