// kda_api.cu -- the extern "C" boundary of libkda (declared in include/kda.h).
//
// Argument marshalling and validation only: every step of the forward runs in
// the CUDA kernels.  Checks follow the "first violated condition" convention
// of fused_kda_unsupported_reason on the kda_fused page of
// nemo_automodel.components.models.kimi_k3: the first failing check is
// reported and nothing is launched; there is no fallback.
#include <cuda_runtime.h>
#include <stdarg.h>
#include <stdint.h>
#include <stdio.h>

#include <mutex>

#include "../../include/kda.h"
#include "kda_internal.h"

namespace {

thread_local char g_err[512] = "";

kda_status fail(kda_status s, const char *fmt, ...) {
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(g_err, sizeof(g_err), fmt, ap);
    va_end(ap);
    return s;
}

// One status word per device; its device address is looked up once per device.
__device__ int g_kda_status_word;

constexpr int kMaxDevices = 64;
int *g_status_ptr[kMaxDevices] = {nullptr};
std::mutex g_status_mu;

kda_status status_ptr(int dev, int **out) {
    if (dev < 0 || dev >= kMaxDevices) return fail(KDA_ERR_UNSUPPORTED_DEVICE, "device id %d out of range", dev);
    std::lock_guard<std::mutex> lock(g_status_mu);
    if (!g_status_ptr[dev]) {
        void *p = nullptr;
        cudaError_t e = cudaGetSymbolAddress(&p, g_kda_status_word);
        if (e != cudaSuccess) return fail(KDA_ERR_CUDA, "cudaGetSymbolAddress: %s", cudaGetErrorString(e));
        g_status_ptr[dev] = static_cast<int *>(p);
    }
    *out = g_status_ptr[dev];
    return KDA_OK;
}

kda_status check_device(int *dev_out) {
    int dev = -1;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return fail(KDA_ERR_CUDA, "cudaGetDevice: %s", cudaGetErrorString(e));
    int major = 0, minor = 0;
    cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev);
    cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev);
    if (major != 10 || minor != 0)
        return fail(KDA_ERR_UNSUPPORTED_DEVICE,
                    "device %d is sm_%d%d; libkda is built for sm_100a (B200) only", dev, major, minor);
    *dev_out = dev;
    return KDA_OK;
}

bool aligned(const void *p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

bool overlaps(const void *a, size_t na, const void *b, size_t nb) {
    const uintptr_t x = reinterpret_cast<uintptr_t>(a), y = reinterpret_cast<uintptr_t>(b);
    return x < y + nb && y < x + na;
}

}  // namespace

namespace kda {

int set_last_error(int status, const char *msg) { return (int)fail((kda_status)status, "%s", msg); }

int device_context(int *dev, int **status) {
    kda_status s = check_device(dev);
    if (s != KDA_OK) return s;
    return status_ptr(*dev, status);
}

}  // namespace kda

extern "C" {

const char *kda_last_error(void) { return g_err; }

int kda_abi_version(void) { return 1; }

}  // extern "C"

namespace {

enum class FwdKernel { kChunk, kRecurrent };

// Validation and launch shared by the chunked and the recurrent forward (same arguments,
// same contract); `which` selects the kernel.
kda_status fwd_common(FwdKernel which, const uint16_t *q, const uint16_t *k, const uint16_t *v, const float *g,
                      const float *beta, const int32_t *cu_seqlens, int n_docs, int64_t T, int H,
                      const float *initial_state, float *final_state, uint16_t *out, void *stream) {
    g_err[0] = '\0';
    if (n_docs < 1) return fail(KDA_ERR_INVALID_ARG, "n_docs must be >= 1 (got %d)", n_docs);
    if (H < 1) return fail(KDA_ERR_INVALID_ARG, "H must be >= 1 (got %d)", H);
    if (T < 0) return fail(KDA_ERR_INVALID_ARG, "T must be >= 0 (got %lld)", (long long)T);
    if (T > (int64_t)INT32_MAX) return fail(KDA_ERR_INVALID_ARG, "T must fit int32 (cu_seqlens is int32)");
    if (!cu_seqlens) return fail(KDA_ERR_INVALID_ARG, "cu_seqlens is NULL");
    const int64_t chains = (int64_t)n_docs * H;
    if (chains > (int64_t)INT32_MAX) return fail(KDA_ERR_INVALID_ARG, "n_docs * H too large for one launch");
    const size_t state_bytes = (size_t)chains * KDA_HEAD_DIM * KDA_HEAD_DIM * sizeof(float);
    if ((initial_state && !aligned(initial_state, 16)) || (final_state && !aligned(final_state, 16)))
        return fail(KDA_ERR_INVALID_ARG, "initial_state and final_state must be 16-byte aligned");
    if (initial_state && final_state && initial_state != final_state &&
        overlaps(initial_state, state_bytes, final_state, state_bytes))
        return fail(KDA_ERR_INVALID_ARG, "initial_state and final_state must be the same buffer or disjoint");
    if (T == 0) {
        // no tokens: the final states are the initial ones
        if (!final_state || final_state == initial_state) return KDA_OK;
        int dev = -1;
        kda_status s = check_device(&dev);
        if (s != KDA_OK) return s;
        cudaStream_t st = static_cast<cudaStream_t>(stream);
        cudaError_t e = initial_state
                            ? cudaMemcpyAsync(final_state, initial_state, state_bytes, cudaMemcpyDeviceToDevice, st)
                            : cudaMemsetAsync(final_state, 0, state_bytes, st);
        if (e != cudaSuccess) return fail(KDA_ERR_CUDA, "final state copy: %s", cudaGetErrorString(e));
        return KDA_OK;
    }
    if (!q || !k || !v || !g || !beta || !out) return fail(KDA_ERR_INVALID_ARG, "a tensor pointer is NULL");
    if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(g, 16) || !aligned(out, 16))
        return fail(KDA_ERR_INVALID_ARG, "q, k, v, g and out must be 16-byte aligned");
    if (!aligned(beta, 4) || !aligned(cu_seqlens, 4))
        return fail(KDA_ERR_INVALID_ARG, "beta and cu_seqlens must be 4-byte aligned");
    const size_t nel = (size_t)T * (size_t)H * KDA_HEAD_DIM;
    const size_t ob = nel * 2;
    if (overlaps(out, ob, q, ob) || overlaps(out, ob, k, ob) || overlaps(out, ob, v, ob) ||
        overlaps(out, ob, g, nel * 4) || overlaps(out, ob, beta, (size_t)T * H * 4))
        return fail(KDA_ERR_INVALID_ARG, "out must not alias an input");
    if (final_state) {
        const void *ins[6] = {q, k, v, g, beta, out};
        const size_t insz[6] = {ob, ob, ob, nel * 4, (size_t)T * H * 4, ob};
        for (int i = 0; i < 6; ++i)
            if (overlaps(final_state, state_bytes, ins[i], insz[i]))
                return fail(KDA_ERR_INVALID_ARG, "final_state must not alias an input or out");
    }
    int dev = -1;
    kda_status s = check_device(&dev);
    if (s != KDA_OK) return s;
    int *status = nullptr;
    s = status_ptr(dev, &status);
    if (s != KDA_OK) return s;
    // one CTA per (document, head) in both kernels
    const cudaStream_t st = static_cast<cudaStream_t>(stream);
    cudaError_t e = which == FwdKernel::kChunk
                        ? kda::launch_fwd_pipe(q, k, v, g, beta, cu_seqlens, n_docs, T, H, initial_state,
                                               final_state, out, status, st)
                        : kda::launch_fwd_recurrent(q, k, v, g, beta, cu_seqlens, n_docs, T, H, initial_state,
                                                    final_state, out, status, st);
    if (e != cudaSuccess) return fail(KDA_ERR_CUDA, "kernel launch: %s", cudaGetErrorString(e));
    return KDA_OK;
}

}  // namespace

extern "C" {

kda_status kda_chunk_fwd_state(const uint16_t *q, const uint16_t *k, const uint16_t *v, const float *g,
                               const float *beta, const int32_t *cu_seqlens, int n_docs, int64_t T, int H,
                               const float *initial_state, float *final_state, uint16_t *out, void *stream) {
    return fwd_common(FwdKernel::kChunk, q, k, v, g, beta, cu_seqlens, n_docs, T, H, initial_state, final_state,
                      out, stream);
}

kda_status kda_recurrent_fwd(const uint16_t *q, const uint16_t *k, const uint16_t *v, const float *g,
                             const float *beta, const int32_t *cu_seqlens, int n_docs, int64_t T, int H,
                             const float *initial_state, float *final_state, uint16_t *out, void *stream) {
    return fwd_common(FwdKernel::kRecurrent, q, k, v, g, beta, cu_seqlens, n_docs, T, H, initial_state,
                      final_state, out, stream);
}

// Device copies of kda_chunk_fwd_host: q, k, v, out (bf16), g (fp32), beta (fp32), cu_seqlens (int32),
// each starting on a 256-byte boundary.
size_t kda_chunk_fwd_host_workspace_size(int n_docs, int64_t T, int H) {
    if (n_docs < 1 || H < 1 || T < 0) return 0;
    auto up = [](size_t x) { return (x + 255) & ~(size_t)255; };
    const size_t nel = (size_t)T * (size_t)H * KDA_HEAD_DIM;
    return 4 * up(nel * 2) + up(nel * 4) + up((size_t)T * H * 4) + up(((size_t)n_docs + 1) * 4);
}

kda_status kda_chunk_fwd_host(const uint16_t *q, const uint16_t *k, const uint16_t *v, const float *g,
                              const float *beta, const int32_t *cu_seqlens, int n_docs, int64_t T, int H,
                              uint16_t *out, void *workspace, size_t workspace_bytes, void *stream) {
    g_err[0] = '\0';
    if (n_docs < 1) return fail(KDA_ERR_INVALID_ARG, "n_docs must be >= 1 (got %d)", n_docs);
    if (H < 1) return fail(KDA_ERR_INVALID_ARG, "H must be >= 1 (got %d)", H);
    if (T < 0) return fail(KDA_ERR_INVALID_ARG, "T must be >= 0 (got %lld)", (long long)T);
    if (T > (int64_t)INT32_MAX) return fail(KDA_ERR_INVALID_ARG, "T must fit int32 (cu_seqlens is int32)");
    if (!cu_seqlens) return fail(KDA_ERR_INVALID_ARG, "cu_seqlens is NULL");
    if (T == 0) return KDA_OK;
    if (!q || !k || !v || !g || !beta || !out) return fail(KDA_ERR_INVALID_ARG, "a tensor pointer is NULL");
    if (!workspace || !aligned(workspace, 256))
        return fail(KDA_ERR_INVALID_ARG, "workspace must be a 256-byte aligned device buffer");
    const size_t need = kda_chunk_fwd_host_workspace_size(n_docs, T, H);
    if (workspace_bytes < need)
        return fail(KDA_ERR_INVALID_ARG, "workspace too small: %zu bytes given, %zu needed", workspace_bytes, need);
    int dev = -1;
    kda_status s = check_device(&dev);
    if (s != KDA_OK) return s;
    auto up = [](size_t x) { return (x + 255) & ~(size_t)255; };
    const size_t nel = (size_t)T * (size_t)H * KDA_HEAD_DIM;
    uint8_t *w = static_cast<uint8_t *>(workspace);
    uint16_t *dq = reinterpret_cast<uint16_t *>(w);
    uint16_t *dk = reinterpret_cast<uint16_t *>(w + up(nel * 2));
    uint16_t *dv = reinterpret_cast<uint16_t *>(w + 2 * up(nel * 2));
    uint16_t *dout = reinterpret_cast<uint16_t *>(w + 3 * up(nel * 2));
    float *dg = reinterpret_cast<float *>(w + 4 * up(nel * 2));
    float *dbeta = reinterpret_cast<float *>(w + 4 * up(nel * 2) + up(nel * 4));
    int32_t *dcu = reinterpret_cast<int32_t *>(w + 4 * up(nel * 2) + up(nel * 4) + up((size_t)T * H * 4));
    const cudaStream_t st = static_cast<cudaStream_t>(stream);
    struct Copy {
        void *dst;
        const void *src;
        size_t bytes;
    } const ins[6] = {{dq, q, nel * 2}, {dk, k, nel * 2}, {dv, v, nel * 2}, {dg, g, nel * 4},
                      {dbeta, beta, (size_t)T * H * 4}, {dcu, cu_seqlens, ((size_t)n_docs + 1) * 4}};
    for (const Copy &c : ins) {
        const cudaError_t e = cudaMemcpyAsync(c.dst, c.src, c.bytes, cudaMemcpyHostToDevice, st);
        if (e != cudaSuccess) return fail(KDA_ERR_CUDA, "host-to-device copy: %s", cudaGetErrorString(e));
    }
    s = kda_chunk_fwd(dq, dk, dv, dg, dbeta, dcu, n_docs, T, H, dout, stream);
    if (s != KDA_OK) return s;
    const cudaError_t e = cudaMemcpyAsync(out, dout, nel * 2, cudaMemcpyDeviceToHost, st);
    if (e != cudaSuccess) return fail(KDA_ERR_CUDA, "device-to-host copy: %s", cudaGetErrorString(e));
    return KDA_OK;
}

kda_status kda_chunk_fwd(const uint16_t *q, const uint16_t *k, const uint16_t *v, const float *g,
                         const float *beta, const int32_t *cu_seqlens, int n_docs, int64_t T, int H,
                         uint16_t *out, void *stream) {
    return kda_chunk_fwd_state(q, k, v, g, beta, cu_seqlens, n_docs, T, H, nullptr, nullptr, out, stream);
}

size_t kda_chunk_bwd_workspace_size(int n_docs, int64_t T, int H) {
    if (n_docs < 1 || H < 1 || T < 0) return 0;
    return kda::bwd_workspace_floats(n_docs, T, H) * sizeof(float);
}

kda_status kda_chunk_bwd(const uint16_t *q, const uint16_t *k, const uint16_t *v, const float *g,
                         const float *beta, const int32_t *cu_seqlens, int n_docs, int64_t T, int H,
                         const uint16_t *dout, uint16_t *dq, uint16_t *dk, uint16_t *dv, float *dg,
                         float *dbeta, void *workspace, size_t workspace_bytes, void *stream) {
    g_err[0] = '\0';
    if (n_docs < 1) return fail(KDA_ERR_INVALID_ARG, "n_docs must be >= 1 (got %d)", n_docs);
    if (H < 1) return fail(KDA_ERR_INVALID_ARG, "H must be >= 1 (got %d)", H);
    if (T < 0) return fail(KDA_ERR_INVALID_ARG, "T must be >= 0 (got %lld)", (long long)T);
    if (T > (int64_t)INT32_MAX) return fail(KDA_ERR_INVALID_ARG, "T must fit int32 (cu_seqlens is int32)");
    if (!cu_seqlens) return fail(KDA_ERR_INVALID_ARG, "cu_seqlens is NULL");
    if (T == 0) return KDA_OK;
    if (!q || !k || !v || !g || !beta || !dout || !dq || !dk || !dv || !dg || !dbeta)
        return fail(KDA_ERR_INVALID_ARG, "a tensor pointer is NULL");
    if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(g, 16) || !aligned(dout, 16) ||
        !aligned(dq, 16) || !aligned(dk, 16) || !aligned(dv, 16) || !aligned(dg, 16))
        return fail(KDA_ERR_INVALID_ARG, "q, k, v, g, dout, dq, dk, dv and dg must be 16-byte aligned");
    if (!aligned(beta, 4) || !aligned(cu_seqlens, 4) || !aligned(dbeta, 4))
        return fail(KDA_ERR_INVALID_ARG, "beta, dbeta and cu_seqlens must be 4-byte aligned");
    if (!workspace || !aligned(workspace, 16))
        return fail(KDA_ERR_INVALID_ARG, "workspace must be a 16-byte aligned device buffer");
    const size_t need = kda_chunk_bwd_workspace_size(n_docs, T, H);
    if (workspace_bytes < need)
        return fail(KDA_ERR_INVALID_ARG, "workspace too small: %zu bytes given, %zu needed", workspace_bytes, need);
    const size_t nel = (size_t)T * (size_t)H * KDA_HEAD_DIM;
    const void *ins[7] = {q, k, v, dout, g, beta, workspace};
    const size_t insz[7] = {nel * 2, nel * 2, nel * 2, nel * 2, nel * 4, (size_t)T * H * 4, need};
    const void *outs[5] = {dq, dk, dv, dg, dbeta};
    const size_t outsz[5] = {nel * 2, nel * 2, nel * 2, nel * 4, (size_t)T * H * 4};
    for (int i = 0; i < 5; ++i) {
        for (int j = 0; j < 7; ++j)
            if (overlaps(outs[i], outsz[i], ins[j], insz[j]))
                return fail(KDA_ERR_INVALID_ARG, "gradient outputs must not alias an input or the workspace");
        for (int j = i + 1; j < 5; ++j)
            if (overlaps(outs[i], outsz[i], outs[j], outsz[j]))
                return fail(KDA_ERR_INVALID_ARG, "gradient outputs must not alias each other");
    }
    if ((int64_t)n_docs * H > (int64_t)INT32_MAX) return fail(KDA_ERR_INVALID_ARG, "n_docs * H too large");
    int dev = -1;
    kda_status s = check_device(&dev);
    if (s != KDA_OK) return s;
    int *status = nullptr;
    s = status_ptr(dev, &status);
    if (s != KDA_OK) return s;
    cudaError_t e = kda::launch_bwd(q, k, v, g, beta, cu_seqlens, n_docs, T, H, dout, dq, dk, dv, dg, dbeta,
                                    static_cast<float *>(workspace), status, static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return fail(KDA_ERR_CUDA, "kernel launch: %s", cudaGetErrorString(e));
    return KDA_OK;
}

kda_status kda_wait_selftest(void *stream) {
    g_err[0] = '\0';
    int dev = -1;
    kda_status s = check_device(&dev);
    if (s != KDA_OK) return s;
    int *status = nullptr;
    s = status_ptr(dev, &status);
    if (s != KDA_OK) return s;
    cudaError_t e = kda::launch_wait_selftest(status, 20000000LL, static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return fail(KDA_ERR_CUDA, "self-test launch: %s", cudaGetErrorString(e));
    return KDA_OK;
}

kda_status kda_device_status(void *stream) {
    g_err[0] = '\0';
    int dev = -1;
    kda_status s = check_device(&dev);
    if (s != KDA_OK) return s;
    int *status = nullptr;
    s = status_ptr(dev, &status);
    if (s != KDA_OK) return s;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    int h = 0;
    const int zero = 0;
    cudaError_t e = cudaMemcpyAsync(&h, status, sizeof(int), cudaMemcpyDeviceToHost, st);
    if (e == cudaSuccess) e = cudaMemcpyAsync(status, &zero, sizeof(int), cudaMemcpyHostToDevice, st);
    if (e == cudaSuccess) e = cudaStreamSynchronize(st);
    if (e != cudaSuccess) return fail(KDA_ERR_CUDA, "device status read: %s", cudaGetErrorString(e));
    if (h == kda::kStatusBadSeqlens) return fail(KDA_ERR_BAD_SEQLENS, "cu_seqlens malformed (seen on device)");
    if (h == kda::kStatusTimeout) return fail(KDA_ERR_TIMEOUT, "a device-side wait timed out");
    return KDA_OK;
}

}  // extern "C"
