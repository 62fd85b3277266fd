// kda_long.cu -- the forward of one long document, its chunk chain split into segments.
//
// The pipelined kernel runs one CTA per (document, head) chain, so a single document with H heads
// keeps only H SMs busy and its time is the length of its serial chunk chain.  The recurrence is
// affine in the state: over a segment of tokens,
//
//   S_out = M S_in + N,   M = A_L ... A_1,  A_t = (I - beta_t k^_t k^_t^T) Diag(e^{g_t}),
//
// where N is the segment run from the zero state and M the same run with v = 0 from the identity
// state (its rows and columns are key channels).  So the document is cut into P segments at chunk
// boundaries and run in three stages, each with at most T/P tokens per chain:
//   1. N_p for segments 0..P-2 (segment 0 from the initial state; its outputs are final), and at
//      the same time, on a second stream, M_p for the middle segments 1..P-2;
//   2. the hand-off, in fp32: S_in(1) = N_0, S_in(p+1) = M_p S_in(p) + N_p;
//   3. segments 1..P-1 again, from their entering states, writing their outputs and the final
//      state.
// Every pass is the pipelined kernel on a cu_seqlens table whose "documents" are segments.
//
// The state hand-off between pieces of one sequence is how the kimi_k3 model page runs KDA under
// context parallelism (KimiDeltaAttention._forward_with_cp: the recurrent state is passed from
// one shard to the next); the transition map lets the pieces run concurrently on one GPU instead
// of one after another.
#include <cuda_runtime.h>
#include <stdarg.h>
#include <stdint.h>
#include <stdio.h>

#include <mutex>

#include "../../include/kda.h"
#include "kda_internal.h"

namespace kda {
namespace longdoc {

constexpr int D = KDA_HEAD_DIM;
constexpr size_t kStateFloats = (size_t)D * D;
constexpr int kMaxSegments = 16;
constexpr int kMinChunksPerSegment = 8;

// Segment p covers chunks [floor(n p / P), floor(n (p + 1) / P)) of the document's n chunks.
int64_t boundary(int64_t T, int P, int p) {
    const int64_t n = (T + 63) / 64;
    return p >= P ? T : 64 * ((n * p) / P);
}

// Workspace carve-up (byte offsets, each 256-byte aligned).
struct Layout {
    size_t tables, sin, nst, mst, ident, fst, vzero, mout, total;
};

size_t up256(size_t x) { return (x + 255) & ~(size_t)255; }

Layout layout(int64_t T, int H, int P) {
    Layout l{};
    size_t off = 0;
    auto take = [&](size_t bytes) {
        const size_t at = off;
        off += up256(bytes);
        return at;
    };
    const size_t st = kStateFloats * sizeof(float) * (size_t)H;   // one state per head
    const int mid = P >= 3 ? P - 2 : 0;
    const int64_t mid_tokens = P >= 3 ? boundary(T, P, P - 1) - boundary(T, P, 1) : 0;
    l.tables = take(3 * (kMaxSegments + 1) * sizeof(int32_t));
    l.sin = take(P >= 2 ? st * (size_t)(P - 1) : 0);
    l.nst = take(P >= 2 ? st * (size_t)(P - 1) : 0);
    l.fst = take(P >= 2 ? st * (size_t)(P - 1) : 0);
    l.mst = take(st * (size_t)mid);
    l.ident = take(st * (size_t)mid);
    l.vzero = take((size_t)mid_tokens * H * D * sizeof(uint16_t));
    l.mout = take((size_t)mid_tokens * H * D * sizeof(uint16_t));
    l.total = off;
    return l;
}

// The three cu_seqlens tables (N pass, M pass, final pass), passed by value.
struct Tables {
    int32_t n[3];
    int32_t v[3][kMaxSegments + 1];
};

__global__ void write_tables(Tables t, int32_t *dst) {
    const int i = threadIdx.x;
#pragma unroll
    for (int j = 0; j < 3; ++j)
        if (i < t.n[j]) dst[j * (kMaxSegments + 1) + i] = t.v[j][i];
}

// count states of 128 x 128: the identity.
__global__ void write_identity(float *dst, size_t count) {
    const size_t total = count * kStateFloats;
    for (size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x; i < total; i += (size_t)gridDim.x * blockDim.x) {
        const size_t e = i % kStateFloats;
        dst[i] = (e / D == e % D) ? 1.f : 0.f;
    }
}

// The hand-off for one head per CTA: sin[0] = nst[0]; sin[s] = mst[s-1] sin[s-1] + nst[s] for
// s = 1..P-2 (slot s of nst/sin belongs to segment s of the N pass / the state entering segment
// s+1; slot s-1 of mst is segment s of the M pass).  States are S[c][v] with c the key channel, so
// the product contracts M's column index with S's row index.  Thread (tr, tc) of a 16 x 16 grid
// owns rows 8 tr.. and columns 8 tc..; M is staged transposed (padded pitch) so that both
// operands are read as float4 rows.
constexpr int kHandThreads = 256;
constexpr int kMtPitch = D + 4;
constexpr size_t kHandSmem = ((size_t)D * kMtPitch + (size_t)D * D) * sizeof(float);

__global__ void __launch_bounds__(kHandThreads) hand_off(const float *__restrict__ nst, const float *__restrict__ mst,
                                                         float *__restrict__ sin, int H, int P) {
    extern __shared__ float4 smem4[];
    float *Mt = reinterpret_cast<float *>(smem4);
    float *S = Mt + D * kMtPitch;
    const int h = blockIdx.x, tid = threadIdx.x;
    const size_t hs = (size_t)h * kStateFloats;
    for (int i = tid; i < D * D / 4; i += kHandThreads) {
        const float4 x = reinterpret_cast<const float4 *>(nst + hs)[i];
        reinterpret_cast<float4 *>(S)[i] = x;
        reinterpret_cast<float4 *>(sin + hs)[i] = x;
    }
    const int r0 = 8 * (tid >> 4), c0 = 8 * (tid & 15);
    for (int s = 1; s <= P - 2; ++s) {
        const float *M = mst + ((size_t)(s - 1) * H + h) * kStateFloats;
        const float *N = nst + ((size_t)s * H + h) * kStateFloats;
        float *out = sin + ((size_t)s * H + h) * kStateFloats;
        for (int i = tid; i < D * D; i += kHandThreads) Mt[(i % D) * kMtPitch + i / D] = M[i];
        __syncthreads();   // Mt staged; S holds the previous entering state
        float acc[8][8];
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            const float4 a = *reinterpret_cast<const float4 *>(N + (size_t)(r0 + i) * D + c0);
            const float4 b = *reinterpret_cast<const float4 *>(N + (size_t)(r0 + i) * D + c0 + 4);
            acc[i][0] = a.x, acc[i][1] = a.y, acc[i][2] = a.z, acc[i][3] = a.w;
            acc[i][4] = b.x, acc[i][5] = b.y, acc[i][6] = b.z, acc[i][7] = b.w;
        }
#pragma unroll 4
        for (int j = 0; j < D; ++j) {
            const float4 m0 = *reinterpret_cast<const float4 *>(Mt + j * kMtPitch + r0);
            const float4 m1 = *reinterpret_cast<const float4 *>(Mt + j * kMtPitch + r0 + 4);
            const float4 s0 = *reinterpret_cast<const float4 *>(S + j * D + c0);
            const float4 s1 = *reinterpret_cast<const float4 *>(S + j * D + c0 + 4);
            const float m[8] = {m0.x, m0.y, m0.z, m0.w, m1.x, m1.y, m1.z, m1.w};
            const float sv[8] = {s0.x, s0.y, s0.z, s0.w, s1.x, s1.y, s1.z, s1.w};
#pragma unroll
            for (int i = 0; i < 8; ++i)
#pragma unroll
                for (int c = 0; c < 8; ++c) acc[i][c] = fmaf(m[i], sv[c], acc[i][c]);
        }
        __syncthreads();   // every read of Mt and S is done
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            const float4 a = make_float4(acc[i][0], acc[i][1], acc[i][2], acc[i][3]);
            const float4 b = make_float4(acc[i][4], acc[i][5], acc[i][6], acc[i][7]);
            *reinterpret_cast<float4 *>(S + (r0 + i) * D + c0) = a;
            *reinterpret_cast<float4 *>(S + (r0 + i) * D + c0 + 4) = b;
            *reinterpret_cast<float4 *>(out + (size_t)(r0 + i) * D + c0) = a;
            *reinterpret_cast<float4 *>(out + (size_t)(r0 + i) * D + c0 + 4) = b;
        }
    }
}

// The second stream and its two events, created once per device.
struct Aux {
    cudaStream_t stream = nullptr;
    cudaEvent_t fork = nullptr, join = nullptr;
};
constexpr int kMaxDevices = 64;
Aux g_aux[kMaxDevices];
std::mutex g_aux_mu;   // held from the aux lookup to the last enqueue of a call

cudaError_t aux_for(int dev, Aux **out) {
    Aux &a = g_aux[dev];
    if (!a.stream) {
        cudaError_t e = cudaStreamCreateWithFlags(&a.stream, cudaStreamNonBlocking);
        if (e == cudaSuccess) e = cudaEventCreateWithFlags(&a.fork, cudaEventDisableTiming);
        if (e == cudaSuccess) e = cudaEventCreateWithFlags(&a.join, cudaEventDisableTiming);
        if (e != cudaSuccess) {
            if (a.join) cudaEventDestroy(a.join);
            if (a.fork) cudaEventDestroy(a.fork);
            if (a.stream) cudaStreamDestroy(a.stream);
            a = Aux{};
            return e;
        }
    }
    *out = &a;
    return cudaSuccess;
}

}  // namespace longdoc
}  // namespace kda

namespace {

using namespace kda::longdoc;

bool aligned(const void *p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

bool overlaps(const void *a, size_t na, const void *b, size_t nb) {
    if (!a || !b) return false;
    const uintptr_t x = reinterpret_cast<uintptr_t>(a), y = reinterpret_cast<uintptr_t>(b);
    return x < y + nb && y < x + na;
}

kda_status fail(kda_status s, const char *fmt, ...) __attribute__((format(printf, 2, 3)));
kda_status fail(kda_status s, const char *fmt, ...) {
    char buf[512];
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(buf, sizeof(buf), fmt, ap);
    va_end(ap);
    return (kda_status)kda::set_last_error((int)s, buf);
}

kda_status cuda_fail(const char *what, cudaError_t e) {
    return fail(KDA_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

}  // namespace

extern "C" {

int kda_chunk_fwd_long_segments(int64_t T, int H, int num_sms) {
    if (T <= 0 || H < 1 || num_sms < 1) return 1;
    const int64_t n = (T + 63) / 64;
    int best = 1;
    for (int P = 3; P <= kMaxSegments; ++P) {
        if ((int64_t)(2 * P - 3) * H > num_sms) break;   // stage 1 must fit one wave, one CTA per SM
        if (n / P < kMinChunksPerSegment) break;
        best = P;
    }
    return best;
}

size_t kda_chunk_fwd_long_workspace_size(int64_t T, int H, int segments) {
    if (T < 0 || H < 1 || segments < 1 || segments > kMaxSegments) return 0;
    return layout(T, H, segments).total;
}

kda_status kda_chunk_fwd_long(const uint16_t *q, const uint16_t *k, const uint16_t *v, const float *g,
                              const float *beta, int64_t T, int H, int segments, const float *initial_state,
                              float *final_state, uint16_t *out, void *workspace, size_t workspace_bytes,
                              void *stream) {
    kda::set_last_error(KDA_OK, "");
    if (H < 1) return fail(KDA_ERR_INVALID_ARG, "H must be >= 1 (got %d)", H);
    if (T < 0) return fail(KDA_ERR_INVALID_ARG, "T must be >= 0 (got %lld)", (long long)T);
    if (T > (int64_t)INT32_MAX) return fail(KDA_ERR_INVALID_ARG, "T must fit int32");
    const int64_t nch = (T + 63) / 64;
    if (segments < 1 || segments > kMaxSegments)
        return fail(KDA_ERR_INVALID_ARG, "segments must be in [1, %d] (got %d)", kMaxSegments, segments);
    if (T > 0 && segments > nch)
        return fail(KDA_ERR_INVALID_ARG, "segments (%d) exceeds the document's %lld chunks", segments,
                    (long long)nch);
    if ((int64_t)segments * H > (int64_t)INT32_MAX) return fail(KDA_ERR_INVALID_ARG, "segments * H too large");
    const int P = segments;
    const size_t st_bytes = kStateFloats * sizeof(float) * (size_t)H;
    if ((initial_state && !aligned(initial_state, 16)) || (final_state && !aligned(final_state, 16)))
        return fail(KDA_ERR_INVALID_ARG, "initial_state and final_state must be 16-byte aligned");
    if (initial_state && final_state && initial_state != final_state &&
        overlaps(initial_state, st_bytes, final_state, st_bytes))
        return fail(KDA_ERR_INVALID_ARG, "initial_state and final_state must be the same buffer or disjoint");
    const cudaStream_t st = static_cast<cudaStream_t>(stream);
    int dev = -1;
    int *status = nullptr;
    if (T == 0) {
        if (!final_state || final_state == initial_state) return KDA_OK;
        kda_status s = (kda_status)kda::device_context(&dev, &status);
        if (s != KDA_OK) return s;
        cudaError_t e = initial_state ? cudaMemcpyAsync(final_state, initial_state, st_bytes, cudaMemcpyDeviceToDevice, st)
                                      : cudaMemsetAsync(final_state, 0, st_bytes, st);
        return e == cudaSuccess ? KDA_OK : cuda_fail("final state copy", e);
    }
    if (!q || !k || !v || !g || !beta || !out) return fail(KDA_ERR_INVALID_ARG, "a tensor pointer is NULL");
    if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(g, 16) || !aligned(out, 16))
        return fail(KDA_ERR_INVALID_ARG, "q, k, v, g and out must be 16-byte aligned");
    if (!aligned(beta, 4)) return fail(KDA_ERR_INVALID_ARG, "beta must be 4-byte aligned");
    const size_t nel = (size_t)T * (size_t)H * D;
    const size_t ob = nel * 2;
    const void *ins[5] = {q, k, v, g, beta};
    const size_t insz[5] = {ob, ob, ob, nel * 4, (size_t)T * H * 4};
    for (int i = 0; i < 5; ++i)
        if (overlaps(out, ob, ins[i], insz[i])) return fail(KDA_ERR_INVALID_ARG, "out must not alias an input");
    if (final_state) {
        for (int i = 0; i < 5; ++i)
            if (overlaps(final_state, st_bytes, ins[i], insz[i]))
                return fail(KDA_ERR_INVALID_ARG, "final_state must not alias an input or out");
        if (overlaps(final_state, st_bytes, out, ob))
            return fail(KDA_ERR_INVALID_ARG, "final_state must not alias an input or out");
    }
    const Layout lay = layout(T, H, P);
    if (!workspace || !aligned(workspace, 256))
        return fail(KDA_ERR_INVALID_ARG, "workspace must be a 256-byte aligned device buffer");
    if (workspace_bytes < lay.total)
        return fail(KDA_ERR_INVALID_ARG, "workspace too small: %zu bytes given, %zu needed", workspace_bytes,
                    lay.total);
    for (int i = 0; i < 5; ++i)
        if (overlaps(workspace, lay.total, ins[i], insz[i]))
            return fail(KDA_ERR_INVALID_ARG, "workspace must not alias an argument");
    if (overlaps(workspace, lay.total, out, ob) || overlaps(workspace, lay.total, initial_state, st_bytes) ||
        overlaps(workspace, lay.total, final_state, st_bytes))
        return fail(KDA_ERR_INVALID_ARG, "workspace must not alias an argument");
    {
        kda_status s = (kda_status)kda::device_context(&dev, &status);
        if (s != KDA_OK) return s;
    }

    uint8_t *ws = static_cast<uint8_t *>(workspace);
    int32_t *tab = reinterpret_cast<int32_t *>(ws + lay.tables);
    int32_t *cuN = tab, *cuM = tab + (kMaxSegments + 1), *cuF = tab + 2 * (kMaxSegments + 1);
    int64_t b[kMaxSegments + 1];
    for (int p = 0; p <= P; ++p) b[p] = boundary(T, P, p);
    Tables t{};
    if (P == 1) {
        t.n[0] = 2;
        t.v[0][0] = 0;
        t.v[0][1] = (int32_t)T;
    } else {
        t.n[0] = P;                                   // N pass: segments 0..P-2, tokens [0, b[P-1])
        for (int p = 0; p < P; ++p) t.v[0][p] = (int32_t)b[p];
        t.n[1] = P - 1;                               // M pass: segments 1..P-2, tokens [b1, b[P-1])
        for (int p = 1; p < P; ++p) t.v[1][p - 1] = (int32_t)(b[p] - b[1]);
        t.n[2] = P;                                   // final pass: segments 1..P-1, tokens [b1, T)
        for (int p = 1; p <= P; ++p) t.v[2][p - 1] = (int32_t)(b[p] - b[1]);
    }
    cudaError_t e;
    write_tables<<<1, 32, 0, st>>>(t, tab);
    if ((e = cudaGetLastError()) != cudaSuccess) return cuda_fail("table launch", e);
    if (P == 1) {
        e = kda::launch_fwd_pipe(q, k, v, g, beta, cuN, 1, T, H, initial_state, final_state, out, status, st);
        return e == cudaSuccess ? KDA_OK : cuda_fail("kernel launch", e);
    }

    float *sin = reinterpret_cast<float *>(ws + lay.sin);
    float *nst = reinterpret_cast<float *>(ws + lay.nst);
    float *fst = reinterpret_cast<float *>(ws + lay.fst);
    float *mst = reinterpret_cast<float *>(ws + lay.mst);
    float *ident = reinterpret_cast<float *>(ws + lay.ident);
    uint16_t *vzero = reinterpret_cast<uint16_t *>(ws + lay.vzero);
    uint16_t *mout = reinterpret_cast<uint16_t *>(ws + lay.mout);
    const size_t row = (size_t)H * D;                  // elements per token
    const size_t o1 = (size_t)b[1] * row;              // first token of segment 1
    const int64_t Tn = b[P - 1], Tm = b[P - 1] - b[1], Tf = T - b[1];

    std::lock_guard<std::mutex> lock(g_aux_mu);
    Aux *aux = nullptr;
    const bool have_mid = P >= 3;
    if (have_mid) {
        if ((e = aux_for(dev, &aux)) != cudaSuccess) return cuda_fail("second stream", e);
    }
    // the N pass starts segment 0 from the initial state and the others from zero
    const float *h0n = nullptr;
    if (initial_state) {
        if ((e = cudaMemcpyAsync(sin, initial_state, st_bytes, cudaMemcpyDeviceToDevice, st)) != cudaSuccess ||
            (e = cudaMemsetAsync(sin + (size_t)H * kStateFloats, 0, st_bytes * (size_t)(P - 2), st)) != cudaSuccess)
            return cuda_fail("initial state copy", e);
        h0n = sin;
    }
    if (have_mid) {
        // stage 1b on the second stream, after the tables (and any earlier use of the workspace)
        if ((e = cudaEventRecord(aux->fork, st)) != cudaSuccess ||
            (e = cudaStreamWaitEvent(aux->stream, aux->fork, 0)) != cudaSuccess)
            return cuda_fail("stream fork", e);
        const char *what = "zero values";
        e = cudaMemsetAsync(vzero, 0, (size_t)Tm * row * sizeof(uint16_t), aux->stream);
        if (e == cudaSuccess) {
            what = "identity launch";
            const size_t n_floats = (size_t)(P - 2) * H * kStateFloats;    // about 4 per thread
            write_identity<<<(unsigned)((n_floats / 4 + 255) / 256), 256, 0, aux->stream>>>(ident,
                                                                                          (size_t)(P - 2) * H);
            e = cudaGetLastError();
        }
        if (e == cudaSuccess) {
            what = "transition pass launch";
            e = kda::launch_fwd_pipe(q + o1, k + o1, vzero, g + o1, beta + (size_t)b[1] * H, cuM, P - 2, Tm, H,
                                     ident, mst, mout, status, aux->stream);
        }
        const cudaError_t ej = cudaEventRecord(aux->join, aux->stream);
        if (e != cudaSuccess || ej != cudaSuccess) {
            // join even after a failure, so that no work of this call stays unordered with `stream`
            if (ej == cudaSuccess) cudaStreamWaitEvent(st, aux->join, 0);
            return e != cudaSuccess ? cuda_fail(what, e) : cuda_fail("stream join", ej);
        }
    }
    // stage 1a: N_p of segments 0..P-2, at the same time as the M pass; segment 0's outputs are
    // final.  `stream` joins the second stream after it (also when the launch failed).
    e = kda::launch_fwd_pipe(q, k, v, g, beta, cuN, P - 1, Tn, H, h0n, nst, out, status, st);
    const cudaError_t ew = have_mid ? cudaStreamWaitEvent(st, aux->join, 0) : cudaSuccess;
    if (e != cudaSuccess) return cuda_fail("segment pass launch", e);
    if (ew != cudaSuccess) return cuda_fail("stream join", ew);
    // stage 2: entering states of segments 1..P-1
    static bool smem_set[kMaxDevices] = {false};
    if (!smem_set[dev]) {
        if ((e = cudaFuncSetAttribute(hand_off, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kHandSmem)) !=
            cudaSuccess)
            return cuda_fail("hand-off attribute", e);
        smem_set[dev] = true;
    }
    hand_off<<<H, kHandThreads, kHandSmem, st>>>(nst, mst, sin, H, P);
    if ((e = cudaGetLastError()) != cudaSuccess) return cuda_fail("hand-off launch", e);
    // stage 3: segments 1..P-1 from their entering states
    e = kda::launch_fwd_pipe(q + o1, k + o1, v + o1, g + o1, beta + (size_t)b[1] * H, cuF, P - 1, Tf, H, sin,
                             final_state ? fst : nullptr, out + o1, status, st);
    if (e != cudaSuccess) return cuda_fail("final pass launch", e);
    if (final_state &&
        (e = cudaMemcpyAsync(final_state, fst + (size_t)(P - 2) * H * kStateFloats, st_bytes,
                             cudaMemcpyDeviceToDevice, st)) != cudaSuccess)
        return cuda_fail("final state copy", e);
    return KDA_OK;
}

}  // extern "C"
