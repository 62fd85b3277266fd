// kda_split.cu -- the forward with long documents cut into segments that run side by side.
//
// The pipelined kernel runs one CTA per (document, head) chain, so a few long documents keep few
// SMs busy and the call takes as long as the longest serial chunk chain.  The recurrence is
// affine in the state: over a segment of tokens,
//
//   S_out = M S_in + N,   M = A_L ... A_1,  A_t = (I - beta_t k^_t k^_t^T) Diag(e^{g_t}),
//
// where N is the segment run from the zero state and M the same run with v = 0 from the identity
// state (its rows and columns are key channels).  A document cut into P segments at chunk
// boundaries runs in three stages, each chain at most ceil(n / P) chunks long:
//   1. N_p for segments 0..P-2 (segment 0 from the document's initial state; its outputs are
//      final) together with the documents that are not cut, and at the same time, on a second
//      stream, M_p for the middle segments 1..P-2 (a transition pass: no v, no outputs);
//   2. the hand-off, in fp32: S_in(1) = N_0, S_in(p+1) = M_p S_in(p) + N_p;
//   3. segments 1..P-1 again, from their entering states, writing their outputs and the
//      document's final state.
// A planner kernel reads cu_seqlens on the device and writes the three segment tables, so the host
// never waits for the document lengths.  It gives the stage-1 CTAs one wave of SMs: documents start
// whole (one chain per head each), and while SMs remain the document with the longest current chain
// gets more segments (P = 1 -> 3 -> 4 ...; a cut document holds 2 P - 3 chains per head in stage 1),
// keeping at least 8 chunks per segment.
//
// The state hand-off between pieces of one sequence is how the kimi_k3 model page runs KDA under
// context parallelism (KimiDeltaAttention._forward_with_cp: the recurrent state is passed from one
// shard to the next); the transition map lets the pieces of one GPU run concurrently instead.
#include <cuda_runtime.h>
#include <stdarg.h>
#include <stdint.h>
#include <stdio.h>

#include <mutex>

#include "../../include/kda.h"
#include "kda_internal.h"

namespace kda {
namespace split {

constexpr int D = KDA_HEAD_DIM;
constexpr size_t kStateFloats = (size_t)D * D;
constexpr int kMaxSegments = 16;
constexpr int kMinChunksPerSegment = 8;
constexpr int kSortMax = 256;       // tables are ordered longest first up to this many entries

// The plan's sizes (host side, before the lengths are known): table capacities and state slots.
struct Caps {
    int n, m, f, hand;   // entries of the N, M and final tables, hand-off records
    int slots;           // workspace states per head
};

// forced_P > 0: one document cut into exactly forced_P segments (kda_chunk_fwd_long)
Caps caps(int n_docs, int H, int num_sms, int forced_P) {
    Caps c{};
    if (forced_P > 0) {
        const int P = forced_P;
        c.n = P;
        c.m = P >= 3 ? P - 2 : 0;
        c.f = P >= 2 ? P - 1 : 0;
        c.hand = P >= 2 ? 1 : 0;
        c.slots = P >= 2 ? 3 * P - 4 : 0;
        return c;
    }
    const int smax = num_sms / H > 1 ? num_sms / H : 1;   // stage-1 chains per head in one wave
    // documents are cut only while stage 1 fits the wave: every cut document adds at least two
    // chains per head, so at most smax / 3 of them, and sum_d (2 P_d - 3) <= smax bounds the segments
    c.n = n_docs + smax;
    c.m = smax;
    c.f = smax;
    c.hand = smax / 3 + 1;
    c.slots = 3 * smax;
    return c;
}

struct Layout {
    size_t counts, tab_n, tab_m, tab_f, hand, states, total;
};

size_t up256(size_t x) { return (x + 255) & ~(size_t)255; }

Layout layout(const Caps &c, int H) {
    Layout l{};
    size_t off = 0;
    auto take = [&](size_t bytes) {
        const size_t at = off;
        off += up256(bytes);
        return at;
    };
    l.counts = take(4 * sizeof(int));
    l.tab_n = take((size_t)c.n * sizeof(int4));
    l.tab_m = take((size_t)c.m * sizeof(int4));
    l.tab_f = take((size_t)c.f * sizeof(int4));
    l.hand = take((size_t)c.hand * sizeof(int4));
    l.states = take((size_t)c.slots * H * kStateFloats * sizeof(float));
    l.total = off;
    return l;
}

struct PlanArgs {
    int n_docs, H, num_sms, forced_P, has_init, has_final;
    int64_t T;
    Caps caps;
};

// longest entries first (stable), for at most kSortMax entries
__device__ void sort_longest_first(int4 *t, int n) {
    if (n > kSortMax) return;
    for (int i = 1; i < n; ++i) {
        const int4 x = t[i];
        int j = i - 1;
        while (j >= 0 && (t[j].y - t[j].x) < (x.y - x.x)) {
            t[j + 1] = t[j];
            --j;
        }
        t[j + 1] = x;
    }
}

// One thread: validate cu_seqlens (NULL means one document [0, T)), choose the segment counts and
// write the tables.  counts = {N entries, M entries, final entries, hand-off records}.  A malformed
// table records KDA_ERR_BAD_SEQLENS and plans nothing.
__global__ void plan_kernel(const int32_t *__restrict__ cu, PlanArgs a, int *counts, int4 *tab_n, int4 *tab_m,
                            int4 *tab_f, int4 *hand, int *status) {
    if (threadIdx.x != 0) return;
    auto cu_at = [&](int d) -> int64_t { return cu ? (int64_t)cu[d] : (d == 0 ? 0 : a.T); };
    counts[0] = counts[1] = counts[2] = counts[3] = 0;
    bool ok = cu_at(0) == 0 && cu_at(a.n_docs) == a.T;
    for (int d = 0; ok && d < a.n_docs; ++d) ok = cu_at(d) <= cu_at(d + 1);
    if (!ok) {
        atomicExch(status, kStatusBadSeqlens);
        return;
    }
    // segment counts: P = 1 everywhere, then cut the document with the longest chain while the
    // stage-1 wave has room (a document cut into P segments holds 2 P - 3 stage-1 chains per head)
    int np = 0;   // documents with P > 1 so far (bounded by the hand-off capacity)
    auto chunks = [&](int d) -> int64_t { return (cu_at(d + 1) - cu_at(d) + 63) / 64; };
    // P_d kept in tab_m's space temporarily is not needed: the counts are recomputed below
    // from a small per-document array (the planner runs for few documents; beyond kSortMax no cuts)
    int Pd[kSortMax];
    const int nd = a.n_docs <= kSortMax ? a.n_docs : 0;
    for (int d = 0; d < nd; ++d) Pd[d] = 1;
    if (a.forced_P > 0) {
        if (nd >= 1) Pd[0] = a.forced_P;
    } else if (nd > 0) {
        int free_slots = (a.num_sms / a.H > 1 ? a.num_sms / a.H : 1) - nd;
        while (free_slots >= 2) {
            int best = -1;
            float best_cost = 0.f;
            for (int d = 0; d < nd; ++d) {
                const float n = (float)chunks(d);
                const float cost = Pd[d] == 1 ? n : 2.f * n / (float)Pd[d];
                if (cost > best_cost) {
                    best_cost = cost;
                    best = d;
                }
            }
            if (best < 0) break;
            const int nxt = Pd[best] == 1 ? 3 : Pd[best] + 1;
            if (nxt > kMaxSegments || chunks(best) / nxt < kMinChunksPerSegment) break;
            if (Pd[best] == 1 && np + 1 > a.caps.hand) break;
            if (Pd[best] == 1) ++np;
            Pd[best] = nxt;
            free_slots -= 2;
        }
    }
    int cn = 0, cm = 0, cf = 0, ch = 0, slot = 0;
    for (int d = 0; d < a.n_docs; ++d) {
        const int init = a.has_init ? kSplitSlotCaller + d : -1;
        const int fin = a.has_final ? kSplitSlotCaller + d : -1;
        const int P = d < nd ? Pd[d] : 1;
        const int64_t s0 = cu_at(d), s1 = cu_at(d + 1);
        if (P == 1) {
            tab_n[cn++] = make_int4((int)s0, (int)s1, init, fin);
            continue;
        }
        const int64_t n = chunks(d);
        auto bnd = [&](int p) -> int64_t { return p >= P ? s1 : s0 + 64 * ((n * p) / P); };
        const int base_n = slot, base_m = base_n + (P - 1), base_s = base_m + (P - 2);
        slot = base_s + (P - 1);
        for (int p = 0; p <= P - 2; ++p) tab_n[cn++] = make_int4((int)bnd(p), (int)bnd(p + 1), p == 0 ? init : -1, base_n + p);
        for (int p = 1; p <= P - 2; ++p) tab_m[cm++] = make_int4((int)bnd(p), (int)bnd(p + 1), -1, base_m + p - 1);
        for (int p = 1; p <= P - 1; ++p)
            tab_f[cf++] = make_int4((int)bnd(p), (int)bnd(p + 1), base_s + p - 1, p == P - 1 ? fin : -1);
        hand[ch++] = make_int4(P, base_n, base_m, base_s);
    }
    sort_longest_first(tab_n, cn);
    sort_longest_first(tab_m, cm);
    sort_longest_first(tab_f, cf);
    counts[0] = cn;
    counts[1] = cm;
    counts[2] = cf;
    counts[3] = ch;
}

// The hand-off of one cut document and head per CTA: sin[0] = nst[0]; sin[p] = mst[p-1] sin[p-1] +
// nst[p] for p = 1..P-2 (nst[p]: segment p's N; mst[p-1]: segment p's M; sin[p]: the state entering
// segment p+1).  States are S[c][v] with c the key channel, so the product contracts M's column
// index with S's row index.  Thread (tr, tc) of a 16 x 16 grid owns rows 8 tr.. and columns 8 tc..;
// M is staged transposed (padded pitch) so that both operands are read as float4 rows.
constexpr int kHandThreads = 256;
constexpr int kMtPitch = D + 4;
constexpr size_t kHandSmem = ((size_t)D * kMtPitch + (size_t)D * D) * sizeof(float);

__global__ void __launch_bounds__(kHandThreads) hand_off(const int4 *__restrict__ hand, const int *__restrict__ counts,
                                                         float *__restrict__ states, int H) {
    extern __shared__ float4 smem4[];
    if ((int)blockIdx.x >= counts[3]) return;
    const int4 rec = hand[blockIdx.x];
    const int P = rec.x, h = blockIdx.y, tid = threadIdx.x;
    auto st = [&](int slot) -> float * { return states + ((size_t)slot * H + h) * kStateFloats; };
    float *Mt = reinterpret_cast<float *>(smem4);
    float *S = Mt + D * kMtPitch;
    {
        const float *n0 = st(rec.y);
        float *s0 = st(rec.w);
        for (int i = tid; i < D * D / 4; i += kHandThreads) {
            const float4 x = reinterpret_cast<const float4 *>(n0)[i];
            reinterpret_cast<float4 *>(S)[i] = x;
            reinterpret_cast<float4 *>(s0)[i] = x;
        }
    }
    const int r0 = 8 * (tid >> 4), c0 = 8 * (tid & 15);
    for (int p = 1; p <= P - 2; ++p) {
        const float *M = st(rec.z + p - 1);
        const float *N = st(rec.y + p);
        float *out = st(rec.w + p);
        for (int i = tid; i < D * D; i += kHandThreads) Mt[(i % D) * kMtPitch + i / D] = M[i];
        __syncthreads();   // Mt staged; S holds the previous entering state
        float acc[8][8];
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            const float4 x = *reinterpret_cast<const float4 *>(N + (size_t)(r0 + i) * D + c0);
            const float4 y = *reinterpret_cast<const float4 *>(N + (size_t)(r0 + i) * D + c0 + 4);
            acc[i][0] = x.x, acc[i][1] = x.y, acc[i][2] = x.z, acc[i][3] = x.w;
            acc[i][4] = y.x, acc[i][5] = y.y, acc[i][6] = y.z, acc[i][7] = y.w;
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
            const float4 x = make_float4(acc[i][0], acc[i][1], acc[i][2], acc[i][3]);
            const float4 y = make_float4(acc[i][4], acc[i][5], acc[i][6], acc[i][7]);
            *reinterpret_cast<float4 *>(S + (r0 + i) * D + c0) = x;
            *reinterpret_cast<float4 *>(S + (r0 + i) * D + c0 + 4) = y;
            *reinterpret_cast<float4 *>(out + (size_t)(r0 + i) * D + c0) = x;
            *reinterpret_cast<float4 *>(out + (size_t)(r0 + i) * D + c0 + 4) = y;
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
bool g_smem_set[kMaxDevices] = {false};
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

}  // namespace split
}  // namespace kda

namespace {

using namespace kda::split;

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

kda_status cuda_fail(const char *what, cudaError_t e) { return fail(KDA_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e)); }

int current_sms() {
    int dev = 0, sms = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return 0;
    if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 0;
    return sms;
}

// The split forward of n_docs documents given by the DEVICE table cu (NULL: one document [0, T)),
// with forced_P > 0 cutting that one document into exactly forced_P segments.
kda_status split_forward(const uint16_t *q, const uint16_t *k, const uint16_t *v, const float *g, const float *beta,
                         const int32_t *cu, int n_docs, int64_t T, int H, int forced_P, const float *initial_state,
                         float *final_state, uint16_t *out, void *workspace, size_t workspace_bytes, void *stream,
                         int num_sms) {
    if (n_docs < 1) return fail(KDA_ERR_INVALID_ARG, "n_docs must be >= 1 (got %d)", n_docs);
    if (H < 1) return fail(KDA_ERR_INVALID_ARG, "H must be >= 1 (got %d)", H);
    if (T < 0) return fail(KDA_ERR_INVALID_ARG, "T must be >= 0 (got %lld)", (long long)T);
    if (T > (int64_t)INT32_MAX) return fail(KDA_ERR_INVALID_ARG, "T must fit int32 (cu_seqlens is int32)");
    if ((int64_t)n_docs * H > (int64_t)INT32_MAX / 2) return fail(KDA_ERR_INVALID_ARG, "n_docs * H too large");
    const size_t st_bytes = kStateFloats * sizeof(float) * (size_t)H * (size_t)n_docs;
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
    if (!aligned(beta, 4) || (cu && !aligned(cu, 4)))
        return fail(KDA_ERR_INVALID_ARG, "beta and cu_seqlens must be 4-byte aligned");
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
    if (num_sms < 1) return fail(KDA_ERR_CUDA, "cannot read the device's SM count");
    const Caps cp = caps(n_docs, H, num_sms, forced_P);
    const Layout lay = layout(cp, H);
    if (!workspace || !aligned(workspace, 256))
        return fail(KDA_ERR_INVALID_ARG, "workspace must be a 256-byte aligned device buffer");
    if (workspace_bytes < lay.total)
        return fail(KDA_ERR_INVALID_ARG, "workspace too small: %zu bytes given, %zu needed", workspace_bytes, lay.total);
    for (int i = 0; i < 5; ++i)
        if (overlaps(workspace, lay.total, ins[i], insz[i]))
            return fail(KDA_ERR_INVALID_ARG, "workspace must not alias an argument");
    if (overlaps(workspace, lay.total, out, ob) || overlaps(workspace, lay.total, initial_state, st_bytes) ||
        overlaps(workspace, lay.total, final_state, st_bytes) ||
        (cu && overlaps(workspace, lay.total, cu, ((size_t)n_docs + 1) * 4)))
        return fail(KDA_ERR_INVALID_ARG, "workspace must not alias an argument");
    {
        kda_status s = (kda_status)kda::device_context(&dev, &status);
        if (s != KDA_OK) return s;
    }
    uint8_t *ws = static_cast<uint8_t *>(workspace);
    int *counts = reinterpret_cast<int *>(ws + lay.counts);
    int4 *tab_n = reinterpret_cast<int4 *>(ws + lay.tab_n);
    int4 *tab_m = reinterpret_cast<int4 *>(ws + lay.tab_m);
    int4 *tab_f = reinterpret_cast<int4 *>(ws + lay.tab_f);
    int4 *hand = reinterpret_cast<int4 *>(ws + lay.hand);
    float *states = reinterpret_cast<float *>(ws + lay.states);

    PlanArgs pa{};
    pa.n_docs = n_docs;
    pa.H = H;
    pa.num_sms = num_sms;
    pa.forced_P = forced_P;
    pa.has_init = initial_state != nullptr;
    pa.has_final = final_state != nullptr;
    pa.T = T;
    pa.caps = cp;
    cudaError_t e;
    plan_kernel<<<1, 32, 0, st>>>(cu, pa, counts, tab_n, tab_m, tab_f, hand, status);
    if ((e = cudaGetLastError()) != cudaSuccess) return cuda_fail("planner launch", e);

    std::lock_guard<std::mutex> lock(g_aux_mu);
    Aux *aux = nullptr;
    const bool have_mid = cp.m > 0;
    if (have_mid && (e = aux_for(dev, &aux)) != cudaSuccess) return cuda_fail("second stream", e);
    if (have_mid) {
        // stage 1b on the second stream, after the planner (and any earlier use of the workspace)
        if ((e = cudaEventRecord(aux->fork, st)) != cudaSuccess ||
            (e = cudaStreamWaitEvent(aux->stream, aux->fork, 0)) != cudaSuccess)
            return cuda_fail("stream fork", e);
        e = kda::launch_fwd_segments(true, q, k, v, g, beta, T, H, tab_m, counts + 1, cp.m, nullptr, nullptr, states,
                                     out, status, aux->stream);
        const cudaError_t ej = cudaEventRecord(aux->join, aux->stream);
        if (e != cudaSuccess || ej != cudaSuccess) {
            // join even after a failure, so that no work of this call stays unordered with `stream`
            if (ej == cudaSuccess) cudaStreamWaitEvent(st, aux->join, 0);
            return e != cudaSuccess ? cuda_fail("transition pass launch", e) : cuda_fail("stream join", ej);
        }
    }
    // stage 1a: whole documents and segments 0..P-2 of the cut ones, at the same time as the
    // transition pass; `stream` joins the second stream after it (also when the launch failed)
    e = kda::launch_fwd_segments(false, q, k, v, g, beta, T, H, tab_n, counts + 0, cp.n, initial_state, final_state,
                                 states, out, status, st);
    const cudaError_t ew = have_mid ? cudaStreamWaitEvent(st, aux->join, 0) : cudaSuccess;
    if (e != cudaSuccess) return cuda_fail("segment pass launch", e);
    if (ew != cudaSuccess) return cuda_fail("stream join", ew);
    if (cp.hand > 0) {
        // stage 2: entering states of segments 1..P-1
        if (!g_smem_set[dev]) {
            if ((e = cudaFuncSetAttribute(hand_off, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kHandSmem)) !=
                cudaSuccess)
                return cuda_fail("hand-off attribute", e);
            g_smem_set[dev] = true;
        }
        hand_off<<<dim3((unsigned)cp.hand, (unsigned)H), kHandThreads, kHandSmem, st>>>(hand, counts, states, H);
        if ((e = cudaGetLastError()) != cudaSuccess) return cuda_fail("hand-off launch", e);
        // stage 3: segments 1..P-1 from their entering states
        e = kda::launch_fwd_segments(false, q, k, v, g, beta, T, H, tab_f, counts + 2, cp.f, initial_state,
                                     final_state, states, out, status, st);
        if (e != cudaSuccess) return cuda_fail("final pass launch", e);
    }
    return KDA_OK;
}

}  // namespace

extern "C" {

size_t kda_chunk_fwd_split_workspace_size(int n_docs, int64_t T, int H) {
    if (n_docs < 1 || H < 1 || T < 0) return 0;
    const int sms = current_sms();
    if (sms < 1) return 0;
    return layout(caps(n_docs, H, sms, 0), H).total;
}

kda_status kda_chunk_fwd_split(const uint16_t *q, const uint16_t *k, const uint16_t *v, const float *g,
                               const float *beta, const int32_t *cu_seqlens, int n_docs, int64_t T, int H,
                               const float *initial_state, float *final_state, uint16_t *out, void *workspace,
                               size_t workspace_bytes, void *stream) {
    kda::set_last_error(KDA_OK, "");
    if (!cu_seqlens) return fail(KDA_ERR_INVALID_ARG, "cu_seqlens is NULL");
    return split_forward(q, k, v, g, beta, cu_seqlens, n_docs, T, H, 0, initial_state, final_state, out, workspace,
                         workspace_bytes, stream, current_sms());
}

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
    return layout(caps(1, H, 1, segments), H).total;
}

kda_status kda_chunk_fwd_long(const uint16_t *q, const uint16_t *k, const uint16_t *v, const float *g,
                              const float *beta, int64_t T, int H, int segments, const float *initial_state,
                              float *final_state, uint16_t *out, void *workspace, size_t workspace_bytes,
                              void *stream) {
    kda::set_last_error(KDA_OK, "");
    if (segments < 1 || segments > kMaxSegments)
        return fail(KDA_ERR_INVALID_ARG, "segments must be in [1, %d] (got %d)", kMaxSegments, segments);
    const int64_t nch = (T + 63) / 64;
    if (T > 0 && segments > nch)
        return fail(KDA_ERR_INVALID_ARG, "segments (%d) exceeds the document's %lld chunks", segments, (long long)nch);
    if (T > 0 && segments * H > INT32_MAX / 4) return fail(KDA_ERR_INVALID_ARG, "segments * H too large");
    return split_forward(q, k, v, g, beta, nullptr, 1, T, H, segments, initial_state, final_state, out, workspace,
                         workspace_bytes, stream, 1);
}

}  // extern "C"
