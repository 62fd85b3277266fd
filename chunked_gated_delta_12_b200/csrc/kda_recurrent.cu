// kda_recurrent.cu -- the token-by-token (recurrent) KDA forward, for decode and short sequences.
//
// The recurrence itself, one token at a time, with no chunking (the alternative to chunk mode
// that the pages' mode switch picks for short sequences: the kda_mode setting and
// KimiDeltaAttention._resolve_mode on the kimi_linear model page):
//
//   S' = Diag(e^{g_t}) S,  p = S'^T k^,  S = S' + beta_t k^ (v_t - p)^T,  o_t = scale S^T q^
//
// A chain's 128 value columns are split over 4 CTAs of 128 threads (the columns of S evolve
// independently given q, k, g and beta, so the split needs no exchange).  Thread (quad, group)
// keeps 4 adjacent columns of 8 rows of the fp32 state in registers, so that the state moves as
// 16-byte vectors and every warp instruction covers four whole 128-byte row pieces.  Per token the
// CTA stages q, k and the decays in shared memory with the norm partial sums, each thread forms
// its rows' share of S'^T k and S'^T q for its 4 columns, the 16 row groups meet by two shuffle
// levels and one exchange between the 4 warps, and every thread applies the rank-one update to
// its rows.  The norms are applied to the dot products rather than to the vectors:
// S'^T k^ = rk S'^T k and likewise for q.  The state may start from an initial state and be
// written out at the end, as in kda_chunk_fwd_state.  Meant for few tokens per document (decode
// after a prefill); the chunked kernel is far faster per token on long documents.
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "kda_common.cuh"
#include "kda_internal.h"

namespace kda {
namespace recurrent {

constexpr int D = 128;
constexpr int kThreads = 128;

__device__ __forceinline__ float bf2f(uint16_t b) { return __uint_as_float((uint32_t)b << 16); }

// One token's inputs as this thread loads them: channel c of q, k and g, its 4 columns of v, beta.
struct Tok {
    float q, k, g, beta;
    uint2 v;   // four bf16
};

constexpr int kSplit = 4;                // CTAs per chain, 32 columns each
constexpr int kCols = D / kSplit;        // columns of a CTA
constexpr int kQuads = kCols / 4;        // 8 column quads
constexpr int kGroups = kThreads / kQuads;   // 16 row groups
constexpr int kRows = D / kGroups;       // 8 rows per group
constexpr int kAhead = 1;                // tokens of inputs in flight

// 6 CTAs per SM (80 registers): enough state bytes in flight for the decoding step to run at ~0.9 of
// the HBM copy rate (4 CTAs at the natural 108-128 registers reached ~0.79)
__global__ void __launch_bounds__(kThreads, 6) kda_recurrent_kernel(const uint16_t *__restrict__ q,
                                                                 const uint16_t *__restrict__ k,
                                                                 const uint16_t *__restrict__ v,
                                                                 const float *__restrict__ g,
                                                                 const float *__restrict__ beta,
                                                                 const int32_t *__restrict__ cu_seqlens, int n_docs,
                                                                 int64_t T, int H, const float *h0, float *ht,
                                                                 uint16_t *__restrict__ out,
                                                                 int *__restrict__ status) {
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int chain = blockIdx.x, doc = chain / H, h = chain % H;
    if (chain == 0 && blockIdx.y == 0 && tid == 0 && (cu_seqlens[0] != 0 || (int64_t)cu_seqlens[n_docs] != T))
        atomicExch(status, kStatusBadSeqlens);
    const int64_t t0 = cu_seqlens[doc], t1 = cu_seqlens[doc + 1];
    if (t0 < 0 || t1 < t0 || t1 > T) {
        if (tid == 0) atomicExch(status, kStatusBadSeqlens);
        return;
    }
    // thread (quad, group): columns col..col+3, rows r0..r0+7; the 4 groups of a warp hold the same
    // quads (lanes 8 apart)
    const int quad = tid & (kQuads - 1), grp = tid / kQuads;
    const int col = blockIdx.y * kCols + 4 * quad, r0 = kRows * grp;
    const size_t soff = (size_t)chain * D * D;
    float4 S[kRows];
#pragma unroll
    for (int j = 0; j < kRows; ++j)
        S[j] = h0 ? *reinterpret_cast<const float4 *>(h0 + soff + (size_t)(r0 + j) * D + col)
                  : make_float4(0.f, 0.f, 0.f, 0.f);

    // Per-token broadcast vectors (raw q, raw k, e^g), the norm partial sums and the warps' column
    // sums, double-buffered by token parity: a thread writing token t+2's buffers has passed both
    // barriers of token t+1, which every reader of token t's buffers reached only after its last
    // read of them.
    __shared__ __align__(16) float sq[2][D], sk[2][D], sa[2][D];
    __shared__ float sred[2][3][4];
    __shared__ __align__(16) float4 spw[2][4][kQuads][2];   // [parity][warp][quad]{S'^T k, S'^T q}
    const float scale = rsqrtf((float)D);
    const int c = tid;                       // key channel of the load phase
    auto load = [&](int64_t t) {
        const size_t row = ((size_t)t * H + h) * D;
        Tok x;
        x.q = bf2f(q[row + c]);
        x.k = bf2f(k[row + c]);
        x.g = g[row + c];
        x.v = *reinterpret_cast<const uint2 *>(v + row + col);
        x.beta = beta[(size_t)t * H + h];
        return x;
    };
    // Inputs run kAhead tokens ahead of the arithmetic: token t's registers are refilled with
    // token t + kAhead right after they are staged.
    Tok x[kAhead];
#pragma unroll
    for (int i = 0; i < kAhead; ++i)
        if (t0 + i < t1) x[i] = load(t0 + i);
    for (int64_t tb = t0; tb < t1; tb += kAhead) {
#pragma unroll
        for (int i = 0; i < kAhead; ++i) {
            const int64_t t = tb + i;
            if (t >= t1) break;
            const int b = (int)((t - t0) & 1);   // buffer parity of this token
            sq[b][c] = x[i].q;
            sk[b][c] = x[i].k;
            sa[b][c] = ex2_ftz(x[i].g * kLog2e);
            float pq = x[i].q * x[i].q, pk = x[i].k * x[i].k, pqk = x[i].q * x[i].k;
#pragma unroll
            for (int o = 16; o; o >>= 1) {
                pq += __shfl_xor_sync(0xffffffffu, pq, o);
                pk += __shfl_xor_sync(0xffffffffu, pk, o);
                pqk += __shfl_xor_sync(0xffffffffu, pqk, o);
            }
            if (lane == 0) {
                sred[b][0][warp] = pq;
                sred[b][1][warp] = pk;
                sred[b][2][warp] = pqk;
            }
            const uint2 v_t = x[i].v;
            const float b_t = x[i].beta;
            if (t + kAhead < t1) x[i] = load(t + kAhead);
            __syncthreads();
            const float rq = rsqrtf(sred[b][0][0] + sred[b][0][1] + sred[b][0][2] + sred[b][0][3] + 1e-6f);
            const float rk = rsqrtf(sred[b][1][0] + sred[b][1][1] + sred[b][1][2] + sred[b][1][3] + 1e-6f);
            const float qk = (sred[b][2][0] + sred[b][2][1] + sred[b][2][2] + sred[b][2][3]) * rq * rk;
            // S' = Diag(e^g) S; this thread's rows' share of p = S'^T k and w = S'^T q (raw k, q)
            float kr[kRows];
            float4 p = make_float4(0.f, 0.f, 0.f, 0.f), w = p;
#pragma unroll
            for (int j4 = 0; j4 < kRows; j4 += 4) {
                const float4 a4 = *reinterpret_cast<const float4 *>(sa[b] + r0 + j4);
                const float4 k4 = *reinterpret_cast<const float4 *>(sk[b] + r0 + j4);
                const float4 q4 = *reinterpret_cast<const float4 *>(sq[b] + r0 + j4);
                const float av[4] = {a4.x, a4.y, a4.z, a4.w}, kv[4] = {k4.x, k4.y, k4.z, k4.w};
                const float qv[4] = {q4.x, q4.y, q4.z, q4.w};
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                    float4 &sj = S[j4 + u];
                    sj.x *= av[u]; sj.y *= av[u]; sj.z *= av[u]; sj.w *= av[u];
                    p.x = fmaf(sj.x, kv[u], p.x); p.y = fmaf(sj.y, kv[u], p.y);
                    p.z = fmaf(sj.z, kv[u], p.z); p.w = fmaf(sj.w, kv[u], p.w);
                    w.x = fmaf(sj.x, qv[u], w.x); w.y = fmaf(sj.y, qv[u], w.y);
                    w.z = fmaf(sj.z, qv[u], w.z); w.w = fmaf(sj.w, qv[u], w.w);
                    kr[j4 + u] = kv[u];
                }
            }
            // the 4 row groups of the warp (lanes 8 apart) meet by shuffles, the 4 warps in shared memory
#pragma unroll
            for (int o = 8; o < 32; o <<= 1) {
                p.x += __shfl_xor_sync(0xffffffffu, p.x, o); p.y += __shfl_xor_sync(0xffffffffu, p.y, o);
                p.z += __shfl_xor_sync(0xffffffffu, p.z, o); p.w += __shfl_xor_sync(0xffffffffu, p.w, o);
                w.x += __shfl_xor_sync(0xffffffffu, w.x, o); w.y += __shfl_xor_sync(0xffffffffu, w.y, o);
                w.z += __shfl_xor_sync(0xffffffffu, w.z, o); w.w += __shfl_xor_sync(0xffffffffu, w.w, o);
            }
            if (lane < kQuads) {
                spw[b][warp][quad][0] = p;
                spw[b][warp][quad][1] = w;
            }
            __syncthreads();
            p = w = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
            for (int ww = 0; ww < 4; ++ww) {
                const float4 pp = spw[b][ww][quad][0], qq = spw[b][ww][quad][1];
                p.x += pp.x; p.y += pp.y; p.z += pp.z; p.w += pp.w;
                w.x += qq.x; w.y += qq.y; w.z += qq.z; w.w += qq.w;
            }
            // e = beta (v - S'^T k^); S = S' + k^ e^T; o = scale S^T q^ = scale (S'^T q^ + (q^.k^) e)
            const float2 v01 = unpack_bf16(v_t.x), v23 = unpack_bf16(v_t.y);
            const float4 e = make_float4(b_t * (v01.x - p.x * rk), b_t * (v01.y - p.y * rk),
                                         b_t * (v23.x - p.z * rk), b_t * (v23.y - p.w * rk));
            if (grp == 0) {
                const uint2 o2 = make_uint2(pack_bf16(scale * (w.x * rq + qk * e.x), scale * (w.y * rq + qk * e.y)),
                                            pack_bf16(scale * (w.z * rq + qk * e.z), scale * (w.w * rq + qk * e.w)));
                *reinterpret_cast<uint2 *>(out + ((size_t)t * H + h) * D + col) = o2;
            }
            const float4 er = make_float4(e.x * rk, e.y * rk, e.z * rk, e.w * rk);
#pragma unroll
            for (int j = 0; j < kRows; ++j) {
                S[j].x = fmaf(kr[j], er.x, S[j].x); S[j].y = fmaf(kr[j], er.y, S[j].y);
                S[j].z = fmaf(kr[j], er.z, S[j].z); S[j].w = fmaf(kr[j], er.w, S[j].w);
            }
        }
    }
    if (ht) {
#pragma unroll
        for (int j = 0; j < kRows; ++j) *reinterpret_cast<float4 *>(ht + soff + (size_t)(r0 + j) * D + col) = S[j];
    }
}

}  // namespace recurrent

cudaError_t launch_fwd_recurrent(const uint16_t *q, const uint16_t *k, const uint16_t *v, const float *g,
                                 const float *beta, const int32_t *cu, int n_docs, int64_t T, int H, const float *h0,
                                 float *ht, uint16_t *out, int *status, cudaStream_t stream) {
    const dim3 grid((unsigned)(n_docs * H), recurrent::kSplit);
    recurrent::kda_recurrent_kernel<<<grid, recurrent::kThreads, 0, stream>>>(q, k, v, g, beta, cu, n_docs, T, H, h0,
                                                                             ht, out, status);
    return cudaGetLastError();
}

}  // namespace kda
