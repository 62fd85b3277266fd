// kda_recurrent.cu -- the token-by-token (recurrent) KDA forward, for decode and short sequences.
//
// The recurrence itself, one token at a time, with no chunking (the alternative to chunk mode
// that the pages' mode switch picks for short sequences: the kda_mode setting and
// KimiDeltaAttention._resolve_mode on the kimi_linear model page):
//
//   S' = Diag(e^{g_t}) S,  p = S'^T k^,  S = S' + beta_t k^ (v_t - p)^T,  o_t = scale S^T q^
//
// A chain's 128 value columns are split over 4 CTAs of 128 threads (the columns of S evolve
// independently given q, k, g and beta, so the split needs no exchange).  Four adjacent lanes
// share value column v and keep 32 rows each of the fp32 state column S[:, v] in registers, so a
// token costs 4 x 32 multiply-adds per thread, with the token's q, k and decays broadcast from
// shared memory, one barrier, and the next token's inputs loaded while this one computes.  The norms are applied
// to the dot products rather than to the vectors: S'^T k^ = rk S'^T k and likewise for q.
// The state may start from an initial state and be written out at the end, as in
// kda_chunk_fwd_state.  Meant for few tokens per document (decode after a prefill); the chunked
// kernel is far faster per token on long documents.
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

// One token's inputs as this thread loads them: channel c of q, k and g, column `col` of v, beta.
struct Tok {
    float q, k, g, v, beta;
};

// kSplit threads share one value column, each holding kRows = 128 / kSplit rows of it; a CTA of
// 128 threads covers kCols = 128 / kSplit columns, so a chain takes kSplit CTAs (the columns of
// S evolve independently given q, k, g and beta, so splitting them needs no exchange).
template <int kSplit, int kAhead>
__global__ void __launch_bounds__(kThreads) kda_recurrent_kernel(const uint16_t *__restrict__ q,
                                                                 const uint16_t *__restrict__ k,
                                                                 const uint16_t *__restrict__ v,
                                                                 const float *__restrict__ g,
                                                                 const float *__restrict__ beta,
                                                                 const int32_t *__restrict__ cu_seqlens, int n_docs,
                                                                 int64_t T, int H, const float *h0, float *ht,
                                                                 uint16_t *__restrict__ out,
                                                                 int *__restrict__ status) {
    static_assert(kAhead % 2 == 0, "the smem double buffer alternates by token parity");
    constexpr int kRows = D / kSplit, kCols = D / kSplit;
    constexpr int kVec = D + 4 * kSplit;    // smem vector: each row block shifted by 4 floats (other banks)
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int chain = blockIdx.x, doc = chain / H, h = chain % H;
    if (chain == 0 && blockIdx.y == 0 && tid == 0 && (cu_seqlens[0] != 0 || (int64_t)cu_seqlens[n_docs] != T))
        atomicExch(status, kStatusBadSeqlens);
    const int64_t t0 = cu_seqlens[doc], t1 = cu_seqlens[doc + 1];
    if (t0 < 0 || t1 < t0 || t1 > T) {
        if (tid == 0) atomicExch(status, kStatusBadSeqlens);
        return;
    }
    // thread (col, part): S[part*kRows + r][col], r < kRows, as kRows/2 packed pairs; the kSplit
    // threads of a column are adjacent lanes and meet with shuffles
    const int part = tid % kSplit, col = blockIdx.y * kCols + tid / kSplit, r0 = part * kRows;
    const size_t soff = (size_t)chain * D * D;
    float2 S[kRows / 2];
#pragma unroll
    for (int j = 0; j < kRows / 2; ++j)
        S[j] = h0 ? make_float2(h0[soff + (size_t)(r0 + 2 * j) * D + col], h0[soff + (size_t)(r0 + 2 * j + 1) * D + col])
                  : make_float2(0.f, 0.f);

    // Per-token broadcast vectors (raw q, raw k, e^g) and the norm partial sums, double-buffered
    // by token parity: a thread writing token t+2's buffers has passed token t+1's barrier,
    // which every reader of token t's buffers reached only after its last read of them.
    __shared__ __align__(16) float sq[2][kVec], sk[2][kVec], sa[2][kVec];
    __shared__ float sred[2][3][4];
    const float scale = rsqrtf((float)D);
    const int c = tid;                       // key channel of the load phase
    const int cs = c + (c / kRows) * 4;      // its smem slot
    auto load = [&](int64_t t) {
        const size_t row = ((size_t)t * H + h) * D;
        Tok x;
        x.q = bf2f(q[row + c]);
        x.k = bf2f(k[row + c]);
        x.g = g[row + c];
        x.v = bf2f(v[row + col]);
        x.beta = beta[(size_t)t * H + h];
        return x;
    };
    // Inputs run kAhead tokens ahead of the arithmetic: token t's registers are refilled with
    // token t + kAhead right after they are staged, and the loop is unrolled kAhead times so
    // that no register copy waits for a load issued less than kAhead tokens earlier.
    Tok x[kAhead];
#pragma unroll
    for (int i = 0; i < kAhead; ++i)
        if (t0 + i < t1) x[i] = load(t0 + i);
    for (int64_t tb = t0; tb < t1; tb += kAhead) {
#pragma unroll
        for (int i = 0; i < kAhead; ++i) {
            const int64_t t = tb + i;
            if (t >= t1) break;
            const int b = i & 1;             // (t - t0) & 1, kAhead being even
            sq[b][cs] = x[i].q;
            sk[b][cs] = x[i].k;
            sa[b][cs] = ex2_ftz(x[i].g * kLog2e);
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
            const float v_t = x[i].v, b_t = x[i].beta;
            if (t + kAhead < t1) x[i] = load(t + kAhead);
            __syncthreads();
            const float rq = rsqrtf(sred[b][0][0] + sred[b][0][1] + sred[b][0][2] + sred[b][0][3] + 1e-6f);
            const float rk = rsqrtf(sred[b][1][0] + sred[b][1][1] + sred[b][1][2] + sred[b][1][3] + 1e-6f);
            const float qk = (sred[b][2][0] + sred[b][2][1] + sred[b][2][2] + sred[b][2][3]) * rq * rk;
            // S' = Diag(e^g) S, p = S'^T k (raw k), w = S'^T q (raw q), over this thread's rows
            float2 pa = make_float2(0.f, 0.f), pb = pa, wa = pa, wb = pa;
            const int base = r0 + part * 4;
            const float4 *a4 = reinterpret_cast<const float4 *>(sa[b] + base);
            const float4 *k4 = reinterpret_cast<const float4 *>(sk[b] + base);
            const float4 *q4 = reinterpret_cast<const float4 *>(sq[b] + base);
#pragma unroll
            for (int j4 = 0; j4 < kRows / 4; ++j4) {
                const float4 a = a4[j4], kk = k4[j4], qq = q4[j4];
                S[2 * j4] = __fmul2_rn(S[2 * j4], make_float2(a.x, a.y));
                S[2 * j4 + 1] = __fmul2_rn(S[2 * j4 + 1], make_float2(a.z, a.w));
                pa = __ffma2_rn(S[2 * j4], make_float2(kk.x, kk.y), pa);
                pb = __ffma2_rn(S[2 * j4 + 1], make_float2(kk.z, kk.w), pb);
                wa = __ffma2_rn(S[2 * j4], make_float2(qq.x, qq.y), wa);
                wb = __ffma2_rn(S[2 * j4 + 1], make_float2(qq.z, qq.w), wb);
            }
            float p = (pa.x + pb.x) + (pa.y + pb.y), w = (wa.x + wb.x) + (wa.y + wb.y);
#pragma unroll
            for (int o = 1; o < kSplit; o <<= 1) {
                p += __shfl_xor_sync(0xffffffffu, p, o);
                w += __shfl_xor_sync(0xffffffffu, w, o);
            }
            // e = beta (v - S'^T k^); S = S' + k^ e^T; o = scale S^T q^ = scale (S'^T q^ + (q^.k^) e)
            const float e = b_t * (v_t - p * rk);
            if (part == 0)
                out[((size_t)t * H + h) * D + col] =
                    __bfloat16_as_ushort(__float2bfloat16_rn(scale * (w * rq + qk * e)));
            const float2 e2 = make_float2(e * rk, e * rk);
#pragma unroll
            for (int j4 = 0; j4 < kRows / 4; ++j4) {
                const float4 kk = k4[j4];
                S[2 * j4] = __ffma2_rn(make_float2(kk.x, kk.y), e2, S[2 * j4]);
                S[2 * j4 + 1] = __ffma2_rn(make_float2(kk.z, kk.w), e2, S[2 * j4 + 1]);
            }
        }
    }
    if (ht) {
#pragma unroll
        for (int j = 0; j < kRows / 2; ++j) {
            ht[soff + (size_t)(r0 + 2 * j) * D + col] = S[j].x;
            ht[soff + (size_t)(r0 + 2 * j + 1) * D + col] = S[j].y;
        }
    }
}

}  // namespace recurrent

#ifndef KDA_RECURRENT_SPLIT
#define KDA_RECURRENT_SPLIT 4
#endif
#ifndef KDA_RECURRENT_AHEAD
#define KDA_RECURRENT_AHEAD 2
#endif

cudaError_t launch_fwd_recurrent(const uint16_t *q, const uint16_t *k, const uint16_t *v, const float *g,
                                 const float *beta, const int32_t *cu, int n_docs, int64_t T, int H, const float *h0,
                                 float *ht, uint16_t *out, int *status, cudaStream_t stream) {
    constexpr int kSplit = KDA_RECURRENT_SPLIT;
    const dim3 grid((unsigned)(n_docs * H), kSplit);
    recurrent::kda_recurrent_kernel<kSplit, KDA_RECURRENT_AHEAD><<<grid, recurrent::kThreads, 0, stream>>>(q, k, v, g, beta, cu, n_docs,
                                                                                           T, H, h0, ht, out, status);
    return cudaGetLastError();
}

}  // namespace kda
