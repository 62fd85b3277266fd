// kda_fwd_mma.cu -- fused chunk-KDA forward, one CTA per (document, head, V-slice).
//
// The CTA walks its document's 64-token chunks in order and keeps the fp32
// state slice S[128 x VS] in registers (warp-level MMA accumulators).  Per
// chunk (rows r, i of the chunk; Gamma = inclusive in-chunk cumsum of g):
//
//   prep    q^, k^ (l2 norm, fp32), Gamma (per-channel cumsum, fp32)
//   intra   A_kk[r,i] = beta_r sum_c k^_rc k^_ic e^{Gamma_rc - Gamma_ic}  (i < r)
//           A_qk[r,i] =        sum_c q^_rc k^_ic e^{Gamma_rc - Gamma_ic}  (i <= r)
//           T = (I + A_kk)^-1 (blocked forward substitution, fp32), T' = T diag(beta)
//           W = T' (K^ e^Gamma),  U = T' V
//   state   U~ = U - W S;  O = (Q^ e^Gamma) S + A_qk U~
//           S <- Diag(e^{Gamma_last}) S + (K^ e^{Gamma_last - Gamma})^T U~
//   output  o = O / sqrt(128) -> bf16, rows inside the document only
//
// Gate range: g >= -5 per token, so Gamma spans up to 320 inside a chunk and
// e^{+-Gamma} alone would overflow fp32.  The exponent is therefore split at
// 16-row sub-block boundaries (block R = rows 16R..16R+15, m_R = 16R, e_R =
// 16R+15):
//   E1[r] = e^{Gamma_r - Gamma_{m_R}} <= 1,  E2[r] = e^{Gamma_{e_R} - Gamma_r} <= 1
//   e^{Gamma_r - Gamma_i} = E1[r] * s_{R,I} * E2[i],  s_{R,I} = e^{Gamma_{m_R} - Gamma_{e_I}}
// where s_{R,I} <= 1 off the diagonal (I < R) and <= e^{75} on it (I = R) --
// every factor stays inside fp32/bf16 range.  Two exp2 per (token, channel).
//
// Rows past the document end are zero-filled on load (never read from
// memory), which makes their g = 0, beta = 0, k = v = 0: they drop out of
// every product and leave Gamma_last = Gamma of the last real row.
#include <cuda_runtime.h>
#include <stdint.h>

#include "kda_common.cuh"
#include "kda_internal.h"

namespace kda {
namespace mma_path {

constexpr int kThreads = 256;

template <int VS>
struct Smem {
    static constexpr int Q = 0;                       // q raw bf16 [64][128]
    static constexpr int K = Q + 16384;               // k raw bf16 [64][128]
    static constexpr int G = K + 16384;               // g raw -> Gamma fp32 [64][128]; later A_kk/T'/X
    static constexpr int V = G + 32768;               // v slice bf16 [64][VS]
    static constexpr int QL = V + 64 * VS * 2;        // q^ E1          -> later W bf16 [64][128]
    static constexpr int KL = QL + 16384;             // k^ E1          -> later U~ bf16 [64][VS]
    static constexpr int KR = KL + 16384;             // k^ E2          -> later T fp32 [64][64]
    static constexpr int QT = KR + 16384;             // q^ e^Gamma
    static constexpr int KG = QT + 16384;             // k^ e^Gamma
    static constexpr int KD = KG + 16384;             // k^ e^{Gamma_last - Gamma}
    static constexpr int SB = KD + 16384;             // S bf16 [128][VS]
    static constexpr int AQK = SB + 128 * VS * 2;     // A_qk bf16 [64][64]
    static constexpr int PS = AQK + 8192;             // s_{R,I} fp32 [10][128]
    static constexpr int DC = PS + 10 * 128 * 4;      // e^{Gamma_last} fp32 [128]
    static constexpr int BETA = DC + 512;             // beta fp32 [64]
    static constexpr int RQ = BETA + 256;             // 1/|q| fp32 [64]
    static constexpr int RK = RQ + 256;               // 1/|k| fp32 [64]
    static constexpr int BYTES = RK + 256;
    // aliases inside G (live from intra onwards, after Gamma is dead)
    static constexpr int AKK = G;                     // A_kk fp32 [64][64] (pitch 256)
    static constexpr int TP = G + 16384;              // T' bf16 [64][64] (pitch 128)
    static constexpr int X = G + 24576;               // solve temporaries fp32 [3][16][16]
    static constexpr int W = QL;
    static constexpr int UT = KL;
    static constexpr int TM = KR;                     // T fp32 [64][64] (pitch 256)
};

// Issue the async loads of q and k rows [tok0, tok0 + L) of head h.
template <int VS>
__device__ __forceinline__ void load_qk(uint8_t *sm, const uint16_t *q, const uint16_t *k,
                                        int64_t tok0, int L, int H, int h) {
    using S = Smem<VS>;
    for (int idx = threadIdx.x; idx < 64 * 16; idx += kThreads) {
        const int row = idx >> 4, ch = idx & 15;
        const bool ok = row < L;
        const int64_t off = ok ? ((tok0 + row) * H + h) * kHeadDim + ch * 8 : 0;
        cp_async16(smem_u32(sm + S::Q) + swz_chunk(row, ch, 256), q + off, ok ? 16 : 0);
        cp_async16(smem_u32(sm + S::K) + swz_chunk(row, ch, 256), k + off, ok ? 16 : 0);
    }
}

// Issue the async loads of g, the v slice and beta for rows [tok0, tok0 + L).
template <int VS>
__device__ __forceinline__ void load_gvb(uint8_t *sm, const float *g, const uint16_t *v,
                                         const float *beta, int64_t tok0, int L, int H, int h,
                                         int v0) {
    using S = Smem<VS>;
    for (int idx = threadIdx.x; idx < 64 * 32; idx += kThreads) {
        const int row = idx >> 5, ch = idx & 31;
        const bool ok = row < L;
        const int64_t off = ok ? ((tok0 + row) * H + h) * kHeadDim + ch * 4 : 0;
        cp_async16(smem_u32(sm + S::G) + swz_chunk(row, ch, 512), g + off, ok ? 16 : 0);
    }
    constexpr int VCH = VS / 8;
    for (int idx = threadIdx.x; idx < 64 * VCH; idx += kThreads) {
        const int row = idx / VCH, ch = idx % VCH;
        const bool ok = row < L;
        const int64_t off = ok ? ((tok0 + row) * H + h) * kHeadDim + v0 + ch * 8 : 0;
        cp_async16(smem_u32(sm + S::V) + swz_chunk(row, ch, VS * 2), v + off, ok ? 16 : 0);
    }
    if (threadIdx.x < 64) {
        const int row = threadIdx.x;
        const bool ok = row < L;
        const float *src = ok ? beta + (tok0 + row) * H + h : beta;
        asm volatile("cp.async.ca.shared.global [%0], [%1], 4, %2;\n" ::"r"(
                         smem_u32(sm + S::BETA + row * 4)),
                     "l"(src), "r"(ok ? 4 : 0)
                     : "memory");
    }
}

template <int VS>
__global__ void __launch_bounds__(kThreads, 1)
    kda_fwd_mma_kernel(const uint16_t *__restrict__ q, const uint16_t *__restrict__ k,
                       const uint16_t *__restrict__ v, const float *__restrict__ g,
                       const float *__restrict__ beta, const int32_t *__restrict__ cu_seqlens,
                       int n_docs, int64_t T, int H, uint16_t *__restrict__ out,
                       int *__restrict__ status) {
    using S = Smem<VS>;
    constexpr int NV = kHeadDim / VS;   // V-slices per chain
    constexpr int NTU = VS / 64;        // n8 tiles of U / O per warp (1 or 2)
    constexpr int NTS = VS / 8;         // n8 tiles of the state per warp
    extern __shared__ __align__(1024) uint8_t sm[];

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int gq = lane >> 2, tq = lane & 3;   // mma fragment row group / thread-in-group
    const int vsl = blockIdx.x % NV;
    const int chain = blockIdx.x / NV;
    const int doc = chain / H, h = chain % H;
    const int v0 = vsl * VS;

    if (blockIdx.x == 0 && tid == 0) {
        if (cu_seqlens[0] != 0 || (int64_t)cu_seqlens[n_docs] != T) atomicExch(status, 6);
    }
    const int64_t doc_start = cu_seqlens[doc], doc_end = cu_seqlens[doc + 1];
    if (doc_start < 0 || doc_end < doc_start || doc_end > T) {
        if (tid == 0) atomicExch(status, 6);
        return;
    }
    if (doc_end == doc_start) return;

    float sacc[NTS][4];
#pragma unroll
    for (int i = 0; i < NTS; ++i) sacc[i][0] = sacc[i][1] = sacc[i][2] = sacc[i][3] = 0.f;
    // S bf16 copy starts at zero
    for (int i = tid; i < 128 * VS * 2 / 16; i += kThreads)
        *reinterpret_cast<uint4 *>(sm + S::SB + i * 16) = make_uint4(0, 0, 0, 0);

    {
        const int L0 = (int)(doc_end - doc_start < 64 ? doc_end - doc_start : 64);
        load_qk<VS>(sm, q, k, doc_start, L0, H, h);
        load_gvb<VS>(sm, g, v, beta, doc_start, L0, H, h, v0);
        cp_async_commit();
    }

    const float out_scale = rsqrtf((float)kHeadDim);

    for (int64_t tok0 = doc_start; tok0 < doc_end; tok0 += 64) {
        const int L = (int)(doc_end - tok0 < 64 ? doc_end - tok0 : 64);
        const int64_t ntok0 = tok0 + 64;
        const int nL = (int)(doc_end - ntok0 < 64 ? doc_end - ntok0 : 64);   // <= 0: no next chunk
        cp_async_wait_all();
        __syncthreads();

        // ---------------- prep: l2 norms (warp per row) ----------------
        for (int r = warp * 8; r < warp * 8 + 8; ++r) {
            const uint32_t off = swz_chunk(r, lane >> 1, 256) + (lane & 1) * 8;
            const uint2 qa = *reinterpret_cast<const uint2 *>(sm + S::Q + off);
            const uint2 ka = *reinterpret_cast<const uint2 *>(sm + S::K + off);
            float2 q01 = unpack_bf16(qa.x), q23 = unpack_bf16(qa.y);
            float2 k01 = unpack_bf16(ka.x), k23 = unpack_bf16(ka.y);
            float sq = q01.x * q01.x + q01.y * q01.y + q23.x * q23.x + q23.y * q23.y;
            float sk = k01.x * k01.x + k01.y * k01.y + k23.x * k23.x + k23.y * k23.y;
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) {
                sq += __shfl_xor_sync(0xffffffffu, sq, o);
                sk += __shfl_xor_sync(0xffffffffu, sk, o);
            }
            if (lane == 0) {
                reinterpret_cast<float *>(sm + S::RQ)[r] = rsqrtf(sq + 1e-6f);
                reinterpret_cast<float *>(sm + S::RK)[r] = rsqrtf(sk + 1e-6f);
            }
        }
        // ---------------- prep: in-chunk cumsum of g, two halves ----------------
        {
            const int c = tid & 127, half = tid >> 7;
            float acc = 0.f;
#pragma unroll 8
            for (int r = half * 32; r < half * 32 + 32; ++r) {
                float *p = reinterpret_cast<float *>(sm + S::G + swz_f32(r, c, 512));
                acc += *p;
                *p = acc;
            }
            __syncthreads();
            if (half) {
                const float base = *reinterpret_cast<const float *>(sm + S::G + swz_f32(31, c, 512));
#pragma unroll 8
                for (int r = 32; r < 64; ++r) {
                    float *p = reinterpret_cast<float *>(sm + S::G + swz_f32(r, c, 512));
                    *p += base;
                }
            }
            __syncthreads();
        }
        auto gam = [&](int r, int c) -> float {
            return *reinterpret_cast<const float *>(sm + S::G + swz_f32(r, c, 512));
        };
        // ---------------- per-channel scalars ----------------
        for (int idx = tid; idx < 10 * 128; idx += kThreads) {
            const int p = idx >> 7, c = idx & 127;
            const int R = p >= 6 ? 3 : p >= 3 ? 2 : p >= 1 ? 1 : 0;
            const int I = p - R * (R + 1) / 2;
            reinterpret_cast<float *>(sm + S::PS)[idx] =
                fast_exp2((gam(16 * R, c) - gam(16 * I + 15, c)) * kLog2e);
        }
        if (tid < 128)
            reinterpret_cast<float *>(sm + S::DC)[tid] = fast_exp2(gam(63, tid) * kLog2e);
        // ---------------- derived operand tiles ----------------
        {
            const int cg = tid & 31, r0 = tid >> 5;
            const int c0 = cg * 4;
            float gm[4][4], ge[4][4];
#pragma unroll
            for (int R = 0; R < 4; ++R) {
                const float4 a = *reinterpret_cast<const float4 *>(sm + S::G + swz_chunk(16 * R, cg, 512));
                const float4 b = *reinterpret_cast<const float4 *>(sm + S::G + swz_chunk(16 * R + 15, cg, 512));
                gm[R][0] = a.x; gm[R][1] = a.y; gm[R][2] = a.z; gm[R][3] = a.w;
                ge[R][0] = b.x; ge[R][1] = b.y; ge[R][2] = b.z; ge[R][3] = b.w;
            }
            const float *rq = reinterpret_cast<const float *>(sm + S::RQ);
            const float *rk = reinterpret_cast<const float *>(sm + S::RK);
#pragma unroll 2
            for (int i = 0; i < 8; ++i) {
                const int r = r0 + 8 * i, R = i >> 1;
                const uint32_t boff = swz_bf16(r, c0, 256);
                const uint2 qa = *reinterpret_cast<const uint2 *>(sm + S::Q + boff);
                const uint2 ka = *reinterpret_cast<const uint2 *>(sm + S::K + boff);
                const float4 G4 = *reinterpret_cast<const float4 *>(sm + S::G + swz_chunk(r, cg, 512));
                const float2 q01 = unpack_bf16(qa.x), q23 = unpack_bf16(qa.y);
                const float2 k01 = unpack_bf16(ka.x), k23 = unpack_bf16(ka.y);
                const float qv[4] = {q01.x, q01.y, q23.x, q23.y};
                const float kv[4] = {k01.x, k01.y, k23.x, k23.y};
                const float Gv[4] = {G4.x, G4.y, G4.z, G4.w};
                const float sq = rq[r], sk = rk[r];
                float ql[4], kl[4], kr[4], qt[4], kg[4], kd[4];
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    const float qh = qv[j] * sq, kh = kv[j] * sk;
                    const float e1 = fast_exp2((Gv[j] - gm[R][j]) * kLog2e);
                    const float e2 = fast_exp2((ge[R][j] - Gv[j]) * kLog2e);
                    const float pm = fast_exp2(gm[R][j] * kLog2e);
                    const float dk = fast_exp2((ge[3][j] - ge[R][j]) * kLog2e);
                    ql[j] = qh * e1;
                    kl[j] = kh * e1;
                    kr[j] = kh * e2;
                    qt[j] = ql[j] * pm;
                    kg[j] = kl[j] * pm;
                    kd[j] = kr[j] * dk;
                }
                auto st4 = [&](int base, const float (&x)[4]) {
                    *reinterpret_cast<uint2 *>(sm + base + boff) =
                        make_uint2(pack_bf16(x[0], x[1]), pack_bf16(x[2], x[3]));
                };
                st4(S::QL, ql);
                st4(S::KL, kl);
                st4(S::KR, kr);
                st4(S::QT, qt);
                st4(S::KG, kg);
                st4(S::KD, kd);
            }
        }
        __syncthreads();
        // q and k raw tiles are dead: prefetch the next chunk's
        if (nL > 0) {
            load_qk<VS>(sm, q, k, ntok0, nL, H, h);
            cp_async_commit();
        }

        // ---------------- intra: A_kk and A_qk, 16x16 blocks ----------------
        {
            const int type = warp & 1;          // 0: A_kk, 1: A_qk
            const int jw = warp >> 1;
            const int left = type ? S::QL : S::KL;
            for (int p = jw; p < 10; p += 4) {
                const int R = p >= 6 ? 3 : p >= 3 ? 2 : p >= 1 ? 1 : 0;
                const int I = p - R * (R + 1) / 2;
                const float *ps = reinterpret_cast<const float *>(sm + S::PS) + p * 128;
                float acc[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
#pragma unroll
                for (int kk = 0; kk < 8; ++kk) {
                    uint32_t a[4];
                    {
                        const int j = lane >> 3;
                        const int row = 16 * R + (lane & 7) + 8 * (j & 1);
                        ldsm_x4(smem_u32(sm + left) + swz_chunk(row, kk * 2 + (j >> 1), 256), a[0],
                                a[1], a[2], a[3]);
                    }
                    const int cb = kk * 16 + 2 * tq;
                    const float2 s0 = *reinterpret_cast<const float2 *>(ps + cb);
                    const float2 s8 = *reinterpret_cast<const float2 *>(ps + cb + 8);
                    {
                        float2 x;
                        x = unpack_bf16(a[0]); a[0] = pack_bf16(x.x * s0.x, x.y * s0.y);
                        x = unpack_bf16(a[1]); a[1] = pack_bf16(x.x * s0.x, x.y * s0.y);
                        x = unpack_bf16(a[2]); a[2] = pack_bf16(x.x * s8.x, x.y * s8.y);
                        x = unpack_bf16(a[3]); a[3] = pack_bf16(x.x * s8.x, x.y * s8.y);
                    }
                    uint32_t b0, b1, b2, b3;
                    {
                        const int j = lane >> 3;
                        const int row = 16 * I + (lane & 7) + 8 * (j >> 1);
                        ldsm_x4(smem_u32(sm + S::KR) + swz_chunk(row, kk * 2 + (j & 1), 256), b0, b1,
                                b2, b3);
                    }
                    mma_bf16(acc[0], a, b0, b1);
                    mma_bf16(acc[1], a, b2, b3);
                }
                const float *bet = reinterpret_cast<const float *>(sm + S::BETA);
#pragma unroll
                for (int nt = 0; nt < 2; ++nt) {
#pragma unroll
                    for (int hh = 0; hh < 2; ++hh) {
                        const int row = 16 * R + gq + 8 * hh;
                        const int col = 16 * I + 8 * nt + 2 * tq;
                        float x0 = acc[nt][2 * hh], x1 = acc[nt][2 * hh + 1];
                        if (type == 0) {
                            const float br = bet[row];
                            x0 = col < row ? x0 * br : 0.f;
                            x1 = col + 1 < row ? x1 * br : 0.f;
                            *reinterpret_cast<float2 *>(sm + S::AKK + swz_f32(row, col, 256)) =
                                make_float2(x0, x1);
                        } else {
                            x0 = col <= row ? x0 : 0.f;
                            x1 = col + 1 <= row ? x1 : 0.f;
                            *reinterpret_cast<uint32_t *>(sm + S::AQK + swz_bf16(row, col, 128)) =
                                pack_bf16(x0, x1);
                        }
                    }
                }
            }
        }
        __syncthreads();

        // ---------------- intra: T = (I + A_kk)^-1 ----------------
        auto akk = [&](int r, int c) -> float {
            return *reinterpret_cast<const float *>(sm + S::AKK + swz_f32(r, c, 256));
        };
        auto tm = [&](int r, int c) -> float & {
            return *reinterpret_cast<float *>(sm + S::TM + swz_f32(r, c, 256));
        };
        if (warp < 4 && lane < 16) {   // diagonal 16x16 blocks, one column per lane
            const int R = warp, col = lane;
            float x[16];
#pragma unroll
            for (int r = 0; r < 16; ++r) {
                float acc = (r == col) ? 1.f : 0.f;
#pragma unroll
                for (int j = 0; j < r; ++j) acc -= akk(16 * R + r, 16 * R + j) * x[j];
                x[r] = acc;
            }
#pragma unroll
            for (int r = 0; r < 16; ++r) tm(16 * R + r, 16 * R + col) = x[r];
        }
        __syncthreads();
        {
            float *X = reinterpret_cast<float *>(sm + S::X);
            const int i = tid >> 4, j = tid & 15;
#pragma unroll 1
            for (int d = 1; d < 4; ++d) {
                // X_R = sum_{J=I}^{R-1} A_{R,J} T_{J,I}, I = R - d
                for (int bi = 0; bi < 4 - d; ++bi) {
                    const int R = d + bi, I = R - d;
                    float acc = 0.f;
                    for (int J = I; J < R; ++J)
#pragma unroll
                        for (int b = 0; b < 16; ++b)
                            acc += akk(16 * R + i, 16 * J + b) * tm(16 * J + b, 16 * I + j);
                    X[bi * 256 + i * 16 + j] = acc;
                }
                __syncthreads();
                // T_{R,I} = -T_{R,R} X_R
                for (int bi = 0; bi < 4 - d; ++bi) {
                    const int R = d + bi, I = R - d;
                    float acc = 0.f;
#pragma unroll
                    for (int a = 0; a < 16; ++a) acc += tm(16 * R + i, 16 * R + a) * X[bi * 256 + a * 16 + j];
                    tm(16 * R + i, 16 * I + j) = -acc;
                }
                __syncthreads();
            }
        }
        // T' = T diag(beta) in bf16, zero above the diagonal
        {
            const float *bet = reinterpret_cast<const float *>(sm + S::BETA);
            const int r = tid >> 2, cb = (tid & 3) * 16;
#pragma unroll
            for (int c = cb; c < cb + 16; c += 2) {
                const float x0 = c <= r ? tm(r, c) * bet[c] : 0.f;
                const float x1 = c + 1 <= r ? tm(r, c + 1) * bet[c + 1] : 0.f;
                *reinterpret_cast<uint32_t *>(sm + S::TP + swz_bf16(r, c, 128)) = pack_bf16(x0, x1);
            }
        }
        __syncthreads();

        // ---------------- intra: W = T' KG (cols 16w..16w+15), U = T' V (warp's tiles) ----------------
        float uacc[4][NTU][4];
        {
            const int uc0 = warp * 8 * NTU;   // first U column of this warp (within the slice)
#pragma unroll
            for (int R = 0; R < 4; ++R) {
                float wacc[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
#pragma unroll
                for (int nt = 0; nt < NTU; ++nt) uacc[R][nt][0] = uacc[R][nt][1] = uacc[R][nt][2] = uacc[R][nt][3] = 0.f;
#pragma unroll
                for (int I = 0; I <= R; ++I) {
                    uint32_t a[4];
                    {
                        const int j = lane >> 3;
                        const int row = 16 * R + (lane & 7) + 8 * (j & 1);
                        ldsm_x4(smem_u32(sm + S::TP) + swz_chunk(row, 2 * I + (j >> 1), 128), a[0], a[1],
                                a[2], a[3]);
                    }
                    {
                        const int j = lane >> 3;
                        const int row = 16 * I + (lane & 7) + 8 * (j & 1);
                        uint32_t b0, b1, b2, b3;
                        ldsm_x4_t(smem_u32(sm + S::KG) + swz_chunk(row, 2 * warp + (j >> 1), 256), b0, b1,
                                  b2, b3);
                        mma_bf16(wacc[0], a, b0, b1);
                        mma_bf16(wacc[1], a, b2, b3);
                    }
                    if (NTU == 1) {
                        const int j = (lane >> 3) & 1;
                        const int row = 16 * I + (lane & 7) + 8 * j;
                        uint32_t b0, b1;
                        ldsm_x2_t(smem_u32(sm + S::V) + swz_chunk(row, uc0 >> 3, VS * 2), b0, b1);
                        mma_bf16(uacc[R][0], a, b0, b1);
                    } else {
                        const int j = lane >> 3;
                        const int row = 16 * I + (lane & 7) + 8 * (j & 1);
                        uint32_t b0, b1, b2, b3;
                        ldsm_x4_t(smem_u32(sm + S::V) + swz_chunk(row, (uc0 >> 3) + (j >> 1), VS * 2), b0,
                                  b1, b2, b3);
                        mma_bf16(uacc[R][0], a, b0, b1);
                        mma_bf16(uacc[R][NTU - 1], a, b2, b3);
                    }
                }
#pragma unroll
                for (int nt = 0; nt < 2; ++nt)
#pragma unroll
                    for (int hh = 0; hh < 2; ++hh) {
                        const int row = 16 * R + gq + 8 * hh;
                        const int col = 16 * warp + 8 * nt + 2 * tq;
                        *reinterpret_cast<uint32_t *>(sm + S::W + swz_bf16(row, col, 256)) =
                            pack_bf16(wacc[nt][2 * hh], wacc[nt][2 * hh + 1]);
                    }
            }
        }
        __syncthreads();
        // g, v, beta, A_kk, T' are dead: prefetch the next chunk's g, v, beta
        if (nL > 0) {
            load_gvb<VS>(sm, g, v, beta, ntok0, nL, H, h, v0);
            cp_async_commit();
        }

        // ---------------- state: U~ = U - W S, O = Qt S + A_qk U~ ----------------
        {
            const int uc0 = warp * 8 * NTU;
            float oacc[4][NTU][4];
#pragma unroll
            for (int R = 0; R < 4; ++R) {
                float ws[NTU][4];
#pragma unroll
                for (int nt = 0; nt < NTU; ++nt)
#pragma unroll
                    for (int e = 0; e < 4; ++e) ws[nt][e] = oacc[R][nt][e] = 0.f;
#pragma unroll
                for (int kk = 0; kk < 8; ++kk) {
                    uint32_t aw[4], aq[4];
                    const int j = lane >> 3;
                    const int arow = 16 * R + (lane & 7) + 8 * (j & 1);
                    const uint32_t aoff = swz_chunk(arow, 2 * kk + (j >> 1), 256);
                    ldsm_x4(smem_u32(sm + S::W) + aoff, aw[0], aw[1], aw[2], aw[3]);
                    ldsm_x4(smem_u32(sm + S::QT) + aoff, aq[0], aq[1], aq[2], aq[3]);
                    if (NTU == 1) {
                        const int jj = (lane >> 3) & 1;
                        const int row = 16 * kk + (lane & 7) + 8 * jj;
                        uint32_t b0, b1;
                        ldsm_x2_t(smem_u32(sm + S::SB) + swz_chunk(row, uc0 >> 3, VS * 2), b0, b1);
                        mma_bf16(ws[0], aw, b0, b1);
                        mma_bf16(oacc[R][0], aq, b0, b1);
                    } else {
                        const int row = 16 * kk + (lane & 7) + 8 * (j & 1);
                        uint32_t b0, b1, b2, b3;
                        ldsm_x4_t(smem_u32(sm + S::SB) + swz_chunk(row, (uc0 >> 3) + (j >> 1), VS * 2), b0,
                                  b1, b2, b3);
                        mma_bf16(ws[0], aw, b0, b1);
                        mma_bf16(ws[NTU - 1], aw, b2, b3);
                        mma_bf16(oacc[R][0], aq, b0, b1);
                        mma_bf16(oacc[R][NTU - 1], aq, b2, b3);
                    }
                }
#pragma unroll
                for (int nt = 0; nt < NTU; ++nt)
#pragma unroll
                    for (int hh = 0; hh < 2; ++hh) {
                        const int row = 16 * R + gq + 8 * hh;
                        const int col = uc0 + 8 * nt + 2 * tq;
                        *reinterpret_cast<uint32_t *>(sm + S::UT + swz_bf16(row, col, VS * 2)) =
                            pack_bf16(uacc[R][nt][2 * hh] - ws[nt][2 * hh],
                                      uacc[R][nt][2 * hh + 1] - ws[nt][2 * hh + 1]);
                    }
            }
            __syncwarp();
            // O += A_qk U~ (this warp's columns; U~ rows of all blocks written by this warp)
#pragma unroll
            for (int R = 0; R < 4; ++R) {
#pragma unroll
                for (int I = 0; I <= R; ++I) {
                    uint32_t a[4];
                    const int j = lane >> 3;
                    const int arow = 16 * R + (lane & 7) + 8 * (j & 1);
                    ldsm_x4(smem_u32(sm + S::AQK) + swz_chunk(arow, 2 * I + (j >> 1), 128), a[0], a[1], a[2],
                            a[3]);
                    if (NTU == 1) {
                        const int jj = (lane >> 3) & 1;
                        const int row = 16 * I + (lane & 7) + 8 * jj;
                        uint32_t b0, b1;
                        ldsm_x2_t(smem_u32(sm + S::UT) + swz_chunk(row, uc0 >> 3, VS * 2), b0, b1);
                        mma_bf16(oacc[R][0], a, b0, b1);
                    } else {
                        const int row = 16 * I + (lane & 7) + 8 * (j & 1);
                        uint32_t b0, b1, b2, b3;
                        ldsm_x4_t(smem_u32(sm + S::UT) + swz_chunk(row, (uc0 >> 3) + (j >> 1), VS * 2), b0,
                                  b1, b2, b3);
                        mma_bf16(oacc[R][0], a, b0, b1);
                        mma_bf16(oacc[R][NTU - 1], a, b2, b3);
                    }
                }
            }
            // epilogue: o = O / sqrt(128) -> bf16, rows inside the document
#pragma unroll
            for (int R = 0; R < 4; ++R)
#pragma unroll
                for (int nt = 0; nt < NTU; ++nt)
#pragma unroll
                    for (int hh = 0; hh < 2; ++hh) {
                        const int row = 16 * R + gq + 8 * hh;
                        if (row < L) {
                            const int col = v0 + uc0 + 8 * nt + 2 * tq;
                            uint32_t *dst = reinterpret_cast<uint32_t *>(
                                out + ((tok0 + row) * H + h) * kHeadDim + col);
                            *dst = pack_bf16(oacc[R][nt][2 * hh] * out_scale,
                                             oacc[R][nt][2 * hh + 1] * out_scale);
                        }
                    }
        }
        __syncthreads();

        // ---------------- state: S <- Diag(e^{Gamma_last}) S + Kd^T U~ ----------------
        {
            const int m0 = 16 * warp;
            const float *dc = reinterpret_cast<const float *>(sm + S::DC);
            const float d0 = dc[m0 + gq], d1 = dc[m0 + gq + 8];
#pragma unroll
            for (int nt = 0; nt < NTS; ++nt) {
                sacc[nt][0] *= d0;
                sacc[nt][1] *= d0;
                sacc[nt][2] *= d1;
                sacc[nt][3] *= d1;
            }
#pragma unroll
            for (int kk = 0; kk < 4; ++kk) {
                uint32_t a[4];
                {
                    const int j = lane >> 3;
                    const int row = 16 * kk + (lane & 7) + 8 * (j >> 1);
                    ldsm_x4_t(smem_u32(sm + S::KD) + swz_chunk(row, (m0 >> 3) + (j & 1), 256), a[0], a[1],
                              a[2], a[3]);
                }
#pragma unroll
                for (int np = 0; np < NTS / 2; ++np) {
                    const int j = lane >> 3;
                    const int row = 16 * kk + (lane & 7) + 8 * (j & 1);
                    uint32_t b0, b1, b2, b3;
                    ldsm_x4_t(smem_u32(sm + S::UT) + swz_chunk(row, 2 * np + (j >> 1), VS * 2), b0, b1, b2,
                              b3);
                    mma_bf16(sacc[2 * np], a, b0, b1);
                    mma_bf16(sacc[2 * np + 1], a, b2, b3);
                }
            }
#pragma unroll
            for (int nt = 0; nt < NTS; ++nt)
#pragma unroll
                for (int hh = 0; hh < 2; ++hh) {
                    const int row = m0 + gq + 8 * hh;
                    const int col = 8 * nt + 2 * tq;
                    *reinterpret_cast<uint32_t *>(sm + S::SB + swz_bf16(row, col, VS * 2)) =
                        pack_bf16(sacc[nt][2 * hh], sacc[nt][2 * hh + 1]);
                }
        }
        // the barrier at the top of the next iteration orders these writes
    }
}

template <int VS>
cudaError_t launch(const uint16_t *q, const uint16_t *k, const uint16_t *v, const float *g,
                   const float *beta, const int32_t *cu, int n_docs, int64_t T, int H,
                   uint16_t *out, int *status, cudaStream_t stream) {
    constexpr int bytes = Smem<VS>::BYTES;
    static_assert(bytes <= 232448, "shared memory budget");
    cudaError_t e = cudaFuncSetAttribute(kda_fwd_mma_kernel<VS>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
    if (e != cudaSuccess) return e;
    const int64_t blocks = (int64_t)n_docs * H * (kHeadDim / VS);
    kda_fwd_mma_kernel<VS><<<(unsigned)blocks, kThreads, bytes, stream>>>(q, k, v, g, beta, cu, n_docs, T,
                                                                         H, out, status);
    return cudaGetLastError();
}

}  // namespace mma_path

cudaError_t launch_fwd_mma(const uint16_t *q, const uint16_t *k, const uint16_t *v, const float *g,
                           const float *beta, const int32_t *cu, int n_docs, int64_t T, int H,
                           uint16_t *out, int *status, int v_slice, cudaStream_t stream) {
    if (v_slice == 128)
        return mma_path::launch<128>(q, k, v, g, beta, cu, n_docs, T, H, out, status, stream);
    return mma_path::launch<64>(q, k, v, g, beta, cu, n_docs, T, H, out, status, stream);
}

}  // namespace kda
