// kda_bwd.cu -- recompute-from-inputs backward of the chunk-KDA forward.
//
// Given the forward's inputs and the upstream gradient dO, computes dq, dk (of the raw,
// un-normalised q and k), dv, dg and dbeta; the pages' fused backward is a recompute backward
// with these outputs (kda_fused page of nemo_automodel.components.models.kimi_k3, the backward
// of fused_chunk_kda).
//
// Per 64-token chunk, with G the in-chunk inclusive cumsum of g, QG = q^ e^G, Kd = k^ e^{G_last - G},
// D = e^{G_last}, T = (I + A_kk)^-1, W = T diag(beta) K^e^G, U~ = U - W S and dS the gradient of the
// state leaving the chunk, the reverse mode is
//
//   dU~ = A_qk^T dO + Kd dS                     dS_in = D dS + QG^T dO - W^T dU~
//   dQG = dO S^T    dA_qk = lower(dO U~^T)      dKd = U~ dS^T     dW = -dU~ S^T
//   dT = dW (beta KG)^T + dU~ (beta V)^T        dA_kk = strict_lower(-T^T dT T^T)
//
// and then the chain rule through beta, the pairwise decays e^{G_r - G_i}, the factors e^G, the
// in-chunk cumsum (dg = reverse cumsum of dG) and the l2 norms.  Only dS crosses chunks, so the
// work splits into three launches:
//
//   1. the pipelined forward kernel (kda_fwd_pipe.cu) in its checkpoint instance: per chunk, the
//      state entering it and its U~ (transposed, bf16), the tensor-core operand tiles it built
//      anyway ([-W^T | scale QG^T], Kd^T, scale A_qk, bf16), T and A_hat (bf16) and D (fp32);
//   2. dstate (one CTA per document and head, chunks in reverse): the dS recurrence on tcgen05
//      with dS^T in tensor memory (fp32), its operands copied from the checkpoint block as flat
//      images, writing dS^T and dU~^T of every chunk;
//   3. grad (one CTA per chunk and head, all chunks at once): every gradient, from the chunk's
//      inputs, S, U~, T, A_hat, dS and dU~, with warp-level bf16 MMAs.
//
// Precision: every product takes bf16 operands with fp32 accumulation; T = (I + A_kk)^-1 and all
// elementwise work are fp32.  The pairwise-decay sums of dg cancel between their row and column
// sides; both sides multiply by the same bf16-rounded operands (k^ E1, q^ E1, k^ E2), so the
// cancellation stays exact and the rounding does not reach dg amplified.
//
// Tiles: every bf16 tile, in shared memory and in the workspace alike, is stored in 128-byte
// swizzled atoms: 64-column halves of rows x 128 bytes, the 16-byte chunk index XORed with
// (row & 7).  That is the tensor core's SWIZZLE_128B layout (K-major with rows = M or N, or
// MN-major with rows = K), and ldmatrix reads it without bank conflicts, so workspace tiles are
// copied to shared memory as flat byte images.  The library allocates nothing.
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "kda_common.cuh"
#include "kda_internal.h"
#include "kda_tc.cuh"

namespace kda {
namespace bwd {

constexpr int C = 64;     // chunk
constexpr int D = 128;    // head dim (K = V)
constexpr float kScale = 0.08838834764831845f;   // 1 / sqrt(128)
constexpr long long kWaitLimit = 2000000000LL;

// ---------------------------------------------------------------------------------------------
// Workspace: three regions, each [n_slots * H] blocks; the slot of chunk j of document d is
// cu[d] / 64 + d + j (unique, below T / 64 + n_docs, found without reading the lengths).
// ---------------------------------------------------------------------------------------------
struct Ws {
    // forward checkpoint block (written by the forward kernel's checkpoint instance)
    static constexpr size_t S = 0;                    // S^T bf16 [128 v][128 c], column groups of 16
    static constexpr size_t UT = 32768;               // U~^T bf16 [128 v][64 s], column groups of 32
    static constexpr size_t B2 = 49152;               // [-W^T | scale QG^T] bf16 [128 c][64 s | 64 t]
    static constexpr size_t KD = 81920;               // Kd^T bf16 [128 c][64 s]
    static constexpr size_t AQ = 98304;               // scale A_qk bf16 [64 t][64 s]
    static constexpr size_t TB = 106496;              // T bf16 [64 r][64 i]
    static constexpr size_t AH = 114688;              // A_hat bf16 [64 r][64 i], valid below the diagonal
    static constexpr size_t DL = 122880;              // D = e^{G_last} fp32 [128]
    static constexpr size_t CK = 123904;
    // dstate outputs
    static constexpr size_t DS = 0;                   // dS^T bf16 [128 v][128 c] (dS leaving the chunk), groups of 32
    static constexpr size_t DU = DS + 32768;          // dU~^T bf16 [128 v][64 s], column groups of 32
    static constexpr size_t DST = DU + 16384;
    static constexpr size_t PER_SLOT = CK + DST;
};

// Row-major tiles written by one thread per row (S^T, U~^T, dS^T, dU~^T in the workspace) are stored
// as column groups: the group's values of row 0, then of row 1, ..., so that the 32 rows of a warp
// land in one contiguous piece.  Byte offset of the 16 bytes holding columns 8m .. 8m + 7 of row r,
// with G columns per group and 128 rows:
__device__ __forceinline__ uint32_t grp_off(int r, int m, int G) {
    return (uint32_t)((8 * m / G) * 128 * G * 2 + r * G * 2 + (8 * m % G) * 2);
}

// byte offset of bf16 element (row, col) in a tile of `rows` rows (128-byte swizzled atoms)
__device__ __forceinline__ uint32_t at(int row, int col, int rows) {
    return (uint32_t)((col >> 6) * rows * 128 + row * 128 + ((((col >> 3) & 7) ^ (row & 7)) << 4) + ((col & 7) << 1));
}

// ---- warp-level bf16 MMA (m16n8k16) fragments from atom tiles --------------------------------
// A fragment (16 x 16 at m0, k0) of a tile stored [m][k] (rows = m) or, kT, [k][m] (rows = k)
template <bool kT>
__device__ __forceinline__ void frag_a(uint32_t base, int rows, int m0, int k0, uint32_t (&a)[4]) {
    const int lane = threadIdx.x & 31, j = lane >> 3, r = lane & 7;
    if constexpr (!kT) {
        ldsm_x4(base + at(m0 + (j & 1) * 8 + r, k0 + (j >> 1) * 8, rows), a[0], a[1], a[2], a[3]);
    } else {
        ldsm_x4_t(base + at(k0 + (j >> 1) * 8 + r, m0 + (j & 1) * 8, rows), a[0], a[1], a[2], a[3]);
    }
}
// B fragments of two n-tiles (k0..k0+15, n0..n0+15) of a tile stored [n][k] (rows = n) or, kT, [k][n]
// (rows = k): b[0], b[1] for columns n0..n0+7, b[2], b[3] for n0+8..n0+15
template <bool kT>
__device__ __forceinline__ void frag_b2(uint32_t base, int rows, int k0, int n0, uint32_t (&b)[4]) {
    const int lane = threadIdx.x & 31, j = lane >> 3, r = lane & 7;
    if constexpr (!kT) {
        ldsm_x4(base + at(n0 + (j >> 1) * 8 + r, k0 + (j & 1) * 8, rows), b[0], b[1], b[2], b[3]);
    } else {
        ldsm_x4_t(base + at(k0 + (j & 1) * 8 + r, n0 + (j >> 1) * 8, rows), b[0], b[1], b[2], b[3]);
    }
}
// acc[NT][4] += A(16 rows from m0, k in [k0, k1)) * B(k, NT * 8 columns from n0); NT even
template <int NT, bool kAT, bool kBT>
__device__ __forceinline__ void mma_rows(float (&acc)[NT][4], uint32_t a_base, int a_rows, int m0, uint32_t b_base,
                                         int b_rows, int n0, int k0, int k1) {
#pragma unroll 2
    for (int k = k0; k < k1; k += 16) {
        uint32_t a[4];
        frag_a<kAT>(a_base, a_rows, m0, k, a);
#pragma unroll
        for (int t = 0; t < NT; t += 2) {
            uint32_t b[4];
            frag_b2<kBT>(b_base, b_rows, k, n0 + 8 * t, b);
            mma_bf16(acc[t], a, b[0], b[1]);
            mma_bf16(acc[t + 1], a, b[2], b[3]);
        }
    }
}
// The same product with compile-time tile heights (AR, BR rows) and k range [K0, K1): addresses are
// per-thread constants plus compile-time offsets.  For a 16-aligned k the swizzled chunk of a lane's
// 16-byte row piece is ((k >> 3) & 7) ^ key with a per-thread key, and moving along the row index
// of a tile is a plain multiple of 128 bytes.
template <int NT, bool kAT, bool kBT, int AR, int BR, int K0, int K1>
__device__ __forceinline__ void mma_fix(float (&acc)[NT][4], uint32_t a_base, int m0, uint32_t b_base, int n0) {
    const int lane = threadIdx.x & 31, r = lane & 7, jlo = (lane >> 3) & 1, jhi = lane >> 4;
    uint32_t a_p, a_key4 = 0;
    if constexpr (!kAT) {
        a_p = a_base + (uint32_t)((m0 + jlo * 8 + r) * 128);
        a_key4 = (uint32_t)((jhi ^ r) << 4);
    } else {
        a_p = a_base + (uint32_t)((m0 >> 6) * AR * 128 + (jhi * 8 + r) * 128 + ((((m0 >> 3) & 7) ^ jlo ^ r) << 4));
    }
    uint32_t b_p[NT / 2];
    const uint32_t b_key4 = (uint32_t)((jlo ^ r) << 4);
#pragma unroll
    for (int tt = 0; tt < NT / 2; ++tt) {
        const int n = n0 + 16 * tt;
        if constexpr (!kBT) b_p[tt] = b_base + (uint32_t)((n + jhi * 8 + r) * 128);
        else b_p[tt] = b_base + (uint32_t)((n >> 6) * BR * 128 + (jlo * 8 + r) * 128 + ((((n >> 3) & 7) ^ jhi ^ r) << 4));
    }
#pragma unroll
    for (int k = K0; k < K1; k += 16) {
        uint32_t a[4];
        if constexpr (!kAT)
            ldsm_x4(a_p + (uint32_t)((k >> 6) * AR * 128) + ((uint32_t)(((k >> 3) & 7) << 4) ^ a_key4), a[0], a[1], a[2], a[3]);
        else
            ldsm_x4_t(a_p + (uint32_t)(k * 128), a[0], a[1], a[2], a[3]);
#pragma unroll
        for (int tt = 0; tt < NT / 2; ++tt) {
            uint32_t b[4];
            if constexpr (!kBT)
                ldsm_x4(b_p[tt] + (uint32_t)((k >> 6) * BR * 128) + ((uint32_t)(((k >> 3) & 7) << 4) ^ b_key4), b[0], b[1],
                        b[2], b[3]);
            else
                ldsm_x4_t(b_p[tt] + (uint32_t)(k * 128), b[0], b[1], b[2], b[3]);
            mma_bf16(acc[2 * tt], a, b[0], b[1]);
            mma_bf16(acc[2 * tt + 1], a, b[2], b[3]);
        }
    }
}
template <int NT>
__device__ __forceinline__ void zero_acc(float (&acc)[NT][4]) {
#pragma unroll
    for (int t = 0; t < NT; ++t) acc[t][0] = acc[t][1] = acc[t][2] = acc[t][3] = 0.f;
}

__device__ __forceinline__ float bfl(uint16_t b) { return __uint_as_float((uint32_t)b << 16); }
__device__ __forceinline__ uint16_t f2b(float x) { return __bfloat16_as_ushort(__float2bfloat16_rn(x)); }
__device__ __forceinline__ float2 bf2(uint32_t u) {
    return make_float2(__uint_as_float(u << 16), __uint_as_float(u & 0xffff0000u));
}

// chunk slot -> (document, first token, length); false when the slot holds no chunk or the
// document's bounds are invalid (the forward pass records KDA_ERR_BAD_SEQLENS for those)
__device__ __forceinline__ bool slot_chunk(const int32_t *cu, int n_docs, int64_t T, int slot, int &doc,
                                           int64_t &tok0, int &L) {
    int lo = 0, hi = n_docs - 1;
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        const int base = (int)((unsigned)cu[mid] / C) + mid;
        if (cu[mid] >= 0 && base <= slot) lo = mid;
        else hi = mid - 1;
    }
    const int64_t d0 = cu[lo], d1 = cu[lo + 1];
    if (d0 < 0 || d1 < d0 || d1 > T) return false;
    const int64_t j = (int64_t)slot - (d0 / C + lo);
    if (j < 0) return false;
    tok0 = d0 + j * C;
    if (tok0 >= d1) return false;
    doc = lo;
    L = (int)((d1 - tok0) < C ? (d1 - tok0) : C);
    return true;
}

// pair index p of block pair (R, I), I <= R, and back
__device__ __forceinline__ int pair_of(int R, int I) { return R * (R + 1) / 2 + I; }
__device__ __forceinline__ int pair_R(int p) { return p >= 6 ? 3 : p >= 3 ? 2 : p >= 1 ? 1 : 0; }

// l2 norms of rows [0, 64) of q and k (rows >= L zero): rq[r] = 1/sqrt(|q_r|^2 + 1e-6), rk likewise;
// one warp per row, nwarps warps
__device__ __forceinline__ void row_norms(const uint16_t *q, const uint16_t *k, int64_t tok0, int L, int H, int h,
                                          float *rq, float *rk, int nwarps) {
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    for (int r = warp; r < C; r += nwarps) {
        float sq = 0.f, sk = 0.f;
        if (r < L) {
            const int64_t off = ((tok0 + r) * H + h) * D + 4 * lane;
            const uint2 q4 = *reinterpret_cast<const uint2 *>(q + off), k4 = *reinterpret_cast<const uint2 *>(k + off);
            const float2 a = bf2(q4.x), b = bf2(q4.y), c = bf2(k4.x), d = bf2(k4.y);
            sq = a.x * a.x + a.y * a.y + b.x * b.x + b.y * b.y;
            sk = c.x * c.x + c.y * c.y + d.x * d.x + d.y * d.y;
        }
#pragma unroll
        for (int o = 16; o; o >>= 1) {
            sq += __shfl_xor_sync(0xffffffffu, sq, o);
            sk += __shfl_xor_sync(0xffffffffu, sk, o);
        }
        if (lane == 0) {
            rq[r] = rsqrtf(sq + 1e-6f);
            rk[r] = rsqrtf(sk + 1e-6f);
        }
    }
}

// flat copy of `bytes` (a multiple of 16) between 16-byte aligned buffers, all threads of the CTA
__device__ __forceinline__ void copy_out(uint8_t *dst, const uint8_t *src, int bytes, int nthreads) {
    for (int i = threadIdx.x; i < bytes / 16; i += nthreads)
        reinterpret_cast<uint4 *>(dst)[i] = reinterpret_cast<const uint4 *>(src)[i];
}

// =============================================================================================
// 2. dstate: one CTA per (document, head), chunks in reverse, dS^T [v][c] fp32 in tensor memory
//    (lane = value column v).  Per chunk, with the operands in shared memory:
//      dU~^T  = dS^T_bf16 Kd^T + dO^T (scale A_qk)          (N = 64)
//      dS^T  <- dS^T Diag(D) + dO^T (scale QG) + dU~^T_bf16 (-W)   (N = 128)
//    dS^T (bf16, before the update) and dU~^T (bf16) go to the chunk's workspace block.
// =============================================================================================
namespace dstate {
constexpr int kThreads = 128;
constexpr uint32_t kTmemCols = 256;
constexpr uint32_t kFS = 0;     // dS^T fp32 [128 v][128 c]
constexpr uint32_t kSB = 128;   // dS^T bf16, packed [128][64]
constexpr uint32_t kUB = 128;   // dU~^T bf16, packed [128][32] (over kSB once the dU~ product has read it)
constexpr uint32_t kDU = 192;   // dU~^T fp32 [128 v][64 s]
struct Sm {
    static constexpr int KD = 0;          // Kd^T [128 c][64 s]          MN-major B (K = c, N = s)
    static constexpr int AQ = 16384;      // scale A_qk [64 t][64 s]     MN-major B (K = t, N = s)
    static constexpr int WN = 24576;      // -W^T [128 c][64 s]          K-major B (N = c, K = s)
    static constexpr int QG = 40960;      // scale QG^T [128 c][64 t]    K-major B (N = c, K = t)
    static constexpr int DO = 57344;      // two buffers: dout [64 t][128 v]   MN-major A (K = t, M = v)
    static constexpr int DL = 90112;      // D fp32 [128]
    static constexpr int MBAR = DL + 512; // mbarriers: Kd/A_qk/D copies, [-W | QG] copy, dU~ product, state product
    static constexpr int TBASE = MBAR + 32, FLAG = TBASE + 8;
    static constexpr int TOTAL = FLAG + 8;
    static constexpr uint32_t kBytesA = 16384 + 8192 + 512;   // Kd^T, A_qk, D
    static constexpr uint32_t kBytesB = 32768;                // [-W^T | scale QG^T]
};

__device__ __forceinline__ void bulk_load(uint32_t dst, const void *src, uint32_t bytes, uint32_t mbar) {
    asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(dst),
                 "l"(src), "r"(bytes), "r"(mbar)
                 : "memory");
}
__device__ __forceinline__ void mma_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t b, uint32_t idesc, uint32_t acc) {
    asm volatile(
        "{\n.reg .pred p;\nsetp.ne.b32 p, %4, 0;\n"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n}\n" ::"r"(d_tmem),
        "r"(a_tmem), "l"(b), "r"(idesc), "r"(acc));
}
__device__ __forceinline__ void st16(uint32_t taddr, const uint32_t (&r)[16]) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};" ::"r"(
            taddr),
        "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]), "r"(r[9]),
        "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15])
        : "memory");
}
template <int N>
__device__ __forceinline__ void reg_fence(float (&v)[N]) {
#pragma unroll
    for (int i = 0; i < N; ++i) asm volatile("" : "+f"(v[i]));
}

__global__ void __launch_bounds__(kThreads, 2)
kda_bwd_dstate_kernel(const uint16_t *dout, const int32_t *cu, int n_docs, int64_t T, int H, const uint8_t *ws_ck,
                      uint8_t *ws_dst, int *status) {
    extern __shared__ __align__(1024) uint8_t sm[];
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int h = blockIdx.x % H;
    const int doc = doc_at_rank(cu, n_docs, blockIdx.x / H, reinterpret_cast<int *>(sm));
    const int64_t d0 = cu[doc], d1 = cu[doc + 1];
    if (d0 < 0 || d1 < d0 || d1 > T || d1 == d0) return;
    const int nch = (int)((d1 - d0 + C - 1) / C);
    const int64_t slot0 = d0 / C + doc;
    const uint32_t sbase = smem_u32(sm);
    const uint32_t mb_a = sbase + Sm::MBAR, mb_b = mb_a + 8, mb_u = mb_a + 16, mb_s = mb_a + 24;
    volatile int *flag = reinterpret_cast<volatile int *>(sm + Sm::FLAG);
    const float *dl = reinterpret_cast<const float *>(sm + Sm::DL);
    if (warp == 0) tc::alloc(sbase + Sm::TBASE, kTmemCols);
    if (tid == 0) {
        tc::mbar_init(mb_a, 1);
        tc::mbar_init(mb_b, 1);
        tc::mbar_init(mb_u, 1);
        tc::mbar_init(mb_s, 1);
        *flag = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    tc::fence_before();
    __syncthreads();
    tc::fence_after();
    const uint32_t tmem = *reinterpret_cast<volatile uint32_t *>(sm + Sm::TBASE);
    const uint32_t lane_base = tmem + ((uint32_t)(32 * warp) << 16);
    const int v = 32 * warp + lane;   // this thread's TMEM lane = value column

    // descriptors: K-major (-W^T, QG^T) and MN-major (dout, A_qk, Kd^T; 64-wide atoms 8 KB apart)
    const uint64_t dK = tc::sdesc(sbase, 16u, 1024u), dM = tc::sdesc(sbase, 64u * 128u, 1024u);
    constexpr uint32_t id_u1 = tc::idesc_bf16(128, 64, false, true, false);    // dS^T_bf16 (TMEM) x Kd^T
    constexpr uint32_t id_u2 = tc::idesc_bf16(128, 64, true, true, false);     // dO^T x A_qk
    constexpr uint32_t id_s1 = tc::idesc_bf16(128, 128, true, false, false);   // dO^T x QG
    constexpr uint32_t id_s2 = tc::idesc_bf16(128, 128, false, false, false);  // dU~^T_bf16 (TMEM) x (-W)

    // Each input group of chunk j is requested as soon as its buffer is free: Kd^T, A_qk and D once
    // chunk j+1's dU~ product and scaling have read them, [-W^T | scale QG^T] once chunk j+1's state
    // product has, and the dout rows a whole step ahead into the second buffer.
    auto load_a = [&](int j) {   // Kd^T, A_qk, D of chunk j (one thread)
        const uint8_t *src = ws_ck + ((size_t)(slot0 + j) * H + h) * Ws::CK;
        tc::mbar_expect_tx(mb_a, Sm::kBytesA);
        bulk_load(sbase + Sm::KD, src + Ws::KD, 16384, mb_a);
        bulk_load(sbase + Sm::AQ, src + Ws::AQ, 8192, mb_a);
        bulk_load(sbase + Sm::DL, src + Ws::DL, 512, mb_a);
    };
    auto load_b = [&](int j) {   // [-W^T | scale QG^T] of chunk j (one thread)
        const uint8_t *src = ws_ck + ((size_t)(slot0 + j) * H + h) * Ws::CK;
        tc::mbar_expect_tx(mb_b, Sm::kBytesB);
        bulk_load(sbase + Sm::WN, src + Ws::B2, 32768, mb_b);
    };
    auto load_do = [&](int j, int b) {   // dout rows of chunk j (zero past the document end) into buffer b
        const int64_t tok = d0 + (int64_t)j * C;
        const int Lj = (int)((d1 - tok) < C ? (d1 - tok) : C);
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            const int idx = tid + i * kThreads, t = idx >> 4, m = idx & 15;
            const bool ok = t < Lj;
            const uint16_t *src = ok ? dout + ((tok + t) * H + h) * D + 8 * m : dout;
            cp_async16(sbase + Sm::DO + b * 16384 + at(t, 8 * m, C), src, ok ? 16 : 0);
        }
        cp_async_commit();
    };
    // dS^T row v as bf16 into the workspace block of chunk j (and, optionally, into TMEM)
    auto store_ds = [&](int j, bool to_tmem) {
        uint8_t *dst = ws_dst + ((size_t)(slot0 + j) * H + h) * Ws::DST + Ws::DS + (size_t)v * 64;
#pragma unroll
        for (int q4 = 0; q4 < 4; ++q4) {
            float x[32];
            tc::ld32(lane_base + kFS + 32 * q4, x);
            tc::wait_ld();
            reg_fence(x);
            uint32_t pk[16];
#pragma unroll
            for (int i = 0; i < 16; ++i) pk[i] = pack_bf16(x[2 * i], x[2 * i + 1]);
            if (to_tmem) st16(lane_base + kSB + 16 * q4, pk);
#pragma unroll
            for (int e = 0; e < 4; ++e)   // channels 32 q4 + 8 e .. (column group q4)
                *reinterpret_cast<uint4 *>(dst + (size_t)q4 * (128 * 64) + 16 * e) =
                    make_uint4(pk[4 * e], pk[4 * e + 1], pk[4 * e + 2], pk[4 * e + 3]);
        }
    };

    // dS leaving the last chunk is zero
    {
        float z[32];
#pragma unroll
        for (int i = 0; i < 32; ++i) z[i] = 0.f;
#pragma unroll
        for (int q4 = 0; q4 < 4; ++q4) tc::st32(lane_base + kFS + 32 * q4, z);
        tc::st32(lane_base + kSB, z);
        tc::st32(lane_base + kSB + 32, z);
        tc::wait_st();
    }
    store_ds(nch - 1, false);
    load_do(nch - 1, 0);
    // the copies are issued by thread 32, so that thread 0 issues the products without waiting
    if (tid == 32) {
        load_a(nch - 1);
        load_b(nch - 1);
    }
    int last_a = nch - 1, last_b = nch - 1;   // the chunks whose copies were issued last

    bool aborted = false;
    int n_commit_s = 0;   // completions of the state-product barrier so far (the next has parity n & 1)
    for (int j = nch - 1; j >= 0; --j) {
        const int b = (nch - 1 - j) & 1;   // dout buffer of chunk j
        const uint32_t par = (uint32_t)b;
        const uint32_t dofs = (uint32_t)(b * (16384 >> 4));
        cp_async_wait_all();   // chunk j's dout rows (the only group in flight)
        tc::fence_proxy_async();
        bool ok = tc::mbar_wait(mb_a, par, kWaitLimit);
        tc::wait_st();
        tc::fence_before();
        if (__syncthreads_or(!ok)) {
            aborted = true;
            break;
        }
        // the other dout buffer was last read by chunk j+1's products, which have completed
        if (j > 0) load_do(j - 1, b ^ 1);
        if (tid == 0) {
            tc::fence_after();
#pragma unroll
            for (int kk = 0; kk < 8; ++kk)
                mma_ts(tmem + kDU, tmem + kSB + 8 * kk, dM + (uint64_t)((Sm::KD + kk * 2048) >> 4), id_u1, kk > 0);
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)
                tc::mma(tmem + kDU, dM + (uint64_t)((Sm::DO + kk * 2048) >> 4) + dofs,
                        dM + (uint64_t)((Sm::AQ + kk * 2048) >> 4), id_u2, 1u);
            tc::commit(mb_u);
        }
        // dS^T <- dS^T Diag(D) (the fp32 columns; the product above reads the bf16 copy)
#pragma unroll
        for (int q4 = 0; q4 < 4; ++q4) {
            float x[32];
            tc::ld32(lane_base + kFS + 32 * q4, x);
            tc::wait_ld();
            reg_fence(x);
#pragma unroll
            for (int i = 0; i < 32; ++i) x[i] *= dl[32 * q4 + i];
            tc::st32(lane_base + kFS + 32 * q4, x);
        }
        ok = tc::mbar_wait(mb_u, par, kWaitLimit);
        tc::fence_after();
        if (ok) {
            // dU~^T -> workspace (bf16 row v) and -> TMEM as the A operand of the update
            uint8_t *dst = ws_dst + ((size_t)(slot0 + j) * H + h) * Ws::DST + Ws::DU + (size_t)v * 64;
#pragma unroll
            for (int h2 = 0; h2 < 2; ++h2) {
                float x[32];
                tc::ld32(lane_base + kDU + 32 * h2, x);
                tc::wait_ld();
                reg_fence(x);
                uint32_t pk[16];
#pragma unroll
                for (int i = 0; i < 16; ++i) pk[i] = pack_bf16(x[2 * i], x[2 * i + 1]);
                st16(lane_base + kUB + 16 * h2, pk);
#pragma unroll
                for (int e = 0; e < 4; ++e)   // s = 32 h2 + 8 e .. (column group h2)
                    *reinterpret_cast<uint4 *>(dst + (size_t)h2 * (128 * 64) + 16 * e) =
                        make_uint4(pk[4 * e], pk[4 * e + 1], pk[4 * e + 2], pk[4 * e + 3]);
            }
        }
        ok = tc::mbar_wait(mb_b, par, kWaitLimit) && ok;   // chunk j's [-W^T | scale QG^T]
        tc::wait_st();
        tc::fence_proxy_async();   // D was read through the generic proxy; its buffer is refilled below
        tc::fence_before();
        if (__syncthreads_or(!ok)) {
            aborted = true;
            break;
        }
        // Kd^T and A_qk (read by the dU~ product, complete) and D (read by every thread above) are free
        if (j > 0 && tid == 32) load_a(j - 1);
        if (j > 0) last_a = j - 1;
        if (tid == 0) {
            tc::fence_after();
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)
                tc::mma(tmem + kFS, dM + (uint64_t)((Sm::DO + kk * 2048) >> 4) + dofs,
                        dK + (uint64_t)((Sm::QG + kk * 32) >> 4), id_s1, 1u);
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)
                mma_ts(tmem + kFS, tmem + kUB + 8 * kk, dK + (uint64_t)((Sm::WN + kk * 32) >> 4), id_s2, 1u);
            tc::commit(mb_s);
        }
        ++n_commit_s;
        ok = tc::mbar_wait(mb_s, par, kWaitLimit);
        tc::fence_after();
        if (__syncthreads_or(!ok)) {
            aborted = true;
            break;
        }
        if (j > 0) {
            if (tid == 32) load_b(j - 1);   // [-W^T | scale QG^T] was read by the state product
            last_b = j - 1;
            store_ds(j - 1, true);
            tc::wait_st();
        }
    }
    if (aborted) {
        // a wait ran out of time: record it, then wait (bounded) for the copies and tensor-core
        // operations still in flight before the CTA's shared memory and columns are released
        if (tid == 0) {
            atomicExch(status, kStatusTimeout);
            tc::mbar_wait(mb_a, (uint32_t)((nch - 1 - last_a) & 1), kWaitLimit);
            tc::mbar_wait(mb_b, (uint32_t)((nch - 1 - last_b) & 1), kWaitLimit);
            tc::commit(mb_s);
            tc::mbar_wait(mb_s, (uint32_t)(n_commit_s & 1), kWaitLimit);
        }
        cp_async_wait_all();
    }
    tc::fence_before();
    __syncthreads();
    tc::fence_after();
    if (warp == 0) tc::dealloc(tmem, kTmemCols);
}
}  // namespace dstate

// =============================================================================================
// 3. grad: one CTA per (chunk slot, head), 16 warps.  For 64 x 128 results warp w owns rows
//    16 (w & 3) .. +15 and columns 32 (w >> 2) .. +31 (four 16 x 8 tiles); the gradients of k^,
//    q^ and G at those positions stay in its registers from the first product to the last.
// =============================================================================================
namespace grad {
constexpr int kThreads = 512;
struct Sm {
    static constexpr int ST = 0;          // S^T [128 v][128 c]; then dW [64 s][128 c]
    static constexpr int DST = 32768;     // dS^T [128 v][128 c]; then dA_qk, dT, Xm, dA_hat (8 KB each)
    static constexpr int DAQ = DST, DT = DST + 8192, XM = DST + 16384, DAH = DST + 24576;
    static constexpr int DUT = 65536;     // dU~^T [128 v][64 s]; then pair scales fp32 [10][128]
    static constexpr int PS = DUT;
    static constexpr int XT = 81920;      // row-group totals of G (prep); then k^ E1 [64][128]
    static constexpr int TB = 98304;      // T [64 r][64 i]
    static constexpr int AH = 106496;     // A_hat [64 r][64 i]
    static constexpr int DO = 114688;     // dout [64 t][128 v]
    static constexpr int BV = 131072;     // beta v [64][128]; then q^ E1
    static constexpr int QT = BV;
    static constexpr int BK = 147456;     // beta k^ e^G [64][128]; then k^ E2
    static constexpr int YT = BK;
    static constexpr int UT = 163840;     // U~^T [128 v][64 s]
    static constexpr int GF = 180224;     // G (log2 units) fp32 [64][128], swizzled; then dG
    // partial sums are kept per producing warp and added in a fixed order (bit-reproducible results):
    // DGLP [6][128] dG_last (2 halves of S.dS, 4 row blocks of dKd Kd); DBP [12][64] dbeta (4 column
    // warps each of dBk.KG, dBv.v, dA_kk.A_hat); RED [2][64][4] the row dots of dq and dk
    static constexpr int RQ = 212992, RK = RQ + 256, BETA = RK + 256, DGLP = BETA + 256, DLS = DGLP + 3072,
                         GLS = DLS + 512, DBP = GLS + 512, RED = DBP + 3072, TOT = RED + 2048;
    static constexpr int TOTAL = TOT + 2048;
};
// fp32 [64][128] tile with the 8-float group index XORed with (row & 7): float2 reads of fragment
// positions (8 rows x 8 columns per warp) touch all 32 banks
__device__ __forceinline__ int gfi(int row, int col) { return row * D + (col ^ ((row & 7) << 3)); }

struct Args {
    const uint16_t *q, *k, *v, *dout;
    const float *g, *beta;
    const int32_t *cu;
    int n_docs;
    int64_t T;
    int H;
    const uint8_t *ws_ck, *ws_dst;
    uint16_t *dq, *dk, *dv;
    float *dg, *dbeta;
};
// TMA maps of dq, dk and dv over [T, H * 128] bf16, 64 x 64 boxes with 128-byte swizzled rows, and of
// dg over [T, H * 128] fp32, 64-row x 128-column boxes, unswizzled
struct OutMaps {
    CUtensorMap dq, dk, dv, dg;
};

__global__ void __launch_bounds__(kThreads, 1) kda_bwd_grad_kernel(const Args a, const __grid_constant__ OutMaps om) {
    extern __shared__ __align__(1024) uint8_t sm[];
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31, gq = lane >> 2, tq = lane & 3;
    const int H = a.H, slot = blockIdx.x / H, h = blockIdx.x % H;
    int doc, L;
    int64_t tok0;
    if (!slot_chunk(a.cu, a.n_docs, a.T, slot, doc, tok0, L)) return;
    const size_t blk = (size_t)slot * H + h;
    // A whole chunk writes dq, dk and dv by TMA stores from staged tiles; a partial chunk, whose rows
    // past the document end belong to the next document, stores its valid rows directly.
    const bool full = L == C;
    const uint8_t *ck = a.ws_ck + blk * Ws::CK, *dsb = a.ws_dst + blk * Ws::DST;
    const uint32_t sbase = smem_u32(sm);
    float *rq = reinterpret_cast<float *>(sm + Sm::RQ), *rk = reinterpret_cast<float *>(sm + Sm::RK);
    float *sbeta = reinterpret_cast<float *>(sm + Sm::BETA), *dglp = reinterpret_cast<float *>(sm + Sm::DGLP);
    float *dls = reinterpret_cast<float *>(sm + Sm::DLS), *gls = reinterpret_cast<float *>(sm + Sm::GLS);
    float *dbp = reinterpret_cast<float *>(sm + Sm::DBP), *red = reinterpret_cast<float *>(sm + Sm::RED);
    float *tot = reinterpret_cast<float *>(sm + Sm::TOT), *gf = reinterpret_cast<float *>(sm + Sm::GF);
    float *ps = reinterpret_cast<float *>(sm + Sm::PS);

    // ---- the prep's rows of q, k, v, g first, so that their latency overlaps the tile copies below
    //      (warp w holds rows 4w .. 4w + 3, lane l channels 4l .. 4l + 3; rows past the end are zero) ----
    const int pc0 = 4 * lane, pr0 = 4 * warp;
    uint2 qr[4], kr[4], vr[4];
    float4 gr[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const int r = pr0 + i;
        if (r < L) {
            const int64_t o = ((tok0 + r) * H + h) * D + pc0;
            qr[i] = __ldg(reinterpret_cast<const uint2 *>(a.q + o));
            kr[i] = __ldg(reinterpret_cast<const uint2 *>(a.k + o));
            vr[i] = __ldg(reinterpret_cast<const uint2 *>(a.v + o));
            gr[i] = __ldg(reinterpret_cast<const float4 *>(a.g + o));
        } else {
            qr[i] = kr[i] = vr[i] = make_uint2(0u, 0u);
            gr[i] = make_float4(0.f, 0.f, 0.f, 0.f);
        }
    }
    // ---- loads: workspace tiles as flat images, dout rows (zero past the document end) ----
    {
        // S^T, U~^T, dS^T, dU~^T: column groups -> swizzled atoms; T, A_hat: flat images.  Consecutive
        // threads take consecutive 16-byte pieces of a group image (piece i of the tile is piece j of
        // row r in group grp, i.e. grp_off(r, grp * G / 8 + j, G) = 16 i), so that every warp reads whole
        // 128-byte lines; reading row by row across the groups instead fills shared memory at half the rate.
        const uint8_t *gsrc[4] = {ck + Ws::S, ck + Ws::UT, dsb + Ws::DS, dsb + Ws::DU};
        const int gdst[4] = {Sm::ST, Sm::UT, Sm::DST, Sm::DUT}, gcols[4] = {128, 64, 128, 64}, ggrp[4] = {16, 32, 32, 32};
#pragma unroll
        for (int t = 0; t < 4; ++t) {
            const int pg = ggrp[t] / 8;   // pieces per row inside a group
            for (int i = tid; i < 16 * gcols[t]; i += kThreads) {
                const int grp = i / (128 * pg), k = i % (128 * pg), r = k / pg, m = grp * pg + k % pg;
                cp_async16(sbase + gdst[t] + at(r, 8 * m, D), gsrc[t] + 16 * i, 16);
            }
        }
        for (int i = tid; i < 8192 / 16; i += kThreads) {
            cp_async16(sbase + Sm::TB + 16 * i, ck + Ws::TB + 16 * i, 16);
            cp_async16(sbase + Sm::AH + 16 * i, ck + Ws::AH + 16 * i, 16);
        }
#pragma unroll
        for (int i = 0; i < 2; ++i) {
            const int idx = tid + i * kThreads, t = idx >> 4, m = idx & 15;
            const bool ok = t < L;
            const uint16_t *s = ok ? a.dout + ((tok0 + t) * H + h) * D + 8 * m : a.dout;
            cp_async16(sbase + Sm::DO + at(t, 8 * m, C), s, ok ? 16 : 0);
        }
        cp_async_commit();
    }
    if (tid < C) sbeta[tid] = tid < L ? __ldg(a.beta + (tok0 + tid) * H + h) : 0.f;
    if (tid < D) dls[tid] = reinterpret_cast<const float *>(ck + Ws::DL)[tid];

    // ---- prep: row norms, G (log2 units), beta k^ e^G and beta v ----
    {
        const int c0 = pc0, r0 = pr0;
        float rkr[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const float2 qa = bf2(qr[i].x), qb = bf2(qr[i].y), ka = bf2(kr[i].x), kb = bf2(kr[i].y);
            float sq = qa.x * qa.x + qa.y * qa.y + qb.x * qb.x + qb.y * qb.y;
            float sk = ka.x * ka.x + ka.y * ka.y + kb.x * kb.x + kb.y * kb.y;
#pragma unroll
            for (int o = 16; o; o >>= 1) {
                sq += __shfl_xor_sync(0xffffffffu, sq, o);
                sk += __shfl_xor_sync(0xffffffffu, sk, o);
            }
            rkr[i] = rsqrtf(sk + 1e-6f);
            if (lane == 0) {
                rq[r0 + i] = rsqrtf(sq + 1e-6f);
                rk[r0 + i] = rkr[i];
            }
        }
        float g2[4][4], run[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const float x[4] = {gr[i].x, gr[i].y, gr[i].z, gr[i].w};
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                run[e] += x[e] * kLog2e;
                g2[i][e] = run[e];
            }
        }
        float *gt = reinterpret_cast<float *>(sm + Sm::XT);   // [16][128] row-group totals
        *reinterpret_cast<float4 *>(gt + warp * D + c0) = make_float4(run[0], run[1], run[2], run[3]);
        __syncthreads();
        float off[4] = {0.f, 0.f, 0.f, 0.f};
        for (int w2 = 0; w2 < warp; ++w2) {
            const float4 t4 = *reinterpret_cast<const float4 *>(gt + w2 * D + c0);
            off[0] += t4.x; off[1] += t4.y; off[2] += t4.z; off[3] += t4.w;
        }
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const int r = r0 + i;
            float bk[4], bv[4];
            const float2 ka = bf2(kr[i].x), kb = bf2(kr[i].y), va = bf2(vr[i].x), vb = bf2(vr[i].y);
            const float kv[4] = {ka.x, ka.y, kb.x, kb.y}, vv[4] = {va.x, va.y, vb.x, vb.y};
            const float br = sbeta[r];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                g2[i][e] += off[e];
                bk[e] = br * kv[e] * rkr[i] * ex2_ftz(g2[i][e]);
                bv[e] = br * vv[e];
            }
            *reinterpret_cast<float4 *>(gf + gfi(r, c0)) = make_float4(g2[i][0], g2[i][1], g2[i][2], g2[i][3]);
            const uint32_t o2 = at(r, c0, C);
            *reinterpret_cast<uint2 *>(sm + Sm::BK + o2) =
                make_uint2(pack_bf16(bk[0], bk[1]), pack_bf16(bk[2], bk[3]));
            *reinterpret_cast<uint2 *>(sm + Sm::BV + o2) =
                make_uint2(pack_bf16(bv[0], bv[1]), pack_bf16(bv[2], bv[3]));
        }
        if (warp == 15) *reinterpret_cast<float4 *>(gls + c0) = make_float4(g2[3][0], g2[3][1], g2[3][2], g2[3][3]);
    }
    cp_async_wait_all();
    __syncthreads();

    // ---- dG_last part 1: D[c] sum_v S[c][v] dS[c][v], from matching B fragments of S^T and dS^T ----
    {
        const int c0 = 16 * (warp & 7), kb = 64 * (warp >> 3);
        float s0 = 0.f, s1 = 0.f;
#pragma unroll
        for (int kk = 0; kk < 64; kk += 16) {
            uint32_t bs[4], bd[4];
            frag_b2<true>(sbase + Sm::ST, D, kb + kk, c0, bs);
            frag_b2<true>(sbase + Sm::DST, D, kb + kk, c0, bd);
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const float2 x = bf2(bs[e]), y = bf2(bd[e]);
                const float p = x.x * y.x + x.y * y.y;
                if (e < 2) s0 += p;
                else s1 += p;
            }
        }
        s0 += __shfl_xor_sync(0xffffffffu, s0, 1);
        s0 += __shfl_xor_sync(0xffffffffu, s0, 2);
        s1 += __shfl_xor_sync(0xffffffffu, s1, 1);
        s1 += __shfl_xor_sync(0xffffffffu, s1, 2);
        if (tq == 0) {
            dglp[(warp >> 3) * D + c0 + gq] = dls[c0 + gq] * s0;
            dglp[(warp >> 3) * D + c0 + 8 + gq] = dls[c0 + 8 + gq] * s1;
        }
    }

    const int rb = warp & 3, cb = warp >> 2, m0 = 16 * rb, n0 = 32 * cb;
    float dkn[4][4], dqn[4][4], dG[4][4];
    zero_acc(dkn);
    zero_acc(dqn);
    zero_acc(dG);
    // element (t, e) of a 64 x 128 result: row m0 + gq + 8 (e >> 1), column n0 + 8 t + 2 tq + (e & 1)
    // raw bf16 pairs (row, col..col+1) of q / k / v at this thread's result positions (zero past the
    // document end), read through the non-coherent path and issued before the product they serve
    auto ld_pairs = [&](const uint16_t *p, uint32_t (&u)[4][2]) {
#pragma unroll
        for (int t = 0; t < 4; ++t)
#pragma unroll
            for (int hh = 0; hh < 2; ++hh) {
                const int row = m0 + gq + 8 * hh, col = n0 + 8 * t + 2 * tq;
                u[t][hh] = row < L ? __ldg(reinterpret_cast<const unsigned int *>(p + ((tok0 + row) * H + h) * D + col))
                                   : 0u;
            }
    };

    // ---- dKd = U~ dS^T: dk^ += dKd e^{G_last - G}, dG -= dKd Kd, dG_last += sum_r dKd Kd ----
    {
        uint32_t kp[4][2];
        ld_pairs(a.k, kp);
        float acc[4][4];
        zero_acc(acc);
        mma_fix<4, true, true, D, D, 0, D>(acc, sbase + Sm::UT, m0, sbase + Sm::DST, n0);
        float cs[4][2];
#pragma unroll
        for (int t = 0; t < 4; ++t) {
            cs[t][0] = cs[t][1] = 0.f;
#pragma unroll
            for (int hh = 0; hh < 2; ++hh) {
                const int row = m0 + gq + 8 * hh, col = n0 + 8 * t + 2 * tq;
                const float2 g2 = *reinterpret_cast<const float2 *>(gf + gfi(row, col));
                const float2 kr = bf2(kp[t][hh]);
                const float ed0 = ex2_ftz(gls[col] - g2.x), ed1 = ex2_ftz(gls[col + 1] - g2.y);
                const float kd0 = kr.x * rk[row] * ed0, kd1 = kr.y * rk[row] * ed1;
                const float x0 = acc[t][2 * hh], x1 = acc[t][2 * hh + 1];
                dkn[t][2 * hh] += x0 * ed0;
                dkn[t][2 * hh + 1] += x1 * ed1;
                dG[t][2 * hh] -= x0 * kd0;
                dG[t][2 * hh + 1] -= x1 * kd1;
                cs[t][0] += x0 * kd0;
                cs[t][1] += x1 * kd1;
            }
        }
#pragma unroll
        for (int t = 0; t < 4; ++t)
#pragma unroll
            for (int e = 0; e < 2; ++e) {
                float x = cs[t][e];
                x += __shfl_xor_sync(0xffffffffu, x, 4);
                x += __shfl_xor_sync(0xffffffffu, x, 8);
                x += __shfl_xor_sync(0xffffffffu, x, 16);
                if (gq == 0) dglp[(2 + rb) * D + n0 + 8 * t + 2 * tq + e] = x;
            }
    }
    // ---- dQG = scale dO S^T: dq^ += dQG e^G, dG += dQG QG ----
    {
        uint32_t qp[4][2];
        ld_pairs(a.q, qp);
        float acc[4][4];
        zero_acc(acc);
        mma_fix<4, false, true, C, D, 0, D>(acc, sbase + Sm::DO, m0, sbase + Sm::ST, n0);
#pragma unroll
        for (int t = 0; t < 4; ++t)
#pragma unroll
            for (int hh = 0; hh < 2; ++hh) {
                const int row = m0 + gq + 8 * hh, col = n0 + 8 * t + 2 * tq;
                const float2 g2 = *reinterpret_cast<const float2 *>(gf + gfi(row, col));
                const float2 qr = bf2(qp[t][hh]);
                const float e0 = ex2_ftz(g2.x), e1 = ex2_ftz(g2.y);
                const float x0 = kScale * acc[t][2 * hh], x1 = kScale * acc[t][2 * hh + 1];
                dqn[t][2 * hh] += x0 * e0;
                dqn[t][2 * hh + 1] += x1 * e1;
                dG[t][2 * hh] += x0 * qr.x * rq[row] * e0;
                dG[t][2 * hh + 1] += x1 * qr.y * rq[row] * e1;
            }
    }
    // ---- dW = -dU~ S^T (kept in registers until every warp is done with S) ----
    float dw[4][4];
    zero_acc(dw);
    mma_fix<4, true, true, D, D, 0, D>(dw, sbase + Sm::DUT, m0, sbase + Sm::ST, n0);
    __syncthreads();   // S^T and dS^T are read: their space takes dW and the 64 x 64 tiles
#pragma unroll
    for (int t = 0; t < 4; ++t)
#pragma unroll
        for (int hh = 0; hh < 2; ++hh)
            *reinterpret_cast<uint32_t *>(sm + Sm::ST + at(m0 + gq + 8 * hh, n0 + 8 * t + 2 * tq, C)) =
                pack_bf16(-dw[t][2 * hh], -dw[t][2 * hh + 1]);

    // 64 x 64 results: warp w owns rows 16 (w & 3) and columns 16 (w >> 2) (two 16 x 8 tiles)
    const int n64 = 16 * cb;
    // ---- dA_qk = scale lower(dO U~^T) ----
    {
        float acc[2][4];
        zero_acc(acc);
        mma_fix<2, false, true, C, D, 0, D>(acc, sbase + Sm::DO, m0, sbase + Sm::UT, n64);
#pragma unroll
        for (int t = 0; t < 2; ++t)
#pragma unroll
            for (int hh = 0; hh < 2; ++hh) {
                const int row = m0 + gq + 8 * hh, col = n64 + 8 * t + 2 * tq;
                const float x0 = col <= row ? kScale * acc[t][2 * hh] : 0.f;
                const float x1 = col + 1 <= row ? kScale * acc[t][2 * hh + 1] : 0.f;
                *reinterpret_cast<uint32_t *>(sm + Sm::DAQ + at(row, col, C)) = pack_bf16(x0, x1);
            }
    }
    __syncthreads();   // dW in place
    // ---- dT = dW (beta KG)^T + dU~ (beta V)^T ----
    {
        float acc[2][4];
        zero_acc(acc);
        mma_fix<2, false, false, C, C, 0, D>(acc, sbase + Sm::ST, m0, sbase + Sm::BK, n64);
        mma_fix<2, true, false, D, C, 0, D>(acc, sbase + Sm::DUT, m0, sbase + Sm::BV, n64);
#pragma unroll
        for (int t = 0; t < 2; ++t)
#pragma unroll
            for (int hh = 0; hh < 2; ++hh)
                *reinterpret_cast<uint32_t *>(sm + Sm::DT + at(m0 + gq + 8 * hh, n64 + 8 * t + 2 * tq, C)) =
                    pack_bf16(acc[t][2 * hh], acc[t][2 * hh + 1]);
    }
    // ---- dBk = T^T dW: dKG = beta dBk; dk^ += dKG e^G, dG += dKG KG, dbeta += dBk . KG ----
    {
        uint32_t kp[4][2];
        ld_pairs(a.k, kp);
        float acc[4][4];
        zero_acc(acc);
        mma_fix<4, true, true, C, C, 0, C>(acc, sbase + Sm::TB, m0, sbase + Sm::ST, n0);
        float rs[2] = {0.f, 0.f};
#pragma unroll
        for (int t = 0; t < 4; ++t)
#pragma unroll
            for (int hh = 0; hh < 2; ++hh) {
                const int row = m0 + gq + 8 * hh, col = n0 + 8 * t + 2 * tq;
                const float2 g2 = *reinterpret_cast<const float2 *>(gf + gfi(row, col));
                const float2 kr = bf2(kp[t][hh]);
                const float e0 = ex2_ftz(g2.x), e1 = ex2_ftz(g2.y);
                const float kg0 = kr.x * rk[row] * e0, kg1 = kr.y * rk[row] * e1;
                const float b = sbeta[row];
                const float x0 = acc[t][2 * hh], x1 = acc[t][2 * hh + 1];
                dkn[t][2 * hh] += b * x0 * e0;
                dkn[t][2 * hh + 1] += b * x1 * e1;
                dG[t][2 * hh] += b * x0 * kg0;
                dG[t][2 * hh + 1] += b * x1 * kg1;
                rs[hh] += x0 * kg0 + x1 * kg1;
            }
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) {
            float x = rs[hh];
            x += __shfl_xor_sync(0xffffffffu, x, 1);
            x += __shfl_xor_sync(0xffffffffu, x, 2);
            if (tq == 0) dbp[(0 + cb) * C + m0 + gq + 8 * hh] = x;
        }
    }
    // ---- dBv = T^T dU~: dv = beta dBv, dbeta += dBv . v ----
    {
        uint32_t vp[4][2];
        ld_pairs(a.v, vp);
        float acc[4][4];
        zero_acc(acc);
        mma_fix<4, true, false, C, D, 0, C>(acc, sbase + Sm::TB, m0, sbase + Sm::DUT, n0);
        float rs[2] = {0.f, 0.f};
#pragma unroll
        for (int t = 0; t < 4; ++t)
#pragma unroll
            for (int hh = 0; hh < 2; ++hh) {
                const int row = m0 + gq + 8 * hh, col = n0 + 8 * t + 2 * tq;
                const float x0 = acc[t][2 * hh], x1 = acc[t][2 * hh + 1];
                if (row < L) {
                    const float2 vr = bf2(vp[t][hh]);
                    rs[hh] += x0 * vr.x + x1 * vr.y;
                    const float b = sbeta[row];
                    const uint32_t pv = pack_bf16(b * x0, b * x1);
                    if (full)   // dout's tile is free since dA_qk
                        *reinterpret_cast<uint32_t *>(sm + Sm::DO + at(row, col, C)) = pv;
                    else
                        *reinterpret_cast<uint32_t *>(a.dv + ((tok0 + row) * H + h) * D + col) = pv;
                }
            }
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) {
            float x = rs[hh];
            x += __shfl_xor_sync(0xffffffffu, x, 1);
            x += __shfl_xor_sync(0xffffffffu, x, 2);
            if (tq == 0) dbp[(4 + cb) * C + m0 + gq + 8 * hh] = x;
        }
    }
    if (full) tc::fence_proxy_async();   // the staged dv tile is read by the TMA engine
    __syncthreads();   // dT in place; dW, dU~^T, beta V, beta KG are read
    if (full && tid == 0) {
        tc::tma_store_2d(&om.dv, h * D, (int)tok0, sbase + Sm::DO);
        tc::tma_store_2d(&om.dv, h * D + 64, (int)tok0, sbase + Sm::DO + 8192);
        tc::bulk_commit();
    }
    // ---- Xm = T^T dT ----
    {
        float acc[2][4];
        zero_acc(acc);
        mma_fix<2, true, true, C, C, 0, C>(acc, sbase + Sm::TB, m0, sbase + Sm::DT, n64);
#pragma unroll
        for (int t = 0; t < 2; ++t)
#pragma unroll
            for (int hh = 0; hh < 2; ++hh)
                *reinterpret_cast<uint32_t *>(sm + Sm::XM + at(m0 + gq + 8 * hh, n64 + 8 * t + 2 * tq, C)) =
                    pack_bf16(acc[t][2 * hh], acc[t][2 * hh + 1]);
    }
    // ---- k^ E1, q^ E1, k^ E2 (the pairwise-decay operands, bf16) and the pair scales: warp w holds
    //      rows 4w .. 4w + 3, lane l channels 4l .. 4l + 3 ----
    {
        const int c0 = 4 * lane, r0 = 4 * warp, BR = warp >> 2;
        uint2 qr[4], kr[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const int r = r0 + i;
            if (r < L) {
                const int64_t o = ((tok0 + r) * H + h) * D + c0;
                qr[i] = __ldg(reinterpret_cast<const uint2 *>(a.q + o));
                kr[i] = __ldg(reinterpret_cast<const uint2 *>(a.k + o));
            } else {
                qr[i] = kr[i] = make_uint2(0u, 0u);
            }
        }
        const float4 gs4 = *reinterpret_cast<const float4 *>(gf + gfi(16 * BR, c0));
        const float4 ge4 = *reinterpret_cast<const float4 *>(gf + gfi(16 * BR + 15, c0));
        const float gs[4] = {gs4.x, gs4.y, gs4.z, gs4.w}, ge[4] = {ge4.x, ge4.y, ge4.z, ge4.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const int r = r0 + i;
            const float4 g4 = *reinterpret_cast<const float4 *>(gf + gfi(r, c0));
            const float gv[4] = {g4.x, g4.y, g4.z, g4.w};
            const float2 qa = bf2(qr[i].x), qb = bf2(qr[i].y), ka = bf2(kr[i].x), kb = bf2(kr[i].y);
            const float qv[4] = {qa.x, qa.y, qb.x, qb.y}, kv[4] = {ka.x, ka.y, kb.x, kb.y};
            const float iq = rq[r], ik = rk[r];
            float x[4], y[4], z[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const float e1 = ex2_ftz(gv[e] - gs[e]);
                x[e] = kv[e] * ik * e1;
                y[e] = qv[e] * iq * e1;
                z[e] = kv[e] * ik * ex2_ftz(ge[e] - gv[e]);
            }
            const uint32_t o2 = at(r, c0, C);
            *reinterpret_cast<uint2 *>(sm + Sm::XT + o2) = make_uint2(pack_bf16(x[0], x[1]), pack_bf16(x[2], x[3]));
            *reinterpret_cast<uint2 *>(sm + Sm::QT + o2) = make_uint2(pack_bf16(y[0], y[1]), pack_bf16(y[2], y[3]));
            *reinterpret_cast<uint2 *>(sm + Sm::YT + o2) = make_uint2(pack_bf16(z[0], z[1]), pack_bf16(z[2], z[3]));
        }
        if (warp < 10) {
            const int PR = pair_R(warp), PI = warp - PR * (PR + 1) / 2;
            const float4 a4 = *reinterpret_cast<const float4 *>(gf + gfi(16 * PR, c0));
            const float4 b4 = *reinterpret_cast<const float4 *>(gf + gfi(16 * PI + 15, c0));
            *reinterpret_cast<float4 *>(ps + warp * D + c0) =
                make_float4(ex2_ftz(a4.x - b4.x), ex2_ftz(a4.y - b4.y), ex2_ftz(a4.z - b4.z), ex2_ftz(a4.w - b4.w));
        }
    }
    __syncthreads();   // Xm in place
    // ---- dA_kk = strict_lower(-Xm T^T): dbeta += dA_kk . A_hat, dA_hat = beta dA_kk ----
    {
        float acc[2][4];
        zero_acc(acc);
        mma_fix<2, false, false, C, C, 0, C>(acc, sbase + Sm::XM, m0, sbase + Sm::TB, n64);
        float rs[2] = {0.f, 0.f};
#pragma unroll
        for (int t = 0; t < 2; ++t)
#pragma unroll
            for (int hh = 0; hh < 2; ++hh) {
                const int row = m0 + gq + 8 * hh, col = n64 + 8 * t + 2 * tq;
                const float x0 = col < row ? -acc[t][2 * hh] : 0.f, x1 = col + 1 < row ? -acc[t][2 * hh + 1] : 0.f;
                // A_hat is defined below the diagonal only: the rest of its tile is never read
                const float2 ah = col < row ? bf2(*reinterpret_cast<const uint32_t *>(sm + Sm::AH + at(row, col, C)))
                                            : make_float2(0.f, 0.f);
                rs[hh] += x0 * ah.x + (col + 1 < row ? x1 * ah.y : 0.f);
                const float b = sbeta[row];
                *reinterpret_cast<uint32_t *>(sm + Sm::DAH + at(row, col, C)) = pack_bf16(b * x0, b * x1);
            }
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) {
            float x = rs[hh];
            x += __shfl_xor_sync(0xffffffffu, x, 1);
            x += __shfl_xor_sync(0xffffffffu, x, 2);
            if (tq == 0) dbp[(8 + cb) * C + m0 + gq + 8 * hh] = x;
        }
    }
    __syncthreads();   // dA_hat, dA_qk, the pairwise operands and scales in place
    // ---- pairwise-decay sums, block pair by block pair (pair scale per column) ----
    //   row side    (rows r in block rb): P1 = sum_{I<=rb} s (dA_hat[rb,I] Y~_I),  P3 likewise with dA_qk
    //   column side (rows i in block rb): P24 = sum_{R>=rb} s (dA_hat[R,rb]^T X~_R + dA_qk[R,rb]^T Q~_R)
    //   dk^ += E1 P1 + E2 P24,  dq^ += E1 P3,  dG += X~ P1 + Q~ P3 - Y~ P24
    {
        float p1[4][4], p3[4][4];
        zero_acc(p1);
        zero_acc(p3);
        for (int I = 0; I <= rb; ++I) {
            const int p = pair_of(rb, I);
            float t1[4][4], t3[4][4];
            zero_acc(t1);
            zero_acc(t3);
            mma_rows<4, false, true>(t1, sbase + Sm::DAH, C, m0, sbase + Sm::YT, C, n0, 16 * I, 16 * I + 16);
            mma_rows<4, false, true>(t3, sbase + Sm::DAQ, C, m0, sbase + Sm::YT, C, n0, 16 * I, 16 * I + 16);
#pragma unroll
            for (int t = 0; t < 4; ++t) {
                const float2 s = *reinterpret_cast<const float2 *>(ps + p * D + n0 + 8 * t + 2 * tq);
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const float se = (e & 1) ? s.y : s.x;
                    p1[t][e] += se * t1[t][e];
                    p3[t][e] += se * t3[t][e];
                }
            }
        }
#pragma unroll
        for (int t = 0; t < 4; ++t)
#pragma unroll
            for (int hh = 0; hh < 2; ++hh) {
                const int row = m0 + gq + 8 * hh, col = n0 + 8 * t + 2 * tq;
                const float2 g2 = *reinterpret_cast<const float2 *>(gf + gfi(row, col));
                const float2 gs = *reinterpret_cast<const float2 *>(gf + gfi(m0, col));
                const float e0 = ex2_ftz(g2.x - gs.x), e1 = ex2_ftz(g2.y - gs.y);
                const float2 xt = bf2(*reinterpret_cast<const uint32_t *>(sm + Sm::XT + at(row, col, C)));
                const float2 qt = bf2(*reinterpret_cast<const uint32_t *>(sm + Sm::QT + at(row, col, C)));
                dkn[t][2 * hh] += e0 * p1[t][2 * hh];
                dkn[t][2 * hh + 1] += e1 * p1[t][2 * hh + 1];
                dqn[t][2 * hh] += e0 * p3[t][2 * hh];
                dqn[t][2 * hh + 1] += e1 * p3[t][2 * hh + 1];
                dG[t][2 * hh] += xt.x * p1[t][2 * hh] + qt.x * p3[t][2 * hh];
                dG[t][2 * hh + 1] += xt.y * p1[t][2 * hh + 1] + qt.y * p3[t][2 * hh + 1];
            }
    }
    uint32_t qf[4][2], kf[4][2];   // q and k at the result positions, for the final phase
    ld_pairs(a.q, qf);
    ld_pairs(a.k, kf);
    {
        float p24[4][4];
        zero_acc(p24);
        for (int R = rb; R < 4; ++R) {
            const int p = pair_of(R, rb);
            float t2[4][4];
            zero_acc(t2);
            mma_rows<4, true, true>(t2, sbase + Sm::DAH, C, m0, sbase + Sm::XT, C, n0, 16 * R, 16 * R + 16);
            mma_rows<4, true, true>(t2, sbase + Sm::DAQ, C, m0, sbase + Sm::QT, C, n0, 16 * R, 16 * R + 16);
#pragma unroll
            for (int t = 0; t < 4; ++t) {
                const float2 s = *reinterpret_cast<const float2 *>(ps + p * D + n0 + 8 * t + 2 * tq);
#pragma unroll
                for (int e = 0; e < 4; ++e) p24[t][e] += ((e & 1) ? s.y : s.x) * t2[t][e];
            }
        }
#pragma unroll
        for (int t = 0; t < 4; ++t)
#pragma unroll
            for (int hh = 0; hh < 2; ++hh) {
                const int row = m0 + gq + 8 * hh, col = n0 + 8 * t + 2 * tq;
                const float2 g2 = *reinterpret_cast<const float2 *>(gf + gfi(row, col));
                const float2 ge = *reinterpret_cast<const float2 *>(gf + gfi(m0 + 15, col));
                const float e0 = ex2_ftz(ge.x - g2.x), e1 = ex2_ftz(ge.y - g2.y);
                const float2 yt = bf2(*reinterpret_cast<const uint32_t *>(sm + Sm::YT + at(row, col, C)));
                dkn[t][2 * hh] += e0 * p24[t][2 * hh];
                dkn[t][2 * hh + 1] += e1 * p24[t][2 * hh + 1];
                dG[t][2 * hh] -= yt.x * p24[t][2 * hh];
                dG[t][2 * hh + 1] -= yt.y * p24[t][2 * hh + 1];
            }
    }

    // ---- dq, dk through the l2 norms (row dots across the four column warps), dG to shared ----
    {
        float sq[2] = {0.f, 0.f}, sk[2] = {0.f, 0.f};
#pragma unroll
        for (int t = 0; t < 4; ++t)
#pragma unroll
            for (int hh = 0; hh < 2; ++hh) {
                const int row = m0 + gq + 8 * hh;
                const float2 qr = bf2(qf[t][hh]), kr = bf2(kf[t][hh]);
                sq[hh] += rq[row] * (qr.x * dqn[t][2 * hh] + qr.y * dqn[t][2 * hh + 1]);
                sk[hh] += rk[row] * (kr.x * dkn[t][2 * hh] + kr.y * dkn[t][2 * hh + 1]);
            }
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) {
            float x = sq[hh], y = sk[hh];
            x += __shfl_xor_sync(0xffffffffu, x, 1);
            x += __shfl_xor_sync(0xffffffffu, x, 2);
            y += __shfl_xor_sync(0xffffffffu, y, 1);
            y += __shfl_xor_sync(0xffffffffu, y, 2);
            if (tq == 0) {
                red[(m0 + gq + 8 * hh) * 4 + cb] = x;
                red[256 + (m0 + gq + 8 * hh) * 4 + cb] = y;
            }
        }
    }
    __syncthreads();   // row dots in place; every read of G is done
    // A whole chunk stages dq and dk as bf16 tiles in the space S^T and dW held (free since dBk),
    // [64 rows][128] each with 128-byte swizzled rows, and writes them with four TMA stores; the
    // per-thread pairs would otherwise leave as scattered 4-byte stores (8 rows x 16 bytes per warp
    // instruction).
#pragma unroll
    for (int t = 0; t < 4; ++t)
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) {
            const int row = m0 + gq + 8 * hh, col = n0 + 8 * t + 2 * tq;
            *reinterpret_cast<float2 *>(gf + gfi(row, col)) = make_float2(dG[t][2 * hh], dG[t][2 * hh + 1]);
            if (row < L) {
                const float4 s4 = *reinterpret_cast<const float4 *>(red + row * 4);
                const float4 k4 = *reinterpret_cast<const float4 *>(red + 256 + row * 4);
                const float sq = s4.x + s4.y + s4.z + s4.w, sk = k4.x + k4.y + k4.z + k4.w;
                const float2 qr = bf2(qf[t][hh]), kr = bf2(kf[t][hh]);
                const float iq = rq[row], ik = rk[row];
                const uint32_t pq =
                    pack_bf16(iq * (dqn[t][2 * hh] - qr.x * iq * sq), iq * (dqn[t][2 * hh + 1] - qr.y * iq * sq));
                const uint32_t pk =
                    pack_bf16(ik * (dkn[t][2 * hh] - kr.x * ik * sk), ik * (dkn[t][2 * hh + 1] - kr.y * ik * sk));
                if (full) {
                    *reinterpret_cast<uint32_t *>(sm + Sm::ST + at(row, col, C)) = pq;
                    *reinterpret_cast<uint32_t *>(sm + Sm::ST + 16384 + at(row, col, C)) = pk;
                } else {
                    const int64_t o = ((tok0 + row) * H + h) * D + col;
                    *reinterpret_cast<uint32_t *>(a.dq + o) = pq;
                    *reinterpret_cast<uint32_t *>(a.dk + o) = pk;
                }
            }
        }
    if (full) tc::fence_proxy_async();   // the staged tiles are read by the TMA engine
    __syncthreads();   // dG in place
    if (full && tid == 0) {
        tc::tma_store_2d(&om.dq, h * D, (int)tok0, sbase + Sm::ST);
        tc::tma_store_2d(&om.dq, h * D + 64, (int)tok0, sbase + Sm::ST + 8192);
        tc::tma_store_2d(&om.dk, h * D, (int)tok0, sbase + Sm::ST + 16384);
        tc::tma_store_2d(&om.dk, h * D + 64, (int)tok0, sbase + Sm::ST + 24576);
        tc::bulk_commit();
    }
    // ---- dg = reverse cumsum of dG over the chunk + dG_last (which reaches every row); dbeta ----
    {
        const int c = tid & (D - 1), qd = tid >> 7;
        float x[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) x[i] = gf[gfi(16 * qd + i, c)];
#pragma unroll
        for (int i = 14; i >= 0; --i) x[i] += x[i + 1];
        tot[qd * D + c] = x[0];
        __syncthreads();
        float off = 0.f;
#pragma unroll
        for (int i = 0; i < 6; ++i) off += dglp[i * D + c];
        for (int q2 = qd + 1; q2 < 4; ++q2) off += tot[q2 * D + c];
        // a whole chunk stages dg row-major in G's space (every read of G is done: barrier above) for
        // one TMA store; a partial chunk stores its valid rows directly
#pragma unroll
        for (int i = 0; i < 16; ++i) {
            const int r = 16 * qd + i;
            if (full) gf[r * D + c] = x[i] + off;
            else if (r < L) a.dg[((tok0 + r) * H + h) * D + c] = x[i] + off;
        }
        if (tid < L) {
            float x = 0.f;
#pragma unroll
            for (int i = 0; i < 12; ++i) x += dbp[i * C + tid];
            a.dbeta[(tok0 + tid) * H + h] = x;
        }
    }
    if (full) {
        tc::fence_proxy_async();   // the staged dg tile is read by the TMA engine
        __syncthreads();
        if (tid == 0) {
            tc::tma_store_2d(&om.dg, h * D, (int)tok0, sbase + Sm::GF);
            tc::bulk_commit();
            tc::bulk_wait_read();   // the TMA stores have read their tiles before shared memory goes away
        }
    }
}
}  // namespace grad


}  // namespace bwd

// workspace bytes of the backward: per chunk slot and head, the forward checkpoint block and the
// dstate outputs
size_t bwd_workspace_floats(int n_docs, int64_t T, int H) {
    return ((size_t)(T / bwd::C) + (size_t)n_docs) * (size_t)H * (bwd::Ws::PER_SLOT / sizeof(float));
}

cudaError_t launch_bwd(const uint16_t *q, const uint16_t *k, const uint16_t *v, const float *g, const float *beta,
                       const int32_t *cu, int n_docs, int64_t T, int H, const uint16_t *dout, uint16_t *dq,
                       uint16_t *dk, uint16_t *dv, float *dg, float *dbeta, float *workspace, int *status,
                       cudaStream_t stream) {
    using namespace bwd;
    const size_t blocks = ((size_t)(T / C) + (size_t)n_docs) * (size_t)H;
    uint8_t *ws = reinterpret_cast<uint8_t *>(workspace);
    uint8_t *ws_ck = ws, *ws_dst = ws + blocks * Ws::CK;
    // 1. forward with checkpoints (this instance forms no output; dq only gives its unused output map a base)
    cudaError_t e = launch_fwd_pipe(q, k, v, g, beta, cu, n_docs, T, H, nullptr, nullptr, dq, status, stream,
                                    reinterpret_cast<uint16_t *>(ws_ck));
    if (e != cudaSuccess) return e;
    // 2. dstate
    e = cudaFuncSetAttribute(dstate::kda_bwd_dstate_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             dstate::Sm::TOTAL);
    if (e != cudaSuccess) return e;
    dstate::kda_bwd_dstate_kernel<<<(unsigned)(n_docs * H), dstate::kThreads, dstate::Sm::TOTAL, stream>>>(
        dout, cu, n_docs, T, H, ws_ck, ws_dst, status);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    // 3. grad
    grad::Args a;
    a.q = q; a.k = k; a.v = v; a.dout = dout; a.g = g; a.beta = beta; a.cu = cu;
    a.n_docs = n_docs; a.T = T; a.H = H;
    a.ws_ck = ws_ck; a.ws_dst = ws_dst;
    a.dq = dq; a.dk = dk; a.dv = dv; a.dg = dg; a.dbeta = dbeta;
    grad::OutMaps om;
    const uint64_t cols = (uint64_t)H * D;
    if (!pipe_path::make_map(&om.dq, dq, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, (uint64_t)T, cols, 64, 64,
                             CU_TENSOR_MAP_SWIZZLE_128B) ||
        !pipe_path::make_map(&om.dk, dk, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, (uint64_t)T, cols, 64, 64,
                             CU_TENSOR_MAP_SWIZZLE_128B) ||
        !pipe_path::make_map(&om.dv, dv, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, (uint64_t)T, cols, 64, 64,
                             CU_TENSOR_MAP_SWIZZLE_128B) ||
        !pipe_path::make_map(&om.dg, dg, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, (uint64_t)T, cols, 64, 128,
                             CU_TENSOR_MAP_SWIZZLE_NONE))
        return cudaErrorInvalidValue;
    e = cudaFuncSetAttribute(grad::kda_bwd_grad_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, grad::Sm::TOTAL);
    if (e != cudaSuccess) return e;
    grad::kda_bwd_grad_kernel<<<(unsigned)blocks, grad::kThreads, grad::Sm::TOTAL, stream>>>(a, om);
    return cudaGetLastError();
}

}  // namespace kda
