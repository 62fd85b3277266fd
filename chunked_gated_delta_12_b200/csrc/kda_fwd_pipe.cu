// kda_fwd_pipe.cu -- pipelined fused chunk-KDA forward (one CTA per (document, head),
// all 128 value columns), for launches with enough chains to cover the SMs.
//
// Two chunks are in flight per CTA.  In step s all 16 warps first prepare chunk
// s; then warps 0-11 finish chunk s's intra-chunk work while warps 12-15 run
// chunk s-1's state update on the tensor cores.  The state is kept transposed,
// S^T[v][c] in fp32 in tensor memory (lane = value column v), so that both the
// bf16 copy of the state and the corrected values U~ are tcgen05 A operands
// read straight from TMEM -- no shared-memory round trip on the state chain.
//
// Per chunk (rows r, i; Gamma = in-chunk cumsum of g; scale-free notation):
//   A_kk[r,i] = beta_r k^_r.(k^_i e^{Gamma_r - Gamma_i}) (i < r),  A_qk (i <= r)
//   T' = (I + A_kk)^-1 diag(beta)
//   W  = T' K^e^Gamma,  U = T' V,  Q' = Q^e^Gamma - A_qk W,  U' = A_qk U
//   U~ = U - W S,  O = Q'S + U'  (= Q^e^Gamma S + A_qk U~)
//   S <- Diag(e^{Gamma_last}) S + (K^ e^{Gamma_last - Gamma})^T U~
// and on the tensor cores (M = 128 everywhere):
//   intra  D_WQ = [0 | Q~^T] - (K^e^Gamma)^T [T'; A_qk T']^T      -> [-W^T | Q'^T]   (B2, shared)
//          D    = V^T [T'; A_qk T']^T                              -> [U^T | U'^T]
//   state  D   += S^T_bf16 (TMEM) B2                               -> [U~^T | O^T]
//          S^T += U~^T_bf16 (TMEM) Kd                               (after S^T <- S^T Diag(e^{Gamma_last}))
// The gate exponent is split at 16-row sub-block boundaries exactly as in the
// non-pipelined kernel (kda_fwd_tc.cu).  Every tensor-core wait is
// time-limited and reports KDA_ERR_TIMEOUT.
#include <cuda_runtime.h>
#include <stdint.h>

#include "kda_common.cuh"
#include "kda_internal.h"
#include "kda_tc.cuh"

namespace kda {
namespace pipe_path {

constexpr int kThreads = 512;
constexpr int kIntraThreads = 384;            // warps 0-11
constexpr int kStateTid0 = 384;               // first thread of warps 12-15
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kSF = 0;                   // S^T fp32          [128 lanes v][128 cols c]
constexpr uint32_t kSB = 128;                 // S^T bf16 packed   [128][64]
constexpr uint32_t kD0 = 192;                 // chunk accumulators, two buffers of 128 columns
constexpr uint32_t kUB = 448;                 // U~^T bf16 packed  [128][32]
constexpr long long kWaitLimit = 2000000000LL;

// A_kk / T as ten 16x16 fp32 blocks (I <= R), rows padded to 20 floats
constexpr int kBlkPitch = 20;
constexpr int kBlkFloats = 16 * kBlkPitch;

struct Smem {
    static constexpr int Q = 0;            // raw q [64][128] bf16 (pitch 256) -> q^E1 [c][r] SW128
    static constexpr int K = 16384;        // raw k                             -> k^E1 [c][r] SW128
    static constexpr int G = 32768;        // raw g [64][128] fp32 (pitch 512)
    static constexpr int V = 65536;        // raw v, MN-major SW128 (64 K-rows, two 64-wide atoms)
    static constexpr int KR = 81920;       // k^E2 [c][r] SW128 -> A1 = [T'; A_qk T'] (K-major, 128 rows)
    static constexpr int KGT = 98304;      // (k^ e^Gamma)^T, K-major [c][r]
    static constexpr int KDT = 114688;     // two buffers: (k^ e^{Gamma_last-Gamma})^T, K-major [c][r]
    static constexpr int B2 = 147456;      // [-W^T | Q'^T], MN-major [c][n], two 64-wide atoms
    static constexpr int AQK = 180224;     // A_qk [r][i], K-major (64 rows)
    static constexpr int AKK = 188416;     // A_kk blocks fp32
    static constexpr int TM = AKK + 10 * kBlkFloats * 4;   // T blocks fp32
    static constexpr int SMALL = TM + 10 * kBlkFloats * 4;
    static constexpr int BETA = SMALL;               // fp32 [2][64]
    static constexpr int RQ = BETA + 512;            // fp32 [64]
    static constexpr int RK = RQ + 256;              // fp32 [64]
    static constexpr int TOT = RK + 256;             // fp32 [4][128]
    static constexpr int PS = TOT + 2048;            // fp32 [10][128]
    static constexpr int DC = PS + 5120;             // fp32 [2][128]
    static constexpr int XT = DC + 1024;             // fp32 [6][16][8]
    static constexpr int MBAR = XT + 3072;           // u64 [4]
    static constexpr int TBASE = MBAR + 32;
    static constexpr int ABORT = TBASE + 16;
    static constexpr int BYTES = ABORT + 16;
    static constexpr int ALLOC = BYTES + 1024;
};
static_assert(Smem::ALLOC <= 232448, "shared memory budget");

__device__ __forceinline__ void bar_intra() { asm volatile("bar.sync 1, 384;" ::: "memory"); }
__device__ __forceinline__ void bar_state() { asm volatile("bar.sync 2, 128;" ::: "memory"); }

__device__ __forceinline__ uint32_t tf32(float x) {
    uint32_t r;
    asm("cvt.rna.tf32.f32 %0, %1;" : "=r"(r) : "f"(x));
    return r;
}
__device__ __forceinline__ void mma_tf32(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                         uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k8.row.col.f32.tf32.tf32.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%0,%1,%2,%3};\n"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}
// tcgen05.mma with A in TMEM
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
__device__ __forceinline__ void st16f(uint32_t taddr, const float (&v)[16]) {
    uint32_t r[16];
#pragma unroll
    for (int i = 0; i < 16; ++i) r[i] = __float_as_uint(v[i]);
    st16(taddr, r);
}
__device__ __forceinline__ uint4 pack8(const float *x, float s) {
    return make_uint4(pack_bf16(x[0] * s, x[1] * s), pack_bf16(x[2] * s, x[3] * s), pack_bf16(x[4] * s, x[5] * s),
                      pack_bf16(x[6] * s, x[7] * s));
}
__device__ __forceinline__ int pair_R(int p) { return p >= 6 ? 3 : p >= 3 ? 2 : p >= 1 ? 1 : 0; }
__device__ __forceinline__ int pair_of(int R, int I) { return R * (R + 1) / 2 + I; }

__device__ __forceinline__ void load_qk(uint8_t *sm, const uint16_t *q, const uint16_t *k, int64_t tok0, int L,
                                        int H, int h, int t0, int nthr) {
    for (int idx = t0; idx < 64 * 16; idx += nthr) {
        const int row = idx >> 4, ch = idx & 15;
        const bool ok = row < L;
        const int64_t off = ok ? ((tok0 + row) * H + h) * kHeadDim + ch * 8 : 0;
        cp_async16(smem_u32(sm + Smem::Q + row * 256 + ch * 16), q + off, ok ? 16 : 0);
        cp_async16(smem_u32(sm + Smem::K + row * 256 + ch * 16), k + off, ok ? 16 : 0);
    }
}
__device__ __forceinline__ void load_gb(uint8_t *sm, const float *g, const float *beta, int64_t tok0, int L, int H,
                                        int h, int buf) {
    for (int idx = threadIdx.x; idx < 64 * 32; idx += kThreads) {
        const int row = idx >> 5, ch = idx & 31;
        const bool ok = row < L;
        const int64_t off = ok ? ((tok0 + row) * H + h) * kHeadDim + ch * 4 : 0;
        cp_async16(smem_u32(sm + Smem::G + row * 512 + ch * 16), g + off, ok ? 16 : 0);
    }
    if (threadIdx.x < 64) {
        const int row = threadIdx.x;
        const bool ok = row < L;
        const float *src = ok ? beta + (tok0 + row) * H + h : beta;
        asm volatile("cp.async.ca.shared.global [%0], [%1], 4, %2;\n" ::"r"(
                         smem_u32(sm + Smem::BETA + buf * 256 + row * 4)),
                     "l"(src), "r"(ok ? 4 : 0)
                     : "memory");
    }
}
__device__ __forceinline__ void load_v(uint8_t *sm, const uint16_t *v, int64_t tok0, int L, int H, int h, int t0,
                                       int nthr) {
    for (int idx = t0; idx < 64 * 16; idx += nthr) {
        const int row = idx >> 4, ch = idx & 15;
        const bool ok = row < L;
        const int64_t off = ok ? ((tok0 + row) * H + h) * kHeadDim + ch * 8 : 0;
        cp_async16(smem_u32(sm + Smem::V) + tc::mnmaj_chunk(ch, row, 64), v + off, ok ? 16 : 0);
    }
}

__global__ void __launch_bounds__(kThreads, 1)
    kda_fwd_pipe_kernel(const uint16_t *__restrict__ q, const uint16_t *__restrict__ k,
                        const uint16_t *__restrict__ v, const float *__restrict__ g,
                        const float *__restrict__ beta, const int32_t *__restrict__ cu_seqlens, int n_docs,
                        int64_t T, int H, uint16_t *__restrict__ out, int *__restrict__ status) {
    using S = Smem;
    extern __shared__ __align__(1024) uint8_t sm_raw[];
    uint8_t *sm = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(sm_raw) + 1023) & ~uintptr_t(1023));

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int gq = lane >> 2, tq = lane & 3;
    const int doc = blockIdx.x / H, h = blockIdx.x % H;

    if (blockIdx.x == 0 && tid == 0) {
        if (cu_seqlens[0] != 0 || (int64_t)cu_seqlens[n_docs] != T) atomicExch(status, kStatusBadSeqlens);
    }
    const int64_t doc_start = cu_seqlens[doc], doc_end = cu_seqlens[doc + 1];
    if (doc_start < 0 || doc_end < doc_start || doc_end > T) {
        if (tid == 0) atomicExch(status, kStatusBadSeqlens);
        return;
    }
    if (doc_end == doc_start) return;
    const int nchunks = (int)((doc_end - doc_start + 63) / 64);

    float *f_rq = reinterpret_cast<float *>(sm + S::RQ);
    float *f_rk = reinterpret_cast<float *>(sm + S::RK);
    float *f_tot = reinterpret_cast<float *>(sm + S::TOT);
    float *f_ps = reinterpret_cast<float *>(sm + S::PS);
    float *f_akk = reinterpret_cast<float *>(sm + S::AKK);
    float *f_tm = reinterpret_cast<float *>(sm + S::TM);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(sm + S::ABORT);
    const uint32_t mbar_wq = smem_u32(sm + S::MBAR), mbar_u = mbar_wq + 8, mbar_2 = mbar_wq + 16,
                   mbar_4 = mbar_wq + 24;
    const uint32_t sbase = smem_u32(sm);

    // ---- setup ----
    if (warp == 0) tc::alloc(smem_u32(sm + S::TBASE), kTmemCols);
    if (tid == 0) {
        tc::mbar_init(mbar_wq, 1);
        tc::mbar_init(mbar_u, 1);
        tc::mbar_init(mbar_2, 1);
        tc::mbar_init(mbar_4, 1);
        *abort_flag = 0;
    }
    {
        const int L0 = (int)(doc_end - doc_start < 64 ? doc_end - doc_start : 64);
        load_qk(sm, q, k, doc_start, L0, H, h, tid, kThreads);
        load_gb(sm, g, beta, doc_start, L0, H, h, 0);
        cp_async_commit();
    }
    tc::fence_before();
    __syncthreads();
    tc::fence_after();
    const uint32_t tmem = *reinterpret_cast<volatile uint32_t *>(sm + S::TBASE);
    const int lq = warp & 3;
    const uint32_t lane_base = tmem + ((uint32_t)(32 * lq) << 16);
    if (warp >= 12) {   // S^T = 0
        float z[32];
#pragma unroll
        for (int i = 0; i < 32; ++i) z[i] = 0.f;
#pragma unroll
        for (int c0 = 0; c0 < 128; c0 += 32) tc::st32(lane_base + kSF + c0, z);
        tc::wait_st();
    }
    tc::fence_before();
    __syncthreads();
    tc::fence_after();

    bool aborted = false;
    const float out_scale = rsqrtf((float)kHeadDim);

    for (int s = 0; s <= nchunks; ++s) {
        const bool have_intra = s < nchunks;        // chunk s: prep + intra
        const bool have_state = s >= 1;             // chunk s-1: state update + output
        const int64_t tok0 = doc_start + 64 * (int64_t)s;
        const int L = have_intra ? (int)(doc_end - tok0 < 64 ? doc_end - tok0 : 64) : 0;
        const int64_t ntok0 = tok0 + 64;
        const int nL = (int)(doc_end - ntok0 < 64 ? doc_end - ntok0 : 64);    // <= 0: no chunk s+1
        const int buf = s & 1;

        // ---- top: raw(s) landed; the previous step's U product is done (V, KR free) ----
        cp_async_wait_all();
        if (have_state) {
            if (!tc::mbar_wait(mbar_u, (uint32_t)((s - 1) & 1), kWaitLimit)) *abort_flag = 1;
        }
        tc::fence_before();
        __syncthreads();
        tc::fence_after();
        if (*abort_flag) { aborted = true; break; }
        // v(s) for this step's U product (intra warps; waited on before that product)
        if (tid < kIntraThreads) {
            if (have_intra) load_v(sm, v, tok0, L, H, h, tid, kIntraThreads);
            cp_async_commit();
        }

        float ql[16], kl[16], kr[16];
        float lg0 = 0.f;
        const int pc = tid & 127, pR = tid >> 7;
        if (have_intra) {
            // ---- norms: warp w handles rows 4w..4w+3 ----
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const int r = warp * 4 + i;
                const uint2 qa = *reinterpret_cast<const uint2 *>(sm + S::Q + r * 256 + lane * 8);
                const uint2 ka = *reinterpret_cast<const uint2 *>(sm + S::K + r * 256 + lane * 8);
                const float2 q01 = unpack_bf16(qa.x), q23 = unpack_bf16(qa.y);
                const float2 k01 = unpack_bf16(ka.x), k23 = unpack_bf16(ka.y);
                float sq = q01.x * q01.x + q01.y * q01.y + q23.x * q23.x + q23.y * q23.y;
                float sk = k01.x * k01.x + k01.y * k01.y + k23.x * k23.x + k23.y * k23.y;
#pragma unroll
                for (int o = 16; o > 0; o >>= 1) {
                    sq += __shfl_xor_sync(0xffffffffu, sq, o);
                    sk += __shfl_xor_sync(0xffffffffu, sk, o);
                }
                if (lane == 0) {
                    f_rq[r] = rsqrtf(sq + 1e-6f);
                    f_rk[r] = rsqrtf(sk + 1e-6f);
                }
            }
        }
        __syncthreads();
        float lg15 = 0.f;
        if (have_intra) {
            // ---- prep pass 1: thread = (channel c, row block R) ----
            float lg[16];
            float acc = 0.f;
#pragma unroll
            for (int j = 0; j < 16; ++j) {
                acc += *reinterpret_cast<const float *>(sm + S::G + (16 * pR + j) * 512 + pc * 4);
                lg[j] = acc;
            }
            lg0 = lg[0];
            lg15 = lg[15];
            f_tot[pR * 128 + pc] = lg15;
#pragma unroll
            for (int j = 0; j < 16; ++j) {
                const int r = 16 * pR + j;
                const float qv = __bfloat162float(*reinterpret_cast<const __nv_bfloat16 *>(sm + S::Q + r * 256 + pc * 2));
                const float kv = __bfloat162float(*reinterpret_cast<const __nv_bfloat16 *>(sm + S::K + r * 256 + pc * 2));
                const float qh = qv * f_rq[r], kh = kv * f_rk[r];
                const float e1 = fast_exp2((lg[j] - lg0) * kLog2e);
                const float e2 = fast_exp2((lg15 - lg[j]) * kLog2e);
                ql[j] = qh * e1;
                kl[j] = kh * e1;
                kr[j] = kh * e2;
            }
        }
        __syncthreads();   // raw q, k, g read; block sums published
        // raw g is dead: the next chunk's g and beta
        if (nL > 0) load_gb(sm, g, beta, ntok0, nL, H, h, buf ^ 1);
        cp_async_commit();
        if (have_intra) {
            // ---- prep pass 2 ----
            float offs[5];
            offs[0] = 0.f;
#pragma unroll
            for (int R = 0; R < 4; ++R) offs[R + 1] = offs[R] + f_tot[R * 128 + pc];
            const float gm = offs[pR] + lg0;
            const float ge = offs[pR + 1];
            const float gl = offs[4];
            const float P = fast_exp2(gm * kLog2e);
            const float Dk = fast_exp2((gl - ge) * kLog2e);
#pragma unroll
            for (int I = 0; I < 4; ++I)
                if (I <= pR) f_ps[pair_of(pR, I) * 128 + pc] = fast_exp2((gm - offs[I + 1]) * kLog2e);
            if (pR == 0) reinterpret_cast<float *>(sm + S::DC)[buf * 128 + pc] = fast_exp2(gl * kLog2e);
#pragma unroll
            for (int half = 0; half < 2; ++half) {
                const int j0 = half * 8;
                const uint32_t off = tc::kmaj_chunk(pc, 2 * pR + half);
                *reinterpret_cast<uint4 *>(sm + S::Q + off) = pack8(ql + j0, 1.f);
                *reinterpret_cast<uint4 *>(sm + S::K + off) = pack8(kl + j0, 1.f);
                *reinterpret_cast<uint4 *>(sm + S::KR + off) = pack8(kr + j0, 1.f);
                *reinterpret_cast<uint4 *>(sm + S::KGT + off) = pack8(kl + j0, P);
                *reinterpret_cast<uint4 *>(sm + S::KDT + buf * 16384 + off) = pack8(kr + j0, Dk);
            }
            // D_WQ init in TMEM (lane c): columns 16R.. = 0, columns 64+16R.. = Q~ rows 16R..16R+15
            {
                float qt[16], z[16];
#pragma unroll
                for (int j = 0; j < 16; ++j) {
                    qt[j] = ql[j] * P;
                    z[j] = 0.f;
                }
                const uint32_t dcol = kD0 + 128 * (uint32_t)buf;
                st16f(lane_base + dcol + 16 * pR, z);
                st16f(lane_base + dcol + 64 + 16 * pR, qt);
                tc::wait_st();
            }
        }
        tc::fence_before();
        __syncthreads();
        tc::fence_after();

        if (warp < 12) {
            // ================= intra (chunk s) =================
            if (have_intra) {
                const float *f_beta = reinterpret_cast<const float *>(sm + S::BETA + buf * 256);
                // ---- A_kk and A_qk, one 16x16 block pair per warp ----
                if (warp < 10) {
                    const int p = warp;
                    const int R = pair_R(p), I = p - R * (R + 1) / 2;
                    const uint32_t kbase = sbase + S::K, qbase = sbase + S::Q, rbase = sbase + S::KR;
                    const float *ps = f_ps + p * 128;
                    float ak[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
                    float aq[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
                    const int j = lane >> 3;
#pragma unroll
                    for (int kk = 0; kk < 8; ++kk) {
                        const uint32_t aoff = tc::kmaj_chunk(16 * kk + (lane & 7) + 8 * (j >> 1), 2 * R + (j & 1));
                        uint32_t fk[4], fq[4], b0, b1, b2, b3;
                        ldsm_x4_t(kbase + aoff, fk[0], fk[1], fk[2], fk[3]);
                        ldsm_x4_t(qbase + aoff, fq[0], fq[1], fq[2], fq[3]);
                        ldsm_x4_t(rbase + tc::kmaj_chunk(16 * kk + (lane & 7) + 8 * (j & 1), 2 * I + (j >> 1)), b0, b1,
                                  b2, b3);
                        const int cb = kk * 16 + 2 * tq;
                        const float2 s0 = *reinterpret_cast<const float2 *>(ps + cb);
                        const float2 s8 = *reinterpret_cast<const float2 *>(ps + cb + 8);
                        const __nv_bfloat162 h0 = __floats2bfloat162_rn(s0.x, s0.y);
                        const __nv_bfloat162 h8 = __floats2bfloat162_rn(s8.x, s8.y);
#pragma unroll
                        for (int e = 0; e < 4; ++e) {
                            const __nv_bfloat162 sc = e < 2 ? h0 : h8;
                            __nv_bfloat162 x = __hmul2(*reinterpret_cast<__nv_bfloat162 *>(&fk[e]), sc);
                            fk[e] = *reinterpret_cast<uint32_t *>(&x);
                            x = __hmul2(*reinterpret_cast<__nv_bfloat162 *>(&fq[e]), sc);
                            fq[e] = *reinterpret_cast<uint32_t *>(&x);
                        }
                        mma_bf16(ak[0], fk, b0, b1);
                        mma_bf16(ak[1], fk, b2, b3);
                        mma_bf16(aq[0], fq, b0, b1);
                        mma_bf16(aq[1], fq, b2, b3);
                    }
                    float *blk = f_akk + p * kBlkFloats;
#pragma unroll
                    for (int nt = 0; nt < 2; ++nt)
#pragma unroll
                        for (int hh = 0; hh < 2; ++hh) {
                            const int i = gq + 8 * hh, jj = 8 * nt + 2 * tq;
                            const int row = 16 * R + i, col = 16 * I + jj;
                            const float br = f_beta[row];
                            const float x0 = col < row ? ak[nt][2 * hh] * br : 0.f;
                            const float x1 = col + 1 < row ? ak[nt][2 * hh + 1] * br : 0.f;
                            *reinterpret_cast<float2 *>(blk + i * kBlkPitch + jj) = make_float2(x0, x1);
                            const float y0 = col <= row ? aq[nt][2 * hh] : 0.f;
                            const float y1 = col + 1 <= row ? aq[nt][2 * hh + 1] : 0.f;
                            *reinterpret_cast<uint32_t *>(sm + S::AQK + tc::kmaj_off(row, col)) = pack_bf16(y0, y1);
                        }
                } else {
                    // warps 10, 11: A_qk is zero above the block diagonal
                    const int t = tid - 320;
                    for (int idx = t; idx < 192; idx += 64) {
                        const int b = idx >> 5, row = (idx & 31) >> 1, half = idx & 1;
                        const int R = b < 3 ? 0 : b < 5 ? 1 : 2;
                        const int I = b < 3 ? b + 1 : b < 5 ? b - 1 : 3;
                        *reinterpret_cast<uint4 *>(sm + S::AQK + tc::kmaj_chunk(16 * R + row, 2 * I + half)) =
                            make_uint4(0, 0, 0, 0);
                    }
                }
            }
            bar_intra();
            // q^E1 / k^E1 consumed: the next chunk's raw q, k
            if (nL > 0) load_qk(sm, q, k, ntok0, nL, H, h, tid, kIntraThreads);
            cp_async_commit();
            if (have_intra) {
                const float *f_beta = reinterpret_cast<const float *>(sm + S::BETA + buf * 256);
                // ---- T = (I + A_kk)^-1: diagonal blocks, one column per lane ----
                if (warp < 4 && lane < 16) {
                    const int R = warp, col = lane;
                    const float *blk = f_akk + pair_of(R, R) * kBlkFloats;
                    float x[16];
#pragma unroll
                    for (int r = 0; r < 16; ++r) {
                        float a[16];
#pragma unroll
                        for (int q4 = 0; q4 < 4; ++q4) {
                            const float4 t4 = *reinterpret_cast<const float4 *>(blk + r * kBlkPitch + 4 * q4);
                            a[4 * q4] = t4.x; a[4 * q4 + 1] = t4.y; a[4 * q4 + 2] = t4.z; a[4 * q4 + 3] = t4.w;
                        }
                        float acc = (r == col) ? 1.f : 0.f;
#pragma unroll
                        for (int jj = 0; jj < r; ++jj) acc -= a[jj] * x[jj];
                        x[r] = acc;
                    }
                    float *tb = f_tm + pair_of(R, R) * kBlkFloats;
#pragma unroll
                    for (int r = 0; r < 16; ++r) tb[r * kBlkPitch + col] = x[r];
                }
                bar_intra();
                // ---- off-diagonal blocks by distance d ----
#pragma unroll 1
                for (int d = 1; d < 4; ++d) {
                    const int njobs = 2 * (4 - d);
                    if (warp < njobs) {
                        const int R = d + (warp >> 1), I = R - d, nt = warp & 1;
                        float xacc[4] = {0.f, 0.f, 0.f, 0.f};
                        for (int J = I; J < R; ++J) {
                            const float *ab = f_akk + pair_of(R, J) * kBlkFloats;
                            const float *tb = f_tm + pair_of(J, I) * kBlkFloats;
#pragma unroll
                            for (int kb = 0; kb < 16; kb += 8) {
                                const uint32_t a0 = tf32(ab[gq * kBlkPitch + kb + tq]);
                                const uint32_t a1 = tf32(ab[(gq + 8) * kBlkPitch + kb + tq]);
                                const uint32_t a2 = tf32(ab[gq * kBlkPitch + kb + tq + 4]);
                                const uint32_t a3 = tf32(ab[(gq + 8) * kBlkPitch + kb + tq + 4]);
                                const uint32_t b0 = tf32(tb[(kb + tq) * kBlkPitch + 8 * nt + gq]);
                                const uint32_t b1 = tf32(tb[(kb + tq + 4) * kBlkPitch + 8 * nt + gq]);
                                mma_tf32(xacc, a0, a1, a2, a3, b0, b1);
                            }
                        }
                        float *xt = reinterpret_cast<float *>(sm + S::XT) + warp * 128;   // X[16][8]
                        xt[gq * 8 + 2 * tq] = xacc[0];
                        xt[gq * 8 + 2 * tq + 1] = xacc[1];
                        xt[(gq + 8) * 8 + 2 * tq] = xacc[2];
                        xt[(gq + 8) * 8 + 2 * tq + 1] = xacc[3];
                        __syncwarp();
                        const float *tr = f_tm + pair_of(R, R) * kBlkFloats;
                        float tacc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
                        for (int kb = 0; kb < 16; kb += 8) {
                            const uint32_t a0 = tf32(tr[gq * kBlkPitch + kb + tq]);
                            const uint32_t a1 = tf32(tr[(gq + 8) * kBlkPitch + kb + tq]);
                            const uint32_t a2 = tf32(tr[gq * kBlkPitch + kb + tq + 4]);
                            const uint32_t a3 = tf32(tr[(gq + 8) * kBlkPitch + kb + tq + 4]);
                            const uint32_t b0 = tf32(xt[(kb + tq) * 8 + gq]);
                            const uint32_t b1 = tf32(xt[(kb + tq + 4) * 8 + gq]);
                            mma_tf32(tacc, a0, a1, a2, a3, b0, b1);
                        }
                        float *to = f_tm + pair_of(R, I) * kBlkFloats;
                        *reinterpret_cast<float2 *>(to + gq * kBlkPitch + 8 * nt + 2 * tq) = make_float2(-tacc[0], -tacc[1]);
                        *reinterpret_cast<float2 *>(to + (gq + 8) * kBlkPitch + 8 * nt + 2 * tq) =
                            make_float2(-tacc[2], -tacc[3]);
                    }
                    bar_intra();
                }
                // ---- T' = T diag(beta) -> bf16 rows 0-63 of A1 ----
                for (int idx = tid; idx < 512; idx += kIntraThreads) {
                    const int r = idx >> 3, ch = idx & 7;
                    const int R = r >> 4, i = r & 15, I = ch >> 1;
                    uint32_t w4[4];
                    if (I <= R) {
                        const float *tb = f_tm + pair_of(R, I) * kBlkFloats + i * kBlkPitch + (ch & 1) * 8;
#pragma unroll
                        for (int e = 0; e < 4; ++e) {
                            const int c0 = ch * 8 + 2 * e;
                            const float x0 = c0 <= r ? tb[2 * e] * f_beta[c0] : 0.f;
                            const float x1 = c0 + 1 <= r ? tb[2 * e + 1] * f_beta[c0 + 1] : 0.f;
                            w4[e] = pack_bf16(x0, x1);
                        }
                    } else {
                        w4[0] = w4[1] = w4[2] = w4[3] = 0u;
                    }
                    *reinterpret_cast<uint4 *>(sm + S::KR + tc::kmaj_chunk(r, ch)) = make_uint4(w4[0], w4[1], w4[2], w4[3]);
                }
                bar_intra();
                // ---- A_qk T' -> bf16 rows 64-127 of A1 (warp-level MMA, warps 0-7) ----
                if (warp < 8) {
                    const int R = warp >> 1, nh = warp & 1;
                    const uint32_t abase = sbase + S::AQK, tbase2 = sbase + S::KR;
                    float acc[4][4];
#pragma unroll
                    for (int a = 0; a < 4; ++a) acc[a][0] = acc[a][1] = acc[a][2] = acc[a][3] = 0.f;
                    const int j = lane >> 3;
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk) {
                        uint32_t fa[4];
                        ldsm_x4(abase + tc::kmaj_chunk(16 * R + (lane & 7) + 8 * (j & 1), 2 * kk + (j >> 1)), fa[0], fa[1],
                                fa[2], fa[3]);
#pragma unroll
                        for (int np = 0; np < 2; ++np) {
                            uint32_t b0, b1, b2, b3;
                            ldsm_x4_t(tbase2 + tc::kmaj_chunk(16 * kk + (lane & 7) + 8 * (j & 1), 4 * nh + 2 * np + (j >> 1)),
                                      b0, b1, b2, b3);
                            mma_bf16(acc[2 * np], fa, b0, b1);
                            mma_bf16(acc[2 * np + 1], fa, b2, b3);
                        }
                    }
#pragma unroll
                    for (int nt = 0; nt < 4; ++nt)
#pragma unroll
                        for (int hh = 0; hh < 2; ++hh) {
                            const int row = 64 + 16 * R + gq + 8 * hh;
                            const int col = 32 * nh + 8 * nt + 2 * tq;
                            *reinterpret_cast<uint32_t *>(sm + S::KR + tc::kmaj_off(row, col)) =
                                pack_bf16(acc[nt][2 * hh], acc[nt][2 * hh + 1]);
                        }
                }
                tc::fence_proxy_async();
                tc::fence_before();
                bar_intra();
                // ---- tcgen05: D_WQ = [0 | Q~^T] - KG^T A1^T ----
                const uint32_t dcol = kD0 + 128 * (uint32_t)buf;
                if (tid == 0) {
                    tc::fence_after();
                    constexpr uint32_t id_wq = tc::idesc_bf16(128, 128, false, false, true);
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk)
                        tc::mma(tmem + dcol, tc::desc_kmaj(sbase + S::KGT, kk), tc::desc_kmaj(sbase + S::KR, kk), id_wq,
                                1u);
                    tc::commit(mbar_wq);
                }
                if (!tc::mbar_wait(mbar_wq, (uint32_t)(s & 1), kWaitLimit)) *abort_flag = 1;
                // B2 is free once the previous chunk's state product has read it
                if (have_state) {
                    if (!tc::mbar_wait(mbar_2, (uint32_t)((s - 1) & 1), kWaitLimit)) *abort_flag = 1;
                }
                tc::fence_after();
                if (warp < 8) {
                    const int c = 32 * lq + lane, cg = warp >> 2;
#pragma unroll
                    for (int h2 = 0; h2 < 2; ++h2) {
                        float w[32];
                        tc::ld32(lane_base + dcol + 64 * cg + 32 * h2, w);
                        tc::wait_ld();
#pragma unroll
                        for (int e = 0; e < 4; ++e)
                            *reinterpret_cast<uint4 *>(sm + S::B2 + tc::mnmaj_chunk(8 * cg + 4 * h2 + e, c, 128)) =
                                pack8(w + 8 * e, 1.f);
                    }
                }
                // v(s) landed (the two groups committed after it may still be in flight)
                asm volatile("cp.async.wait_group 2;\n" ::: "memory");
                tc::fence_proxy_async();
                tc::fence_before();
                bar_intra();
                // ---- tcgen05: D = V^T A1^T = [U^T | (A_qk U)^T] ----
                if (tid == 0) {
                    tc::fence_after();
                    constexpr uint32_t id_u = tc::idesc_bf16(128, 128, true, false, false);
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk)
                        tc::mma(tmem + dcol, tc::desc_mnmaj(sbase + S::V, kk, 64), tc::desc_kmaj(sbase + S::KR, kk), id_u,
                                kk > 0);
                    tc::commit(mbar_u);
                }
            } else {
                bar_intra();   // keep the intra barrier count uniform for a step without a chunk
            }
        } else if (have_state) {
            // ================= state (chunk s-1), warps 12-15 =================
            const int n = s - 1, nbuf = n & 1;
            const int64_t ptok0 = tok0 - 64;
            const int pL = (int)(doc_end - ptok0 < 64 ? doc_end - ptok0 : 64);
            const uint32_t dcol = kD0 + 128 * (uint32_t)nbuf;
            const float *dc = reinterpret_cast<const float *>(sm + S::DC) + nbuf * 128;
            // S^T -> bf16 copy (A operand), then S^T <- S^T Diag(e^{Gamma_last})
#pragma unroll 1
            for (int c0 = 0; c0 < 128; c0 += 32) {
                float sv[32];
                tc::ld32(lane_base + kSF + c0, sv);
                tc::wait_ld();
                uint32_t pk[16];
#pragma unroll
                for (int i = 0; i < 16; ++i) pk[i] = pack_bf16(sv[2 * i], sv[2 * i + 1]);
                st16(lane_base + kSB + c0 / 2, pk);
#pragma unroll
                for (int i = 0; i < 32; i += 4) {
                    const float4 d4 = *reinterpret_cast<const float4 *>(dc + c0 + i);
                    sv[i] *= d4.x; sv[i + 1] *= d4.y; sv[i + 2] *= d4.z; sv[i + 3] *= d4.w;
                }
                tc::st32(lane_base + kSF + c0, sv);
            }
            tc::wait_st();
            tc::fence_before();
            bar_state();
            if (tid == kStateTid0) {
                tc::fence_after();
                constexpr uint32_t id2 = tc::idesc_bf16(128, 128, false, true, false);
#pragma unroll
                for (int kk = 0; kk < 8; ++kk)
                    mma_ts(tmem + dcol, tmem + kSB + 8 * kk, tc::desc_mnmaj(sbase + S::B2, kk, 128), id2, 1u);
                tc::commit(mbar_2);
            }
            if (!tc::mbar_wait(mbar_2, (uint32_t)(n & 1), kWaitLimit)) *abort_flag = 1;
            tc::fence_after();
            // U~^T (columns 0-63) -> bf16 copy (A operand of the state update)
            {
                float u[32];
                uint32_t pk[16];
#pragma unroll
                for (int h2 = 0; h2 < 2; ++h2) {
                    tc::ld32(lane_base + dcol + 32 * h2, u);
                    tc::wait_ld();
#pragma unroll
                    for (int i = 0; i < 16; ++i) pk[i] = pack_bf16(u[2 * i], u[2 * i + 1]);
                    st16(lane_base + kUB + 16 * h2, pk);
                }
                tc::wait_st();
            }
            tc::fence_before();
            bar_state();
            if (tid == kStateTid0) {
                tc::fence_after();
                constexpr uint32_t id4 = tc::idesc_bf16(128, 128, false, false, false);
#pragma unroll
                for (int kk = 0; kk < 4; ++kk)
                    mma_ts(tmem + kSF, tmem + kUB + 8 * kk, tc::desc_kmaj(sbase + S::KDT + nbuf * 16384, kk), id4, 1u);
                tc::commit(mbar_4);
            }
            // O^T (columns 64-127): lane v holds o[r][v] for the 64 rows of chunk s-1
            {
                const int vcol = 32 * lq + lane;
#pragma unroll
                for (int h2 = 0; h2 < 2; ++h2) {
                    float o[32];
                    tc::ld32(lane_base + dcol + 64 + 32 * h2, o);
                    tc::wait_ld();
#pragma unroll
                    for (int i = 0; i < 32; ++i) {
                        const int r = 32 * h2 + i;
                        if (r < pL) {
                            const __nv_bfloat16 b = __float2bfloat16_rn(o[i] * out_scale);
                            out[((ptok0 + r) * H + h) * kHeadDim + vcol] = *reinterpret_cast<const uint16_t *>(&b);
                        }
                    }
                }
            }
            if (!tc::mbar_wait(mbar_4, (uint32_t)(n & 1), kWaitLimit)) *abort_flag = 1;
            tc::fence_after();
        }
        tc::fence_before();
        __syncthreads();
        tc::fence_after();
        if (*abort_flag) { aborted = true; break; }
    }

    // ---- teardown ----
    cp_async_wait_all();
    if (aborted) {
        if (tid == 0) atomicExch(status, kStatusTimeout);
        tc::mbar_wait(mbar_wq, 0, kWaitLimit / 8);
        tc::mbar_wait(mbar_wq, 1, kWaitLimit / 8);
    }
    tc::fence_before();
    __syncthreads();
    tc::fence_after();
    if (warp == 0) tc::dealloc(tmem, kTmemCols);
}

}  // namespace pipe_path

cudaError_t launch_fwd_pipe(const uint16_t *q, const uint16_t *k, const uint16_t *v, const float *g,
                            const float *beta, const int32_t *cu, int n_docs, int64_t T, int H, uint16_t *out,
                            int *status, cudaStream_t stream) {
    constexpr int bytes = pipe_path::Smem::ALLOC;
    cudaError_t e = cudaFuncSetAttribute(pipe_path::kda_fwd_pipe_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         bytes);
    if (e != cudaSuccess) return e;
    const int64_t blocks = (int64_t)n_docs * H;
    pipe_path::kda_fwd_pipe_kernel<<<(unsigned)blocks, pipe_path::kThreads, bytes, stream>>>(q, k, v, g, beta, cu,
                                                                                             n_docs, T, H, out, status);
    return cudaGetLastError();
}

}  // namespace kda
