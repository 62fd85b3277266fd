// kda_fwd_tc.cu -- fused chunk-KDA forward on the 5th-generation tensor cores.
//
// One CTA (512 threads) per (document, head, value slice of VS columns) walks
// the document's 64-token chunks.  The fp32 state S[128 x VS] lives in tensor
// memory (TMEM lane = key channel c) for the whole document; the chunk
// contractions run as tcgen05.mma (bf16 operands in 128-byte-swizzled shared
// memory, fp32 accumulators in TMEM).  Per chunk (rows r, i; Gamma = in-chunk
// inclusive cumsum of g per channel):
//
//   norms    1/|q_r|, 1/|k_r| (warp reductions)
//   prep     thread = (channel c, 16-row block R): Gamma, E1 = e^{Gamma_r - Gamma_{16R}},
//            E2 = e^{Gamma_{16R+15} - Gamma_r}; bf16 tiles q^E1, k^E1, k^E2 (for the
//            intra products), -q^e^Gamma, (k^e^Gamma)^T, (k^e^{Gamma_last-Gamma})^T
//   intra    A_kk, A_qk as 16x16 blocks on warp-level bf16 MMA; T = (I + A_kk)^-1:
//            diagonal blocks by forward substitution (fp32), off-diagonal blocks in
//            three rounds of tf32 warp MMA; T' = T diag(beta)
//   tcgen05  W^T = (K^e^Gamma)^T T'^T          (M=128 channels, N=64, K=64)
//            D   = [T'; 0] V                   (M=128, N=VS, K=64)      -> rows 0-63: U
//   state    S <- Diag(e^{Gamma_last}) S in TMEM; bf16 copy of the old S to shared
//            D  += -[W; -Q~] S                 (M=128, N=VS, K=128)     -> [U~; Q~S]
//            D  += [* ; A_qk] U~               (M=128, N=VS, K=64)      -> rows 64-127: O
//            S  += Kd^T U~                     (M=128, N=VS, K=64)
//   output   o = O / sqrt(128) -> bf16, rows inside the document
//
// The exponent split at 16-row sub-block boundaries keeps every exp factor
// inside fp32/bf16 range for a gate bounded below by -5 per token (a chunk's
// cumsum reaches -320): E1, E2 <= 1 and the per-channel pair scales
// s_{R,I} = e^{Gamma_{16R} - Gamma_{16I+15}} are <= 1 off the diagonal and
// <= e^{75} on it.  Rows past the document end are zero-filled at load.
//
// Every wait on the tensor core has a time limit; on expiry the CTA records
// KDA_ERR_TIMEOUT in the status word, stops, frees its TMEM and returns.
#include <cuda_runtime.h>
#include <stdint.h>

#include "kda_common.cuh"
#include "kda_internal.h"
#include "kda_tc.cuh"

namespace kda {
namespace tc_path {

constexpr int kThreads = 512;
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kTmemS = 0, kTmemD = 128, kTmemW = 256;
constexpr long long kWaitLimit = 2000000000LL;   // ~1 s of SM clocks

template <int VS>
struct Smem {
    static constexpr int Q = 0;                       // raw q [64][128] bf16 (pitch 256) -> q^E1 [c][r] SW128
    static constexpr int K = Q + 16384;               // raw k                             -> k^E1 [c][r] SW128
    static constexpr int G = K + 16384;               // raw g [64][128] fp32 (pitch 512)
    static constexpr int AKK = G;                     //   later A_kk fp32 [64][64] (swizzled, pitch 256)
    static constexpr int TM = G + 16384;              //   later T    fp32 [64][64]
    static constexpr int V = G + 32768;               // raw v slice, MN-major SW128, 64 K-rows
    static constexpr int SB = V + 64 * VS * 2;        // bf16 copy of the state, MN-major, 128 K-rows
    static constexpr int KR = SB + 128 * VS * 2;      // k^E2 [c][r] SW128 -> [T'; 0] (K-major) -> U~ (MN-major)
    static constexpr int KGT = KR + 16384;            // (k^ e^Gamma)^T, K-major [c][r]
    static constexpr int KDT = KGT + 16384;           // (k^ e^{Gamma_last - Gamma})^T, K-major [c][r]
    static constexpr int A2 = KDT + 16384;            // [W; -Q~], MN-major, 128 K-rows, two M atoms
    static constexpr int AQK = A2 + 32768;            // A_qk rows (K-major, 64 rows); A3 = AQK - 8192
    static constexpr int SMALL = AQK + 8192;
    static constexpr int BETA = SMALL;                // fp32 [64]
    static constexpr int RQ = BETA + 256;             // fp32 [64]
    static constexpr int RK = RQ + 256;               // fp32 [64]
    static constexpr int TOT = RK + 256;              // fp32 [4][128] block sums of g
    static constexpr int PS = TOT + 2048;             // fp32 [10][128] pair scales
    static constexpr int DC = PS + 5120;              // fp32 [128] e^{Gamma_last}
    static constexpr int XT = DC + 512;               // fp32 [6][16][8] solve temporaries
    static constexpr int MBAR = XT + 3072;            // u64 [4]
    static constexpr int TBASE = MBAR + 32;           // u32 TMEM base
    static constexpr int ABORT = TBASE + 16;          // int
    static constexpr int BYTES = ABORT + 16;
    static constexpr int ALLOC = BYTES + 1024;        // slack for 1024-byte alignment
};

// Warps 0-11 run the intra-chunk work; warps 12-15 (one full warpgroup, all
// 128 TMEM lanes) prepare the state at the same time.  Named barrier 1 syncs
// the intra warps only.
constexpr int kIntraThreads = 384;
__device__ __forceinline__ void bar_intra() { asm volatile("bar.sync 1, 384;" ::: "memory"); }

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

// Async loads of one chunk's rows [tok0, tok0 + L) of head h (rows >= L zero-filled).
template <int VS>
__device__ __forceinline__ void load_qk(uint8_t *sm, const uint16_t *q, const uint16_t *k, int64_t tok0,
                                        int L, int H, int h, int t0, int nthr) {
    using S = Smem<VS>;
    for (int idx = t0; idx < 64 * 16; idx += nthr) {
        const int row = idx >> 4, ch = idx & 15;
        const bool ok = row < L;
        const int64_t off = ok ? ((tok0 + row) * H + h) * kHeadDim + ch * 8 : 0;
        cp_async16(smem_u32(sm + S::Q + row * 256 + ch * 16), q + off, ok ? 16 : 0);
        cp_async16(smem_u32(sm + S::K + row * 256 + ch * 16), k + off, ok ? 16 : 0);
    }
}
template <int VS>
__device__ __forceinline__ void load_gb(uint8_t *sm, const float *g, const float *beta, int64_t tok0, int L,
                                        int H, int h) {
    using S = Smem<VS>;
    for (int idx = threadIdx.x; idx < 64 * 32; idx += kThreads) {
        const int row = idx >> 5, ch = idx & 31;
        const bool ok = row < L;
        const int64_t off = ok ? ((tok0 + row) * H + h) * kHeadDim + ch * 4 : 0;
        cp_async16(smem_u32(sm + S::G + row * 512 + ch * 16), g + off, ok ? 16 : 0);
    }
    if (threadIdx.x < 64) {
        const int row = threadIdx.x;
        const bool ok = row < L;
        const float *src = ok ? beta + (tok0 + row) * H + h : beta;
        asm volatile("cp.async.ca.shared.global [%0], [%1], 4, %2;\n" ::"r"(smem_u32(sm + S::BETA + row * 4)),
                     "l"(src), "r"(ok ? 4 : 0)
                     : "memory");
    }
}
template <int VS>
__device__ __forceinline__ void load_v(uint8_t *sm, const uint16_t *v, int64_t tok0, int L, int H, int h,
                                       int v0) {
    using S = Smem<VS>;
    constexpr int VCH = VS / 8;
    for (int idx = threadIdx.x; idx < 64 * VCH; idx += kThreads) {
        const int row = idx / VCH, ch = idx % VCH;
        const bool ok = row < L;
        const int64_t off = ok ? ((tok0 + row) * H + h) * kHeadDim + v0 + ch * 8 : 0;
        cp_async16(smem_u32(sm + S::V) + tc::mnmaj_chunk(ch, row, 64), v + off, ok ? 16 : 0);
    }
}

// pair p = R(R+1)/2 + I  (I <= R)
__device__ __forceinline__ int pair_R(int p) { return p >= 6 ? 3 : p >= 3 ? 2 : p >= 1 ? 1 : 0; }

__device__ __forceinline__ uint4 pack8(const float *x, float s) {
    return make_uint4(pack_bf16(x[0] * s, x[1] * s), pack_bf16(x[2] * s, x[3] * s), pack_bf16(x[4] * s, x[5] * s),
                      pack_bf16(x[6] * s, x[7] * s));
}

// Output rows 64-127 of the chunk accumulator (O) -> o = O / sqrt(128) in bf16.
template <int VS>
__device__ __forceinline__ void store_output(uint32_t lane_base, int lq, int lane, int cgw, int64_t tok0, int L,
                                             int H, int h, int v0, uint16_t *out) {
    constexpr int CW = VS / 4;
    const float out_scale = rsqrtf((float)kHeadDim);
    const int r = 32 * (lq - 2) + lane;
    float o[32];
    if (CW == 32) {
        tc::ld32(lane_base + kTmemD + 32 * cgw, o);
    } else {
        float o16[16];
        tc::ld16(lane_base + kTmemD + 16 * cgw, o16);
#pragma unroll
        for (int i = 0; i < 16; ++i) o[i] = o16[i];
    }
    tc::wait_ld();
    if (r < L) {
        uint16_t *dst = out + ((tok0 + r) * H + h) * kHeadDim + v0 + CW * cgw;
#pragma unroll
        for (int e = 0; e < CW / 8; ++e) *reinterpret_cast<uint4 *>(dst + 8 * e) = pack8(o + 8 * e, out_scale);
    }
}

template <int VS>
__global__ void __launch_bounds__(kThreads, 1)
    kda_fwd_tc_kernel(const uint16_t *__restrict__ q, const uint16_t *__restrict__ k,
                      const uint16_t *__restrict__ v, const float *__restrict__ g,
                      const float *__restrict__ beta, const int32_t *__restrict__ cu_seqlens, int n_docs,
                      int64_t T, int H, uint16_t *__restrict__ out, int *__restrict__ status) {
    using S = Smem<VS>;
    constexpr int NV = kHeadDim / VS;
    constexpr int CW = VS / 4;            // TMEM columns per warp in the U~ / O passes
    static_assert(CW == 32 || CW == 16, "VS must be 128 or 64");
    extern __shared__ __align__(1024) uint8_t sm_raw[];
    // align by offsetting the shared array itself, so every access stays in the shared window (LDS/STS)
    uint8_t *sm = sm_raw + (((smem_u32(sm_raw) + 1023u) & ~1023u) - smem_u32(sm_raw));

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int gq = lane >> 2, tq = lane & 3;
    const int vsl = blockIdx.x % NV;
    const int chain = blockIdx.x / NV;
    const int doc = chain / H, h = chain % H;
    const int v0 = vsl * VS;

    if (blockIdx.x == 0 && tid == 0) {
        if (cu_seqlens[0] != 0 || (int64_t)cu_seqlens[n_docs] != T) atomicExch(status, kStatusBadSeqlens);
    }
    const int64_t doc_start = cu_seqlens[doc], doc_end = cu_seqlens[doc + 1];
    if (doc_start < 0 || doc_end < doc_start || doc_end > T) {
        if (tid == 0) atomicExch(status, kStatusBadSeqlens);
        return;
    }
    if (doc_end == doc_start) return;

    float *f_beta = reinterpret_cast<float *>(sm + S::BETA);
    float *f_rq = reinterpret_cast<float *>(sm + S::RQ);
    float *f_rk = reinterpret_cast<float *>(sm + S::RK);
    float *f_tot = reinterpret_cast<float *>(sm + S::TOT);
    float *f_ps = reinterpret_cast<float *>(sm + S::PS);
    float *f_dc = reinterpret_cast<float *>(sm + S::DC);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(sm + S::ABORT);
    const uint32_t mbar0 = smem_u32(sm + S::MBAR);
    const uint32_t sbase = smem_u32(sm);

    // ---- setup: TMEM, mbarriers, the zero state, the first chunk's loads ----
    if (warp == 0) tc::alloc(smem_u32(sm + S::TBASE), kTmemCols);
    if (tid == 0) {
        for (int i = 0; i < 3; ++i) tc::mbar_init(mbar0 + 8 * i, 1);
        *abort_flag = 0;
    }
    {
        const int L0 = (int)(doc_end - doc_start < 64 ? doc_end - doc_start : 64);
        load_qk<VS>(sm, q, k, doc_start, L0, H, h, tid, kThreads);
        load_gb<VS>(sm, g, beta, doc_start, L0, H, h);
        load_v<VS>(sm, v, doc_start, L0, H, h, v0);
        cp_async_commit();
    }
    tc::fence_before();
    __syncthreads();
    tc::fence_after();
    const uint32_t tmem = *reinterpret_cast<volatile uint32_t *>(sm + S::TBASE);
    const int lq = warp & 3;                   // TMEM lane quarter of this warp
    const int cgw = warp >> 2;                 // column group of this warp (0..3)
    const uint32_t lane_base = tmem + ((uint32_t)(32 * lq) << 16);
    if (warp >= 12) {
        float z[32];
#pragma unroll
        for (int i = 0; i < 32; ++i) z[i] = 0.f;
#pragma unroll
        for (int c0 = 0; c0 < VS; c0 += 32) tc::st32(lane_base + kTmemS + c0, z);
        tc::wait_st();
    }
    tc::fence_before();
    __syncthreads();
    tc::fence_after();

    uint32_t iter = 0;
    bool aborted = false;
    int64_t prev_tok0 = 0;
    int prev_L = 0;

    for (int64_t tok0 = doc_start; tok0 < doc_end; tok0 += 64, ++iter) {
        const int L = (int)(doc_end - tok0 < 64 ? doc_end - tok0 : 64);
        const int64_t ntok0 = tok0 + 64;
        const int nL = (int)(doc_end - ntok0 < 64 ? doc_end - ntok0 : 64);   // <= 0: no next chunk
        const uint32_t par = iter & 1;
        cp_async_wait_all();
        __syncthreads();

        // ---- previous chunk's output (lanes 64-127) || this chunk's norms (lanes 0-63 warps) ----
        if (lq >= 2) {
            if (iter > 0) {
                if (!tc::mbar_wait(mbar0 + 16, par ^ 1u, kWaitLimit)) *abort_flag = 1;
                tc::fence_after();
                store_output<VS>(lane_base, lq, lane, cgw, prev_tok0, prev_L, H, h, v0, out);
            }
        } else {
            const int nidx = cgw * 2 + lq;     // 0..7: rows 8 nidx .. 8 nidx + 7
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                const int r = nidx * 8 + i;
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
        tc::fence_before();
        __syncthreads();
        tc::fence_after();
        if (*abort_flag) { aborted = true; break; }

        // ---------------- prep pass 1: thread = (channel c, row block R) ----------------
        const int pc = tid & 127, pR = tid >> 7;
        float ql[16], kl[16], kr[16];
        float lg0, lg15;
        {
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
        __syncthreads();   // raw q, k, g fully read; block sums of g published
        // ---------------- prep pass 2 ----------------
        {
            float offs[5];
            offs[0] = 0.f;
#pragma unroll
            for (int R = 0; R < 4; ++R) offs[R + 1] = offs[R] + f_tot[R * 128 + pc];
            const float gm = offs[pR] + lg0;                   // Gamma at row 16R
            const float ge = offs[pR + 1];                     // Gamma at row 16R+15
            const float gl = offs[4];                          // Gamma at the last row
            const float P = fast_exp2(gm * kLog2e);            // e^{Gamma_16R} (<= 1)
            const float Dk = fast_exp2((gl - ge) * kLog2e);    // e^{Gamma_last - Gamma_16R+15} (<= 1)
#pragma unroll
            for (int I = 0; I < 4; ++I)
                if (I <= pR) f_ps[(pR * (pR + 1) / 2 + I) * 128 + pc] = fast_exp2((gm - offs[I + 1]) * kLog2e);
            if (pR == 0) f_dc[pc] = fast_exp2(gl * kLog2e);
#pragma unroll
            for (int half = 0; half < 2; ++half) {
                const int j0 = half * 8;
                const uint32_t off = tc::kmaj_chunk(pc, 2 * pR + half);
                // q^E1 and k^E1 overwrite the raw q / k tiles; k^E2 has its own tile
                *reinterpret_cast<uint4 *>(sm + S::Q + off) = pack8(ql + j0, 1.f);
                *reinterpret_cast<uint4 *>(sm + S::K + off) = pack8(kl + j0, 1.f);
                *reinterpret_cast<uint4 *>(sm + S::KR + off) = pack8(kr + j0, 1.f);
                *reinterpret_cast<uint4 *>(sm + S::KGT + off) = pack8(kl + j0, P);
                *reinterpret_cast<uint4 *>(sm + S::KDT + off) = pack8(kr + j0, Dk);
                // -Q~ into rows 64.. of A2 (MN-major: K-row c, M = 64 + r)
                *reinterpret_cast<uint4 *>(sm + S::A2 + tc::mnmaj_chunk(8 + 2 * pR + half, pc, 128)) =
                    pack8(ql + j0, -P);
            }
        }
        __syncthreads();

        if (warp >= 12) {
            // ---------------- state warpgroup: S <- Diag(e^{Gamma_last}) S, bf16 copy of the old S ----------------
            const int c = 32 * lq + lane;
            const float dcy = f_dc[c];
#pragma unroll 1
            for (int col0 = 0; col0 < VS; col0 += 32) {
                float s[32];
                tc::ld32(lane_base + kTmemS + col0, s);
                tc::wait_ld();
#pragma unroll
                for (int e = 0; e < 4; ++e)
                    *reinterpret_cast<uint4 *>(sm + S::SB + tc::mnmaj_chunk(col0 / 8 + e, c, 128)) = pack8(s + 8 * e, 1.f);
#pragma unroll
                for (int i = 0; i < 32; ++i) s[i] *= dcy;
                tc::st32(lane_base + kTmemS + col0, s);
            }
            tc::wait_st();
            tc::fence_proxy_async();
            tc::fence_before();
        } else {
            // ---------------- intra: A_kk and A_qk, one 16x16 block pair per warp ----------------
            if (warp < 10) {
                const int p = warp;
                const int R = pair_R(p), I = p - R * (R + 1) / 2;
                const uint32_t kbase = smem_u32(sm + S::K), qbase = smem_u32(sm + S::Q);
                const uint32_t rbase = smem_u32(sm + S::KR);
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
                    ldsm_x4_t(rbase + tc::kmaj_chunk(16 * kk + (lane & 7) + 8 * (j & 1), 2 * I + (j >> 1)), b0, b1, b2,
                              b3);
                    const int cb = kk * 16 + 2 * tq;
                    const float2 s0 = *reinterpret_cast<const float2 *>(ps + cb);
                    const float2 s8 = *reinterpret_cast<const float2 *>(ps + cb + 8);
                    // pair scale on the channel pairs of the fragment, packed bf16x2 multiply
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
#pragma unroll
                for (int nt = 0; nt < 2; ++nt)
#pragma unroll
                    for (int hh = 0; hh < 2; ++hh) {
                        const int row = 16 * R + gq + 8 * hh;
                        const int col = 16 * I + 8 * nt + 2 * tq;
                        const float br = f_beta[row];
                        const float x0 = col < row ? ak[nt][2 * hh] * br : 0.f;
                        const float x1 = col + 1 < row ? ak[nt][2 * hh + 1] * br : 0.f;
                        *reinterpret_cast<float2 *>(sm + S::AKK + swz_f32(row, col, 256)) = make_float2(x0, x1);
                        const float y0 = col <= row ? aq[nt][2 * hh] : 0.f;
                        const float y1 = col + 1 <= row ? aq[nt][2 * hh + 1] : 0.f;
                        *reinterpret_cast<uint32_t *>(sm + S::AQK + tc::kmaj_off(row, col)) = pack_bf16(y0, y1);
                    }
            }
            bar_intra();
            // q^E1 / k^E1 consumed: prefetch the next chunk's raw q, k
            if (nL > 0) {
                load_qk<VS>(sm, q, k, ntok0, nL, H, h, tid, kIntraThreads);
                cp_async_commit();
            }
            // ---------------- intra: T = (I + A_kk)^-1, diagonal 16x16 blocks ----------------
            if (warp < 4 && lane < 16) {
                const int R = warp, col = lane;
                float x[16];
#pragma unroll
                for (int r = 0; r < 16; ++r) {
                    float a[16];
#pragma unroll
                    for (int q4 = 0; q4 < 4; ++q4) {
                        const float4 t4 =
                            *reinterpret_cast<const float4 *>(sm + S::AKK + swz_chunk(16 * R + r, 4 * R + q4, 256));
                        a[4 * q4] = t4.x; a[4 * q4 + 1] = t4.y; a[4 * q4 + 2] = t4.z; a[4 * q4 + 3] = t4.w;
                    }
                    float acc = (r == col) ? 1.f : 0.f;
#pragma unroll
                    for (int jj = 0; jj < r; ++jj) acc -= a[jj] * x[jj];
                    x[r] = acc;
                }
#pragma unroll
                for (int r = 0; r < 16; ++r)
                    *reinterpret_cast<float *>(sm + S::TM + swz_f32(16 * R + r, 16 * R + col, 256)) = x[r];
            }
            bar_intra();
            auto akk = [&](int r, int c) -> float {
                return *reinterpret_cast<const float *>(sm + S::AKK + swz_f32(r, c, 256));
            };
            auto tmf = [&](int r, int c) -> float * {
                return reinterpret_cast<float *>(sm + S::TM + swz_f32(r, c, 256));
            };
            // off-diagonal blocks by distance d: T_{R,R-d} = -T_RR sum_{J=R-d}^{R-1} A_{R,J} T_{J,R-d}
#pragma unroll 1
            for (int d = 1; d < 4; ++d) {
                const int njobs = 2 * (4 - d);
                if (warp < njobs) {
                    const int R = d + (warp >> 1), I = R - d, nt = warp & 1;
                    float xacc[4] = {0.f, 0.f, 0.f, 0.f};
                    for (int J = I; J < R; ++J) {
#pragma unroll
                        for (int kb = 0; kb < 16; kb += 8) {
                            const uint32_t a0 = tf32(akk(16 * R + gq, 16 * J + kb + tq));
                            const uint32_t a1 = tf32(akk(16 * R + gq + 8, 16 * J + kb + tq));
                            const uint32_t a2 = tf32(akk(16 * R + gq, 16 * J + kb + tq + 4));
                            const uint32_t a3 = tf32(akk(16 * R + gq + 8, 16 * J + kb + tq + 4));
                            const uint32_t b0 = tf32(*tmf(16 * J + kb + tq, 16 * I + 8 * nt + gq));
                            const uint32_t b1 = tf32(*tmf(16 * J + kb + tq + 4, 16 * I + 8 * nt + gq));
                            mma_tf32(xacc, a0, a1, a2, a3, b0, b1);
                        }
                    }
                    float *xt = reinterpret_cast<float *>(sm + S::XT) + warp * 128;   // X[16][8]
                    xt[gq * 8 + 2 * tq] = xacc[0];
                    xt[gq * 8 + 2 * tq + 1] = xacc[1];
                    xt[(gq + 8) * 8 + 2 * tq] = xacc[2];
                    xt[(gq + 8) * 8 + 2 * tq + 1] = xacc[3];
                    __syncwarp();
                    float tacc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
                    for (int kb = 0; kb < 16; kb += 8) {
                        const uint32_t a0 = tf32(*tmf(16 * R + gq, 16 * R + kb + tq));
                        const uint32_t a1 = tf32(*tmf(16 * R + gq + 8, 16 * R + kb + tq));
                        const uint32_t a2 = tf32(*tmf(16 * R + gq, 16 * R + kb + tq + 4));
                        const uint32_t a3 = tf32(*tmf(16 * R + gq + 8, 16 * R + kb + tq + 4));
                        const uint32_t b0 = tf32(xt[(kb + tq) * 8 + gq]);
                        const uint32_t b1 = tf32(xt[(kb + tq + 4) * 8 + gq]);
                        mma_tf32(tacc, a0, a1, a2, a3, b0, b1);
                    }
                    const int col = 16 * I + 8 * nt + 2 * tq;
                    *reinterpret_cast<float2 *>(tmf(16 * R + gq, col)) = make_float2(-tacc[0], -tacc[1]);
                    *reinterpret_cast<float2 *>(tmf(16 * R + gq + 8, col)) = make_float2(-tacc[2], -tacc[3]);
                }
                bar_intra();
            }
            // T' = T diag(beta) -> bf16 rows 0-63 of A1 (K-major); rows 64-127 zero
            for (int idx = tid; idx < 512; idx += kIntraThreads) {
                const int r = idx >> 3, ch = idx & 7;
                uint32_t w4[4];
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const int c0 = ch * 8 + 2 * e;
                    const float x0 = c0 <= r ? *tmf(r, c0) * f_beta[c0] : 0.f;
                    const float x1 = c0 + 1 <= r ? *tmf(r, c0 + 1) * f_beta[c0 + 1] : 0.f;
                    w4[e] = pack_bf16(x0, x1);
                }
                *reinterpret_cast<uint4 *>(sm + S::KR + tc::kmaj_chunk(r, ch)) = make_uint4(w4[0], w4[1], w4[2], w4[3]);
                *reinterpret_cast<uint4 *>(sm + S::KR + tc::kmaj_chunk(64 + r, ch)) = make_uint4(0, 0, 0, 0);
            }
            // A_qk above the block diagonal is zero (the tensor-core product reads all 64 columns)
            if (tid < 192) {
                const int b = tid >> 5, row = (tid & 31) >> 1, half = tid & 1;
                const int R = b < 3 ? 0 : b < 5 ? 1 : 2;                 // (0,1) (0,2) (0,3) (1,2) (1,3) (2,3)
                const int I = b < 3 ? b + 1 : b < 5 ? b - 1 : 3;
                *reinterpret_cast<uint4 *>(sm + S::AQK + tc::kmaj_chunk(16 * R + row, 2 * I + half)) =
                    make_uint4(0, 0, 0, 0);
            }
            tc::fence_proxy_async();
            tc::fence_before();
        }
        __syncthreads();
        tc::fence_after();
        // g, beta, A_kk and T are dead: prefetch the next chunk's g and beta
        if (nL > 0) {
            load_gb<VS>(sm, g, beta, ntok0, nL, H, h);
            cp_async_commit();
        }
        // ---------------- tcgen05: W^T = KG^T T'^T and D = [T'; 0] V ----------------
        if (tid == 0) {
            constexpr uint32_t id_w = tc::idesc_bf16(128, 64, false, false, false);
            constexpr uint32_t id_u = tc::idesc_bf16(128, VS, false, true, false);
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)
                tc::mma(tmem + kTmemW, tc::desc_kmaj(sbase + S::KGT, kk), tc::desc_kmaj(sbase + S::KR, kk), id_w,
                        kk > 0);
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)
                tc::mma(tmem + kTmemD, tc::desc_kmaj(sbase + S::KR, kk), tc::desc_mnmaj(sbase + S::V, kk, 64), id_u,
                        kk > 0);
            tc::commit(mbar0);
        }
        // ---------------- W^T -> bf16 rows 0-63 of A2 ----------------
        {
            if (!tc::mbar_wait(mbar0, par, kWaitLimit)) *abort_flag = 1;
            tc::fence_after();
            const int c = 32 * lq + lane;
            float w[16];
            tc::ld16(lane_base + kTmemW + 16 * cgw, w);
            tc::wait_ld();
#pragma unroll
            for (int half = 0; half < 2; ++half)
                *reinterpret_cast<uint4 *>(sm + S::A2 + tc::mnmaj_chunk(2 * cgw + half, c, 128)) = pack8(w + 8 * half, 1.f);
        }
        tc::fence_proxy_async();
        tc::fence_before();
        __syncthreads();
        tc::fence_after();
        if (*abort_flag) { aborted = true; break; }
        // v is consumed (U done): prefetch the next chunk's v
        if (nL > 0) {
            load_v<VS>(sm, v, ntok0, nL, H, h, v0);
            cp_async_commit();
        }
        // ---------------- tcgen05: D += -[W; -Q~] S ----------------
        if (tid == 0) {
            constexpr uint32_t id2 = tc::idesc_bf16(128, VS, true, true, true);
#pragma unroll
            for (int kk = 0; kk < 8; ++kk)
                tc::mma(tmem + kTmemD, tc::desc_mnmaj(sbase + S::A2, kk, 128), tc::desc_mnmaj(sbase + S::SB, kk, 128),
                        id2, 1u);
            tc::commit(mbar0 + 8);
        }
        // ---------------- U~ (rows 0-63 of D) -> bf16 shared ----------------
        {
            if (!tc::mbar_wait(mbar0 + 8, par, kWaitLimit)) *abort_flag = 1;
            tc::fence_after();
            if (lq < 2) {
                const int r = 32 * lq + lane;
                if (CW == 32) {
                    float u[32];
                    tc::ld32(lane_base + kTmemD + 32 * cgw, u);
                    tc::wait_ld();
#pragma unroll
                    for (int e = 0; e < 4; ++e)
                        *reinterpret_cast<uint4 *>(sm + S::KR + tc::mnmaj_chunk(4 * cgw + e, r, 64)) = pack8(u + 8 * e, 1.f);
                } else {
                    float u[16];
                    tc::ld16(lane_base + kTmemD + 16 * cgw, u);
                    tc::wait_ld();
#pragma unroll
                    for (int e = 0; e < 2; ++e)
                        *reinterpret_cast<uint4 *>(sm + S::KR + tc::mnmaj_chunk(2 * cgw + e, r, 64)) = pack8(u + 8 * e, 1.f);
                }
            }
        }
        tc::fence_proxy_async();
        tc::fence_before();
        __syncthreads();
        tc::fence_after();
        if (*abort_flag) { aborted = true; break; }
        // ---------------- tcgen05: O = Q~S + A_qk U~ ;  S += Kd^T U~ ----------------
        if (tid == 0) {
            constexpr uint32_t id3 = tc::idesc_bf16(128, VS, false, true, false);
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)
                tc::mma(tmem + kTmemD, tc::desc_kmaj(sbase + S::AQK - 8192, kk), tc::desc_mnmaj(sbase + S::KR, kk, 64),
                        id3, 1u);
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)
                tc::mma(tmem + kTmemS, tc::desc_kmaj(sbase + S::KDT, kk), tc::desc_mnmaj(sbase + S::KR, kk, 64), id3,
                        1u);
            tc::commit(mbar0 + 16);
        }
        prev_tok0 = tok0;
        prev_L = L;
        // the output of this chunk is stored at the top of the next iteration (or below)
    }

    if (!aborted && iter > 0) {
        if (lq >= 2) {
            if (!tc::mbar_wait(mbar0 + 16, (iter - 1) & 1u, kWaitLimit)) *abort_flag = 1;
            tc::fence_after();
            store_output<VS>(lane_base, lq, lane, cgw, prev_tok0, prev_L, H, h, v0, out);
        }
        tc::fence_before();
        __syncthreads();
        if (*abort_flag) aborted = true;
    }
    // ---- teardown: no copy or MMA may still be in flight when TMEM is freed ----
    cp_async_wait_all();
    if (aborted) {
        if (tid == 0) atomicExch(status, kStatusTimeout);
        for (int i = 0; i < 3; ++i) tc::mbar_wait(mbar0 + 8 * i, (iter & 1), kWaitLimit / 4);
    }
    tc::fence_before();
    __syncthreads();
    tc::fence_after();
    if (warp == 0) tc::dealloc(tmem, kTmemCols);
}

template <int VS>
cudaError_t launch(const uint16_t *q, const uint16_t *k, const uint16_t *v, const float *g, const float *beta,
                   const int32_t *cu, int n_docs, int64_t T, int H, uint16_t *out, int *status,
                   cudaStream_t stream) {
    constexpr int bytes = Smem<VS>::ALLOC;
    static_assert(bytes <= 232448, "shared memory budget");
    cudaError_t e =
        cudaFuncSetAttribute(kda_fwd_tc_kernel<VS>, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
    if (e != cudaSuccess) return e;
    const int64_t blocks = (int64_t)n_docs * H * (kHeadDim / VS);
    kda_fwd_tc_kernel<VS><<<(unsigned)blocks, kThreads, bytes, stream>>>(q, k, v, g, beta, cu, n_docs, T, H, out,
                                                                        status);
    return cudaGetLastError();
}

}  // namespace tc_path

cudaError_t launch_fwd_tc(const uint16_t *q, const uint16_t *k, const uint16_t *v, const float *g,
                          const float *beta, const int32_t *cu, int n_docs, int64_t T, int H, uint16_t *out,
                          int *status, int v_slice, cudaStream_t stream) {
    if (v_slice == 128) return tc_path::launch<128>(q, k, v, g, beta, cu, n_docs, T, H, out, status, stream);
    return tc_path::launch<64>(q, k, v, g, beta, cu, n_docs, T, H, out, status, stream);
}

}  // namespace kda
