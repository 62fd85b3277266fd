// kda_fwd_pipe.cu -- pipelined fused chunk-KDA forward (one CTA per (document, head),
// all 128 value columns); kda_chunk_fwd launches it for every call.
//
// Two chunks are in flight per CTA.  In step s all 16 warps first prepare chunk s (gate factors
// and every bf16 operand tile); then warps 0-11 finish chunk s's intra-chunk work while warps
// 12-15 run chunk s-1's state update and output.  Every chunk product runs on the tensor cores
// with tcgen05.mma (accumulators in tensor memory); only the UT solve's 16 x 16 block products
// use warp-level MMA.
//
// Per chunk, with raw q and k, Gamma the inclusive in-chunk cumsum of g, and the row norms
// n_r = 1/|q_r|, m_r = 1/|k_r| applied outside the products:
//   L_qk[r,i] = sum_c q_rc k_ic e^{Gamma_rc - Gamma_ic} (i <= r),  L_kk likewise (i < r)
//   A_kk = diag(beta m) L_kk diag(m),   T = (I + A_kk)^-1
//   T_U  = diag(m) T diag(beta),        T_W = T_U diag(m)
//   U' = T_U V,   W' = T_W (K e^Gamma),   U~ = U' - W' S       (U~ is diag(m) times the usual U~)
//   O  = (Q e^Gamma) S + L_qk U~,          o = scale diag(n) O
//   S <- Diag(e^{Gamma_63}) S + (K e^{Gamma_63 - Gamma})^T U~
// which is the recurrence unrolled over the chunk with q^ = diag(n) q and k^ = diag(m) k.
//
// L_qk and L_kk come from one tcgen05 product.  The exponent is split at a reference row in the
// middle of each 32-row half (rows 15 and 47): the row side carries e^{Gamma_r - Gamma_ref(r)},
// the column side e^{Gamma_ref - Gamma_i}; with gates in [-5, 0] every factor lies within
// e^{+-80}, inside the fp32 / bf16 range, and each product term keeps its true size
// |q_rc k_ic| e^{Gamma_rc - Gamma_ic} <= |q_rc k_ic|.  The product is
//   D[128 rows: q rows | k rows][96 cols] = X Y^T,
//   X rows r: (q_r | k_r) e^{Gamma_r - Gamma_ref(r)},
//   Y cols 0..63: k_i e^{Gamma_47 - Gamma_i} (the reference of rows 32..63),
//   Y cols 64..95: k_i e^{Gamma_15 - Gamma_i}, i < 32 (the reference of rows 0..31);
// entries of other pairs are never read.
//
// The state is kept transposed, S^T[v][c] in fp32 in tensor memory (lane = value column v), so
// that both its bf16 copy and U~ are tcgen05 A operands read straight from tensor memory:
//   state  D   = [U'^T | 0] + S^T_bf16 [-W'^T | Q~^T]   -> [U~^T | (Q~ S)^T]
//          O^T += U~^T_bf16 L_qk^T,   S^T += U~^T_bf16 Kd     (after S^T <- S^T Diag(e^{Gamma_63}))
// q, k and v tiles arrive by TMA (2-D tensor maps over [T, H*128]); each prep thread reads its
// channel of g straight from global memory one step ahead (the tiles are prefetched into L2
// two chunks ahead).  A tile may reach into the next document; rows past the document end are
// read as zero (q, k, g, beta) or zeroed in shared memory (v), so poisoned neighbours cannot
// leak.  Every wait is time-limited and reports KDA_ERR_TIMEOUT.
#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>
#include <stdint.h>

#include <mutex>

#include "kda_common.cuh"
#include "kda_internal.h"
#include "kda_tc.cuh"

namespace kda {
namespace pipe_path {

constexpr int kThreads = 512;
constexpr int kStateTid0 = 384;               // first thread of warps 12-15
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kSF = 0;                   // S^T fp32                   [128 lanes v][128 cols c]
constexpr uint32_t kSB = 128;                 // S^T bf16 packed            [128][64]
constexpr uint32_t kUB = 128;                 // U~^T bf16 packed [128][32], over S^T bf16 once the state product is done
constexpr uint32_t kDA = 192;                 // L product [128][96]; then -W'^T [128 c][64 r]
constexpr uint32_t kQT = 288;                 // Q~^T fp32 [128 c][64 r]
constexpr uint32_t kDS = 352;                 // [U'^T -> U~^T | O^T]       [128 v][64 + 64]
constexpr long long kWaitLimit = 2000000000LL;

// A_kk / T as ten 16x16 fp32 blocks (I <= R), rows padded to 20 floats
constexpr int kBlkPitch = 20;
constexpr int kBlkFloats = 16 * kBlkPitch;

struct Smem {
    static constexpr int AX = 0;           // raw q, k: TMA boxes [64 rows][64 ch] at +0, +8192 (q), +16384, +24576 (k);
                                           // then the row side X, MN-major [c][r], atoms q | k
    static constexpr int BY = 32768;       // column side Y, MN-major [c][n], two 64-wide atoms (N = 96 used)
    static constexpr int TU = BY;          // after the L product: T_U bf16, K-major [r][i]
    static constexpr int TW = BY + 8192;   //                      T_W bf16, K-major [r][i]
    static constexpr int V = 65536;        // raw v: two TMA boxes, 128B-swizzled = MN-major SW128 atoms
    static constexpr int KGT = 81920;      // (K e^Gamma)^T, K-major [c][i]
    static constexpr int KDT = 98304;      // two buffers: (K e^{Gamma_63 - Gamma})^T, K-major [c][r]; output staging
    static constexpr int B2 = 131072;      // [-W'^T | Q~^T], MN-major [c][n], two 64-wide atoms
    static constexpr int AQK = 163840;     // two buffers: L_qk [r][i], K-major (64 rows)
    static constexpr int SMALL = 180224;
    static constexpr int BETA = SMALL;               // fp32 [2][64]
    static constexpr int RQ = BETA + 512;            // fp32 [4][64]  scale / |q_r|
    static constexpr int RK = RQ + 1024;             // fp32 [2][64]  1 / |k_r|
    static constexpr int TOT = RK + 512;             // fp32 [4][128] per 16-row block sums of log2e g
    static constexpr int DL = TOT + 2048;            // fp32 [2][128] e^{Gamma_63}
    static constexpr int MBAR = DL + 1024;           // u64 [16]
    static constexpr int TBASE = MBAR + 128;
    static constexpr int ABORT = TBASE + 16;
    static constexpr int AKK = 186368;               // A_kk blocks fp32 (after the small arrays, 1024-aligned)
    static constexpr int TM = AKK + 10 * kBlkFloats * 4;   // T blocks fp32
    // raw g of the next chunk: four TMA boxes [64 rows][32 ch] fp32, landing over the A_kk / T blocks
    // once the solve is done with them and read by the next step's prep before the next read-back
    static constexpr int G = AKK;
    static constexpr int BYTES = G + 32768;
    static constexpr int ALLOC = BYTES + 1024;
};
static_assert(Smem::ALLOC <= 232448, "shared memory budget");
static_assert(Smem::ABORT + 16 <= Smem::AKK && Smem::TM + 10 * kBlkFloats * 4 <= Smem::BYTES, "layout");

// every barrier completes by tcgen05.commit or by TMA transaction bytes
enum Mbar { kMbA = 0, kMbW, kMbU, kMb2, kMb4, kMbQK, kMbG, kMbV, kNumMbar };

__device__ __forceinline__ void bar_intra() { asm volatile("bar.sync 1, 384;" ::: "memory"); }
__device__ __forceinline__ void bar_state() { asm volatile("bar.sync 2, 128;" ::: "memory"); }
__device__ __forceinline__ void bar_solve() { asm volatile("bar.sync 3, 256;" ::: "memory"); }   // warps 0-7

// tf32 warp MMA on fp32 bit patterns (the tensor core ignores the low mantissa bits)
__device__ __forceinline__ void mma_tf32(float (&d)[4], float a0, float a1, float a2, float a3, float b0, float b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k8.row.col.f32.tf32.tf32.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%0,%1,%2,%3};\n"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(__float_as_uint(a0)), "r"(__float_as_uint(a1)), "r"(__float_as_uint(a2)), "r"(__float_as_uint(a3)),
          "r"(__float_as_uint(b0)), "r"(__float_as_uint(b1)));
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
__device__ __forceinline__ void st8(uint32_t taddr, const uint32_t (&r)[8]) {
    asm volatile("tcgen05.st.sync.aligned.32x32b.x8.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8};" ::"r"(taddr), "r"(r[0]),
                 "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7])
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
// eight values held as four row pairs, as bf16
__device__ __forceinline__ uint4 pack8x2(const float2 *x) {
    return make_uint4(pack_bf16(x[0].x, x[0].y), pack_bf16(x[1].x, x[1].y), pack_bf16(x[2].x, x[2].y),
                      pack_bf16(x[3].x, x[3].y));
}
// 1/x by the hardware approximation (PTX rcp.approx.ftz; x here is a product of decays in
// [e^-80, 1], far from the denormal range)
__device__ __forceinline__ float rcp_approx(float x) {
    float y;
    asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}
// registers filled by tcgen05.ld are valid only after tcgen05.wait::ld: this empty asm, placed after
// the wait, keeps the compiler from moving their first use above it
template <int N>
__device__ __forceinline__ void reg_fence(float (&v)[N]) {
#pragma unroll
    for (int i = 0; i < N; ++i) asm volatile("" : "+f"(v[i]));
}
__device__ __forceinline__ int pair_of(int R, int I) { return R * (R + 1) / 2 + I; }

// beta rows [tok0, tok0 + L) of head h, one row per calling thread (row in [0, 64); rows >= L zero-filled)
__device__ __forceinline__ void load_beta(uint8_t *sm, const float *beta, int64_t tok0, int L, int H, int h, int buf,
                                          int row) {
    const bool ok = row < L;
    const float *src = ok ? beta + (tok0 + row) * H + h : beta;
    asm volatile("cp.async.ca.shared.global [%0], [%1], 4, %2;\n" ::"r"(smem_u32(sm + Smem::BETA + buf * 256 + row * 4)),
                 "l"(src), "r"(ok ? 4 : 0)
                 : "memory");
}

struct Maps {
    CUtensorMap q, k, g, v, o;
};

// kCkpt: also store the state entering every chunk into `ckpt` (the backward's checkpoints); a
// separate instance, so that the plain forward carries no trace of it
template <bool kCkpt>
__global__ void __launch_bounds__(kThreads, 1)
    kda_fwd_pipe_kernel(const __grid_constant__ Maps maps, const float *__restrict__ g, const float *__restrict__ beta,
                        const int32_t *__restrict__ cu_seqlens, int n_docs, int64_t T, int H, const float *h0,
                        float *ht, float *ckpt, uint16_t *__restrict__ out, int *__restrict__ status) {
    using S = Smem;
    extern __shared__ __align__(1024) uint8_t sm_raw[];
    // align by offsetting the shared array itself, so every access stays in the shared window (LDS/STS)
    uint8_t *sm = sm_raw + (((smem_u32(sm_raw) + 1023u) & ~1023u) - smem_u32(sm_raw));

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int gq = lane >> 2, tq = lane & 3;
    // CTA -> (document, head), longest documents first; the AX area is free until the first TMA load
    const int doc = doc_at_rank(cu_seqlens, n_docs, blockIdx.x / H, reinterpret_cast<int *>(sm)), h = blockIdx.x % H;

    if (blockIdx.x == 0 && tid == 0) {
        if (cu_seqlens[0] != 0 || (int64_t)cu_seqlens[n_docs] != T) atomicExch(status, kStatusBadSeqlens);
    }
    const int64_t doc_start = cu_seqlens[doc], doc_end = cu_seqlens[doc + 1];
    if (doc_start < 0 || doc_end < doc_start || doc_end > T) {
        if (tid == 0) atomicExch(status, kStatusBadSeqlens);
        return;
    }
    // initial / final state of this chain: [n_docs * H][128 key channels][128 value columns] fp32
    const size_t state_off = ((size_t)doc * H + h) * kHeadDim * kHeadDim;
    if (doc_end == doc_start) {
        // nothing to process: the final state is the initial one
        if (ht)
            for (int idx = tid; idx < kHeadDim * kHeadDim; idx += kThreads)
                ht[state_off + idx] = h0 ? h0[state_off + idx] : 0.f;
        return;
    }
    const int nchunks = (int)((doc_end - doc_start + 63) / 64);
    auto chunk_len = [&](int i) -> int {
        const int64_t rem = doc_end - (doc_start + 64 * (int64_t)i);
        return rem <= 0 ? 0 : (rem < 64 ? (int)rem : 64);
    };

    float *f_rq = reinterpret_cast<float *>(sm + S::RQ);
    float *f_rk = reinterpret_cast<float *>(sm + S::RK);
    float *f_tot = reinterpret_cast<float *>(sm + S::TOT);
    float *f_dl = reinterpret_cast<float *>(sm + S::DL);
    float *f_akk = reinterpret_cast<float *>(sm + S::AKK);
    float *f_tm = reinterpret_cast<float *>(sm + S::TM);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(sm + S::ABORT);
    const uint32_t mb = smem_u32(sm + S::MBAR);
    auto mbar = [&](int i) -> uint32_t { return mb + 8u * (uint32_t)i; };
    const uint32_t sbase = smem_u32(sm);
    // UMMA shared-memory descriptors of the tile area; every operand descriptor is one of these plus the
    // tile's constant byte offset / 16 (addresses stay below 256 KB, so the 14-bit field cannot carry)
    const uint64_t dK = tc::sdesc(sbase, 16u, 1024u);           // K-major, 128-byte swizzled rows
    const uint64_t dM128 = tc::sdesc(sbase, 128u * 128u, 1024u); // MN-major, 128 K rows per 64-wide atom
    const uint64_t dM64 = tc::sdesc(sbase, 64u * 128u, 1024u);   // MN-major, 64 K rows per 64-wide atom
    const int xq = h * kHeadDim;          // TMA x coordinate of this head's channel 0

    auto issue_qk = [&](int i) {          // q, k tiles of chunk i (one thread)
        const int y = (int)(doc_start + 64 * (int64_t)i);
        tc::mbar_expect_tx(mbar(kMbQK), 32768u);
        tc::tma_load_2d(sbase + S::AX, &maps.q, xq, y, mbar(kMbQK));
        tc::tma_load_2d(sbase + S::AX + 8192, &maps.q, xq + 64, y, mbar(kMbQK));
        tc::tma_load_2d(sbase + S::AX + 16384, &maps.k, xq, y, mbar(kMbQK));
        tc::tma_load_2d(sbase + S::AX + 24576, &maps.k, xq + 64, y, mbar(kMbQK));
    };
    auto issue_g = [&](int i) {
        const int y = (int)(doc_start + 64 * (int64_t)i);
        tc::mbar_expect_tx(mbar(kMbG), 32768u);
#pragma unroll
        for (int b = 0; b < 4; ++b) tc::tma_load_2d(sbase + S::G + 8192 * b, &maps.g, xq + 32 * b, y, mbar(kMbG));
    };
    auto issue_v = [&](int i) {
        const int y = (int)(doc_start + 64 * (int64_t)i);
        tc::mbar_expect_tx(mbar(kMbV), 16384u);
        tc::tma_load_2d(sbase + S::V, &maps.v, xq, y, mbar(kMbV));
        tc::tma_load_2d(sbase + S::V + 8192, &maps.v, xq + 64, y, mbar(kMbV));
    };
    // prep thread: channel pc, rows 16 pR .. 16 pR + 15 of the chunk
    const int pc = tid & 127, pR = tid >> 7;
    // scale/|q_r| and 1/|k_r| for rows r0..r0+15 of the raw tiles (rows >= Li count as zero), into
    // the buffers of chunk i.  Lane = (tensor, row): lanes 0-15 sum a q row, lanes 16-31 a k row,
    // reading its sixteen 16-byte chunks in an order rotated by the lane, so that every load
    // instruction touches each bank group only as often as its width requires.
    auto norms16 = [&](int r0, int Li, int i) {
        const int r = r0 + (lane & 15);
        const uint8_t *rowp = sm + S::AX + (lane >> 4) * 16384 + r * 128;
        float acc0 = 0.f, acc1 = 0.f;
        if (r < Li) {
#pragma unroll 1
            for (int j = 0; j < 16; ++j) {
                const int ch = (j + lane) & 15;
                const uint4 u = *reinterpret_cast<const uint4 *>(rowp + (ch >> 3) * 8192 + (ch & 7) * 16);
                const float2 x0 = unpack_bf16(u.x), x1 = unpack_bf16(u.y), x2 = unpack_bf16(u.z), x3 = unpack_bf16(u.w);
                acc0 = fmaf(x0.x, x0.x, fmaf(x0.y, x0.y, fmaf(x1.x, x1.x, fmaf(x1.y, x1.y, acc0))));
                acc1 = fmaf(x2.x, x2.x, fmaf(x2.y, x2.y, fmaf(x3.x, x3.x, fmaf(x3.y, x3.y, acc1))));
            }
        }
        const float rn = rsqrtf(acc0 + acc1 + 1e-6f);
        if (lane < 16) f_rq[(i & 3) * 64 + r] = rn * rsqrtf((float)kHeadDim);
        else f_rk[(i & 1) * 64 + r] = rn;
    };

    // ---- setup ----
    if (warp == 0) tc::alloc(smem_u32(sm + S::TBASE), kTmemCols);
    if (tid == 0) {
        for (int i = 0; i < kNumMbar; ++i) tc::mbar_init(mbar(i), 1);
        *abort_flag = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    __syncthreads();
    if (tid == 0) {
        issue_qk(0);
        issue_g(0);
    }
    if (tid < 64) load_beta(sm, beta, doc_start, chunk_len(0), H, h, 0, tid);
    cp_async_commit();
    tc::fence_before();
    __syncthreads();
    tc::fence_after();
    const uint32_t tmem = *reinterpret_cast<volatile uint32_t *>(sm + S::TBASE);
    const int lq = warp & 3;
    const uint32_t lane_base = tmem + ((uint32_t)(32 * lq) << 16);
    if (warp >= 12) {
        // S^T[v][c] (lane v) = h0[c][v], or zero; the O columns start at zero
        const int vcol = 32 * lq + lane;
#pragma unroll 1
        for (int c0 = 0; c0 < 128; c0 += 32) {
            float z[32];
#pragma unroll
            for (int i = 0; i < 32; ++i) z[i] = h0 ? h0[state_off + (size_t)(c0 + i) * kHeadDim + vcol] : 0.f;
            tc::st32(lane_base + kSF + c0, z);
        }
        float z[32];
#pragma unroll
        for (int i = 0; i < 32; ++i) z[i] = 0.f;
        tc::st32(lane_base + kDS + 64, z);
        tc::st32(lane_base + kDS + 96, z);
        tc::wait_st();
    }
    // chunk 0's q, k, g (one thread polls the barriers; the CTA barrier releases the rest), then its norms
    cp_async_wait_all();
    if (tid == 0) {
        bool ok = tc::mbar_wait(mbar(kMbQK), 0u, kWaitLimit);
        ok = tc::mbar_wait(mbar(kMbG), 0u, kWaitLimit) && ok;
        if (!ok) *abort_flag = 1;
    }
    __syncthreads();
    if (warp < 4) norms16(warp * 16, chunk_len(0), 0);
    tc::fence_before();
    __syncthreads();
    tc::fence_after();

    bool aborted = *abort_flag != 0;

    for (int s = 0; s <= nchunks && !aborted; ++s) {
        const bool have_intra = s < nchunks;        // chunk s: prep + intra
        const bool have_state = s >= 1;             // chunk s-1: state update + output
        const bool have_next = s + 1 < nchunks;     // chunk s+1 exists
        const int L = chunk_len(s);
        const int nL = chunk_len(s + 1);
        const int buf = s & 1;
        const uint32_t par = (uint32_t)(s & 1);

        // q, k, g and beta of chunk s landed before the previous step's closing barrier

        // ---- prep pass 1: raw q, k (zero past the document end), per-row decays, in-block products ----
        uint32_t qp[8], kp[8];     // rows (2j, 2j+1) of this thread's block as packed bf16 pairs
        float a[16], sa[16];
        if (have_intra) {
            const uint8_t *qcol = sm + S::AX + (pc >> 6) * 8192 + (pc & 63) * 2;
            const uint8_t *kcol = qcol + 16384;
#pragma unroll
            for (int j2 = 0; j2 < 8; ++j2) {
                const int r = 16 * pR + 2 * j2;
                const uint32_t q0 = r < L ? *reinterpret_cast<const uint16_t *>(qcol + r * 128) : 0u;
                const uint32_t q1 = r + 1 < L ? *reinterpret_cast<const uint16_t *>(qcol + (r + 1) * 128) : 0u;
                const uint32_t k0 = r < L ? *reinterpret_cast<const uint16_t *>(kcol + r * 128) : 0u;
                const uint32_t k1 = r + 1 < L ? *reinterpret_cast<const uint16_t *>(kcol + (r + 1) * 128) : 0u;
                qp[j2] = q0 | (q1 << 16);
                kp[j2] = k0 | (k1 << 16);
            }
            // a_j = 2^{log2e g_j}; the block's log2 sum; then sa_j = a_{j+1} .. a_15 and, in place,
            // a_j <- a_0 .. a_j (every such product lies in [e^-80, 1])
            const uint8_t *gcol = sm + S::G + (pc >> 5) * 8192 + (pc & 31) * 4;
            float tl = 0.f;
#pragma unroll
            for (int j2 = 0; j2 < 8; ++j2) {
                const int r = 16 * pR + 2 * j2;
                const float g0 = r < L ? *reinterpret_cast<const float *>(gcol + r * 128) : 0.f;
                const float g1 = r + 1 < L ? *reinterpret_cast<const float *>(gcol + (r + 1) * 128) : 0.f;
                const float2 t2 = __fmul2_rn(make_float2(g0, g1), make_float2(kLog2e, kLog2e));
                tl += t2.x;
                tl += t2.y;
                a[2 * j2] = ex2_ftz(t2.x);
                a[2 * j2 + 1] = ex2_ftz(t2.y);
            }
            sa[15] = 1.f;
#pragma unroll
            for (int j = 14; j >= 0; --j) sa[j] = sa[j + 1] * a[j + 1];
#pragma unroll
            for (int j = 1; j < 16; ++j) a[j] *= a[j - 1];
            f_tot[pR * 128 + pc] = tl;
        }
        // the previous step's U product is done: the column-side tile (T_U, T_W), KGT and V are free
        if (tid == 0 && have_state && !tc::mbar_wait(mbar(kMbU), (uint32_t)((s - 1) & 1), kWaitLimit)) *abort_flag = 1;
        // the previous step's output store has read its staging buffer (KDT[buf], rewritten below)
        if (tid == kStateTid0) tc::bulk_wait_read();
        tc::fence_before();
        // raw q, k read (the row-side tile may be written over them); block sums published.  The abort
        // decision is taken by the barrier itself, so that every thread leaves the loop together.
        const bool stop = __syncthreads_or(*abort_flag != 0);
        tc::fence_after();
        if (stop) { aborted = true; break; }
        if (have_intra) {
            // ---- prep pass 2: factors and operand tiles ----
            // log2 sums of the four 16-row blocks of this channel (pR is warp-uniform: no divergence)
            const float t0 = f_tot[pc], t1 = f_tot[128 + pc], t2 = f_tot[256 + pc], t3 = f_tot[384 + pc];
            const float before = pR == 0 ? 0.f : pR == 1 ? t0 : pR == 2 ? t0 + t1 : (t0 + t1) + t2;
            const float after = pR == 3 ? 0.f : pR == 2 ? t3 : pR == 1 ? t2 + t3 : (t1 + t2) + t3;
            const float to47 = pR == 0 ? t1 + t2 : pR == 1 ? t2 : 0.f;
            const float pre = ex2_ftz(before);   // e^{Gamma before this block}
            const float suf = ex2_ftz(after);    // e^{Gamma_63 - Gamma at this block's end}
            const float y1s = ex2_ftz(to47);     // e^{Gamma_47 - Gamma at this block's end} (1 for pR >= 2)
            if (pR == 0) f_dl[buf * 128 + pc] = ex2_ftz(((t0 + t1) + t2) + t3);
            const bool even = (pR & 1) == 0;
            const float2 pre2 = make_float2(pre, pre), suf2 = make_float2(suf, suf), y12 = make_float2(y1s, y1s);
            auto put = [&](int off, const float2 (&x)[4]) { *reinterpret_cast<uint4 *>(sm + off) = pack8x2(x); };
#pragma unroll 1
            for (int hh = 0; hh < 2; ++hh) {
                // rows 8 hh .. 8 hh + 7 sit in entries 0..7 (the upper half is shifted down below)
                const int ch = 2 * pR + hh;   // 16-byte chunk of these 8 rows within a 64-row atom
                // even blocks end at a reference row: X = 1/sa there; odd blocks start right after one:
                // Y = 1/pa there (one reciprocal per element either way)
                float inv[8];
#pragma unroll
                for (int t = 0; t < 8; ++t) inv[t] = rcp_approx(even ? sa[t] : a[t]);
                float2 qv[4], kv[4];   // rows 8 hh .. 8 hh + 7 as fp32 pairs (bf16 widens exactly)
#pragma unroll
                for (int p = 0; p < 4; ++p) {
                    qv[p] = unpack_bf16(qp[p]);
                    kv[p] = unpack_bf16(kp[p]);
                }
                float2 x[4], y[4];
#pragma unroll
                for (int p = 0; p < 4; ++p) {   // row side e^{Gamma_r - Gamma_ref(r)}
                    const int j = 2 * p;
                    const float2 fx = even ? make_float2(inv[2 * p], inv[2 * p + 1]) : make_float2(a[j], a[j + 1]);
                    x[p] = __fmul2_rn(qv[p], fx);
                    y[p] = __fmul2_rn(kv[p], fx);
                }
                put(S::AX + tc::mnmaj_chunk(ch, pc, 128), x);
                put(S::AX + tc::mnmaj_chunk(8 + ch, pc, 128), y);
#pragma unroll
                for (int p = 0; p < 4; ++p) {   // column side e^{Gamma_47 - Gamma_i} and e^{Gamma_15 - Gamma_i}
                    const int j = 2 * p;
                    const float2 sa2 = make_float2(sa[j], sa[j + 1]);
                    const float2 fy1 = pR == 3 ? make_float2(inv[2 * p], inv[2 * p + 1]) : __fmul2_rn(sa2, y12);
                    const float2 fy0 = even ? sa2 : make_float2(inv[2 * p], inv[2 * p + 1]);
                    x[p] = __fmul2_rn(kv[p], fy1);
                    y[p] = __fmul2_rn(kv[p], fy0);
                }
                put(S::BY + tc::mnmaj_chunk(ch, pc, 128), x);
                if (pR < 2) put(S::BY + tc::mnmaj_chunk(8 + ch, pc, 128), y);
                float qt[8];
#pragma unroll
                for (int p = 0; p < 4; ++p) {   // e^{Gamma_r} (K e^Gamma, Q~) and e^{Gamma_63 - Gamma_r} (Kd)
                    const int j = 2 * p;
                    const float2 e = __fmul2_rn(make_float2(a[j], a[j + 1]), pre2);
                    const float2 fd = __fmul2_rn(make_float2(sa[j], sa[j + 1]), suf2);
                    x[p] = __fmul2_rn(kv[p], e);
                    y[p] = __fmul2_rn(kv[p], fd);
                    const float2 qe = __fmul2_rn(qv[p], e);
                    qt[2 * p] = qe.x;
                    qt[2 * p + 1] = qe.y;
                }
                put(S::KGT + tc::kmaj_chunk(pc, ch), x);
                put(S::KDT + buf * 16384 + tc::kmaj_chunk(pc, ch), y);
                uint32_t qr[8];
#pragma unroll
                for (int i = 0; i < 8; ++i) qr[i] = __float_as_uint(qt[i]);
                st8(lane_base + kQT + 16 * pR + 8 * hh, qr);   // lane = channel pc, columns = rows
#pragma unroll
                for (int t = 0; t < 8; ++t) {
                    a[t] = a[t + 8];
                    sa[t] = sa[t + 8];
                }
#pragma unroll
                for (int p = 0; p < 4; ++p) {
                    qp[p] = qp[p + 4];
                    kp[p] = kp[p + 4];
                }
            }
            tc::wait_st();
        }
        // operand tiles written through the generic proxy are read by the tensor core
        tc::fence_proxy_async();
        tc::fence_before();
        __syncthreads();
        tc::fence_after();

        if (warp < 12) {
            // ================= intra (chunk s) =================
            if (have_intra) {
                const float *f_beta = reinterpret_cast<const float *>(sm + S::BETA + buf * 256);
                const float *rk = f_rk + buf * 64;
                // ---- tcgen05: D[128 rows: q | k][96] = X Y^T ----
                if (tid == 0) {
                    constexpr uint32_t idA = tc::idesc_bf16(128, 96, true, true, false);
#pragma unroll
                    for (int kk = 0; kk < 8; ++kk)
                        tc::mma(tmem + kDA, dM128 + (uint64_t)((S::AX + kk * 2048) >> 4),
                                dM128 + (uint64_t)((S::BY + kk * 2048) >> 4), idA, kk > 0);
                    tc::commit(mbar(kMbA));
                }
                if (warp >= 10) {
                    // V is free (the previous U product is done): this chunk's v; the next chunk's beta;
                    // warm L2 with the tiles of the next steps' loads (v of chunk s+1; q, k, g of s+2)
                    if (tid == 320) {
                        issue_v(s);
                        if (have_next) {
                            const int y1 = (int)(doc_start + 64 * (int64_t)(s + 1));
                            tc::tma_prefetch_2d(&maps.v, xq, y1);
                            tc::tma_prefetch_2d(&maps.v, xq + 64, y1);
                        }
                        if (s + 2 < nchunks) {
                            const int y2 = (int)(doc_start + 64 * (int64_t)(s + 2));
                            tc::tma_prefetch_2d(&maps.q, xq, y2);
                            tc::tma_prefetch_2d(&maps.q, xq + 64, y2);
                            tc::tma_prefetch_2d(&maps.k, xq, y2);
                            tc::tma_prefetch_2d(&maps.k, xq + 64, y2);
#pragma unroll
                            for (int b = 0; b < 4; ++b) tc::tma_prefetch_2d(&maps.g, xq + 32 * b, y2);
                        }
                    }
                    if (have_next) load_beta(sm, beta, doc_start + 64 * (int64_t)(s + 1), nL, H, h, buf ^ 1, tid - 320);
                    cp_async_commit();
                }
                if (tid == 0) {
                    if (!tc::mbar_wait(mbar(kMbA), par, kWaitLimit)) *abort_flag = 1;
                    tc::fence_before();
                }
                bar_intra();
                tc::fence_after();
                // the row-side tile has been read: the next chunk's raw q, k
                if (tid == 320 && have_next) {
                    tc::fence_proxy_async();
                    issue_qk(s + 1);
                }
                if (warp >= 8) {
                    // warps 8-11: row norms of chunk s+1, once warps 0-3 are through the solve (its
                    // shared-memory chains are the critical path; the norms are needed only next step)
                    asm volatile("bar.sync 5, %0;" ::"r"(have_state ? 384 : 256) : "memory");
                    if (have_next) {
                        if (lane == 0 && !tc::mbar_wait(mbar(kMbQK), (uint32_t)((s + 1) & 1), kWaitLimit)) *abort_flag = 1;
                        __syncwarp();
                        norms16((warp - 8) * 16, nL, s + 1);
                    }
                } else {
                    // ---- read back L_qk (lanes 0-63) and L_kk (lanes 64-127) ----
                    // lane quarter qd: q rows 0-31 | q rows 32-63 | k rows 0-31 | k rows 32-63; rows of the
                    // first half use columns 64..95 (i < 32), rows of the second half columns 0..63.  Warp
                    // pairs split the columns (hf = 0: the first half of them), read 8 columns at a time.
                    {
                        const int qd = warp & 3, hf = warp >> 2;
                        const int row = 32 * (qd & 1) + lane;
                        const bool second = (qd & 1) != 0;
                        const int nI = second ? 32 : 16;
                        const int i0 = nI * hf;
                        const uint32_t c0 = (second ? 0u : 64u) + (uint32_t)i0;
                        const int R = row >> 4, rr = row & 15;
                        const float br = f_beta[row] * rk[row];
                        uint8_t *aqk = sm + S::AQK + buf * 8192;
#pragma unroll 1
                        for (int g8 = 0; g8 < nI; g8 += 8) {
                            float d[8];
                            tc::ld8(lane_base + kDA + c0 + (uint32_t)g8, d);
                            tc::wait_ld();
                            reg_fence(d);
                            const int ib = i0 + g8;   // first column i of this group
                            if (qd < 2) {
                                // L_qk row, bf16 K-major [r][i], i <= r (no scaling: n rides on the output,
                                // m on U~)
                                float x[8];
#pragma unroll
                                for (int t = 0; t < 8; ++t) x[t] = ib + t <= row ? d[t] : 0.f;
                                *reinterpret_cast<uint4 *>(aqk + tc::kmaj_chunk(row, ib >> 3)) = pack8(x, 1.f);
                            } else {
                                // A_kk[r][i] = beta_r m_r m_i L_kk[r][i] (i < r) into the block (R, i / 16):
                                // off-diagonal blocks row-major, the diagonal block transposed (column j at
                                // j * 20) for the substitution's column reads
                                const int I = ib >> 4, jb = ib & 15;
                                float x[8];
#pragma unroll
                                for (int t = 0; t < 8; ++t) x[t] = d[t] * br * rk[ib + t];
                                if (I < R) {
                                    float *dst = f_akk + pair_of(R, I) * kBlkFloats + rr * kBlkPitch + jb;
                                    *reinterpret_cast<float4 *>(dst) = make_float4(x[0], x[1], x[2], x[3]);
                                    *reinterpret_cast<float4 *>(dst + 4) = make_float4(x[4], x[5], x[6], x[7]);
                                } else if (I == R) {
                                    float *dst = f_akk + pair_of(R, R) * kBlkFloats + jb * kBlkPitch + rr;
#pragma unroll
                                    for (int t = 0; t < 8; ++t) dst[t * kBlkPitch] = jb + t < rr ? x[t] : 0.f;
                                }
                            }
                        }
                        // rows of the first half: L_qk is zero for i >= 32
                        if (qd == 0)
#pragma unroll
                            for (int e = 0; e < 2; ++e)
                                *reinterpret_cast<uint4 *>(aqk + tc::kmaj_chunk(row, 4 + 2 * hf + e)) = make_uint4(0u, 0u, 0u, 0u);
                    }
                    bar_solve();
                    // ---- T = (I + A_kk)^-1, diagonal blocks: lane = column, right-looking substitution:
                    // once x[j] is final, every later row takes its term, x[r] -= A[r][j] x[j] (r > j), with
                    // column j of A (stored transposed) read as float4; the dependent chain is one
                    // multiply-add per row.  T (fp32) is kept for the off-diagonal pass; T_U = diag(m) T
                    // diag(beta) and T_W = T_U diag(m) are written as bf16.
                    if (warp < 4) {
                        if (lane < 16) {
                            const int R = warp, col = lane;
                            const float *blkT = f_akk + pair_of(R, R) * kBlkFloats;
                            float x[16];
#pragma unroll
                            for (int r = 0; r < 16; ++r) x[r] = (r == col) ? 1.f : 0.f;
#pragma unroll
                            for (int j = 0; j < 15; ++j) {
                                const float xj = x[j];
#pragma unroll
                                for (int r4 = (j + 1) & ~3; r4 < 16; r4 += 4) {
                                    const float4 av = *reinterpret_cast<const float4 *>(blkT + j * kBlkPitch + r4);
                                    if (r4 > j) x[r4] -= av.x * xj;
                                    if (r4 + 1 > j) x[r4 + 1] -= av.y * xj;
                                    if (r4 + 2 > j) x[r4 + 2] -= av.z * xj;
                                    if (r4 + 3 > j) x[r4 + 3] -= av.w * xj;
                                }
                            }
                            float *tb = f_tm + pair_of(R, R) * kBlkFloats;
#pragma unroll
                            for (int r = 0; r < 16; ++r) tb[r * kBlkPitch + col] = x[r];
                            const float bc = f_beta[16 * R + col], mc = rk[16 * R + col];
#pragma unroll 1
                            for (int r = 0; r < 16; ++r) {
                                const float tu = tb[r * kBlkPitch + col] * rk[16 * R + r] * bc;
                                const uint32_t o = tc::kmaj_off(16 * R + r, 16 * R + col);
                                *reinterpret_cast<__nv_bfloat16 *>(sm + S::TU + o) = __float2bfloat16_rn(tu);
                                *reinterpret_cast<__nv_bfloat16 *>(sm + S::TW + o) = __float2bfloat16_rn(tu * mc);
                            }
                        }
                    } else {
                        // T_U and T_W are zero above the block diagonal (warps 4-7)
                        const int t = tid - 128;
                        for (int idx = t; idx < 384; idx += 128) {
                            const int tile = idx >= 192 ? 1 : 0, id = idx - 192 * tile;
                            const int b = id >> 5, row = (id & 31) >> 1, half = id & 1;
                            const int R = b < 3 ? 0 : b < 5 ? 1 : 2;
                            const int I = b < 3 ? b + 1 : b < 5 ? b - 1 : 3;
                            *reinterpret_cast<uint4 *>(sm + (tile ? S::TW : S::TU) +
                                                       tc::kmaj_chunk(16 * R + row, 2 * I + half)) = make_uint4(0, 0, 0, 0);
                        }
                    }
                    bar_solve();
                    // ---- off-diagonal blocks of T as a two-level block inverse (tf32 warp MMA) ----
                    // T = [[T_a, 0], [-T_b A_ba T_a, T_b]] with T_a, T_b the 32x32 inverses, each
                    // [[T_00, 0], [-T_11 A_10 T_00, T_11]] at the 16-row level.  Level 32: T_10 and T_32
                    // (warps 0-3, one 16x8 strip each); level 64: the lower-left 32x32 block (warps 0-3,
                    // one 32x8 column strip each).  Accumulators become B fragments (rows tq, tq+4,
                    // 8+tq, 12+tq; column gq) by two shuffles per register.
                    const int src_lo = 4 * tq + (gq >> 1);          // holder of rows tq (and 8+tq), column gq
                    const int src_hi = 4 * (tq + 4) + (gq >> 1);    // holder of rows tq+4 (and 12+tq)
                    const bool odd_col = gq & 1;
                    auto to_bfrag = [&](const float (&c)[4], float (&b)[4]) {
#pragma unroll
                        for (int ks = 0; ks < 2; ++ks) {
                            const float e0 = __shfl_sync(0xffffffffu, c[2 * ks], src_lo);
                            const float o0 = __shfl_sync(0xffffffffu, c[2 * ks + 1], src_lo);
                            const float e1 = __shfl_sync(0xffffffffu, c[2 * ks], src_hi);
                            const float o1 = __shfl_sync(0xffffffffu, c[2 * ks + 1], src_hi);
                            b[2 * ks] = odd_col ? o0 : e0;
                            b[2 * ks + 1] = odd_col ? o1 : e1;
                        }
                    };
                    // B fragment of column strip 8nt..8nt+7 of an fp32 16x16 block
                    auto load_bfrag = [&](const float *blk, int nt, float (&b)[4]) {
                        const float *t = blk + 8 * nt + gq;
                        b[0] = t[tq * kBlkPitch];
                        b[1] = t[(tq + 4) * kBlkPitch];
                        b[2] = t[(8 + tq) * kBlkPitch];
                        b[3] = t[(12 + tq) * kBlkPitch];
                    };
                    // acc += blk (16x16, fp32 A fragment) * b (16x8 B fragment)
                    auto mma16 = [&](float (&acc)[4], const float *blk, const float (&b)[4]) {
#pragma unroll
                        for (int ks = 0; ks < 2; ++ks) {
                            const int k0 = 8 * ks;
                            mma_tf32(acc, blk[gq * kBlkPitch + k0 + tq], blk[(gq + 8) * kBlkPitch + k0 + tq],
                                     blk[gq * kBlkPitch + k0 + tq + 4], blk[(gq + 8) * kBlkPitch + k0 + tq + 4],
                                     b[2 * ks], b[2 * ks + 1]);
                        }
                    };
                    // T_RI strip = -y: T_U = -m_row y beta_col and T_W = T_U m_col, bf16
                    auto store_tp = [&](int R, int I, int nt, const float (&y)[4]) {
                        const int cl = 8 * nt + 2 * tq;
                        const float b0 = f_beta[16 * I + cl], b1 = f_beta[16 * I + cl + 1];
                        const float m0 = rk[16 * I + cl], m1 = rk[16 * I + cl + 1];
#pragma unroll
                        for (int hr = 0; hr < 2; ++hr) {
                            const int r = 16 * R + gq + 8 * hr;
                            const float mr = rk[r];
                            const float u0 = -y[2 * hr] * mr * b0, u1 = -y[2 * hr + 1] * mr * b1;
                            const uint32_t o = tc::kmaj_off(r, 16 * I + cl);
                            *reinterpret_cast<uint32_t *>(sm + S::TU + o) = pack_bf16(u0, u1);
                            *reinterpret_cast<uint32_t *>(sm + S::TW + o) = pack_bf16(u0 * m0, u1 * m1);
                        }
                    };
                    if (warp < 4) {
                        // level 32: T_RI = -T_RR (A_RI T_II), (R, I) = (1, 0) or (3, 2)
                        const int R = warp < 2 ? 1 : 3, I = R - 1, nt = warp & 1;
                        float tb[4], xacc[4] = {0.f, 0.f, 0.f, 0.f}, xb[4], y[4] = {0.f, 0.f, 0.f, 0.f};
                        load_bfrag(f_tm + pair_of(I, I) * kBlkFloats, nt, tb);
                        mma16(xacc, f_akk + pair_of(R, I) * kBlkFloats, tb);
                        to_bfrag(xacc, xb);
                        mma16(y, f_tm + pair_of(R, R) * kBlkFloats, xb);
                        store_tp(R, I, nt, y);
                        float *to = f_tm + pair_of(R, I) * kBlkFloats;
                        const int cl = 8 * nt + 2 * tq;
                        *reinterpret_cast<float2 *>(to + gq * kBlkPitch + cl) = make_float2(-y[0], -y[1]);
                        *reinterpret_cast<float2 *>(to + (gq + 8) * kBlkPitch + cl) = make_float2(-y[2], -y[3]);
                    }
                    bar_solve();
                    if (warp < 4) {
                        // level 64: column strip (I, nt) of rows 32..63:
                        //   X = A_ba T_a[:, strip]:  X_2 = A_20 T_0I + A_21 T_1I,  X_3 = A_30 T_0I + A_31 T_1I
                        //   Y = T_b X:               Y_2 = T_22 X_2,  Y_3 = T_32 X_2 + T_33 X_3;  T_RI = -Y_R
                        const int I = warp >> 1, nt = warp & 1;
                        float t1[4], x2[4] = {0.f, 0.f, 0.f, 0.f}, x3[4] = {0.f, 0.f, 0.f, 0.f};
                        load_bfrag(f_tm + pair_of(1, I) * kBlkFloats, nt, t1);
                        if (I == 0) {
                            float t0[4];
                            load_bfrag(f_tm + pair_of(0, 0) * kBlkFloats, nt, t0);
                            mma16(x2, f_akk + pair_of(2, 0) * kBlkFloats, t0);
                            mma16(x3, f_akk + pair_of(3, 0) * kBlkFloats, t0);
                        }
                        mma16(x2, f_akk + pair_of(2, 1) * kBlkFloats, t1);
                        mma16(x3, f_akk + pair_of(3, 1) * kBlkFloats, t1);
                        float xb2[4], xb3[4], y2[4] = {0.f, 0.f, 0.f, 0.f}, y3[4] = {0.f, 0.f, 0.f, 0.f};
                        to_bfrag(x2, xb2);
                        to_bfrag(x3, xb3);
                        mma16(y2, f_tm + pair_of(2, 2) * kBlkFloats, xb2);
                        mma16(y3, f_tm + pair_of(3, 2) * kBlkFloats, xb2);
                        mma16(y3, f_tm + pair_of(3, 3) * kBlkFloats, xb3);
                        store_tp(2, I, nt, y2);
                        store_tp(3, I, nt, y3);
                        // the solve is through: release the norms (warps 8-11) and the output read-back
                        asm volatile("bar.arrive 5, %0;" ::"r"(have_state ? 384 : 256) : "memory");
                    }
                    tc::fence_proxy_async();   // all of T_U, T_W (diagonal, zeros, off-diagonal) to the tensor core
                    bar_solve();
                    // ---- tcgen05: -W'^T = -(K e^Gamma)^T T_W^T, over the read-back L product ----
                    // the A_kk / T blocks are done with: the next chunk's g lands over them
                    if (tid == 128 && have_next) issue_g(s + 1);
                    if (tid == 0) {
                        tc::fence_after();
                        constexpr uint32_t id_w = tc::idesc_bf16(128, 64, false, false, true);
#pragma unroll
                        for (int kk = 0; kk < 4; ++kk)
                            tc::mma(tmem + kDA, dK + (uint64_t)((S::KGT + kk * 32) >> 4),
                                    dK + (uint64_t)((S::TW + kk * 32) >> 4), id_w, kk > 0);
                        tc::commit(mbar(kMbW));
                    }
                }   // warps 0-7
                if (tid == 0) {
                    bool ok = tc::mbar_wait(mbar(kMbW), par, kWaitLimit);
                    // B2 is free once the previous chunk's state product has read it
                    if (have_state) ok = tc::mbar_wait(mbar(kMb2), (uint32_t)((s - 1) & 1), kWaitLimit) && ok;
                    ok = tc::mbar_wait(mbar(kMbV), par, kWaitLimit) && ok;    // v(s) landed
                    if (!ok) *abort_flag = 1;
                    tc::fence_before();
                }
                bar_intra();
                tc::fence_after();
                if (warp < 8) {
                    // B2 = [-W'^T | Q~^T] (bf16, MN-major [c][n]): warps 0-3 from -W'^T, warps 4-7 from Q~^T
                    const int c = 32 * lq + lane, part = warp >> 2;
                    const uint32_t src = part ? kQT : kDA;
#pragma unroll 1
                    for (int h2 = 0; h2 < 2; ++h2) {
                        float w[32];
                        tc::ld32(lane_base + src + 32 * h2, w);
                        tc::wait_ld();
                        reg_fence(w);
#pragma unroll
                        for (int e = 0; e < 4; ++e)
                            *reinterpret_cast<uint4 *>(sm + S::B2 + tc::mnmaj_chunk(8 * part + 4 * h2 + e, c, 128)) =
                                pack8(w + 8 * e, 1.f);
                    }
                } else if (L < 64) {
                    // rows of v past the document end are zero (the tile may reach the next document)
                    for (int idx = tid - 256; idx < (64 - L) * 16; idx += 128) {
                        const int row = L + (idx >> 4), ch = idx & 15;
                        *reinterpret_cast<uint4 *>(sm + S::V + (ch >> 3) * 8192 + row * 128 + (ch & 7) * 16) =
                            make_uint4(0, 0, 0, 0);
                    }
                }
                tc::fence_proxy_async();
                tc::fence_before();
                bar_intra();
                // ---- tcgen05: U'^T = V^T T_U^T into the state accumulator, once the state side has
                // finished with the previous chunk's U~ and O there ----
                if (warp == 0) {
                    if (have_state) asm volatile("bar.sync 4, 160;" ::: "memory");
                    if (lane == 0) {
                        tc::fence_after();
                        constexpr uint32_t id_u = tc::idesc_bf16(128, 64, true, false, false);
#pragma unroll
                        for (int kk = 0; kk < 4; ++kk)
                            tc::mma(tmem + kDS, dM64 + (uint64_t)((S::V + kk * 2048) >> 4),
                                    dK + (uint64_t)((S::TU + kk * 32) >> 4), id_u, kk > 0);
                        tc::commit(mbar(kMbU));
                    }
                    __syncwarp();
                }
            }
            // the beta rows (issued by warps 10-11) and the g tile of chunk s+1 have landed before the step ends
            cp_async_wait_all();
            if (tid == 256 && have_next && !tc::mbar_wait(mbar(kMbG), (uint32_t)((s + 1) & 1), kWaitLimit))
                *abort_flag = 1;
        } else {
            // ================= state warps (12-15) =================
            if (have_state) {
                // ---- chunk s-1: state update and output ----
                const int n = s - 1, nbuf = n & 1;
                const int64_t ptok0 = doc_start + 64 * (int64_t)n;
                const int pL = chunk_len(n);
                const float *dc = f_dl + nbuf * 128;
                // S^T -> bf16 copy (A operand), then S^T <- S^T Diag(e^{Gamma_63})
                auto sprep = [&](float (&sv)[16], int c0) {
                    uint32_t pk[8];
#pragma unroll
                    for (int i = 0; i < 8; ++i) pk[i] = pack_bf16(sv[2 * i], sv[2 * i + 1]);
                    st8(lane_base + kSB + c0 / 2, pk);
#pragma unroll
                    for (int i = 0; i < 16; i += 4) {
                        const float4 d4 = *reinterpret_cast<const float4 *>(dc + c0 + i);
                        const float2 x = __fmul2_rn(make_float2(sv[i], sv[i + 1]), make_float2(d4.x, d4.y));
                        const float2 y = __fmul2_rn(make_float2(sv[i + 2], sv[i + 3]), make_float2(d4.z, d4.w));
                        sv[i] = x.x; sv[i + 1] = x.y; sv[i + 2] = y.x; sv[i + 3] = y.y;
                    }
                    st16f(lane_base + kSF + c0, sv);
                };
                // two loads in flight: the next 16 columns are read while the current ones are converted;
                // the product's first four k-steps (key channels 0-63) start once their bf16 copy is in
                // place, while the second half is converted
                constexpr uint32_t id2 = tc::idesc_bf16(128, 128, false, true, false);
                auto state_mma = [&](int kk0) {   // [U~^T | (Q~ S)^T] accumulated onto [U'^T | 0]
                    tc::wait_st();
                    tc::fence_before();
                    bar_state();
                    if (tid == kStateTid0) {
                        tc::fence_after();
#pragma unroll
                        for (int kk = kk0; kk < kk0 + 4; ++kk)
                            mma_ts(tmem + kDS, tmem + kSB + 8 * kk, dM128 + (uint64_t)((S::B2 + kk * 2048) >> 4), id2, 1u);
                    }
                };
                {
                    float sa16[16], sb16[16];
                    tc::ld16(lane_base + kSF, sa16);
                    tc::wait_ld();
                    reg_fence(sa16);
                    // the state entering chunk n, S[c][v] fp32, into its checkpoint slot
                    auto ckpt_store = [&](const float (&cur)[16], int c0) {
                        if constexpr (kCkpt) {
                            float *ck = ckpt + ((size_t)(doc_start / 64 + doc + n) * H + h) * (kHeadDim * kHeadDim) +
                                        (size_t)c0 * kHeadDim + 32 * lq + lane;
#pragma unroll
                            for (int i = 0; i < 16; ++i) ck[(size_t)i * kHeadDim] = cur[i];
                        }
                    };
#pragma unroll 1
                    for (int cp = 0; cp < 4; ++cp) {
                        const int c0 = 32 * cp;
                        tc::ld16(lane_base + kSF + c0 + 16, sb16);
                        ckpt_store(sa16, c0);
                        sprep(sa16, c0);
                        tc::wait_ld();
                        reg_fence(sb16);
                        if (cp < 3) tc::ld16(lane_base + kSF + c0 + 32, sa16);
                        ckpt_store(sb16, c0 + 16);
                        sprep(sb16, c0 + 16);
                        if (cp == 1) state_mma(0);   // key channels 0-63 converted
                        if (cp < 3) {
                            tc::wait_ld();
                            reg_fence(sa16);
                        }
                    }
                    state_mma(4);
                    if (tid == kStateTid0) tc::commit(mbar(kMb2));
                }
                if (tid == kStateTid0) {
                    if (!tc::mbar_wait(mbar(kMb2), (uint32_t)(n & 1), kWaitLimit)) *abort_flag = 1;
                    tc::fence_before();
                }
                bar_state();
                tc::fence_after();
                // U~^T (columns 0-63) -> bf16 copy (A operand of the O and state products), over the S^T bf16
                // copy that the state product has finished reading
                {
                    float u[32];
                    uint32_t pk[16];
#pragma unroll 1
                    for (int h2 = 0; h2 < 2; ++h2) {
                        tc::ld32(lane_base + kDS + 32 * h2, u);
                        tc::wait_ld();
                        reg_fence(u);
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
                    // O^T += U~^T L_qk^T (L_qk [r][i] is the K-major B operand), then the state update
                    constexpr uint32_t id_o = tc::idesc_bf16(128, 64, false, false, false);
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk)
                        mma_ts(tmem + kDS + 64, tmem + kUB + 8 * kk,
                               dK + (uint64_t)((S::AQK + kk * 32) >> 4) + (uint64_t)(nbuf * (8192 >> 4)), id_o, 1u);
                    constexpr uint32_t id4 = tc::idesc_bf16(128, 128, false, false, false);
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk)
                        mma_ts(tmem + kSF, tmem + kUB + 8 * kk,
                               dK + (uint64_t)((S::KDT + kk * 32) >> 4) + (uint64_t)(nbuf * (16384 >> 4)), id4, 1u);
                    tc::commit(mbar(kMb4));
                    // the output tile is staged in Kd's buffer, which the state update reads
                    if (!tc::mbar_wait(mbar(kMb4), (uint32_t)(n & 1), kWaitLimit)) *abort_flag = 1;
                    tc::fence_before();
                }
                bar_state();
                tc::fence_after();
                // wait until the intra warps are through the UT solve (its latency-bound chains are the
                // step's critical path; the output has slack until the next U product)
                if (have_intra) asm volatile("bar.sync 5, 384;" ::: "memory");
                // O^T (columns 64-127): lane v holds O[r][v]; o = (scale / |q_r|) O, taken eight rows at a
                // time.  Each thread writes its column v of every row (lanes = consecutive v, so one store
                // instruction covers a contiguous run of a row).
                {
                    const int vcol = 32 * lq + lane;
                    const float *rq = f_rq + (n & 3) * 64;
                    if (pL == 64) {
                        // whole chunk: stage o[r][v] as bf16 in Kd's buffer (free now, rewritten only by the
                        // next step's prep; two 64-channel boxes, 128-B swizzled rows) and write it with one
                        // TMA store per box
                        const uint32_t vb = (uint32_t)(vcol & 63) * 2;          // byte of v in its row
                        const uint32_t stage_off = S::KDT + (uint32_t)nbuf * 16384u;
                        uint8_t *stage = sm + stage_off + (vcol >> 6) * 8192;
#pragma unroll 1
                        for (int r0 = 0; r0 < 64; r0 += 8) {
                            float o[8];
                            tc::ld8(lane_base + kDS + 64 + (uint32_t)r0, o);
                            tc::wait_ld();
                            reg_fence(o);
                            const float4 ra = *reinterpret_cast<const float4 *>(rq + r0);
                            const float4 rb = *reinterpret_cast<const float4 *>(rq + r0 + 4);
                            const float sc[8] = {ra.x, ra.y, ra.z, ra.w, rb.x, rb.y, rb.z, rb.w};
#pragma unroll
                            for (int i = 0; i < 8; ++i) {
                                const int r = r0 + i;
                                const uint32_t off = (uint32_t)r * 128u + ((((vb >> 4) ^ (uint32_t)(r & 7)) << 4) | (vb & 15u));
                                *reinterpret_cast<__nv_bfloat16 *>(stage + off) = __float2bfloat16_rn(o[i] * sc[i]);
                            }
                        }
                        tc::fence_proxy_async();
                        bar_state();
                        if (tid == kStateTid0) {
                            tc::tma_store_2d(&maps.o, xq, (int)ptok0, sbase + stage_off);
                            tc::tma_store_2d(&maps.o, xq + 64, (int)ptok0, sbase + stage_off + 8192);
                            tc::bulk_commit();   // its reads of the staging buffer are awaited in the next step
                        }
                    } else {
                        // partial chunk: rows past the document end belong to the next document, so
                        // store the valid rows directly
#pragma unroll 1
                        for (int r0 = 0; r0 < 64; r0 += 8) {
                            float o[8];
                            tc::ld8(lane_base + kDS + 64 + (uint32_t)r0, o);
                            tc::wait_ld();
                            reg_fence(o);
#pragma unroll
                            for (int i = 0; i < 8; ++i) {
                                const int r = r0 + i;
                                if (r < pL)
                                    reinterpret_cast<__nv_bfloat16 *>(out)[((ptok0 + r) * H + h) * kHeadDim + vcol] =
                                        __float2bfloat16_rn(o[i] * rq[r]);
                            }
                        }
                    }
                    // the O columns start the next chunk's state product from zero
                    float z[32];
#pragma unroll
                    for (int i = 0; i < 32; ++i) z[i] = 0.f;
                    tc::st32(lane_base + kDS + 64, z);
                    tc::st32(lane_base + kDS + 96, z);
                    tc::wait_st();
                }
                // U~ and O have been read: the state accumulator is free for the next U product
                tc::fence_before();
                if (have_intra) asm volatile("bar.arrive 4, 160;" ::: "memory");
            }
        }
        tc::fence_before();
        const bool stop_end = __syncthreads_or(*abort_flag != 0);
        tc::fence_after();
        if (stop_end) { aborted = true; break; }
    }

    // ---- final state: ht[c][v] = S^T[v][c] (the last state update has completed) ----
    if (!aborted && ht && warp >= 12) {
        const int vcol = 32 * lq + lane;
#pragma unroll 1
        for (int c0 = 0; c0 < 128; c0 += 32) {
            float z[32];
            tc::ld32(lane_base + kSF + c0, z);
            tc::wait_ld();
#pragma unroll
            for (int i = 0; i < 32; ++i) ht[state_off + (size_t)(c0 + i) * kHeadDim + vcol] = z[i];
        }
    }

    // ---- teardown ----
    cp_async_wait_all();
    if (tid == kStateTid0) tc::bulk_wait();   // output tiles written before shared memory goes away
    if (aborted) {
        if (tid == 0) atomicExch(status, kStatusTimeout);
        // let any tensor-core work or copy still in flight land before TMEM and shared memory go away
        for (int i = 0; i < kNumMbar; ++i) {
            tc::mbar_wait(mbar(i), 0u, kWaitLimit / 16);
            tc::mbar_wait(mbar(i), 1u, kWaitLimit / 16);
        }
    }
    tc::fence_before();
    __syncthreads();
    tc::fence_after();
    if (warp == 0) tc::dealloc(tmem, kTmemCols);
}

// ---- host: TMA descriptors ----
PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    });
    return fn;
}

// 2-D map over a [rows, cols] row-major tensor (cols contiguous), box [box_rows, box_cols]
bool make_map(CUtensorMap *m, const void *base, CUtensorMapDataType dt, int elem_bytes, uint64_t rows, uint64_t cols,
              uint32_t box_rows, uint32_t box_cols, CUtensorMapSwizzle swz) {
    auto fn = encode_fn();
    if (!fn) return false;
    cuuint64_t dims[2] = {cols, rows};
    cuuint64_t strides[1] = {cols * (cuuint64_t)elem_bytes};
    cuuint32_t box[2] = {box_cols, box_rows};
    cuuint32_t estr[2] = {1, 1};
    return fn(m, dt, 2, const_cast<void *>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, swz,
              CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace pipe_path

cudaError_t launch_fwd_pipe(const uint16_t *q, const uint16_t *k, const uint16_t *v, const float *g,
                            const float *beta, const int32_t *cu, int n_docs, int64_t T, int H, const float *h0,
                            float *ht, uint16_t *out, int *status, cudaStream_t stream, float *ckpt) {
    using namespace pipe_path;
    Maps maps;
    const uint64_t cols = (uint64_t)H * kHeadDim;
    if (!make_map(&maps.q, q, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, (uint64_t)T, cols, 64, 64, CU_TENSOR_MAP_SWIZZLE_NONE) ||
        !make_map(&maps.k, k, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, (uint64_t)T, cols, 64, 64, CU_TENSOR_MAP_SWIZZLE_NONE) ||
        !make_map(&maps.g, g, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, (uint64_t)T, cols, 64, 32, CU_TENSOR_MAP_SWIZZLE_NONE) ||
        !make_map(&maps.v, v, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, (uint64_t)T, cols, 64, 64, CU_TENSOR_MAP_SWIZZLE_128B) ||
        !make_map(&maps.o, out, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, (uint64_t)T, cols, 64, 64, CU_TENSOR_MAP_SWIZZLE_128B))
        return cudaErrorInvalidValue;
    constexpr int bytes = Smem::ALLOC;
    auto kernel = ckpt ? kda_fwd_pipe_kernel<true> : kda_fwd_pipe_kernel<false>;
    cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
    if (e != cudaSuccess) return e;
    const int64_t blocks = (int64_t)n_docs * H;
    kernel<<<(unsigned)blocks, kThreads, bytes, stream>>>(maps, g, beta, cu, n_docs, T, H, h0, ht, ckpt, out, status);
    return cudaGetLastError();
}

}  // namespace kda
