// kda_fwd_pipe.cu -- pipelined fused chunk-KDA forward (one CTA per (document, head),
// all 128 value columns); kda_chunk_fwd launches it for every call.
//
// Two chunks are in flight per CTA.  In step s all 16 warps first prepare chunk
// s; then warps 0-11 finish chunk s's intra-chunk work while warps 12-15 run
// chunk s-1's state update on the tensor cores and the row norms of chunk s+1.
// The state is kept transposed, S^T[v][c] in fp32 in tensor memory (lane =
// value column v), so that both the bf16 copy of the state and the corrected
// values U~ are tcgen05 A operands read straight from TMEM.
//
// Per chunk (rows r, i; Gamma = in-chunk cumsum of g):
//   A_kk[r,i] = beta_r k^_r.(k^_i e^{Gamma_r - Gamma_i}) (i < r),  A_qk (i <= r)
//   T' = (I + A_kk)^-1 diag(beta)
//   W  = T' K^e^Gamma,  U = T' V,  U~ = U - W S
//   O  = Q^e^Gamma S + A_qk U~
//   S <- Diag(e^{Gamma_last}) S + (K^ e^{Gamma_last - Gamma})^T U~
// and on the tensor cores (M = 128 everywhere):
//   intra  D[:, 0:64] = -(K^e^Gamma)^T T'^T = -W^T, next to Q~^T (written by the prep)
//          -> B2 = [-W^T | Q~^T] (bf16, shared);  then D[:, 0:64] = V^T T'^T = U^T
//   state  D   += S^T_bf16 (TMEM) B2                -> [U~^T | (Q~ S)^T]
//          O^T += U~^T_bf16 (TMEM) A_qk^T
//          S^T += U~^T_bf16 (TMEM) Kd               (after S^T <- S^T Diag(e^{Gamma_last}))
// The output scale is carried by Q~ and A_qk.
// q, k, g and v tiles arrive by TMA (2-D tensor maps over [T, H*128], each CTA loading its own
// tiles).  A tile may reach into the next document, so the rows past the document end are zeroed
// in shared memory (q, k and g when the step starts, v before the U product) and count as zero
// in the row norms.  The gate exponent is split at 16-row sub-block boundaries
// (e^{G_r - G_i} = E1_r s_RI E2_i, every factor within the fp32/bf16 range).  Every wait is
// time-limited and reports KDA_ERR_TIMEOUT.
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
// The backward's checkpoint block per chunk and head (bytes): S^T and U~^T (bf16, stored as column
// groups of 16 (S^T) or 32 (U~^T) values per row v, rows v consecutive inside a group, so that a
// warp's stores cover whole contiguous pieces), the chunk's tensor-core operands [-W^T | Q~^T] (B2)
// and Kd^T, A_qk, T = (I + A_kk)^-1 and A_hat (bf16, A_hat without beta and valid below the diagonal
// only), and e^{Gamma_last} (fp32)
constexpr size_t kCkS = 0, kCkU = 32768, kCkB2 = 49152, kCkKD = 81920, kCkAQ = 98304, kCkT = 106496,
                 kCkAH = 114688, kCkDL = 122880, kCkptBytes = 123904;
constexpr int kStateTid0 = 384;               // first thread of warps 12-15
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kSF = 0;                   // S^T fp32          [128 lanes v][128 cols c]
constexpr uint32_t kSB = 128;                 // S^T bf16 packed   [128][64]
constexpr uint32_t kD0 = 192;                 // chunk accumulators, two buffers of 128 columns
constexpr uint32_t kUB = 448;                 // U~^T bf16 packed  [128][32]
constexpr long long kWaitLimit = 2000000000LL;
// kernel modes (what a CTA's token range is) and the segment-table state slot encoding
constexpr int kDocs = 0, kSegs = 1, kTransition = 2;
constexpr int kSlotCaller = kSplitSlotCaller;

// A_kk / T as ten 16x16 fp32 blocks (I <= R), rows padded to 20 floats
constexpr int kBlkPitch = 20;
constexpr int kBlkFloats = 16 * kBlkPitch;

struct Smem {
    static constexpr int Q = 0;            // raw q: two TMA boxes [64 rows][64 ch] (128 B rows) -> q^E1 [c][r] SW128
    static constexpr int K = 16384;        // raw k                                                -> k^E1 [c][r] SW128
    static constexpr int G = 32768;        // raw g: four TMA boxes [64 rows][32 ch] fp32
    static constexpr int V = 65536;        // raw v: two TMA boxes, 128B-swizzled = MN-major SW128 atoms
    static constexpr int KR = 81920;       // k^E2 [c][r] SW128 -> T' (rows 0-63) and the A_qk staging tile
    static constexpr int KGT = 98304;      // (k^ e^Gamma)^T, K-major [c][r]
    static constexpr int KDT = 114688;     // two buffers: (k^ e^{Gamma_last-Gamma})^T, K-major [c][r]
    static constexpr int B2 = 147456;      // [-W^T | Q'^T], MN-major [c][n], two 64-wide atoms
    static constexpr int AQK = 180224;     // two buffers: A_qk [r][i], K-major (64 rows), read by the state side
    static constexpr int AKK = 196608;     // A_kk blocks fp32
    static constexpr int TM = AKK + 10 * kBlkFloats * 4;   // T blocks fp32
    static constexpr int SMALL = TM + 10 * kBlkFloats * 4;
    static constexpr int BETA = SMALL;               // fp32 [2][64]
    static constexpr int RQ = BETA + 512;            // fp32 [64]
    static constexpr int RK = RQ + 256;              // fp32 [64]
    static constexpr int TOT = RK + 256;             // fp32 [4][128]
    static constexpr int PS = TOT + 2048;            // bf16 [10][128] pair scales
    static constexpr int DC = PS + 2560;             // fp32 [2][128]
    static constexpr int MBAR = DC + 1024;           // u64 [16]
    static constexpr int TBASE = MBAR + 128;
    static constexpr int ABORT = TBASE + 16;
    static constexpr int HTP = ABORT + 16;           // this chain's final-state pointer (read after the loop)
    static constexpr int BYTES = HTP + 16;
    static constexpr int ALLOC = BYTES + 1024;
};
static_assert(Smem::ALLOC <= 232448, "shared memory budget");

// every barrier completes by tcgen05.commit or by TMA transaction bytes
enum Mbar { kMbWQ = 0, kMbU, kMb2, kMb4, kMbQK, kMbG, kMbV, kNumMbar };

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
// eight values held as four row pairs, as bf16 (optionally scaled by a packed multiply)
__device__ __forceinline__ uint4 pack8x2(const float2 *x) {
    return make_uint4(pack_bf16(x[0].x, x[0].y), pack_bf16(x[1].x, x[1].y), pack_bf16(x[2].x, x[2].y),
                      pack_bf16(x[3].x, x[3].y));
}
__device__ __forceinline__ uint4 pack8x2s(const float2 *x, float2 s) {
    const float2 a = __fmul2_rn(x[0], s), b = __fmul2_rn(x[1], s), c = __fmul2_rn(x[2], s), d = __fmul2_rn(x[3], s);
    return make_uint4(pack_bf16(a.x, a.y), pack_bf16(b.x, b.y), pack_bf16(c.x, c.y), pack_bf16(d.x, d.y));
}
// registers filled by tcgen05.ld are valid only after tcgen05.wait::ld: this empty asm, placed after
// the wait, keeps the compiler from moving their first use above it
template <int N>
__device__ __forceinline__ void reg_fence(float (&v)[N]) {
#pragma unroll
    for (int i = 0; i < N; ++i) asm volatile("" : "+f"(v[i]));
}
__device__ __forceinline__ int pair_R(int p) { return p >= 6 ? 3 : p >= 3 ? 2 : p >= 1 ? 1 : 0; }
// bulk copy shared -> global (16-byte aligned, size a multiple of 16), tracked by the issuing thread's bulk group
__device__ __forceinline__ void bulk_store(void *gdst, uint32_t ssrc, uint32_t bytes) {
    asm volatile("cp.async.bulk.global.shared::cta.bulk_group [%0], [%1], %2;" ::"l"(gdst), "r"(ssrc), "r"(bytes)
                 : "memory");
}
__device__ __forceinline__ int pair_of(int R, int I) { return R * (R + 1) / 2 + I; }

// beta rows [tok0, tok0 + L) of head h, one row per calling thread (row in [0, 64); rows >= L zero-filled)
__device__ __forceinline__ void load_beta(uint8_t *sm, const float *beta, int64_t tok0, int L, int H, int h, int buf,
                                          int row) {
    {
        const bool ok = row < L;
        const float *src = ok ? beta + (tok0 + row) * H + h : beta;
        asm volatile("cp.async.ca.shared.global [%0], [%1], 4, %2;\n" ::"r"(
                         smem_u32(sm + Smem::BETA + buf * 256 + row * 4)),
                     "l"(src), "r"(ok ? 4 : 0)
                     : "memory");
    }
}

struct Maps {
    CUtensorMap q, k, g, v, o;
};

// kCkpt: the backward's forward pass: store, per chunk and head, the checkpoint block described at
// kCkS..kCkptBytes into `ckpt` (the state entering the chunk, U~ and the chunk's operand tiles), and
// form no output (neither O nor the (Q~ S)^T half of the state product); a separate instance, so that
// the plain forward carries no trace of it.
// kMode: what a CTA's token range is -- kDocs: document blockIdx.x / H of cu_seqlens (every plain
// forward); kSegs: entry blockIdx.x / H of a segment table built on the device (a document cut into
// pieces, see kda_split.cu), outputs written; kTransition: the same with v taken as zero, the
// identity as the entering state and no outputs (a segment's transition map M, its final state).
template <bool kCkpt, int kMode>
__global__ void __launch_bounds__(kThreads, 1)
    kda_fwd_pipe_kernel(const __grid_constant__ Maps maps, const float *__restrict__ beta,
                        const int32_t *__restrict__ cu_seqlens, int n_docs, int64_t T, int H,
                        const float *h0, float *ht, uint16_t *ckpt, uint16_t *__restrict__ out,
                        int *__restrict__ status, const int4 *__restrict__ seg, const int *__restrict__ seg_count,
                        float *ws_states) {
    using S = Smem;
    extern __shared__ __align__(1024) uint8_t sm_raw[];
    // align by offsetting the shared array itself, so every access stays in the shared window (LDS/STS)
    uint8_t *sm = sm_raw + (((smem_u32(sm_raw) + 1023u) & ~1023u) - smem_u32(sm_raw));

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int gq = lane >> 2, tq = lane & 3;
    const int h = blockIdx.x % H;
    int doc = 0;
    int64_t doc_start, doc_end;
    // initial / final state of this chain, [128 key channels][128 value columns] fp32, or NULL
    const float *h0p = nullptr;
    float *htp = nullptr;
    if constexpr (kMode == kDocs) {
        // CTA -> (document, head), longest documents first; the Q tile area is free until the first TMA load
        doc = doc_at_rank(cu_seqlens, n_docs, blockIdx.x / H, reinterpret_cast<int *>(sm));
        if (blockIdx.x == 0 && tid == 0) {
            if (cu_seqlens[0] != 0 || (int64_t)cu_seqlens[n_docs] != T) atomicExch(status, kStatusBadSeqlens);
        }
        doc_start = cu_seqlens[doc];
        doc_end = cu_seqlens[doc + 1];
        const size_t state_off = ((size_t)doc * H + h) * kHeadDim * kHeadDim;   // [n_docs * H] states
        if (h0) h0p = h0 + state_off;
        if (ht) htp = ht + state_off;
    } else {
        // CTA -> (table entry, head); entries past the count written by the planner have no work
        const int rank = blockIdx.x / H;
        if (rank >= *seg_count) return;
        const int4 e = seg[rank];
        doc_start = e.x;
        doc_end = e.y;
        auto slot = [&](int sl, const float *caller) -> const float * {
            if (sl < 0) return nullptr;
            if (sl < kSlotCaller) return ws_states + ((size_t)sl * H + h) * kHeadDim * kHeadDim;
            return caller ? caller + ((size_t)(sl - kSlotCaller) * H + h) * kHeadDim * kHeadDim : nullptr;
        };
        if constexpr (kMode == kSegs) h0p = slot(e.z, h0);
        htp = const_cast<float *>(slot(e.w, ht));
    }
    if (doc_start < 0 || doc_end < doc_start || doc_end > T) {
        if (tid == 0) atomicExch(status, kStatusBadSeqlens);
        return;
    }
    if (doc_end == doc_start) {
        // nothing to process: the final state is the initial one
        if (htp)
            for (int idx = tid; idx < kHeadDim * kHeadDim; idx += kThreads)
                htp[idx] = h0p ? h0p[idx] : (kMode == kTransition && idx / kHeadDim == idx % kHeadDim ? 1.f : 0.f);
        return;
    }
    const int nchunks = (int)((doc_end - doc_start + 63) / 64);
    // barrier waits poll in the plain forward and park the thread in the segment passes (measured)
    constexpr bool kSuspendWaits = kMode != kDocs;
    // the checkpoint block of chunk i of this chain (kCkpt)
    auto ck_block = [&](int i) -> uint8_t * {
        return reinterpret_cast<uint8_t *>(ckpt) + ((size_t)(doc_start / 64 + doc + i) * H + h) * kCkptBytes;
    };
    auto chunk_len = [&](int i) -> int {
        const int64_t rem = doc_end - (doc_start + 64 * (int64_t)i);
        return rem <= 0 ? 0 : (rem < 64 ? (int)rem : 64);
    };

    float *f_rq = reinterpret_cast<float *>(sm + S::RQ);
    float *f_rk = reinterpret_cast<float *>(sm + S::RK);
    float *f_tot = reinterpret_cast<float *>(sm + S::TOT);
    __nv_bfloat16 *f_ps = reinterpret_cast<__nv_bfloat16 *>(sm + S::PS);
    float *f_akk = reinterpret_cast<float *>(sm + S::AKK);
    float *f_tm = reinterpret_cast<float *>(sm + S::TM);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(sm + S::ABORT);
    const uint32_t mb = smem_u32(sm + S::MBAR);
    auto mbar = [&](int i) -> uint32_t { return mb + 8u * (uint32_t)i; };
    const uint32_t sbase = smem_u32(sm);
    // UMMA shared-memory descriptors of the tile area; every operand descriptor is one of these plus the
    // tile's byte offset / 16 (addresses stay below 256 KB, so the 14-bit field cannot carry).  Built
    // once, so that issuing a product is a 64-bit add per instruction.
    const uint64_t dK = tc::sdesc(sbase, 16u, 1024u);            // K-major, 128-byte swizzled rows
    const uint64_t dM128 = tc::sdesc(sbase, 128u * 128u, 1024u); // MN-major, 128 K rows per 64-wide atom
    const uint64_t dM64 = tc::sdesc(sbase, 64u * 128u, 1024u);   // MN-major, 64 K rows per 64-wide atom
    const int xq = h * kHeadDim;          // TMA x coordinate of this head's channel 0

    auto issue_qk = [&](int i) {          // q, k tiles of chunk i (one thread)
        const int y = (int)(doc_start + 64 * (int64_t)i);
        tc::mbar_expect_tx(mbar(kMbQK), 32768u);
        tc::tma_load_2d(sbase + S::Q, &maps.q, xq, y, mbar(kMbQK));
        tc::tma_load_2d(sbase + S::Q + 8192, &maps.q, xq + 64, y, mbar(kMbQK));
        tc::tma_load_2d(sbase + S::K, &maps.k, xq, y, mbar(kMbQK));
        tc::tma_load_2d(sbase + S::K + 8192, &maps.k, xq + 64, y, mbar(kMbQK));
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
    // 1/|q_r| and 1/|k_r| for rows r0..r0+15 of the raw tiles (rows >= Li count as zero).
    // Each lane sums its 4 channels for all 32 (tensor, row) pairs, then a transposed
    // butterfly (31 shuffles) leaves lane l with the total of pair l.
    auto norms16 = [&](int r0, int Li) {
        float v[32];
#pragma unroll
        for (int i = 0; i < 16; ++i) {
            const int r = r0 + i;
            const uint32_t off = (lane >> 4) * 8192 + r * 128 + (lane & 15) * 8;
            uint2 qa = *reinterpret_cast<const uint2 *>(sm + S::Q + off);
            uint2 ka = *reinterpret_cast<const uint2 *>(sm + S::K + off);
            if (r >= Li) qa = ka = make_uint2(0u, 0u);
            const float2 q01 = unpack_bf16(qa.x), q23 = unpack_bf16(qa.y);
            const float2 k01 = unpack_bf16(ka.x), k23 = unpack_bf16(ka.y);
            v[i] = q01.x * q01.x + q01.y * q01.y + q23.x * q23.x + q23.y * q23.y;
            v[16 + i] = k01.x * k01.x + k01.y * k01.y + k23.x * k23.x + k23.y * k23.y;
        }
#pragma unroll
        for (int lv = 0; lv < 5; ++lv) {
            const int o = 16 >> lv, half = 16 >> lv;
            const bool up = (lane & o) != 0;
#pragma unroll
            for (int j = 0; j < half; ++j) {
                const float send = up ? v[j] : v[j + half];
                const float keep = up ? v[j + half] : v[j];
                v[j] = keep + __shfl_xor_sync(0xffffffffu, send, o);
            }
        }
        float *dst = lane < 16 ? f_rq : f_rk;
        dst[r0 + (lane & 15)] = rsqrtf(v[0] + 1e-6f);
    };

    // ---- setup ----
    // the final-state pointer waits in shared memory until after the loop (one register pair less there)
    if (tid == 0) *reinterpret_cast<float **>(sm + S::HTP) = htp;
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
        // S^T[v][c] (lane v) = h0[c][v], or zero (the identity for a transition pass)
        const int vcol = 32 * lq + lane;
#pragma unroll 1
        for (int c0 = 0; c0 < 128; c0 += 32) {
            float z[32];
#pragma unroll
            for (int i = 0; i < 32; ++i)
                z[i] = kMode == kTransition ? (c0 + i == vcol ? 1.f : 0.f)
                                            : (h0p ? h0p[(size_t)(c0 + i) * kHeadDim + vcol] : 0.f);
            tc::st32(lane_base + kSF + c0, z);
        }
        tc::wait_st();
    }
    // chunk 0's inputs (one thread polls the barriers; the CTA barrier releases the rest), then its norms
    cp_async_wait_all();
    if (tid == 0) {
        bool ok = tc::mbar_wait<kSuspendWaits>(mbar(kMbQK), 0u, kWaitLimit);
        ok = tc::mbar_wait<kSuspendWaits>(mbar(kMbG), 0u, kWaitLimit) && ok;
        if (!ok) *abort_flag = 1;
    }
    __syncthreads();
    if (warp < 4) norms16(warp * 16, chunk_len(0));
    tc::fence_before();
    __syncthreads();
    tc::fence_after();

    bool aborted = *abort_flag != 0;
    const float out_scale = rsqrtf((float)kHeadDim);

    for (int s = 0; s <= nchunks && !aborted; ++s) {
        const bool have_intra = s < nchunks;        // chunk s: prep + intra
        const bool have_state = s >= 1;             // chunk s-1: state update + output
        const bool have_next = s + 1 < nchunks;     // chunk s+1 exists
        const int L = chunk_len(s);
        const int nL = chunk_len(s + 1);
        const int buf = s & 1;
        const uint32_t par = (uint32_t)(s & 1);

        // beta(s), q, k and g of chunk s landed before the previous step's closing barrier

        // a partial last chunk: rows past the document end (the TMA tile reaches into the next
        // document) are zeroed, so the prep below needs no per-element masks
        if (have_intra && L < 64) {
            for (int idx = tid; idx < (64 - L) * 16; idx += kThreads) {
                const int row = L + (idx >> 4), ch = idx & 15;             // 16 chunks of 16 B per row
                const uint32_t o = (uint32_t)row * 128u + (uint32_t)(ch & 7) * 16u;
                const uint4 z = make_uint4(0, 0, 0, 0);
                *reinterpret_cast<uint4 *>(sm + S::Q + (ch >> 3) * 8192 + o) = z;
                *reinterpret_cast<uint4 *>(sm + S::K + (ch >> 3) * 8192 + o) = z;
                *reinterpret_cast<uint4 *>(sm + S::G + (ch >> 3) * 16384 + o) = z;
                *reinterpret_cast<uint4 *>(sm + S::G + (ch >> 3) * 16384 + 8192 + o) = z;
            }
            __syncthreads();
        }
        float2 ql[8], kl[8], kr[8];      // row pairs (2j, 2j+1) of this thread's 16-row block
        float lg0 = 0.f;
        const int pc = tid & 127, pR = tid >> 7;
        if (have_intra) {
            // ---- prep pass 1: thread = (channel c, row block R) ----
            // per-row decays a_j = 2^{log2e g_j} (one exp2 each); E1 and E2 are running products
            // inside the 16-row block: E1_j = a_1..a_j, E2_j = a_{j+1}..a_15 (both in [e^-75, 1])
            float2 a[8];
            float gsum = 0.f;
            const uint8_t *gcol = sm + S::G + (pc >> 5) * 8192 + (pc & 31) * 4;
#pragma unroll
            for (int j2 = 0; j2 < 8; ++j2) {
                const int r = 16 * pR + 2 * j2;
                const float g0 = *reinterpret_cast<const float *>(gcol + r * 128);
                const float g1 = *reinterpret_cast<const float *>(gcol + (r + 1) * 128);
                gsum += g0;
                gsum += g1;
                const float2 gl2 = __fmul2_rn(make_float2(g0, g1), make_float2(kLog2e, kLog2e));   // log2-scaled
                if (j2 == 0) lg0 = gl2.x;
                a[j2] = make_float2(ex2_ftz(gl2.x), ex2_ftz(gl2.y));
            }
            f_tot[pR * 128 + pc] = gsum * kLog2e;
            float2 e1[8], e2[8];
            e1[0] = make_float2(1.f, a[0].y);
#pragma unroll
            for (int j2 = 1; j2 < 8; ++j2) {
                e1[j2].x = e1[j2 - 1].y * a[j2].x;
                e1[j2].y = e1[j2].x * a[j2].y;
            }
            e2[7] = make_float2(a[7].y, 1.f);
#pragma unroll
            for (int j2 = 6; j2 >= 0; --j2) {
                e2[j2].y = e2[j2 + 1].x * a[j2 + 1].x;
                e2[j2].x = e2[j2].y * a[j2].y;
            }
            const uint8_t *qcol = sm + S::Q + (pc >> 6) * 8192 + (pc & 63) * 2;
            const uint8_t *kcol = sm + S::K + (pc >> 6) * 8192 + (pc & 63) * 2;
#pragma unroll
            for (int j4 = 0; j4 < 4; ++j4) {
                const float4 rq4 = *reinterpret_cast<const float4 *>(f_rq + 16 * pR + 4 * j4);
                const float4 rk4 = *reinterpret_cast<const float4 *>(f_rk + 16 * pR + 4 * j4);
#pragma unroll
                for (int h2 = 0; h2 < 2; ++h2) {
                    const int j2 = 2 * j4 + h2, r = 16 * pR + 2 * j2;
                    const float2 qv = make_float2(bf16_bits_to_float(*reinterpret_cast<const uint16_t *>(qcol + r * 128)),
                                                  bf16_bits_to_float(*reinterpret_cast<const uint16_t *>(qcol + (r + 1) * 128)));
                    const float2 kv = make_float2(bf16_bits_to_float(*reinterpret_cast<const uint16_t *>(kcol + r * 128)),
                                                  bf16_bits_to_float(*reinterpret_cast<const uint16_t *>(kcol + (r + 1) * 128)));
                    const float2 qh = __fmul2_rn(qv, h2 ? make_float2(rq4.z, rq4.w) : make_float2(rq4.x, rq4.y));
                    const float2 kh = __fmul2_rn(kv, h2 ? make_float2(rk4.z, rk4.w) : make_float2(rk4.x, rk4.y));
                    ql[j2] = __fmul2_rn(qh, e1[j2]);
                    kl[j2] = __fmul2_rn(kh, e1[j2]);
                    kr[j2] = __fmul2_rn(kh, e2[j2]);
                }
            }
        }
        // the previous step's U product is done: V, KR and its accumulator are free
        if (tid == 0 && have_state && !tc::mbar_wait<kSuspendWaits>(mbar(kMbU), (uint32_t)((s - 1) & 1), kWaitLimit)) *abort_flag = 1;
        // the previous step's output store has read its staging buffer (Kd's buffer, rewritten below)
        if (tid == kStateTid0) tc::bulk_wait_read();
        tc::fence_before();
        // raw q, k, g read; block sums published.  The abort decision is taken by the barrier itself, so
        // that every thread leaves the loop together.
        const bool stop = __syncthreads_or(*abort_flag != 0);
        tc::fence_after();
        if (stop) { aborted = true; break; }
        if (have_intra) {
            // ---- prep pass 2 (log2-scaled Gamma) ----
            float offs[5];
            offs[0] = 0.f;
#pragma unroll
            for (int R = 0; R < 4; ++R) offs[R + 1] = offs[R] + f_tot[R * 128 + pc];
            const float gm = offs[pR] + lg0;
            const float ge = offs[pR + 1];
            const float gl = offs[4];
            const float P = ex2_ftz(gm);
            const float2 Pq = make_float2(P * out_scale, P * out_scale);   // the output scale rides on Q~ and A_qk
            // Q~ into TMEM first (lane c, columns 64+16R..), next to -W^T of the W product
            {
                float qtf[16];
#pragma unroll
                for (int j2 = 0; j2 < 8; ++j2) {
                    const float2 t = __fmul2_rn(ql[j2], Pq);
                    qtf[2 * j2] = t.x;
                    qtf[2 * j2 + 1] = t.y;
                }
                const uint32_t dcol = kD0 + 128 * (uint32_t)buf;
                st16f(lane_base + dcol + 64 + 16 * pR, qtf);
            }
            const float2 P2 = make_float2(P, P);
            const float Dkv = ex2_ftz(gl - ge);
            const float2 Dk = make_float2(Dkv, Dkv);
#pragma unroll
            for (int I = 0; I < 4; ++I)
                if (I <= pR) f_ps[pair_of(pR, I) * 128 + pc] = __float2bfloat16_rn(ex2_ftz(gm - offs[I + 1]));
            if (pR == 0) reinterpret_cast<float *>(sm + S::DC)[buf * 128 + pc] = ex2_ftz(gl);
#pragma unroll
            for (int half = 0; half < 2; ++half) {
                const int j0 = half * 4;
                const uint32_t off = tc::kmaj_chunk(pc, 2 * pR + half);
                *reinterpret_cast<uint4 *>(sm + S::Q + off) = pack8x2(ql + j0);
                *reinterpret_cast<uint4 *>(sm + S::K + off) = pack8x2(kl + j0);
                *reinterpret_cast<uint4 *>(sm + S::KR + off) = pack8x2(kr + j0);
                *reinterpret_cast<uint4 *>(sm + S::KGT + off) = pack8x2s(kl + j0, P2);
                *reinterpret_cast<uint4 *>(sm + S::KDT + buf * 16384 + off) = pack8x2s(kr + j0, Dk);
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
                // ---- A_kk and A_qk, one 16x16 block pair per warp ----
                const int aqk = S::AQK + buf * 8192;      // A_qk(s); the other buffer holds A_qk(s-1)
                if (warp < 10) {
                    const int p = warp;
                    const int R = pair_R(p), I = p - R * (R + 1) / 2;
                    const uint32_t kbase = sbase + S::K, qbase = sbase + S::Q, rbase = sbase + S::KR;
                    const __nv_bfloat16 *ps = f_ps + p * 128;
                    float ak[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
                    float aq[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
                    const int j = lane >> 3;
                    // the pair scale of this thread's fragment channels, as bf16x2, for all 8 k-steps
                    __nv_bfloat162 hs[8][2];
#pragma unroll
                    for (int kk = 0; kk < 8; ++kk) {
                        const int cb = kk * 16 + 2 * tq;
                        hs[kk][0] = *reinterpret_cast<const __nv_bfloat162 *>(ps + cb);
                        hs[kk][1] = *reinterpret_cast<const __nv_bfloat162 *>(ps + cb + 8);
                    }
#pragma unroll
                    for (int kk = 0; kk < 8; ++kk) {
                        const uint32_t aoff = tc::kmaj_chunk(16 * kk + (lane & 7) + 8 * (j >> 1), 2 * R + (j & 1));
                        uint32_t fk[4], fq[4], b0, b1, b2, b3;
                        ldsm_x4_t(kbase + aoff, fk[0], fk[1], fk[2], fk[3]);
                        ldsm_x4_t(qbase + aoff, fq[0], fq[1], fq[2], fq[3]);
                        ldsm_x4_t(rbase + tc::kmaj_chunk(16 * kk + (lane & 7) + 8 * (j & 1), 2 * I + (j >> 1)), b0, b1,
                                  b2, b3);
#pragma unroll
                        for (int e = 0; e < 4; ++e) {
                            const __nv_bfloat162 sc = hs[kk][e >> 1];
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
                            if constexpr (kCkpt)
                                *reinterpret_cast<uint32_t *>(ck_block(s) + kCkAH + tc::kmaj_off(row, col)) =
                                    pack_bf16(col < row ? ak[nt][2 * hh] : 0.f, col + 1 < row ? ak[nt][2 * hh + 1] : 0.f);
                            const float y0 = col <= row ? aq[nt][2 * hh] * out_scale : 0.f;
                            const float y1 = col + 1 <= row ? aq[nt][2 * hh + 1] * out_scale : 0.f;
                            *reinterpret_cast<uint32_t *>(sm + aqk + tc::kmaj_off(row, col)) = pack_bf16(y0, y1);
                        }
                } else {
                    // warps 10-11 have no A_kk block: raw g and the beta(s+1) buffer are free (prep pass 1
                    // is done) and so is V (the previous U product is done): the next chunk's g and
                    // beta, this chunk's v
                    if (tid == 320) {
                        tc::fence_proxy_async();
                        if (have_next) issue_g(s + 1);
                        if constexpr (kMode != kTransition) issue_v(s);
                        // warm L2 with the tiles of the next steps' loads (v of chunk s+1; q, k, g of s+2)
                        if (kMode != kTransition && have_next) {
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
                    // A_qk is zero above the block diagonal
                    for (int idx = tid - 320; idx < 192; idx += 64) {
                        const int b = idx >> 5, row = (idx & 31) >> 1, half = idx & 1;
                        const int R = b < 3 ? 0 : b < 5 ? 1 : 2;
                        const int I = b < 3 ? b + 1 : b < 5 ? b - 1 : 3;
                        *reinterpret_cast<uint4 *>(sm + aqk + tc::kmaj_chunk(16 * R + row, 2 * I + half)) =
                            make_uint4(0, 0, 0, 0);
                    }
                }
                bar_intra();
                // the state side's tcgen05 product waits for the warp-level A_kk products to finish
                if (have_state && warp == 0) asm volatile("bar.arrive 4, 160;" ::: "memory");
                // q^E1 / k^E1 consumed: the next chunk's raw q, k
                if (tid == 320 && have_next) {
                    tc::fence_proxy_async();
                    issue_qk(s + 1);
                }
                const uint32_t dcol = kD0 + 128 * (uint32_t)buf;
                // warps 8-11: row norms of chunk s+1 while warps 0-7 solve for T (they rejoin at the
                // barrier before the W readback)
                if (warp >= 8) {
                    if (have_next) {
                        if (lane == 0 && !tc::mbar_wait<kSuspendWaits>(mbar(kMbQK), (uint32_t)((s + 1) & 1), kWaitLimit)) *abort_flag = 1;
                        __syncwarp();
                        norms16((warp - 8) * 16, nL);
                    }
                } else {
                    // ---- T = (I + A_kk)^-1, diagonal blocks: lane = column, left-looking substitution
                    // x[r] = delta_rc - sum_{j<r} A[r][j] x[j] with the rows of A read as float4.
                    // T (fp32) is kept for the off-diagonal pass, T' = T diag(beta) is written as bf16.
                    if (warp < 4) {
                        if (lane < 16) {
                            const int R = warp, col = lane;
                            const float *blk = f_akk + pair_of(R, R) * kBlkFloats;
                            float x[16];
    #pragma unroll
                            for (int r = 0; r < 16; ++r) {
                                float acc = (r == col) ? 1.f : 0.f;
    #pragma unroll
                                for (int j4 = 0; j4 < r; j4 += 4) {
                                    const float4 a = *reinterpret_cast<const float4 *>(blk + r * kBlkPitch + j4);
                                    acc -= a.x * x[j4];
                                    if (j4 + 1 < r) acc -= a.y * x[j4 + 1];
                                    if (j4 + 2 < r) acc -= a.z * x[j4 + 2];
                                    if (j4 + 3 < r) acc -= a.w * x[j4 + 3];
                                }
                                x[r] = acc;
                            }
                            float *tb = f_tm + pair_of(R, R) * kBlkFloats;
                            const float bc = f_beta[16 * R + col];
    #pragma unroll
                            for (int r = 0; r < 16; ++r) {
                                tb[r * kBlkPitch + col] = x[r];
                                if constexpr (kCkpt)
                                    *reinterpret_cast<__nv_bfloat16 *>(ck_block(s) + kCkT + tc::kmaj_off(16 * R + r, 16 * R + col)) =
                                        __float2bfloat16_rn(x[r]);
                                const __nv_bfloat16 t1 = __float2bfloat16_rn(x[r] * bc);
                                *reinterpret_cast<__nv_bfloat16 *>(sm + S::KR + tc::kmaj_off(16 * R + r, 16 * R + col)) = t1;
                            }
                        }
                    } else {
                        // T' is zero above the block diagonal (warps 4-7)
                        const int t = tid - 128;
                        for (int idx = t; idx < 192; idx += 128) {
                            const int b = idx >> 5, row = (idx & 31) >> 1, half = idx & 1;
                            const int R = b < 3 ? 0 : b < 5 ? 1 : 2;
                            const int I = b < 3 ? b + 1 : b < 5 ? b - 1 : 3;
                            *reinterpret_cast<uint4 *>(sm + S::KR + tc::kmaj_chunk(16 * R + row, 2 * I + half)) =
                                make_uint4(0, 0, 0, 0);
                            if constexpr (kCkpt)
                                *reinterpret_cast<uint4 *>(ck_block(s) + kCkT + tc::kmaj_chunk(16 * R + row, 2 * I + half)) =
                                    make_uint4(0, 0, 0, 0);
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
                    // T'_RI strip = -y diag(beta), bf16, into the B operand of the W and U products
                    auto store_tp = [&](int R, int I, int nt, const float (&y)[4]) {
                        const int cl = 8 * nt + 2 * tq;
                        const float b0 = f_beta[16 * I + cl], b1 = f_beta[16 * I + cl + 1];
                        *reinterpret_cast<uint32_t *>(sm + S::KR + tc::kmaj_off(16 * R + gq, 16 * I + cl)) =
                            pack_bf16(-y[0] * b0, -y[1] * b1);
                        *reinterpret_cast<uint32_t *>(sm + S::KR + tc::kmaj_off(16 * R + gq + 8, 16 * I + cl)) =
                            pack_bf16(-y[2] * b0, -y[3] * b1);
                        if constexpr (kCkpt) {
                            uint8_t *tt = ck_block(s) + kCkT;
                            *reinterpret_cast<uint32_t *>(tt + tc::kmaj_off(16 * R + gq, 16 * I + cl)) = pack_bf16(-y[0], -y[1]);
                            *reinterpret_cast<uint32_t *>(tt + tc::kmaj_off(16 * R + gq + 8, 16 * I + cl)) =
                                pack_bf16(-y[2], -y[3]);
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
                    }
                    tc::fence_proxy_async();   // all of T' (diagonal, zeros, off-diagonal) to the tensor core
                    bar_solve();
                    // T' is complete: the W product can start now
                    if (tid == 0) {
                        tc::fence_after();
                        constexpr uint32_t id_w = tc::idesc_bf16(128, 64, false, false, true);
    #pragma unroll
                        for (int kk = 0; kk < 4; ++kk)
                            tc::mma(tmem + dcol, dK + (uint64_t)((S::KGT + kk * 32) >> 4), dK + (uint64_t)((S::KR + kk * 32) >> 4), id_w,
                                    kk > 0);
                        tc::commit(mbar(kMbWQ));
                    }
                }   // warps 0-7
                if (tid == 0) {
                    if constexpr (kCkpt) tc::bulk_wait_read();   // the previous chunk's B2 copy has read it
                    bool ok = tc::mbar_wait<kSuspendWaits>(mbar(kMbWQ), par, kWaitLimit);
                    // B2 is free once the previous chunk's state product has read it
                    if (have_state) ok = tc::mbar_wait<kSuspendWaits>(mbar(kMb2), (uint32_t)((s - 1) & 1), kWaitLimit) && ok;
                    if constexpr (kMode != kTransition) ok = tc::mbar_wait<kSuspendWaits>(mbar(kMbV), par, kWaitLimit) && ok;   // v(s) landed
                    if (!ok) *abort_flag = 1;
                    tc::fence_before();
                }
                bar_intra();
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
                    if (cg == 1 || kMode == kTransition) {
                        // Q~ has been read: zero its columns, so that the state product can accumulate
                        // [U~^T | (Q~ S)^T] onto [U^T | 0] with one N = 128 instruction per k-step.  With
                        // v = 0 (a transition pass) U = 0 too, and -W^T's columns are zeroed instead of
                        // running the U product.
                        float z[32];
#pragma unroll
                        for (int i = 0; i < 32; ++i) z[i] = 0.f;
                        tc::st32(lane_base + dcol + 64 * cg, z);
                        tc::st32(lane_base + dcol + 64 * cg + 32, z);
                        tc::wait_st();
                    }
                } else if (kMode != kTransition && L < 64) {
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
                // ---- tcgen05: D[:, 0:64] = V^T T'^T = U^T ----
                if (tid == 0) {
                    tc::fence_after();
                    if constexpr (kCkpt) {
                        // [-W^T | Q~^T] and A_qk of chunk s, complete now, to its checkpoint block
                        bulk_store(ck_block(s) + kCkB2, sbase + S::B2, 32768);
                        bulk_store(ck_block(s) + kCkAQ, sbase + S::AQK + buf * 8192, 8192);
                        tc::bulk_commit();
                    }
                    if constexpr (kMode != kTransition) {
                        constexpr uint32_t id_u = tc::idesc_bf16(128, 64, true, false, false);
#pragma unroll
                        for (int kk = 0; kk < 4; ++kk)
                            tc::mma(tmem + dcol, dM64 + (uint64_t)((S::V + kk * 2048) >> 4),
                                    dK + (uint64_t)((S::KR + kk * 32) >> 4), id_u, kk > 0);
                    }
                    // (with no product issued the commit tracks the W product alone: the step's tensor
                    // work is done when it arrives)
                    tc::commit(mbar(kMbU));
                }
            }
            // the beta rows of chunk s+1 (issued by warps 10-11) have landed before the step ends
            cp_async_wait_all();
        } else {
            // ================= state warps (12-15) =================
            if (have_state) {
                // ---- chunk s-1: state update and output ----
                const int n = s - 1, nbuf = n & 1;
                const int64_t ptok0 = doc_start + 64 * (int64_t)n;
                const int pL = chunk_len(n);
                const uint32_t dcol = kD0 + 128 * (uint32_t)nbuf;
                const float *dc = reinterpret_cast<const float *>(sm + S::DC) + nbuf * 128;
                if constexpr (kCkpt) {
                    // Kd^T and e^{Gamma_last} of chunk n to its checkpoint block (bulk copies, read-awaited
                    // before this step's output is staged in Kd's buffer)
                    if (tid == kStateTid0) {
                        bulk_store(ck_block(n) + kCkKD, sbase + S::KDT + nbuf * 16384, 16384);
                        bulk_store(ck_block(n) + kCkDL, sbase + S::DC + nbuf * 512, 512);
                        tc::bulk_commit();
                    }
                }
                // S^T -> bf16 copy (A operand), then S^T <- S^T Diag(e^{Gamma_last})
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
                // two loads in flight: the next 32 columns are read while the current ones are converted;
                // the product's first four k-steps (key channels 0-63) start once their bf16 copy is in
                // place, while the second half is converted
                // (the backward's checkpoint pass has no output: its state product needs U~ alone)
                constexpr uint32_t id2 = tc::idesc_bf16(128, kCkpt ? 64 : 128, false, true, false);
                auto state_mma = [&](int kk0) {   // [U~^T | (Q~ S)^T] accumulated onto [U^T | 0]
                    if (kk0 == 0 && have_intra) asm volatile("bar.sync 4, 160;" ::: "memory");
                    tc::wait_st();
                    tc::fence_before();
                    bar_state();
                    if (tid == kStateTid0) {
                        tc::fence_after();
#pragma unroll
                        for (int kk = kk0; kk < kk0 + 4; ++kk)
                            mma_ts(tmem + dcol, tmem + kSB + 8 * kk, dM128 + (uint64_t)((S::B2 + kk * 2048) >> 4), id2, 1u);
                    }
                };
                {
                    float sa[16], sb[16];
                    tc::ld16(lane_base + kSF, sa);
                    tc::wait_ld();
                    reg_fence(sa);
#pragma unroll
                    for (int ch = 0; ch < 8; ++ch) {
                        float(&cur)[16] = (ch & 1) ? sb : sa;
                        float(&nxt)[16] = (ch & 1) ? sa : sb;
                        if (ch < 7) tc::ld16(lane_base + kSF + 16 * (ch + 1), nxt);
                        if constexpr (kCkpt) {
                            // the state entering chunk n into its checkpoint slot: row v of S^T, channels
                            // 16ch..16ch+15 as bf16, in column group ch
                            const int vrow = 32 * lq + lane;
                            uint8_t *ck = ck_block(n) + kCkS + (size_t)ch * (128 * 32) + (size_t)vrow * 32;
                            *reinterpret_cast<uint4 *>(ck) = pack8(cur, 1.f);
                            *reinterpret_cast<uint4 *>(ck + 16) = pack8(cur + 8, 1.f);
                        }
                        sprep(cur, 16 * ch);
                        if (ch == 3) state_mma(0);
                        if (ch < 7) {
                            tc::wait_ld();
                            reg_fence(nxt);
                        }
                    }
                    state_mma(4);
                    if (tid == kStateTid0) tc::commit(mbar(kMb2));
                }
                if (tid == kStateTid0) {
                    if (!tc::mbar_wait<kSuspendWaits>(mbar(kMb2), (uint32_t)(n & 1), kWaitLimit)) *abort_flag = 1;
                    tc::fence_before();
                }
                bar_state();
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
                        if constexpr (kCkpt) {
                            // U~^T row v, s = 32 h2 .. 32 h2 + 31 (column group h2), after the chunk's S^T
                            const int vrow = 32 * lq + lane;
                            uint8_t *cu8 = ck_block(n) + kCkU + (size_t)h2 * (128 * 64) + (size_t)vrow * 64;
#pragma unroll
                            for (int e = 0; e < 4; ++e)
                                *reinterpret_cast<uint4 *>(cu8 + 16 * e) =
                                    make_uint4(pk[4 * e], pk[4 * e + 1], pk[4 * e + 2], pk[4 * e + 3]);
                        }
                    }
                    tc::wait_st();
                }
                tc::fence_before();
                bar_state();
                if (tid == kStateTid0) {
                    tc::fence_after();
                    // O^T += U~^T A_qk^T (A_qk [r][i] is the K-major B operand), then the state update
                    if constexpr (!kCkpt) {
                        constexpr uint32_t id_o = tc::idesc_bf16(128, 64, false, false, false);
#pragma unroll
                        for (int kk = 0; kk < 4; ++kk)
                            mma_ts(tmem + dcol + 64, tmem + kUB + 8 * kk,
                                   dK + (uint64_t)((S::AQK + kk * 32) >> 4) + (uint64_t)(nbuf * (8192 >> 4)), id_o,
                                   1u);
                    }
                    constexpr uint32_t id4 = tc::idesc_bf16(128, 128, false, false, false);
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk)
                        mma_ts(tmem + kSF, tmem + kUB + 8 * kk,
                               dK + (uint64_t)((S::KDT + kk * 32) >> 4) + (uint64_t)(nbuf * (16384 >> 4)), id4, 1u);
                    tc::commit(mbar(kMb4));
                    // the output tile is staged in Kd's buffer, which the state update reads
                    if (!tc::mbar_wait<kSuspendWaits>(mbar(kMb4), (uint32_t)(n & 1), kWaitLimit)) *abort_flag = 1;
                    if constexpr (kCkpt) tc::bulk_wait_read();   // and the checkpoint copy of Kd^T
                    tc::fence_before();
                }
                bar_state();
                tc::fence_after();
                // O^T (columns 64-127; the output scale is already applied): lane v holds o[r][v].
                // Lane pairs swap values so that each thread writes the pair (v, v+1) of one row.  (A
                // transition pass and the backward's checkpoint pass have no output.)
                if constexpr (kMode != kTransition && !kCkpt) {
                    const int vcol = 32 * lq + lane;
                    const bool odd = lane & 1;
                    if (pL == 64) {
                        // whole chunk: stage o[r][v] as bf16 in Kd's buffer (free now, rewritten only by the
                        // next step's prep; two 64-channel boxes, 128-B swizzled rows) and write it with one
                        // TMA store per box.  Even lanes take rows with
                        // (r & 4) == 0, odd lanes the row 4 below, so one store instruction covers 32 banks.
                        const uint32_t vb = (uint32_t)(vcol & 62) * 2;          // byte of the pair in its row
                        const uint32_t stage_off = S::KDT + (uint32_t)nbuf * 16384u;
                        uint8_t *stage = sm + stage_off + (vcol >> 6) * 8192;
#pragma unroll
                        for (int h2 = 0; h2 < 2; ++h2) {
                            float o[32];
                            tc::ld32(lane_base + dcol + 64 + 32 * h2, o);
                            tc::wait_ld();
#pragma unroll
                            for (int i = 0; i < 16; ++i) {
                                const int ja = (i & 3) + 8 * (i >> 2), jb = ja + 4;
                                const float send = odd ? o[ja] : o[jb];
                                const float recv = __shfl_xor_sync(0xffffffffu, send, 1);
                                const float lo = odd ? recv : o[ja];
                                const float hi = odd ? o[jb] : recv;
                                const int r = 32 * h2 + (odd ? jb : ja);
                                const uint32_t off = (uint32_t)r * 128u + ((((vb >> 4) ^ (uint32_t)(r & 7)) << 4) | (vb & 15u));
                                *reinterpret_cast<uint32_t *>(stage + off) = pack_bf16(lo, hi);
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
#pragma unroll
                        for (int h2 = 0; h2 < 2; ++h2) {
                            float o[32];
                            tc::ld32(lane_base + dcol + 64 + 32 * h2, o);
                            tc::wait_ld();
                            // even lanes store rows 32h2 + [0,16), odd lanes rows 32h2 + [16,32)
#pragma unroll
                            for (int i = 0; i < 16; ++i) {
                                const float mine_for_partner = odd ? o[i] : o[16 + i];
                                const float from_partner = __shfl_xor_sync(0xffffffffu, mine_for_partner, 1);
                                const int r = 32 * h2 + (odd ? 16 + i : i);
                                const float lo = odd ? from_partner : o[i];
                                const float hi = odd ? o[16 + i] : from_partner;
                                if (r < pL) {
                                    uint32_t *dst = reinterpret_cast<uint32_t *>(
                                        out + ((ptok0 + r) * H + h) * kHeadDim + (vcol & ~1));
                                    *dst = pack_bf16(lo, hi);
                                }
                            }
                        }
                    }
                }
            }
            // the raw q, k and g of chunk s+1 have landed before the step ends
            if (tid == kStateTid0 && have_next) {
                bool ok = tc::mbar_wait<kSuspendWaits>(mbar(kMbQK), (uint32_t)((s + 1) & 1), kWaitLimit);
                ok = tc::mbar_wait<kSuspendWaits>(mbar(kMbG), (uint32_t)((s + 1) & 1), kWaitLimit) && ok;
                if (!ok) *abort_flag = 1;
            }
        }
        tc::fence_before();
        const bool stop_end = __syncthreads_or(*abort_flag != 0);
        tc::fence_after();
        if (stop_end) { aborted = true; break; }
    }

    // ---- final state: ht[c][v] = S^T[v][c] (the last state update has completed) ----
    htp = *reinterpret_cast<float *volatile *>(sm + S::HTP);
    if (!aborted && htp && warp >= 12) {
        const int vcol = 32 * lq + lane;
#pragma unroll 1
        for (int c0 = 0; c0 < 128; c0 += 32) {
            float z[32];
            tc::ld32(lane_base + kSF + c0, z);
            tc::wait_ld();
#pragma unroll
            for (int i = 0; i < 32; ++i) htp[(size_t)(c0 + i) * kHeadDim + vcol] = z[i];
        }
    }

    // ---- teardown ----
    cp_async_wait_all();
    if (tid == kStateTid0) tc::bulk_wait();   // output tiles written before shared memory goes away
    if constexpr (kCkpt)
        if (tid == 0) tc::bulk_wait();       // and the checkpoint copies
    if (aborted) {
        if (tid == 0) atomicExch(status, kStatusTimeout);
        // let any tensor-core work or copy still in flight land before TMEM and shared memory go away
        for (int i = 0; i < kNumMbar; ++i) {
            tc::mbar_wait<kSuspendWaits>(mbar(i), 0u, kWaitLimit / 16);
            tc::mbar_wait<kSuspendWaits>(mbar(i), 1u, kWaitLimit / 16);
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

namespace {

// TMA maps of one launch; `v` and `out` may be NULL for a transition pass (never loaded or stored:
// their maps are then built over q, only to have a valid descriptor)
bool make_maps(pipe_path::Maps &maps, const uint16_t *q, const uint16_t *k, const uint16_t *v, const float *g,
               uint16_t *out, int64_t T, int H) {
    using namespace pipe_path;
    const uint64_t cols = (uint64_t)H * kHeadDim;
    const void *vb = v ? static_cast<const void *>(v) : q;
    const void *ob = out ? static_cast<const void *>(out) : q;
    return make_map(&maps.q, q, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, (uint64_t)T, cols, 64, 64, CU_TENSOR_MAP_SWIZZLE_NONE) &&
           make_map(&maps.k, k, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, (uint64_t)T, cols, 64, 64, CU_TENSOR_MAP_SWIZZLE_NONE) &&
           make_map(&maps.g, g, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, (uint64_t)T, cols, 64, 32, CU_TENSOR_MAP_SWIZZLE_NONE) &&
           make_map(&maps.v, vb, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, (uint64_t)T, cols, 64, 64, CU_TENSOR_MAP_SWIZZLE_128B) &&
           make_map(&maps.o, ob, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, (uint64_t)T, cols, 64, 64, CU_TENSOR_MAP_SWIZZLE_128B);
}

template <bool kCkpt, int kMode>
cudaError_t launch_mode(const pipe_path::Maps &maps, const float *beta, const int32_t *cu, int n_docs, int64_t T,
                        int H, const float *h0, float *ht, uint16_t *ckpt, uint16_t *out, int *status, const int4 *seg,
                        const int *seg_count, float *ws_states, int64_t ctas, cudaStream_t stream) {
    using namespace pipe_path;
    constexpr int bytes = Smem::ALLOC;
    auto kernel = kda_fwd_pipe_kernel<kCkpt, kMode>;
    cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
    if (e != cudaSuccess) return e;
    kernel<<<(unsigned)ctas, kThreads, bytes, stream>>>(maps, beta, cu, n_docs, T, H, h0, ht, ckpt, out, status, seg,
                                                          seg_count, ws_states);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_fwd_pipe(const uint16_t *q, const uint16_t *k, const uint16_t *v, const float *g,
                            const float *beta, const int32_t *cu, int n_docs, int64_t T, int H, const float *h0,
                            float *ht, uint16_t *out, int *status, cudaStream_t stream, uint16_t *ckpt) {
    using namespace pipe_path;
    Maps maps;
    if (!make_maps(maps, q, k, v, g, out, T, H)) return cudaErrorInvalidValue;
    const int64_t ctas = (int64_t)n_docs * H;
    return ckpt ? launch_mode<true, kDocs>(maps, beta, cu, n_docs, T, H, h0, ht, ckpt, out, status, nullptr, nullptr,
                                           nullptr, ctas, stream)
                : launch_mode<false, kDocs>(maps, beta, cu, n_docs, T, H, h0, ht, nullptr, out, status, nullptr,
                                            nullptr, nullptr, ctas, stream);
}

cudaError_t launch_fwd_segments(bool transition, const uint16_t *q, const uint16_t *k, const uint16_t *v,
                                const float *g, const float *beta, int64_t T, int H, const int4 *seg,
                                const int *seg_count, int max_segs, const float *h0, float *ht, float *ws_states,
                                uint16_t *out, int *status, cudaStream_t stream) {
    using namespace pipe_path;
    if (max_segs <= 0) return cudaSuccess;
    Maps maps;
    if (!make_maps(maps, q, k, transition ? nullptr : v, g, transition ? nullptr : out, T, H))
        return cudaErrorInvalidValue;
    const int64_t ctas = (int64_t)max_segs * H;
    return transition ? launch_mode<false, kTransition>(maps, beta, nullptr, 0, T, H, nullptr, ht, nullptr, nullptr,
                                                        status, seg, seg_count, ws_states, ctas, stream)
                      : launch_mode<false, kSegs>(maps, beta, nullptr, 0, T, H, h0, ht, nullptr, out, status, seg,
                                                  seg_count, ws_states, ctas, stream);
}

}  // namespace kda
