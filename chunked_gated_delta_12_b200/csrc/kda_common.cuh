// kda_common.cuh -- small device helpers shared by the libkda kernels:
// shared-memory tile addressing (XOR-swizzled 16-byte chunks), cp.async with
// zero fill, ldmatrix, warp-level bf16 MMA, bf16 packing, exp2.
#pragma once

#include <cuda_bf16.h>
#include <stdint.h>

namespace kda {

constexpr int kHeadDim = 128;   // K = V = 128
constexpr int kChunk = 64;      // tokens per chunk
constexpr float kLog2e = 1.4426950408889634f;

// ---------------------------------------------------------------------------
// Swizzled shared-memory tiles.  Rows are `pitch` bytes (a multiple of 128);
// the 16-byte chunk index inside a row is XORed with (row & 7), so 8
// consecutive rows read at the same logical column land in 8 distinct
// 16-byte bank groups (conflict-free ldmatrix and row-strided accesses).
// ---------------------------------------------------------------------------
__device__ __forceinline__ uint32_t swz_chunk(int row, int chunk16, int pitch) {
    return (uint32_t)(row * pitch + ((chunk16 ^ (row & 7)) << 4));
}
// bf16 element (row, col)
__device__ __forceinline__ uint32_t swz_bf16(int row, int col, int pitch) {
    return swz_chunk(row, col >> 3, pitch) + (uint32_t)((col & 7) << 1);
}
// fp32 element (row, col)
__device__ __forceinline__ uint32_t swz_f32(int row, int col, int pitch) {
    return swz_chunk(row, col >> 2, pitch) + (uint32_t)((col & 3) << 2);
}

__device__ __forceinline__ uint32_t smem_u32(const void *p) {
    return (uint32_t)__cvta_generic_to_shared(p);
}

// 16-byte async copy global -> shared; src_bytes < 16 zero-fills the rest
// (src_bytes == 0 reads nothing and writes 16 zero bytes).
__device__ __forceinline__ void cp_async16(uint32_t dst, const void *src, int src_bytes) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;\n" ::"r"(dst), "l"(src),
                 "r"(src_bytes)
                 : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;\n" ::: "memory"); }
__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_group 0;\n" ::: "memory"); }

// ---------------------------------------------------------------------------
// ldmatrix / mma.sync (m16n8k16, bf16 inputs, fp32 accumulate)
// ---------------------------------------------------------------------------
__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t &r0, uint32_t &r1, uint32_t &r2,
                                        uint32_t &r3) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];\n"
                 : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
                 : "r"(addr));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t &r0, uint32_t &r1, uint32_t &r2,
                                          uint32_t &r3) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];\n"
                 : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
                 : "r"(addr));
}
__device__ __forceinline__ void ldsm_x2_t(uint32_t addr, uint32_t &r0, uint32_t &r1) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x2.trans.shared.b16 {%0,%1}, [%2];\n"
                 : "=r"(r0), "=r"(r1)
                 : "r"(addr));
}
__device__ __forceinline__ void ldsm_x2(uint32_t addr, uint32_t &r0, uint32_t &r1) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x2.shared.b16 {%0,%1}, [%2];\n"
                 : "=r"(r0), "=r"(r1)
                 : "r"(addr));
}

// D += A * B, A 16x16 (4 regs), B 16x8 (2 regs), D 16x8 fp32 (4 regs)
__device__ __forceinline__ void mma_bf16(float (&d)[4], const uint32_t (&a)[4], uint32_t b0,
                                         uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
        "{%8,%9}, {%0,%1,%2,%3};\n"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
    __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t *>(&h);
}
__device__ __forceinline__ float2 unpack_bf16(uint32_t u) {
    __nv_bfloat162 h = *reinterpret_cast<__nv_bfloat162 *>(&u);
    return __bfloat1622float2(h);
}

// 2^x through the SFU (CUDA's exp2f intrinsic path).
__device__ __forceinline__ float fast_exp2(float x) { return exp2f(x); }
// 2^x by the hardware approximation (PTX ex2.approx.ftz): results below 2^-126 flush to zero,
// which only drops decay factors that are negligible anyway (every exponent here is <= 0)
__device__ __forceinline__ float ex2_ftz(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}
// Longest-first document order for grids of one CTA per (document, head), CTA b covering
// (document doc_at_rank(b / H), head b % H).  The hardware starts CTAs in index order, so the
// longest chains start in the first wave and the short ones fill the tail (list scheduling in
// decreasing order).  Ranks documents by (length descending, index ascending), a permutation for
// any cu_seqlens content; with more than kLongestFirstMaxDocs documents the order is the identity.
// Every thread of the CTA must call it (it holds a CTA barrier); `scratch` is n_docs + 2 ints of
// shared memory that the caller does not use yet.
constexpr int kLongestFirstMaxDocs = 256;
__device__ __forceinline__ int doc_at_rank(const int32_t *cu, int n_docs, int rank, int *scratch) {
    if (n_docs <= 1 || n_docs > kLongestFirstMaxDocs) return rank;
    for (int i = threadIdx.x; i <= n_docs; i += blockDim.x) scratch[1 + i] = cu[i];
    __syncthreads();
    for (int d = threadIdx.x; d < n_docs; d += blockDim.x) {
        const int len = scratch[2 + d] - scratch[1 + d];
        int r = 0;
        for (int e = 0; e < n_docs; ++e) {
            const int le = scratch[2 + e] - scratch[1 + e];
            r += (le > len) || (le == len && e < d);
        }
        if (r == rank) scratch[0] = d;
    }
    __syncthreads();
    const int doc = scratch[0];
    __syncthreads();   // scratch may be reused by the caller
    return doc;
}

// bf16 bit pattern -> fp32 (exact)
__device__ __forceinline__ float bf16_bits_to_float(uint16_t b) { return __uint_as_float((uint32_t)b << 16); }

}  // namespace kda
