// kda_internal.h -- launchers shared between the libkda kernel files and its C ABI.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace kda {

// Device status codes written by kernels (same values as kda_status).
constexpr int kStatusBadSeqlens = 6;
constexpr int kStatusTimeout = 5;

// Pipelined fused forward: one CTA per (document, head) covering all 128 value
// columns, two chunks in flight (intra-chunk work of chunk s overlapped with the
// state update of chunk s-1).
// h0 / ht: optional initial / final states, [n_docs * H][128][128] fp32 (NULL: zero / not written).
// ckpt: optional, receives per chunk a 123904-byte block in slot (cu[d] / 64 + d + j) * H + h for chunk j
// of document d (the backward's checkpoint layout, kda_fwd_pipe.cu): the state entering the chunk S^T[v][c]
// and its U~^T[v][s] (bf16, column groups of 16 and 32 values per row), the operand tiles [-W^T | Q~^T],
// Kd^T and A_qk, T and A_hat (bf16) and e^{Gamma_last} (fp32).  With ckpt set no output is formed: out
// only gives the unused output map a valid base.
cudaError_t launch_fwd_pipe(const uint16_t *q, const uint16_t *k, const uint16_t *v, const float *g,
                            const float *beta, const int32_t *cu, int n_docs, int64_t T, int H,
                            const float *h0, float *ht, uint16_t *out, int *status, cudaStream_t stream,
                            uint16_t *ckpt = nullptr);

// Segment-table forward (kda_split.cu builds the tables on the device): CTA (entry, head) runs
// entry blockIdx.x / H of `seg`, {first token, end token, entering-state slot, final-state slot},
// for entries below *seg_count; max_segs bounds the count (the grid is max_segs * H CTAs).  A slot
// is -1 (zero entering state / no final state), a workspace slot s < kSplitSlotCaller (the state at
// ws_states + (s * H + head) * 128 * 128), or kSplitSlotCaller + d (document d of h0 / ht).
// transition: v taken as zero, the identity as every entering state, no outputs (the transition
// map M of each segment lands in its final-state slot).
constexpr int kSplitSlotCaller = 1 << 24;
cudaError_t launch_fwd_segments(bool transition, const uint16_t *q, const uint16_t *k, const uint16_t *v,
                                const float *g, const float *beta, int64_t T, int H, const int4 *seg,
                                const int *seg_count, int max_segs, const float *h0, float *ht, float *ws_states,
                                uint16_t *out, int *status, cudaStream_t stream);

// Token-by-token forward (the recurrence itself, no chunking): one CTA of 128 threads per
// (document, head), the state in registers.  Same arguments and contract as launch_fwd_pipe.
cudaError_t launch_fwd_recurrent(const uint16_t *q, const uint16_t *k, const uint16_t *v, const float *g,
                                 const float *beta, const int32_t *cu, int n_docs, int64_t T, int H,
                                 const float *h0, float *ht, uint16_t *out, int *status, cudaStream_t stream);

// 2-D TMA map over a row-major [rows, cols] tensor (cols contiguous) with box [box_rows, box_cols]
// (kda_fwd_pipe.cu); false when the driver's encoder is unavailable or rejects the arguments.
namespace pipe_path {
bool make_map(CUtensorMap *m, const void *base, CUtensorMapDataType dt, int elem_bytes, uint64_t rows, uint64_t cols,
              uint32_t box_rows, uint32_t box_cols, CUtensorMapSwizzle swz);
}

// Recompute backward: dq, dk, dv (bf16), dg, dbeta (fp32) from the forward inputs and dout.
// workspace holds bwd_workspace_floats(n_docs, T, H) floats (entering states of every chunk
// and per-chain scratch).
size_t bwd_workspace_floats(int n_docs, int64_t T, int H);
cudaError_t launch_bwd(const uint16_t *q, const uint16_t *k, const uint16_t *v, const float *g, const float *beta,
                       const int32_t *cu, int n_docs, int64_t T, int H, const uint16_t *dout, uint16_t *dq,
                       uint16_t *dk, uint16_t *dv, float *dg, float *dbeta, float *workspace, int *status,
                       cudaStream_t stream);

// Records `msg` as the thread's kda_last_error() text and returns `status` (for entry points
// defined outside kda_api.cu).
int set_last_error(int status, const char *msg);

// Checks that the current device is sm_100 and returns it with its device status word (the
// word kernels record KDA_ERR_BAD_SEQLENS / KDA_ERR_TIMEOUT in); a kda_status, with the
// message recorded on failure.
int device_context(int *dev, int **status);

// Runs one time-limited mbarrier wait that can never complete (self-test of the
// timeout path): records kStatusTimeout in *status after about limit_cycles.
cudaError_t launch_wait_selftest(int *status, long long limit_cycles, cudaStream_t stream);

}  // namespace kda
