/*
 * kda.h -- C ABI of libkda, the B200 (sm_100a) chunk-KDA forward.
 *
 * Kimi Delta Attention (KDA) is the gated delta rule with a per-key-channel
 * decay.  Per document and head, with the 128 x 128 fp32 state S starting at 0:
 *
 *   S_t = (I - beta_t k_t k_t^T) Diag(exp(g_t)) S_{t-1} + beta_t k_t v_t^T
 *   o_t = scale * S_t^T q_t,          scale = 1/sqrt(128)
 *
 * with q_t and k_t l2-normalised inside the op (q / sqrt(|q|^2 + 1e-6)).
 *
 * Scope follows the fused-kernel contract of the kda_fused page of
 * nemo_automodel.components.models.kimi_k3 (module description and
 * fused_chunk_kda): head dims K = V = 128, packed layout (batch 1, int32
 * cu_seqlens; a dense batch of B equal-length sequences is passed as B packed
 * documents with cu_seqlens = [0, L, 2L, ..., BL]), q/k l2-normalised inside
 * the kernel, a bounded log gate, no initial or final state, no context
 * parallelism, chunk mode only (kda_chunk_fwd).  Entry points that widen it:
 * kda_chunk_fwd_state adds an initial and a final state per chain;
 * kda_recurrent_fwd is the token-by-token mode (the "recurrent" alternative to
 * "chunk" that the kda_mode setting and KimiDeltaAttention._resolve_mode of
 * the kimi_linear model page choose between) for decoding and short inputs;
 * kda_chunk_fwd_split (and kda_chunk_fwd_long, its one-document form) cuts long
 * documents into segments joined through the state hand-off; kda_chunk_bwd (and kda_chunk_bwd_noalloc) is the backward.
 * Like fused_kda_unsupported_reason on the kda_fused page, every call that
 * falls outside this scope is rejected with the first violated condition
 * (kda_last_error); there is no fallback path of any kind.
 */
#ifndef KDA_H_
#define KDA_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    KDA_OK = 0,
    KDA_ERR_INVALID_ARG = 1,        /* bad pointer, size or alignment (see kda_last_error) */
    KDA_ERR_UNSUPPORTED_DEVICE = 2, /* current device is not sm_100 (B200-class)          */
    KDA_ERR_CUDA = 3,               /* a CUDA runtime call or launch failed               */
    KDA_ERR_NO_MEMORY = 4,          /* reserved: libkda allocates no device memory        */
    KDA_ERR_TIMEOUT = 5,            /* a device-side bounded wait gave up                 */
    KDA_ERR_BAD_SEQLENS = 6         /* cu_seqlens content found malformed on the device   */
} kda_status;

/* Head dimension the kernels are specialised to (K = V). */
#define KDA_HEAD_DIM 128

/*
 * kda_chunk_fwd -- chunked KDA forward, o = KDA(q, k, v, g, beta) per document.
 *
 * Operation: the recurrence in the header comment, evaluated chunk-wise
 * (64-token chunks starting at each document start) in the exact UT/WY
 * algebra; output equal to the token recurrence up to rounding.  This is
 * fused_chunk_kda(q, k, v, g, beta, cu_seqlens) of the kda_fused page, whose
 * return convention is (o, None): no final state.
 *
 * Arguments (all arrays DEVICE memory, C-contiguous, 16-byte aligned):
 *   q, k, v    [T, H, 128] bf16 (uint16 bit patterns), token-major, then head, then channel
 *   g          [T, H, 128] fp32 per-key-channel log decay; precondition -5 <= g <= 0
 *              (the bounded gate; values outside are not checked and may lose accuracy)
 *   beta       [T, H] fp32 write strength, expected in [0, 1]
 *   cu_seqlens [n_docs + 1] int32, cu[0] = 0, non-decreasing, cu[n_docs] = T;
 *              zero-length documents are allowed and produce nothing
 *   n_docs     >= 1
 *   T          total tokens (>= 0); T = 0 returns KDA_OK without launching
 *   H          heads (>= 1); q, k and v share H (no grouped heads)
 *   out        [T, H, 128] bf16 (uint16), written for every token in [0, T); must not
 *              alias any input
 *   stream     cudaStream_t (NULL = legacy default stream); the call is asynchronous
 *
 * Ownership: the caller owns every buffer; libkda keeps no pointer after the
 * enqueued work and allocates no device memory.
 *
 * Errors: argument and device checks return KDA_ERR_INVALID_ARG /
 * KDA_ERR_UNSUPPORTED_DEVICE with a message in kda_last_error() and launch
 * nothing.  A malformed cu_seqlens table cannot be seen from the host without
 * a sync; the kernel detects it, skips the affected documents and records
 * KDA_ERR_BAD_SEQLENS, which kda_device_status() reports.
 */
kda_status kda_chunk_fwd(const uint16_t *q, const uint16_t *k, const uint16_t *v,
                         const float *g, const float *beta, const int32_t *cu_seqlens,
                         int n_docs, int64_t T, int H, uint16_t *out, void *stream);

/*
 * kda_chunk_fwd_host -- kda_chunk_fwd on HOST buffers: the end-to-end call.
 *
 * Enqueues on `stream`, in this order: one cudaMemcpyAsync per input (q, k, v, g, beta,
 * cu_seqlens) from host memory into the caller's device workspace, the forward of kda_chunk_fwd
 * on those device copies, and one cudaMemcpyAsync of the output back into host `out`.  The
 * operation and its result are kda_chunk_fwd's (bit-identical on the same inputs).
 *
 * Arguments: q, k, v, g, beta, cu_seqlens, out, n_docs, T, H as kda_chunk_fwd, except that the
 * seven arrays are HOST memory (page-locked for the copies to run asynchronously at the link's
 * rate; pageable memory works but CUDA stages it and the call may block); no alignment rule.
 *   workspace        DEVICE memory, 256-byte aligned, at least
 *                    kda_chunk_fwd_host_workspace_size(n_docs, T, H) bytes; it receives the
 *                    device copies (content on entry ignored).
 *   workspace_bytes  its size.
 * Ownership: the caller owns every buffer.  The call is asynchronous: the host arrays must stay
 * valid and unchanged until the stream has passed the copies, and out is complete only after the
 * stream is synchronised.
 * Errors: as kda_chunk_fwd, checked before anything is enqueued, plus KDA_ERR_INVALID_ARG for a
 * missing, misaligned or small workspace and KDA_ERR_CUDA when a copy cannot be enqueued.  As in
 * kda_chunk_fwd, cu_seqlens is validated on the device (KDA_ERR_BAD_SEQLENS via
 * kda_device_status).
 */
kda_status kda_chunk_fwd_host(const uint16_t *q, const uint16_t *k, const uint16_t *v, const float *g,
                              const float *beta, const int32_t *cu_seqlens, int n_docs, int64_t T, int H,
                              uint16_t *out, void *workspace, size_t workspace_bytes, void *stream);

/* Device workspace bytes of kda_chunk_fwd_host (0 for invalid sizes). */
size_t kda_chunk_fwd_host_workspace_size(int n_docs, int64_t T, int H);

/*
 * kda_chunk_fwd_state -- kda_chunk_fwd with an initial and a final state per chain.
 *
 * The same forward, except that the state of each (document, head) chain starts from
 * initial_state instead of zero, and the state after the document's last token is written
 * to final_state.  This is FLA's initial/final state convention, which the fused-kernel
 * contract of the kda_fused page leaves out (it fixes "no initial or final state"); it makes
 * stateful use possible (a long sequence in pieces, or decoding after a prefill).
 *
 * Arguments: as kda_chunk_fwd, plus
 *   initial_state [n_docs, H, 128, 128] fp32 DEVICE memory: S_0 of chain (doc, head), rows are
 *                 key channels, columns value columns; NULL means zero.
 *   final_state   [n_docs, H, 128, 128] fp32 DEVICE memory, written for every chain (an empty
 *                 document gets its initial state); NULL means not written.  It may be the same
 *                 buffer as initial_state (updated in place) but must not overlap it otherwise,
 *                 nor any input or out.  Both 16-byte aligned.
 * With T = 0 only final_state is written (a copy of initial_state, or zero).
 * Errors: as kda_chunk_fwd.
 */
kda_status kda_chunk_fwd_state(const uint16_t *q, const uint16_t *k, const uint16_t *v, const float *g,
                               const float *beta, const int32_t *cu_seqlens, int n_docs, int64_t T, int H,
                               const float *initial_state, float *final_state, uint16_t *out, void *stream);

/*
 * kda_recurrent_fwd -- token-by-token KDA forward (recurrent mode), with optional states.
 *
 * Operation: the recurrence in the header comment taken one token at a time, no chunking
 * (the "recurrent" kernel choice of the kda_mode setting on the kimi_linear model page, which
 * KimiDeltaAttention._resolve_mode picks by sequence length).  The result is the same as
 * kda_chunk_fwd_state's up to rounding; the state stays fp32 throughout.  One CTA of 128
 * threads per (document, head) chain; its cost per token is a fixed 128 x 128 state update,
 * so it suits few tokens per document (decoding a token after a prefill, short documents),
 * while kda_chunk_fwd is far faster on long documents.
 *
 * Arguments, layouts, ownership and errors: exactly as kda_chunk_fwd_state (initial_state and
 * final_state optional, final_state may be initial_state for an in-place update).  Only
 * 2-byte alignment is needed by this kernel, but the same 16-byte rule is enforced so that a
 * buffer valid for one mode is valid for the other.
 */
kda_status kda_recurrent_fwd(const uint16_t *q, const uint16_t *k, const uint16_t *v, const float *g,
                             const float *beta, const int32_t *cu_seqlens, int n_docs, int64_t T, int H,
                             const float *initial_state, float *final_state, uint16_t *out, void *stream);

/*
 * kda_chunk_fwd_split -- kda_chunk_fwd_state with long documents cut into segments that run side
 * by side (for calls with few (document, head) chains: one long document, or a few long documents
 * packed with short ones).
 *
 * Why: the chunked kernel runs one CTA per (document, head) chain, so a call with few chains keeps
 * few SMs busy and takes as long as its longest serial chain of chunk steps.
 *
 * Operation: the same result as kda_chunk_fwd_state, up to rounding.  The recurrence in the header
 * comment is affine in the state: a segment of tokens maps its entering state to
 * S_out = M S_in + N, where N is the segment run from the zero state and M the product of its
 * per-token maps (I - beta k k^T) Diag(exp(g)) (the same run with v = 0 from the identity state).
 * A planner kernel reads cu_seqlens on the device and cuts the documents with the longest chains
 * into P segments at chunk boundaries (at least 8 chunks each, P <= 16), as many as keep the first
 * stage within one wave of the GPU's SMs (a cut document holds 2 P - 3 chains per head there);
 * documents that are not cut run whole in the first stage.  A cut document runs as
 *   1. N_p of segments 0..P-2 (segment 0 from its initial state; its outputs are final), while a
 *      second, library-owned stream computes M_p of the middle segments 1..P-2;
 *   2. the hand-off, in fp32: S_in(1) = N_0, S_in(p + 1) = M_p S_in(p) + N_p;
 *   3. segments 1..P-1 from their entering states: their outputs and the final state.
 * The state hand-off between pieces of one sequence is how the kimi_k3 model page runs KDA under
 * context parallelism (KimiDeltaAttention._forward_with_cp passes the recurrent state from one shard
 * to the next); the transition map M lets the pieces run at the same time on one GPU.  Outputs of
 * documents that are not cut, and of every first segment, are bit-identical to kda_chunk_fwd_state's.
 *
 * Arguments: as kda_chunk_fwd_state, plus
 *   workspace       DEVICE memory, 256-byte aligned, at least
 *                   kda_chunk_fwd_split_workspace_size(n_docs, T, H) bytes for the current device,
 *                   overlapping no other argument; its contents on entry do not matter.  Calls that
 *                   share a workspace must be ordered (one stream).
 * Streams: the M pass runs on a non-blocking stream that libkda creates, with two events, once per
 * device at the first call that needs it, with that device current; `stream` forks to it and joins
 * it through the events, so the call stays asynchronous and ordered on `stream`.  That second stream
 * is shared by every call on the device: while a call is being captured into a CUDA graph, the shared
 * stream belongs to that capture until the capture ends, so no other split call on the same device
 * (from another thread or another stream) may run between the captured call and the end of its
 * capture.
 * Ownership and errors: as kda_chunk_fwd_state (a malformed cu_seqlens table is found by the planner
 * on the device, nothing runs, and kda_device_status() reports KDA_ERR_BAD_SEQLENS); bad sizes,
 * pointers, alignment, aliasing or a small workspace return KDA_ERR_INVALID_ARG and launch nothing.
 */
kda_status kda_chunk_fwd_split(const uint16_t *q, const uint16_t *k, const uint16_t *v, const float *g,
                               const float *beta, const int32_t *cu_seqlens, int n_docs, int64_t T, int H,
                               const float *initial_state, float *final_state, uint16_t *out, void *workspace,
                               size_t workspace_bytes, void *stream);

/*
 * kda_chunk_fwd_split_workspace_size -- bytes of workspace kda_chunk_fwd_split needs for these sizes
 * on the current device (it depends on the device's SM count, not on the document lengths); 0 for
 * invalid sizes.  About 3 (SMs / H) states of 64 KB per head plus the segment tables.
 */
size_t kda_chunk_fwd_split_workspace_size(int n_docs, int64_t T, int H);

/*
 * kda_chunk_fwd_long -- kda_chunk_fwd_state for ONE document, its chunk chain split into
 * `segments` pieces that run side by side.
 *
 * Why: the chunked kernel runs one CTA per (document, head) chain, so one long document with H
 * heads occupies only H SMs and takes as long as its serial chain of T/64 chunk steps.
 *
 * Operation: the same result as kda_chunk_fwd_state with cu_seqlens = [0, T], up to rounding.
 * The recurrence in the header comment is affine in the state: a segment of tokens maps its
 * entering state to S_out = M S_in + N, where N is the segment run from the zero state and M the
 * product of its per-token maps (I - beta k k^T) Diag(exp(g)) (the same run with v = 0 from the
 * identity state).  The document is cut at chunk boundaries into P segments (segment p covers
 * chunks [floor(n p / P), floor(n (p + 1) / P)) of its n = ceil(T / 64) chunks) and run as
 *   1. N_p of segments 0..P-2, segment 0 from initial_state (its outputs are final), while a
 *      second, library-owned stream computes M_p of the middle segments 1..P-2;
 *   2. the hand-off, in fp32: S_in(1) = N_0, S_in(p + 1) = M_p S_in(p) + N_p;
 *   3. segments 1..P-1 from their entering states: their outputs and the final state.
 * Each stage's chains are at most ceil(n / P) chunks long, so the document takes about 2 n / P
 * chunk steps instead of n.  The state hand-off between pieces of one sequence is how the kimi_k3
 * model page runs KDA under context parallelism (KimiDeltaAttention._forward_with_cp passes the
 * recurrent state from one shard to the next); the transition map M lets the pieces run at the
 * same time on one GPU.  Outputs of segment 0 are bit-identical to kda_chunk_fwd_state's.
 *
 * Arguments: q, k, v, g, beta, out, T, H, initial_state, final_state and stream as
 * kda_chunk_fwd_state with n_docs = 1 (states [1, H, 128, 128]; no cu_seqlens: the document is
 * [0, T)), plus
 *   segments        P, 1..16 and at most ceil(T / 64); 1 runs the document unsplit.
 *                   kda_chunk_fwd_long_segments gives the choice that fits the GPU.
 *   workspace       DEVICE memory, 256-byte aligned, at least
 *                   kda_chunk_fwd_long_workspace_size(T, H, segments) bytes, overlapping no
 *                   other argument; its contents on entry do not matter.  Calls that share a
 *                   workspace must be ordered (one stream).
 * Streams: as kda_chunk_fwd_split (this is that call with one document and a fixed segment count).
 * Ownership and errors: as kda_chunk_fwd_state; bad sizes, pointers, alignment, aliasing or a
 * small workspace return KDA_ERR_INVALID_ARG and launch nothing.
 */
kda_status kda_chunk_fwd_long(const uint16_t *q, const uint16_t *k, const uint16_t *v, const float *g,
                              const float *beta, int64_t T, int H, int segments, const float *initial_state,
                              float *final_state, uint16_t *out, void *workspace, size_t workspace_bytes,
                              void *stream);

/*
 * kda_chunk_fwd_long_workspace_size -- bytes of workspace kda_chunk_fwd_long needs for these
 * sizes (0 for invalid sizes): the segment tables and, for P >= 2, per head 3 P - 4 states of
 * 64 KB (N and entering states of P - 1 segments, M of P - 2).
 */
size_t kda_chunk_fwd_long_workspace_size(int64_t T, int H, int segments);

/*
 * kda_chunk_fwd_long_segments -- the segment count for kda_chunk_fwd_long on a GPU with
 * num_sms SMs: the largest P <= 16 whose stage 1, (2 P - 3) H chains of one CTA each, fits on
 * the SMs at once and whose segments keep at least 8 chunks; 1 (no split) when that P is below
 * 3, where splitting does not shorten the chain (P = 2 takes n / 2 + n / 2 steps).
 */
int kda_chunk_fwd_long_segments(int64_t T, int H, int num_sms);

/*
 * kda_chunk_bwd_workspace_size -- bytes of device workspace kda_chunk_bwd needs for a call
 * with these sizes (an upper bound that does not depend on the cu_seqlens content).
 */
size_t kda_chunk_bwd_workspace_size(int n_docs, int64_t T, int H);

/*
 * kda_chunk_bwd -- recompute-from-inputs backward of kda_chunk_fwd.
 *
 * Operation: the gradients of L = sum(dout * o), o = KDA(q, k, v, g, beta) per document as in
 * kda_chunk_fwd, with respect to the raw (un-normalised) q and k, to v, g and beta.  This is the
 * backward of fused_chunk_kda on the kda_fused page: nothing is saved by the forward, every
 * intermediate is recomputed from the inputs.  Evaluated chunk-wise in exact algebra (64-token
 * chunks from each document start); equal to the reverse-mode derivative of the token
 * recurrence up to rounding.
 *
 * Arguments (DEVICE memory, C-contiguous):
 *   q, k, v, g, beta, cu_seqlens, n_docs, T, H   exactly as for kda_chunk_fwd
 *   dout       [T, H, 128] bf16 (uint16 bit patterns): the upstream gradient of o
 *   dq, dk, dv [T, H, 128] bf16 outputs; dg [T, H, 128] fp32; dbeta [T, H] fp32.  Every row in
 *              [0, T) is written.  Outputs must not alias an input or each other.
 *   workspace  device buffer of at least kda_chunk_bwd_workspace_size(n_docs, T, H) bytes,
 *              16-byte aligned, owned by the caller; its content on entry is ignored and on
 *              return is unspecified.  It holds, per chunk and head (about 169 KB), what the
 *              forward pass saves (the state entering the chunk, U~, the chunk's operand tiles,
 *              T and A_hat) and what the reverse dS sweep writes (dS and dU~).  libkda allocates
 *              no memory of its own.
 *
 * Work: three launches on `stream` -- the forward kernel in its checkpoint instance, the reverse
 * sweep over dS (one CTA per document and head, tcgen05 with dS^T in tensor memory), and the
 * gradient kernel (one CTA per chunk and head).  Results are bit-reproducible: no atomics, fixed
 * summation orders.
 *   stream     cudaStream_t (NULL = legacy default stream); the call is asynchronous
 *
 * Errors: as kda_chunk_fwd; a workspace smaller than required is KDA_ERR_INVALID_ARG.
 */
kda_status kda_chunk_bwd(const uint16_t *q, const uint16_t *k, const uint16_t *v, const float *g,
                         const float *beta, const int32_t *cu_seqlens, int n_docs, int64_t T, int H,
                         const uint16_t *dout, uint16_t *dq, uint16_t *dk, uint16_t *dv, float *dg,
                         float *dbeta, void *workspace, size_t workspace_bytes, void *stream);

/* Bytes of device scratch that kda_chunk_bwd_noalloc holds on each GPU (64 MiB). */
#define KDA_BWD_NOALLOC_SCRATCH_BYTES (64u * 1024u * 1024u)

/*
 * kda_chunk_bwd_noalloc -- kda_chunk_bwd for callers that cannot allocate device memory.
 *
 * The reference pages have no counterpart to this entry point; it is a convenience of this
 * library.  Some callers cannot call cudaMalloc when they run the backward: their device
 * memory is owned by another allocator (for instance a framework's caching pool that has
 * already reserved the free memory, so a fresh cudaMalloc fails), or they must not allocate
 * after start-up because cudaMalloc and cudaFree synchronise the device and can stall the
 * work of every other stream.  This entry point computes exactly what kda_chunk_bwd computes,
 * with the same kernel, but takes its workspace from a fixed scratch array of
 * KDA_BWD_NOALLOC_SCRATCH_BYTES that lives in the library's own device image.  It calls no
 * cudaMalloc, cudaFree or other allocating routine.
 *
 * Arguments, layouts and errors: as kda_chunk_bwd without the workspace pair.  The caller
 * still provides every input and output buffer.
 *
 * Limit: calls whose kda_chunk_bwd_workspace_size(n_docs, T, H) exceeds
 * KDA_BWD_NOALLOC_SCRATCH_BYTES are rejected with KDA_ERR_INVALID_ARG and a message naming
 * the sizes (for example 1 document of 2048 tokens with 8 heads fits; 4096 tokens with 32
 * heads does not); those callers need kda_chunk_bwd.  The results are bit-identical to
 * kda_chunk_bwd's.
 *
 * Memory held: every GPU that loads libkda's device code keeps the array until the process
 * exits.  Its device address is looked up on the first call made on each device (with that
 * device current), so make that first call before any stream capture.
 *
 * Sharing: every call on a device uses the same array, which keeps the last call's contents
 * (the kernel sets every value it reads, so nothing needs clearing between calls).  Calls
 * whose executions overlap on the GPU -- on different streams, or from different host
 * threads without ordering -- race on the array and give wrong results; order them on one
 * stream or use kda_chunk_bwd with separate workspaces.
 */
kda_status kda_chunk_bwd_noalloc(const uint16_t *q, const uint16_t *k, const uint16_t *v, const float *g,
                                 const float *beta, const int32_t *cu_seqlens, int n_docs, int64_t T, int H,
                                 const uint16_t *dout, uint16_t *dq, uint16_t *dk, uint16_t *dv, float *dg,
                                 float *dbeta, void *stream);

/* Thread-local description of the first violated condition of the last failing call. */
const char *kda_last_error(void);

/*
 * kda_device_status -- synchronise `stream`, then return and clear the
 * device-side status word of the current device (KDA_OK, KDA_ERR_BAD_SEQLENS or
 * KDA_ERR_TIMEOUT), or KDA_ERR_CUDA if the synchronisation itself failed.
 */
kda_status kda_device_status(void *stream);

/*
 * kda_wait_selftest -- enqueue on `stream` a one-warp kernel whose time-limited
 * device wait can never be satisfied, so that it gives up (after ~10 ms of SM
 * clock) and records KDA_ERR_TIMEOUT exactly as the forward kernels do when a
 * tensor-core or TMA completion never arrives.  A following kda_device_status()
 * returns KDA_ERR_TIMEOUT and clears it; the CUDA context stays usable.  This is
 * a diagnostic of the failure-reporting path (the kda_fused page's rule: report
 * the condition, never hang or fall back), not part of the forward.
 */
kda_status kda_wait_selftest(void *stream);

/* ABI version of this header (bumped on any signature change). */
int kda_abi_version(void);

#ifdef __cplusplus
}
#endif

#endif /* KDA_H_ */
