"""ctypes binding of libkda (include/kda.h): argument marshalling only.

Every step of the forward runs in the CUDA library; nothing here computes.
If libkda.so is missing or the device is not sm_100, calls raise -- there is
no fallback path.
"""
from __future__ import annotations

import ctypes
import os

import torch

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libkda.so")

STATUS = {0: "KDA_OK", 1: "KDA_ERR_INVALID_ARG", 2: "KDA_ERR_UNSUPPORTED_DEVICE", 3: "KDA_ERR_CUDA",
          4: "KDA_ERR_NO_MEMORY", 5: "KDA_ERR_TIMEOUT", 6: "KDA_ERR_BAD_SEQLENS"}

_lib = None


class KdaError(RuntimeError):
    def __init__(self, code: int, msg: str):
        super().__init__(f"{STATUS.get(code, code)}: {msg}")
        self.code = code


def lib() -> ctypes.CDLL:
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(f"libkda.so not built ({LIB_PATH}); run "
                              "`python -m chunked_gated_delta_12_b200.build` (needs nvcc)")
        L = ctypes.CDLL(LIB_PATH)
        vp, i32, i64 = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64
        L.kda_chunk_fwd.restype = i32
        L.kda_chunk_fwd.argtypes = [vp, vp, vp, vp, vp, vp, i32, i64, i32, vp, vp]
        L.kda_chunk_fwd_state.restype = i32
        L.kda_chunk_fwd_state.argtypes = [vp, vp, vp, vp, vp, vp, i32, i64, i32, vp, vp, vp, vp]
        L.kda_recurrent_fwd.restype = i32
        L.kda_recurrent_fwd.argtypes = [vp, vp, vp, vp, vp, vp, i32, i64, i32, vp, vp, vp, vp]
        L.kda_last_error.restype = ctypes.c_char_p
        L.kda_last_error.argtypes = []
        L.kda_device_status.restype = i32
        L.kda_device_status.argtypes = [vp]
        L.kda_wait_selftest.restype = i32
        L.kda_wait_selftest.argtypes = [vp]
        L.kda_chunk_bwd_workspace_size.restype = ctypes.c_size_t
        L.kda_chunk_bwd_workspace_size.argtypes = [i32, i64, i32]
        L.kda_chunk_bwd.restype = i32
        L.kda_chunk_bwd.argtypes = [vp, vp, vp, vp, vp, vp, i32, i64, i32, vp, vp, vp, vp, vp, vp, vp,
                                    ctypes.c_size_t, vp]
        L.kda_chunk_bwd_noalloc.restype = i32
        L.kda_chunk_bwd_noalloc.argtypes = [vp, vp, vp, vp, vp, vp, i32, i64, i32, vp, vp, vp, vp, vp, vp, vp]
        L.kda_chunk_fwd_split.restype = i32
        L.kda_chunk_fwd_split.argtypes = [vp, vp, vp, vp, vp, vp, i32, i64, i32, vp, vp, vp, vp, ctypes.c_size_t, vp]
        L.kda_chunk_fwd_split_workspace_size.restype = ctypes.c_size_t
        L.kda_chunk_fwd_split_workspace_size.argtypes = [i32, i64, i32]
        L.kda_chunk_fwd_long.restype = i32
        L.kda_chunk_fwd_long.argtypes = [vp, vp, vp, vp, vp, i64, i32, i32, vp, vp, vp, vp, ctypes.c_size_t, vp]
        L.kda_chunk_fwd_long_workspace_size.restype = ctypes.c_size_t
        L.kda_chunk_fwd_long_workspace_size.argtypes = [i64, i32, i32]
        L.kda_chunk_fwd_long_segments.restype = i32
        L.kda_chunk_fwd_long_segments.argtypes = [i64, i32, i32]
        L.kda_abi_version.restype = i32
        L.kda_abi_version.argtypes = []
        L.kda_chunk_fwd_host.restype = i32
        L.kda_chunk_fwd_host.argtypes = [vp, vp, vp, vp, vp, vp, i32, i64, i32, vp, vp, ctypes.c_size_t, vp]
        L.kda_chunk_fwd_host_workspace_size.restype = ctypes.c_size_t
        L.kda_chunk_fwd_host_workspace_size.argtypes = [i32, i64, i32]
        _lib = L
    return _lib


def _check(rc: int) -> None:
    if rc != 0:
        raise KdaError(rc, lib().kda_last_error().decode())


def _stream_handle(stream) -> int:
    if stream is None:
        stream = torch.cuda.current_stream()
    return int(stream.cuda_stream)


def _ptr(t):
    return ctypes.c_void_p(t.data_ptr()) if t is not None else None


def _fwd_checked(q, k, v, g, beta, cu_seqlens, out, initial_state, output_final_state, final_state):
    """Shape/dtype checks shared by the forwards; returns the marshalled tensors and sizes.
    cu_seqlens None means one document [0, T) (kda_chunk_fwd_long)."""
    if q.dim() == 4:
        q, k, v, g = (x.squeeze(0) for x in (q, k, v, g))
        beta = beta.squeeze(0)
    T, H, D = q.shape
    for name, t, dt, shape in (("q", q, torch.bfloat16, (T, H, D)), ("k", k, torch.bfloat16, (T, H, D)),
                               ("v", v, torch.bfloat16, (T, H, D)), ("g", g, torch.float32, (T, H, D)),
                               ("beta", beta, torch.float32, (T, H))):
        if t.dtype != dt or tuple(t.shape) != shape or not t.is_contiguous() or not t.is_cuda:
            raise KdaError(1, f"{name} must be a contiguous CUDA {dt} tensor of shape {shape} "
                              f"(got {t.dtype} {tuple(t.shape)})")
    if cu_seqlens is not None and (cu_seqlens.dtype != torch.int32 or not cu_seqlens.is_cuda
                                   or cu_seqlens.dim() != 1):
        raise KdaError(1, "cu_seqlens must be a 1-d int32 CUDA tensor")
    if out is None:
        out = torch.empty_like(q)
    n_docs = 1 if cu_seqlens is None else cu_seqlens.numel() - 1
    shape_s = (n_docs, H, D, D)
    for name, t in (("initial_state", initial_state), ("final_state", final_state)):
        if t is not None and (t.dtype != torch.float32 or tuple(t.shape) != shape_s or not t.is_contiguous()
                              or not t.is_cuda):
            raise KdaError(1, f"{name} must be a contiguous CUDA float32 tensor of shape {shape_s}")
    if final_state is None and output_final_state:
        final_state = torch.empty(shape_s, dtype=torch.float32, device=q.device)
    return q, k, v, g, beta, out, n_docs, T, H, final_state


# Documents shorter than this many tokens are never cut (three segments of at least 8 chunks).
SPLIT_MIN_TOKENS = 3 * 8 * 64


def use_split(n_docs: int, T: int, H: int, num_sms: int | None = None) -> bool:
    """Whether ``kda_chunk_fwd`` routes a call through kda_chunk_fwd_split: when its (document, head)
    chains fill less than half of the GPU's SMs and it has enough tokens for a cut to exist.  The
    device-side planner then decides which documents (if any) are cut."""
    if num_sms is None:
        num_sms = torch.cuda.get_device_properties(torch.cuda.current_device()).multi_processor_count
    return T >= SPLIT_MIN_TOKENS and 2 * n_docs * H < num_sms


def split_workspace_bytes(n_docs: int, T: int, H: int) -> int:
    """Device workspace bytes kda_chunk_fwd_split needs on the current device
    (kda_chunk_fwd_split_workspace_size)."""
    return int(lib().kda_chunk_fwd_split_workspace_size(n_docs, T, H))


def kda_chunk_fwd(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, g: torch.Tensor,
                  beta: torch.Tensor, cu_seqlens: torch.Tensor, out: torch.Tensor | None = None,
                  stream: torch.cuda.Stream | None = None, initial_state: torch.Tensor | None = None,
                  output_final_state: bool = False, final_state: torch.Tensor | None = None,
                  split: bool | None = None, workspace: torch.Tensor | None = None):
    """Chunked KDA forward through libkda: kda_chunk_fwd (kda_chunk_fwd_state with states), or
    kda_chunk_fwd_split when the call has few (document, head) chains.

    q, k, v: [T, H, 128] bf16 (a leading batch dim of 1 is accepted); g: [T, H, 128] fp32;
    beta: [T, H] fp32; cu_seqlens: [n_docs + 1] int32, all on the same CUDA device.
    initial_state: optional [n_docs, H, 128, 128] fp32 starting states (zero if None).
    split: None chooses by ``use_split``; True / False force kda_chunk_fwd_split / the plain call.
    workspace: a CUDA uint8 tensor of at least ``split_workspace_bytes`` bytes for the split call,
    allocated by torch when not given.
    Returns out [T, H, 128] bf16 (allocated by torch if not given), or (out, final_state
    [n_docs, H, 128, 128] fp32) when output_final_state (or a final_state buffer) is given.
    """
    want_state = initial_state is not None or final_state is not None or output_final_state
    q, k, v, g, beta, out, n_docs, T, H, final_state = _fwd_checked(q, k, v, g, beta, cu_seqlens, out, initial_state,
                                                                     output_final_state, final_state)
    if split is None:
        split = use_split(n_docs, T, H)
    if split:
        need = split_workspace_bytes(n_docs, T, H)
        if workspace is None:
            workspace = torch.empty(max(need, 256), dtype=torch.uint8, device=q.device)
        rc = lib().kda_chunk_fwd_split(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta), _ptr(cu_seqlens), n_docs, T, H,
                                       _ptr(initial_state), _ptr(final_state), _ptr(out), _ptr(workspace),
                                       workspace.numel() * workspace.element_size(),
                                       ctypes.c_void_p(_stream_handle(stream)))
        _check(rc)
        return (out, final_state) if final_state is not None else out
    if not want_state:
        rc = lib().kda_chunk_fwd(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta), _ptr(cu_seqlens),
                                 n_docs, T, H, _ptr(out), ctypes.c_void_p(_stream_handle(stream)))
        _check(rc)
        return out
    rc = lib().kda_chunk_fwd_state(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta), _ptr(cu_seqlens), n_docs, T, H,
                                   _ptr(initial_state), _ptr(final_state), _ptr(out),
                                   ctypes.c_void_p(_stream_handle(stream)))
    _check(rc)
    return (out, final_state) if final_state is not None else out


def host_workspace_bytes(n_docs: int, T: int, H: int) -> int:
    """Device workspace bytes of ``kda_chunk_fwd_host``."""
    return int(lib().kda_chunk_fwd_host_workspace_size(n_docs, T, H))


def kda_chunk_fwd_host(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, g: torch.Tensor, beta: torch.Tensor,
                       cu_seqlens: torch.Tensor, out: torch.Tensor, workspace: torch.Tensor,
                       stream: torch.cuda.Stream | None = None) -> torch.Tensor:
    """kda_chunk_fwd_host: the forward on HOST tensors (copies to the device workspace, the forward and
    the copy of the output back are enqueued on `stream`).

    q, k, v, g, beta, cu_seqlens, out: contiguous CPU tensors with kda_chunk_fwd's dtypes and shapes
    (pinned memory for asynchronous copies); workspace: a CUDA uint8 tensor of at least
    ``host_workspace_bytes`` bytes.  Returns out, complete once the stream is synchronised.
    """
    T, H, D = q.shape
    for name, t, dt, shape in (("q", q, torch.bfloat16, (T, H, D)), ("k", k, torch.bfloat16, (T, H, D)),
                               ("v", v, torch.bfloat16, (T, H, D)), ("g", g, torch.float32, (T, H, D)),
                               ("beta", beta, torch.float32, (T, H)), ("out", out, torch.bfloat16, (T, H, D))):
        if t.dtype != dt or tuple(t.shape) != shape or not t.is_contiguous() or t.is_cuda:
            raise KdaError(1, f"{name} must be a contiguous host {dt} tensor of shape {shape}")
    if cu_seqlens.dtype != torch.int32 or cu_seqlens.is_cuda or cu_seqlens.dim() != 1:
        raise KdaError(1, "cu_seqlens must be a 1-d int32 host tensor")
    if workspace.dtype != torch.uint8 or not workspace.is_cuda:
        raise KdaError(1, "workspace must be a CUDA uint8 tensor")
    n_docs = cu_seqlens.numel() - 1
    rc = lib().kda_chunk_fwd_host(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta), _ptr(cu_seqlens), n_docs, T, H,
                                  _ptr(out), _ptr(workspace), workspace.numel(),
                                  ctypes.c_void_p(_stream_handle(stream)))
    _check(rc)
    return out


def kda_recurrent_fwd(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, g: torch.Tensor,
                      beta: torch.Tensor, cu_seqlens: torch.Tensor, out: torch.Tensor | None = None,
                      stream: torch.cuda.Stream | None = None, initial_state: torch.Tensor | None = None,
                      output_final_state: bool = False, final_state: torch.Tensor | None = None):
    """Token-by-token KDA forward through libkda's kda_recurrent_fwd (decode, short inputs).

    Same arguments and return convention as ``kda_chunk_fwd``.
    """
    q, k, v, g, beta, out, n_docs, T, H, final_state = _fwd_checked(q, k, v, g, beta, cu_seqlens, out, initial_state,
                                                                     output_final_state, final_state)
    rc = lib().kda_recurrent_fwd(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta), _ptr(cu_seqlens), n_docs, T, H,
                                 _ptr(initial_state), _ptr(final_state), _ptr(out),
                                 ctypes.c_void_p(_stream_handle(stream)))
    _check(rc)
    return (out, final_state) if final_state is not None else out


def long_segments(T: int, H: int, num_sms: int | None = None) -> int:
    """Segment count kda_chunk_fwd_long uses by default (kda_chunk_fwd_long_segments) on a GPU with
    ``num_sms`` SMs (the current device's if None)."""
    if num_sms is None:
        num_sms = torch.cuda.get_device_properties(torch.cuda.current_device()).multi_processor_count
    return int(lib().kda_chunk_fwd_long_segments(T, H, num_sms))


def long_workspace_bytes(T: int, H: int, segments: int) -> int:
    """Device workspace bytes kda_chunk_fwd_long needs (kda_chunk_fwd_long_workspace_size)."""
    return int(lib().kda_chunk_fwd_long_workspace_size(T, H, segments))


def kda_chunk_fwd_long(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, g: torch.Tensor,
                       beta: torch.Tensor, out: torch.Tensor | None = None, segments: int | None = None,
                       initial_state: torch.Tensor | None = None, output_final_state: bool = False,
                       final_state: torch.Tensor | None = None, workspace: torch.Tensor | None = None,
                       stream: torch.cuda.Stream | None = None):
    """Forward of ONE document [0, T) through libkda's kda_chunk_fwd_long: its chunk chain is split
    into ``segments`` pieces (``long_segments`` if None) that run side by side, joined through the
    state hand-off S_out = M S_in + N.

    Tensors as ``kda_chunk_fwd`` with one document (no cu_seqlens); states [1, H, 128, 128] fp32.
    ``workspace`` (a CUDA uint8 tensor of at least ``long_workspace_bytes`` bytes) is allocated by
    torch when not given.  Returns out, or (out, final_state) as ``kda_chunk_fwd`` does.
    """
    q, k, v, g, beta, out, _, T, H, final_state = _fwd_checked(q, k, v, g, beta, None, out, initial_state,
                                                               output_final_state, final_state)
    if segments is None:
        segments = long_segments(T, H)
    need = long_workspace_bytes(T, H, segments)
    if workspace is None:
        workspace = torch.empty(max(need, 256), dtype=torch.uint8, device=q.device)
    rc = lib().kda_chunk_fwd_long(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta), T, H, segments,
                                  _ptr(initial_state), _ptr(final_state), _ptr(out), _ptr(workspace),
                                  workspace.numel() * workspace.element_size(),
                                  ctypes.c_void_p(_stream_handle(stream)))
    _check(rc)
    return (out, final_state) if final_state is not None else out


# Longest document (tokens) for which the token-by-token kernel beats the chunked one.  Measured
# on B200 with 64 documents x 32 heads and states in and out: 4 tokens 124 us vs 229 us, 16
# tokens 378 us vs 236 us; the crossover lies near 8.
RECURRENT_MAX_LEN = 8


def resolve_mode(seq_len: int) -> str:
    """Kernel for documents of at most ``seq_len`` tokens: "recurrent" (kda_recurrent_fwd) for
    short inputs such as decoding, "chunk" (kda_chunk_fwd) otherwise.  The same choice as
    KimiDeltaAttention._resolve_mode on the kimi_linear model page, with the threshold measured
    here (the page does not print one)."""
    if seq_len < 0:
        raise ValueError("seq_len must be >= 0")
    return "recurrent" if seq_len <= RECURRENT_MAX_LEN else "chunk"


def kda_chunk_bwd(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, g: torch.Tensor, beta: torch.Tensor,
                  cu_seqlens: torch.Tensor, dout: torch.Tensor, workspace: torch.Tensor | None = None,
                  stream: torch.cuda.Stream | None = None):
    """Recompute backward through libkda's kda_chunk_bwd.

    Same inputs as ``kda_chunk_fwd`` plus dout [T, H, 128] bf16.  Returns (dq, dk, dv, dg, dbeta):
    bf16 [T, H, 128] x3, fp32 [T, H, 128], fp32 [T, H].  ``workspace`` (a CUDA uint8 tensor of at
    least ``bwd_workspace_bytes`` bytes) is allocated by torch when not given.
    """
    T, H, D = q.shape
    for name, t, dt, shape in (("q", q, torch.bfloat16, (T, H, D)), ("k", k, torch.bfloat16, (T, H, D)),
                               ("v", v, torch.bfloat16, (T, H, D)), ("g", g, torch.float32, (T, H, D)),
                               ("beta", beta, torch.float32, (T, H)), ("dout", dout, torch.bfloat16, (T, H, D))):
        if t.dtype != dt or tuple(t.shape) != shape or not t.is_contiguous() or not t.is_cuda:
            raise KdaError(1, f"{name} must be a contiguous CUDA {dt} tensor of shape {shape} "
                              f"(got {t.dtype} {tuple(t.shape)})")
    if cu_seqlens.dtype != torch.int32 or not cu_seqlens.is_cuda or cu_seqlens.dim() != 1:
        raise KdaError(1, "cu_seqlens must be a 1-d int32 CUDA tensor")
    n_docs = cu_seqlens.numel() - 1
    need = bwd_workspace_bytes(n_docs, T, H)
    if workspace is None:
        workspace = torch.empty(max(need, 16), dtype=torch.uint8, device=q.device)
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    dg, dbeta = torch.empty_like(g), torch.empty_like(beta)
    rc = lib().kda_chunk_bwd(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta), _ptr(cu_seqlens), n_docs, T, H,
                             _ptr(dout), _ptr(dq), _ptr(dk), _ptr(dv), _ptr(dg), _ptr(dbeta), _ptr(workspace),
                             workspace.numel() * workspace.element_size(), ctypes.c_void_p(_stream_handle(stream)))
    _check(rc)
    return dq, dk, dv, dg, dbeta


def kda_chunk_bwd_noalloc(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, g: torch.Tensor, beta: torch.Tensor,
                          cu_seqlens: torch.Tensor, dout: torch.Tensor, dq: torch.Tensor, dk: torch.Tensor,
                          dv: torch.Tensor, dg: torch.Tensor, dbeta: torch.Tensor,
                          stream: torch.cuda.Stream | None = None) -> None:
    """Recompute backward through libkda's kda_chunk_bwd_noalloc, for callers that cannot
    allocate device memory: the caller passes every input and output (dq, dk, dv bf16
    [T, H, 128]; dg fp32 [T, H, 128]; dbeta fp32 [T, H]) and the library's own fixed scratch
    (``NOALLOC_SCRATCH_BYTES``) serves as the workspace.  Nothing is allocated here either.
    Calls on one device share that scratch, so calls that overlap on the GPU race."""
    T, H, D = q.shape
    for name, t, dt, shape in (("q", q, torch.bfloat16, (T, H, D)), ("k", k, torch.bfloat16, (T, H, D)),
                               ("v", v, torch.bfloat16, (T, H, D)), ("g", g, torch.float32, (T, H, D)),
                               ("beta", beta, torch.float32, (T, H)), ("dout", dout, torch.bfloat16, (T, H, D)),
                               ("dq", dq, torch.bfloat16, (T, H, D)), ("dk", dk, torch.bfloat16, (T, H, D)),
                               ("dv", dv, torch.bfloat16, (T, H, D)), ("dg", dg, torch.float32, (T, H, D)),
                               ("dbeta", dbeta, torch.float32, (T, H))):
        if t.dtype != dt or tuple(t.shape) != shape or not t.is_contiguous() or not t.is_cuda:
            raise KdaError(1, f"{name} must be a contiguous CUDA {dt} tensor of shape {shape} "
                              f"(got {t.dtype} {tuple(t.shape)})")
    if cu_seqlens.dtype != torch.int32 or not cu_seqlens.is_cuda or cu_seqlens.dim() != 1:
        raise KdaError(1, "cu_seqlens must be a 1-d int32 CUDA tensor")
    rc = lib().kda_chunk_bwd_noalloc(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta), _ptr(cu_seqlens),
                                     cu_seqlens.numel() - 1, T, H, _ptr(dout), _ptr(dq), _ptr(dk), _ptr(dv),
                                     _ptr(dg), _ptr(dbeta), ctypes.c_void_p(_stream_handle(stream)))
    _check(rc)


# Scratch bytes kda_chunk_bwd_noalloc holds per GPU (KDA_BWD_NOALLOC_SCRATCH_BYTES in kda.h).
NOALLOC_SCRATCH_BYTES = 64 * 1024 * 1024


def bwd_workspace_bytes(n_docs: int, T: int, H: int) -> int:
    """Device workspace bytes kda_chunk_bwd needs (kda_chunk_bwd_workspace_size)."""
    return int(lib().kda_chunk_bwd_workspace_size(n_docs, T, H))


def wait_selftest(stream: torch.cuda.Stream | None = None) -> None:
    """Enqueue the self-test whose device wait must time out (see kda_wait_selftest)."""
    _check(lib().kda_wait_selftest(ctypes.c_void_p(_stream_handle(stream))))


def device_status(stream: torch.cuda.Stream | None = None) -> None:
    """Synchronise the stream and raise if a kernel flagged bad cu_seqlens or a timeout."""
    _check(lib().kda_device_status(ctypes.c_void_p(_stream_handle(stream))))
