"""fp64 CPU oracle for the chunk-KDA forward -- TEST INFRASTRUCTURE ONLY.

Only tests/, ``__graft_entry__.smoke()`` and bench.py's cpu_baseline /
``--impl reference`` legs may import this package.  The product path
(``chunked_gated_delta_12_b200`` and its CUDA library) never does, and shares
no code with it: the only thing both sides read is the seeded input generator,
which holds no KDA arithmetic.

``kda_fwd`` is the plain token-by-token recurrence in ``kda_oracle.c`` (C,
fp64, pthreads over independent (document, head) chains).  ``chunked.py`` is a
second, independent formulation (chunked UT/WY algebra in numpy fp64) used
only to cross-check the recurrence.  ``kda_bwd`` (``kda_oracle_bwd.c``) is the
reverse-mode derivative of the same recurrence, with ``kda_fwd64`` (the
forward on fp64 inputs) for finite-difference checks.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "kda_oracle.c")
_SRC_BWD = os.path.join(_HERE, "kda_oracle_bwd.c")
_LIB_PATH = os.path.join(_HERE, "libkda_oracle.so")
_lib = None


def build(force: bool = False) -> str:
    """Compile the oracle sources with gcc into oracle/libkda_oracle.so (no GPU needed)."""
    newest = max(os.path.getmtime(_SRC), os.path.getmtime(_SRC_BWD))
    if force or not os.path.exists(_LIB_PATH) or os.path.getmtime(_LIB_PATH) < newest:
        tmp = _LIB_PATH + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-std=c11", "-shared", "-fPIC", "-pthread",
                               "-o", tmp, _SRC, _SRC_BWD, "-lm"])
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _load():
    global _lib
    if _lib is None:
        lib = ctypes.CDLL(build())
        f = lib.kda_oracle_fwd
        f.restype = ctypes.c_int
        f.argtypes = [ctypes.c_void_p] * 6 + [ctypes.c_int, ctypes.c_int64, ctypes.c_int,
                                              ctypes.c_int, ctypes.c_int, ctypes.c_double,
                                              ctypes.c_double, ctypes.c_int, ctypes.c_void_p,
                                              ctypes.c_int, ctypes.c_void_p, ctypes.c_void_p,
                                              ctypes.c_void_p, ctypes.c_int]
        f = lib.kda_oracle_fwd64
        f.restype = ctypes.c_int
        f.argtypes = [ctypes.c_void_p] * 6 + [ctypes.c_int, ctypes.c_int64, ctypes.c_int, ctypes.c_int,
                                              ctypes.c_int, ctypes.c_double, ctypes.c_double,
                                              ctypes.c_void_p, ctypes.c_int, ctypes.c_void_p, ctypes.c_int]
        f = lib.kda_oracle_bwd
        f.restype = ctypes.c_int
        f.argtypes = [ctypes.c_void_p] * 7 + [ctypes.c_int, ctypes.c_int64, ctypes.c_int, ctypes.c_int,
                                              ctypes.c_int, ctypes.c_double, ctypes.c_double,
                                              ctypes.c_void_p, ctypes.c_int] + [ctypes.c_void_p] * 5 + [
                                                  ctypes.c_int]
        _lib = lib
    return _lib


def _f32(x) -> np.ndarray:
    return np.ascontiguousarray(x, dtype=np.float32)


def _ptr(a: np.ndarray | None):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def kda_fwd(q, k, v, g, beta, cu_seqlens, scale: float | None = None, eps: float = 1e-6,
            erase: bool = True, chains=None, n_threads: int | None = None,
            return_state: bool = False, initial_state=None):
    """Token-recurrence KDA forward in fp64.

    q, k, g: [T, H, K] (any float dtype; widened exactly to fp32 then fp64 inside)
    v: [T, H, V]; beta: [T, H]; cu_seqlens: [n_docs + 1] int.
    chains: optional list of chain ids (doc * H + head) to compute; other rows of
    the result are NaN.  initial_state: optional [n_docs, H, K, V] starting states (zero if
    None).  Returns o [T, H, V] fp64 (and the final states [n_chains, K, V] if
    ``return_state``).
    """
    q, k, v, g = _f32(q), _f32(k), _f32(v), _f32(g)
    beta = _f32(beta)
    cu = np.ascontiguousarray(cu_seqlens, dtype=np.int32)
    T, H, K = q.shape
    V = v.shape[2]
    assert k.shape == (T, H, K) and g.shape == (T, H, K) and v.shape[:2] == (T, H)
    assert beta.shape == (T, H)
    n_docs = len(cu) - 1
    if scale is None:
        scale = 1.0 / np.sqrt(K)
    ch = None if chains is None else np.ascontiguousarray(chains, dtype=np.int32)
    n_chains = n_docs * H if ch is None else len(ch)
    out = np.full((T, H, V), np.nan, dtype=np.float64)
    fs = np.zeros((n_chains, K, V), dtype=np.float64) if return_state else None
    if n_threads is None:
        n_threads = os.cpu_count() or 1
    h0 = None
    if initial_state is not None:
        h0 = _f32(initial_state).reshape(n_docs * H, K, V)
    rc = _load().kda_oracle_fwd(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta), _ptr(cu),
                                n_docs, T, H, K, V, float(scale), float(eps), int(bool(erase)),
                                _ptr(ch), n_chains, _ptr(out), _ptr(fs), _ptr(h0), int(n_threads))
    if rc != 0:
        raise ValueError("oracle rejected the arguments (cu_seqlens or sizes malformed)")
    return (out, fs) if return_state else out


def _f64(x) -> np.ndarray:
    return np.ascontiguousarray(x, dtype=np.float64)


def _shapes(q, v, beta, cu_seqlens):
    T, H, K = q.shape
    V = v.shape[2]
    assert v.shape[:2] == (T, H) and beta.shape == (T, H)
    return T, H, K, V, len(cu_seqlens) - 1


def kda_fwd64(q, k, v, g, beta, cu_seqlens, scale: float | None = None, eps: float = 1e-6,
              chains=None, n_threads: int | None = None):
    """The same token recurrence as ``kda_fwd`` on fp64 inputs (no widening from fp32),
    so that finite differences of it can check ``kda_bwd``.  Returns o [T, H, V] fp64."""
    q, k, v, g, beta = _f64(q), _f64(k), _f64(v), _f64(g), _f64(beta)
    cu = np.ascontiguousarray(cu_seqlens, dtype=np.int32)
    T, H, K, V, n_docs = _shapes(q, v, beta, cu)
    scale = 1.0 / np.sqrt(K) if scale is None else scale
    ch = None if chains is None else np.ascontiguousarray(chains, dtype=np.int32)
    out = np.full((T, H, V), np.nan)
    rc = _load().kda_oracle_fwd64(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta), _ptr(cu), n_docs, T, H, K, V,
                                  float(scale), float(eps), _ptr(ch), n_docs * H if ch is None else len(ch),
                                  _ptr(out), int(n_threads or os.cpu_count() or 1))
    if rc != 0:
        raise ValueError("oracle rejected the arguments (cu_seqlens or sizes malformed)")
    return out


def kda_bwd(q, k, v, g, beta, dout, cu_seqlens, scale: float | None = None, eps: float = 1e-6,
            chains=None, n_threads: int | None = None):
    """Reverse-mode gradients of o = KDA(q, k, v, g, beta) against dout, in fp64.

    Inputs of any float dtype are widened exactly to fp64.  Returns a dict with dq, dk ([T, H, K],
    gradients of the raw, un-normalised q and k), dv [T, H, V], dg [T, H, K] and dbeta [T, H];
    rows outside the selected chains are NaN."""
    q, k, v, g, beta, dout = (_f64(x) for x in (q, k, v, g, beta, dout))
    cu = np.ascontiguousarray(cu_seqlens, dtype=np.int32)
    T, H, K, V, n_docs = _shapes(q, v, beta, cu)
    assert dout.shape == v.shape
    scale = 1.0 / np.sqrt(K) if scale is None else scale
    ch = None if chains is None else np.ascontiguousarray(chains, dtype=np.int32)
    res = {n: np.full(s, np.nan) for n, s in (("dq", (T, H, K)), ("dk", (T, H, K)), ("dv", (T, H, V)),
                                               ("dg", (T, H, K)), ("dbeta", (T, H)))}
    rc = _load().kda_oracle_bwd(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta), _ptr(dout), _ptr(cu), n_docs, T,
                                H, K, V, float(scale), float(eps), _ptr(ch), n_docs * H if ch is None else len(ch),
                                _ptr(res["dq"]), _ptr(res["dk"]), _ptr(res["dv"]), _ptr(res["dg"]),
                                _ptr(res["dbeta"]), int(n_threads or os.cpu_count() or 1))
    if rc != 0:
        raise ValueError("oracle rejected the arguments (cu_seqlens or sizes malformed)")
    return res


def chain_rows(cu_seqlens, H: int, chain: int) -> tuple[int, int, int]:
    """(first token, end token, head) of chain id doc * H + head."""
    doc, h = divmod(int(chain), H)
    return int(cu_seqlens[doc]), int(cu_seqlens[doc + 1]), h
