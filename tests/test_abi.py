"""libkda loads, exports every entry point include/kda.h declares, and rejects
bad arguments on the host before touching a device.  CPU only."""
import ctypes
import os
import re

import pytest

from chunked_gated_delta_12_b200 import _lib
from chunked_gated_delta_12_b200.build import build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def L():
    build()
    return _lib.lib()


def declared_functions():
    src = open(os.path.join(ROOT, "include", "kda.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(kda_[a-z0-9_]+)\s*\(", src)))


def test_exports_every_declared_symbol(L):
    names = declared_functions()
    assert "kda_chunk_fwd" in names and "kda_last_error" in names
    for n in names:
        assert hasattr(L, n), f"libkda.so does not export {n}"


def test_abi_version(L):
    assert L.kda_abi_version() == 1


FAKE = 0x10000000  # never dereferenced: every case below fails a host-side check first


def call(L, q=FAKE, k=FAKE, v=FAKE, g=FAKE, beta=FAKE, cu=FAKE, n_docs=1, T=64, H=1, out=FAKE + (1 << 30)):
    vp = ctypes.c_void_p
    return L.kda_chunk_fwd(vp(q), vp(k), vp(v), vp(g), vp(beta), vp(cu), n_docs, T, H, vp(out), None)


def test_rejects_bad_sizes(L):
    assert call(L, n_docs=0) == 1 and b"n_docs" in L.kda_last_error()
    assert call(L, H=0) == 1 and b"H must" in L.kda_last_error()
    assert call(L, T=-1) == 1
    assert call(L, cu=0) == 1 and b"cu_seqlens" in L.kda_last_error()


def test_empty_is_noop(L):
    assert call(L, T=0) == 0


def test_rejects_null_misaligned_and_aliasing(L):
    assert call(L, q=0) == 1 and b"NULL" in L.kda_last_error()
    assert call(L, k=FAKE + 8) == 1 and b"aligned" in L.kda_last_error()
    assert call(L, beta=FAKE + 2) == 1
    assert call(L, out=FAKE) == 1 and b"alias" in L.kda_last_error()


def test_no_device_is_an_error_not_a_fallback(L):
    import torch
    if torch.cuda.is_available():
        pytest.skip("a GPU is present")
    rc = call(L)
    assert rc in (2, 3), rc            # UNSUPPORTED_DEVICE or CUDA error, never OK
    assert L.kda_last_error()


def call_rec(L, q=FAKE, k=FAKE, v=FAKE, g=FAKE, beta=FAKE, cu=FAKE, n_docs=1, T=64, H=1, h0=None, ht=None,
             out=FAKE + (1 << 30)):
    vp = ctypes.c_void_p
    return L.kda_recurrent_fwd(vp(q), vp(k), vp(v), vp(g), vp(beta), vp(cu), n_docs, T, H, vp(h0), vp(ht), vp(out),
                               None)


def test_recurrent_entry_validates_like_the_chunked_one(L):
    assert call_rec(L, n_docs=0) == 1 and b"n_docs" in L.kda_last_error()
    assert call_rec(L, H=0) == 1 and b"H must" in L.kda_last_error()
    assert call_rec(L, q=0) == 1 and b"NULL" in L.kda_last_error()
    assert call_rec(L, v=FAKE + 8) == 1 and b"aligned" in L.kda_last_error()
    assert call_rec(L, out=FAKE) == 1 and b"alias" in L.kda_last_error()
    st = FAKE + (2 << 30)
    assert call_rec(L, h0=st, ht=st + 64) == 1 and b"same buffer or disjoint" in L.kda_last_error()
    assert call_rec(L, h0=st + 4) == 1 and b"16-byte" in L.kda_last_error()
    assert call_rec(L, ht=FAKE) == 1 and b"alias" in L.kda_last_error()
    assert call_rec(L, T=0) == 0                       # no tokens and no final state: nothing to do


def test_resolve_mode():
    from chunked_gated_delta_12_b200 import RECURRENT_MAX_LEN, resolve_mode
    assert resolve_mode(1) == "recurrent" and resolve_mode(RECURRENT_MAX_LEN) == "recurrent"
    assert resolve_mode(RECURRENT_MAX_LEN + 1) == "chunk" and resolve_mode(65536) == "chunk"
    with pytest.raises(ValueError):
        resolve_mode(-1)


def test_backward_workspace_size(L):
    """The backward's workspace is one block per chunk slot and head: the forward pass's checkpoint
    block (S^T and U~^T, B2, Kd^T, A_qk, T, A_hat, D: 123904 bytes) and the dS sweep's block (dS^T
    and dU~^T: 49152 bytes); slots are T / 64 + n_docs per head, an upper bound that does not read
    cu_seqlens."""
    per = 123904 + 49152
    for n_docs, T, H in ((1, 64, 1), (5, 1328, 4), (16, 32768, 32), (1, 65536, 32)):
        assert L.kda_chunk_bwd_workspace_size(n_docs, T, H) == (T // 64 + n_docs) * H * per


def test_host_entry_point_checks_before_any_copy(L):
    """kda_chunk_fwd_host (host inputs, device workspace) rejects bad sizes, pointers and workspaces
    on the host, before anything is enqueued; its workspace holds the device copies of the inputs and
    the output, each on a 256-byte boundary."""
    vp = ctypes.c_void_p
    need = L.kda_chunk_fwd_host_workspace_size(1, 64, 1)
    up = lambda x: (x + 255) // 256 * 256
    assert need == 4 * up(64 * 128 * 2) + up(64 * 128 * 4) + up(64 * 4) + up(2 * 4)
    assert L.kda_chunk_fwd_host_workspace_size(0, 64, 1) == 0

    def host(ws=FAKE, ws_bytes=need, n_docs=1, T=64, q=FAKE):
        return L.kda_chunk_fwd_host(vp(q), vp(FAKE), vp(FAKE), vp(FAKE), vp(FAKE), vp(FAKE), n_docs, T, 1,
                                    vp(FAKE), vp(ws), ws_bytes, None)
    assert host(n_docs=0) == 1 and b"n_docs" in L.kda_last_error()
    assert host(T=0) == 0
    assert host(q=0) == 1 and b"NULL" in L.kda_last_error()
    assert host(ws=0) == 1 and b"workspace" in L.kda_last_error()
    assert host(ws=FAKE + 16) == 1 and b"256-byte" in L.kda_last_error()
    assert host(ws_bytes=need - 1) == 1 and b"too small" in L.kda_last_error()
