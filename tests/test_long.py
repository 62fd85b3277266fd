"""kda_chunk_fwd_long on the host: the segment choice, the workspace size and the argument checks
that reject a call before any device work.  CPU only."""
import ctypes

import pytest

from chunked_gated_delta_12_b200 import _lib
from chunked_gated_delta_12_b200.build import build

FAKE = 0x10000000            # never dereferenced: every case below fails a host-side check first
WS = FAKE + (4 << 30)        # a fake workspace far from the fake tensors
STATE = 128 * 128 * 4


@pytest.fixture(scope="module")
def L():
    build()
    return _lib.lib()


def bounds(T, P):
    """Segment p covers chunks [floor(n p / P), floor(n (p + 1) / P)) of n = ceil(T / 64)."""
    n = -(-T // 64)
    return [64 * (n * p // P) for p in range(P)] + [T]


def test_segment_choice(L):
    seg = L.kda_chunk_fwd_long_segments
    assert seg(65536, 32, 148) == 3          # (2P - 3) * 32 <= 148 allows P = 3
    assert seg(65536, 16, 148) == 6          # 9 * 16 = 144 <= 148 < 11 * 16
    assert seg(65536, 8, 148) == 10
    assert seg(1 << 20, 1, 148) == 16        # capped
    assert seg(65536, 64, 148) == 1          # P = 3 needs 192 SMs: no split
    assert seg(64 * 23, 1, 148) == 1         # 23 chunks: P = 3 leaves segments of 7 chunks
    assert seg(64 * 24, 1, 148) == 3         # 24 chunks: 8 per segment
    assert seg(0, 32, 148) == 1 and seg(100, 0, 148) == 1 and seg(100, 1, 0) == 1


def test_workspace_size(L):
    size = L.kda_chunk_fwd_long_workspace_size
    assert size(65536, 32, 0) == 0 and size(65536, 32, 17) == 0 and size(65536, 0, 3) == 0
    up = lambda x: (x + 255) // 256 * 256
    assert size(100, 2, 1) == 256 + up(16)   # the table counts and one table entry
    for T, H, P in ((65536, 32, 3), (1937, 2, 5), (4096, 8, 2), (100, 3, 1)):
        # counts; N, M and final tables and the hand-off record (16 bytes per entry); per head
        # 3 P - 4 states (N and entering states of P - 1 segments, M of P - 2)
        want = 256 + up(P * 16) + up(max(P - 2, 0) * 16) + up(max(P - 1, 0) * 16) + up((P >= 2) * 16) \
            + up(max(3 * P - 4, 0) * H * STATE)
        assert size(T, H, P) == want, (T, H, P)


def call(L, T=64 * 30, H=2, P=3, q=FAKE, out=FAKE + (1 << 30), h0=None, ht=None, ws=WS, ws_bytes=None):
    vp = ctypes.c_void_p
    if ws_bytes is None:
        ws_bytes = L.kda_chunk_fwd_long_workspace_size(T, H, P) if 1 <= P <= 16 else 1 << 30
    return L.kda_chunk_fwd_long(vp(q), vp(FAKE), vp(FAKE), vp(FAKE), vp(FAKE), T, H, P, vp(h0), vp(ht), vp(out),
                                vp(ws), ws_bytes, None)


def test_rejections(L):
    assert call(L, P=0) == 1 and b"segments" in L.kda_last_error()
    assert call(L, P=17) == 1 and b"segments" in L.kda_last_error()
    assert call(L, T=64 * 2, P=3) == 1 and b"chunks" in L.kda_last_error()
    assert call(L, H=0) == 1 and b"H must" in L.kda_last_error()
    assert call(L, T=-1) == 1
    assert call(L, q=0) == 1 and b"NULL" in L.kda_last_error()
    assert call(L, q=FAKE + 8) == 1 and b"aligned" in L.kda_last_error()
    assert call(L, out=FAKE) == 1 and b"alias" in L.kda_last_error()
    assert call(L, ws=0) == 1 and b"workspace" in L.kda_last_error()
    assert call(L, ws=WS + 16) == 1 and b"256-byte" in L.kda_last_error()
    assert call(L, ws_bytes=1024) == 1 and b"too small" in L.kda_last_error()
    assert call(L, ws=FAKE + (1 << 30)) == 1 and b"alias" in L.kda_last_error()    # workspace over out
    st = FAKE + (2 << 30)
    assert call(L, h0=st, ht=st + 64) == 1 and b"same buffer or disjoint" in L.kda_last_error()
    assert call(L, ht=FAKE) == 1 and b"alias" in L.kda_last_error()
    assert call(L, T=0) == 0                 # no tokens and no final state: nothing to do


def test_no_device_is_an_error_not_a_fallback(L):
    import torch
    if torch.cuda.is_available():
        pytest.skip("a GPU is present")
    rc = call(L)
    assert rc in (2, 3), rc
    assert L.kda_last_error()
