"""Pins of the fp64 backward oracle (``oracle.kda_bwd``) against facts that do not come from it.

* Central finite differences of the fp64-input forward (``oracle.kda_fwd64``) along random
  directions, for every input; one of them is the pages' check (T=32, H=1, K=V=128).
* The closed form of a one-token document (S_0 = 0, so o = scale beta (q^.k^) v).
* Packed documents equal separate runs; the state (and its gradient) resets at a boundary.
* A document longer than the oracle's recompute stride (64 tokens) gives the same
  gradients as finite differences, so the checkpoint bookkeeping is pinned too.
"""
import numpy as np
import pytest

import oracle

NAMES = ("q", "k", "v", "g", "beta")


def make(rng, lengths, H, K, V):
    T = int(sum(lengths))
    x = dict(
        q=rng.normal(size=(T, H, K)),
        k=rng.normal(size=(T, H, K)),
        v=rng.normal(size=(T, H, V)),
        g=-5.0 / (1.0 + np.exp(-rng.normal(size=(T, H, K)))),
        beta=1.0 / (1.0 + np.exp(-rng.normal(size=(T, H)))),
    )
    cu = np.concatenate([[0], np.cumsum(lengths)]).astype(np.int32)
    do = rng.normal(size=(T, H, V))
    return x, cu, do


def loss(x, cu, do):
    return float((oracle.kda_fwd64(**x, cu_seqlens=cu) * do).sum())


def fd_check(x, cu, do, rng, h=1e-6, rtol=2e-7):
    gr = oracle.kda_bwd(**x, dout=do, cu_seqlens=cu)
    for n in NAMES:
        d = rng.normal(size=x[n].shape)
        xp, xm = dict(x), dict(x)
        xp[n] = x[n] + h * d
        xm[n] = x[n] - h * d
        fd = (loss(xp, cu, do) - loss(xm, cu, do)) / (2 * h)
        an = float((gr["d" + n] * d).sum())
        assert abs(fd - an) <= rtol * max(1.0, abs(an)), (n, fd, an)
    return gr


def test_finite_differences_T32_H1_full_width():
    """The pages' validation instance: T=32, H=1, K=V=128."""
    rng = np.random.default_rng(1)
    x, cu, do = make(rng, [32], 1, 128, 128)
    fd_check(x, cu, do, rng)


def test_finite_differences_packed_across_recompute_stride():
    """Two documents, one longer than 64 tokens, two heads, small head dims."""
    rng = np.random.default_rng(2)
    x, cu, do = make(rng, [37, 150], 2, 16, 12)
    fd_check(x, cu, do, rng)


def test_single_token_closed_form():
    rng = np.random.default_rng(3)
    K = V = 8
    x, cu, do = make(rng, [1], 1, K, V)
    eps, scale = 1e-6, 1.0 / np.sqrt(K)
    q, k, v, b = x["q"][0, 0], x["k"][0, 0], x["v"][0, 0], x["beta"][0, 0]
    o_ = do[0, 0]
    rq, rk = 1 / np.sqrt(q @ q + eps), 1 / np.sqrt(k @ k + eps)
    qn, kn = q * rq, k * rk
    qk, vo = qn @ kn, v @ o_
    dqn = scale * b * vo * kn
    dkn = scale * b * vo * qn
    want = dict(
        dv=scale * b * qk * o_,
        dbeta=scale * qk * vo,
        dq=rq * (dqn - qn * (qn @ dqn)),
        dk=rk * (dkn - kn * (kn @ dkn)),
        dg=np.zeros(K),
    )
    gr = oracle.kda_bwd(**x, dout=do, cu_seqlens=cu)
    for n, w in want.items():
        got = gr[n][0, 0] if n != "dbeta" else gr[n][0, 0]
        np.testing.assert_allclose(got, w, rtol=1e-12, atol=1e-14)


def test_packed_equals_separate():
    rng = np.random.default_rng(4)
    lengths = [5, 70, 1]
    x, cu, do = make(rng, lengths, 2, 8, 8)
    packed = oracle.kda_bwd(**x, dout=do, cu_seqlens=cu)
    for d in range(len(lengths)):
        s0, s1 = cu[d], cu[d + 1]
        xs = {n: x[n][s0:s1] for n in NAMES}
        sep = oracle.kda_bwd(**xs, dout=do[s0:s1], cu_seqlens=np.array([0, s1 - s0], np.int32))
        for n in sep:
            np.testing.assert_allclose(packed[n][s0:s1], sep[n], rtol=0, atol=0)


def test_chain_subset_and_bad_seqlens():
    rng = np.random.default_rng(5)
    x, cu, do = make(rng, [10, 20], 2, 8, 8)
    full = oracle.kda_bwd(**x, dout=do, cu_seqlens=cu)
    sub = oracle.kda_bwd(**x, dout=do, cu_seqlens=cu, chains=[3])     # doc 1, head 1
    np.testing.assert_array_equal(sub["dq"][10:, 1], full["dq"][10:, 1])
    assert np.isnan(sub["dq"][:, 0]).all() and np.isnan(sub["dq"][:10, 1]).all()
    with pytest.raises(ValueError):
        oracle.kda_bwd(**x, dout=do, cu_seqlens=np.array([0, 40, 30], np.int32))


def test_chunked_backward_formulation_matches_token_backward():
    """The chunked (WY) reverse-mode formulation the CUDA backward follows equals the token
    recurrence's reverse mode in fp64, across partial chunks, several documents and heads."""
    from oracle.chunked import kda_bwd_chunked
    rng = np.random.default_rng(6)
    x, cu, do = make(rng, [37, 150, 64, 1], 2, 16, 12)
    a = oracle.kda_bwd(**x, dout=do, cu_seqlens=cu)
    b = kda_bwd_chunked(**x, dout=do, cu_seqlens=cu)
    for n in a:
        np.testing.assert_allclose(b[n], a[n], rtol=1e-9, atol=1e-12)
