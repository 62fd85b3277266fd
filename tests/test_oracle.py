"""Pins for the fp64 oracle: closed forms, special cases, invariants and an
independent chunked formulation.  CPU only.

Each test is chosen so that a plausible slip in the oracle (a dropped term, a
flipped sign, decay applied after instead of before the write, a transposed
state, a missing normalisation, a state that leaks across documents) fails at
least one of them.
"""
import json
import os

import numpy as np
import pytest

import oracle
from oracle.chunked import kda_fwd_chunked

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def rand_case(T, H, K, V, seed, g_lo=-5.0, beta=None):
    rng = np.random.default_rng(seed)
    q = rng.standard_normal((T, H, K)).astype(np.float32)
    k = rng.standard_normal((T, H, K)).astype(np.float32)
    v = rng.standard_normal((T, H, V)).astype(np.float32)
    g = (g_lo / (1 + np.exp(-rng.standard_normal((T, H, K))))).astype(np.float32)
    b = (1 / (1 + np.exp(-rng.standard_normal((T, H))))).astype(np.float32) if beta is None \
        else np.full((T, H), beta, dtype=np.float32)
    return q, k, v, g, b


def l2n(x, eps=1e-6):
    x = np.asarray(x, dtype=np.float64)
    return x / np.sqrt((x * x).sum(-1, keepdims=True) + eps)


def test_worked_example_by_hand():
    """Hand-derived 3-token example (tests/golden/worked_example_d2.json)."""
    with open(os.path.join(GOLDEN, "worked_example_d2.json")) as f:
        ex = json.load(f)
    a = lambda key: np.asarray(ex[key], dtype=np.float32)[:, None, :]
    o = oracle.kda_fwd(a("q"), a("k"), a("v"), a("g"), np.asarray(ex["beta"], np.float32)[:, None],
                       [0, 3], scale=ex["scale"], eps=ex["eps"])
    np.testing.assert_allclose(o[:, 0, :], np.asarray(ex["o"]), atol=ex["tolerance_abs"], rtol=0)


def test_single_token_closed_form():
    """T = 1: the state is beta k^ v^T, so o = scale * beta (q^ . k^) v."""
    q, k, v, g, b = rand_case(1, 3, 128, 128, 1)
    o = oracle.kda_fwd(q, k, v, g, b, [0, 1])
    qn, kn = l2n(q), l2n(k)
    ref = (1 / np.sqrt(128)) * b[..., None] * (qn * kn).sum(-1, keepdims=True) * v
    np.testing.assert_allclose(o, ref, rtol=1e-13, atol=1e-15)


def test_two_token_closed_form():
    """T = 2, unrolled by hand:
    o2 = scale [ b1 ((k1 * e^{g2}) . q2) v1 + b2 (k2 . q2) (v2 - b1 ((k1 * e^{g2}) . k2) v1) ]
    (decay of token 2 hits the stored key before the erase; the erase reads S^T k, not S k)."""
    q, k, v, g, b = rand_case(2, 2, 16, 12, 2)
    o = oracle.kda_fwd(q, k, v, g, b, [0, 2], scale=0.37)
    qn, kn = l2n(q), l2n(k)
    for h in range(2):
        k1d = kn[0, h] * np.exp(g[1, h].astype(np.float64))
        b1, b2 = float(b[0, h]), float(b[1, h])
        v1, v2 = v[0, h].astype(np.float64), v[1, h].astype(np.float64)
        ref = 0.37 * (b1 * (k1d @ qn[1, h]) * v1
                      + b2 * (kn[1, h] @ qn[1, h]) * (v2 - b1 * (k1d @ kn[1, h]) * v1))
        np.testing.assert_allclose(o[1, h], ref, rtol=1e-12, atol=1e-14)


def test_beta_zero_gives_zero():
    """beta = 0 disables both the write and the erase, so the state stays 0 and o == 0."""
    q, k, v, g, b = rand_case(50, 2, 128, 128, 3, beta=0.0)
    o = oracle.kda_fwd(q, k, v, g, b, [0, 20, 50])
    assert np.all(o == 0.0)


def test_gla_switch_matches_closed_form():
    """Without the erase term the recurrence is gated linear attention:
    o_t = scale sum_{j<=t} b_j sum_c q^_tc k^_jc prod_{i=j+1..t} e^{g_ic} v_j
    (product of per-token decays, written as an explicit product, not a cumsum)."""
    T, K, V = 20, 8, 5
    q, k, v, g, b = rand_case(T, 1, K, V, 4)
    o = oracle.kda_fwd(q, k, v, g, b, [0, T], erase=False, scale=0.5)
    qn, kn = l2n(q)[:, 0], l2n(k)[:, 0]
    eg = np.exp(g[:, 0].astype(np.float64))
    for t in range(T):
        acc = np.zeros(V)
        for j in range(t + 1):
            dec = np.ones(K)
            for i in range(j + 1, t + 1):
                dec = dec * eg[i]
            acc += float(b[j, 0]) * float((qn[t] * kn[j] * dec).sum()) * v[j, 0].astype(np.float64)
        np.testing.assert_allclose(o[t, 0], 0.5 * acc, rtol=1e-12, atol=1e-14)


@pytest.mark.parametrize("eps,tol", [(0.0, 1e-7), (1e-6, 2e-6)])  # keys orthonormal only to fp32 rounding
def test_overwrite_with_orthonormal_keys(eps, tol):
    """beta = 1, g = 0 and orthonormal keys: each write replaces the value stored
    under its key, so S^T k_i is the latest value written for key i and reading
    with q = k_i returns scale * that value."""
    K = V = 128
    rng = np.random.default_rng(5)
    Qm, _ = np.linalg.qr(rng.standard_normal((K, K)))
    keys = Qm.T.astype(np.float32)               # rows orthonormal (to fp32 rounding)
    keys = keys / np.sqrt((keys.astype(np.float64) ** 2).sum(1, keepdims=True)).astype(np.float32)
    T = 300
    idx = rng.integers(0, 40, size=T)
    read = rng.integers(0, 40, size=T)
    k = keys[idx][:, None, :]
    v = rng.standard_normal((T, 1, V)).astype(np.float32)
    q = keys[read][:, None, :]
    g = np.zeros((T, 1, K), np.float32)
    b = np.ones((T, 1), np.float32)
    o, S = oracle.kda_fwd(q, k, v, g, b, [0, T], scale=1.0, eps=eps, return_state=True)
    latest = {}
    for t in range(T):
        latest[idx[t]] = v[t, 0].astype(np.float64)
        want = latest.get(read[t], np.zeros(V))
        np.testing.assert_allclose(o[t, 0], want, atol=tol * 10, rtol=0)
    for key, val in latest.items():
        np.testing.assert_allclose(S[0].T @ keys[key].astype(np.float64), val, atol=tol * 10)


def test_packed_equals_separate_runs_bitwise():
    """Packed documents reset the state at each boundary: identical to separate runs."""
    lens = [1, 63, 64, 65, 7]
    T = sum(lens)
    q, k, v, g, b = rand_case(T, 3, 32, 16, 6)
    cu = np.concatenate([[0], np.cumsum(lens)])
    o = oracle.kda_fwd(q, k, v, g, b, cu)
    for d in range(len(lens)):
        s, e = cu[d], cu[d + 1]
        od = oracle.kda_fwd(q[s:e], k[s:e], v[s:e], g[s:e], b[s:e], [0, e - s])
        assert np.array_equal(o[s:e], od)


def test_thread_count_does_not_change_result():
    q, k, v, g, b = rand_case(100, 4, 32, 32, 7)
    o1 = oracle.kda_fwd(q, k, v, g, b, [0, 30, 100], n_threads=1)
    o8 = oracle.kda_fwd(q, k, v, g, b, [0, 30, 100], n_threads=8)
    assert np.array_equal(o1, o8)


def test_chain_subset_matches_full():
    q, k, v, g, b = rand_case(90, 4, 32, 32, 8)
    cu = [0, 40, 90]
    full = oracle.kda_fwd(q, k, v, g, b, cu)
    part = oracle.kda_fwd(q, k, v, g, b, cu, chains=[5, 2])   # doc 1 head 1, doc 0 head 2
    assert np.array_equal(part[40:90, 1], full[40:90, 1])
    assert np.array_equal(part[0:40, 2], full[0:40, 2])
    assert np.isnan(part[0:40, 0]).all()


@pytest.mark.parametrize("chunk", [16, 64])
@pytest.mark.parametrize("L", [1, 15, 16, 17, 63, 64, 65, 130, 256])
def test_chunked_wy_matches_recurrence(L, chunk):
    """The chunked UT/WY algebra (a different algorithm) agrees with the recurrence."""
    q, k, v, g, b = rand_case(L, 1, 32, 24, 100 + L)
    o = oracle.kda_fwd(q, k, v, g, b, [0, L])
    oc = kda_fwd_chunked(q, k, v, g, b, [0, L], chunk=chunk)
    err = np.linalg.norm(o - oc) / np.linalg.norm(o)
    assert err < 1e-10


def test_chunked_wy_strong_decay_and_packing():
    """g = -5 everywhere (64-token cumsum reaches -320) and several packed documents."""
    lens = [70, 3, 64, 129]
    T = sum(lens)
    q, k, v, g, b = rand_case(T, 2, 128, 128, 9)
    g[:] = -5.0
    cu = np.concatenate([[0], np.cumsum(lens)])
    o = oracle.kda_fwd(q, k, v, g, b, cu)
    oc = kda_fwd_chunked(q, k, v, g, b, cu, chunk=64)
    assert np.linalg.norm(o - oc) / np.linalg.norm(o) < 1e-10


def test_linear_in_values_and_column_separable():
    """o is linear in v, and each value column evolves on its own (the state's
    columns never mix), which is what makes splitting V across CTAs exact."""
    from chunked_gated_delta_12_b200.inputs import bf16_bits_to_f32, f32_to_bf16_bits
    T, K, V = 40, 16, 12
    q, k, v, g, b = rand_case(T, 2, K, V, 10)
    rb = lambda x: bf16_bits_to_f32(f32_to_bf16_bits(x)).reshape(x.shape)
    v = rb(v)
    v2 = rb(np.random.default_rng(11).standard_normal(v.shape).astype(np.float32))
    v12 = (v + np.float32(2) * v2).astype(np.float32)
    # 8-bit mantissas: the fp32 sum is exact, so linearity can be checked tightly
    assert np.array_equal(v12.astype(np.float64), v.astype(np.float64) + 2 * v2.astype(np.float64))
    cu = [0, 25, 40]
    o1 = oracle.kda_fwd(q, k, v, g, b, cu)
    o2 = oracle.kda_fwd(q, k, v2, g, b, cu)
    o12 = oracle.kda_fwd(q, k, v12, g, b, cu)
    np.testing.assert_allclose(o12, o1 + 2 * o2, rtol=1e-12, atol=1e-13)
    cols = [3, 7, 8]
    osub = oracle.kda_fwd(q, k, np.ascontiguousarray(v[:, :, cols]), g, b, cu)
    np.testing.assert_allclose(osub, o1[:, :, cols], rtol=1e-13, atol=1e-15)


def test_qk_scale_invariance():
    """q and k are l2-normalised inside the op: positive rescaling changes nothing (eps = 0)."""
    q, k, v, g, b = rand_case(30, 2, 16, 8, 12)
    o = oracle.kda_fwd(q, k, v, g, b, [0, 30], eps=0.0)
    o2 = oracle.kda_fwd(q * np.float32(4.0), k * np.float32(0.25), v, g, b, [0, 30], eps=0.0)
    np.testing.assert_allclose(o2, o, rtol=1e-12, atol=1e-14)


def test_state_norm_growth_bound():
    """(I - beta k k^T) has spectral norm <= 1 for beta in [0,1], |k| = 1, and the decay
    is a contraction, so |S_t|_2 <= |S_{t-1}|_2 + beta_t |v_t|."""
    T, K, V = 25, 8, 6
    q, k, v, g, b = rand_case(T, 1, K, V, 13)
    prev = 0.0
    for t in range(1, T + 1):
        _, S = oracle.kda_fwd(q[:t], k[:t], v[:t], g[:t], b[:t], [0, t], return_state=True)
        nrm = np.linalg.norm(S[0], 2)
        bound = prev + float(b[t - 1, 0]) * np.linalg.norm(v[t - 1, 0].astype(np.float64))
        assert nrm <= bound + 1e-12
        prev = nrm


def test_rejects_malformed_seqlens():
    q, k, v, g, b = rand_case(10, 1, 8, 8, 14)
    for cu in ([1, 10], [0, 9], [0, 6, 4, 10]):
        with pytest.raises(ValueError):
            oracle.kda_fwd(q, k, v, g, b, cu)


def test_empty_documents_allowed():
    q, k, v, g, b = rand_case(10, 1, 8, 8, 15)
    o = oracle.kda_fwd(q, k, v, g, b, [0, 0, 4, 4, 10])
    o2 = oracle.kda_fwd(q, k, v, g, b, [0, 4, 10])
    assert np.array_equal(o, o2)


# ---- initial / final state (FLA's convention, an extension of the fused contract) ----

def _rand_inputs(rng, T, H, K, V, decay_scale=5.0):
    return dict(q=rng.normal(size=(T, H, K)), k=rng.normal(size=(T, H, K)), v=rng.normal(size=(T, H, V)),
                g=-decay_scale / (1.0 + np.exp(-rng.normal(size=(T, H, K)))),
                beta=1.0 / (1.0 + np.exp(-rng.normal(size=(T, H)))))


def test_zero_initial_state_is_the_default():
    rng = np.random.default_rng(11)
    x = _rand_inputs(rng, 40, 2, 8, 6)
    cu = np.array([0, 15, 40], np.int32)
    a, sa = oracle.kda_fwd(**x, cu_seqlens=cu, return_state=True)
    b, sb = oracle.kda_fwd(**x, cu_seqlens=cu, return_state=True, initial_state=np.zeros((2, 2, 8, 6), np.float32))
    assert np.array_equal(a, b) and np.array_equal(sa, sb)


def test_state_hand_off_equals_one_run():
    """Running tokens [0, L1) and handing the final state to a second run over [L1, L) gives the
    outputs and final state of one run over [0, L) (up to the fp32 rounding of the handed state).
    Mild decay keeps the handed state significant."""
    rng = np.random.default_rng(12)
    T, H, K, V, L1 = 90, 2, 8, 6, 37
    x = _rand_inputs(rng, T, H, K, V, decay_scale=0.05)
    o, s = oracle.kda_fwd(**x, cu_seqlens=np.array([0, T], np.int32), return_state=True)
    oa, sa = oracle.kda_fwd(**{k: v[:L1] for k, v in x.items()}, cu_seqlens=np.array([0, L1], np.int32),
                            return_state=True)
    ob, sb = oracle.kda_fwd(**{k: v[L1:] for k, v in x.items()}, cu_seqlens=np.array([0, T - L1], np.int32),
                            return_state=True, initial_state=sa.reshape(1, H, K, V))
    assert np.abs(sa).max() > 0.1
    np.testing.assert_allclose(np.concatenate([oa, ob]), o, rtol=0, atol=1e-6)
    np.testing.assert_allclose(sb, s, rtol=0, atol=1e-6)


def test_segment_transition_is_affine():
    """A segment maps its entering state affinely: S_out = M S_in + N, where N is the segment run
    from the zero state and M the same run with v = 0 from the identity state (the key-channel
    transition product).  Three segments chained this way give the outputs and final state of one
    run (up to the fp32 rounding of the handed states).  Mild decay keeps M significant."""
    rng = np.random.default_rng(14)
    T, H, K, b1, b2 = 120, 2, 8, 40, 85
    x = _rand_inputs(rng, T, H, K, K, decay_scale=0.05)
    one = lambda a, b: np.array([0, b - a], np.int32)
    seg = lambda a, b, **kw: {key: (val[a:b] if key != "v" else kw.get("v", val)[a:b]) for key, val in x.items()}
    o, s = oracle.kda_fwd(**x, cu_seqlens=np.array([0, T], np.int32), return_state=True)
    _, n0 = oracle.kda_fwd(**seg(0, b1), cu_seqlens=one(0, b1), return_state=True)
    _, n1 = oracle.kda_fwd(**seg(b1, b2), cu_seqlens=one(b1, b2), return_state=True)
    eye = np.broadcast_to(np.eye(K), (1, H, K, K)).astype(np.float32)
    _, m1 = oracle.kda_fwd(**seg(b1, b2, v=np.zeros_like(x["v"])), cu_seqlens=one(b1, b2), return_state=True,
                           initial_state=eye)
    assert 0.05 < np.abs(m1).max() < 1.0 + 1e-9 and np.abs(m1 - np.eye(K)).max() > 0.05
    s2 = np.einsum("hij,hjv->hiv", m1, n0) + n1             # state entering the third segment
    o2, s_end = oracle.kda_fwd(**seg(b2, T), cu_seqlens=one(b2, T), return_state=True,
                               initial_state=s2.reshape(1, H, K, K))
    np.testing.assert_allclose(o2, o[b2:], rtol=0, atol=1e-6)
    np.testing.assert_allclose(s_end, s, rtol=0, atol=1e-6)
    # the homogeneous part is linear: from the true entering state with v = 0 the run gives M S_in
    _, ms = oracle.kda_fwd(**seg(b1, b2, v=np.zeros_like(x["v"])), cu_seqlens=one(b1, b2), return_state=True,
                           initial_state=n0.reshape(1, H, K, K))
    np.testing.assert_allclose(ms, np.einsum("hij,hjv->hiv", m1, n0.astype(np.float32)), rtol=0, atol=1e-12)


def test_initial_state_one_token_closed_form():
    """S_1 = (I - b k^ k^T) Diag(e^g) S_0 + b k^ v^T, o = scale S_1^T q^ with S_0 given (K x V:
    rows are key channels)."""
    rng = np.random.default_rng(13)
    K, V = 6, 5
    x = _rand_inputs(rng, 1, 1, K, V)
    S0 = rng.normal(size=(K, V)).astype(np.float32).astype(np.float64)
    o, s = oracle.kda_fwd(**x, cu_seqlens=np.array([0, 1], np.int32), return_state=True,
                          initial_state=S0.reshape(1, 1, K, V))
    q, k, v, g, b = (x["q"][0, 0], x["k"][0, 0], x["v"][0, 0], x["g"][0, 0], x["beta"][0, 0])
    eps = 1e-6
    q32, k32, v32, g32 = (np.float64(np.float32(t)) for t in (q, k, v, g))
    b32 = np.float64(np.float32(b))
    qn, kn = q32 / np.sqrt(q32 @ q32 + eps), k32 / np.sqrt(k32 @ k32 + eps)
    S1 = (np.eye(K) - b32 * np.outer(kn, kn)) @ (np.exp(g32)[:, None] * S0) + b32 * np.outer(kn, v32)
    np.testing.assert_allclose(s[0], S1, rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(o[0, 0], S1.T @ qn / np.sqrt(K), rtol=1e-12, atol=1e-13)
