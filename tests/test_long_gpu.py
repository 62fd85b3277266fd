"""kda_chunk_fwd_long (one document split into segments joined through the state hand-off
S_out = M S_in + N) vs the fp64 oracle, through the C ABI (gpu).

Bar as test_parity_gpu: rel-L2 <= 1e-2 and max-abs <= 5e-2 on the bf16 outputs, final states
rel-L2 <= 1e-2 and max-abs <= 5e-2 of their largest magnitude; the first segment's outputs
bit-identical to kda_chunk_fwd's (the same chunks from the same state).
"""
import numpy as np
import pytest

from chunked_gated_delta_12_b200.inputs import custom_workload, generate, workload
from tests.helpers import ATOL_MAX, RTOL_L2, compare, oracle_out, out_to_f64, to_device

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def kda():
    import torch
    import chunked_gated_delta_12_b200 as m
    torch.cuda.init()
    return m


def first_boundary(T, P):
    return 64 * ((-(-T // 64)) // P)


def slow_gates(d, seed, scale=0.001, beta_mean=0.1):
    """Gates near 0 and weak writes, so that the state survives a segment and the transition map M
    matters (dropping it moves the last segment's outputs by 28 % (P = 3) to 47 % (P = 5))."""
    z = np.random.default_rng(seed).standard_normal(d["g"].shape)
    d["g"][:] = (-scale / (1.0 + np.exp(-z))).astype(np.float32)
    d["beta"][:] = (d["beta"] * (beta_mean / d["beta"].mean())).astype(np.float32)


def segment(d, a, b):
    e = {k: v[a:b] for k, v in d.items() if k != "cu_seqlens"}
    e["cu_seqlens"] = np.array([0, b - a], np.int32)
    return e


def run_long(kda, d, P, h0=None, final=False, workspace=None, in_place=False):
    import torch
    t = to_device(d)
    h0_t = None if h0 is None else torch.from_numpy(h0).cuda()
    r = kda.kda_chunk_fwd_long(t["q"], t["k"], t["v"], t["g"], t["beta"], segments=P, initial_state=h0_t,
                               output_final_state=final and not in_place,
                               final_state=h0_t if in_place else None, workspace=workspace)
    kda.device_status()
    torch.cuda.synchronize()
    o, ht = r if isinstance(r, tuple) else (r, None)
    return out_to_f64(o), (None if ht is None else ht.cpu().numpy().astype(np.float64))


def run_plain(kda, d):
    """The unsplit forward (kda_chunk_fwd itself, whatever the chain count)."""
    import torch
    t = to_device(d)
    o = kda.kda_chunk_fwd(t["q"], t["k"], t["v"], t["g"], t["beta"], t["cu_seqlens"], split=False)
    kda.device_status()
    torch.cuda.synchronize()
    return out_to_f64(o)


def check_state(got, ref):
    rel = np.linalg.norm(got - ref) / np.linalg.norm(ref)
    mx = np.abs(got - ref).max() / np.abs(ref).max()
    assert rel <= RTOL_L2 and mx <= 5e-2, (rel, mx)


@pytest.mark.parametrize("P", [2, 3, 5])
def test_matches_oracle_with_slow_decay(kda, P):
    T, H = 64 * 30 + 17, 2
    w = custom_workload("long", [T], H, seed=61)
    d = generate(w)
    slow_gates(d, 62)
    ref = oracle_out(d)
    # the hand-off matters here: the last segment entered with N of the previous segment alone
    # (its M dropped), or from zero when P = 2, is far from the true outputs
    n = -(-T // 64)
    b_prev, b_last = 64 * (n * (P - 2) // P), 64 * (n * (P - 1) // P)
    h_wrong = None
    if P >= 3:
        _, n_prev = oracle_out(segment(d, b_prev, b_last), return_state=True)
        h_wrong = n_prev.reshape(1, H, 128, 128).astype(np.float32)
    wrong = oracle_out(segment(d, b_last, T), initial_state=h_wrong)
    assert np.linalg.norm(wrong - ref[b_last:]) / np.linalg.norm(ref[b_last:]) > 0.2
    got, _ = run_long(kda, d, P)
    rel, mx = compare(got, ref, d["cu_seqlens"], H)
    assert rel <= RTOL_L2 and mx <= ATOL_MAX, (rel, mx)
    b1 = first_boundary(T, P)
    assert np.array_equal(got[:b1], run_plain(kda, d)[:b1])


@pytest.mark.parametrize("in_place", [False, True])
def test_initial_and_final_state(kda, in_place):
    import torch
    T, H, P = 64 * 24 + 5, 3, 4
    w = custom_workload("long_state", [T], H, seed=63)
    d = generate(w)
    slow_gates(d, 64)
    h0 = (np.random.default_rng(65).normal(size=(1, H, 128, 128)) * 0.3).astype(np.float32)
    ref, rs = oracle_out(d, initial_state=h0, return_state=True)
    if in_place:
        h0_t = torch.from_numpy(h0).cuda()
        t = to_device(d)
        o = kda.kda_chunk_fwd_long(t["q"], t["k"], t["v"], t["g"], t["beta"], segments=P, initial_state=h0_t,
                                   final_state=h0_t)[0]
        kda.device_status()
        torch.cuda.synchronize()
        got, ht = out_to_f64(o), h0_t.cpu().numpy().astype(np.float64)
    else:
        got, ht = run_long(kda, d, P, h0=h0, final=True)
    rel, mx = compare(got, ref, d["cu_seqlens"], H)
    assert rel <= RTOL_L2 and mx <= ATOL_MAX, (rel, mx)
    check_state(ht.reshape(-1, 128, 128), rs)


def test_one_segment_is_the_plain_forward_and_calls_repeat(kda):
    import torch
    T, H = 64 * 40 + 33, 4
    w = custom_workload("long_one", [T], H, seed=66)
    d = generate(w)
    plain = run_plain(kda, d)
    one, _ = run_long(kda, d, 1)
    assert np.array_equal(one, plain)
    ws = torch.empty(kda.long_workspace_bytes(T, H, 4), dtype=torch.uint8, device="cuda")
    a, _ = run_long(kda, d, 4, workspace=ws)
    b, _ = run_long(kda, d, 4, workspace=ws)
    assert np.array_equal(a, b)
    rel = np.linalg.norm(a - plain) / np.linalg.norm(plain)
    assert rel <= RTOL_L2, rel


def test_long_document_workload_default_split_all_chains(kda):
    """One document of 65536 tokens, H = 32, with the default segment count (3 on 148 SMs);
    the oracle recomputes all 32 chains and every output row is compared."""
    w = workload(3)
    d = generate(w)
    got, _ = run_long(kda, d, None)
    assert np.isfinite(got).all()
    ref = oracle_out(d)
    rel, mx = compare(got, ref, d["cu_seqlens"], w.H)
    assert rel <= RTOL_L2 and mx <= ATOL_MAX, (rel, mx)
