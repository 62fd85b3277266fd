"""Initial / final state (kda_chunk_fwd_state) vs the fp64 oracle, through the C ABI (gpu).

Bar: outputs as in test_parity_gpu (rel-L2 <= 1e-2, max-abs <= 5e-2); final states rel-L2 <= 1e-2
and max-abs <= 5e-2 of their largest magnitude.
"""
import numpy as np
import pytest

from chunked_gated_delta_12_b200.inputs import custom_workload, generate
from tests.helpers import ATOL_MAX, RTOL_L2, compare, oracle_out, out_to_f64, to_device

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def kda():
    import torch
    import chunked_gated_delta_12_b200 as m
    torch.cuda.init()
    return m


def states(n_docs, H, seed, scale=0.3):
    rng = np.random.default_rng(seed)
    return (rng.normal(size=(n_docs, H, 128, 128)) * scale).astype(np.float32)


def run(kda, d, h0=None, final=True):
    import torch
    t = to_device(d)
    h0_t = None if h0 is None else torch.from_numpy(h0).cuda()
    r = kda.kda_chunk_fwd(t["q"], t["k"], t["v"], t["g"], t["beta"], t["cu_seqlens"], initial_state=h0_t,
                          output_final_state=final)
    kda.device_status()
    torch.cuda.synchronize()
    o, ht = r if final else (r, None)
    return out_to_f64(o), (None if ht is None else ht.cpu().numpy().astype(np.float64))


def check_state(got, ref):
    rel = np.linalg.norm(got - ref) / np.linalg.norm(ref)
    mx = np.abs(got - ref).max() / np.abs(ref).max()
    assert rel <= RTOL_L2 and mx <= 5e-2, (rel, mx)


# the last case has more documents than the kernels rank longest-first (256): they keep index order
@pytest.mark.parametrize("lens,H", [([256], 2), ([1, 63, 64, 0, 65, 129, 2], 3), ([64] * 8 + [100] * 8, 8),
                                    ([(7 * i) % 10 for i in range(300)], 2)])
def test_initial_and_final_state(kda, lens, H):
    w = custom_workload("state", lens, H, seed=51)
    d = generate(w)
    h0 = states(w.n_docs, H, 52)
    got, ht = run(kda, d, h0)
    ref, rs = oracle_out(d, initial_state=h0, return_state=True)
    rel, mx = compare(got, ref, d["cu_seqlens"], H)
    assert rel <= RTOL_L2 and mx <= ATOL_MAX, (rel, mx)
    check_state(ht.reshape(-1, 128, 128), rs)
    # an empty document hands its initial state through unchanged
    for doc, L in enumerate(lens):
        if L == 0:
            assert np.array_equal(ht[doc], h0[doc].astype(np.float64))


def test_state_hand_off(kda):
    """[0, L1) then [L1, L) with the final state handed over equals one run over [0, L)."""
    L, L1, H = 300, 130, 4
    w = custom_workload("handoff", [L], H, seed=53)
    d = generate(w)
    full, s_full = run(kda, d)
    da = {k: (v[:L1] if k not in ("cu_seqlens",) else np.array([0, L1], np.int32)) for k, v in d.items()}
    db = {k: (v[L1:] if k not in ("cu_seqlens",) else np.array([0, L - L1], np.int32)) for k, v in d.items()}
    oa, sa = run(kda, da)
    ob, sb = run(kda, db, sa.astype(np.float32))
    both = np.concatenate([oa, ob])
    rel = np.linalg.norm(both - full) / np.linalg.norm(full)
    assert rel <= 1e-2, rel
    check_state(sb, s_full)


def test_in_place_state_update(kda):
    import torch
    w = custom_workload("inplace", [70, 10], 2, seed=54)
    d = generate(w)
    h0 = states(w.n_docs, 2, 55)
    _, ht_ref = run(kda, d, h0)
    t = to_device(d)
    buf = torch.from_numpy(h0).cuda()
    kda.kda_chunk_fwd(t["q"], t["k"], t["v"], t["g"], t["beta"], t["cu_seqlens"], initial_state=buf, final_state=buf)
    kda.device_status()
    assert np.array_equal(buf.cpu().numpy().astype(np.float64), ht_ref)


def test_no_tokens_copies_initial_state(kda):
    import torch
    w = custom_workload("empty", [0, 0], 2, seed=56)
    d = generate(w)
    h0 = states(2, 2, 57)
    t = to_device(d)
    o, ht = kda.kda_chunk_fwd(t["q"], t["k"], t["v"], t["g"], t["beta"], t["cu_seqlens"],
                              initial_state=torch.from_numpy(h0).cuda(), output_final_state=True)
    torch.cuda.synchronize()
    assert np.array_equal(ht.cpu().numpy(), h0)
