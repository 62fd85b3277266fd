"""kda_chunk_fwd_split (long documents cut into segments planned on the device from cu_seqlens,
joined through the state hand-off S_out = M S_in + N) vs the fp64 oracle, through the C ABI (gpu).

Bar as test_parity_gpu: rel-L2 <= 1e-2 and max-abs <= 5e-2 on the bf16 outputs over every chain;
final states rel-L2 <= 1e-2 and max-abs <= 5e-2 of their largest magnitude; documents that are not
cut bit-identical to the unsplit forward.
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


def slow_gates(d, seed, scale=0.001, beta_mean=0.1):
    """Gates near 0 and weak writes, so that the state survives a segment and the transition map M
    matters (with the workloads' gates in (-5, 0) the state forgets a segment within a few chunks)."""
    z = np.random.default_rng(seed).standard_normal(d["g"].shape)
    d["g"][:] = (-scale / (1.0 + np.exp(-z))).astype(np.float32)
    d["beta"][:] = (d["beta"] * (beta_mean / d["beta"].mean())).astype(np.float32)


def run(kda, d, split, h0=None, final=False):
    import torch
    t = to_device(d)
    h0_t = None if h0 is None else torch.from_numpy(h0).cuda()
    r = kda.kda_chunk_fwd(t["q"], t["k"], t["v"], t["g"], t["beta"], t["cu_seqlens"], split=split,
                          initial_state=h0_t, output_final_state=final)
    kda.device_status()
    torch.cuda.synchronize()
    o, ht = r if isinstance(r, tuple) else (r, None)
    return out_to_f64(o), (None if ht is None else ht.cpu().numpy().astype(np.float64))


LONG_SHORT = [3000] + [37 + 41 * i for i in range(15)] + [2500] + [90 + 23 * i for i in range(15)]


def test_two_long_thirty_short_every_chain(kda):
    """2 long and 30 short documents (H = 2: 64 chains, few enough for the split): the planner cuts
    the long ones; every chain matches the oracle, and the short documents are bit-identical to the
    unsplit forward."""
    assert kda.use_split(len(LONG_SHORT), sum(LONG_SHORT), 2, 148)
    w = custom_workload("long_short", LONG_SHORT, 2, seed=81)
    d = generate(w)
    slow_gates(d, 82)
    ref = oracle_out(d)
    got, _ = run(kda, d, True)
    rel, mx = compare(got, ref, d["cu_seqlens"], w.H)
    assert rel <= RTOL_L2 and mx <= ATOL_MAX, (rel, mx)
    plain, _ = run(kda, d, False)
    cu = d["cu_seqlens"]
    for doc, n in enumerate(LONG_SHORT):
        if n < 2000:
            assert np.array_equal(got[cu[doc]:cu[doc + 1]], plain[cu[doc]:cu[doc + 1]]), doc
    # the cut documents differ from the unsplit forward only by rounding
    for doc in (0, 16):
        a, b = got[cu[doc]:cu[doc + 1]], plain[cu[doc]:cu[doc + 1]]
        assert np.linalg.norm(a - b) / np.linalg.norm(b) < RTOL_L2


def test_workload_gates_every_chain(kda):
    """The same layout with the workloads' gates and betas."""
    w = custom_workload("long_short_g", LONG_SHORT, 2, seed=83)
    d = generate(w)
    ref = oracle_out(d)
    got, _ = run(kda, d, True)
    rel, mx = compare(got, ref, d["cu_seqlens"], w.H)
    assert rel <= RTOL_L2 and mx <= ATOL_MAX, (rel, mx)


def test_initial_and_final_states(kda):
    lens = [2200, 64, 0, 1900, 5]
    w = custom_workload("split_state", lens, 3, seed=84)
    d = generate(w)
    slow_gates(d, 85)
    h0 = (np.random.default_rng(86).normal(size=(len(lens), 3, 128, 128)) * 0.3).astype(np.float32)
    ref, rs = oracle_out(d, initial_state=h0, return_state=True)
    got, ht = run(kda, d, True, h0=h0, final=True)
    rel, mx = compare(got, ref, d["cu_seqlens"], w.H)
    assert rel <= RTOL_L2 and mx <= ATOL_MAX, (rel, mx)
    ht = ht.reshape(-1, 128, 128)
    assert np.linalg.norm(ht - rs) / np.linalg.norm(rs) <= RTOL_L2
    assert np.abs(ht - rs).max() / np.abs(rs).max() <= 5e-2
    # the empty document hands its initial state through unchanged
    assert np.array_equal(ht.reshape(len(lens), 3, 128, 128)[2], h0[2].astype(np.float64))


def test_malformed_seqlens_reported_not_faulted(kda):
    import torch
    w = custom_workload("split_bad", [1600, 64], 2, seed=87)
    d = generate(w)
    t = to_device(d)
    t["cu_seqlens"] = torch.tensor([0, 1700, 1664], dtype=torch.int32, device="cuda")
    kda.kda_chunk_fwd(t["q"], t["k"], t["v"], t["g"], t["beta"], t["cu_seqlens"], split=True)
    with pytest.raises(kda.KdaError) as ei:
        kda.device_status()
    assert ei.value.code == 6
    # the context is still usable
    t["cu_seqlens"] = torch.tensor([0, 1600, 1664], dtype=torch.int32, device="cuda")
    kda.kda_chunk_fwd(t["q"], t["k"], t["v"], t["g"], t["beta"], t["cu_seqlens"], split=True)
    kda.device_status()


def test_repeat_calls_share_a_workspace(kda):
    import torch
    w = custom_workload("split_rep", [4000, 700], 4, seed=88)
    d = generate(w)
    t = to_device(d)
    ws = torch.empty(kda.split_workspace_bytes(2, w.T, 4), dtype=torch.uint8, device="cuda")
    a = kda.kda_chunk_fwd(t["q"], t["k"], t["v"], t["g"], t["beta"], t["cu_seqlens"], split=True, workspace=ws)
    b = kda.kda_chunk_fwd(t["q"], t["k"], t["v"], t["g"], t["beta"], t["cu_seqlens"], split=True, workspace=ws)
    kda.device_status()
    assert torch.equal(a, b)
