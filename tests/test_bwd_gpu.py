"""CUDA backward (kda_chunk_bwd) vs the fp64 reverse-mode oracle, through the C ABI (gpu).

Bar for every gradient (dq, dk, dv bf16; dg, dbeta fp32): relative L2 error <= 1e-2 and max
absolute error <= 5e-2 of the largest reference magnitude, over the compared rows; document
isolation bit-exact.
"""
import numpy as np
import pytest

from chunked_gated_delta_12_b200.inputs import custom_workload, generate, workload
from tests.helpers import compare_grad, oracle_grads, out_to_f64, to_device

pytestmark = pytest.mark.gpu

RTOL_L2 = 1e-2
RMAX = 5e-2


@pytest.fixture(scope="module")
def kda():
    import torch
    import chunked_gated_delta_12_b200 as m
    torch.cuda.init()
    return m


def run_bwd(kda, d):
    import torch
    t = to_device(d)
    grads = kda.kda_chunk_bwd(t["q"], t["k"], t["v"], t["g"], t["beta"], t["cu_seqlens"], t["do"])
    kda.device_status()
    torch.cuda.synchronize()
    dq, dk, dv, dg, db = grads
    return dict(dq=out_to_f64(dq), dk=out_to_f64(dk), dv=out_to_f64(dv),
                dg=dg.cpu().numpy().astype(np.float64), dbeta=db.cpu().numpy().astype(np.float64)), grads


def check(got, ref, cu, H, chains=None):
    for n in ("dq", "dk", "dv", "dg"):
        rel, mx = compare_grad(got[n], ref[n], cu, H, chains)
        assert rel <= RTOL_L2 and mx <= RMAX, (n, rel, mx)
    rel, mx = compare_grad(got["dbeta"][..., None], ref["dbeta"][..., None], cu, H, chains)
    assert rel <= RTOL_L2 and mx <= RMAX, ("dbeta", rel, mx)


def test_single_document_all_chains(kda):
    w = workload(0)
    d = generate(w, with_grad=True)
    got, _ = run_bwd(kda, d)
    check(got, oracle_grads(d), d["cu_seqlens"], w.H)


def test_edge_lengths_and_empty_docs(kda):
    w = custom_workload("bwd_edges", [1, 63, 64, 0, 65, 129, 2], 2, seed=41)
    d = generate(w, with_grad=True)
    got, _ = run_bwd(kda, d)
    check(got, oracle_grads(d), d["cu_seqlens"], w.H)


def test_many_short_documents(kda):
    """More documents than the grid ranks longest-first (256), including empty ones: every chain is
    computed once, in index order."""
    w = custom_workload("bwd_many", [(5 * i) % 7 for i in range(260)], 1, seed=43)
    d = generate(w, with_grad=True)
    got, _ = run_bwd(kda, d)
    check(got, oracle_grads(d), d["cu_seqlens"], w.H)


def test_packed_forward_backward_workload_all_chains(kda):
    """16 packed documents, H = 32 (the forward + backward workload); the oracle recomputes the
    gradients of all 512 (document, head) chains."""
    w = workload(4)
    d = generate(w, with_grad=True)
    got, _ = run_bwd(kda, d)
    check(got, oracle_grads(d), d["cu_seqlens"], w.H)


def test_poisoned_workspace_gives_the_same_gradients(kda):
    """The backward sets every workspace value it reads: a workspace filled with NaN bytes gives
    gradients bit-identical to those of a zeroed one, on a layout with an empty document and
    lengths that are not multiples of 64."""
    import torch
    w = custom_workload("bwd_poison", [130, 0, 77, 64, 1], 3, seed=44)
    d = generate(w, with_grad=True)
    t = to_device(d)
    need = kda.bwd_workspace_bytes(w.n_docs, w.T, w.H)
    outs = []
    for fill in (0x00, 0xFF):
        ws = torch.full((need,), fill, dtype=torch.uint8, device="cuda")
        g = kda.kda_chunk_bwd(t["q"], t["k"], t["v"], t["g"], t["beta"], t["cu_seqlens"], t["do"], workspace=ws)
        kda.device_status()
        torch.cuda.synchronize()
        for x in g:
            assert torch.isfinite(x.float()).all()
        outs.append([x.view(torch.int32 if x.dtype == torch.float32 else torch.int16).cpu().numpy() for x in g])
    for a, b in zip(*outs):
        assert np.array_equal(a, b)


def test_document_isolation_bitwise(kda):
    import torch
    lens = [65, 64, 30]
    w = custom_workload("bwd_iso", lens, 2, seed=42)
    d = generate(w, with_grad=True)
    cu = d["cu_seqlens"]
    _, base = run_bwd(kda, d)
    base = [x.view(torch.int32 if x.dtype == torch.float32 else torch.int16).cpu().numpy() for x in base]
    s0, s1 = int(cu[1]), int(cu[2])
    e = {k: (v.copy() if isinstance(v, np.ndarray) else v) for k, v in d.items()}
    e["q"][s0:s1] = 0x7FC0
    e["k"][s0:s1] = 0x7F80
    e["v"][s0:s1] ^= 0x1234
    e["g"][s0:s1] = np.nan
    e["beta"][s0:s1] = 0.3
    e["do"][s0:s1] = 0x7FC0
    _, got = run_bwd(kda, e)
    got = [x.view(torch.int32 if x.dtype == torch.float32 else torch.int16).cpu().numpy() for x in got]
    for a, b in zip(got, base):
        assert np.array_equal(a[:s0], b[:s0]) and np.array_equal(a[s1:], b[s1:])


def test_workspace_too_small_is_rejected(kda):
    import torch
    w = workload(0)
    d = generate(w, with_grad=True)
    t = to_device(d)
    ws = torch.empty(1024, dtype=torch.uint8, device="cuda")
    with pytest.raises(kda.KdaError) as ei:
        kda.kda_chunk_bwd(t["q"], t["k"], t["v"], t["g"], t["beta"], t["cu_seqlens"], t["do"], workspace=ws)
    assert ei.value.code == 1
