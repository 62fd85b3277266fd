"""CUDA path vs the fp64 oracle, through the C ABI (gpu).

Bar: relative L2 error <= 1e-2 and max abs error <= 5e-2 on the bf16 outputs;
cu_seqlens indexing and document isolation bit-exact.
"""
import numpy as np
import pytest

from chunked_gated_delta_12_b200.inputs import custom_workload, generate, workload
from tests.helpers import ATOL_MAX, RTOL_L2, bf16_out, compare, oracle_out, out_to_f64, to_device

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def kda():
    import torch
    import chunked_gated_delta_12_b200 as m
    torch.cuda.init()
    return m


def run(kda, d, out=None):
    import torch
    t = to_device(d)
    o = kda.kda_chunk_fwd(t["q"], t["k"], t["v"], t["g"], t["beta"], t["cu_seqlens"], out=out)
    kda.device_status()
    torch.cuda.synchronize()
    return o


@pytest.mark.parametrize("idx", [0, 1])
def test_small_workloads_all_chains(kda, idx):
    w = workload(idx)
    d = generate(w)
    got = out_to_f64(run(kda, d))
    ref = oracle_out(d)
    rel, mx = compare(got, ref, d["cu_seqlens"], w.H)
    assert rel <= RTOL_L2 and mx <= ATOL_MAX, (rel, mx)


@pytest.mark.parametrize("idx", [2, 3, 4])
def test_full_size_all_chains(kda, idx):
    """Full-size workloads in the benchmark's launch configuration (dense 4 x 8192, one document of
    65536 tokens, 16 packed documents; H = 32): the oracle recomputes every (document, head) chain
    and every output row is compared."""
    w = workload(idx)
    d = generate(w)
    got = out_to_f64(run(kda, d))
    assert np.isfinite(got).all()
    ref = oracle_out(d)
    rel, mx = compare(got, ref, d["cu_seqlens"], w.H)
    assert rel <= RTOL_L2 and mx <= ATOL_MAX, (rel, mx)


def test_edge_lengths_and_empty_docs(kda):
    lens = [1, 63, 64, 0, 65, 127, 128, 129, 2, 0]
    w = custom_workload("edges", lens, 3, seed=31)
    d = generate(w)
    got = out_to_f64(run(kda, d))
    ref = oracle_out(d)
    rel, mx = compare(got, ref, d["cu_seqlens"], w.H)
    assert rel <= RTOL_L2 and mx <= ATOL_MAX, (rel, mx)


def test_many_chains(kda):
    """60 documents x 2 heads: 120 chains, several waves of CTAs."""
    lens = [70] * 60
    w = custom_workload("many", lens, 2, seed=32)
    d = generate(w)
    got = out_to_f64(run(kda, d))
    ref = oracle_out(d, chains=list(range(0, 120, 7)))
    rel, mx = compare(got, ref, d["cu_seqlens"], w.H, list(range(0, 120, 7)))
    assert rel <= RTOL_L2 and mx <= ATOL_MAX, (rel, mx)


@pytest.mark.parametrize("gval", [-5.0, 0.0])
def test_extreme_gates(kda, gval):
    w = custom_workload("gate", [200, 77], 2, seed=33)
    d = generate(w)
    d["g"][:] = np.float32(gval)
    got = out_to_f64(run(kda, d))
    ref = oracle_out(d)
    rel, mx = compare(got, ref, d["cu_seqlens"], w.H)
    assert rel <= RTOL_L2 and mx <= ATOL_MAX, (rel, mx)


def test_beta_zero_gives_exact_zeros(kda):
    w = custom_workload("b0", [100, 30], 2, seed=34)
    d = generate(w)
    d["beta"][:] = 0.0
    got = out_to_f64(run(kda, d))
    assert np.all(got == 0.0)


def test_document_isolation_bitwise_and_full_coverage(kda):
    """Poisoning document d+1 (NaN/Inf, other values) leaves document d's
    output bit-identical; every output row is written exactly inside [0, T)."""
    import torch
    lens = [65, 129, 64, 1, 127]
    w = custom_workload("iso", lens, 2, seed=35)
    d = generate(w)
    cu = d["cu_seqlens"]
    T, H = w.T, w.H
    guard = 4096
    buf = torch.full((guard + T * H * 128 + guard,), float("nan"), dtype=torch.bfloat16, device="cuda")
    out = buf[guard:guard + T * H * 128].view(T, H, 128)
    base = run(kda, d, out=out).clone()
    assert not torch.isnan(base).any(), "some output row was not written"
    assert torch.isnan(buf[:guard]).all() and torch.isnan(buf[-guard:]).all(), "write outside out"
    base_np = base.view(torch.int16).cpu().numpy()
    for victim in range(1, len(lens)):
        e = dict(d)
        s0, s1 = int(cu[victim]), int(cu[victim + 1])
        e["q"] = d["q"].copy(); e["k"] = d["k"].copy(); e["v"] = d["v"].copy()
        e["g"] = d["g"].copy(); e["beta"] = d["beta"].copy()
        e["q"][s0:s1] = 0x7FC0                      # bf16 NaN
        e["k"][s0:s1] = 0x7F80                      # bf16 +Inf
        e["v"][s0:s1] ^= 0x1234
        e["g"][s0:s1] = np.nan
        e["beta"][s0:s1] = 0.77
        got = run(kda, e).view(torch.int16).cpu().numpy()
        assert np.array_equal(got[:s0], base_np[:s0]), f"doc {victim} leaked backwards"
        assert np.array_equal(got[s1:], base_np[s1:]), f"doc {victim} leaked forwards"


def test_deterministic(kda):
    import torch
    w = workload(1)
    d = generate(w)
    a = run(kda, d).view(torch.int16).cpu().numpy()
    b = run(kda, d).view(torch.int16).cpu().numpy()
    assert np.array_equal(a, b)


def test_malformed_seqlens_reported_not_faulted(kda):
    """A bad cu_seqlens table is caught on the device (no out-of-range access)
    and reported by kda_device_status."""
    import torch
    w = custom_workload("bad", [64, 64, 64], 1, seed=36)
    d = generate(w)
    t = to_device(d)
    for bad in ([0, 100, 50, 192], [0, 64, 128, 500], [5, 64, 128, 192]):
        t["cu_seqlens"] = torch.tensor(bad, dtype=torch.int32, device="cuda")
        kda.kda_chunk_fwd(t["q"], t["k"], t["v"], t["g"], t["beta"], t["cu_seqlens"])
        with pytest.raises(kda.KdaError) as ei:
            kda.device_status()
        assert ei.value.code == 6
    # the context is still usable and the status word was cleared
    t["cu_seqlens"] = torch.tensor([0, 64, 128, 192], dtype=torch.int32, device="cuda")
    kda.kda_chunk_fwd(t["q"], t["k"], t["v"], t["g"], t["beta"], t["cu_seqlens"])
    kda.device_status()


def test_rejects_wrong_dtype(kda):
    import torch
    x = torch.zeros(64, 1, 128, device="cuda", dtype=torch.float16)
    g = torch.zeros(64, 1, 128, device="cuda")
    b = torch.zeros(64, 1, device="cuda")
    cu = torch.tensor([0, 64], dtype=torch.int32, device="cuda")
    with pytest.raises(kda.KdaError):
        kda.kda_chunk_fwd(x, x, x, g, b, cu)


def test_pipelined_path_isolation_bitwise(kda):
    """Same isolation check on a launch with 128 chains: the TMA tiles read
    past document ends, so poisoned rows of the next document must be zeroed,
    never used."""
    import torch
    lens = [1, 64, 65, 129, 63, 200, 64, 14]
    w = custom_workload("iso_pipe", lens, 16, seed=37)       # 8 docs x 16 heads = 128 chains
    d = generate(w)
    cu = d["cu_seqlens"]
    T, H = w.T, w.H
    guard = 4096
    buf = torch.full((guard + T * H * 128 + guard,), float("nan"), dtype=torch.bfloat16, device="cuda")
    out = buf[guard:guard + T * H * 128].view(T, H, 128)
    run(kda, d, out=out)
    assert not torch.isnan(out).any(), "some output row was not written"
    assert torch.isnan(buf[:guard]).all() and torch.isnan(buf[-guard:]).all(), "write outside out"
    base = out.view(torch.int16).cpu().numpy()
    ref = oracle_out(d, chains=list(range(0, 128, 5)))
    rel, mx = compare(bf16_out(base), ref, cu, w.H, list(range(0, 128, 5)))
    assert rel <= RTOL_L2 and mx <= ATOL_MAX, (rel, mx)
    for victim in (1, 3, 6):
        e = dict(d)
        s0, s1 = int(cu[victim]), int(cu[victim + 1])
        for key in ("q", "k", "v", "g", "beta"):
            e[key] = d[key].copy()
        e["q"][s0:s1] = 0x7FC0
        e["k"][s0:s1] = 0x7F80
        e["v"][s0:s1] = 0x7FC0
        e["g"][s0:s1] = np.nan
        e["beta"][s0:s1] = np.inf
        got = run(kda, e).view(torch.int16).cpu().numpy()
        assert np.array_equal(got[:s0], base[:s0]), f"doc {victim} leaked backwards"
        assert np.array_equal(got[s1:], base[s1:]), f"doc {victim} leaked forwards"


@pytest.mark.parametrize("lens", [[64] * 8, [1] * 8, [65, 63, 128, 127, 1, 64, 192, 2]])
def test_pipelined_path_lengths(kda, lens):
    """Chunk-aligned, single-token and mixed documents on the pipelined kernel."""
    w = custom_workload("pipe_lens", lens, 16, seed=38)
    d = generate(w)
    got = out_to_f64(run(kda, d))
    chains = list(range(0, 8 * 16, 3))
    ref = oracle_out(d, chains=chains)
    rel, mx = compare(got, ref, d["cu_seqlens"], w.H, chains)
    assert rel <= RTOL_L2 and mx <= ATOL_MAX, (rel, mx)


def test_device_wait_timeout_is_reported_and_context_survives(kda):
    """A device wait that can never complete gives up, reports KDA_ERR_TIMEOUT
    through kda_device_status, and the next forward runs normally."""
    kda.wait_selftest()
    with pytest.raises(kda.KdaError) as ei:
        kda.device_status()
    assert ei.value.code == 5
    kda.device_status()                      # cleared
    w = workload(0)
    d = generate(w)
    got = out_to_f64(run(kda, d))
    ref = oracle_out(d)
    rel, mx = compare(got, ref, d["cu_seqlens"], w.H)
    assert rel <= RTOL_L2 and mx <= ATOL_MAX, (rel, mx)


def test_host_entry_point_matches_device_call(kda):
    """kda_chunk_fwd_host (pinned host inputs and output, device workspace, copies on the stream) gives
    the bytes kda_chunk_fwd gives on the same inputs (8 packed documents of ragged lengths, H = 8)."""
    import torch
    w = workload(1)
    d = generate(w)
    t = to_device(d)
    want = kda.kda_chunk_fwd(t["q"], t["k"], t["v"], t["g"], t["beta"], t["cu_seqlens"], split=False)
    h = {key: x.cpu().pin_memory() for key, x in t.items()}
    out = torch.empty(want.shape, dtype=torch.bfloat16).pin_memory()
    ws = torch.empty(kda.host_workspace_bytes(w.n_docs, w.T, w.H), dtype=torch.uint8, device="cuda")
    kda.kda_chunk_fwd_host(h["q"], h["k"], h["v"], h["g"], h["beta"], h["cu_seqlens"], out, ws)
    kda.device_status()
    torch.cuda.synchronize()
    assert torch.equal(out.view(torch.int16), want.view(torch.int16).cpu())
