"""Token-by-token forward (kda_recurrent_fwd) vs the fp64 oracle, through the C ABI (gpu).

Bar: outputs rel-L2 <= 1e-2 and max-abs <= 5e-2 as in test_parity_gpu; final states rel-L2 <= 1e-2
and max-abs <= 5e-2 of their largest magnitude; isolation and coverage bit-exact.
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


def run(kda, d, h0=None, final=True, out=None, fn="kda_recurrent_fwd"):
    import torch
    t = to_device(d)
    h0_t = None if h0 is None else torch.from_numpy(h0).cuda()
    r = getattr(kda, fn)(t["q"], t["k"], t["v"], t["g"], t["beta"], t["cu_seqlens"], out=out, initial_state=h0_t,
                         output_final_state=final)
    kda.device_status()
    torch.cuda.synchronize()
    o, ht = r if final else (r, None)
    return o, (None if ht is None else ht.cpu().numpy().astype(np.float64))


def check_state(got, ref):
    rel = np.linalg.norm(got - ref) / np.linalg.norm(ref)
    mx = np.abs(got - ref).max() / np.abs(ref).max()
    assert rel <= RTOL_L2 and mx <= 5e-2, (rel, mx)


@pytest.mark.parametrize("lens,H,with_h0", [([1] * 64, 8, True), ([1] * 64, 8, False),
                                            ([1, 2, 5, 17, 0, 64, 100], 3, True),
                                            ([300], 2, False)])
def test_recurrent_matches_oracle(kda, lens, H, with_h0):
    w = custom_workload("rec", lens, H, seed=61)
    d = generate(w)
    h0 = states(w.n_docs, H, 62) if with_h0 else None
    o, ht = run(kda, d, h0)
    ref, rs = oracle_out(d, initial_state=h0, return_state=True)
    rel, mx = compare(out_to_f64(o), ref, d["cu_seqlens"], H)
    assert rel <= RTOL_L2 and mx <= ATOL_MAX, (rel, mx)
    check_state(ht.reshape(-1, 128, 128), rs)
    for doc, L in enumerate(lens):
        if L == 0:
            want = h0[doc].astype(np.float64) if h0 is not None else np.zeros((H, 128, 128))
            assert np.array_equal(ht[doc], want)


def test_decode_after_chunked_prefill(kda):
    """Prefill with the chunked kernel (final state out), then decode 3 tokens per document one
    at a time with the recurrent kernel updating the state in place; the decoded outputs and the
    state equal the oracle run over the whole documents."""
    import torch
    prefill, n_dec, H = [300, 1000, 65, 1, 0], 3, 4
    lens = [L + n_dec for L in prefill]
    w = custom_workload("decode", lens, H, seed=63)
    d = generate(w)
    cu = d["cu_seqlens"]
    ref, rs = oracle_out(d, return_state=True)
    pre_idx = np.concatenate([np.arange(cu[i], cu[i] + L) for i, L in enumerate(prefill)])
    take = lambda idx, cu_new: {**{k: d[k][idx] for k in ("q", "k", "v", "g", "beta")},
                                "cu_seqlens": np.asarray(cu_new, np.int32)}
    dp = take(pre_idx, np.concatenate([[0], np.cumsum(prefill)]))
    tp = to_device(dp)
    _, state = kda.kda_chunk_fwd(tp["q"], tp["k"], tp["v"], tp["g"], tp["beta"], tp["cu_seqlens"],
                                 output_final_state=True)
    n = len(lens)
    for j in range(n_dec):
        idx = np.array([cu[i] + prefill[i] + j for i in range(n)])
        dj = take(idx, np.arange(n + 1))
        tj = to_device(dj)
        o = kda.kda_recurrent_fwd(tj["q"], tj["k"], tj["v"], tj["g"], tj["beta"], tj["cu_seqlens"],
                                  initial_state=state, final_state=state)[0]
        kda.device_status()
        got = out_to_f64(o)
        want = ref[idx]
        rel = np.linalg.norm(got - want) / np.linalg.norm(want)
        assert rel <= RTOL_L2 and np.abs(got - want).max() <= ATOL_MAX, (j, rel)
    torch.cuda.synchronize()
    check_state(state.cpu().numpy().astype(np.float64).reshape(-1, 128, 128), rs)


def test_recurrent_and_chunked_agree_on_short_documents(kda):
    import torch
    lens, H = [1, 2, 3, 4, 8, 16, 31, 64, 65], 4
    w = custom_workload("agree", lens, H, seed=64)
    d = generate(w)
    h0 = states(w.n_docs, H, 65)
    o_r, s_r = run(kda, d, h0)
    o_c, s_c = run(kda, d, h0, fn="kda_chunk_fwd")
    a, b = out_to_f64(o_r), out_to_f64(o_c)
    rel = np.linalg.norm(a - b) / np.linalg.norm(b)
    assert rel <= RTOL_L2 and np.abs(a - b).max() <= ATOL_MAX, rel
    check_state(s_r, s_c)
    del torch


def test_recurrent_isolation_bitwise_and_full_coverage(kda):
    import torch
    lens = [1, 65, 3, 1, 20]
    w = custom_workload("riso", lens, 2, seed=66)
    d = generate(w)
    cu = d["cu_seqlens"]
    T, H = w.T, w.H
    guard = 4096
    buf = torch.full((guard + T * H * 128 + guard,), float("nan"), dtype=torch.bfloat16, device="cuda")
    out = buf[guard:guard + T * H * 128].view(T, H, 128)
    base, _ = run(kda, d, final=False, out=out)
    base = base.clone()
    assert not torch.isnan(base).any(), "some output row was not written"
    assert torch.isnan(buf[:guard]).all() and torch.isnan(buf[-guard:]).all(), "write outside out"
    base_np = base.view(torch.int16).cpu().numpy()
    for victim in range(1, len(lens)):
        e = {k: v.copy() for k, v in d.items()}
        s0, s1 = int(cu[victim]), int(cu[victim + 1])
        e["q"][s0:s1] = 0x7FC0                      # bf16 NaN
        e["k"][s0:s1] = 0x7F80                      # bf16 +Inf
        e["v"][s0:s1] ^= 0x1234
        e["g"][s0:s1] = np.nan
        e["beta"][s0:s1] = 0.77
        got = run(kda, e, final=False)[0].view(torch.int16).cpu().numpy()
        assert np.array_equal(got[:s0], base_np[:s0]), f"doc {victim} leaked backwards"
        assert np.array_equal(got[s1:], base_np[s1:]), f"doc {victim} leaked forwards"


def test_recurrent_in_place_state_and_no_tokens(kda):
    import torch
    w = custom_workload("rinplace", [5, 1], 2, seed=67)
    d = generate(w)
    h0 = states(w.n_docs, 2, 68)
    _, ht_ref = run(kda, d, h0)
    t = to_device(d)
    buf = torch.from_numpy(h0).cuda()
    kda.kda_recurrent_fwd(t["q"], t["k"], t["v"], t["g"], t["beta"], t["cu_seqlens"], initial_state=buf,
                          final_state=buf)
    kda.device_status()
    assert np.array_equal(buf.cpu().numpy().astype(np.float64), ht_ref)
    w0 = custom_workload("rempty", [0, 0], 2, seed=69)
    t0 = to_device(generate(w0))
    o, ht = kda.kda_recurrent_fwd(t0["q"], t0["k"], t0["v"], t0["g"], t0["beta"], t0["cu_seqlens"],
                                  initial_state=torch.from_numpy(h0).cuda(), output_final_state=True)
    torch.cuda.synchronize()
    assert np.array_equal(ht.cpu().numpy(), h0)


def test_recurrent_malformed_seqlens_reported(kda):
    import torch
    w = custom_workload("rbad", [4, 4, 4], 1, seed=70)
    t = to_device(generate(w))
    for bad in ([0, 8, 2, 12], [0, 4, 8, 500], [3, 4, 8, 12]):
        t["cu_seqlens"] = torch.tensor(bad, dtype=torch.int32, device="cuda")
        kda.kda_recurrent_fwd(t["q"], t["k"], t["v"], t["g"], t["beta"], t["cu_seqlens"])
        with pytest.raises(kda.KdaError) as ei:
            kda.device_status()
        assert ei.value.code == 6
    t["cu_seqlens"] = torch.tensor([0, 4, 8, 12], dtype=torch.int32, device="cuda")
    kda.kda_recurrent_fwd(t["q"], t["k"], t["v"], t["g"], t["beta"], t["cu_seqlens"])
    kda.device_status()
