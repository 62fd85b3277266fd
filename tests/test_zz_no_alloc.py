"""kda_chunk_bwd_noalloc: the backward for callers that cannot allocate device memory.

Some callers cannot call cudaMalloc when they run the backward: their device memory belongs to
another allocator (a framework's caching pool that has already reserved the free memory), or
they must not allocate after start-up because cudaMalloc and cudaFree synchronise the device.
kda_chunk_bwd_noalloc serves them with a fixed scratch array held in the library's device
image instead of a caller-owned workspace.  These tests call it through the C ABI and check
that it gives exactly what kda_chunk_bwd gives (the same kernel on the same inputs, so the
gradients must be bit-identical), on two calls in a row (the second one of another size, so that
it starts from the first call's leftover scratch), that the first call's gradients also meet the
fp64 reverse-mode oracle, and that sizes beyond the array are rejected on the host.

This file is named to be collected last: if its GPU test fails, a run that stops at the first
failure has already run every other test.
"""
import ctypes

import numpy as np
import pytest

from chunked_gated_delta_12_b200 import _lib
from chunked_gated_delta_12_b200.build import build
from chunked_gated_delta_12_b200.inputs import custom_workload, generate
from tests.helpers import compare_grad, oracle_grads, out_to_f64, to_device

# the bar of the other backward tests against the oracle: rel-L2 <= 1e-2, max-abs <= 5e-2 of
# max |reference|
RTOL_L2 = 1e-2
RMAX = 5e-2


def test_rejects_sizes_beyond_the_scratch_on_the_host():
    """Checked before any device work (CPU): a call that needs more scratch than the array holds
    is refused with a message naming the sizes; pointers are never dereferenced."""
    build()
    L = _lib.lib()
    n_docs, T, H = 1, 4096, 32
    assert L.kda_chunk_bwd_workspace_size(n_docs, T, H) > _lib.NOALLOC_SCRATCH_BYTES
    fake = ctypes.c_void_p(0x10000000)
    rc = L.kda_chunk_bwd_noalloc(fake, fake, fake, fake, fake, fake, n_docs, T, H, fake, fake, fake, fake, fake,
                                 fake, None)
    assert rc == 1
    msg = L.kda_last_error()
    assert b"scratch" in msg and b"T=4096" in msg and b"H=32" in msg
    # a size that fits: 1 document of 2048 tokens with 8 heads (the example the header gives)
    assert L.kda_chunk_bwd_workspace_size(1, 2048, 8) <= _lib.NOALLOC_SCRATCH_BYTES
    # the size arguments are checked as kda_chunk_bwd checks them
    assert L.kda_chunk_bwd_noalloc(fake, fake, fake, fake, fake, fake, 0, 64, 1, fake, fake, fake, fake, fake,
                                   fake, None) == 1
    assert b"n_docs" in L.kda_last_error()


def _grads_host(grads):
    dq, dk, dv, dg, db = grads
    return dict(dq=out_to_f64(dq), dk=out_to_f64(dk), dv=out_to_f64(dv),
                dg=dg.cpu().numpy().astype(np.float64), dbeta=db.cpu().numpy().astype(np.float64))


def _bits(grads):
    import torch
    return [x.view(torch.int32 if x.dtype == torch.float32 else torch.int16).cpu().numpy() for x in grads]


@pytest.mark.gpu
def test_noalloc_matches_kda_chunk_bwd_on_two_calls_in_a_row():
    import torch
    import chunked_gated_delta_12_b200 as kda
    torch.cuda.init()
    cases = [custom_workload("noalloc_a", [1000, 63, 65, 0, 200], 4, seed=71),
             custom_workload("noalloc_b", [130, 64, 1], 2, seed=72)]
    for i, w in enumerate(cases):
        d = generate(w, with_grad=True)
        assert _lib.bwd_workspace_bytes(len(d["cu_seqlens"]) - 1, int(d["cu_seqlens"][-1]), w.H) \
            <= kda.NOALLOC_SCRATCH_BYTES
        t = to_device(d)
        ref = kda.kda_chunk_bwd(t["q"], t["k"], t["v"], t["g"], t["beta"], t["cu_seqlens"], t["do"])
        kda.device_status()
        outs = (torch.full_like(t["q"], float("nan")), torch.full_like(t["k"], float("nan")),
                torch.full_like(t["v"], float("nan")), torch.full_like(t["g"], float("nan")),
                torch.full_like(t["beta"], float("nan")))
        kda.kda_chunk_bwd_noalloc(t["q"], t["k"], t["v"], t["g"], t["beta"], t["cu_seqlens"], t["do"], *outs)
        kda.device_status()
        torch.cuda.synchronize()
        # the same kernel on the same inputs: every gradient bit-identical (a stale scratch value
        # read anywhere would show here)
        for name, a, b in zip(("dq", "dk", "dv", "dg", "dbeta"), _bits(outs), _bits(ref)):
            assert np.array_equal(a, b), (w.name, name)
        if i == 0:
            # and the gradients themselves meet the fp64 reverse mode of the token recurrence
            got, exp = _grads_host(outs), oracle_grads(d)
            cu = d["cu_seqlens"]
            for n in ("dq", "dk", "dv", "dg"):
                rel, mx = compare_grad(got[n], exp[n], cu, w.H)
                assert rel <= RTOL_L2 and mx <= RMAX, (w.name, n, rel, mx)
            rel, mx = compare_grad(got["dbeta"][..., None], exp["dbeta"][..., None], cu, w.H)
            assert rel <= RTOL_L2 and mx <= RMAX, (w.name, "dbeta", rel, mx)
