"""Shared test helpers: workload -> device tensors, oracle comparison."""
from __future__ import annotations

import numpy as np

import oracle
from chunked_gated_delta_12_b200.inputs import bf16_bits_to_f32

RTOL_L2 = 1e-2      # relative L2 error bound on bf16 outputs
ATOL_MAX = 5e-2     # max absolute error bound on bf16 outputs


def to_device(d: dict):
    import torch
    dev = torch.device("cuda")
    t = {}
    for key in ("q", "k", "v"):
        t[key] = torch.from_numpy(np.ascontiguousarray(d[key]).view(np.int16)).view(torch.bfloat16).to(dev)
    t["g"] = torch.from_numpy(np.ascontiguousarray(d["g"])).to(dev)
    t["beta"] = torch.from_numpy(np.ascontiguousarray(d["beta"])).to(dev)
    t["cu_seqlens"] = torch.from_numpy(np.ascontiguousarray(d["cu_seqlens"], dtype=np.int32)).to(dev)
    if "do" in d:
        t["do"] = torch.from_numpy(np.ascontiguousarray(d["do"]).view(np.int16)).view(torch.bfloat16).to(dev)
    return t


def out_to_f64(o) -> np.ndarray:
    import torch
    bits = o.view(torch.int16).cpu().numpy().view(np.uint16)
    return bf16_bits_to_f32(bits).reshape(bits.shape).astype(np.float64)


def bf16_out(bits_i16: np.ndarray) -> np.ndarray:
    """int16 view of bf16 output bits -> float64."""
    b = np.ascontiguousarray(bits_i16).view(np.uint16)
    return bf16_bits_to_f32(b).reshape(b.shape).astype(np.float64)


def oracle_out(d: dict, chains=None, **kw) -> np.ndarray:
    f = lambda key: bf16_bits_to_f32(d[key]).reshape(d[key].shape)
    return oracle.kda_fwd(f("q"), f("k"), f("v"), d["g"], d["beta"], d["cu_seqlens"], chains=chains, **kw)


def chain_slices(cu, H, chains):
    for ch in chains:
        doc, h = divmod(int(ch), H)
        yield int(cu[doc]), int(cu[doc + 1]), h


def compare(got: np.ndarray, ref: np.ndarray, cu, H, chains=None) -> tuple[float, float]:
    """rel-L2 and max-abs error over the rows of `chains` (all chains if None)."""
    if chains is None:
        chains = range((len(cu) - 1) * H)
    num = den = 0.0
    mx = 0.0
    for s, e, h in chain_slices(cu, H, chains):
        if e == s:
            continue
        a, b = got[s:e, h], ref[s:e, h]
        assert np.isfinite(a).all(), "non-finite output"
        num += float(((a - b) ** 2).sum())
        den += float((b ** 2).sum())
        mx = max(mx, float(np.abs(a - b).max()))
    return (num ** 0.5) / max(den ** 0.5, 1e-300), mx


def oracle_grads(d: dict, chains=None) -> dict:
    """fp64 reverse-mode gradients of the oracle on the exact input values of `d`."""
    f = lambda key: bf16_bits_to_f32(d[key]).reshape(d[key].shape)
    return oracle.kda_bwd(f("q"), f("k"), f("v"), d["g"], d["beta"], f("do"), d["cu_seqlens"], chains=chains)


def compare_grad(got: np.ndarray, ref: np.ndarray, cu, H, chains=None) -> tuple[float, float]:
    """rel-L2 error and max-abs error relative to max |ref|, over the rows of `chains`."""
    if chains is None:
        chains = range((len(cu) - 1) * H)
    num = den = mx = top = 0.0
    for s, e, h in chain_slices(cu, H, chains):
        if e == s:
            continue
        a, b = got[s:e, h], ref[s:e, h]
        assert np.isfinite(a).all(), "non-finite gradient"
        num += float(((a - b) ** 2).sum())
        den += float((b ** 2).sum())
        mx = max(mx, float(np.abs(a - b).max()))
        top = max(top, float(np.abs(b).max()))
    return (num / den) ** 0.5 if den > 0 else num ** 0.5, mx / top if top > 0 else mx
