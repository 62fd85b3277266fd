"""Seeded synthetic inputs for chunk-KDA workloads.

This module only draws random numbers and lays them out; it holds none of the
KDA arithmetic.  Both the CUDA path (tests, bench) and the CPU oracle read the
same arrays from here, so a parity failure can never come from two generators
disagreeing.

Layout (batch-1 packed documents, as the kda_fused page of
nemo_automodel.components.models.kimi_k3 specifies for its fused kernels):

* q, k, v : [T, H, 128] bf16, stored as uint16 bit patterns (RNE from fp32 draws)
* g       : [T, H, 128] fp32 per-key-channel log decay, -5*sigmoid(N(0,1)) in (-5, 0)
* beta    : [T, H] fp32, sigmoid(N(0,1))
* cu_seqlens : [n_docs + 1] int32, cu[0] = 0, cu[n_docs] = T
* do      : [T, H, 128] bf16 upstream gradient (backward workloads only)

Every tensor has its own stream: numpy's PCG64 seeded with (seed, tensor_id),
seed = 20260 + workload index.
"""
from __future__ import annotations

from concurrent.futures import ThreadPoolExecutor
from dataclasses import dataclass

import numpy as np

HEAD_DIM = 128

_TENSOR_IDS = {"q": 1, "k": 2, "v": 3, "g": 4, "beta": 5, "lengths": 6, "do": 7}


def _rng(seed: int, name: str) -> np.random.Generator:
    return np.random.default_rng([seed, _TENSOR_IDS[name]])


def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round fp32 to bf16 (round-to-nearest-even); returns uint16 bit patterns.  Finite inputs
    only: the 32-bit sum below cannot wrap for any finite value (largest 0xFF7FFFFF + 0x8000)."""
    b = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    rounded = (b + np.uint32(0x7FFF) + ((b >> np.uint32(16)) & np.uint32(1))) >> np.uint32(16)
    return rounded.astype(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    """Exact widening of bf16 bit patterns to fp32."""
    return (np.ascontiguousarray(b, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


def _normal_f32(rng: np.random.Generator, n: int) -> np.ndarray:
    return rng.standard_normal(n, dtype=np.float32)


def _sigmoid(z: np.ndarray) -> np.ndarray:
    return (1.0 / (1.0 + np.exp(-z.astype(np.float64))))


@dataclass
class Workload:
    """One synthetic chunk-KDA forward (and optionally backward) problem."""

    name: str
    seed: int
    lengths: list[int]
    H: int
    with_grad: bool = False

    @property
    def T(self) -> int:
        return int(sum(self.lengths))

    @property
    def n_docs(self) -> int:
        return len(self.lengths)

    def cu_seqlens(self) -> np.ndarray:
        cu = np.zeros(self.n_docs + 1, dtype=np.int32)
        cu[1:] = np.cumsum(np.asarray(self.lengths, dtype=np.int64))
        return cu

    def describe(self) -> dict:
        return {
            "workload": self.name,
            "n_docs": self.n_docs,
            "T": self.T,
            "H": self.H,
            "K": HEAD_DIM,
            "V": HEAD_DIM,
            "seed": self.seed,
        }


def _lengths_uniform_to_sum(rng: np.random.Generator, n: int, lo: int, hi: int,
                            total: int, avoid_all_multiple_of: int | None) -> list[int]:
    """Draw n ints in [lo, hi], rescale to sum exactly to `total`, staying in [max(lo,1), hi].

    The residual left by flooring is spread one token at a time over documents in
    order, cycling, never leaving the bounds.
    """
    lo_b = max(lo, 1)
    while True:
        raw = rng.integers(lo, hi + 1, size=n).astype(np.int64)
        scaled = np.floor(raw * (total / raw.sum())).astype(np.int64)
        scaled = np.clip(scaled, lo_b, hi)
        resid = total - int(scaled.sum())
        i = 0
        guard = 0
        while resid != 0:
            step = 1 if resid > 0 else -1
            nv = scaled[i % n] + step
            if lo_b <= nv <= hi:
                scaled[i % n] = nv
                resid -= step
            i += 1
            guard += 1
            if guard > 100 * total:
                raise RuntimeError("cannot meet the length sum within bounds")
        if avoid_all_multiple_of and all(int(x) % avoid_all_multiple_of == 0 for x in scaled):
            continue
        return [int(x) for x in scaled]


def workload(index: int) -> Workload:
    """The five synthetic chunk-KDA workloads, by index.

    0: one document T=256, H=2 (small; the oracle finishes in well under a second)
    1: 8 packed documents of random length summing to 4096, H=8
    2: dense batch 4 x 8192 viewed as 4 packed documents, H=32 (throughput headline)
    3: one long document T=65536, H=32
    4: 16 packed documents, lengths in [512, 4096] summing to 32768, H=32, with dO
    """
    seed = 20260 + index
    if index == 0:
        return Workload("single_doc_T256_H2", seed, [256], 2)
    if index == 1:
        lens = _lengths_uniform_to_sum(_rng(seed, "lengths"), 8, 1, 1000, 4096, 64)
        return Workload("packed_8docs_T4096_H8", seed, lens, 8)
    if index == 2:
        return Workload("dense_4x8192_H32", seed, [8192] * 4, 32)
    if index == 3:
        return Workload("single_doc_T65536_H32", seed, [65536], 32)
    if index == 4:
        lens = _lengths_uniform_to_sum(_rng(seed, "lengths"), 16, 512, 4096, 32768, None)
        return Workload("packed_16docs_T32768_H32", seed, lens, 32, with_grad=True)
    raise ValueError(f"no workload {index}")


def custom_workload(name: str, lengths: list[int], H: int, seed: int = 777) -> Workload:
    return Workload(name, seed, list(lengths), H)


def generate(w: Workload, with_grad: bool | None = None) -> dict[str, np.ndarray]:
    """Draw the tensors of workload `w` (host numpy arrays, layouts in the module doc)."""
    T, H, d = w.T, w.H, HEAD_DIM
    n = T * H * d

    def draw(name: str) -> np.ndarray:
        if name == "g":
            return (-5.0 * _sigmoid(_normal_f32(_rng(w.seed, "g"), n))).astype(np.float32).reshape(T, H, d)
        if name == "beta":
            return _sigmoid(_normal_f32(_rng(w.seed, "beta"), T * H)).astype(np.float32).reshape(T, H)
        return f32_to_bf16_bits(_normal_f32(_rng(w.seed, name), n)).reshape(T, H, d)

    names = ["q", "k", "v", "g", "beta"]
    if with_grad if with_grad is not None else w.with_grad:
        names.append("do")
    # every tensor has its own random stream, so drawing them side by side (numpy releases the
    # interpreter lock inside these loops) gives the same arrays as drawing them in turn
    with ThreadPoolExecutor(max_workers=len(names)) as ex:
        arrays = list(ex.map(draw, names))
    out: dict[str, np.ndarray] = dict(zip(names, arrays))
    out["cu_seqlens"] = w.cu_seqlens()
    return out
