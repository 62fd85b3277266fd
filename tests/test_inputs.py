"""The seeded workload generator follows the stated recipes (host logic, CPU only)."""
import numpy as np
import pytest

from chunked_gated_delta_12_b200.inputs import (bf16_bits_to_f32, f32_to_bf16_bits, generate,
                                                workload)


def test_bf16_rounding_is_rne():
    x = np.array([1.0, 1.00390625, 1.01171875, -2.5, 3.0e38, 1e-40], dtype=np.float32)
    b = f32_to_bf16_bits(x)
    back = bf16_bits_to_f32(b)
    # 1 + 2^-8 is a tie between 1 and 1 + 2^-7 -> rounds to even (1.0)
    assert back[0] == 1.0 and back[1] == 1.0 and back[2] == np.float32(1.015625)
    assert back[3] == -2.5
    normal = np.abs(x) > 1e-37
    assert np.all(np.abs(back - x)[normal] <= np.abs(x)[normal] * 2.0 ** -8)


@pytest.mark.parametrize("idx", [0, 1, 2, 3, 4])
def test_workload_shapes_and_lengths(idx):
    w = workload(idx)
    cu = w.cu_seqlens()
    assert cu[0] == 0 and cu[-1] == w.T and np.all(np.diff(cu) >= 1)
    expect = {0: (1, 256, 2), 1: (8, 4096, 8), 2: (4, 32768, 32), 3: (1, 65536, 32),
              4: (16, 32768, 32)}[idx]
    assert (w.n_docs, w.T, w.H) == expect
    if idx == 1:
        assert all(1 <= L <= 1000 for L in w.lengths)
        assert not all(L % 64 == 0 for L in w.lengths)
    if idx == 4:
        assert all(512 <= L <= 4096 for L in w.lengths)
    assert w.lengths == workload(idx).lengths          # deterministic


def test_generated_distributions_small():
    w = workload(0)
    d = generate(w)
    assert d["q"].shape == (256, 2, 128) and d["q"].dtype == np.uint16
    g, b = d["g"], d["beta"]
    assert g.dtype == np.float32 and (g < 0).all() and (g > -5).all()
    assert b.shape == (256, 2) and (b > 0).all() and (b < 1).all()
    q = bf16_bits_to_f32(d["q"])
    assert abs(float(q.mean())) < 0.05 and abs(float(q.std()) - 1) < 0.05
    d2 = generate(w)
    for key in ("q", "k", "v", "g", "beta"):
        assert np.array_equal(d[key], d2[key])
