"""Seeded input generator: shapes, determinism and the planted-key structure (CPU)."""
import json
import os

import numpy as np
import torch

import oracle
from gqa_decode_attention_attend_b200 import workloads

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def test_shapes_and_dtypes():
    w = workloads.make("t", [3, 0, 5], 8, 2, 64, dist="normal", seed=7, carry=True)
    assert w.q.shape == (3, 8, 64) and w.q.dtype == torch.bfloat16
    assert w.k.shape == (8, 2, 64) and w.v.shape == (8, 2, 64)
    assert w.offsets.tolist() == [0, 3, 3, 8] and w.offsets.dtype == torch.int32
    m, l, acc = w.carry
    assert m.shape == (24,) and l.shape == (24,) and acc.shape == (24, 64)
    assert float(l.min()) >= 1.0 and float(l.max()) <= 100.0
    assert w.kv_bytes() == 8 * 2 * 64 * 2 * 2


def test_deterministic():
    a = workloads.make("t", [17, 4], 4, 4, 128, dist="uniform", seed=3)
    b = workloads.make("t", [17, 4], 4, 4, 128, dist="uniform", seed=3)
    assert torch.equal(a.k, b.k) and torch.equal(a.q, b.q)
    c = workloads.make("t", [17, 4], 4, 4, 128, dist="uniform", seed=4)
    assert not torch.equal(a.k, c.k)


def test_bf16_is_rne_of_fp32_draw():
    gen = torch.Generator().manual_seed(9)
    x = torch.randn((5, 2, 64), generator=gen)
    w = workloads.make("t", [5], 2, 2, 64, dist="normal", seed=9, q_dtype=torch.float32)
    # the first draw is q [1, 2, 64]; k comes next from the same stream
    gen = torch.Generator().manual_seed(9)
    q = torch.randn((1, 2, 64), generator=gen)
    k = torch.randn((5, 2, 64), generator=gen)
    assert torch.equal(w.q, q)
    assert torch.equal(w.k, k.to(torch.bfloat16))
    del x


def test_needle_structure():
    w = workloads.make("n", [300, 100], 6, 2, 16, dist="needle", seed=5,
                       needle=dict(amp=8.0, depth=40))
    v = w.v.float()
    rows = {p for p, _ in w.needle_rows}
    assert rows == {260, 300 + 60}
    for p, g in w.needle_rows:
        assert float(v[p, g, 0]) == 1.0
    mask = torch.ones(400, dtype=torch.bool)
    mask[list(rows)] = False
    assert float(v[mask, :, 0].abs().max()) == 0.0
    qn = w.q.float().norm(dim=-1)
    assert torch.allclose(qn, torch.full_like(qn, 4.0), rtol=1e-2)


def test_config_sizes():
    w = workloads.config("fp32_b1_n512")
    assert w.q.dtype == torch.float32 and w.kv_bytes() == 1 << 20
    lengths = workloads.ragged_lengths(64, 1, 16384, 4)
    assert len(lengths) == 64 and min(lengths) >= 1 and max(lengths) <= 16384


def test_golden_rows_reproduced_by_oracle():
    g = json.load(open(os.path.join(GOLDEN, "fp32_b1_n512_rows.json")))
    w = workloads.config("fp32_b1_n512")
    st = oracle.decode_attend(w.q.numpy(), w.k.numpy(), w.v.numpy(), w.offsets.numpy(), 8, 4, 1 / 8)
    assert np.array_equal(st.out, np.array(g["out"])) and np.array_equal(st.m, np.array(g["m"]))


def test_golden_needle_reproduced_by_oracle():
    g = json.load(open(os.path.join(GOLDEN, "needle_small.json")))
    w = workloads.make(g["workload"], g["lengths"], g["heads"], g["kv_heads"], g["head_dim"], dist="needle",
                       seed=g["seed"], needle=dict(amp=g["amp"], depth=g["depth"]))
    st = oracle.decode_attend(workloads.host_array(w.q), workloads.host_array(w.k), workloads.host_array(w.v),
                              w.offsets.numpy(), g["heads"], g["kv_heads"])
    assert np.array_equal(st.out[:, 0], np.array(g["out0"]))
