"""GPU parity: the CUDA path through the C ABI against the f64 oracle.

Full-size named workloads run in the launch configuration the benchmark times
(the library's own split heuristic); a sweep of small shapes spans several
pipeline stages and chunks with ragged tails; edge cases cover empty batches,
empty sequences, a too-small length hint, forced split counts and the split
pipeline partials -> gqa_softmax_merge -> gqa_state_finalize.
"""
import math

import numpy as np
import pytest
import torch

import gpu_util as gu
import gqa_decode_attention_attend_b200 as gqa
from gqa_decode_attention_attend_b200 import workloads

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def dev():
    return gu.device()


# ------------------------------------------------------------------ full-size workloads

@pytest.mark.parametrize("name", ["fp32_b1_n512", "bf16_b16_n4096", "bf16_b1_n131072"])
def test_full_config(dev, name):
    w = workloads.config(name)
    dw = gu.DevWorkload(w, dev)
    out, st = gu.run(dw, with_state=True)
    ref = gu.oracle_state(w)
    gu.check_out(out, ref, w, what=f"{name} out")
    gu.check_state(st, ref, w, what=f"{name} state")
    if name == "bf16_b1_n131072":
        # the planted key dominates channel 0 of the first head of every group
        hpk = w.num_heads // w.num_kv_heads
        for g in range(w.num_kv_heads):
            assert ref.out[g * hpk, 0] > 0.0
            assert abs(float(out[0, g * hpk, 0]) - ref.out[g * hpk, 0]) <= 2e-3 + 4e-3 * ref.out[g * hpk, 0]


def test_full_config_ragged_with_carry(dev):
    w = workloads.config("bf16_b64_ragged16384")
    dw = gu.DevWorkload(w, dev)
    out, st = gu.run(dw, with_state=True)
    rows = list(range(0, w.batch * w.num_heads, 3))       # sampled query rows
    ref = gu.oracle_state(w, rows=rows)
    gu.check_out(out, ref, w, rows=rows, what="ragged out")
    gu.check_state(st, ref, w, rows=rows, what="ragged state")


def test_full_config_split_pipeline(dev):
    """partials_out -> gqa_softmax_merge -> gqa_state_finalize on the split-KV stress workload."""
    w = workloads.config("bf16_b4_n32768")
    dw = gu.DevWorkload(w, dev)
    rows = w.batch * w.num_heads
    _, S, chunk = gqa.gqa_decode_workspace_size(dw.q, dw.k, dw.v, dw.offsets, w.num_heads,
                                                w.num_kv_heads, want_out=False,
                                                partials_out=gqa.State.empty(rows, 128, dev, (1,)),
                                                max_seq_len=w.max_seq_len)
    parts = gqa.State.empty(rows, w.head_dim, dev, (S,))
    gqa.gqa_decode_attend(dw.q, dw.k, dw.v, dw.offsets, w.num_heads, w.num_kv_heads,
                          partials_out=parts, num_splits=S, max_seq_len=w.max_seq_len)
    merged = gqa.State.empty(rows, w.head_dim, dev)
    gqa.gqa_softmax_merge(parts, merged_out=merged, want_out=False)
    out = gqa.gqa_state_finalize(merged, out_dtype=torch.bfloat16)
    ref = gu.oracle_state(w)
    gu.check_out(out, ref, w, what="split pipeline finalize")
    gu.check_state(merged, ref, w, what="split pipeline merged")
    # sampled partial states against the oracle over each split's own key range
    ranges = gu.split_ranges(w, chunk, S)
    pm, pl, pacc = parts.m.cpu().numpy(), parts.l.cpu().numpy(), parts.acc.cpu().numpy()
    for b in (0, w.batch - 1):
        for s in sorted({0, 1, S // 2, S - 1}):
            lo, hi = ranges[b][s]
            heads = [0, 7, 8, 63]
            st = gu.oracle_partial(w, b, lo, hi, heads)
            r = [b * w.num_heads + h for h in heads]
            gu.assert_close(pm[r, s], st.m, torch.bfloat16, f"partial m b{b} s{s}")
            gu.assert_close(pl[r, s], st.l, torch.bfloat16, f"partial l b{b} s{s}")
            gu.assert_acc_close(pacc[r, s], st.acc, st.l, torch.bfloat16, f"partial acc b{b} s{s}")


# ------------------------------------------------------------------ sweep of small shapes

SWEEP = []
for D in (64, 128):
    for H, G in ((4, 4), (8, 4), (16, 4), (24, 4), (32, 4), (64, 4)):
        SWEEP.append((D, H, G))


@pytest.mark.parametrize("D,H,G", SWEEP, ids=lambda x: str(x))
@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32], ids=["bf16", "f32"])
def test_sweep_heads_and_dims(dev, D, H, G, dtype):
    lengths = [1, 2, 63, 64, 65, 127, 129, 300, 0, 1000]
    w = workloads.make("sweep", lengths, H, G, D, dtype=dtype, dist="normal", seed=D + H,
                       carry=True)
    dw = gu.DevWorkload(w, dev)
    ref = gu.oracle_state(w)
    for ns in (0, 1, 3):
        out, st = gu.run(dw, with_state=True, num_splits=ns, out_dtype=torch.float32)
        gu.check_out(out, ref, w, what=f"D{D} H{H} G{G} splits{ns} out")
        gu.check_state(st, ref, w, what=f"D{D} H{H} G{G} splits{ns} state")
    out, _ = gu.run(dw)            # native output dtype
    assert out.dtype == dtype
    gu.check_out(out, ref, w, what=f"D{D} H{H} G{G} native out")


@pytest.mark.parametrize("n", [1, 15, 16, 17, 63, 64, 65, 191, 192, 193, 4095, 4097])
def test_lengths_around_stage_and_warp_boundaries(dev, n):
    w = workloads.make("len", [n, max(1, n // 2)], 32, 8, 128, dist="normal", seed=n)
    dw = gu.DevWorkload(w, dev)
    ref = gu.oracle_state(w, carry=False)
    for ns in (0, 2):
        out, st = gu.run(dw, with_state=True, num_splits=ns, out_dtype=torch.float32)
        gu.check_out(out, ref, w, what=f"n{n} splits{ns}")
        gu.check_state(st, ref, w, what=f"n{n} splits{ns} state")


def test_many_splits_and_hint_too_small(dev):
    w = workloads.make("splits", [5000, 3000, 64], 16, 2, 128, dist="normal", seed=77)
    dw = gu.DevWorkload(w, dev)
    ref = gu.oracle_state(w)
    for ns in (1, 2, 7, 40, 79):
        out, _ = gu.run(dw, num_splits=ns, out_dtype=torch.float32)
        gu.check_out(out, ref, w, what=f"splits {ns}")
    # a max_seq_len hint below the real longest sequence stays correct
    out, _ = gu.run(dw, max_seq_len=1000, out_dtype=torch.float32)
    gu.check_out(out, ref, w, what="hint too small")


def test_uniform_distribution_fp32_long(dev):
    w = workloads.make("f32long", [20000, 7], 8, 2, 64, dtype=torch.float32, dist="uniform",
                       seed=31, carry=True)
    dw = gu.DevWorkload(w, dev)
    ref = gu.oracle_state(w)
    out, st = gu.run(dw, with_state=True)
    gu.check_out(out, ref, w, what="fp32 long")
    gu.check_state(st, ref, w, what="fp32 long state")


# ------------------------------------------------------------------ edge cases

def test_empty_batch_is_noop(dev):
    w = workloads.make("empty", [], 8, 2, 128)
    dw = gu.DevWorkload(w, dev)
    dw.k = torch.zeros((4, 2, 128), dtype=torch.bfloat16, device=dev)
    dw.v = torch.zeros_like(dw.k)
    out = gqa.gqa_decode_attend(dw.q, dw.k, dw.v, dw.offsets, 8, 2)
    torch.cuda.synchronize()
    assert out.shape == (0, 8, 128)


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32], ids=["bf16", "f32"])
def test_all_sequences_empty(dev, dtype):
    w = workloads.make("allempty", [0, 0, 0], 8, 2, 64, dtype=dtype, carry=True, seed=5)
    dw = gu.DevWorkload(w, dev)
    # a cache with rows, but no sequence owns any
    dw.k = torch.randn((10, 2, 64), device=dev).to(dtype)
    dw.v = torch.randn((10, 2, 64), device=dev).to(dtype)
    out, st = gu.run(dw, with_state=True, carry=False, out_dtype=torch.float32)
    assert torch.all(out == 0)
    assert torch.all(st.l == 0) and torch.all(torch.isneginf(st.m)) and torch.all(st.acc == 0)
    # with a carry the carry passes through: out = acc / l
    out, st = gu.run(dw, with_state=True, out_dtype=torch.float32)
    m, l, acc = (t.to(dev) for t in w.carry)
    torch.testing.assert_close(out.reshape(-1, 64), acc / l[:, None], rtol=1e-6, atol=1e-6)
    assert torch.equal(st.m, m) and torch.equal(st.l, l) and torch.equal(st.acc, acc)


def test_zero_row_cache(dev):
    w = workloads.make("zerorows", [0, 0], 4, 4, 128, carry=True, seed=6)
    dw = gu.DevWorkload(w, dev)
    assert dw.k.shape[0] == 0
    out, st = gu.run(dw, with_state=True, out_dtype=torch.float32)
    m, l, acc = (t.to(dev) for t in w.carry)
    torch.testing.assert_close(out.reshape(-1, 128), acc / l[:, None], rtol=1e-6, atol=1e-6)


def test_partials_mark_empty_splits(dev):
    w = workloads.make("pe", [10, 300], 8, 2, 128, seed=8)
    dw = gu.DevWorkload(w, dev)
    rows = w.batch * w.num_heads
    parts = gqa.State.empty(rows, 128, dev, (4,))
    parts.m.fill_(123.0)
    parts.l.fill_(5.0)
    gqa.gqa_decode_attend(dw.q, dw.k, dw.v, dw.offsets, 8, 2, partials_out=parts, num_splits=4,
                          max_seq_len=300)
    # chunk = 128 -> sequence 0 (10 keys) fills split 0 only
    assert torch.all(parts.l[:8, 1:] == 0) and torch.all(torch.isneginf(parts.m[:8, 1:]))
    assert torch.all(parts.acc[:8, 1:] == 0)
    # sequence 1 (300 keys) fills splits 0..2; split 3 has no keys left
    assert torch.all(parts.l[8:, :3] > 0) and torch.all(parts.l[8:, 3] == 0)
    out = gqa.gqa_softmax_merge(parts)
    ref = gu.oracle_state(w)
    gu.assert_close(out.cpu().numpy(), ref.out, torch.bfloat16, "merge of partials")


def test_merge_with_carry_and_alias(dev):
    """gqa_softmax_merge folding a carry, writing the merged state over the carry."""
    w = workloads.make("mc", [700, 33], 16, 4, 64, carry=True, seed=9)
    dw = gu.DevWorkload(w, dev)
    rows = w.batch * w.num_heads
    parts = gqa.State.empty(rows, 64, dev, (3,))
    gqa.gqa_decode_attend(dw.q, dw.k, dw.v, dw.offsets, 16, 4, partials_out=parts, num_splits=3,
                          max_seq_len=700)
    carry = gqa.State(*(t.clone() for t in (dw.carry.m, dw.carry.l, dw.carry.acc)))
    out = gqa.gqa_softmax_merge(parts, carry=carry, merged_out=carry, want_out=True)
    ref = gu.oracle_state(w)
    gu.assert_close(out.cpu().numpy(), ref.out, torch.bfloat16, "merge+carry out")
    gu.check_state(carry, ref, w, what="merged state over carry")


def test_state_out_aliases_carry(dev):
    w = workloads.make("alias", [513, 2], 8, 8, 128, carry=True, seed=10)
    dw = gu.DevWorkload(w, dev)
    ref = gu.oracle_state(w)
    out = gqa.gqa_decode_attend(dw.q, dw.k, dw.v, dw.offsets, 8, 8, carry=dw.carry,
                                state_out=dw.carry, out_dtype=torch.float32, want_out=True)
    gu.check_out(out, ref, w, what="aliased out")
    gu.check_state(dw.carry, ref, w, what="aliased state")


def test_explicit_scale_equals_default(dev):
    w = workloads.make("scale", [777], 16, 4, 128, seed=12)
    dw = gu.DevWorkload(w, dev)
    a, _ = gu.run(dw, out_dtype=torch.float32, score_scale=0.0)
    b, _ = gu.run(dw, out_dtype=torch.float32,
                  score_scale=float(np.float32(1.0) / np.sqrt(np.float32(128))))
    assert torch.equal(a, b)
    c, _ = gu.run(dw, out_dtype=torch.float32, score_scale=0.3)
    ref = gu.oracle_state(w, score_scale=0.3)
    gu.check_out(c, ref, w, what="scale 0.3")


def test_final_output_dtype_bf16_from_fp32_inputs(dev):
    w = workloads.make("f32bf", [100, 257], 8, 2, 128, dtype=torch.float32, seed=13)
    dw = gu.DevWorkload(w, dev)
    ref = gu.oracle_state(w)
    out, _ = gu.run(dw, out_dtype=torch.bfloat16)
    assert out.dtype == torch.bfloat16
    gu.check_out(out, ref, w, what="fp32 in, bf16 out")


def test_stored_golden_values(dev):
    """The fp32 workload against the oracle's stored values (tests/golden)."""
    import json
    import os
    g = json.load(open(os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden",
                                    "fp32_b1_n512_rows.json")))
    w = workloads.config("fp32_b1_n512")
    dw = gu.DevWorkload(w, dev)
    out, st = gu.run(dw, with_state=True)
    ref = __import__("oracle").State(np.array(g["m"]), np.array(g["l"]), np.array(g["out"]) * np.array(g["l"])[:, None],
                                     np.array(g["out"]))
    gu.check_out(out, ref, w, what="golden fp32_b1_n512")
    gu.assert_close(st.m.cpu().numpy(), ref.m, torch.float32, "golden fp32_b1_n512 m")


def test_stored_needle_trial(dev):
    """The planted-key trial at 1024 keys (cortiq_engine NystromState example
    `trial`: 6 Q / 2 KV heads, d 64, key planted at depth 64 with amplitude 8,
    V[., 0] = 0 except the planted row) against the oracle's stored out[:, 0]
    (tests/golden/needle_small.json): channel 0 of each output is the weight
    the softmax gives the planted key, which dominates for each group's first
    head (heads 0 and 3)."""
    import json
    import os
    g = json.load(open(os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden",
                                    "needle_small.json")))
    w = workloads.make(g["workload"], g["lengths"], g["heads"], g["kv_heads"], g["head_dim"], dist="needle",
                       seed=g["seed"], needle=dict(amp=g["amp"], depth=g["depth"]))
    dw = gu.DevWorkload(w, dev)
    out, _ = gu.run(dw, out_dtype=torch.float32)
    got0 = out.reshape(-1, g["head_dim"])[:, 0].cpu().numpy()
    gu.assert_close(got0, np.array(g["out0"]), torch.bfloat16, "golden needle_small out[:, 0]")
    hpk = g["heads"] // g["kv_heads"]
    for h in range(0, g["heads"], hpk):
        assert got0[h] > 0.5


def test_more_segments_than_the_fixed_ticket_region(dev):
    """9000 sequences x 8 KV heads = 72000 (sequence, KV head) segments: the merge
    tickets then live in a region cleared on every call."""
    g = torch.Generator().manual_seed(31)
    lengths = torch.randint(1, 9, (9000,), generator=g).tolist()
    lengths[5] = 300                       # one sequence long enough to split
    w = workloads.make("many", lengths, 8, 8, 64, seed=32, carry=True)
    dw = gu.DevWorkload(w, dev)
    rows = list(range(0, 9000 * 8, 97)) + list(range(40, 48))
    ref = gu.oracle_state(w, rows=rows)
    for _ in range(2):                     # the second call must see cleared tickets again
        out, st = gu.run(dw, with_state=True, out_dtype=torch.float32)
        gu.check_out(out, ref, w, rows=rows, what="72000 segments")
        gu.check_state(st, ref, w, rows=rows, what="72000 segments state")


def test_partials_and_merged_output_together(dev):
    w = workloads.make("both", [3000, 17, 1], 16, 4, 128, seed=33, carry=True)
    dw = gu.DevWorkload(w, dev)
    rows = w.batch * w.num_heads
    parts = gqa.State.empty(rows, 128, dev, (5,))
    out = gqa.gqa_decode_attend(dw.q, dw.k, dw.v, dw.offsets, 16, 4, carry=dw.carry, partials_out=parts,
                                num_splits=5, max_seq_len=3000, out_dtype=torch.float32, want_out=True)
    ref = gu.oracle_state(w)
    gu.check_out(out, ref, w, what="out beside partials")
    # the partials alone (no carry) merge to the carry-free result
    merged = gqa.gqa_softmax_merge(parts)
    gu.assert_close(merged.cpu().numpy(), gu.oracle_state(w, carry=False).out, torch.bfloat16,
                    "partials beside out")


def test_zero_kv_heads_means_one_per_query_head(dev):
    w = workloads.make("mha", [500, 64], 8, 8, 64, seed=34)
    dw = gu.DevWorkload(w, dev)
    a = gqa.gqa_decode_attend(dw.q, dw.k, dw.v, dw.offsets, 8, 0, out_dtype=torch.float32)
    b = gqa.gqa_decode_attend(dw.q, dw.k, dw.v, dw.offsets, 8, 8, out_dtype=torch.float32)
    assert torch.equal(a, b)
