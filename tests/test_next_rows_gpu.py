"""GPU parity for the rows beyond plain attend: the additive bias row
(needle_core attn.rs, attn_bias), index rows turned into a mask (metrale
glm5next_dsa_ref, topk_to_mask) and the fused append + attend step
(needle_core attn.rs, KvCache::push_kv then self_attn_incremental), each
against the f64 oracle on the same inputs."""
import numpy as np
import pytest
import torch

import gpu_util as gu
import oracle
import gqa_decode_attention_attend_b200 as gqa
from gqa_decode_attention_attend_b200 import workloads

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def dev():
    return gu.device()


def _bias_for(w, seed, masked_frac=0.2):
    g = torch.Generator().manual_seed(seed)
    b = torch.randn(w.total_rows, generator=g)
    mask = torch.rand(w.total_rows, generator=g) < masked_frac
    b[mask] = float("-inf")
    return b


# ------------------------------------------------------------------ bias row

@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32], ids=["bf16", "f32"])
@pytest.mark.parametrize("D,H,G", [(128, 32, 8), (64, 16, 2), (128, 12, 1)])
def test_bias_row(dev, dtype, D, H, G):
    w = workloads.make("bias", [1, 17, 300, 1000, 4097], H, G, D, dtype=dtype, seed=D + H, carry=True)
    bias = _bias_for(w, 5)
    dw = gu.DevWorkload(w, dev)
    db = bias.to(dev)
    ref = oracle.decode_attend(workloads.host_array(w.q), workloads.host_array(w.k),
                               workloads.host_array(w.v), w.offsets.numpy(), H, G,
                               carry=tuple(t.numpy() for t in w.carry), bias=bias.numpy())
    for ns in (0, 3):
        st = gqa.State.empty(w.batch * H, D, dev)
        out = gqa.gqa_decode_attend(dw.q, dw.k, dw.v, dw.offsets, H, G, carry=dw.carry, state_out=st,
                                    out_dtype=torch.float32, want_out=True, num_splits=ns,
                                    max_seq_len=w.max_seq_len, bias=db)
        gu.check_out(out, ref, w, what=f"bias splits {ns}")
        gu.check_state(st, ref, w, what=f"bias state splits {ns}")


def test_bias_masks_whole_sequence(dev):
    w = workloads.make("mask", [200, 50], 8, 2, 128, seed=3, carry=True)
    dw = gu.DevWorkload(w, dev)
    bias = torch.zeros(w.total_rows)
    bias[:200] = float("-inf")                # sequence 0 fully masked
    out = gqa.gqa_decode_attend(dw.q, dw.k, dw.v, dw.offsets, 8, 2, out_dtype=torch.float32,
                                bias=bias.to(dev))
    assert torch.all(out[0] == 0), "a fully masked sequence without carry gives 0"
    ref = gu.oracle_state(w, carry=False)
    gu.check_out(out[1], ref.__class__(ref.m[8:], ref.l[8:], ref.acc[8:], ref.out[8:]), w,
                 what="unmasked sequence")
    # with its carry the fully masked sequence returns the carry alone
    out = gqa.gqa_decode_attend(dw.q, dw.k, dw.v, dw.offsets, 8, 2, carry=dw.carry,
                                out_dtype=torch.float32, bias=bias.to(dev))
    m, l, acc = w.carry
    torch.testing.assert_close(out[0].cpu(), (acc[:8] / l[:8, None]), rtol=1e-5, atol=1e-6)


def test_constant_bias_is_a_shift(dev):
    w = workloads.make("cb", [3000, 700], 32, 8, 128, seed=4)
    dw = gu.DevWorkload(w, dev)
    a = gqa.gqa_decode_attend(dw.q, dw.k, dw.v, dw.offsets, 32, 8, out_dtype=torch.float32)
    st = gqa.State.empty(64, 128, dev)
    b = gqa.gqa_decode_attend(dw.q, dw.k, dw.v, dw.offsets, 32, 8, out_dtype=torch.float32,
                              state_out=st, want_out=True,
                              bias=torch.full((w.total_rows,), 3.0, device=dev))
    torch.testing.assert_close(a, b, rtol=2e-5, atol=2e-6)


# ------------------------------------------------------------------ index rows -> mask

def test_topk_to_bias_matches_oracle(dev):
    lengths = [5, 0, 12, 300]
    off = np.zeros(5, np.int32)
    off[1:] = np.cumsum(lengths)
    rng = np.random.default_rng(6)
    width = 9
    idx = rng.integers(-2, 20, (4, width)).astype(np.int32)
    idx[0, :3] = [4, 4, -1]                   # a repeat and the INVALID sentinel
    idx[3] = rng.integers(0, 300, width)
    rows = int(off[-1]) + 7
    want = oracle.topk_to_bias(idx, off, rows, fill=0.5)
    got = torch.full((rows,), 0.5, device=dev)
    gqa.gqa_topk_to_bias(torch.from_numpy(idx).to(dev), torch.from_numpy(off).to(dev), rows, bias=got)
    torch.cuda.synchronize()
    assert np.array_equal(got.cpu().numpy(), want), "top-k bias must match bit for bit"


def test_index_selected_attention(dev):
    """decode attention over the keys an index row selects (the DSA reading:
    index row -> mask -> attention), full 16-sequence bf16 shape."""
    w = workloads.make("sel", [4096] * 16, 32, 8, 128, seed=7)
    dw = gu.DevWorkload(w, dev)
    rng = np.random.default_rng(7)
    idx = rng.integers(-1, 4200, (16, 512)).astype(np.int32)     # some -1, some out of range
    bias = gqa.gqa_topk_to_bias(torch.from_numpy(idx).to(dev), dw.offsets, w.total_rows)
    out = gqa.gqa_decode_attend(dw.q, dw.k, dw.v, dw.offsets, 32, 8, bias=bias)
    hb = oracle.topk_to_bias(idx, w.offsets.numpy(), w.total_rows)
    ref = oracle.decode_attend(workloads.host_array(w.q), workloads.host_array(w.k),
                               workloads.host_array(w.v), w.offsets.numpy(), 32, 8, bias=hb)
    gu.check_out(out, ref, w, what="index-selected")


# ------------------------------------------------------------------ append + attend

def _append_case(dev, w, seed, **kw):
    g = torch.Generator().manual_seed(seed)
    kn = torch.randn((w.batch, w.num_kv_heads, w.head_dim), generator=g).to(w.k.dtype)
    vn = torch.randn((w.batch, w.num_kv_heads, w.head_dim), generator=g).to(w.k.dtype)
    dw = gu.DevWorkload(w, dev)
    k_before = dw.k.clone()
    st = gqa.State.empty(w.batch * w.num_heads, w.head_dim, dev)
    out = gqa.gqa_decode_append_attend(dw.q, dw.k, dw.v, dw.offsets, kn.to(dev), vn.to(dev),
                                       w.num_heads, w.num_kv_heads, carry=dw.carry, state_out=st,
                                       out_dtype=torch.float32, want_out=True,
                                       max_seq_len=w.max_seq_len, **kw)
    torch.cuda.synchronize()
    ref, k2, v2 = oracle.append_then_attend(
        workloads.host_array(w.q), workloads.host_array(w.k), workloads.host_array(w.v),
        w.offsets.numpy(), workloads.host_array(kn), workloads.host_array(vn), w.num_heads,
        w.num_kv_heads, carry=None if w.carry is None else tuple(t.numpy() for t in w.carry))
    # the caches now hold exactly the appended rows, and nothing else changed
    assert np.array_equal(workloads.host_array(dw.k.cpu()), k2)
    assert np.array_equal(workloads.host_array(dw.v.cpu()), v2)
    assert not torch.equal(dw.k, k_before) or w.batch == 0
    gu.check_out(out, ref, w, what="append+attend out")
    gu.check_state(st, ref, w, what="append+attend state")


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32], ids=["bf16", "f32"])
def test_append_then_attend(dev, dtype):
    # lengths include the new token: 1 (only it), stage/chunk edges and a long one
    w = workloads.make("app", [1, 2, 64, 65, 129, 3000], 32, 8, 128, dtype=dtype, seed=8, carry=True)
    _append_case(dev, w, 80)
    _append_case(dev, w, 81, num_splits=4)


def test_append_then_attend_small_heads(dev):
    w = workloads.make("app2", [7, 1000], 6, 3, 64, seed=9)
    _append_case(dev, w, 90, num_splits=3)


def test_append_full_batch_shape(dev):
    w = workloads.make("app3", [4096] * 16, 32, 8, 128, seed=10)
    _append_case(dev, w, 100)


def test_append_without_a_row_is_flagged(dev):
    w = workloads.make("app4", [5, 0], 8, 2, 128, seed=11)
    dw = gu.DevWorkload(w, dev)
    ws = gqa.Workspace(dev, 1 << 20)
    kn = torch.randn((2, 2, 128), device=dev).to(torch.bfloat16)
    vn = torch.randn((2, 2, 128), device=dev).to(torch.bfloat16)
    k_before = dw.k.clone()
    gqa.gqa_decode_append_attend(dw.q, dw.k, dw.v, dw.offsets, kn, vn, 8, 2, workspace=ws)
    assert gqa.gqa_get_device_error(ws) == gqa.GQA_ERR_BAD_OFFSETS
    assert torch.equal(dw.k[:4], k_before[:4]) and torch.equal(dw.k[4], kn[0])
