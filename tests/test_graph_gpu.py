"""A decode call allocates nothing and never synchronises, so it can be
captured in a CUDA graph once and replayed per token; the replay must give what
the eager call gives (bitwise: same kernels, same split plan)."""
import pytest
import torch

import gpu_util as gu
import gqa_decode_attention_attend_b200 as gqa
from gqa_decode_attention_attend_b200 import workloads

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32], ids=["bf16", "f32"])
def test_captured_decode_matches_eager(dtype):
    dev = gu.device()
    w = workloads.make("graph", [3000, 1, 700, 4096], 32, 8, 128, dtype=dtype, seed=21, carry=True)
    dw = gu.DevWorkload(w, dev)
    ws = gqa.Workspace(dev, 1 << 20)
    rows = w.batch * w.num_heads
    eager_state = gqa.State.empty(rows, 128, dev)
    eager = gqa.gqa_decode_attend(dw.q, dw.k, dw.v, dw.offsets, 32, 8, carry=dw.carry,
                                  state_out=eager_state, want_out=True, workspace=ws,
                                  max_seq_len=w.max_seq_len)
    torch.cuda.synchronize()
    out = torch.empty_like(eager)
    st = gqa.State.empty(rows, 128, dev)
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        for _ in range(3):      # three decode steps in one graph
            gqa.gqa_decode_attend(dw.q, dw.k, dw.v, dw.offsets, 32, 8, carry=dw.carry, state_out=st,
                                  out=out, workspace=ws, max_seq_len=w.max_seq_len)
    for _ in range(2):
        out.zero_()
        graph.replay()
        torch.cuda.synchronize()
        assert torch.equal(out, eager)
        assert torch.equal(st.l, eager_state.l) and torch.equal(st.acc, eager_state.acc)
    assert gqa.gqa_get_device_error(ws) == gqa.GQA_OK


def test_captured_append_step():
    dev = gu.device()
    w = workloads.make("graph_app", [65, 2000], 16, 4, 64, seed=22)
    dw = gu.DevWorkload(w, dev)
    kn = torch.randn((2, 4, 64), device=dev).to(torch.bfloat16)
    vn = torch.randn((2, 4, 64), device=dev).to(torch.bfloat16)
    ws = gqa.Workspace(dev, 1 << 20)
    eager = gqa.gqa_decode_append_attend(dw.q, dw.k, dw.v, dw.offsets, kn, vn, 16, 4, workspace=ws,
                                         max_seq_len=2000)
    torch.cuda.synchronize()
    out = torch.empty_like(eager)
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        gqa.gqa_decode_append_attend(dw.q, dw.k, dw.v, dw.offsets, kn, vn, 16, 4, out=out,
                                     workspace=ws, max_seq_len=2000)
    graph.replay()
    torch.cuda.synchronize()
    assert torch.equal(out, eager)


@pytest.mark.parametrize("graph", [False, True], ids=["eager", "graph"])
def test_early_start_respects_a_carry_chain(graph):
    """Three calls where each folds the previous one's state as its carry: with
    GQA_FLAG_EARLY_START the kernel may start early, but it must read the carry
    only after the previous kernel is done, so the chain matches plain order."""
    dev = gu.device()
    w = workloads.make("chain", [5000, 300, 64], 32, 8, 128, seed=23)
    dw = gu.DevWorkload(w, dev)
    rows = w.batch * w.num_heads
    ws = gqa.Workspace(dev, 1 << 20)

    def chain(flags, states, out):
        carry = None
        for st in states:
            gqa.gqa_decode_attend(dw.q, dw.k, dw.v, dw.offsets, 32, 8, carry=carry, state_out=st,
                                  want_out=False, workspace=ws, max_seq_len=5000, flags=flags)
            carry = st
        gqa.gqa_decode_attend(dw.q, dw.k, dw.v, dw.offsets, 32, 8, carry=carry, out=out,
                              workspace=ws, max_seq_len=5000, flags=flags)

    ref_states = [gqa.State.empty(rows, 128, dev) for _ in range(3)]
    ref = torch.empty_like(dw.q)
    chain(0, ref_states, ref)
    torch.cuda.synchronize()
    states = [gqa.State.empty(rows, 128, dev) for _ in range(3)]
    out = torch.empty_like(dw.q)
    if graph:
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            chain(gqa.GQA_FLAG_EARLY_START, states, out)
        g.replay()
    else:
        chain(gqa.GQA_FLAG_EARLY_START, states, out)
    torch.cuda.synchronize()
    assert torch.equal(out, ref)
    for a, b in zip(states, ref_states):
        assert torch.equal(a.acc, b.acc) and torch.equal(a.l, b.l)
