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
