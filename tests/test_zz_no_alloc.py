"""gqa_decode_attend_static_workspace: decode attention for callers that cannot
allocate device memory (for instance a plugin inside an engine that owns all
device buffers and gives it no workspace, or a service that forbids allocation
after start-up). Its scratch is a fixed device array inside the library, so the
test checks that two calls in a row, on different inputs, give what the
workspace-taking entry point gives, and that an oversized call is refused.

This file is collected last on purpose: it exercises the library's shared
device array, so every other test has already run when it does.
"""
import ctypes

import pytest
import torch

import gqa_decode_attention_attend_b200 as gqa
from gqa_decode_attention_attend_b200 import workloads

pytestmark = pytest.mark.gpu

TOL = {torch.float32: (1e-5, 1e-5), torch.bfloat16: (2e-3, 2e-3)}


def _static_entry():
    fn = gqa.load_library().gqa_decode_attend_static_workspace
    fn.argtypes = [ctypes.POINTER(gqa._CParams), ctypes.c_void_p]
    fn.restype = ctypes.c_int
    return fn


def _inputs(w, dev):
    carry = gqa.State(*(t.to(dev) for t in w.carry)) if w.carry is not None else None
    return w.q.to(dev), w.k.to(dev), w.v.to(dev), w.offsets.to(dev), carry


def _close(a, b, dtype):
    atol, rtol = TOL[dtype]
    a = a.float()
    b = b.float()
    # both outputs went through the same output rounding; allow the bf16 step on top
    extra = 2.0 ** -8 * b.abs() if a.dtype == torch.bfloat16 else 0.0
    assert torch.all((a - b).abs() <= atol + rtol * b.abs() + extra)


def test_two_calls_match_workspace_entry_point():
    dev = torch.device("cuda:0")
    fn = _static_entry()
    stream = torch.cuda.current_stream()
    cases = [
        workloads.make("na", [700, 33, 4096, 1], 32, 8, 128, dist="normal", seed=41, carry=True),
        workloads.make("nb", [5000, 0, 129], 16, 2, 64, dtype=torch.float32, dist="uniform", seed=42),
    ]
    for w in cases:
        q, k, v, off, carry = _inputs(w, dev)
        ref_state = gqa.State.empty(w.batch * w.num_heads, w.head_dim, dev)
        ref = gqa.gqa_decode_attend(q, k, v, off, w.num_heads, w.num_kv_heads, carry=carry,
                                    state_out=ref_state, want_out=True, max_seq_len=w.max_seq_len)
        out = torch.full_like(ref, float("nan"))
        st = gqa.State(torch.full_like(ref_state.m, float("nan")), torch.full_like(ref_state.l, float("nan")),
                       torch.full_like(ref_state.acc, float("nan")))
        p = gqa._params(q, k, v, off, w.num_heads, w.num_kv_heads, 0.0, carry, st, out,
                        gqa._dtype_code(out), None, 0, w.max_seq_len, None)
        p.workspace = None
        p.workspace_bytes = 0
        status = fn(ctypes.byref(p), ctypes.c_void_p(stream.cuda_stream))
        assert status == gqa.GQA_OK, gqa.gqa_status_string(status)
        torch.cuda.synchronize()
        _close(out, ref, w.k.dtype)
        _close(st.l, ref_state.l, w.k.dtype)
        assert torch.equal(torch.isneginf(st.m), torch.isneginf(ref_state.m))


def test_binding_wrapper_and_oversize_refusal():
    dev = torch.device("cuda:0")
    w = workloads.make("nc", [300, 2000], 8, 4, 128, dist="normal", seed=43)
    q, k, v, off, _ = _inputs(w, dev)
    a = gqa.gqa_decode_attend_static_workspace(q, k, v, off, 8, 4, max_seq_len=2000)
    b = gqa.gqa_decode_attend(q, k, v, off, 8, 4, max_seq_len=2000)
    torch.cuda.synchronize()
    _close(a, b, torch.bfloat16)
    # 2 sequences x 8 heads x 4096 splits x 130 floats x 4 B > 16 MiB of scratch
    with pytest.raises(gqa.GqaError) as e:
        gqa.gqa_decode_attend_static_workspace(q, k, v, off, 8, 4, num_splits=4096, max_seq_len=2000)
    assert e.value.status == gqa.GQA_ERR_WORKSPACE
