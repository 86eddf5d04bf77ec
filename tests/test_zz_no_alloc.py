"""gqa_decode_attend_static_workspace: decode attention for callers that cannot
allocate device memory (for instance a plugin inside an engine that owns all
device buffers and gives it no workspace, or a service that forbids allocation
after start-up). Its scratch is a fixed device array inside the library.

It runs the same kernel with the same split plan as gqa_decode_attend, so the
tests expect the very same bits: output, and the state's m, l and acc, on two
calls in a row with different inputs, and after the array's ticket region was
left soiled (written from the host through the array's symbol address by a
test-only hook in a test copy of the library), which each call must clear.

This file is collected last on purpose: it exercises the library's shared
device array, so every other test has already run when it does.
"""
import ctypes

import pytest
import torch

import gqa_decode_attention_attend_b200 as gqa
from gqa_decode_attention_attend_b200 import build as gbuild
from gqa_decode_attention_attend_b200 import workloads

pytestmark = pytest.mark.gpu


def _bind(lib):
    fn = lib.gqa_decode_attend_static_workspace
    fn.argtypes = [ctypes.POINTER(gqa._CParams), ctypes.c_void_p]
    fn.restype = ctypes.c_int
    return fn


def _inputs(w, dev):
    carry = gqa.State(*(t.to(dev) for t in w.carry)) if w.carry is not None else None
    return w.q.to(dev), w.k.to(dev), w.v.to(dev), w.offsets.to(dev), carry


def _nan_like(ref, ref_state):
    out = torch.full_like(ref, float("nan"))
    st = gqa.State(torch.full_like(ref_state.m, float("nan")), torch.full_like(ref_state.l, float("nan")),
                   torch.full_like(ref_state.acc, float("nan")))
    return out, st


def _static_call(fn, w, q, k, v, off, carry, out, st):
    p = gqa._params(q, k, v, off, w.num_heads, w.num_kv_heads, 0.0, carry, st, out,
                    gqa._dtype_code(out), None, 0, w.max_seq_len, None)
    p.workspace = None
    p.workspace_bytes = 0
    return fn(ctypes.byref(p), ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))


def _same_bits(out, st, ref, ref_state):
    assert torch.equal(out, ref)
    assert torch.equal(st.m, ref_state.m)
    assert torch.equal(st.l, ref_state.l)
    assert torch.equal(st.acc, ref_state.acc)


CASES = [
    dict(name="na", lengths=[700, 33, 4096, 1], H=32, G=8, D=128, dtype=torch.bfloat16, dist="normal",
         seed=41, carry=True),
    dict(name="nb", lengths=[5000, 0, 129], H=16, G=2, D=64, dtype=torch.float32, dist="uniform",
         seed=42, carry=False),
]


def _make(c):
    return workloads.make(c["name"], c["lengths"], c["H"], c["G"], c["D"], dtype=c["dtype"],
                          dist=c["dist"], seed=c["seed"], carry=c["carry"])


def test_two_calls_match_workspace_entry_point():
    dev = torch.device("cuda:0")
    fn = _bind(gqa.load_library())
    for c in CASES:
        w = _make(c)
        q, k, v, off, carry = _inputs(w, dev)
        ref_state = gqa.State.empty(w.batch * w.num_heads, w.head_dim, dev)
        ref = gqa.gqa_decode_attend(q, k, v, off, w.num_heads, w.num_kv_heads, carry=carry,
                                    state_out=ref_state, want_out=True, max_seq_len=w.max_seq_len)
        out, st = _nan_like(ref, ref_state)
        status = _static_call(fn, w, q, k, v, off, carry, out, st)
        assert status == gqa.GQA_OK, gqa.gqa_status_string(status)
        torch.cuda.synchronize()
        _same_bits(out, st, ref, ref_state)


def test_binding_wrapper_and_oversize_refusal():
    dev = torch.device("cuda:0")
    w = workloads.make("nc", [300, 2000], 8, 4, 128, dist="normal", seed=43)
    q, k, v, off, _ = _inputs(w, dev)
    a = gqa.gqa_decode_attend_static_workspace(q, k, v, off, 8, 4, max_seq_len=2000)
    b = gqa.gqa_decode_attend(q, k, v, off, 8, 4, max_seq_len=2000)
    torch.cuda.synchronize()
    assert torch.equal(a, b)
    # 2 sequences x 8 heads x 4096 splits x 130 floats x 4 B > 16 MiB of scratch
    with pytest.raises(gqa.GqaError) as e:
        gqa.gqa_decode_attend_static_workspace(q, k, v, off, 8, 4, num_splits=4096, max_seq_len=2000)
    assert e.value.status == gqa.GQA_ERR_WORKSPACE


def test_soiled_ticket_region_is_cleared():
    """Fill the array's error word and merge tickets with junk (as a call that
    stopped half way could leave them), then call: the result must still be the
    workspace entry point's, bit for bit, on two calls in a row. Both entry
    points are taken from the test copy of the library, which carries the hook."""
    dev = torch.device("cuda:0")
    lib = gqa.load_library(gbuild.build_test_lib())
    fn = _bind(lib)
    soil = lib.gqa_test_soil_static_scratch
    soil.argtypes = [ctypes.c_int32, ctypes.c_void_p]
    soil.restype = ctypes.c_int
    attend = lib.gqa_decode_attend
    attend.argtypes = [ctypes.POINTER(gqa._CParams), ctypes.c_void_p]
    attend.restype = ctypes.c_int
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    for fill, c in zip((0x01, 0xFF), CASES):
        w = _make(c)
        q, k, v, off, carry = _inputs(w, dev)
        ref_state = gqa.State.empty(w.batch * w.num_heads, w.head_dim, dev)
        ref = torch.empty(q.shape, dtype=q.dtype, device=dev)
        p = gqa._params(q, k, v, off, w.num_heads, w.num_kv_heads, 0.0, carry, ref_state, ref,
                        gqa._dtype_code(ref), None, 0, w.max_seq_len, None)
        nbytes = ctypes.c_size_t()
        assert lib.gqa_decode_workspace_size(ctypes.byref(p), ctypes.byref(nbytes), None, None) == gqa.GQA_OK
        ws = torch.zeros(nbytes.value + 256, dtype=torch.uint8, device=dev)
        p.workspace = ctypes.c_void_p((ws.data_ptr() + 255) & ~255)
        p.workspace_bytes = nbytes.value
        assert attend(ctypes.byref(p), stream) == gqa.GQA_OK
        assert soil(fill, stream) == gqa.GQA_OK
        out, st = _nan_like(ref, ref_state)
        status = _static_call(fn, w, q, k, v, off, carry, out, st)
        assert status == gqa.GQA_OK, gqa.gqa_status_string(status)
        torch.cuda.synchronize()
        _same_bits(out, st, ref, ref_state)
