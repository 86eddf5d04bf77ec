"""Refusals and device-side findings on a GPU: host pointers, too-small
workspace, and malformed offsets reported through the device error word (the
kernels clamp and return; nothing faults)."""
import ctypes

import pytest
import torch

import gpu_util as gu
import gqa_decode_attention_attend_b200 as gqa
from gqa_decode_attention_attend_b200 import workloads

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def dev():
    return gu.device()


def test_host_pointer_refused(dev):
    w = workloads.make("h", [100], 8, 2, 128, seed=1)
    dw = gu.DevWorkload(w, dev)
    with pytest.raises(gqa.GqaError) as e:
        gqa.gqa_decode_attend(w.q, dw.k, dw.v, dw.offsets, 8, 2)     # q still on the host
    assert e.value.status == gqa.GQA_ERR_DEVICE


def test_workspace_too_small(dev):
    w = workloads.make("ws", [5000], 8, 2, 128, seed=2)
    dw = gu.DevWorkload(w, dev)
    ws = gqa.Workspace(dev, 256)
    lib = gqa.load_library()
    out = torch.empty_like(dw.q)
    p = gqa._params(dw.q, dw.k, dw.v, dw.offsets, 8, 2, 0.0, None, None, out, gqa.GQA_BF16, None,
                    7, 0, None)
    p.workspace = ws.ptr
    p.workspace_bytes = 256
    st = lib.gqa_decode_attend(ctypes.byref(p), None)
    assert st == gqa.GQA_ERR_WORKSPACE


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32], ids=["bf16", "f32"])
def test_bad_offsets_flagged_not_faulted(dev, dtype):
    w = workloads.make("bad", [64, 64, 64], 8, 2, 128, dtype=dtype, seed=3)
    dw = gu.DevWorkload(w, dev)
    ws = gqa.Workspace(dev, 1 << 20)
    bad = torch.tensor([0, 64, 10_000, 192], dtype=torch.int32, device=dev)   # beyond max_len
    out = gqa.gqa_decode_attend(dw.q, dw.k, dw.v, bad, 8, 2, workspace=ws, out_dtype=torch.float32)
    status = gqa.gqa_get_device_error(ws)
    assert status == gqa.GQA_ERR_BAD_OFFSETS
    assert gqa.gqa_get_device_error(ws) == gqa.GQA_OK          # read clears it
    # the well-formed first sequence is still right; the malformed ones are empty (0)
    ref = gu.oracle_state(w, rows=list(range(8)))
    gu.check_out(out[0], ref, w, what="sequence before the bad offsets")
    assert torch.all(out[1:] == 0)
    # decreasing offsets
    dec = torch.tensor([0, 64, 32, 192], dtype=torch.int32, device=dev)
    gqa.gqa_decode_attend(dw.q, dw.k, dw.v, dec, 8, 2, workspace=ws)
    assert gqa.gqa_get_device_error(ws) == gqa.GQA_ERR_BAD_OFFSETS


def test_clean_run_reports_ok(dev):
    w = workloads.make("ok", [300, 20], 8, 2, 64, seed=4)
    dw = gu.DevWorkload(w, dev)
    ws = gqa.Workspace(dev, 1 << 20)
    gqa.gqa_decode_attend(dw.q, dw.k, dw.v, dw.offsets, 8, 2, workspace=ws)
    assert gqa.gqa_get_device_error(ws) == gqa.GQA_OK
