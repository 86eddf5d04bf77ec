"""The C-ABI library: it loads, exports every declared entry point, and refuses
malformed arguments on the host before touching a device (CPU only)."""
import ctypes
import os
import re

import pytest

import gqa_decode_attention_attend_b200 as gqa

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "gqa_decode.h")


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(gqa_[a-z0-9_]+)\s*\(", text)))


def test_library_exports_every_declared_symbol():
    lib = gqa.load_library()
    names = declared_functions()
    assert "gqa_decode_attend" in names and "gqa_softmax_merge" in names
    assert "gqa_state_finalize" in names
    for n in names:
        assert hasattr(lib, n), f"{n} declared in gqa_decode.h but not exported"


def test_params_struct_layout_matches_header():
    # the ctypes mirror must have the size the C side checks in struct_size
    p = gqa._CParams()
    assert ctypes.sizeof(p) == ctypes.sizeof(gqa._CParams)
    offs = {name: getattr(gqa._CParams, name).offset for name, _ in gqa._CParams._fields_}
    assert offs["q"] == 8 and offs["carry_in"] % 8 == 0 and offs["workspace_bytes"] % 8 == 0


def test_status_strings_and_version():
    assert gqa.gqa_status_string(0) == "GQA_OK"
    assert gqa.gqa_status_string(2) == "GQA_ERR_SHAPE_MISMATCH"
    assert gqa.gqa_status_string(6) == "GQA_ERR_TIMEOUT"
    assert gqa.gqa_status_string(99) == "GQA_ERR_UNKNOWN"
    assert gqa.gqa_version() >= 100


def _base_params(**kw):
    p = gqa._CParams()
    p.struct_size = ctypes.sizeof(gqa._CParams)
    p.q, p.k, p.v, p.offsets = 0x1000, 0x2000, 0x3000, 0x4000
    p.q_dtype = p.kv_dtype = p.out_dtype = gqa.GQA_BF16
    p.batch, p.max_len, p.max_seq_len = 2, 100, 50
    p.num_heads, p.num_kv_heads, p.head_dim = 8, 2, 128
    p.out = 0x5000
    for k, v in kw.items():
        setattr(p, k, v)
    return p


@pytest.mark.parametrize("field,value,status", [
    ("struct_size", 8, gqa.GQA_ERR_INVALID_ARGUMENT),
    ("num_heads", 6, gqa.GQA_ERR_INVALID_ARGUMENT),          # 6 % 4 != 0 with num_kv_heads 4
    ("head_dim", 96, gqa.GQA_ERR_INVALID_ARGUMENT),
    ("batch", -1, gqa.GQA_ERR_INVALID_ARGUMENT),
    ("q", None, gqa.GQA_ERR_INVALID_ARGUMENT),
    ("offsets", None, gqa.GQA_ERR_INVALID_ARGUMENT),
    ("out", None, gqa.GQA_ERR_INVALID_ARGUMENT),              # nothing requested
    ("q_dtype", gqa.GQA_F32, gqa.GQA_ERR_SHAPE_MISMATCH),     # fp32 q with bf16 K/V
    ("kv_dtype", 7, gqa.GQA_ERR_SHAPE_MISMATCH),
    ("k", 0x2002, gqa.GQA_ERR_SHAPE_MISMATCH),                # misaligned cache
    ("score_scale", float("nan"), gqa.GQA_ERR_INVALID_ARGUMENT),
    ("num_splits", -3, gqa.GQA_ERR_INVALID_ARGUMENT),
])
def test_host_refusals(field, value, status):
    lib = gqa.load_library()
    kw = {field: value}
    if field == "num_heads":
        kw["num_kv_heads"] = 4
    p = _base_params(**kw)
    assert lib.gqa_decode_attend(ctypes.byref(p), None) == status
    assert lib.gqa_decode_workspace_size(ctypes.byref(p), None, None, None) == status


def test_too_many_heads_per_kv_head():
    lib = gqa.load_library()
    p = _base_params(num_heads=64, num_kv_heads=2)   # 32 > 16
    assert lib.gqa_decode_attend(ctypes.byref(p), None) == gqa.GQA_ERR_INVALID_ARGUMENT


def test_partial_state_struct_refused():
    lib = gqa.load_library()
    p = _base_params()
    p.carry_in = gqa._CState(0x6000, None, 0x7000)   # l missing
    assert lib.gqa_decode_attend(ctypes.byref(p), None) == gqa.GQA_ERR_INVALID_ARGUMENT


def test_merge_refusals():
    lib = gqa.load_library()
    st = gqa._CState(0x1000, 0x2000, 0x3000)
    none = gqa._CState(None, None, None)
    # head_dim 32 unsupported; no output at all; bad dtype
    assert lib.gqa_softmax_merge(ctypes.byref(st), 4, 2, 32, ctypes.byref(none), ctypes.byref(none),
                                 0x9000, 0, None) == gqa.GQA_ERR_INVALID_ARGUMENT
    assert lib.gqa_softmax_merge(ctypes.byref(st), 4, 2, 64, ctypes.byref(none), ctypes.byref(none),
                                 None, 0, None) == gqa.GQA_ERR_INVALID_ARGUMENT
    assert lib.gqa_softmax_merge(ctypes.byref(st), 4, 2, 64, ctypes.byref(none), ctypes.byref(none),
                                 0x9000, 5, None) == gqa.GQA_ERR_SHAPE_MISMATCH
    assert lib.gqa_state_finalize(None, 4, 64, 0x9000, 0, None) == gqa.GQA_ERR_INVALID_ARGUMENT


def test_workspace_init_refuses_small():
    lib = gqa.load_library()
    assert lib.gqa_workspace_init(None, 4096, None) == gqa.GQA_ERR_WORKSPACE
    assert lib.gqa_workspace_init(ctypes.c_void_p(0x1000), 16, None) == gqa.GQA_ERR_WORKSPACE


# ------------------------------------------------------------------ split heuristic (host only)

def test_plan_uniform_configs():
    # 148 SMs x 2 resident CTAs
    for B, G, N in [(16, 8, 4096), (4, 8, 32768), (1, 8, 131072), (1, 4, 512), (64, 8, 4096),
                    (3, 2, 1000)]:
        chunk, splits = gqa.gqa_plan_splits(B, G, N, B * N, 148, 2)
        assert chunk % 64 == 0 and chunk >= 64
        assert splits == -(-N // chunk)
        assert (splits - 1) * chunk < N <= splits * chunk
        ctas = B * G * splits
        # never a last wave that leaves most SMs idle
        rem = ctas % 296
        assert rem == 0 or rem >= 128 or ctas < 296


def test_plan_matches_measured_best():
    # split counts that measured fastest on B200 for these equal-length batches
    # 16 x 8 segments fill 128 of 148 SMs with one split each: no merge (B200:
    # equal back to back, ~4 us sooner as a lone call than two splits)
    assert gqa.gqa_plan_splits(16, 8, 4096, 16 * 4096, 148, 2) == (4096, 1)
    assert 5 <= gqa.gqa_plan_splits(4, 8, 32768, 4 * 32768, 148, 2)[1] <= 9
    assert gqa.gqa_plan_splits(1, 8, 131072, 131072, 148, 2)[1] in (18, 19, 37)


def test_plan_ragged_uses_more_ctas():
    c_u, s_u = gqa.gqa_plan_splits(64, 8, 16384, 64 * 16384, 148, 2)
    c_r, s_r = gqa.gqa_plan_splits(64, 8, 16384, 524320, 148, 2)
    assert c_r <= c_u and s_r >= s_u


def test_plan_degenerate():
    assert gqa.gqa_plan_splits(0, 8, 100, 0) == (64, 1)
    assert gqa.gqa_plan_splits(3, 8, 0, 0) == (64, 1)
    assert gqa.gqa_plan_splits(1, 1, 1, 1) == (64, 1)
    with pytest.raises(gqa.GqaError):
        gqa.gqa_plan_splits(1, 0, 10, 10)
    with pytest.raises(gqa.GqaError):
        gqa.gqa_plan_splits(1, 1, 10, 10, 0, 2)


_B, _H, _G, _D, _N = 2, 8, 2, 64, 10


def _bad(name):
    """One mismatched argument of a small decode call (CPU tensors)."""
    import torch
    rows = _B * _H
    return {
        "q": ("q", torch.zeros(_B, _H - 1, _D)),
        "k_heads": ("k", torch.zeros(_B * _N, _G + 1, _D)),
        "v_dim": ("v", torch.zeros(_B * _N, _G, _D // 2)),
        "offsets_dtype": ("offsets", torch.tensor([0, _N, 2 * _N])),
        "out": ("out", torch.zeros(rows * _D - 1)),
        "carry": ("carry", gqa.State(torch.zeros(rows - 1), torch.zeros(rows - 1), torch.zeros(rows - 1, _D))),
        "partials": ("partials_out", gqa.State(torch.zeros(rows * 3 + 1), torch.zeros(rows * 3 + 1),
                                               torch.zeros(rows * 3 + 1, _D))),
        "bias": ("bias", torch.zeros(_B * _N - 1)),
        "max_len": ("max_len", 1000),
    }[name]


@pytest.mark.parametrize("name", ["q", "k_heads", "v_dim", "offsets_dtype", "out", "carry", "partials",
                                  "bias", "max_len"])
def test_binding_refuses_mismatched_tensors(name):
    """The C ABI sees pointers only; the binding refuses tensors that do not
    hold what the call would read or write, before anything runs."""
    import torch
    args = dict(q=torch.zeros(_B, _H, _D), k=torch.zeros(_B * _N, _G, _D), v=torch.zeros(_B * _N, _G, _D),
                offsets=torch.tensor([0, _N, 2 * _N], dtype=torch.int32))
    kw = {}
    key, val = _bad(name)
    (args if key in args else kw)[key] = val
    with pytest.raises(gqa.GqaError) as e:
        gqa.gqa_decode_attend(args["q"], args["k"], args["v"], args["offsets"], _H, _G, **kw)
    assert e.value.status == gqa.GQA_ERR_SHAPE_MISMATCH


def test_binding_takes_the_split_count_from_partials():
    import torch
    B, H, D = 2, 8, 64
    parts = gqa.State(torch.zeros(B * H, 3), torch.zeros(B * H, 3), torch.zeros(B * H, 3, D))
    n = gqa._check_shapes(torch.zeros(B, H, D), torch.zeros(20, 2, D), torch.zeros(20, 2, D),
                          torch.tensor([0, 10, 20], dtype=torch.int32), H, 2, None, None, None, parts,
                          0, None, None)
    assert n == 3
    with pytest.raises(gqa.GqaError):
        gqa._check_shapes(torch.zeros(B, H, D), torch.zeros(20, 2, D), torch.zeros(20, 2, D),
                          torch.tensor([0, 10, 20], dtype=torch.int32), H, 2, None, None, None, parts,
                          4, None, None)


def test_sizing_query_keeps_the_library_plan():
    """A sizing query only marks partials_out as wanted: a placeholder of any
    shape neither fails nor fixes the split count."""
    import torch
    B, H, D = 2, 8, 64
    one = gqa.State(torch.zeros(1), torch.zeros(1), torch.zeros(1, D))
    n = gqa._check_shapes(torch.zeros(B, H, D), torch.zeros(20, 2, D), torch.zeros(20, 2, D),
                          torch.tensor([0, 10, 20], dtype=torch.int32), H, 2, None, None,
                          torch.zeros(1), one, 0, None, None, sizing=True)
    assert n == 0


def test_plan_invariants_over_random_shapes():
    """For any batch the split plan is a valid cover of the longest sequence:
    chunks of whole 64-row stages, ceil(N / chunk) of them, none empty."""
    import random
    rnd = random.Random(2024)
    for _ in range(2000):
        B = rnd.randint(1, 512)
        G = rnd.choice([1, 2, 4, 8, 16])
        N = rnd.randint(1, 300000)
        full = B * N
        total = rnd.choice([full, rnd.randint(1, full)])
        sm = rnd.choice([1, 8, 132, 148, 160])
        per_sm = rnd.choice([1, 2, 3])
        chunk, splits = gqa.gqa_plan_splits(B, G, N, total, sm, per_sm)
        assert chunk % 64 == 0 and chunk >= 64
        assert splits >= 1 and splits == -(-N // chunk)
        assert (splits - 1) * chunk < N <= splits * chunk
