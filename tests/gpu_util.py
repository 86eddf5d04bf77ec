"""Helpers for the GPU parity tests: move a workload to the device, run the
library through its C ABI, run the f64 oracle on the same stored inputs, and
compare element by element.

Tolerances (per element, |gpu - oracle| <= atol + rtol * |oracle|):
  fp32 K/V: 1e-5 + 1e-5 rel;  bf16 K/V: 2e-3 + 2e-3 rel  (fp32 accumulation).
These apply to the output requested in fp32 and to the state's m and l. The
state's acc is the unnormalised value sum (acc = out * l), so its bound is the
output bound carried into those units: atol * l + rtol * |acc|. An output
requested in bf16 is additionally rounded to nearest-even by the format itself,
which can move it by up to 2^-8 relative; for bf16 outputs the bound is widened
by exactly that.
"""
import math

import numpy as np
import torch

import oracle
import gqa_decode_attention_attend_b200 as gqa
from gqa_decode_attention_attend_b200 import workloads

TOL = {torch.float32: (1e-5, 1e-5), torch.bfloat16: (2e-3, 2e-3)}
BF16_RNE_REL = 2.0 ** -8


def device():
    if not torch.cuda.is_available():
        raise RuntimeError("GPU test run without a CUDA device")
    return torch.device("cuda:0")


class DevWorkload:
    def __init__(self, w, dev):
        self.w = w
        self.q = w.q.to(dev)
        self.k = w.k.to(dev)
        self.v = w.v.to(dev)
        self.offsets = w.offsets.to(dev)
        self.carry = None
        if w.carry is not None:
            self.carry = gqa.State(*(c.to(dev).contiguous() for c in w.carry))


def run(dw, *, out_dtype=None, with_state=False, carry=True, num_splits=0, max_seq_len=None,
        partials=None, score_scale=None):
    w = dw.w
    rows = w.batch * w.num_heads
    st = gqa.State.empty(rows, w.head_dim, dw.q.device) if with_state else None
    out = gqa.gqa_decode_attend(
        dw.q, dw.k, dw.v, dw.offsets, w.num_heads, w.num_kv_heads,
        score_scale=w.score_scale if score_scale is None else score_scale,
        carry=dw.carry if carry else None, state_out=st, out_dtype=out_dtype,
        partials_out=partials, num_splits=num_splits, want_out=partials is None,
        max_seq_len=w.max_seq_len if max_seq_len is None else max_seq_len)
    return out, st


def oracle_state(w, rows=None, carry=True, score_scale=None):
    c = None
    if carry and w.carry is not None:
        c = tuple(t.numpy() for t in w.carry)
    return oracle.decode_attend(
        workloads.host_array(w.q), workloads.host_array(w.k), workloads.host_array(w.v),
        w.offsets.numpy(), w.num_heads, w.num_kv_heads,
        w.score_scale if score_scale is None else score_scale, carry=c, rows=rows)


def assert_close(got, ref, kv_dtype, what, bf16_out=False):
    atol, rtol = TOL[kv_dtype]
    g = np.asarray(got, np.float64)
    r = np.asarray(ref, np.float64)
    assert g.shape == r.shape, f"{what}: shape {g.shape} vs {r.shape}"
    bound = atol + rtol * np.abs(r)
    if bf16_out:
        bound = bound + BF16_RNE_REL * np.abs(r)
    both_inf = np.isinf(g) & np.isinf(r) & (np.sign(g) == np.sign(r))
    err = np.where(both_inf, 0.0, np.abs(g - r))
    bad = ~(err <= bound)
    if bad.any():
        i = np.unravel_index(np.argmax(np.where(bad, err - bound, -np.inf)), err.shape)
        raise AssertionError(f"{what}: {int(bad.sum())} of {bad.size} elements out of tolerance; "
                             f"worst at {i}: gpu {g[i]!r} oracle {r[i]!r} bound {bound[i]!r}")


def check_out(out, ref_state, w, rows=None, what="out"):
    o = out.float().reshape(-1, w.head_dim).cpu().numpy()
    if rows is not None:
        o = o[rows]
    assert_close(o, ref_state.out, w.k.dtype, what, bf16_out=(out.dtype == torch.bfloat16))


def assert_acc_close(acc, ref_acc, ref_l, kv_dtype, what):
    """acc is the UNnormalised value sum (acc = out * l): its tolerance is the
    output tolerance carried into those units, atol * l + rtol * |acc|."""
    atol, rtol = TOL[kv_dtype]
    g = np.asarray(acc, np.float64)
    r = np.asarray(ref_acc, np.float64)
    lr = np.asarray(ref_l, np.float64)[..., None]
    bound = atol * np.maximum(lr, 1.0) + rtol * np.abs(r)
    err = np.abs(g - r)
    bad = ~(err <= bound)
    if bad.any():
        i = np.unravel_index(np.argmax(np.where(bad, err - bound, -np.inf)), err.shape)
        raise AssertionError(f"{what}: {int(bad.sum())} of {bad.size} elements out of tolerance; "
                             f"worst at {i}: gpu {g[i]!r} oracle {r[i]!r} bound {bound[i]!r}")


def check_state(st, ref_state, w, rows=None, what="state"):
    m = st.m.cpu().numpy().astype(np.float64)
    l = st.l.cpu().numpy().astype(np.float64)
    acc = st.acc.cpu().numpy().astype(np.float64)
    if rows is not None:
        m, l, acc = m[rows], l[rows], acc[rows]
    assert_close(m, ref_state.m, w.k.dtype, what + ".m")
    assert_close(l, ref_state.l, w.k.dtype, what + ".l")
    assert_acc_close(acc, ref_state.acc, ref_state.l, w.k.dtype, what + ".acc")


def split_ranges(w, chunk_len, num_splits):
    """Key range [lo, hi) of each split of each sequence, as the library defines it:
    split s covers keys [s*chunk_len, (s+1)*chunk_len), the last one also any rest."""
    out = []
    for n in w.lengths:
        rs = []
        for s in range(num_splits):
            lo = min(n, s * chunk_len)
            hi = n if s == num_splits - 1 else min(n, (s + 1) * chunk_len)
            rs.append((lo, max(lo, hi)))
        out.append(rs)
    return out


def oracle_partial(w, b, lo, hi, heads):
    """f64 state of query heads `heads` of sequence b over its keys [lo, hi)."""
    base = int(w.offsets[b])
    off = np.array([base + lo, base + hi], np.int32)
    q = workloads.host_array(w.q)[b:b + 1]
    st = oracle.decode_attend(q, workloads.host_array(w.k), workloads.host_array(w.v), off,
                              w.num_heads, w.num_kv_heads, w.score_scale, rows=list(heads))
    return st


def default_scale(d):
    return 1.0 / math.sqrt(d)
