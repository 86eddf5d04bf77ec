"""f64 CPU oracle for grouped-query decode attention -- TEST INFRASTRUCTURE.

Only the test suite, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package. The library's product path never calls
it and shares no code with it (the CUDA sources live in
``gqa_decode_attention_attend_b200/csrc`` and are never included here).

The arithmetic lives in ``gqa_oracle.cpp`` (plain C++17, f64, two passes per
query row); this module only marshals numpy arrays through ctypes.

What it computes, with its sources:
  * decode attention of one query token per sequence over a KV cache laid out
    ``[rows, num_kv_heads, head_dim]``; Q head h reads KV head
    ``h // (H // G)`` -- needle_core ``attn.rs``, ``KvCache`` and
    ``self_attn_incremental``;
  * scale ``score_scale`` or ``head_dim ** -0.5`` when it is 0 -- USearch
    linear algebra, ``DenseAttendConfig::score_scale``;
  * ragged sequences as Arrow offsets, the carry ``(m, l, acc)`` folded by
    partial-softmax rescaling, and outputs divided by the partition -- USearch
    linear algebra, § Attention and ``DenseSoftmaxState``;
  * an empty softmax gives weight 0 (output 0, not NaN) -- metrale
    glm5next_dsa_ref ``pool_states``.

Every function here is pinned by tests/test_oracle_pins.py against brute force,
closed forms and invariants; none is "parity unpinned".
"""
import ctypes
import os

import numpy as np

from . import build as _build

_HERE = os.path.dirname(os.path.abspath(__file__))
_LIB_CACHE = {}

_f32p = ctypes.POINTER(ctypes.c_float)
_f64p = ctypes.POINTER(ctypes.c_double)
_i32p = ctypes.POINTER(ctypes.c_int32)
_i64p = ctypes.POINTER(ctypes.c_int64)


def load(path=None):
    """Load (building first if stale) the oracle shared library."""
    path = path or _build.DEFAULT_OUT
    if path == _build.DEFAULT_OUT and _build.needs_build(path):
        _build.build(path)
    if path in _LIB_CACHE:
        return _LIB_CACHE[path]
    lib = ctypes.CDLL(path)
    lib.oracle_decode_attend.restype = ctypes.c_int
    lib.oracle_decode_attend.argtypes = [
        ctypes.c_void_p, ctypes.c_int, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int,
        _i32p, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_double,
        _f32p, _f32p, _f32p, _f32p, _i64p, ctypes.c_int64, _f64p, _f64p, _f64p, _f64p,
        ctypes.c_int]
    lib.oracle_topk_to_bias.restype = ctypes.c_int
    lib.oracle_topk_to_bias.argtypes = [_i32p, ctypes.c_int, ctypes.c_int, _i32p, _f32p,
                                        ctypes.c_int64]
    lib.oracle_softmax_merge.restype = ctypes.c_int
    lib.oracle_softmax_merge.argtypes = [
        _f32p, _f32p, _f32p, ctypes.c_int64, ctypes.c_int, ctypes.c_int,
        _f32p, _f32p, _f32p, _f64p, _f64p, _f64p, _f64p, ctypes.c_int]
    lib.oracle_reconstruct_words.restype = ctypes.c_int
    lib.oracle_reconstruct_words.argtypes = [ctypes.POINTER(ctypes.c_uint32), ctypes.c_int64, ctypes.c_int,
                                             _f32p, ctypes.c_int, ctypes.c_int, _f64p]
    lib.oracle_f16_to_f64.restype = ctypes.c_double
    lib.oracle_f16_to_f64.argtypes = [ctypes.c_uint16]
    lib.oracle_bf16_to_f64.restype = ctypes.c_double
    lib.oracle_bf16_to_f64.argtypes = [ctypes.c_uint16]
    lib.oracle_default_threads.restype = ctypes.c_int
    lib.oracle_default_threads.argtypes = []
    _LIB_CACHE[path] = lib
    return lib


def _ptr(a, t):
    return None if a is None else a.ctypes.data_as(t)


def _as_stored(x):
    """Return (contiguous ndarray, kind) for an fp32 array (0), bf16 bits (1)
    or f64 (2, e.g. a reconstructed cache).

    bf16 data is passed as its raw uint16 bit patterns (numpy has no bf16).
    """
    x = np.ascontiguousarray(x)
    if x.dtype == np.uint16:
        return x, 1
    if x.dtype == np.float32:
        return x, 0
    if x.dtype == np.float64:
        return x, 2
    raise TypeError(f"oracle inputs are float32, f64 or bf16 bits (uint16), got {x.dtype}")


class State:
    """An online-softmax state in f64: m, l [n]; acc [n, D]; out = acc / l."""

    def __init__(self, m, l, acc, out):
        self.m, self.l, self.acc, self.out = m, l, acc, out


def decode_attend(q, k, v, offsets, num_heads, num_kv_heads, score_scale=0.0,
                  carry=None, rows=None, n_threads=0, lib=None, bias=None):
    """Exact decode attention in f64.

    q: [B, H, D]; k, v: [rows, G, D] (float32 or bf16 bits as uint16);
    offsets: int32 [B+1]; carry: optional (m [B*H], l [B*H], acc [B*H, D]) fp32;
    rows: optional list of flat (b*H + h) rows to evaluate (default all);
    bias: optional fp32 [rows of the cache], added to the scaled logit of each
    cache row (-inf masks a key out).
    Returns a State whose arrays follow ``rows`` order.
    """
    lib = lib or load()
    q, q_bf16 = _as_stored(q)
    k, kv_bf16 = _as_stored(k)
    v, v_bf16 = _as_stored(v)
    if v_bf16 != kv_bf16:
        raise TypeError("k and v must share a dtype")
    offsets = np.ascontiguousarray(offsets, dtype=np.int32)
    B = offsets.shape[0] - 1
    D = q.shape[-1]
    H, G = int(num_heads), int(num_kv_heads)
    if rows is None:
        row_arr = None
        n = B * H
    else:
        row_arr = np.ascontiguousarray(rows, dtype=np.int64)
        n = row_arr.shape[0]
    om = np.empty(n, np.float64)
    ol = np.empty(n, np.float64)
    oacc = np.empty((n, D), np.float64)
    out = np.empty((n, D), np.float64)
    cm = cl = cacc = None
    if carry is not None:
        cm, cl, cacc = (np.ascontiguousarray(c, dtype=np.float32) for c in carry)
    bias_arr = None if bias is None else np.ascontiguousarray(bias, dtype=np.float32)
    rc = lib.oracle_decode_attend(
        q.ctypes.data, q_bf16, k.ctypes.data, v.ctypes.data, kv_bf16, _ptr(offsets, _i32p),
        B, H, G, D, float(score_scale), _ptr(bias_arr, _f32p),
        _ptr(cm, _f32p), _ptr(cl, _f32p), _ptr(cacc, _f32p),
        _ptr(row_arr, _i64p), n, _ptr(om, _f64p), _ptr(ol, _f64p), _ptr(oacc, _f64p),
        _ptr(out, _f64p), int(n_threads))
    if rc != 0:
        raise ValueError("oracle_decode_attend refused its arguments")
    return State(om, ol, oacc, out)


def softmax_merge(m, l, acc, carry=None, n_threads=0, lib=None):
    """Exact f64 merge of fp32 states m, l [rows, S], acc [rows, S, D] (+carry)."""
    lib = lib or load()
    m = np.ascontiguousarray(m, dtype=np.float32)
    l = np.ascontiguousarray(l, dtype=np.float32)
    acc = np.ascontiguousarray(acc, dtype=np.float32)
    rows, S = m.shape
    D = acc.shape[-1]
    om = np.empty(rows, np.float64)
    ol = np.empty(rows, np.float64)
    oacc = np.empty((rows, D), np.float64)
    out = np.empty((rows, D), np.float64)
    cm = cl = cacc = None
    if carry is not None:
        cm, cl, cacc = (np.ascontiguousarray(c, dtype=np.float32) for c in carry)
    rc = lib.oracle_softmax_merge(
        _ptr(m, _f32p), _ptr(l, _f32p), _ptr(acc, _f32p), rows, S, D,
        _ptr(cm, _f32p), _ptr(cl, _f32p), _ptr(cacc, _f32p),
        _ptr(om, _f64p), _ptr(ol, _f64p), _ptr(oacc, _f64p), _ptr(out, _f64p), int(n_threads))
    if rc != 0:
        raise ValueError("oracle_softmax_merge refused its arguments")
    return State(om, ol, oacc, out)


def topk_to_bias(idx, offsets, rows, lib=None, fill=0.0):
    """Additive bias per cache row from index rows idx [B, width] (int32,
    positions relative to each sequence, -1 = INVALID): 0 for selected keys,
    -inf for the other rows of each sequence, `fill` outside every sequence."""
    lib = lib or load()
    idx = np.ascontiguousarray(idx, dtype=np.int32)
    offsets = np.ascontiguousarray(offsets, dtype=np.int32)
    B = offsets.shape[0] - 1
    width = idx.shape[1] if idx.ndim == 2 else 0
    bias = np.full(int(rows), fill, np.float32)
    rc = lib.oracle_topk_to_bias(_ptr(idx, _i32p), B, width, _ptr(offsets, _i32p),
                                 _ptr(bias, _f32p), int(rows))
    if rc != 0:
        raise ValueError("oracle_topk_to_bias refused its arguments")
    return bias


def append_then_attend(q, k, v, offsets, k_new, v_new, num_heads, num_kv_heads, score_scale=0.0,
                       **kw):
    """A decode step with the new token appended first (needle_core attn.rs:
    KvCache::push_kv, then self_attn_incremental): row offsets[b+1]-1 of the
    cache takes k_new[b], v_new[b]; then exact attention over the updated cache.
    Returns (State, k_after, v_after) on host copies; the inputs are not modified."""
    k2 = np.array(k, copy=True)
    v2 = np.array(v, copy=True)
    offsets = np.asarray(offsets, dtype=np.int64)
    for b in range(offsets.shape[0] - 1):
        if offsets[b + 1] > offsets[b]:
            k2[offsets[b + 1] - 1] = k_new[b]
            v2[offsets[b + 1] - 1] = v_new[b]
    st = decode_attend(q, k2, v2, offsets.astype(np.int32), num_heads, num_kv_heads, score_scale,
                       **kw)
    return st, k2, v2


def reconstruct_words(codes, atoms, lib=None):
    """f64 rows from dictionary code words: codes uint32 [..., words] (atom index
    in the high 16 bits, f16 coefficient bits in the low 16), atoms fp32
    [n_atoms, D]. Returns f64 [..., D]."""
    lib = lib or load()
    codes = np.ascontiguousarray(codes, dtype=np.uint32)
    atoms = np.ascontiguousarray(atoms, dtype=np.float32)
    words = codes.shape[-1]
    n = int(np.prod(codes.shape[:-1]))
    D = atoms.shape[1]
    out = np.empty((n, D), np.float64)
    rc = lib.oracle_reconstruct_words(codes.ctypes.data_as(ctypes.POINTER(ctypes.c_uint32)), n, words,
                                      _ptr(atoms, _f32p), atoms.shape[0], D, _ptr(out, _f64p))
    if rc != 0:
        raise ValueError("oracle_reconstruct_words refused its arguments")
    return out.reshape(*codes.shape[:-1], D)


def coded_decode_attend(q, k_codes, v_codes, k_atoms, v_atoms, offsets, num_heads, num_kv_heads,
                        score_scale=0.0, lib=None, **kw):
    """Decode attention over a dictionary-coded cache: reconstruct K and V
    (f64, from the code words) and apply the plain definition."""
    k = reconstruct_words(k_codes, k_atoms, lib=lib)
    v = reconstruct_words(v_codes, v_atoms, lib=lib)
    return decode_attend(q, k, v, offsets, num_heads, num_kv_heads, score_scale, lib=lib, **kw)


def f16_to_f64(bits, lib=None):
    lib = lib or load()
    return lib.oracle_f16_to_f64(int(bits))


def bf16_to_f64(bits, lib=None):
    lib = lib or load()
    return lib.oracle_bf16_to_f64(int(bits))


def default_threads(lib=None):
    lib = lib or load()
    return lib.oracle_default_threads()
