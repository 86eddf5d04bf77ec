"""Python binding of the B200 grouped-query decode-attention library.

Thin ctypes marshalling over the C ABI declared in ``include/gqa_decode.h``:
every step of the computation runs in the library's CUDA kernels. PyTorch
provides device memory (the tensors passed in, and outputs/workspace allocated
here when the caller gives none) and the current CUDA stream.

The entry points keep the C names:
  gqa_decode_attend, gqa_decode_append_attend, gqa_topk_to_bias,
  gqa_decode_workspace_size, gqa_workspace_init, gqa_softmax_merge,
  gqa_state_finalize, gqa_get_device_error, gqa_plan_splits,
  gqa_status_string, gqa_version, gqa_decode_attend_static_workspace,
  gqa_softmax_merge_gathered, gqa_decode_attend_coded.

If the compiled library is missing the first call raises ``LibraryMissing``;
there is no fallback implementation.
"""
import ctypes
import os

__all__ = [
    "GqaError", "LibraryMissing", "State", "Workspace", "gqa_decode_attend",
    "gqa_decode_append_attend", "gqa_topk_to_bias", "gqa_decode_attend_static_workspace",
    "gqa_softmax_merge_gathered", "gqa_decode_attend_coded",
    "gqa_decode_workspace_size", "gqa_workspace_init", "gqa_softmax_merge", "gqa_state_finalize",
    "gqa_get_device_error", "gqa_plan_splits", "gqa_status_string", "gqa_version", "lib_path",
    "load_library",
]

_PKG = os.path.dirname(os.path.abspath(__file__))
_LIB_PATH = os.path.join(_PKG, "lib", "libgqa_decode.so")

GQA_OK = 0
GQA_ERR_INVALID_ARGUMENT = 1
GQA_ERR_SHAPE_MISMATCH = 2
GQA_ERR_DEVICE = 3
GQA_ERR_WORKSPACE = 4
GQA_ERR_BAD_OFFSETS = 5
GQA_ERR_TIMEOUT = 6
GQA_ERR_BAD_CODES = 7
GQA_F32 = 0
GQA_BF16 = 1
GQA_FLAG_EARLY_START = 1


class LibraryMissing(RuntimeError):
    pass


class GqaError(RuntimeError):
    def __init__(self, status, where=""):
        self.status = int(status)
        super().__init__(f"{where}: {gqa_status_string(self.status)} ({self.status})")


class _CState(ctypes.Structure):
    _fields_ = [("m", ctypes.c_void_p), ("l", ctypes.c_void_p), ("acc", ctypes.c_void_p)]


class _CParams(ctypes.Structure):
    _fields_ = [
        ("struct_size", ctypes.c_uint32),
        ("q", ctypes.c_void_p), ("q_dtype", ctypes.c_int32),
        ("k", ctypes.c_void_p), ("v", ctypes.c_void_p), ("kv_dtype", ctypes.c_int32),
        ("offsets", ctypes.c_void_p),
        ("batch", ctypes.c_int32), ("max_len", ctypes.c_int32), ("max_seq_len", ctypes.c_int32),
        ("num_heads", ctypes.c_int32), ("num_kv_heads", ctypes.c_int32), ("head_dim", ctypes.c_int32),
        ("score_scale", ctypes.c_float),
        ("carry_in", _CState), ("state_out", _CState),
        ("out", ctypes.c_void_p), ("out_dtype", ctypes.c_int32),
        ("partials_out", _CState),
        ("num_splits", ctypes.c_int32),
        ("workspace", ctypes.c_void_p), ("workspace_bytes", ctypes.c_size_t),
        ("bias", ctypes.c_void_p),
        ("flags", ctypes.c_uint32),
    ]


class _CCodes(ctypes.Structure):
    _fields_ = [("k_codes", ctypes.c_void_p), ("v_codes", ctypes.c_void_p), ("words", ctypes.c_int32),
                ("k_atoms", ctypes.c_void_p), ("v_atoms", ctypes.c_void_p), ("n_atoms", ctypes.c_int32)]


_lib = None


def lib_path():
    return _LIB_PATH


def load_library(path=None):
    """Load libgqa_decode.so (once). Raises LibraryMissing if it was never built."""
    global _lib
    if _lib is not None and path is None:
        return _lib
    p = path or _LIB_PATH
    if not os.path.exists(p):
        raise LibraryMissing(
            f"{p} not found: build it with `python -m gqa_decode_attention_attend_b200.build`")
    lib = ctypes.CDLL(p)
    sp = ctypes.c_void_p
    i32, i64 = ctypes.c_int32, ctypes.c_int64
    ps = ctypes.POINTER(_CState)
    lib.gqa_decode_workspace_size.argtypes = [ctypes.POINTER(_CParams), ctypes.POINTER(ctypes.c_size_t),
                                              ctypes.POINTER(i32), ctypes.POINTER(i32)]
    lib.gqa_workspace_init.argtypes = [sp, ctypes.c_size_t, sp]
    lib.gqa_decode_attend.argtypes = [ctypes.POINTER(_CParams), sp]
    lib.gqa_decode_append_attend.argtypes = [ctypes.POINTER(_CParams), sp, sp, sp]
    lib.gqa_decode_attend_coded.argtypes = [ctypes.POINTER(_CParams), ctypes.POINTER(_CCodes), sp]
    lib.gqa_decode_coded_workspace_size.argtypes = [ctypes.POINTER(_CParams), ctypes.POINTER(_CCodes),
                                                    ctypes.POINTER(ctypes.c_size_t), ctypes.POINTER(i32),
                                                    ctypes.POINTER(i32)]
    lib.gqa_topk_to_bias.argtypes = [sp, i32, i32, sp, i32, sp, sp, sp]
    lib.gqa_softmax_merge.argtypes = [ps, i32, i32, i32, ps, ps, sp, i32, sp]
    lib.gqa_softmax_merge_gathered.argtypes = [ps, i32, i32, i32, ps, ps, sp, i32, sp]
    lib.gqa_state_finalize.argtypes = [ps, i32, i32, sp, i32, sp]
    lib.gqa_get_device_error.argtypes = [sp, sp]
    lib.gqa_plan_splits.argtypes = [i32, i32, i32, i64, i32, i32, ctypes.POINTER(i32), ctypes.POINTER(i32)]
    lib.gqa_status_string.argtypes = [ctypes.c_int]
    lib.gqa_status_string.restype = ctypes.c_char_p
    lib.gqa_version.argtypes = []
    for fn in ("gqa_decode_workspace_size", "gqa_workspace_init", "gqa_decode_attend", "gqa_softmax_merge",
               "gqa_state_finalize", "gqa_get_device_error", "gqa_plan_splits",
               "gqa_decode_append_attend", "gqa_topk_to_bias", "gqa_softmax_merge_gathered",
               "gqa_decode_attend_coded", "gqa_decode_coded_workspace_size"):
        getattr(lib, fn).restype = ctypes.c_int
    lib.gqa_version.restype = ctypes.c_int32
    if path is None:
        _lib = lib
    return lib


def gqa_status_string(status):
    return load_library().gqa_status_string(int(status)).decode()


def gqa_version():
    return int(load_library().gqa_version())


def _check(status, where):
    if status != GQA_OK:
        raise GqaError(status, where)


# ------------------------------------------------------------------ torch marshalling

def _torch():
    import torch
    return torch


def _dtype_code(t):
    torch = _torch()
    if t.dtype == torch.float32:
        return GQA_F32
    if t.dtype == torch.bfloat16:
        return GQA_BF16
    raise GqaError(GQA_ERR_SHAPE_MISMATCH, f"dtype {t.dtype}")


def _torch_dtype(code):
    torch = _torch()
    return torch.bfloat16 if code == GQA_BF16 else torch.float32


def _ptr(t):
    if t is None:
        return None
    if not t.is_contiguous():
        raise GqaError(GQA_ERR_INVALID_ARGUMENT, "tensors must be contiguous")
    return t.data_ptr()


def _stream_handle(stream):
    torch = _torch()
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


class State:
    """An online-softmax state (m [n], l [n], acc [n, D]) of fp32 device tensors."""

    def __init__(self, m, l, acc):
        self.m, self.l, self.acc = m, l, acc

    @classmethod
    def empty(cls, rows, head_dim, device, extra=()):
        torch = _torch()
        shape = (rows, *extra)
        return cls(torch.empty(shape, dtype=torch.float32, device=device),
                   torch.empty(shape, dtype=torch.float32, device=device),
                   torch.empty((*shape, head_dim), dtype=torch.float32, device=device))

    def _c(self):
        return _CState(_ptr(self.m), _ptr(self.l), _ptr(self.acc))


def _c_state(s):
    return _CState(None, None, None) if s is None else s._c()


class Workspace:
    """Scratch memory for gqa_decode_attend: a uint8 device tensor, 256-byte
    aligned, zeroed once by gqa_workspace_init (error word and merge tickets).
    It grows on demand (and is then re-initialised); growing frees the old
    buffer in the current stream's order, so a workspace belongs to one stream.
    Calls that may run at the same time (other streams, other threads) need
    workspaces of their own: the functions below fall back to one default
    workspace per device when none is given."""

    def __init__(self, device, nbytes=256):
        self.device = device
        self.tensor = None
        self.reserve(nbytes)

    def reserve(self, nbytes, stream=None):
        torch = _torch()
        if self.tensor is not None and self.tensor.numel() >= nbytes + 256:
            return
        n = max(int(nbytes), 256) + 256
        self.tensor = torch.empty(n, dtype=torch.uint8, device=self.device)
        _check(load_library().gqa_workspace_init(ctypes.c_void_p(self.ptr), self.nbytes,
                                                 _stream_handle(stream)), "gqa_workspace_init")

    @property
    def ptr(self):
        p = self.tensor.data_ptr()
        return (p + 255) & ~255

    @property
    def nbytes(self):
        return self.tensor.numel() - (self.ptr - self.tensor.data_ptr())


_default_ws = {}


def _default_workspace(device):
    key = str(device)
    if key not in _default_ws:
        _default_ws[key] = Workspace(device)
    return _default_ws[key]


def _shape_error(what):
    raise GqaError(GQA_ERR_SHAPE_MISMATCH, what)


def _check_shapes(q, k, v, offsets, num_heads, num_kv_heads, carry, state_out, out, partials_out,
                  num_splits, max_len, bias, kv_is_cache=True, sizing=False):
    """The C ABI sees pointers only: check here that every tensor holds the
    elements the call will touch, so a mismatched tensor is refused instead of
    read or written past its end. Returns the split count to pass (the one
    partials_out is laid out for, when num_splits is 0). A sizing query
    (sizing=True) only marks out / partials_out as wanted: their shapes are
    not checked and the library's own split plan is reported."""
    if offsets.dim() != 1 or offsets.numel() < 1 or str(offsets.dtype) != "torch.int32":
        _shape_error("offsets must be a 1-D int32 tensor of batch + 1 entries")
    B = offsets.numel() - 1
    H = int(num_heads)
    G = int(num_kv_heads) or H
    D = q.shape[-1]
    rows = B * H
    if q.numel() != rows * D:
        _shape_error(f"q holds {q.numel()} elements, expected batch*heads*head_dim = {rows * D}")
    if kv_is_cache:
        for name, t in (("k", k), ("v", v)):
            if t.dim() != 3 or t.shape[1] != G or t.shape[2] != D:
                _shape_error(f"{name} must be [max_len, {G}, {D}], got {list(t.shape)}")
            if max_len is not None and int(max_len) > t.shape[0]:
                _shape_error(f"max_len {int(max_len)} exceeds the {t.shape[0]} rows of {name}")
    if not sizing and out is not None and out.numel() != rows * D:
        _shape_error(f"out holds {out.numel()} elements, expected {rows * D}")
    for name, st in (("carry", carry), ("state_out", state_out)):
        if st is not None and (st.m.numel() != rows or st.l.numel() != rows or st.acc.numel() != rows * D):
            _shape_error(f"{name} must hold m, l [{rows}] and acc [{rows}, {D}]")
    if partials_out is not None and rows > 0 and not sizing:
        S, rem = divmod(partials_out.m.numel(), rows)
        if rem or S < 1 or partials_out.l.numel() != rows * S or partials_out.acc.numel() != rows * S * D:
            _shape_error(f"partials_out must hold m, l [{rows}, S] and acc [{rows}, S, {D}]")
        if int(num_splits) == 0:
            num_splits = S
        elif int(num_splits) != S:
            _shape_error(f"partials_out holds {S} splits per row, num_splits is {int(num_splits)}")
    if bias is not None:
        rows_needed = int(max_len) if max_len is not None else (k.shape[0] if kv_is_cache else 0)
        if bias.numel() < rows_needed:
            _shape_error(f"bias holds {bias.numel()} rows, the cache has {rows_needed}")
    return int(num_splits)


def _params(q, k, v, offsets, num_heads, num_kv_heads, score_scale, carry, state_out, out,
            out_dtype, partials_out, num_splits, max_seq_len, max_len, bias=None, flags=0,
            kv_is_cache=True, sizing=False):
    num_splits = _check_shapes(q, k, v, offsets, num_heads, num_kv_heads, carry, state_out, out,
                               partials_out, num_splits, max_len, bias, kv_is_cache, sizing)
    p = _CParams()
    p.struct_size = ctypes.sizeof(_CParams)
    p.q, p.q_dtype = _ptr(q), _dtype_code(q)
    p.k, p.v, p.kv_dtype = _ptr(k), _ptr(v), _dtype_code(k)
    if v.dtype != k.dtype:
        raise GqaError(GQA_ERR_SHAPE_MISMATCH, "k and v dtypes differ")
    p.offsets = _ptr(offsets)
    p.batch = offsets.numel() - 1
    p.max_len = k.shape[0] if max_len is None else int(max_len)
    p.max_seq_len = int(max_seq_len)
    p.num_heads = int(num_heads)
    p.num_kv_heads = int(num_kv_heads)
    p.head_dim = q.shape[-1]
    p.score_scale = float(score_scale)
    p.carry_in = _c_state(carry)
    p.state_out = _c_state(state_out)
    p.out = _ptr(out)
    p.out_dtype = out_dtype
    p.partials_out = _c_state(partials_out)
    p.num_splits = int(num_splits)
    if bias is not None:
        torch = _torch()
        if bias.dtype != torch.float32:
            raise GqaError(GQA_ERR_SHAPE_MISMATCH, "bias must be float32")
    p.bias = _ptr(bias)
    p.flags = int(flags)
    return p


def gqa_decode_workspace_size(q, k, v, offsets, num_heads, num_kv_heads=0, *, score_scale=0.0,
                              carry=None, state_out=None, want_out=True, partials_out=None,
                              num_splits=0, max_seq_len=0, max_len=None):
    """(bytes, num_splits, chunk_len) the library will use for such a call."""
    torch = _torch()
    # sizing never dereferences out; a one-element placeholder marks it as wanted
    placeholder = torch.empty(1, dtype=q.dtype, device=q.device) if want_out else None
    p = _params(q, k, v, offsets, num_heads, num_kv_heads, score_scale, carry, state_out,
                placeholder, _dtype_code(q), partials_out, num_splits, max_seq_len, max_len,
                sizing=True)
    nbytes = ctypes.c_size_t()
    ns = ctypes.c_int32()
    cl = ctypes.c_int32()
    _check(load_library().gqa_decode_workspace_size(ctypes.byref(p), ctypes.byref(nbytes),
                                                    ctypes.byref(ns), ctypes.byref(cl)),
           "gqa_decode_workspace_size")
    return nbytes.value, ns.value, cl.value


def _attend_call(entry, q, k, v, offsets, num_heads, num_kv_heads, score_scale, carry, state_out, out,
                 out_dtype, partials_out, want_out, num_splits, max_seq_len, max_len, workspace, stream,
                 bias, extra=(), flags=0):
    torch = _torch()
    if want_out is None:
        want_out = out is not None or (state_out is None and partials_out is None)
    odt = _dtype_code(q) if out_dtype is None else (out_dtype if isinstance(out_dtype, int)
                                                    else _dtype_code(torch.empty(0, dtype=out_dtype)))
    if want_out and out is None:
        out = torch.empty(q.shape, dtype=_torch_dtype(odt), device=q.device)
    if out is not None:
        odt = _dtype_code(out)
    p = _params(q, k, v, offsets, num_heads, num_kv_heads, score_scale, carry, state_out, out, odt,
                partials_out, num_splits, max_seq_len, max_len, bias, flags)
    lib = load_library()
    ws = workspace or _default_workspace(q.device)
    sh = _stream_handle(stream)
    p.workspace = ws.ptr
    p.workspace_bytes = ws.nbytes
    st = getattr(lib, entry)(ctypes.byref(p), *extra, sh)
    if st == GQA_ERR_WORKSPACE:
        # too small (checked before anything is launched): size it, grow, retry
        nbytes = ctypes.c_size_t()
        _check(lib.gqa_decode_workspace_size(ctypes.byref(p), ctypes.byref(nbytes), None, None),
               "gqa_decode_workspace_size")
        ws.reserve(nbytes.value, stream)
        p.workspace = ws.ptr
        p.workspace_bytes = ws.nbytes
        st = getattr(lib, entry)(ctypes.byref(p), *extra, sh)
    _check(st, entry)
    return out


def gqa_decode_attend(q, k, v, offsets, num_heads, num_kv_heads=0, *, score_scale=0.0, carry=None,
                      state_out=None, out=None, out_dtype=None, partials_out=None, want_out=None,
                      num_splits=0, max_seq_len=0, max_len=None, workspace=None, stream=None,
                      bias=None, flags=0):
    """Decode attention over a KV cache; see include/gqa_decode.h.

    q [B, H, D]; k, v [max_len, G, D]; offsets int32 [B+1] on the device.
    carry / state_out / partials_out: ``State`` objects or None. ``out`` is
    allocated ([B, H, D], out_dtype or q's dtype) unless given, or unless only
    state_out / partials_out are wanted (want_out=False). bias: optional fp32
    [max_len] additive logit bias per cache row. Returns out (or None).
    """
    return _attend_call("gqa_decode_attend", q, k, v, offsets, num_heads, num_kv_heads, score_scale,
                        carry, state_out, out, out_dtype, partials_out, want_out, num_splits,
                        max_seq_len, max_len, workspace, stream, bias, flags=flags)


def gqa_decode_append_attend(q, k, v, offsets, k_new, v_new, num_heads, num_kv_heads=0, *,
                             score_scale=0.0, carry=None, state_out=None, out=None, out_dtype=None,
                             want_out=None, num_splits=0, max_seq_len=0, max_len=None,
                             workspace=None, stream=None, bias=None, flags=0):
    """Append k_new/v_new [B, G, D] at row offsets[b+1]-1 of the caches (which
    are written), then attend with the new key included; see include/gqa_decode.h."""
    if k_new.dtype != k.dtype or v_new.dtype != k.dtype:
        raise GqaError(GQA_ERR_SHAPE_MISMATCH, "k_new/v_new must have the cache dtype")
    rows_new = (offsets.numel() - 1) * k.shape[1] * k.shape[2]
    if k_new.numel() != rows_new or v_new.numel() != rows_new:
        _shape_error(f"k_new/v_new must be [batch, {k.shape[1]}, {k.shape[2]}]")
    return _attend_call("gqa_decode_append_attend", q, k, v, offsets, num_heads, num_kv_heads,
                        score_scale, carry, state_out, out, out_dtype, None, want_out, num_splits,
                        max_seq_len, max_len, workspace, stream, bias,
                        extra=(ctypes.c_void_p(_ptr(k_new)), ctypes.c_void_p(_ptr(v_new))), flags=flags)


def _coded_params(q, k_codes, v_codes, k_atoms, v_atoms, offsets, num_heads, num_kv_heads, score_scale,
                  carry, state_out, out, odt, partials_out, num_splits, max_seq_len, bias, flags):
    torch = _torch()
    max_len = k_codes.shape[0]
    G = int(num_kv_heads) or int(num_heads)
    D = q.shape[-1]
    for name, t in (("k_codes", k_codes), ("v_codes", v_codes)):
        if t.dim() != 3 or t.shape[0] != max_len or t.shape[1] != G or t.shape[2] != k_codes.shape[2]:
            _shape_error(f"{name} must be [max_len, {G}, words], got {list(t.shape)}")
    for name, t in (("k_atoms", k_atoms), ("v_atoms", v_atoms)):
        if t.dim() != 2 or t.shape[1] != D or t.shape[0] != k_atoms.shape[0] or t.dtype != torch.float32:
            _shape_error(f"{name} must be float32 [n_atoms, {D}], got {list(t.shape)}")
    p = _params(q, q, q, offsets, num_heads, num_kv_heads, score_scale, carry, state_out, out, odt,
                partials_out, num_splits, max_seq_len, max_len, bias, flags, kv_is_cache=False)
    p.k = p.v = None
    codes = _CCodes(_ptr(k_codes), _ptr(v_codes), k_codes.shape[-1], _ptr(k_atoms), _ptr(v_atoms),
                    k_atoms.shape[0])
    return p, codes


def gqa_decode_coded_workspace_size(q, k_codes, v_codes, k_atoms, v_atoms, offsets, num_heads, num_kv_heads=0,
                                    *, score_scale=0.0, carry=None, state_out=None, want_out=True,
                                    partials_out=None, num_splits=0, max_seq_len=0):
    """(bytes, num_splits, chunk_len) of a gqa_decode_attend_coded call (the
    coded kernel's own split plan)."""
    torch = _torch()
    # sizing never dereferences out; a one-element placeholder marks it as wanted
    out = torch.empty(1, dtype=q.dtype, device=q.device) if want_out else None
    p, codes = _coded_params(q, k_codes, v_codes, k_atoms, v_atoms, offsets, num_heads, num_kv_heads,
                             score_scale, carry, state_out, None, _dtype_code(q), partials_out, num_splits,
                             max_seq_len, None, 0)
    p.out = _ptr(out)
    nbytes, ns, cl = ctypes.c_size_t(), ctypes.c_int32(), ctypes.c_int32()
    _check(load_library().gqa_decode_coded_workspace_size(ctypes.byref(p), ctypes.byref(codes),
                                                          ctypes.byref(nbytes), ctypes.byref(ns),
                                                          ctypes.byref(cl)), "gqa_decode_coded_workspace_size")
    return nbytes.value, ns.value, cl.value


def gqa_decode_attend_coded(q, k_codes, v_codes, k_atoms, v_atoms, offsets, num_heads, num_kv_heads=0,
                            *, score_scale=0.0, carry=None, state_out=None, out=None, out_dtype=None,
                            partials_out=None, want_out=None, num_splits=0, max_seq_len=0,
                            workspace=None, stream=None, bias=None, flags=0):
    """Decode attention over a dictionary-coded cache: k_codes / v_codes int32
    or uint32-as-int32 [max_len, G, words] (atom index << 16 | f16 coefficient
    bits), k_atoms / v_atoms fp32 [n_atoms, D]; see include/gqa_decode.h."""
    torch = _torch()
    if want_out is None:
        want_out = out is not None or (state_out is None and partials_out is None)
    odt = _dtype_code(q) if out_dtype is None else _dtype_code(torch.empty(0, dtype=out_dtype))
    if want_out and out is None:
        out = torch.empty(q.shape, dtype=_torch_dtype(odt), device=q.device)
    if out is not None:
        odt = _dtype_code(out)
    p, codes = _coded_params(q, k_codes, v_codes, k_atoms, v_atoms, offsets, num_heads, num_kv_heads,
                             score_scale, carry, state_out, out, odt, partials_out, num_splits, max_seq_len,
                             bias, flags)
    lib = load_library()
    nbytes = ctypes.c_size_t()
    _check(lib.gqa_decode_coded_workspace_size(ctypes.byref(p), ctypes.byref(codes), ctypes.byref(nbytes),
                                               None, None), "gqa_decode_coded_workspace_size")
    ws = workspace or _default_workspace(q.device)
    ws.reserve(nbytes.value, stream)
    p.workspace = ws.ptr
    p.workspace_bytes = ws.nbytes
    _check(lib.gqa_decode_attend_coded(ctypes.byref(p), ctypes.byref(codes), _stream_handle(stream)),
           "gqa_decode_attend_coded")
    return out


def gqa_topk_to_bias(idx, offsets, max_len, bias=None, workspace=None, stream=None):
    """fp32 bias [max_len] from index rows idx [B, width] (int32, relative key
    positions, -1 = INVALID): selected keys 0, the sequences' other rows -inf.
    Rows outside every sequence keep their value (0 when bias is allocated here)."""
    torch = _torch()
    if bias is None:
        bias = torch.zeros(int(max_len), dtype=torch.float32, device=offsets.device)
    B = offsets.numel() - 1
    width = idx.shape[1] if idx.dim() == 2 else 0
    _check(load_library().gqa_topk_to_bias(ctypes.c_void_p(_ptr(idx)), B, width,
                                           ctypes.c_void_p(_ptr(offsets)), int(max_len),
                                           ctypes.c_void_p(_ptr(bias)),
                                           ctypes.c_void_p(workspace.ptr) if workspace else None,
                                           _stream_handle(stream)), "gqa_topk_to_bias")
    return bias


def gqa_softmax_merge(states, carry=None, merged_out=None, out=None, out_dtype=None, want_out=None,
                      stream=None):
    """Merge states (m, l [rows, S]; acc [rows, S, D]) with an optional carry.
    Returns out [rows, D] (allocated unless given or want_out=False)."""
    torch = _torch()
    rows, S = states.m.shape
    D = states.acc.shape[-1]
    if want_out is None:
        want_out = out is not None or merged_out is None
    if want_out and out is None:
        out = torch.empty((rows, D), dtype=out_dtype or torch.float32, device=states.m.device)
    odt = _dtype_code(out) if out is not None else GQA_F32
    cs = states._c()
    cc = _c_state(carry)
    cm = _c_state(merged_out)
    _check(load_library().gqa_softmax_merge(ctypes.byref(cs), rows, S, D, ctypes.byref(cc),
                                            ctypes.byref(cm), _ptr(out), odt, _stream_handle(stream)),
           "gqa_softmax_merge")
    return out


def gqa_softmax_merge_gathered(states, carry=None, merged_out=None, out=None, out_dtype=None,
                               want_out=None, stream=None):
    """Merge states gathered as m, l [S, rows]; acc [S, rows, D] (one block per
    contributor, as an all-gather lays them out) with an optional carry."""
    torch = _torch()
    S, rows = states.m.shape
    D = states.acc.shape[-1]
    if want_out is None:
        want_out = out is not None or merged_out is None
    if want_out and out is None:
        out = torch.empty((rows, D), dtype=out_dtype or torch.float32, device=states.m.device)
    odt = _dtype_code(out) if out is not None else GQA_F32
    cs = states._c()
    cc = _c_state(carry)
    cm = _c_state(merged_out)
    _check(load_library().gqa_softmax_merge_gathered(ctypes.byref(cs), rows, S, D, ctypes.byref(cc),
                                                     ctypes.byref(cm), _ptr(out), odt,
                                                     _stream_handle(stream)),
           "gqa_softmax_merge_gathered")
    return out


def gqa_state_finalize(state, out=None, out_dtype=None, stream=None):
    """out = acc / l for a state (m, l [rows]; acc [rows, D])."""
    torch = _torch()
    rows = state.m.shape[0]
    D = state.acc.shape[-1]
    if out is None:
        out = torch.empty((rows, D), dtype=out_dtype or torch.float32, device=state.m.device)
    cs = state._c()
    _check(load_library().gqa_state_finalize(ctypes.byref(cs), rows, D, _ptr(out), _dtype_code(out),
                                             _stream_handle(stream)), "gqa_state_finalize")
    return out


def gqa_get_device_error(workspace=None, device=None, stream=None):
    """Synchronise and return (and clear) the workspace's device error status."""
    ws = workspace or _default_workspace(device if device is not None else _torch().device("cuda"))
    return load_library().gqa_get_device_error(ctypes.c_void_p(ws.ptr), _stream_handle(stream))


def gqa_workspace_init(workspace, stream=None):
    _check(load_library().gqa_workspace_init(ctypes.c_void_p(workspace.ptr), workspace.nbytes,
                                             _stream_handle(stream)), "gqa_workspace_init")


def gqa_plan_splits(batch, num_kv_heads, max_seq_len, total_rows, sm_count=148, ctas_per_sm=2):
    """(chunk_len, num_splits) of the library's split heuristic (host only)."""
    c = ctypes.c_int32()
    s = ctypes.c_int32()
    _check(load_library().gqa_plan_splits(int(batch), int(num_kv_heads), int(max_seq_len),
                                          int(total_rows), int(sm_count), int(ctas_per_sm),
                                          ctypes.byref(c), ctypes.byref(s)), "gqa_plan_splits")
    return c.value, s.value


def gqa_decode_attend_static_workspace(q, k, v, offsets, num_heads, num_kv_heads=0, *, score_scale=0.0,
                                       carry=None, state_out=None, out=None, out_dtype=None,
                                       partials_out=None, want_out=None, num_splits=0, max_seq_len=0,
                                       max_len=None, stream=None):
    """gqa_decode_attend for callers that cannot provide scratch memory.

    Same arguments and result as gqa_decode_attend minus the workspace: the
    library keeps its scratch in a fixed 16 MiB device array of its own (see
    include/gqa_decode.h for who needs this and its limits). Calls that may run
    concurrently on the GPU share that array and must be serialised.
    """
    torch = _torch()
    lib = load_library()
    fn = lib.gqa_decode_attend_static_workspace
    fn.argtypes = [ctypes.POINTER(_CParams), ctypes.c_void_p]
    fn.restype = ctypes.c_int
    if want_out is None:
        want_out = out is not None or (state_out is None and partials_out is None)
    odt = _dtype_code(q) if out_dtype is None else _dtype_code(torch.empty(0, dtype=out_dtype))
    if want_out and out is None:
        out = torch.empty(q.shape, dtype=_torch_dtype(odt), device=q.device)
    if out is not None:
        odt = _dtype_code(out)
    p = _params(q, k, v, offsets, num_heads, num_kv_heads, score_scale, carry, state_out, out, odt,
                partials_out, num_splits, max_seq_len, max_len)
    _check(fn(ctypes.byref(p), _stream_handle(stream)), "gqa_decode_attend_static_workspace")
    return out
