"""Pins for the f64 oracle: checks that do not go through the oracle's own formula.

Each pin takes an oracle handle (the ``oracle`` package functions bound to one
compiled library, so mutated builds can be pinned too) and raises
AssertionError when the oracle disagrees with:
  * brute force on tiny inputs -- a numpy matrix-form softmax with explicit
    per-head K/V expansion and *unshifted* exponentials, the carry entering as
    one extra pseudo-key of weight l_c e^{m_c} and value acc_c / l_c;
  * closed forms -- a single key returns its value row; constant values return
    that constant; a zero query averages the values; two keys with logit gap
    delta take weights 1/(1+e^delta) and e^delta/(1+e^delta);
  * invariants -- heads of one group with identical queries agree; permuting
    the KV heads permutes the outputs; merging the states of two disjoint key
    sets equals attending over their union; an empty carry changes nothing;
    adding a constant to every logit changes nothing; a planted high-logit key
    dominates; ``score_scale = 0`` means ``1/sqrt(head_dim)``;
  * the additive bias row -- brute force with the bias added after the scale; a
    constant bias only shifts m; a -inf bias equals removing the key; index rows
    turned into a mask keep exactly the distinct in-range indices; appending a
    token writes only its row and attends over it;
  * the dictionary-coded cache -- binary16 coefficients on fixed bit patterns;
    reconstruction against numpy's sum of coefficient * atom; one-hot codes
    over the cache's own rows give plain attention exactly.

Sources: needle_core ``attn.rs`` (``KvCache`` layout, ``self_attn_incremental``
head map and scale); USearch linear algebra § Attention (online softmax folded
into the walk, carry by partial-softmax rescaling, outputs divided by the
partition, ``score_scale`` zero derives it); cortiq_engine ``NystromState``
example ``trial`` (planted key); metrale glm5next_dsa_ref ``pool_states``
(empty softmax gives 0, not NaN) and ``topk_to_mask`` (index rows -> mask);
needle_core ``attn.rs`` ``attn_bias`` and ``KvCache::push_kv``; qualiaDB
``KvDictionary`` ``reconstruct`` / ``reconstruct_from_words``.
"""
import math

import numpy as np


class OracleHandle:
    """The oracle's two entry points bound to one compiled library."""

    def __init__(self, oracle_pkg, lib):
        self.pkg = oracle_pkg
        self.lib = lib

    def attend(self, *a, **kw):
        kw.setdefault("lib", self.lib)
        return self.pkg.decode_attend(*a, **kw)

    def merge(self, *a, **kw):
        kw.setdefault("lib", self.lib)
        return self.pkg.softmax_merge(*a, **kw)

    def bf16(self, bits):
        return self.pkg.bf16_to_f64(bits, lib=self.lib)

    def topk_to_bias(self, *a, **kw):
        kw.setdefault("lib", self.lib)
        return self.pkg.topk_to_bias(*a, **kw)

    def reconstruct(self, *a, **kw):
        kw.setdefault("lib", self.lib)
        return self.pkg.reconstruct_words(*a, **kw)


def _rng(seed):
    return np.random.default_rng(seed)


def _offsets(lengths):
    o = np.zeros(len(lengths) + 1, np.int32)
    o[1:] = np.cumsum(lengths)
    return o


def _tiny(seed, lengths, H, G, D, scale=0.7):
    r = _rng(seed)
    R = int(sum(lengths))
    q = r.uniform(-1, 1, (len(lengths), H, D)).astype(np.float32)
    k = r.uniform(-1, 1, (R, G, D)).astype(np.float32)
    v = r.uniform(-1, 1, (R, G, D)).astype(np.float32)
    return q, k, v, _offsets(lengths)


def brute_force(q, k, v, offsets, H, G, scale, carry=None, bias=None):
    """softmax(q K^T * scale + bias) V per (b, h), matrix form, unshifted exp, in f64.
    A bias of -inf gives its key weight exactly 0."""
    q = q.astype(np.float64)
    k = k.astype(np.float64)
    v = v.astype(np.float64)
    B, _, D = q.shape
    rep = H // G
    out = np.zeros((B * H, D))
    for b in range(B):
        kb = k[offsets[b]:offsets[b + 1]]            # [n, G, D]
        vb = v[offsets[b]:offsets[b + 1]]
        # explicit repeat-copy of each KV head to its Q heads: [n, H, D]
        k_h = np.repeat(kb, rep, axis=1)
        v_h = np.repeat(vb, rep, axis=1)
        logits = np.einsum("hd,nhd->hn", q[b], k_h) * scale        # [H, n]
        if bias is not None:
            logits = logits + np.asarray(bias, np.float64)[offsets[b]:offsets[b + 1]][None, :]
        w = np.exp(logits)
        num = np.einsum("hn,nhd->hd", w, v_h)
        den = w.sum(axis=1)
        if carry is not None:
            cm, cl, cacc = (np.asarray(c, np.float64) for c in carry)
            sl = slice(b * H, (b + 1) * H)
            wc = np.where(cl[sl] != 0, cl[sl] * np.exp(cm[sl]), 0.0)
            vc = np.where(cl[sl, None] != 0, cacc[sl] / np.where(cl[sl, None] != 0, cl[sl, None], 1), 0)
            num = num + wc[:, None] * vc
            den = den + wc
        out[b * H:(b + 1) * H] = np.where(den[:, None] > 0, num / np.where(den[:, None] > 0, den[:, None], 1), 0)
    return out


def _close(a, b, rtol=1e-12, atol=1e-12, what=""):
    a = np.asarray(a, np.float64)
    b = np.asarray(b, np.float64)
    if a.shape != b.shape or not np.allclose(a, b, rtol=rtol, atol=atol, equal_nan=False):
        err = np.max(np.abs(a - b)) if a.shape == b.shape else "shape"
        raise AssertionError(f"{what}: max err {err}")


# ----------------------------------------------------------------------------- pins

def pin_bf16_widening(o):
    cases = {0x3F80: 1.0, 0xC000: -2.0, 0x0000: 0.0, 0x4049: 3.140625, 0x0001: 2.0 ** -133,
             0x7F7F: 3.3895313892515355e38, 0x3C00: 2.0 ** -7, 0xBF40: -0.75}
    for bits, want in cases.items():
        got = o.bf16(bits)
        assert got == want, f"bf16 0x{bits:04x}: {got} != {want}"
    assert o.bf16(0x7F80) == math.inf and o.bf16(0xFF80) == -math.inf


def pin_brute_force_tiny(o):
    shapes = [([5], 1, 1, 3), ([3, 8, 1], 4, 2, 4), ([6, 2], 6, 3, 2), ([7, 0, 4], 8, 2, 5),
              ([2, 5], 4, 4, 3)]
    for i, (lengths, H, G, D) in enumerate(shapes):
        q, k, v, off = _tiny(100 + i, lengths, H, G, D)
        for scale in (0.7, 0.0):
            st = o.attend(q, k, v, off, H, G, score_scale=scale)
            eff = scale if scale != 0.0 else 1.0 / math.sqrt(D)
            _close(st.out, brute_force(q, k, v, off, H, G, eff), what=f"brute force {i}")
        # with a carry: m ~ N(0,1), l ~ U(1,3), acc ~ U(-1,1); one row's carry empty
        r = _rng(200 + i)
        n = len(lengths) * H
        cm = r.normal(0, 1, n).astype(np.float32)
        cl = r.uniform(1, 3, n).astype(np.float32)
        cl[0] = 0.0
        cacc = r.uniform(-1, 1, (n, D)).astype(np.float32)
        st = o.attend(q, k, v, off, H, G, score_scale=0.7, carry=(cm, cl, cacc))
        _close(st.out, brute_force(q, k, v, off, H, G, 0.7, carry=(cm, cl, cacc)),
               what=f"brute force + carry {i}")
        # the partition and the running max against their definitions
        for row in range(n):
            b, h = divmod(row, H)
            g = h // (H // G)
            ks = k[off[b]:off[b + 1], g].astype(np.float64)
            logits = list(ks @ q[b, h].astype(np.float64) * 0.7)
            if cl[row] != 0:
                logits.append(float(cm[row]))
            if not logits:
                assert st.m[row] == -math.inf and st.l[row] == 0.0
                continue
            mx = max(logits)
            assert abs(st.m[row] - mx) <= 1e-12 * max(1.0, abs(mx)), "running max"
            lsum = sum(math.exp(x - mx) for x in logits[: len(ks)])
            if cl[row] != 0:
                lsum += float(cl[row]) * math.exp(float(cm[row]) - mx)
            assert abs(st.l[row] - lsum) <= 1e-12 * lsum, "partition"
            _close(st.acc[row], st.out[row] * st.l[row], rtol=1e-12, atol=1e-13, what="acc = out*l")


def pin_single_key(o):
    for D in (1, 4, 64):
        for G, H in ((1, 1), (2, 4), (4, 8)):
            q, k, v, off = _tiny(300 + D + H, [1, 1, 1], H, G, D)
            st = o.attend(q, k, v, off, H, G)
            for row in range(3 * H):
                b, h = divmod(row, H)
                g = h // (H // G)
                assert np.array_equal(st.out[row], v[off[b], g].astype(np.float64)), "single key"
                assert st.l[row] == 1.0


def pin_constant_v(o):
    q, k, v, off = _tiny(400, [9, 33], 6, 2, 8)
    c = np.linspace(-3, 3, 8).astype(np.float32)
    v[:] = c
    st = o.attend(q, k, v, off, 6, 2, score_scale=1.3)
    for row in range(12):
        _close(st.out[row], c, rtol=1e-14, atol=1e-15, what="constant V")


def pin_zero_query_mean(o):
    # all logits 0 => every weight is 1/N and out is the mean of the group's values
    q, k, v, off = _tiny(500, [4, 7], 4, 2, 3)
    q[:] = 0.0
    st = o.attend(q, k, v, off, 4, 2)
    for row in range(8):
        b, h = divmod(row, 4)
        g = h // 2
        want = v[off[b]:off[b + 1], g].astype(np.float64).mean(axis=0)
        _close(st.out[row], want, rtol=1e-14, atol=1e-15, what="zero query")
        assert st.m[row] == 0.0 and st.l[row] == off[b + 1] - off[b]


def pin_two_key_closed_form(o):
    # D = 1, q = 1, keys 0 and delta/scale => logits 0 and delta
    for delta in (0.5, 2.0, -3.0):
        scale = 0.25
        q = np.ones((1, 1, 1), np.float32)
        k = np.array([[[0.0]], [[delta / scale]]], np.float32)
        v = np.array([[[2.0]], [[-6.0]]], np.float32)
        st = o.attend(q, k, v, np.array([0, 2], np.int32), 1, 1, score_scale=scale)
        d = float(k[1, 0, 0]) * scale
        w1 = math.exp(d) / (1.0 + math.exp(d))
        _close(st.out[0, 0], 2.0 * (1 - w1) - 6.0 * w1, rtol=1e-14, what="two keys")
        _close(st.m[0], max(0.0, d), what="two keys m")


def pin_group_symmetry(o):
    H, G, D = 8, 2, 6
    q, k, v, off = _tiny(600, [13, 5], H, G, D)
    q[:, 1] = q[:, 0]
    q[:, 2] = q[:, 0]
    q[:, 3] = q[:, 0]                 # heads 0..3 form group 0
    st = o.attend(q, k, v, off, H, G)
    for b in range(2):
        for h in (1, 2, 3):
            assert np.array_equal(st.out[b * H + h], st.out[b * H]), "group symmetry"
    # swapping the two KV heads swaps which Q heads see which keys
    q2 = q.copy()
    q2[:, :4], q2[:, 4:] = q[:, 4:], q[:, :4]
    st2 = o.attend(q2, k[:, ::-1].copy(), v[:, ::-1].copy(), off, H, G)
    for b in range(2):
        for h in range(H):
            _close(st2.out[b * H + (h + 4) % 8], st.out[b * H + h], rtol=1e-13, atol=1e-14,
                   what="KV head permutation")


def pin_merge_union(o):
    H, G, D = 4, 2, 5
    q, k, v, off = _tiny(700, [20, 9], H, G, D)
    full = o.attend(q, k, v, off, H, G, score_scale=0.9)
    # split every sequence at a cut; attend over each part separately
    cut = [7, 4]
    offA = np.array([0, cut[0], cut[0] + cut[1]], np.int32)
    kA = np.concatenate([k[0:7], k[20:24]])
    vA = np.concatenate([v[0:7], v[20:24]])
    kB = np.concatenate([k[7:20], k[24:29]])
    vB = np.concatenate([v[7:20], v[24:29]])
    offB = np.array([0, 13, 18], np.int32)
    sa = o.attend(q, kA, vA, offA, H, G, score_scale=0.9)
    sb = o.attend(q, kB, vB, offB, H, G, score_scale=0.9)
    n = 2 * H
    m = np.stack([sa.m, sb.m], 1).astype(np.float32)
    l = np.stack([sa.l, sb.l], 1).astype(np.float32)
    acc = np.stack([sa.acc, sb.acc], 1).astype(np.float32)
    merged = o.merge(m, l, acc)
    _close(merged.out, full.out, rtol=1e-6, atol=1e-7, what="merge = union")   # fp32 storage
    _close(merged.l * np.exp(merged.m - full.m), full.l, rtol=1e-6, what="merged partition")
    # an empty third state changes nothing
    m3 = np.concatenate([m, np.full((n, 1), 5.0, np.float32)], 1)
    l3 = np.concatenate([l, np.zeros((n, 1), np.float32)], 1)
    acc3 = np.concatenate([acc, np.full((n, 1, D), 7.0, np.float32)], 1)
    merged3 = o.merge(m3, l3, acc3)
    assert np.array_equal(merged3.out, merged.out), "empty state in merge"
    assert np.array_equal(merged3.m, merged.m) and np.array_equal(merged3.l, merged.l), "empty state's m in merge"
    # the same union through the carry of attend
    sc = o.attend(q, kB, vB, offB, H, G, score_scale=0.9,
                  carry=(sa.m.astype(np.float32), sa.l.astype(np.float32), sa.acc.astype(np.float32)))
    _close(sc.out, full.out, rtol=1e-6, atol=1e-7, what="carry = union")
    # merge is symmetric in its states
    mr = o.merge(m[:, ::-1].copy(), l[:, ::-1].copy(), acc[:, ::-1].copy())
    _close(mr.out, merged.out, rtol=1e-14, atol=1e-15, what="merge order")


def pin_carry_identity(o):
    H, G, D = 6, 3, 4
    q, k, v, off = _tiny(800, [11, 3], H, G, D)
    n = 2 * H
    r = _rng(801)
    base = o.attend(q, k, v, off, H, G)
    cm = r.normal(0, 3, n).astype(np.float32)
    cl = np.zeros(n, np.float32)
    cacc = r.normal(0, 1, (n, D)).astype(np.float32)
    st = o.attend(q, k, v, off, H, G, carry=(cm, cl, cacc))
    assert np.array_equal(st.out, base.out) and np.array_equal(st.l, base.l), "empty carry"
    assert np.array_equal(st.m, base.m), "empty carry's m"
    # the carry of an empty sequence passes through as acc/l
    cl = r.uniform(1, 2, n).astype(np.float32)
    st = o.attend(q[:1], k[:0], v[:0], np.array([0, 0], np.int32), H, G,
                  carry=(cm[:H], cl[:H], cacc[:H]))
    _close(st.out, cacc[:H].astype(np.float64) / cl[:H, None], rtol=1e-14, what="carry only")
    # no keys and no carry: weight 0, output 0, not NaN
    st = o.attend(q[:1], k[:0], v[:0], np.array([0, 0], np.int32), H, G)
    assert np.all(st.out == 0.0) and np.all(st.l == 0.0) and np.all(np.isneginf(st.m))


def pin_shift_invariance(o):
    # an extra channel with q = c and k = 1/scale on every key adds c to every logit
    H, G, D = 4, 2, 6
    q, k, v, off = _tiny(900, [17, 6], H, G, D)
    base = o.attend(q, k, v, off, H, G, score_scale=0.5)
    for c in (50.0, 1000.0, -1000.0):
        q2 = np.concatenate([q, np.full((2, H, 1), c, np.float32)], axis=2)
        k2 = np.concatenate([k, np.full((23, G, 1), 2.0, np.float32)], axis=2)
        v2 = np.concatenate([v, np.zeros((23, G, 1), np.float32)], axis=2)
        st = o.attend(q2, k2, v2, off, H, G, score_scale=0.5)
        assert np.all(np.isfinite(st.out)), "overflow under a logit shift"
        _close(st.out[:, :D], base.out, rtol=1e-9, atol=1e-12, what=f"shift {c}")


def pin_needle(o):
    # planted-key trial: V[:,0] = 0 except at the needle, so out[h,0] is its weight
    H, G, D, N = 6, 2, 16, 200
    r = _rng(1000)
    u = r.uniform(-1, 1, (1, H, D))
    u /= np.linalg.norm(u, axis=-1, keepdims=True)
    q = (u * math.sqrt(D)).astype(np.float32)
    k = (r.uniform(-1, 1, (N, G, D)) * 1.732).astype(np.float32)
    v = r.uniform(-1, 1, (N, G, D)).astype(np.float32)
    v[:, :, 0] = 0.0
    p = N - 40
    for g in range(G):
        k[p, g] += (8.0 * u[0, g * 3]).astype(np.float32)
        v[p, g, 0] = 1.0
    st = o.attend(q, k, v, np.array([0, N], np.int32), H, G)
    bf = brute_force(q, k, v, np.array([0, N], np.int32), H, G, 1.0 / math.sqrt(D))
    for g in range(G):
        h = g * 3
        logits = k[:, g].astype(np.float64) @ q[0, h].astype(np.float64) / math.sqrt(D)
        w = math.exp(logits[p]) / np.exp(logits).sum()
        _close(st.out[h, 0], w, rtol=1e-12, what="needle weight")
        assert st.out[h, 0] > 0.5, "planted key does not dominate"
    _close(st.out, bf, what="needle brute force")


def pin_rows_subset(o):
    H, G, D = 4, 1, 3
    q, k, v, off = _tiny(1100, [5, 9, 2], H, G, D)
    full = o.attend(q, k, v, off, H, G)
    rows = [11, 0, 5, 5, 7]
    sub = o.attend(q, k, v, off, H, G, rows=rows)
    assert np.array_equal(sub.out, full.out[rows]) and np.array_equal(sub.m, full.m[rows])


def pin_bias_brute_force(o):
    # additive bias row after the scale (attn.rs attn_bias), incl. masked keys
    for i, (lengths, H, G, D) in enumerate([([6, 9], 4, 2, 3), ([5, 0, 7], 6, 3, 4)]):
        q, k, v, off = _tiny(1200 + i, lengths, H, G, D)
        r = _rng(1300 + i)
        bias = r.normal(0, 1, off[-1]).astype(np.float32)
        bias[::4] = -np.inf
        st = o.attend(q, k, v, off, H, G, score_scale=0.6, bias=bias)
        _close(st.out, brute_force(q, k, v, off, H, G, 0.6, bias=bias), what=f"bias brute force {i}")


def pin_bias_constant_is_shift(o):
    q, k, v, off = _tiny(1400, [13, 4], 8, 2, 5)
    base = o.attend(q, k, v, off, 8, 2, score_scale=0.4)
    st = o.attend(q, k, v, off, 8, 2, score_scale=0.4, bias=np.full(off[-1], 7.5, np.float32))
    _close(st.out, base.out, rtol=1e-13, atol=1e-14, what="constant bias")
    _close(st.m, base.m + 7.5, rtol=1e-14, what="constant bias shifts m")


def pin_bias_mask_is_subset(o):
    # masking rows with -inf equals attending over the cache without them
    H, G, D = 4, 2, 4
    q, k, v, off = _tiny(1500, [10, 6], H, G, D)
    keep = np.ones(off[-1], bool)
    keep[[1, 2, 7, 11, 15]] = False
    bias = np.where(keep, 0.0, -np.inf).astype(np.float32)
    st = o.attend(q, k, v, off, H, G, bias=bias)
    sub_off = np.array([0, keep[:10].sum(), keep.sum()], np.int32)
    ref = o.attend(q, k[keep], v[keep], sub_off, H, G)
    assert np.array_equal(st.out, ref.out) and np.array_equal(st.l, ref.l), "mask = subset"
    # every key of a sequence masked: weight 0, output 0 (or the carry alone)
    bias[:10] = -np.inf
    st = o.attend(q, k, v, off, H, G, bias=bias)
    assert np.all(st.out[:H] == 0.0) and np.all(np.isneginf(st.m[:H]))


def pin_topk_to_bias(o):
    # index rows: repeated indices collapse, -1 (INVALID) and out-of-range entries drop
    off = np.array([0, 5, 5, 12], np.int32)
    idx = np.array([[4, 0, 4, -1, 5, 2],
                    [0, 1, -1, -1, -1, -1],
                    [6, 6, 7, -3, 3, 0]], np.int32)
    bias = o.topk_to_bias(idx, off, 14, fill=1.25)
    for b in range(3):
        n = off[b + 1] - off[b]
        selected = {int(t) for t in idx[b] if 0 <= t < n}
        for t in range(n):
            want = 0.0 if t in selected else -np.inf
            assert bias[off[b] + t] == want, f"topk bias seq {b} key {t}"
    assert np.all(bias[12:] == 1.25), "rows outside every sequence are left alone"


def pin_append_then_attend(o):
    H, G, D = 4, 2, 3
    q, k, v, off = _tiny(1600, [5, 1, 3], H, G, D)
    r = _rng(1601)
    kn = r.uniform(-1, 1, (3, G, D)).astype(np.float32)
    vn = r.uniform(-1, 1, (3, G, D)).astype(np.float32)
    st, k2, v2 = o.pkg.append_then_attend(q, k, v, off, kn, vn, H, G, lib=o.lib)
    for b in range(3):
        assert np.array_equal(k2[off[b + 1] - 1], kn[b]) and np.array_equal(v2[off[b + 1] - 1], vn[b])
    untouched = np.ones(off[-1], bool)
    untouched[off[1:] - 1] = False
    assert np.array_equal(k2[untouched], k[untouched]), "append touched other rows"
    _close(st.out, brute_force(q, k2, v2, off, H, G, 1 / math.sqrt(D)), what="append then attend")


def _pack(idx, coeff):
    """Code word: atom index high 16 bits, coefficient's binary16 bits low 16."""
    bits = np.asarray(coeff, np.float16).view(np.uint16).astype(np.uint32)
    return (np.asarray(idx, np.uint32) << 16) | bits


def pin_f16_coefficients(o):
    cases = {0x3C00: 1.0, 0xC000: -2.0, 0x7BFF: 65504.0, 0x0001: 2.0 ** -24, 0x0400: 2.0 ** -14,
             0x3555: 0.333251953125, 0x0000: 0.0, 0x8000: -0.0}
    for bits, want in cases.items():
        assert o.pkg.f16_to_f64(bits, lib=o.lib) == want, f"f16 0x{bits:04x}"
    assert math.isinf(o.pkg.f16_to_f64(0x7C00, lib=o.lib))


def pin_reconstruct_words(o):
    r = _rng(1700)
    atoms = r.normal(0, 1, (40, 6)).astype(np.float32)
    idx = r.integers(0, 40, (5, 3, 4))
    coeff = r.normal(0, 1, (5, 3, 4)).astype(np.float16)
    coeff[0, 0, 3] = 0.0                                        # a padding word
    idx[0, 0, 3] = 39
    got = o.reconstruct(_pack(idx, coeff), atoms)
    want = np.einsum("rgw,rgwd->rgd", coeff.astype(np.float64), atoms[idx].astype(np.float64))
    _close(got, want, rtol=1e-14, atol=1e-14, what="reconstruct")
    # one-hot codes with coefficient 1 give the atom back exactly
    one = o.reconstruct(_pack(np.array([[7], [3]]), np.array([[1.0], [1.0]])), atoms)
    assert np.array_equal(one, atoms[[7, 3]].astype(np.float64))


def pin_coded_attention_is_plain_attention(o):
    # atoms = the cache's own rows and one-hot codes: the coded path must equal
    # plain attention over that cache
    H, G, D = 4, 2, 5
    q, k, v, off = _tiny(1800, [6, 9], H, G, D)
    R = off[-1]
    k_atoms = k.reshape(R * G, D)
    v_atoms = v.reshape(R * G, D)
    codes = _pack(np.arange(R * G).reshape(R, G, 1), np.ones((R, G, 1)))
    st = o.pkg.coded_decode_attend(q, codes, codes, k_atoms, v_atoms, off, H, G, 0.8, lib=o.lib)
    ref = o.attend(q, k, v, off, H, G, score_scale=0.8)
    assert np.array_equal(st.out, ref.out), "coded one-hot = plain"


ALL_PINS = [pin_bf16_widening, pin_brute_force_tiny, pin_single_key, pin_constant_v,
            pin_zero_query_mean, pin_two_key_closed_form, pin_group_symmetry, pin_merge_union,
            pin_carry_identity, pin_shift_invariance, pin_needle, pin_rows_subset,
            pin_bias_brute_force, pin_bias_constant_is_shift, pin_bias_mask_is_subset,
            pin_topk_to_bias, pin_append_then_attend, pin_f16_coefficients, pin_reconstruct_words,
            pin_coded_attention_is_plain_attention]


def run_all(o):
    """Run every pin; return the names of those that failed (with their messages)."""
    failed = []
    for pin in ALL_PINS:
        try:
            pin(o)
        except (AssertionError, ValueError, FloatingPointError) as e:
            failed.append(f"{pin.__name__}: {e}")
    return failed
