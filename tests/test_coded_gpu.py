"""GPU parity for the dictionary-coded cache read path (qualiaDB KvDictionary:
code words of atom index + f16 coefficient): gqa_decode_attend_coded against
the oracle, which rebuilds the rows in f64 and applies the plain attention."""
import numpy as np
import pytest
import torch

import gpu_util as gu
import oracle
import gqa_decode_attention_attend_b200 as gqa
from gqa_decode_attention_attend_b200 import workloads

pytestmark = pytest.mark.gpu


def make_codes(rows, G, words, n_atoms, D, seed, pad_frac=0.2):
    """Synthetic dictionary (unit-norm atoms) and codes (random atoms, N(0,1)
    coefficients rounded to binary16, some zero padding words)."""
    rng = np.random.default_rng(seed)
    ka = rng.normal(0, 1, (n_atoms, D))
    va = rng.normal(0, 1, (n_atoms, D))
    ka = (ka / np.linalg.norm(ka, axis=1, keepdims=True)).astype(np.float32)
    va = (va / np.linalg.norm(va, axis=1, keepdims=True)).astype(np.float32)

    def codes():
        idx = rng.integers(0, n_atoms, (rows, G, words)).astype(np.uint32)
        cf = rng.normal(0, 1, (rows, G, words)).astype(np.float16)
        cf[rng.random((rows, G, words)) < pad_frac] = 0
        return (idx << 16) | cf.view(np.uint16).astype(np.uint32)

    return codes(), codes(), ka, va


def run_coded(w, kc, vc, ka, va, dev, **kw):
    t = lambda a: torch.from_numpy(a.view(np.int32) if a.dtype == np.uint32 else a).to(dev)
    carry = gqa.State(*(c.to(dev) for c in w.carry)) if w.carry is not None else None
    return gqa.gqa_decode_attend_coded(w.q.to(dev), t(kc), t(vc), t(ka), t(va), w.offsets.to(dev),
                                       w.num_heads, w.num_kv_heads, carry=carry,
                                       max_seq_len=w.max_seq_len, **kw)


@pytest.mark.parametrize("D,H,G,words,n_atoms", [(128, 32, 8, 8, 256), (64, 16, 2, 4, 1024),
                                                 (128, 16, 1, 1, 64), (128, 48, 8, 16, 512),
                                                 (64, 16, 4, 4, 512)])
@pytest.mark.parametrize("qdt", [torch.bfloat16, torch.float32], ids=["bf16q", "f32q"])
def test_coded_attention(D, H, G, words, n_atoms, qdt):
    dev = gu.device()
    lengths = [1, 0, 300, 2049, 5000]
    w = workloads.make("coded", lengths, H, G, D, dtype=qdt, seed=D + words, carry=True)
    kc, vc, ka, va = make_codes(w.total_rows, G, words, n_atoms, D, seed=n_atoms)
    ref = oracle.coded_decode_attend(workloads.host_array(w.q), kc, vc, ka, va, w.offsets.numpy(), H, G,
                                     carry=tuple(t.numpy() for t in w.carry))
    for ns in (0, 3):
        out = run_coded(w, kc, vc, ka, va, dev, out_dtype=torch.float32, num_splits=ns)
        gu.assert_close(out.reshape(-1, D).cpu().numpy(), ref.out, torch.float32,
                        f"coded D{D} H{H} G{G} words{words} atoms{n_atoms} splits{ns}")


def test_one_hot_codes_equal_plain_attention():
    dev = gu.device()
    w = workloads.make("onehot", [700, 33], 16, 4, 128, dtype=torch.float32, seed=5)
    R, G, D = w.total_rows, 4, 128
    rows = np.arange(R * G, dtype=np.uint32).reshape(R, G, 1)
    ones = np.ones((R, G, 1), np.float16).view(np.uint16).astype(np.uint32)
    codes = (rows << 16) | ones
    atoms_k = w.k.numpy().reshape(R * G, D)
    atoms_v = w.v.numpy().reshape(R * G, D)
    # R*G = 2932 atoms x 4 heads per KV head fits the table limit
    out = run_coded(w, codes, codes, atoms_k, atoms_v, dev, out_dtype=torch.float32)
    plain = gqa.gqa_decode_attend(w.q.to(dev), w.k.to(dev), w.v.to(dev), w.offsets.to(dev), 16, 4)
    torch.testing.assert_close(out, plain, rtol=2e-5, atol=2e-6)


def test_bad_code_is_flagged():
    dev = gu.device()
    w = workloads.make("bad", [40], 8, 2, 64, dtype=torch.float32, seed=6)
    kc, vc, ka, va = make_codes(w.total_rows, 2, 4, 32, 64, seed=7, pad_frac=0.0)
    kc[5, 1, 2] = (np.uint32(32) << 16) | np.uint32(0x3C00)     # atom 32 of 32: out of range
    ws = gqa.Workspace(dev, 1 << 20)
    run_coded(w, kc, vc, ka, va, dev, workspace=ws)
    assert gqa.gqa_get_device_error(ws) == gqa.GQA_ERR_BAD_CODES


def test_coded_is_deterministic():
    """The value weights are summed in fixed point by integer atomics, whose
    sums do not depend on their order: repeated calls give identical bits."""
    dev = gu.device()
    w = workloads.make("cdet", [4096] * 4, 32, 8, 128, seed=8, carry=True)
    kc, vc, ka, va = make_codes(w.total_rows, 8, 8, 256, 128, seed=9)
    outs = [run_coded(w, kc, vc, ka, va, dev, out_dtype=torch.float32) for _ in range(4)]
    torch.cuda.synchronize()
    for o in outs[1:]:
        assert torch.equal(o, outs[0])


@pytest.mark.parametrize("words", [6, 3])
def test_coded_sharp_softmax_and_wide_coefficients(words):
    """Peaked logits (score scale 1 instead of 1/sqrt(128): few keys carry the
    weight) and coefficients spread over four and a half orders of magnitude,
    at the fp32 tolerance: the fixed-point scale of each round follows the
    weights actually present."""
    dev = gu.device()
    D, H, G, NA = 128, 16, 4, 96
    lengths = [1500, 257, 2100]
    w = workloads.make("csharp", lengths, H, G, D, dtype=torch.float32, seed=10 + words,
                       score_scale=1.0, carry=True)
    rng = np.random.default_rng(11 + words)
    ka = rng.normal(0, 1, (NA, D))
    va = rng.normal(0, 1, (NA, D))
    ka = (ka / np.linalg.norm(ka, axis=1, keepdims=True)).astype(np.float32)
    va = (va / np.linalg.norm(va, axis=1, keepdims=True)).astype(np.float32)

    def codes():
        idx = rng.integers(0, NA, (w.total_rows, G, words)).astype(np.uint32)
        mag = 10.0 ** rng.uniform(-4, 0.5, (w.total_rows, G, words))
        cf = (mag * rng.choice([-1.0, 1.0], mag.shape)).astype(np.float16)
        return (idx << 16) | cf.view(np.uint16).astype(np.uint32)

    kc, vc = codes(), codes()
    ref = oracle.coded_decode_attend(workloads.host_array(w.q), kc, vc, ka, va, w.offsets.numpy(), H, G,
                                     score_scale=1.0, carry=tuple(t.numpy() for t in w.carry))
    out = run_coded(w, kc, vc, ka, va, dev, out_dtype=torch.float32, score_scale=1.0)
    gu.assert_close(out.reshape(-1, D).cpu().numpy(), ref.out, torch.float32, f"sharp coded words{words}")


@pytest.mark.parametrize("D", [128, 64])
def test_coded_at_the_table_limit(D):
    """heads_per_kv * n_atoms = 12288 with 16 words per row: the largest
    shared-memory footprint the kernel accepts; one atom more is refused."""
    dev = gu.device()
    H, G, NA, words = 16, 1, 768, 16
    w = workloads.make("climit", [300, 17, 0], H, G, D, dtype=torch.float32, seed=12, carry=True)
    kc, vc, ka, va = make_codes(w.total_rows, G, words, NA, D, seed=13)
    ref = oracle.coded_decode_attend(workloads.host_array(w.q), kc, vc, ka, va, w.offsets.numpy(), H, G,
                                     carry=tuple(t.numpy() for t in w.carry))
    out = run_coded(w, kc, vc, ka, va, dev, out_dtype=torch.float32)
    gu.assert_close(out.reshape(-1, D).cpu().numpy(), ref.out, torch.float32, f"coded at the limit D{D}")
    ka2 = np.concatenate([ka, ka[:1]])
    with pytest.raises(gqa.GqaError):
        run_coded(w, kc, vc, ka2, ka2, dev, out_dtype=torch.float32)


def test_coded_many_heads_rounds_and_bias():
    """16 query heads per KV head (the values every thread shares then live in
    shared memory), three rounds of keys on the longest sequence (one split of
    2600 keys, rounds of 1024), and a bias row: finite values, and -inf over the
    first 1100 keys of sequence 0, so that its first round is masked out
    entirely and its second in part."""
    dev = gu.device()
    D, H, G, words, NA = 128, 32, 2, 8, 256
    lengths = [2600, 1, 1100]
    w = workloads.make("cbias", lengths, H, G, D, dtype=torch.float32, seed=14, carry=True)
    kc, vc, ka, va = make_codes(w.total_rows, G, words, NA, D, seed=15)
    rng = np.random.default_rng(16)
    bias = rng.normal(0, 1, w.total_rows).astype(np.float32)
    off = w.offsets.numpy()
    bias[off[0]:off[0] + 1100] = -np.inf
    ref = oracle.coded_decode_attend(workloads.host_array(w.q), kc, vc, ka, va, off, H, G,
                                     carry=tuple(t.numpy() for t in w.carry), bias=bias)
    for ns in (0, 1):
        out = run_coded(w, kc, vc, ka, va, dev, out_dtype=torch.float32, num_splits=ns,
                        bias=torch.from_numpy(bias).to(dev))
        gu.assert_close(out.reshape(-1, D).cpu().numpy(), ref.out, torch.float32,
                        f"coded 16 heads per KV head, rounds, bias, splits{ns}")


def test_coded_long_single_split_over_rounds():
    """8 words, 256 atoms, 4 heads per KV head (rounds of 6656 keys): one split
    of 14000 keys takes three rounds, the last one ragged, beside a short
    sequence; the planned splits as well."""
    dev = gu.device()
    D, H, G, words, NA = 128, 32, 8, 8, 256
    w = workloads.make("clong", [14000, 130], H, G, D, dtype=torch.bfloat16, seed=17, carry=True)
    kc, vc, ka, va = make_codes(w.total_rows, G, words, NA, D, seed=18)
    ref = oracle.coded_decode_attend(workloads.host_array(w.q), kc, vc, ka, va, w.offsets.numpy(), H, G,
                                     carry=tuple(t.numpy() for t in w.carry))
    for ns in (1, 0):
        out = run_coded(w, kc, vc, ka, va, dev, out_dtype=torch.float32, num_splits=ns)
        gu.assert_close(out.reshape(-1, D).cpu().numpy(), ref.out, torch.float32,
                        f"coded long single split, splits{ns}")
