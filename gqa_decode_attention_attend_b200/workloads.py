"""Seeded synthetic inputs for grouped-query decode attention.

This module only draws random numbers and lays them out; it holds none of the
attention arithmetic. Both the CUDA path's tests/benchmark and the f64 oracle
consume what it returns, so it is the one piece they share.

Layouts (needle_core ``attn.rs`` ``KvCache``; USearch linear algebra):
  q        [B, H, D]              query row b*H + h is head h of sequence b
  k, v     [R, G, D]              packed cache; sequence b owns rows
                                  offsets[b] .. offsets[b+1]  (Arrow offsets)
  offsets  int32 [B+1]
  carry    (m [B*H], l [B*H], acc [B*H, D]) fp32, optional

Every draw is fp32 from a CPU ``torch.Generator`` with the stated seed, in the
order lengths, q, k, v, carry; bf16 tensors are the fp32 draws rounded to
nearest-even. The named workloads follow the five decode configurations this
library is measured on; the needle workload follows the planted-key trial of
the cortiq_engine ``NystromState`` example (``examples/o1_recovery.rs``).
"""
from dataclasses import dataclass, field
import math
from typing import Optional, Sequence

import torch


@dataclass
class Workload:
    name: str
    q: torch.Tensor
    k: torch.Tensor
    v: torch.Tensor
    offsets: torch.Tensor
    num_heads: int
    num_kv_heads: int
    head_dim: int
    score_scale: float = 0.0
    carry: Optional[tuple] = None
    max_seq_len: int = 0
    needle_rows: Optional[list] = None      # (row index into k/v, kv head) of planted keys
    meta: dict = field(default_factory=dict)

    @property
    def batch(self):
        return self.offsets.numel() - 1

    @property
    def lengths(self):
        return (self.offsets[1:] - self.offsets[:-1]).tolist()

    @property
    def total_rows(self):
        return int(self.offsets[-1])

    def kv_bytes(self):
        """Algorithmic KV-cache bytes one decode call reads: sum_b N_b * G * D * 2 * elem."""
        return self.total_rows * self.num_kv_heads * self.head_dim * 2 * self.k.element_size()


def _uniform(gen, shape, lo=-1.0, hi=1.0):
    return torch.rand(shape, generator=gen, dtype=torch.float32) * (hi - lo) + lo


def _normal(gen, shape):
    return torch.randn(shape, generator=gen, dtype=torch.float32)


def _unit_rows(x):
    return x / x.norm(dim=-1, keepdim=True)


def make(name, lengths: Sequence[int], num_heads, num_kv_heads, head_dim, dtype=torch.bfloat16,
         dist="normal", seed=0, score_scale=0.0, carry=False, needle=None, q_dtype=None,
         gen=None):
    """Build one workload.

    dist: "normal" (iid N(0,1)), "uniform" (iid U(-1,1)) or "needle".
    needle: dict(amp=8.0, depth=4096) for dist="needle": per sequence the key at
      position N_b - depth of every KV head g is moved by amp * unit(u) along the
      direction u of that group's first Q head, and its value's channel 0 is set
      to 1 while channel 0 of every other value is 0.
    """
    gen = gen or torch.Generator().manual_seed(seed)
    lengths = [int(n) for n in lengths]
    B, H, G, D = len(lengths), int(num_heads), int(num_kv_heads), int(head_dim)
    offsets = torch.zeros(B + 1, dtype=torch.int32)
    if B:
        offsets[1:] = torch.cumsum(torch.tensor(lengths, dtype=torch.int64), 0).to(torch.int32)
    R = int(offsets[-1])
    needle_rows = None
    if dist == "normal":
        q = _normal(gen, (B, H, D))
        k = _normal(gen, (R, G, D))
        v = _normal(gen, (R, G, D))
    elif dist == "uniform":
        q = _uniform(gen, (B, H, D))
        k = _uniform(gen, (R, G, D))
        v = _uniform(gen, (R, G, D))
    elif dist == "needle":
        needle = dict(needle or {})
        amp = float(needle.get("amp", 8.0))
        depth = int(needle.get("depth", 4096))
        u = _unit_rows(_uniform(gen, (B, H, D)))
        q = u * math.sqrt(D)
        k = _uniform(gen, (R, G, D)) * 1.732
        v = _uniform(gen, (R, G, D))
        v[:, :, 0] = 0.0
        hpk = H // G
        needle_rows = []
        for b in range(B):
            n = lengths[b]
            if n == 0:
                continue
            p = int(offsets[b]) + max(0, n - depth)
            for g in range(G):
                k[p, g, :] += amp * u[b, g * hpk, :]
                v[p, g, 0] = 1.0
                needle_rows.append((p, g))
    else:
        raise ValueError(f"unknown dist {dist!r}")
    qd = q_dtype or dtype
    c = None
    if carry:
        cm = _normal(gen, (B * H,))
        cl = _uniform(gen, (B * H,), 1.0, 100.0)
        cacc = _normal(gen, (B * H, D))
        c = (cm, cl, cacc)
    return Workload(name=name, q=q.to(qd).contiguous(), k=k.to(dtype).contiguous(),
                    v=v.to(dtype).contiguous(), offsets=offsets, num_heads=H, num_kv_heads=G,
                    head_dim=D, score_scale=score_scale, carry=c,
                    max_seq_len=max(lengths) if lengths else 0, needle_rows=needle_rows,
                    meta=dict(dist=dist, seed=seed))


# ---------------------------------------------------------------- named configurations

CONFIG_NAMES = ("fp32_b1_n512", "bf16_b16_n4096", "bf16_b4_n32768", "bf16_b64_ragged16384",
                "bf16_b1_n131072")

CONFIG_TEXT = {
    "fp32_b1_n512":
        "fp32 GQA decode, batch 1, 8 Q / 4 KV heads, head_dim 64, cache len 512; "
        "q,K,V iid U(-1,1); scale 1/sqrt(64); no carry",
    "bf16_b16_n4096":
        "bf16 K/V, fp32 accumulation, bf16 q/out; batch 16, 32 Q / 8 KV heads, "
        "head_dim 128, every sequence 4096 keys; q,K,V iid N(0,1)",
    "bf16_b4_n32768":
        "bf16 split-KV stress; batch 4, 64 Q / 8 KV heads, head_dim 128, 32768 keys "
        "each; q,K,V iid N(0,1); partial states merged by gqa_softmax_merge",
    "bf16_b64_ragged16384":
        "ragged bf16 batch of 64 sequences, lengths uniform in [1,16384], 32 Q / 8 KV "
        "heads, head_dim 128; carry m~N(0,1), l~U(1,100), acc~N(0,1) folded in",
    "bf16_b1_n131072":
        "bf16 long context; batch 1, 48 Q / 8 KV heads, head_dim 128, 131072 keys; "
        "K 1.732*U(-1,1), V U(-1,1); planted key at depth 4096, amp 8",
}


def ragged_lengths(batch, lo, hi, seed):
    gen = torch.Generator().manual_seed(seed)
    return torch.randint(lo, hi + 1, (batch,), generator=gen, dtype=torch.int64).tolist()


def config(name):
    """The full-size named workloads (seeds 1..5)."""
    if name == "fp32_b1_n512":
        w = make(name, [512], 8, 4, 64, dtype=torch.float32, dist="uniform", seed=1,
                 score_scale=1.0 / 8.0)
    elif name == "bf16_b16_n4096":
        w = make(name, [4096] * 16, 32, 8, 128, dist="normal", seed=2)
    elif name == "bf16_b4_n32768":
        w = make(name, [32768] * 4, 64, 8, 128, dist="normal", seed=3)
    elif name == "bf16_b64_ragged16384":
        gen = torch.Generator().manual_seed(4)
        lengths = torch.randint(1, 16385, (64,), generator=gen, dtype=torch.int64).tolist()
        w = make(name, lengths, 32, 8, 128, dist="normal", carry=True, gen=gen, seed=4)
    elif name == "bf16_b1_n131072":
        w = make(name, [131072], 48, 8, 128, dist="needle", seed=5,
                 needle=dict(amp=8.0, depth=4096))
    else:
        raise ValueError(f"unknown config {name!r}; expected one of {CONFIG_NAMES}")
    w.meta["text"] = CONFIG_TEXT[name]
    return w


def bf16_bits(t: torch.Tensor):
    """Raw bit patterns of a bf16 tensor as a numpy uint16 array (for the oracle)."""
    return t.contiguous().view(torch.int16).numpy().view("uint16")


def host_array(t: torch.Tensor):
    """numpy view of a CPU tensor as stored: fp32 stays fp32, bf16 becomes uint16 bits."""
    if t.dtype == torch.bfloat16:
        return bf16_bits(t)
    return t.contiguous().numpy()
