"""Write the stored expected values under tests/golden/ by calling only the oracle.

The pages this library follows print no worked numeric example, so every stored
value here is the f64 oracle's, on seeded inputs from the shared generator:

  fp32_b1_n512_rows.json  config "fp32, batch 1, 8 Q / 4 KV heads, head_dim 64,
                     512 keys, U(-1,1), scale 1/8": all 8 output rows and their
                     (m, l) -- needle_core attn.rs `self_attn_incremental`
                     (GQA decode), USearch linear algebra § Attention (m, l).
  needle_small.json  planted-key trial at 1024 keys, 6 Q / 2 KV heads, d 64,
                     depth 64, amp 8 (cortiq_engine NystromState example
                     `trial`): out[:, 0] of every head.

Usage: python tests/golden/make_golden.py
"""
import json
import os
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(os.path.dirname(HERE))
sys.path.insert(0, ROOT)

import oracle  # noqa: E402
from gqa_decode_attention_attend_b200 import workloads  # noqa: E402


def fp32_b1_n512_rows():
    w = workloads.config("fp32_b1_n512")
    st = oracle.decode_attend(workloads.host_array(w.q), workloads.host_array(w.k),
                              workloads.host_array(w.v), w.offsets.numpy(), w.num_heads,
                              w.num_kv_heads, w.score_scale)
    return dict(workload="fp32_b1_n512", text=w.meta["text"], m=st.m.tolist(), l=st.l.tolist(),
                out=st.out.tolist())


def needle_small():
    w = workloads.make("needle_small", [1024], 6, 2, 64, dist="needle", seed=11,
                       needle=dict(amp=8.0, depth=64))
    st = oracle.decode_attend(workloads.host_array(w.q), workloads.host_array(w.k),
                              workloads.host_array(w.v), w.offsets.numpy(), 6, 2)
    return dict(workload="needle_small", lengths=[1024], heads=6, kv_heads=2, head_dim=64,
                seed=11, amp=8.0, depth=64, out0=st.out[:, 0].tolist())


def main():
    for name, fn in (("fp32_b1_n512_rows.json", fp32_b1_n512_rows), ("needle_small.json", needle_small)):
        with open(os.path.join(HERE, name), "w") as f:
            json.dump(fn(), f, indent=1)
        print("wrote", name)


if __name__ == "__main__":
    main()
