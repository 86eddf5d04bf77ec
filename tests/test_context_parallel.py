"""Context-parallel split-KV: key slices per rank, state exchange, merge.

CPU (gloo, two ranks): every rank computes the f64-exact state of its slice
with the oracle, exchange_states all-gathers them, and the gathered states
merge (oracle) to attention over the whole sequences. GPU (one device): the
ranks' slices are run one after another through gqa_decode_attend and merged
with gqa_softmax_merge_gathered, against the oracle.
"""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import oracle
from gqa_decode_attention_attend_b200 import State, context_parallel as cp, workloads


def test_shard_bounds_cover_every_key_once():
    lengths = [0, 1, 5, 4096, 7]
    for world in (1, 2, 3, 8):
        seen = [np.zeros(n, int) for n in lengths]
        for r in range(world):
            for b, (lo, hi) in enumerate(cp.shard_bounds(lengths, world, r)):
                seen[b][lo:hi] += 1
            off = cp.local_offsets(lengths, world, r)
            assert off[0] == 0 and np.all(np.diff(off) >= 0)
        assert all(np.all(s == 1) for s in seen)


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _rank(rank, world, port, q):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=__import__("datetime").timedelta(seconds=60))
    try:
        w = workloads.make("cp", [300, 1, 0, 77], 8, 2, 64, dtype=torch.float32, dist="uniform",
                           seed=3, carry=True)
        k, v, off = cp.shard_cache(w.k, w.v, w.offsets.tolist(), world, rank)
        st = oracle.decode_attend(w.q.numpy(), k.numpy(), v.numpy(), off.numpy(), 8, 2)
        local = State(torch.from_numpy(st.m.astype(np.float32)), torch.from_numpy(st.l.astype(np.float32)),
                      torch.from_numpy(st.acc.astype(np.float32)))
        g = cp.exchange_states(local)
        merged = oracle.softmax_merge(g.m.numpy().T, g.l.numpy().T, g.acc.numpy().transpose(1, 0, 2),
                                      carry=tuple(t.numpy() for t in w.carry))
        full = oracle.decode_attend(w.q.numpy(), w.k.numpy(), w.v.numpy(), w.offsets.numpy(), 8, 2,
                                    carry=tuple(t.numpy() for t in w.carry))
        q.put((rank, float(np.max(np.abs(merged.out - full.out))), tuple(g.m.shape)))
    finally:
        dist.barrier()
        dist.destroy_process_group()


def test_exchange_and_merge_two_gloo_ranks():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, err, shape in res:
        assert shape == (2, 32)
        assert err < 1e-6, f"rank {rank}: merged slices differ from the whole by {err}"


@pytest.mark.gpu
@pytest.mark.parametrize("world", [2, 3, 4])
@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32], ids=["bf16", "f32"])
def test_ranks_emulated_on_one_gpu(world, dtype):
    import gpu_util as gu
    import gqa_decode_attention_attend_b200 as gqa
    dev = gu.device()
    w = workloads.make("cpg", [4096, 3, 1, 9000], 32, 8, 128, dtype=dtype, seed=4, carry=True)
    rows = w.batch * w.num_heads
    gathered = State(torch.empty((world, rows), device=dev), torch.empty((world, rows), device=dev),
                     torch.empty((world, rows, 128), device=dev))
    for r in range(world):
        k, v, off = cp.shard_cache(w.k, w.v, w.offsets.tolist(), world, r)
        st = State(gathered.m[r], gathered.l[r], gathered.acc[r])
        gqa.gqa_decode_attend(w.q.to(dev), k.to(dev), v.to(dev), off.to(dev), 32, 8, state_out=st,
                              want_out=False, max_seq_len=9000)
    carry = State(*(t.to(dev) for t in w.carry))
    out = gqa.gqa_softmax_merge_gathered(gathered, carry=carry, out_dtype=torch.float32)
    ref = gu.oracle_state(w)
    gu.check_out(out, ref, w, what=f"context parallel x{world}")


@pytest.mark.gpu
def test_cp_decode_attend_single_rank():
    import gpu_util as gu
    dev = gu.device()
    w = workloads.make("cp1", [2000, 64], 16, 4, 128, seed=5, carry=True)
    dw = gu.DevWorkload(w, dev)
    out = cp.cp_decode_attend(dw.q, dw.k, dw.v, dw.offsets, 16, 4, carry=dw.carry, max_seq_len=2000,
                              out_dtype=torch.float32)
    ref = gu.oracle_state(w)
    gu.check_out(out, ref, w, what="cp single rank")
