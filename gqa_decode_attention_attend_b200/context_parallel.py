"""Context-parallel decode attention across ranks (split-KV over GPUs).

Every rank holds a contiguous slice of every sequence's keys and computes the
online-softmax state (m, l, acc) of its slice with gqa_decode_attend, the
carry left out. The states -- B*H*(D+2) floats per rank -- are exchanged with
one all-gather over the process group (NCCL over NVLink / NVSwitch on B200),
and every rank folds them, with the carry, by gqa_softmax_merge_gathered. The
merge is exact up to rounding (USearch linear algebra, DenseAttendConfig::carry:
partial-softmax rescaling folds one call into another over the same queries),
so every rank ends with attention over the whole sequences.

The all-gather is the only data-path collective; it moves a few tens of KB per
call, so it is latency-bound, and NCCL's all-gather is used as is.
"""
import numpy as np

from . import State, gqa_decode_attend, gqa_softmax_merge_gathered


def shard_bounds(lengths, world, rank):
    """Keys [lo, hi) of every sequence that `rank` of `world` holds: the
    sequence of n keys is cut into `world` contiguous, near-equal slices."""
    return [(n * rank // world, n * (rank + 1) // world) for n in lengths]


def local_offsets(lengths, world, rank):
    """Arrow offsets of the rank's local packed cache (its slices, in order)."""
    bounds = shard_bounds(lengths, world, rank)
    off = np.zeros(len(lengths) + 1, np.int32)
    off[1:] = np.cumsum([hi - lo for lo, hi in bounds])
    return off


def shard_cache(k, v, offsets, world, rank):
    """The rank's slice of a packed cache: (k_local, v_local, local_offsets).
    k, v: [rows, G, D] tensors; offsets: host int sequence [B+1]."""
    import torch
    offsets = [int(x) for x in offsets]
    lengths = [offsets[b + 1] - offsets[b] for b in range(len(offsets) - 1)]
    rows = []
    for b, (lo, hi) in enumerate(shard_bounds(lengths, world, rank)):
        rows.extend(range(offsets[b] + lo, offsets[b] + hi))
    index = torch.tensor(rows, dtype=torch.long, device=k.device)
    return (k.index_select(0, index).contiguous(), v.index_select(0, index).contiguous(),
            torch.from_numpy(local_offsets(lengths, world, rank)))


def exchange_states(state, group=None):
    """All-gather every rank's state: returns m, l [world, rows], acc
    [world, rows, D], block r holding rank r's state."""
    import torch
    import torch.distributed as dist
    if group is None and not dist.is_initialized():
        return State(state.m[None], state.l[None], state.acc[None])
    world = dist.get_world_size(group)
    rows = state.m.shape[0]

    def gather(t):
        # concatenated along dim 0 (the form every backend accepts), then viewed per rank
        buf = torch.empty((world * rows, *t.shape[1:]), dtype=t.dtype, device=t.device)
        dist.all_gather_into_tensor(buf, t.contiguous(), group=group)
        return buf.view(world, rows, *t.shape[1:])

    return State(gather(state.m), gather(state.l), gather(state.acc))


def cp_decode_attend(q, k_local, v_local, local_offsets, num_heads, num_kv_heads=0, *, group=None,
                     carry=None, out=None, out_dtype=None, score_scale=0.0, max_seq_len=0,
                     workspace=None, stream=None):
    """Decode attention over sequences whose keys are split across the ranks of
    `group`: local partial state, all-gather of the states, merge with the
    carry. Every rank passes the same q and carry and receives the same out."""
    B, H, D = q.shape
    local = State.empty(B * H, D, q.device)
    gqa_decode_attend(q, k_local, v_local, local_offsets, num_heads, num_kv_heads,
                      score_scale=score_scale, state_out=local, want_out=False,
                      max_seq_len=max_seq_len, workspace=workspace, stream=stream)
    gathered = exchange_states(local, group)
    flat = gqa_softmax_merge_gathered(gathered, carry=carry, out=None if out is None else out.view(B * H, D),
                                      out_dtype=out_dtype or q.dtype, stream=stream)
    return flat.view(B, H, D)
