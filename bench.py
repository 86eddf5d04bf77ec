#!/usr/bin/env python
"""Benchmark of the decode-attention hot path on B200.

One step = one gqa_decode_attend call over the whole batch (one launch of the
split-KV partition kernel, whose last CTA per sequence and KV head merges the
splits and the carry and writes the output). The default workload is the
largest one: a ragged bf16 batch of 64 sequences with lengths uniform in
[1, 16384] (Arrow offsets), 32 Q / 8 KV heads, head_dim 128, q/K/V iid N(0,1),
a per-query-row carry (m ~ N(0,1), l ~ U(1,100), acc ~ N(0,1)) folded in,
bf16 output: ~2.15 GB of KV cache per step, resident in HBM before the timed
region and far larger than the 126 MB L2. Smaller caches are duplicated and
the copies alternated so no step reads a cache L2 could still hold.

The K timed steps are captured once into a CUDA graph and replayed (the call
allocates nothing and never synchronises), each launched with
GQA_FLAG_EARLY_START (no step writes the cache rows or offsets the next one
reads); --eager and --no-early-start turn either off.

Prints ONE JSON line (rank 0). `value` is the KV-cache bytes read per step,
summed over ranks, divided by the max-over-ranks device time (GB/s); `e2e` is
the same metric through the same public call when every step also copies its
inputs from pinned host memory and its output back. `targets` times, in the
same run, the three long-context bf16 workloads that must each hold >= 70 % of
the nominal 8 TB/s in KV bytes read: the 4 x 32768 split stress batch through
the three-call path it names (partial states, gqa_softmax_merge with the
carry, gqa_state_finalize), the ragged batch, and the 131072-key sequence;
each with its step time back to back and as one isolated call after an L2
flush, and its clock record.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                  [--workload NAME] [--op OP] [--splits S] [--eager] [--no-early-start]
                  [--no-cpu-baseline] [--no-targets] [--quick]

--impl reference times the f64 CPU oracle (the library's reference
implementation) on a bounded sample of the same workload, on rank 0 only.
"""
import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "GQA decode attention: KV-cache HBM GB/s (% of B200 peak) and queries·heads/s"
NOMINAL_HBM_GBS = 8000.0
FALLBACK_HBM_GBS = 6650.0


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default="bf16_b64_ragged16384")
    ap.add_argument("--op", choices=sorted(LAUNCHES), default="attend",
                    help="attend: plain decode attention (the default line); append_attend: "
                         "append the new token's K/V then attend; masked_attend: index rows -> "
                         "bias (gqa_topk_to_bias) then attend with it; coded_attend: the "
                         "same shape as a dictionary-coded cache (8 code words per row, 256 "
                         "atoms), KV bytes = code bytes read; split_pipeline: the three-call "
                         "path (partial states, gqa_softmax_merge with the carry, "
                         "gqa_state_finalize)")
    ap.add_argument("--splits", type=int, default=0,
                    help="force this many splits per sequence (0: the library's heuristic)")
    ap.add_argument("--no-targets", action="store_true",
                    help="skip timing the long-context workloads beside the line")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=5.0)
    ap.add_argument("--e2e-steps", type=int, default=30)
    ap.add_argument("--no-early-start", action="store_true",
                    help="launch every call in plain stream order instead of with "
                         "GQA_FLAG_EARLY_START (steps here never write the cache rows or "
                         "offsets the next step reads, which is that flag's contract)")
    ap.add_argument("--eager", action="store_true",
                    help="launch every step from Python instead of replaying a CUDA graph "
                         "of the K steps")
    ap.add_argument("--quick", action="store_true",
                    help="timed loop and kernel timing only (no clock sampling, e2e or CPU "
                         "baseline); for profiler launch lists")
    return ap.parse_args()


def dist_env():
    return (int(os.environ.get("RANK", "0")), int(os.environ.get("WORLD_SIZE", "1")),
            int(os.environ.get("LOCAL_RANK", "0")))


def measured_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(p) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    except (OSError, KeyError, ValueError):
        return FALLBACK_HBM_GBS, "fallback"


# The sources that define the profiled launch of the bf16 partition kernel:
# its body, the tile logic and fused merge it includes, the PTX wrappers, and
# the host code that plans and launches it.
PROFILED_SOURCES = ("gqa_decode.cu", "partition_bf16.cuh", "ptx.cuh", "tile.cuh")


def kernel_source_hash():
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "gqa_decode_attention_attend_b200", "csrc")
    for name in PROFILED_SOURCES:
        with open(os.path.join(csrc, name), "rb") as f:
            h.update(name.encode() + f.read())
    return h.hexdigest()[:16]


def recorded_traffic(workload):
    """dram read+write bytes per launch of the partition kernel from the committed
    ncu summary, or None if there is none or the kernel sources changed since."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    try:
        with open(p) as f:
            d = json.load(f)
    except (OSError, ValueError):
        return None
    e = d.get(workload)
    if not e or e.get("kernel_source_hash") != kernel_source_hash():
        return None
    return int(e["dram_bytes_per_launch"])


class ClockSampler:
    """nvidia-smi clock / throttle sampling in the background."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index):
        self.gpu = gpu_index
        self.proc = None
        self.lines = []

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-i", str(self.gpu), "-lms", "100"], stdout=subprocess.PIPE,
                stderr=subprocess.DEVNULL, text=True)
            self.t = threading.Thread(target=self._read, daemon=True)
            self.t.start()
        except OSError:
            self.proc = None

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self.t.join(timeout=5)
        return self.summarize(self.lines)

    @staticmethod
    def summarize(lines):
        """Median SM clock, max clock and the throttle reasons seen in
        `nvidia-smi --format=csv,noheader,nounits` lines of FIELDS."""
        sm, mx, reasons = [], [], set()
        names = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")
        for ln in lines:
            parts = [x.strip() for x in ln.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                mx.append(float(parts[2]))
            except ValueError:
                continue
            for n, v in zip(names, parts[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(mx), "reasons": sorted(reasons),
                "samples": len(sm)}


# ------------------------------------------------------------------ CPU oracle (baseline)

def oracle_sample(w, seconds):
    """Time the f64 oracle on whole copies of the workload until `seconds` pass.
    Returns (GB/s, queries*heads/s, threads, sample description)."""
    import oracle
    from gqa_decode_attention_attend_b200 import workloads
    q, k, v = (workloads.host_array(t) for t in (w.q, w.k, w.v))
    off = w.offsets.numpy()
    carry = tuple(t.numpy() for t in w.carry) if w.carry is not None else None
    reps, t0 = 0, time.perf_counter()
    while True:
        oracle.decode_attend(q, k, v, off, w.num_heads, w.num_kv_heads, w.score_scale, carry=carry)
        reps += 1
        dt = time.perf_counter() - t0
        if dt >= seconds:
            break
    gbs = w.kv_bytes() * reps / dt / 1e9
    qh = w.batch * w.num_heads * reps / dt
    return gbs, qh, oracle.default_threads(), f"{reps} full passes of {w.name} ({dt:.1f} s wall)"


# ------------------------------------------------------------------ multi-rank plumbing

def rank_workload(name, rank, world):
    """The workload a rank times: the named one on a single GPU; under weak
    scaling every rank gets its own batch of the same shape (seed 1000+rank)."""
    from gqa_decode_attention_attend_b200 import workloads
    base = workloads.config(name)
    if world == 1:
        return base
    w = workloads.make(base.name, base.lengths, base.num_heads, base.num_kv_heads, base.head_dim,
                       dtype=base.k.dtype, dist=base.meta["dist"], seed=1000 + rank,
                       score_scale=base.score_scale, carry=base.carry is not None,
                       needle=dict(amp=8.0, depth=4096) if base.meta["dist"] == "needle" else None)
    w.meta["text"] = base.meta.get("text", "")
    return w


def max_over_ranks(x, device, dist=None):
    """Max of a float over all ranks (identity on one rank)."""
    import torch
    if dist is None or not dist.is_initialized() or dist.get_world_size() == 1:
        return float(x)
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def whole_job_gbs(kv_bytes_per_rank, world, ms_per_step_max):
    """Whole-job throughput: every rank's KV bytes over the slowest rank's step time."""
    return kv_bytes_per_rank * world / (ms_per_step_max / 1e3) / 1e9


# ------------------------------------------------------------------ ours

# Launches of the library's kernels per step of each op.
LAUNCHES = {"attend": 1, "append_attend": 1, "masked_attend": 2, "coded_attend": 1, "split_pipeline": 3}

# The long-context bf16 workloads that must hold >= 70 % of the nominal HBM
# bandwidth in KV-cache bytes read, each timed through the call its
# description names (the split stress workload through the three-call path).
TARGETS = (("bf16_b4_n32768", "split_pipeline"), ("bf16_b64_ragged16384", "attend"),
           ("bf16_b1_n131072", "attend"))


class Op:
    """One step of `op` on workload `w`, its inputs resident on `dev`.

    attend: plain decode attention; append_attend: append the new token's K/V
    then attend; masked_attend: index rows -> bias (gqa_topk_to_bias) then
    attend with it; coded_attend: the same shape as a dictionary-coded cache
    (8 code words per row, 256 atoms; KV bytes = code bytes read);
    split_pipeline: the three-call path (partial states, gqa_softmax_merge with
    the carry, gqa_state_finalize)."""

    def __init__(self, w, op, dev, flags, num_splits=0):
        import torch
        import gqa_decode_attention_attend_b200 as gqa
        self.gqa, self.w, self.op, self.flags, self.forced = gqa, w, op, flags, int(num_splits)
        H, G, D = w.num_heads, w.num_kv_heads, w.head_dim
        self.kv_bytes = w.kv_bytes()
        self.q = w.q.to(dev)
        self.offsets = w.offsets.to(dev)
        # two cache copies, alternated step by step, unless one is already > 4x L2
        self.caches = [(w.k.to(dev), w.v.to(dev))]
        if self.kv_bytes < 4 * 126e6:
            self.caches.append((self.caches[0][0].clone(), self.caches[0][1].clone()))
        self.carry = gqa.State(*(t.to(dev) for t in w.carry)) if w.carry is not None else None
        self.out = torch.empty(self.q.shape, dtype=self.q.dtype, device=dev)
        self.ws = gqa.Workspace(dev)
        gen = torch.Generator().manual_seed(77)
        self.k_new = torch.randn((w.batch, G, D), generator=gen).to(w.k.dtype).to(dev)
        self.v_new = torch.randn((w.batch, G, D), generator=gen).to(w.k.dtype).to(dev)
        self.idx = torch.randint(-1, max(w.max_seq_len, 1), (w.batch, 512), generator=gen,
                                 dtype=torch.int32).to(dev)
        self.bias = torch.zeros(w.total_rows, dtype=torch.float32, device=dev)
        self.kernel = ("gqa_partition_bf16_kernel" if w.k.dtype == torch.bfloat16
                       else "gqa_partition_f32_kernel")
        if op == "coded_attend":
            words, n_atoms = 8, 256
            cg = torch.Generator().manual_seed(78)
            idx = torch.randint(0, n_atoms, (w.total_rows, G, words), generator=cg, dtype=torch.int64)
            cf = torch.randn((w.total_rows, G, words), generator=cg).to(torch.float16).view(torch.int16)
            code = ((idx << 16) | (cf.to(torch.int64) & 0xFFFF)).to(torch.int64)
            code = torch.where(code >= 2**31, code - 2**32, code).to(torch.int32)
            self.kcodes = code.to(dev).contiguous()
            self.vcodes = torch.roll(code, 1, 0).to(dev).contiguous()
            self.atoms = torch.nn.functional.normalize(torch.randn((n_atoms, D), generator=cg), dim=1).to(dev)
            self.kv_bytes = 2 * self.kcodes.numel() * 4
            # the codes are small: enough copies, taken in turn, that each
            # step's codes come from HBM (more than twice the L2 in all)
            ncopy = min(16, max(2, -(-2 * 126_000_000 // self.kv_bytes)))
            self.code_sets = [(self.kcodes, self.vcodes)] + [
                (self.kcodes.clone(), self.vcodes.clone()) for _ in range(ncopy - 1)]
            self.kernel = "gqa_partition_coded_kernel"
        # the split plan of the plain call, and the three-call path's buffers
        self.S_ws, self.S, self.chunk = gqa.gqa_decode_workspace_size(
            self.q, self.caches[0][0], self.caches[0][1], self.offsets, H, G, score_scale=w.score_scale,
            want_out=True, num_splits=self.forced, max_seq_len=w.max_seq_len)
        if op == "coded_attend":
            _, self.S, self.chunk = gqa.gqa_decode_coded_workspace_size(
                self.q, self.kcodes, self.vcodes, self.atoms, self.atoms, self.offsets, H, G,
                score_scale=w.score_scale, carry=self.carry, num_splits=self.forced, max_seq_len=w.max_seq_len)
        if op == "split_pipeline":
            self.parts = gqa.State.empty(w.batch * H, D, dev, (self.S,))
            self.merged = gqa.State.empty(w.batch * H, D, dev)
        self.launches = LAUNCHES[op]

    def run(self, i, st=None, flags=None):
        gqa, w = self.gqa, self.w
        H, G = w.num_heads, w.num_kv_heads
        k, v = self.caches[i % len(self.caches)]
        fl = self.flags if flags is None else flags
        common = dict(score_scale=w.score_scale, max_seq_len=w.max_seq_len, workspace=self.ws, stream=st,
                      flags=fl)
        if self.op == "coded_attend":
            kc, vc = self.code_sets[i % len(self.code_sets)]
            gqa.gqa_decode_attend_coded(self.q, kc, vc, self.atoms, self.atoms, self.offsets,
                                        H, G, carry=self.carry, out=self.out, num_splits=self.forced, **common)
        elif self.op == "append_attend":
            gqa.gqa_decode_append_attend(self.q, k, v, self.offsets, self.k_new, self.v_new, H, G,
                                         carry=self.carry, out=self.out, num_splits=self.forced, **common)
        elif self.op == "split_pipeline":
            gqa.gqa_decode_attend(self.q, k, v, self.offsets, H, G, partials_out=self.parts,
                                  num_splits=self.S, **common)
            gqa.gqa_softmax_merge(self.parts, carry=self.carry, merged_out=self.merged, want_out=False,
                                  stream=st)
            gqa.gqa_state_finalize(self.merged, out=self.out.view(w.batch * H, w.head_dim), stream=st)
        elif self.op == "masked_attend":
            gqa.gqa_topk_to_bias(self.idx, self.offsets, w.total_rows, bias=self.bias, stream=st)
            gqa.gqa_decode_attend(self.q, k, v, self.offsets, H, G, carry=self.carry, out=self.out,
                                  bias=self.bias, num_splits=self.forced, **common)
        else:
            gqa.gqa_decode_attend(self.q, k, v, self.offsets, H, G, carry=self.carry, out=self.out,
                                  num_splits=self.forced, **common)

    def partials_only(self, i, st=None):
        """The partition launch alone (partial states out, no merge)."""
        gqa, w = self.gqa, self.w
        if not hasattr(self, "parts_only"):
            self.parts_only = gqa.State.empty(w.batch * w.num_heads, w.head_dim, self.q.device, (self.S,))
        if self.op == "coded_attend":
            kc, vc = self.code_sets[i % len(self.code_sets)]
            gqa.gqa_decode_attend_coded(self.q, kc, vc, self.atoms, self.atoms, self.offsets, w.num_heads,
                                        w.num_kv_heads, score_scale=w.score_scale, partials_out=self.parts_only,
                                        num_splits=self.S, max_seq_len=w.max_seq_len, workspace=self.ws,
                                        stream=st)
            return
        k, v = self.caches[i % len(self.caches)]
        gqa.gqa_decode_attend(self.q, k, v, self.offsets, w.num_heads, w.num_kv_heads,
                              score_scale=w.score_scale, partials_out=self.parts_only, num_splits=self.S,
                              max_seq_len=w.max_seq_len, workspace=self.ws, stream=st)


def time_steps(op, steps, warmup, eager):
    """Device time (ms) of `steps` steps after `warmup` untimed ones, by CUDA
    events on the launching stream. Unless `eager`, the K steps are captured
    once into a CUDA graph and replayed (the calls allocate nothing and never
    synchronise, so they capture as they are): the host's per-call marshalling
    is then off the critical path, as in a serving loop. Returns (ms, replay)
    where replay() re-runs the same timed work untimed."""
    import torch
    stream = torch.cuda.current_stream()
    for i in range(warmup):
        op.run(i)
    torch.cuda.synchronize()
    assert op.gqa.gqa_get_device_error(op.ws) == 0
    graph = None
    if not eager:
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph):
            cap = torch.cuda.current_stream()
            for i in range(steps):
                op.run(i, cap)
        torch.cuda.synchronize()
        graph.replay()                   # one untimed replay
        torch.cuda.synchronize()

    def replay():
        if graph is not None:
            graph.replay()
        else:
            for i in range(steps):
                op.run(i)

    torch.cuda.synchronize()
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    ev0.record(stream)
    replay()
    ev1.record(stream)
    torch.cuda.synchronize()
    return ev0.elapsed_time(ev1), replay, graph


def time_isolated(op, reps=20):
    """Median device time (ms) of one lone step: L2 flushed first (a 512 MiB
    write), the GPU kept busy by a spin kernel while the host enqueues the call
    (so no host gap is timed), plain stream order, no call before or after it
    in flight."""
    import torch
    stream = torch.cuda.current_stream()
    flush = torch.empty(512 << 20, dtype=torch.uint8, device=op.q.device)
    times = []
    for i in range(reps + 2):
        flush.zero_()
        torch.cuda._sleep(400000)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        op.run(i, flags=0)
        e1.record(stream)
        torch.cuda.synchronize()
        if i >= 2:
            times.append(e0.elapsed_time(e1))
    del flush
    return statistics.median(times)


def sampled(fn, sampler_gpu, min_s=1.5):
    """Run fn() (timed work) under the clock sampler, then keep the same load
    (fn's replay) for at least min_s seconds so the sampler sees it."""
    import torch
    sampler = ClockSampler(sampler_gpu)
    sampler.start()
    time.sleep(0.3)
    t0 = time.perf_counter()
    res = fn()
    ms, replay = res[0], res[1]
    while ms / 1e3 + (time.perf_counter() - t0) < min_s:
        replay()
        torch.cuda.synchronize()
    return res, sampler.stop()


def run_ours(args):
    import torch
    import torch.distributed as dist
    import gqa_decode_attention_attend_b200 as gqa

    rank, world, local = dist_env()
    if world > 1:
        dist.init_process_group("nccl", timeout=__import__("datetime").timedelta(seconds=120))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    stream = torch.cuda.current_stream()
    flags = 0 if args.no_early_start else gqa.GQA_FLAG_EARLY_START
    peak, peak_src = measured_peaks()

    w = rank_workload(args.workload, rank, world)
    op = Op(w, args.op, dev, flags, args.splits)
    kv_bytes = op.kv_bytes
    H, D = w.num_heads, w.head_dim

    def barrier():
        if world > 1:
            dist.barrier()

    args.warmup = max(args.warmup, 3)        # at least three untimed warm-up steps

    def timed():
        barrier()
        res = time_steps(op, args.steps, args.warmup, args.eager)
        torch.cuda.synchronize()
        barrier()
        return res

    if args.quick:
        (ms_total, _, graph), clocks = timed(), None
    else:
        (ms_total, _, graph), clocks = sampled(timed, local)
    del graph
    ms_max = max_over_ranks(ms_total, dev, dist if world > 1 else None)
    ms_per_step = ms_max / args.steps
    value = whole_job_gbs(kv_bytes, world, ms_per_step)

    # ---- the dominant kernel: one decode call is one launch of the partition
    # kernel (the split merge runs inside it), so its launch duration is this
    # rank's step time; the partials-only launch is reported beside it.
    launch_ms = ms_total / args.steps
    achieved = kv_bytes / (launch_ms / 1e3) / 1e9
    for i in range(5):
        op.partials_only(i)
    n_part = args.steps if args.quick else max(args.steps, 50)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for i in range(n_part):
        op.partials_only(i)
    e1.record(stream)
    torch.cuda.synchronize()
    part_ms = e0.elapsed_time(e1) / n_part
    iso_ms = None if args.quick else time_isolated(op)

    # ---- end to end: pinned host inputs -> device, call, output -> pinned host
    n_e2e = 0 if args.quick else args.e2e_steps
    e2e = None
    if n_e2e:
        dev_in = [op.q, op.offsets]
        dev_in += [op.kcodes, op.vcodes] if args.op == "coded_attend" else list(op.caches[0])
        if op.carry is not None:
            dev_in += [op.carry.m, op.carry.l, op.carry.acc]
        host_in = [t.cpu().pin_memory() for t in dev_in]
        hout = torch.empty(op.out.shape, dtype=op.out.dtype).pin_memory()
        h2d = sum(t.numel() * t.element_size() for t in host_in)
        d2h = hout.numel() * hout.element_size()

        def e2e_step():
            for d, h in zip(dev_in, host_in):
                d.copy_(h, non_blocking=True)
            op.run(0)
            hout.copy_(op.out, non_blocking=True)

        for _ in range(2):
            e2e_step()
        torch.cuda.synchronize()
        barrier()
        x0, x1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        x0.record(stream)
        for _ in range(n_e2e):
            e2e_step()
        x1.record(stream)
        torch.cuda.synchronize()
        e2e_ms = max_over_ranks(x0.elapsed_time(x1) / n_e2e, dev, dist if world > 1 else None)
        e2e = {"value": round(whole_job_gbs(kv_bytes, world, e2e_ms), 2), "unit": "GB/s",
               "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "ms_per_step": e2e_ms}
        del host_in, hout

    # ---- the long-context targets, each through the call its workload names
    targets = None
    if rank == 0 and world == 1 and not args.quick and not args.no_targets:
        targets = {}
        for name, top in TARGETS:
            if name == w.name and top == args.op and not args.splits:
                t_ms, t_iso, t_clk, t_op = launch_ms, iso_ms, clocks, op
            else:
                t_op = Op(rank_workload(name, 0, 1), top, dev, flags)
                (t_total, _, g), t_clk = sampled(lambda: time_steps(t_op, args.steps, args.warmup,
                                                                    args.eager), local)
                del g
                t_ms = t_total / args.steps
                t_iso = time_isolated(t_op)
            gbs = t_op.kv_bytes / (t_ms / 1e3) / 1e9
            targets[name] = {
                "op": top, "ms_per_step": t_ms, "gbs": round(gbs, 1),
                "frac_of_measured": round(gbs / peak, 4), "frac_of_nominal_8tbs": round(gbs / NOMINAL_HBM_GBS, 4),
                "isolated_ms": t_iso,
                "isolated_gbs": round(t_op.kv_bytes / (t_iso / 1e3) / 1e9, 1) if t_iso else None,
                "num_splits": t_op.S, "chunk_len": t_op.chunk, "launches_per_step": t_op.launches,
                "clocks": t_clk,
            }
            if t_op is not op:
                del t_op
                torch.cuda.empty_cache()

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline and not args.quick:
        gbs, qh, cores, sample = oracle_sample(w, args.cpu_seconds)
        cpu = {"value": gbs, "unit": "GB/s", "cores": cores, "kind": "oracle", "sample": sample,
               "queries_heads_per_s": qh}

    if rank == 0:
        line = {
            "metric": METRIC,
            "value": round(value, 1),
            "unit": "GB/s",
            "n_gpus": world,
            "steps": args.steps,
            "warmup": args.warmup,
            "ms_per_step": ms_per_step,
            "higher_is_better": True,
            "scaling": "weak",
            "vs_baseline": None,
            "dtype": "bf16" if w.k.dtype == torch.bfloat16 else "f32",
            "data": "synthetic (seeded, no dataset)",
            "config": {
                "workload": w.name, "op": args.op, "text": w.meta.get("text", ""), "batch": w.batch,
                "num_heads": H, "num_kv_heads": w.num_kv_heads, "head_dim": D, "seq_len": w.max_seq_len,
                "total_rows": w.total_rows, "kv_bytes_per_step": kv_bytes, "num_splits": op.S,
                "chunk_len": op.chunk,
                "l2": (f"inputs larger than L2: {len(op.code_sets)} copies of the {kv_bytes / 2**20:.0f} MiB "
                       f"of codes taken in turn" if args.op == "coded_attend" else
                       f"inputs larger than L2: {len(op.caches)} cache copies of "
                       f"{kv_bytes / 2**20:.0f} MiB alternated" if len(op.caches) > 1 else
                       f"inputs larger than L2: one {kv_bytes / 2**20:.0f} MiB cache, > 4x the 126 MB L2"),
                "parallelism": f"replicas x{world} (independent batches, no collective)",
            },
            "queries_heads_per_s": w.batch * H * world / (ms_per_step / 1e3),
            "pct_of_nominal_8tbs": round(100.0 * value / world / NOMINAL_HBM_GBS, 2),
            "pct_of_measured_peak": round(100.0 * value / world / peak, 2),
            "roofline": {
                "bound": "hbm", "kernel": op.kernel,
                "achieved": round(achieved, 1), "peak": peak, "peak_source": peak_src, "unit": "GB/s",
                "frac": round(achieved / peak, 4),
                "traffic": recorded_traffic(w.name) if args.op == "attend" and not args.splits else None,
                "algorithmic_bytes_per_launch": kv_bytes, "launch_ms": launch_ms,
                "isolated_launch_ms": iso_ms,
                "partials_only_launch_ms": part_ms,
                "partials_only_gbs": round(kv_bytes / (part_ms / 1e3) / 1e9, 1),
            },
            "cpu_baseline": cpu,
            "e2e": e2e,
            "gpu_launches": args.steps * op.launches,
            "launch_mode": ("eager" if args.eager else "cuda_graph_of_timed_steps") +
                           ("" if args.no_early_start else "+early_start"),
            "clocks": clocks,
        }
        if targets is not None:
            line["targets"] = targets
            line["targets_met_70pct_of_nominal"] = all(t["frac_of_nominal_8tbs"] >= 0.70
                                                       for t in targets.values())
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()


# ------------------------------------------------------------------ reference arm (CPU oracle)

def run_reference(args):
    rank, world, _ = dist_env()
    if rank != 0:
        return
    from gqa_decode_attention_attend_b200 import workloads
    import oracle
    w = workloads.config(args.workload)
    # each step: the oracle over a bounded sample of the workload (the first
    # sequences of the batch, all their heads), sized to a few hundred ms
    nseq = max(1, min(w.batch, 4))
    o = w.offsets[: nseq + 1]
    ws = workloads.make(w.name, w.lengths[:nseq], w.num_heads, w.num_kv_heads, w.head_dim,
                        dtype=w.k.dtype, seed=0)
    ws.q, ws.k, ws.v = w.q[:nseq], w.k[: int(o[-1])], w.v[: int(o[-1])]
    ws.carry = None if w.carry is None else tuple(t[: nseq * w.num_heads] for t in w.carry)
    ws.score_scale = w.score_scale
    q, k, v = (workloads.host_array(t) for t in (ws.q, ws.k, ws.v))
    off = ws.offsets.numpy()
    carry = tuple(t.numpy() for t in ws.carry) if ws.carry is not None else None

    def step():
        oracle.decode_attend(q, k, v, off, w.num_heads, w.num_kv_heads, w.score_scale, carry=carry)

    for _ in range(max(args.warmup, 1)):
        step()
    steps = args.steps
    t0 = time.perf_counter()
    for _ in range(steps):
        step()
        if time.perf_counter() - t0 > 120:        # keep the arm within a few minutes
            steps = _ + 1
            break
    dt = (time.perf_counter() - t0) / steps
    kvb = ws.kv_bytes()
    value = kvb / dt / 1e9
    cores = oracle.default_threads()
    sample = f"first {nseq} of {w.batch} sequences of {w.name}, all heads ({kvb / 2**20:.0f} MiB KV)"
    print(json.dumps({
        "impl": "reference", "metric": METRIC, "value": round(value, 3), "unit": "GB/s",
        "n_gpus": world, "steps": steps, "warmup": args.warmup, "ms_per_step": dt * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "f64", "data": "synthetic (seeded, no dataset)",
        "config": {"workload": w.name, "text": w.meta.get("text", ""), "batch": w.batch,
                   "num_heads": w.num_heads, "num_kv_heads": w.num_kv_heads,
                   "head_dim": w.head_dim, "seq_len": w.max_seq_len},
        "cpu_baseline": {"value": round(value, 3), "unit": "GB/s", "cores": cores, "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": round(value, 3), "unit": "GB/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }), flush=True)


def main():
    args = parse()
    if args.impl == "reference":
        run_reference(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
