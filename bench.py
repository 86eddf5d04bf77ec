#!/usr/bin/env python
"""Benchmark of the decode-attention hot path on B200.

One step = one gqa_decode_attend call over the whole batch (one launch of the
split-KV partition kernel, whose last CTA per sequence and KV head merges the
splits and writes the output) on the 16-sequence bf16 workload: batch 16,
32 Q / 8 KV heads, head_dim 128, 4096 cached keys per sequence, q/K/V iid
N(0,1), bf16 output. Inputs are resident in HBM before the timed region; two
copies of the 256 MiB cache are alternated so consecutive steps never read a
cache the 126 MB L2 could still hold.

The K timed steps are captured once into a CUDA graph and replayed (the call
allocates nothing and never synchronises), each launched with
GQA_FLAG_EARLY_START (no step writes the cache rows or offsets the next one
reads); --eager and --no-early-start turn either off.

Prints ONE JSON line (rank 0). `value` is the KV-cache bytes read per step,
summed over ranks, divided by the max-over-ranks device time (GB/s); `e2e` is
the same metric through the same public call when every step also copies its
inputs from pinned host memory and its output back.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                  [--workload NAME] [--op OP] [--eager] [--no-early-start]
                  [--no-cpu-baseline] [--quick]

--impl reference times the f64 CPU oracle (the library's reference
implementation) on a bounded sample of the same workload, on rank 0 only.
"""
import argparse
import hashlib
import json
import math
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
    ap.add_argument("--workload", default="bf16_b16_n4096")
    ap.add_argument("--op", choices=["attend", "append_attend", "masked_attend", "coded_attend",
                                     "split_pipeline"],
                    default="attend",
                    help="attend: plain decode attention (the default line); append_attend: "
                         "append the new token's K/V then attend; masked_attend: index rows -> "
                         "bias (gqa_topk_to_bias) then attend with it; coded_attend: the "
                         "same shape as a dictionary-coded cache (8 code words per row, 256 "
                         "atoms), KV bytes = code bytes read; split_pipeline: the three-call "
                         "path (partial states, gqa_softmax_merge with the carry, "
                         "gqa_state_finalize)")
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

def run_ours(args):
    import torch
    import torch.distributed as dist
    import gqa_decode_attention_attend_b200 as gqa
    from gqa_decode_attention_attend_b200 import workloads

    rank, world, local = dist_env()
    if world > 1:
        dist.init_process_group("nccl", timeout=__import__("datetime").timedelta(seconds=120))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    stream = torch.cuda.current_stream()

    w = rank_workload(args.workload, rank, world)
    H, G, D = w.num_heads, w.num_kv_heads, w.head_dim
    kv_bytes = w.kv_bytes()
    q = w.q.to(dev)
    offsets = w.offsets.to(dev)
    # two cache copies, alternated step by step (together > 2x L2)
    caches = [(w.k.to(dev), w.v.to(dev))]
    if kv_bytes < 4 * 126e6:
        caches.append((caches[0][0].clone(), caches[0][1].clone()))
    carry = gqa.State(*(t.to(dev) for t in w.carry)) if w.carry is not None else None
    out = torch.empty(q.shape, dtype=q.dtype, device=dev)
    ws = gqa.Workspace(dev)

    gen = torch.Generator().manual_seed(77)
    k_new = torch.randn((w.batch, G, D), generator=gen).to(w.k.dtype).to(dev)
    v_new = torch.randn((w.batch, G, D), generator=gen).to(w.k.dtype).to(dev)
    width = 512
    idx = torch.randint(-1, max(w.max_seq_len, 1), (w.batch, width), generator=gen,
                        dtype=torch.int32).to(dev)
    bias = torch.zeros(w.total_rows, dtype=torch.float32, device=dev)

    if args.op == "coded_attend":
        # synthetic dictionary and codes of the workload's shape: 8 words per row
        words, n_atoms = 8, 256
        cg = torch.Generator().manual_seed(78)
        idx = torch.randint(0, n_atoms, (w.total_rows, G, words), generator=cg, dtype=torch.int64)
        cf = torch.randn((w.total_rows, G, words), generator=cg).to(torch.float16).view(torch.int16)
        code = ((idx << 16) | (cf.to(torch.int64) & 0xFFFF)).to(torch.int64)
        code = torch.where(code >= 2**31, code - 2**32, code).to(torch.int32)
        kcodes = [code.to(dev).contiguous()]
        vcodes = [torch.roll(code, 1, 0).to(dev).contiguous()]
        atoms = torch.nn.functional.normalize(torch.randn((n_atoms, D), generator=cg), dim=1).to(dev)
        kv_bytes = 2 * kcodes[0].numel() * 4

    def step(i):
        run_op(*caches[i % len(caches)])

    def step_on(i, st):
        run_op(*caches[i % len(caches)], st)

    flags = 0 if args.no_early_start else gqa.GQA_FLAG_EARLY_START
    if args.op == "split_pipeline":
        # the heuristic's split count (a sizing query), and the three calls' buffers
        _, sp_splits, _ = gqa.gqa_decode_workspace_size(
            q, caches[0][0], caches[0][1], offsets, H, G, score_scale=w.score_scale, want_out=False,
            partials_out=gqa.State.empty(1, D, dev, (1,)), max_seq_len=w.max_seq_len)
        sp_parts = gqa.State.empty(w.batch * H, D, dev, (sp_splits,))
        sp_merged = gqa.State.empty(w.batch * H, D, dev)

    def run_op(k, v, st=None):
        st = st or stream
        if args.op == "coded_attend":
            gqa.gqa_decode_attend_coded(q, kcodes[0], vcodes[0], atoms, atoms, offsets, H, G,
                                        score_scale=w.score_scale, carry=carry, out=out,
                                        max_seq_len=w.max_seq_len, workspace=ws, stream=st, flags=flags)
        elif args.op == "append_attend":
            gqa.gqa_decode_append_attend(q, k, v, offsets, k_new, v_new, H, G, score_scale=w.score_scale,
                                         carry=carry, out=out, max_seq_len=w.max_seq_len, workspace=ws,
                                         stream=st, flags=flags)
        elif args.op == "split_pipeline":
            gqa.gqa_decode_attend(q, k, v, offsets, H, G, score_scale=w.score_scale, partials_out=sp_parts,
                                  num_splits=sp_splits, max_seq_len=w.max_seq_len, workspace=ws, stream=st,
                                  flags=flags)
            gqa.gqa_softmax_merge(sp_parts, carry=carry, merged_out=sp_merged, want_out=False, stream=st)
            gqa.gqa_state_finalize(sp_merged, out=out.view(w.batch * H, D), stream=st)
        elif args.op == "masked_attend":
            gqa.gqa_topk_to_bias(idx, offsets, w.total_rows, bias=bias, stream=st)
            gqa.gqa_decode_attend(q, k, v, offsets, H, G, score_scale=w.score_scale, carry=carry,
                                  out=out, max_seq_len=w.max_seq_len, workspace=ws, stream=st,
                                  bias=bias, flags=flags)
        else:
            gqa.gqa_decode_attend(q, k, v, offsets, H, G, score_scale=w.score_scale, carry=carry,
                                  out=out, max_seq_len=w.max_seq_len, workspace=ws, stream=st, flags=flags)

    def barrier():
        if world > 1:
            dist.barrier()

    args.warmup = max(args.warmup, 3)        # at least three untimed warm-up steps
    for i in range(args.warmup):
        step(i)
    torch.cuda.synchronize()
    assert gqa.gqa_get_device_error(ws) == 0

    # The timed K steps are captured once into a CUDA graph (the calls allocate
    # nothing and never synchronise, so they capture as-is) and replayed: the
    # host's per-call marshalling is then off the critical path, as in a serving
    # loop. --eager launches them one by one instead.
    graph = None
    if not args.eager:
        torch.cuda.synchronize()
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph):
            cap_stream = torch.cuda.current_stream()
            for i in range(args.steps):
                step_on(i, cap_stream)
        torch.cuda.synchronize()
        graph.replay()                   # one untimed replay
        torch.cuda.synchronize()

    def timed_steps():
        if graph is not None:
            graph.replay()
        else:
            for i in range(args.steps):
                step(i)

    sampler = ClockSampler(local) if not args.quick else None
    if sampler:
        sampler.start()
        time.sleep(0.3)
    barrier()
    torch.cuda.synchronize()
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    ev0.record(stream)
    timed_steps()
    ev1.record(stream)
    torch.cuda.synchronize()
    barrier()
    ms_total = ev0.elapsed_time(ev1)
    # keep the same load for at least ~1.5 s so the clock sampler sees it
    extra_t0 = time.perf_counter()
    i = 0
    while sampler and ms_total / 1e3 + (time.perf_counter() - extra_t0) < 1.5:
        timed_steps()
        torch.cuda.synchronize()
    clocks = sampler.stop() if sampler else None

    ms_max = max_over_ranks(ms_total, dev, dist if world > 1 else None)
    ms_per_step = ms_max / args.steps
    value = whole_job_gbs(kv_bytes, world, ms_per_step)

    # ---- dominant kernel alone: the partition launch (partials-only call)
    S_ws, S, chunk = gqa.gqa_decode_workspace_size(q, caches[0][0], caches[0][1], offsets, H, G,
                                                   score_scale=w.score_scale, want_out=True,
                                                   max_seq_len=w.max_seq_len)
    parts = gqa.State.empty(w.batch * H, D, dev, (S,))

    def part_only(i):
        k, v = caches[i % len(caches)]
        gqa.gqa_decode_attend(q, k, v, offsets, H, G, score_scale=w.score_scale, partials_out=parts,
                              num_splits=S, max_seq_len=w.max_seq_len, workspace=ws, stream=stream)

    for i in range(5):
        part_only(i)
    n_part = args.steps if args.quick else max(args.steps, 50)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for i in range(n_part):
        part_only(i)
    e1.record(stream)
    torch.cuda.synchronize()
    part_ms = e0.elapsed_time(e1) / n_part
    peak, peak_src = measured_peaks()
    # A decode call is one launch of the partition kernel (the split merge runs
    # inside it), so the dominant kernel's launch duration is the step time of
    # this rank; the partials-only launch is reported beside it.
    launch_ms = ms_total / args.steps
    achieved = kv_bytes / (launch_ms / 1e3) / 1e9

    # ---- end to end: pinned host inputs -> device, call, output -> pinned host
    hq = w.q.pin_memory()
    hoff = w.offsets.pin_memory()
    hout = torch.empty(out.shape, dtype=out.dtype).pin_memory()
    # the step's cache inputs: the raw K/V, or the code arrays for the coded op
    if args.op == "coded_attend":
        dev_cache = [kcodes[0], vcodes[0]]
    else:
        dev_cache = list(caches[0])
    host_cache = [t.cpu().pin_memory() for t in dev_cache]
    h2d = (hq.numel() * hq.element_size() + sum(t.numel() * t.element_size() for t in host_cache) +
           hoff.numel() * 4)
    d2h = hout.numel() * hout.element_size()

    def e2e_step():
        q.copy_(hq, non_blocking=True)
        for d, h in zip(dev_cache, host_cache):
            d.copy_(h, non_blocking=True)
        offsets.copy_(hoff, non_blocking=True)
        run_op(*caches[0])
        hout.copy_(out, non_blocking=True)

    n_e2e = 0 if args.quick else args.e2e_steps
    for _ in range(2 if n_e2e else 0):
        e2e_step()
    torch.cuda.synchronize()
    barrier()
    x0, x1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    x0.record(stream)
    for _ in range(n_e2e):
        e2e_step()
    x1.record(stream)
    torch.cuda.synchronize()
    e2e_ms = max_over_ranks(x0.elapsed_time(x1) / max(n_e2e, 1), dev, dist if world > 1 else None)
    e2e_value = whole_job_gbs(kv_bytes, world, e2e_ms)

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
                "num_heads": H, "num_kv_heads": G, "head_dim": D, "seq_len": w.max_seq_len,
                "kv_bytes_per_step": kv_bytes, "num_splits": S, "chunk_len": chunk,
                "l2": f"inputs larger than L2: {len(caches)} cache copies of {kv_bytes / 2**20:.0f} MiB alternated",
                "parallelism": f"replicas x{world} (independent batches, no collective)",
            },
            "queries_heads_per_s": w.batch * H * world / (ms_per_step / 1e3),
            "pct_of_nominal_8tbs": round(100.0 * value / world / NOMINAL_HBM_GBS, 2),
            "pct_of_measured_peak": round(100.0 * value / world / peak, 2),
            "roofline": {
                "bound": "hbm",
                "kernel": ("gqa_partition_coded_kernel" if args.op == "coded_attend" else
                           "gqa_partition_bf16_kernel" if w.k.dtype == torch.bfloat16
                           else "gqa_partition_f32_kernel"),
                "achieved": round(achieved, 1), "peak": peak, "peak_source": peak_src, "unit": "GB/s",
                "frac": round(achieved / peak, 4), "traffic": recorded_traffic(w.name) if args.op == "attend" else None,
                "algorithmic_bytes_per_launch": kv_bytes, "launch_ms": launch_ms,
                "partials_only_launch_ms": part_ms,
                "partials_only_gbs": round(kv_bytes / (part_ms / 1e3) / 1e9, 1),
            },
            "cpu_baseline": cpu,
            "e2e": {"value": round(e2e_value, 2), "unit": "GB/s", "h2d_bytes_per_step": h2d,
                    "d2h_bytes_per_step": d2h, "ms_per_step": e2e_ms},
            "gpu_launches": args.steps * {"masked_attend": 2, "split_pipeline": 3}.get(args.op, 1),
            "launch_mode": ("eager" if args.eager else "cuda_graph_of_timed_steps") +
                           ("" if args.no_early_start else "+early_start"),
            "clocks": clocks,
        }
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
