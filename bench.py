"""Decode attention-stage benchmark of the JSSA hot path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl jssa|reference] [--workload NAME]

A step is one decode step of one attention layer at the workload's shape:
append the new token's low-rank key row, score the low-rank cache, select a
top-k token set per (batch, KV head), and run gather-free indexed attention
(jssa_decode_step: one launch of the fused streaming kernel where that form
applies, else three or four kernels).  The default workload is the
128K-context, batch-16 GQA layer (B=16, Hq=32, Hkv=8, d=128, T=131072, r=32,
k=256).

value  = steps/s of the whole job (N replicas, one per GPU, each running the
         full workload: weak scaling, no collective on the data path), timed
         on the device with CUDA events over exactly K steps, max over ranks;
         each step is a replay of a CUDA graph of jssa_decode_step (one graph
         per rotating query; --eager times the plain call loop instead).
e2e    = the same metric through the public session API with host buffers:
         every step copies q and the new K/V rows from pinned host memory and
         reads the output back (synchronising per step).
roofline = the dominant kernel against the measured HBM copy bandwidth: the
         fused step kernel itself when the step is one launch (algorithmic bytes
         of the step / its duration in the timed loop), else the selection pass
         (jssa_select) timed alone.
cpu_baseline / --impl reference = the fp64 C oracle on the host cores over a
         bounded sample of (batch, KV head) pairs, scaled to a whole step.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "decode attn-stage steps/s at 128K ctx, batch 16; achieved HBM GB/s vs peak"
FALLBACK_HBM_GBS = 6650.0


def log(*a):
    print(*a, file=sys.stderr, flush=True)


def measured_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return float(d.get("hbm_gbs", FALLBACK_HBM_GBS)), "measured"
    return FALLBACK_HBM_GBS, "fallback"


def algorithmic_bytes(w):
    """Bytes the method must move per step: the low-rank key cache, the k
    selected K and V rows per (b, h), the queries and the outputs."""
    es = 2
    kt = w.B * w.Hkv * w.T * w.r * es
    row = w.d if w.latent else w.d + w.Dv  # a latent row is key and value at once
    sel = w.B * w.Hkv * min(w.k, w.T) * row * es
    qo = w.B * w.Hq * (w.d + w.Dv) * es
    return kt + sel + qo, kt


def select_bytes(w):
    """Algorithmic bytes of the fused score + top-k pass: the low-rank cache,
    the queries and the index lists it writes."""
    return w.B * w.Hkv * w.T * w.r * 2 + w.B * w.Hq * w.d * 2 + w.B * w.Hkv * (w.k + 1) * 4


def profile_traffic(kernel_file, summary):
    """DRAM bytes per launch from a committed ncu summary (profiles/<summary>),
    if the summary's source hash matches the kernel source as it is now (else
    None)."""
    path = os.path.join(ROOT, "profiles", summary)
    src = os.path.join(ROOT, "token_level_sparse_kv_b200", "csrc", kernel_file)
    if not (os.path.exists(path) and os.path.exists(src)):
        return None
    h = hashlib.sha256(open(src, "rb").read()).hexdigest()[:16]
    vals = {}
    for line in open(path):
        if ":" in line:
            k, v = line.split(":", 1)
            vals[k.strip()] = v.strip()
    if vals.get("source_sha256_16") != h:
        return None
    try:
        return float(vals["dram_bytes_per_launch"])
    except (KeyError, ValueError):
        return None


class ClockSampler:
    """nvidia-smi clock / throttle sampling while the timed region runs."""

    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.hw_slowdown,"
              "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
              "clocks_event_reasons.sw_power_cap")

    def __init__(self, index):
        self.index = index
        self.proc = None

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.index), "--query-gpu=" + self.FIELDS, "--format=csv,noheader,nounits",
                 "-lms", "100"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except (OSError, ValueError):
            self.proc = None
        return self

    def __exit__(self, *exc):
        self.lines = []
        if self.proc is not None:
            self.proc.terminate()
            try:
                out, _ = self.proc.communicate(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
                out, _ = self.proc.communicate()
            self.lines = [l for l in out.splitlines() if l.strip()]

    def summary(self):
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for l in getattr(self, "lines", []):
            parts = [p.strip() for p in l.split(",")]
            if len(parts) < 7:
                continue
            try:
                sm.append(float(parts[0]))
                mx = float(parts[1])
            except ValueError:
                continue
            for n, v in zip(names, parts[3:7]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": mx, "reasons": sorted(reasons), "samples": len(sm)}


def setup_dist(args):
    import torch

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime

        import torch.distributed as dist

        backend = "nccl" if torch.cuda.is_available() else "gloo"
        if torch.cuda.is_available():
            torch.cuda.set_device(local)
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120))
    elif torch.cuda.is_available():
        torch.cuda.set_device(local)
    return world, rank, local


def max_over_ranks(x, world):
    if world == 1:
        return x
    import torch
    import torch.distributed as dist

    dev = "cuda" if torch.cuda.is_available() else "cpu"
    t = torch.tensor([float(x)], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def barrier(world):
    if world > 1:
        import torch.distributed as dist

        dist.barrier()


# --------------------------------------------------------------- CPU oracle
class OracleSample:
    """The fp64 C oracle on a bounded sample of one workload: n_rows batch rows
    drawn on the host (all KV heads), the prefix low-rank cache built by the
    oracle itself; a timed unit is one decode step (append one row, score,
    select, attend) over a chosen number of (batch, KV head) pairs."""

    def __init__(self, w, n_rows, threads):
        import oracle
        from token_level_sparse_kv_b200.inputs import Workload, make_inputs

        self.w = w
        self.threads = threads
        oracle.set_threads(threads)
        ws = Workload(**{**w.__dict__, "B": n_rows, "name": w.name + "_sample"})
        self.q, self.K, self.V, self.P, self.sl = make_inputs(ws, device="cpu")
        self.Kt = oracle.append_lowrank(self.K, self.P, [0] * n_rows, ws.T)
        self.pos = (self.sl - 1).clamp_min(0).tolist()
        self.n_pairs_avail = n_rows * w.Hkv
        self.cursor = 0

    def run(self, n_pairs):
        """One timed oracle step over n_pairs (b, h) pairs; returns seconds."""
        import oracle

        w = self.w
        bh = [(self.cursor + i) % self.n_pairs_avail for i in range(n_pairs)]
        self.cursor = (self.cursor + n_pairs) % self.n_pairs_avail
        rows = sorted(set(x // w.Hkv for x in bh))
        t0 = time.perf_counter()
        Kt = self.Kt  # the append touches only the sampled rows' newest position
        oracle.append_lowrank(self.K[rows[0]:rows[-1] + 1], self.P, [self.pos[r] for r in range(rows[0], rows[-1] + 1)],
                              1, Kt=Kt[rows[0]:rows[-1] + 1])
        s = oracle.score(self.q, self.P, Kt, self.sl, bh_list=bh)
        idx, cnt = oracle.topk(s, self.sl, w.k, bh_list=bh)
        oracle.attend(self.q, self.K, self.V, idx, cnt, self.sl, w.scale, dv=w.Dv, bh_list=bh,
                      v_aliases_k=self.V is None)
        return time.perf_counter() - t0

    def describe(self, n_pairs, repeats):
        w = self.w
        return ("%d of %d (batch, KV head) pairs per timed step (T=%d, r=%d, k=%d): append 1 row, score, select, "
                "attend; mean of %d, scaled x%g to a full step" % (n_pairs, w.B * w.Hkv, w.T, w.r, w.k, repeats,
                                                                  w.B * w.Hkv / n_pairs))


def oracle_baseline(w, budget_s, n_rows, threads):
    """Oracle steps/s over about budget_s seconds of host work."""
    smp = OracleSample(w, n_rows, threads)
    n_pairs = smp.n_pairs_avail
    smp.run(n_pairs)  # warm
    times = []
    t_end = time.perf_counter() + budget_s
    while time.perf_counter() < t_end or len(times) < 3:
        times.append(smp.run(n_pairs))
    per_step = statistics.mean(times) * (w.B * w.Hkv / n_pairs)
    return 1.0 / per_step, smp.describe(n_pairs, len(times)), threads


def run_reference(args, world, rank):
    if rank != 0:
        return 0
    w = workload_of(args)
    threads = os.cpu_count() or 1
    smp = OracleSample(w, max(1, min(w.B, args.cpu_rows)), threads)
    # size the per-step sample so that warm-up + timed steps take about 2 minutes
    t1 = smp.run(1)
    t1 = min(t1, smp.run(1))
    n_pairs = int(max(1, min(smp.n_pairs_avail, 120.0 / (args.steps + args.warmup) / max(t1, 1e-6))))
    for _ in range(args.warmup):
        smp.run(n_pairs)
    times = [smp.run(n_pairs) for _ in range(args.steps)]
    sec = statistics.mean(times) * (w.B * w.Hkv / n_pairs)
    v = 1.0 / sec
    line = {"impl": "reference", "metric": METRIC, "value": v, "unit": "steps/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": sec * 1e3, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": config_of(w, world),
            "cpu_baseline": {"value": v, "unit": "steps/s", "cores": threads, "kind": "oracle",
                             "sample": smp.describe(n_pairs, args.steps)},
            "e2e": {"value": v, "unit": "steps/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


def workload_of(args):
    from token_level_sparse_kv_b200.inputs import WORKLOADS, Workload

    w = WORKLOADS[args.workload]
    over = {}
    if args.batch is not None and args.batch != w.B:
        over["B"] = args.batch
    if args.topk is not None and args.topk != w.k:
        over["k"] = args.topk
    if over:
        name = w.name + "".join("_%s%d" % (("b" if k == "B" else "k"), v) for k, v in over.items())
        w = Workload(**{**w.__dict__, **over, "name": name})
    return w


def flushes_l2(w, l2_bytes):
    """Whether a timed step of workload w needs an L2 flush before it: its
    streamed bytes would otherwise sit in the L2 from the step before."""
    step_bytes, _ = algorithmic_bytes(w)
    return step_bytes < 2 * l2_bytes


def config_of(w, world, flush=False):
    return {"workload": w.name, "B": w.B, "Hq": w.Hq, "Hkv": w.Hkv, "d": w.d, "dv": w.Dv, "T": w.T, "r": w.r,
            "k": w.k, "inputs": ("N(0,1) Gaussian" if w.kind == "plain" else
                                 "spiked Gaussian (q spike 2, key spike 3 along one direction on 1% of tokens)"),
            "l2": (("L2 flushed before every timed step (a %.0f MiB step fits in L2); per-step CUDA events"
                    % (algorithmic_bytes(w)[0] / 2**20)) if flush else
                   ("inputs larger than L2 (%.0f MiB low-rank cache streamed per step; 4 rotating queries)"
                    % (w.B * w.Hkv * w.T * w.r * 2 / 2**20))),
            "parallelism": "replicas x%d (one full workload per GPU)" % world}


# --------------------------------------------------------------- GPU timing
def time_loop(fn, steps, stream, events_inside=None):
    import torch

    torch.cuda.synchronize()
    start = torch.cuda.Event(enable_timing=True)
    end = torch.cuda.Event(enable_timing=True)
    start.record(stream)
    for i in range(steps):
        fn(i)
    end.record(stream)
    torch.cuda.synchronize()
    return start.elapsed_time(end) / 1e3


def time_steps(fn, steps, stream, flush_buf=None):
    """Per-step CUDA-event durations (seconds) of steps calls fn(i).  Without
    flush_buf the events sit back to back (their sum is the loop's device
    time); with it the L2 is flushed (a write of a buffer twice its size)
    before each step, outside the step's events."""
    import torch

    torch.cuda.synchronize()
    if flush_buf is None:
        evs = [torch.cuda.Event(enable_timing=True) for _ in range(steps + 1)]
        evs[0].record(stream)
        for i in range(steps):
            fn(i)
            evs[i + 1].record(stream)
        torch.cuda.synchronize()
        return [evs[i].elapsed_time(evs[i + 1]) / 1e3 for i in range(steps)]
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
    for i, (a, b) in enumerate(evs):
        flush_buf.fill_(i & 255)
        a.record(stream)
        fn(i)
        b.record(stream)
    torch.cuda.synchronize()
    return [a.elapsed_time(b) / 1e3 for a, b in evs]


def percentile(xs, q):
    ys = sorted(xs)
    if not ys:
        return float("nan")
    pos = (len(ys) - 1) * q
    lo = int(pos)
    hi = min(lo + 1, len(ys) - 1)
    return ys[lo] + (ys[hi] - ys[lo]) * (pos - lo)


def latency_summary(durs):
    return {"p10_us": percentile(durs, 0.1) * 1e6, "p50_us": percentile(durs, 0.5) * 1e6,
            "p90_us": percentile(durs, 0.9) * 1e6, "mean_us": sum(durs) / len(durs) * 1e6, "n": len(durs)}


def graphed(fn, dev, n=4):
    """One CUDA graph per rotating input (fn(j), j < n), replayed by index."""
    from token_level_sparse_kv_b200 import ops

    graphs = [ops.StepGraph(lambda j=j: fn(j), dev) for j in range(n)]
    return lambda i: graphs[i % n].replay()


def measure_decode_loop(dev, n_layers, steps, stream):
    """Steady-state steps/s of an n_layers attention stack at the 4K/B1 GQA
    layer shape (each layer's output is the next layer's query), eager calls
    vs one CUDA graph per step (every layer plus the position advance)."""
    import torch

    from token_level_sparse_kv_b200 import ops
    from token_level_sparse_kv_b200.inputs import WORKLOADS, Workload, make_inputs

    w0 = WORKLOADS["gqa_4k_b1"]
    room = 2 * steps + 16
    layers = []
    for l in range(n_layers):
        w = Workload(**{**w0.__dict__, "seed": w0.seed + 7000 + l})
        q, K, V, P, sl = make_inputs(w, device=dev)
        layers.append((K, V, P, ops.build_lowrank_cache(K, P)))
    res = {"layers": n_layers, "shape": "GQA layer B=1, Hq=32, Hkv=8, d=128, T=4096, r=32, k=256"}
    for mode in ("eager", "graph"):
        sl = torch.full((w0.B,), w0.T - room, dtype=torch.int32, device=dev)
        pos = sl - 1
        loop = ops.DecodeLoop(layers, sl, pos, w0.k, w0.scale)
        loop.set_query(q)
        g = mode == "graph"
        for _ in range(3):
            loop.step(graph=g)
        torch.cuda.synchronize()
        secs = time_loop(lambda i: loop.step(graph=g), steps, stream)
        res[mode] = {"steps_per_s": steps / secs, "us_per_step": secs / steps * 1e6,
                     "us_per_layer": secs / steps / n_layers * 1e6}
    res["launches_per_step"] = n_layers * ops.plan_info(ops.make_dims(q, layers[0][0], layers[0][1], P=layers[0][2],
                                                                       Kt=layers[0][3]), w0.k,
                                                        ops.OP_DECODE_STEP)[0] + 2
    del layers
    torch.cuda.empty_cache()
    return res


def screening_comparison(w, qs, K, V, P, Kt, sl, pos, dims, dev, stream, flush_buf, steps, world, use_graph):
    """The decode step with exact block screening (per-128-token norm bounds
    of the low-rank cache): its time and the tiles it skipped per step, on
    the same inputs as the timed step (results are bit-identical)."""
    import torch

    from token_level_sparse_kv_b200 import ops

    nrm = ops.block_norms(Kt)
    ws = ops.new_workspace(dims, w.k, ops.OP_DECODE_STEP, dev)
    idx = torch.empty((w.B, w.Hkv, w.k), dtype=torch.int32, device=dev)
    cnt = torch.empty((w.B, w.Hkv), dtype=torch.int32, device=dev)
    out = torch.empty((w.B, w.Hq, w.Dv), dtype=qs[0].dtype, device=dev)
    lse = torch.empty((w.B, w.Hq), dtype=torch.float32, device=dev)

    ws_plain = ops.new_workspace(dims, w.k, ops.OP_DECODE_STEP, dev)

    def step(i):
        ops.decode_step(qs[i & 3], K, V, P, Kt, sl, pos, w.k, w.scale, ws=ws, idx=idx, count=cnt, out=out, lse=lse,
                        block_norms=nrm)

    def plain(i):
        ops.decode_step(qs[i & 3], K, V, P, Kt, sl, pos, w.k, w.scale, ws=ws_plain, idx=idx, count=cnt, out=out,
                        lse=lse)

    fns = {}
    for name, fn in (("screened", step), ("plain", plain)):
        for i in range(3):
            fn(i)
        fns[name] = graphed(fn, dev) if use_graph else fn
        for i in range(3):
            fns[name](i)
    torch.cuda.synchronize()
    before = ops.skip_count(ws)
    # alternate the two in blocks so that clock and power drift hit both alike
    ds, dp = [], []
    blk = max(1, steps // 4)
    for _ in range(4):
        ds += time_steps(fns["screened"], blk, stream, flush_buf)
        dp += time_steps(fns["plain"], blk, stream, flush_buf)
    skipped = ops.skip_count(ws) - before
    med = max_over_ranks(percentile(ds, 0.5), world)
    medp = max_over_ranks(percentile(dp, 0.5), world)
    tiles = w.B * w.Hkv * ((w.T * w.r * 2 + 32767) // 32768)
    return {"steps_per_s": world / med, "ms_per_step": med * 1e3, "plain_ms_per_step": medp * 1e3,
            "skipped_tiles_per_step": skipped / len(ds), "tiles_per_step": tiles,
            "note": "Cauchy-Schwarz bound ||qbar|| * max ||Kt_t|| per 128-token block against the segment's k-th "
                    "key; on these inputs the bound rarely falls below it"}


def calibration_recall(w, q, K, P, sl, dev, stream, n_keys=4096, iters=30):
    """Selection quality against the exact top-k of the full-width group
    scores (sum_g q_g . K_t, by the library's own selection with an identity
    basis, r = d): recall of the k selected tokens per (b, h) with the random
    orthonormal basis and with the basis calibrated from the step's queries
    and sampled keys (jssa_calibrate_basis), and the calibration's time."""
    import torch

    from token_level_sparse_kv_b200 import ops

    eye = torch.eye(w.d, dtype=torch.float32, device=dev).expand(w.Hkv, w.d, w.d).contiguous()
    Kt_full = ops.build_lowrank_cache(K, eye)
    idx_exact, _ = ops.select(q, eye, Kt_full, sl, w.k)
    del Kt_full
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    ops.calibrate_basis(q, K, sl, P, n_keys=n_keys, iters=iters)  # warm (planning)
    a.record(stream)
    P_cal = ops.calibrate_basis(q, K, sl, P, n_keys=n_keys, iters=iters)
    b.record(stream)
    torch.cuda.synchronize()
    cal_ms = a.elapsed_time(b)

    def recall(basis):
        Kt = ops.build_lowrank_cache(K, basis)
        idx, _ = ops.select(q, basis, Kt, sl, w.k)
        hit = (idx.unsqueeze(-1) == idx_exact.unsqueeze(-2)).any(-1) & (idx >= 0)
        r = float(hit.sum().item() / max(1, int((idx_exact >= 0).sum().item())))
        del Kt
        torch.cuda.empty_cache()
        return r

    res = {"recall_random_P": recall(P), "recall_calibrated_P": recall(P_cal), "calibration_ms": cal_ms,
           "samples": "the step's queries (%d rows) and %d evenly spaced keys per batch row; %d iterations"
                      % (w.B, n_keys, iters),
           "reference": "exact top-k of the full-width group scores (identity basis, r = d)"}
    torch.cuda.synchronize()
    return res


def per_head_comparison(w, q, K, V, P, Kt, sl, pos, dims, dev, stream, flush_buf, steps, world, use_graph):
    """The per-query-head selection variant (every query head its own top-k)
    against the method's per-KV-head selection on the same inputs: step time
    of both as separate calls (append, selection, indexed attention), bytes of
    selected rows each reads, the recall of the shared per-KV-head set against
    each query head's own top-k, and each output's distance to dense full-KV
    attention (a proxy for what sharing one set per KV head costs)."""
    import torch

    from token_level_sparse_kv_b200 import ops

    G = w.G
    ws_a = ops.new_workspace(dims, 1, ops.OP_APPEND, dev)
    ws_s = ops.new_workspace(dims, w.k, ops.OP_SELECT, dev)
    ws_i = ops.new_workspace(dims, w.k, ops.OP_INDEXED_DECODE, dev)
    ws_sh = ops.new_workspace(dims, w.k, ops.OP_SELECT_HEADS, dev)
    ws_ih = ops.new_workspace(dims, w.k, ops.OP_INDEXED_DECODE_HEADS, dev)
    idx = torch.empty((w.B, w.Hkv, w.k), dtype=torch.int32, device=dev)
    cnt = torch.empty((w.B, w.Hkv), dtype=torch.int32, device=dev)
    idh = torch.empty((w.B, w.Hq, w.k), dtype=torch.int32, device=dev)
    cnh = torch.empty((w.B, w.Hq), dtype=torch.int32, device=dev)
    out_kv = torch.empty((w.B, w.Hq, w.Dv), dtype=q.dtype, device=dev)
    out_q = torch.empty_like(out_kv)
    lse = torch.empty((w.B, w.Hq), dtype=torch.float32, device=dev)

    def kv_step(i):
        ops.append_lowrank(K, P, Kt, pos, 1, ws=ws_a)
        ops.select(q, P, Kt, sl, w.k, ws=ws_s, idx=idx, count=cnt)
        ops.indexed_decode(q, K, V, idx, cnt, sl, w.scale, ws=ws_i, out=out_kv, lse=lse)

    def head_step(i):
        ops.append_lowrank(K, P, Kt, pos, 1, ws=ws_a)
        ops.select_heads(q, P, Kt, sl, w.k, ws=ws_sh, idx=idh, count=cnh)
        ops.indexed_decode_heads(q, K, V, idh, cnh, sl, w.scale, ws=ws_ih, out=out_q, lse=lse)

    res = {}
    for name, fn in (("per_kv_head_calls", kv_step), ("per_query_head_calls", head_step)):
        for i in range(3):
            fn(i)
        rep_fn = graphed(fn, dev, 1) if use_graph else fn
        for i in range(3):
            rep_fn(i)
        d = time_steps(rep_fn, steps, stream, flush_buf)
        med = max_over_ranks(percentile(d, 0.5), world)
        res[name] = {"steps_per_s": world / med, "ms_per_step": med * 1e3}
    torch.cuda.synchronize()
    # recall of the shared set against each query head's own top-k
    kv_sets = idx.repeat_interleave(G, 1)  # [B, Hq, k]
    hit = (idh.unsqueeze(-1) == kv_sets.unsqueeze(-2)).any(-1) & (idh >= 0)
    res["recall_of_per_kv_head_sets"] = float(hit.sum().item() / max(1, int((idh >= 0).sum().item())))
    od, _ = ops.dense_decode(q, K, V, sl, w.scale)
    torch.cuda.synchronize()
    res["mean_abs_err_vs_dense"] = {"per_kv_head": float((out_kv.float() - od.float()).abs().mean().item()),
                                    "per_query_head": float((out_q.float() - od.float()).abs().mean().item())}
    row = (w.d + w.Dv) * 2
    res["selected_bytes_per_step"] = {"per_kv_head": w.B * w.Hkv * min(w.k, w.T) * row,
                                      "per_query_head": w.B * w.Hq * min(w.k, w.T) * row}
    res["note"] = ("per-query-head selection reads G = %d times the selected rows; recall = share of each query "
                   "head's own top-k that its KV head's shared set contains" % G)
    return res


def run_jssa(args, world, rank, local):
    import torch

    from token_level_sparse_kv_b200 import ops
    from token_level_sparse_kv_b200.inputs import Workload, make_inputs, make_queries

    w0 = workload_of(args)
    w = Workload(**{**w0.__dict__, "seed": w0.seed + 1000 * rank})
    dev = torch.device("cuda", local)
    stream = torch.cuda.current_stream(dev)
    t_setup = time.perf_counter()
    q, K, V, P, sl = make_inputs(w, device=dev)
    qs = [q] + make_queries(w, 3, device=dev)
    Kt = ops.build_lowrank_cache(K, P)
    pos = (sl - 1).clamp_min(0).contiguous()
    dims = ops.make_dims(q, K, V, P=P, Kt=Kt)
    ws = ops.new_workspace(dims, w.k, ops.OP_DECODE_STEP, dev)
    launches, step_form = ops.plan_info(dims, w.k, ops.OP_DECODE_STEP)
    sel_form = ops.plan_info(dims, w.k, ops.OP_SELECT)[1]
    idx = torch.empty((w.B, w.Hkv, w.k), dtype=torch.int32, device=dev)
    cnt = torch.empty((w.B, w.Hkv), dtype=torch.int32, device=dev)
    out = torch.empty((w.B, w.Hq, w.Dv), dtype=q.dtype, device=dev)
    lse = torch.empty((w.B, w.Hq), dtype=torch.float32, device=dev)
    Vv = V
    torch.cuda.synchronize()
    log("rank %d: setup %.1f s" % (rank, time.perf_counter() - t_setup))

    def step(i):
        ops.decode_step(qs[i & 3], K, Vv, P, Kt, sl, pos, w.k, w.scale, ws=ws, idx=idx, count=cnt, out=out, lse=lse)

    for i in range(args.warmup):
        step(i)
    torch.cuda.synchronize()
    status = ops.device_status(ws)
    if status:
        raise RuntimeError("device status 0x%x after warm-up" % status)
    # the timed loop replays one CUDA graph per rotating query (the step's
    # launches without host planning), as a serving decode loop would
    graphs, launch_mode = None, "eager"
    if not args.eager:
        try:
            graphs = [ops.StepGraph(lambda j=j: step(j), dev) for j in range(4)]
            launch_mode = "cuda graph (one replay per step)"
        except Exception as e:  # capture unsupported: time the eager loop
            log("graph capture failed (%s); timing the eager loop" % e)
            graphs = None
    if graphs:
        def timed(i):
            graphs[i & 3].replay()

        for i in range(max(3, args.warmup)):
            timed(i)
        torch.cuda.synchronize()
    else:
        timed = step

    l2 = torch.cuda.get_device_properties(dev).L2_cache_size
    flush = flushes_l2(w, l2)
    flush_buf = torch.empty(2 * l2, dtype=torch.uint8, device=dev) if flush else None
    sampler = ClockSampler(local)
    with sampler:
        barrier(world)
        durs = time_steps(timed, args.steps, stream, flush_buf)
        barrier(world)
        secs = sum(durs)
        eager_steps = max(5, min(args.steps, 200))
        eager_secs = time_loop(step, eager_steps, stream) if graphs else None
        # dominant kernel alone: the fused score + top-k pass (jssa_select)
        ws_sel = ops.new_workspace(dims, w.k, ops.OP_SELECT, dev)
        sel_steps = max(args.steps, 20)

        def sel(i):
            ops.select(qs[i & 3], P, Kt, sl, w.k, ws=ws_sel, idx=idx, count=cnt)

        for i in range(3):
            sel(i)
        sel_secs = time_loop(sel, sel_steps, stream)
    clocks = sampler.summary()
    secs_max = max_over_ranks(secs, world)
    # steps/s = 1 / median step latency (the slowest rank's median), whole job
    med_max = max_over_ranks(percentile(durs, 0.5), world)
    ms = med_max * 1e3
    value = world / med_max
    value_mean = world * args.steps / secs_max

    peak, peak_kind = measured_peaks()
    step_bytes, kt_bytes = algorithmic_bytes(w)
    step_flops = 2 * w.B * w.Hq * min(w.k, w.T) * (w.d + w.Dv)  # q.k and p.v of the selected rows
    sel_s = sel_secs / sel_steps
    if launches == 1:
        # the step is one launch of the fused streaming kernel: it is the dominant kernel
        kname = "stream_select_kernel (fused decode step: append, projection, score, top-k, attention)"
        kbytes, k_s = step_bytes, secs_max / args.steps
        traffic = profile_traffic("jssa_stream.cu", "stream_step_%s.txt" % w.name)
    else:
        kname = "selection pass (jssa_select: %s)" % sel_form
        kbytes, k_s = select_bytes(w), sel_s
        traffic = None
    achieved = kbytes / k_s / 1e9

    line = {"metric": METRIC, "value": value, "unit": "steps/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "bf16", "data": "synthetic", "config": config_of(w, world, flush),
            "roofline": {"bound": "hbm", "kernel": kname,
                         "achieved": achieved, "peak": peak, "unit": "GB/s", "frac": achieved / peak,
                         "peak_kind": peak_kind + " (burst copy)", "traffic": traffic,
                         "algorithmic_bytes_per_launch": kbytes, "us_per_launch": k_s * 1e6},
            "select_alone": {"us_per_call": sel_s * 1e6, "algorithmic_bytes": select_bytes(w),
                             "achieved_gbs": select_bytes(w) / sel_s / 1e9, "form": sel_form},
            "step_hbm": {"algorithmic_bytes_per_step": step_bytes, "achieved_gbs": step_bytes / (ms / 1e3) / 1e9,
                         "frac_of_peak": step_bytes / (ms / 1e3) / 1e9 / peak, "peak_gbs": peak,
                         "attention_flops_per_step": step_flops},
            "latency": latency_summary(durs),
            "steps_per_s_mean": value_mean,
            "step_form": step_form,
            "launch": launch_mode,
            "eager_ms_per_step": (max_over_ranks(eager_secs, world) / eager_steps * 1e3) if graphs else ms,
            "gpu_launches": launches * args.steps}
    if clocks:
        line["clocks"] = clocks

    if not args.quick:
        # comparison paths from the same build, same inputs
        ws_d = ops.new_workspace(dims, 1, ops.OP_DENSE_DECODE, dev)
        ws_a = ops.new_workspace(dims, 1, ops.OP_APPEND, dev)
        ws_g = ops.new_workspace(dims, w.k, ops.OP_GATHER_THEN_DENSE, dev)
        ws_i = ops.new_workspace(dims, w.k, ops.OP_INDEXED_DECODE, dev)
        gbuf = torch.empty(ops.gather_buffer_bytes(dims, w.k), dtype=torch.uint8, device=dev)
        cmp_steps = max(5, min(args.steps, args.cmp_steps))

        def dense(i):
            ops.dense_decode(qs[i & 3], K, Vv, sl, w.scale, window=0, ws=ws_d, out=out, lse=lse)

        def local(i):  # the sliding-window layer of a hybrid global/local pair
            ops.dense_decode(qs[i & 3], K, Vv, sl, w.scale, window=w.window, ws=ws_d, out=out, lse=lse)

        def gather(i):
            ops.append_lowrank(K, P, Kt, pos, 1, ws=ws_a)
            ops.select(qs[i & 3], P, Kt, sl, w.k, ws=ws_sel, idx=idx, count=cnt)
            ops.gather_then_dense(qs[i & 3], K, Vv, idx, cnt, sl, w.scale, gather_buf=gbuf, ws=ws_g, out=out,
                                  lse=lse)

        def split(i):
            ops.append_lowrank(K, P, Kt, pos, 1, ws=ws_a)
            ops.select(qs[i & 3], P, Kt, sl, w.k, ws=ws_sel, idx=idx, count=cnt)
            ops.indexed_decode(qs[i & 3], K, Vv, idx, cnt, sl, w.scale, ws=ws_i, out=out, lse=lse)

        res = {}
        paths = [("dense_full_kv", dense), ("gather_then_dense", gather), ("split_calls_gather_free", split)]
        if w.window:
            paths.append(("local_window_layer", local))
        for name, fn in paths:
            for i in range(3):
                fn(i)
            rep_fn = graphed(fn, dev) if graphs else fn
            for i in range(3):
                rep_fn(i)
            # the window layer is small enough for the L2: flush it like a small step
            fb = flush_buf
            if fb is None and name == "local_window_layer":
                fb = torch.empty(2 * l2, dtype=torch.uint8, device=dev)
            d = time_steps(rep_fn, cmp_steps, stream, fb)
            med = max_over_ranks(percentile(d, 0.5), world)
            res[name] = {"steps_per_s": world / med, "ms_per_step": med * 1e3, "latency": latency_summary(d),
                         "launch": "cuda graph replay" if graphs else "eager"}
        if not w.latent:
            res["block_screening"] = screening_comparison(w, qs, K, Vv, P, Kt, sl, pos, dims, dev, stream, flush_buf,
                                                          cmp_steps, world, graphs is not None)
        if not w.latent and w.d <= 128:
            res["calibration_of_P"] = calibration_recall(w, q, K, P, sl, dev, stream)
        if not w.latent:
            res["per_query_head_selection"] = per_head_comparison(w, q, K, Vv, P, Kt, sl, pos, dims, dev, stream,
                                                                  flush_buf, cmp_steps, world, graphs is not None)
        res["speedup_vs_dense"] = value / res["dense_full_kv"]["steps_per_s"]
        res["speedup_vs_gather_then_dense"] = value / res["gather_then_dense"]["steps_per_s"]
        if w.window:
            res["local_window_layer"]["note"] = "dense sliding window %d over the same cache shape" % w.window
            pair_ms = ms + res["local_window_layer"]["ms_per_step"]
            res["hybrid_pair"] = {"steps_per_s": world * 1e3 / pair_ms, "ms_per_step": pair_ms,
                                  "note": "sparse global layer (the timed step) + dense sliding-window local layer"}
        line["comparison"] = res

    if not args.quick:
        # end to end through the C-ABI call with host buffers: every step copies
        # the packed [q | new K rows | new V rows] block from pinned host memory,
        # writes the new rows into the cache, runs the step and copies the
        # output back to pinned host memory; the host waits for it every step
        nbytes = ops.host_step_bytes(dims)
        g = torch.Generator().manual_seed(1234 + rank)
        hosts = []
        for j in range(4):
            kn = torch.randn((w.B, w.Hkv, w.d), generator=g).to(q.dtype)
            parts = [qs[j].cpu().reshape(-1), kn.reshape(-1)]
            if not w.latent:
                parts.append(torch.randn((w.B, w.Hkv, w.Dv), generator=g).to(q.dtype).reshape(-1))
            blob = torch.cat(parts).view(torch.uint8)
            hosts.append(torch.empty(nbytes, dtype=torch.uint8).pin_memory().copy_(blob))
        stage = torch.empty(nbytes, dtype=torch.uint8, device=dev)
        out_host = torch.empty(out.shape, dtype=out.dtype).pin_memory()
        e2e_steps = max(5, min(args.steps, args.e2e_steps))

        def host_step(i):
            ops.decode_step_host(hosts[i & 3], stage, K, Vv, P, Kt, sl, pos, w.k, w.scale, out_host, ws, idx, cnt,
                                 out, lse, dims=dims)
            stream.synchronize()  # the host reads the output every step

        for i in range(3):
            host_step(i)
        barrier(world)
        t0 = time.perf_counter()
        for i in range(e2e_steps):
            host_step(i)
        te = max_over_ranks(time.perf_counter() - t0, world)
        line["e2e"] = {"value": world * e2e_steps / te, "unit": "steps/s", "h2d_bytes_per_step": nbytes,
                       "d2h_bytes_per_step": out_host.numel() * out_host.element_size(),
                       "api": "jssa_decode_step_host (C ABI; pinned host in/out, one stream sync per step)"}

    if not args.quick and world == 1:
        line["decode_loop"] = measure_decode_loop(dev, 32, 20, stream)

    if rank == 0 and not args.no_cpu:
        v, desc, thr = oracle_baseline(w0, args.cpu_seconds, max(1, min(w0.B, args.cpu_rows)), os.cpu_count() or 1)
        line["cpu_baseline"] = {"value": v, "unit": "steps/s", "cores": thr, "kind": "oracle", "sample": desc}
    if status := ops.device_status(ws):
        raise RuntimeError("device status 0x%x after the timed region" % status)
    if rank == 0:
        print(json.dumps(line), flush=True)
    return 0


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", default="jssa", choices=["jssa", "reference"])
    ap.add_argument("--workload", default="gqa_128k_b16")
    ap.add_argument("--batch", type=int, default=None, help="override the workload's batch size (sweeps)")
    ap.add_argument("--topk", type=int, default=None, help="override the workload's k (sweeps)")
    ap.add_argument("--cmp-steps", type=int, default=200)
    ap.add_argument("--e2e-steps", type=int, default=500)
    ap.add_argument("--cpu-rows", type=int, default=2, help="batch rows in the oracle's timed sample")
    ap.add_argument("--cpu-seconds", type=float, default=10.0, help="host seconds of oracle work to time")
    ap.add_argument("--quick", action="store_true", help="skip the comparison and end-to-end passes")
    ap.add_argument("--eager", action="store_true", help="time the eager call loop instead of CUDA graph replays")
    ap.add_argument("--no-cpu", action="store_true", help="skip the CPU oracle baseline")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3
    world, rank, local = setup_dist(args)
    try:
        if args.impl == "reference":
            return run_reference(args, world, rank)
        return run_jssa(args, world, rank, local)
    finally:
        if world > 1:
            import torch.distributed as dist

            dist.destroy_process_group()


if __name__ == "__main__":
    sys.exit(main())
