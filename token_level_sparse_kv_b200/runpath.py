"""Run one call of the library repeatedly on a synthetic workload.

    python -m token_level_sparse_kv_b200.runpath --workload gqa_32k_b4 --path dense --iters 3

Draws the workload's seeded inputs on cuda:0, builds the low-rank cache,
selects once, then runs `--path` `--iters` times and prints each call's
device time (CUDA events on the launching stream).  It exists so that a
profiler can capture one path of the decode step in isolation (e.g. ncu with
`-k` and `-c` on the kernel of interest) without the rest of the benchmark.

Paths: step (jssa_decode_step), select, score, topk (over a score array),
append (one new row), indexed (jssa_indexed_decode on the selection), dense
(full KV), window (dense over the workload's sliding window, or --window),
gather (jssa_gather_then_dense).
"""
from __future__ import annotations

import argparse
import sys

import torch

from . import ops
from .inputs import WORKLOADS, Workload, make_inputs


def main(argv=None) -> int:
    ap = argparse.ArgumentParser()
    ap.add_argument("--workload", default="gqa_32k_b4", choices=sorted(WORKLOADS))
    ap.add_argument("--path", default="step",
                    choices=["step", "select", "score", "topk", "append", "indexed", "dense", "window", "gather"])
    ap.add_argument("--iters", type=int, default=3)
    ap.add_argument("--batch", type=int, default=None)
    ap.add_argument("--topk", type=int, default=None)
    ap.add_argument("--window", type=int, default=None)
    ap.add_argument("--form", default="auto", choices=sorted(ops.FORMS))
    ap.add_argument("--unfused", action="store_true")
    args = ap.parse_args(argv)

    w = WORKLOADS[args.workload]
    over = {}
    if args.batch is not None:
        over["B"] = args.batch
    if args.topk is not None:
        over["k"] = args.topk
    if over:
        w = Workload(**{**w.__dict__, **over})
    dev = torch.device("cuda", 0)
    q, K, V, P, sl = make_inputs(w, device=dev)
    Kt = ops.build_lowrank_cache(K, P)
    pos = (sl - 1).clamp_min(0).contiguous()
    dims = ops.make_dims(q, K, V, P=P, Kt=Kt)
    idx, cnt = ops.select(q, P, Kt, sl, w.k, form=args.form)
    out = torch.empty((w.B, w.Hq, w.Dv), dtype=q.dtype, device=dev)
    lse = torch.empty((w.B, w.Hq), dtype=torch.float32, device=dev)
    window = w.window if args.window is None else args.window
    scores = ops.score(q, P, Kt, sl) if args.path == "topk" else None
    gbuf = (torch.empty(ops.gather_buffer_bytes(dims, w.k), dtype=torch.uint8, device=dev)
            if args.path == "gather" else None)
    op = {"step": ops.OP_DECODE_STEP, "select": ops.OP_SELECT, "score": ops.OP_SCORE, "topk": ops.OP_TOPK,
          "append": ops.OP_APPEND, "indexed": ops.OP_INDEXED_DECODE, "dense": ops.OP_DENSE_DECODE,
          "window": ops.OP_DENSE_DECODE, "gather": ops.OP_GATHER_THEN_DENSE}[args.path]
    ws = ops.new_workspace(dims, w.k, op, dev)

    def call():
        if args.path == "step":
            ops.decode_step(q, K, V, P, Kt, sl, pos, w.k, w.scale, ws=ws, idx=idx, count=cnt, out=out, lse=lse,
                            form=args.form, unfused=args.unfused)
        elif args.path == "select":
            ops.select(q, P, Kt, sl, w.k, ws=ws, idx=idx, count=cnt, form=args.form)
        elif args.path == "score":
            ops.score(q, P, Kt, sl, ws=ws)
        elif args.path == "topk":
            ops.topk(scores, sl, w.k, Hq=w.Hq, d=w.d, ws=ws, form=args.form)
        elif args.path == "append":
            ops.append_lowrank(K, P, Kt, pos, 1, ws=ws)
        elif args.path == "indexed":
            ops.indexed_decode(q, K, V, idx, cnt, sl, w.scale, ws=ws, out=out, lse=lse)
        elif args.path in ("dense", "window"):
            ops.dense_decode(q, K, V, sl, w.scale, window=window if args.path == "window" else 0, ws=ws, out=out,
                             lse=lse)
        else:
            ops.gather_then_dense(q, K, V, idx, cnt, sl, w.scale, gather_buf=gbuf, ws=ws, out=out, lse=lse)

    stream = torch.cuda.current_stream(dev)
    for i in range(args.iters):
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        call()
        b.record(stream)
        torch.cuda.synchronize()
        print("%s %s iter %d: %.1f us" % (w.name, args.path, i, a.elapsed_time(b) * 1e3))
    status = ops.device_status(ws)
    if status:
        print("device status 0x%x" % status, file=sys.stderr)
        return 1
    return 0


if __name__ == "__main__":
    sys.exit(main())
