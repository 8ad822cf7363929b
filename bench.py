#!/usr/bin/env python
"""Benchmark of the block-sparse attention path (stage 1 plan + stage 2 forward).

One step = sparse_attn_plan + sparse_attn_fwd over one batch of resident bf16
Q/K/V of the chosen workload (default: the largest configured shape, the
HunyuanVideo-13B-shaped layer B=1 H=24 N=118,800 d=128 with centroid weight 1.5,
tau=0.95, lambda=-12). Prints ONE JSON line on rank 0.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload hunyuan|wan|lm|small|tiny]
                    [--tau T] [--lam L|off] [--recall R] [--impl ours|reference]

On rank 0 of a one-GPU run the line also carries the CPU oracle's timing
(cpu_baseline) and, from the same oracle runs, the parity of the timed
configuration (parity): mask rows differing from the oracle's plan and the
blocks the 1e-4 tau band excuses, the output error against the oracle run on
the GPU's mask and filter decisions, and the sparse-vs-dense error.

Multi-GPU: the path has no exchange step; N ranks run N independent replicas of
the same workload (weak scaling), timed on the device, max over ranks.
"""
from __future__ import annotations

import argparse
import dataclasses
import json
import math
import os
import statistics
import subprocess
import sys
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

from free_block_sparse_mean_b200 import workloads as wl  # noqa: E402

METRIC = "sparse attn ms/call & dense-equiv TFLOPS at τ; sparsity %; % of BF16 peak"
UNIT = "TFLOP/s dense-equivalent"
L2_BYTES = 126 * 1024 * 1024
FLUSH_BYTES = 512 * 1024 * 1024
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default="hunyuan", choices=sorted(wl.WORKLOADS))
    ap.add_argument("--tau", type=float, default=0.95)
    ap.add_argument("--lam", default="-12")
    ap.add_argument("--centroid-weight", type=float, default=None)
    ap.add_argument("--seed", type=int, default=0)
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=12.0)
    ap.add_argument("--heads", type=int, default=None,
                    help="run only the first H heads of the workload (profiling captures)")
    ap.add_argument("--no-dense", action="store_true", help="skip the dense (full-mask) reference timing")
    ap.add_argument("--sweep", action="store_true",
                    help="one JSON line per configured (workload, tau, lambda, centroid weight); kernel timing only")
    ap.add_argument("--qk", default="bf16", choices=["bf16", "fp8", "int8"],
                    help="score operands: bf16 Q and K, or their per-block FP8 E4M3 or INT8 codes "
                         "(P.V stays bf16)")
    ap.add_argument("--recall", type=float, default=None,
                    help="P.V filter: the cumulative-energy test keeping this recall per row "
                         "(sparse_attn_fwd_recall) instead of the lambda test")
    ap.add_argument("--cluster-iters", type=int, default=None,
                    help="reorder the tokens by interaction clustering (this many k-means iterations) "
                         "before the plan, and the output back after the forward (non-causal workloads)")
    ap.add_argument("--no-graph", action="store_true",
                    help="launch plan and forward directly instead of replaying CUDA graphs")
    return ap.parse_args()


def lam_value(s):
    return None if s in ("off", "none", "None", "-inf") else float(s)


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return FALLBACK_PEAKS, "fallback"


def measured_traffic(w, tau, lam, qk="bf16", recall=None, centroid_weight=None):
    """DRAM bytes per launch of the forward kernel from the committed ncu capture,
    or None if the kernel source changed since (or the workload differs: for the
    video workloads the key names the centroid weight, which sets the sparsity)."""
    import hashlib
    p = os.path.join(ROOT, "profiles", "fwd_kernel_traffic.json")
    if not os.path.exists(p):
        return None
    with open(p) as f:
        d = json.load(f)
    h = hashlib.sha256()
    for src in d.get("sources", []):
        with open(os.path.join(ROOT, src), "rb") as f:
            h.update(f.read())
    if h.hexdigest() != d.get("source_sha256"):
        return None
    key = f"{w.name}: B={w.B} H={w.H} N={w.N} d={w.D} tau={tau:g} lambda={lam if lam is not None else 'off'}"
    key = key.replace("lambda=-12.0", "lambda=-12") + ("" if qk == "bf16" else f" qk={qk}")
    if recall is not None:
        key = key.split(" lambda=")[0] + f" recall={recall:g}"
    if w.kind == "video":
        cw = w.centroid_weight if centroid_weight is None else centroid_weight
        key += f" centroid_weight={cw:g}"
    ent = d.get("traffic_bytes_per_launch", {}).get(key)
    return None if ent is None else float(ent["total"])


def plan_batches(BH, Nb):
    """Strip batches of one plan call: the pooled scores are computed and selected in
    strips of 128 query blocks, as many per batch as fit in 64 MiB (at least one),
    as the library lays out its workspace."""
    strips = BH * ((Nb + 127) // 128)
    strip_bytes = 128 * ((Nb + 31) // 32 * 32) * 4
    per = max(1, min(strips, (64 << 20) // strip_bytes))
    return (strips + per - 1) // per


def dense_flops(w):
    if w.causal:
        return 2.0 * w.B * w.H * w.N * (w.N + 1) * w.D
    return 4.0 * w.B * w.H * w.N * w.N * w.D


# --------------------------------------------------------------------------- dist
def dist_setup(args):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    pg = None
    if world > 1:
        import torch.distributed as dist
        from datetime import timedelta
        backend = "nccl" if torch.cuda.is_available() else "gloo"
        if backend == "nccl":
            torch.cuda.set_device(local)
        dist.init_process_group(backend, timeout=timedelta(seconds=120))
        pg = dist
    return world, rank, local, pg


def reduce_max(pg, x: float, device) -> float:
    if pg is None:
        return x
    t = torch.tensor([x], dtype=torch.float64, device=device)
    pg.all_reduce(t, op=pg.ReduceOp.MAX)
    return float(t.item())


def barrier(pg, device=None):
    if pg is not None:
        if device is not None and device.type == "cuda":
            pg.barrier(device_ids=[device.index])
        else:
            pg.barrier()


# --------------------------------------------------------------------------- clocks
class ClockSampler:
    """nvidia-smi sampling of SM clocks and throttle reasons during the timed region."""
    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.proc = None
        self.path = os.path.join("/tmp", f"sa_clocks_{os.getpid()}.csv")

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.index), f"--query-gpu={self.Q}", "--format=csv,noheader,nounits",
                 "-lms", "200"], stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        time.sleep(0.25)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        rows = []
        try:
            for line in open(self.path):
                parts = [p.strip() for p in line.split(",")]
                if len(parts) >= 9:
                    rows.append(parts)
            os.remove(self.path)
        except Exception:
            return None
        if not rows:
            return None
        sm = [float(r[1]) for r in rows if r[1].replace(".", "").isdigit()]
        smax = max(float(r[2]) for r in rows)
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if r[5 + i].lower() == "active"})
        loaded = [x for x in sm if x > 0.5 * smax] or sm
        return {"sm_mhz": statistics.median(loaded), "sm_max_mhz": smax, "reasons": reasons,
                "samples": len(rows)}


# --------------------------------------------------------------------------- CPU oracle leg
def oracle_qblocks(w):
    """The query blocks the oracle's forward covers per head: all of them for
    short heads, else 16 spread over the head (the first and the last included)."""
    nb = -(-w.N // 64)
    if w.N <= 8192:
        return None
    step = max(1, nb // 15)
    return sorted(set(list(range(0, nb, step))[:15]) | {nb - 1})


def time_oracle(w, tau, lam, budget_s, seed, recall=None, cluster_iters=None, gpu=None):
    """The oracle as it stands (fp64 NumPy, host cores) on a bounded sample of the
    workload: whole heads of plan + forward (the forward on oracle_qblocks for long
    heads) until the time budget is used, at least one head.

    gpu, if given, holds host copies of the timed configuration's device tensors
    (q, k, v, out, mask, dec: inputs, output, mask and recorded filter decisions)
    by head; the oracle then runs on those exact inputs, its forward on the GPU's
    mask replaying the GPU's decisions, and the same runs give the parity fields
    (returned as a dict, else None): the GPU mask against the oracle's plan (exact
    outside the 1e-4 tau band), the GPU output against the oracle's, and the
    sparse-vs-dense error (the oracle with every block kept, on up to 4 of the
    sampled query blocks; not timed)."""
    from oracle import sparse_attn_oracle as orc
    try:
        import threadpoolctl
        cores = max(v.get("num_threads", 1) for v in threadpoolctl.threadpool_info()) or os.cpu_count()
    except Exception:
        cores = os.cpu_count()
    per_head_dense = dense_flops(w) / (w.B * w.H)
    nb = -(-w.N // 64)
    qblocks = oracle_qblocks(w)
    t_total = 0.0
    flops = 0.0
    heads = 0
    par = None
    if gpu is not None:
        from tests.helpers import BAND, compare_masks, output_errors
        par = {"heads": [], "mask_rows": 0, "mask_rows_differing": 0, "excused_blocks": 0, "max_abs": 0.0,
               "rel_fro": 0.0, "dense_max_abs": 0.0, "dense_rel_fro": 0.0, "band": BAND,
               "qblocks_per_head": nb if qblocks is None else len(qblocks)}
    for h in range(w.H):
        if gpu is not None:
            q, k, v = gpu["q"][:, h:h + 1], gpu["k"][:, h:h + 1], gpu["v"][:, h:h + 1]
        else:
            q, k, v = wl.generate(w, seed=seed, device="cpu", heads=[h])
        t0 = time.perf_counter()
        if cluster_iters is not None:      # clustering, plan and forward of whole heads
            orc.clustered_attention(q, k, v, tau, lam, cluster_iters)
            t_total += time.perf_counter() - t0
            flops += per_head_dense
            heads += 1
            if t_total >= budget_s:
                break
            continue
        p = orc.plan(q, k, tau, None, w.causal)
        mask = p["mask"] if gpu is None else gpu["mask"][:, h:h + 1]
        forced = None if gpu is None else gpu["dec"][:, h:h + 1]
        if recall is not None:
            ref = orc.attention_recall(q, k, v, mask, recall, None, w.causal, qblocks=qblocks, forced=forced)
        else:
            ref = orc.fwd(q, k, v, mask, lam, None, w.causal, qblocks=qblocks, forced=forced)
        dt = time.perf_counter() - t0
        t_total += dt
        frac = 1.0 if qblocks is None else len(qblocks) / nb
        # attention part scales with the sampled query blocks; plan is whole-head
        flops += per_head_dense * frac
        heads += 1
        if par is not None:
            rows, exc = compare_masks(mask, p, tau)
            got = gpu["out"][:, h:h + 1].float().numpy()
            ma, rel = output_errors(got, ref)
            dq = (qblocks or list(range(nb)))
            dq = [dq[i] for i in np.linspace(0, len(dq) - 1, min(4, len(dq))).round().astype(int)]
            dense = orc.attention_masked(q, k, v, np.ones_like(mask), None, w.causal, qblocks=dq)
            dma, drel = output_errors(got, dense)
            par["heads"].append(h)
            par["mask_rows"] += nb
            par["mask_rows_differing"] += rows
            par["excused_blocks"] += exc
            par["max_abs"] = max(par["max_abs"], ma)
            par["rel_fro"] = max(par["rel_fro"], rel)
            par["dense_max_abs"] = max(par["dense_max_abs"], dma)
            par["dense_rel_fro"] = max(par["dense_rel_fro"], drel)
        if t_total >= budget_s:
            break
    if cluster_iters is not None:
        return flops / t_total / 1e12, t_total, cores, f"{heads} of {w.H} heads, clustering + plan + forward", None
    sample = (f"{heads} of {w.H} heads, full plan"
              + ("" if qblocks is None else f", forward on {len(qblocks)} of {nb} query blocks"))
    if par is not None:
        par["tolerance"] = {"max_abs": 2e-2, "rel_fro": 1e-2}
        par["within_tolerance"] = par["max_abs"] <= 2e-2 and par["rel_fro"] <= 1e-2
        par["note"] = ("per sampled head: mask against the oracle's plan; output against the oracle on the "
                       "GPU's mask replaying its filter decisions (worst head); sparse-vs-dense: oracle with "
                       "every block kept on up to 4 sampled query blocks")
    return flops / t_total / 1e12, t_total, cores, sample, par


# --------------------------------------------------------------------------- main arms
def run_reference(args, w, world, rank, pg):
    lam = lam_value(args.lam)
    if rank != 0:
        return
    per_step = []
    vals = []
    budget = max(2.0, min(args.cpu_seconds, 240.0 / max(1, args.steps + args.warmup)))
    for i in range(args.warmup + args.steps):
        v, t, cores, sample, _ = time_oracle(w, args.tau, lam, budget, args.seed, args.recall, args.cluster_iters)
        if i >= args.warmup:
            per_step.append(t)
            vals.append(v)
    value = statistics.median(vals)
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * statistics.median(per_step),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic", "config": config_dict(w, args, world),
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": cores, "kind": "oracle", "sample": sample},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
        "gpu_launches": 0,
    }
    print(json.dumps(line), flush=True)


def config_dict(w, args, world):
    return {"workload": f"{w.name}: B={w.B} H={w.H} N={w.N} d={w.D} block=64 "
                        f"{'causal' if w.causal else 'non-causal'}",
            "tau": args.tau, "lambda": None if getattr(args, "recall", None) is not None else lam_value(args.lam),
            "pv_filter": "recall" if getattr(args, "recall", None) is not None else "lambda",
            "recall": getattr(args, "recall", None), "seq_len": w.N, "heads": w.H, "head_dim": w.D,
            "qk": getattr(args, "qk", "bf16"),
            "cluster_iters": getattr(args, "cluster_iters", None),
            "global_batch": w.B * world, "parallelism": f"replicas{world}",
            "l2": "flushed between timed steps" if 3 * w.B * w.H * w.N * w.D * 2 < 2 * L2_BYTES
            else "inputs larger than L2 (flushed too)",
            "centroid_weight": args.centroid_weight if args.centroid_weight is not None
            else (w.centroid_weight if w.kind == "video" else None)}


def check_device(sa, where):
    """A bounded wait that ran out or a range check makes every number void."""
    code = sa.sparse_attn_device_error()
    if code:
        raise RuntimeError(f"device-side check fired during {where}: error word {code}")


def run_ours(args, w, world, rank, local, pg):
    import free_block_sparse_mean_b200 as sa
    if not torch.cuda.is_available():
        raise RuntimeError("no CUDA device: the benchmark needs a B200")
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    rec = args.recall
    lam = None if rec is not None else lam_value(args.lam)   # the recall test replaces lambda
    q, k, v = wl.generate(w, seed=args.seed, device=dev, centroid_weight=args.centroid_weight)
    torch.cuda.synchronize()
    B, H, N, D = w.B, w.H, w.N, w.D
    Nb = -(-N // 64)
    # buffers reused by every step (resident, allocated once)
    q8 = args.qk in ("fp8", "int8")
    i8 = args.qk == "int8"
    if q8 and rec is not None:
        raise SystemExit("--recall runs on bf16 scores: drop --qk")
    cl = args.cluster_iters
    if cl is not None and (q8 or w.causal):
        raise SystemExit("--cluster-iters needs bf16 scores and a non-causal workload")
    plan = sa.sparse_attn_plan(q, k, args.tau, None, w.causal, with_idx=False, quantize=args.qk if q8 else False)
    ws = torch.empty(sa.sparse_attn_plan_workspace_size(B, H, N, D), dtype=torch.uint8, device=dev)
    out = torch.empty_like(q)
    flush = torch.empty(FLUSH_BYTES // 4, dtype=torch.float32, device=dev)
    stream = torch.cuda.current_stream(dev)

    if cl is not None:
        # the clustered path: both orders, the reordered q, k, v, then the plan on them;
        # the forward on the reordered tensors and its rows put back in token order
        ws_c = torch.empty(sa.sparse_attn_cluster_workspace_size(B, H, N, D), dtype=torch.uint8, device=dev)
        cq = sa.Clustering(perm=torch.empty((B, H, N), dtype=torch.int32, device=dev))
        ck = sa.Clustering(perm=torch.empty((B, H, N), dtype=torch.int32, device=dev))
        qs, ks, vs, os_ = (torch.empty_like(q) for _ in range(4))

        def run_plan():
            sa.sparse_attn_cluster(q, k, cl, out=cq, workspace=ws_c)
            sa.sparse_attn_cluster(k, q, cl, out=ck, workspace=ws_c)
            sa.sparse_attn_permute_rows(q, cq.perm, out=qs)
            sa.sparse_attn_permute_rows(k, ck.perm, out=ks)
            sa.sparse_attn_permute_rows(v, ck.perm, out=vs)
            sa.sparse_attn_plan(qs, ks, args.tau, None, False, out=plan, workspace=ws, with_idx=False)

        def run_fwd(stats=None):
            sa.sparse_attn_fwd(qs, ks, vs, plan, lam, out=os_, stats=stats, recall=rec)
            sa.sparse_attn_permute_rows(os_, cq.perm, inverse=True, out=out)
        # kernels per step: per clustering 4, then 8 per iteration less the last
        # iteration's centroid pass (with none, the 4 kernels of the order), 3 row moves,
        # the plan (pool, a score and a selection kernel per strip batch, the pairing),
        # the forward, the move back
        plan_launches = 2 + 2 * plan_batches(w.B * w.H, -(-w.N // 64))
        launches_per_step = 2 * (4 + (8 * cl - 1 if cl > 0 else 4)) + 3 + plan_launches + 1 + 1
    else:
        def run_plan():
            sa.sparse_attn_plan(q, k, args.tau, None, w.causal, out=plan, workspace=ws, with_idx=False,
                                quantize=args.qk if q8 else False)

        def run_fwd(stats=None):
            sa.sparse_attn_fwd(q, k, v, plan, lam, out=out, stats=stats, qk_fp8=q8 and not i8, qk_int8=i8,
                               recall=rec)
        # the plan (pool, a score and a selection kernel per strip batch, the pairing)
        # and the forward
        launches_per_step = 2 + 2 * plan_batches(w.B * w.H, -(-w.N // 64)) + 1

    def step():
        run_plan()
        run_fwd()

    # stats (outside timing): kept pairs, skipped P.V, union tiles, algorithmic FLOPs
    # of the forward; on the bf16 path the same launch also records the filter's
    # decisions for the parity check of the oracle leg
    stats = torch.zeros(4, dtype=torch.int64, device=dev)
    run_plan()
    dec = None
    if not q8 and cl is None:
        dec = torch.zeros((B, H, Nb, Nb), dtype=torch.uint8, device=dev)
        sa.sparse_attn_fwd(q, k, v, plan, lam, out=out, stats=stats, recall=rec, decisions=dec)
    else:
        run_fwd(stats)
    torch.cuda.synchronize()
    check_device(sa, "the stats pass")
    st = [int(x) for x in stats.cpu()]
    n_tok = torch.full((Nb,), 64, dtype=torch.float64, device=dev)
    n_tok[-1] = N - 64 * (Nb - 1)
    m = plan.mask.to(torch.float64)
    if w.causal:
        m = m * torch.tril(torch.ones(Nb, Nb, dtype=torch.float64, device=dev))
    pair_tokens = float(torch.einsum("bhij,i,j->", m, n_tok, n_tok))   # sum over kept pairs n_i n_j
    kept_pairs = float(m.sum())
    total_pairs = B * H * (Nb * (Nb + 1) / 2 if w.causal else Nb * Nb)
    skipped = st[1]
    avg_pair_tokens = pair_tokens / max(kept_pairs, 1)
    exec_flops = 2.0 * D * pair_tokens + 2.0 * D * avg_pair_tokens * (kept_pairs - skipped)
    dflops = dense_flops(w)

    # dense reference time of our own kernel (full mask), for the predictor budget
    dense_ms = None
    if not args.no_dense:
        full = torch.ones((B, H, Nb, Nb), dtype=torch.uint8, device=dev)
        if q8:   # the same score operands, every block kept
            full = dataclasses.replace(plan, mask=full, work=None)
        for _ in range(2):
            sa.sparse_attn_fwd(q, k, v, full, None, out=out, causal=w.causal, qk_fp8=q8 and not i8, qk_int8=i8)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        flush.zero_()
        e0.record(stream)
        sa.sparse_attn_fwd(q, k, v, full, None, out=out, causal=w.causal, qk_fp8=q8 and not i8, qk_int8=i8)
        e1.record(stream)
        torch.cuda.synchronize()
        dense_ms = e0.elapsed_time(e1)
        check_device(sa, "the dense (full-mask) reference")
        del full

    for _ in range(args.warmup):
        flush.zero_()
        step()
    torch.cuda.synchronize()
    if not args.no_graph:
        # Each stage is one CUDA graph (its kernels only), so the timed steps replay
        # two launches instead of paying host launch overhead per kernel.
        g_plan, g_fwd = torch.cuda.CUDAGraph(), torch.cuda.CUDAGraph()
        with torch.cuda.graph(g_plan):
            run_plan()
        with torch.cuda.graph(g_fwd):
            run_fwd()
        g_plan.replay()
        g_fwd.replay()
        torch.cuda.synchronize()
        run_plan, run_fwd = g_plan.replay, g_fwd.replay
        stream = torch.cuda.current_stream(dev)
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True),
           torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    sampler = ClockSampler(local)
    barrier(pg, dev)
    torch.cuda.synchronize()
    sampler.start()
    time.sleep(0.3)
    for i in range(args.steps):
        flush.zero_()                       # L2 flush, outside the timed events
        a, b, c = ev[i]
        a.record(stream)
        run_plan()
        b.record(stream)
        run_fwd()
        c.record(stream)
    torch.cuda.synchronize()
    barrier(pg, dev)
    clocks = sampler.stop()
    check_device(sa, "the timed steps")
    plan_ms = [a.elapsed_time(b) for a, b, _ in ev]
    fwd_ms = [b.elapsed_time(c) for _, b, c in ev]
    step_ms_local = sum(p + f for p, f in zip(plan_ms, fwd_ms)) / args.steps
    step_ms = reduce_max(pg, step_ms_local, dev)
    value = world * dflops / (step_ms * 1e-3) / 1e12
    fwd_avg = statistics.mean(fwd_ms)
    plan_avg = statistics.mean(plan_ms)

    # end to end through the public API from pinned host buffers
    e2e = None
    if not args.no_e2e and cl is None:
        qh, kh, vh = (x.cpu().pin_memory() for x in (q, k, v))
        # warm-up calls exactly like the timed ones, so that the caching pinned
        # allocator holds the output blocks the timed calls cycle through
        for _ in range(max(3, args.warmup)):
            o_host = sa.sparse_attention(qh, kh, vh, args.tau, lam, None, w.causal, device=dev,
                                         qk_fp8=q8 and not i8, qk_int8=i8, recall=rec)
            torch.cuda.synchronize()
        barrier(pg, dev)
        t = []
        for _ in range(max(3, min(args.steps, 20))):
            flush.zero_()
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(stream)
            o_host = sa.sparse_attention(qh, kh, vh, args.tau, lam, None, w.causal, device=dev,
                                         qk_fp8=q8 and not i8, qk_int8=i8, recall=rec)
            b.record(stream)
            torch.cuda.synchronize()
            t.append(a.elapsed_time(b))
        check_device(sa, "the end-to-end calls")
        e2e_ms = reduce_max(pg, statistics.mean(t), dev)
        e2e = {"value": world * dflops / (e2e_ms * 1e-3) / 1e12, "unit": UNIT,
               "ms_per_call": e2e_ms, "median_ms_per_call": statistics.median(t), "calls": len(t),
               "h2d_bytes_per_step": 3 * q.numel() * 2, "d2h_bytes_per_step": o_host.numel() * 2}
        del qh, kh, vh

    pk, pk_kind = peaks()
    peak_t = float(pk["bf16_tflops"])
    peak_source = f"{pk_kind} bf16_tflops (burst)"
    if q8:
        # QK^T on FP8 / INT8 at twice the bf16 peak (the nominal 8-bit : bf16 ratio), P.V at the
        # bf16 peak: the peak of this mix is the FLOPs over the time each part needs
        s_flops = 2.0 * D * pair_tokens
        peak_t = exec_flops / (s_flops / (2.0 * peak_t) + (exec_flops - s_flops) / peak_t)
        peak_source = (f"{pk_kind} bf16_tflops (burst) for P.V, x2 (nominal {args.qk}:bf16) for QK^T, "
                       "combined over the executed FLOPs")
    achieved = exec_flops / (fwd_avg * 1e-3) / 1e12
    # predictor: compulsory bytes (Q and K read once; mask and counts written; with
    # FP8 scores also the codes and scales) over the plan time, against the HBM copy peak
    pred_bytes = 2.0 * B * H * N * D * 2 + B * H * Nb * Nb + 4.0 * B * H * Nb
    if q8:
        pred_bytes += 2.0 * B * H * N * D + 8.0 * B * H * Nb
    hbm = float(pk.get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"]))
    pred_gbs = pred_bytes / (plan_avg * 1e-3) / 1e9
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": step_ms, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": (f"{'int8' if i8 else 'fp8 e4m3'} QK^T, bf16 P.V") if q8 else "bf16",
        "data": "synthetic (seeded cluster-centroid generator)",
        "config": config_dict(w, args, world),
        "plan_ms": plan_avg, "fwd_ms": fwd_avg, "dense_fwd_ms": dense_ms,
        "sparsity_pct": 100.0 * (1.0 - kept_pairs / total_pairs),
        "lambda_skip_pct" if rec is None else "recall_skip_pct": 100.0 * skipped / max(kept_pairs, 1),
        "executed_tflops": achieved, "pct_of_bf16_peak_executed": 100.0 * achieved / peak_t,
        "predictor_pct_of_dense": None if dense_ms is None else 100.0 * plan_avg / dense_ms,
        "predictor": {"bound": "hbm", "achieved": pred_gbs, "peak": hbm, "unit": "GB/s", "frac": pred_gbs / hbm,
                      "bytes": pred_bytes, "peak_source": f"{pk_kind} hbm_gbs"},
        "roofline": {"bound": "tensor", "achieved": achieved, "peak": peak_t, "unit": "TFLOP/s",
                     "frac": achieved / peak_t, "traffic": None if cl is not None else measured_traffic(w, args.tau, lam, args.qk, rec, args.centroid_weight),
                     "kernel": (f"fwd_kernel<{D}, int8 scores> (sparse_attn_fwd_i8)" if i8
                                else f"fwd_kernel<{D}, fp8 scores> (sparse_attn_fwd_q8)") if q8
                     else (f"fwd_kernel<{D}, recall filter> (sparse_attn_fwd_recall)" if rec is not None
                           else f"fwd_kernel<{D}> (sparse_attn_fwd)"),
                     "peak_source": peak_source},
        "e2e": e2e, "gpu_launches": launches_per_step * args.steps, "cuda_graphs": not args.no_graph, "clocks": clocks,
    }
    line["union"] = {"score_tiles": st[2], "pv_tiles": st[3], "kept_pairs": kept_pairs,
                     "waste_pct": 100.0 * (st[2] - kept_pairs / 2) / max(kept_pairs / 2, 1),
                     "note": "128x64 score tiles computed (one per union entry of a 128-row tile) against "
                             "kept pairs / 2, the count with no union waste"}
    if rank == 0 and world == 1 and not args.no_cpu:
        gpu = None
        if dec is not None:
            # the timed configuration's inputs, output (of the last timed step), mask and
            # recorded decisions, copied to the host for the oracle leg
            gpu = {"q": q.cpu(), "k": k.cpu(), "v": v.cpu(), "out": out.cpu(),
                   "mask": plan.mask.cpu().numpy(), "dec": dec.cpu().numpy()}
        v_cpu, t_cpu, cores, sample, par = time_oracle(w, args.tau, lam, args.cpu_seconds, args.seed, rec, cl,
                                                        gpu=gpu)
        line["cpu_baseline"] = {"value": v_cpu, "unit": UNIT, "cores": cores, "kind": "oracle",
                                "sample": sample, "seconds": t_cpu}
        line["parity"] = par
    if rank == 0:
        print(json.dumps(line), flush=True)


def sweep(args):
    """Every configured point of every workload (one GPU, kernel timing only)."""
    base = dict(vars(args))
    for name, w in wl.WORKLOADS.items():
        if args.qk != "bf16" and w.D != 128:
            continue                                  # 8-bit scores are for d = 128
        cws = w.centroid_weights or (None,)
        for tau in w.taus:
            for lam in w.lams:
                for cw in cws:
                    a = argparse.Namespace(**base)
                    a.workload, a.tau, a.lam, a.centroid_weight = name, tau, "off" if lam is None else str(lam), cw
                    a.no_e2e, a.no_cpu, a.steps, a.warmup = True, True, min(args.steps, 5), 3
                    run_ours(a, w, 1, 0, 0, None)
                    torch.cuda.empty_cache()


def main():
    args = parse()
    if args.sweep:
        sweep(args)
        return
    w = wl.WORKLOADS[args.workload]
    if args.heads:
        w = w.with_(H=min(args.heads, w.H))
    world, rank, local, pg = dist_setup(args)
    try:
        if args.impl == "reference":
            run_reference(args, w, world, rank, pg)
        else:
            run_ours(args, w, world, rank, local, pg)
    finally:
        if pg is not None:
            pg.destroy_process_group()


if __name__ == "__main__":
    main()
