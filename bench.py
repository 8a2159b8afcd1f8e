"""Benchmark of the ZHA decode hot path (routed decode queries per second).

One step = one decode step of the streaming workload: the newest token is in the
cache, zha_append_chunk runs when a chunk completes (every C steps), then
zha_route and zha_sparse_attend process the step's batch of queries at the
current context length. Inputs are resident in HBM; L2 is flushed (a 512 MiB
memset) between timed steps, outside the timed events.

The timed window starts 2C - 5 tokens past the workload's context, so that level
1 holds one node more than at the context itself (16385 at 1M tokens: the
wide-level selection) and a chunk completes at the window's fifth step (the
append is timed with the step). Before it, a traced pass (CUDA events around
every library kernel) gives each kernel's share of the step; inside it, events
around the dominant kernel's launches give the roofline figure.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload 1m|256k|32k|deep|tiny]
                    [--impl zha|reference]

With N > 1 (torchrun) every rank runs an independent replica (its own seeded
problem): weak scaling, no data-path collective. Rank 0 prints one JSON line.
``--impl reference`` times the CPU oracle on the same workload instead.
"""

from __future__ import annotations

import argparse
import datetime
import json
import os
import subprocess
import sys
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from hierarchical_sparse_attention_zha_b200 import workloads as W  # noqa: E402

METRIC = "routed decode queries/sec/GPU at context N; achieved HBM GB/s vs roofline"
UNIT = "queries/s"
L2_NOTE = "GPU arm: L2 flushed between timed steps; CPU arm: not applicable"


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=256)
    ap.add_argument("--warmup", type=int, default=8)
    ap.add_argument("--workload", default="1m", choices=list(W.WORKLOADS))
    ap.add_argument("--impl", default="zha", choices=["zha", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--context", type=int, default=0,
                    help="override the workload's context length (profiling runs)")
    ap.add_argument("--flush-mb", type=int, default=512, help="L2 flush buffer between steps")
    ap.add_argument("--dump-bytes", default="",
                    help="write the algorithmic bytes of every timed step (JSON) to this path")
    ap.add_argument("--trace-steps", type=int, default=32,
                    help="steps of the traced pass before the timed region (0: none)")
    ap.add_argument("--cpu-budget", type=float, default=12.0,
                    help="seconds of oracle work per leg of the CPU baseline")
    return ap.parse_args()


def measured_traffic(workload: str, kernel_key: str, alg_bytes: float):
    """DRAM bytes per launch of `kernel_key` measured by ncu on this workload
    (profiles/traffic_<workload>.json), or None. The record names the kernel's
    source file and its SHA-256 when captured; a changed source voids it. A
    record taken on a smaller context of the same configuration holds the ratio
    of DRAM bytes to the launch's algorithmic bytes instead, and the traffic of
    a full launch is that ratio times `alg_bytes` (the launch's algorithmic
    bytes here)."""
    import hashlib
    path = os.path.join(ROOT, "profiles", f"traffic_{workload.lower().replace(' ', '_')}.json")
    if not os.path.exists(path):
        return None, None
    with open(path) as f:
        d = json.load(f)
    rec = d.get("kernels", {}).get(kernel_key)
    if d.get("workload") != workload or rec is None:
        return None, None
    src = os.path.join(ROOT, rec["source"])
    if not os.path.exists(src) or hashlib.sha256(open(src, "rb").read()).hexdigest() != rec["source_sha256"]:
        return None, f"ncu traffic of {kernel_key} predates the current {rec['source']}"
    if "dram_per_algorithmic" in rec:
        return float(rec["dram_per_algorithmic"]) * alg_bytes, (
            f"ncu dram__bytes_read.sum + dram__bytes_write.sum of one {kernel_key} launch = "
            f"{rec['dram_per_algorithmic']:.4f} x its algorithmic bytes, scaled to this launch's "
            f"algorithmic bytes ({rec.get('note', 'see profiles/')})")
    return float(rec["dram_bytes_per_launch"]), (
        f"ncu dram__bytes_read.sum + dram__bytes_write.sum of one {kernel_key} launch "
        f"({rec.get('note', 'see profiles/')})")


def measured_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    return 6650.0, "fallback"


# ---------------------------------------------------------------------------
# Algorithmic bytes of one step, from the kept bitmaps and chunk lists
# ---------------------------------------------------------------------------

def step_bytes(spec: W.Workload, bits: np.ndarray, ids: np.ndarray, cnt: np.ndarray,
               n_tokens: int, batch: int) -> dict:
    """Bytes the step must move: unique summaries visited per KV head and level,
    unique selected K/V rows per KV head (sink and tail included), Q in, O and
    lse out; per level also the (query head, candidate) pairs scored."""
    C, L, R, d, G = spec.chunk, spec.levels, spec.n_ref, spec.head_dim, spec.group
    nb = C * (n_tokens // C)
    node_bytes = R * (d + 1) * 4
    n_l = {l: nb // C ** l for l in range(1, L + 2)}
    n_l[L + 1] = 0
    words = {l: (n_l[l] + 31) // 32 for l in range(1, L + 1)}
    offs, o = {}, 0
    for l in range(1, L + 1):
        offs[l] = o
        o += batch * spec.n_q_heads * words[l]
    kept = {}
    for l in range(1, L + 1):
        blk = bits[offs[l]: offs[l] + batch * spec.n_q_heads * words[l]].reshape(batch, spec.n_q_heads, words[l])
        kept[l] = np.unpackbits(blk.view(np.uint8), axis=-1, bitorder="little")[..., : n_l[l]].astype(bool)
    levels = {l: {"nodes": 0, "pairs": 0} for l in range(1, L + 1)}
    for g in range(spec.n_kv_heads):
        hs = slice(g * G, (g + 1) * G)
        for l in range(1, L + 1):
            if n_l[l] == 0:
                continue
            orphan0 = C * n_l[l + 1]
            cand = np.zeros((batch, G, n_l[l]), bool)
            cand[..., orphan0:] = True
            if l < L and orphan0 > 0:
                cand[..., :orphan0] = np.repeat(kept[l + 1][:, hs, : n_l[l + 1]], C, axis=-1)
            levels[l]["nodes"] += int(cand.any(axis=(0, 1)).sum())
            levels[l]["pairs"] += int(cand.sum())
    summ_nodes = sum(v["nodes"] for v in levels.values())
    kv_tokens = 0
    tail = n_tokens - nb
    for g in range(spec.n_kv_heads):
        sel = np.zeros(nb // C, bool)
        sink_needed = False
        for b in range(batch):
            for h in range(g * G, (g + 1) * G):
                c = ids[b, h, : cnt[b, h]]
                sel[c] = True
                if nb > 0 and (cnt[b, h] == 0 or c[0] != 0):
                    sink_needed = True
        kv_tokens += int(sel.sum()) * C + tail + (1 if sink_needed and not sel[0] else 0)
    elt = spec.elt_bytes
    q_bytes = batch * spec.n_q_heads * d * 4
    return {
        "summary_bytes": summ_nodes * node_bytes,
        "summary_nodes": summ_nodes,
        "score_pairs": sum(v["pairs"] for v in levels.values()),
        "levels": levels,
        "node_bytes": node_bytes,
        "q_bytes": q_bytes,
        "kv_bytes": kv_tokens * 2 * d * elt,
        "kv_tokens": kv_tokens,
        "route_bytes": summ_nodes * node_bytes + q_bytes,
        "attend_bytes": kv_tokens * 2 * d * elt + q_bytes + q_bytes + batch * spec.n_q_heads * 4,
    }


def kernel_bytes(name: str, tag: int, by: dict) -> float | None:
    """Algorithmic bytes of one launch of a library kernel in a step whose
    step_bytes() are `by` (None for kernels without a byte model): a scoring
    launch reads its level's visited node records and the queries and writes one
    score per (query head, candidate) pair; a selection launch reads those scores;
    the attention kernels read the selected K/V rows and the queries."""
    if name in ("score_dense_kernel", "select_top_kernel"):
        return None                    # several levels in one launch (latency-bound)
    if name.startswith("score") and tag in by["levels"]:
        lv = by["levels"][tag]
        return lv["nodes"] * by["node_bytes"] + lv["pairs"] * 4 + by["q_bytes"]
    if name.startswith("select") and tag in by["levels"]:
        return by["levels"][tag]["pairs"] * 4
    if name in ("attend_split_kernel", "attend_kernel"):
        return by["kv_bytes"] + by["q_bytes"]
    return None


# ---------------------------------------------------------------------------
# Clock sampling during the timed region
# ---------------------------------------------------------------------------

class Clocks:
    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.proc = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.index), f"--query-gpu={self.Q}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None

    def stop(self) -> dict | None:
        if self.proc is None:
            return None
        time.sleep(0.25)
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
            out, _ = self.proc.communicate()
        sm, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in out.strip().splitlines():
            f = [x.strip() for x in line.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                mx.append(float(f[2]))
            except ValueError:
                continue
            for nm, v in zip(names, f[5:9]):
                if v.lower() == "active":
                    reasons.add(nm)
        if not sm:
            return None
        return {"sm_mhz": float(np.median(sm)), "sm_max_mhz": float(max(mx)),
                "reasons": sorted(reasons), "samples": len(sm)}


# ---------------------------------------------------------------------------
# The oracle on a bounded sample (cpu_baseline leg and --impl reference)
# ---------------------------------------------------------------------------

def oracle_setup(inp: W.Inputs, n_tokens: int, g: int = 0):
    import oracle as O
    spec = inp.spec
    Kf = O.bf16_bits_to_f64(inp.K[g, :n_tokens]) if spec.kv_dtype == "bf16" else inp.K[g, :n_tokens].astype(np.float64)
    Vf = O.bf16_bits_to_f64(inp.V[g, :n_tokens]) if spec.kv_dtype == "bf16" else inp.V[g, :n_tokens].astype(np.float64)
    tree = O.build_tree(Kf, inp.ref_q[g], spec.chunk, spec.levels, n_tokens)
    return O, Kf, Vf, tree


def oracle_head(O, Kf, Vf, tree, q, p):
    tr = O.route(q, tree, p)
    return O.attend(q, Kf, Vf, tr.tokens)


def blas_threads() -> int:
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads", 1) for i in threadpool_info() if i.get("user_api") == "blas"]
        return int(max(n)) if n else 1
    except Exception:
        return os.cpu_count() or 1


def cpu_baseline(inp: W.Inputs, n_tokens: int, q_index: int, budget_s: float,
                 gpu_kept: dict | None = None) -> dict:
    """The oracle on this host, on a bounded sample of the workload at context
    n_tokens (the first timed step's context and queries): route + attend of the
    query heads of KV head 0 on all cores and on one thread, the oracle's build
    of KV head 0's tree, and dense fp64 attention of one head over the whole
    context. With `gpu_kept` ({(b, h): {level: ids}} of the same step) the
    sampled heads' routes are also compared with the GPU's (ties counted)."""
    from threadpoolctl import threadpool_limits

    from oracle.parity import RouteReport, compare_route_head
    spec = inp.spec
    import oracle as O
    t0 = time.perf_counter()
    O, Kf, Vf, tree = oracle_setup(inp, n_tokens, 0)
    build_s = time.perf_counter() - t0
    heads = [(b, h) for b in range(spec.batch) for h in range(spec.group)]
    report = RouteReport()

    def run(limit_s, max_heads):
        t = time.perf_counter()
        done = 0
        for (b, h) in heads[:max_heads]:
            q = inp.Q[q_index, b, h].astype(np.float64)
            tr = O.route(q, tree, spec.p)
            O.attend(q, Kf, Vf, tr.tokens)
            if gpu_kept is not None and (b, h) in gpu_kept and done >= report.heads:
                compare_route_head(q, tree, spec.p, gpu_kept[(b, h)], report, (b, h))
            done += 1
            if time.perf_counter() - t > limit_s:
                break
        return done, time.perf_counter() - t

    n_all, t_all = run(budget_s, len(heads))
    with threadpool_limits(limits=1):
        n_one, t_one = run(budget_s / 2, len(heads))
        t = time.perf_counter()
        O.sdpa(inp.Q[q_index, 0, 0].astype(np.float64)[None], Kf, Vf)
        dense_1t = time.perf_counter() - t
    t = time.perf_counter()
    O.sdpa(inp.Q[q_index, 0, 0].astype(np.float64)[None], Kf, Vf)
    dense_all = time.perf_counter() - t
    out = {"value": n_all / spec.n_q_heads / t_all, "unit": UNIT, "cores": blas_threads(),
           "kind": "oracle",
           "sample": (f"fp64 numpy oracle: route + attend of {n_all} query heads of KV head 0 at "
                      f"context {n_tokens} (queries of the first timed step; tree prebuilt, "
                      f"untimed); a query = {spec.n_q_heads} heads"),
           "single_thread": {"value": n_one / spec.n_q_heads / t_one, "unit": UNIT, "cores": 1,
                             "heads": n_one},
           "os_cpu_count": os.cpu_count(),
           "oracle_build_s": {"kv_heads": 1, "tokens": n_tokens, "seconds": build_s,
                              "whole_tree_estimate_s": build_s * spec.n_kv_heads},
           "dense_attention_ms_per_head": {"all_cores": dense_all * 1e3, "one_thread": dense_1t * 1e3,
                                           "tokens": n_tokens}}
    if gpu_kept is not None:
        out["route_parity_sample"] = report.summary()
        out["route_parity_sample"]["hard_examples"] = [str(x) for x in report.hard[:3]]
    return out


# ---------------------------------------------------------------------------
# Distributed plumbing
# ---------------------------------------------------------------------------

def dist_setup(n_gpus: int):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import torch.distributed as dist
        backend = "nccl" if torch.cuda.is_available() else "gloo"
        if torch.cuda.is_available():
            torch.cuda.set_device(local)
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120))
    elif torch.cuda.is_available():
        torch.cuda.set_device(local)
    return world, rank, local


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def allreduce_max(x: float, world: int) -> float:
    if world == 1:
        return x
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64, device="cuda" if torch.cuda.is_available() else "cpu")
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def dist_close(world):
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


# ---------------------------------------------------------------------------
# The reference arm: the oracle on the host cores
# ---------------------------------------------------------------------------

def run_reference(args, world, rank):
    if rank != 0:
        return
    spec = W.WORKLOADS[args.workload]
    inp = W.generate(spec, n_batches=1)
    n_tokens = spec.n_tokens
    O, Kf, Vf, tree = oracle_setup(inp, n_tokens, 0)
    heads = [(b, h) for b in range(spec.batch) for h in range(spec.group)]
    times = []
    for s in range(args.warmup + args.steps):
        b, h = heads[s % len(heads)]
        t0 = time.perf_counter()
        oracle_head(O, Kf, Vf, tree, inp.Q[0, b, h].astype(np.float64), spec.p)
        if s >= args.warmup:
            times.append(time.perf_counter() - t0)
    step = float(np.mean(times))
    value = 1.0 / (spec.n_q_heads * step)
    sample = (f"each step: fp64 numpy oracle route + attend of one query head of KV head 0 at "
              f"context {n_tokens} (tree prebuilt, untimed); a query = {spec.n_q_heads} heads")
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": step * 1e3,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic (seeded generators in hierarchical_sparse_attention_zha_b200/workloads.py)",
            "config": {"workload": spec.name, **spec.describe(), "l2": L2_NOTE},
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": blas_threads(), "kind": "oracle",
                             "sample": sample},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


# ---------------------------------------------------------------------------
# The CUDA path
# ---------------------------------------------------------------------------

def _kernel_key(name: str, tag: int) -> str:
    return f"{name}/L{tag}" if name.startswith(("score", "select")) else name


def run_zha(args, world, rank, local):
    from hierarchical_sparse_attention_zha_b200 import zha

    dev = torch.device("cuda", local)
    base = W.WORKLOADS[args.workload]
    if args.context:
        base = W.scaled(base, n_tokens=args.context)
    C = base.chunk
    K_steps, W_steps = args.steps, args.warmup
    T_steps = max(0, args.trace_steps)
    n_e2e = 0 if args.no_e2e else min(K_steps, 64)
    e2e_warm = 4 if n_e2e else 0
    # First timed context: 2C - 5 tokens past the workload's context (level 1
    # then holds one node more; a chunk completes at the fifth timed step).
    p_first = base.n_tokens + 2 * C - min(5, C)
    N0 = p_first - 1 - W_steps - T_steps
    if N0 < 1:
        raise SystemExit("bench: the warm-up and traced steps do not fit before the timed window")
    n_batches = W_steps + T_steps + K_steps + e2e_warm + n_e2e
    last = p_first + K_steps + e2e_warm + n_e2e + 1
    spec = W.scaled(base, stream_tokens=-(-(last - base.n_tokens) // C) * C)
    t_gen = time.perf_counter()
    inp = W.generate(spec, n_batches=n_batches, rank=rank)
    t_gen = time.perf_counter() - t_gen
    B = spec.batch
    kv_t = torch.bfloat16 if spec.kv_dtype == "bf16" else torch.float32
    if spec.kv_dtype == "bf16":
        K = torch.from_numpy(inp.K.view(np.int16)).to(dev).view(torch.bfloat16)
        V = torch.from_numpy(inp.V.view(np.int16)).to(dev).view(torch.bfloat16)
    else:
        K = torch.from_numpy(inp.K).to(dev)
        V = torch.from_numpy(inp.V).to(dev)
    refq = torch.from_numpy(inp.ref_q).to(dev)
    Qall = torch.from_numpy(inp.Q).to(dev)
    cap = spec.capacity
    cfg = zha.make_config(spec.n_kv_heads, spec.n_q_heads, spec.head_dim, C, spec.levels, spec.n_ref,
                          kv_t, cap)
    tree = zha.Tree(cfg, refq)

    # prefill build, timed on its own (after one untimed build)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    tree.build(K, N0)
    torch.cuda.synchronize()
    tree = zha.Tree(cfg, refq)
    e0.record()
    tree.build(K, N0)
    e1.record()
    torch.cuda.synchronize()
    build_ms = e0.elapsed_time(e1)

    max_sel = cap // C
    ids = torch.empty(B, spec.n_q_heads, max_sel, dtype=torch.int32, device=dev)
    cnt = torch.empty(B, spec.n_q_heads, dtype=torch.int32, device=dev)
    words = zha.route_kept_words(cfg, B, cap)
    bits = torch.zeros(n_batches, words + 1, dtype=torch.int32, device=dev)
    ids_keep = torch.empty(K_steps, B, spec.n_q_heads, max_sel, dtype=torch.int32, device=dev)
    cnt_keep = torch.empty(K_steps, B, spec.n_q_heads, dtype=torch.int32, device=dev)
    ws_r = torch.empty(zha.route_workspace_bytes(cfg, B, cap) // 4 + 64, dtype=torch.float32, device=dev)
    ws_a = torch.empty(zha.attend_workspace_bytes(cfg, B, cap) // 4 + 64, dtype=torch.float32, device=dev)
    out = torch.empty(B, spec.n_q_heads, spec.head_dim, dtype=torch.float32, device=dev)
    lse = torch.empty(B, spec.n_q_heads, dtype=torch.float32, device=dev)
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    flush = torch.empty(max(1, args.flush_mb) << 20, dtype=torch.uint8, device=dev)

    def step(s, n_tok, ev=None):
        if ev is not None:
            ev[0].record()
        appended = False
        if n_tok % C == 0:
            tree.append_chunk(K, n_tok)
            appended = True
        if ev is not None:
            ev[1].record()
        tree.route(Qall[s], n_tok, spec.p, max_sel, chunk_ids=ids, n_chunks=cnt,
                   kept_bits=bits[s], ws=ws_r, status=status)
        if ev is not None:
            ev[2].record()
        tree.sparse_attend(Qall[s], K, V, n_tok, ids, cnt, out=out, lse=lse, ws=ws_a, status=status)
        if ev is not None:
            ev[3].record()
        return appended

    pos = N0
    s = 0
    for _ in range(W_steps):
        pos += 1
        step(s, pos)
        s += 1
        flush.zero_()
    torch.cuda.synchronize()

    # traced pass: CUDA events around every library kernel (shares of the step)
    kernels, dominant = {}, ("score_tma_kernel", 1)
    if T_steps:
        zha.trace_enable(64 * T_steps)
        trace_bytes = []
        for _ in range(T_steps):
            pos += 1
            step(s, pos)
            trace_bytes.append((s, pos))
            s += 1
            flush.zero_()
        torch.cuda.synchronize()
        recs = zha.trace_records()
        zha.trace_enable(0)
        tot = sum(ms for _, _, ms in recs)
        for name, tag, ms in recs:
            k = kernels.setdefault(_kernel_key(name, tag), {"name": name, "tag": tag, "launches": 0,
                                                           "total_us": 0.0})
            k["launches"] += 1
            k["total_us"] += ms * 1e3
        for k in kernels.values():
            k["mean_us"] = k["total_us"] / k["launches"]
            k["share"] = k["total_us"] / (tot * 1e3) if tot > 0 else 0.0
        if kernels:
            top = max(kernels.values(), key=lambda k: k["total_us"])
            dominant = (top["name"], top["tag"])
    torch.cuda.synchronize()

    # timed region; events also bracket the dominant kernel's launches
    zha.trace_enable(4 * K_steps + 16, dominant[0], dominant[1])
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(K_steps)]
    positions, appended, s_timed = [], [], []
    clocks = Clocks(torch.cuda.current_device()) if rank == 0 else None
    launches0 = zha.launch_count()
    barrier(world)
    torch.cuda.synchronize()
    if clocks:
        clocks.start()
    t_wall = time.perf_counter()
    for k in range(K_steps):
        pos += 1
        positions.append(pos)
        s_timed.append(s)
        appended.append(step(s, pos, evs[k]))
        s += 1
        ids_keep[k].copy_(ids)
        cnt_keep[k].copy_(cnt)
        flush.zero_()
    torch.cuda.synchronize()
    barrier(world)
    t_wall = time.perf_counter() - t_wall
    clk = clocks.stop() if clocks else None
    launches = zha.launch_count() - launches0
    dom_recs = zha.trace_records()
    zha.trace_enable(0)
    st = int(status.item())

    step_ms = np.array([e[0].elapsed_time(e[3]) for e in evs])
    app_ms = np.array([e[0].elapsed_time(e[1]) for e in evs])
    route_ms = np.array([e[1].elapsed_time(e[2]) for e in evs])
    att_ms = np.array([e[2].elapsed_time(e[3]) for e in evs])
    total_ms = float(step_ms.sum())
    total_ms_max = allreduce_max(total_ms, world)
    ms_per_step = total_ms_max / K_steps

    # algorithmic bytes, per step, from the recorded selections
    bits_h = bits.cpu().numpy().view(np.uint32)
    ids_h, cnt_h = ids_keep.cpu().numpy(), cnt_keep.cpu().numpy()
    by = [step_bytes(spec, bits_h[s_timed[k]], ids_h[k], cnt_h[k], positions[k], B)
          for k in range(K_steps)]
    route_b = np.array([x["route_bytes"] for x in by], float)
    att_b = np.array([x["attend_bytes"] for x in by], float)
    peak, peak_kind = measured_peaks()
    route_gbs = route_b.sum() / (route_ms.sum() * 1e-3) / 1e9
    att_gbs = att_b.sum() / (att_ms.sum() * 1e-3) / 1e9
    step_gbs = (route_b.sum() + att_b.sum()) / (total_ms * 1e-3) / 1e9

    # the dominant kernel: one launch per step, bytes from that step's selection
    dom_key = _kernel_key(*dominant)
    dom_ms = [ms for _, _, ms in dom_recs]
    dom_b = [kernel_bytes(dominant[0], dominant[1], by[k]) for k in range(K_steps)]
    roofline = None
    if len(dom_ms) == K_steps and all(b is not None for b in dom_b) and sum(dom_ms) > 0:
        ach = sum(dom_b) / (sum(dom_ms) * 1e-3) / 1e9
        traffic, traffic_note = measured_traffic(spec.name, dom_key, float(np.mean(dom_b)))
        roofline = {"bound": "hbm", "achieved": ach, "peak": peak, "unit": "GB/s", "frac": ach / peak,
                    "traffic": traffic, "traffic_note": traffic_note, "kernel": dom_key,
                    "bytes_per_launch": float(np.mean(dom_b)), "mean_us": float(np.mean(dom_ms)) * 1e3,
                    "launches": len(dom_ms), "peak_source": f"{peak_kind} (MEASURED_PEAKS.json hbm_gbs)"
                    if peak_kind == "measured" else "fallback 6650 GB/s"}
    if args.dump_bytes and rank == 0:
        with open(args.dump_bytes, "w") as f:
            json.dump({"first_timed_step": W_steps + T_steps, "route_bytes": route_b.tolist(),
                       "attend_bytes": att_b.tolist(),
                       "levels": [{str(l): v for l, v in x["levels"].items()} for x in by]}, f)
    # per-kernel achieved bandwidth of the traced pass (scoring and selection
    # kernels run once per step and level; their bytes follow from the bitmaps)
    if T_steps and kernels:
        no_ids = np.zeros((B, spec.n_q_heads, 1), np.int32)
        no_cnt = np.zeros((B, spec.n_q_heads), np.int32)
        by_t = [step_bytes(spec, bits_h[st_], no_ids, no_cnt, p_, B) for st_, p_ in trace_bytes]
        for k in kernels.values():
            name, tag = k.pop("name"), k["tag"]
            bt = [kernel_bytes(name, tag, x) for x in by_t]
            if name.startswith(("score", "select")) and all(b is not None for b in bt) and \
                    k["launches"] == len(by_t):
                k["gbs"] = sum(bt) / (k["total_us"] * 1e-6) / 1e9
                k["frac"] = k["gbs"] / peak
    append_frac = float(app_ms[np.array(appended)].sum() / step_ms.sum()) if any(appended) else 0.0

    # end to end through the API with host buffers
    e2e = None
    if n_e2e:
        # One pinned input block per step (the step's queries, then the new
        # token's K and V rows) goes H2D in one copy; O and lse come back in
        # one copy from one device block.
        Qh = torch.from_numpy(inp.Q)
        elt_kv = 2 if spec.kv_dtype == "bf16" else 4
        q_nbytes = Qall[0].numel() * 4
        row_nbytes = spec.n_kv_heads * spec.head_dim * elt_kv
        in_h = torch.empty(q_nbytes + 2 * row_nbytes, dtype=torch.uint8).pin_memory()
        in_d = torch.empty(in_h.numel(), dtype=torch.uint8, device=dev)

        def in_views(buf):
            q_v = buf[:q_nbytes].view(torch.float32).view(Qall[0].shape)
            k_v = buf[q_nbytes: q_nbytes + row_nbytes].view(kv_t).view(spec.n_kv_heads, 1, spec.head_dim)
            v_v = buf[q_nbytes + row_nbytes:].view(kv_t).view(spec.n_kv_heads, 1, spec.head_dim)
            return q_v, k_v, v_v

        q_h, k_h, v_h = in_views(in_h)
        q_dev, k_dev, v_dev = in_views(in_d)
        n_out = out.numel()
        res_d = torch.empty(n_out + lse.numel(), dtype=torch.float32, device=dev)
        res_h = torch.empty(res_d.numel(), dtype=torch.float32).pin_memory()
        out_d, lse_d = res_d[:n_out].view(out.shape), res_d[n_out:].view(lse.shape)
        h2d = in_h.numel()
        d2h = res_h.numel() * 4
        src_k = torch.from_numpy(inp.K.view(np.int16)).view(torch.bfloat16) if spec.kv_dtype == "bf16" else torch.from_numpy(inp.K)
        src_v = torch.from_numpy(inp.V.view(np.int16)).view(torch.bfloat16) if spec.kv_dtype == "bf16" else torch.from_numpy(inp.V)
        ee = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(n_e2e)]
        host_s, host_calls = 0.0, 0
        barrier(world)
        torch.cuda.synchronize()
        for k in range(e2e_warm + n_e2e):
            timed = k >= e2e_warm
            t_new = pos           # index of the token written this step
            pos += 1
            q_h.copy_(Qh[s])
            k_h.copy_(src_k[:, t_new: t_new + 1])
            v_h.copy_(src_v[:, t_new: t_new + 1])
            if timed:
                ee[k - e2e_warm][0].record()
            in_d.copy_(in_h, non_blocking=True)
            K[:, t_new: t_new + 1].copy_(k_dev)
            V[:, t_new: t_new + 1].copy_(v_dev)
            th = time.perf_counter()
            n_calls = 2
            if pos % C == 0:
                tree.append_chunk(K, pos)
                n_calls += 1
            tree.route(q_dev, pos, spec.p, max_sel, chunk_ids=ids, n_chunks=cnt, ws=ws_r,
                       kept_bits=bits[s], status=status)
            tree.sparse_attend(q_dev, K, V, pos, ids, cnt, out=out_d, lse=lse_d, ws=ws_a, status=status)
            if timed:
                host_s += time.perf_counter() - th
                host_calls += n_calls
            res_h.copy_(res_d, non_blocking=True)
            if timed:
                ee[k - e2e_warm][1].record()
                ee[k - e2e_warm][1].synchronize()
            else:
                torch.cuda.synchronize()
            s += 1
            flush.zero_()
        torch.cuda.synchronize()
        e2e_ms = float(np.sum([a.elapsed_time(b) for a, b in ee]))
        e2e_ms = allreduce_max(e2e_ms, world) / n_e2e
        e2e = {"value": world * B / (e2e_ms * 1e-3), "unit": UNIT, "h2d_bytes_per_step": int(h2d),
               "d2h_bytes_per_step": int(d2h), "ms_per_step": e2e_ms, "steps": n_e2e,
               "warmup": e2e_warm, "host_us_per_call": host_s * 1e6 / max(1, host_calls),
               "note": "timed region: one H2D copy of the step's queries and new K/V row from pinned "
                       "memory (the row then written into the cache on the device), the library calls "
                       "(Python binding -> C ABI), one D2H copy of O and lse, then a host "
                       "synchronisation"}

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        kept0 = {}           # the GPU's kept sets of KV head 0's heads at the first timed step
        nb0 = C * (positions[0] // C)
        offs, o = {}, 0
        for l in range(1, spec.levels + 1):
            offs[l] = o
            o += B * spec.n_q_heads * ((nb0 // C ** l + 31) // 32)
        for b in range(B):
            for h in range(spec.group):
                per = {}
                for l in range(1, spec.levels + 1):
                    n_l = nb0 // C ** l
                    w = (n_l + 31) // 32
                    blk = bits_h[s_timed[0]][offs[l] + (b * spec.n_q_heads + h) * w:
                                             offs[l] + (b * spec.n_q_heads + h + 1) * w]
                    nz = np.nonzero(np.unpackbits(blk.view(np.uint8), bitorder="little"))[0]
                    per[l] = nz[nz < n_l]
                kept0[(b, h)] = per
        cpu = cpu_baseline(inp, positions[0], s_timed[0], args.cpu_budget, gpu_kept=kept0)

    value = world * K_steps * B / (total_ms_max * 1e-3)
    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": K_steps,
            "warmup": W_steps, "ms_per_step": ms_per_step, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f32",
            "data": "synthetic (seeded generators in hierarchical_sparse_attention_zha_b200/workloads.py)",
            "config": {"workload": spec.name, **base.describe(), "l2": L2_NOTE},
            "parallelism": f"replicas x{world}" if world > 1 else "1 GPU",
            "window": {"decode_from": N0, "steps_context": [positions[0], positions[-1]],
                       "level1_nodes": [positions[0] // C, positions[-1] // C],
                       "appends": int(sum(appended)),
                       "l2_flush": f"{args.flush_mb} MiB memset between timed steps, outside the events"},
            "roofline": roofline,
            "step_roofline": {"achieved": step_gbs, "frac": step_gbs / peak,
                              "route_gbs": route_gbs, "attend_gbs": att_gbs,
                              "route_ms": float(route_ms.mean()), "attend_ms": float(att_ms.mean()),
                              "append_share": append_frac,
                              "append_ms_when_appending": float(app_ms[np.array(appended)].mean())
                              if any(appended) else None,
                              "bytes_per_step": float((route_b + att_b).mean()),
                              "summary_mb": float(np.mean([x["summary_bytes"] for x in by]) / 1e6),
                              "kv_mb": float(np.mean([x["kv_bytes"] for x in by]) / 1e6),
                              "kv_tokens": float(np.mean([x["kv_tokens"] for x in by])),
                              "score_pairs": float(np.mean([x["score_pairs"] for x in by]))},
            "kernels": {"source": f"traced pass of {T_steps} steps before the timed region "
                                  "(CUDA events around each library launch)", "by_kernel": kernels},
            "build_ms": build_ms, "build_tokens": N0, "gen_s": t_gen, "wall_s_timed_region": t_wall,
            "gpu_launches": int(launches), "device_status": st,
            "clocks": clk, "e2e": e2e, "cpu_baseline": cpu,
        }
        print(json.dumps(line), flush=True)


def main():
    args = parse()
    world, rank, local = dist_setup(args.gpus)
    try:
        if args.impl == "reference":
            run_reference(args, world, rank)
        else:
            run_zha(args, world, rank, local)
    finally:
        dist_close(world)


if __name__ == "__main__":
    main()
