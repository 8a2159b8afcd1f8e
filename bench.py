"""Benchmark of the ZHA decode hot path (routed decode queries per second).

One step = one decode step of the streaming workload: the newest token is in the
cache, zha_append_chunk runs when a chunk completes (every C steps), then
zha_route and zha_sparse_attend process the step's batch of queries at the
current context length. Inputs are resident in HBM; L2 is flushed (a 512 MiB
memset) between timed steps, outside the timed events.

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
    return ap.parse_args()


def measured_traffic(workload: str):
    """DRAM bytes per call measured by ncu on this workload (profiles/), if any."""
    path = os.path.join(ROOT, "profiles", "traffic_1m_context.json")
    if not os.path.exists(path):
        return None
    with open(path) as f:
        d = json.load(f)
    return d if d.get("workload") == workload else None


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
    lse out."""
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
    summ_nodes = 0
    pairs = 0
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
            summ_nodes += int(cand.any(axis=(0, 1)).sum())
            pairs += int(cand.sum())
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
        "score_pairs": pairs,
        "kv_bytes": kv_tokens * 2 * d * elt,
        "kv_tokens": kv_tokens,
        "route_bytes": summ_nodes * node_bytes + q_bytes,
        "attend_bytes": kv_tokens * 2 * d * elt + q_bytes + q_bytes + batch * spec.n_q_heads * 4,
    }


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


def cpu_baseline(inp: W.Inputs, n_tokens: int, budget_s: float = 20.0) -> dict:
    spec = inp.spec
    O, Kf, Vf, tree = oracle_setup(inp, n_tokens, 0)
    t0 = time.perf_counter()
    done = 0
    for b in range(spec.batch):
        for h in range(spec.group):
            oracle_head(O, Kf, Vf, tree, inp.Q[0, b, h].astype(np.float64), spec.p)
            done += 1
            if time.perf_counter() - t0 > budget_s:
                break
        if time.perf_counter() - t0 > budget_s:
            break
    dt = time.perf_counter() - t0
    return {"value": done / spec.n_q_heads / dt, "unit": UNIT, "cores": blas_threads(),
            "kind": "oracle",
            "sample": (f"fp64 numpy oracle: route + attend of {done} query heads of KV head 0 at "
                       f"context {n_tokens} (tree prebuilt, untimed); a query = {spec.n_q_heads} heads")}


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
            "data": "synthetic", "config": {"workload": spec.name, **spec.describe(), "l2": "n/a (CPU)"},
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": blas_threads(), "kind": "oracle",
                             "sample": sample},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


# ---------------------------------------------------------------------------
# The CUDA path
# ---------------------------------------------------------------------------

def run_zha(args, world, rank, local):
    from hierarchical_sparse_attention_zha_b200 import zha

    dev = torch.device("cuda", local)
    base = W.WORKLOADS[args.workload]
    K_steps, W_steps = args.steps, args.warmup
    n_e2e = 0 if args.no_e2e else min(K_steps, 64)
    total_steps = W_steps + K_steps + n_e2e
    if args.context:
        base = W.scaled(base, n_tokens=args.context)
    spec = W.scaled(base, stream_tokens=-(-(total_steps + 2) // base.chunk) * base.chunk)
    t_gen = time.perf_counter()
    inp = W.generate(spec, n_batches=total_steps, rank=rank)
    t_gen = time.perf_counter() - t_gen
    N0, C, B = spec.n_tokens, spec.chunk, spec.batch
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
    stream = torch.cuda.current_stream(dev)

    # prefill build, timed on its own
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
    bits = torch.zeros(total_steps, words + 1, dtype=torch.int32, device=dev)
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
    for s in range(W_steps):
        pos += 1
        step(s, pos)
        flush.zero_()
    torch.cuda.synchronize()

    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(K_steps)]
    positions, appended = [], []
    clocks = Clocks(torch.cuda.current_device()) if rank == 0 else None
    launches0 = zha.launch_count()
    barrier(world)
    torch.cuda.synchronize()
    if clocks:
        clocks.start()
    t_wall = time.perf_counter()
    for k in range(K_steps):
        s = W_steps + k
        pos += 1
        positions.append(pos)
        appended.append(step(s, pos, evs[k]))
        ids_keep[k].copy_(ids)
        cnt_keep[k].copy_(cnt)
        flush.zero_()
    torch.cuda.synchronize()
    barrier(world)
    t_wall = time.perf_counter() - t_wall
    clk = clocks.stop() if clocks else None
    launches = zha.launch_count() - launches0
    st = int(status.item())

    step_ms = np.array([e[0].elapsed_time(e[3]) for e in evs])
    app_ms = np.array([e[0].elapsed_time(e[1]) for e in evs])
    route_ms = np.array([e[1].elapsed_time(e[2]) for e in evs])
    att_ms = np.array([e[2].elapsed_time(e[3]) for e in evs])
    total_ms = float(step_ms.sum())
    total_ms_max = allreduce_max(total_ms, world)
    ms_per_step = total_ms_max / K_steps

    # algorithmic bytes, per step, from the recorded selections
    bits_h = bits[W_steps: W_steps + K_steps].cpu().numpy().view(np.uint32)
    ids_h, cnt_h = ids_keep.cpu().numpy(), cnt_keep.cpu().numpy()
    by = [step_bytes(spec, bits_h[k], ids_h[k], cnt_h[k], positions[k], B) for k in range(K_steps)]
    route_b = np.array([x["route_bytes"] for x in by], float)
    att_b = np.array([x["attend_bytes"] for x in by], float)
    peak, peak_kind = measured_peaks()
    route_gbs = route_b.sum() / (route_ms.sum() * 1e-3) / 1e9
    att_gbs = att_b.sum() / (att_ms.sum() * 1e-3) / 1e9
    step_gbs = (route_b.sum() + att_b.sum()) / (total_ms * 1e-3) / 1e9
    dominant = "zha_route" if route_ms.sum() >= att_ms.sum() else "zha_sparse_attend"
    ach = route_gbs if dominant == "zha_route" else att_gbs
    per_launch = (route_b.mean() if dominant == "zha_route" else att_b.mean())
    if args.dump_bytes and rank == 0:
        with open(args.dump_bytes, "w") as f:
            json.dump({"first_timed_step": W_steps, "route_bytes": route_b.tolist(),
                       "attend_bytes": att_b.tolist()}, f)
    traffic, traffic_note = None, None
    mt = measured_traffic(spec.name)
    if mt is not None and dominant in mt:
        traffic = float(mt[dominant]["dram_bytes"])
        traffic_note = (f"ncu dram bytes of one {dominant} call (step {mt['step']}, whose algorithmic "
                        f"bytes were {mt[dominant]['algorithmic_bytes']:.0f}); see profiles/")
    non_app = ~np.array(appended)
    append_frac = float(app_ms[np.array(appended)].sum() / step_ms.sum()) if any(appended) else 0.0

    # end to end through the API with host buffers
    e2e = None
    if n_e2e:
        Qh = torch.from_numpy(inp.Q).pin_memory()
        kv_new_k = torch.empty(spec.n_kv_heads, 1, spec.head_dim, dtype=kv_t).pin_memory()
        kv_new_v = torch.empty_like(kv_new_k).pin_memory()
        out_h = torch.empty(B, spec.n_q_heads, spec.head_dim, dtype=torch.float32).pin_memory()
        lse_h = torch.empty(B, spec.n_q_heads, dtype=torch.float32).pin_memory()
        q_dev = torch.empty_like(Qall[0])
        h2d = q_dev.numel() * 4 + 2 * kv_new_k.numel() * kv_new_k.element_size()
        d2h = out_h.numel() * 4 + lse_h.numel() * 4
        src_k = torch.from_numpy(inp.K.view(np.int16)).view(torch.bfloat16) if spec.kv_dtype == "bf16" else torch.from_numpy(inp.K)
        src_v = torch.from_numpy(inp.V.view(np.int16)).view(torch.bfloat16) if spec.kv_dtype == "bf16" else torch.from_numpy(inp.V)
        ee = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(n_e2e)]
        barrier(world)
        torch.cuda.synchronize()
        for k in range(n_e2e):
            s = W_steps + K_steps + k
            t_new = pos           # index of the token written this step
            pos += 1
            kv_new_k.copy_(src_k[:, t_new: t_new + 1])
            kv_new_v.copy_(src_v[:, t_new: t_new + 1])
            ee[k][0].record()
            K[:, t_new: t_new + 1].copy_(kv_new_k, non_blocking=True)
            V[:, t_new: t_new + 1].copy_(kv_new_v, non_blocking=True)
            q_dev.copy_(Qh[s], non_blocking=True)
            if pos % C == 0:
                tree.append_chunk(K, pos)
            tree.route(q_dev, pos, spec.p, max_sel, chunk_ids=ids, n_chunks=cnt, ws=ws_r,
                       kept_bits=bits[s], status=status)
            tree.sparse_attend(q_dev, K, V, pos, ids, cnt, out=out, lse=lse, ws=ws_a, status=status)
            out_h.copy_(out, non_blocking=True)
            lse_h.copy_(lse, non_blocking=True)
            ee[k][1].record()
            ee[k][1].synchronize()
            flush.zero_()
        torch.cuda.synchronize()
        e2e_ms = float(np.sum([a.elapsed_time(b) for a, b in ee]))
        e2e_ms = allreduce_max(e2e_ms, world) / n_e2e
        e2e = {"value": world * B / (e2e_ms * 1e-3), "unit": UNIT, "h2d_bytes_per_step": int(h2d),
               "d2h_bytes_per_step": int(d2h), "ms_per_step": e2e_ms, "steps": n_e2e}

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline(inp, positions[0])

    value = world * K_steps * B / (total_ms_max * 1e-3)
    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": K_steps,
            "warmup": W_steps, "ms_per_step": ms_per_step, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f32",
            "data": "synthetic (seeded generators; see DESIGN.md)",
            "config": {"workload": spec.name, **base.describe(), "decode_from": N0,
                       "steps_context": [positions[0], positions[-1]],
                       "l2": f"flushed between timed steps ({args.flush_mb} MiB memset outside the events)",
                       "parallelism": f"replicas x{world}" if world > 1 else "1 GPU"},
            "roofline": {"bound": "hbm", "achieved": ach, "peak": peak, "unit": "GB/s",
                         "frac": ach / peak, "traffic": traffic, "traffic_note": traffic_note,
                         "kernel": dominant,
                         "bytes_per_launch": float(per_launch), "peak_source": peak_kind},
            "step_roofline": {"achieved": step_gbs, "frac": step_gbs / peak,
                              "route_gbs": route_gbs, "attend_gbs": att_gbs,
                              "route_ms": float(route_ms.mean()), "attend_ms": float(att_ms.mean()),
                              "append_share": append_frac,
                              "bytes_per_step": float((route_b + att_b).mean()),
                              "summary_mb": float(np.mean([x["summary_bytes"] for x in by]) / 1e6),
                              "kv_mb": float(np.mean([x["kv_bytes"] for x in by]) / 1e6),
                              "kv_tokens": float(np.mean([x["kv_tokens"] for x in by])),
                              "score_pairs": float(np.mean([x["score_pairs"] for x in by]))},
            "build_ms": build_ms, "gen_s": t_gen, "wall_s_timed_region": t_wall,
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
