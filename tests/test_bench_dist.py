"""bench.py's multi-process plumbing on CPU (gloo, world size 2): replicas
each run their own problem, rank 0 alone prints, and times are reduced as the
maximum over ranks. No GPU is involved."""

import json
import os
import socket
import subprocess
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    os.environ.update(RANK=str(rank), WORLD_SIZE=str(world), LOCAL_RANK=str(rank),
                      MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    sys.path.insert(0, ROOT)
    import bench
    w, r, _ = bench.dist_setup(world)
    assert (w, r) == (world, rank)
    bench.barrier(w)
    got = bench.allreduce_max(float(10 * rank + 1), w)
    out.put((rank, got))
    bench.dist_close(w)


def test_allreduce_max_over_two_gloo_ranks():
    port = _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    res = dict(q.get(timeout=10) for _ in range(2))
    assert res == {0: 11.0, 1: 11.0}


def test_reference_arm_under_torchrun_prints_one_line():
    port = _free_port()
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node", "2",
           "--master-addr", "127.0.0.1", "--master-port", str(port), "bench.py", "--impl", "reference",
           "--gpus", "2", "--workload", "tiny", "--steps", "2", "--warmup", "1"]
    env = dict(os.environ, OMP_NUM_THREADS="1")
    r = subprocess.run(cmd, cwd=ROOT, capture_output=True, text=True, timeout=600, env=env)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [l for l in r.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1
    line = json.loads(lines[0])
    assert line["impl"] == "reference" and line["n_gpus"] == 2 and line["value"] > 0
    assert line["config"]["workload"] == "Tiny NoPE"
    assert set(line["e2e"]) >= {"value", "unit", "h2d_bytes_per_step", "d2h_bytes_per_step"}


def test_step_bytes_counts_unique_summaries_and_rows():
    """The algorithmic-bytes accounting on a hand-made selection."""
    sys.path.insert(0, ROOT)
    import numpy as np
    import bench
    from hierarchical_sparse_attention_zha_b200 import workloads as W
    spec = W.scaled("tiny", n_kv_heads=1, n_q_heads=2, chunk=4, levels=2, n_ref=4, head_dim=64,
                    kv_dtype="f32", batch=1)
    n_tokens = 70                     # N_b = 68: 17 level-1 nodes, 4 level-2 nodes, tail 2 tokens
    w1, w2 = 1, 1                     # bitmap words per head at levels 1 and 2
    bits = np.zeros(2 * w1 + 2 * w2, np.uint32)
    bits[0] = 0b101                   # head 0 keeps level-1 nodes 0 and 2
    bits[1] = 0b1000                  # head 1 keeps level-1 node 3
    bits[2] = 0b1                     # head 0 keeps level-2 node 0
    bits[3] = 0b11                    # head 1 keeps level-2 nodes 0 and 1
    ids = np.array([[[0, 2, -1], [3, -1, -1]]], np.int32)
    cnt = np.array([[2, 1]], np.int32)
    by = bench.step_bytes(spec, bits, ids, cnt, n_tokens, batch=1)
    node = 4 * 65 * 4
    # level 2: every node is a candidate (4); level 1: children of kept level-2
    # nodes (head 0: 0..3, head 1: 0..7) plus the orphan 16 -> union 0..7 and 16
    assert by["summary_nodes"] == 4 + 9
    assert by["summary_bytes"] == 13 * node
    # K/V rows: chunks {0, 2, 3} (12 tokens) + tail (2); the sink is in chunk 0
    assert by["kv_tokens"] == 14
    assert by["kv_bytes"] == 14 * 2 * 64 * 4
