"""Parity of the CUDA path (through the C ABI) with the CPU oracle.

Every case draws seeded inputs, runs build -> route -> sparse attend on the GPU
and checks, against the oracle on the same bytes:
  * every summary of every level (norm-wise relative 1e-4);
  * the kept set of every level of every query head, the level conditioned on
    the GPU's kept set one level up; disagreements are allowed only as ties
    (score within 1e-5 of the cut, or cumulative mass within 1e-5 of p), which
    are counted and reported;
  * the attention output and log-normaliser over the GPU's leaf set (absolute
    2e-2 bf16 / 1e-4 fp32, and a tighter fp32-accumulation bound).
Small cases are checked exhaustively; the full-size workloads on sampled nodes
and heads (the oracle computes those one by one).
"""

import math

import numpy as np
import pytest
import torch

import oracle as O
from hierarchical_sparse_attention_zha_b200 import workloads as W
from _parity import (O_ATOL, SUMMARY_RTOL, RouteReport, attend_errors, cache_f64, compare_route_head,
                     config_for, derived_lse_bound, derived_o_bound, kept_from_bits, summary_errors,
                     to_device, values_f64)

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def zha():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from hierarchical_sparse_attention_zha_b200 import zha as z
    return z


def run_pipeline(zha, inp, n_tokens, p=None, max_sel=None, batch_index=0, stream=None, tree=None,
                 dev=None):
    """Build (unless ``tree`` is given: a tree already built to ``n_tokens``),
    route and attend on the GPU; ``dev`` = (K, V, ref_q, Q) device tensors."""
    spec = inp.spec
    K, V, refq, Q = dev if dev is not None else to_device(inp)
    if tree is None:
        cfg = config_for(spec)
        tree = zha.Tree(cfg, refq)
        tree.build(K, n_tokens, stream=stream)
    cfg = tree.cfg
    q = Q[batch_index].contiguous()
    B = q.shape[0]
    p = spec.p if p is None else p
    max_sel = max_sel or max(1, n_tokens // spec.chunk)
    bits = torch.zeros(zha.route_kept_words(cfg, B, n_tokens) + 1, dtype=torch.int32, device="cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    ids, cnt = tree.route(q, n_tokens, p, max_sel, kept_bits=bits, status=status, stream=stream)
    out, lse = tree.sparse_attend(q, K, V, n_tokens, ids, cnt, status=status, stream=stream)
    torch.cuda.synchronize()
    return dict(tree=tree, K=K, V=V, Q=q, ids=ids.cpu().numpy(), cnt=cnt.cpu().numpy(),
                bits=bits.cpu().numpy().view(np.uint32), out=out.cpu().numpy().astype(np.float64),
                lse=lse.cpu().numpy().astype(np.float64), status=int(status.item()), p=p)


def check_case(zha, inp, n_tokens, p=None, heads=None, all_nodes=True, batch_index=0, tree=None,
               dev=None, oracle_p=None, oracle_build=None):
    """Full comparison; returns the route report. ``p`` goes to the GPU route
    (a mass or a zha.RoutePolicy), ``oracle_p`` (default: ``p``) to the oracle's."""
    spec = inp.spec
    res = run_pipeline(zha, inp, n_tokens, p=p, batch_index=batch_index, tree=tree, dev=dev)
    p = res["p"] if oracle_p is None else oracle_p
    assert res["status"] == 0
    G = spec.group
    B = spec.batch
    kept = kept_from_bits(res["bits"], spec, B, n_tokens)
    report = RouteReport()
    for g in range(spec.n_kv_heads):
        Kf = cache_f64(inp, g, n_tokens)
        Vf = values_f64(inp, g, n_tokens)
        build = oracle_build or O.build_tree
        otree = build(Kf, inp.ref_q[g], spec.chunk, spec.levels, n_tokens)
        # summaries, every level
        for lvl in range(1, spec.levels + 1):
            n_l = otree.n_nodes(lvl)
            if n_l == 0:
                continue
            kh, bh = res["tree"].level(lvl)
            kh = kh[g, :n_l].cpu().numpy().astype(np.float64)
            bh = bh[g, :n_l].cpu().numpy().astype(np.float64)
            ek, eb = summary_errors(kh, bh, *otree.nodes[lvl])
            assert ek <= SUMMARY_RTOL and eb <= SUMMARY_RTOL, (g, lvl, ek, eb)
        for b in range(B):
            for h in range(g * G, (g + 1) * G):
                if heads is not None and (b, h) not in heads:
                    continue
                q = inp.Q[batch_index, b, h].astype(np.float64)
                gpu_kept = {lvl: kept[lvl][(b, h)] for lvl in kept}
                compare_route_head(q, otree, p, gpu_kept, report, (b, h))
                # the chunk list equals the level-1 bitmap, ascending
                n = int(res["cnt"][b, h])
                assert list(res["ids"][b, h, :n]) == list(gpu_kept[1])
                S = O.leaf_token_set(res["ids"][b, h, :n], spec.chunk, n_tokens)
                do, dl, vmax, lse_ref = attend_errors(q, Kf, Vf, S, res["out"][b, h], res["lse"][b, h])
                assert do <= O_ATOL[spec.kv_dtype], (b, h, do)
                assert do <= derived_o_bound(vmax), (b, h, do, vmax)
                assert dl <= derived_lse_bound(lse_ref), (b, h, dl, lse_ref)
    assert not report.hard, report.hard[:10]
    return report


# ---------------------------------------------------------------------------
# Small and mid-size cases, exhaustively compared
# ---------------------------------------------------------------------------

CASES = {
    "tiny": (W.WORKLOADS["tiny"], 4096),
    "tiny_ragged": (W.WORKLOADS["tiny"], 4091),
    "32k": (W.WORKLOADS["32k"], 32768),
    "256k_small": (W.scaled("256k", n_kv_heads=2, n_q_heads=8, n_tokens=65536, stream_tokens=64), 65536 + 37),
    "deep_small": (W.scaled("deep", n_kv_heads=2, n_q_heads=8, n_tokens=16384, stream_tokens=16), 16384 + 9),
    "1m_small": (W.scaled("1m", n_kv_heads=1, n_q_heads=8, n_tokens=262144, stream_tokens=128,
                          n_needles=4), 262144 + 100),
}


@pytest.mark.parametrize("name", list(CASES))
def test_parity_small_and_mid(zha, parity_log, name):
    spec, n_tokens = CASES[name]
    inp = W.generate(spec)
    rep = check_case(zha, inp, n_tokens)
    parity_log(name, rep)
    print(f"{name}: heads {rep.heads} levels {rep.levels_compared} ties {rep.ties} "
          f"exact heads {len(rep.exact_heads)}")
    assert rep.heads == spec.batch * spec.n_q_heads


@pytest.mark.parametrize("n_tokens", [1, 3, 4, 5, 15, 16, 17, 63, 64, 65, 83, 200, 257])
def test_edge_token_counts(zha, parity_log, n_tokens):
    """C=4, L=3: no chunk, only a tail, exact chunk boundaries, orphans at every level."""
    spec = W.scaled("tiny", chunk=4, levels=3, n_tokens=260, n_needles=0, batch=3)
    inp = W.generate(spec)
    parity_log(f"edge_{n_tokens}", check_case(zha, inp, n_tokens))


@pytest.mark.parametrize("p", [1e-6, 0.3, 0.999])
def test_extreme_p(zha, parity_log, p):
    spec = W.scaled("tiny", n_tokens=2048, n_needles=2, batch=4)
    parity_log(f"p_{p}", check_case(zha, W.generate(spec), 2048 - 3, p=p))


@pytest.mark.parametrize("name", ["tiny_ragged", "256k_small"])
def test_p1_routes_everything_and_equals_dense_attention(zha, name):
    spec, n_tokens = CASES[name]
    if spec.n_kv_heads > 1:
        spec = W.scaled(spec, n_kv_heads=1, n_q_heads=spec.group)
    inp = W.generate(spec)
    res = run_pipeline(zha, inp, n_tokens, p=1.0)
    nb = spec.chunk * (n_tokens // spec.chunk)
    for b in range(spec.batch):
        for h in range(spec.n_q_heads):
            assert list(res["ids"][b, h, : res["cnt"][b, h]]) == list(range(nb // spec.chunk))
            Kf, Vf = cache_f64(inp, 0, n_tokens), values_f64(inp, 0, n_tokens)
            q = inp.Q[0, b, h].astype(np.float64)
            _, dense = O.sdpa(q[None], Kf, Vf)
            assert np.max(np.abs(res["out"][b, h] - dense[0])) <= O_ATOL[spec.kv_dtype]
            assert np.max(np.abs(res["out"][b, h] - dense[0])) <= derived_o_bound(np.abs(Vf).max())


def test_selection_overflow_is_flagged_and_truncated(zha):
    spec = W.scaled("deep", n_kv_heads=1, n_q_heads=4, n_tokens=4096, batch=2)
    inp = W.generate(spec)
    full = run_pipeline(zha, inp, 4096)
    small = run_pipeline(zha, inp, 4096, max_sel=3)
    assert small["status"] & zha.ZHA_DEV_SELECTION_TRUNCATED
    assert np.array_equal(small["cnt"], full["cnt"])
    assert np.array_equal(small["ids"][..., :3], full["ids"][..., :3])


def test_bad_external_selection_is_flagged_not_fatal(zha):
    spec = W.scaled("tiny", n_tokens=1024, n_needles=0, batch=2)
    inp = W.generate(spec)
    K, V, refq, Q = to_device(inp)
    cfg = config_for(spec)
    tree = zha.Tree(cfg, refq)
    tree.build(K, 1024)
    q = Q[0].contiguous()
    ids = torch.tensor([[[5, 3, 70, -1]] * 4] * 2, dtype=torch.int32, device="cuda")
    cnt = torch.full((2, 4), 4, dtype=torch.int32, device="cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    out, lse = tree.sparse_attend(q, K, V, 1024, ids, cnt, status=status)
    torch.cuda.synchronize()
    assert status.item() & zha.ZHA_DEV_BAD_SELECTION
    assert torch.isfinite(out).all() and torch.isfinite(lse).all()


def test_external_selection_parity(zha):
    """sparse_attend on oracle-chosen chunk lists (random sorted subsets)."""
    spec = W.scaled("32k", n_kv_heads=2, n_q_heads=8, n_tokens=8192 + 64)
    inp = W.generate(spec)
    K, V, refq, Q = to_device(inp)
    tree = zha.Tree(config_for(spec), refq)
    n_tokens = 8192 + 40
    rng = np.random.default_rng(11)
    n_ch = n_tokens // spec.chunk
    max_sel = 40
    ids = np.full((spec.batch, spec.n_q_heads, max_sel), -7, np.int32)
    cnt = np.zeros((spec.batch, spec.n_q_heads), np.int32)
    for b in range(spec.batch):
        for h in range(spec.n_q_heads):
            k = int(rng.integers(0, max_sel + 1))
            sel = np.sort(rng.choice(n_ch, size=k, replace=False))
            ids[b, h, :k] = sel
            cnt[b, h] = k
    out, lse = tree.sparse_attend(Q[0].contiguous(), K, V, n_tokens,
                                  torch.from_numpy(ids).cuda(), torch.from_numpy(cnt).cuda())
    out, lse = out.cpu().numpy(), lse.cpu().numpy()
    for b in range(spec.batch):
        for h in range(spec.n_q_heads):
            g = h // spec.group
            S = O.leaf_token_set(ids[b, h, : cnt[b, h]], spec.chunk, n_tokens)
            do, dl, vmax, lse_ref = attend_errors(inp.Q[0, b, h].astype(np.float64),
                                                  cache_f64(inp, g, n_tokens), values_f64(inp, g, n_tokens),
                                                  S, out[b, h], lse[b, h])
            assert do <= derived_o_bound(vmax) and dl <= derived_lse_bound(lse_ref)


def test_append_matches_a_fresh_build_and_the_oracle(zha):
    spec = W.scaled("tiny", chunk=4, levels=3, n_tokens=300, n_needles=0, batch=2, stream_tokens=0)
    inp = W.generate(spec)
    K, V, refq, Q = to_device(inp)
    cfg = config_for(spec)
    inc = zha.Tree(cfg, refq)
    inc.build(K, 37)
    for n in range(38, 300):
        inc.append_chunk(K, n)            # summarises chunks as they complete
    assert inc.built_tokens == 296
    big = zha.Tree(cfg, refq)
    big.build(K, 40)
    big.append_chunk(K, 299)              # many chunks at once: the bulk path
    fresh = zha.Tree(cfg, refq)
    fresh.build(K, 299)
    torch.cuda.synchronize()
    otree = O.build_tree(inp.K[0].astype(np.float64), inp.ref_q[0], 4, 3, 299)
    for lvl in (1, 2, 3):
        n_l = 296 // 4 ** lvl
        for t in (inc, big):
            assert torch.equal(t.level(lvl)[0][:, :n_l], fresh.level(lvl)[0][:, :n_l])
            assert torch.equal(t.level(lvl)[1][:, :n_l], fresh.level(lvl)[1][:, :n_l])
        kh, bh = fresh.level(lvl)
        ek, eb = summary_errors(kh[0, :n_l].cpu().numpy(), bh[0, :n_l].cpu().numpy(), *otree.nodes[lvl])
        assert ek <= SUMMARY_RTOL and eb <= SUMMARY_RTOL
    with pytest.raises(zha.ZhaError) as e:
        inc.append_chunk(K, 200)
    assert e.value.status == zha.ZHA_ERR_STATE


def test_deterministic_and_stream_ordered(zha):
    spec = W.scaled("256k", n_kv_heads=1, n_q_heads=4, n_tokens=16384)
    inp = W.generate(spec)
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        a = run_pipeline(zha, inp, 16384 - 5, stream=s)
        b = run_pipeline(zha, inp, 16384 - 5, stream=s)
    for k in ("cnt", "bits", "out", "lse"):
        assert np.array_equal(a[k], b[k]), k
    for b_ in range(spec.batch):
        for h in range(spec.n_q_heads):
            n = a["cnt"][b_, h]
            assert np.array_equal(a["ids"][b_, h, :n], b["ids"][b_, h, :n])


# ---------------------------------------------------------------------------
# Full-size workloads: sampled nodes and heads
# ---------------------------------------------------------------------------

def _sampled_heads(spec, inp, g, rng, n_random=4):
    """Random heads of KV head g plus every needle head of g (the needles are
    planted for batch 0's queries; they give the narrowest selections)."""
    G = spec.group
    heads = {(b, h) for (b, h, _) in inp.meta.get("needles", []) if h // G == g}
    target = min(spec.batch * G, len(heads) + n_random)
    while len(heads) < target:
        heads.add((int(rng.integers(spec.batch)), g * G + int(rng.integers(G))))
    return sorted(heads)


def _check_sampled(zha, inp, res, g, otree, Kf, Vf, n_tokens, heads, report):
    spec = inp.spec
    kept = kept_from_bits(res["bits"], spec, spec.batch, n_tokens)
    for (b, h) in heads:
        q = inp.Q[0, b, h].astype(np.float64)
        compare_route_head(q, otree, spec.p, {l: kept[l][(b, h)] for l in kept}, report, (b, h))
        n = int(res["cnt"][b, h])
        assert list(res["ids"][b, h, :n]) == list(kept[1][(b, h)])
        S = O.leaf_token_set(res["ids"][b, h, :n], spec.chunk, n_tokens)
        do, dl, vmax, lse_ref = attend_errors(q, Kf, Vf, S, res["out"][b, h], res["lse"][b, h])
        assert do <= O_ATOL[spec.kv_dtype] and do <= derived_o_bound(vmax), (b, h, do)
        assert dl <= derived_lse_bound(lse_ref), (b, h, dl)


@pytest.mark.slow
@pytest.mark.parametrize("key", ["32k", "256k", "deep", "1m"])
def test_parity_full_size_sampled(zha, parity_log, key):
    """The full-size workloads: sampled summaries of every level against the
    direct summary of the raw keys under them, and routing + attention of
    sampled heads (random ones and the needle heads) of one KV head. For the
    1M-context workload the stream then goes on: 101 more tokens through
    zha_append_chunk one token per call (one new chunk: 16385 level-1 nodes,
    so level 1 is routed by the wide-level selection), and the appended node
    and the sampled heads are checked again at the new length."""
    spec = W.WORKLOADS[key]
    inp = W.generate(spec)
    n_tokens = spec.n_tokens
    dev = to_device(inp)
    res = run_pipeline(zha, inp, n_tokens, dev=dev)
    assert res["status"] == 0
    rng = np.random.default_rng(5)
    C = spec.chunk
    g = int(rng.integers(spec.n_kv_heads))
    n_end = n_tokens + (101 if key == "1m" else 0)
    Kf = cache_f64(inp, g, n_end)
    Vf = values_f64(inp, g, n_end)
    # sampled summaries of every level vs the direct summary of the raw keys under them
    for lvl in range(1, spec.levels + 1):
        n_l = n_tokens // C ** lvl
        kh, bh = res["tree"].level(lvl)
        for i in rng.choice(n_l, size=min(n_l, 16 if lvl > 1 else 64), replace=False):
            span = C ** lvl
            kd, bd = O.summarise_chunk(inp.ref_q[g], Kf[i * span:(i + 1) * span])
            ek, eb = summary_errors(kh[g, i].cpu().numpy()[None], bh[g, i].cpu().numpy()[None],
                                    kd[None], bd[None])
            assert ek <= SUMMARY_RTOL and eb <= SUMMARY_RTOL, (lvl, i, ek, eb)
    otree = O.build_tree(Kf[:n_tokens], inp.ref_q[g], C, spec.levels, n_tokens)
    heads = _sampled_heads(spec, inp, g, rng)
    report = RouteReport()
    _check_sampled(zha, inp, res, g, otree, Kf[:n_tokens], Vf[:n_tokens], n_tokens, heads, report)
    assert not report.hard, report.hard[:10]
    parity_log(f"full_{key}", report)
    if key != "1m":
        return
    tree = res["tree"]
    for n in range(n_tokens + 1, n_end + 1):
        tree.append_chunk(dev[0], n)
    assert tree.built_tokens == n_tokens + C
    res2 = run_pipeline(zha, inp, n_end, tree=tree, dev=dev)
    assert res2["status"] == 0
    # the appended level-1 node against the direct summary of its keys; levels
    # 2 and 3 gain no node (their next parents are incomplete)
    i_new = n_tokens // C
    kd, bd = O.summarise_chunk(inp.ref_q[g], Kf[i_new * C:(i_new + 1) * C])
    kh, bh = tree.level(1)
    ek, eb = summary_errors(kh[g, i_new].cpu().numpy()[None], bh[g, i_new].cpu().numpy()[None],
                            kd[None], bd[None])
    assert ek <= SUMMARY_RTOL and eb <= SUMMARY_RTOL, (ek, eb)
    otree2 = O.OracleTree(chunk=C, levels=spec.levels, n_tokens=n_end, qhat=otree.qhat,
                          nodes=dict(otree.nodes))
    otree2.nodes[1] = (np.concatenate([otree.nodes[1][0], kd[None]]),
                       np.concatenate([otree.nodes[1][1], bd[None]]))
    assert otree2.n_nodes(1) == i_new + 1 > 16384
    report2 = RouteReport()
    _check_sampled(zha, inp, res2, g, otree2, Kf, Vf, n_end, heads, report2)
    assert not report2.hard, report2.hard[:10]
    parity_log("full_1m_stream_16385_nodes", report2)


@pytest.mark.parametrize("n_ref,head_dim,kv", [(1, 64, "f32"), (3, 64, "f32"), (16, 64, "bf16"),
                                               (32, 128, "bf16"), (1, 128, "bf16"), (7, 128, "f32")])
def test_reference_query_counts_and_head_dims(zha, n_ref, head_dim, kv):
    """Every plane-count / head-dim variant of the scoring kernel, and both
    attention kernels (tensor cores for bf16 d=128, CUDA cores otherwise)."""
    spec = W.scaled("tiny", n_ref=n_ref, head_dim=head_dim, kv_dtype=kv, n_kv_heads=2, n_q_heads=8,
                    n_tokens=3000, chunk=8, levels=3, batch=5, n_needles=0)
    check_case(zha, W.generate(spec), 2990)


@pytest.mark.gpu
def test_one_group_spread_over_every_cta_matches_dense(zha):
    """One KV head with <= 32 query heads is one attention group; with every
    chunk listed its tiles outnumber the CTAs, so every CTA's span meets the
    group and the combine merges more states than one pass of its warps holds."""
    spec = W.scaled("32k", n_kv_heads=1, n_q_heads=4, n_tokens=40000 + 64, batch=2)
    inp = W.generate(spec)
    K, V, refq, Q = to_device(inp)
    tree = zha.Tree(config_for(spec), refq)
    n_tokens = 40000 + 17
    n_ch = n_tokens // spec.chunk
    ids = torch.arange(n_ch, dtype=torch.int32, device="cuda").repeat(spec.batch, spec.n_q_heads, 1)
    cnt = torch.full((spec.batch, spec.n_q_heads), n_ch, dtype=torch.int32, device="cuda")
    out, lse = tree.sparse_attend(Q[0].contiguous(), K, V, n_tokens, ids.contiguous(), cnt)
    out, lse = out.cpu().numpy(), lse.cpu().numpy()
    Kf, Vf = cache_f64(inp, 0, n_tokens), values_f64(inp, 0, n_tokens)
    for b in range(spec.batch):
        for h in range(spec.n_q_heads):
            q = inp.Q[0, b, h].astype(np.float64)
            _, dense = O.sdpa(q[None], Kf, Vf)
            assert np.max(np.abs(out[b, h] - dense[0])) <= derived_o_bound(np.abs(Vf).max())


@pytest.mark.gpu
def test_more_than_32_queries_per_kv_head(zha):
    """64 query heads per KV head (batch 8 x GQA 8): each KV head's queries
    form two attention groups and two scoring groups."""
    spec = W.scaled("1m", n_kv_heads=2, n_q_heads=16, n_tokens=8192, stream_tokens=128, batch=8,
                    n_needles=2)
    check_case(zha, W.generate(spec), 8192 + 77)


# ---------------------------------------------------------------------------
# Levels wider than 16384 nodes (the wide-level selection) and the incremental
# path of the 1M-context configuration
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("levels,p", [(1, 0.9), (2, 0.9), (2, 0.999)])
def test_levels_wider_than_16384_nodes(zha, parity_log, levels, p):
    """17499 level-1 nodes (C = 4, 69999 tokens). L = 1: every node is a
    candidate (17499 > 16384: scores read from the route workspace). L = 2,
    p = 0.9: ~14.6K candidates (cached in shared memory). L = 2, p = 0.999:
    ~17.4K candidates (not cached)."""
    spec = W.scaled("deep", n_kv_heads=1, n_q_heads=4, n_tokens=70000, levels=levels, batch=2,
                    stream_tokens=0)
    rep = check_case(zha, W.generate(spec), 70000 - 1, p=p)
    parity_log(f"wide_L{levels}_p{p}", rep)


def plane_terms(zha, tree):
    """Views [H, 2, cap, R, d] fp16 of the store's second copy of each level's
    planes (head_dim 128, R = 16; the operand of the tensor-core scoring),
    laid out after the status block as the header documents."""
    cfg = tree.cfg
    H, R, d, C, L = cfg.n_kv_heads, cfg.n_ref, cfg.head_dim, cfg.chunk, cfg.levels
    caps = [cfg.max_tokens // C ** lvl for lvl in range(1, L + 1)]
    sizes = [H * 2 * cap * R * d * 2 for cap in caps]
    off = zha.tree_bytes(cfg) - sum(sizes)
    raw = tree.store.view(torch.uint8)
    out = {}
    for lvl, cap, size in zip(range(1, L + 1), caps, sizes):
        out[lvl] = raw[off: off + size].view(torch.float16).view(H, 2, cap, R, d)
        off += size
    return out


def split_terms(x):
    """Term 0 = x rounded to fp16, term 1 = (x - term 0) rounded to fp16."""
    t0 = x.half()
    return t0, (x - t0.float()).half()


def check_plane_terms(zha, tree, n_tokens):
    """Both fp16 terms of every built node of every level, bit for bit."""
    C = tree.cfg.chunk
    nb = C * (n_tokens // C)
    for lvl, terms in plane_terms(zha, tree).items():
        n_l = nb // C ** lvl
        t0, t1 = split_terms(tree.level(lvl)[0][:, :n_l])
        assert torch.equal(terms[:, 0, :n_l].view(torch.int16), t0.view(torch.int16)), lvl
        assert torch.equal(terms[:, 1, :n_l].view(torch.int16), t1.view(torch.int16)), lvl


def test_append_bf16_d128_c64_r16_matches_the_oracle(zha, parity_log):
    """The incremental build of the 1M-context configuration (bf16 keys,
    head_dim 128, R = 16, C = 64): a tensor-core prefill to an odd chunk count,
    then one chunk per call across a level-2 boundary (fused append kernel),
    6 chunks in one call (the same kernel), and 13 chunks from an odd chunk
    index in one call (the tensor-core level-1 build with c_begin > 0 and a
    tile whose second chunk lies past the new prefix). Every node of every
    level is compared with the oracle and with a fresh build (norm-wise
    relative 1e-4 each); then routing and attention at the final length."""
    C = 64
    spec = W.scaled("1m", n_kv_heads=2, n_q_heads=16, n_tokens=C * 90, stream_tokens=0, levels=2,
                    batch=2, n_needles=2)
    inp = W.generate(spec)
    dev = to_device(inp)
    K, V, refq, Q = dev
    cfg = config_for(spec)
    inc = zha.Tree(cfg, refq)
    inc.build(K, C * 37 + 5)
    for n in range(C * 37 + 6, C * 65 + 4):
        inc.append_chunk(K, n)                   # one chunk at each boundary
    assert inc.built_tokens == C * 65
    inc.append_chunk(K, C * 71 + 2)              # 6 chunks in one call
    assert inc.built_tokens == C * 71
    inc.append_chunk(K, C * 84 + 9)              # 13 chunks from chunk 71 (odd)
    assert inc.built_tokens == C * 84
    n_final = C * 84 + 9
    fresh = zha.Tree(cfg, refq)
    fresh.build(K, n_final)
    torch.cuda.synchronize()
    for g in range(spec.n_kv_heads):
        otree = O.build_tree(cache_f64(inp, g, n_final), inp.ref_q[g], C, spec.levels, n_final)
        for lvl in (1, 2):
            n_l = otree.n_nodes(lvl)
            for t in (inc, fresh):
                kh, bh = t.level(lvl)
                ek, eb = summary_errors(kh[g, :n_l].cpu().numpy().astype(np.float64),
                                        bh[g, :n_l].cpu().numpy().astype(np.float64), *otree.nodes[lvl])
                assert ek <= SUMMARY_RTOL and eb <= SUMMARY_RTOL, (g, lvl, ek, eb)
    for t in (inc, fresh):
        check_plane_terms(zha, t, n_final)
    rep = check_case(zha, inp, n_final, tree=inc, dev=dev)
    parity_log("append_bf16_c64", rep)


@pytest.mark.parametrize("C,levels,c0", [(16, 3, 261), (32, 2, 101), (128, 2, 131)])
def test_tensor_core_build_other_chunk_sizes(zha, parity_log, C, levels, c0):
    """The tensor-core level-1 build at C = 16 (a chunk is half a warp's rows),
    32 (one warp) and 128 (a whole tile), bf16 keys, head_dim 128, R = 16: a
    prefill to an odd chunk count, then 13 chunks in one call from that odd
    chunk (c_begin > 0, a tile partly past the new prefix). Every node of every
    level against the oracle (norm-wise relative 1e-4), then routing and
    attention at the final length. The kernel must have run."""
    spec = W.scaled("1m", n_kv_heads=2, n_q_heads=16, n_tokens=C * (c0 + 14), stream_tokens=0, chunk=C,
                    levels=levels, batch=2, n_needles=2)
    inp = W.generate(spec)
    dev = to_device(inp)
    K, V, refq, Q = dev
    tree = zha.Tree(config_for(spec), refq)
    zha.trace_enable(64, "build_l1_tc")
    try:
        tree.build(K, C * c0 + 3)
        tree.append_chunk(K, C * (c0 + 13) + 7)    # 13 chunks from chunk c0 (odd)
        torch.cuda.synchronize()
        launched = len(zha.trace_records())
    finally:
        zha.trace_enable(0)
    assert launched == 2
    n_final = C * (c0 + 13) + 7
    assert tree.built_tokens == C * (c0 + 13)
    for g in range(spec.n_kv_heads):
        otree = O.build_tree(cache_f64(inp, g, n_final), inp.ref_q[g], C, levels, n_final)
        for lvl in range(1, levels + 1):
            n_l = otree.n_nodes(lvl)
            assert n_l > 0
            kh, bh = tree.level(lvl)
            ek, eb = summary_errors(kh[g, :n_l].cpu().numpy().astype(np.float64),
                                    bh[g, :n_l].cpu().numpy().astype(np.float64), *otree.nodes[lvl])
            assert ek <= SUMMARY_RTOL and eb <= SUMMARY_RTOL, (g, lvl, ek, eb)
    check_plane_terms(zha, tree, n_final)
    rep = check_case(zha, inp, n_final, tree=tree, dev=dev)
    parity_log(f"build_tc_c{C}", rep)


def test_scores_beyond_the_fp16_range_are_recomputed_in_fp32(zha, parity_log):
    """Level scoring on the tensor cores splits each value into two fp16 terms;
    an element of magnitude >= 65520 (fp16 overflow) makes a row's products
    non-finite and the kernel recomputes that row in fp32. Plant such elements
    in level-1 summaries and in one query, route, and compare every level's
    kept set with the oracle's routing over the same summaries."""
    spec = W.scaled("1m", n_kv_heads=1, n_q_heads=8, n_tokens=8192, stream_tokens=64, levels=2, batch=2,
                    n_needles=0)
    inp = W.generate(spec)
    K, V, refq, Q = to_device(inp)
    n_tokens = 8192 + 5
    tree = zha.Tree(config_for(spec), refq)
    tree.build(K, n_tokens)
    kh, _ = tree.level(1)
    kh[0, 3, 2, 5] = 7.0e4                 # one element of one plane
    kh[0, 40, 0, 100] = -2.0e5
    kh[0, 77, :, 17] = 9.0e4               # every plane of a node
    # (a caller that writes planes itself rewrites their fp16 terms too)
    t0, t1 = split_terms(kh)
    terms = plane_terms(zha, tree)[1]
    terms[:, 0] = t0
    terms[:, 1] = t1
    Qm = Q.clone()
    Qm[0, 1, 5] = 1.0e5                    # a query head with an element beyond the range
    torch.cuda.synchronize()
    q = Qm[0].contiguous()
    B = q.shape[0]
    max_sel = n_tokens // spec.chunk
    bits = torch.zeros(zha.route_kept_words(tree.cfg, B, n_tokens) + 1, dtype=torch.int32, device="cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    ids, cnt = tree.route(q, n_tokens, spec.p, max_sel, kept_bits=bits, status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    kept = kept_from_bits(bits.cpu().numpy().view(np.uint32), spec, B, n_tokens)
    otree = O.OracleTree(chunk=spec.chunk, levels=spec.levels, n_tokens=n_tokens, qhat=inp.ref_q[0])
    for lvl in range(1, spec.levels + 1):
        k_l, b_l = tree.level(lvl)
        n_l = otree.n_nodes(lvl)
        otree.nodes[lvl] = (k_l[0, :n_l].cpu().numpy().astype(np.float64),
                            b_l[0, :n_l].cpu().numpy().astype(np.float64))
    qh = Qm[0].cpu().numpy().astype(np.float64)
    report = RouteReport()
    for b in range(B):
        for h in range(spec.n_q_heads):
            compare_route_head(qh[b, h], otree, spec.p, {lvl: kept[lvl][(b, h)] for lvl in kept}, report,
                               (b, h))
    assert not report.hard, report.hard[:10]
    assert report.heads == B * spec.n_q_heads
    parity_log("fp16_range_fallback", report)


def test_build_status_is_clean_and_reaches_the_route(zha):
    """The tree's device status word (build time-outs) starts at zero after a
    build and a route over it reports no bit."""
    spec = W.scaled("1m", n_kv_heads=1, n_q_heads=8, n_tokens=4096, stream_tokens=64, batch=2,
                    n_needles=0)
    inp = W.generate(spec)
    res = run_pipeline(zha, inp, 4096 + 3)
    assert res["status"] == 0
    st = res["tree"].store.view(torch.int32)
    # the 256-byte block after the levels (the fp16 plane terms follow it)
    cfg = res["tree"].cfg
    terms = sum(cfg.n_kv_heads * 2 * (cfg.max_tokens // cfg.chunk ** lvl) * cfg.n_ref * cfg.head_dim * 2
                for lvl in range(1, cfg.levels + 1)) if (cfg.head_dim, cfg.n_ref) == (128, 16) else 0
    off = (zha.tree_bytes(cfg) - terms - 256) // 4
    assert int(st[off].item()) == 0


# ---------------------------------------------------------------------------
# Routing policies: per-level p and fixed-budget top-K [ZHA: 전제와 한계]
# ---------------------------------------------------------------------------

POLICY_CASES = {
    "depth_scaled_p": ("top_p", [0.75 ** (1 / 3)] * 3),
    "per_level_p": ("top_p", [0.95, 0.8, 0.5]),          # levels 1, 2, 3
    "top_k_small": ("top_k", [40, 12, 3]),               # counting path (<= 512 candidates)
    "top_k_wide": ("top_k", [700, 150, 20]),             # radix path at level 1
}


@pytest.mark.parametrize("case", list(POLICY_CASES))
def test_route_policies_match_the_oracle(zha, parity_log, case):
    """zha_route_ex against the oracle's route under the same policy, every
    level of every head (C = 16, L = 3, 65557 tokens, clustered keys)."""
    mode, vals = POLICY_CASES[case]
    spec = W.scaled("256k", n_kv_heads=2, n_q_heads=8, n_tokens=65536, stream_tokens=64)
    inp = W.generate(spec)
    if mode == "top_p":
        gpu_p = zha.top_p_policy(vals)
        oracle_p = O.RoutePolicy(mode="top_p", p={l + 1: float(np.float32(v)) for l, v in enumerate(vals)})
    else:
        gpu_p = zha.top_k_policy(vals)
        oracle_p = O.RoutePolicy(mode="top_k", k={l + 1: v for l, v in enumerate(vals)})
    rep = check_case(zha, inp, 65536 + 21, p=gpu_p, oracle_p=oracle_p)
    parity_log(f"policy_{case}", rep)
    if mode == "top_k":
        res = run_pipeline(zha, inp, 65536 + 21, p=gpu_p)
        assert (res["cnt"] <= vals[0]).all()


# ---------------------------------------------------------------------------
# Rotary positions [ZHA: 무엇과 다른가]: summaries at rotated reference queries,
# the merge's correction term; routing and attention unchanged
# ---------------------------------------------------------------------------

ROPE_CASES = {
    "f32_d64_full": (W.scaled("tiny", n_tokens=3000, chunk=8, levels=3, n_ref=4, batch=3,
                              n_needles=0), 2990, 32, 10000.0),
    "bf16_d128_partial": (W.scaled("1m", n_kv_heads=2, n_q_heads=16, n_tokens=8192, stream_tokens=128,
                                   levels=2, batch=2, n_needles=2), 8192 + 77, 16, 10000.0),
    "bf16_c4_deep": (W.scaled("deep", n_kv_heads=1, n_q_heads=4, n_tokens=4096, levels=4, batch=2,
                              stream_tokens=16), 4096 + 3, 64, 500000.0),
    "bf16_262k_positions": (W.scaled("1m", n_kv_heads=1, n_q_heads=8, n_tokens=262144,
                                     stream_tokens=128, n_needles=4), 262144 + 100, 64, 10000.0),
}


@pytest.mark.parametrize("name", list(ROPE_CASES))
def test_rotary_positions_match_the_oracle(zha, parity_log, name):
    """Every summary of every level against the oracle's build with rotated
    reference queries (norm-wise 1e-4), then routing and attention on that tree."""
    spec, n_tokens, pairs, base = ROPE_CASES[name]
    inp = W.generate(spec)
    dev = to_device(inp)
    tree = zha.Tree(config_for(spec, rope_pairs=pairs, rope_base=base), dev[2])
    tree.build(dev[0], n_tokens)
    build = lambda K, q, C, L, n: O.build_tree_rope(K, q, C, L, n, base, pairs)
    rep = check_case(zha, inp, n_tokens, tree=tree, dev=dev, oracle_build=build)
    parity_log(f"rope_{name}", rep)


def test_rotary_positions_append_matches_the_oracle(zha):
    """Appends with rotary positions (one chunk per call across a level-2
    boundary, then a bulk append) against the oracle's build."""
    spec = W.scaled("1m", n_kv_heads=1, n_q_heads=8, n_tokens=64 * 70, stream_tokens=0, levels=2,
                    batch=2, n_needles=0)
    inp = W.generate(spec)
    K, V, refq, Q = to_device(inp)
    tree = zha.Tree(config_for(spec, rope_pairs=48, rope_base=10000.0), refq)
    tree.build(K, 64 * 61 + 3)
    for n in range(64 * 61 + 4, 64 * 66 + 1):
        tree.append_chunk(K, n)
    tree.append_chunk(K, 64 * 70)                     # 4 chunks in one call
    torch.cuda.synchronize()
    otree = O.build_tree_rope(cache_f64(inp, 0, 64 * 70), inp.ref_q[0], 64, 2, 64 * 70, 10000.0, 48)
    for lvl in (1, 2):
        n_l = otree.n_nodes(lvl)
        kh, bh = tree.level(lvl)
        ek, eb = summary_errors(kh[0, :n_l].cpu().numpy().astype(np.float64),
                                bh[0, :n_l].cpu().numpy().astype(np.float64), *otree.nodes[lvl])
        assert ek <= SUMMARY_RTOL and eb <= SUMMARY_RTOL, (lvl, ek, eb)


# ---------------------------------------------------------------------------
# Routing diagnostics [ZHA: 어떻게 쓰나; 전제와 한계]
# ---------------------------------------------------------------------------

DIAG_CASES = {
    "f32_d64": (W.scaled("tiny", n_tokens=2048, n_needles=2, batch=4), 2048 - 3, 0),
    "bf16_c64": (W.scaled("1m", n_kv_heads=2, n_q_heads=16, n_tokens=8192, stream_tokens=128, levels=2,
                          batch=2, n_needles=2), 8192 + 77, 0),
    "bf16_rope_c4": (W.scaled("deep", n_kv_heads=1, n_q_heads=4, n_tokens=4096, levels=4, batch=2,
                              stream_tokens=16), 4096 + 3, 64),
}


@pytest.mark.parametrize("name", list(DIAG_CASES))
def test_route_diagnostics_match_the_oracle(zha, name):
    """KL(target || estimate) per level and head against the oracle's fp64
    value: |dKL| <= 2e-4 + 2e-3 KL (fp32 log-masses and scores, each within
    ~1e-5 of the oracle's, move KL by a few 1e-5). Plane-usage counts per
    level: identical except for nodes whose two best planes lie within 1e-5
    (counted; each may move one count)."""
    spec, n_tokens, pairs = DIAG_CASES[name]
    inp = W.generate(spec)
    K, V, refq, Q = to_device(inp)
    tree = zha.Tree(config_for(spec, rope_pairs=pairs, rope_base=10000.0), refq)
    tree.build(K, n_tokens)
    kl, usage = tree.diagnostics(Q[0].contiguous(), K, n_tokens)
    torch.cuda.synchronize()
    kl, usage = kl.cpu().numpy(), usage.cpu().numpy()
    G = spec.group
    want = np.zeros_like(usage)
    near = np.zeros(spec.levels, int)
    for g in range(spec.n_kv_heads):
        Kf = cache_f64(inp, g, n_tokens)
        if pairs:
            otree = O.build_tree_rope(Kf, inp.ref_q[g], spec.chunk, spec.levels, n_tokens, 10000.0, pairs)
        else:
            otree = O.build_tree(Kf, inp.ref_q[g], spec.chunk, spec.levels, n_tokens)
        for b in range(spec.batch):
            for h in range(g * G, (g + 1) * G):
                q = inp.Q[0, b, h].astype(np.float64)
                for lvl in range(1, spec.levels + 1):
                    if otree.n_nodes(lvl) == 0:
                        continue
                    ref = O.level_kl(q, Kf, otree, lvl)
                    assert abs(kl[lvl - 1, b, h] - ref) <= 2e-4 + 2e-3 * ref, (lvl, b, h, kl[lvl - 1, b, h], ref)
                    want[lvl - 1] += O.plane_usage(q, otree, lvl)
                    t = np.sort(O.tangent_planes(q, *otree.nodes[lvl]), axis=-1)
                    if t.shape[-1] > 1:
                        near[lvl - 1] += int(np.sum(t[:, -1] - t[:, -2] <= 1e-5))
    for lvl in range(spec.levels):
        assert np.abs(usage[lvl] - want[lvl]).sum() <= 2 * near[lvl], (lvl, usage[lvl], want[lvl], near[lvl])
    assert usage.sum(axis=1)[0] == spec.batch * spec.n_q_heads * (n_tokens // spec.chunk)


# ---------------------------------------------------------------------------
# Paged K/V caches [Attention: "KV cache 를 담는 방식을 바꾼다: PagedAttention,
# 양자화"]: pages of C tokens in a shuffled pool, a block table per KV head
# ---------------------------------------------------------------------------

def _paged(K, V, C, n_visible, seed, extra_pages=7):
    """Pools [n_pages, C, d] holding the first n_visible tokens of each KV head
    in shuffled pages (every other slot, unused pages included, is NaN), and the
    block table [Hkv, max_blocks]."""
    Hkv, cap, d = K.shape
    blocks = -(-cap // C)
    n_pages = Hkv * blocks + extra_pages
    rng = np.random.default_rng(seed)
    table = rng.permutation(n_pages)[: Hkv * blocks].reshape(Hkv, blocks).astype(np.int32)
    Kp = torch.full((n_pages, C, d), float("nan"), dtype=K.dtype, device=K.device)
    Vp = torch.full_like(Kp, float("nan"))
    for g in range(Hkv):
        for b in range(blocks):
            rows = min(C, n_visible - b * C)
            if rows <= 0:
                break
            Kp[int(table[g, b]), :rows] = K[g, b * C: b * C + rows]
            Vp[int(table[g, b]), :rows] = V[g, b * C: b * C + rows]
    return Kp, Vp, torch.from_numpy(table).to(K.device), table


PAGED_CASES = {
    "bf16_c64_tma": (W.scaled("1m", n_kv_heads=2, n_q_heads=16, n_tokens=8192, stream_tokens=128, levels=2,
                              batch=2, n_needles=2), 8192 + 77),
    "bf16_c4_cp_async": (W.scaled("deep", n_kv_heads=1, n_q_heads=4, n_tokens=4096, levels=4, batch=2,
                                  stream_tokens=16), 4096 + 3),
    "f32_d64": (W.scaled("tiny", n_tokens=2048, n_needles=2, batch=4), 2048 - 3),
}


@pytest.mark.parametrize("name", list(PAGED_CASES))
def test_paged_cache_matches_the_oracle_and_the_contiguous_cache(zha, parity_log, name):
    """Tree built from the pages: every summary and the routing against the
    oracle; attention over the pages against the oracle and against the
    contiguous cache's attention on the same selection (same arithmetic)."""
    spec, n_tokens = PAGED_CASES[name]
    inp = W.generate(spec)
    dev = to_device(inp)
    K, V, refq, Q = dev
    Kp, Vp, table, _ = _paged(K, V, spec.chunk, n_tokens, seed=3)
    kv = zha.kv_cache(Kp, Vp, table)
    tree = zha.Tree(config_for(spec), refq)
    tree.build_kv(kv, n_tokens)
    if (tree.cfg.head_dim, tree.cfg.n_ref) == (128, 16):
        check_plane_terms(zha, tree, n_tokens)
    rep = check_case(zha, inp, n_tokens, tree=tree, dev=dev)
    parity_log(f"paged_{name}", rep)
    res = run_pipeline(zha, inp, n_tokens, tree=tree, dev=dev)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    ids = torch.from_numpy(res["ids"]).cuda()
    cnt = torch.from_numpy(res["cnt"]).cuda()
    out, lse = tree.sparse_attend_kv(Q[0].contiguous(), kv, n_tokens, ids, cnt, status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    out, lse = out.cpu().numpy(), lse.cpu().numpy()
    assert np.isfinite(out).all() and np.isfinite(lse).all()
    assert np.max(np.abs(out - res["out"])) <= 1e-6 and np.max(np.abs(lse - res["lse"])) <= 1e-5


def test_paged_append_and_a_page_outside_the_pool(zha):
    """Appends through the block table as pages fill (one chunk per call), then
    an entry naming a page outside the pool: the build marks the tree (the next
    route reports ZHA_DEV_BAD_PAGE), attention over it reports the bit too, and
    every output stays finite."""
    C = 64
    spec = W.scaled("1m", n_kv_heads=1, n_q_heads=8, n_tokens=C * 40, stream_tokens=C * 4, levels=2,
                    batch=2, n_needles=0)
    inp = W.generate(spec)
    K, V, refq, Q = to_device(inp)
    n0, n1 = C * 40 + 5, C * 43 + 9
    Kp, Vp, table_t, table = _paged(K, V, C, n1, seed=8)
    kv = zha.kv_cache(Kp, Vp, table_t)
    tree = zha.Tree(config_for(spec), refq)
    tree.build_kv(kv, n0)
    for n in range(n0 + 1, n1 + 1):
        tree.append_chunk_kv(kv, n)
    fresh = zha.Tree(config_for(spec), refq)
    fresh.build(K, n1)
    torch.cuda.synchronize()
    otree = O.build_tree(cache_f64(inp, 0, n1), inp.ref_q[0], C, 2, n1)
    for lvl in (1, 2):
        n_l = otree.n_nodes(lvl)
        kh, bh = tree.level(lvl)
        ek, eb = summary_errors(kh[0, :n_l].cpu().numpy().astype(np.float64),
                                bh[0, :n_l].cpu().numpy().astype(np.float64), *otree.nodes[lvl])
        assert ek <= SUMMARY_RTOL and eb <= SUMMARY_RTOL, (lvl, ek, eb)
    # a table entry outside the pool
    bad = table_t.clone()
    bad[0, 3] = Kp.shape[0] + 10
    kv_bad = zha.kv_cache(Kp, Vp, bad)
    t2 = zha.Tree(config_for(spec), refq)
    t2.build_kv(kv_bad, n1)
    q = Q[0].contiguous()
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    ids, cnt = t2.route(q, n1, 0.9, n1 // C, status=st)
    torch.cuda.synchronize()
    assert int(st.item()) & zha.ZHA_DEV_BAD_PAGE
    all_ids = torch.arange(n1 // C, dtype=torch.int32, device="cuda").repeat(spec.batch, spec.n_q_heads, 1)
    all_cnt = torch.full((spec.batch, spec.n_q_heads), n1 // C, dtype=torch.int32, device="cuda")
    st2 = torch.zeros(1, dtype=torch.int32, device="cuda")
    out, lse = fresh.sparse_attend_kv(q, kv_bad, n1, all_ids.contiguous(), all_cnt, status=st2)
    torch.cuda.synchronize()
    assert int(st2.item()) & zha.ZHA_DEV_BAD_PAGE
    assert torch.isfinite(out).all() and torch.isfinite(lse).all()


def test_bounded_wait_times_out_cleanly_and_the_next_call_is_clean(zha, parity_log):
    """The level scoring's producer withholds everything (test hook), so its
    consumers' bounded waits (16 polls, ~1 ms) run out with nothing in flight:
    the route returns within the bound with ZHA_DEV_TIMEOUT set. With the hook
    cleared, the next route on the same tree is clean and matches the oracle."""
    import time
    spec = W.scaled("1m", n_kv_heads=1, n_q_heads=8, n_tokens=8192, stream_tokens=64, batch=2,
                    n_needles=0)
    inp = W.generate(spec)
    dev = to_device(inp)
    K, V, refq, Q = dev
    n_tokens = 8192 + 5
    tree = zha.Tree(config_for(spec), refq)
    tree.build(K, n_tokens)
    q = Q[0].contiguous()
    torch.cuda.synchronize()
    assert zha.lib.zha_tree_debug(tree.handle, 16, 1) == zha.ZHA_OK
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    t0 = time.perf_counter()
    tree.route(q, n_tokens, spec.p, n_tokens // spec.chunk, status=st)
    torch.cuda.synchronize()
    elapsed = time.perf_counter() - t0
    assert int(st.item()) & zha.ZHA_DEV_TIMEOUT
    assert elapsed < 5.0
    assert zha.lib.zha_tree_debug(tree.handle, 0, 0) == zha.ZHA_OK
    rep = check_case(zha, inp, n_tokens, tree=tree, dev=dev)       # asserts a zero status
    parity_log("after_timeout", rep)
