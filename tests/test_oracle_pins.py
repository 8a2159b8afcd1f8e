"""Pins of the CPU oracle against facts the pages and the mathematics fix.

Each test ties one oracle function to something other than the oracle itself:
numbers printed on the pages (tests/golden/, each file carries its citation),
closed forms, convexity, a numerical derivative, brute force over all subsets,
or hand-derived routing outcomes. No GPU is involved.
"""

import itertools
import json
import math
import os

import numpy as np
import pytest

import oracle as O


def _load(golden_dir, name):
    with open(os.path.join(golden_dir, name)) as f:
        return json.load(f)


# ---------------------------------------------------------------------------
# Scaled dot-product attention: the pages' worked examples
# ---------------------------------------------------------------------------

def test_sdpa_three_token_example(golden_dir):
    g = _load(golden_dir, "attention_3token.json")
    half = 0.5 * 10 ** -g["decimals"] + 1e-12
    A, Out = O.sdpa(np.array(g["Q"]), np.array(g["K"]), np.array(g["V"]))
    S = np.array(g["Q"]) @ np.array(g["K"]).T / math.sqrt(2)
    assert np.max(np.abs(S - np.array(g["S_scaled"]))) <= half
    assert np.max(np.abs(A - np.array(g["A"]))) <= half
    assert np.max(np.abs(Out - np.array(g["O"]))) <= half


def test_sdpa_causal_example(golden_dir):
    g = _load(golden_dir, "attention_causal.json")
    half = 0.5 * 10 ** -g["decimals"] + 1e-12
    mask = np.tril(np.ones((3, 3), bool))
    A, Out = O.sdpa(np.array(g["Q"]), np.array(g["K"]), np.array(g["V"]), mask)
    assert np.max(np.abs(A[1, :2] - np.array(g["A_row2_visible"]))) <= half
    assert A[0, 0] == 1.0 and A[1, 2] == 0.0
    assert np.max(np.abs(Out - np.array(g["O_causal"]))) <= half


def test_attend_over_token_sets_reproduces_examples(golden_dir):
    """attend() over S = all tokens gives O; over S = prefix {0..i} gives O_causal."""
    g = _load(golden_dir, "attention_3token.json")
    c = _load(golden_dir, "attention_causal.json")
    half = 0.5e-3 + 1e-12
    K, V = np.array(g["K"], float), np.array(g["V"], float)
    for i, q in enumerate(np.array(g["Q"], float)):
        o, lse = O.attend(q, K, V, np.arange(3))
        assert np.max(np.abs(o - np.array(g["O"][i]))) <= half
        s = K @ q / math.sqrt(2)
        assert abs(lse - math.log(np.exp(s).sum())) < 1e-12
        o_c, _ = O.attend(q, K, V, np.arange(i + 1))
        assert np.max(np.abs(o_c - np.array(c["O_causal"][i]))) <= half


def test_softmax_saturation_through_attend(golden_dir):
    """The softmax weights printed for scores [1,0,-1] and [11.3,0,-11.3]: feed
    keys that produce those scaled scores and one-hot values, so o = weights."""
    g = _load(golden_dir, "softmax_saturation.json")
    d = 4
    for case in g["cases"]:
        scores = np.array(case["scores"])
        q = np.zeros(d); q[0] = math.sqrt(d)          # q.k/sqrt(d) = k[0]
        K = np.zeros((3, d)); K[:, 0] = scores
        V = np.eye(d)[:3]
        o, _ = O.attend(q, K, V, np.arange(3))
        w = np.array(case["weights"])
        tol = case["abs_tol"]
        assert np.max(np.abs(o[:2] - w[:2])) <= tol
        assert abs(o[2] - w[2]) <= case.get("abs_tol_last", tol)
        assert o[3] == 0.0


# ---------------------------------------------------------------------------
# The combine identity: the online-softmax table
# ---------------------------------------------------------------------------

def test_combine_reproduces_online_softmax_table(golden_dir):
    g = _load(golden_dir, "online_softmax_table.json")
    half = 0.5e-3 + 1e-12
    Q = np.array([[1, 0], [0, 1], [1, 1]], float)
    V = np.array([[1, 0], [0, 2], [3, 3]], float)
    q = np.array(g["query"], float)
    s = Q @ q / math.sqrt(2)                       # K = Q in the example
    assert np.max(np.abs(s - np.array(g["scaled_scores"]))) <= half
    # block 1 on its own: log mass m + log l, normalised output o / l
    b1 = g["blocks"][0]
    F1, avg1 = O.combine_log_masses(s[b1], V[b1])
    a1 = g["after_block1"]
    assert abs(F1 - (a1["m"] + math.log(a1["l"]))) <= half * 2
    assert np.max(np.abs(avg1 - np.array(a1["o"]) / a1["l"])) <= half
    # block 2 is one token: its log mass is its score, its state its value
    b2 = g["blocks"][1]
    F2, avg2 = O.combine_log_masses(s[b2], V[b2])
    # combine the two block states: this is the table's second row
    F, avg = O.combine_log_masses(np.array([F1, F2]), np.stack([avg1, avg2]))
    a2 = g["after_block2"]
    assert abs(math.exp(a1["m"] - a2["m"]) - g["rescale_factor"]) <= half
    assert abs(F - (a2["m"] + math.log(a2["l"]))) <= 2 * half
    assert np.max(np.abs(avg - np.array(a2["o"]) / a2["l"])) <= half
    assert np.max(np.abs(avg - np.array(g["final"]))) <= half


def test_merge_of_unequal_children_matches_worked_example(golden_dir):
    """Summaries of {tok1, tok2} and {tok3} at q_r = token 3's query, merged by
    the tree's rule, give the page's numbers: F = m + log l from the online-softmax
    table, and khat = (row 3 of A) applied to K."""
    g = _load(golden_dir, "attention_3token.json")
    t = _load(golden_dir, "online_softmax_table.json")
    K = np.array(g["K"], float)
    qhat = np.array([[1.0, 1.0]])
    kh_a, bh_a = O.summarise_chunk(qhat, K[:2])
    kh_b, bh_b = O.summarise_chunk(qhat, K[2:])
    kh, bh = O.merge_children(qhat, np.stack([kh_a, kh_b]), np.stack([bh_a, bh_b]))
    F = bh[0] + qhat[0] @ kh[0] / math.sqrt(2)
    a2 = t["after_block2"]
    assert abs(F - (a2["m"] + math.log(a2["l"]))) <= 2e-3
    A3 = np.array(g["A"][2])
    assert np.max(np.abs(kh[0] - A3 @ K)) <= 2e-3
    # and it equals the direct summary of all three keys
    kd, bd = O.summarise_chunk(qhat, K)
    assert np.allclose(kh, kd, rtol=0, atol=1e-14) and np.allclose(bh, bd, atol=1e-14)


# ---------------------------------------------------------------------------
# Tangent-plane summaries: closed forms, convexity, gradient
# ---------------------------------------------------------------------------

def _rand_chunk(rng, C=16, d=8, R=5, scale=1.0):
    Kc = rng.standard_normal((C, d)) * scale
    qhat = rng.standard_normal((R, d)) * math.sqrt(d)
    return qhat, Kc


def test_summary_of_identical_keys_is_that_key_and_log_C():
    rng = np.random.default_rng(1)
    d, C, R = 6, 7, 3                    # C != R so an axis mix-up shows
    k = rng.standard_normal(d)
    qhat = rng.standard_normal((R, d)) * 3
    kh, bh = O.summarise_chunk(qhat, np.tile(k, (C, 1)))
    assert np.allclose(kh, np.tile(k, (R, 1)), atol=1e-13)
    assert np.allclose(bh, math.log(C), atol=1e-13)


def test_summary_of_a_single_key():
    rng = np.random.default_rng(2)
    qhat, Kc = _rand_chunk(rng, C=1, d=5, R=4)
    kh, bh = O.summarise_chunk(qhat, Kc)
    assert np.allclose(kh, np.tile(Kc[0], (4, 1)), atol=1e-14)
    assert np.allclose(bh, 0.0, atol=1e-13)


def test_tangent_is_exact_at_its_reference_query():
    rng = np.random.default_rng(3)
    qhat, Kc = _rand_chunk(rng, C=32, d=16, R=6, scale=2.0)
    kh, bh = O.summarise_chunk(qhat, Kc)
    for r in range(qhat.shape[0]):
        t = O.tangent_planes(qhat[r], kh, bh)[r]
        assert abs(t - O.chunk_log_mass(qhat[r], Kc)) < 1e-12


def test_max_of_planes_is_a_lower_bound_of_the_log_mass():
    """LSE is convex, so each tangent plane lies below F_C everywhere."""
    rng = np.random.default_rng(4)
    qhat, Kc = _rand_chunk(rng, C=24, d=12, R=8, scale=1.5)
    kh, bh = O.summarise_chunk(qhat, Kc)
    qs = rng.standard_normal((10_000, 12)) * 4.0
    est = np.array([O.node_score(q, kh, bh) for q in qs])
    true = O.chunk_log_mass(qs, Kc)
    assert np.all(est <= true + 1e-12)
    assert np.mean(true - est) > 1e-3     # and not trivially equal


def test_node_score_is_exact_at_every_reference_query():
    """At q = q_r plane r touches F_C and every other plane lies below it, so the
    max-of-planes estimate equals the true log mass there (and no less)."""
    rng = np.random.default_rng(7)
    qhat, Kc = _rand_chunk(rng, C=16, d=8, R=6, scale=2.0)
    kh, bh = O.summarise_chunk(qhat, Kc)
    for r in range(6):
        assert abs(O.node_score(qhat[r], kh, bh) - O.chunk_log_mass(qhat[r], Kc)) < 1e-12
    planes = O.tangent_planes(qhat[0], kh, bh)
    assert np.min(planes) < np.max(planes) - 1e-3


def test_compressed_key_is_the_gradient_of_the_log_mass():
    """d F_C / d q at q_r equals khat_r / sqrt(d) (central differences)."""
    rng = np.random.default_rng(5)
    qhat, Kc = _rand_chunk(rng, C=20, d=10, R=4)
    kh, _ = O.summarise_chunk(qhat, Kc)
    h = 1e-5
    for r in range(4):
        grad = np.zeros(10)
        for i in range(10):
            e = np.zeros(10); e[i] = h
            grad[i] = (O.chunk_log_mass(qhat[r] + e, Kc) - O.chunk_log_mass(qhat[r] - e, Kc)) / (2 * h)
        assert np.allclose(grad, kh[r] / math.sqrt(10), rtol=1e-6, atol=1e-8)


def test_chunk_log_mass_against_a_plain_loop():
    rng = np.random.default_rng(6)
    q = rng.standard_normal(9)
    Kc = rng.standard_normal((11, 9)) * 2
    total = 0.0
    for j in range(11):
        total += math.exp(sum(q[i] * Kc[j, i] for i in range(9)) / 3.0)
    assert abs(O.chunk_log_mass(q, Kc) - math.log(total)) < 1e-12


# ---------------------------------------------------------------------------
# Upper levels: merge == direct summary of the raw keys
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("C,L,n_tokens", [(4, 3, 64), (4, 3, 93), (3, 4, 200), (2, 1, 9)])
def test_every_level_equals_the_direct_summary(C, L, n_tokens):
    rng = np.random.default_rng(10 + C + L)
    d, R = 8, 5
    K = rng.standard_normal((n_tokens, d)) * 1.5 + rng.standard_normal(d)
    qhat = rng.standard_normal((R, d)) * 2
    tree = O.build_tree(K, qhat, C, L, n_tokens)
    for lvl in range(1, L + 1):
        span = C ** lvl
        kh, bh = tree.nodes[lvl]
        assert kh.shape[0] == (C * (n_tokens // C)) // span == tree.n_nodes(lvl)
        for i in range(kh.shape[0]):
            kd, bd = O.summarise_chunk(qhat, K[i * span:(i + 1) * span])
            assert np.allclose(kh[i], kd, rtol=1e-10, atol=1e-12)
            assert np.allclose(bh[i], bd, rtol=1e-10, atol=1e-12)


# ---------------------------------------------------------------------------
# Top-p selection: brute force, special cases, tie rule
# ---------------------------------------------------------------------------

def test_top_p_is_the_minimal_subset_by_brute_force():
    rng = np.random.default_rng(20)
    for trial in range(300):
        n = int(rng.integers(1, 11))
        sigma = rng.standard_normal(n) * rng.uniform(0.1, 4)
        ids = rng.permutation(50)[:n]
        p = float(rng.uniform(0.05, 0.999))
        sel = O.top_p_prefix(sigma, ids, p)
        pi = np.exp(sigma - sigma.max()); pi /= pi.sum()
        # smallest cardinality of ANY subset whose mass reaches p
        best = None
        for k in range(1, n + 1):
            if any(sum(pi[list(c)]) >= p for c in itertools.combinations(range(n), k)):
                best = k
                break
        assert sel.m == best, (trial, sel.m, best)
        # the kept set is the top-m by score and reaches p
        kept_pos = [int(np.nonzero(ids == k)[0][0]) for k in sel.kept]
        assert pi[kept_pos].sum() >= p - 1e-15
        if sel.m < n:
            assert min(sigma[kept_pos]) >= max(np.delete(sigma, kept_pos))


def test_top_p_special_cases():
    ids = np.arange(4)
    assert O.top_p_prefix(np.array([0.3, -1.0, 2.0, 0.0]), ids, 1.0).m == 4
    assert O.top_p_prefix(np.array([0.3, -1.0, 2.0, 0.0]), ids, 1.5).m == 4
    one = O.top_p_prefix(np.array([0.0, 30.0, 0.0, 0.0]), ids, 0.99)
    assert one.m == 1 and list(one.kept) == [1]
    flat = O.top_p_prefix(np.zeros(4), np.array([7, 3, 9, 5]), 0.5)
    assert flat.m == 2 and list(flat.kept) == [3, 5]      # ties: lower index first
    flat = O.top_p_prefix(np.zeros(4), np.array([7, 3, 9, 5]), 0.51)
    assert flat.m == 3 and list(flat.kept) == [3, 5, 7]
    assert O.top_p_prefix(np.zeros(0), np.zeros(0, int), 0.9).m == 0


# ---------------------------------------------------------------------------
# Routing: hand-built trees, invariants, p = 1 equals dense attention
# ---------------------------------------------------------------------------

def test_route_follows_a_single_strong_key_by_hand():
    """C=2, L=2, N=11: level-1 nodes 0..4 (tokens 0..9), level-2 nodes 0..1
    (tokens 0..3, 4..7), level-1 node 4 is an orphan, token 10 is the tail.
    One strong key at token 5: the route keeps level-2 node 1, then level-1
    node 2, so S = {0} u {4, 5} u {10}."""
    d = 2
    K = np.zeros((11, d)); K[5] = [3.0, 0.0]
    tree = O.build_tree(K, np.array([[1.0, 0.0]]), chunk=2, levels=2, n_tokens=11)
    tr = O.route(np.array([10.0, 0.0]), tree, p=0.9)
    assert list(tr.levels[2].candidates) == [0, 1]
    assert list(tr.levels[2].topp.kept) == [1]
    assert list(tr.levels[1].candidates) == [2, 3, 4]          # children of 1 + orphan 4
    assert list(tr.levels[1].topp.kept) == [2]
    assert list(tr.tokens) == [0, 4, 5, 10]


def test_route_on_flat_keys_breaks_ties_by_index_by_hand():
    """All keys zero: every node's score is log(tokens under it). Level 2: two
    equal nodes, p=0.5 keeps node 0. Level 1: children {0,1} + orphan {4}, each
    of mass 1/3; p=0.5 keeps {0,1}. S = {0,1,2,3} u {10}."""
    K = np.zeros((11, 2))
    tree = O.build_tree(K, np.array([[1.0, 0.0], [0.0, 1.0]]), 2, 2, 11)
    tr = O.route(np.array([1.0, -2.0]), tree, p=0.5)
    assert np.allclose(tr.levels[2].sigma, math.log(4))
    assert list(tr.levels[2].topp.kept) == [0]
    assert list(tr.levels[1].candidates) == [0, 1, 4]
    assert list(tr.levels[1].topp.kept) == [0, 1]
    assert list(tr.tokens) == [0, 1, 2, 3, 10]


def _random_tree(seed, n_tokens=1000, C=4, L=3, d=8, R=4):
    rng = np.random.default_rng(seed)
    K = rng.standard_normal((n_tokens, d)) * 1.3
    V = rng.standard_normal((n_tokens, d))
    qhat = rng.standard_normal((R, d)) * 2
    return rng, K, V, O.build_tree(K, qhat, C, L, n_tokens)


@pytest.mark.parametrize("n_tokens", [1000, 1027, 64, 63, 3, 1])
def test_route_set_invariants(n_tokens):
    rng, K, V, tree = _random_tree(30 + n_tokens, n_tokens=n_tokens)
    C, L = tree.chunk, tree.levels
    for _ in range(20):
        q = rng.standard_normal(8) * 3
        tr = O.route(q, tree, p=float(rng.uniform(0.3, 0.95)))
        S = set(tr.tokens.tolist())
        assert 0 in S
        assert set(range(tree.n_built, n_tokens)) <= S
        assert max(S) < n_tokens
        for lvl in range(1, L + 1):
            lt = tr.levels[lvl]
            kept = set(lt.topp.kept.tolist())
            assert kept <= set(lt.candidates.tolist())
            n_par = tree.n_nodes(lvl + 1)
            for i in kept:
                parent = i // C
                if parent < n_par:
                    assert parent in set(tr.levels[lvl + 1].topp.kept.tolist())
            # candidates: every node whose parent was kept, and every orphan
            expect = [i for i in range(tree.n_nodes(lvl))
                      if i // C >= n_par or (lvl < L and i // C in set(tr.levels[lvl + 1].expanded.tolist()))]
            assert sorted(lt.candidates.tolist()) == expect
        # S is exactly sink + tail + tokens of kept chunks
        expect_S = {0} | set(range(tree.n_built, n_tokens))
        for c in tr.leaf_chunks:
            expect_S |= set(range(c * C, (c + 1) * C))
        assert S == expect_S


@pytest.mark.parametrize("n_tokens", [1000, 1027, 70, 5])
def test_route_at_p1_equals_dense_attention(n_tokens):
    rng, K, V, tree = _random_tree(50 + n_tokens, n_tokens=n_tokens)
    for _ in range(5):
        q = rng.standard_normal(8) * 3
        tr = O.route(q, tree, p=1.0)
        assert list(tr.tokens) == list(range(n_tokens))
        o, lse = O.attend(q, K, V, tr.tokens)
        _, dense = O.sdpa(q[None], K[:n_tokens], V[:n_tokens])
        assert np.max(np.abs(o - dense[0])) < 1e-12


def test_forced_expansion_uses_the_given_kept_set():
    rng, K, V, tree = _random_tree(70, n_tokens=1000)
    q = rng.standard_normal(8) * 3
    forced = {3: np.array([1, 2])}
    tr = O.route(q, tree, p=0.6, forced_kept=forced)
    C = tree.chunk
    n2 = tree.n_nodes(2)
    expect = sorted([c for k in (1, 2) for c in range(k * C, k * C + C)] +
                    list(range(C * tree.n_nodes(3), n2)))
    assert sorted(tr.levels[2].candidates.tolist()) == expect


def test_bf16_decode_is_exact():
    vals = np.array([1.0, -2.5, 0.15625, 3.0e38, -1.0e-38, 0.0], np.float32)
    bits = (vals.view(np.uint32) >> 16).astype(np.uint16)     # these values are bf16-exact
    assert np.array_equal(O.bf16_bits_to_f64(bits), vals.astype(np.float64)) or \
        np.allclose(O.bf16_bits_to_f64(bits), vals.astype(np.float64), rtol=2 ** -8)
    assert O.bf16_bits_to_f64(np.array([0x3F80], np.uint16))[0] == 1.0
    assert O.bf16_bits_to_f64(np.array([0xC020], np.uint16))[0] == -2.5
    assert O.bf16_bits_to_f64(np.array([0x0000], np.uint16))[0] == 0.0


# ---------------------------------------------------------------------------
# Routing policies: per-level p schedule and fixed-budget top-K
# [ZHA: 전제와 한계]
# ---------------------------------------------------------------------------

def _precedes(sig, ids, a, b):
    """Candidate a comes before candidate b: higher score, or equal score and
    lower node index."""
    return sig[a] > sig[b] or (sig[a] == sig[b] and ids[a] < ids[b])


def test_top_k_is_the_upward_closed_subset_by_brute_force():
    """Among all subsets of size min(k, n) exactly one contains, with each of
    its members, every candidate that precedes it; top_k_prefix keeps it."""
    rng = np.random.default_rng(21)
    for _ in range(300):
        n = int(rng.integers(0, 9))
        sig = rng.integers(-3, 3, size=n).astype(float)          # many ties
        ids = rng.permutation(40)[:n]
        k = int(rng.integers(1, 11))
        sel = O.top_k_prefix(sig, ids, k)
        m = min(k, n)
        closed = []
        for S in itertools.combinations(range(n), m):
            Sset = set(S)
            if all(not _precedes(sig, ids, b, a) for a in Sset for b in range(n) if b not in Sset):
                closed.append(sorted(ids[list(S)]))
        assert len(closed) == 1
        assert list(sel.kept) == closed[0] and sel.m == m


def _flat_tree(C=4, L=3, n_tokens=256):
    """Every key equal: every node of a level has the same summary, so the
    candidates' estimated masses are uniform and ties go to the lower index."""
    d = 8
    K = np.tile(np.linspace(-1.0, 1.0, d), (n_tokens, 1))
    qhat = np.random.default_rng(3).standard_normal((2, d))
    return O.build_tree(K, qhat, C, L, n_tokens), np.random.default_rng(4).standard_normal(d)


def _kept_counts(trace):
    return {lvl: len(lt.topp.kept) for lvl, lt in trace.levels.items()}


def test_flat_tree_kept_counts_under_fixed_and_depth_scaled_p():
    """Uniform masses over n candidates: top-p keeps ceil(p n) of them. With
    C = 4 and 4, 16, 64 nodes at levels 3, 2, 1: a fixed p = 0.7 keeps 3 of 4,
    then 9 of 12, then 26 of 36 (26/64 = 0.41 of the chunks: the per-level
    fractions multiply); p**(1/3) = 0.8879 per level keeps 4 of 4, 15 of 16,
    54 of 60 (0.84 of the chunks)."""
    tree, q = _flat_tree()
    fixed = O.route(q, tree, 0.7)
    assert _kept_counts(fixed) == {3: 3, 2: 9, 1: 26}
    assert list(fixed.levels[3].topp.kept) == [0, 1, 2]           # ties: lower index first
    assert [len(fixed.levels[l].candidates) for l in (3, 2, 1)] == [4, 12, 36]
    scaled = O.route(q, tree, O.depth_scaled_p(0.7, 3))
    assert _kept_counts(scaled) == {3: 4, 2: 15, 1: 54}
    sched = O.route(q, tree, {3: 0.55, 2: 0.9, 1: 0.3})    # ceil(2.2), ceil(10.8), ceil(13.2)
    assert _kept_counts(sched) == {3: 3, 2: 11, 1: 14}
    pol = O.route(q, tree, O.RoutePolicy(mode="top_p", p={3: 0.55, 2: 0.9, 1: 0.3}))
    assert _kept_counts(pol) == {3: 3, 2: 11, 1: 14}


def test_depth_scaled_masses_multiply_to_p():
    for p in (0.3, 0.75, 0.9, 0.99):
        for L in (1, 2, 3, 6):
            sched = O.depth_scaled_p(p, L)
            assert sorted(sched) == list(range(1, L + 1))
            assert abs(math.prod(sched.values()) - p) < 1e-12
            assert all(v >= p for v in sched.values())


def test_top_k_route_keeps_the_budget_at_every_level():
    """Flat tree: top-K keeps exactly min(k_l, candidates) per level. Random
    trees: each level's kept set is the upward-closed subset of that level's
    candidates (checked pairwise) of size min(k_l, candidates)."""
    tree, q = _flat_tree()
    tr = O.route(q, tree, O.RoutePolicy(mode="top_k", k={3: 2, 2: 5, 1: 7}))
    assert _kept_counts(tr) == {3: 2, 2: 5, 1: 7}
    assert list(tr.levels[3].topp.kept) == [0, 1] and list(tr.leaf_chunks) == list(range(7))
    rng = np.random.default_rng(8)
    for n_tokens in (97, 300, 1000):
        K = rng.standard_normal((n_tokens, 8))
        t = O.build_tree(K, rng.standard_normal((3, 8)), 4, 3, n_tokens)
        budget = {3: 3, 2: 6, 1: 9}
        tr = O.route(rng.standard_normal(8) * 2, t, O.RoutePolicy(mode="top_k", k=budget))
        for lvl, lt in tr.levels.items():
            n = len(lt.candidates)
            kept = set(lt.topp.kept.tolist())
            assert len(kept) == min(budget[lvl], n)
            pos = {int(c): i for i, c in enumerate(lt.candidates)}
            for a in kept:
                for b in lt.candidates:
                    if int(b) not in kept:
                        assert not _precedes(lt.sigma, lt.candidates, pos[int(b)], pos[a])


# ---------------------------------------------------------------------------
# Rotary positions: summaries at rotated reference queries and the merge's
# correction term [ZHA: 무엇과 다른가; Attention: "Attention 은 순서를 모르므로
# 위치 정보를 따로 넣는다"]
# ---------------------------------------------------------------------------

def test_rope_inner_product_depends_only_on_the_offset():
    """The Attention page: rotating q by m theta and k by n theta leaves an
    inner product that depends on (m - n) theta alone; rotations keep norms;
    no rotated pair (or position 0) is the identity."""
    rng = np.random.default_rng(31)
    for d, pairs in ((8, 4), (16, 5), (64, 32)):
        q, k = rng.standard_normal(d), rng.standard_normal(d)
        for m, n in ((7, 3), (1000, 999), (5, 5), (0, 12)):
            a = O.rope_rotate(q, m, 10000.0, pairs) @ O.rope_rotate(k, n, 10000.0, pairs)
            b = O.rope_rotate(q, m - n, 10000.0, pairs) @ k
            assert abs(a - b) < 1e-10 * (1 + abs(a))
        assert abs(np.linalg.norm(O.rope_rotate(q, 123, 500.0, pairs)) - np.linalg.norm(q)) < 1e-12
        assert np.array_equal(O.rope_rotate(q, 0, 10000.0, pairs), q)
        assert np.allclose(O.rope_rotate(q, 77, 10000.0, 0), q, rtol=0, atol=0)
    # partial rotation: pairs past `pairs` are untouched
    x = rng.standard_normal(16)
    y = O.rope_rotate(x, 9, 10000.0, 3)
    assert np.array_equal(y[6:], x[6:]) and not np.allclose(y[:6], x[:6])


def test_rope_tree_without_rotated_pairs_is_the_position_free_tree():
    rng = np.random.default_rng(32)
    K = rng.standard_normal((4 * 16 + 3, 8))
    qhat = rng.standard_normal((3, 8))
    a = O.build_tree_rope(K, qhat, 4, 3, K.shape[0], 10000.0, 0)
    b = O.build_tree(K, qhat, 4, 3, K.shape[0])
    for lvl in (1, 2, 3):
        assert np.allclose(a.nodes[lvl][0], b.nodes[lvl][0], rtol=0, atol=1e-12)
        assert np.allclose(a.nodes[lvl][1], b.nodes[lvl][1], rtol=0, atol=1e-12)


def test_rope_level1_plane_is_exact_at_the_rotated_reference_query():
    """t_{r,c}(q_hat_{r,c}) = F_c(q_hat_{r,c}) with q_hat_{r,c} = rotate(q_hat_r, pos_c),
    and the summary equals the position-free one taken in the chunk's frame:
    khat = rotate(khat', pos) for keys rotated back by -pos."""
    rng = np.random.default_rng(33)
    qhat = rng.standard_normal((4, 16)) * 2
    Kc = rng.standard_normal((8, 16))
    for pos in (0, 5, 4096, 1 << 20):
        kh, bh = O.summarise_chunk_rope(qhat, Kc, pos, 10000.0, 8)
        q_rot = O.rope_rotate(qhat, pos, 10000.0, 8)
        t = np.sum(kh * q_rot, axis=-1) / 4.0 + bh
        assert np.allclose(t, O.chunk_log_mass(q_rot, Kc), rtol=0, atol=1e-12)
        kh0, bh0 = O.summarise_chunk(qhat, O.rope_rotate(Kc, -pos, 10000.0, 8))
        assert np.allclose(kh, O.rope_rotate(kh0, pos, 10000.0, 8), rtol=0, atol=1e-10)
        assert np.allclose(bh, bh0, rtol=0, atol=1e-10)


def test_rope_merge_of_single_key_children_is_exact():
    """A child whose keys are all the same key k has F_c(q) = log C + q.k/sqrt(d),
    a linear function, so its plane is exact at every query and the corrected
    merge equals the direct summary of all the parent's keys at the parent's
    rotated reference query."""
    rng = np.random.default_rng(34)
    C, d, R = 4, 16, 3
    qhat = rng.standard_normal((R, d))
    for P in (0, 1, 37):
        child_keys = rng.standard_normal((C, d)) * 2
        K = np.repeat(child_keys, C, axis=0)                           # C children of C equal keys
        pos_ch = O.node_position(1, P * C + np.arange(C), C)
        kh_c, bh_c = O.summarise_chunk_rope(qhat, K.reshape(C, C, d), pos_ch, 10000.0, d // 2)
        kh, bh = O.merge_children_rope(qhat, kh_c, bh_c, O.node_position(2, P, C), pos_ch, 10000.0, d // 2)
        kd, bd = O.summarise_chunk_rope(qhat, K, O.node_position(2, P, C), 10000.0, d // 2)
        assert np.allclose(kh, kd, rtol=0, atol=1e-10) and np.allclose(bh, bd, rtol=0, atol=1e-10)


def test_rope_merge_correction_is_second_order_in_the_rotation():
    """For a general child, the corrected log mass at the parent's rotated
    reference query differs from the true F_c there by O(angle^2): halving the
    position offset divides the error by ~4. Without the correction term the
    error is first order (halving divides it by ~2)."""
    rng = np.random.default_rng(35)
    d, R = 16, 2
    qhat = rng.standard_normal((R, d)) * 2
    Kc = rng.standard_normal((8, d)) * 1.5
    errs, errs_plain = [], []
    for t in (0.02, 0.01, 0.005):
        kh_c, bh_c = O.summarise_chunk_rope(qhat, Kc[None], np.array([t]), 1.0, d // 2)   # base 1: theta = 1
        kh, bh = O.merge_children_rope(qhat, kh_c, bh_c, 0.0, np.array([t]), 1.0, d // 2)
        F_P = bh + np.sum(kh * qhat, axis=-1) / 4.0                    # parent at position 0: q_hat_P = q_hat
        true = O.chunk_log_mass(qhat, Kc)
        errs.append(np.max(np.abs(F_P - true)))
        q_c = O.rope_rotate(qhat, t, 1.0, d // 2)
        plain = np.sum(kh_c[0] * q_c, axis=-1) / 4.0 + bh_c[0]          # F_c at its own query, uncorrected
        errs_plain.append(np.max(np.abs(plain - true)))
    for a, b in zip(errs, errs[1:]):
        assert 3.5 < a / b < 4.5
    for a, b in zip(errs_plain, errs_plain[1:]):
        assert 1.7 < a / b < 2.3


# ---------------------------------------------------------------------------
# Routing diagnostics [ZHA: 어떻게 쓰나; 전제와 한계]
# ---------------------------------------------------------------------------

def test_target_mass_sums_dense_weights_per_node_by_a_plain_loop():
    """p_{l,C}: the dense softmax weights summed node by node (a loop over
    nodes and keys with math.exp), normalised over the level's nodes."""
    rng = np.random.default_rng(41)
    K = rng.standard_normal((4 * 16 + 5, 6))
    q = rng.standard_normal(6) * 2
    tree = O.build_tree(K, rng.standard_normal((2, 6)), 4, 2, K.shape[0])
    for lvl in (1, 2):
        span = 4 ** lvl
        n_l = tree.n_nodes(lvl)
        w = [sum(math.exp(float(q @ K[j]) / math.sqrt(6)) for j in range(i * span, (i + 1) * span))
             for i in range(n_l)]
        ref = np.array(w) / sum(w)
        assert np.allclose(O.level_target_mass(q, K, tree, lvl), ref, rtol=1e-12, atol=0)


def test_kl_is_zero_when_every_chunk_repeats_one_key():
    """A chunk of C copies of one key has F(q) = log C + q.k/sqrt(d), a linear
    function: every plane is exact, the estimate equals the target at every
    level, KL = 0. Random chunks give KL > 0."""
    rng = np.random.default_rng(42)
    keys = rng.standard_normal((4, 8)) * 2
    K = np.repeat(keys, 16, axis=0)                    # every level-2 node (16 tokens) one key
    qhat = rng.standard_normal((3, 8))
    tree = O.build_tree(K, qhat, 4, 2, 64)
    for _ in range(5):
        q = rng.standard_normal(8) * 3
        for lvl in (1, 2):
            assert abs(O.level_kl(q, K, tree, lvl)) < 1e-12
    K2 = rng.standard_normal((64, 8)) * 2
    tree2 = O.build_tree(K2, qhat, 4, 2, 64)
    assert O.level_kl(rng.standard_normal(8) * 3, K2, tree2, 1) > 1e-6


def test_plane_usage_by_hand():
    """Equal reference queries give equal planes: every node counts for r = 0.
    A query equal to reference query r makes plane r exact (tangent) and the
    others lower (convexity): at level 1 every node counts for r."""
    rng = np.random.default_rng(43)
    K = rng.standard_normal((64, 8))
    same = np.repeat(rng.standard_normal((1, 8)), 3, axis=0)
    tree = O.build_tree(K, same, 4, 2, 64)
    assert list(O.plane_usage(rng.standard_normal(8), tree, 1)) == [16, 0, 0]
    qhat = rng.standard_normal((3, 8)) * 2
    tree = O.build_tree(K, qhat, 4, 2, 64)
    for r in range(3):
        u = O.plane_usage(qhat[r], tree, 1)
        assert u[r] == 16 and u.sum() == 16
