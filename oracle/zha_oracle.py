"""Plain fp64 CPU oracle of the ZHA decode hot path -- TEST INFRASTRUCTURE.

Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py`` (its ``cpu_baseline``
leg and ``--impl reference`` arm) may import this module. It is slow on purpose:
each function writes out what the pages define, in fp64, with numpy library
primitives (matmul, sort, cumulative sum) as its only building blocks and no
blocking, fusion or reordering beyond the definitions.

Citations
---------
[ZHA: <section>]  page "ZHA는 KV 캐시를 트리로 요약해 어텐션 비용을 준(sub)이차로 낮춘다"
                  (onedev.kr/papers/1556), the named section:
                  "무엇과 다른가" (what differs: summaries, merge, GQA, schedule),
                  "전제와 한계" (assumptions and limits: top-p routing, sink, tail).
[Attention: <section>]  page "Attention"
                  (zzong2006.github.io/machine_learning/nlp/attention-function),
                  the named section: "Scaled dot-product attention 의 식",
                  "토큰 세 개로 직접 계산하기" (3-token worked example),
                  "Causal mask 는 뒤에 오는 토큰을 가린다",
                  "같은 계산을 메모리 IO 를 줄여서 한다: FlashAttention 계열"
                  (online-softmax table), "Attention 은 순서를 모르므로 위치
                  정보를 따로 넣는다" (RoPE).
[ASM: 방법론]     page "효율적인 긴 컨텍스트 생성을 위한 컨텍스트 기억화"
                  (aitrends.kr/articles/59378), section "방법론": the merge of two
                  attention states, used only as a second statement of the identity
                  behind ``combine_log_masses``.

Readings taken where the pages are silent:
  * Level l of the tree covers C**l tokens; level 0 is the tokens. Node (l, i)
    exists iff (i+1)*C**l <= N_b with N_b = C*floor(N/C).
  * Merge rule: child c's log mass at reference query q_r is its own plane r
    evaluated there; the parent combines these log masses and the children's
    compressed keys with the softmax-weighted average (``merge_children``).
  * Routing starts from every top-level node; an orphan (a node whose parent
    does not exist yet) is a candidate at its own level; the kept prefix is the
    shortest prefix of (score desc, node index asc) with softmax mass >= p;
    p >= 1 keeps everything; top-p runs on levels L..1 and every token of a kept
    level-1 chunk is attended, plus token 0 and the in-progress tail [N_b, N).
  * Routing is per query head; the tree is shared by the query heads of a KV head.

Pins (tests/test_oracle_pins.py): the 3-token worked example (A and O), the
causal example, the online-softmax table, the softmax-saturation numbers, tangent
exactness, the convexity lower bound, the finite-difference gradient
dF/dq = khat/sqrt(d), identical-key and single-key chunks, merge == direct
summary over raw keys, brute-force minimal prefix over all subsets, hand-built
routing trees, set invariants, and p=1 routed == dense attention; for the
routing policies, brute force over all subsets (top-K), the closed-form kept
counts of a flat tree under a fixed p and under p**(1/L), and the product of
the depth-scaled masses.
``captured_mass`` is a diagnostic only: parity unpinned.
"""

from __future__ import annotations

from dataclasses import dataclass, field

import numpy as np


# ----------------------------------------------------------------------------
# Elementary pieces
# ----------------------------------------------------------------------------

def bf16_bits_to_f64(bits: np.ndarray) -> np.ndarray:
    """Exact value of bfloat16 numbers given as their 16-bit patterns.

    A bfloat16 is the top half of an IEEE fp32; widening is exact.
    """
    b = np.ascontiguousarray(bits, dtype=np.uint16)
    return (b.astype(np.uint32) << np.uint32(16)).view(np.float32).astype(np.float64)


def logsumexp(x: np.ndarray, axis: int = -1) -> np.ndarray:
    """log(sum(exp(x))) along ``axis``, shifted by the maximum for range."""
    x = np.asarray(x, dtype=np.float64)
    m = np.max(x, axis=axis, keepdims=True)
    m_safe = np.where(np.isfinite(m), m, 0.0)
    s = np.sum(np.exp(x - m_safe), axis=axis, keepdims=True)
    with np.errstate(divide="ignore"):
        out = np.log(s) + m_safe
    return np.squeeze(out, axis=axis)


def sdpa(Q: np.ndarray, K: np.ndarray, V: np.ndarray,
         mask: np.ndarray | None = None) -> tuple[np.ndarray, np.ndarray]:
    """Scaled dot-product attention, softmax(Q K^T / sqrt(d_k) + M) V.

    [Attention: "Scaled dot-product attention 의 식"] -- scores, scaling by
    sqrt(d_k), row-wise softmax, weighted average of the value rows.
    [Attention: "Causal mask 는 뒤에 오는 토큰을 가린다"] -- ``mask`` is a boolean
    matrix, False where the score is replaced by -inf.
    Returns (A, O).
    """
    Q = np.asarray(Q, np.float64)
    K = np.asarray(K, np.float64)
    V = np.asarray(V, np.float64)
    d_k = Q.shape[-1]
    S = (Q @ K.T) / np.sqrt(d_k)
    if mask is not None:
        S = np.where(mask, S, -np.inf)
    S_max = np.max(S, axis=-1, keepdims=True)
    E = np.exp(S - S_max)
    A = E / np.sum(E, axis=-1, keepdims=True)
    return A, A @ V


def combine_log_masses(u: np.ndarray, rows: np.ndarray) -> tuple[np.ndarray, np.ndarray]:
    """Combine parts given by their log masses ``u`` and their averaged rows.

    u: [..., n] log masses; rows: [..., n, d]. Returns (F, avg) with
    F = log sum_c exp(u_c) and avg = sum_c softmax(u)_c rows_c.

    This is the identity behind the online softmax: two blocks with running
    maxima, exp-sums and unnormalised outputs combine into the softmax over
    their union ([Attention: "FlashAttention 계열"], the two-block table for
    token 3), restated as a merge of (mass, normalised state) pairs by
    [ASM: 방법론]. Over single keys (u_j = q.k_j/sqrt(d), rows = k_j or v_j)
    it is one row of scaled dot-product attention with its log-normaliser.
    """
    u = np.asarray(u, np.float64)
    rows = np.asarray(rows, np.float64)
    F = logsumexp(u, axis=-1)
    w = np.exp(u - F[..., None])
    avg = np.einsum("...c,...cd->...d", w, rows)
    return F, avg


# ----------------------------------------------------------------------------
# Summaries: level 1 and the merge of upper levels   [ZHA: 무엇과 다른가]
# ----------------------------------------------------------------------------

def chunk_log_mass(q: np.ndarray, Kc: np.ndarray) -> np.ndarray:
    """F_C(q) = LSE_j(q . k_j / sqrt(d)), the unnormalised log attention mass of
    a key chunk K_C for query q. [ZHA: 무엇과 다른가]

    q: [..., d] (one or many queries), Kc: [C, d]. Returns [...].
    """
    q = np.asarray(q, np.float64)
    Kc = np.asarray(Kc, np.float64)
    d = Kc.shape[-1]
    s = (q @ Kc.T) / np.sqrt(d)
    return logsumexp(s, axis=-1)


def summarise_chunk(qhat: np.ndarray, Kc: np.ndarray) -> tuple[np.ndarray, np.ndarray]:
    """Tangent-plane summary of a key chunk at each reference query.
    [ZHA: 무엇과 다른가]

    The first-order expansion of F_C around q_r gives the plane
    t_r(q) = q . khat_r / sqrt(d) + bhat_r, where khat_r = Attn(q_r, K_C, K_C)
    (the attention output of q_r over the chunk, values = keys) and
    bhat_r = F_C(q_r) - q_r . khat_r / sqrt(d).

    qhat: [R, d]; Kc: [..., C, d] (one chunk or a stack of chunks).
    Returns khat [..., R, d], bhat [..., R].
    """
    qhat = np.asarray(qhat, np.float64)
    Kc = np.asarray(Kc, np.float64)
    d = Kc.shape[-1]
    # log mass of each single key j at each q_r: u[..., r, j] = q_r . k_j / sqrt(d)
    u = np.swapaxes(Kc @ qhat.T, -1, -2) / np.sqrt(d)            # [..., R, C]
    keys = np.broadcast_to(Kc[..., None, :, :], u.shape + (d,))    # [..., R, C, d]
    F, khat = combine_log_masses(u, keys)                          # [..., R], [..., R, d]
    bhat = F - np.sum(khat * qhat, axis=-1) / np.sqrt(d)
    return khat, bhat


def tangent_planes(q: np.ndarray, khat: np.ndarray, bhat: np.ndarray) -> np.ndarray:
    """t_r(q) = q . khat_r / sqrt(d) + bhat_r for every plane r. [ZHA: 무엇과 다른가]

    q: [d]; khat: [..., R, d]; bhat: [..., R]. Returns [..., R].
    """
    q = np.asarray(q, np.float64)
    d = q.shape[-1]
    return np.asarray(khat, np.float64) @ q / np.sqrt(d) + np.asarray(bhat, np.float64)


def node_score(q: np.ndarray, khat: np.ndarray, bhat: np.ndarray) -> np.ndarray:
    """A node's estimated log mass for a future query: the maximum of its R
    tangent planes, max_r t_r(q). [ZHA: 무엇과 다른가]"""
    return np.max(tangent_planes(q, khat, bhat), axis=-1)


def merge_children(qhat: np.ndarray, khat_ch: np.ndarray,
                   bhat_ch: np.ndarray) -> tuple[np.ndarray, np.ndarray]:
    """Parent summary from its children's summaries ("merged in the same way").
    [ZHA: 무엇과 다른가]

    For each reference query q_r: the child's log mass there is its own plane r,
    u_c = q_r . khat_{r,c} / sqrt(d) + bhat_{r,c}  (= F_c(q_r) by construction);
    F_P = LSE_c u_c, khat_{r,P} = sum_c softmax(u)_c khat_{r,c},
    bhat_{r,P} = F_P - q_r . khat_{r,P} / sqrt(d).
    With no positional rotation this equals ``summarise_chunk`` over all the
    raw keys under the parent (the combine identity applied twice).

    qhat: [R, d]; khat_ch: [..., C, R, d]; bhat_ch: [..., C, R].
    Returns khat [..., R, d], bhat [..., R].
    """
    qhat = np.asarray(qhat, np.float64)
    khat_ch = np.asarray(khat_ch, np.float64)
    bhat_ch = np.asarray(bhat_ch, np.float64)
    d = qhat.shape[-1]
    u = np.sum(khat_ch * qhat, axis=-1) / np.sqrt(d) + bhat_ch      # [..., C, R]
    u_rc = np.swapaxes(u, -1, -2)                                   # [..., R, C]
    rows = np.moveaxis(khat_ch, -3, -2)                             # [..., R, C, d]
    F, khat = combine_log_masses(u_rc, rows)
    bhat = F - np.sum(khat * qhat, axis=-1) / np.sqrt(d)
    return khat, bhat


@dataclass
class OracleTree:
    """Summary tree of one KV head. ``nodes[l] = (khat [n_l, R, d], bhat [n_l, R])``."""
    chunk: int
    levels: int
    n_tokens: int
    qhat: np.ndarray
    nodes: dict = field(default_factory=dict)

    @property
    def n_built(self) -> int:
        return self.chunk * (self.n_tokens // self.chunk)

    def n_nodes(self, level: int) -> int:
        if level < 1 or level > self.levels:
            return 0
        return self.n_built // (self.chunk ** level)


def build_tree(K: np.ndarray, qhat: np.ndarray, chunk: int, levels: int,
               n_tokens: int) -> OracleTree:
    """Build levels 1..L over the complete chunks of the first ``n_tokens`` keys
    of one KV head. [ZHA: 무엇과 다른가]

    Level 1 summarises each contiguous chunk of C keys; level l >= 2 merges
    groups of C consecutive level-(l-1) nodes. Only complete nodes exist.
    """
    K = np.asarray(K, np.float64)
    qhat = np.asarray(qhat, np.float64)
    d = K.shape[1]
    tree = OracleTree(chunk=chunk, levels=levels, n_tokens=int(n_tokens), qhat=qhat)
    n1 = tree.n_nodes(1)
    Kc = K[: n1 * chunk].reshape(n1, chunk, d)
    tree.nodes[1] = summarise_chunk(qhat, Kc)
    for lvl in range(2, levels + 1):
        n_here = tree.n_nodes(lvl)
        kh, bh = tree.nodes[lvl - 1]
        kh = kh[: n_here * chunk].reshape(n_here, chunk, *kh.shape[1:])
        bh = bh[: n_here * chunk].reshape(n_here, chunk, bh.shape[-1])
        tree.nodes[lvl] = merge_children(qhat, kh, bh)
    return tree


# ----------------------------------------------------------------------------
# Rotary positions   [ZHA: 무엇과 다른가; Attention: "Attention 은 순서를 모르므로 위치 정보를 따로 넣는다"]
# ----------------------------------------------------------------------------

def rope_angles(d: int, base: float, pairs: int) -> np.ndarray:
    """Rotation speed theta_i of each element pair i = (2i, 2i+1).

    [Attention: "Attention 은 순서를 모르므로 위치 정보를 따로 넣는다"] pairs the
    elements of a query or key two by
    two, reads each pair as a point of a plane, and turns pair i of the token
    at position m by the angle m * theta_i, a different speed per pair (Su et
    al., 2021). Reading: theta_i = base**(-2i/d), the first ``pairs`` pairs
    turn, the others (partial RoPE) stay as they are (theta = 0).
    """
    i = np.arange(d // 2, dtype=np.float64)
    theta = np.power(float(base), -2.0 * i / d)
    theta[int(pairs):] = 0.0
    return theta


def rope_rotate(x: np.ndarray, pos, base: float, pairs: int) -> np.ndarray:
    """Turn pair i of x (elements 2i, 2i+1) by pos * theta_i. x: [..., d];
    pos: a number or an array broadcasting against x[..., 0]."""
    x = np.asarray(x, np.float64)
    d = x.shape[-1]
    ang = np.asarray(pos, np.float64)[..., None] * rope_angles(d, base, pairs)     # [..., d/2]
    c, s = np.cos(ang), np.sin(ang)
    a, b = x[..., 0::2], x[..., 1::2]
    out = np.empty(np.broadcast_shapes(x.shape, ang.shape[:-1] + (d,)), np.float64)
    out[..., 0::2] = a * c - b * s
    out[..., 1::2] = a * s + b * c
    return out


def node_position(level: int, index, chunk: int):
    """Position of node (level, index): its first token, index * chunk**level
    (reading: a node's rotated reference query sits where its span starts)."""
    return np.asarray(index, np.int64) * chunk ** level


def summarise_chunk_rope(qhat: np.ndarray, Kc: np.ndarray, pos, base: float,
                         pairs: int) -> tuple[np.ndarray, np.ndarray]:
    """Level-1 summary with rotary positions: the tangent plane of F_C taken at
    the chunk's rotated reference queries q_hat_{r,c} = rotate(q_hat_r, pos_c),
    over the keys as the cache stores them (already rotated at their own
    positions). [ZHA: 무엇과 다른가]

    qhat: [R, d]; Kc: [..., C, d]; pos: [...] chunk positions.
    """
    qhat = np.asarray(qhat, np.float64)
    Kc = np.asarray(Kc, np.float64)
    pos = np.asarray(pos, np.float64)
    q_rot = rope_rotate(qhat, pos[..., None], base, pairs)        # [..., R, d]
    d = Kc.shape[-1]
    u = np.einsum("...rd,...jd->...rj", q_rot, Kc) / np.sqrt(d)    # [..., R, C]
    keys = np.broadcast_to(Kc[..., None, :, :], u.shape + (d,))
    F, khat = combine_log_masses(u, keys)
    bhat = F - np.sum(khat * q_rot, axis=-1) / np.sqrt(d)
    return khat, bhat


def merge_children_rope(qhat: np.ndarray, khat_ch: np.ndarray, bhat_ch: np.ndarray,
                        pos_parent, pos_children, base: float,
                        pairs: int) -> tuple[np.ndarray, np.ndarray]:
    """Parent summary from its children's with rotary positions. [ZHA: 무엇과
    다른가]: each child is re-evaluated at the parent's rotated reference query
    q_hat_{r,P}; its log mass there is its tangent value at its own rotated
    reference query, F_c(q_hat_{r,c}) = q_hat_{r,c}.khat_{r,c}/sqrt(d) + bhat_{r,c},
    plus the correction 1/sqrt(d) <khat_{r,c}, q_hat_{r,P} - q_hat_{r,c}>; the
    parent then combines these log masses and the children's compressed keys
    as in the position-free merge.

    khat_ch: [..., C, R, d]; bhat_ch: [..., C, R]; pos_parent: [...];
    pos_children: [..., C].
    """
    qhat = np.asarray(qhat, np.float64)
    khat_ch = np.asarray(khat_ch, np.float64)
    bhat_ch = np.asarray(bhat_ch, np.float64)
    d = qhat.shape[-1]
    q_P = rope_rotate(qhat, np.asarray(pos_parent, np.float64)[..., None], base, pairs)     # [..., R, d]
    q_c = rope_rotate(qhat, np.asarray(pos_children, np.float64)[..., None], base, pairs)   # [..., C, R, d]
    F_c = np.sum(khat_ch * q_c, axis=-1) / np.sqrt(d) + bhat_ch                # [..., C, R]
    corr = np.sum(khat_ch * (q_P[..., None, :, :] - q_c), axis=-1) / np.sqrt(d)
    u = F_c + corr
    F, khat = combine_log_masses(np.swapaxes(u, -1, -2), np.moveaxis(khat_ch, -3, -2))
    bhat = F - np.sum(khat * q_P, axis=-1) / np.sqrt(d)
    return khat, bhat


def build_tree_rope(K: np.ndarray, qhat: np.ndarray, chunk: int, levels: int, n_tokens: int,
                    base: float, pairs: int) -> OracleTree:
    """``build_tree`` for a model with rotary positions: level-1 summaries at
    each chunk's rotated reference queries, upper levels by
    ``merge_children_rope``. [ZHA: 무엇과 다른가]"""
    K = np.asarray(K, np.float64)
    qhat = np.asarray(qhat, np.float64)
    d = K.shape[1]
    tree = OracleTree(chunk=chunk, levels=levels, n_tokens=int(n_tokens), qhat=qhat)
    n1 = tree.n_nodes(1)
    Kc = K[: n1 * chunk].reshape(n1, chunk, d)
    tree.nodes[1] = summarise_chunk_rope(qhat, Kc, node_position(1, np.arange(n1), chunk), base, pairs)
    for lvl in range(2, levels + 1):
        n_here = tree.n_nodes(lvl)
        kh, bh = tree.nodes[lvl - 1]
        kh = kh[: n_here * chunk].reshape(n_here, chunk, *kh.shape[1:])
        bh = bh[: n_here * chunk].reshape(n_here, chunk, bh.shape[-1])
        par = np.arange(n_here)
        ch = par[:, None] * chunk + np.arange(chunk)[None, :]
        tree.nodes[lvl] = merge_children_rope(qhat, kh, bh, node_position(lvl, par, chunk),
                                              node_position(lvl - 1, ch, chunk), base, pairs)
    return tree


# ----------------------------------------------------------------------------
# Routing   [ZHA: 전제와 한계]
# ----------------------------------------------------------------------------

@dataclass
class TopP:
    """Outcome of one top-p selection.

    order: candidate positions in selection order (score desc, node index asc);
    pi: softmax of the scores over the candidates; cum: cumulative pi along
    ``order``; m: number kept; kept: the kept node ids, ascending.
    """
    kept: np.ndarray
    order: np.ndarray
    pi: np.ndarray
    cum: np.ndarray
    m: int


def top_p_prefix(sigma: np.ndarray, ids: np.ndarray, p: float) -> TopP:
    """Minimal prefix holding estimated mass >= p. [ZHA: 전제와 한계]

    Candidates are softmaxed over their scores and sorted by score (ties:
    lower node index first); the kept set is the shortest prefix whose summed
    probability reaches p (sum in fp64). p >= 1 keeps every candidate; no
    candidates keeps nothing.
    """
    sigma = np.asarray(sigma, np.float64)
    ids = np.asarray(ids, np.int64)
    n = sigma.shape[0]
    if n == 0:
        e = np.zeros(0, np.int64)
        return TopP(kept=e, order=e, pi=np.zeros(0), cum=np.zeros(0), m=0)
    order = np.lexsort((ids, -sigma))
    pi = np.exp(sigma - logsumexp(sigma))
    cum = np.cumsum(pi[order])
    if p >= 1.0:
        m = n
    else:
        reached = np.nonzero(cum >= p)[0]
        m = int(reached[0]) + 1 if reached.size else n
    kept = np.sort(ids[order[:m]])
    return TopP(kept=kept, order=order, pi=pi, cum=cum, m=m)


def top_k_prefix(sigma: np.ndarray, ids: np.ndarray, k: int) -> TopP:
    """Fixed-budget selection: the first min(k, n) candidates in the order
    score descending, node index ascending. [ZHA: 전제와 한계] sets top-p
    routing against a fixed-budget top-K, which keeps the same number of nodes
    whether the mass is concentrated or flat; this is that comparison mode.
    ``pi`` and ``cum`` are the softmax masses along the order, as for top-p.
    """
    sigma = np.asarray(sigma, np.float64)
    ids = np.asarray(ids, np.int64)
    n = sigma.shape[0]
    if n == 0:
        e = np.zeros(0, np.int64)
        return TopP(kept=e, order=e, pi=np.zeros(0), cum=np.zeros(0), m=0)
    order = np.lexsort((ids, -sigma))
    pi = np.exp(sigma - logsumexp(sigma))
    cum = np.cumsum(pi[order])
    m = min(int(k), n)
    return TopP(kept=np.sort(ids[order[:m]]), order=order, pi=pi, cum=cum, m=m)


@dataclass
class RoutePolicy:
    """How each level's kept prefix is chosen. [ZHA: 전제와 한계]

    mode "top_p": level l keeps the minimal prefix holding estimated mass
    ``p[l]`` (one p for every level when ``p`` is a number).
    mode "top_k": level l keeps the first ``k[l]`` candidates (fixed budget).
    """
    mode: str = "top_p"
    p: object = 0.9
    k: object = None

    def at(self, level: int):
        v = self.p if self.mode == "top_p" else self.k
        return v[level] if isinstance(v, dict) else v


def depth_scaled_p(p: float, levels: int) -> dict:
    """Per-level mass p_l = p**(1/L) for l = 1..L, so that the product of the
    per-level masses is p. [ZHA: 전제와 한계] names both ends of the depth
    scaling: a fixed p per level gives an effective p**L, which goes to 0 with
    depth, while correcting with p**(1/L) drives each level's p towards 1."""
    return {lvl: float(p) ** (1.0 / levels) for lvl in range(1, levels + 1)}


def select_level(sigma: np.ndarray, ids: np.ndarray, level: int, policy) -> TopP:
    """One level's selection under ``policy`` (a number p, a {level: p} dict,
    or a RoutePolicy)."""
    if isinstance(policy, RoutePolicy):
        if policy.mode == "top_k":
            return top_k_prefix(sigma, ids, policy.at(level))
        return top_p_prefix(sigma, ids, policy.at(level))
    if isinstance(policy, dict):
        return top_p_prefix(sigma, ids, policy[level])
    return top_p_prefix(sigma, ids, policy)


@dataclass
class LevelTrace:
    candidates: np.ndarray      # node ids at this level, ascending
    sigma: np.ndarray           # score of each candidate (same order)
    topp: TopP                  # this level's own selection
    expanded: np.ndarray        # kept set whose children form the next level's candidates


@dataclass
class RouteTrace:
    levels: dict                # level -> LevelTrace
    leaf_chunks: np.ndarray     # level-1 chunks whose tokens are attended
    tokens: np.ndarray          # leaf token set S (ascending)


def leaf_token_set(leaf_chunks: np.ndarray, chunk: int, n_tokens: int) -> np.ndarray:
    """S = {0} u tokens(kept level-1 chunks) u [N_b, N). [ZHA: 전제와 한계]

    Token 0 is the attention sink and the tail [N_b, N) is the visible part of
    the chunk still being filled; both are always attended. S is a set.
    """
    nb = chunk * (n_tokens // chunk)
    parts = [np.zeros(1, np.int64) if n_tokens > 0 else np.zeros(0, np.int64),
             np.arange(nb, n_tokens, dtype=np.int64)]
    for c in np.asarray(leaf_chunks, np.int64):
        parts.append(np.arange(c * chunk, (c + 1) * chunk, dtype=np.int64))
    return np.unique(np.concatenate(parts))


def route(q: np.ndarray, tree: OracleTree, p,
          forced_kept: dict | None = None) -> RouteTrace:
    """Per-level top-p routing of one query head through one tree.
    [ZHA: 전제와 한계]

    Level L starts with every level-L node as candidate. At each level the
    candidates are scored (``node_score``), softmaxed and cut by
    ``top_p_prefix``; the next level's candidates are the children of the kept
    nodes plus that level's orphans (nodes whose parent does not exist).
    ``p`` is one mass for every level, a {level: p_l} schedule, or a
    RoutePolicy (per-level p, or the fixed-budget top-K comparison mode).

    ``forced_kept`` (level -> node ids) makes the expansion below that level use
    the given kept set instead of this oracle's own; each level still records its
    own selection. Tests use it to compare a level conditioned on the GPU's
    choice one level up.
    """
    C, L = tree.chunk, tree.levels
    levels: dict = {}
    parent_kept = np.zeros(0, np.int64)
    for lvl in range(L, 0, -1):
        n_here = tree.n_nodes(lvl)
        n_parent = tree.n_nodes(lvl + 1)          # 0 above the top level
        children = (parent_kept[:, None] * C + np.arange(C)[None, :]).reshape(-1)
        orphans = np.arange(C * n_parent, n_here, dtype=np.int64)
        cand = np.concatenate([children.astype(np.int64), orphans])
        khat, bhat = tree.nodes[lvl]
        sigma = node_score(q, khat[cand], bhat[cand]) if cand.size else np.zeros(0)
        sel = select_level(sigma, cand, lvl, p)
        if forced_kept is not None and lvl in forced_kept:
            expanded = np.sort(np.asarray(forced_kept[lvl], np.int64))
        else:
            expanded = sel.kept
        levels[lvl] = LevelTrace(candidates=cand, sigma=sigma, topp=sel, expanded=expanded)
        parent_kept = expanded
    leaf_chunks = parent_kept
    return RouteTrace(levels=levels, leaf_chunks=leaf_chunks,
                      tokens=leaf_token_set(leaf_chunks, C, tree.n_tokens))


# ----------------------------------------------------------------------------
# Attention over the leaf set
# ----------------------------------------------------------------------------

def attend(q: np.ndarray, K: np.ndarray, V: np.ndarray,
           tokens: np.ndarray) -> tuple[np.ndarray, float]:
    """Exact softmax attention of one query head over the gathered tokens S.

    [Attention: "Scaled dot-product attention 의 식"] restricted to the rows in
    S ([ZHA: 무엇인가 / 전제와 한계]: keys are picked per query, there is no value
    summary). Returns (o [d], lse) with lse = log sum_{j in S} exp(q.k_j/sqrt(d)).
    """
    q = np.asarray(q, np.float64)
    tokens = np.asarray(tokens, np.int64)
    Ks = np.asarray(K, np.float64)[tokens]
    Vs = np.asarray(V, np.float64)[tokens]
    _, O = sdpa(q[None, :], Ks, Vs)
    s = Ks @ q / np.sqrt(q.shape[-1])
    return O[0], float(logsumexp(s))


# ----------------------------------------------------------------------------
# Routing diagnostics   [ZHA: 어떻게 쓰나; 전제와 한계]
# ----------------------------------------------------------------------------

def level_target_mass(q: np.ndarray, K: np.ndarray, tree: OracleTree, level: int) -> np.ndarray:
    """Target distribution p_{l,C}(q) over the complete nodes of `level`:
    the dense attention weights of q over the keys, summed node by node.
    [ZHA: 어떻게 쓰나] (the target of the reference queries' KL training).
    Reading: the weights are taken over the keys the level's nodes cover and
    normalised over the nodes (keys of the in-progress tail are in no node)."""
    n_l = tree.n_nodes(level)
    span = tree.chunk ** level
    A, _ = sdpa(np.asarray(q, np.float64)[None], np.asarray(K, np.float64)[: n_l * span],
                np.zeros((n_l * span, 1)))
    return A[0].reshape(n_l, span).sum(axis=1)


def level_estimate(q: np.ndarray, tree: OracleTree, level: int) -> np.ndarray:
    """Estimate p_hat_{l,C}(q): softmax over the level's nodes of their scores
    max_r t_r(q). [ZHA: 어떻게 쓰나]"""
    khat, bhat = tree.nodes[level]
    sigma = node_score(q, khat, bhat)
    return np.exp(sigma - logsumexp(sigma))


def level_kl(q: np.ndarray, K: np.ndarray, tree: OracleTree, level: int) -> float:
    """KL(p_{l,C}(q) || p_hat_{l,C}(q)) over the level's nodes. [ZHA: 어떻게 쓰나]"""
    p = level_target_mass(q, K, tree, level)
    ph = level_estimate(q, tree, level)
    nz = p > 0
    return float(np.sum(p[nz] * (np.log(p[nz]) - np.log(ph[nz]))))


def plane_usage(q: np.ndarray, tree: OracleTree, level: int) -> np.ndarray:
    """How often each reference query gives a node's score: for every node of
    the level the plane r attaining max_r t_r(q) (lowest r on ties), counted
    per r. [ZHA: 전제와 한계] reports that few reference queries serve the upper
    levels and the use evens out towards the leaves."""
    khat, bhat = tree.nodes[level]
    t = tangent_planes(q, khat, bhat)                    # [n, R]
    return np.bincount(np.argmax(t, axis=-1), minlength=khat.shape[-2])


def captured_mass(q: np.ndarray, K: np.ndarray, tokens: np.ndarray,
                  n_tokens: int) -> float:
    """Share of the dense attention mass over [0, n_tokens) that S holds.
    Diagnostic only -- parity unpinned (the pages bound nothing here)."""
    q = np.asarray(q, np.float64)
    s = np.asarray(K, np.float64)[:n_tokens] @ q / np.sqrt(q.shape[-1])
    lse_all = logsumexp(s)
    return float(np.exp(logsumexp(s[np.asarray(tokens, np.int64)]) - lse_all))
