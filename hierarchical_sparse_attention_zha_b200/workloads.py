"""Seeded synthetic inputs for the ZHA decode hot path.

This module only draws data (NumPy PCG64, fixed seeds) in the shapes, value
distributions and structure of the five workloads below; it contains none of
the method's arithmetic, and both the CUDA path and the CPU oracle read the
same bytes from it. Values are drawn in fp32 and, for bf16 caches, rounded once
to bfloat16 (round to nearest, ties to even) and handed out as 16-bit patterns.

The pages evaluate on long novels, RULER and SWE-bench; those are not used.
The generators stand in for them with the structure the pages describe:
attention mass concentrated on a few tokens (planted keys and needles), mass
concentrated by a power law (Zipf-popular key clusters laid out in contiguous
runs), and near-flat mass (i.i.d. keys) that forces wide top-p selections.

Workloads (all NoPE: no positional rotation):

  tiny  -- Tiny NoPE: 1 KV head / 4 query heads, d=64, fp32 K/V, 4096 tokens,
           C=16, L=2, R=4, p=0.9, 16 queries. K, V ~ N(0,1) + 3*mu_g; 8 needle
           keys, each aligned with one query and 6 logits above that query's
           best other key. Seed 0.
  32k   -- NoPE 32K: 8/32 heads, d=128, bf16, 32768 tokens, C=64, L=2, R=16,
           p=0.9, 8 queries. 1% of the keys (8 spans of 41) planted as
           z + gamma*mu_g, gamma giving +8 logits for the group's queries. Seed 1.
  256k  -- NoPE 256K: 4/16 heads, d=128, bf16, 262144 tokens, C=16, L=3, R=16,
           p=0.75, 4 queries. Keys from 512 Gaussian clusters (key = centre +
           0.3 N(0,I)); the centres lie in the head's cone (norm sqrt(d), the
           anisotropy of real keys) and are laid out in contiguous runs
           (geometric length, mean 256) with Zipf(1.1) cluster popularity. Seed 2.
  deep  -- Deep tree: 8/32 heads, d=128, bf16, 65536 tokens, C=4, L=6, R=16,
           p=0.9, 8 queries. K, V ~ N(0,1); queries of norm sqrt(d) in random
           directions (near-flat mass). Seed 3.
  1m    -- 1M context: 4/32 heads, d=128, bf16, 1048576 tokens, C=64, L=3,
           R=16, p=0.75, 4 queries per decode step, as 256k plus 16 needles, and
           4*C further tokens for streaming decode (appends every C steps). Seed 4.

Queries of the clustered workloads: for each (batch element, KV head) one
cluster is drawn uniformly; each of the G query heads of that KV head gets
28 * normalise(centre_dir + 0.5 z / sqrt(d)), so a group's heads look at the
same cluster with per-head noise. Reference queries of every workload lie in a
cone around a per-head direction mu_g: normalise(mu_g + 1.13 z / sqrt(d)),
mean pairwise cosine about 0.44, scaled to the workload's query norm.
"""

from __future__ import annotations

from dataclasses import dataclass, field, replace

import numpy as np


@dataclass(frozen=True)
class Workload:
    key: str
    name: str
    n_kv_heads: int
    n_q_heads: int
    head_dim: int
    kv_dtype: str          # "f32" or "bf16"
    n_tokens: int
    chunk: int
    levels: int
    n_ref: int
    p: float
    batch: int
    seed: int
    recipe: str            # "needles" | "planted" | "clusters" | "uniform"
    n_needles: int = 0
    stream_tokens: int = 0  # tokens beyond n_tokens for streaming decode

    @property
    def group(self) -> int:
        return self.n_q_heads // self.n_kv_heads

    @property
    def elt_bytes(self) -> int:
        return 4 if self.kv_dtype == "f32" else 2

    @property
    def capacity(self) -> int:
        return self.n_tokens + self.stream_tokens

    def describe(self) -> dict:
        return {
            "workload": self.name, "n_kv_heads": self.n_kv_heads,
            "n_q_heads": self.n_q_heads, "head_dim": self.head_dim,
            "kv_dtype": self.kv_dtype, "context": self.n_tokens, "chunk": self.chunk,
            "levels": self.levels, "n_ref": self.n_ref, "p": self.p,
            "batch": self.batch, "seed": self.seed,
        }


WORKLOADS = {
    "tiny": Workload("tiny", "Tiny NoPE", 1, 4, 64, "f32", 4096, 16, 2, 4, 0.9, 16, 0,
                     "needles", n_needles=8),
    "32k": Workload("32k", "NoPE 32K", 8, 32, 128, "bf16", 32768, 64, 2, 16, 0.9, 8, 1,
                    "planted"),
    "256k": Workload("256k", "NoPE 256K", 4, 16, 128, "bf16", 262144, 16, 3, 16, 0.75, 4, 2,
                     "clusters"),
    "deep": Workload("deep", "Deep tree", 8, 32, 128, "bf16", 65536, 4, 6, 16, 0.9, 8, 3,
                     "uniform"),
    "1m": Workload("1m", "1M context", 4, 32, 128, "bf16", 1048576, 64, 3, 16, 0.75, 4, 4,
                   "clusters", n_needles=16, stream_tokens=256),
}

# Frozen generator constants (see the module docstring).
CONE_SPREAD = 1.13          # reference-query cone: mean pairwise cosine ~ 0.44
TINY_OFFSET = 3.0           # per-head mean offset of Tiny NoPE keys and values
NEEDLE_MARGIN = 6.0         # needle logit above the query's best other key
PLANTED_FRACTION = 0.01     # NoPE 32K planted keys
PLANTED_SPANS = 8
PLANTED_LOGIT = 8.0
N_CLUSTERS = 512
CLUSTER_SIGMA = 0.3
RUN_MEAN = 256
ZIPF_S = 1.1
CLUSTER_QUERY_NORM = 28.0
CLUSTER_QUERY_NOISE = 0.5


@dataclass
class Inputs:
    """One workload's arrays. K, V: [Hkv, capacity, d] (float32, or uint16
    bfloat16 patterns); ref_q: [Hkv, R, d] float32; Q: [n_batches, B, Hq, d]
    float32 (batch t is decode step t's queries)."""
    spec: Workload
    K: np.ndarray
    V: np.ndarray
    ref_q: np.ndarray
    Q: np.ndarray
    meta: dict = field(default_factory=dict)


def to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """fp32 -> bfloat16 bit patterns, round to nearest, ties to even."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    rounded = u + np.uint32(0x7FFF) + ((u >> np.uint32(16)) & np.uint32(1))
    return (rounded >> np.uint32(16)).astype(np.uint16)


def bf16_bits_to_f32(bits: np.ndarray) -> np.ndarray:
    """bfloat16 bit patterns -> fp32 (exact widening)."""
    return (np.ascontiguousarray(bits, np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


def _unit(v: np.ndarray, axis: int = -1) -> np.ndarray:
    return v / np.linalg.norm(v, axis=axis, keepdims=True)


def _cone(rng, mu: np.ndarray, n: int, norm: float) -> np.ndarray:
    d = mu.shape[-1]
    z = rng.standard_normal((n, d))
    return (norm * _unit(mu[None, :] + CONE_SPREAD * z / np.sqrt(d))).astype(np.float32)


def _store(x: np.ndarray, kv_dtype: str) -> np.ndarray:
    return x.astype(np.float32) if kv_dtype == "f32" else to_bf16_bits(x)


_BLOCK = 1 << 16


def _fill(rng, out: np.ndarray, kv_dtype: str, scale: float = 1.0, base=None) -> None:
    """out[t] = store(base(t) + scale * N(0, I)), drawn block by block so that
    no full-size fp32 temporary is needed. ``base(lo, hi)`` returns the fp32
    mean rows of tokens [lo, hi) (or None for zero mean)."""
    n, d = out.shape
    for lo in range(0, n, _BLOCK):
        hi = min(n, lo + _BLOCK)
        x = rng.standard_normal((hi - lo, d), dtype=np.float32)
        if scale != 1.0:
            x *= np.float32(scale)
        if base is not None:
            x += base(lo, hi)
        out[lo:hi] = _store(x, kv_dtype)


def _stored_f32(x: np.ndarray, kv_dtype: str) -> np.ndarray:
    return x if kv_dtype == "f32" else bf16_bits_to_f32(x)


def _cluster_layout(rng, n: int) -> np.ndarray:
    """Cluster id of each of n tokens: contiguous runs of geometric length
    (mean RUN_MEAN), cluster per run drawn with Zipf(ZIPF_S) popularity."""
    pop = 1.0 / np.arange(1, N_CLUSTERS + 1) ** ZIPF_S
    pop /= pop.sum()
    perm = rng.permutation(N_CLUSTERS)           # popularity rank -> cluster id
    n_runs = n // RUN_MEAN * 2 + 16
    lengths = rng.geometric(1.0 / RUN_MEAN, size=n_runs)
    while lengths.sum() < n:
        lengths = np.concatenate([lengths, rng.geometric(1.0 / RUN_MEAN, size=n_runs)])
    clusters = perm[rng.choice(N_CLUSTERS, size=lengths.size, p=pop)]
    return np.repeat(clusters, lengths)[:n].astype(np.int32)


def generate(spec: Workload | str, n_batches: int = 1, rank: int = 0) -> Inputs:
    """Draw the workload's K, V, reference queries and ``n_batches`` query
    batches. ``rank`` offsets the seed so replicas get independent problems."""
    if isinstance(spec, str):
        spec = WORKLOADS[spec]
    rng = np.random.default_rng(spec.seed + 1000 * rank)
    Hkv, Hq, d, G = spec.n_kv_heads, spec.n_q_heads, spec.head_dim, spec.group
    cap, R, B = spec.capacity, spec.n_ref, spec.batch
    K = np.empty((Hkv, cap, d), np.float32 if spec.kv_dtype == "f32" else np.uint16)
    V = np.empty_like(K)
    ref_q = np.empty((Hkv, R, d), np.float32)
    Q = np.empty((n_batches, B, Hq, d), np.float32)
    mu = _unit(rng.standard_normal((Hkv, d)))
    meta: dict = {}

    if spec.recipe == "needles":
        qn = 2.0 * np.sqrt(d)
        for g in range(Hkv):
            ref_q[g] = _cone(rng, mu[g], R, qn)
            off = (TINY_OFFSET * mu[g]).astype(np.float32)
            _fill(rng, K[g], spec.kv_dtype, base=lambda lo, hi: off)
            _fill(rng, V[g], spec.kv_dtype, base=lambda lo, hi: off)
        for t in range(n_batches):
            for h in range(Hq):
                Q[t, :, h] = _cone(rng, mu[h // G], B, qn)
    elif spec.recipe == "planted":
        qn = np.sqrt(d)
        n_plant = int(round(PLANTED_FRACTION * spec.n_tokens))
        span = -(-n_plant // PLANTED_SPANS)
        for g in range(Hkv):
            ref_q[g] = _cone(rng, mu[g], R, qn)
            # disjoint spans, clear of token 0 and of the last chunk
            n_slots = (spec.n_tokens - spec.chunk - 1) // span
            starts = 1 + span * np.sort(rng.choice(n_slots, size=PLANTED_SPANS, replace=False))
            # gamma so that a cone query (cos(q, mu) ~ 1/sqrt(1+CONE_SPREAD^2)) gains PLANTED_LOGIT
            gamma = PLANTED_LOGIT * np.sqrt(d) / (qn / np.sqrt(1.0 + CONE_SPREAD ** 2))
            planted = np.zeros(cap, bool)
            for s0 in starts:
                planted[s0:s0 + span] = True
            shift = (gamma * mu[g]).astype(np.float32)
            _fill(rng, K[g], spec.kv_dtype,
                  base=lambda lo, hi: planted[lo:hi, None] * shift[None, :])
            _fill(rng, V[g], spec.kv_dtype)
            meta.setdefault("planted_starts", []).append(starts.tolist())
        meta["planted_span"] = span
        for t in range(n_batches):
            for h in range(Hq):
                Q[t, :, h] = _cone(rng, mu[h // G], B, qn)
    elif spec.recipe == "uniform":
        qn = np.sqrt(d)
        for g in range(Hkv):
            ref_q[g] = _cone(rng, mu[g], R, qn)
            _fill(rng, K[g], spec.kv_dtype)
            _fill(rng, V[g], spec.kv_dtype)
        for t in range(n_batches):
            Q[t] = (qn * _unit(rng.standard_normal((B, Hq, d)))).astype(np.float32)
    elif spec.recipe == "clusters":
        qn = CLUSTER_QUERY_NORM
        # cluster centres lie in the head's cone (anisotropic keys), norm sqrt(d)
        centres = np.stack([_cone(rng, mu[g], N_CLUSTERS, np.sqrt(d)) for g in range(Hkv)])
        layouts = []
        for g in range(Hkv):
            ref_q[g] = _cone(rng, mu[g], R, qn)
            lay = _cluster_layout(rng, cap)
            layouts.append(lay)
            cg = centres[g]
            _fill(rng, K[g], spec.kv_dtype, scale=CLUSTER_SIGMA,
                  base=lambda lo, hi: cg[lay[lo:hi]])
            _fill(rng, V[g], spec.kv_dtype)
        for t in range(n_batches):
            for b in range(B):
                for g in range(Hkv):
                    c = centres[g][rng.integers(N_CLUSTERS)]
                    z = rng.standard_normal((G, d))
                    Q[t, b, g * G:(g + 1) * G] = (qn * _unit(_unit(c)[None, :] + CLUSTER_QUERY_NOISE * z / np.sqrt(d))).astype(np.float32)
        meta["cluster_layout_head0"] = layouts[0]
    else:
        raise ValueError(spec.recipe)

    if spec.n_needles:
        # needles: one per chosen (batch, query head) of batch 0; key aligned
        # with that query, NEEDLE_MARGIN logits above its best other key.
        picks = rng.choice(B * Hq, size=spec.n_needles, replace=False)
        lo, hi = 1, spec.n_tokens - spec.chunk
        needles = []
        for idx in picks:
            b, h = divmod(int(idx), Hq)
            g = h // G
            q = Q[0, b, h].astype(np.float64)
            pos = int(rng.integers(lo, hi))
            Kg = _stored_f32(K[g, : spec.n_tokens], spec.kv_dtype)
            best = float(np.max(Kg @ q.astype(np.float32))) / np.sqrt(d)
            beta = (best + NEEDLE_MARGIN) * np.sqrt(d) / np.linalg.norm(q)
            K[g, pos] = _store((beta * q / np.linalg.norm(q))[None, :].astype(np.float32), spec.kv_dtype)[0]
            needles.append((b, h, pos))
        meta["needles"] = needles
    return Inputs(spec=spec, K=K, V=V, ref_q=ref_q, Q=Q, meta=meta)


def scaled(spec: Workload | str, **changes) -> Workload:
    """A copy of a workload with some fields changed (smaller parity cases)."""
    if isinstance(spec, str):
        spec = WORKLOADS[spec]
    return replace(spec, **changes)
