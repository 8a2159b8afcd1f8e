"""The seeded input generators: determinism, encodings, and the structure each
workload promises (cone of reference queries, needles, planted spans)."""

import numpy as np
import pytest
import torch

from hierarchical_sparse_attention_zha_b200 import workloads as W


def test_bf16_rounding_matches_torch():
    rng = np.random.default_rng(0)
    x = (rng.standard_normal(100_000) * np.exp(rng.uniform(-20, 20, 100_000))).astype(np.float32)
    x[:4] = [1.0, -0.0, 1.0 + 2 ** -8, 1.0 + 3 * 2 ** -8]      # exact ties both ways
    ours = W.to_bf16_bits(x)
    ref = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(ours, ref)
    assert np.array_equal(W.bf16_bits_to_f32(ours), torch.from_numpy(x).to(torch.bfloat16).float().numpy())


@pytest.mark.parametrize("key", ["tiny", "32k", "256k", "deep", "1m"])
def test_shapes_dtypes_and_determinism(key):
    spec = W.scaled(key, n_tokens=2048 if key != "1m" else 4096, stream_tokens=64 if key == "1m" else 0)
    if spec.recipe == "clusters":
        spec = W.scaled(spec, n_kv_heads=2, n_q_heads=2 * spec.group)
    a = W.generate(spec, n_batches=2)
    b = W.generate(spec, n_batches=2)
    Hkv, Hq, d = spec.n_kv_heads, spec.n_q_heads, spec.head_dim
    assert a.K.shape == (Hkv, spec.capacity, d) and a.V.shape == a.K.shape
    assert a.K.dtype == (np.float32 if spec.kv_dtype == "f32" else np.uint16)
    assert a.ref_q.shape == (Hkv, spec.n_ref, d) and a.ref_q.dtype == np.float32
    assert a.Q.shape == (2, spec.batch, Hq, d) and a.Q.dtype == np.float32
    for x, y in [(a.K, b.K), (a.V, b.V), (a.ref_q, b.ref_q), (a.Q, b.Q)]:
        assert np.array_equal(x, y)
    c = W.generate(spec, n_batches=2, rank=1)
    assert not np.array_equal(a.K, c.K)


def test_reference_queries_form_a_cone():
    spec = W.scaled("32k", n_tokens=4096)
    inp = W.generate(spec)
    cos = []
    for g in range(spec.n_kv_heads):
        u = inp.ref_q[g] / np.linalg.norm(inp.ref_q[g], axis=1, keepdims=True)
        cos.append((u @ u.T)[np.triu_indices(spec.n_ref, 1)])
    assert abs(np.mean(cos) - 0.44) < 0.03


def test_tiny_needles_stand_out():
    inp = W.generate("tiny")
    d = inp.spec.head_dim
    for b, h, pos in inp.meta["needles"]:
        q = inp.Q[0, b, h].astype(np.float64)
        logits = inp.K[0, : inp.spec.n_tokens].astype(np.float64) @ q / np.sqrt(d)
        others = np.delete(logits, [p for _, _, p in inp.meta["needles"]])
        assert logits[pos] >= others.max() + 6.0 - 1e-3
        assert 0 < pos < inp.spec.n_tokens - inp.spec.chunk


def test_planted_spans_are_disjoint_and_clear_of_sink_and_tail():
    spec = W.WORKLOADS["32k"]
    inp = W.generate(W.scaled(spec, n_kv_heads=2, n_q_heads=8))
    span = inp.meta["planted_span"]
    for starts in inp.meta["planted_starts"]:
        starts = np.array(starts)
        assert len(starts) == W.PLANTED_SPANS and span * W.PLANTED_SPANS >= 0.01 * spec.n_tokens
        assert np.all(np.diff(starts) >= span) and starts[0] >= 1
        assert starts[-1] + span <= spec.n_tokens - spec.chunk
