"""zha_route_noalloc: routing for callers that cannot allocate device memory.

Some callers of this library have no way to hand it a workspace: a plugin in an
inference server that owns every device allocation, a serving loop with a fixed
memory plan, or a plain C host program without a device allocator. For them
zha_route_noalloc keeps zha_route's scratch in a fixed array inside the library.
These tests call it through the C ABI and check that, on two calls in a row, it
returns exactly what zha_route returns with a caller workspace (the outputs are
integers, so the comparison is exact), with and without caller-provided kept
bitmaps, and that a call needing more scratch than the array holds is refused
before anything is launched.
"""

import ctypes

import numpy as np
import pytest
import torch

from hierarchical_sparse_attention_zha_b200 import workloads as W

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def zha():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from hierarchical_sparse_attention_zha_b200 import zha as z
    return z


def _inputs(spec, n_batches):
    inp = W.generate(spec, n_batches=n_batches)
    K = torch.from_numpy(inp.K.view(np.int16)).cuda().view(torch.bfloat16)
    return inp, K, torch.from_numpy(inp.ref_q).cuda(), torch.from_numpy(inp.Q).cuda()


def test_noalloc_route_matches_zha_route_on_two_calls_in_a_row(zha):
    spec = W.scaled("32k", n_kv_heads=2, n_q_heads=8, n_tokens=16384, stream_tokens=64)
    inp, K, refq, Q = _inputs(spec, n_batches=2)
    n_tokens = 16384 + 17
    cfg = zha.make_config(spec.n_kv_heads, spec.n_q_heads, spec.head_dim, spec.chunk, spec.levels,
                          spec.n_ref, torch.bfloat16, spec.capacity)
    tree = zha.Tree(cfg, refq)
    tree.build(K, n_tokens)
    B, Hq = spec.batch, spec.n_q_heads
    max_sel = n_tokens // spec.chunk
    words = zha.route_kept_words(cfg, B, n_tokens)
    stream = zha.stream_ptr()
    for call in range(2):
        q = Q[call].contiguous()
        bits_ref = torch.zeros(words, dtype=torch.int32, device="cuda")
        st_ref = torch.zeros(1, dtype=torch.int32, device="cuda")
        ids_ref, cnt_ref = tree.route(q, n_tokens, spec.p, max_sel, kept_bits=bits_ref, status=st_ref)
        outs = []
        for with_bits in (True, False):
            ids = torch.full((B, Hq, max_sel), -1, dtype=torch.int32, device="cuda")
            cnt = torch.full((B, Hq), -1, dtype=torch.int32, device="cuda")
            bits = torch.zeros(words, dtype=torch.int32, device="cuda") if with_bits else None
            st = torch.zeros(1, dtype=torch.int32, device="cuda")
            rc = zha.lib.zha_route_noalloc(tree.handle, zha.ptr(q), B, n_tokens, spec.p,
                                           zha.ptr(ids), zha.ptr(cnt), max_sel, zha.ptr(bits),
                                           zha.ptr(st), stream)
            assert rc == zha.ZHA_OK, zha.last_error()
            outs.append((ids, cnt, bits, st))
        torch.cuda.synchronize()
        for ids, cnt, bits, st in outs:
            assert torch.equal(cnt, cnt_ref)
            for b in range(B):
                for h in range(Hq):
                    n = int(cnt_ref[b, h])
                    assert torch.equal(ids[b, h, :n], ids_ref[b, h, :n])
            if bits is not None:
                assert torch.equal(bits, bits_ref)
            assert int(st.item()) == int(st_ref.item())


def test_noalloc_route_refuses_calls_beyond_its_fixed_scratch(zha):
    spec = W.scaled("tiny", n_needles=0)
    inp = W.generate(spec)
    cfg = zha.make_config(spec.n_kv_heads, spec.n_q_heads, spec.head_dim, spec.chunk, spec.levels,
                          spec.n_ref, torch.float32, spec.capacity)
    tree = zha.Tree(cfg, torch.from_numpy(inp.ref_q).cuda())
    tree.build(torch.from_numpy(inp.K).cuda(), spec.n_tokens)
    batch = 65535                      # scores alone need ~285 MB here
    assert zha.route_workspace_bytes(cfg, batch, spec.n_tokens) > (32 << 20)
    q = torch.zeros(1, spec.n_q_heads, spec.head_dim, dtype=torch.float32, device="cuda")
    ids = torch.zeros(1, dtype=torch.int32, device="cuda")
    before = zha.launch_count()
    rc = zha.lib.zha_route_noalloc(tree.handle, zha.ptr(q), batch, spec.n_tokens, spec.p,
                                   zha.ptr(ids), zha.ptr(ids), 1, None, None, zha.stream_ptr())
    assert rc == zha.ZHA_ERR_CAPACITY
    assert "scratch" in zha.last_error() and "zha_route" in zha.last_error()
    assert zha.launch_count() == before


def test_noalloc_route_allocates_nothing(zha):
    """The property the entry point exists for: after a first call (which may
    load the library's module on the device and reserve its fixed scratch), a
    further call changes neither the device's free memory nor torch's caching
    allocator (no cudaMalloc, no torch allocation)."""
    spec = W.scaled("32k", n_kv_heads=1, n_q_heads=4, n_tokens=8192, stream_tokens=64)
    inp, K, refq, Q = _inputs(spec, n_batches=1)
    n_tokens = 8192 + 5
    cfg = zha.make_config(spec.n_kv_heads, spec.n_q_heads, spec.head_dim, spec.chunk, spec.levels,
                          spec.n_ref, torch.bfloat16, spec.capacity)
    tree = zha.Tree(cfg, refq)
    tree.build(K, n_tokens)
    B, Hq = spec.batch, spec.n_q_heads
    max_sel = n_tokens // spec.chunk
    q = Q[0].contiguous()
    ids = torch.empty((B, Hq, max_sel), dtype=torch.int32, device="cuda")
    cnt = torch.empty((B, Hq), dtype=torch.int32, device="cuda")
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    stream = zha.stream_ptr()

    def call():
        rc = zha.lib.zha_route_noalloc(tree.handle, zha.ptr(q), B, n_tokens, spec.p, zha.ptr(ids),
                                       zha.ptr(cnt), max_sel, None, zha.ptr(st), stream)
        assert rc == zha.ZHA_OK, zha.last_error()
        torch.cuda.synchronize()

    call()                                     # first call on the device: set-up
    free0, _ = torch.cuda.mem_get_info()
    stats0 = torch.cuda.memory_stats()
    call()
    free1, _ = torch.cuda.mem_get_info()
    stats1 = torch.cuda.memory_stats()
    assert free1 == free0
    for key in ("allocation.all.allocated", "segment.all.allocated", "allocated_bytes.all.allocated"):
        assert stats1.get(key, 0) == stats0.get(key, 0), key
    assert int(st.item()) == 0
