"""The C-ABI library on the host (no GPU): it loads, exports every symbol that
include/zha.h declares, and its host-side checks and layout arithmetic behave as
documented. Calls that would launch kernels are only made with arguments the
host checks reject before any CUDA call."""

import ctypes
import os
import re
import subprocess

import pytest
import torch

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "zha.h")


@pytest.fixture(scope="module")
def zha():
    from hierarchical_sparse_attention_zha_b200 import zha as z
    return z


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(zha_\w+)\s*\(", text)))


def test_header_declares_the_four_hot_path_calls():
    names = declared_functions()
    for n in ("zha_build", "zha_append_chunk", "zha_route", "zha_sparse_attend"):
        assert n in names


def test_library_exports_every_declared_symbol(zha):
    names = declared_functions()
    assert len(names) >= 16
    out = subprocess.run(["nm", "-D", "--defined-only", zha.LIB_PATH], capture_output=True,
                         text=True, check=True).stdout
    exported = set(re.findall(r" T (zha_\w+)", out))
    missing = [n for n in names if n not in exported]
    assert not missing, missing
    lib = ctypes.CDLL(zha.LIB_PATH)
    for n in names:
        assert getattr(lib, n) is not None


def test_version_and_status_strings(zha):
    assert zha.lib.zha_abi_version() == 3
    assert zha.status_str(0) == "ok"
    assert "state" in zha.status_str(zha.ZHA_ERR_STATE)
    assert zha.status_str(-99) == "unknown status"


def _cfg(zha, **kw):
    base = dict(n_kv_heads=4, n_q_heads=32, head_dim=128, chunk=64, levels=3, n_ref=16,
                kv_dtype=torch.bfloat16, max_tokens=1 << 20)
    base.update(kw)
    return zha.make_config(**base)


def test_tree_bytes_matches_the_documented_layout(zha):
    for (H, d, C, L, R, T) in [(4, 128, 64, 3, 16, 1 << 20), (1, 64, 16, 2, 4, 4096),
                               (8, 128, 4, 6, 16, 65536 + 7), (2, 64, 3, 4, 5, 1000)]:
        cfg = _cfg(zha, n_kv_heads=H, n_q_heads=H * 2, head_dim=d, chunk=C, levels=L, n_ref=R,
                   max_tokens=T)
        node = R * d + (R + 3) // 4 * 4
        floats = sum(H * (T // C ** l) * node for l in range(1, L + 1))
        # the levels, then a 256-byte block (the tree's device status word) at
        # the next 256-byte boundary, then (head_dim 128, R = 16) the planes
        # again as two fp16 terms
        terms = sum(H * 2 * (T // C ** l) * R * d * 2 for l in range(1, L + 1)) if (d, R) == (128, 16) else 0
        assert zha.tree_bytes(cfg) == (floats * 4 + 255) // 256 * 256 + 256 + terms


@pytest.mark.parametrize("field,value", [("head_dim", 96), ("chunk", 1), ("chunk", 129),
                                         ("levels", 0), ("levels", 9), ("n_ref", 0),
                                         ("n_ref", 33), ("n_q_heads", 30), ("max_tokens", 0)])
def test_invalid_configs_have_no_size(zha, field, value):
    cfg = _cfg(zha)
    setattr(cfg, field, value)
    assert zha.tree_bytes(cfg) == 0
    assert zha.route_workspace_bytes(cfg, 4, 1000) == 0


def test_route_workspace_and_kept_words_arithmetic(zha):
    cfg = _cfg(zha)
    n = (1 << 20) + 100
    nb = 64 * (n // 64)
    heads = 4 * 32
    words = sum(heads * ((nb // 64 ** l + 31) // 32) for l in (1, 2, 3))
    assert zha.route_kept_words(cfg, 4, n) == words
    ws = zha.route_workspace_bytes(cfg, 4, n)
    sig = sum(-(-heads * (nb // 64 ** l) // 64) * 64 for l in (1, 2, 3))
    assert ws >= sig * 4 + words * 4
    assert zha.route_workspace_bytes(cfg, 4, 1000) < ws        # grows with n_tokens
    # attend (bf16, d = 128: tensor-core path): union lists per (KV head, block of
    # 32 query heads) laid out in blocks of <= 2048 chunks (a multiple of 32),
    # a count per (group, block), the tile split, and one state per (CTA piece, head)
    r256 = lambda x: -(-x // 256) * 256
    groups, n_ch = 4 * 1, n // 64
    n_blocks = -(-n_ch // 2048)
    block = -(-(-(-n_ch // n_blocks)) // 32) * 32
    cap, units = n_blocks * block, groups * n_blocks
    lists = 2 * r256(groups * cap * 4)
    slots = r256((296 + groups) * 32 * 132 * 4)
    assert zha.attend_workspace_bytes(cfg, 4, n) == lists + r256(units * 4) + r256((units + 3) * 4) + slots


def test_host_checks_reject_before_any_launch(zha):
    cfg = _cfg(zha)
    handle = ctypes.c_void_p()
    st = zha.lib.zha_tree_create(ctypes.byref(cfg), None, 1 << 30, ctypes.c_void_p(256),
                                 ctypes.byref(handle))
    assert st == zha.ZHA_ERR_INVALID and "store" in zha.last_error()
    st = zha.lib.zha_tree_create(ctypes.byref(cfg), ctypes.c_void_p(4096 + 16), 1 << 30,
                                 ctypes.c_void_p(256), ctypes.byref(handle))
    assert st == zha.ZHA_ERR_INVALID                                  # misaligned store
    st = zha.lib.zha_tree_create(ctypes.byref(cfg), ctypes.c_void_p(4096), 1024,
                                 ctypes.c_void_p(256), ctypes.byref(handle))
    assert st == zha.ZHA_ERR_CAPACITY
    # a handle over fake (never dereferenced) pointers exercises the call checks
    st = zha.lib.zha_tree_create(ctypes.byref(cfg), ctypes.c_void_p(1 << 40), 1 << 34,
                                 ctypes.c_void_p(1 << 41), ctypes.byref(handle))
    assert st == zha.ZHA_OK
    try:
        P = ctypes.c_void_p
        assert zha.lib.zha_tree_built_tokens(handle) == 0
        assert zha.lib.zha_build(handle, None, 100, 10, None) == zha.ZHA_ERR_INVALID
        assert zha.lib.zha_build(handle, P(1 << 42), 100, 101, None) == zha.ZHA_ERR_INVALID
        # routing at 1000 tokens needs the tree built to 960 tokens
        rc = zha.lib.zha_route(handle, P(1 << 42), 4, 1000, 0.9, P(1 << 43), P(1 << 44), 16, None,
                               P(1 << 45), 1 << 30, None, None)
        assert rc == zha.ZHA_ERR_STATE and "960" in zha.last_error()
        rc = zha.lib.zha_route(handle, P(1 << 42), 4, 10, 0.0, P(1 << 43), P(1 << 44), 16, None,
                               P(1 << 45), 1 << 30, None, None)
        assert rc == zha.ZHA_ERR_INVALID                               # p must be > 0
        rc = zha.lib.zha_route(handle, P(1 << 42), 4, 10, 0.9, P(1 << 43), P(1 << 44), 16, None,
                               P(1 << 45), 16, None, None)
        assert rc == zha.ZHA_ERR_CAPACITY                              # workspace too small
        rc = zha.lib.zha_sparse_attend(handle, P(1 << 42), P(1 << 42), P(1 << 42), 100, 200, 4,
                                       P(1 << 43), P(1 << 44), 16, P(1 << 42), None, P(1 << 45),
                                       1 << 30, None, None)
        assert rc == zha.ZHA_ERR_INVALID                               # n_tokens > ld
        rc = zha.lib.zha_sparse_attend(handle, P(1 << 42), P(1 << 42), P(1 << 42), 100, 50, 4,
                                       P(1 << 43), P(1 << 44), 16, P(1 << 42), None, P(1 << 45),
                                       8, None, None)
        assert rc == zha.ZHA_ERR_CAPACITY
        assert zha.lib.zha_append_chunk(handle, P(1 << 42), 100, 5, None) == zha.ZHA_OK  # no new chunk
    finally:
        zha.lib.zha_tree_destroy(handle)


def test_no_cpu_fallback_exists():
    """The package ships no alternative implementation: the binding's only
    compute entry points are the C calls."""
    import hierarchical_sparse_attention_zha_b200 as pkg
    src = open(os.path.join(os.path.dirname(pkg.__file__), "zha.py")).read()
    assert "import oracle" not in src and "from oracle" not in src
    assert "numpy" not in src


def test_split_arithmetic_of_the_tensor_core_attention():
    """The combine finds the CTAs whose span met a group from the tile offsets
    alone: CTA c covers tiles [c T / n, (c + 1) T / n), so tile t belongs to CTA
    ((t + 1) n - 1) / T, and a CTA between two such CTAs wrote a state iff its
    span is non-empty. Checked exhaustively for small T and the launch sizes."""
    for n in (1, 2, 7, 148, 296):
        for T in range(1, 700):
            start = [c * T // n for c in range(n + 1)]
            for t in range(T):
                c = ((t + 1) * n - 1) // T
                assert start[c] <= t < start[c + 1]
            # a group occupying tiles [lo, hi): the CTAs the combine visits are
            # exactly those whose span intersects it
            for lo, hi in ((0, T), (T // 3, T // 3 + 1), (T // 2, T)):
                if lo >= hi:
                    continue
                c_lo, c_hi = ((lo + 1) * n - 1) // T, (hi * n - 1) // T
                visited = {c for c in range(c_lo, c_hi + 1) if (c + 1) * T // n > c * T // n}
                meets = {c for c in range(n) if max(start[c], lo) < min(start[c + 1], hi)}
                assert visited == meets


def test_route_ex_rejects_bad_policies_before_any_launch(zha):
    """zha_route_ex checks its policy on the host: NULL, unknown mode, reserved
    != 0, p <= 0 or not finite, k < 1 on a level of the tree; entries past the
    tree's levels are ignored."""
    cfg = _cfg(zha)
    handle = ctypes.c_void_p()
    assert zha.lib.zha_tree_create(ctypes.byref(cfg), ctypes.c_void_p(1 << 40), 1 << 34,
                                   ctypes.c_void_p(1 << 41), ctypes.byref(handle)) == zha.ZHA_OK
    P = ctypes.c_void_p
    before = zha.launch_count()
    try:
        def call(pol):
            return zha.lib.zha_route_ex(handle, P(1 << 42), 4, 10, pol, P(1 << 43), P(1 << 44), 16, None,
                                        P(1 << 45), 16, None, None)
        assert call(None) == zha.ZHA_ERR_INVALID and "policy" in zha.last_error()
        bad_mode = zha.top_p_policy([0.9] * 3)
        bad_mode.mode = 7
        assert call(ctypes.byref(bad_mode)) == zha.ZHA_ERR_INVALID
        res = zha.top_p_policy([0.9] * 3)
        res.reserved = 1
        assert call(ctypes.byref(res)) == zha.ZHA_ERR_INVALID
        for ps in ([0.9, 0.0, 0.9], [0.9, 0.9, float("nan")], [-1.0, 0.9, 0.9]):
            assert call(ctypes.byref(zha.top_p_policy(ps))) == zha.ZHA_ERR_INVALID
        assert call(ctypes.byref(zha.top_k_policy([5, 0, 2]))) == zha.ZHA_ERR_INVALID
        # valid policies (levels 4..8 unset) pass the policy checks and then
        # fail on the tiny workspace
        assert call(ctypes.byref(zha.top_p_policy([0.9, 0.9, 0.9]))) == zha.ZHA_ERR_CAPACITY
        assert call(ctypes.byref(zha.top_k_policy([5, 3, 2]))) == zha.ZHA_ERR_CAPACITY
        assert zha.launch_count() == before
    finally:
        zha.lib.zha_tree_destroy(handle)


def test_rotary_config_is_validated(zha):
    """rope_pairs in [0, head_dim / 2]; a base > 1 (finite) when rope_pairs > 0;
    the base is ignored without rotated pairs."""
    assert zha.tree_bytes(_cfg(zha, rope_pairs=64, rope_base=10000.0)) > 0
    assert zha.tree_bytes(_cfg(zha, rope_pairs=65, rope_base=10000.0)) == 0
    assert zha.tree_bytes(_cfg(zha, rope_pairs=-1)) == 0
    assert zha.tree_bytes(_cfg(zha, rope_pairs=8, rope_base=1.0)) == 0
    assert zha.tree_bytes(_cfg(zha, rope_pairs=8, rope_base=float("inf"))) == 0
    cfg = _cfg(zha)
    cfg.rope_base = -3.0                  # no rotated pairs: not read
    assert zha.tree_bytes(cfg) > 0
    # the rotary fields do not change the store's size
    assert zha.tree_bytes(_cfg(zha, rope_pairs=64, rope_base=10000.0)) == zha.tree_bytes(_cfg(zha))
