"""Python binding of libzha (the C ABI in include/zha.h).

Argument marshalling only: every step of the hot path runs in the library's
CUDA kernels. Tensors are torch CUDA tensors (PyTorch supplies device memory
and streams); their data pointers and the current stream are handed to the C
calls. Importing this module raises if libzha.so has not been built -- there is
no fallback implementation.
"""

from __future__ import annotations

import ctypes
import os
from ctypes import POINTER, byref, c_char_p, c_float, c_int32, c_int64, c_size_t, c_uint64, c_void_p

import torch

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libzha.so")

ZHA_OK = 0
ZHA_ERR_INVALID = -1
ZHA_ERR_CAPACITY = -2
ZHA_ERR_STATE = -3
ZHA_ERR_CUDA = -4
ZHA_ERR_UNSUPPORTED = -6
ZHA_F32 = 0
ZHA_BF16 = 1
ZHA_DEV_SELECTION_TRUNCATED = 1
ZHA_DEV_BAD_SELECTION = 2
ZHA_DEV_TIMEOUT = 4
ZHA_DEV_BAD_PAGE = 8


class ZhaError(RuntimeError):
    def __init__(self, status: int, message: str):
        super().__init__(message)
        self.status = status


ZHA_SELECT_TOP_P = 0
ZHA_SELECT_TOP_K = 1


class RoutePolicy(ctypes.Structure):
    """zha_route_policy: per-level top-p masses or top-k budgets (level l at index l-1)."""
    _fields_ = [("mode", c_int32), ("reserved", c_int32), ("p", c_float * 8), ("k", c_int32 * 8)]


def top_p_policy(p_by_level) -> RoutePolicy:
    """Top-p with p_by_level[l-1] at level l (a sequence of up to 8 masses)."""
    pol = RoutePolicy()
    pol.mode = ZHA_SELECT_TOP_P
    for i, v in enumerate(p_by_level):
        pol.p[i] = float(v)
    return pol


def top_k_policy(k_by_level) -> RoutePolicy:
    """Fixed-budget top-K with k_by_level[l-1] nodes kept at level l."""
    pol = RoutePolicy()
    pol.mode = ZHA_SELECT_TOP_K
    for i, v in enumerate(k_by_level):
        pol.k[i] = int(v)
    return pol


class KvCache(ctypes.Structure):
    """zha_kv_cache: a contiguous [Hkv, ld, d] cache, or page pools [n_pages, C, d]
    with a block table [Hkv, max_blocks] (int32 page ids)."""
    _fields_ = [("k", c_void_p), ("v", c_void_p), ("ld", c_int64), ("block_table", c_void_p),
                ("max_blocks", c_int64)]


def kv_cache(K: torch.Tensor, V: torch.Tensor | None = None,
             block_table: torch.Tensor | None = None) -> KvCache:
    """A zha_kv_cache over torch tensors: contiguous when block_table is None
    (K [Hkv, ld, d]), else page pools K, V [n_pages, C, d] and block_table
    [Hkv, max_blocks] int32."""
    c = KvCache()
    c.k = K.data_ptr()
    c.v = V.data_ptr() if V is not None else None
    c.ld = K.shape[0] if block_table is not None else K.shape[1]
    if block_table is not None:
        if not (block_table.is_cuda and block_table.dtype == torch.int32 and block_table.is_contiguous()):
            raise ValueError("block_table must be a contiguous int32 CUDA tensor [Hkv, max_blocks]")
        c.block_table = block_table.data_ptr()
        c.max_blocks = block_table.shape[1]
    return c


class Config(ctypes.Structure):
    _fields_ = [
        ("n_kv_heads", c_int32), ("n_q_heads", c_int32), ("head_dim", c_int32),
        ("chunk", c_int32), ("levels", c_int32), ("n_ref", c_int32),
        ("kv_dtype", c_int32), ("rope_pairs", c_int32), ("max_tokens", c_int64),
        ("rope_base", c_float), ("reserved", c_int32),
    ]


def _load() -> ctypes.CDLL:
    if not os.path.exists(LIB_PATH):
        raise ImportError(
            f"{LIB_PATH} is missing: build it with `python -m "
            "hierarchical_sparse_attention_zha_b200.build` (there is no CPU fallback)")
    lib = ctypes.CDLL(LIB_PATH)
    P = c_void_p
    sig = {
        "zha_abi_version": (c_int32, []),
        "zha_status_str": (c_char_p, [c_int32]),
        "zha_last_error": (c_char_p, []),
        "zha_launch_count": (c_uint64, []),
        "zha_tree_bytes": (c_size_t, [POINTER(Config)]),
        "zha_tree_create": (c_int32, [POINTER(Config), P, c_size_t, P, POINTER(P)]),
        "zha_tree_destroy": (None, [P]),
        "zha_tree_built_tokens": (c_int64, [P]),
        "zha_tree_level_layout": (c_int32, [P, c_int32, POINTER(c_int64), POINTER(c_int64),
                                            POINTER(c_int32)]),
        "zha_build": (c_int32, [P, P, c_int64, c_int64, P]),
        "zha_append_chunk": (c_int32, [P, P, c_int64, c_int64, P]),
        "zha_route_workspace_bytes": (c_size_t, [POINTER(Config), c_int32, c_int64]),
        "zha_route_kept_words": (c_size_t, [POINTER(Config), c_int32, c_int64]),
        "zha_route": (c_int32, [P, P, c_int32, c_int64, c_float, P, P, c_int32, P, P, c_size_t,
                                P, P]),
        "zha_route_noalloc": (c_int32, [P, P, c_int32, c_int64, c_float, P, P, c_int32, P, P, P]),
        "zha_route_ex": (c_int32, [P, P, c_int32, c_int64, POINTER(RoutePolicy), P, P, c_int32, P, P,
                                   c_size_t, P, P]),
        "zha_attend_workspace_bytes": (c_size_t, [POINTER(Config), c_int32, c_int64]),
        "zha_sparse_attend": (c_int32, [P, P, P, P, c_int64, c_int64, c_int32, P, P, c_int32, P,
                                        P, P, c_size_t, P, P]),
        "zha_build_kv": (c_int32, [P, POINTER(KvCache), c_int64, P]),
        "zha_append_chunk_kv": (c_int32, [P, POINTER(KvCache), c_int64, P]),
        "zha_sparse_attend_kv": (c_int32, [P, P, POINTER(KvCache), c_int64, c_int32, P, P, c_int32, P, P,
                                           P, c_size_t, P, P]),
        "zha_diagnostics_workspace_bytes": (c_size_t, [POINTER(Config), c_int32, c_int64]),
        "zha_route_diagnostics": (c_int32, [P, P, P, c_int64, c_int32, c_int64, P, P, P, c_size_t, P]),
        "zha_tree_debug": (c_int32, [P, ctypes.c_uint32, c_int32]),
        "zha_trace_enable": (c_int32, [c_int32, c_char_p, c_int32]),
        "zha_trace_count": (c_int32, []),
        "zha_trace_dropped": (c_int32, []),
        "zha_trace_read": (c_int32, [c_int32, POINTER(c_char_p), POINTER(c_int32), POINTER(c_float)]),
        "zha_trace_clear": (None, []),
    }
    for name, (res, args) in sig.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    return lib


lib = _load()


def status_str(status: int) -> str:
    return lib.zha_status_str(status).decode()


def last_error() -> str:
    return lib.zha_last_error().decode()


def launch_count() -> int:
    return int(lib.zha_launch_count())


def check(status: int, what: str) -> None:
    if status != ZHA_OK:
        raise ZhaError(status, f"{what}: {status_str(status)}: {last_error()}")


def ptr(t: torch.Tensor | None):
    return None if t is None else c_void_p(t.data_ptr())


def stream_ptr(stream: torch.cuda.Stream | None = None):
    s = stream if stream is not None else torch.cuda.current_stream()
    return c_void_p(s.cuda_stream)


def trace_enable(max_records: int, name_filter: str | None = None, tag_filter: int = -1) -> None:
    """Record CUDA events around the library's kernel launches (see zha.h)."""
    check(lib.zha_trace_enable(max_records, name_filter.encode() if name_filter else None, tag_filter),
          "zha_trace_enable")


def trace_records() -> list[tuple[str, int, float]]:
    """(kernel name, tag, device ms) of every recorded launch; synchronise first."""
    out = []
    for i in range(int(lib.zha_trace_count())):
        name, tag, ms = c_char_p(), c_int32(), c_float()
        check(lib.zha_trace_read(i, byref(name), byref(tag), byref(ms)), "zha_trace_read")
        out.append((name.value.decode(), int(tag.value), float(ms.value)))
    return out


def trace_dropped() -> int:
    return int(lib.zha_trace_dropped())


def trace_clear() -> None:
    lib.zha_trace_clear()


def make_config(n_kv_heads: int, n_q_heads: int, head_dim: int, chunk: int, levels: int,
                n_ref: int, kv_dtype: torch.dtype, max_tokens: int, rope_pairs: int = 0,
                rope_base: float = 10000.0) -> Config:
    """zha_config; rope_pairs > 0 declares rotary positions (see zha.h)."""
    dt = {torch.float32: ZHA_F32, torch.bfloat16: ZHA_BF16}[kv_dtype]
    return Config(n_kv_heads, n_q_heads, head_dim, chunk, levels, n_ref, dt, rope_pairs, max_tokens,
                  rope_base if rope_pairs > 0 else 0.0, 0)


def tree_bytes(cfg: Config) -> int:
    return int(lib.zha_tree_bytes(byref(cfg)))


def route_workspace_bytes(cfg: Config, batch: int, n_tokens: int) -> int:
    return int(lib.zha_route_workspace_bytes(byref(cfg), batch, n_tokens))


def route_kept_words(cfg: Config, batch: int, n_tokens: int) -> int:
    return int(lib.zha_route_kept_words(byref(cfg), batch, n_tokens))


def attend_workspace_bytes(cfg: Config, batch: int, n_tokens: int) -> int:
    return int(lib.zha_attend_workspace_bytes(byref(cfg), batch, n_tokens))


def _bytes_tensor(nbytes: int, device) -> torch.Tensor:
    return torch.empty(max(1, (nbytes + 255) // 256) * 64, dtype=torch.float32, device=device)


class Tree:
    """One summary store (all KV heads) plus its C handle.

    ``ref_q``: float32 CUDA tensor [n_kv_heads, n_ref, head_dim], kept alive here.
    """

    def __init__(self, cfg: Config, ref_q: torch.Tensor):
        if not (ref_q.is_cuda and ref_q.dtype == torch.float32 and ref_q.is_contiguous()):
            raise ValueError("ref_q must be a contiguous float32 CUDA tensor")
        if tuple(ref_q.shape) != (cfg.n_kv_heads, cfg.n_ref, cfg.head_dim):
            raise ValueError("ref_q shape does not match the config")
        self.cfg = cfg
        self.ref_q = ref_q
        self.device = ref_q.device
        nbytes = tree_bytes(cfg)
        if nbytes == 0:
            check(ZHA_ERR_INVALID, "zha_tree_bytes")
        self.store = _bytes_tensor(nbytes, self.device)
        handle = c_void_p()
        check(lib.zha_tree_create(byref(cfg), ptr(self.store), self.store.numel() * 4, ptr(ref_q),
                                  byref(handle)), "zha_tree_create")
        self.handle = handle

    def __del__(self):
        h = getattr(self, "handle", None)
        # (at interpreter exit the module's globals may already be gone)
        if h is not None and h.value and lib is not None:
            lib.zha_tree_destroy(h)
            self.handle = None

    @property
    def built_tokens(self) -> int:
        return int(lib.zha_tree_built_tokens(self.handle))

    def _kv(self, K: torch.Tensor) -> None:
        want = torch.float32 if self.cfg.kv_dtype == ZHA_F32 else torch.bfloat16
        if not (K.is_cuda and K.dtype == want and K.is_contiguous() and K.dim() == 3
                and K.shape[0] == self.cfg.n_kv_heads and K.shape[2] == self.cfg.head_dim):
            raise ValueError(f"cache must be a contiguous {want} CUDA tensor [Hkv, ld, d]")

    def build(self, K: torch.Tensor, n_tokens: int, stream=None) -> None:
        self._kv(K)
        check(lib.zha_build(self.handle, ptr(K), K.shape[1], n_tokens, stream_ptr(stream)),
              "zha_build")

    def append_chunk(self, K: torch.Tensor, n_tokens: int, stream=None) -> None:
        self._kv(K)
        check(lib.zha_append_chunk(self.handle, ptr(K), K.shape[1], n_tokens, stream_ptr(stream)),
              "zha_append_chunk")

    def build_kv(self, kv: KvCache, n_tokens: int, stream=None) -> None:
        """zha_build_kv over a zha_kv_cache (see kv_cache())."""
        check(lib.zha_build_kv(self.handle, byref(kv), n_tokens, stream_ptr(stream)), "zha_build_kv")

    def append_chunk_kv(self, kv: KvCache, n_tokens: int, stream=None) -> None:
        check(lib.zha_append_chunk_kv(self.handle, byref(kv), n_tokens, stream_ptr(stream)),
              "zha_append_chunk_kv")

    def sparse_attend_kv(self, Q: torch.Tensor, kv: KvCache, n_tokens: int, chunk_ids: torch.Tensor,
                         n_chunks: torch.Tensor, out: torch.Tensor | None = None,
                         lse: torch.Tensor | None = None, ws: torch.Tensor | None = None,
                         status: torch.Tensor | None = None, stream=None):
        B = Q.shape[0]
        if out is None:
            out = torch.empty(B, self.cfg.n_q_heads, self.cfg.head_dim, dtype=torch.float32,
                              device=self.device)
        if lse is None:
            lse = torch.empty(B, self.cfg.n_q_heads, dtype=torch.float32, device=self.device)
        if ws is None:
            ws = _bytes_tensor(attend_workspace_bytes(self.cfg, B, n_tokens), self.device)
        check(lib.zha_sparse_attend_kv(self.handle, ptr(Q), byref(kv), n_tokens, B, ptr(chunk_ids),
                                       ptr(n_chunks), chunk_ids.shape[-1], ptr(out), ptr(lse), ptr(ws),
                                       ws.numel() * ws.element_size(), ptr(status), stream_ptr(stream)),
              "zha_sparse_attend_kv")
        return out, lse

    def level(self, level: int) -> tuple[torch.Tensor, torch.Tensor]:
        """Views of level `level`'s summaries: khat [Hkv, cap, R, d], bhat [Hkv, cap, R]."""
        off, cap, nf = c_int64(), c_int64(), c_int32()
        check(lib.zha_tree_level_layout(self.handle, level, byref(off), byref(cap), byref(nf)),
              "zha_tree_level_layout")
        H, R, d = self.cfg.n_kv_heads, self.cfg.n_ref, self.cfg.head_dim
        blk = self.store[off.value: off.value + H * cap.value * nf.value].view(H, cap.value, nf.value)
        return blk[:, :, : R * d].reshape(H, cap.value, R, d), blk[:, :, R * d: R * d + R]

    def route(self, Q: torch.Tensor, n_tokens: int, p: "float | RoutePolicy", max_sel: int,
              chunk_ids: torch.Tensor | None = None, n_chunks: torch.Tensor | None = None,
              kept_bits: torch.Tensor | None = None, ws: torch.Tensor | None = None,
              status: torch.Tensor | None = None, stream=None):
        B = Q.shape[0]
        if chunk_ids is None:
            chunk_ids = torch.empty(B, self.cfg.n_q_heads, max_sel, dtype=torch.int32, device=self.device)
        if n_chunks is None:
            n_chunks = torch.empty(B, self.cfg.n_q_heads, dtype=torch.int32, device=self.device)
        if ws is None:
            ws = _bytes_tensor(route_workspace_bytes(self.cfg, B, n_tokens), self.device)
        if isinstance(p, RoutePolicy):
            check(lib.zha_route_ex(self.handle, ptr(Q), B, n_tokens, byref(p), ptr(chunk_ids),
                                   ptr(n_chunks), max_sel, ptr(kept_bits), ptr(ws),
                                   ws.numel() * ws.element_size(), ptr(status), stream_ptr(stream)),
                  "zha_route_ex")
        else:
            check(lib.zha_route(self.handle, ptr(Q), B, n_tokens, p, ptr(chunk_ids), ptr(n_chunks),
                                max_sel, ptr(kept_bits), ptr(ws), ws.numel() * ws.element_size(),
                                ptr(status), stream_ptr(stream)), "zha_route")
        return chunk_ids, n_chunks

    def diagnostics(self, Q: torch.Tensor, K: torch.Tensor, n_tokens: int, usage: bool = True,
                    stream=None):
        """zha_route_diagnostics: (kl [L, B, Hq] float32, usage [L, R] int64 or None)."""
        self._kv(K)
        B = Q.shape[0]
        L = self.cfg.levels
        kl = torch.empty(L, B, self.cfg.n_q_heads, dtype=torch.float32, device=self.device)
        use = torch.zeros(L, self.cfg.n_ref, dtype=torch.int32, device=self.device) if usage else None
        ws = _bytes_tensor(int(lib.zha_diagnostics_workspace_bytes(byref(self.cfg), B, n_tokens)),
                           self.device)
        check(lib.zha_route_diagnostics(self.handle, ptr(Q), ptr(K), K.shape[1], B, n_tokens, ptr(kl),
                                        ptr(use), ptr(ws), ws.numel() * 4, stream_ptr(stream)),
              "zha_route_diagnostics")
        return kl, (use.to(torch.int64) if use is not None else None)

    def sparse_attend(self, Q: torch.Tensor, K: torch.Tensor, V: torch.Tensor, n_tokens: int,
                      chunk_ids: torch.Tensor, n_chunks: torch.Tensor,
                      out: torch.Tensor | None = None, lse: torch.Tensor | None = None,
                      ws: torch.Tensor | None = None, status: torch.Tensor | None = None,
                      stream=None):
        self._kv(K)
        self._kv(V)
        B = Q.shape[0]
        if out is None:
            out = torch.empty(B, self.cfg.n_q_heads, self.cfg.head_dim, dtype=torch.float32,
                              device=self.device)
        if lse is None:
            lse = torch.empty(B, self.cfg.n_q_heads, dtype=torch.float32, device=self.device)
        if ws is None:
            ws = _bytes_tensor(attend_workspace_bytes(self.cfg, B, n_tokens), self.device)
        check(lib.zha_sparse_attend(self.handle, ptr(Q), ptr(K), ptr(V), K.shape[1], n_tokens, B,
                                    ptr(chunk_ids), ptr(n_chunks), chunk_ids.shape[-1], ptr(out),
                                    ptr(lse), ptr(ws), ws.numel() * ws.element_size(), ptr(status),
                                    stream_ptr(stream)), "zha_sparse_attend")
        return out, lse
