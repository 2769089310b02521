"""ctypes binding of libbasiskv.so (include/basiskv.h).

Argument marshalling only: torch tensors are checked for device, dtype,
shape and contiguity and their device pointers are passed to the C ABI.
Every step of the decode path runs in the library's CUDA kernels; there is
no fallback.  ``lib()`` raises if the shared library is missing.
"""
from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass
from typing import Optional

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libbasiskv.so")

OK, ERR_INVALID_ARG, ERR_UNSUPPORTED, ERR_CUDA, ERR_WORKSPACE = 0, 1, 2, 3, 4
F32, BF16 = 0, 1
GROUP_SUM, GROUP_MAX = 1, 2
DEVERR_BLOCK_TABLE, DEVERR_SELECTION, DEVERR_SEQ_LEN, DEVERR_TIMEOUT, DEVERR_WORKSPACE = 1, 2, 4, 8, 16

# every function include/basiskv.h declares
SYMBOLS = [
    "basiskv_append", "basiskv_route", "basiskv_decode_attn", "basiskv_out_proj",
    "basiskv_fuse_out_factor", "basiskv_workspace_bytes", "basiskv_status_string",
    "basiskv_abi_version", "basiskv_decode_attn_noalloc", "basiskv_route_group", "basiskv_prefill",
    "basiskv_copy", "basiskv_append_route",
]


class CConfig(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int32) for n in
                ["num_q_heads", "num_kv_heads", "head_dim", "rank_v", "rank_k", "page_size",
                 "hidden", "top_k", "dtype"]]


class CCache(ctypes.Structure):
    _fields_ = [("k_raw", ctypes.c_void_p), ("c_lat", ctypes.c_void_p), ("r_res", ctypes.c_void_p),
                ("summary", ctypes.c_void_p), ("block_table", ctypes.c_void_p),
                ("seq_len", ctypes.c_void_p), ("num_phys_pages", ctypes.c_int32),
                ("max_pages", ctypes.c_int32)]


class CFactors(ctypes.Structure):
    _fields_ = [("A", ctypes.c_void_p), ("P", ctypes.c_void_p), ("E", ctypes.c_void_p),
                ("Gt", ctypes.c_void_p)]


_lib = None


def lib():
    """Load libbasiskv.so (once) and declare its signatures."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise RuntimeError(f"libbasiskv.so not built ({LIB_PATH}); run "
                           "`python -m long_context_decode_basiskv_b200.build`")
    L = ctypes.CDLL(LIB_PATH)
    vp, i32, sz = ctypes.c_void_p, ctypes.c_int32, ctypes.c_size_t
    pc, pk, pf = ctypes.POINTER(CConfig), ctypes.POINTER(CCache), ctypes.POINTER(CFactors)
    L.basiskv_append.argtypes = [pc, pk, pf, vp, vp, i32, i32, vp, vp]
    L.basiskv_prefill.argtypes = [pc, pk, pf, vp, vp, i32, i32, vp, vp]
    L.basiskv_route.argtypes = [pc, pk, vp, i32, vp, vp, vp, vp, sz, vp, vp]
    L.basiskv_route_group.argtypes = [pc, pk, vp, i32, i32, vp, vp, vp, vp, sz, vp, vp]
    L.basiskv_decode_attn.argtypes = [pc, pk, vp, i32, vp, vp, vp, vp, sz, vp, vp]
    L.basiskv_out_proj.argtypes = [pc, pf, vp, i32, vp, vp, sz, vp]
    L.basiskv_decode_attn_noalloc.argtypes = [pc, pk, vp, i32, vp, vp, vp, vp, vp]
    L.basiskv_fuse_out_factor.argtypes = [pc, vp, vp, vp, vp]
    L.basiskv_copy.argtypes = [vp, vp, sz, vp]
    L.basiskv_append_route.argtypes = [pc, pk, pf, vp, vp, vp, i32, i32, vp, vp, vp, sz, vp, vp]
    L.basiskv_workspace_bytes.argtypes = [pc, i32, i32]
    L.basiskv_workspace_bytes.restype = sz
    L.basiskv_status_string.argtypes = [i32]
    L.basiskv_status_string.restype = ctypes.c_char_p
    L.basiskv_abi_version.argtypes = []
    for name in ["basiskv_append", "basiskv_route", "basiskv_decode_attn", "basiskv_out_proj",
                 "basiskv_fuse_out_factor", "basiskv_abi_version", "basiskv_decode_attn_noalloc",
                 "basiskv_route_group", "basiskv_prefill", "basiskv_copy", "basiskv_append_route"]:
        getattr(L, name).restype = i32
    _lib = L
    return L


class BasisKVError(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = status
        super().__init__(f"{what}: {lib().basiskv_status_string(status).decode()} (status {status})")


def _check(status: int, what: str):
    if status != OK:
        raise BasisKVError(status, what)


@dataclass(frozen=True)
class Config:
    num_q_heads: int
    num_kv_heads: int
    head_dim: int
    rank_v: int
    rank_k: int
    page_size: int
    hidden: int
    top_k: int
    dtype: torch.dtype

    @property
    def group(self) -> int:
        return self.num_q_heads // self.num_kv_heads

    def c(self) -> CConfig:
        return CConfig(self.num_q_heads, self.num_kv_heads, self.head_dim, self.rank_v, self.rank_k,
                       self.page_size, self.hidden, self.top_k,
                       BF16 if self.dtype == torch.bfloat16 else F32)


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _need(t: torch.Tensor, name: str, dtype=None, shape=None):
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if dtype is not None and t.dtype != dtype:
        raise ValueError(f"{name}: dtype {t.dtype}, expected {dtype}")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name}: shape {tuple(t.shape)}, expected {tuple(shape)}")


def _need_reachable(t: torch.Tensor, name: str, dtype=None, shape=None):
    """_need, but a page-locked CPU tensor is also accepted (the kernels reach it
    through the runtime's mapping of pinned host memory)."""
    if isinstance(t, torch.Tensor) and not t.is_cuda:
        if not t.is_pinned():
            raise ValueError(f"{name} must be a CUDA tensor or a pinned CPU tensor")
        if not t.is_contiguous():
            raise ValueError(f"{name} must be contiguous")
        if dtype is not None and t.dtype != dtype:
            raise ValueError(f"{name}: dtype {t.dtype}, expected {dtype}")
        if shape is not None and tuple(t.shape) != tuple(shape):
            raise ValueError(f"{name}: shape {tuple(t.shape)}, expected {tuple(shape)}")
        return
    _need(t, name, dtype, shape)


def _stream(stream) -> ctypes.c_void_p:
    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


class PagedCache:
    """Device tensors of the paged cache (allocated by torch, owned by this object)."""

    def __init__(self, cfg: Config, num_phys_pages: int, block_table: torch.Tensor,
                 seq_len: torch.Tensor, device="cuda"):
        self.cfg = cfg
        Hkv, P, d, r, s = cfg.num_kv_heads, cfg.page_size, cfg.head_dim, cfg.rank_v, cfg.rank_k
        self.k_raw = torch.empty((num_phys_pages, Hkv, P, d), dtype=cfg.dtype, device=device)
        self.c_lat = torch.empty((num_phys_pages, Hkv, P, r), dtype=cfg.dtype, device=device)
        self.r_res = torch.empty((num_phys_pages, Hkv, P, s), dtype=cfg.dtype, device=device)
        self.summary = torch.empty((num_phys_pages, Hkv, d), dtype=torch.float32, device=device)
        self.block_table = block_table.to(device=device, dtype=torch.int32).contiguous()
        self.seq_len = seq_len.to(device=device, dtype=torch.int32).contiguous()
        self.num_phys_pages = num_phys_pages

    @property
    def batch(self) -> int:
        return self.block_table.shape[0]

    @property
    def max_pages(self) -> int:
        return self.block_table.shape[1]

    def c(self) -> CCache:
        return CCache(self.k_raw.data_ptr(), self.c_lat.data_ptr(), self.r_res.data_ptr(),
                      self.summary.data_ptr(), self.block_table.data_ptr(), self.seq_len.data_ptr(),
                      self.num_phys_pages, self.max_pages)


@dataclass
class Factors:
    A: torch.Tensor    # [Hkv, d, r]
    P: torch.Tensor    # [Hkv, r, d]
    E: torch.Tensor    # [Hkv, d, s]
    Gt: torch.Tensor   # [hidden, Hq, r]

    def c(self) -> CFactors:
        return CFactors(self.A.data_ptr(), self.P.data_ptr(), self.E.data_ptr(), self.Gt.data_ptr())


def workspace_bytes(cfg: Config, batch: int, max_pages: int) -> int:
    return int(lib().basiskv_workspace_bytes(ctypes.byref(cfg.c()), batch, max_pages))


def alloc_workspace(cfg: Config, batch: int, max_pages: int, device="cuda") -> torch.Tensor:
    """A zero-filled workspace (the library keeps its counters at zero between calls)."""
    return torch.zeros(max(workspace_bytes(cfg, batch, max_pages), 256), dtype=torch.uint8, device=device)


def fuse_out_factor(cfg: Config, Bf: torch.Tensor, W_O: torch.Tensor, Gt: torch.Tensor, stream=None):
    _need(Bf, "Bf", cfg.dtype, (cfg.num_kv_heads, cfg.rank_v, cfg.head_dim))
    _need(W_O, "W_O", cfg.dtype, (cfg.num_q_heads * cfg.head_dim, cfg.hidden))
    _need(Gt, "Gt", cfg.dtype, (cfg.hidden, cfg.num_q_heads, cfg.rank_v))
    _check(lib().basiskv_fuse_out_factor(ctypes.byref(cfg.c()), _ptr(Bf), _ptr(W_O), _ptr(Gt),
                                         _stream(stream)), "basiskv_fuse_out_factor")


def append(cfg: Config, cache: PagedCache, f: Factors, k_new: torch.Tensor, v_new: torch.Tensor,
           err: torch.Tensor, stream=None):
    """k_new, v_new: [B, n_new, Hkv, d]; cache.seq_len must already count them."""
    B, n_new = k_new.shape[0], k_new.shape[1]
    shape = (B, n_new, cfg.num_kv_heads, cfg.head_dim)
    _need(k_new, "k_new", cfg.dtype, shape)
    _need(v_new, "v_new", cfg.dtype, shape)
    _need(err, "err", torch.int32)
    _check(lib().basiskv_append(ctypes.byref(cfg.c()), ctypes.byref(cache.c()), ctypes.byref(f.c()),
                                _ptr(k_new), _ptr(v_new), B, n_new, _ptr(err), _stream(stream)),
           "basiskv_append")


def prefill(cfg: Config, cache: PagedCache, f: Factors, k_new: torch.Tensor, v_new: torch.Tensor,
            err: torch.Tensor, stream=None):
    """basiskv_append for long appends on the tensor cores (bf16): k_new, v_new [B, n_new, Hkv, d]."""
    B, n_new = k_new.shape[0], k_new.shape[1]
    shape = (B, n_new, cfg.num_kv_heads, cfg.head_dim)
    _need(k_new, "k_new", cfg.dtype, shape)
    _need(v_new, "v_new", cfg.dtype, shape)
    _need(err, "err", torch.int32)
    _check(lib().basiskv_prefill(ctypes.byref(cfg.c()), ctypes.byref(cache.c()), ctypes.byref(f.c()),
                                 _ptr(k_new), _ptr(v_new), B, n_new, _ptr(err), _stream(stream)),
           "basiskv_prefill")


def route(cfg: Config, cache: PagedCache, q: torch.Tensor, sel: torch.Tensor, sel_cnt: torch.Tensor,
          ws: torch.Tensor, err: torch.Tensor, scores: Optional[torch.Tensor] = None, stream=None):
    B = q.shape[0]
    _need(q, "q", cfg.dtype, (B, cfg.num_q_heads, cfg.head_dim))
    _need(sel, "sel", torch.int32, (B, cfg.num_q_heads, cfg.top_k + 2))
    _need(sel_cnt, "sel_cnt", torch.int32, (B, cfg.num_q_heads))
    _need(ws, "workspace", torch.uint8)
    _need(err, "err", torch.int32)
    if scores is not None:
        _need(scores, "scores", torch.float32, (B, cfg.num_q_heads, cache.max_pages))
    _check(lib().basiskv_route(ctypes.byref(cfg.c()), ctypes.byref(cache.c()), _ptr(q), B, _ptr(sel),
                               _ptr(sel_cnt), _ptr(scores), _ptr(ws), ws.numel(), _ptr(err),
                               _stream(stream)), "basiskv_route")


def append_route(cfg: Config, cache: PagedCache, f: Factors, k_new: torch.Tensor, v_new: torch.Tensor,
                 q: torch.Tensor, reduce: int, sel: torch.Tensor, sel_cnt: torch.Tensor, ws: torch.Tensor,
                 err: torch.Tensor, stream=None):
    """append (one token per sequence) then route (reduce = 0) or route_group in one call,
    the scoring running beside the append (basiskv_append_route)."""
    B = q.shape[0]
    _need(k_new, "k_new", cfg.dtype, (B, 1, cfg.num_kv_heads, cfg.head_dim))
    _need(v_new, "v_new", cfg.dtype, (B, 1, cfg.num_kv_heads, cfg.head_dim))
    _need(q, "q", cfg.dtype, (B, cfg.num_q_heads, cfg.head_dim))
    _need(sel, "sel", torch.int32, (B, cfg.num_q_heads, cfg.top_k + 2))
    _need(sel_cnt, "sel_cnt", torch.int32, (B, cfg.num_q_heads))
    _need(ws, "workspace", torch.uint8)
    _need(err, "err", torch.int32)
    _check(lib().basiskv_append_route(ctypes.byref(cfg.c()), ctypes.byref(cache.c()), ctypes.byref(f.c()),
                                      _ptr(k_new), _ptr(v_new), _ptr(q), B, reduce, _ptr(sel), _ptr(sel_cnt),
                                      _ptr(ws), ws.numel(), _ptr(err), _stream(stream)), "basiskv_append_route")


def route_group(cfg: Config, cache: PagedCache, q: torch.Tensor, reduce: int, sel: torch.Tensor,
                sel_cnt: torch.Tensor, ws: torch.Tensor, err: torch.Tensor,
                scores: Optional[torch.Tensor] = None, stream=None):
    """One selection per KV group (reduce = GROUP_SUM or GROUP_MAX of its heads' scores),
    written to the sel rows of every head of the group; scores [B][Hkv][max_pages]."""
    B = q.shape[0]
    _need(q, "q", cfg.dtype, (B, cfg.num_q_heads, cfg.head_dim))
    _need(sel, "sel", torch.int32, (B, cfg.num_q_heads, cfg.top_k + 2))
    _need(sel_cnt, "sel_cnt", torch.int32, (B, cfg.num_q_heads))
    _need(ws, "workspace", torch.uint8)
    _need(err, "err", torch.int32)
    if scores is not None:
        _need(scores, "scores", torch.float32, (B, cfg.num_kv_heads, cache.max_pages))
    _check(lib().basiskv_route_group(ctypes.byref(cfg.c()), ctypes.byref(cache.c()), _ptr(q), B, reduce,
                                     _ptr(sel), _ptr(sel_cnt), _ptr(scores), _ptr(ws), ws.numel(),
                                     _ptr(err), _stream(stream)), "basiskv_route_group")


def decode_attn(cfg: Config, cache: PagedCache, q: torch.Tensor, sel: Optional[torch.Tensor],
                sel_cnt: Optional[torch.Tensor], o_lat: torch.Tensor, ws: torch.Tensor, err: torch.Tensor,
                stream=None):
    """Attention over the pages in sel / sel_cnt, or (both None) over the selection the
    last route / route_group call left in the same workspace."""
    B = q.shape[0]
    _need(q, "q", cfg.dtype, (B, cfg.num_q_heads, cfg.head_dim))
    if (sel is None) != (sel_cnt is None):
        raise ValueError("sel and sel_cnt are given together or not at all")
    if sel is not None:
        _need(sel, "sel", torch.int32, (B, cfg.num_q_heads, cfg.top_k + 2))
        _need(sel_cnt, "sel_cnt", torch.int32, (B, cfg.num_q_heads))
    _need(o_lat, "o_lat", torch.float32, (B, cfg.num_q_heads, cfg.rank_v))
    _need(ws, "workspace", torch.uint8)
    _need(err, "err", torch.int32)
    _check(lib().basiskv_decode_attn(ctypes.byref(cfg.c()), ctypes.byref(cache.c()), _ptr(q), B,
                                     _ptr(sel), _ptr(sel_cnt), _ptr(o_lat), _ptr(ws), ws.numel(),
                                     _ptr(err), _stream(stream)), "basiskv_decode_attn")


def out_proj(cfg: Config, f: Factors, o_lat: torch.Tensor, y: torch.Tensor, ws: torch.Tensor,
             stream=None):
    B = o_lat.shape[0]
    _need(o_lat, "o_lat", torch.float32, (B, cfg.num_q_heads, cfg.rank_v))
    _need_reachable(y, "y", torch.float32, (B, cfg.hidden))  # device, or pinned host: stored there directly
    _need(ws, "workspace", torch.uint8)
    _check(lib().basiskv_out_proj(ctypes.byref(cfg.c()), ctypes.byref(f.c()), _ptr(o_lat), B, _ptr(y),
                                  _ptr(ws), ws.numel(), _stream(stream)), "basiskv_out_proj")


def copy(dst: torch.Tensor, src: torch.Tensor, stream=None):
    """dst <- src (same dtype and element count) by a kernel: either may be a CUDA tensor
    or a pinned CPU tensor (basiskv_copy)."""
    _need_reachable(dst, "dst")
    _need_reachable(src, "src", dst.dtype)
    if dst.numel() != src.numel():
        raise ValueError(f"copy: {src.numel()} elements into {dst.numel()}")
    _check(lib().basiskv_copy(_ptr(dst), _ptr(src), src.numel() * src.element_size(), _stream(stream)),
           "basiskv_copy")


def decode_attn_noalloc(cfg: Config, cache: PagedCache, q: torch.Tensor, sel: torch.Tensor,
                        sel_cnt: torch.Tensor, o_lat: torch.Tensor, err: torch.Tensor, stream=None):
    """decode_attn for callers that cannot allocate: the library's fixed 16 MiB scratch
    stands in for the workspace (see basiskv_decode_attn_noalloc in include/basiskv.h)."""
    B = q.shape[0]
    _need(q, "q", cfg.dtype, (B, cfg.num_q_heads, cfg.head_dim))
    _need(sel, "sel", torch.int32, (B, cfg.num_q_heads, cfg.top_k + 2))
    _need(sel_cnt, "sel_cnt", torch.int32, (B, cfg.num_q_heads))
    _need(o_lat, "o_lat", torch.float32, (B, cfg.num_q_heads, cfg.rank_v))
    _need(err, "err", torch.int32)
    _check(lib().basiskv_decode_attn_noalloc(ctypes.byref(cfg.c()), ctypes.byref(cache.c()), _ptr(q), B,
                                             _ptr(sel), _ptr(sel_cnt), _ptr(o_lat), _ptr(err),
                                             _stream(stream)), "basiskv_decode_attn_noalloc")
