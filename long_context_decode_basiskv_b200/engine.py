"""One decode step of BasisKV on the GPU, driven through the C ABI.

``DecodeEngine`` owns the device state of a batch: the paged cache (built by
the library's own append kernel in prefill mode), the factors with the fused
out-projection factor (built by the library's fusion kernel), the step's
inputs and outputs, and one workspace.  ``step()`` enqueues one decode step:
append and route (one basiskv_append_route call, or the two calls on two
streams), decode_attn, out_proj.  ``routing`` picks one
selection per query head ("head") or per KV group from the sum ("group_sum")
or maximum ("group_max") of its heads' page scores.  ``prefill_mode`` builds
the cache with basiskv_append ("exact", fp64 sums) or basiskv_prefill ("tc",
the tensor-core path for long appends).  ``overlap`` picks how append and
route overlap: "pdl" (one call, basiskv_append_route: the scoring runs
beside the append as its programmatic dependent, one stream) or "streams"
(basiskv_append on a forked stream beside basiskv_route, then a join).
"""
from __future__ import annotations

import torch

from . import binding as bk
from .workloads import Case


def config_of(case: Case) -> bk.Config:
    wl = case.wl
    return bk.Config(wl.num_q_heads, wl.num_kv_heads, wl.head_dim, wl.rank_v, wl.rank_k,
                     wl.page_size, wl.hidden, wl.top_k, wl.torch_dtype)


_GROUP_REDUCE = {"group_sum": bk.GROUP_SUM, "group_max": bk.GROUP_MAX}


class DecodeEngine:
    def __init__(self, case: Case, device="cuda", stream=None, routing: str = "head",
                 prefill_mode: str = "exact", overlap: str = "pdl"):
        if routing != "head" and routing not in _GROUP_REDUCE:
            raise ValueError(f"routing must be 'head', 'group_sum' or 'group_max', not {routing!r}")
        if overlap not in ("pdl", "streams"):
            raise ValueError(f"overlap must be 'pdl' or 'streams', not {overlap!r}")
        self.overlap = overlap
        if prefill_mode not in ("exact", "tc"):
            raise ValueError(f"prefill_mode must be 'exact' or 'tc', not {prefill_mode!r}")
        self.routing = routing
        self.prefill_mode = prefill_mode
        self.case = case
        self.cfg = cfg = config_of(case)
        self.device = torch.device(device)
        dev = self.device
        B = case.wl.batch
        lengths = torch.tensor(case.lengths, dtype=torch.int32)
        self.cache = bk.PagedCache(cfg, case.num_phys_pages, case.block_table, lengths, device=dev)
        self.factors = bk.Factors(case.A.to(dev).contiguous(), case.P.to(dev).contiguous(),
                                  case.E.to(dev).contiguous(),
                                  torch.empty((cfg.hidden, cfg.num_q_heads, cfg.rank_v),
                                              dtype=cfg.dtype, device=dev))
        bk.fuse_out_factor(cfg, case.Bf.to(dev).contiguous(), case.W_O.to(dev).contiguous(),
                           self.factors.Gt, stream)
        self.err = torch.zeros(1, dtype=torch.int32, device=dev)
        self.ws = bk.alloc_workspace(cfg, B, self.cache.max_pages, device=dev)
        # step inputs: the last token of every sequence, and the query; q, k_new
        # and v_new are views of one device buffer, so a caller can refresh all
        # three with one host-to-device copy (input_buffer)
        k_new = torch.stack([k[-1] for k in case.keys]).unsqueeze(1)
        v_new = torch.stack([v[-1] for v in case.values]).unsqueeze(1)
        q = case.q
        parts = [q, k_new, v_new]
        sizes = [t.numel() for t in parts]
        self._inbuf = torch.empty(sum(sizes), dtype=cfg.dtype, device=dev)
        views, off = [], 0
        for t, n in zip(parts, sizes):
            v = self._inbuf[off:off + n].view(t.shape)
            v.copy_(t.to(dev))
            views.append(v)
            off += n
        self.q, self.k_new, self.v_new = views
        # step outputs
        self.sel = torch.empty((B, cfg.num_q_heads, cfg.top_k + 2), dtype=torch.int32, device=dev)
        self.sel_cnt = torch.empty((B, cfg.num_q_heads), dtype=torch.int32, device=dev)
        self.o_lat = torch.empty((B, cfg.num_q_heads, cfg.rank_v), dtype=torch.float32, device=dev)
        self.y = torch.empty((B, cfg.hidden), dtype=torch.float32, device=dev)
        self.prefill(stream)

    def input_buffer(self) -> torch.Tensor:
        """The device buffer holding q, k_new and v_new back to back (in that order)."""
        return self._inbuf

    def prefill(self, stream=None):
        """Append every token but the last of each sequence (one call per sequence)."""
        cfg, case = self.cfg, self.case
        dev = self.device
        for b, L in enumerate(case.lengths):
            if L <= 1:
                continue
            sub = bk.PagedCache.__new__(bk.PagedCache)
            sub.__dict__.update(self.cache.__dict__)
            sub.block_table = self.cache.block_table[b:b + 1]
            sub.seq_len = torch.tensor([L - 1], dtype=torch.int32, device=dev)
            k = case.keys[b][:-1].to(dev).unsqueeze(0).contiguous()
            v = case.values[b][:-1].to(dev).unsqueeze(0).contiguous()
            fn = bk.prefill if self.prefill_mode == "tc" else bk.append
            fn(cfg, sub, self.factors, k, v, self.err, stream)

    def append(self, stream=None):
        bk.append(self.cfg, self.cache, self.factors, self.k_new, self.v_new, self.err, stream)

    def route(self, scores=None, stream=None):
        if self.routing == "head":
            bk.route(self.cfg, self.cache, self.q, self.sel, self.sel_cnt, self.ws, self.err, scores, stream)
        else:
            bk.route_group(self.cfg, self.cache, self.q, _GROUP_REDUCE[self.routing], self.sel,
                           self.sel_cnt, self.ws, self.err, scores, stream)

    def decode_attn(self, stream=None, from_route: bool = True):
        """Attention over the step's selection: by default the union lists route() left in
        the workspace; from_route=False passes sel / sel_cnt (the library rebuilds them)."""
        sel, cnt = (None, None) if from_route else (self.sel, self.sel_cnt)
        bk.decode_attn(self.cfg, self.cache, self.q, sel, cnt, self.o_lat, self.ws, self.err, stream)

    def out_proj(self, stream=None, y=None):
        """y defaults to the engine's device tensor; a pinned CPU tensor of its shape
        receives the result straight from the kernel."""
        bk.out_proj(self.cfg, self.factors, self.o_lat, self.y if y is None else y, self.ws, stream)

    def append_route(self, stream=None, host_in=None):
        """Append (on a forked stream) concurrently with route, then join.

        Without a scores output, route reads nothing the step's append writes
        (only the recent page changes, and it is kept whatever it scores).
        With `host_in` (pinned, input_buffer()'s layout) the step's inputs are
        first brought in by basiskv_copy: with overlap "pdl" all of them in one
        copy before the combined call; with "streams" k_new and v_new on the
        forked stream before the append and q on the calling stream before
        route.  (Measured in the step graph, the single copy before the
        combined call is the faster of the two on every workload but the
        64-sequence ragged batch.)
        """
        main = torch.cuda.current_stream(self.device) if stream is None else stream
        if not hasattr(self, "_aux"):
            self._aux = torch.cuda.Stream(device=self.device)
            self._fork = torch.cuda.Event()
            self._join = torch.cuda.Event()
        nq = self.q.numel()
        if self.overlap == "pdl":
            if host_in is not None:
                bk.copy(self._inbuf, host_in, main)
            bk.append_route(self.cfg, self.cache, self.factors, self.k_new, self.v_new, self.q,
                            0 if self.routing == "head" else _GROUP_REDUCE[self.routing], self.sel,
                            self.sel_cnt, self.ws, self.err, main)
            return
        self._fork.record(main)
        self._aux.wait_event(self._fork)
        if host_in is not None:
            bk.copy(self._inbuf[nq:], host_in[nq:], self._aux)
        self.append(self._aux)
        self._join.record(self._aux)
        if host_in is not None:
            bk.copy(self._inbuf[:nq], host_in[:nq], main)
        self.route(stream=main)
        main.wait_event(self._join)

    def step(self, stream=None, y=None, host_in=None):
        """One decode step: (append || route) -> decode_attn -> out_proj (into y, by
        default the engine's device tensor; inputs from `host_in` when given, see
        append_route)."""
        self.append_route(stream, host_in)
        self.decode_attn(stream)
        self.out_proj(stream, y)
        return self.y if y is None else y

    def graph_step(self):
        """step() replayed from a CUDA graph captured on first use (the inputs are
        read from and the outputs written to the engine's tensors, so a caller
        refreshes q / k_new / v_new in place between steps)."""
        if not hasattr(self, "_graph"):
            side = torch.cuda.Stream(device=self.device)
            side.wait_stream(torch.cuda.current_stream(self.device))
            with torch.cuda.stream(side):
                self.step()  # first launches (shared-memory attributes) outside the capture
            torch.cuda.current_stream(self.device).wait_stream(side)
            self._graph = torch.cuda.CUDAGraph()
            with torch.cuda.graph(self._graph, stream=side):
                self.step()
        self._graph.replay()
        return self.y

    def graph_step_host(self, host_in: torch.Tensor, host_y: torch.Tensor):
        """One decode step with host buffers, replayed from one CUDA graph: the step's
        inputs come from `host_in` (pinned, input_buffer()'s layout and dtype) through
        basiskv_copy (see append_route), the step's calls, the out-projection storing y
        straight into
        `host_y` (pinned, y's shape and dtype); no copy-engine transfer.  The graph is
        captured on the first call for these two buffers; the caller refills host_in before
        a call and reads host_y once the current stream is synchronised."""
        if not (host_in.is_pinned() and host_y.is_pinned()):
            raise ValueError("host buffers must be pinned")
        if host_in.shape != self._inbuf.shape or host_in.dtype != self._inbuf.dtype:
            raise ValueError("host_in must match input_buffer()")
        if host_y.shape != self.y.shape or host_y.dtype != self.y.dtype:
            raise ValueError("host_y must match y")
        key = (host_in.data_ptr(), host_y.data_ptr())
        if getattr(self, "_io_key", None) != key:
            side = torch.cuda.Stream(device=self.device)
            side.wait_stream(torch.cuda.current_stream(self.device))
            with torch.cuda.stream(side):
                self.step()  # first launches (shared-memory attributes) outside the capture
            torch.cuda.current_stream(self.device).wait_stream(side)
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g, stream=side):
                self.step(y=host_y, host_in=host_in)
            self._io_graph, self._io_key = g, key
        self._io_graph.replay()
        return host_y

    def kc_swizzled(self) -> bool:
        """bf16 K and C pages are stored with 16-byte chunks XOR-swizzled per row."""
        c = self.cfg
        return c.dtype == torch.bfloat16 and c.head_dim % 16 == 0 and c.rank_v % 16 == 0

    def logical(self, tensor: torch.Tensor, b: int) -> torch.Tensor:
        """Gather a per-page cache tensor [phys, Hkv, P, x] of sequence b into [Hkv, L, x],
        in token order and with the row swizzle of K and C pages undone."""
        L = self.case.lengths[b]
        n = -(-L // self.cfg.page_size)
        phys = self.cache.block_table[b, :n].long()
        t = tensor[phys]                       # [n, Hkv, P, x]
        if self.kc_swizzled() and (tensor is self.cache.k_raw or tensor is self.cache.c_lat):
            x = t.shape[-1]
            chunks = x // 8
            mask = 7 if chunks % 8 == 0 else 3 if chunks % 4 == 0 else 1 if chunks % 2 == 0 else 0
            row = torch.arange(t.shape[2], device=t.device)[:, None]
            src = ((torch.arange(chunks, device=t.device)[None, :] ^ (row & mask)) * 8)[..., None] \
                + torch.arange(8, device=t.device)                          # [P, chunks, 8]
            t = torch.gather(t, 3, src.reshape(1, 1, t.shape[2], x).expand_as(t))
        t = t.permute(1, 0, 2, 3).reshape(t.shape[1], n * self.cfg.page_size, -1)
        return t[:, :L]
