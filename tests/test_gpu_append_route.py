"""basiskv_append_route (the append with the route's scoring beside it as a
programmatic dependent, one stream) against the two calls on forked streams:
the same selections, latents and outputs, bit for bit, for per-head and
per-group routing; and its host-side refusals."""
import ctypes

import pytest
import torch

pytestmark = pytest.mark.gpu

from long_context_decode_basiskv_b200 import binding as bk  # noqa: E402
from long_context_decode_basiskv_b200.engine import DecodeEngine  # noqa: E402
from long_context_decode_basiskv_b200.workloads import WORKLOADS, make_case, shrink  # noqa: E402

CASES = [
    ("llama3_8b_32k", dict(batch=3, context=16 * 300 + 7, top_k=24)),
    ("llama3_70b_64k", dict(batch=2, context=16 * 260 + 3, top_k=40)),
    ("single_seq_131k", dict(batch=1, context=64 * 90 + 1, top_k=16)),
    ("tiny_fp32", dict(batch=2, context=700, top_k=6)),
    ("ragged_serving", dict(batch=6, ragged=(1, 900), top_k=12)),
]


@pytest.mark.parametrize("routing", ["head", "group_sum", "group_max"])
@pytest.mark.parametrize("base,kw", CASES, ids=[c[0] for c in CASES])
def test_append_route_matches_two_streams(base, kw, routing):
    wl = shrink(WORKLOADS[base], name=f"ar_{base}", **kw)
    outs = []
    for overlap in ("streams", "pdl"):
        eng = DecodeEngine(make_case(wl, "cuda"), routing=routing, overlap=overlap)
        for _ in range(2):  # the second step rewrites the recent page: the same values again
            eng.step()
        eng.graph_step()
        torch.cuda.synchronize()
        assert int(eng.err.item()) == 0
        # the cache compared through each sequence's pages (physical pages no sequence
        # uses are never written and hold whatever the allocation held)
        lat = [torch.cat([eng.logical(t, b).flatten() for b in range(wl.batch)])
               for t in (eng.cache.c_lat, eng.cache.k_raw, eng.cache.r_res)]
        P = wl.page_size
        summ = torch.cat([eng.cache.summary[eng.cache.block_table[b, :-(-L // P)].long()].flatten()
                          for b, L in enumerate(eng.case.lengths)])
        outs.append((eng.sel.clone(), eng.sel_cnt.clone(), eng.o_lat.clone(), eng.y.clone(), summ, *lat))
    names = ["sel", "sel_cnt", "o_lat", "y", "summary", "c_lat", "k_raw", "r_res"]
    for nm, a, b in zip(names, *outs):
        assert torch.equal(a, b), f"{nm} differs at {int((a != b).sum())} places"


def test_append_route_refusals():
    wl = shrink(WORKLOADS["llama3_8b_32k"], batch=2, context=2000, top_k=8, name="ar_refuse")
    eng = DecodeEngine(make_case(wl, "cuda"))
    L = bk.lib()
    s = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)

    def call(reduce=0, k_new=eng.k_new, ws_bytes=None):
        return L.basiskv_append_route(ctypes.byref(eng.cfg.c()), ctypes.byref(eng.cache.c()),
                                      ctypes.byref(eng.factors.c()), ctypes.c_void_p(k_new.data_ptr())
                                      if k_new is not None else None,
                                      ctypes.c_void_p(eng.v_new.data_ptr()), ctypes.c_void_p(eng.q.data_ptr()),
                                      2, reduce, ctypes.c_void_p(eng.sel.data_ptr()),
                                      ctypes.c_void_p(eng.sel_cnt.data_ptr()), ctypes.c_void_p(eng.ws.data_ptr()),
                                      eng.ws.numel() if ws_bytes is None else ws_bytes,
                                      ctypes.c_void_p(eng.err.data_ptr()), s)

    assert call(reduce=7) == bk.ERR_INVALID_ARG
    assert call(k_new=None) == bk.ERR_INVALID_ARG
    assert call(ws_bytes=16) == bk.ERR_WORKSPACE
    assert call() == bk.OK
    torch.cuda.synchronize()
    assert int(eng.err.item()) == 0
