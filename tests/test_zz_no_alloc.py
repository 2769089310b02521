"""basiskv_decode_attn_noalloc: sparse attention for callers that cannot
allocate device memory (an engine plugin whose host owns every allocation,
work enqueued while a stream is being captured, a fixed memory budget).

It must give what basiskv_decode_attn gives with a caller workspace, on two
calls in a row (the second reuses the library's fixed scratch as the first
left it), and must refuse shapes whose scratch would not fit.  This file is
collected last; it builds its own inputs, so it also passes on its own in a
fresh process.
"""
import ctypes

import pytest
import torch

from tests.harness import assert_close, storage_of

pytestmark = pytest.mark.gpu

from long_context_decode_basiskv_b200 import binding as bk  # noqa: E402
from long_context_decode_basiskv_b200.engine import DecodeEngine  # noqa: E402
from long_context_decode_basiskv_b200.workloads import WORKLOADS, make_case, shrink  # noqa: E402


@pytest.mark.parametrize("wl", [
    shrink(WORKLOADS["llama3_8b_32k"], batch=4, context=6001, top_k=64, name="noalloc_bf16"),
    WORKLOADS["tiny_fp32"],
], ids=["bf16", "fp32"])
def test_noalloc_matches_workspace_call_twice(wl):
    eng = DecodeEngine(make_case(wl, "cuda"))
    eng.append()
    eng.route()
    eng.decode_attn()                       # the call with a caller workspace
    torch.cuda.synchronize()
    want = eng.o_lat.cpu().numpy()
    for _ in range(2):
        o = torch.full_like(eng.o_lat, float("nan"))
        bk.decode_attn_noalloc(eng.cfg, eng.cache, eng.q, eng.sel, eng.sel_cnt, o, eng.err)
        torch.cuda.synchronize()
        assert int(eng.err.item()) == 0
        assert_close(o.cpu().numpy(), want, storage_of(wl), "noalloc o_lat vs workspace o_lat")


def test_noalloc_refuses_shapes_beyond_its_scratch():
    """A batch whose scratch would not fit the fixed array is refused before any launch.  Every
    buffer is sized for that batch (empty sequences), so even a call that got through would only
    touch valid memory."""
    wl = shrink(WORKLOADS["llama3_8b_32k"], batch=2, context=2000, top_k=16, name="noalloc_big")
    eng = DecodeEngine(make_case(wl, "cuda"))
    too_many = 4096                         # sequences whose partials need far more than 16 MiB
    cfg = eng.cfg
    q = torch.zeros((too_many, cfg.num_q_heads, cfg.head_dim), dtype=cfg.dtype, device="cuda")
    sel = torch.full((too_many, cfg.num_q_heads, cfg.top_k + 2), -1, dtype=torch.int32, device="cuda")
    cnt = torch.zeros((too_many, cfg.num_q_heads), dtype=torch.int32, device="cuda")
    o = torch.zeros((too_many, cfg.num_q_heads, cfg.rank_v), dtype=torch.float32, device="cuda")
    bt = torch.zeros((too_many, eng.cache.max_pages), dtype=torch.int32, device="cuda")
    sl = torch.zeros((too_many,), dtype=torch.int32, device="cuda")
    c = eng.cache.c()
    big = bk.CCache(c.k_raw, c.c_lat, c.r_res, c.summary, bt.data_ptr(), sl.data_ptr(), c.num_phys_pages,
                    c.max_pages)
    st = bk.lib().basiskv_decode_attn_noalloc(
        ctypes.byref(cfg.c()), ctypes.byref(big), q.data_ptr(), too_many, sel.data_ptr(), cnt.data_ptr(),
        o.data_ptr(), eng.err.data_ptr(), None)
    assert st == bk.ERR_WORKSPACE
