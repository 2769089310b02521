"""CUDA path vs the fp64 oracle, step by step and end to end, on small
workloads that keep the oracle within seconds but still span many tiles,
partial last pages and (for the ragged batch) shuffled block tables.
"""
import numpy as np
import pytest
import torch

from tests.harness import (OracleCase, assert_close, assert_stored_equal, gt_plain, oracle_on_selection,
                           selection_ok, storage_of, to64)

pytestmark = pytest.mark.gpu

from long_context_decode_basiskv_b200 import binding as bk  # noqa: E402
from long_context_decode_basiskv_b200.engine import DecodeEngine  # noqa: E402
from long_context_decode_basiskv_b200.workloads import WORKLOADS, make_case, shrink  # noqa: E402

SMALL = {
    "tiny_fp32": WORKLOADS["tiny_fp32"],
    "l8b_small": shrink(WORKLOADS["llama3_8b_32k"], batch=3, context=8001, name="l8b_small"),
    "hot_small": shrink(WORKLOADS["single_seq_131k"], context=64 * 300 + 17, name="hot_small"),
    "l70b_small": shrink(WORKLOADS["llama3_70b_64k"], batch=2, context=9000, name="l70b_small"),
    "ragged_small": shrink(WORKLOADS["ragged_serving"], batch=6, ragged=(100, 3000), top_k=32,
                           name="ragged_small"),
}


class Run:
    def __init__(self, wl):
        self.wl = wl
        self.case = make_case(wl, "cuda")
        self.eng = DecodeEngine(self.case)
        self.scores = torch.full((wl.batch, wl.num_q_heads, self.eng.cache.max_pages), float("nan"),
                                 device="cuda")
        self.eng.append()
        self.eng.route(scores=self.scores)
        self.eng.decode_attn()
        self.eng.out_proj()
        torch.cuda.synchronize()
        self.oc = OracleCase(self.case)
        self.ref = [self.oc.sequence(b) for b in range(wl.batch)]
        self.outputs = (self.eng.sel.clone(), self.eng.sel_cnt.clone(), self.eng.o_lat.clone(), self.eng.y.clone())


@pytest.fixture(scope="module", params=sorted(SMALL))
def run(request):
    r = Run(SMALL[request.param])
    yield r
    del r
    torch.cuda.empty_cache()


def test_no_device_error(run):
    assert int(run.eng.err.item()) == 0


def test_append_stores_exact_latents_and_summaries(run):
    eng, wl = run.eng, run.wl
    for b, (cache, _) in enumerate(run.ref):
        L = run.case.lengths[b]
        n = -(-L // wl.page_size)
        C = to64(eng.logical(eng.cache.c_lat, b))
        R = to64(eng.logical(eng.cache.r_res, b))
        K = to64(eng.logical(eng.cache.k_raw, b))
        st = storage_of(wl)
        assert_stored_equal(C, cache.C[:, :L], st, f"C b={b}")
        assert_stored_equal(R, cache.R[:, :L], st, f"R b={b}")
        np.testing.assert_array_equal(K, to64(run.case.keys[b]).transpose(1, 0, 2))
        phys = eng.cache.block_table[b, :n].long()
        S = to64(eng.cache.summary[phys]).transpose(1, 0, 2)
        assert_stored_equal(S, cache.S[:, :n], "f32", f"summary b={b}", max_frac=1e-3)


def test_route_selection_and_scores(run):
    eng, wl = run.eng, run.wl
    sel = eng.sel.cpu().numpy()
    cnt = eng.sel_cnt.cpu().numpy()
    scores = run.scores.cpu().numpy()
    exact = 0
    for b, (_, out) in enumerate(run.ref):
        n = -(-run.case.lengths[b] // wl.page_size)
        for h in range(wl.num_q_heads):
            ok, ex = selection_ok(sel[b, h], cnt[b, h], out["sel"][h], out["scores"][h])
            assert ok, f"b={b} h={h}: gpu {sel[b, h][:cnt[b, h]]} oracle {out['sel'][h]}"
            exact += ex
            ref = out["scores"][h]
            tol = 1e-5 * np.max(np.abs(ref))
            assert np.max(np.abs(scores[b, h, :n] - ref)) <= tol
    assert exact >= 0.99 * wl.batch * wl.num_q_heads


def test_route_on_oracle_summaries(run):
    """Step-wise: route over summaries written by the oracle, not by the GPU append."""
    eng, wl = run.eng, run.wl
    saved = eng.cache.summary.clone()
    try:
        for b, (cache, _) in enumerate(run.ref):
            n = -(-run.case.lengths[b] // wl.page_size)
            phys = eng.cache.block_table[b, :n].long()
            eng.cache.summary[phys] = torch.from_numpy(cache.S[:, :n].transpose(1, 0, 2).copy()).float().cuda()
        sel = torch.empty_like(eng.sel)
        cnt = torch.empty_like(eng.sel_cnt)
        bk.route(eng.cfg, eng.cache, eng.q, sel, cnt, eng.ws, eng.err)
        sel, cnt = sel.cpu().numpy(), cnt.cpu().numpy()
        for b, (_, out) in enumerate(run.ref):
            for h in range(wl.num_q_heads):
                ok, _ = selection_ok(sel[b, h], cnt[b, h], out["sel"][h], out["scores"][h])
                assert ok
    finally:
        eng.cache.summary.copy_(saved)


def test_decode_attn_on_oracle_selection(run):
    """Step-wise: the oracle's page selection drives the GPU sparse attention."""
    eng, wl = run.eng, run.wl
    sel = torch.full_like(eng.sel, -1)
    cnt = torch.zeros_like(eng.sel_cnt)
    for b, (_, out) in enumerate(run.ref):
        for h in range(wl.num_q_heads):
            s = out["sel"][h]
            sel[b, h, :len(s)] = torch.from_numpy(s.astype(np.int32))
            cnt[b, h] = len(s)
    o_lat = torch.empty_like(eng.o_lat)
    bk.decode_attn(eng.cfg, eng.cache, eng.q, sel.contiguous(), cnt.contiguous(), o_lat, eng.ws, eng.err)
    got = o_lat.cpu().numpy()
    want = np.stack([out["o_lat"] for _, out in run.ref])
    assert_close(got, want, storage_of(wl), "o_lat (oracle selection)")
    assert int(eng.err.item()) == 0


def test_fused_factor_is_exact(run):
    cfg = run.eng.cfg
    got = gt_plain(run.eng.factors.Gt, cfg.num_q_heads, cfg.rank_v, cfg.hidden)   # [hidden, Hq, r]
    assert_stored_equal(got, run.oc.G.transpose(2, 0, 1), storage_of(run.wl), "Gt")


def test_out_proj_on_oracle_latents(run):
    eng, wl = run.eng, run.wl
    o = torch.from_numpy(np.stack([out["o_lat"] for _, out in run.ref])).float().cuda().contiguous()
    y = torch.empty_like(eng.y)
    bk.out_proj(eng.cfg, eng.factors, o, y, eng.ws)
    want = np.stack([O_y(run.oc.G, to64(o)[b]) for b in range(wl.batch)])
    assert_close(y.cpu().numpy(), want, storage_of(wl), "y (oracle latents)")


def O_y(G, o_lat):
    from oracle import basiskv_oracle as O
    return O.out_projection(o_lat, G)


def test_end_to_end(run):
    """Every sequence and head: the selection under the near-tie rule, then o_lat and y
    against the oracle's attention and out-projection over the GPU's own selection (the
    oracle's results themselves wherever the two selections are identical)."""
    eng, wl = run.eng, run.wl
    sel, cnt, o_lat, y = (t.cpu().numpy() for t in run.outputs)
    for b, (cache, out) in enumerate(run.ref):
        for h in range(wl.num_q_heads):
            assert selection_ok(sel[b, h], cnt[b, h], out["sel"][h], out["scores"][h])[0], f"b={b} h={h}"
        o_want, y_want = oracle_on_selection(run.oc, b, cache, out, sel[b], cnt[b])
        assert_close(o_lat[b], o_want, storage_of(wl), f"o_lat b={b}")
        assert_close(y[b], y_want, storage_of(wl), f"y b={b}")


def test_step_repeats(run):
    """A second step on the same inputs gives bitwise identical selections and outputs (the
    split of the attention work depends only on the union sizes)."""
    eng = run.eng
    s0, c0, o0, y0 = run.outputs
    eng.step()
    torch.cuda.synchronize()
    assert torch.equal(eng.sel, s0) and torch.equal(eng.sel_cnt, c0)
    assert torch.equal(eng.o_lat, o0) and torch.equal(eng.y, y0)
