"""Per-KV-group routing (basiskv_route_group) against the oracle.

One selection per (sequence, KV group) from the sum or the maximum of the
group's query-head scores, copied to every head of the group.  End to end on
small workloads (the attention then reads k + 2 pages per group), and exactly
on crafted integer scores, including block tables wide enough for the other
selection kernels.
"""
import numpy as np
import pytest
import torch

from oracle import basiskv_oracle as O
from tests.harness import OracleCase, assert_close, selection_ok, storage_of

pytestmark = pytest.mark.gpu

from long_context_decode_basiskv_b200 import binding as bk  # noqa: E402
from long_context_decode_basiskv_b200.engine import DecodeEngine  # noqa: E402
from long_context_decode_basiskv_b200.workloads import WORKLOADS, make_case, shrink  # noqa: E402

SMALL = {
    "tiny_fp32": WORKLOADS["tiny_fp32"],
    "l8b_small": shrink(WORKLOADS["llama3_8b_32k"], batch=3, context=8001, name="l8b_small"),
    "l70b_small": shrink(WORKLOADS["llama3_70b_64k"], batch=2, context=9000, name="l70b_small"),
    "ragged_small": shrink(WORKLOADS["ragged_serving"], batch=6, ragged=(100, 3000), top_k=32,
                           name="ragged_small"),
}
ROUTINGS = ["group_sum", "group_max"]


class GroupRun:
    def __init__(self, wl, routing):
        self.wl, self.routing = wl, routing
        self.case = make_case(wl, "cuda")
        self.eng = DecodeEngine(self.case, routing=routing)
        self.scores = torch.full((wl.batch, wl.num_kv_heads, self.eng.cache.max_pages), float("nan"),
                                 device="cuda")
        self.eng.append()
        self.eng.route(scores=self.scores)
        self.eng.decode_attn()
        self.eng.out_proj()
        torch.cuda.synchronize()
        oc = OracleCase(self.case)
        self.ref = [oc.sequence(b, routing) for b in range(wl.batch)]


@pytest.fixture(scope="module", params=[(w, r) for w in sorted(SMALL) for r in ROUTINGS],
                ids=lambda p: f"{p[0]}-{p[1]}")
def run(request):
    w, r = request.param
    gr = GroupRun(SMALL[w], r)
    yield gr
    del gr
    torch.cuda.empty_cache()


def test_group_selection_and_scores(run):
    eng, wl = run.eng, run.wl
    G = wl.num_q_heads // wl.num_kv_heads
    sel = eng.sel.cpu().numpy()
    cnt = eng.sel_cnt.cpu().numpy()
    scores = run.scores.cpu().numpy()
    assert int(eng.err.item()) == 0
    for b, (_, out) in enumerate(run.ref):
        n = -(-run.case.lengths[b] // wl.page_size)
        for g in range(wl.num_kv_heads):
            ref = out["scores"][g]
            tol = 1e-5 * np.max(np.abs(ref))
            assert np.max(np.abs(scores[b, g, :n] - ref)) <= tol
            for h in range(g * G, (g + 1) * G):
                np.testing.assert_array_equal(sel[b, h], sel[b, g * G])  # one selection per group
                assert cnt[b, h] == cnt[b, g * G]
                ok, _ = selection_ok(sel[b, h], cnt[b, h], out["sel"][h], ref)
                assert ok, f"b={b} h={h}: gpu {sel[b, h][:cnt[b, h]]} oracle {out['sel'][h]}"
            assert cnt[b, g * G] == min(n, wl.top_k + 2)


def test_group_end_to_end(run):
    st = storage_of(run.wl)
    want_o = np.stack([out["o_lat"] for _, out in run.ref])
    want_y = np.stack([out["y"] for _, out in run.ref])
    assert_close(run.eng.o_lat.cpu().numpy().astype(np.float64), want_o, st, "o_lat (group routing)")
    assert_close(run.eng.y.cpu().numpy().astype(np.float64), want_y, st, "y (group routing)")


@pytest.fixture(scope="module", params=["llama3_8b_32k", "llama3_70b_64k"])
def int_eng(request):
    """Query head h of a group is the unit vector e_(h mod G); summaries hold
    small integers in dimensions 0..G-1, so group sums and maxima are exact."""
    wl = shrink(WORKLOADS[request.param], batch=2, context=16 * 700 + 5, top_k=32, name="group_cases")
    e = DecodeEngine(make_case(wl, "cuda"))
    G = wl.num_q_heads // wl.num_kv_heads
    e.q.zero_()
    for h in range(wl.num_q_heads):
        e.q[:, h, h % G] = 1.0
    return e


def _plant_integer_summaries(eng, rng, kind):
    cfg, cache = eng.cfg, eng.cache
    G = cfg.num_q_heads // cfg.num_kv_heads
    per_seq = []
    for b in range(cache.batch):
        n = -(-eng.case.lengths[b] // cfg.page_size)
        phys = cache.block_table[b, :n].long()
        Sg = []
        for g in range(cfg.num_kv_heads):
            S = np.zeros((n, cfg.head_dim), dtype=np.float32)
            if kind == "ties":
                S[:, :G] = rng.integers(0, 3, size=(n, G))
            else:
                S[:, :G] = rng.integers(-60, 60, size=(n, G))
            cache.summary[phys, g] = torch.from_numpy(S).cuda()
            Sg.append(S.astype(np.float64))
        per_seq.append(Sg)
    return per_seq


@pytest.mark.parametrize("reduce", ["sum", "max"])
@pytest.mark.parametrize("kind", ["spread", "ties"])
@pytest.mark.parametrize("width", [None, 6000, 8192 + 40])
def test_group_selection_exact(int_eng, reduce, kind, width):
    eng = int_eng
    cfg, cache = eng.cfg, eng.cache
    G = cfg.num_q_heads // cfg.num_kv_heads
    rng = np.random.default_rng(2 * ["sum", "max"].index(reduce) + ["spread", "ties"].index(kind))
    per_seq = _plant_integer_summaries(eng, rng, kind)
    qs = np.eye(cfg.head_dim)[:G]
    route_cache, ws = cache, eng.ws
    if width is not None:
        route_cache = bk.PagedCache.__new__(bk.PagedCache)
        route_cache.__dict__.update(cache.__dict__)
        bt = torch.full((cache.batch, width), -1, dtype=torch.int32, device="cuda")
        bt[:, :cache.max_pages] = cache.block_table
        route_cache.block_table = bt
        ws = bk.alloc_workspace(cfg, cache.batch, width, device="cuda")
    eng.err.zero_()
    eng.sel.fill_(-7)
    red = bk.GROUP_SUM if reduce == "sum" else bk.GROUP_MAX
    bk.route_group(cfg, route_cache, eng.q, red, eng.sel, eng.sel_cnt, ws, eng.err)
    torch.cuda.synchronize()
    assert int(eng.err.item()) == 0
    sel = eng.sel.cpu().numpy()
    cnt = eng.sel_cnt.cpu().numpy()
    for b in range(cache.batch):
        for g in range(cfg.num_kv_heads):
            want, _ = O.route_pages_group(qs, per_seq[b][g], cfg.top_k, reduce)
            for h in range(g * G, (g + 1) * G):
                np.testing.assert_array_equal(sel[b, h, :cnt[b, h]], want, err_msg=f"b={b} h={h}")
                assert np.all(sel[b, h, cnt[b, h]:] == -1)
