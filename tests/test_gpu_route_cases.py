"""Page selection on crafted score distributions (GPU vs oracle, exact).

The query is one-hot and each page summary carries an integer in dimension
0, so every routing score is an exact integer on both sides and the selection
must match the oracle's total order (score descending, page ascending)
exactly: all scores equal, more pages tied at the top than k, one huge
outlier (the rest crowd into one histogram bucket), heavy duplication, mixed
signs."""
import numpy as np
import pytest
import torch

from oracle import basiskv_oracle as O

pytestmark = pytest.mark.gpu

from long_context_decode_basiskv_b200 import binding as bk  # noqa: E402
from long_context_decode_basiskv_b200.engine import DecodeEngine  # noqa: E402
from long_context_decode_basiskv_b200.workloads import WORKLOADS, make_case, shrink  # noqa: E402


@pytest.fixture(scope="module")
def eng():
    wl = shrink(WORKLOADS["llama3_8b_32k"], batch=2, context=16 * 700 + 5, top_k=32, name="route_cases")
    e = DecodeEngine(make_case(wl, "cuda"))
    e.q.zero_()
    e.q[..., 0] = 1.0
    return e


def _values(kind, n, rng):
    if kind == "all_equal":
        return np.full(n, 5.0)
    if kind == "top_ties":
        v = np.ones(n)
        v[rng.choice(np.arange(1, n - 1), size=80, replace=False)] = 7.0
        return v
    if kind == "outlier":
        v = rng.integers(0, 100, size=n).astype(np.float64)
        v[n // 3] = 1e30
        return v
    if kind == "duplicates":
        return rng.integers(0, 10, size=n).astype(np.float64)
    if kind == "mixed_sign":
        return rng.integers(-1000, 1000, size=n).astype(np.float64)
    if kind == "tiny_spread":
        return 1.0 + rng.integers(0, 3, size=n) * 2.0 ** -20
    raise ValueError(kind)


@pytest.mark.parametrize("kind", ["all_equal", "top_ties", "outlier", "duplicates", "mixed_sign", "tiny_spread"])
def test_selection_on_crafted_scores(eng, kind):
    rng = np.random.default_rng(abs(hash(kind)) % 2**32)
    cfg, cache = eng.cfg, eng.cache
    B = cache.batch
    wants = []
    for b in range(B):
        n = -(-eng.case.lengths[b] // cfg.page_size)
        vals = _values(kind, n, rng).astype(np.float32)
        S = np.zeros((n, cfg.head_dim), dtype=np.float32)
        S[:, 0] = vals
        phys = cache.block_table[b, :n].long()
        for g in range(cfg.num_kv_heads):
            cache.summary[phys, g] = torch.from_numpy(S).cuda()
        sel, scores = O.route_pages(np.eye(cfg.head_dim)[0], S.astype(np.float64), cfg.top_k)
        wants.append(sel)
    eng.err.zero_()
    bk.route(cfg, cache, eng.q, eng.sel, eng.sel_cnt, eng.ws, eng.err)
    torch.cuda.synchronize()
    assert int(eng.err.item()) == 0
    sel = eng.sel.cpu().numpy()
    cnt = eng.sel_cnt.cpu().numpy()
    for b in range(B):
        for h in range(cfg.num_q_heads):
            got = sel[b, h, :cnt[b, h]]
            np.testing.assert_array_equal(got, wants[b], err_msg=f"{kind} b={b} h={h}")
            assert np.all(sel[b, h, cnt[b, h]:] == -1)


@pytest.mark.parametrize("width", [6000, 8192 + 40])
def test_wide_block_tables(eng, width):
    """Wider block tables select with other kernel instances (32 register keys
    per thread up to 8192 pages, the shared-memory histogram kernel beyond);
    they must select exactly the pages of the narrow table."""
    rng = np.random.default_rng(7)
    cfg, cache = eng.cfg, eng.cache
    B = cache.batch
    for b in range(B):
        n = -(-eng.case.lengths[b] // cfg.page_size)
        S = np.zeros((n, cfg.head_dim), dtype=np.float32)
        S[:, 0] = rng.integers(-50, 50, size=n)
        phys = cache.block_table[b, :n].long()
        for g in range(cfg.num_kv_heads):
            cache.summary[phys, g] = torch.from_numpy(S).cuda()
    eng.err.zero_()
    bk.route(cfg, cache, eng.q, eng.sel, eng.sel_cnt, eng.ws, eng.err)
    torch.cuda.synchronize()
    ref_sel, ref_cnt = eng.sel.clone(), eng.sel_cnt.clone()

    wide = bk.PagedCache.__new__(bk.PagedCache)
    wide.__dict__.update(cache.__dict__)
    bt = torch.full((B, width), -1, dtype=torch.int32, device="cuda")
    bt[:, :cache.max_pages] = cache.block_table
    wide.block_table = bt
    ws = bk.alloc_workspace(cfg, B, width, device="cuda")
    eng.sel.fill_(-7)
    bk.route(cfg, wide, eng.q, eng.sel, eng.sel_cnt, ws, eng.err)
    torch.cuda.synchronize()
    assert int(eng.err.item()) == 0
    assert torch.equal(eng.sel, ref_sel)
    assert torch.equal(eng.sel_cnt, ref_cnt)
