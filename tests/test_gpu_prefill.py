"""basiskv_prefill (the tensor-core append for long appends) against the oracle.

Stored values: raw keys exact; C and R differ from the oracle's correctly
rounded fp64 values on a small fraction of them, each by at most one bf16 ulp
plus 2^-14 of the largest value of its row (the products accumulate in fp32
and the chained intermediate travels as a bf16 hi + lo pair, ~2^-16 relative
to the terms, so a result can land on the other side of a bf16 rounding
midpoint, or, where the terms cancel, a few ulps of a small value away); the page
summaries, recomputed in fp64 from the stored C and R, within 1e-3 relative
L2 per page (one flipped C value of a page moves its mean by at most
2^-8 / page size of that component).  Then a decode step on the prefilled
cache matches the oracle run on that same stored cache at the usual
tolerances.
"""
import numpy as np
import pytest
import torch

from oracle import basiskv_oracle as O
from tests.harness import OracleCase, assert_close, selection_ok, storage_of, to64, ulp

pytestmark = pytest.mark.gpu

from long_context_decode_basiskv_b200 import binding as bk  # noqa: E402
from long_context_decode_basiskv_b200.engine import DecodeEngine  # noqa: E402
from long_context_decode_basiskv_b200.workloads import WORKLOADS, make_case, shrink  # noqa: E402

C_FRAC = 4e-3    # fraction of stored C values allowed one bf16 ulp off
R_FRAC = 2e-2    # R: the residual k - C P cancels, which scales its relative error up
S_REL = 1e-3

SMALL = {
    "l8b_small": shrink(WORKLOADS["llama3_8b_32k"], batch=3, context=8001, name="l8b_small"),
    "hot_small": shrink(WORKLOADS["single_seq_131k"], context=64 * 300 + 17, name="hot_small"),
    "l70b_small": shrink(WORKLOADS["llama3_70b_64k"], batch=2, context=9000, name="l70b_small"),
    "ragged_small": shrink(WORKLOADS["ragged_serving"], batch=6, ragged=(100, 3000), top_k=32,
                           name="ragged_small"),
}


def _ulp_check(got, want, storage, frac, what):
    """Every value within one ulp of its own, plus 2^-14 of its row's largest
    magnitude (fp32 accumulation error is relative to the terms summed, not to
    a small result of cancelling terms); at most `frac` of the values differ."""
    diff = np.abs(got - want)
    tol = ulp(want, storage) + 2.0 ** -14 * np.max(np.abs(want), axis=-1, keepdims=True)
    assert np.all(diff <= tol * 1.0000001), f"{what}: {np.max(diff / tol):.2f} x tolerance"
    f = (diff > 0).mean()
    assert f <= frac, f"{what}: {f:.2e} of values differ (allowed {frac:.0e})"
    return f


class PrefillRun:
    def __init__(self, wl):
        self.wl = wl
        self.case = make_case(wl, "cuda")
        self.eng = DecodeEngine(self.case, prefill_mode="tc")
        torch.cuda.synchronize()
        self.oc = OracleCase(self.case)
        self.fracs = {}


@pytest.fixture(scope="module", params=sorted(SMALL))
def run(request):
    pr = PrefillRun(SMALL[request.param])
    yield pr
    del pr
    torch.cuda.empty_cache()


def test_prefill_cache_matches_oracle(run):
    eng, wl, oc = run.eng, run.wl, run.oc
    assert int(eng.err.item()) == 0
    st = storage_of(wl)
    for b in range(wl.batch):
        L = run.case.lengths[b]
        K = to64(run.case.keys[b])
        V = to64(run.case.values[b])
        ref = O.prefill(K[:-1], V[:-1], oc.A, oc.P, oc.E, wl.page_size, oc.storage, capacity=L)
        Lp = L - 1
        n = -(-Lp // wl.page_size)
        C = to64(eng.logical(eng.cache.c_lat, b))[:, :Lp]
        R = to64(eng.logical(eng.cache.r_res, b))[:, :Lp]
        Kc = to64(eng.logical(eng.cache.k_raw, b))[:, :Lp]
        np.testing.assert_array_equal(Kc, K[:-1].transpose(1, 0, 2))
        run.fracs[f"C{b}"] = _ulp_check(C, ref.C[:, :Lp], st, C_FRAC, f"C b={b}")
        run.fracs[f"R{b}"] = _ulp_check(R, ref.R[:, :Lp], st, R_FRAC, f"R b={b}")
        phys = eng.cache.block_table[b, :n].long()
        S = to64(eng.cache.summary[phys]).transpose(1, 0, 2)   # [Hkv, n, d]
        err = np.linalg.norm(S - ref.S[:, :n], axis=-1) / np.maximum(np.linalg.norm(ref.S[:, :n], axis=-1), 1e-30)
        assert err.max() <= S_REL, f"summary b={b}: {err.max():.2e}"
        # the summaries are exactly the fp64 page means of the stored C and R
        Sx = np.stack([O.page_summaries(C[g], R[g], oc.P[g], oc.E[g], wl.page_size, storage="f32")
                       for g in range(wl.num_kv_heads)])
        np.testing.assert_allclose(S, Sx, rtol=2e-7, atol=1e-30)


def test_decode_step_on_prefilled_cache(run):
    """The decode step on the tensor-core-prefilled cache, against the oracle run
    on that same stored cache (its K, C, R and summaries)."""
    eng, wl, oc = run.eng, run.wl, run.oc
    eng.step()
    torch.cuda.synchronize()
    assert int(eng.err.item()) == 0
    sel = eng.sel.cpu().numpy()
    cnt = eng.sel_cnt.cpu().numpy()
    st = storage_of(wl)
    o_want, y_want = [], []
    for b in range(wl.batch):
        L = run.case.lengths[b]
        Lp = L - 1
        n = -(-Lp // wl.page_size)
        cache = O.SequenceCache(wl.num_kv_heads, wl.head_dim, wl.rank_v, wl.rank_k, wl.page_size, L, oc.storage)
        cache.K[:, :Lp] = to64(run.case.keys[b])[:-1].transpose(1, 0, 2)
        full_C = to64(eng.logical(eng.cache.c_lat, b))
        full_R = to64(eng.logical(eng.cache.r_res, b))
        cache.C[:, :Lp] = full_C[:, :Lp]
        cache.R[:, :Lp] = full_R[:, :Lp]
        phys = eng.cache.block_table[b, :n].long()
        # the step's append rewrote only the tail page's summary, which the oracle's step recomputes too
        cache.S[:, :n] = to64(eng.cache.summary[phys]).transpose(1, 0, 2)
        cache.length = Lp
        out = O.decode_step(cache, to64(run.case.keys[b])[-1], to64(run.case.values[b])[-1],
                            to64(run.case.q[b]), oc.A, oc.P, oc.E, oc.G, wl.top_k)
        for h in range(wl.num_q_heads):
            ok, _ = selection_ok(sel[b, h], cnt[b, h], out["sel"][h], out["scores"][h])
            assert ok, f"b={b} h={h}"
        o_want.append(out["o_lat"])
        y_want.append(out["y"])
    assert_close(eng.o_lat.cpu().numpy().astype(np.float64), np.stack(o_want), st, "o_lat after tc prefill")
    assert_close(eng.y.cpu().numpy().astype(np.float64), np.stack(y_want), st, "y after tc prefill")


@pytest.mark.parametrize("first,n_new", [(37, 500), (40, 1), (16, 127), (5, 129), (0, 3000)])
def test_prefill_after_earlier_tokens(first, n_new):
    """Appends that start inside a page, span a partial tile, or follow an exact append:
    tokens [0, first) by basiskv_append, then [first, first + n_new) by basiskv_prefill,
    into a cache zeroed beforehand."""
    wl = shrink(WORKLOADS["llama3_8b_32k"], batch=2, context=first + n_new, name="pf_unaligned")
    case = make_case(wl, "cuda")
    eng = DecodeEngine(case)
    cfg, dev = eng.cfg, "cuda"
    oc = OracleCase(case)
    for t in (eng.cache.k_raw, eng.cache.c_lat, eng.cache.r_res, eng.cache.summary):
        t.zero_()
    for b in range(wl.batch):
        sub = bk.PagedCache.__new__(bk.PagedCache)
        sub.__dict__.update(eng.cache.__dict__)
        sub.block_table = eng.cache.block_table[b:b + 1]
        if first:
            sub.seq_len = torch.tensor([first], dtype=torch.int32, device=dev)
            bk.append(cfg, sub, eng.factors, case.keys[b][:first].unsqueeze(0).contiguous(),
                      case.values[b][:first].unsqueeze(0).contiguous(), eng.err)
        sub.seq_len = torch.tensor([first + n_new], dtype=torch.int32, device=dev)
        bk.prefill(cfg, sub, eng.factors, case.keys[b][first:].unsqueeze(0).contiguous(),
                   case.values[b][first:].unsqueeze(0).contiguous(), eng.err)
    torch.cuda.synchronize()
    assert int(eng.err.item()) == 0
    L = first + n_new
    n = -(-L // wl.page_size)
    for b in range(wl.batch):
        K, V = to64(case.keys[b]), to64(case.values[b])
        ref = O.prefill(K, V, oc.A, oc.P, oc.E, wl.page_size, oc.storage, capacity=L)
        C = to64(eng.logical(eng.cache.c_lat, b))
        R = to64(eng.logical(eng.cache.r_res, b))
        if first:  # the exact append's tokens, untouched by the prefill
            _ulp_check(C[:, :first], ref.C[:, :first], "bf16", max(1e-4, 2.0 / C[:, :first].size), "C exact")
        _ulp_check(C, ref.C[:, :L], "bf16", max(C_FRAC, 2.0 / C.size), "C")
        _ulp_check(R, ref.R[:, :L], "bf16", max(R_FRAC, 2.0 / R.size), "R")
        np.testing.assert_array_equal(to64(eng.logical(eng.cache.k_raw, b)), K.transpose(1, 0, 2))
        phys = eng.cache.block_table[b, :n].long()
        S = to64(eng.cache.summary[phys]).transpose(1, 0, 2)
        Sx = np.stack([O.page_summaries(C[g], R[g], oc.P[g], oc.E[g], wl.page_size, storage="f32")
                       for g in range(wl.num_kv_heads)])
        np.testing.assert_allclose(S, Sx, rtol=2e-7, atol=1e-30)


def test_prefill_rejects_unsupported_shapes():
    wl = WORKLOADS["tiny_fp32"]
    case = make_case(wl, "cuda")
    eng = DecodeEngine(case)
    k = case.keys[0][:10].unsqueeze(0).contiguous()
    with pytest.raises(bk.BasisKVError) as e:
        bk.prefill(eng.cfg, eng.cache, eng.factors, k, k.clone(), eng.err)
    assert e.value.status == bk.ERR_UNSUPPORTED
