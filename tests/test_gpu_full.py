"""The five decode workloads at full size, through the same engine and launch
configuration the benchmark times.  Sampled sequences are checked against the
oracle (every query head of them); every head of every sequence is checked
for the selection invariants (count, order, sink and recent pages)."""
import numpy as np
import pytest
import torch

from tests.harness import OracleCase, assert_close, oracle_on_selection, selection_ok, storage_of

pytestmark = pytest.mark.gpu

from long_context_decode_basiskv_b200.engine import DecodeEngine  # noqa: E402
from long_context_decode_basiskv_b200.workloads import WORKLOADS, make_case  # noqa: E402

SAMPLES = {
    "tiny_fp32": [0],
    "llama3_8b_32k": [0, 5],
    "single_seq_131k": [0],
    "llama3_70b_64k": [2],
    "ragged_serving": [3, 40],
}


@pytest.mark.parametrize("name", list(SAMPLES))
def test_full_workload(name):
    wl = WORKLOADS[name]
    case = make_case(wl, "cuda")
    eng = DecodeEngine(case)
    eng.step()
    torch.cuda.synchronize()
    assert int(eng.err.item()) == 0
    sel = eng.sel.cpu().numpy()
    cnt = eng.sel_cnt.cpu().numpy()
    for b, L in enumerate(case.lengths):
        n = -(-L // wl.page_size)
        want = min(n, wl.top_k + 2)
        assert np.all(cnt[b] == want)
        for h in range(wl.num_q_heads):
            s = sel[b, h, :want]
            assert s[0] == 0 and s[-1] == n - 1 and np.all(np.diff(s) > 0)
            assert np.all(sel[b, h, want:] == -1)
    o_lat = eng.o_lat.cpu().numpy()
    y = eng.y.cpu().numpy()
    oc = OracleCase(case)
    storage = storage_of(wl)
    for b in SAMPLES[name]:
        cache, out = oc.sequence(b)
        for h in range(wl.num_q_heads):
            assert selection_ok(sel[b, h], cnt[b, h], out["sel"][h], out["scores"][h])[0], f"{name} b={b} h={h}"
        # every head and y, against the oracle over the GPU's own selection (a near-tie swap
        # is a correct selection; where there is none these are the oracle's own outputs)
        o_want, y_want = oracle_on_selection(oc, b, cache, out, sel[b], cnt[b])
        assert_close(o_lat[b], o_want, storage, f"{name} o_lat b={b}")
        assert_close(y[b], y_want, storage, f"{name} y b={b}")
    if case.hot_pages is not None:
        print(f"{name}: hot pages {len(case.hot_pages)}, alpha {case.hot_alpha:.3f}, dense mass {case.hot_mass:.3f}")
    del eng, case
    torch.cuda.empty_cache()
