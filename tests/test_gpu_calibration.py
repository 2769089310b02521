"""Joint cross-partition factor fitting (offline calibration) on the GPU.

calibrate.fit_value_factors runs on whatever device its tensors are on; here
it runs on cuda:0 in fp64 and must reproduce the oracle's fit (least squares
on the written-out design matrices, numpy on the host).  Then a decode step of
the CUDA path on a case whose Value factors were fitted that way (and whose
key factors were refitted to them) must match the oracle's decode step on the
same factors."""
import numpy as np
import pytest
import torch

from oracle import basiskv_oracle as O
from tests.harness import OracleCase, assert_close, oracle_on_selection, selection_ok, storage_of

pytestmark = pytest.mark.gpu

from long_context_decode_basiskv_b200 import calibrate as CAL  # noqa: E402
from long_context_decode_basiskv_b200.engine import DecodeEngine  # noqa: E402
from long_context_decode_basiskv_b200.workloads import WORKLOADS, make_case, shrink  # noqa: E402


@pytest.mark.parametrize("Hq,Hkv,parts,objective", [
    (8, 2, [[0], [1]], "joint"), (8, 2, [[0], [1]], "isolated"), (6, 3, [[0, 1], [2]], "joint"),
])
def test_fit_on_the_gpu_matches_the_oracle(Hq, Hkv, parts, objective):
    rng = np.random.default_rng(Hq * 7 + Hkv)
    N, d, r, hid = 64, 8, 3, 12
    shared = rng.standard_normal((N, d))
    Z = np.stack([0.7 * shared + rng.standard_normal((N, d)) * rng.uniform(0.3, 2.0, size=d) for _ in range(Hq)])
    W_O = rng.standard_normal((Hq * d, hid)) / np.sqrt(d)
    A0, B0, h0 = O.fit_value_factors(Z, W_O, Hkv, parts, r, 3, objective)
    Zc, Wc = torch.from_numpy(Z).cuda(), torch.from_numpy(W_O).cuda()
    A1, B1, h1 = CAL.fit_value_factors(Zc, Wc, Hkv, parts, r, 3, objective)
    assert A1.is_cuda and B1.is_cuda
    np.testing.assert_allclose(np.array(h1), h0, rtol=1e-9)
    for g in range(Hkv):
        P0 = A0[g] @ B0[g]
        P1 = (A1[g] @ B1[g]).cpu().numpy()
        np.testing.assert_allclose(P1, P0, atol=1e-8 * np.abs(P0).max())


@pytest.mark.parametrize("base", ["tiny_fp32", "l8b"])
def test_decode_step_with_calibrated_factors(base):
    wl = WORKLOADS["tiny_fp32"] if base == "tiny_fp32" else \
        shrink(WORKLOADS["llama3_8b_32k"], batch=2, context=16 * 300 + 5, top_k=32, name="cal_gpu")
    case = make_case(wl, "cuda")
    # calibration queries and the exact attention outputs of sequence 0, fit on the GPU
    g = torch.Generator(device="cuda").manual_seed(11)
    q = torch.randn((256, wl.num_q_heads, wl.head_dim), generator=g, device="cuda", dtype=torch.float64)
    K = case.keys[0].to(torch.float64)
    V = case.values[0].to(torch.float64)
    Z = CAL.calibration_outputs(q, K, V)
    parts = [[i] for i in range(wl.num_kv_heads)]
    A, B, hist = CAL.fit_value_factors(Z, case.W_O.to(torch.float64), wl.num_kv_heads, parts, wl.rank_v, 2, "joint")
    assert hist[-1] <= hist[0]
    cal = CAL.with_value_factors(case, A, B)
    eng = DecodeEngine(cal)
    eng.step()
    torch.cuda.synchronize()
    assert int(eng.err.item()) == 0
    oc = OracleCase(cal)
    sel, cnt = eng.sel.cpu().numpy(), eng.sel_cnt.cpu().numpy()
    for b in range(wl.batch):
        cache, out = oc.sequence(b)
        for h in range(wl.num_q_heads):
            assert selection_ok(sel[b, h], cnt[b, h], out["sel"][h], out["scores"][h])[0], f"b={b} h={h}"
        o_want, y_want = oracle_on_selection(oc, b, cache, out, sel[b], cnt[b])
        assert_close(eng.o_lat[b].cpu().numpy(), o_want, storage_of(wl), f"calibrated o_lat b={b}")
        assert_close(eng.y[b].cpu().numpy(), y_want, storage_of(wl), f"calibrated y b={b}")
