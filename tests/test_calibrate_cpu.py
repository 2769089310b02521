"""Calibration (calibrate.py) against the oracle on CPU: the same factors, errors
and sweeps from an independent implementation (normal equations with Kronecker
blocks in torch vs least squares on the written-out design matrix in numpy),
and the calibration attention outputs against the oracle's attention."""
import numpy as np
import pytest
import torch

from oracle import basiskv_oracle as O
from long_context_decode_basiskv_b200 import calibrate as CAL


def _case(seed, Hq, Hkv, N, d, hid):
    rng = np.random.default_rng(seed)
    shared = rng.standard_normal((N, d))  # a component common to every head (correlated partitions)
    Z = np.stack([0.7 * shared + rng.standard_normal((N, d)) * rng.uniform(0.3, 2.0, size=d)
                  for _ in range(Hq)])
    W_O = rng.standard_normal((Hq * d, hid)) / np.sqrt(d)
    return Z, W_O


@pytest.mark.parametrize("Hq,Hkv,parts,objective", [
    (4, 2, [[0], [1]], "joint"), (4, 2, [[0], [1]], "isolated"),
    (8, 2, [[0], [1]], "joint"), (6, 3, [[0, 1], [2]], "isolated"), (6, 3, [[0, 1], [2]], "joint"),
])
def test_fit_matches_oracle(Hq, Hkv, parts, objective):
    N, d, r, hid = 48, 6, 2, 9
    Z, W_O = _case(Hq * 10 + Hkv, Hq, Hkv, N, d, hid)
    A0, B0, h0 = O.fit_value_factors(Z, W_O, Hkv, parts, r, 3, objective)
    A1, B1, h1 = CAL.fit_value_factors(torch.from_numpy(Z), torch.from_numpy(W_O), Hkv, parts, r, 3, objective)
    np.testing.assert_allclose(np.array(h1), h0, rtol=1e-9)
    for g in range(Hkv):
        P0 = A0[g] @ B0[g]
        P1 = (A1[g] @ B1[g]).numpy()
        np.testing.assert_allclose(P1, P0, atol=1e-8 * np.abs(P0).max())
    assert abs(CAL.output_error(torch.from_numpy(Z), torch.from_numpy(W_O), A1, B1) - h0[-1]) <= 1e-9 * h0[-1]


def test_fit_rejects_unknown_objective():
    Z, W_O = _case(1, 2, 1, 10, 4, 5)
    with pytest.raises(ValueError):
        CAL.fit_value_factors(torch.from_numpy(Z), torch.from_numpy(W_O), 1, [[0]], 2, 1, "partition")


def test_calibration_outputs_match_oracle_attention():
    rng = np.random.default_rng(3)
    N, Hq, Hkv, T, d = 5, 4, 2, 37, 8
    q = rng.standard_normal((N, Hq, d))
    K = rng.standard_normal((T, Hkv, d))
    V = rng.standard_normal((T, Hkv, d))
    Z = CAL.calibration_outputs(torch.from_numpy(q), torch.from_numpy(K), torch.from_numpy(V)).numpy()
    for h in range(Hq):
        g = h // (Hq // Hkv)
        for n in range(N):
            o, _, _ = O.sparse_attention(q[n, h], K[:, g], V[:, g], np.arange(O.num_pages(T, 4)), 4)
            np.testing.assert_allclose(Z[h, n], o, atol=1e-12)


def test_with_value_factors_refits_the_key_factors_like_the_workloads():
    """Given the workloads' own (unrounded) Value encoders, the refit reproduces their P and E."""
    from long_context_decode_basiskv_b200.workloads import WORKLOADS, _top_eigvecs, gram_matrices, make_case, shrink

    for wl in (WORKLOADS["tiny_fp32"], shrink(WORKLOADS["llama3_8b_32k"], batch=2, context=700, name="cal")):
        case = make_case(wl, "cpu")
        gvv, _, _ = gram_matrices(case.keys, case.values)
        A = torch.stack([_top_eigvecs(gvv[h], wl.rank_v) for h in range(wl.num_kv_heads)])
        out = CAL.with_value_factors(case, A, A.transpose(1, 2))
        for a, b in ((out.A, case.A), (out.Bf, case.Bf), (out.P, case.P), (out.E, case.E)):
            assert a.dtype == b.dtype and torch.equal(a, b)


def test_calibrated_case_runs_through_the_oracle():
    """Joint factors fitted on calibration outputs of a case, then one oracle decode step on it."""
    from long_context_decode_basiskv_b200.workloads import WORKLOADS, make_case

    case = make_case(WORKLOADS["tiny_fp32"], "cpu")
    wl = case.wl
    g = torch.Generator().manual_seed(3)
    q = torch.randn((64, wl.num_q_heads, wl.head_dim), generator=g, dtype=torch.float64) * 2
    K = case.keys[0].to(torch.float64)
    V = case.values[0].to(torch.float64)
    Z = CAL.calibration_outputs(q, K, V)
    W = case.W_O.to(torch.float64)
    A, B, hist = CAL.fit_value_factors(Z, W, wl.num_kv_heads, [[0], [1]], wl.rank_v, 2, "joint")
    assert hist[-1] <= hist[0]
    cal = CAL.with_value_factors(case, A, B)
    f64 = lambda t: t.to(torch.float64).numpy()  # noqa: E731
    G = O.fuse_out_factor(f64(cal.Bf), f64(cal.W_O), wl.num_q_heads, "f32")
    cache = O.prefill(f64(K)[:-1], f64(V)[:-1], f64(cal.A), f64(cal.P), f64(cal.E), wl.page_size, "f32",
                      capacity=K.shape[0])
    out = O.decode_step(cache, f64(K)[-1], f64(V)[-1], f64(case.q[0]), f64(cal.A), f64(cal.P), f64(cal.E), G,
                        wl.top_k)
    assert np.all(np.isfinite(out["y"])) and np.allclose(out["weight_sums"], 1.0)
