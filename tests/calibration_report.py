"""Quality of the Value factors: fitted in isolation per partition or jointly
against the complete attention output (reported, not gated; CPU, fp64).

Synthetic layer (seeded): per KV group g, values V_g = Z_g U_g^T + 0.05 N
(rank `data_rank`), keys K_g = V_g M_g + 0.3 N, as in the decode workloads;
the latent Z_g is either drawn per group ("independent") or mixes a component
shared by all groups ("shared", weight rho), which correlates the partitions.
Calibration and held-out queries are N(0, q_scale^2); the attention outputs
and the fits use calibrate.py (the oracle's fit is pinned against it on small
cases).  For each tensor-parallel split the held-out relative error of the
complete output sum_h Z_h A_g B_g W_O,h is reported for: PCA of the values
(the factors the decode workloads use), the per-group SVD of the attention
outputs (the fits' start), the isolated fit and the joint fit.

    python -m tests.calibration_report [--out FILE]
"""
from __future__ import annotations

import argparse
import json
import math

import torch

from long_context_decode_basiskv_b200 import calibrate as CAL


def synthetic_layer(seed, Hq=32, Hkv=8, d=64, data_rank=16, T=2048, hidden=1024, shared=0.0):
    g = torch.Generator().manual_seed(seed)
    f64 = torch.float64
    U = torch.linalg.qr(torch.randn((Hkv, d, data_rank), generator=g, dtype=f64)).Q
    M = torch.randn((Hkv, d, d), generator=g, dtype=f64) / math.sqrt(d)
    common = torch.randn((T, 1, data_rank), generator=g, dtype=f64)
    own = torch.randn((T, Hkv, data_rank), generator=g, dtype=f64)
    Z = math.sqrt(shared) * common + math.sqrt(1.0 - shared) * own
    V = torch.einsum("thr,hdr->thd", Z, U) + 0.05 * torch.randn((T, Hkv, d), generator=g, dtype=f64)
    K = torch.einsum("thd,hde->the", V, M) + 0.3 * torch.randn((T, Hkv, d), generator=g, dtype=f64)
    W_O = torch.randn((Hq * d, hidden), generator=g, dtype=f64) / math.sqrt(hidden)
    return K, V, W_O, g


def relative_error(Z, W_O, A, B):
    Hq, N, d = Z.shape
    y = sum(Z[h] @ W_O[h * d:(h + 1) * d] for h in range(Hq))
    return math.sqrt(CAL.output_error(Z, W_O, A, B) / float((y * y).sum()))


def measure(shared, rank=8, n_calib=4096, n_test=1024, q_scale=2.0, sweeps=5, splits=(2, 4, 8), seed=7, **kw):
    K, V, W_O, g = synthetic_layer(seed, shared=shared, **kw)
    T, Hkv, d = V.shape
    Hq = W_O.shape[0] // d
    q_cal = q_scale * torch.randn((n_calib, Hq, d), generator=g, dtype=torch.float64)
    q_test = q_scale * torch.randn((n_test, Hq, d), generator=g, dtype=torch.float64)
    Z_cal = CAL.calibration_outputs(q_cal, K, V)
    Z_test = CAL.calibration_outputs(q_test, K, V)
    # PCA of the values (uncentred): the factors the decode workloads are built with
    A_pca = torch.stack([torch.linalg.svd(V[:, h], full_matrices=False).Vh[:rank].T for h in range(Hkv)])
    res = {"pca_of_values": relative_error(Z_test, W_O, A_pca, A_pca.transpose(1, 2))}
    for n in splits:
        per = Hkv // n
        parts = [list(range(i * per, (i + 1) * per)) for i in range(n)]
        row = {}
        for objective in ("isolated", "joint"):
            A, B, _ = CAL.fit_value_factors(Z_cal, W_O, Hkv, parts, rank, sweeps, objective)
            row[objective] = relative_error(Z_test, W_O, A, B)
        A0, B0, _ = CAL.fit_value_factors(Z_cal, W_O, Hkv, parts, rank, 0, "joint")
        row["svd_of_outputs"] = relative_error(Z_test, W_O, A0, B0)
        res[f"tp{n}"] = {k: round(v, 5) for k, v in row.items()}
    res["pca_of_values"] = round(res["pca_of_values"], 5)
    return res


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--out", default=None)
    args = ap.parse_args()
    report = {}
    for name, shared in [("independent", 0.0), ("shared_0.5", 0.5)]:
        report[name] = measure(shared)
        print(name, json.dumps(report[name]), flush=True)
    if args.out:
        with open(args.out, "w") as f:
            json.dump(report, f, indent=1)


if __name__ == "__main__":
    main()
