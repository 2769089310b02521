"""Offline calibration: Value factors fitted against the complete attention output.

Under tensor parallelism each rank holds the low-rank factors of its own
attention heads.  The BasisKV pages (kongchang.com explainer, section
"联合优化而非逐分区拟合"; BasisKV abstract) fit those factors jointly across
the partitions against the complete attention output instead of letting every
partition fit its own output.  With the Value factor bound to the output
projection, head h of KV group g contributes Z_h A_g B_g W_O,h to the layer
output, Z_h being the head's exact attention outputs (softmax-weighted raw
values) on calibration queries; the target is sum_h Z_h W_O,h.

``fit_value_factors`` starts from a per-group SVD (A_g = top right singular
vectors of the group's Z rows, B_g = A_g^T) and runs sweeps of alternating
least squares: for each group in turn, B_g then A_g solve their linear
least-squares problem against the target, which is

  "joint":    the complete output minus the other groups' current approximations;
  "isolated": the same restricted to the heads of the group's own partition.

Each solve uses the normal equations, whose (r d) x (r d) matrix is a sum of
Kronecker products of the G x G head-pair Gram blocks, so nothing of size
N x hidden x r x d is formed.  Runs on whatever device the tensors are on
(calibration is offline; the matrices are small dense solves).
"""
from __future__ import annotations

import dataclasses

import torch

from .workloads import Case, gram_matrices, key_factors_from_grams


def output_error(Z: torch.Tensor, W_O: torch.Tensor, A: torch.Tensor, B: torch.Tensor) -> float:
    """Squared Frobenius error of sum_h Z_h A_g B_g W_O,h against sum_h Z_h W_O,h."""
    Hq, N, d = Z.shape
    group = Hq // A.shape[0]
    W = W_O.view(Hq, d, -1)
    err = torch.zeros((N, W.shape[2]), dtype=Z.dtype, device=Z.device)
    for h in range(Hq):
        g = h // group
        err += Z[h] @ W[h] - (Z[h] @ A[g]) @ (B[g] @ W[h])
    return float((err * err).sum())


def _solve_two_sided(X, Ys, rhs):
    """Solve sum_{i,j} X[i][j] M Ys[i][j]^T-form normal equations for M.

    X[i][j]: left Gram blocks (p x p); Ys[i][j]: right Gram blocks (q x q), both
    for the term pair (i, j); the system matrix is sum_ij kron(X[i][j], Ys[i][j])
    acting on M flattened row-major (p x q); rhs: p x q."""
    n = len(X)
    p, q = rhs.shape
    N = torch.zeros((p * q, p * q), dtype=rhs.dtype, device=rhs.device)
    for i in range(n):
        for j in range(n):
            N += torch.kron(X[i][j], Ys[i][j])
    return torch.linalg.solve(N, rhs.reshape(-1)).reshape(p, q)


def fit_value_factors(Z: torch.Tensor, W_O: torch.Tensor, num_kv_heads: int, partitions, rank: int,
                      sweeps: int, objective: str):
    """Z [Hq, N, d], W_O [Hq*d, hidden] (same dtype and device); partitions: lists of KV
    groups.  Returns (A [Hkv, d, r], B [Hkv, r, d], complete-output error after the
    start and after every sweep)."""
    if objective not in ("joint", "isolated"):
        raise ValueError(f"objective must be 'joint' or 'isolated', not {objective!r}")
    Hq, N, d = Z.shape
    group = Hq // num_kv_heads
    W = W_O.view(Hq, d, -1)
    A = torch.zeros((num_kv_heads, d, rank), dtype=Z.dtype, device=Z.device)
    B = torch.zeros((num_kv_heads, rank, d), dtype=Z.dtype, device=Z.device)
    for g in range(num_kv_heads):
        rows = Z[g * group:(g + 1) * group].reshape(-1, d)
        Vh = torch.linalg.svd(rows, full_matrices=False).Vh
        A[g] = Vh[:rank].T
        B[g] = Vh[:rank]
    part_of = {g: tuple(p) for p in partitions for g in p}
    # right Gram blocks of the B step depend on W_O only
    WW = [[[W[g * group + i] @ W[g * group + j].T for j in range(group)] for i in range(group)]
          for g in range(num_kv_heads)]
    hist = [output_error(Z, W_O, A, B)]
    for _ in range(sweeps):
        for g in range(num_kv_heads):
            scope = range(Hq) if objective == "joint" else [h for h in range(Hq) if h // group in part_of[g]]
            t = torch.zeros((N, W.shape[2]), dtype=Z.dtype, device=Z.device)
            for h in scope:
                t += Z[h] @ W[h]
                if h // group != g:
                    t -= (Z[h] @ A[h // group]) @ (B[h // group] @ W[h])
            own = list(range(g * group, (g + 1) * group))
            U = [Z[h] @ A[g] for h in own]                                   # N x r
            B[g] = _solve_two_sided([[U[i].T @ U[j] for j in range(group)] for i in range(group)], WW[g],
                                    sum(U[i].T @ t @ W[own[i]].T for i in range(group)))
            M = [B[g] @ W[h] for h in own]                                   # r x hidden
            A[g] = _solve_two_sided([[Z[own[i]].T @ Z[own[j]] for j in range(group)] for i in range(group)],
                                    [[M[i] @ M[j].T for j in range(group)] for i in range(group)],
                                    sum(Z[own[i]].T @ t @ M[i].T for i in range(group)))
        hist.append(output_error(Z, W_O, A, B))
    return A, B, hist


def calibration_outputs(q: torch.Tensor, keys: torch.Tensor, values: torch.Tensor) -> torch.Tensor:
    """Exact attention outputs Z [Hq, N, d] of N calibration queries per head over one
    sequence: q [N, Hq, d]; keys, values [T, Hkv, d] (GQA: head h reads group h // G)."""
    N, Hq, d = q.shape
    Hkv = keys.shape[1]
    group = Hq // Hkv
    out = torch.empty((Hq, N, d), dtype=q.dtype, device=q.device)
    for h in range(Hq):
        g = h // group
        s = (q[:, h] @ keys[:, g].T) / d ** 0.5
        out[h] = torch.softmax(s, dim=-1) @ values[:, g]
    return out


def with_value_factors(case: Case, A: torch.Tensor, B: torch.Tensor) -> Case:
    """`case` with the Value factors A [Hkv, d, r] and B [Hkv, r, d] (for instance from
    fit_value_factors) and the key factors refitted to them as the workloads fit them:
    P_g by least squares of K on C = V A_g, E_g the top rank_k directions of the
    residual, over every token of the case.  All four are rounded to the case's
    storage dtype, so the decode path (basiskv_fuse_out_factor builds G_h = B_g W_O,h)
    runs on them directly."""
    gvv, gvk, gkk = gram_matrices(case.keys, case.values)
    P, E = key_factors_from_grams(gvv, gvk, gkk, A.detach().to("cpu", torch.float64), case.wl.rank_k)
    td, dev = case.A.dtype, case.A.device
    return dataclasses.replace(case, A=A.to(dev, td), Bf=B.to(dev, td), P=P.to(dev, td), E=E.to(dev, td))

