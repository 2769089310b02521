"""Shared helpers of the GPU parity tests: run the oracle on a workload's
sequences and compare the CUDA path's outputs with it.

Tolerances (stated for the decode step's outputs): bf16 workloads
max |err| <= 2e-2 and relative L2 <= 5e-3; fp32 workloads relative L2
<= 1e-4.  Page selections must be identical except for pairs of pages whose
oracle routing scores differ by less than 1e-5 of the head's largest |score|.
"""
from __future__ import annotations

import numpy as np
import torch

from oracle import basiskv_oracle as O

BF16_MAX_ABS = 2e-2
BF16_REL_L2 = 5e-3
F32_REL_L2 = 1e-4
NEAR_TIE_REL = 1e-5


def storage_of(wl) -> str:
    return "f32" if wl.dtype == "f32" else "bf16"


def to64(t: torch.Tensor) -> np.ndarray:
    return t.detach().to("cpu").to(torch.float64).numpy()


class OracleCase:
    """The oracle's view of a Case: factors in fp64 and the fused G."""

    def __init__(self, case):
        self.case = case
        self.wl = case.wl
        self.storage = storage_of(case.wl)
        self.A, self.P, self.E = to64(case.A), to64(case.P), to64(case.E)
        self.G = O.fuse_out_factor(to64(case.Bf), to64(case.W_O), case.wl.num_q_heads, self.storage)

    def sequence(self, b: int, routing: str = "head"):
        """Prefill all but the last token of sequence b, then one decode step."""
        wl = self.wl
        K = to64(self.case.keys[b])
        V = to64(self.case.values[b])
        L = K.shape[0]
        cache = O.prefill(K[:-1], V[:-1], self.A, self.P, self.E, wl.page_size, self.storage, capacity=L)
        out = O.decode_step(cache, K[-1], V[-1], to64(self.case.q[b]), self.A, self.P, self.E,
                            self.G, wl.top_k, routing=routing)
        return cache, out


def oracle_on_selection(oc: OracleCase, b: int, cache, out, gpu_sel: np.ndarray, gpu_cnt: np.ndarray):
    """The oracle's attention and out-projection of sequence b's decode step over the
    GPU's page selection.  Where the two selections differ only by pages whose routing
    scores tie within the near-tie rule, both are correct selections; the outputs the GPU
    must then match are the oracle's on the pages the GPU chose.  Heads whose selection
    is the oracle's keep the oracle's own results.  cache and out come from
    oc.sequence(b) (the cache holds the step's new token).
    Returns (o_lat [Hq, r], y [hidden])."""
    wl = oc.wl
    group = wl.num_q_heads // wl.num_kv_heads
    q = to64(oc.case.q[b])
    L = cache.length
    o = np.array(out["o_lat"], dtype=np.float64, copy=True)
    for h in range(wl.num_q_heads):
        s = np.asarray(gpu_sel[h, :gpu_cnt[h]], dtype=np.int64)
        if not np.array_equal(s, out["sel"][h]):
            g = h // group
            o[h] = O.sparse_attention(q[h], cache.K[g, :L], cache.C[g, :L], s, cache.page_size)[0]
    return o, O.out_projection(o, oc.G)


def selection_ok(gpu_sel: np.ndarray, gpu_cnt: int, want: np.ndarray, scores: np.ndarray,
                 rel: float = NEAR_TIE_REL):
    """(ok, exact): GPU selection vs oracle selection under the near-tie rule."""
    g = gpu_sel[:gpu_cnt]
    if gpu_cnt != len(want) or np.any(gpu_sel[gpu_cnt:] != -1):
        return False, False
    if np.any(np.diff(g) <= 0):
        return False, False
    if np.array_equal(g, want):
        return True, True
    only_g = sorted(set(g.tolist()) - set(want.tolist()))
    only_o = sorted(set(want.tolist()) - set(g.tolist()))
    if len(only_g) != len(only_o):
        return False, False
    tol = rel * float(np.max(np.abs(scores)))
    ok = all(abs(scores[a] - scores[b]) < tol for a in only_g for b in only_o)
    return ok, False


def close_report(got: np.ndarray, want: np.ndarray):
    err = np.asarray(got, np.float64) - np.asarray(want, np.float64)
    max_abs = float(np.max(np.abs(err))) if err.size else 0.0
    denom = float(np.linalg.norm(want))
    rel = float(np.linalg.norm(err)) / denom if denom > 0 else float(np.linalg.norm(err))
    return max_abs, rel


def assert_close(got, want, storage: str, what: str):
    max_abs, rel = close_report(got, want)
    if storage == "bf16":
        assert max_abs <= BF16_MAX_ABS and rel <= BF16_REL_L2, \
            f"{what}: max|err| {max_abs:.3e} (<= {BF16_MAX_ABS}), rel L2 {rel:.3e} (<= {BF16_REL_L2})"
    else:
        assert rel <= F32_REL_L2, f"{what}: rel L2 {rel:.3e} (<= {F32_REL_L2})"
    return max_abs, rel


def ulp(x: np.ndarray, storage: str) -> np.ndarray:
    """Spacing of the storage type's values at |x|."""
    x = np.abs(np.asarray(x, np.float64))
    if storage == "f32":
        return np.spacing(x.astype(np.float32)).astype(np.float64)
    _, e = np.frexp(x)
    return np.ldexp(1.0, np.maximum(e, -125) - 8)


def assert_stored_equal(got, want, storage: str, what: str, max_frac: float = 1e-4):
    """Stored values: identical except <= 1 ulp on a small fraction of elements.

    Both sides round an fp64 result once; the two fp64 sums run in different
    orders, so an exact value within ~1e-12 (relative) of a rounding midpoint
    can round to neighbouring values.
    """
    got = np.asarray(got, np.float64)
    want = np.asarray(want, np.float64)
    assert got.shape == want.shape, what
    diff = got != want
    nd = int(diff.sum())
    if nd == 0:
        return 0
    bad = np.abs(got - want)[diff] > ulp(want, storage)[diff] * 1.0000001
    assert not np.any(bad), f"{what}: {int(bad.sum())} values differ by more than 1 ulp"
    assert nd <= max(1, max_frac * got.size), f"{what}: {nd} of {got.size} values differ by 1 ulp"
    return nd


def gt_plain(Gt: torch.Tensor, num_q_heads: int, rank_v: int, hidden: int) -> np.ndarray:
    """Values of the fused factor as [hidden][Hq][r], whatever its storage layout.

    bf16 shapes with K = Hq*r % 64 == 0 and hidden % 128 == 0 are stored in
    128 x 64 tiles with XOR-swizzled 16-byte chunks (include/basiskv.h).
    """
    K = num_q_heads * rank_v
    flat = Gt.detach().reshape(-1).cpu()
    if Gt.dtype == torch.bfloat16 and K % 64 == 0 and hidden % 128 == 0:
        t = flat.reshape(hidden // 128, K // 64, 128, 8, 8)          # [mt][kc][m][pos][e]
        m = torch.arange(128)[:, None]
        pos = torch.arange(8)[None, :] ^ (m % 8)                    # chunk j of row m sits at j ^ (m % 8)
        t = t[:, :, m, pos, :]                                       # [mt][kc][m][j][e]
        t = t.permute(0, 2, 1, 3, 4).reshape(hidden, K)
    else:
        t = flat.reshape(hidden, K)
    return t.to(torch.float64).numpy().reshape(hidden, num_q_heads, rank_v)
