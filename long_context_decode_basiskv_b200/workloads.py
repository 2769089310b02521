"""Seeded synthetic workloads for the BasisKV decode step.

This module draws the inputs that both the CUDA path and the fp64 oracle
consume: queries, raw keys and values, the low-rank factors, the output
projection and the paged-cache block tables.  It holds none of the decode
step's arithmetic (no latent append, no page summary, no routing, no sparse
attention, no out-projection); the factor fit below is the calibration that
produces the factors those steps take as inputs.

Generative model (BasisKV abstract, "Value latents for communication and key
routing"; the five decode workloads it is exercised on are listed in
``WORKLOADS``):

* per KV head g: ``U_g`` (d x r) random orthonormal, ``M_g`` (d x d) with
  i.i.d. N(0, std 1/sqrt(d)) entries;
* per token: ``V = Z U_g^T + 0.05 N1`` with ``Z ~ N(0, 1)`` of width r and
  ``K = V M_g + 0.3 N2``;
* ``q ~ N(0, 1)``; ``W_O ~ N(0, std 1/sqrt(hidden))``;
* factors: ``A_g`` = top-r (uncentred) principal directions of all context
  values of head g, ``B_g = A_g^T``; ``P_g`` = least-squares map from the
  latents ``V A_g`` to the keys; ``E_g`` = top-s principal directions of the
  key residual ``K - V A_g P_g``.
* the single-sequence 131K workload adds ``alpha * u_g`` (``u_g`` the unit
  mean query direction of group g) to the keys of 5% of the pages, chosen
  uniformly among the non-sink, non-recent pages, with alpha bisected so that
  those pages carry 80% of the dense softmax mass.

Bulk per-token draws use ``torch.Generator`` on the requested device (one
generator per sequence, seeded from the workload seed and the sequence index);
small host-side draws (U, M, lengths, page permutation, hot pages) use
``numpy.random.default_rng(seed)``.  Everything is drawn in fp32 and rounded
to the storage dtype (bf16 round-to-nearest-even) before anything else sees it.
"""
from __future__ import annotations

import dataclasses
import math
from dataclasses import dataclass, field
from typing import Optional

import numpy as np
import torch

__all__ = ["Workload", "WORKLOADS", "Case", "make_case", "shrink"]


@dataclass(frozen=True)
class Workload:
    name: str
    batch: int
    num_q_heads: int
    num_kv_heads: int
    head_dim: int
    context: int                 # tokens per sequence after the decode append
    page_size: int
    rank_v: int                  # r
    rank_k: int                  # s
    top_k: int
    hidden: int
    dtype: str                   # "f32" or "bf16" storage / weight dtype
    seed: int
    ragged: Optional[tuple] = None     # (lo, hi) inclusive per-sequence lengths
    hot_fraction: float = 0.0          # fraction of pages made "hot"
    hot_mass: float = 0.0              # dense softmax mass the hot pages carry

    @property
    def group(self) -> int:
        return self.num_q_heads // self.num_kv_heads

    @property
    def torch_dtype(self):
        return torch.float32 if self.dtype == "f32" else torch.bfloat16


WORKLOADS = {
    "tiny_fp32": Workload(
        "tiny_fp32", batch=1, num_q_heads=8, num_kv_heads=2, head_dim=64, context=2048,
        page_size=32, rank_v=16, rank_k=8, top_k=8, hidden=512, dtype="f32", seed=0),
    "llama3_8b_32k": Workload(
        "llama3_8b_32k", batch=8, num_q_heads=32, num_kv_heads=8, head_dim=128, context=32768,
        page_size=16, rank_v=64, rank_k=32, top_k=128, hidden=4096, dtype="bf16", seed=1),
    "single_seq_131k": Workload(
        "single_seq_131k", batch=1, num_q_heads=32, num_kv_heads=8, head_dim=128, context=131072,
        page_size=64, rank_v=64, rank_k=32, top_k=64, hidden=4096, dtype="bf16", seed=2,
        hot_fraction=0.05, hot_mass=0.80),
    "llama3_70b_64k": Workload(
        "llama3_70b_64k", batch=4, num_q_heads=64, num_kv_heads=8, head_dim=128, context=65536,
        page_size=16, rank_v=96, rank_k=32, top_k=256, hidden=8192, dtype="bf16", seed=3),
    "ragged_serving": Workload(
        "ragged_serving", batch=64, num_q_heads=32, num_kv_heads=8, head_dim=128, context=32768,
        page_size=16, rank_v=64, rank_k=32, top_k=128, hidden=4096, dtype="bf16", seed=4,
        ragged=(2048, 32768)),
}


def shrink(wl: Workload, *, batch: Optional[int] = None, context: Optional[int] = None,
           ragged: Optional[tuple] = None, top_k: Optional[int] = None,
           seed: Optional[int] = None, name: Optional[str] = None) -> Workload:
    """Same head geometry, ranks and dtype as ``wl`` with a smaller batch/context."""
    kw = {}
    if batch is not None:
        kw["batch"] = batch
    if context is not None:
        kw["context"] = context
    if ragged is not None:
        kw["ragged"] = ragged
    if top_k is not None:
        kw["top_k"] = top_k
    if seed is not None:
        kw["seed"] = seed
    kw["name"] = name or f"{wl.name}_small"
    return dataclasses.replace(wl, **kw)


@dataclass
class Case:
    """One seeded decode-step instance.

    Token tensors are per sequence: ``keys[b]``/``values[b]`` are
    ``[L_b, Hkv, d]`` in the storage dtype; the last row is the token the
    decode step appends, the others form the prefilled context.
    Factor tensors are in the storage dtype:
    ``A [Hkv, d, r]``, ``Bf [Hkv, r, d]``, ``P [Hkv, r, d]``, ``E [Hkv, d, s]``,
    ``W_O [Hq*d, hidden]``; ``q [B, Hq, d]``.
    ``block_table [B, max_pages]`` holds physical page ids (-1 past the end).
    """
    wl: Workload
    lengths: list
    q: torch.Tensor
    keys: list
    values: list
    A: torch.Tensor
    Bf: torch.Tensor
    P: torch.Tensor
    E: torch.Tensor
    W_O: torch.Tensor
    block_table: torch.Tensor
    num_phys_pages: int
    max_pages: int
    hot_pages: Optional[np.ndarray] = None
    hot_alpha: float = 0.0
    hot_mass: float = 0.0
    info: dict = field(default_factory=dict)

    def pages(self, b: int) -> int:
        return -(-self.lengths[b] // self.wl.page_size)


def _orthonormal(rng: np.random.Generator, d: int, r: int) -> np.ndarray:
    qmat, rmat = np.linalg.qr(rng.standard_normal((d, r)))
    return qmat * np.sign(np.diag(rmat))[None, :]


def _fix_signs(vecs: torch.Tensor) -> torch.Tensor:
    """Deterministic sign: the largest-magnitude entry of each column is positive."""
    idx = vecs.abs().argmax(dim=0)
    s = torch.sign(vecs[idx, torch.arange(vecs.shape[1])])
    s[s == 0] = 1
    return vecs * s[None, :]


def _top_eigvecs(gram: torch.Tensor, k: int) -> torch.Tensor:
    w, v = torch.linalg.eigh(gram)           # ascending eigenvalues
    order = torch.argsort(w, descending=True)[:k]
    return _fix_signs(v[:, order])


def _seq_generator(device, seed: int, b: int) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(int(seed) * 1_000_003 + 7919 * int(b) + 17)
    return g


def make_case(wl: Workload, device="cpu") -> Case:
    """Draw the workload ``wl`` on ``device`` (token tensors stay there)."""
    device = torch.device(device)
    rng = np.random.default_rng(wl.seed)
    B, Hq, Hkv, d, r, s = wl.batch, wl.num_q_heads, wl.num_kv_heads, wl.head_dim, wl.rank_v, wl.rank_k
    G = wl.group
    assert Hq % Hkv == 0 and r <= d and s <= d

    # host-side draws, fixed order: U, M, lengths, permutation, hot pages
    U = np.stack([_orthonormal(rng, d, r) for _ in range(Hkv)])                  # [Hkv, d, r]
    M = rng.standard_normal((Hkv, d, d)) / math.sqrt(d)                          # [Hkv, d, d]
    if wl.ragged is not None:
        lo, hi = wl.ragged
        lengths = [int(x) for x in rng.integers(lo, hi, size=B, endpoint=True)]
    else:
        lengths = [wl.context] * B
    P_ = wl.page_size
    npages = [-(-L // P_) for L in lengths]
    num_phys = int(sum(npages))
    perm = rng.permutation(num_phys).astype(np.int32)
    max_pages = max(npages)
    bt = np.full((B, max_pages), -1, dtype=np.int32)
    off = 0
    for b in range(B):
        bt[b, :npages[b]] = perm[off:off + npages[b]]
        off += npages[b]

    gq = _seq_generator(device, wl.seed, 1 << 20)
    q32 = torch.randn((B, Hq, d), generator=gq, device=device, dtype=torch.float32)
    wo32 = torch.randn((Hq * d, wl.hidden), generator=gq, device=device,
                       dtype=torch.float32) / math.sqrt(wl.hidden)

    U_t = torch.from_numpy(U).to(device=device, dtype=torch.float32)
    M_t = torch.from_numpy(M).to(device=device, dtype=torch.float32)
    keys32, vals32 = [], []
    for b in range(B):
        g = _seq_generator(device, wl.seed, b)
        L = lengths[b]
        Z = torch.randn((L, Hkv, r), generator=g, device=device, dtype=torch.float32)
        N1 = torch.randn((L, Hkv, d), generator=g, device=device, dtype=torch.float32)
        N2 = torch.randn((L, Hkv, d), generator=g, device=device, dtype=torch.float32)
        V = torch.einsum("thr,hdr->thd", Z, U_t) + 0.05 * N1
        del Z, N1
        K = torch.einsum("thd,hde->the", V, M_t) + 0.3 * N2
        del N2
        keys32.append(K)
        vals32.append(V)

    hot_pages = None
    alpha = 0.0
    mass = 0.0
    if wl.hot_fraction > 0:
        hot_pages, alpha, mass = _plant_hot_pages(wl, rng, q32, keys32, lengths)

    td = wl.torch_dtype
    keys = [k.to(td) for k in keys32]
    values = [v.to(td) for v in vals32]
    del keys32, vals32
    q = q32.to(td)
    W_O = wo32.to(td)

    A, Bf, Pm, E = _fit_factors(wl, keys, values)
    return Case(wl=wl, lengths=lengths, q=q, keys=keys, values=values,
                A=A.to(device=device, dtype=td), Bf=Bf.to(device=device, dtype=td),
                P=Pm.to(device=device, dtype=td), E=E.to(device=device, dtype=td),
                W_O=W_O, block_table=torch.from_numpy(bt).to(device),
                num_phys_pages=num_phys, max_pages=max_pages,
                hot_pages=hot_pages, hot_alpha=alpha, hot_mass=mass)


def _fit_factors(wl: Workload, keys, values):
    """Calibration stand-in for the pages' joint factor fit (uncentred PCA + least squares).

    Works from per-head Gram matrices (V^T V, V^T K, K^T K) accumulated in
    fp64 over every context token of every sequence, so it never holds an
    fp64 copy of the cache.
    """
    Hkv, d, r, s = wl.num_kv_heads, wl.head_dim, wl.rank_v, wl.rank_k
    gvv, gvk, gkk = gram_matrices(keys, values)
    A = torch.zeros((Hkv, d, r), dtype=torch.float64)
    for h in range(Hkv):
        A[h] = _top_eigvecs(gvv[h], r)                   # d x r
    Pm, E = key_factors_from_grams(gvv, gvk, gkk, A, s)
    Bf = A.transpose(1, 2).contiguous()
    return A, Bf, Pm, E


def gram_matrices(keys, values):
    """Per-KV-head fp64 Gram matrices V^T V, V^T K, K^T K over every token of the
    given sequences (lists of [T, Hkv, d]), accumulated in chunks; on the host."""
    Hkv, d = keys[0].shape[1], keys[0].shape[2]
    dev = keys[0].device
    gvv = torch.zeros((Hkv, d, d), dtype=torch.float64, device=dev)
    gvk = torch.zeros_like(gvv)
    gkk = torch.zeros_like(gvv)
    for K, V in zip(keys, values):
        for t0 in range(0, K.shape[0], 1 << 16):
            k = K[t0:t0 + (1 << 16)].to(torch.float64)
            v = V[t0:t0 + (1 << 16)].to(torch.float64)
            gvv += torch.einsum("thd,the->hde", v, v)
            gvk += torch.einsum("thd,the->hde", v, k)
            gkk += torch.einsum("thd,the->hde", k, k)
    return gvv.cpu(), gvk.cpu(), gkk.cpu()


def key_factors_from_grams(gvv, gvk, gkk, A, s: int):
    """Key factors for given Value encoders A [Hkv, d, r]: P_g by least squares of K on
    C = V A_g, E_g the top-s directions of the residual K - C P_g (from the Gram matrices)."""
    Hkv, d, r = A.shape
    Pm = torch.zeros((Hkv, r, d), dtype=torch.float64)
    E = torch.zeros((Hkv, d, s), dtype=torch.float64)
    for h in range(Hkv):
        a = A[h].to(torch.float64)
        ctc = a.T @ gvv[h] @ a                           # C^T C
        ctk = a.T @ gvk[h]                               # C^T K
        p = torch.linalg.solve(ctc, ctk)                 # r x d
        res = gkk[h] - ctk.T @ p - p.T @ ctk + p.T @ ctc @ p
        res = 0.5 * (res + res.T)
        Pm[h], E[h] = p, _top_eigvecs(res, s)
    return Pm, E


def _plant_hot_pages(wl: Workload, rng, q32, keys32, lengths):
    """Make 5% of the pages carry ~80% of the dense softmax mass (keys shifted along q)."""
    B, Hq, Hkv, d, P_ = wl.batch, wl.num_q_heads, wl.num_kv_heads, wl.head_dim, wl.page_size
    G = wl.group
    assert B == 1, "hot-page planting is defined for a single sequence"
    L = lengths[0]
    n = -(-L // P_)
    nhot = int(math.ceil(wl.hot_fraction * n))
    hot = np.sort(rng.choice(np.arange(1, n - 1), size=nhot, replace=False)).astype(np.int64)
    K = keys32[0]                                               # [L, Hkv, d] fp32
    dev = K.device
    tok_hot = torch.zeros(L, dtype=torch.bool, device=dev)
    hot_t = torch.from_numpy(hot).to(dev)
    for j in range(P_):
        idx = hot_t * P_ + j
        tok_hot[idx[idx < L]] = True
    qg = q32[0].view(Hkv, G, d)
    u = qg.mean(dim=1)
    u = u / u.norm(dim=1, keepdim=True)                         # [Hkv, d]
    scale = 1.0 / math.sqrt(d)
    base = torch.einsum("hgd,thd->hgt", qg.double(), K.double()) * scale      # [Hkv, G, L]
    qu = torch.einsum("hgd,hd->hg", qg.double(), u.double()) * scale         # [Hkv, G]
    hotf = tok_hot.double()

    def mass(alpha: float) -> float:
        sc = base + alpha * qu[:, :, None] * hotf[None, None, :]
        w = torch.softmax(sc, dim=-1)
        return float((w * hotf).sum(-1).mean())

    lo, hi = 0.0, 1.0
    while mass(hi) < wl.hot_mass:
        hi *= 2.0
        if hi > 1e4:
            break
    for _ in range(60):
        mid = 0.5 * (lo + hi)
        if mass(mid) < wl.hot_mass:
            lo = mid
        else:
            hi = mid
        if hi - lo < 1e-6:
            break
    alpha = 0.5 * (lo + hi)
    K += alpha * tok_hot[:, None, None].float() * u[None, :, :].float()
    return hot, float(alpha), mass(alpha)
