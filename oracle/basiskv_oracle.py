"""fp64 CPU oracle of the BasisKV decode step.  TEST INFRASTRUCTURE ONLY.

Only the tests, the smoke check and the benchmark's CPU-baseline leg may import
this module.  The product path (the CUDA library and its binding) never does;
the two share no code.

What it computes follows the BasisKV abstract ("BasisKV: Value Latents for
Communication and Key Routing", weekinpapers.com/paper/2611.02583v1, Abstract)
and the kongchang.com explainer of it (sections "用Value潜变量辅助Key路由" on
key routing, and the opening section on binding the Value latent to the output
projection), with the decode-step order of the machinelearning.ru
"KV-кэширование" page (section "Фаза Decode": the new K/V are appended first,
then the new query attends over every cached token) and its attention formula
(section "Математическая формализация").  The formulas of the five steps are
the plainest reading of those passages:

  1. append       C = v A_g,  R = (k - C P_g) E_g           (stored rounded)
  2. summary      S_p = mean_t(C_t) P_g + mean_t(R_t) E_g^T  over the page's
                  valid tokens (the mean predicted key), stored fp32
  3. route        score_p = q_h . S_p ; top-k of pages 1..n-2 by
                  (score desc, page asc), plus sink page 0 and recent page n-1
  4. attention    exact softmax(q K^T / sqrt(d)) over the selected pages'
                  original keys, weights applied to the stored latents C
  5. out-proj     y = sum_h o_h G_h  with  G_h = B_g W_O,h

A variant of step 3 routes once per KV group: the pages only say that routing
picks key pages whose original keys are then read back (explainer, section
"用Value潜变量辅助Key路由"), and under grouped-query attention the G query
heads of a group share one cached key head (cloud.baidu.com article
"大模型KV缓存压缩架构解析", section "1. 分组查询注意力（GQA）").  The variant
scores page p for the whole group by the sum, or the maximum, over the group's
heads of q_h . S_p and applies step 3's selection rule to that one score row;
every head of the group then attends over the same pages.

All arithmetic is fp64 numpy; a matmul is used as a library primitive where
a step is a plain matrix product.  Rounding to the storage type (bf16
round-to-nearest-even, or fp32) happens exactly where a value is stored.

Pins (tests/test_oracle_pins.py): dense-attention special case against
torch's scaled_dot_product_attention, identity factors, closed-form page
means, a full-sort and brute-force check of the selection, softmax weights
summing to one, associativity of the fused out-projection, a hand-worked
golden example; for the per-group routing a hand-worked two-head example and
reductions to per-head routing; for the factor fit the Eckart-Young error,
exact low-rank recovery, closed-form least-squares steps and monotone sweeps.
Every function below is pinned by at least one of them.
"""
from __future__ import annotations

import math

import numpy as np

__all__ = [
    "round_storage", "append_latents", "page_summaries", "route_pages", "route_pages_group",
    "sparse_attention", "fuse_out_factor", "out_projection",
    "SequenceCache", "prefill", "decode_step", "num_pages", "fit_value_factors", "output_error",
]


# --------------------------------------------------------------------------
# storage rounding
# --------------------------------------------------------------------------
def _round_bf16(x: np.ndarray) -> np.ndarray:
    """Nearest bf16 value (ties to even) of fp64 ``x``, returned as fp64.

    bf16 keeps 8 significant bits and the fp32 exponent range.  For
    |x| in [2^(e-1), 2^e) the spacing of bf16 values is 2^(e-8); below the
    smallest normal 2^-126 it stays 2^-133.  Dividing by a power of two and
    ``rint`` (round half to even) are exact in fp64, so this is one correct
    rounding of the fp64 input.
    """
    x = np.asarray(x, dtype=np.float64)
    _, e = np.frexp(x)
    e = np.maximum(e, -125)
    spacing = np.ldexp(1.0, e - 8)
    out = np.rint(x / spacing) * spacing
    big = np.abs(out) >= 2.0 ** 128
    if np.any(big):
        out = np.where(big, np.copysign(np.inf, x), out)
    return out


def round_storage(x: np.ndarray, storage: str) -> np.ndarray:
    """Round fp64 values to the storage type ``storage`` ("bf16", "f32" or "f64")."""
    x = np.asarray(x, dtype=np.float64)
    if storage == "bf16":
        return _round_bf16(x)
    if storage == "f32":
        return x.astype(np.float32).astype(np.float64)
    if storage == "f64":
        return x.copy()
    raise ValueError(f"unknown storage type {storage!r}")


def num_pages(length: int, page_size: int) -> int:
    return -(-length // page_size)


# --------------------------------------------------------------------------
# step 1: append (Value latent and key-specific residual)
# --------------------------------------------------------------------------
def append_latents(k, v, A, P, E, storage: str):
    """Latent and residual of new tokens of one KV head.

    k, v: [T, d] (the new tokens' key and value rows); A: [d, r]; P: [r, d];
    E: [d, s].  The Value latent is C = v A; the key residual is what the
    latent's key prediction C P misses, projected on the residual basis:
    R = (k - C P) E.  R is formed from the unrounded C; only then are C and R
    rounded to the storage type.  Returns (C_stored [T, r], R_stored [T, s]).
    """
    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    C = v @ A
    R = (k - C @ P) @ E
    return round_storage(C, storage), round_storage(R, storage)


# --------------------------------------------------------------------------
# step 2: page summary (mean predicted key)
# --------------------------------------------------------------------------
def page_summaries(C_st, R_st, P, E, page_size: int, pages=None, storage: str = "f32"):
    """Mean predicted key of each page of one KV head.

    C_st: [T, r] and R_st: [T, s] are the stored latents/residuals of the T
    valid tokens.  The predicted key of a token is C P + R E^T; by linearity
    its page mean is mean(C) P + mean(R) E^T, the mean taken over the page's
    valid tokens only (a partial last page is not zero-padded).
    ``pages`` restricts the computation to the listed page indices.
    Returns [n_pages or len(pages), d], rounded to ``storage``.
    """
    T = C_st.shape[0]
    n = num_pages(T, page_size)
    idx = range(n) if pages is None else pages
    d = P.shape[1]
    out = np.empty((len(idx), d), dtype=np.float64)
    for i, p in enumerate(idx):
        lo, hi = p * page_size, min(T, (p + 1) * page_size)
        mean_c = C_st[lo:hi].mean(axis=0)
        mean_r = R_st[lo:hi].mean(axis=0)
        out[i] = mean_c @ P + mean_r @ E.T
    return round_storage(out, storage)


# --------------------------------------------------------------------------
# step 3: key routing
# --------------------------------------------------------------------------
def route_pages(q, S, top_k: int):
    """Pages one query head attends to.

    q: [d]; S: [n, d] stored page summaries.  score_p = q . S_p (unscaled:
    1/sqrt(d) would not change the order).  The sink page 0 and the recent
    page n-1 are always kept and do not compete; of pages 1..n-2 the top_k
    are taken under the total order (score descending, page index ascending).
    With n <= top_k + 2 every page is kept.  Returns (selected pages in
    ascending order, fp64 scores of all n pages).
    """
    q = np.asarray(q, dtype=np.float64)
    scores = S @ q
    return _select_pages(scores, top_k), scores


def _select_pages(scores, top_k: int):
    """Step 3's selection rule on one row of page scores (see route_pages)."""
    n = scores.shape[0]
    if n <= top_k + 2:
        return np.arange(n, dtype=np.int64)
    candidates = list(range(1, n - 1))
    candidates.sort(key=lambda p: (-scores[p], p))
    chosen = set(candidates[:top_k])
    chosen.add(0)
    chosen.add(n - 1)
    return np.array(sorted(chosen), dtype=np.int64)


def route_pages_group(qs, S, top_k: int, reduce: str):
    """Pages a whole KV group attends to: one selection for its G query heads.

    qs: [G, d] the group's query rows; S: [n, d].  The group's score of page p
    is the sum (reduce="sum") or the maximum (reduce="max") over the heads h
    of q_h . S_p; step 3's rule then selects from that one row.  Returns
    (selected pages in ascending order, fp64 group scores of all n pages).
    """
    qs = np.asarray(qs, dtype=np.float64)
    per_head = S @ qs.T  # [n, G]
    if reduce == "sum":
        scores = per_head.sum(axis=1)
    elif reduce == "max":
        scores = per_head.max(axis=1)
    else:
        raise ValueError(f"reduce must be 'sum' or 'max', not {reduce!r}")
    return _select_pages(scores, top_k), scores


# --------------------------------------------------------------------------
# step 4: exact attention on the selected pages
# --------------------------------------------------------------------------
def sparse_attention(q, K, C_st, sel, page_size: int):
    """Exact attention of one query head over the tokens of the selected pages.

    q: [d]; K: [T, d] original keys; C_st: [T, r] stored Value latents;
    sel: page indices.  s_j = q . K_j / sqrt(d) over the valid tokens j of
    the selected pages, w = softmax(s), o = sum_j w_j C_j (rank r).
    Returns (o [r], w, token indices).
    """
    q = np.asarray(q, dtype=np.float64)
    T, d = K.shape
    tok = np.concatenate([np.arange(p * page_size, min(T, (p + 1) * page_size)) for p in sel])
    s = (K[tok] @ q) / math.sqrt(d)
    w = np.exp(s - s.max())
    w = w / w.sum()
    return w @ C_st[tok], w, tok


# --------------------------------------------------------------------------
# step 5: out-projection through the bound factor
# --------------------------------------------------------------------------
def fuse_out_factor(Bf, W_O, num_q_heads: int, storage: str):
    """G_h = B_g(h) W_O,h for every query head, rounded to ``storage``.

    Bf: [Hkv, r, d] (the Value reconstruction factors); W_O: [Hq*d, hidden],
    whose rows h*d .. h*d+d-1 are W_O,h.  g(h) = h // (Hq/Hkv).
    Returns [Hq, r, hidden].
    """
    Hkv, r, d = Bf.shape
    group = num_q_heads // Hkv
    hidden = W_O.shape[1]
    G = np.empty((num_q_heads, r, hidden), dtype=np.float64)
    for h in range(num_q_heads):
        G[h] = Bf[h // group] @ W_O[h * d:(h + 1) * d]
    return round_storage(G, storage)


def out_projection(o_lat, G):
    """y = sum_h o_h G_h.  o_lat: [Hq, r]; G: [Hq, r, hidden].  Returns [hidden]."""
    y = np.zeros(G.shape[2], dtype=np.float64)
    for h in range(G.shape[0]):
        y += o_lat[h] @ G[h]
    return y


# --------------------------------------------------------------------------
# a decode step over one sequence
# --------------------------------------------------------------------------
class SequenceCache:
    """The compressed cache of one sequence, in logical token order.

    Per KV head g: raw keys K[g] [cap, d], stored latents C[g] [cap, r],
    stored residuals R[g] [cap, s] and page summaries S[g] [cap_pages, d];
    ``length`` tokens are valid.  Paging here is only the grouping of token
    rows into pages; physical placement does not change any result.
    """

    def __init__(self, num_kv_heads, head_dim, rank_v, rank_k, page_size, capacity,
                 storage, summary_storage="f32"):
        self.page_size = page_size
        self.storage = storage
        self.summary_storage = summary_storage
        self.length = 0
        npg = num_pages(capacity, page_size)
        self.K = np.zeros((num_kv_heads, capacity, head_dim))
        self.C = np.zeros((num_kv_heads, capacity, rank_v))
        self.R = np.zeros((num_kv_heads, capacity, rank_k))
        self.S = np.zeros((num_kv_heads, npg, head_dim))

    @property
    def pages(self) -> int:
        return num_pages(self.length, self.page_size)

    def append(self, k, v, A, P, E):
        """Steps 1-2 for new tokens k, v: [T, Hkv, d] (rows in token order)."""
        k = np.asarray(k, dtype=np.float64)
        v = np.asarray(v, dtype=np.float64)
        T = k.shape[0]
        lo, hi = self.length, self.length + T
        for g in range(self.K.shape[0]):
            C, R = append_latents(k[:, g], v[:, g], A[g], P[g], E[g], self.storage)
            self.K[g, lo:hi] = k[:, g]
            self.C[g, lo:hi] = C
            self.R[g, lo:hi] = R
        self.length = hi
        touched = list(range(lo // self.page_size, num_pages(hi, self.page_size)))
        for g in range(self.K.shape[0]):
            self.S[g, touched] = page_summaries(
                self.C[g, :hi], self.R[g, :hi], P[g], E[g], self.page_size,
                pages=touched, storage=self.summary_storage)


def prefill(keys, values, A, P, E, page_size, storage, capacity=None):
    """Cache of one sequence holding every row of ``keys``/``values`` [T, Hkv, d]."""
    T, Hkv, d = keys.shape
    cache = SequenceCache(Hkv, d, A.shape[2], E.shape[2], page_size,
                          capacity or T, storage)
    if T:
        cache.append(keys, values, A, P, E)
    return cache


def decode_step(cache: SequenceCache, k_new, v_new, q, A, P, E, G, top_k: int, routing: str = "head"):
    """One decode step of one sequence: append, summary, route, attend, project.

    k_new, v_new: [Hkv, d] (the new token); q: [Hq, d]; G: [Hq, r, hidden].
    routing: "head" (one selection per query head), or "group_sum" /
    "group_max" (one selection per KV group, see route_pages_group).
    Returns a dict with per-head selections ``sel`` (list of arrays),
    routing ``scores`` (list: per head, or per KV group in the group modes),
    latent outputs ``o_lat`` [Hq, r], the softmax weight sums and the output
    ``y`` [hidden].
    """
    cache.append(np.asarray(k_new)[None], np.asarray(v_new)[None], A, P, E)
    Hq = q.shape[0]
    Hkv = cache.K.shape[0]
    group = Hq // Hkv
    L, n = cache.length, cache.pages
    sels, scores, wsum = [], [], []
    if routing not in ("head", "group_sum", "group_max"):
        raise ValueError(f"unknown routing {routing!r}")
    group_sel = []
    if routing != "head":
        for g in range(Hkv):
            gsel, gsc = route_pages_group(q[g * group:(g + 1) * group], cache.S[g, :n], top_k, routing[6:])
            group_sel.append(gsel)
            scores.append(gsc)
    o_lat = np.zeros((Hq, cache.C.shape[2]))
    for h in range(Hq):
        g = h // group
        if routing == "head":
            sel, sc = route_pages(q[h], cache.S[g, :n], top_k)
            scores.append(sc)
        else:
            sel = group_sel[g]
        o, w, _ = sparse_attention(q[h], cache.K[g, :L], cache.C[g, :L], sel, cache.page_size)
        sels.append(sel)
        wsum.append(w.sum())
        o_lat[h] = o
    y = out_projection(o_lat, G)
    return {"sel": sels, "scores": scores, "o_lat": o_lat, "weight_sums": np.array(wsum), "y": y}


# --------------------------------------------------------------------------
# calibration: Value factors fitted against the complete attention output
# --------------------------------------------------------------------------
# The explainer's section "联合优化而非逐分区拟合" (and the BasisKV abstract)
# contrast two ways of fitting the low-rank factors when the heads are split
# over tensor-parallel partitions: each partition fitting its own (partial)
# attention output in isolation, or all partitions' factors optimised together
# against the complete attention output.  With the Value factor bound to the
# output projection, head h (KV group g) contributes Z_h A_g B_g W_O,h to the
# layer output, where Z_h holds the head's exact attention outputs (softmax-
# weighted raw values) on calibration queries; the target is sum_h Z_h W_O,h.

def output_error(Z, W_O, A, B, heads=None):
    """Squared Frobenius error of sum_h Z_h A_g B_g W_O,h against sum_h Z_h W_O,h.

    Z: [Hq, N, d]; W_O: [Hq*d, hidden]; A: [Hkv, d, r]; B: [Hkv, r, d];
    heads: the heads summed (default: all).  g(h) = h // (Hq / Hkv).
    """
    Hq, N, d = Z.shape
    group = Hq // A.shape[0]
    heads = range(Hq) if heads is None else heads
    err = np.zeros((N, W_O.shape[1]))
    for h in heads:
        g = h // group
        W = W_O[h * d:(h + 1) * d]
        err += Z[h] @ W - Z[h] @ A[g] @ B[g] @ W
    return float(np.sum(err * err))


def _lstsq_B(us, Ws, t):
    """argmin_B || t - sum_i us[i] B Ws[i] ||_F  (design matrix written out, np.linalg.lstsq)."""
    D = sum(np.kron(u, W.T) for u, W in zip(us, Ws))
    x = np.linalg.lstsq(D, t.reshape(-1), rcond=None)[0]
    return x.reshape(us[0].shape[1], Ws[0].shape[0])


def _lstsq_A(Zs, Ms, t):
    """argmin_A || t - sum_i Zs[i] A Ms[i] ||_F  (design matrix written out, np.linalg.lstsq)."""
    D = sum(np.kron(z, M.T) for z, M in zip(Zs, Ms))
    x = np.linalg.lstsq(D, t.reshape(-1), rcond=None)[0]
    return x.reshape(Zs[0].shape[1], Ms[0].shape[0])


def fit_value_factors(Z, W_O, num_kv_heads: int, partitions, rank: int, sweeps: int, objective: str):
    """Low-rank Value factors A_g [d, r], B_g [r, d] of every KV group.

    Z: [Hq, N, d] attention outputs of every query head on N calibration
    queries; W_O: [Hq*d, hidden]; partitions: lists of KV groups (the
    tensor-parallel ranks).  Start: A_g = the top-`rank` right singular
    vectors of the group's stacked Z rows, B_g = A_g^T (a per-partition SVD).
    Each sweep visits the groups in order; for group g the target is

      "joint":    the complete output, sum over all heads of Z_h W_O,h, minus
                  the current approximations of every other group's heads;
      "isolated": the same restricted to the heads of g's own partition,

    and the update solves the linear least-squares problem for B_g with A_g
    fixed, then for A_g with the new B_g fixed.  Returns (A, B, the complete-
    output error after the start and after every sweep).
    """
    Hq, N, d = Z.shape
    group = Hq // num_kv_heads
    hidden = W_O.shape[1]
    W = [W_O[h * d:(h + 1) * d] for h in range(Hq)]
    A = np.zeros((num_kv_heads, d, rank))
    B = np.zeros((num_kv_heads, rank, d))
    for g in range(num_kv_heads):
        rows = np.concatenate([Z[h] for h in range(g * group, (g + 1) * group)])
        Vt = np.linalg.svd(rows, full_matrices=False)[2]
        A[g] = Vt[:rank].T
        B[g] = Vt[:rank]
    part_of = {g: tuple(p) for p in partitions for g in p}
    history = [output_error(Z, W_O, A, B)]
    for _ in range(sweeps):
        for g in range(num_kv_heads):
            if objective == "joint":
                scope = range(Hq)
            elif objective == "isolated":
                scope = [h for h in range(Hq) if h // group in part_of[g]]
            else:
                raise ValueError(f"objective must be 'joint' or 'isolated', not {objective!r}")
            t = np.zeros((N, hidden))
            for h in scope:
                t += Z[h] @ W[h]
                if h // group != g:
                    t -= Z[h] @ A[h // group] @ B[h // group] @ W[h]
            own = range(g * group, (g + 1) * group)
            B[g] = _lstsq_B([Z[h] @ A[g] for h in own], [W[h] for h in own], t)
            A[g] = _lstsq_A([Z[h] for h in own], [B[g] @ W[h] for h in own], t)
        history.append(output_error(Z, W_O, A, B))
    return A, B, np.array(history)

