"""Planted mistakes in the oracle (CPU only): every one must fail at least one pin.

A mutation replaces one oracle function with a plausible wrong version (a
dropped term, a wrong sign, a wrong index or tie-break, a missing scale);
the pins of tests/test_oracle_pins.py are then run against the mutated module.
"""
import math

import numpy as np
import pytest

from oracle import basiskv_oracle as ORACLE
from tests.test_oracle_pins import ALL_CHECKS

_orig = {name: getattr(ORACLE, name) for name in
         ["append_latents", "page_summaries", "route_pages", "route_pages_group", "sparse_attention",
          "fit_value_factors", "_lstsq_B", "_lstsq_A",
          "fuse_out_factor", "out_projection", "round_storage", "_round_bf16"]}


def _summary_no_residual(C_st, R_st, P, E, page_size, pages=None, storage="f32"):
    return _orig["page_summaries"](C_st, np.zeros_like(R_st), P, E, page_size, pages, storage)


def _summary_zero_padded(C_st, R_st, P, E, page_size, pages=None, storage="f32"):
    T = C_st.shape[0]
    n = ORACLE.num_pages(T, page_size)
    idx = range(n) if pages is None else pages
    out = np.empty((len(idx), P.shape[1]))
    for i, p in enumerate(idx):
        lo, hi = p * page_size, min(T, (p + 1) * page_size)
        out[i] = C_st[lo:hi].sum(0) / page_size @ P + R_st[lo:hi].sum(0) / page_size @ E.T
    return ORACLE.round_storage(out, storage)


def _summary_transposed_E(C_st, R_st, P, E, page_size, pages=None, storage="f32"):
    if E.shape[0] != E.shape[1]:
        return _orig["page_summaries"](C_st, R_st, P, E, page_size, pages, storage)
    return _orig["page_summaries"](C_st, R_st, P, E.T.copy() + 0.0, page_size, pages, storage) \
        if not np.allclose(E, E.T) else _summary_no_residual(C_st, R_st, P, E, page_size, pages, storage)


def _append_wrong_sign(k, v, A, P, E, storage):
    C = np.asarray(v, np.float64) @ A
    R = (np.asarray(k, np.float64) + C @ P) @ E
    return ORACLE.round_storage(C, storage), ORACLE.round_storage(R, storage)


def _append_rounded_c(k, v, A, P, E, storage):
    C = ORACLE.round_storage(np.asarray(v, np.float64) @ A, storage)
    R = (np.asarray(k, np.float64) - C @ P) @ E
    return C, ORACLE.round_storage(R, storage)


def _route_no_recent(q, S, top_k):
    sel, sc = _orig["route_pages"](q, S, top_k)
    n = S.shape[0]
    if n > 1 and len(sel) > 1:
        sel = sel[sel != n - 1]
    return sel, sc


def _route_tie_high_index(q, S, top_k):
    n = S.shape[0]
    scores = S @ np.asarray(q, np.float64)
    if n <= top_k + 2:
        return np.arange(n), scores
    cand = sorted(range(1, n - 1), key=lambda p: (-scores[p], -p))
    return np.array(sorted(set(cand[:top_k]) | {0, n - 1})), scores


def _route_lowest(q, S, top_k):
    return _orig["route_pages"](-np.asarray(q, np.float64), S, top_k)[0], S @ np.asarray(q, np.float64)


def _route_k_plus_one(q, S, top_k):
    return _orig["route_pages"](q, S, top_k + 1)


def _attn_no_scale(q, K, C_st, sel, page_size):
    d = K.shape[1]
    return _orig["sparse_attention"](np.asarray(q, np.float64) * math.sqrt(d), K, C_st, sel, page_size)


def _attn_skip_partial_page(q, K, C_st, sel, page_size):
    T = K.shape[0]
    full = [p for p in sel if (p + 1) * page_size <= T]
    return _orig["sparse_attention"](q, K, C_st, np.array(full or sel[:1]), page_size)


def _fuse_wrong_group(Bf, W_O, num_q_heads, storage):
    Hkv, r, d = Bf.shape
    G = np.empty((num_q_heads, r, W_O.shape[1]))
    for h in range(num_q_heads):
        G[h] = Bf[h % Hkv] @ W_O[h * d:(h + 1) * d]
    return ORACLE.round_storage(G, storage)


def _fuse_transposed_wo(Bf, W_O, num_q_heads, storage):
    Hkv, r, d = Bf.shape
    hid = W_O.shape[1]
    Wt = W_O.reshape(d, num_q_heads, hid).transpose(1, 0, 2).reshape(num_q_heads * d, hid)
    return _orig["fuse_out_factor"](Bf, Wt, num_q_heads, storage)


def _group_first_head_only(qs, S, top_k, reduce):
    return _orig["route_pages_group"](np.asarray(qs)[:1], S, top_k, reduce)


def _group_max_as_min(qs, S, top_k, reduce):
    if reduce != "max":
        return _orig["route_pages_group"](qs, S, top_k, reduce)
    sc = (S @ np.asarray(qs, np.float64).T).min(axis=1)
    return ORACLE._select_pages(sc, top_k), sc


def _group_sum_as_mean(qs, S, top_k, reduce):
    sel, sc = _orig["route_pages_group"](qs, S, top_k, reduce)
    return sel, (sc / len(qs) if reduce == "sum" else sc)


def _lstsq_B_untransposed(us, Ws, t):
    D = sum(np.kron(u, W) for u, W in zip(us, Ws))
    x = np.linalg.lstsq(D, t.reshape(-1), rcond=None)[0]
    return x.reshape(us[0].shape[1], Ws[0].shape[0])


def _lstsq_A_drops_last_term(Zs, Ms, t):
    return _orig["_lstsq_A"](Zs[:1], Ms[:1], t) if len(Zs) > 1 else _orig["_lstsq_A"](Zs, Ms, 0.5 * t)


def _fit_with(init_last: bool = False, keep_others: bool = False):
    """fit_value_factors with one planted change (see MUTATIONS)."""
    def fit(Z, W_O, num_kv_heads, partitions, rank, sweeps, objective):
        Hq, N, d = Z.shape
        group = Hq // num_kv_heads
        W = [W_O[h * d:(h + 1) * d] for h in range(Hq)]
        A = np.zeros((num_kv_heads, d, rank))
        B = np.zeros((num_kv_heads, rank, d))
        for g in range(num_kv_heads):
            rows = np.concatenate([Z[h] for h in range(g * group, (g + 1) * group)])
            Vt = np.linalg.svd(rows, full_matrices=False)[2]
            sel = Vt[-rank:] if init_last else Vt[:rank]
            A[g], B[g] = sel.T, sel
        part_of = {g: tuple(p) for p in partitions for g in p}
        hist = [ORACLE.output_error(Z, W_O, A, B)]
        for _ in range(sweeps):
            for g in range(num_kv_heads):
                scope = range(Hq) if objective == "joint" else [h for h in range(Hq) if h // group in part_of[g]]
                t = np.zeros((N, W_O.shape[1]))
                for h in scope:
                    t += Z[h] @ W[h]
                    if h // group != g and not keep_others:
                        t -= Z[h] @ A[h // group] @ B[h // group] @ W[h]
                own = range(g * group, (g + 1) * group)
                B[g] = ORACLE._lstsq_B([Z[h] @ A[g] for h in own], [W[h] for h in own], t)
                A[g] = ORACLE._lstsq_A([Z[h] for h in own], [B[g] @ W[h] for h in own], t)
            hist.append(ORACLE.output_error(Z, W_O, A, B))
        return A, B, np.array(hist)
    return fit


def _outproj_first_head_only(o_lat, G):
    return o_lat[0] @ G[0]


def _bf16_truncate(x):
    x = np.asarray(x, np.float64)
    _, e = np.frexp(x)
    sp = np.ldexp(1.0, np.maximum(e, -125) - 8)
    return np.trunc(x / sp) * sp


MUTATIONS = {
    "summary_drops_residual": ("page_summaries", _summary_no_residual),
    "summary_zero_padded_mean": ("page_summaries", _summary_zero_padded),
    "summary_transposed_E": ("page_summaries", _summary_transposed_E),
    "append_residual_sign": ("append_latents", _append_wrong_sign),
    "append_residual_from_rounded_latent": ("append_latents", _append_rounded_c),
    "route_drops_recent_page": ("route_pages", _route_no_recent),
    "route_tie_prefers_high_index": ("route_pages", _route_tie_high_index),
    "route_picks_lowest_scores": ("route_pages", _route_lowest),
    "route_keeps_one_too_many": ("route_pages", _route_k_plus_one),
    "group_route_first_head_only": ("route_pages_group", _group_first_head_only),
    "group_route_max_as_min": ("route_pages_group", _group_max_as_min),
    "group_route_sum_as_mean": ("route_pages_group", _group_sum_as_mean),
    "fit_start_from_smallest_directions": ("fit_value_factors", _fit_with(init_last=True)),
    "fit_target_keeps_other_groups_outputs": ("fit_value_factors", _fit_with(keep_others=True)),
    "fit_B_step_untransposed_W_O": ("_lstsq_B", _lstsq_B_untransposed),
    "fit_A_step_drops_a_head": ("_lstsq_A", _lstsq_A_drops_last_term),
    "attention_missing_sqrt_d": ("sparse_attention", _attn_no_scale),
    "attention_skips_partial_page": ("sparse_attention", _attn_skip_partial_page),
    "fuse_wrong_head_group": ("fuse_out_factor", _fuse_wrong_group),
    "fuse_transposed_W_O_rows": ("fuse_out_factor", _fuse_transposed_wo),
    "out_projection_one_head": ("out_projection", _outproj_first_head_only),
    "bf16_truncates": ("_round_bf16", _bf16_truncate),
}


@pytest.mark.parametrize("name", sorted(MUTATIONS))
def test_planted_mistake_is_caught(name, monkeypatch):
    attr, bad = MUTATIONS[name]
    monkeypatch.setattr(ORACLE, attr, bad)
    failed = []
    for check in ALL_CHECKS:
        try:
            check(ORACLE)
        except Exception as exc:  # an AssertionError, or a crash on a wrong shape
            failed.append((check.__name__, type(exc).__name__))
    assert failed, f"mutation {name} passed every pin"


def test_unmutated_oracle_passes_every_pin():
    for check in ALL_CHECKS:
        check(ORACLE)
