"""Pins of the fp64 oracle against things other than itself (CPU only).

Each ``check_*`` takes the oracle module so that tests/test_oracle_mutations.py
can run the same checks against an oracle with a planted mistake and show
that at least one of them fails.
"""
import itertools
import json
import math
import os

import numpy as np
import pytest
import torch

from oracle import basiskv_oracle as ORACLE

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "worked_example.json")


def _rand_orth(rng, d, r):
    qm, _ = np.linalg.qr(rng.standard_normal((d, r)))
    return qm


def _sdpa(q, K, V):
    """Textbook softmax(q K^T / sqrt(d)) V via torch's library routine (fp64, CPU)."""
    qt = torch.from_numpy(np.asarray(q, np.float64))[None, None, None, :]
    kt = torch.from_numpy(np.asarray(K, np.float64))[None, None]
    vt = torch.from_numpy(np.asarray(V, np.float64))[None, None]
    return torch.nn.functional.scaled_dot_product_attention(qt, kt, vt)[0, 0, 0].numpy()


# ---------------------------------------------------------------------------
# storage rounding
# ---------------------------------------------------------------------------
def check_bf16_rounding(o):
    rng = np.random.default_rng(11)
    x32 = np.concatenate([
        rng.standard_normal(20000).astype(np.float32) * np.float32(3.0),
        (rng.standard_normal(2000) * 1e-39).astype(np.float32),          # subnormal range
        (rng.standard_normal(2000) * 1e37).astype(np.float32),
        np.array([1 + 2 ** -8, 1 + 3 * 2 ** -8, -(1 + 2 ** -8), 0.0, -0.0,
                  2 ** -126, 2 ** -133, 3.3e38], dtype=np.float32),      # ties, tiny, huge
    ])
    want = torch.from_numpy(x32).to(torch.bfloat16).to(torch.float64).numpy()
    got = o.round_storage(x32.astype(np.float64), "bf16")
    np.testing.assert_array_equal(got, want)
    # fp64 inputs just above / below a bf16 midpoint must not double-round
    assert o.round_storage(np.array([1 + 2 ** -8 + 2 ** -40]), "bf16")[0] == 1 + 2 ** -7
    assert o.round_storage(np.array([1 + 2 ** -8 - 2 ** -40]), "bf16")[0] == 1.0
    f = rng.standard_normal(1000)
    np.testing.assert_array_equal(o.round_storage(f, "f32"), f.astype(np.float32).astype(np.float64))


def test_bf16_rounding_matches_torch():
    check_bf16_rounding(ORACLE)


# ---------------------------------------------------------------------------
# step 1: append
# ---------------------------------------------------------------------------
def check_append_identity(o):
    """A = I (r = d), P = I, E = I (s = d): C = v and R = k - v exactly."""
    rng = np.random.default_rng(1)
    d = 8
    k = rng.standard_normal((5, d))
    v = rng.standard_normal((5, d))
    eye = np.eye(d)
    C, R = o.append_latents(k, v, eye, eye, eye, "f64")
    np.testing.assert_array_equal(C, v)
    np.testing.assert_allclose(R, k - v, rtol=0, atol=1e-15)
    # the residual is taken from the unrounded latent
    v_b = o.round_storage(v * 1.001, "bf16")
    C2, R2 = o.append_latents(k, v_b * (1 + 2 ** -12), eye, eye, eye, "bf16")
    np.testing.assert_array_equal(R2, o.round_storage(k - v_b * (1 + 2 ** -12), "bf16"))


def check_append_projection(o):
    """Rank-r latent of a value lying in span(A) recovers its coordinates exactly."""
    rng = np.random.default_rng(2)
    d, r, s = 16, 4, 3
    A = _rand_orth(rng, d, r)
    coords = rng.standard_normal((6, r))
    v = coords @ A.T
    P = rng.standard_normal((r, d))
    E = _rand_orth(rng, d, s)
    resid = rng.standard_normal((6, s))
    k = coords @ P + resid @ E.T           # key = predicted part + residual in span(E)
    C, R = o.append_latents(k, v, A, P, E, "f64")
    np.testing.assert_allclose(C, coords, atol=1e-12)
    np.testing.assert_allclose(R, resid, atol=1e-12)


def test_append_identity():
    check_append_identity(ORACLE)


def test_append_projection():
    check_append_projection(ORACLE)


# ---------------------------------------------------------------------------
# step 2: page summaries
# ---------------------------------------------------------------------------
def check_summary_closed_form(o):
    """s = d, E = I: the predicted key is the key itself, so S_p = mean of the page's keys.

    The length is not a multiple of the page size: the last page's mean is
    over its valid tokens only.
    """
    rng = np.random.default_rng(3)
    d, r, ps, T = 8, 3, 4, 14
    A = _rand_orth(rng, d, r)
    P = rng.standard_normal((r, d))
    E = np.eye(d)
    k = rng.standard_normal((T, d))
    v = rng.standard_normal((T, d))
    C, R = o.append_latents(k, v, A, P, E, "f64")
    S = o.page_summaries(C, R, P, E, ps, storage="f64")
    assert S.shape == (4, d)
    for p in range(4):
        np.testing.assert_allclose(S[p], k[p * ps:min(T, (p + 1) * ps)].mean(axis=0), atol=1e-12)
    # a subset of pages gives the same rows
    S2 = o.page_summaries(C, R, P, E, ps, pages=[3, 1], storage="f64")
    np.testing.assert_allclose(S2, S[[3, 1]], atol=0)


def check_summary_low_rank_residual(o):
    """With a key that is exactly C P + R E^T, the summary is the page mean of the keys."""
    rng = np.random.default_rng(4)
    d, r, s, ps, T = 12, 3, 2, 5, 13
    A = _rand_orth(rng, d, r)
    E = _rand_orth(rng, d, s)
    P = rng.standard_normal((r, d))
    P = P - (P @ E) @ E.T                   # prediction orthogonal to the residual basis
    coords = rng.standard_normal((T, r))
    resid = rng.standard_normal((T, s))
    v = coords @ A.T
    k = coords @ P + resid @ E.T
    C, R = o.append_latents(k, v, A, P, E, "f64")
    S = o.page_summaries(C, R, P, E, ps, storage="f64")
    for p in range(3):
        np.testing.assert_allclose(S[p], k[p * ps:min(T, (p + 1) * ps)].mean(axis=0), atol=1e-12)


def test_summary_closed_form():
    check_summary_closed_form(ORACLE)


def test_summary_low_rank_residual():
    check_summary_low_rank_residual(ORACLE)


# ---------------------------------------------------------------------------
# step 3: routing
# ---------------------------------------------------------------------------
def _sort_reference(scores, k):
    n = len(scores)
    if n <= k + 2:
        return np.arange(n)
    cand = np.arange(1, n - 1)
    order = np.lexsort((cand, -scores[1:n - 1]))      # primary: score desc, then index asc
    return np.unique(np.concatenate([[0, n - 1], cand[order[:k]]]))


def check_route_full_sort(o):
    rng = np.random.default_rng(5)
    for n, k in [(64, 8), (200, 17), (2048, 128), (10, 8), (11, 8)]:
        S = rng.standard_normal((n, 16))
        q = rng.standard_normal(16)
        sel, scores = o.route_pages(q, S, k)
        np.testing.assert_allclose(scores, S @ q, atol=1e-12)
        np.testing.assert_array_equal(sel, _sort_reference(scores, k))
        assert len(sel) == min(n, k + 2)
        assert sel[0] == 0 and sel[-1] == n - 1
        assert np.all(np.diff(sel) > 0)


def check_route_ties(o):
    """Equal scores: the lower page index wins."""
    S = np.zeros((8, 2))
    S[:, 0] = [0, 1, 2, 2, 2, 1, 0, -5]
    sel, _ = o.route_pages(np.array([1.0, 0.0]), S, 2)
    np.testing.assert_array_equal(sel, [0, 2, 3, 7])


def check_route_bruteforce(o):
    """n <= 12: the kept non-sink, non-recent pages are the k-subset of largest total score."""
    rng = np.random.default_rng(6)
    for n in range(4, 13):
        for k in range(1, n - 2):
            S = rng.standard_normal((n, 4))
            q = rng.standard_normal(4)
            sel, scores = o.route_pages(q, S, k)
            best = max(itertools.combinations(range(1, n - 1), k),
                       key=lambda c: sum(scores[list(c)]))
            np.testing.assert_array_equal(sel, sorted(set(best) | {0, n - 1}))


def check_route_small_n(o):
    q = np.array([1.0, -1.0])
    for n in [1, 2, 3, 5]:
        S = np.random.default_rng(n).standard_normal((n, 2))
        sel, _ = o.route_pages(q, S, 3)
        np.testing.assert_array_equal(sel, np.arange(n))
    # sink and recent are kept however low they score
    S = np.array([[-100.0, 0], [1, 0], [2, 0], [3, 0], [-100.0, 0]])
    sel, _ = o.route_pages(np.array([1.0, 0.0]), S, 1)
    np.testing.assert_array_equal(sel, [0, 3, 4])


def check_route_group_worked_example(o):
    """Two heads reading one coordinate each; the group scores worked by hand.

    Per page (1..4) the head scores are (5, -9), (-9, 4), (1, 1), (3, 3):
    max over heads = 5, 4, 1, 3 and sum = -4, -5, 2, 6.  With k = 2 the max
    keeps pages 1 and 2, the sum pages 3 and 4 (head 0 alone would keep 1 and 4).
    """
    S = np.array([[0.0, 0], [5, -9], [-9, 4], [1, 1], [3, 3], [0, 0]])
    qs = np.eye(2)
    sel, sc = o.route_pages_group(qs, S, 2, "max")
    np.testing.assert_array_equal(sel, [0, 1, 2, 5])
    np.testing.assert_allclose(sc[1:5], [5, 4, 1, 3], atol=0)
    sel, sc = o.route_pages_group(qs, S, 2, "sum")
    np.testing.assert_array_equal(sel, [0, 3, 4, 5])
    np.testing.assert_allclose(sc[1:5], [-4, -5, 2, 6], atol=0)
    np.testing.assert_array_equal(o.route_pages(qs[0], S, 2)[0], [0, 1, 4, 5])


def check_route_group_reductions(o):
    """Group routing against identities: one head is per-head routing; the sum
    is the score of the summed query (linearity); identical heads select what
    one of them selects; the max is at least every head's score."""
    rng = np.random.default_rng(11)
    for n, k, G in [(64, 8, 4), (300, 17, 8), (12, 3, 2), (9, 8, 4)]:
        S = rng.standard_normal((n, 16))
        qs = rng.standard_normal((G, 16))
        for red in ("sum", "max"):
            sel1, sc1 = o.route_pages_group(qs[:1], S, k, red)
            sel_h, sc_h = o.route_pages(qs[0], S, k)
            np.testing.assert_array_equal(sel1, sel_h)
            np.testing.assert_allclose(sc1, sc_h, atol=1e-12)
            same = np.repeat(qs[:1], G, axis=0)
            np.testing.assert_array_equal(o.route_pages_group(same, S, k, red)[0], sel_h)
        sel, sc = o.route_pages_group(qs, S, k, "sum")
        qsum = qs.sum(axis=0)
        np.testing.assert_allclose(sc, S @ qsum, atol=1e-11)
        np.testing.assert_array_equal(sel, _sort_reference(S @ qsum, k))
        sel, sc = o.route_pages_group(qs, S, k, "max")
        for h in range(G):
            assert np.all(sc >= S @ qs[h] - 1e-12)
        assert np.all(np.isclose(sc[:, None], S @ qs.T, atol=1e-12).any(axis=1))  # attained by a head
        np.testing.assert_array_equal(sel, _sort_reference(sc, k))
        assert len(sel) == min(n, k + 2)


def test_route_group_worked_example():
    check_route_group_worked_example(ORACLE)


def test_route_group_reductions():
    check_route_group_reductions(ORACLE)


def test_route_full_sort():
    check_route_full_sort(ORACLE)


def test_route_ties():
    check_route_ties(ORACLE)


def test_route_bruteforce():
    check_route_bruteforce(ORACLE)


def test_route_small_n():
    check_route_small_n(ORACLE)


# ---------------------------------------------------------------------------
# step 4: exact sparse attention
# ---------------------------------------------------------------------------
def check_attention_dense_reduction(o):
    """Selecting every page with r = d and A = I reduces to textbook attention over V."""
    rng = np.random.default_rng(7)
    d, ps, T = 16, 4, 23
    K = rng.standard_normal((T, d))
    V = rng.standard_normal((T, d))
    q = rng.standard_normal(d) * 2.0
    n = o.num_pages(T, ps)
    out, w, tok = o.sparse_attention(q, K, V, np.arange(n), ps)
    np.testing.assert_array_equal(tok, np.arange(T))
    np.testing.assert_allclose(out, _sdpa(q, K, V), atol=1e-12)
    assert abs(w.sum() - 1.0) < 1e-12


def check_attention_subset(o):
    """A page subset equals textbook attention over the subset's tokens (partial last page)."""
    rng = np.random.default_rng(8)
    d, r, ps, T = 8, 3, 4, 19
    K = rng.standard_normal((T, d))
    C = rng.standard_normal((T, r))
    q = rng.standard_normal(d)
    sel = np.array([0, 2, 4])
    out, w, tok = o.sparse_attention(q, K, C, sel, ps)
    want_tok = np.array([0, 1, 2, 3, 8, 9, 10, 11, 16, 17, 18])
    np.testing.assert_array_equal(tok, want_tok)
    np.testing.assert_allclose(out, _sdpa(q, K[want_tok], C[want_tok]), atol=1e-12)
    assert abs(w.sum() - 1.0) < 1e-12


def test_attention_dense_reduction():
    check_attention_dense_reduction(ORACLE)


def test_attention_subset():
    check_attention_subset(ORACLE)


# ---------------------------------------------------------------------------
# step 5 and the whole step
# ---------------------------------------------------------------------------
def check_out_projection_associativity(o):
    """sum_h o_h (B_g W_O,h) == sum_h (o_h B_g) W_O,h (the fusion does not change y)."""
    rng = np.random.default_rng(9)
    Hq, Hkv, d, r, hid = 6, 2, 8, 3, 10
    Bf = rng.standard_normal((Hkv, r, d))
    W_O = rng.standard_normal((Hq * d, hid))
    o_lat = rng.standard_normal((Hq, r))
    G = o.fuse_out_factor(Bf, W_O, Hq, "f64")
    y = o.out_projection(o_lat, G)
    want = np.zeros(hid)
    for h in range(Hq):
        want += (o_lat[h] @ Bf[h // (Hq // Hkv)]) @ W_O[h * d:(h + 1) * d]
    np.testing.assert_allclose(y, want, atol=1e-12)
    # concatenated-heads form of the textbook out-projection
    v_hat = np.concatenate([o_lat[h] @ Bf[h // (Hq // Hkv)] for h in range(Hq)])
    np.testing.assert_allclose(y, v_hat @ W_O, atol=1e-12)


def test_out_projection_associativity():
    check_out_projection_associativity(ORACLE)


def _tiny_sequence(rng, T, Hkv, d):
    K = rng.standard_normal((T, Hkv, d))
    V = rng.standard_normal((T, Hkv, d))
    return K, V


def check_decode_dense_special_case(o):
    """k >= n-2, r = d, A = B = P = I, E = I: the decode step is dense GQA attention then W_O."""
    rng = np.random.default_rng(10)
    Hq, Hkv, d, ps, T, hid = 4, 2, 8, 4, 22, 6
    K, V = _tiny_sequence(rng, T, Hkv, d)
    q = rng.standard_normal((Hq, d))
    eye = np.stack([np.eye(d)] * Hkv)
    W_O = rng.standard_normal((Hq * d, hid))
    G = o.fuse_out_factor(eye, W_O, Hq, "f64")
    cache = o.prefill(K[:-1], V[:-1], eye, eye, eye, ps, "f64", capacity=T)
    out = o.decode_step(cache, K[-1], V[-1], q, eye, eye, eye, G, top_k=100)
    heads = []
    for h in range(Hq):
        g = h // (Hq // Hkv)
        heads.append(_sdpa(q[h], K[:, g], V[:, g]))
        np.testing.assert_allclose(out["o_lat"][h], heads[-1], atol=1e-12)
    np.testing.assert_allclose(out["y"], np.concatenate(heads) @ W_O, atol=1e-11)
    np.testing.assert_allclose(out["weight_sums"], 1.0, atol=1e-12)


def check_decode_all_pages_real_factors(o):
    """All pages selected, real low-rank factors: y = sum_h softmax(q K^T/sqrt d)(C B) W_O,h."""
    rng = np.random.default_rng(12)
    Hq, Hkv, d, r, s, ps, T, hid = 4, 2, 16, 5, 3, 8, 37, 7
    K, V = _tiny_sequence(rng, T, Hkv, d)
    q = rng.standard_normal((Hq, d))
    A = np.stack([_rand_orth(rng, d, r) for _ in range(Hkv)])
    Bf = A.transpose(0, 2, 1).copy()
    P = rng.standard_normal((Hkv, r, d))
    E = np.stack([_rand_orth(rng, d, s) for _ in range(Hkv)])
    W_O = rng.standard_normal((Hq * d, hid))
    G = o.fuse_out_factor(Bf, W_O, Hq, "f64")
    cache = o.prefill(K[:-1], V[:-1], A, P, E, ps, "f64", capacity=T)
    out = o.decode_step(cache, K[-1], V[-1], q, A, P, E, G, top_k=1000)
    y = np.zeros(hid)
    for h in range(Hq):
        g = h // (Hq // Hkv)
        v_hat = (V[:, g] @ A[g]) @ Bf[g]
        y += _sdpa(q[h], K[:, g], v_hat) @ W_O[h * d:(h + 1) * d]
    np.testing.assert_allclose(out["y"], y, atol=1e-11)


def check_new_token_is_attended(o):
    """The appended token is in the recent page and is attended in the same step."""
    rng = np.random.default_rng(13)
    Hq, Hkv, d, ps, T = 2, 1, 8, 4, 41
    K, V = _tiny_sequence(rng, T, Hkv, d)
    q = rng.standard_normal((Hq, d))
    K[-1, 0] = 40.0 * q[0] / np.linalg.norm(q[0])       # dominant key for head 0
    eye = np.eye(d)[None]
    G = o.fuse_out_factor(eye, np.eye(Hq * d), Hq, "f64")
    cache = o.prefill(K[:-1], V[:-1], eye, eye, eye, ps, "f64", capacity=T)
    out = o.decode_step(cache, K[-1], V[-1], q, eye, eye, eye, G, top_k=2)
    assert cache.length == T and out["sel"][0][-1] == o.num_pages(T, ps) - 1
    np.testing.assert_allclose(out["o_lat"][0], V[-1, 0], atol=1e-6)


def check_decode_group_routing(o):
    """Group routing in a decode step: with every page selected it is dense GQA
    attention; with few pages every head of a group attends, by textbook
    softmax, over the tokens of the pages its group's summed or max score
    keeps (computed here from the summed query and an elementwise maximum)."""
    rng = np.random.default_rng(15)
    Hq, Hkv, d, ps, T, hid = 4, 2, 8, 4, 41, 5
    G_ = Hq // Hkv
    K, V = _tiny_sequence(rng, T, Hkv, d)
    q = rng.standard_normal((Hq, d))
    eye = np.stack([np.eye(d)] * Hkv)
    W_O = rng.standard_normal((Hq * d, hid))
    G = o.fuse_out_factor(eye, W_O, Hq, "f64")
    n = o.num_pages(T, ps)
    for routing in ("group_sum", "group_max"):
        cache = o.prefill(K[:-1], V[:-1], eye, eye, eye, ps, "f64", capacity=T)
        out = o.decode_step(cache, K[-1], V[-1], q, eye, eye, eye, G, top_k=100, routing=routing)
        heads = [_sdpa(q[h], K[:, h // G_], V[:, h // G_]) for h in range(Hq)]
        np.testing.assert_allclose(out["y"], np.concatenate(heads) @ W_O, atol=1e-11)
        cache = o.prefill(K[:-1], V[:-1], eye, eye, eye, ps, "f64", capacity=T)
        out = o.decode_step(cache, K[-1], V[-1], q, eye, eye, eye, G, top_k=3, routing=routing)
        for g in range(Hkv):
            Sg = cache.S[g, :n]  # the stored (fp32) summaries: with E = I, the mean key of each page
            mean_k = np.stack([K[p * ps:(p + 1) * ps, g].mean(axis=0) for p in range(n)])
            np.testing.assert_allclose(Sg, mean_k, rtol=1e-6, atol=1e-6)
            qg = q[g * G_:(g + 1) * G_]
            gs = Sg @ qg.sum(axis=0) if routing == "group_sum" else np.maximum.reduce(Sg @ qg.T, axis=1)
            np.testing.assert_allclose(out["scores"][g], gs, atol=1e-12)
            want = _sort_reference(gs, 3)
            for h in range(g * G_, (g + 1) * G_):
                np.testing.assert_array_equal(out["sel"][h], want)
                tok = np.concatenate([np.arange(p * ps, min(T, (p + 1) * ps)) for p in want])
                np.testing.assert_allclose(out["o_lat"][h], _sdpa(q[h], K[tok, g], V[tok, g]), atol=1e-12)


def check_golden(o):
    with open(GOLDEN) as f:
        gx = json.load(f)
    ex = gx["expect"]
    A = np.array(gx["A"])[None]
    P = np.array(gx["P"])[None]
    E = np.array(gx["E"])[None]
    Bf = np.array(gx["B"])[None]
    keys = np.array(gx["keys"], dtype=np.float64)[:, None, :]
    vals = np.array(gx["values"], dtype=np.float64)[:, None, :]
    q = np.array(gx["q"])[None]
    for storage in ["bf16", "f32", "f64"]:
        G = o.fuse_out_factor(Bf, np.array(gx["W_O"]), 1, storage)
        np.testing.assert_array_equal(G[0], ex["G"])
        cache = o.prefill(keys[:-1], vals[:-1], A, P, E, gx["page_size"], storage, capacity=7)
        out = o.decode_step(cache, keys[-1], vals[-1], q, A, P, E, G, gx["top_k"])
        np.testing.assert_array_equal(cache.C[0, :7, 0], ex["C"])
        np.testing.assert_array_equal(cache.R[0, :7, 0], ex["R"])
        np.testing.assert_array_equal(cache.S[0, :4], ex["S"])
        np.testing.assert_array_equal(out["scores"][0], ex["scores"])
        np.testing.assert_array_equal(out["sel"][0], ex["sel"])
        s = math.sqrt(2.0)
        num = [math.exp(x / s) for x in ex["logit_numerators"]]
        cvals = [ex["C"][t] for t in ex["attended_tokens"]]
        o_want = sum(a * b for a, b in zip(num, cvals)) / sum(num)
        np.testing.assert_allclose(out["o_lat"][0, 0], o_want, rtol=1e-14)
        np.testing.assert_allclose(out["y"], [o_want, 2 * o_want], rtol=1e-14)


def test_decode_dense_special_case():
    check_decode_dense_special_case(ORACLE)


def test_decode_all_pages_real_factors():
    check_decode_all_pages_real_factors(ORACLE)


def test_new_token_is_attended():
    check_new_token_is_attended(ORACLE)


def test_decode_group_routing():
    check_decode_group_routing(ORACLE)


def test_golden_worked_example():
    check_golden(ORACLE)


def check_incremental_equals_batch(o):
    """Appending token by token gives the same cache as one batched append."""
    rng = np.random.default_rng(14)
    Hkv, d, r, s, ps, T = 2, 8, 3, 2, 4, 11
    K, V = _tiny_sequence(rng, T, Hkv, d)
    A = np.stack([_rand_orth(rng, d, r) for _ in range(Hkv)])
    P = rng.standard_normal((Hkv, r, d))
    E = np.stack([_rand_orth(rng, d, s) for _ in range(Hkv)])
    c1 = o.prefill(K, V, A, P, E, ps, "bf16")
    c2 = o.SequenceCache(Hkv, d, r, s, ps, T, "bf16")
    for t in range(T):
        c2.append(K[t:t + 1], V[t:t + 1], A, P, E)
    np.testing.assert_array_equal(c1.C, c2.C)
    np.testing.assert_array_equal(c1.R, c2.R)
    np.testing.assert_array_equal(c1.S, c2.S)


def test_incremental_equals_batch():
    check_incremental_equals_batch(ORACLE)


# ---------------------------------------------------------------------------
# calibration: Value factors against the complete attention output
# ---------------------------------------------------------------------------
def check_fit_eckart_young(o):
    """One head, W_O = I: the best rank-r factors give the Eckart-Young error
    (sum of the squared singular values past r), from the start and after sweeps."""
    rng = np.random.default_rng(21)
    N, d, r = 60, 7, 3
    Z = rng.standard_normal((1, N, d)) * np.array([5.0, 3, 2, 1.5, 1, 0.5, 0.2])
    sv = np.linalg.svd(Z[0], compute_uv=False)
    ey = float(np.sum(sv[r:] ** 2))
    for objective in ("joint", "isolated"):
        A, B, hist = o.fit_value_factors(Z, np.eye(d), 1, [[0]], r, 0, objective)
        assert abs(hist[0] - ey) <= 1e-9 * ey
        A, B, hist = o.fit_value_factors(Z, np.eye(d), 1, [[0]], r, 4, objective)
        assert np.all(np.abs(hist - ey) <= 1e-8 * ey)
        assert abs(o.output_error(Z, np.eye(d), A, B) - ey) <= 1e-8 * ey


def check_fit_exact_low_rank(o):
    """Each group's attention outputs lie in an r-dimensional subspace: the
    factors reproduce the complete output exactly under both objectives."""
    rng = np.random.default_rng(22)
    Hq, Hkv, N, d, r, hid = 4, 2, 50, 6, 2, 9
    basis = [np.linalg.qr(rng.standard_normal((d, r)))[0] for _ in range(Hkv)]
    Z = np.stack([rng.standard_normal((N, r)) @ basis[h // 2].T for h in range(Hq)])
    W_O = rng.standard_normal((Hq * d, hid))
    scale = o.output_error(Z, W_O, np.zeros((Hkv, d, r)), np.zeros((Hkv, r, d)))
    for objective in ("joint", "isolated"):
        A, B, hist = o.fit_value_factors(Z, W_O, Hkv, [[0], [1]], r, 2, objective)
        assert hist[-1] <= 1e-20 * scale


def check_fit_least_squares_steps(o):
    """One term: the B and A updates equal the two-sided least-squares closed forms."""
    rng = np.random.default_rng(23)
    N, r, d, hid = 30, 3, 5, 8
    U = rng.standard_normal((N, r))
    W = rng.standard_normal((d, hid))
    t = rng.standard_normal((N, hid))
    want_B = np.linalg.solve(U.T @ U, U.T @ t @ W.T) @ np.linalg.inv(W @ W.T)
    np.testing.assert_allclose(o._lstsq_B([U], [W], t), want_B, atol=1e-10)
    Zs = rng.standard_normal((N, d))
    M = rng.standard_normal((r, hid))
    want_A = np.linalg.solve(Zs.T @ Zs, Zs.T @ t @ M.T) @ np.linalg.inv(M @ M.T)
    np.testing.assert_allclose(o._lstsq_A([Zs], [M], t), want_A, atol=1e-10)


def check_fit_sweeps(o):
    """Joint sweeps never increase the complete-output error (each update is an
    exact minimisation of it); with one partition the two objectives coincide."""
    rng = np.random.default_rng(24)
    Hq, Hkv, N, d, r, hid = 6, 3, 40, 5, 2, 8
    Z = rng.standard_normal((Hq, N, d))
    W_O = rng.standard_normal((Hq * d, hid))
    _, _, hist = o.fit_value_factors(Z, W_O, Hkv, [[0], [1], [2]], r, 6, "joint")
    assert np.all(np.diff(hist) <= 1e-9 * hist[0])
    assert hist[-1] < 0.9 * hist[0]
    _, _, h1 = o.fit_value_factors(Z, W_O, Hkv, [[0, 1, 2]], r, 3, "isolated")
    _, _, h2 = o.fit_value_factors(Z, W_O, Hkv, [[0, 1, 2]], r, 3, "joint")
    np.testing.assert_allclose(h1, h2, rtol=1e-12)


def test_fit_eckart_young():
    check_fit_eckart_young(ORACLE)


def test_fit_exact_low_rank():
    check_fit_exact_low_rank(ORACLE)


def test_fit_least_squares_steps():
    check_fit_least_squares_steps(ORACLE)


def test_fit_sweeps():
    check_fit_sweeps(ORACLE)


ALL_CHECKS = [
    check_bf16_rounding, check_append_identity, check_append_projection,
    check_summary_closed_form, check_summary_low_rank_residual,
    check_route_full_sort, check_route_ties, check_route_bruteforce, check_route_small_n,
    check_route_group_worked_example, check_route_group_reductions, check_decode_group_routing,
    check_attention_dense_reduction, check_attention_subset,
    check_out_projection_associativity, check_decode_dense_special_case,
    check_decode_all_pages_real_factors, check_new_token_is_attended, check_golden,
    check_incremental_equals_batch,
    check_fit_eckart_young, check_fit_exact_low_rank, check_fit_least_squares_steps, check_fit_sweeps,
]
