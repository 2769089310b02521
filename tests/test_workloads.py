"""The seeded generator (CPU): determinism, shapes, factor-fit sanity, hot pages."""
import numpy as np
import torch

from long_context_decode_basiskv_b200.workloads import WORKLOADS, make_case, shrink


def test_tiny_case_shapes_and_determinism():
    wl = WORKLOADS["tiny_fp32"]
    a = make_case(wl)
    b = make_case(wl)
    assert a.lengths == [2048] and a.pages(0) == 64 and a.max_pages == 64
    assert a.q.shape == (1, 8, 64) and a.q.dtype == torch.float32
    assert a.keys[0].shape == (2048, 2, 64)
    assert a.A.shape == (2, 64, 16) and a.P.shape == (2, 16, 64) and a.E.shape == (2, 64, 8)
    assert a.W_O.shape == (8 * 64, 512)
    for x, y in [(a.q, b.q), (a.keys[0], b.keys[0]), (a.values[0], b.values[0]),
                 (a.A, b.A), (a.P, b.P), (a.E, b.E), (a.W_O, b.W_O), (a.block_table, b.block_table)]:
        assert torch.equal(x, y)
    # block table: a permutation of the physical pool
    bt = a.block_table.numpy()
    assert sorted(bt[0].tolist()) == list(range(64))


def test_factor_fit_is_a_good_basis():
    wl = WORKLOADS["tiny_fp32"]
    c = make_case(wl)
    for g in range(wl.num_kv_heads):
        A = c.A[g].double().numpy()
        np.testing.assert_allclose(A.T @ A, np.eye(wl.rank_v), atol=1e-5)
        V = c.values[0][:, g].double().numpy()
        rel = np.linalg.norm(V - V @ A @ A.T) / np.linalg.norm(V)
        assert rel < 0.1            # V is rank r plus 5% noise
        E = c.E[g].double().numpy()
        np.testing.assert_allclose(E.T @ E, np.eye(wl.rank_k), atol=1e-5)


def test_ragged_lengths_and_bf16_storage():
    wl = shrink(WORKLOADS["ragged_serving"], batch=5, ragged=(17, 90), name="ragged_tiny")
    c = make_case(wl)
    assert len(c.lengths) == 5 and all(17 <= L <= 90 for L in c.lengths)
    assert c.keys[0].dtype == torch.bfloat16 and c.A.dtype == torch.bfloat16
    npg = [-(-L // 16) for L in c.lengths]
    bt = c.block_table.numpy()
    used = np.concatenate([bt[b, :npg[b]] for b in range(5)])
    assert sorted(used.tolist()) == list(range(sum(npg)))
    for b in range(5):
        assert np.all(bt[b, npg[b]:] == -1)


def test_hot_pages_carry_the_requested_mass():
    wl = shrink(WORKLOADS["single_seq_131k"], context=64 * 200, name="hot_small")
    c = make_case(wl)
    assert len(c.hot_pages) == 10
    assert c.hot_pages.min() >= 1 and c.hot_pages.max() <= 198
    assert abs(c.hot_mass - 0.80) < 0.01 and c.hot_alpha > 0
