"""Head-sharded (tensor-parallel) decomposition on CPU: slicing a case by KV
groups, and the sum of the ranks' partial outputs equal to the full step's
output (oracle, fp64), directly and through a gloo all-reduce of world size 2."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

from oracle import basiskv_oracle as O
from long_context_decode_basiskv_b200.tensor_parallel import head_range, reduce_y, shard_case
from long_context_decode_basiskv_b200.workloads import WORKLOADS, make_case, shrink


def _f64(t):
    return t.detach().to("cpu").to(torch.float64).numpy()


def _oracle_y(case):
    """The oracle's decode-step output y of every sequence of `case` ([B, hidden])."""
    wl = case.wl
    storage = "f32" if wl.dtype == "f32" else "bf16"
    A, P, E = _f64(case.A), _f64(case.P), _f64(case.E)
    G = O.fuse_out_factor(_f64(case.Bf), _f64(case.W_O), wl.num_q_heads, storage)
    ys = []
    for b in range(wl.batch):
        K, V = _f64(case.keys[b]), _f64(case.values[b])
        L = K.shape[0]
        cache = O.prefill(K[:-1], V[:-1], A, P, E, wl.page_size, storage, capacity=L)
        out = O.decode_step(cache, K[-1], V[-1], _f64(case.q[b]), A, P, E, G, wl.top_k)
        ys.append(out["y"])
    return np.stack(ys)


def test_head_range():
    assert [head_range(8, r, 4) for r in range(4)] == [(0, 2), (2, 4), (4, 6), (6, 8)]
    with pytest.raises(ValueError):
        head_range(8, 0, 3)


def test_shard_slices():
    wl = shrink(WORKLOADS["llama3_8b_32k"], batch=2, context=300, name="tp_slices")
    case = make_case(wl, "cpu")
    for world in (2, 4, 8):
        for rank in range(world):
            s = shard_case(case, rank, world)
            g0, g1 = head_range(8, rank, world)
            assert s.wl.num_kv_heads == g1 - g0 and s.wl.num_q_heads == 4 * (g1 - g0)
            assert torch.equal(s.q, case.q[:, 4 * g0:4 * g1])
            assert torch.equal(s.keys[1], case.keys[1][:, g0:g1])
            assert torch.equal(s.A, case.A[g0:g1]) and torch.equal(s.E, case.E[g0:g1])
            assert torch.equal(s.W_O, case.W_O[4 * g0 * 128:4 * g1 * 128])
            assert torch.equal(s.block_table, case.block_table)


@pytest.mark.parametrize("name,world", [("tiny_fp32", 2), ("l8b", 4)])
def test_partial_outputs_sum_to_the_full_step(name, world):
    wl = WORKLOADS["tiny_fp32"] if name == "tiny_fp32" else \
        shrink(WORKLOADS["llama3_8b_32k"], batch=1, context=700, top_k=8, name="tp_l8b")
    case = make_case(wl, "cpu")
    full = _oracle_y(case)
    part = sum(_oracle_y(shard_case(case, r, world)) for r in range(world))
    np.testing.assert_allclose(part, full, rtol=0, atol=1e-10 * np.abs(full).max())


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    os.environ.update({"MASTER_ADDR": "127.0.0.1", "MASTER_PORT": str(port)})
    torch.distributed.init_process_group("gloo", rank=rank, world_size=world)
    try:
        case = make_case(WORKLOADS["tiny_fp32"], "cpu")
        y = torch.from_numpy(_oracle_y(shard_case(case, rank, world)))
        reduce_y(y, world)
        torch.save(y, os.path.join(out, f"{rank}.pt"))
    finally:
        torch.distributed.destroy_process_group()


def test_gloo_all_reduce_of_partials(tmp_path):
    world = 2
    mp.spawn(_worker, args=(world, _free_port(), str(tmp_path)), nprocs=world, join=True)
    full = _oracle_y(make_case(WORKLOADS["tiny_fp32"], "cpu"))
    for r in range(world):
        y = torch.load(tmp_path / f"{r}.pt").numpy()
        np.testing.assert_allclose(y, full, rtol=0, atol=1e-10 * np.abs(full).max())


def test_engine_rejects_unknown_modes():
    """Engine options are checked before any device work."""
    from long_context_decode_basiskv_b200.engine import DecodeEngine

    case = make_case(WORKLOADS["tiny_fp32"], "cpu")
    with pytest.raises(ValueError):
        DecodeEngine(case, device="cpu", routing="per_page")
    with pytest.raises(ValueError):
        DecodeEngine(case, device="cpu", prefill_mode="fast")
