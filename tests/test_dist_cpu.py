"""Multi-process host logic of bench.py on CPU (gloo, world size 2).

The decode path has no exchange step: N GPUs run N independent replicas
(weak scaling), each on its own sequences, and the step time reported is the
maximum over ranks.  These tests run that plumbing as two gloo ranks on
127.0.0.1: rendezvous from the torchrun environment variables, the
max-over-ranks reduction, the barrier, distinct replica workloads per rank,
and the reference arm printing only on rank 0.
"""
import contextlib
import io
import json
import os
import socket

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

import bench
from long_context_decode_basiskv_b200.workloads import WORKLOADS, make_case, shrink

WORLD = 2


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, outdir):
    os.environ.update({"RANK": str(rank), "WORLD_SIZE": str(world), "LOCAL_RANK": str(rank),
                       "MASTER_ADDR": "127.0.0.1", "MASTER_PORT": str(port)})
    w, r, local = bench.dist_env()
    bench.init_dist(w, "gloo")
    try:
        res = {"env": [w, r, local]}
        res["max"] = bench.max_over_ranks(1.5 + 10.0 * r, w, "cpu")
        bench.barrier(w)
        wl = bench.replica_workload(shrink(WORKLOADS["tiny_fp32"], batch=2, context=40, name="dist"), r, w)
        case = make_case(wl, "cpu")
        res["seed"] = wl.seed
        res["q_sum"] = float(case.q.double().sum())
        res["k0"] = case.keys[0][:4, 0, 0].double().tolist()
        # the reference arm runs on rank 0 only; other ranks print nothing
        if r != 0:
            buf = io.StringIO()
            with contextlib.redirect_stdout(buf):
                bench.run_reference(type("A", (), {"workload": "tiny_fp32", "warmup": 0, "steps": 1, "routing": "head"})(), w, r)
            res["ref_out"] = buf.getvalue()
        bench.barrier(w)
    finally:
        torch.distributed.destroy_process_group()
    with open(os.path.join(outdir, f"{rank}.json"), "w") as f:
        json.dump(res, f)


@pytest.fixture(scope="module")
def results(tmp_path_factory):
    out = tmp_path_factory.mktemp("dist")
    mp.spawn(_worker, args=(WORLD, _free_port(), str(out)), nprocs=WORLD, join=True)
    return [json.load(open(out / f"{r}.json")) for r in range(WORLD)]


def test_env_and_rendezvous(results):
    for r, res in enumerate(results):
        assert res["env"] == [WORLD, r, r]


def test_max_over_ranks(results):
    for res in results:
        assert res["max"] == 11.5


def test_replicas_differ(results):
    assert results[0]["seed"] != results[1]["seed"]
    assert results[0]["q_sum"] != results[1]["q_sum"]
    assert not np.allclose(results[0]["k0"], results[1]["k0"])


def test_reference_arm_silent_off_rank0(results):
    assert results[1]["ref_out"] == ""


def test_single_rank_is_identity():
    assert bench.max_over_ranks(3.25, 1, "cpu") == 3.25
    wl = WORKLOADS["llama3_8b_32k"]
    assert bench.replica_workload(wl, 0, 1) is wl
