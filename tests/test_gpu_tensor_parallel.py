"""Head-sharded tensor parallelism (the pages' deployment setting) on one GPU.

Rank i of N computes the whole decode path for its slice of the KV groups
(shard_case) with the single-GPU calls and produces a partial output y_i; the
layer output is the sum of the partials (reduce_y adds them with one
all-reduce).  Here the N shard engines run one after another on cuda:0 and
their partials are summed on the host, which is what the all-reduce computes,
and compared with the unsharded fp64 oracle: selections head by head under
the near-tie rule, o_lat and the summed y at the bf16 tolerances."""
import numpy as np
import pytest
import torch

from tests.harness import OracleCase, assert_close, oracle_on_selection, selection_ok, storage_of

pytestmark = pytest.mark.gpu

from long_context_decode_basiskv_b200.engine import DecodeEngine  # noqa: E402
from long_context_decode_basiskv_b200.tensor_parallel import head_range, shard_case  # noqa: E402
from long_context_decode_basiskv_b200.workloads import WORKLOADS, make_case, shrink  # noqa: E402


@pytest.fixture(scope="module")
def full_case():
    wl = shrink(WORKLOADS["llama3_8b_32k"], batch=3, context=16 * 700 + 9, top_k=48, name="tp_gpu")
    case = make_case(wl, "cuda")
    oc = OracleCase(case)
    return case, oc, [oc.sequence(b) for b in range(wl.batch)]


@pytest.mark.parametrize("world", [2, 4, 8])
def test_sharded_steps_sum_to_the_unsharded_oracle(full_case, world):
    case, oc, ref = full_case
    wl = case.wl
    B, Hq, G = wl.batch, wl.num_q_heads, wl.num_q_heads // wl.num_kv_heads
    sel = np.full((B, Hq, wl.top_k + 2), -1, dtype=np.int64)
    cnt = np.zeros((B, Hq), dtype=np.int64)
    o_lat = np.zeros((B, Hq, wl.rank_v))
    y = np.zeros((B, wl.hidden))
    for r in range(world):
        eng = DecodeEngine(shard_case(case, r, world))
        eng.step()
        torch.cuda.synchronize()
        assert int(eng.err.item()) == 0, f"rank {r}"
        g0, g1 = head_range(wl.num_kv_heads, r, world)
        h0, h1 = g0 * G, g1 * G
        sel[:, h0:h1] = eng.sel.cpu().numpy()
        cnt[:, h0:h1] = eng.sel_cnt.cpu().numpy()
        o_lat[:, h0:h1] = eng.o_lat.cpu().numpy()
        y += eng.y.to(torch.float64).cpu().numpy()     # what the all-reduce of the partials sums
        del eng
    for b, (cache, out) in enumerate(ref):
        for h in range(Hq):
            assert selection_ok(sel[b, h], cnt[b, h], out["sel"][h], out["scores"][h])[0], f"b={b} h={h}"
        o_want, y_want = oracle_on_selection(oc, b, cache, out, sel[b], cnt[b])
        assert_close(o_lat[b], o_want, storage_of(wl), f"tp{world} o_lat b={b}")
        assert_close(y[b], y_want, storage_of(wl), f"tp{world} summed y b={b}")
