"""Edge cases on the GPU: tiny and degenerate sequences, empty batches, and the
device error flags (planted on the host; every kernel checks before it reads,
so none of these faults the GPU)."""
import numpy as np
import pytest
import torch

from tests.harness import OracleCase, assert_close, selection_ok, storage_of

pytestmark = pytest.mark.gpu

from long_context_decode_basiskv_b200 import binding as bk  # noqa: E402
from long_context_decode_basiskv_b200.engine import DecodeEngine  # noqa: E402
from long_context_decode_basiskv_b200.workloads import WORKLOADS, make_case, shrink  # noqa: E402


@pytest.mark.parametrize("top_k,ragged,base", [
    (1, (1, 70), "ragged_serving"),       # n from 1 to 5 pages: n <= k+2 and n > k+2
    (2, (1, 70), "ragged_serving"),
    (3, (15, 130), "tiny_fp32"),          # pages of 32, fp32
    (1, (63, 200), "single_seq_131k"),    # pages of 64
])
def test_short_and_partial_sequences(top_k, ragged, base):
    wl = shrink(WORKLOADS[base], batch=12, ragged=ragged, top_k=top_k, name=f"edge_{base}_{top_k}")
    if wl.hot_fraction:
        wl = shrink(wl, name=wl.name)
        import dataclasses
        wl = dataclasses.replace(wl, hot_fraction=0.0, hot_mass=0.0)
    case = make_case(wl, "cuda")
    eng = DecodeEngine(case)
    eng.step()
    torch.cuda.synchronize()
    assert int(eng.err.item()) == 0
    oc = OracleCase(case)
    sel, cnt = eng.sel.cpu().numpy(), eng.sel_cnt.cpu().numpy()
    o_lat, y = eng.o_lat.cpu().numpy(), eng.y.cpu().numpy()
    for b in range(wl.batch):
        _, out = oc.sequence(b)
        for h in range(wl.num_q_heads):
            ok, _ = selection_ok(sel[b, h], cnt[b, h], out["sel"][h], out["scores"][h])
            assert ok
        assert_close(o_lat[b], out["o_lat"], storage_of(wl), f"o_lat b={b} L={case.lengths[b]}")
        assert_close(y[b], out["y"], storage_of(wl), f"y b={b}")


def _engine():
    wl = shrink(WORKLOADS["llama3_8b_32k"], batch=2, context=3000, top_k=16, name="flags")
    return DecodeEngine(make_case(wl, "cuda"))


def test_block_table_out_of_range_sets_flag():
    eng = _engine()
    eng.step()
    torch.cuda.synchronize()
    assert int(eng.err.item()) == 0
    eng.cache.block_table[1, 0] = eng.cache.num_phys_pages + 7      # sink page of sequence 1
    eng.route()
    eng.decode_attn()
    torch.cuda.synchronize()
    assert int(eng.err.item()) & bk.DEVERR_BLOCK_TABLE
    # sequence 0 is untouched and still correct
    assert torch.isfinite(eng.o_lat[0]).all()


def test_selection_out_of_range_sets_flag():
    eng = _engine()
    eng.step()
    torch.cuda.synchronize()
    sel = eng.sel.clone()
    sel[0, 3, 1] = 100000
    eng.err.zero_()
    o = torch.empty_like(eng.o_lat)
    bk.decode_attn(eng.cfg, eng.cache, eng.q, sel, eng.sel_cnt, o, eng.ws, eng.err)
    torch.cuda.synchronize()
    assert int(eng.err.item()) & bk.DEVERR_SELECTION


def test_seq_len_too_long_sets_flag():
    eng = _engine()
    eng.step()
    torch.cuda.synchronize()
    eng.cache.seq_len[0] = eng.cache.max_pages * eng.cfg.page_size + 5
    eng.err.zero_()
    eng.append()
    eng.route()
    torch.cuda.synchronize()
    assert int(eng.err.item()) & bk.DEVERR_SEQ_LEN


def test_empty_batch_through_binding():
    eng = _engine()
    cfg = eng.cfg
    q0 = torch.empty((0, cfg.num_q_heads, cfg.head_dim), dtype=cfg.dtype, device="cuda")
    sel0 = torch.empty((0, cfg.num_q_heads, cfg.top_k + 2), dtype=torch.int32, device="cuda")
    cnt0 = torch.empty((0, cfg.num_q_heads), dtype=torch.int32, device="cuda")
    o0 = torch.empty((0, cfg.num_q_heads, cfg.rank_v), dtype=torch.float32, device="cuda")
    y0 = torch.empty((0, cfg.hidden), dtype=torch.float32, device="cuda")
    bk.route(cfg, eng.cache, q0, sel0, cnt0, eng.ws, eng.err)
    bk.decode_attn(cfg, eng.cache, q0, sel0, cnt0, o0, eng.ws, eng.err)
    bk.out_proj(cfg, eng.factors, o0, y0, eng.ws)
    torch.cuda.synchronize()
    assert int(eng.err.item()) == 0


def test_workspace_too_small_is_rejected():
    eng = _engine()
    small = torch.empty(64, dtype=torch.uint8, device="cuda")
    with pytest.raises(bk.BasisKVError) as ei:
        bk.route(eng.cfg, eng.cache, eng.q, eng.sel, eng.sel_cnt, small, eng.err)
    assert ei.value.status == bk.ERR_WORKSPACE


def test_graph_step_matches_step():
    """The engine's CUDA-graph step gives exactly the eager step's outputs, also when replayed."""
    wl = shrink(WORKLOADS["llama3_8b_32k"], batch=3, context=16 * 300 + 7, top_k=24, name="graph_step")
    eng = DecodeEngine(make_case(wl, "cuda"))
    eng.step()
    torch.cuda.synchronize()
    ref = (eng.sel.clone(), eng.o_lat.clone(), eng.y.clone())
    for _ in range(2):
        eng.y.zero_()
        eng.o_lat.zero_()
        eng.graph_step()
        torch.cuda.synchronize()
        assert int(eng.err.item()) == 0
        assert torch.equal(eng.sel, ref[0])
        assert torch.equal(eng.o_lat, ref[1])
        assert torch.equal(eng.y, ref[2])
