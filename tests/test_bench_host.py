"""bench.py host logic on CPU: algorithmic bytes from a step's selection (per head
and per group), the measured-peak fallback, and the rule that committed DRAM
traffic is reported only while the profiled kernel source is unchanged."""
import hashlib
import json
import os
import types

import torch

import bench
from long_context_decode_basiskv_b200.workloads import WORKLOADS, shrink


def _fake_engine(routing):
    wl = shrink(WORKLOADS["llama3_8b_32k"], batch=1, context=16 * 10, top_k=2, name="bytes")
    B, Hq, k = 1, wl.num_q_heads, wl.top_k
    sel = torch.full((B, Hq, k + 2), -1, dtype=torch.int32)
    cnt = torch.full((B, Hq), k + 2, dtype=torch.int32)
    for h in range(Hq):  # head h of group g keeps pages {0, 9, 1 + (h % 4), 5 + g % 3}
        g = h // 4
        sel[0, h, :4] = torch.tensor(sorted({0, 9, 1 + h % 4, 5 + g % 3}), dtype=torch.int32)
        cnt[0, h] = len({0, 9, 1 + h % 4, 5 + g % 3})
    case = types.SimpleNamespace(wl=wl, lengths=[160])
    return types.SimpleNamespace(case=case, cfg=None, sel=sel, sel_cnt=cnt, routing=routing), wl


def test_algorithmic_bytes_counts_the_union_per_group():
    eng, wl = _fake_engine("head")
    nb = bench.algorithmic_bytes(eng)
    # every group: pages 0, 9, 1..4 and its 5 + g % 3 (which is outside 1..4) -> 7 pages
    assert nb["union_pages"] == 8 * 7
    P, d, r = wl.page_size, wl.head_dim, wl.rank_v
    q_bytes = wl.num_q_heads * d * 2
    sel_bytes = wl.num_q_heads * (wl.top_k + 2) * 4
    assert nb["decode_attn"] == 56 * P * (d + r) * 2 + q_bytes + sel_bytes + wl.num_q_heads * r * 4
    pages = 10
    assert nb["route"] == pages * 8 * d * 4 + 2 * pages * wl.num_q_heads * 4 + q_bytes + sel_bytes


def test_group_routing_writes_one_score_row_per_group():
    head, _ = _fake_engine("head")
    group, wl = _fake_engine("group_sum")
    diff = bench.algorithmic_bytes(head)["route"] - bench.algorithmic_bytes(group)["route"]
    assert diff == 2 * 10 * (wl.num_q_heads - wl.num_kv_heads) * 4


def test_measured_peak_fallback(tmp_path, monkeypatch):
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    assert bench.measured_peak() == (bench.FALLBACK_HBM_GBS, "fallback")
    (tmp_path / "MEASURED_PEAKS.json").write_text(json.dumps({"hbm_gbs": 6000.5}))
    assert bench.measured_peak() == (6000.5, "measured")


def test_profiled_traffic_only_for_the_profiled_source(tmp_path, monkeypatch):
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    src = tmp_path / "long_context_decode_basiskv_b200" / "csrc"
    src.mkdir(parents=True)
    (src / "k.cu").write_text("// kernel v1\\n")
    (tmp_path / "profiles").mkdir()
    sha = hashlib.sha256((src / "k.cu").read_bytes()).hexdigest()
    (tmp_path / "profiles" / "traffic.json").write_text(json.dumps({"source_sha256": sha,
                                                                    "dram_bytes_per_launch": 123}))
    assert bench.profiled_traffic("k.cu")["dram_bytes_per_launch"] == 123
    (src / "k.cu").write_text("// kernel v2\\n")
    assert bench.profiled_traffic("k.cu") is None
