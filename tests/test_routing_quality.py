"""The routing-quality report (tests/routing_quality.py) on a tiny workload:
its figures are well formed, and selecting every page has no routing error."""
from long_context_decode_basiskv_b200.workloads import WORKLOADS, shrink
from tests.routing_quality import ROUTINGS, measure


def test_report_is_well_formed():
    wl = shrink(WORKLOADS["tiny_fp32"], context=700, name="rq_tiny")
    rep = measure(wl, 1)
    n = -(-wl.context // wl.page_size)
    for r in ROUTINGS:
        row = rep[r]
        assert 0.0 < row["mass_on_selected"] <= 1.0
        assert row["y_rel_vs_all_pages"] >= 0.0
        assert wl.top_k + 2 <= row["pages_per_group"] <= min(n, wl.group * wl.top_k + 2)
        if r != "head":
            assert row["pages_per_group"] == wl.top_k + 2
    assert rep["all_pages_y_rel_vs_dense"] < 0.05


def test_every_page_selected_has_no_routing_error():
    wl = shrink(WORKLOADS["tiny_fp32"], context=300, top_k=64, name="rq_all")
    rep = measure(wl, 1)
    for r in ROUTINGS:
        assert rep[r]["y_rel_vs_all_pages"] < 1e-12
        assert abs(rep[r]["mass_on_selected"] - 1.0) < 1e-9
