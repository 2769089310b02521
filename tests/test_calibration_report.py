"""The calibration quality report (tests/calibration_report.py) at a small size:
its figures are well formed and the fits beat nothing they should not."""
import math

from tests.calibration_report import measure


def test_report_is_well_formed():
    rep = measure(0.5, rank=4, n_calib=256, n_test=128, sweeps=2, splits=(2, 4),
                  Hq=8, Hkv=4, d=16, data_rank=8, T=256, hidden=64)
    assert 0.0 < rep["pca_of_values"] < 1.5
    for n in (2, 4):
        row = rep[f"tp{n}"]
        for k in ("isolated", "joint", "svd_of_outputs"):
            assert math.isfinite(row[k]) and 0.0 < row[k] < 1.5


def test_full_rank_fit_is_exact():
    rep = measure(0.0, rank=16, n_calib=128, n_test=64, sweeps=1, splits=(2,),
                  Hq=4, Hkv=2, d=16, data_rank=4, T=64, hidden=32)
    assert rep["tp2"]["joint"] < 1e-5 and rep["tp2"]["isolated"] < 1e-5
