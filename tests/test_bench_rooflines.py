"""The bench's stage rooflines on the host: each stage's algorithmic work for
the 4096 x 4096 layer with 262,144 calibration rows (4-bit, groups of 128),
checked against the closed forms, and the achieved rates as work over time."""
import os
import sys
from types import SimpleNamespace

import pytest

sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
import bench  # noqa: E402

D, N, B = 4096, 262144, 128


def _layer():
    return SimpleNamespace(d_out=D, d_in=D, n=N, bits=4, groupsize=128, blocksize=B)


def test_stage_work_matches_closed_forms():
    stages = {"hessian": 4.0, "prepare_hinv": 2.0, "quantize_layer": 1.0}    # ms
    r = bench.stage_rooflines(_layer(), stages, peak=1600.0, hbm=6500.0)
    # X^T X: the upper triangle with its diagonal, 2 flops per multiply-add
    assert r["hessian"]["achieved"] == pytest.approx(N * D * (D + 1) / 4e-3 / 1e12)
    assert N * D * (D + 1) == pytest.approx(4.40e12, rel=1e-3)
    # Cholesky and triangular inverse, d^3 / 3 flops each
    assert r["prepare_hinv"]["achieved"] == pytest.approx(2 * D ** 3 / 3 / 2e-3 / 1e12)
    assert r["prepare_hinv"]["issued_tflops"] == pytest.approx(3 * r["prepare_hinv"]["achieved"])
    # sweep: W in, E out (fp32 each), 4-bit codes, fp16 scale + zero per row and group, U's diagonal blocks
    sweep = D * D * (4 + 4 + 0.5) + D * (D // 128) * 4 + (D // B) * B * B * 4
    q = r["quantize_layer"]
    assert q["sweep_gbs_over_stage"] == pytest.approx(sweep / 1e-3 / 1e9)
    assert q["sweep_frac_over_stage"] == pytest.approx(sweep / 1e-3 / 1e9 / 6500.0)
    assert q["sweep_issued_gbs_over_stage"] == pytest.approx((sweep + D * D * 4) / 1e-3 / 1e9)
    # trailing products: sum over blocks of 2 d_out (d_in - B (i + 1)) B = d_out d_in (d_in - B)
    t = 2 * D * B * sum(D - B * (i + 1) for i in range(D // B))
    assert t == D * D * (D - B)
    assert q["trailing_tflops_over_stage"] == pytest.approx(t / 1e-3 / 1e12)
    assert q["trailing_issued_tflops_over_stage"] == pytest.approx(3 * t / 1e-3 / 1e12)
    for k, v in (("hessian", r["hessian"]), ("prepare_hinv", r["prepare_hinv"])):
        assert v["frac"] == pytest.approx(v["achieved"] / 1600.0), k


def test_per_row_grid_counts_one_group():
    p = _layer()
    p.groupsize = -1
    stages = {"hessian": 1.0, "prepare_hinv": 1.0, "quantize_layer": 1.0}
    r = bench.stage_rooflines(p, stages, peak=1.0, hbm=1.0)
    sweep = D * D * 8.5 + D * 4 + (D // B) * B * B * 4
    assert r["quantize_layer"]["sweep_gbs_over_stage"] == pytest.approx(sweep / 1e-3 / 1e9)
