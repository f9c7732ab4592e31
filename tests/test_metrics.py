"""The benchmark's FLOP convention, pinned to the MLX fused-SDPA "After"
table (MLX PR "Nax Refactor"): printed tflops = mlx_flops / (t_fus / 64)."""

import csv
import os

import pytest

import oracle
from mixed_precision_attention_tm_b200 import metrics

GOLD = os.path.join(os.path.dirname(__file__), "golden", "mlx_sdpa_after_table.csv")


def _rows():
    lines = [l for l in open(GOLD) if not l.startswith("#")]
    return list(csv.DictReader(lines))


def test_mlx_table_flop_convention():
    rows = _rows()
    assert len(rows) == 18
    for r in rows:
        f = metrics.mlx_flops(int(r["B"]), int(r["n_qh"]), int(r["qsl"]), int(r["ksl"]), int(r["hdim"]),
                              int(r["causal"]) == 1)
        tflops = f / (float(r["t_fus"]) / 64) / 1e12
        # t_fus is printed with 3 decimals (e.g. 0.022 s): allow its rounding
        rel_t = 0.0005 / float(r["t_fus"])
        assert abs(tflops / float(r["tflops"]) - 1) <= rel_t + 1e-3, r


def test_causal_rows_of_the_table_cost_like_bottom_right():
    # qsl=512, ksl=4096: causal and non-causal times are close (bottom-right
    # alignment keeps ~94% of the pairs; top-left would keep ~6%)
    rows = {(r["qsl"], r["ksl"], r["hdim"], r["causal"]): float(r["t_fus"]) for r in _rows()}
    for d in ("64", "128"):
        t_nc, t_c = rows[("512", "4096", d, "0")], rows[("512", "4096", d, "1")]
        frac_br = metrics.visible_pairs(512, 4096, True) / (512 * 4096)
        assert frac_br > 0.9 and t_c / t_nc > 0.9


@pytest.mark.parametrize("Lq,Lk,causal", [(10, 10, True), (5, 12, True), (12, 5, True), (7, 9, False), (1, 1, True),
                                          (16384, 16384, True), (512, 4096, True)])
def test_visible_pairs_closed_form(Lq, Lk, causal):
    if Lq * Lk <= 200:
        brute = sum(1 for i in range(Lq) for j in range(Lk) if oracle.visible(i, j, Lq, Lk, causal))
        assert metrics.visible_pairs(Lq, Lk, causal) == brute
    n, _ = oracle.route_stats(None, oracle.seq_table(Lq, Lk), 1, 128, 128, 1, causal)
    assert metrics.visible_pairs(Lq, Lk, causal) == n


def test_mixed_roofline_closed_forms():
    """T_roof = 2d E16 / P16 + 2d E8 / P8 + 2d N / P16 with P8 = 2 P16: all-FP16
    pairs give the FP16 peak, all-INT8 pairs 4/3 of it, and the routing
    sweep's realised INT8 fraction the bench line's effective peak."""
    import bench
    d, n, p16 = 128, 1.0e9, 1673.8e12
    eff = lambda e8: 4 * d * n / bench.roofline_time(d, n, e8, p16, 2 * p16) / 1e12   # noqa: E731
    assert abs(eff(0.0) - 1673.8) < 1e-6
    assert abs(eff(n) - 1673.8 * 4 / 3) < 1e-6
    f = 0.6801647848642051                      # realised INT8 fraction at p = 0.75
    assert abs(eff(f * n) - 2 * 1673.8 / (1 + (1 - f) + f / 2)) < 1e-6
    assert abs(eff(f * n) - 2016.73) < 0.01
