"""Pins of the oracle's per-tile quantiser (symmetric absmax/127, fp32 scale,
round-to-nearest-even codes, clamp to [-127, 127]).

Source: TileMix (Lattice paper page), abstract -- INT8 score computation over
score tiles; the scale rule is the symmetric per-tile absmax/127 reading.
"""

import numpy as np
import pytest

import oracle
from bruteforce import quant_block


def _one_tile(vals, d=None):
    vals = np.asarray(vals, dtype=np.float16)
    x = vals.reshape(len(vals) // (d or len(vals)), 1, d or len(vals))
    seqs = oracle.seq_table(x.shape[0], x.shape[0])
    codes, scales = oracle.quantize_tiles(x, seqs, 128, "q")
    return codes.reshape(-1), scales[0, 0]


def test_integer_tile_is_identity():
    vals = np.arange(-127, 128, dtype=np.float32)         # contains +-127
    codes, s = _one_tile(vals)
    assert s == np.float32(1.0)
    assert np.array_equal(codes.astype(np.int32), vals.astype(np.int32))


def test_round_half_to_even():
    vals = [127.0, 2.5, 3.5, -2.5, 0.5, -0.5, 1.5, -1.5, 126.5]
    codes, s = _one_tile(vals)
    assert s == 1.0
    assert codes.tolist() == [127, 2, 4, -2, 0, 0, 2, -2, 126]


def test_zero_tile():
    codes, s = _one_tile([0.0] * 16)
    assert s == 0.0 and not codes.any()


def test_single_outlier_flattens_the_rest():
    vals = [1000.0] + [0.25, -0.5, 1.0, -2.0, 3.0, 3.9375, -3.9375]
    codes, s = _one_tile(vals)
    assert s == np.float32(np.float32(1000.0) / np.float32(127.0))
    assert codes[0] == 127
    # |x| / s < 0.5 for |x| <= 3.9 (s = 7.874...): every other code is 0
    assert codes[1:].tolist() == [0, 0, 0, 0, 0, 1, -1]


def test_scale_is_fp32_division():
    # amax values whose quotient by 127 is inexact: s must be the RN fp32 quotient
    for amax in [1.0, 3.0, 0.1, 65504.0, 6.1e-05, 2.0 ** -24]:
        a = np.float32(np.float16(amax))
        codes, s = _one_tile([float(a), 0.0])
        exact = float(a) / 127.0                    # binary64 quotient, then one rounding
        assert s == np.float32(exact)
        assert codes[0] == 127


@pytest.mark.parametrize("seed", range(6))
def test_random_tiles_vs_scalar_bruteforce(seed):
    rng = np.random.default_rng(seed)
    T, H, d, tile = 23, 2, 8, 5                     # ragged last tile (23 = 4*5 + 3)
    x = (rng.standard_normal((T, H, d)) * rng.choice([0.01, 1.0, 30.0])).astype(np.float16)
    if seed % 2:
        x[3, 1, 5] = np.float16(-700.0)             # outlier in one tile
    if seed == 4:
        x[5:10, 0, :] = 0                           # an all-zero tile
    seqs = oracle.seq_table(T, T)
    codes, scales = oracle.quantize_tiles(x, seqs, tile, "q")
    for ti, r0 in enumerate(range(0, T, tile)):
        for h in range(H):
            rows = range(r0, min(T, r0 + tile))
            vals = [float(x[r, h, c]) for r in rows for c in range(d)]
            s, cs = quant_block(vals)
            assert scales[ti, h] == np.float32(s)
            got = [int(codes[r, h, c]) for r in rows for c in range(d)]
            assert got == cs


def test_varlen_tiles_restart_per_sequence():
    rng = np.random.default_rng(7)
    cu = [0, 7, 7, 20]                              # includes an empty sequence
    T, H, d, tile = 20, 1, 4, 4
    x = rng.standard_normal((T, H, d)).astype(np.float16)
    seqs = oracle.seq_table(T, T, cu)
    codes, scales = oracle.quantize_tiles(x, seqs, tile, "k")
    # tiles: seq0 rows 0-3, 4-6; seq2 rows 7-10, 11-14, 15-18, 19
    bounds = [(0, 4), (4, 7), (7, 11), (11, 15), (15, 19), (19, 20)]
    assert scales.shape == (len(bounds), 1)
    for t, (a, b) in enumerate(bounds):
        s, cs = quant_block([float(v) for v in x[a:b, 0, :].reshape(-1)])
        assert scales[t, 0] == np.float32(s)
        assert codes[a:b, 0, :].reshape(-1).tolist() == cs


def test_reconstruction_error_bound():
    rng = np.random.default_rng(3)
    x = rng.standard_normal((128, 1, 128)).astype(np.float16)
    seqs = oracle.seq_table(128, 128)
    codes, scales = oracle.quantize_tiles(x, seqs, 128, "q")
    s = float(scales[0, 0])
    err = np.abs(codes.astype(np.float64) * s - x.astype(np.float64))
    assert err.max() <= 0.5 * s * (1 + 1e-6)
