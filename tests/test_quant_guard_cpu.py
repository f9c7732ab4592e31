"""CPU check of the rule the quantiser kernel uses to form INT8 codes without
one IEEE division per element (tm_quant.cu, int8_code): with r the correctly
rounded reciprocal of the tile scale s, code = rne(fl32(x * r)) unless that
product lies within 2^-15 of a half-integer, where fl32(x / s) decides.  The
rule is emulated here in numpy float32 and compared, over every fp16 value of
a tile's range and over constructed near-ties, with the oracle's codes (one
IEEE fp32 division per element).  GPU parity tests compare the kernel itself."""

import numpy as np
import pytest

import oracle
from quant_cases import AMAXES, all_f16_up_to, near_tie_values


def _guarded_codes(x16, s):
    """The kernel's rule: v = fl32(x * r); code = rne(v) unless
    |v - rne(v)| > 1/2 - 2^-15, where the IEEE quotient fl32(x / s) decides."""
    x = x16.astype(np.float32)
    s = np.float32(s)
    r = np.float32(np.float64(1.0) / np.float64(s))       # RN(1/s): exact 1/s rounded once
    v = (x * r).astype(np.float32)
    n = np.rint(v)
    near = np.abs((v - n).astype(np.float32)) > np.float32(0.5 - 2.0 ** -15)
    exact = np.rint((x.astype(np.float64) / np.float64(s)).astype(np.float32))   # fl32(x / s)
    n = np.where(near, exact, n)
    assert np.abs(n).max() <= 127                              # no clamp needed off the fallback
    return np.clip(n, -127, 127).astype(np.int8), int(near.sum())


@pytest.mark.parametrize("amax", AMAXES)
def test_guarded_reciprocal_rule_matches_oracle_on_every_fp16_value(amax):
    a = np.float16(amax)
    x = all_f16_up_to(a)
    x = np.concatenate([x, near_tie_values(a)])
    # one tile holding every value (amax included), as [T, 1, 1]
    seqs = oracle.seq_table(len(x), len(x))
    codes, scales = oracle.quantize_tiles(x.reshape(-1, 1, 1), seqs, len(x), "q")
    s = scales[0, 0]
    assert s == np.float32(np.float32(a) / np.float32(127.0))
    got, n_fallback = _guarded_codes(x, s)
    assert np.array_equal(got, codes.reshape(-1))
    if float(a) in (127.0, 1.984375, 2.0 ** -3 * 127):
        assert n_fallback > 0          # exact ties go through the division


def test_near_tie_construction_finds_exact_and_inexact_ties():
    # power-of-two scale: every x = (n + 0.5) * s is an exact tie
    v = near_tie_values(np.float16(127.0))
    assert np.any((v.astype(np.float64) / 1.0) % 1.0 == 0.5)
    # a scale that is not a power of two still yields near-ties
    assert near_tie_values(np.float16(3.140625)).size > 0
