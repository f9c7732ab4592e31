"""Pins of the oracle's FP8 E4M3 third precision (reading (p) of the oracle):
the format's published facts, a brute-force check of the encoder's
rounding, the tile quantiser on cases whose answer is known, and the FP8
route's wiring on inputs that the format represents exactly."""

import math

import numpy as np
import pytest

import oracle
from mixed_precision_attention_tm_b200 import inputs

ALL = np.arange(256)


# ---------------------------------------------------------------- the format
def test_e4m3_format_facts():
    v = oracle.e4m3_decode(ALL)
    nan = np.isnan(v)
    assert list(np.nonzero(nan)[0]) == [0x7F, 0xFF]           # one NaN per sign, no infinities
    assert v[0x7E] == 448.0 and oracle.E4M3_MAX == 448.0      # largest finite value
    assert v[0x08] == 2.0 ** -6                               # smallest normal
    assert v[0x01] == 2.0 ** -9                               # smallest subnormal
    assert v[0x00] == 0.0 and math.copysign(1.0, v[0x80]) == -1.0
    pos = v[:0x7F]
    assert np.all(np.diff(pos) > 0)                           # codes order the magnitudes
    assert np.array_equal(v[0x80:0xFF], -v[0x00:0x7F])        # sign bit
    # 8 equally spaced values per binade [2^k, 2^(k+1)) for k = -6 .. 7,
    # 7 in the top binade [256, 448]; the subnormals step by 2^-9
    for k in range(-6, 8):
        b = pos[(pos >= 2.0 ** k) & (pos < 2.0 ** (k + 1))]
        assert len(b) == 8 and np.allclose(np.diff(b), 2.0 ** (k - 3), rtol=0, atol=0)
    top = pos[pos >= 256]
    assert len(top) == 7 and top[-1] == 448
    assert np.array_equal(pos[:8], np.arange(8) * 2.0 ** -9)


def test_e4m3_round_trip():
    v = oracle.e4m3_decode(ALL)
    fin = ~np.isnan(v)
    assert np.array_equal(oracle.e4m3_encode(v[fin]), ALL[fin].astype(np.uint8))


def _brute(x):
    """Nearest finite E4M3 value by exhaustive search, ties to the even code,
    saturating; the sign of a zero result is the sign of x."""
    v = oracle.e4m3_decode(ALL)
    out = []
    for xi in np.asarray(x, dtype=np.float32).astype(np.float64):
        best, bd = None, None
        for c in range(0x7F):                       # non-negative finite codes
            dist = abs(abs(xi) - v[c])
            if best is None or dist < bd or (dist == bd and c % 2 == 0):
                best, bd = c, dist
        if np.signbit(xi):
            best |= 0x80
        out.append(best)
    return np.array(out, dtype=np.uint8)


def test_e4m3_encoder_matches_exhaustive_search():
    rng = np.random.default_rng(3)
    x = np.concatenate([rng.uniform(-500, 500, 600), rng.normal(0, 1e-2, 300), rng.normal(0, 3, 300),
                        np.exp2(rng.uniform(-12, 9, 300)) * rng.choice([-1, 1], 300)]).astype(np.float32)
    assert np.array_equal(oracle.e4m3_encode(x), _brute(x))


@pytest.mark.parametrize("x,code", [
    (1.0625, 0x38),          # halfway 1 .. 1.125: even mantissa (1.0)
    (1.1875, 0x3A),          # halfway 1.125 .. 1.25: even mantissa (1.25)
    (15.5, 0x58),            # halfway 15 (0x57, m=7) .. 16 (0x58, next binade, m=0): the even code
    (2.0 ** -10, 0x00),      # halfway 0 .. 2^-9: zero
    (3 * 2.0 ** -10, 0x02),  # halfway 2^-9 .. 2^-8: 2^-8
    (464.0, 0x7E),           # above 448: saturates
    (1e30, 0x7E),
    (-1e30, 0xFE),
    (-1e-20, 0x80),          # negative underflow keeps its sign
])
def test_e4m3_hand_cases(x, code):
    assert int(oracle.e4m3_encode(np.array([x]))[0]) == code


# ---------------------------------------------------------------- the tile quantiser
def test_fp8_tile_quantiser_known_cases():
    # one sequence of 192 rows, 64-row tiles, 2 heads, d = 16
    seqs = oracle.seq_table(192, 192)
    rng = np.random.default_rng(5)
    codes = rng.integers(0, 0x7F, size=(192, 2, 16)).astype(np.uint8)
    codes |= (rng.integers(0, 2, size=codes.shape) << 7).astype(np.uint8)
    codes[(codes & 0x7F) == 0x7F] = 0x10
    val = oracle.e4m3_decode(codes) * 2.0 ** -4                 # E4M3 values x 2^-4, exact in fp16
    x = val.astype(np.float16)
    assert np.array_equal(x.astype(np.float64), val)
    # tile 0 of head 0 reaches amax = 448 * 2^-4: its scale is 2^-4 exactly and
    # every code comes back; tile 1 of head 1 is all zero: scale 0, codes 0
    x[0, 0, 0] = np.float16(448 * 2.0 ** -4)
    x[64:128, 1, :] = 0
    c, s = oracle.quantize_tiles_fp8(x, seqs, 64, "q")
    assert s.shape == (3, 2) and s.dtype == np.float32
    assert s[0, 0] == np.float32(2.0 ** -4)
    exp0 = oracle.e4m3_encode(x[:64, 0, :].astype(np.float32) / np.float32(2.0 ** -4))
    assert np.array_equal(c[:64, 0, :], exp0)
    assert np.array_equal(oracle.e4m3_decode(c[1:64, 0, :]) * 2.0 ** -4, val[1:64, 0, :])
    assert s[1, 1] == 0 and not c[64:128, 1, :].any()
    # every scale is amax / 448 in fp32 and every code is within half a step
    for ig in range(3):
        for h in range(2):
            blk = x[ig * 64:(ig + 1) * 64, h, :].astype(np.float32)
            assert s[ig, h] == np.float32(np.float32(np.abs(blk).max()) / np.float32(448))


# ---------------------------------------------------------------- the FP8 route
def _fp8_exact_inputs(L, hq, hkv, d, tile, seed):
    """Q, K whose every value is an E4M3 value x 2^-4 and whose every tile
    holds +-448 x 2^-4, so each tile scale is 2^-4 and the codes are exact."""
    rng = np.random.default_rng(seed)
    out = []
    for h in (hq, hkv):
        c = rng.integers(0x20, 0x60, size=(L, h, d)).astype(np.uint8)   # moderate magnitudes
        c |= (rng.integers(0, 2, size=c.shape) << 7).astype(np.uint8)
        for r0 in range(0, L, tile):
            c[r0, :, 0] = 0x7E
        out.append((oracle.e4m3_decode(c) * 2.0 ** -4).astype(np.float16))
    return out


@pytest.mark.parametrize("causal", [False, True])
def test_fp8_route_on_exact_inputs_equals_fp16(causal):
    L, hq, hkv, d, tile, g = 200, 4, 2, 32, 64, 1
    q, k = _fp8_exact_inputs(L, hq, hkv, d, tile, 9)
    v = inputs.randn_f16((L, hkv, d), 10).numpy()
    seqs = oracle.seq_table(L, L)
    plain = oracle.attention(q, k, v, causal=causal, tile_m=tile, tile_n=tile, g=g)
    zero = np.zeros((hq, oracle.n_tiles(L, tile), oracle.mask_words(L, tile, g)), dtype=np.uint32)
    f8 = oracle.build_mask(hq, seqs, tile, tile, g, causal, 1.0, 4)      # every legal group FP8
    qf = oracle.quantize_tiles_fp8(q, seqs, tile, "q")
    kf = oracle.quantize_tiles_fp8(k, seqs, tile, "k")
    assert np.all(qf[1] == np.float32(2.0 ** -4)) and np.all(kf[1] == np.float32(2.0 ** -4))
    routed = oracle.attention(q, k, v, causal=causal, tile_m=tile, tile_n=tile, g=g, mask=zero,
                              q_quant=oracle.quantize_tiles(q, seqs, tile, "q"),
                              k_quant=oracle.quantize_tiles(k, seqs, tile, "k"),
                              mask_fp8=f8, qf8_quant=qf, kf8_quant=kf)
    assert np.array_equal(routed, plain)


def test_fp8_route_changes_scores_and_int8_takes_precedence():
    L, hq, hkv, d, tile, g = 192, 2, 1, 32, 64, 1
    q, k, v = (inputs.randn_f16((L, h, d), s).numpy() for h, s in ((hq, 1), (hkv, 2), (hkv, 3)))
    seqs = oracle.seq_table(L, L)
    qq, kq = oracle.quantize_tiles(q, seqs, tile, "q"), oracle.quantize_tiles(k, seqs, tile, "k")
    qf, kf = oracle.quantize_tiles_fp8(q, seqs, tile, "q"), oracle.quantize_tiles_fp8(k, seqs, tile, "k")
    ones = oracle.build_mask(hq, seqs, tile, tile, g, False, 1.0, 7)
    zero = np.zeros_like(ones)
    kw = dict(tile_m=tile, tile_n=tile, g=g, q_quant=qq, k_quant=kq, qf8_quant=qf, kf8_quant=kf)
    plain = oracle.attention(q, k, v, tile_m=tile, tile_n=tile, g=g)
    only8 = oracle.attention(q, k, v, mask=ones, mask_fp8=zero, **kw)
    both = oracle.attention(q, k, v, mask=ones, mask_fp8=ones, **kw)
    onlyf8 = oracle.attention(q, k, v, mask=zero, mask_fp8=ones, **kw)
    assert np.array_equal(both, only8)                        # INT8 wins over FP8
    e8, ef8 = np.abs(only8 - plain).max(), np.abs(onlyf8 - plain).max()
    assert 0 < ef8 and 0 < e8                                 # both routes quantise
    # E4M3 keeps 3 mantissa bits against the 7 of the per-tile INT8 codes on
    # unit-variance data: its score error, hence output error, is larger
    assert ef8 > e8
