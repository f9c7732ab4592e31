"""GPU parity of the FP8 third precision against the oracle: the E4M3 tile
quantiser bit for bit, and attention routed three ways (FP16, INT8, FP8)
element by element within the 3e-3 bound."""

import numpy as np
import pytest
import torch

import oracle
from gpu_helpers import TOL
from mixed_precision_attention_tm_b200 import inputs, ops

pytestmark = pytest.mark.gpu


def _seqs(L, cu):
    return oracle.seq_table(L, L, None if cu is None else list(cu))


# ---------------------------------------------------------------- quantiser
@pytest.mark.parametrize("T,H,d,tile,cu,scale", [
    (256, 2, 128, 128, None, 1.0),
    (300, 3, 128, 64, None, 1.0),                  # ragged last tile
    (777, 2, 64, 128, [0, 100, 555, 777], 1.0),    # varlen
    (512, 1, 128, 128, None, 1e-3),                # small values: subnormal codes and negative underflow
    (384, 2, 128, 128, None, 40.0),                # large values
])
def test_fp8_quantiser_bit_exact(T, H, d, tile, cu, scale):
    x = inputs.randn_f16((T, H, d), 7, scale=scale)
    if scale == 1.0:
        x[5, 0, :4] = torch.tensor([30.0, -25.0, 1e-4, -1e-7], dtype=torch.float16)   # outliers, tiny values
    seqs = _seqs(T, cu)
    ref_c, ref_s = oracle.quantize_tiles_fp8(x.numpy(), seqs, tile, "q")
    cu_t = None if cu is None else torch.tensor(cu, dtype=torch.int32, device="cuda")
    qc, qs, _, _ = ops.quantize_qk_fp8(x.cuda(), None, tile_m=tile, cu_seqlens=cu_t)
    torch.cuda.synchronize()
    assert ops.get_device_error() == ops.TM_OK
    assert np.array_equal(qs.cpu().numpy(), ref_s)
    got = qc.cpu().numpy()
    if cu is not None:                              # rows outside every sequence are not written
        got = got[:cu[-1]]
        ref_c = ref_c[:cu[-1]]
    assert np.array_equal(got, ref_c), f"{np.count_nonzero(got != ref_c)} codes differ"


# ---------------------------------------------------------------- attention
FP8_CASES = [
    # name, L or cu, hq, hkv, causal, g, p_int8 (None: no INT8 plane), p_fp8
    ("mixed3_noncausal", 640, 4, 2, False, 2, 0.3, 0.6),
    ("fp8_only_causal_ragged", 777, 4, 1, True, 1, None, 0.7),
    ("all_fp8", 512, 2, 2, True, 1, None, 1.0),
    ("mixed3_varlen", [0, 300, 1100, 1400], 4, 2, True, 1, 0.4, 0.5),
]


def _run(L, hq, hkv, causal, g, p8, pf8, cu=None, seed=0, qk=None):
    d = 128
    if qk is None:
        q, k, _ = inputs.qk_with_outliers(L, L, hq, hkv, d, seed)
    else:
        q, k = qk
    v = inputs.randn_f16((L, hkv, d), seed + 2)
    seqs = _seqs(L, cu)
    cu_t = None if cu is None else torch.tensor(cu, dtype=torch.int32, device="cuda")
    mk = dict(tile_m=128, tile_n=128, g=g, causal=causal, Lq=L, Lk=L, cu_seqlens=cu_t, force_diag=True,
              force_sink=True)
    qd, kd, vd = q.cuda(), k.cuda(), v.cuda()
    m8 = None if p8 is None else ops.build_mask(hq, p=p8, seed=seed + 4, **mk)
    mf8 = ops.build_mask(hq, p=pf8, seed=seed + 5, **mk)
    qq = kq = None
    if m8 is not None:
        qc, qs, kc, ks = ops.quantize_qk(qd, kd, cu_seqlens=cu_t)
        qq, kq = (qc, qs), (kc, ks)
    qf = ops.quantize_qk_fp8(qd, kd, cu_seqlens=cu_t)
    out = ops.attn_fwd_fp8(qd, kd, vd, bitmask_fp8=mf8, qf8_quant=qf[:2], kf8_quant=qf[2:], g=g, causal=causal,
                           bitmask=m8, q_quant=qq, k_quant=kq, cu_seqlens=cu_t)
    torch.cuda.synchronize()
    assert ops.get_device_error() == ops.TM_OK
    # oracle on the same bits
    cu_l = None if cu is None else list(cu)
    om8 = None if p8 is None else oracle.build_mask(hq, seqs, 128, 128, g, causal, p8, seed + 4, True, True)
    omf8 = oracle.build_mask(hq, seqs, 128, 128, g, causal, pf8, seed + 5, True, True)
    assert np.array_equal(mf8.cpu().numpy().view(np.uint32), omf8)
    qn, kn = q.numpy(), k.numpy()
    kw = dict(cu_seqlens=cu_l, causal=causal, tile_m=128, tile_n=128, g=g, mask_fp8=omf8,
              qf8_quant=oracle.quantize_tiles_fp8(qn, seqs, 128, "q"),
              kf8_quant=oracle.quantize_tiles_fp8(kn, seqs, 128, "k"))
    if om8 is not None:
        kw.update(mask=om8, q_quant=oracle.quantize_tiles(qn, seqs, 128, "q"),
                  k_quant=oracle.quantize_tiles(kn, seqs, 128, "k"))
    ref = oracle.attention(qn, kn, v.numpy(), **kw)
    return out.cpu(), ref, omf8, om8


@pytest.fixture(params=[ops.ATTN_KERNEL_TWO_TILE, ops.ATTN_KERNEL_ONE_TILE], ids=["two_tile", "one_tile"])
def attn_kernel(request):
    """FP8 launches without an INT8 plane run on either d = 128 kernel (the
    two-tile kernel with its 8-bit route in E4M3, or the one-tile kernel);
    three-way launches always take the one-tile kernel."""
    ops.set_attn_kernel(request.param)
    yield request.param
    ops.set_attn_kernel(ops.ATTN_KERNEL_AUTO)


@pytest.mark.parametrize("case", FP8_CASES, ids=[c[0] for c in FP8_CASES])
def test_fp8_routed_attention_matches_oracle(case, attn_kernel):
    name, L, hq, hkv, causal, g, p8, pf8 = case
    cu = None
    if isinstance(L, list):
        cu, L = L, L[-1]
    out, ref, mf8, m8 = _run(L, hq, hkv, causal, g, p8, pf8, cu=cu)
    o = out.double().numpy()
    if cu is not None:
        o, ref = o[:cu[-1]], ref[:cu[-1]]
    err = float(np.abs(o - ref).max())
    assert mf8.any()
    assert err <= TOL, f"{name}: max abs err {err}"


def test_fp8_route_on_exact_inputs_matches_fp16(attn_kernel):
    """Q, K whose values are E4M3 values x 2^-4 with every tile reaching
    448 x 2^-4: each tile scale is 2^-4, the codes are exact and the FP8 route
    computes the FP16 route's scores; the two outputs agree up to the fp32
    accumulation order of the tensor core."""
    L, hq, hkv, d = 384, 2, 1, 128
    rng = np.random.default_rng(1)
    qk = []
    for h in (hq, hkv):
        c = rng.integers(0x20, 0x58, size=(L, h, d)).astype(np.uint8)
        c |= (rng.integers(0, 2, size=c.shape) << 7).astype(np.uint8)
        c[0::128, :, 0] = 0x7E
        qk.append(torch.from_numpy((oracle.e4m3_decode(c) * 2.0 ** -4).astype(np.float16)))
    out, ref, _, _ = _run(L, hq, hkv, True, 1, None, 1.0, qk=qk)
    plain = oracle.attention(qk[0].numpy(), qk[1].numpy(), inputs.randn_f16((L, hkv, d), 2).numpy(), causal=True)
    assert np.abs(ref - plain).max() < 1e-12            # the oracle's FP8 route is exact here
    assert float(np.abs(out.double().numpy() - plain).max()) <= 1e-3
