"""CPU checks of the C-ABI library: it loads, exports every function that
include/tm.h declares, its host-side routing functions agree bit for bit with
the oracle, and argument validation rejects bad calls before any launch.
No GPU compute is called here."""

import ctypes
import os
import shutil
import subprocess

import numpy as np
import pytest

import oracle
from mixed_precision_attention_tm_b200 import build as tmbuild

tmbuild.build()
from mixed_precision_attention_tm_b200 import ops  # noqa: E402


def test_library_exports_every_declared_symbol():
    names = ops.header_functions()
    assert len(names) >= 10
    lib = ops._lib()
    for n in names:
        assert hasattr(lib, n), n
    out = subprocess.run(["nm", "-D", "--defined-only", ops.LIB_PATH], capture_output=True, text=True).stdout
    exported = {l.split()[-1] for l in out.splitlines() if l.strip()}
    assert set(names) <= exported


def test_header_is_plain_c(tmp_path):
    """include/tm.h is a C header: it compiles as strict C99 with no CUDA or
    C++ header on the include path."""
    gcc = shutil.which("gcc")
    if gcc is None:
        pytest.skip("gcc not found")
    src = tmp_path / "use_header.c"
    src.write_text('#include "tm.h"\nint main(void) { tm_tensor t; (void)t; return tm_status_string(0) == 0; }\n')
    inc = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "include")
    r = subprocess.run([gcc, "-std=c99", "-Wall", "-Wextra", "-pedantic", "-Werror", "-I", inc, "-c", str(src),
                        "-o", str(tmp_path / "use_header.o")], capture_output=True, text=True)
    assert r.returncode == 0, r.stderr


def test_status_strings_and_version():
    lib = ops._lib()
    assert lib.tm_status_string(0) == b"ok"
    assert lib.tm_status_string(4) == b"device wait timed out"
    assert lib.tm_version().count(b".") == 2


@pytest.mark.parametrize("L,tile_n,g", [(16384, 128, 4), (16385, 128, 4), (65536, 128, 8), (256, 64, 1),
                                        (1, 128, 1), (0, 64, 3)])
def test_mask_words_matches_oracle(L, tile_n, g):
    assert ops.mask_words(L, tile_n, g) == oracle.mask_words(L, tile_n, g)


def test_count_tiles():
    assert ops.count_tiles(1000, 128) == 8
    assert ops.count_tiles(None, 64, [0, 70, 70, 231, 300]) == 2 + 0 + 3 + 2


MASK_CASES = [
    # (Hq, Lq, Lk, cu, tm, tn, g, causal, p, fd, fs)
    (2, 256, 256, None, 64, 64, 1, False, 0.5, False, False),
    (32, 16384, 16384, None, 128, 128, 4, True, 0.75, True, True),
    (3, 700, 2100, None, 128, 64, 3, True, 0.4, True, False),
    (4, 1500, 300, None, 64, 128, 1, True, 0.9, False, True),
    (5, 0, 0, [0, 1000, 1000, 5000, 5001], 128, 128, 4, True, 0.75, True, True),
    (28, 65536, 65536, None, 128, 128, 8, True, 0.5, True, True),
    (2, 4096, 4096, None, 128, 128, 1, False, 1.0, False, False),
    (2, 4096, 4096, None, 128, 128, 1, True, 0.0, False, False),
]


@pytest.mark.parametrize("case", MASK_CASES)
def test_host_mask_builder_bit_exact_vs_oracle(case):
    Hq, Lq, Lk, cu, tm, tn, g, causal, p, fd, fs = case
    seed = 0xC0FFEE + Hq
    got = ops.build_mask_host(Hq, tile_m=tm, tile_n=tn, g=g, causal=causal, p=p, seed=seed,
                              force_diag=fd, force_sink=fs, Lq=Lq, Lk=Lk, cu_seqlens_host=cu)
    if cu is not None:
        Lq = Lk = cu[-1]
    seqs = oracle.seq_table(Lq, Lk, cu)
    ref = oracle.build_mask(Hq, seqs, tm, tn, g, causal, p, seed, fd, fs)
    assert got.shape == ref.shape
    assert np.array_equal(got, ref)


@pytest.mark.parametrize("case", MASK_CASES[:5])
def test_route_stats_matches_oracle(case):
    Hq, Lq, Lk, cu, tm, tn, g, causal, p, fd, fs = case
    m = ops.build_mask_host(Hq, tile_m=tm, tile_n=tn, g=g, causal=causal, p=p, seed=3,
                            force_diag=fd, force_sink=fs, Lq=Lq, Lk=Lk, cu_seqlens_host=cu)
    nv, e8 = ops.route_stats(m, Hq=Hq, tile_m=tm, tile_n=tn, g=g, causal=causal, Lq=Lq, Lk=Lk,
                             cu_seqlens_host=cu)
    if cu is not None:
        Lq = Lk = cu[-1]
    seqs = oracle.seq_table(Lq, Lk, cu)
    rnv, re8 = oracle.route_stats(m, seqs, Hq, tm, tn, g, causal)
    assert (nv, e8) == (rnv, re8)


@pytest.mark.parametrize("case", MASK_CASES[:5])
def test_route_stats_of_two_planes_partition_the_pairs(case):
    """The FP8 pairs of a three-way launch are counted on the plane 'FP8 bit
    and not INT8 bit': the INT8 count and that count add up to the count of
    the union plane, and never exceed the visible pairs."""
    Hq, Lq, Lk, cu, tm, tn, g, causal, p, fd, fs = case
    kw = dict(tile_m=tm, tile_n=tn, g=g, causal=causal, force_diag=fd, force_sink=fs, Lq=Lq, Lk=Lk,
              cu_seqlens_host=cu)
    m8 = ops.build_mask_host(Hq, p=p, seed=3, **kw)
    mf8 = ops.build_mask_host(Hq, p=0.6, seed=4, **kw)
    st = dict(Hq=Hq, tile_m=tm, tile_n=tn, g=g, causal=causal, Lq=Lq, Lk=Lk, cu_seqlens_host=cu)
    nv, e8 = ops.route_stats(m8, **st)
    _, ef8 = ops.route_stats(mf8 & ~m8, **st)
    _, eu = ops.route_stats(m8 | mf8, **st)
    assert e8 + ef8 == eu and eu <= nv


def _t(T=256, H=2, d=64, data=1 << 20):
    return ops.TmTensor(data, T, H, d, H * d, d, None, None, 0)


def test_validation_rejects_before_launch():
    lib = ops._lib()
    q, k, v, o = _t(), _t(H=1), _t(H=1), _t()
    by = ctypes.byref
    # d outside {64, 128}
    bad = _t(d=96)
    assert lib.tm_attn_fwd(by(bad), by(k), by(v), by(o), None, 0, 0, None, 0, 64, 64, 1, 0, None) == ops.TM_ERR_UNSUPPORTED
    # tile sizes
    assert lib.tm_attn_fwd(by(q), by(k), by(v), by(o), None, 0, 0, None, 0, 32, 64, 1, 0, None) == ops.TM_ERR_UNSUPPORTED
    # Hq not a multiple of Hkv
    k3, v3 = _t(H=3), _t(H=3)
    assert lib.tm_attn_fwd(by(q), by(k3), by(v3), by(o), None, 0, 0, None, 0, 64, 64, 1, 0, None) == ops.TM_ERR_INVALID_ARG
    # misaligned pointer
    qm = _t(data=(1 << 20) + 2)
    assert lib.tm_attn_fwd(by(qm), by(k), by(v), by(o), None, 0, 0, None, 0, 64, 64, 1, 0, None) == ops.TM_ERR_INVALID_ARG
    # bitmask without codes / scales
    assert lib.tm_attn_fwd(by(q), by(k), by(v), by(o), None, 0, 0, ctypes.c_void_p(1 << 20), 0, 64, 64, 1, 0,
                           None) == ops.TM_ERR_INVALID_ARG
    # g < 1
    assert lib.tm_attn_fwd(by(q), by(k), by(v), by(o), None, 0, 0, None, 0, 64, 64, 0, 0, None) == ops.TM_ERR_INVALID_ARG
    # varlen without batch
    assert lib.tm_attn_fwd(by(q), by(k), by(v), by(o), ctypes.c_void_p(1 << 20), 0, 16, None, 0, 64, 64, 1, 0,
                           None) == ops.TM_ERR_INVALID_ARG
    # quantiser: null outputs, bad tile
    assert lib.tm_quantize_qk(by(q), None, None, None, None, None, None, 0, 0, 64, 64, None) == ops.TM_ERR_INVALID_ARG
    assert lib.tm_quantize_qk(by(q), None, None, None, None, None, None, 0, 0, 48, 64, None) == ops.TM_ERR_UNSUPPORTED
    # mask builder: p outside [0, 1]
    assert lib.tm_build_mask(ctypes.c_void_p(1 << 20), 2, None, 0, 0, 256, 256, 64, 64, 1, 0, 1.5,
                             ctypes.c_uint64(0), 0, 0, 8, None) == ops.TM_ERR_INVALID_ARG


def test_fp8_validation_rejects_before_launch():
    """tm_attn_fwd_fp8 / tm_quantize_qk_fp8 argument checks: every case below
    returns its status before any CUDA call."""
    lib = ops._lib()
    by = ctypes.byref
    P = ctypes.c_void_p
    q, k, v, o = _t(d=128), _t(H=1, d=128), _t(H=1, d=128), _t(d=128)
    ok = P(1 << 20)                                     # an aligned stand-in pointer

    def fwd(q=q, k=k, v=v, o=o, bm8=None, bmf8=ok, qc=ok, qs=ok, kc=ok, ks=ok, g=1):
        return lib.tm_attn_fwd_fp8(by(q), by(k), by(v), by(o), None, 0, 0, bm8, bmf8, 0, qc, qs, kc, ks, g, 1, None)

    # the FP8 route runs at d = 128 only
    assert fwd(q=_t(d=64), k=_t(H=1, d=64), v=_t(H=1, d=64), o=_t(d=64)) == ops.TM_ERR_UNSUPPORTED
    # an INT8 K/V cache is not an FP8 operand
    kc8 = ops.TmTensor(0, 256, 1, 128, 128, 128, P(1 << 20), P(1 << 21), ops.TM_SCALE_TOKEN)
    assert fwd(k=kc8, v=kc8) == ops.TM_ERR_UNSUPPORTED
    # the FP8 plane, codes and scales are required and aligned
    assert fwd(bmf8=None) == ops.TM_ERR_INVALID_ARG
    assert fwd(bmf8=P((1 << 20) + 2)) == ops.TM_ERR_INVALID_ARG
    for name in ("qc", "kc"):
        assert fwd(**{name: None}) == ops.TM_ERR_INVALID_ARG
        assert fwd(**{name: P((1 << 20) + 8)}) == ops.TM_ERR_INVALID_ARG
    for name in ("qs", "ks"):
        assert fwd(**{name: None}) == ops.TM_ERR_INVALID_ARG
        assert fwd(**{name: P((1 << 20) + 2)}) == ops.TM_ERR_INVALID_ARG
    # an INT8 plane needs the INT8 codes on Q and K
    assert fwd(bm8=ok) == ops.TM_ERR_INVALID_ARG
    assert fwd(g=0) == ops.TM_ERR_INVALID_ARG
    # quantiser: tile sizes, null and misaligned outputs
    assert lib.tm_quantize_qk_fp8(by(q), None, ok, ok, None, None, None, 0, 0, 96, 128, None) == ops.TM_ERR_UNSUPPORTED
    assert lib.tm_quantize_qk_fp8(by(q), None, None, ok, None, None, None, 0, 0, 128, 128, None) == \
        ops.TM_ERR_INVALID_ARG
    assert lib.tm_quantize_qk_fp8(by(q), None, P((1 << 20) + 4), ok, None, None, None, 0, 0, 128, 128, None) == \
        ops.TM_ERR_INVALID_ARG
    assert lib.tm_quantize_qk_fp8(by(q), None, ok, P((1 << 20) + 1), None, None, None, 0, 0, 128, 128, None) == \
        ops.TM_ERR_INVALID_ARG
    # K of another head width
    assert lib.tm_quantize_qk_fp8(by(q), by(_t(H=1, d=64)), ok, ok, ok, ok, None, 0, 0, 128, 128, None) == \
        ops.TM_ERR_INVALID_ARG


def test_prefill_plan_buffers_match_library_sizes():
    """The plan preallocates codes, tile scales and the routing mask once; their
    shapes must be the ones the library writes (tile counts per sequence, mask
    words from the longest sequence)."""
    import torch
    from mixed_precision_attention_tm_b200.api import TileMixPrefill
    lens = [300, 129, 1000]
    cu = torch.tensor(np.concatenate([[0], np.cumsum(lens)]), dtype=torch.int32)
    T = int(cu[-1])
    pl = TileMixPrefill(T, T, 8, 2, 128, causal=True, tile_m=64, tile_n=128, g=2, p=0.5,
                        cu_seqlens=cu, device="cpu")
    nqt = sum(-(-n // 64) for n in lens)
    nkt = sum(-(-n // 128) for n in lens)
    assert pl.q_quant[0].shape == (T, 8, 128) and pl.q_quant[1].shape == (nqt, 8)
    assert pl.k_quant[0].shape == (T, 2, 128) and pl.k_quant[1].shape == (nkt, 2)
    assert pl.bitmask.shape == (8, nqt, oracle.mask_words(max(lens), 128, 2))
    cache = TileMixPrefill(T, T, 8, 2, 128, p=0.5, cu_seqlens=cu, int8_cache=True, device="cpu")
    # quantise Q, build the mask, expand the cache into the workspace, attend
    assert cache.k_quant is None and cache.launches_per_step == 4
    assert cache.cache_ws.numel() == ops.cache_workspace_bytes(T, 2, len(lens))
    plain = TileMixPrefill(256, 256, 8, 2, 128, device="cpu")
    assert plain.bitmask is None and plain.launches_per_step == 1


def test_attn_kernel_choice_rejects_unknown_values():
    lib = ops._lib()
    assert lib.tm_set_attn_kernel(3) == ops.TM_ERR_INVALID_ARG
    assert lib.tm_set_attn_kernel(-1) == ops.TM_ERR_INVALID_ARG
    for c in (ops.ATTN_KERNEL_TWO_TILE, ops.ATTN_KERNEL_ONE_TILE, ops.ATTN_KERNEL_AUTO):
        assert lib.tm_set_attn_kernel(c) == ops.TM_OK


def test_kernel_choice_follows_the_documented_rule():
    """tm_attn_kernel_choice (host-only with an explicit SM count) returns the
    kernel tm_attn_fwd would launch, by the rule include/tm.h states: d = 64
    and routed d = 128 launches take the one-query-tile kernel, as do
    all-FP16 rows of fewer than 64 key tiles; longer all-FP16 rows keep the
    two-query-tile kernel unless it leaves SMs idle or fills its last wave
    clearly worse; tm_set_attn_kernel overrides."""
    one, two = ops.ATTN_KERNEL_ONE_TILE, ops.ATTN_KERNEL_TWO_TILE
    ch = ops.attn_kernel_choice
    sms = 148
    try:
        ops.set_attn_kernel(ops.ATTN_KERNEL_AUTO)
        # d = 64: the dual-stream one-tile kernel, whatever the shape
        for L, h, causal in ((1024, 32, False), (16384, 32, True), (65536, 8, False)):
            assert ch(L, L, h, 64, causal=causal, sm_count=sms) == one
        # d = 128 routed: the ping-pong one-tile kernel at every length
        for L in (640, 16384, 65536):
            assert ch(L, L, 32, 128, routed=True, sm_count=sms) == one
        # d = 128 all-FP16 rows under 64 key tiles (8191 keys: 64 tiles minus one key)
        assert ch(4096, 4096, 32, 128, causal=True, sm_count=sms) == one
        assert ch(512, 8064, 32, 128, causal=False, sm_count=sms) == one
        # 64 key tiles or more, causal, enough CTAs: the two-tile kernel (chunked)
        assert ch(16384, 16384, 32, 128, causal=True, sm_count=sms) == two
        assert ch(8192, 8192, 32, 128, causal=True, sm_count=sms) == two
        # ... unless its CTAs leave SMs idle: 8192 rows, 2 heads = 64 two-tile CTAs
        assert ch(8192, 8192, 2, 128, causal=True, sm_count=sms) == one
        # non-causal long rows: the kernel whose last wave is fuller (32 heads x 64
        # query tiles: 1024 pair CTAs fill 7 waves 0.99, 2048 one-tile CTAs 14 waves 0.99)
        assert ch(8192, 8192, 32, 128, causal=False, sm_count=sms) == two
        # the SM count enters the rule: 64 two-tile CTAs fill a 64-SM part
        assert ch(8192, 8192, 2, 128, causal=True, sm_count=64) == two
        # overrides
        ops.set_attn_kernel(ops.ATTN_KERNEL_TWO_TILE)
        assert ch(4096, 4096, 32, 64, sm_count=sms) == two
        ops.set_attn_kernel(ops.ATTN_KERNEL_ONE_TILE)
        assert ch(16384, 16384, 32, 128, sm_count=sms) == one
    finally:
        ops.set_attn_kernel(ops.ATTN_KERNEL_AUTO)
    lib = ops._lib()
    for bad in ((0, 1, 1, 8, 128, 0, 1, sms), (1, 1, 1, 8, 96, 0, 1, sms), (1, 1, 0, 8, 128, 0, 1, sms),
                (1, 1, 1, 8, 128, 0, 1, -1)):
        assert lib.tm_attn_kernel_choice(*bad) == 0, bad


def test_noalloc_validates_every_argument_before_any_cuda_call():
    """tm_attn_fwd_routed_noalloc rejects a bad call before it looks up its
    scratch array or launches anything: each case below returns its status
    without a CUDA call.  With no GPU present, a well-formed call gets as far
    as the first CUDA call (the array's address) and returns TM_ERR_CUDA, which
    shows the order."""
    import torch
    lib = ops._lib()
    by = ctypes.byref
    q, k, v, o = _t(d=128, H=4), _t(H=2, d=128), _t(H=2, d=128), _t(d=128, H=4)

    def call(q=q, k=k, v=v, o=o, tm=128, tn=128, g=2, p=0.5):
        return lib.tm_attn_fwd_routed_noalloc(by(q), by(k), by(v), by(o), tm, tn, g, 1, p, ctypes.c_uint64(1), 1, 1,
                                              None)

    assert lib.tm_attn_fwd_routed_noalloc(None, by(k), by(v), by(o), 128, 128, 1, 1, 0.5, ctypes.c_uint64(1), 1, 1,
                                          None) == ops.TM_ERR_INVALID_ARG
    assert call(tm=96) == ops.TM_ERR_UNSUPPORTED
    assert call(g=0) == ops.TM_ERR_INVALID_ARG
    assert call(p=1.5) == ops.TM_ERR_INVALID_ARG
    assert call(p=float("nan")) == ops.TM_ERR_INVALID_ARG
    # head width outside {64, 128}, and K / V / out of another head width than Q
    assert call(q=_t(d=96, H=4), o=_t(d=96, H=4)) == ops.TM_ERR_UNSUPPORTED
    assert call(k=_t(H=2, d=64)) == ops.TM_ERR_INVALID_ARG
    assert call(v=_t(H=2, d=64)) == ops.TM_ERR_INVALID_ARG
    assert call(o=_t(H=4, d=64)) == ops.TM_ERR_INVALID_ARG
    # Hq not a multiple of Hkv; V's shape differs from K's
    assert call(k=_t(H=3, d=128), v=_t(H=3, d=128)) == ops.TM_ERR_INVALID_ARG
    assert call(v=_t(T=255, H=2, d=128)) == ops.TM_ERR_INVALID_ARG
    assert call(v=_t(H=1, d=128)) == ops.TM_ERR_INVALID_ARG
    assert call(o=_t(T=128, H=4, d=128)) == ops.TM_ERR_INVALID_ARG
    # misaligned data and strides
    assert call(v=ops.TmTensor((1 << 20) + 8, 256, 2, 128, 256, 128, None, None, 0)) == ops.TM_ERR_INVALID_ARG
    assert call(k=ops.TmTensor(1 << 20, 256, 2, 128, 260, 128, None, None, 0)) == ops.TM_ERR_INVALID_ARG
    assert call(o=ops.TmTensor(1 << 20, 256, 4, 128, 256, 64, None, None, 0)) == ops.TM_ERR_INVALID_ARG
    # beyond the fixed array (codes alone: 16384 * 32 * 128 bytes = 64 MiB)
    big_q = _t(T=16384, H=32, d=128)
    assert call(q=big_q, o=big_q, k=_t(T=16384, H=8, d=128), v=_t(T=16384, H=8, d=128)) == ops.TM_ERR_UNSUPPORTED
    if not torch.cuda.is_available():
        assert call() == ops.TM_ERR_CUDA


def test_policy_entries_validate_before_launch():
    """tm_build_mask_scale_policy_varlen and tm_key_tile_scales return their
    status for bad arguments before any CUDA call."""
    lib = ops._lib()
    P = ctypes.c_void_p
    bm, cu, ck, sc = P(1 << 20), P(2 << 20), P(3 << 20), P(4 << 20)
    inf = ctypes.c_float(float("inf"))
    pol = lib.tm_build_mask_scale_policy_varlen
    # missing key offsets, missing query offsets
    assert pol(bm, 4, 2, cu, None, 2, 64, 64, 128, 128, 1, 1, sc, sc, inf, 0, 0, 8, None) == ops.TM_ERR_INVALID_ARG
    assert pol(bm, 4, 2, None, ck, 2, 64, 64, 128, 128, 1, 1, sc, sc, inf, 0, 0, 8, None) == ops.TM_ERR_INVALID_ARG
    # Hq not a multiple of Hkv, NaN tau, null scales, max_seqlen_k <= 0, batch <= 0
    assert pol(bm, 3, 2, cu, ck, 2, 64, 64, 128, 128, 1, 1, sc, sc, inf, 0, 0, 8, None) == ops.TM_ERR_INVALID_ARG
    assert pol(bm, 4, 2, cu, ck, 2, 64, 64, 128, 128, 1, 1, sc, sc, ctypes.c_float(float("nan")), 0, 0, 8,
               None) == ops.TM_ERR_INVALID_ARG
    assert pol(bm, 4, 2, cu, ck, 2, 64, 64, 128, 128, 1, 1, None, sc, inf, 0, 0, 8, None) == ops.TM_ERR_INVALID_ARG
    assert pol(bm, 4, 2, cu, ck, 2, 64, 0, 128, 128, 1, 1, sc, sc, inf, 0, 0, 8, None) == ops.TM_ERR_INVALID_ARG
    assert pol(bm, 4, 2, cu, ck, 0, 64, 64, 128, 128, 1, 1, sc, sc, inf, 0, 0, 8, None) == ops.TM_ERR_INVALID_ARG
    kts = lib.tm_key_tile_scales
    # null output / input, misaligned output, Hkv <= 0, tile_n <= 0, offsets without batch, negative length
    assert kts(None, sc, 2, None, 0, 0, 256, 128, None) == ops.TM_ERR_INVALID_ARG
    assert kts(sc, None, 2, None, 0, 0, 256, 128, None) == ops.TM_ERR_INVALID_ARG
    assert kts(P((4 << 20) + 2), sc, 2, None, 0, 0, 256, 128, None) == ops.TM_ERR_INVALID_ARG
    assert kts(sc, sc, 0, None, 0, 0, 256, 128, None) == ops.TM_ERR_INVALID_ARG
    assert kts(sc, sc, 2, None, 0, 0, 256, 0, None) == ops.TM_ERR_INVALID_ARG
    assert kts(sc, sc, 2, ck, 0, 256, 0, 128, None) == ops.TM_ERR_INVALID_ARG
    assert kts(sc, sc, 2, None, 0, 0, -1, 128, None) == ops.TM_ERR_INVALID_ARG
    # nothing to do: no launch, TM_OK
    assert kts(sc, sc, 2, None, 0, 0, 0, 128, None) == ops.TM_OK


def test_cache_workspace_entry_validates_before_launch():
    """tm_attn_fwd_cache_ws: a null or short workspace, or K / V that are not
    an INT8 cache, return TM_ERR_INVALID_ARG before any CUDA call."""
    lib = ops._lib()
    by = ctypes.byref
    q, o = _t(d=128), _t(d=128)
    kc = ops.TmTensor(None, 256, 1, 128, 128, 128, 2 << 20, 3 << 20, ops.TM_SCALE_TOKEN)
    need = lib.tm_cache_workspace_bytes(256, 1, 0)
    assert need >= 2 * 256 * 128 * 2 + 2 * 128 * 4
    P = ctypes.c_void_p
    call = lambda k, ws, nbytes: lib.tm_attn_fwd_cache_ws(by(q), by(k), by(k), by(o), None, None, 0, 0, 0, None, 0,
                                                          128, 128, 1, 1, ws, nbytes, None)
    assert call(kc, None, need) == ops.TM_ERR_INVALID_ARG
    assert call(kc, P(4 << 20), need - 256) == ops.TM_ERR_INVALID_ARG
    assert call(kc, P((4 << 20) + 16), need) == ops.TM_ERR_INVALID_ARG      # not 256-byte aligned
    assert call(_t(H=1, d=128), P(4 << 20), need) == ops.TM_ERR_INVALID_ARG  # fp16 K / V, not a cache
    assert lib.tm_cache_workspace_bytes(-1, 1, 0) < 0 and lib.tm_cache_workspace_bytes(10, 0, 0) < 0
