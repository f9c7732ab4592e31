"""Thin Python binding of libtm (ctypes).

Argument marshalling only: every step of tile-routed attention runs in the
library's CUDA kernels.  PyTorch supplies device memory and the current
stream; outputs are allocated here with torch and passed to the library as
raw pointers.  There is no CPU fallback: if libtm.so is missing the import
fails, and a CUDA tensor is required wherever the library expects device
memory.
"""

from __future__ import annotations

import ctypes
import math
import os
import re

import numpy as np
import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libtm.so")
HEADER = os.path.join(_HERE, "..", "include", "tm.h")

TM_OK, TM_ERR_INVALID_ARG, TM_ERR_UNSUPPORTED, TM_ERR_CUDA, TM_ERR_TIMEOUT = range(5)
TM_SCALE_NONE, TM_SCALE_TILE, TM_SCALE_TOKEN = range(3)


class TmError(RuntimeError):
    def __init__(self, status, what):
        self.status = status
        super().__init__(f"{what}: {_lib().tm_status_string(status).decode()} (status {status}"
                         + (f", cuda {_lib().tm_last_cuda_error()})" if status == TM_ERR_CUDA else ")"))


class TmTensor(ctypes.Structure):
    _fields_ = [
        ("data", ctypes.c_void_p),
        ("T", ctypes.c_int64), ("H", ctypes.c_int64), ("d", ctypes.c_int64),
        ("stride_t", ctypes.c_int64), ("stride_h", ctypes.c_int64),
        ("codes", ctypes.c_void_p),
        ("scales", ctypes.c_void_p),
        ("scale_kind", ctypes.c_int32),
    ]


_LIB = None


def _lib():
    global _LIB
    if _LIB is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(f"libtm.so not built at {LIB_PATH}; run "
                              "`python -m mixed_precision_attention_tm_b200.build`")
        lib = ctypes.CDLL(LIB_PATH)
        P, I32, I64, U64, D = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_uint64, ctypes.c_double
        TP = ctypes.POINTER(TmTensor)
        sig = {
            "tm_quantize_qk": (I32, [TP, TP, P, P, P, P, P, I32, I32, I32, I32, P]),
            "tm_mask_words": (I32, [I64, I32, I32]),
            "tm_count_tiles": (I64, [P, I32, I64, I32]),
            "tm_build_mask": (I32, [P, I32, P, I32, I32, I64, I64, I32, I32, I32, I32, D, U64, I32, I32,
                                    I64, P]),
            "tm_build_mask_host": (I32, [P, I32, P, I32, I64, I64, I32, I32, I32, I32, D, U64, I32, I32]),
            "tm_build_mask_scale_policy": (I32, [P, I32, I32, P, I32, I32, I64, I64, I32, I32, I32, I32, P, P,
                                                 ctypes.c_float, I32, I32, I64, P]),
            "tm_build_mask_scale_policy_varlen": (I32, [P, I32, I32, P, P, I32, I32, I32, I32, I32, I32, I32,
                                                        P, P, ctypes.c_float, I32, I32, I64, P]),
            "tm_key_tile_scales": (I32, [P, P, I32, P, I32, I32, I64, I32, P]),
            "tm_cache_workspace_bytes": (I64, [I64, I32, I32]),
            "tm_attn_fwd_cache_ws": (I32, [TP, TP, TP, TP, P, P, I32, I32, I32, P, I64, I32, I32, I32, I32, P, I64,
                                           P]),
            "tm_route_stats": (I32, [P, I64, I32, P, I32, I64, I64, I32, I32, I32, I32,
                                     ctypes.POINTER(D), ctypes.POINTER(D)]),
            "tm_attn_fwd": (I32, [TP, TP, TP, TP, P, I32, I32, P, I64, I32, I32, I32, I32, P]),
            "tm_attn_fwd_varlen": (I32, [TP, TP, TP, TP, P, P, I32, I32, I32, P, I64, I32, I32, I32, I32, P]),
            "tm_quantize_qk_varlen": (I32, [TP, TP, P, P, P, P, P, P, I32, I32, I32, I32, I32, P]),
            "tm_build_mask_varlen": (I32, [P, I32, P, P, I32, I32, I32, I32, I32, I32, I32, D, U64, I32, I32,
                                           I64, P]),
            "tm_route_stats_varlen": (I32, [P, I64, I32, P, P, I32, I32, I32, I32, I32,
                                            ctypes.POINTER(D), ctypes.POINTER(D)]),
            "tm_attn_fwd_routed_noalloc": (I32, [TP, TP, TP, TP, I32, I32, I32, I32, D, U64, I32, I32, P]),
            "tm_selftest_wait_timeout": (I32, [U64, P]),
            "tm_get_device_error": (I32, [P]),
            "tm_status_string": (ctypes.c_char_p, [I32]),
            "tm_last_cuda_error": (I32, []),
            "tm_version": (ctypes.c_char_p, []),
            "tm_probe_scratch_bytes": (I64, []),
            "tm_probe_rates": (I32, [ctypes.POINTER(D), I32, P, I64, P]),
            "tm_merge_head_shards": (I32, [P, I64, P, I64, I32, I32, I32, I32, P, P]),
            "tm_set_attn_kernel": (I32, [I32]),
            "tm_attn_kernel_choice": (I32, [I64, I64, I32, I32, I32, I32, I32, I32]),
            "tm_quantize_qk_fp8": (I32, [TP, TP, P, P, P, P, P, I32, I32, I32, I32, P]),
            "tm_attn_fwd_fp8": (I32, [TP, TP, TP, TP, P, I32, I32, P, P, I64, P, P, P, P, I32, I32, P]),
        }
        for name, (res, args) in sig.items():
            f = getattr(lib, name)
            f.restype = res
            f.argtypes = args
        _LIB = lib
    return _LIB


def header_functions():
    """Names of the functions declared in include/tm.h."""
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(tm_[a-z0-9_]+)\s*\(", src)))


def _check(st, what):
    if st != TM_OK:
        raise TmError(st, what)


def _stream():
    return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _cuda(t, name):
    if t is not None and not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")


def _desc(x, codes=None, scales=None, scale_kind=TM_SCALE_NONE, shape_from=None):
    """tm_tensor for a [T, H, d] tensor (x may be None for an INT8 cache)."""
    ref = x if x is not None else shape_from
    T, H, d = ref.shape
    if x is not None:
        if x.dtype != torch.float16:
            raise ValueError("fp16 tensor expected")
        if x.stride(2) != 1:
            raise ValueError("innermost dimension must be contiguous")
        st, sh = x.stride(0), x.stride(1)
    else:
        st, sh = H * d, d
    return TmTensor(None if x is None else x.data_ptr(), T, H, d, st, sh,
                    None if codes is None else codes.data_ptr(),
                    None if scales is None else scales.data_ptr(), scale_kind)


def _cu_host(cu_seqlens, cu_seqlens_host=None):
    """Host int32 copy of cu_seqlens.  Callers that run many steps pass the
    host copy they keep (cu_seqlens_host) so no step reads the device array
    back (a blocking copy)."""
    if cu_seqlens is None:
        return None
    if cu_seqlens_host is not None:
        return torch.as_tensor(cu_seqlens_host, dtype=torch.int32).contiguous()
    return cu_seqlens.detach().to("cpu", torch.int32).contiguous()


def _check_buf(t, shape, dtype, name):
    if t is None or tuple(t.shape) != tuple(shape) or t.dtype != dtype or not t.is_contiguous():
        raise ValueError(f"{name}: expected a contiguous {dtype} tensor of shape {tuple(shape)}")


def count_tiles(L=None, tile=128, cu_seqlens_host=None):
    lib = _lib()
    if cu_seqlens_host is not None:
        cu = np.ascontiguousarray(np.asarray(cu_seqlens_host, dtype=np.int32))
        return int(lib.tm_count_tiles(cu.ctypes.data, len(cu) - 1, 0, tile))
    return int(lib.tm_count_tiles(None, 0, int(L), tile))


def mask_words(max_lk, tile_n, g):
    return int(_lib().tm_mask_words(int(max_lk), int(tile_n), int(g)))


def _need(t, n, dtype, name):
    """t holds at least n contiguous elements of dtype."""
    if t is None or t.dtype != dtype or not t.is_contiguous() or t.numel() < n:
        got = "None" if t is None else f"{tuple(t.shape)} {t.dtype}"
        raise ValueError(f"{name}: at least {n} contiguous {dtype} elements expected, got {got}")


def _check_routing(Tq, Hq, Tk, Hkv, d, tile_m, tile_n, g, maxk, cu_h, ck_h, bitmask, mask_head_stride,
                   q_quant, k_quant, codes_dtype=torch.int8, what=""):
    """Sizes of the buffers an attention launch reads (the library receives
    plain pointers): codes [T, H, d]; tile scales n_tiles x H fp32, tiles
    counted per sequence; mask words (Hm - 1) x head stride + n_qtiles x W,
    W = mask_words(longest key row, tile_n, g) as the kernels compute it.
    ck_h: host key offsets (cu_h when keys share the query offsets), or None
    when only the device holds them (then the key scales are not counted)."""
    nqt = count_tiles(Tq, tile_m, None if cu_h is None else cu_h.numpy())
    if bitmask is not None:
        rows = nqt * mask_words(maxk, tile_n, g)
        _need(bitmask, rows + (Hq - 1) * int(mask_head_stride or 0), torch.int32, what + "bitmask")
    if q_quant is not None:
        _need(q_quant[0], Tq * Hq * d, codes_dtype, what + "q codes")
        _need(q_quant[1], nqt * Hq, torch.float32, what + "q scales")
    if k_quant is not None:
        _need(k_quant[0], Tk * Hkv * d, codes_dtype, what + "k codes")
        if ck_h is not None or cu_h is None:
            nkt = count_tiles(Tk, tile_n, None if ck_h is None else ck_h.numpy())
            _need(k_quant[1], nkt * Hkv, torch.float32, what + "k scales")


# ---------------------------------------------------------------- quantise
def quantize_qk(q, k=None, *, tile_m=128, tile_n=128, cu_seqlens=None, max_seqlen=None,
                cu_seqlens_host=None, out=None, cu_seqlens_k=None, max_seqlen_k=None, cu_seqlens_k_host=None):
    """Per-tile INT8 codes and fp32 scales of Q (tile_m rows) and K (tile_n
    rows): returns (q_codes [Tq,Hq,d] int8, q_scales [n_qt, Hq] fp32,
    k_codes, k_scales) (the K pair is None when k is None).  out: the same
    4-tuple of preallocated tensors to write into (reused across steps)."""
    _cuda(q, "q")
    _cuda(k, "k")
    lib = _lib()
    cu_h = _cu_host(cu_seqlens, cu_seqlens_host)
    batch = 0 if cu_h is None else cu_h.numel() - 1
    if cu_seqlens is not None and max_seqlen is None:
        max_seqlen = int((cu_h[1:] - cu_h[:-1]).max()) if batch else 0
    nqt = count_tiles(q.shape[0], tile_m, None if cu_h is None else cu_h.numpy())
    ck_h = cu_h if cu_seqlens_k is None else _cu_host(cu_seqlens_k, cu_seqlens_k_host)
    if cu_seqlens_k is not None and max_seqlen_k is None:
        max_seqlen_k = int((ck_h[1:] - ck_h[:-1]).max()) if batch else 0
    if out is not None:
        qc, qs, kc, ks = out
        _check_buf(qc, q.shape, torch.int8, "q_codes")
        _check_buf(qs, (nqt, q.shape[1]), torch.float32, "q_scales")
        if k is None:
            kc = ks = None
    else:
        qc = torch.empty(q.shape, dtype=torch.int8, device=q.device)
        qs = torch.empty((nqt, q.shape[1]), dtype=torch.float32, device=q.device)
        kc = ks = None
    if k is not None and out is not None:
        nkt = count_tiles(k.shape[0], tile_n, None if ck_h is None else ck_h.numpy())
        _check_buf(kc, k.shape, torch.int8, "k_codes")
        _check_buf(ks, (nkt, k.shape[1]), torch.float32, "k_scales")
    elif k is not None:
        nkt = count_tiles(k.shape[0], tile_n, None if ck_h is None else ck_h.numpy())
        kc = torch.empty(k.shape, dtype=torch.int8, device=k.device)
        ks = torch.empty((nkt, k.shape[1]), dtype=torch.float32, device=k.device)
    qd = _desc(q)
    kd = _desc(k) if k is not None else None
    if cu_seqlens_k is not None:       # separate key offsets (prefix-cached prefill)
        st = lib.tm_quantize_qk_varlen(ctypes.byref(qd), None if kd is None else ctypes.byref(kd),
                                       _ptr(qc), _ptr(qs), _ptr(kc), _ptr(ks), _ptr(cu_seqlens), _ptr(cu_seqlens_k),
                                       batch, int(max_seqlen or 0), int(max_seqlen_k or 0), tile_m, tile_n,
                                       _stream())
        _check(st, "tm_quantize_qk_varlen")
        return qc, qs, kc, ks
    st = lib.tm_quantize_qk(ctypes.byref(qd), None if kd is None else ctypes.byref(kd),
                            _ptr(qc), _ptr(qs), _ptr(kc), _ptr(ks), _ptr(cu_seqlens), batch,
                            int(max_seqlen or 0), tile_m, tile_n, _stream())
    _check(st, "tm_quantize_qk")
    return qc, qs, kc, ks


def quantize_qk_fp8(q, k=None, *, tile_m=128, tile_n=128, cu_seqlens=None, max_seqlen=None,
                    cu_seqlens_host=None, out=None):
    """Per-tile FP8 E4M3 codes and fp32 scales of Q and K (the third
    precision; tm_quantize_qk_fp8): returns (q_codes [Tq,Hq,d] uint8,
    q_scales [n_qt, Hq] fp32, k_codes, k_scales); the K pair is None when k
    is None.  out: the same 4-tuple of preallocated tensors."""
    _cuda(q, "q")
    _cuda(k, "k")
    cu_h = _cu_host(cu_seqlens, cu_seqlens_host)
    batch = 0 if cu_h is None else cu_h.numel() - 1
    if cu_seqlens is not None and max_seqlen is None:
        max_seqlen = int((cu_h[1:] - cu_h[:-1]).max()) if batch else 0
    cu_np = None if cu_h is None else cu_h.numpy()
    nqt = count_tiles(q.shape[0], tile_m, cu_np)
    if out is not None:
        qc, qs, kc, ks = out
        _check_buf(qc, q.shape, torch.uint8, "q_codes")
        _check_buf(qs, (nqt, q.shape[1]), torch.float32, "q_scales")
    else:
        qc = torch.empty(q.shape, dtype=torch.uint8, device=q.device)
        qs = torch.empty((nqt, q.shape[1]), dtype=torch.float32, device=q.device)
        kc = ks = None
    if k is not None:
        nkt = count_tiles(k.shape[0], tile_n, cu_np)
        if out is not None:
            _check_buf(kc, k.shape, torch.uint8, "k_codes")
            _check_buf(ks, (nkt, k.shape[1]), torch.float32, "k_scales")
        else:
            kc = torch.empty(k.shape, dtype=torch.uint8, device=k.device)
            ks = torch.empty((nkt, k.shape[1]), dtype=torch.float32, device=k.device)
    else:
        kc = ks = None
    qd = _desc(q)
    kd = _desc(k) if k is not None else None
    st = _lib().tm_quantize_qk_fp8(ctypes.byref(qd), None if kd is None else ctypes.byref(kd), _ptr(qc), _ptr(qs),
                                   _ptr(kc), _ptr(ks), _ptr(cu_seqlens), batch, int(max_seqlen or 0), tile_m,
                                   tile_n, _stream())
    _check(st, "tm_quantize_qk_fp8")
    return qc, qs, kc, ks


# ---------------------------------------------------------------- mask
def build_mask(Hq, *, tile_m, tile_n, g, causal, p, seed, force_diag=False, force_sink=False,
               Lq=None, Lk=None, cu_seqlens=None, max_seqlen=None, device="cuda",
               cu_seqlens_host=None, out=None, cu_seqlens_k=None, max_seqlen_k=None, cu_seqlens_k_host=None):
    """Seeded routing bitmask on the device, int32 view [Hq, n_qt, W] of the
    uint32 words (bit 1 = INT8).  The library writes every word, so the
    buffer (out, or a new one) needs no initialisation."""
    lib = _lib()
    cu_h = _cu_host(cu_seqlens, cu_seqlens_host)
    batch = 0 if cu_h is None else cu_h.numel() - 1
    if cu_h is not None:
        lens = (cu_h[1:] - cu_h[:-1])
        maxk = int(lens.max()) if batch else 0
        if max_seqlen is None:
            max_seqlen = maxk
        nqt = count_tiles(None, tile_m, cu_h.numpy())
        if cu_seqlens_k is not None:       # key lengths from the key offsets
            ck_h = _cu_host(cu_seqlens_k, cu_seqlens_k_host)
            maxk = int((ck_h[1:] - ck_h[:-1]).max()) if batch else 0
            if max_seqlen_k is None:
                max_seqlen_k = maxk
            maxk = max_seqlen_k
    else:
        maxk = Lk
        nqt = count_tiles(Lq, tile_m)
    W = mask_words(maxk, tile_n, g)
    if out is None:
        out = torch.empty((Hq, nqt, W), dtype=torch.int32, device=device)
    else:
        _check_buf(out, (Hq, nqt, W), torch.int32, "bitmask")
    if cu_seqlens_k is not None:
        st = lib.tm_build_mask_varlen(_ptr(out), Hq, _ptr(cu_seqlens), _ptr(cu_seqlens_k), batch,
                                      int(max_seqlen or 0), int(max_seqlen_k or 0), tile_m, tile_n, g,
                                      int(bool(causal)), float(p), ctypes.c_uint64(int(seed) & (2 ** 64 - 1)),
                                      int(bool(force_diag)), int(bool(force_sink)), nqt * W, _stream())
        _check(st, "tm_build_mask_varlen")
        return out
    st = lib.tm_build_mask(_ptr(out), Hq, _ptr(cu_seqlens), batch, int(max_seqlen or 0),
                           int(Lq or 0), int(Lk or 0), tile_m, tile_n, g, int(bool(causal)),
                           float(p), ctypes.c_uint64(int(seed) & (2 ** 64 - 1)),
                           int(bool(force_diag)), int(bool(force_sink)), nqt * W, _stream())
    _check(st, "tm_build_mask")
    return out


def build_mask_scale_policy(q_scales, k_scales, Hq, Hkv, *, tile_m, tile_n, g, causal, tau, force_diag=False,
                            force_sink=False, Lq=None, Lk=None, cu_seqlens=None, max_seqlen=None,
                            cu_seqlens_host=None, out=None, cu_seqlens_k=None, max_seqlen_k=None,
                            cu_seqlens_k_host=None):
    """Content-driven routing bitmask (int32 view [Hq, n_qt, W]): group G of
    query tile I goes INT8 iff s_q[I] * max s_k over its visible key tiles
    <= tau (see tm_build_mask_scale_policy).  q_scales / k_scales: the device
    tile scales from quantize_qk, or k_scales from key_tile_scales for an INT8
    cache.  cu_seqlens_k: key offsets when they differ from cu_seqlens."""
    _cuda(q_scales, "q_scales")
    _cuda(k_scales, "k_scales")
    lib = _lib()
    cu_h = _cu_host(cu_seqlens, cu_seqlens_host)
    batch = 0 if cu_h is None else cu_h.numel() - 1
    if cu_seqlens_k is not None and cu_h is None:
        raise ValueError("cu_seqlens_k needs cu_seqlens")
    if cu_h is not None:
        maxk = int((cu_h[1:] - cu_h[:-1]).max()) if batch else 0
        if max_seqlen is None:
            max_seqlen = maxk
        nqt = count_tiles(None, tile_m, cu_h.numpy())
        if cu_seqlens_k is not None:
            ck_h = _cu_host(cu_seqlens_k, cu_seqlens_k_host)
            if max_seqlen_k is None:
                max_seqlen_k = int((ck_h[1:] - ck_h[:-1]).max()) if batch else 0
            maxk = max_seqlen_k
    else:
        maxk = Lk
        nqt = count_tiles(Lq, tile_m)
    W = mask_words(maxk, tile_n, g)
    if out is None:
        out = torch.empty((Hq, nqt, W), dtype=torch.int32, device=q_scales.device)
    else:
        _check_buf(out, (Hq, nqt, W), torch.int32, "bitmask")
    if cu_seqlens_k is not None:
        st = lib.tm_build_mask_scale_policy_varlen(
            _ptr(out), Hq, Hkv, _ptr(cu_seqlens), _ptr(cu_seqlens_k), batch, int(max_seqlen or 0),
            int(max_seqlen_k or 0), tile_m, tile_n, g, int(bool(causal)), _ptr(q_scales), _ptr(k_scales),
            float(tau), int(bool(force_diag)), int(bool(force_sink)), nqt * W, _stream())
        _check(st, "tm_build_mask_scale_policy_varlen")
        return out
    st = lib.tm_build_mask_scale_policy(_ptr(out), Hq, Hkv, _ptr(cu_seqlens), batch, int(max_seqlen or 0),
                                        int(Lq or 0), int(Lk or 0), tile_m, tile_n, g, int(bool(causal)),
                                        _ptr(q_scales), _ptr(k_scales), float(tau), int(bool(force_diag)),
                                        int(bool(force_sink)), nqt * W, _stream())
    _check(st, "tm_build_mask_scale_policy")
    return out


def key_tile_scales(k_token_scales, *, tile_n, cu_seqlens_k=None, max_seqlen_k=None, cu_seqlens_k_host=None,
                    out=None):
    """Largest per-token key scale of every key tile and kv head (fp32
    [n_ktiles, Hkv]) from an INT8 cache's fp16 scales [Tk, Hkv]: the k_scales
    of the scale policy for that cache (see tm_key_tile_scales)."""
    _cuda(k_token_scales, "k_token_scales")
    if k_token_scales.dtype != torch.float16 or k_token_scales.dim() != 2 or not k_token_scales.is_contiguous():
        raise ValueError("k_token_scales: contiguous fp16 [Tk, Hkv]")
    Tk, Hkv = k_token_scales.shape
    lib = _lib()
    ck_h = _cu_host(cu_seqlens_k, cu_seqlens_k_host)
    batch = 0 if ck_h is None else ck_h.numel() - 1
    if ck_h is not None:
        if max_seqlen_k is None:
            max_seqlen_k = int((ck_h[1:] - ck_h[:-1]).max()) if batch else 0
        nkt = count_tiles(None, tile_n, ck_h.numpy())
    else:
        nkt = count_tiles(Tk, tile_n)
    if out is None:
        out = torch.empty((nkt, Hkv), dtype=torch.float32, device=k_token_scales.device)
    else:
        _check_buf(out, (nkt, Hkv), torch.float32, "k_tile_scales")
    st = lib.tm_key_tile_scales(_ptr(out), _ptr(k_token_scales), Hkv, _ptr(cu_seqlens_k), batch,
                                int(max_seqlen_k or 0), int(Tk), tile_n, _stream())
    _check(st, "tm_key_tile_scales")
    return out


def build_mask_host(Hq, *, tile_m, tile_n, g, causal, p, seed, force_diag=False, force_sink=False,
                    Lq=None, Lk=None, cu_seqlens_host=None):
    """Host twin of build_mask: numpy uint32 [Hq, n_qt, W]."""
    lib = _lib()
    cu = None if cu_seqlens_host is None else np.ascontiguousarray(np.asarray(cu_seqlens_host, np.int32))
    batch = 0 if cu is None else len(cu) - 1
    if cu is not None:
        maxk = int((cu[1:] - cu[:-1]).max()) if batch else 0
        nqt = count_tiles(None, tile_m, cu)
    else:
        maxk = Lk
        nqt = count_tiles(Lq, tile_m)
    W = mask_words(maxk, tile_n, g)
    out = np.zeros((Hq, nqt, W), dtype=np.uint32)
    st = lib.tm_build_mask_host(out.ctypes.data, Hq, None if cu is None else cu.ctypes.data, batch,
                                int(Lq or 0), int(Lk or 0), tile_m, tile_n, g, int(bool(causal)),
                                float(p), ctypes.c_uint64(int(seed) & (2 ** 64 - 1)),
                                int(bool(force_diag)), int(bool(force_sink)))
    _check(st, "tm_build_mask_host")
    return out


def route_stats(mask_host, *, Hq, tile_m, tile_n, g, causal, Lq=None, Lk=None, cu_seqlens_host=None,
                cu_seqlens_k_host=None):
    """(n_vis, e8) from a host mask (numpy uint32 [Hm, n_qt, W]) or None."""
    lib = _lib()
    cu = None if cu_seqlens_host is None else np.ascontiguousarray(np.asarray(cu_seqlens_host, np.int32))
    if cu_seqlens_k_host is not None:
        ck = np.ascontiguousarray(np.asarray(cu_seqlens_k_host, np.int32))
        nv, e8 = ctypes.c_double(), ctypes.c_double()
        ptr, hs = None, 0
        if mask_host is not None:
            m = np.ascontiguousarray(mask_host.astype(np.uint32, copy=False))
            ptr, hs = m.ctypes.data, (0 if m.shape[0] == 1 else m.shape[1] * m.shape[2])
        st = lib.tm_route_stats_varlen(ptr, hs, Hq, cu.ctypes.data, ck.ctypes.data, len(cu) - 1, tile_m, tile_n,
                                       g, int(bool(causal)), ctypes.byref(nv), ctypes.byref(e8))
        _check(st, "tm_route_stats_varlen")
        return nv.value, e8.value
    batch = 0 if cu is None else len(cu) - 1
    nv, e8 = ctypes.c_double(), ctypes.c_double()
    ptr, hs = None, 0
    if mask_host is not None:
        m = np.ascontiguousarray(mask_host.astype(np.uint32, copy=False))
        ptr = m.ctypes.data
        hs = 0 if m.shape[0] == 1 else m.shape[1] * m.shape[2]
    st = lib.tm_route_stats(ptr, hs, Hq, None if cu is None else cu.ctypes.data, batch, int(Lq or 0),
                            int(Lk or 0), tile_m, tile_n, g, int(bool(causal)), ctypes.byref(nv),
                            ctypes.byref(e8))
    _check(st, "tm_route_stats")
    return nv.value, e8.value


# ---------------------------------------------------------------- attention
def attn_fwd(q, k=None, v=None, *, out=None, tile_m=128, tile_n=128, g=1, causal=False,
             bitmask=None, mask_head_stride=None, q_quant=None, k_quant=None, kv_cache=None,
             cu_seqlens=None, max_seqlen=None, cu_seqlens_host=None, cu_seqlens_k=None, max_seqlen_k=None,
             cache_workspace=None):
    """Fused tile-routed attention.  q: fp16 [Tq,Hq,d]; k, v: fp16 [Tk,Hkv,d]
    (or kv_cache = (k_codes, k_scale16, v_codes, v_scale16)); bitmask: int32
    view [Hm, n_qt, W] (Hm = Hq or 1) or None (all FP16); q_quant / k_quant:
    (codes, scales) from quantize_qk, needed with a bitmask.
    cache_workspace: with kv_cache, a uint8 device tensor of at least
    cache_workspace_bytes(...) bytes; the cache is then expanded into it once
    and read from there (tm_attn_fwd_cache_ws).  Returns out."""
    _cuda(q, "q")
    lib = _lib()
    if out is None:
        out = torch.empty_like(q)
    cu_h = _cu_host(cu_seqlens, cu_seqlens_host)
    batch = 0 if cu_h is None else cu_h.numel() - 1
    if cu_seqlens is not None and max_seqlen is None:
        max_seqlen = int((cu_h[1:] - cu_h[:-1]).max()) if batch else 0
    if bitmask is not None and mask_head_stride is None:
        mask_head_stride = 0 if bitmask.shape[0] == 1 else bitmask.shape[1] * bitmask.shape[2]
    ck_h = None
    if cu_seqlens_k is not None and max_seqlen_k is None:
        ck_h = _cu_host(cu_seqlens_k, None)
        max_seqlen_k = int((ck_h[1:] - ck_h[:-1]).max()) if batch else 0
    kshape = (kv_cache[0] if kv_cache is not None else k).shape
    maxk = (max_seqlen_k if cu_seqlens_k is not None else max_seqlen) if cu_seqlens is not None else kshape[0]
    _check_routing(q.shape[0], q.shape[1], kshape[0], kshape[1], q.shape[2], tile_m, tile_n, g, maxk or 0, cu_h,
                   ck_h if cu_seqlens_k is not None else cu_h, bitmask, mask_head_stride, q_quant, k_quant)
    qd = _desc(q, *(q_quant if q_quant is not None else (None, None)),
               scale_kind=TM_SCALE_TILE if q_quant is not None else TM_SCALE_NONE)
    if kv_cache is not None:
        kcod, ksc, vcod, vsc = kv_cache
        kd = _desc(None, kcod, ksc, TM_SCALE_TOKEN, shape_from=kcod)
        vd = _desc(None, vcod, vsc, TM_SCALE_TOKEN, shape_from=vcod)
    else:
        _cuda(k, "k")
        _cuda(v, "v")
        kd = _desc(k, *(k_quant if k_quant is not None else (None, None)),
                   scale_kind=TM_SCALE_TILE if k_quant is not None else TM_SCALE_NONE)
        vd = _desc(v)
    od = _desc(out)
    if cache_workspace is not None:
        if kv_cache is None:
            raise ValueError("cache_workspace is for an INT8 K/V cache")
        _cuda(cache_workspace, "cache_workspace")
        need = cache_workspace_bytes(kshape[0], kshape[1], batch)
        if cache_workspace.dtype != torch.uint8 or cache_workspace.numel() < need \
                or not cache_workspace.is_contiguous():
            raise ValueError(f"cache_workspace: contiguous uint8 of at least {need} bytes expected")
        st = lib.tm_attn_fwd_cache_ws(ctypes.byref(qd), ctypes.byref(kd), ctypes.byref(vd), ctypes.byref(od),
                                      _ptr(cu_seqlens), _ptr(cu_seqlens_k), batch, int(max_seqlen or 0),
                                      int(max_seqlen_k or 0), _ptr(bitmask), int(mask_head_stride or 0), tile_m,
                                      tile_n, g, int(bool(causal)), _ptr(cache_workspace),
                                      int(cache_workspace.numel()), _stream())
        _check(st, "tm_attn_fwd_cache_ws")
        return out
    if cu_seqlens_k is not None:
        st = lib.tm_attn_fwd_varlen(ctypes.byref(qd), ctypes.byref(kd), ctypes.byref(vd), ctypes.byref(od),
                                    _ptr(cu_seqlens), _ptr(cu_seqlens_k), batch, int(max_seqlen or 0),
                                    int(max_seqlen_k or 0), _ptr(bitmask), int(mask_head_stride or 0), tile_m,
                                    tile_n, g, int(bool(causal)), _stream())
        _check(st, "tm_attn_fwd_varlen")
        return out
    st = lib.tm_attn_fwd(ctypes.byref(qd), ctypes.byref(kd), ctypes.byref(vd), ctypes.byref(od),
                         _ptr(cu_seqlens), batch, int(max_seqlen or 0), _ptr(bitmask),
                         int(mask_head_stride or 0), tile_m, tile_n, g, int(bool(causal)), _stream())
    _check(st, "tm_attn_fwd")
    return out


def cache_workspace_bytes(Tk, Hkv, batch=0):
    """Bytes of the workspace tm_attn_fwd_cache_ws needs for a cache of Tk
    tokens and Hkv heads (batch: sequences, 0 for one without offsets)."""
    n = int(_lib().tm_cache_workspace_bytes(int(Tk), int(Hkv), int(batch)))
    if n < 0:
        raise ValueError("bad cache shape")
    return n


def attn_fwd_fp8(q, k, v, *, bitmask_fp8, qf8_quant, kf8_quant, out=None, g=1, causal=False, bitmask=None,
                 q_quant=None, k_quant=None, cu_seqlens=None, max_seqlen=None, cu_seqlens_host=None):
    """Attention with the FP8 third precision (tm_attn_fwd_fp8): d = 128,
    128 x 128 tiles; bitmask_fp8 (int32 view [Hm, n_qt, W], layout of the
    INT8 bitmask) routes a group to FP8 when its INT8 bit (bitmask, may be
    None) is clear; qf8_quant / kf8_quant = (codes, scales) from
    quantize_qk_fp8; q_quant / k_quant the INT8 (codes, scales) when bitmask
    is given.  Returns out."""
    for t, n in ((q, "q"), (k, "k"), (v, "v"), (bitmask_fp8, "bitmask_fp8")):
        _cuda(t, n)
    if out is None:
        out = torch.empty_like(q)
    cu_h = _cu_host(cu_seqlens, cu_seqlens_host)
    batch = 0 if cu_h is None else cu_h.numel() - 1
    if cu_seqlens is not None and max_seqlen is None:
        max_seqlen = int((cu_h[1:] - cu_h[:-1]).max()) if batch else 0
    qd = _desc(q, *(q_quant if q_quant is not None else (None, None)),
               scale_kind=TM_SCALE_TILE if q_quant is not None else TM_SCALE_NONE)
    kd = _desc(k, *(k_quant if k_quant is not None else (None, None)),
               scale_kind=TM_SCALE_TILE if k_quant is not None else TM_SCALE_NONE)
    vd, od = _desc(v), _desc(out)
    mhs = 0 if bitmask_fp8.shape[0] == 1 else bitmask_fp8.shape[1] * bitmask_fp8.shape[2]
    if bitmask is not None and tuple(bitmask.shape) != tuple(bitmask_fp8.shape):
        raise ValueError("bitmask and bitmask_fp8 must have the same layout")
    maxk = max_seqlen if cu_seqlens is not None else k.shape[0]
    _check_routing(q.shape[0], q.shape[1], k.shape[0], k.shape[1], q.shape[2], 128, 128, g, maxk or 0, cu_h, cu_h,
                   bitmask, mhs, q_quant, k_quant)
    _check_routing(q.shape[0], q.shape[1], k.shape[0], k.shape[1], q.shape[2], 128, 128, g, maxk or 0, cu_h, cu_h,
                   bitmask_fp8, mhs, qf8_quant, kf8_quant, codes_dtype=torch.uint8, what="fp8 ")
    st = _lib().tm_attn_fwd_fp8(ctypes.byref(qd), ctypes.byref(kd), ctypes.byref(vd), ctypes.byref(od),
                                _ptr(cu_seqlens), batch, int(max_seqlen or 0), _ptr(bitmask), _ptr(bitmask_fp8), mhs,
                                _ptr(qf8_quant[0]), _ptr(qf8_quant[1]), _ptr(kf8_quant[0]), _ptr(kf8_quant[1]),
                                g, int(bool(causal)), _stream())
    _check(st, "tm_attn_fwd_fp8")
    return out


def attn_fwd_routed_noalloc(q, k, v, *, out=None, tile_m=128, tile_n=128, g=1, causal=False, p=0.5,
                            seed=0, force_diag=False, force_sink=False):
    """Routed prefill (quantise, mask, attend) for one sequence with the
    library's fixed device scratch array instead of caller-allocated codes,
    scales and mask; only out is allocated here (by torch) when not given."""
    for t, n in ((q, "q"), (k, "k"), (v, "v")):
        _cuda(t, n)
    if out is None:
        out = torch.empty_like(q)
    qd, kd, vd, od = _desc(q), _desc(k), _desc(v), _desc(out)
    st = _lib().tm_attn_fwd_routed_noalloc(ctypes.byref(qd), ctypes.byref(kd), ctypes.byref(vd), ctypes.byref(od),
                                           tile_m, tile_n, g, int(bool(causal)), float(p),
                                           ctypes.c_uint64(int(seed) & (2 ** 64 - 1)), int(bool(force_diag)),
                                           int(bool(force_sink)), _stream())
    _check(st, "tm_attn_fwd_routed_noalloc")
    return out


ATTN_KERNEL_AUTO, ATTN_KERNEL_TWO_TILE, ATTN_KERNEL_ONE_TILE = 0, 1, 2


def set_attn_kernel(choice):
    """Kernel for 128 x 128-tile attention with fp16 K / V, d = 64 or 128
    (tm_set_attn_kernel): ATTN_KERNEL_AUTO (default), ATTN_KERNEL_TWO_TILE or
    ATTN_KERNEL_ONE_TILE.  Process-wide."""
    _check(_lib().tm_set_attn_kernel(int(choice)), "tm_set_attn_kernel")


def attn_kernel_choice(max_q, max_k, hq, d, *, batch=1, routed=False, causal=True, sm_count=0):
    """Kernel tm_attn_fwd would run for 128 x 128 tiles with fp16 K / V
    (tm_attn_kernel_choice): ATTN_KERNEL_TWO_TILE or ATTN_KERNEL_ONE_TILE.
    sm_count 0 queries the current device."""
    r = int(_lib().tm_attn_kernel_choice(int(max_q), int(max_k), int(batch), int(hq), int(d), int(bool(routed)),
                                         int(bool(causal)), int(sm_count)))
    if r == 0:
        raise ValueError("tm_attn_kernel_choice: invalid arguments")
    return r


def merge_head_shards(out, gathered, head_start):
    """Interleave the all-gathered output slices of a head-sharded prefill
    back into token-major order (tm_merge_head_shards): gathered fp16
    [world, T, h_cap, d] contiguous, rank r's heads head_start[r] ..
    head_start[r+1]-1 in its first slots; out fp16 [T, Hq, d] (heads
    contiguous, rows may be strided).  Returns out."""
    _cuda(out, "out")
    _cuda(gathered, "gathered")
    if out.dtype != torch.float16 or gathered.dtype != torch.float16:
        raise ValueError("fp16 tensors expected")
    if gathered.dim() != 4 or not gathered.is_contiguous():
        raise ValueError("gathered: contiguous [world, T, h_cap, d] expected")
    world, T, h_cap, d = gathered.shape
    if out.dim() != 3 or out.shape[0] != T or out.shape[2] != d or out.stride(2) != 1 or out.stride(1) != d:
        raise ValueError("out: [T, Hq, d] with contiguous heads expected")
    hs = np.ascontiguousarray(np.asarray(head_start, dtype=np.int32))
    if hs.shape != (world + 1,):
        raise ValueError("head_start must hold world + 1 entries")
    st = _lib().tm_merge_head_shards(_ptr(out), int(out.stride(0)), _ptr(gathered), int(T), int(out.shape[1]),
                                     int(d), int(world), int(h_cap), hs.ctypes.data, _stream())
    _check(st, "tm_merge_head_shards")
    return out


def probe_rates():
    """Instruction rates behind the kernels' secondary bounds, measured on the
    current GPU (see tm_probe_rates in include/tm.h): cycles per warp
    instruction per SM sub-partition for MUFU ex2, cvt int32->fp32 and the
    kernels' exact conversion; cycles per tcgen05 MMA (f16 M128N128K16, i8
    M128N128K32) on one SM."""
    lib = _lib()
    n = int(lib.tm_probe_scratch_bytes())
    scratch = torch.empty(n, dtype=torch.uint8, device="cuda")
    out = (ctypes.c_double * 5)()
    _check(lib.tm_probe_rates(out, 5, _ptr(scratch), n, _stream()), "tm_probe_rates")
    keys = ("ex2_cycles_per_warp_instr", "cvt_s32_f32_cycles_per_warp_instr", "magic_conversion_cycles_per_warp_value",
            "mma_f16_m128n128k16_cycles", "mma_i8_m128n128k32_cycles")
    return dict(zip(keys, list(out)))


def selftest_wait_timeout(limit_ns=1_000_000):
    """Launch the bounded-wait self-test (a wait that must time out)."""
    _check(_lib().tm_selftest_wait_timeout(int(limit_ns), _stream()), "tm_selftest_wait_timeout")


def get_device_error():
    return int(_lib().tm_get_device_error(_stream()))


def sm_scale(d):
    return 1.0 / math.sqrt(d)
