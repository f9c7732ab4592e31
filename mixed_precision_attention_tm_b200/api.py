"""User-facing prefill plan: device buffers plus the three library calls.

``TileMixPrefill`` owns the device tensors of one problem shape (Q, K, V or
the INT8 cache, INT8 codes and tile scales, the routing bitmask, the output)
and runs one prefill step:

    tm_quantize_qk  ->  tm_build_mask  ->  tm_attn_fwd

on the current CUDA stream.  ``run_host`` is the same step fed from host
memory: pinned host -> device copies of the inputs, the step, and a device ->
host copy of the output.  Everything that computes is in libtm; this module
only allocates and passes pointers.
"""

from __future__ import annotations

import torch

from . import ops


class TileMixPrefill:
    def __init__(self, Lq, Lk, hq, hkv, d, *, causal=True, tile_m=128, tile_n=128, g=1, p=None,
                 seed=0, force_diag=False, force_sink=False, cu_seqlens=None, int8_cache=False,
                 tau=None, cu_seqlens_k=None, device="cuda"):
        """p: Bernoulli INT8 probability per eligible group (seeded mask);
        tau: instead of p, the content-driven policy (INT8 iff the tile
        scales' score-error bound s_q * s_k is at most tau).  Neither: all
        FP16.  cu_seqlens_k: key offsets per sequence when they differ from
        cu_seqlens (prefix-cached prefill: Lq = total new queries, Lk = total
        keys)."""
        self.shape = (Lq, Lk, hq, hkv, d)
        self.causal, self.tile_m, self.tile_n, self.g = causal, tile_m, tile_n, g
        if p is not None and tau is not None:
            raise ValueError("give either p (random routing) or tau (scale policy), not both")
        if tau is not None and int8_cache:
            raise ValueError("the scale policy needs tile scales of K; the INT8 cache has per-token scales")
        self.p, self.seed, self.force_diag, self.force_sink = p, seed, force_diag, force_sink
        self.tau = tau
        self.int8_cache = int8_cache
        self.device = torch.device(device)
        self.cu = None if cu_seqlens is None else cu_seqlens.to(self.device, torch.int32)
        cu_h = None if cu_seqlens is None else cu_seqlens.to("cpu", torch.int32).contiguous()
        self.cu_h = cu_h
        self.max_seqlen = None if cu_h is None else int((cu_h[1:] - cu_h[:-1]).max())
        if cu_seqlens_k is not None and cu_seqlens is None:
            raise ValueError("cu_seqlens_k needs cu_seqlens")
        if cu_seqlens_k is not None and tau is not None:
            raise ValueError("the scale policy takes shared query / key offsets")
        self.cu_k = None if cu_seqlens_k is None else cu_seqlens_k.to(self.device, torch.int32)
        self.ck_h = None if cu_seqlens_k is None else cu_seqlens_k.to("cpu", torch.int32).contiguous()
        self.max_seqlen_k = None if self.ck_h is None else int((self.ck_h[1:] - self.ck_h[:-1]).max())
        dev = self.device
        self.q = torch.empty((Lq, hq, d), dtype=torch.float16, device=dev)
        if int8_cache:
            self.k = self.v = None
            self.kc = torch.empty((Lk, hkv, d), dtype=torch.int8, device=dev)
            self.vc = torch.empty((Lk, hkv, d), dtype=torch.int8, device=dev)
            self.ks = torch.empty((Lk, hkv), dtype=torch.float16, device=dev)
            self.vs = torch.empty((Lk, hkv), dtype=torch.float16, device=dev)
        else:
            self.k = torch.empty((Lk, hkv, d), dtype=torch.float16, device=dev)
            self.v = torch.empty((Lk, hkv, d), dtype=torch.float16, device=dev)
        self.out = torch.empty((Lq, hq, d), dtype=torch.float16, device=dev)
        self.routed = p is not None or tau is not None
        self.q_quant = self.k_quant = self.bitmask = None
        if self.routed:
            # codes, tile scales and the routing mask: allocated once, rewritten every step
            cu_np = None if cu_h is None else cu_h.numpy()
            nqt = ops.count_tiles(Lq, tile_m, cu_np)
            self.q_quant = (torch.empty((Lq, hq, d), dtype=torch.int8, device=dev),
                            torch.empty((nqt, hq), dtype=torch.float32, device=dev))
            if not int8_cache:
                ck_np = cu_np if self.ck_h is None else self.ck_h.numpy()
                nkt = ops.count_tiles(Lk, tile_n, ck_np)
                self.k_quant = (torch.empty((Lk, hkv, d), dtype=torch.int8, device=dev),
                                torch.empty((nkt, hkv), dtype=torch.float32, device=dev))
            maxk = Lk if cu_h is None else (self.max_seqlen if self.ck_h is None else self.max_seqlen_k)
            self.bitmask = torch.empty((hq, nqt, ops.mask_words(maxk, tile_n, g)), dtype=torch.int32,
                                       device=dev)
        self.launches_per_step = 1 + (3 if self.routed and not int8_cache else 2 if self.routed else 0)

    # -- inputs -----------------------------------------------------------
    def load(self, q, k=None, v=None, kv_cache=None):
        """Copy device or host tensors into the plan's resident buffers."""
        self.q.copy_(q, non_blocking=True)
        if self.int8_cache:
            kc, ks, vc, vs = kv_cache
            self.kc.copy_(kc, non_blocking=True)
            self.ks.copy_(ks, non_blocking=True)
            self.vc.copy_(vc, non_blocking=True)
            self.vs.copy_(vs, non_blocking=True)
        else:
            self.k.copy_(k, non_blocking=True)
            self.v.copy_(v, non_blocking=True)

    def input_bytes(self):
        t = [self.q] + ([self.kc, self.ks, self.vc, self.vs] if self.int8_cache else [self.k, self.v])
        return sum(x.numel() * x.element_size() for x in t)

    def output_bytes(self):
        return self.out.numel() * self.out.element_size()

    # -- the step ---------------------------------------------------------
    def quantize(self):
        kq = (None, None) if self.k_quant is None else self.k_quant
        ops.quantize_qk(self.q, None if self.int8_cache else self.k, tile_m=self.tile_m, tile_n=self.tile_n,
                        cu_seqlens=self.cu, max_seqlen=self.max_seqlen, cu_seqlens_host=self.cu_h,
                        out=(*self.q_quant, *kq), cu_seqlens_k=self.cu_k, max_seqlen_k=self.max_seqlen_k,
                        cu_seqlens_k_host=self.ck_h)

    def mask(self):
        Lq, Lk = self.shape[0], self.shape[1]
        if self.tau is not None:
            ops.build_mask_scale_policy(self.q_quant[1], self.k_quant[1], self.shape[2], self.shape[3],
                                        tile_m=self.tile_m, tile_n=self.tile_n, g=self.g, causal=self.causal,
                                        tau=self.tau, force_diag=self.force_diag, force_sink=self.force_sink,
                                        Lq=Lq, Lk=Lk, cu_seqlens=self.cu, max_seqlen=self.max_seqlen,
                                        cu_seqlens_host=self.cu_h, out=self.bitmask)
            return
        ops.build_mask(self.shape[2], tile_m=self.tile_m, tile_n=self.tile_n, g=self.g,
                       causal=self.causal, p=self.p, seed=self.seed, force_diag=self.force_diag,
                       force_sink=self.force_sink, Lq=Lq, Lk=Lk, cu_seqlens=self.cu,
                       max_seqlen=self.max_seqlen, device=self.device, cu_seqlens_host=self.cu_h,
                       out=self.bitmask, cu_seqlens_k=self.cu_k, max_seqlen_k=self.max_seqlen_k,
                       cu_seqlens_k_host=self.ck_h)

    def attend(self):
        kv = (self.kc, self.ks, self.vc, self.vs) if self.int8_cache else None
        return ops.attn_fwd(self.q, self.k, self.v, out=self.out, tile_m=self.tile_m, tile_n=self.tile_n,
                            g=self.g, causal=self.causal,
                            bitmask=self.bitmask if self.routed else None,
                            q_quant=self.q_quant if self.routed else None,
                            k_quant=self.k_quant if self.routed else None, kv_cache=kv,
                            cu_seqlens=self.cu, max_seqlen=self.max_seqlen, cu_seqlens_host=self.cu_h,
                            cu_seqlens_k=self.cu_k, max_seqlen_k=self.max_seqlen_k)

    def run(self):
        """One prefill step on the resident inputs; returns the device output."""
        if self.routed:
            self.quantize()
            self.mask()
        return self.attend()

    def run_host(self, q, k=None, v=None, kv_cache=None, out_host=None):
        """Step fed from (pinned) host tensors; the output lands in out_host."""
        self.load(q, k, v, kv_cache)
        self.run()
        if out_host is None:
            out_host = torch.empty(self.out.shape, dtype=self.out.dtype, pin_memory=True)
        out_host.copy_(self.out, non_blocking=True)
        return out_host


class HostPipeline:
    """Prefill steps fed from pinned host memory with the copies overlapped.

    Holds `depth` plans (device buffer sets) and three streams: host->device
    copies of step i+1 and device->host copies of step i-1 run while step i
    computes.  Events order each buffer set: a step's inputs are uploaded
    after the buffer's previous output has been downloaded, computed after
    its upload, and downloaded after its compute.  Every step still moves its
    own inputs and output across PCIe.
    """

    def __init__(self, *plan_args, depth=2, device="cuda", **plan_kw):
        self.device = torch.device(device)
        self.plans = [TileMixPrefill(*plan_args, device=self.device, **plan_kw) for _ in range(depth)]
        self.h2d = torch.cuda.Stream(device=self.device)
        self.comp = torch.cuda.Stream(device=self.device)
        self.d2h = torch.cuda.Stream(device=self.device)
        self.depth = depth
        self.freed = [None] * depth

    def input_bytes(self):
        return self.plans[0].input_bytes()

    def output_bytes(self):
        return self.plans[0].output_bytes()

    def run(self, host_inputs, host_outputs):
        """host_inputs: list of (q, k, v, kv_cache) pinned host tensors per step
        (k, v or kv_cache may be None); host_outputs: list of pinned host
        tensors receiving each step's output.  Returns the d2h stream's last
        event (completion of the final download)."""
        last = None
        for i, (inp, out_h) in enumerate(zip(host_inputs, host_outputs)):
            b = i % self.depth
            plan = self.plans[b]
            q, k, v, kv = inp
            with torch.cuda.stream(self.h2d):
                if self.freed[b] is not None:
                    self.h2d.wait_event(self.freed[b])
                plan.load(q, k, v, kv)
                loaded = torch.cuda.Event()
                loaded.record(self.h2d)
            with torch.cuda.stream(self.comp):
                self.comp.wait_event(loaded)
                plan.run()
                done = torch.cuda.Event()
                done.record(self.comp)
            with torch.cuda.stream(self.d2h):
                self.d2h.wait_event(done)
                out_h.copy_(plan.out, non_blocking=True)
                freed = torch.cuda.Event()
                freed.record(self.d2h)
            self.freed[b] = freed
            last = freed
        return last
