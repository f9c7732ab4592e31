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

from . import dist, ops


class TileMixPrefill:
    def __init__(self, Lq, Lk, hq, hkv, d, *, causal=True, tile_m=128, tile_n=128, g=1, p=None,
                 seed=0, force_diag=False, force_sink=False, cu_seqlens=None, int8_cache=False,
                 tau=None, cu_seqlens_k=None, out=None, bitmask=None, device="cuda"):
        """p: Bernoulli INT8 probability per eligible group (seeded mask);
        tau: instead of p, the content-driven policy (INT8 iff the tile
        scales' score-error bound s_q * s_k is at most tau; with the INT8
        cache s_k is the largest per-token key scale of the group's tiles).
        Neither: all FP16.  cu_seqlens_k: key offsets per sequence when they differ from
        cu_seqlens (prefix-cached prefill: Lq = total new queries, Lk = total
        keys).  out: an fp16 [Lq, hq, d] device tensor to write the output
        into (heads contiguous; rows may be strided) instead of a new one.
        bitmask: routing bits the caller writes before each step (an int32
        [hq, n_qt, W] device tensor); the step then routes by it and builds
        no mask of its own (p and tau must be None)."""
        self.shape = (Lq, Lk, hq, hkv, d)
        self.causal, self.tile_m, self.tile_n, self.g = causal, tile_m, tile_n, g
        if p is not None and tau is not None:
            raise ValueError("give either p (random routing) or tau (scale policy), not both")
        if bitmask is not None and (p is not None or tau is not None):
            raise ValueError("a caller-written bitmask replaces p and tau")
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
            # the cache's fp16 view and per-token K scales by key tile, written
            # once per step (tm_attn_fwd_cache_ws; 128 x 128 tiles, d = 128)
            self.cache_ws = None
            if tile_m == 128 and tile_n == 128 and d == 128:
                nb = 0 if cu_h is None else cu_h.numel() - 1
                self.cache_ws = torch.empty(ops.cache_workspace_bytes(Lk, hkv, nb), dtype=torch.uint8, device=dev)
        else:
            self.k = torch.empty((Lk, hkv, d), dtype=torch.float16, device=dev)
            self.v = torch.empty((Lk, hkv, d), dtype=torch.float16, device=dev)
        if out is not None:
            same_dev = out.device.type == dev.type and (dev.index is None or out.device.index == dev.index)
            if tuple(out.shape) != (Lq, hq, d) or out.dtype != torch.float16 or not same_dev \
                    or out.stride(2) != 1:
                raise ValueError("out: fp16 [Lq, hq, d] on the plan's device, innermost contiguous")
            self.out = out
        else:
            self.out = torch.empty((Lq, hq, d), dtype=torch.float16, device=dev)
        self.external_mask = bitmask is not None
        self.routed = p is not None or tau is not None or self.external_mask
        self.q_quant = self.k_quant = self.bitmask = self.k_tile_sc = None
        if self.routed:
            # codes, tile scales and the routing mask: allocated once, rewritten every step
            cu_np = None if cu_h is None else cu_h.numpy()
            nqt = ops.count_tiles(Lq, tile_m, cu_np)
            self.q_quant = (torch.empty((Lq, hq, d), dtype=torch.int8, device=dev),
                            torch.empty((nqt, hq), dtype=torch.float32, device=dev))
            ck_np = cu_np if self.ck_h is None else self.ck_h.numpy()
            nkt = ops.count_tiles(Lk, tile_n, ck_np)
            if not int8_cache:
                self.k_quant = (torch.empty((Lk, hkv, d), dtype=torch.int8, device=dev),
                                torch.empty((nkt, hkv), dtype=torch.float32, device=dev))
            elif tau is not None:
                # the policy's key statistic from the cache's per-token scales
                self.k_tile_sc = torch.empty((nkt, hkv), dtype=torch.float32, device=dev)
            maxk = Lk if cu_h is None else (self.max_seqlen if self.ck_h is None else self.max_seqlen_k)
            shape = (hq, nqt, ops.mask_words(maxk, tile_n, g))
            if self.external_mask:
                if tuple(bitmask.shape) != shape or bitmask.dtype != torch.int32 or not bitmask.is_contiguous():
                    raise ValueError(f"bitmask: contiguous int32 {shape} expected")
                self.bitmask = bitmask
            else:
                self.bitmask = torch.empty(shape, dtype=torch.int32, device=dev)
        n_quant = 1 if self.routed else 0          # Q and K are quantised in one launch
        n_mask = 1 if self.routed and not self.external_mask else 0
        n_mask += 1 if self.k_tile_sc is not None else 0
        n_mask += 1 if int8_cache and self.cache_ws is not None else 0   # the cache expansion
        self.launches_per_step = 1 + n_quant + n_mask

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
            k_sc = self.k_quant[1] if self.k_tile_sc is None else self.k_tile_sc
            if self.k_tile_sc is not None:
                shared = self.cu_k is None
                ops.key_tile_scales(self.ks, tile_n=self.tile_n, cu_seqlens_k=self.cu if shared else self.cu_k,
                                    max_seqlen_k=self.max_seqlen if shared else self.max_seqlen_k,
                                    cu_seqlens_k_host=self.cu_h if shared else self.ck_h, out=k_sc)
            ops.build_mask_scale_policy(self.q_quant[1], k_sc, self.shape[2], self.shape[3],
                                        tile_m=self.tile_m, tile_n=self.tile_n, g=self.g, causal=self.causal,
                                        tau=self.tau, force_diag=self.force_diag, force_sink=self.force_sink,
                                        Lq=Lq, Lk=Lk, cu_seqlens=self.cu, max_seqlen=self.max_seqlen,
                                        cu_seqlens_host=self.cu_h, out=self.bitmask, cu_seqlens_k=self.cu_k,
                                        max_seqlen_k=self.max_seqlen_k, cu_seqlens_k_host=self.ck_h)
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
                            cu_seqlens_k=self.cu_k, max_seqlen_k=self.max_seqlen_k,
                            cache_workspace=self.cache_ws if self.int8_cache else None)

    def run(self):
        """One prefill step on the resident inputs; returns the device output."""
        if self.routed:
            self.quantize()
            if not self.external_mask:
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


class HeadShardedPrefill:
    """One prefill problem split by query heads over the ranks of a process
    group (one process per GPU; strong scaling).

    Rank ``rank`` computes the block of consecutive query heads
    ``dist.head_shards(hq, world)[rank]``, cut into ``dist.kv_segments`` so
    that each segment is one ``TileMixPrefill`` whose heads keep the
    library's GQA map; the segments write straight into this rank's output
    slice ``out_local`` [Lq, h_cap, d].  With a seeded mask (p) the routing
    bits of the whole problem are built once per step and each segment reads
    its own heads' rows of them, so every head is routed exactly as in the
    unsharded problem (the bits hash the global head index); with the scale
    policy (tau) each segment's bits depend only on its own heads' scales.
    ``run`` then all-gathers the slices over the group and interleaves them
    into ``out`` [Lq, hq, d] (tm_merge_head_shards).  Ranks exchange nothing
    else.
    """

    def __init__(self, Lq, Lk, hq, hkv, d, *, rank=0, world=1, group=None, causal=True, tile_m=128,
                 tile_n=128, g=1, p=None, seed=0, force_diag=False, force_sink=False, cu_seqlens=None,
                 int8_cache=False, tau=None, cu_seqlens_k=None, device="cuda"):
        if hq % hkv:
            raise ValueError("hq must be a multiple of hkv")
        if not 0 <= rank < world:
            raise ValueError("rank out of range")
        self.shape = (Lq, Lk, hq, hkv, d)
        self.rank, self.world, self.group = rank, world, group
        self.device = torch.device(device)
        shards = dist.head_shards(hq, world)
        self.head_start = [a for a, _ in shards] + [hq]
        self.h0, self.h1 = shards[rank]
        self.h_cap = max(b - a for a, b in shards)
        self.out_local = torch.empty((Lq, self.h_cap, d), dtype=torch.float16, device=self.device)
        self.segments = dist.kv_segments(self.h0, self.h1, hq // hkv)
        kw = dict(causal=causal, tile_m=tile_m, tile_n=tile_n, g=g, force_diag=force_diag,
                  force_sink=force_sink, cu_seqlens=cu_seqlens, int8_cache=int8_cache,
                  cu_seqlens_k=cu_seqlens_k, device=self.device)
        self.p, self.seed = p, seed
        self.full_mask = None
        if p is not None and self.segments:
            # the whole problem's routing bits, one row block per query head
            self._mask_kw = dict(tile_m=tile_m, tile_n=tile_n, g=g, causal=causal, p=p, seed=seed,
                                 force_diag=force_diag, force_sink=force_sink, Lq=Lq, Lk=Lk,
                                 cu_seqlens=None if cu_seqlens is None else cu_seqlens.to(self.device, torch.int32),
                                 cu_seqlens_host=None if cu_seqlens is None else cu_seqlens.to("cpu", torch.int32),
                                 cu_seqlens_k=None if cu_seqlens_k is None
                                 else cu_seqlens_k.to(self.device, torch.int32),
                                 cu_seqlens_k_host=None if cu_seqlens_k is None
                                 else cu_seqlens_k.to("cpu", torch.int32),
                                 device=self.device)
            self.full_mask = ops.build_mask(hq, **self._mask_kw)
        self.subs = []
        for s0, s1, k0, k1 in self.segments:
            out_view = self.out_local[:, s0 - self.h0:s1 - self.h0]
            if p is not None:
                sub = TileMixPrefill(Lq, Lk, s1 - s0, k1 - k0, d, bitmask=self.full_mask[s0:s1], out=out_view,
                                     **kw)
            else:
                sub = TileMixPrefill(Lq, Lk, s1 - s0, k1 - k0, d, tau=tau, out=out_view, **kw)
            self.subs.append(sub)
        if world > 1:
            self.gathered = torch.empty((world, Lq, self.h_cap, d), dtype=torch.float16, device=self.device)
            self.out = torch.empty((Lq, hq, d), dtype=torch.float16, device=self.device)
        else:
            self.gathered = None
            self.out = self.out_local
        self.launches_per_step = (sum(x.launches_per_step for x in self.subs)
                                  + (1 if self.full_mask is not None else 0) + (1 if world > 1 else 0))

    def slice_inputs(self, q, k=None, v=None, kv_cache=None, pin=False):
        """This rank's heads of the whole problem's inputs (q [Lq, hq, d];
        k, v [Lk, hkv, d] or the INT8 cache (k_codes, k_scales, v_codes,
        v_scales)), one contiguous (q, k, v, kv_cache) per segment; pinned
        when pin is set (host tensors that a step then uploads)."""
        def cut(x, a, b):
            if x is None:
                return None
            y = x[:, a:b].contiguous()
            return y.pin_memory() if pin else y
        out = []
        for s0, s1, k0, k1 in self.segments:
            kv = None if kv_cache is None else tuple(cut(x, k0, k1) for x in kv_cache)
            out.append((cut(q, s0, s1), cut(k, k0, k1), cut(v, k0, k1), kv))
        return out

    def load_slices(self, slices):
        """Copy per-segment inputs (as returned by slice_inputs) into the
        segments' buffers."""
        for (q, k, v, kv), sub in zip(slices, self.subs):
            sub.load(q, k, v, kv)

    def load(self, q, k=None, v=None, kv_cache=None):
        """Copy this rank's heads of the whole problem's inputs (device or
        host tensors) into the segments' buffers."""
        for (s0, s1, k0, k1), sub in zip(self.segments, self.subs):
            kv = None if kv_cache is None else tuple(x[:, k0:k1] for x in kv_cache)
            sub.load(q[:, s0:s1], None if k is None else k[:, k0:k1], None if v is None else v[:, k0:k1], kv)

    def input_bytes(self):
        return sum(sub.input_bytes() for sub in self.subs)

    def output_bytes(self):
        return self.out.numel() * self.out.element_size()

    def run_local(self):
        """This rank's heads: routing bits, then every segment's step, into
        out_local."""
        if self.full_mask is not None:
            ops.build_mask(self.shape[2], out=self.full_mask, **self._mask_kw)
        for sub in self.subs:
            sub.run()
        return self.out_local

    def gather(self):
        return dist.all_gather_heads(self.gathered, self.out_local, self.group)

    def merge(self):
        return ops.merge_head_shards(self.out, self.gathered, self.head_start)

    def run(self):
        """One step: this rank's heads, the all-gather, the interleaving copy.
        Returns the whole [Lq, hq, d] output (every rank holds it)."""
        self.run_local()
        if self.world > 1:
            self.gather()
            self.merge()
        return self.out


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
