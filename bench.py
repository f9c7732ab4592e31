#!/usr/bin/env python
"""Benchmark of tile-routed FP16/INT8 fused prefill attention on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload sweep|long|varlen|mlx|tiny] [--p P]

One step = one pass of the whole hot path over one seeded synthetic batch:
per-tile INT8 quantisation of Q and K, the seeded routing bitmask, and the
fused attention kernel (for an all-FP16 workload only the attention kernel).
Default workload: the TileMix routing sweep shape (L = 16384, Hq = 32,
Hkv = 8, d = 128, causal, 128x128 tiles, g = 4, outlier channels x20,
diagonal and sink groups FP16) at INT8 group probability 0.75.

Prints ONE JSON line (rank 0).  `value` is the whole-job algorithmic
TFLOP/s: 4 * d FLOP per visible query-key pair (QK^T and P.V, causal-aware),
the same convention as the tflops column of the MLX fused-SDPA tables,
summed over all ranks and divided by the max-over-ranks device time.
With N > 1 every rank processes its own independently seeded batch of the
same shape (weak scaling, no collective on the data path).

`--impl reference` times the CPU oracle (fp64 NumPy) on the host cores
instead, one sampled (query tile, head) pair of the same workload per step.
"""

from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import threading
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from mixed_precision_attention_tm_b200 import dist, inputs  # noqa: E402

# ncu summaries of the kernel each workload's attention runs: the routing
# sweep's routed launches run the one-query-tile kernel (tm_attn3.cu), the
# INT8-cache workload the two-query-tile kernel on the expanded cache
# (tm_attn2.cu) after the expansion (tm_cache_expand.cu).  A summary records
# the hash of those sources; a changed kernel reports no traffic.
PROFILE = os.path.join(ROOT, "profiles", "attn_split_routing_sweep.md")
PROFILE_CACHE = os.path.join(ROOT, "profiles", "attn_pair_toks_varlen_int8_cache.md")
KERNEL_SOURCES = [os.path.join(ROOT, "mixed_precision_attention_tm_b200", "csrc", f)
                  for f in ("tm_attn3.cu", "tm_device.cuh")]
CACHE_SOURCES = [os.path.join(ROOT, "mixed_precision_attention_tm_b200", "csrc", f)
                 for f in ("tm_attn2.cu", "tm_device.cuh", "tm_cache_expand.cu")]


def kernel_source_hash(sources=None):
    import hashlib
    h = hashlib.sha256()
    for f in (sources or KERNEL_SOURCES):
        with open(f, "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def profiled_traffic(profile=PROFILE, sources=None):
    """DRAM bytes per attention launch from the committed ncu summary, or
    None when the kernel sources changed since that capture."""
    if not os.path.exists(profile):
        return None, "no committed capture"
    fields = {}
    for line in open(profile):
        if line.startswith("- ") and ":" in line:
            k, v = line[2:].split(":", 1)
            fields[k.strip().strip("`")] = v.strip().strip("`")
    if fields.get("kernel_source_sha256") != kernel_source_hash(sources):
        return None, "kernel changed since the committed capture"
    try:
        return float(fields["dram_bytes_per_launch"]), fields.get("workload", "")
    except (KeyError, ValueError):
        return None, "capture summary unreadable"

FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
NOMINAL = {"f16_tflops": 2250.0, "i8_tops": 4500.0}


# ---------------------------------------------------------------------------
def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


class ClockSampler:
    """nvidia-smi clock / throttle sampling while the timed region runs."""
    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.hw_slowdown,"
              "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
              "clocks_event_reasons.sw_power_cap")
    NAMES = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")

    def __init__(self, device_index):
        self.samples = []
        self.proc = None
        try:
            uuid = str(torch.cuda.get_device_properties(device_index).uuid)
            ident = uuid if uuid.startswith("GPU-") else f"GPU-{uuid}"
        except Exception:
            ident = str(device_index)
        self.cmd = ["nvidia-smi", "-i", ident, f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                    "-lms", "100"]

    def start(self):
        try:
            self.proc = subprocess.Popen(self.cmd, stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
        except Exception:
            self.proc = None

    def _read(self):
        for line in self.proc.stdout:
            parts = [x.strip() for x in line.split(",")]
            if len(parts) >= 7:
                self.samples.append(parts)

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        return self.summary()

    def summary(self):
        """Median SM clock, the highest max clock seen and every throttle
        reason reported active, from the parsed nvidia-smi rows."""
        sm = [float(s[0]) for s in self.samples if s[0].replace(".", "").isdigit()]
        mx = [float(s[1]) for s in self.samples if s[1].replace(".", "").isdigit()]
        reasons = set()
        for s in self.samples:
            for name, val in zip(self.NAMES, s[3:7]):
                if val.lower().startswith("active"):
                    reasons.add(name)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(mx) if mx else None,
                "reasons": sorted(reasons), "samples": len(self.samples)}


# ---------------------------------------------------------------------------
def make_workload(name, p, seed):
    """p: INT8 group probability; None takes the workload's configured one
    (routing sweep 0.75, long context 0.5, varlen and prefix 0.75)."""
    if name == "sweep":
        return inputs.routing_sweep(p if p is not None else 0.75, seed=seed)
    if name == "long":
        return inputs.long_context(p=p if p is not None else 0.5, seed=seed)
    if name == "varlen":
        return inputs.varlen_int8_cache(p=p if p is not None else 0.75, seed=seed)
    if name == "prefix":
        return inputs.prefix_int8_cache(p=p if p is not None else 0.75, seed=seed)
    if name == "mlx":
        return inputs.mlx_shape(4096, 4096, 128, 32, 8, True, seed=seed)
    if name == "tiny":
        return inputs.tiny(seed=seed, p=p)
    raise ValueError(name)


L2_BYTES = 126 * 1000 * 1000
FLUSH_BYTES = 256 << 20


def flush_l2(buf):
    """Evicts the inputs from L2 before a timed step (outside its events):
    writes a buffer of twice the L2 size and then reads it back, so that the
    lines left in L2 are clean and the timed step does not pay for writing
    the flush buffer back to HBM."""
    buf.zero_()
    buf.view(torch.int64).amax()


def step_input_bytes(w):
    """Bytes a step reads from its resident inputs (Q, K, V or the cache)."""
    t = [w.q] + ([w.k, w.v] if w.kv_cache is None else list(w.kv_cache))
    return sum(x.numel() * x.element_size() for x in t if x is not None)


def needs_flush(w):
    return step_input_bytes(w) < 2 * L2_BYTES


def data_note(w):
    """How the workload's synthetic inputs were drawn."""
    parts = ["seeded N(0,1) fp16"]
    if "outlier_channels" in w.extra:
        parts.append("4 outlier channels per KV head x20")
    if "outlier_tokens" in w.extra:
        parts.append(f"{w.extra['outlier_tokens']} outlier key tokens x20")
    if w.kv_cache is not None:
        parts.append("K/V as a per-token INT8 cache")
    return "synthetic (" + ", ".join(parts) + ")"


def describe(w):
    cfg = {"workload": w.name, "Lq": w.Lq, "Lk": w.Lk, "Hq": w.hq, "Hkv": w.hkv, "d": w.d, "causal": w.causal,
           "tile_m": w.tile_m, "tile_n": w.tile_n, "g": w.g, "int8_group_probability": w.p,
           "force_diag": w.force_diag, "force_sink": w.force_sink,
           "l2": ("inputs smaller than twice L2: a 256 MiB buffer is written and read back before every timed "
                  "step, outside the per-step events" if needs_flush(w) else "inputs larger than L2 (126 MB), no flush")}
    if w.lens is not None:
        cfg["seq_lens"] = [int(x) for x in w.lens]
        cfg["int8_kv_cache"] = w.kv_cache is not None
    if w.lens_k is not None:
        cfg["key_lens"] = [int(x) for x in w.lens_k]
    return cfg


def route_stats_of(w, mask_host):
    from mixed_precision_attention_tm_b200 import ops
    cu = None if w.cu_seqlens is None else w.cu_seqlens.numpy()
    ck = None if w.cu_seqlens_k is None else w.cu_seqlens_k.numpy()
    return ops.route_stats(mask_host, Hq=w.hq, tile_m=w.tile_m, tile_n=w.tile_n, g=w.g, causal=w.causal,
                           Lq=w.Lq, Lk=w.Lk, cu_seqlens_host=cu, cu_seqlens_k_host=ck)


def quant_bytes(plan):
    """Algorithmic HBM bytes of one quantiser launch: the fp16 operands read
    once, their int8 codes and fp32 tile scales written once."""
    n = 0
    for x, quant in ((plan.q, plan.q_quant), (plan.k, plan.k_quant)):
        if x is None or quant is None:
            continue
        n += x.numel() * 2 + quant[0].numel() + quant[1].numel() * 4
    return n


def roofline_time(d, n_vis, e8, p16, p8):
    """Mix-weighted tensor roofline (seconds): QK^T of FP16 pairs at p16, of
    INT8 pairs at p8, and P.V of every pair at p16 (FLOP/s)."""
    e16 = n_vis - e8
    return 2 * d * e16 / p16 + 2 * d * e8 / p8 + 2 * d * n_vis / p16


# ---------------------------------------------------------------------------
def run_ours(args, rank, world, local_rank):
    from mixed_precision_attention_tm_b200 import ops
    from mixed_precision_attention_tm_b200.api import TileMixPrefill

    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    peaks, peak_src = load_peaks()
    ops.set_attn_kernel({"auto": ops.ATTN_KERNEL_AUTO, "two": ops.ATTN_KERNEL_TWO_TILE,
                         "one": ops.ATTN_KERNEL_ONE_TILE}[args.attn_kernel])
    w = make_workload(args.workload, args.p, seed=dist.rank_seed(args.seed, rank))
    plan = TileMixPrefill(w.Lq, w.Lk, w.hq, w.hkv, w.d, causal=w.causal, tile_m=w.tile_m, tile_n=w.tile_n,
                          g=w.g, p=w.p, seed=w.mask_seed, force_diag=w.force_diag, force_sink=w.force_sink,
                          cu_seqlens=w.cu_seqlens, int8_cache=w.kv_cache is not None, device=dev,
                          cu_seqlens_k=w.cu_seqlens_k)
    plan.load(w.q, w.k, w.v, w.kv_cache)
    torch.cuda.synchronize()

    stream = torch.cuda.current_stream()
    for _ in range(args.warmup):
        plan.run()
    torch.cuda.synchronize()
    if ops.get_device_error() != ops.TM_OK:
        raise RuntimeError("device error after warm-up")

    # routing statistics of the mask the step builds
    mask_host = None
    if plan.routed:
        mask_host = plan.bitmask.cpu().numpy().view(np.uint32)
    n_vis, e8 = route_stats_of(w, mask_host)
    flops = 4.0 * w.d * n_vis

    K = args.steps
    ev_a = [torch.cuda.Event(enable_timing=True) for _ in range(K)]
    ev_b = [torch.cuda.Event(enable_timing=True) for _ in range(K)]
    ev_qa = [torch.cuda.Event(enable_timing=True) for _ in range(K)]
    ev_qb = [torch.cuda.Event(enable_timing=True) for _ in range(K)]
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    clocks = ClockSampler(local_rank)
    dist.barrier()
    torch.cuda.synchronize()
    flush = torch.empty(FLUSH_BYTES, dtype=torch.uint8, device=dev) if needs_flush(w) else None
    st_a = [torch.cuda.Event(enable_timing=True) for _ in range(K)] if flush is not None else None
    st_b = [torch.cuda.Event(enable_timing=True) for _ in range(K)] if flush is not None else None
    clocks.start()
    time.sleep(0.3)
    t0.record(stream)
    for i in range(K):
        if flush is not None:
            flush_l2(flush)                    # evict the inputs from L2 (outside the step's events)
            st_a[i].record(stream)
        if plan.routed:
            ev_qa[i].record(stream)
            plan.quantize()
            ev_qb[i].record(stream)
            plan.mask()
        ev_a[i].record(stream)
        plan.attend()
        ev_b[i].record(stream)
        if flush is not None:
            st_b[i].record(stream)
    t1.record(stream)
    torch.cuda.synchronize()
    clk = clocks.stop()
    dist.barrier()
    total_ms = t0.elapsed_time(t1)
    if flush is not None:
        total_ms = sum(a.elapsed_time(b) for a, b in zip(st_a, st_b))
    attn_ms = sum(a.elapsed_time(b) for a, b in zip(ev_a, ev_b)) / K
    quant_ms = sum(a.elapsed_time(b) for a, b in zip(ev_qa, ev_qb)) / K if plan.routed else 0.0
    if ops.get_device_error() != ops.TM_OK:
        raise RuntimeError("device error in timed region")
    total_ms, attn_ms, quant_ms = dist.max_over_ranks([total_ms, attn_ms, quant_ms], device=dev)
    ms_step = total_ms / K
    value = dist.job_throughput(world, flops, ms_step)
    if world == 1:
        w.extra["gpu_out"] = plan.out.cpu()      # the last timed step's output, for the parity sample

    # roofline of the attention kernel (dominant launch)
    p16 = float(peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"])) * 1e12
    p8 = 2.0 * p16                              # nominal INT8 : FP16 dense ratio (4.5 : 2.25)
    t_roof = roofline_time(w.d, n_vis, e8, p16, p8)
    peak_eff = flops / t_roof / 1e12
    achieved = flops / (attn_ms * 1e-3) / 1e12
    t_roof_nom = roofline_time(w.d, n_vis, e8, NOMINAL["f16_tflops"] * 1e12, NOMINAL["i8_tops"] * 1e12)

    # end-to-end through the public API from pinned host memory: every step
    # uploads its inputs and downloads its output (HostPipeline overlaps the
    # copies of neighbouring steps with the compute of the current one)
    e2e = None
    if not args.no_e2e:
        from mixed_precision_attention_tm_b200.api import HostPipeline
        qh = w.q.pin_memory()
        kh = None if w.k is None else w.k.pin_memory()
        vh = None if w.v is None else w.v.pin_memory()
        kvh = None if w.kv_cache is None else tuple(x.pin_memory() for x in w.kv_cache)
        pipe = HostPipeline(w.Lq, w.Lk, w.hq, w.hkv, w.d, causal=w.causal, tile_m=w.tile_m, tile_n=w.tile_n,
                            g=w.g, p=w.p, seed=w.mask_seed, force_diag=w.force_diag, force_sink=w.force_sink,
                            cu_seqlens=w.cu_seqlens, int8_cache=w.kv_cache is not None, device=dev,
                          cu_seqlens_k=w.cu_seqlens_k)
        outs = [torch.empty(plan.out.shape, dtype=torch.float16, pin_memory=True) for _ in range(2)]
        ke = max(4, min(K, 20))
        step_in = [(qh, kh, vh, kvh)]
        pipe.run(step_in * 2, outs)
        torch.cuda.synchronize()
        dist.barrier()
        s0, s1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        s0.record(pipe.h2d)
        last = pipe.run(step_in * ke, [outs[i % 2] for i in range(ke)])
        pipe.d2h.wait_event(last)
        s1.record(pipe.d2h)
        torch.cuda.synchronize()
        if ops.get_device_error() != ops.TM_OK:
            raise RuntimeError("device error in the end-to-end run")
        (te,) = dist.max_over_ranks([s0.elapsed_time(s1) / ke], device=dev)
        e2e = {"value": dist.job_throughput(world, flops, te), "unit": "TFLOP/s",
               "ms_per_step": te, "h2d_bytes_per_step": pipe.input_bytes(),
               "d2h_bytes_per_step": pipe.output_bytes(), "steps": ke,
               "path": "api.HostPipeline (pinned host -> device, prefill step, device -> host; copies of "
                       "neighbouring steps overlapped)"}
        del pipe

    # INT8-fraction sweep (outside the timed region; context for the metric)
    sweep = None
    if args.workload == "sweep" and not args.no_sweep:
        sweep = []
        for ps in (0.0, 0.25, 0.5, 0.75, 1.0):
            ws = inputs.Workload(w.name, w.q, w.k, w.v, w.hq, w.hkv, w.d, w.causal, w.tile_m, w.tile_n, w.g, ps,
                                 mask_seed=w.mask_seed, force_diag=True, force_sink=True)
            pl = TileMixPrefill(ws.Lq, ws.Lk, ws.hq, ws.hkv, ws.d, causal=True, tile_m=128, tile_n=128, g=ws.g,
                                p=ps, seed=ws.mask_seed, force_diag=True, force_sink=True, device=dev)
            pl.q, pl.k, pl.v = plan.q, plan.k, plan.v
            for _ in range(3):
                pl.run()
            torch.cuda.synchronize()
            mh = pl.bitmask.cpu().numpy().view(np.uint32)
            nv_s, e8_s = route_stats_of(ws, mh)
            ns = max(5, min(K, 30))
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a_ms = 0.0
            for _ in range(ns):
                pl.quantize()
                pl.mask()
                a.record(stream)
                pl.attend()
                b.record(stream)
                b.synchronize()
                a_ms += a.elapsed_time(b)
            a_ms /= ns
            fl = 4.0 * ws.d * nv_s
            tr = roofline_time(ws.d, nv_s, e8_s, p16, p8)
            sweep.append({"p": ps, "realised_int8_fraction": e8_s / nv_s, "attn_ms": a_ms,
                          "tflops": fl / (a_ms * 1e-3) / 1e12, "mixed_roofline_frac": tr / (a_ms * 1e-3),
                          "tokens_per_s": ws.Lq / (a_ms * 1e-3)})
            del pl

    # secondary bounds: instruction rates probed on this GPU, turned into
    # floors for this workload at the clock sampled during the timed region
    secondary = None
    try:
        rates = ops.probe_rates()
        sms = torch.cuda.get_device_properties(dev).multi_processor_count
        f_hz = float(clk.get("sm_mhz") or clk.get("sm_max_mhz") or 1965.0) * 1e6
        per_sm_clk = lambda cyc: 4 * 32 / cyc            # values per clock per SM (4 sub-partitions)
        ex2 = per_sm_clk(rates["ex2_cycles_per_warp_instr"])
        cvt = per_sm_clk(rates["cvt_s32_f32_cycles_per_warp_instr"])
        mag = per_sm_clk(rates["magic_conversion_cycles_per_warp_value"])
        secondary = {
            "probe": rates,
            "sm_clock_mhz": f_hz / 1e6,
            "exp2_per_clk_per_sm": ex2,
            "exp_floor_ms_all_mufu": n_vis / (ex2 * sms * f_hz) * 1e3,
            "exp_floor_ms_mufu_share": 5.0 / 8.0 * n_vis / (ex2 * sms * f_hz) * 1e3,
            "int8_pair_conversion_floor_ms_cvt": e8 / (cvt * sms * f_hz) * 1e3,
            "int8_pair_conversion_floor_ms_kernel": e8 / (mag * sms * f_hz) * 1e3,
            "mma_f16_tflops_back_to_back": 2.0 * 128 * 128 * 16 / rates["mma_f16_m128n128k16_cycles"]
                                           * sms * f_hz / 1e12,
            "note": "exp: one exp2 per visible pair; the kernels evaluate 3 of every 8 on the FMA pipe "
                    "(mufu_share); conversion: the floor one int32->fp32 per INT8-routed pair would set "
                    "in the softmax -- the two-tile and one-tile kernels take INT8 scores from the "
                    "tensor core already in fp32 (exact seed / unseed MMAs) and pay none of it; the "
                    "64-row kernel and the in-kernel INT8-cache conversion kernel still convert",
        }
    except Exception as exc:                                   # a probe failure must not hide the run
        secondary = {"unavailable": str(exc)}

    # roofline of the quantiser launch (Q and K in one launch): HBM-bound,
    # 2 bytes read + 1 byte of code written per element, plus the tile scales
    roofline_quant = None
    if plan.routed and quant_ms > 0:
        qbytes = quant_bytes(plan)
        hbm = float(peaks.get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"]))
        ach = qbytes / (quant_ms * 1e-3) / 1e9
        roofline_quant = {"bound": "hbm", "achieved": ach, "peak": hbm, "unit": "GB/s", "frac": ach / hbm,
                          "traffic": None, "bytes_per_launch": qbytes, "ms_per_launch": quant_ms,
                          "peak_source": f"{peak_src} copy bandwidth",
                          "traffic_note": "algorithmic bytes: fp16 Q and K read once, int8 codes and fp32 "
                                          "tile scales written once"}

    launches = plan.launches_per_step * K
    traffic, traffic_note = (None, "traffic captured for the routing-sweep and INT8-cache workloads only")
    if args.workload == "sweep" and w.p == 0.75:
        traffic, traffic_note = profiled_traffic()
    elif args.workload == "varlen" and w.p == 0.75:
        traffic, traffic_note = profiled_traffic(PROFILE_CACHE, CACHE_SOURCES)
    line = {
        "metric": "prefill attention TFLOPS (tile-routed FP16/INT8 QK^T, FP16 P.V)",
        "value": value,
        "unit": "TFLOP/s",
        "n_gpus": world,
        "steps": K,
        "warmup": args.warmup,
        "ms_per_step": ms_step,
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "f16+i8 (fp32 accumulate)",
        "data": data_note(w),
        "config": describe(w),
        "tokens_per_s": world * w.Lq / (ms_step * 1e-3),
        "realised_int8_fraction": e8 / n_vis,
        "visible_pairs": n_vis,
        "attn_ms": attn_ms,
        "attn_launches": ("cache expansion + attention (the INT8 cache's fp16 view written once into the plan's "
                          "workspace, then the attention kernel); the roofline charges both"
                          if getattr(plan, "cache_ws", None) is not None else "attention kernel"),
        "mixed_roofline_frac_of_measured": t_roof / (attn_ms * 1e-3),
        "mixed_roofline_frac_of_nominal": t_roof_nom / (attn_ms * 1e-3),
        "quant_ms": quant_ms,
        "roofline_quant": roofline_quant,
        "roofline": {"bound": "tensor", "achieved": achieved, "peak": peak_eff, "unit": "TFLOP/s",
                     "frac": achieved / peak_eff, "traffic": traffic, "traffic_note": traffic_note,
                     "peak_source": f"{peak_src} bf16 burst {p16 / 1e12:.1f} TFLOP/s for FP16 pairs, x2 "
                                    "(nominal INT8:FP16 ratio) for INT8 QK^T, mix-weighted by visible pairs"},
        "gpu_launches": launches,
        "clocks": clk,
        "secondary_bounds": secondary,
    }
    if e2e is not None:
        line["e2e"] = e2e
    if sweep is not None:
        line["sweep"] = sweep
    if args.attn_kernel != "auto":
        line["config"]["attn_kernel"] = args.attn_kernel
    if w.kv_cache is None and w.cu_seqlens is None and w.tile_m == 128 and w.tile_n == 128:
        # which 128 x 128-tile kernel the step's attention ran (tm_attn_kernel_choice)
        kc = ops.attn_kernel_choice(w.Lq, w.Lk, w.hq, w.d, routed=plan.routed, causal=w.causal)
        line["attn_kernel"] = {ops.ATTN_KERNEL_TWO_TILE: "two query tiles per CTA",
                               ops.ATTN_KERNEL_ONE_TILE: "one query tile per CTA"}[kc]
    return line, w


def run_sharded(args, rank, world, local_rank):
    """One problem split by query heads over the ranks (strong scaling):
    every rank holds the same seeded workload, computes its block of query
    heads (api.HeadShardedPrefill) and ends each step with the whole output,
    through one all-gather and the library's interleaving copy, both inside
    the timed step."""
    from mixed_precision_attention_tm_b200 import ops
    from mixed_precision_attention_tm_b200.api import HeadShardedPrefill

    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    peaks, peak_src = load_peaks()
    w = make_workload(args.workload, args.p, seed=args.seed)     # one problem, the same on every rank
    plan = HeadShardedPrefill(w.Lq, w.Lk, w.hq, w.hkv, w.d, rank=rank, world=world, causal=w.causal,
                              tile_m=w.tile_m, tile_n=w.tile_n, g=w.g, p=w.p, seed=w.mask_seed,
                              force_diag=w.force_diag, force_sink=w.force_sink, cu_seqlens=w.cu_seqlens,
                              int8_cache=w.kv_cache is not None, cu_seqlens_k=w.cu_seqlens_k, device=dev)
    plan.load(w.q, w.k, w.v, w.kv_cache)
    torch.cuda.synchronize()
    stream = torch.cuda.current_stream()
    for _ in range(args.warmup):
        plan.run()
    torch.cuda.synchronize()
    if ops.get_device_error() != ops.TM_OK:
        raise RuntimeError("device error after warm-up")

    # work of the whole problem and of this rank's heads
    cu = None if w.cu_seqlens is None else w.cu_seqlens.numpy()
    ck = None if w.cu_seqlens_k is None else w.cu_seqlens_k.numpy()
    full_host = None if plan.full_mask is None else plan.full_mask.cpu().numpy().view(np.uint32)

    def stats(h0, h1):
        if h1 <= h0:
            return 0.0, 0.0
        m = None if full_host is None else np.ascontiguousarray(full_host[h0:h1])
        return ops.route_stats(m, Hq=h1 - h0, tile_m=w.tile_m, tile_n=w.tile_n, g=w.g, causal=w.causal,
                               Lq=w.Lq, Lk=w.Lk, cu_seqlens_host=cu, cu_seqlens_k_host=ck)
    n_vis_r, e8_r = stats(plan.h0, plan.h1)
    n_vis, e8 = n_vis_r, e8_r
    if world > 1:
        t = torch.tensor([n_vis_r, e8_r], dtype=torch.float64, device=dev)
        torch.distributed.all_reduce(t)
        n_vis, e8 = float(t[0]), float(t[1])
    flops = 4.0 * w.d * n_vis

    K = args.steps
    st_a = [torch.cuda.Event(enable_timing=True) for _ in range(K)]
    st_b = [torch.cuda.Event(enable_timing=True) for _ in range(K)]
    at_a = [[torch.cuda.Event(enable_timing=True) for _ in plan.subs] for _ in range(K)]
    at_b = [[torch.cuda.Event(enable_timing=True) for _ in plan.subs] for _ in range(K)]
    flush = torch.empty(FLUSH_BYTES, dtype=torch.uint8, device=dev) if needs_flush(w) else None
    clocks = ClockSampler(local_rank)
    dist.barrier()
    torch.cuda.synchronize()
    clocks.start()
    time.sleep(0.3)
    for i in range(K):
        if flush is not None:
            flush_l2(flush)
        st_a[i].record(stream)
        if plan.full_mask is not None:
            ops.build_mask(w.hq, out=plan.full_mask, **plan._mask_kw)
        for j, sub in enumerate(plan.subs):
            if sub.routed:
                sub.quantize()
            at_a[i][j].record(stream)
            sub.attend()
            at_b[i][j].record(stream)
        if world > 1:
            plan.gather()
            plan.merge()
        st_b[i].record(stream)
    torch.cuda.synchronize()
    clk = clocks.stop()
    dist.barrier()
    if ops.get_device_error() != ops.TM_OK:
        raise RuntimeError("device error in timed region")
    step_ms = sum(a.elapsed_time(b) for a, b in zip(st_a, st_b)) / K
    attn_ms = sum(a.elapsed_time(b) for i in range(K) for a, b in zip(at_a[i], at_b[i])) / K
    step_max, attn_max = dist.max_over_ranks([step_ms, attn_ms], device=dev)
    value = flops / (step_max * 1e-3) / 1e12

    p16 = float(peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"])) * 1e12
    p8 = 2.0 * p16
    flops_r = 4.0 * w.d * n_vis_r
    t_roof_r = roofline_time(w.d, n_vis_r, e8_r, p16, p8) if n_vis_r else 0.0
    peak_eff = flops_r / t_roof_r / 1e12 if t_roof_r else None
    achieved = flops_r / (attn_ms * 1e-3) / 1e12 if attn_ms > 0 else 0.0

    e2e = None
    if not args.no_e2e:
        slices = plan.slice_inputs(w.q, w.k, w.v, w.kv_cache, pin=True)
        out_h = torch.empty(plan.out.shape, dtype=torch.float16, pin_memory=True)
        ke = max(4, min(K, 20))
        for _ in range(2):
            plan.load_slices(slices)
            plan.run()
            out_h.copy_(plan.out, non_blocking=True)
        torch.cuda.synchronize()
        dist.barrier()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(ke):
            plan.load_slices(slices)
            plan.run()
            out_h.copy_(plan.out, non_blocking=True)
        e1.record(stream)
        torch.cuda.synchronize()
        (te,) = dist.max_over_ranks([e0.elapsed_time(e1) / ke], device=dev)
        e2e = {"value": flops / (te * 1e-3) / 1e12, "unit": "TFLOP/s", "ms_per_step": te,
               "h2d_bytes_per_step": plan.input_bytes(), "d2h_bytes_per_step": plan.output_bytes(),
               "steps": ke, "path": "api.HeadShardedPrefill (this rank's heads from pinned host memory, "
                                    "its step, the all-gather and interleave, the whole output to the host; "
                                    "no overlap between steps)"}

    cfg = describe(w)
    cfg["parallelism"] = f"query heads over {world} rank(s)"
    cfg["head_shards"] = [plan.head_start[r + 1] - plan.head_start[r] for r in range(world)]
    line = {
        "metric": "prefill attention TFLOPS (tile-routed FP16/INT8 QK^T, FP16 P.V)",
        "value": value,
        "unit": "TFLOP/s",
        "n_gpus": world,
        "steps": K,
        "warmup": args.warmup,
        "ms_per_step": step_max,
        "higher_is_better": True,
        "scaling": "strong",
        "vs_baseline": None,
        "dtype": "f16+i8 (fp32 accumulate)",
        "data": data_note(w),
        "config": cfg,
        "tokens_per_s": w.Lq / (step_max * 1e-3),
        "realised_int8_fraction": e8 / n_vis,
        "visible_pairs": n_vis,
        "attn_ms_rank_max": attn_max,
        "roofline": {"bound": "tensor", "achieved": achieved, "peak": peak_eff, "unit": "TFLOP/s",
                     "frac": None if not peak_eff else achieved / peak_eff, "traffic": None,
                     "traffic_note": "rank 0's attention launches over its own heads; no capture of this mode",
                     "peak_source": f"{peak_src} bf16 burst {p16 / 1e12:.1f} TFLOP/s for FP16 pairs, x2 "
                                    "(nominal INT8:FP16 ratio) for INT8 QK^T, mix-weighted by visible pairs"},
        "gpu_launches": plan.launches_per_step * K,
        "clocks": clk,
    }
    if e2e is not None:
        line["e2e"] = e2e
    return line, w


def cpu_sample_spec(w, n_pairs):
    """Evenly spaced (query tile, head) pairs of the workload."""
    import oracle
    cu = None if w.cu_seqlens is None else w.cu_seqlens.tolist()
    ck = None if w.cu_seqlens_k is None else w.cu_seqlens_k.tolist()
    seqs = oracle.seq_table(w.Lq, w.Lk, cu, ck)
    qt = oracle.tile_table(seqs, w.tile_m, "q")
    out = []
    n = len(qt) * w.hq
    for i in range(n_pairs):
        idx = (i * n) // n_pairs + (n // (2 * n_pairs))
        out.append((qt[(idx // w.hq) % len(qt)], idx % w.hq))
    return seqs, out


def oracle_pair(w, seqs, tile, h, prep):
    """Run the oracle on one (query tile, head): all rows of the tile, the
    head's slice of Q; returns the pair's algorithmic FLOPs and the oracle's
    output rows [rows, d] (fp64)."""
    import oracle
    b, I, r0, rows, ig = tile
    q1 = w.q.numpy()[:, h:h + 1]
    kw = dict(prep)
    if kw.get("mask") is not None:
        kw["mask"] = kw["mask"][h:h + 1]
        qc, qs = kw["q_quant"]
        kw["q_quant"] = (qc[:, h:h + 1], qs[:, h:h + 1])
    hk = h // (w.hq // w.hkv)
    if w.kv_cache is not None:
        kc, ks, vc, vs = kw["kv_cache"]
        kw["kv_cache"] = (kc[:, hk:hk + 1], ks[:, hk:hk + 1], vc[:, hk:hk + 1], vs[:, hk:hk + 1])
        k1 = v1 = None
    else:
        k1, v1 = w.k.numpy()[:, hk:hk + 1], w.v.numpy()[:, hk:hk + 1]
        if kw.get("k_quant") is not None:
            kc, ks = kw["k_quant"]
            kw["k_quant"] = (kc[:, hk:hk + 1], ks[:, hk:hk + 1])
    ref = oracle.attention(q1, k1, v1, rows=range(r0, r0 + rows), **kw)[r0:r0 + rows, 0]
    _qs, lq, _ks, lk = seqs[b]
    ii = I * w.tile_m + np.arange(rows)
    lim = np.minimum(lk - 1, ii + lk - lq) if w.causal else np.full(rows, lk - 1)
    return 4.0 * w.d * float(np.maximum(lim + 1, 0).sum()), ref


def oracle_prep(w, seqs):
    import oracle
    cu = None if w.cu_seqlens is None else w.cu_seqlens.tolist()
    ck = None if w.cu_seqlens_k is None else w.cu_seqlens_k.tolist()
    prep = dict(cu_seqlens=cu, cu_seqlens_k=ck, causal=w.causal, tile_m=w.tile_m, tile_n=w.tile_n, g=w.g)
    if w.kv_cache is not None:
        prep["kv_cache"] = tuple(t.numpy() for t in w.kv_cache)
    if w.p is not None:
        prep["mask"] = oracle.build_mask(w.hq, seqs, w.tile_m, w.tile_n, w.g, w.causal, w.p, w.mask_seed,
                                         w.force_diag, w.force_sink)
        prep["q_quant"] = oracle.quantize_tiles(w.q.numpy(), seqs, w.tile_m, "q")
        if w.kv_cache is None:
            prep["k_quant"] = oracle.quantize_tiles(w.k.numpy(), seqs, w.tile_n, "k")
    return prep


PARITY_BOUND = 3e-3   # max-abs output error of the parity tests (fp16 output, unit-variance inputs)


def cpu_baseline(w, target_s):
    """Time the oracle as it stands on evenly spaced (query tile, head) pairs
    until about target_s seconds of oracle time have run.  When the GPU
    output of the timed steps is at hand (w.extra["gpu_out"]), the same
    sampled rows are compared with it (outside the oracle's time).  Returns
    (cpu_baseline dict, parity dict or None)."""
    cores = len(os.sched_getaffinity(0))
    seqs, _ = cpu_sample_spec(w, 1)
    prep = oracle_prep(w, seqs)            # quantisation and mask: not timed
    n_try = 64
    _, pairs = cpu_sample_spec(w, n_try)
    gpu = w.extra.get("gpu_out")
    flops, dt, err, n_rows, done = 0.0, 0.0, 0.0, 0, 0
    for tile, h in pairs:
        t0 = time.perf_counter()
        f, ref = oracle_pair(w, seqs, tile, h, prep)
        dt += time.perf_counter() - t0
        flops += f
        done += 1
        if gpu is not None:
            r0, rows = tile[2], tile[3]
            got = gpu[r0:r0 + rows, h].to(torch.float64).numpy()
            err = max(err, float(np.abs(got - ref).max()))
            n_rows += rows
        if dt > target_s:
            break
    base = {"value": flops / dt / 1e12, "unit": "TFLOP/s", "cores": cores, "kind": "oracle",
            "sample": f"{done} evenly spaced (query tile, head) pairs of {w.name} (all rows of each tile, "
                      f"fp64 NumPy/BLAS), {dt:.1f} s; quantisation and mask built beforehand, untimed"}
    parity = None
    if gpu is not None:
        parity = {"max_abs_err": err, "bound": PARITY_BOUND, "pass": bool(err <= PARITY_BOUND),
                  "rows_compared": n_rows,
                  "sample": "the cpu_baseline pairs: every row of each sampled (query tile, head), the GPU output "
                            "of the last timed step against the fp64 oracle on the same inputs"}
    return base, parity


def run_reference(args):
    """CPU oracle arm: one (query tile, head) pair of the workload per step."""
    w = make_workload(args.workload, args.p, seed=args.seed)
    cores = len(os.sched_getaffinity(0))
    seqs, pairs = cpu_sample_spec(w, max(1, args.steps + args.warmup))
    prep = oracle_prep(w, seqs)
    for tile, h in pairs[:args.warmup]:
        oracle_pair(w, seqs, tile, h, prep)
    flops = 0.0
    t0 = time.perf_counter()
    for tile, h in pairs[args.warmup:args.warmup + args.steps]:
        flops += oracle_pair(w, seqs, tile, h, prep)[0]
    dt = time.perf_counter() - t0
    value = flops / dt / 1e12
    line = {
        "impl": "reference",
        "metric": "prefill attention TFLOPS (tile-routed FP16/INT8 QK^T, FP16 P.V)",
        "value": value, "unit": "TFLOP/s", "n_gpus": 1, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": dt * 1e3 / max(1, args.steps), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": data_note(w),
        "config": describe(w),
        "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": cores, "kind": "oracle",
                         "sample": f"one (query tile, head) pair of {w.name} per step, fp64 NumPy/BLAS; "
                                   "quantisation and mask built beforehand, untimed"},
        "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    return line


def run_mlx_table(args):
    """All 48 runs of the MLX-shaped all-FP16 configuration (24 shapes x
    causal / non-causal), timed as the MLX table times them: 10 warm-up and
    64 timed calls, median and mean of per-call CUDA-event times.  A 256 MiB
    buffer is written between timed calls so that no call finds its inputs
    in L2 (the flush is outside the timed region)."""
    from mixed_precision_attention_tm_b200 import metrics, ops
    from mixed_precision_attention_tm_b200.api import TileMixPrefill

    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    peaks, peak_src = load_peaks()
    p16 = float(peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"]))
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    rows = []
    for (Lq, Lk, d, hq, hkv) in inputs.MLX_SHAPES:
        for causal in (False, True):
            w = inputs.mlx_shape(Lq, Lk, d, hq, hkv, causal, seed=args.seed)
            plan = TileMixPrefill(w.Lq, w.Lk, w.hq, w.hkv, w.d, causal=w.causal, device=dev)
            plan.load(w.q, w.k, w.v)
            for _ in range(10):
                plan.run()
            torch.cuda.synchronize()
            ts = []
            for _ in range(64):
                flush_l2(flush)
                a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                a.record()
                plan.run()
                b.record()
                b.synchronize()
                ts.append(a.elapsed_time(b))
            if ops.get_device_error() != ops.TM_OK:
                raise RuntimeError(f"device error on {w.name}")
            med, mean = float(np.median(ts)), float(np.mean(ts))
            nvis = metrics.visible_pairs(Lq, Lk, causal) * hq
            alg = metrics.algorithmic_flops(d, nvis) / (med * 1e-3) / 1e12
            mlx = metrics.mlx_flops(1, hq, Lq, Lk, d, causal) / (med * 1e-3) / 1e12
            rows.append({"qsl": Lq, "ksl": Lk, "hdim": d, "n_qh": hq, "n_kvh": hkv, "causal": int(causal),
                         "ms_median": round(med, 4), "ms_mean": round(mean, 4),
                         "tflops_alg": round(alg, 1), "tflops_mlx": round(mlx, 1),
                         "tokens_per_s": round(Lq / (med * 1e-3), 0),
                         "frac_of_fp16_roofline": round(alg / p16, 3)})
            del plan
    return {"metric": "prefill attention TFLOPS, MLX-shaped all-FP16 table", "unit": "TFLOP/s",
            "n_gpus": 1, "dtype": "f16 (fp32 accumulate)", "data": "synthetic (seeded N(0,1) fp16)",
            "timing": "10 warm-up + 64 calls, per-call CUDA events, 256 MiB L2 flush (written, read back) between calls",
            "peak": {"bf16_tflops": p16, "source": peak_src}, "table": rows}


def run_frontier(args):
    """Accuracy-efficiency curve on the routing-sweep inputs: for random
    routing (Bernoulli p) and for the scale policy (INT8 iff s_q * s_k <=
    tau, tau at quantiles of the tile-scale products), the realised INT8
    fraction, the attention time (median of 20 calls) and the output error
    against the all-FP16 output of the same kernel (max, mean and rms of the
    absolute difference over every output element)."""
    from mixed_precision_attention_tm_b200 import ops
    from mixed_precision_attention_tm_b200.api import TileMixPrefill

    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    peaks, peak_src = load_peaks()
    p16 = float(peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"])) * 1e12
    w = (inputs.routing_sweep_token_outliers(0.0, seed=args.seed) if args.frontier_input == "tokens"
         else inputs.routing_sweep(0.0, seed=args.seed))
    common = dict(causal=True, tile_m=128, tile_n=128, g=w.g, force_diag=True, force_sink=True, device=dev)

    def run(**kw):
        pl = TileMixPrefill(w.Lq, w.Lk, w.hq, w.hkv, w.d, **common, **kw)
        pl.load(w.q, w.k, w.v)
        for _ in range(3):
            pl.run()
        torch.cuda.synchronize()
        ts = []
        for _ in range(20):
            if pl.routed:
                pl.quantize()
                pl.mask()
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record()
            pl.attend()
            b.record()
            b.synchronize()
            ts.append(a.elapsed_time(b))
        if ops.get_device_error() != ops.TM_OK:
            raise RuntimeError("device error in the frontier run")
        mh = pl.bitmask.cpu().numpy().view(np.uint32) if pl.routed else None
        nv, e8 = route_stats_of(w, mh)
        return pl, float(np.median(ts)), nv, e8

    ref_plan, ref_ms, nv, _ = run(p=None)
    ref = ref_plan.out.float()

    def point(kind, knob, pl, ms, nv_, e8_):
        diff = (pl.out.float() - ref).abs()
        t_roof = roofline_time(w.d, nv_, e8_, p16, 2.0 * p16)
        return {"policy": kind, "knob": knob, "realised_int8_fraction": e8_ / nv_, "attn_ms": ms,
                "tflops": 4.0 * w.d * nv_ / (ms * 1e-3) / 1e12, "mixed_roofline_frac": t_roof / (ms * 1e-3),
                "err_max_abs": float(diff.max()), "err_mean_abs": float(diff.mean()),
                "err_rms": float(diff.pow(2).mean().sqrt())}

    rows = [point("fp16", None, ref_plan, ref_ms, nv, 0.0)]
    for p in (0.25, 0.5, 0.75, 1.0):
        pl, ms, nv_, e8_ = run(p=p, seed=w.mask_seed)
        rows.append(point("random", p, pl, ms, nv_, e8_))
        del pl
    # tau at quantiles of s_q * s_k over (query tile, head) x (key tile, kv head)
    qc, qs, kc, ks = ops.quantize_qk(ref_plan.q, ref_plan.k, tile_m=128, tile_n=128)
    prods = (qs.reshape(-1, 1) * ks.reshape(1, -1)).flatten()
    qv = torch.tensor([0.2, 0.4, 0.6, 0.8, 0.9, 0.97], device=dev)
    taus = torch.quantile(prods[torch.randperm(prods.numel(), device=dev)[:1 << 20]], qv).tolist()
    for tau in taus + [float("inf")]:
        pl, ms, nv_, e8_ = run(tau=tau)
        rows.append(point("scale", tau, pl, ms, nv_, e8_))
        del pl
    return {"metric": "accuracy-efficiency frontier: output error vs realised INT8 fraction", "unit": "mixed",
            "n_gpus": 1, "workload": w.name, "config": describe(w), "inputs": args.frontier_input,
            "reference": "all-FP16 output of the same kernel on the same inputs",
            "peak": {"bf16_tflops": p16 / 1e12, "source": peak_src}, "points": rows}


def run_fp8_table(args):
    """The FP8 third precision on the routing-sweep inputs: attention time,
    mix-weighted roofline fraction and output error against the all-FP16
    output for FP16-only, INT8-only, FP8-only and three-way routing.  Each
    point's kernel is named: FP8 / FP16 routing runs in the two-tile kernel
    (auto) and in the one-tile kernel; three-way routing in the one-tile
    kernel.  E4M3 QK^T runs at the INT8
    rate, so FP8 pairs take p8 = 2 p16 in the roofline like INT8 pairs.
    Only the attention launch is timed (median of 20 calls, a 256 MiB buffer
    written before each)."""
    from mixed_precision_attention_tm_b200 import ops

    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    peaks, peak_src = load_peaks()
    p16 = float(peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"])) * 1e12
    w = inputs.routing_sweep(0.0, seed=args.seed)
    q, k, v = (x.to(dev) for x in (w.q, w.k, w.v))
    mk = dict(tile_m=128, tile_n=128, g=w.g, causal=True, Lq=w.Lq, Lk=w.Lk, force_diag=True, force_sink=True)
    i8 = ops.quantize_qk(q, k)
    f8 = ops.quantize_qk_fp8(q, k)
    flush = torch.empty(FLUSH_BYTES, dtype=torch.uint8, device=dev)
    out = torch.empty_like(q)

    def timed(fn):
        for _ in range(3):
            fn()
        torch.cuda.synchronize()
        ts = []
        for _ in range(20):
            flush_l2(flush)
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record()
            fn()
            b.record()
            b.synchronize()
            ts.append(a.elapsed_time(b))
        if ops.get_device_error() != ops.TM_OK:
            raise RuntimeError("device error in the FP8 report")
        return float(np.median(ts))

    ref = None
    rows = []

    def point(name, kernel, p8, pf8):
        nonlocal ref
        m8 = None if p8 is None else ops.build_mask(w.hq, p=p8, seed=w.mask_seed, **mk)
        mf8 = None if pf8 is None else ops.build_mask(w.hq, p=pf8, seed=w.mask_seed + 1, **mk)
        ops.set_attn_kernel(kernel)
        try:
            if mf8 is None:
                fn = lambda: ops.attn_fwd(q, k, v, out=out, g=w.g, causal=True, bitmask=m8,  # noqa: E731
                                          q_quant=None if m8 is None else i8[:2],
                                          k_quant=None if m8 is None else i8[2:])
            else:
                fn = lambda: ops.attn_fwd_fp8(q, k, v, out=out, g=w.g, causal=True, bitmask_fp8=mf8,  # noqa: E731
                                              qf8_quant=f8[:2], kf8_quant=f8[2:], bitmask=m8,
                                              q_quant=None if m8 is None else i8[:2],
                                              k_quant=None if m8 is None else i8[2:])
            ms = timed(fn)
        finally:
            ops.set_attn_kernel(ops.ATTN_KERNEL_AUTO)
        h8 = None if m8 is None else m8.cpu().numpy().view(np.uint32)
        hf8 = None if mf8 is None else mf8.cpu().numpy().view(np.uint32)
        nv, e8 = route_stats_of(w, h8)
        ef8 = 0.0
        if hf8 is not None:                           # FP8 where the INT8 bit is clear
            _, ef8 = route_stats_of(w, hf8 if h8 is None else hf8 & ~h8)
        t_roof = roofline_time(w.d, nv, e8 + ef8, p16, 2.0 * p16)
        o = out.float()
        if ref is None:
            ref = o.clone()
        diff = (o - ref).abs()
        rows.append({"point": name, "kernel": {ops.ATTN_KERNEL_AUTO: "auto", ops.ATTN_KERNEL_ONE_TILE: "one-tile",
                                                ops.ATTN_KERNEL_TWO_TILE: "two-tile"}[kernel],
                     "int8_group_probability": p8, "fp8_group_probability": pf8,
                     "realised_int8_fraction": round(e8 / nv, 4), "realised_fp8_fraction": round(ef8 / nv, 4),
                     "attn_ms": round(ms, 4), "tflops": round(4.0 * w.d * nv / (ms * 1e-3) / 1e12, 1),
                     "mixed_roofline_frac": round(t_roof / (ms * 1e-3), 3),
                     "err_max_abs": float(diff.max()), "err_rms": float(diff.pow(2).mean().sqrt())})

    AUTO, ONE = ops.ATTN_KERNEL_AUTO, ops.ATTN_KERNEL_ONE_TILE
    if args.fp8_only is not None:
        # one FP8-only point (no error reference: its error fields are
        # against its own output)
        point("fp8", AUTO, None, args.fp8_only)
        return {"metric": "FP8 third precision: attention time by route mix", "unit": "mixed", "n_gpus": 1,
                "workload": w.name, "config": describe(w),
                "peak": {"bf16_tflops": p16 / 1e12, "source": peak_src}, "points": rows}
    point("fp16", AUTO, None, None)                   # the error reference
    point("fp16", ONE, None, None)
    point("int8", AUTO, 0.75, None)
    point("int8", ONE, 0.75, None)
    point("fp8 plane empty", AUTO, None, 0.0)         # the two-tile kernel's FP8 variant, nothing routed to FP8
    for pf8 in (0.25, 0.5, 0.75, 1.0):
        point("fp8", AUTO, None, pf8)                 # FP8 and FP16 only: the two-tile kernel
    point("fp8 plane empty", ONE, None, 0.0)          # the one-tile kernel's FP8 variant
    for pf8 in (0.25, 0.5, 0.75, 1.0):
        point("fp8", ONE, None, pf8)
    point("int8 + fp8", ONE, 0.5, 0.5)                # three-way routing: the one-tile kernel
    point("int8 + fp8", ONE, 0.75, 1.0)
    return {"metric": "FP8 third precision: attention time and error by route mix", "unit": "mixed",
            "n_gpus": 1, "workload": w.name, "config": describe(w),
            "reference": "all-FP16 output of the automatically chosen kernel on the same inputs",
            "peak": {"bf16_tflops": p16 / 1e12, "source": peak_src}, "points": rows}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=100)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default="sweep",
                    choices=["sweep", "long", "varlen", "prefix", "mlx", "tiny", "mlx_table", "frontier", "fp8_table"])
    ap.add_argument("--p", type=float, default=None,
                    help="INT8 group probability (default: the workload's configuration: 0.75, long context 0.5)")
    ap.add_argument("--seed", type=int, default=0)
    ap.add_argument("--no-sweep", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=15.0)
    ap.add_argument("--shard", default="batch", choices=["batch", "heads"],
                    help="batch: every rank runs its own seeded problem (weak scaling); heads: one problem "
                         "split by query heads over the ranks, output all-gathered (strong scaling)")
    ap.add_argument("--fp8-only", type=float, default=None,
                    help="FP8 report: time only the FP8-only route at this group probability")
    ap.add_argument("--attn-kernel", default="auto", choices=["auto", "two", "one"],
                    help="128 x 128-tile attention kernel: the library's automatic choice (default), the "
                         "two-query-tile or the one-query-tile kernel (tm_set_attn_kernel)")
    ap.add_argument("--frontier-input", default="channels", choices=["channels", "tokens"],
                    help="frontier report: outlier channels in every token (the routing sweep's inputs) "
                         "or outliers in 0.2%% of the key tokens")
    args = ap.parse_args()
    args.warmup = max(args.warmup, 3)

    rank, local_rank, world = dist.world_info()

    if args.workload in ("mlx_table", "frontier", "fp8_table"):   # reports, not the contract's bench line
        if rank == 0:
            fn = {"mlx_table": run_mlx_table, "frontier": run_frontier, "fp8_table": run_fp8_table}[args.workload]
            print(json.dumps(fn(args)), flush=True)
        return

    if args.impl == "reference":
        if rank == 0:
            print(json.dumps(run_reference(args)), flush=True)
        return

    if world > 1:
        import datetime
        torch.cuda.set_device(local_rank)
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                             device_id=torch.device("cuda", local_rank))
    try:
        line, w = (run_sharded if args.shard == "heads" else run_ours)(args, rank, world, local_rank)
        if rank == 0 and world == 1 and not args.no_cpu_baseline:
            line["cpu_baseline"], parity = cpu_baseline(w, args.cpu_seconds)
            if parity is not None:
                line["parity"] = parity
        if rank == 0:
            print(json.dumps(line), flush=True)
    finally:
        if world > 1:
            torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
