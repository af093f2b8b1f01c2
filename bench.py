#!/usr/bin/env python
"""Benchmark: exact tiled GQA attention on B200, Qwen3-8B shapes.

One step = the whole hot path once: attn_prefill on the Qwen3-8B-shaped causal
prefill (B=4, Hq=32, Hkv=8, Lq=Lk=8192, D=128) followed by attn_decode on the
Qwen3-8B-shaped decode batch (B=64, Hq=32, Hkv=8, D=128, cache lengths drawn
uniform in [1024, 32768]).  Inputs are seeded synthetic N(0,1) bf16 tensors,
resident in HBM before the timed region, each larger than the 126 MB L2.

The JSON line's `value` is prefill TFLOP/s (algorithmic FLOPs: visible
query/key pairs only), `decode` holds decode HBM GB/s; both are timed with
CUDA events on the launching stream, per call.  `e2e` repeats the step
through the public Python API with host buffers: pinned-host -> device copies
of the step's inputs (prefill q/k/v, decode q) and device -> host copies of
the outputs (out, lse) inside the timed region; the decode KV cache is
resident device state, as in serving.

Multi-GPU (torchrun): every rank runs the same per-rank workload on its own
GPU (independent sequences -- the path has no exchange step), timing is the
max over ranks, and `value` sums the work of all ranks ("scaling": "weak").

`--impl reference` times the fp64 CPU oracle on a bounded sample of the same
workloads on this host's cores (rank 0 only).
"""
from __future__ import annotations

import argparse
import dataclasses
import json
import os
import statistics
import sys
import threading
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from exact_tiled_attention_gqa_b200 import roofline as RL          # noqa: E402
from exact_tiled_attention_gqa_b200.multigpu import max_over_ranks as _max_over_ranks, rank_seed  # noqa: E402
from exact_tiled_attention_gqa_b200 import workloads as W          # noqa: E402

METRIC = "prefill TFLOP/s & decode HBM GB/s (frac. of roofline), Qwen3-8B GQA shapes"
PREFILL = W.QWEN_PREFILL_8K_B4
DECODE = W.QWEN_DECODE
PREFILL_WORKLOADS = {"qwen3_8b_b4_l8192": W.QWEN_PREFILL_8K_B4, "qwen3_8b_b1_l4096": W.QWEN_PREFILL_4K,
                     "chunked_16k": W.CHUNKED_16K, "chunked_32k": W.CHUNKED_32K, "hd64_b4_l8192": W.HD64_PREFILL,
                     "hd256_b2_l8192": W.HD256_PREFILL}


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=100)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--seed", type=int, default=0)
    ap.add_argument("--no-cpu-baseline", action="store_true", help="skip the oracle timing leg")
    ap.add_argument("--cpu-seconds", type=float, default=12.0, help="target CPU seconds per oracle sample")
    ap.add_argument("--ref-seconds", type=float, default=120.0,
                    help="--impl reference: target CPU seconds for the whole run (warm-up + timed samples)")
    ap.add_argument("--e2e-steps", type=int, default=3)
    ap.add_argument("--only", choices=["prefill", "decode"], default=None,
                    help="profiling aid: time one call type only (the JSON line is then partial)")
    ap.add_argument("--decode-batch", type=int, default=None,
                    help="profiling aid: use the first N sequences of the decode batch")
    ap.add_argument("--decode-cache", choices=["bf16", "e4m3", "q8_0"], default="bf16",
                    help="with --only decode: the cache element format (8-bit caches use attn_decode_kv8)")
    ap.add_argument("--decode-group", type=int, default=None,
                    help="profiling aid: with --only decode, use the group-size sweep shape with this G")
    ap.add_argument("--prefill-workload", choices=sorted(PREFILL_WORKLOADS), default="qwen3_8b_b4_l8192",
                    help="profiling aid: with --only prefill, the prefill workload to time")
    ap.add_argument("--no-sweeps", action="store_true",
                    help="skip the other workloads (group-size decode sweep, other prefill shapes)")
    return ap.parse_args()


# --------------------------------------------------------------------------
# clocks sampled during the timed region
# --------------------------------------------------------------------------
class ClockSampler:
    """Polls SM clock, power and throttle reasons through NVML every ~10 ms
    while the timed region runs.  Without NVML the line's clocks record says
    why and holds no samples."""
    REASONS = {0x4: "sw_power_cap", 0x8: "hw_slowdown", 0x20: "sw_thermal_slowdown",
               0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown"}

    def __init__(self, torch_device_index: int):
        self.dev_index = torch_device_index
        self.samples = []          # (sm_mhz, max_mhz, power_w, reason_bits)
        self._stop = threading.Event()
        self.thread = None
        self.nvml = None
        self.handle = None
        self.error = None

    def _open(self):
        import pynvml
        pynvml.nvmlInit()
        uuid = str(torch.cuda.get_device_properties(self.dev_index).uuid)
        uuid = uuid if uuid.startswith("GPU-") else "GPU-" + uuid
        self.handle = pynvml.nvmlDeviceGetHandleByUUID(uuid.encode())
        self.nvml = pynvml

    def start(self):
        try:
            self._open()
        except Exception as e:   # NVML missing or the UUID lookup failed
            self.error = f"nvml unavailable: {e}"
            return
        self.thread = threading.Thread(target=self._poll, daemon=True)
        self.thread.start()

    def _poll(self):
        n, h = self.nvml, self.handle
        while not self._stop.is_set():
            try:
                sm = n.nvmlDeviceGetClockInfo(h, n.NVML_CLOCK_SM)
                mx = n.nvmlDeviceGetMaxClockInfo(h, n.NVML_CLOCK_SM)
                pw = n.nvmlDeviceGetPowerUsage(h) / 1000.0
                rs = n.nvmlDeviceGetCurrentClocksEventReasons(h)
                self.samples.append((float(sm), float(mx), pw, int(rs)))
            except Exception as e:
                self.error = str(e)
                return
            time.sleep(0.01)

    def stop(self):
        self._stop.set()
        if self.thread is not None:
            self.thread.join(timeout=5)
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [self.error or "no samples"], "samples": 0}
        reasons = set()
        for *_, bits in self.samples:
            for bit, name in self.REASONS.items():
                if bits & bit:
                    reasons.add(name)
        loaded = [s[0] for s in self.samples if s[2] > 300.0] or [s[0] for s in self.samples]
        return {"sm_mhz": statistics.median(loaded), "sm_max_mhz": max(s[1] for s in self.samples),
                "reasons": sorted(reasons), "samples": len(self.samples),
                "power_w_max": round(max(s[2] for s in self.samples), 1)}


# --------------------------------------------------------------------------
# our arm
# --------------------------------------------------------------------------
def run_ours(args, rank, world, local_rank):
    import exact_tiled_attention_gqa_b200 as attn
    from exact_tiled_attention_gqa_b200 import build

    global PREFILL
    if args.prefill_workload != "qwen3_8b_b4_l8192":
        if args.only != "prefill":
            raise SystemExit("--prefill-workload applies to --only prefill")
        PREFILL = PREFILL_WORKLOADS[args.prefill_workload]

    build.build()
    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    dist = None
    if world > 1:
        import torch.distributed as dist_mod
        dist = dist_mod
    peaks = RL.measured_peaks()

    # ---- inputs (per rank: its own sequences; seeds differ by rank) ----
    seed = rank_seed(args.seed, rank)
    if args.only != "decode":
        q_h, k_h, v_h = W.prefill_inputs_for(PREFILL, seed=seed, device="cpu")
        q, k, v = q_h.to(dev), k_h.to(dev), v_h.to(dev)
    if args.only == "prefill":
        dshape = W.DecodeShape(DECODE.name, 1, DECODE.Hq, DECODE.Hkv, 64, DECODE.D, 64, 64)
    elif args.decode_group:
        dshape = W.group_sweep_decode(args.decode_group)
    elif args.decode_batch:
        dshape = W.DecodeShape(DECODE.name + f" (first {args.decode_batch})", args.decode_batch, DECODE.Hq,
                               DECODE.Hkv, DECODE.Lmax, DECODE.D, DECODE.seqlen_lo, DECODE.seqlen_hi)
    else:
        dshape = DECODE
    if args.only == "decode":
        q_h, k_h, v_h = W.prefill_inputs(1, PREFILL.Hq, PREFILL.Hkv, 128, 128, PREFILL.D, seed=seed)
        q, k, v = q_h.to(dev), k_h.to(dev), v_h.to(dev)
    if args.decode_cache != "bf16" and args.only != "decode":
        raise SystemExit("--decode-cache applies to --only decode")
    kv8 = args.decode_cache != "bf16"
    if kv8:
        dshape = dataclasses.replace(dshape, name=dshape.name + f", {args.decode_cache} KV cache")
        dq, dk, dv, dks, dvs, dsl = W.decode_inputs_kv8(dshape.B, dshape.Hq, dshape.Hkv, dshape.Lmax, dshape.D,
                                                        dshape.seqlen_lo, dshape.seqlen_hi, args.decode_cache,
                                                        seed=seed, device=dev)
        dq = dq[:, :, 0].contiguous()
    else:
        dq, dk, dv, dsl = W.decode_inputs_for(dshape, seed=seed, device=dev)
    if args.only is not None:
        print(json.dumps({"profiling_workload": dshape.name if args.only == "decode" else PREFILL.name}), flush=True)
    seqlens_host = dsl.cpu()
    p_flops = RL.prefill_flops(PREFILL.B, PREFILL.Hq, PREFILL.Lq, PREFILL.Lk, PREFILL.D, PREFILL.is_causal)
    d_bytes = (RL.decode_kv8_bytes(seqlens_host.tolist(), dshape.B, dshape.Hq, dshape.Hkv, dshape.D,
                                   args.decode_cache == "q8_0") if kv8 else
               RL.decode_bytes(seqlens_host.tolist(), dshape.B, dshape.Hq, dshape.Hkv, dshape.D))
    p_out = torch.empty_like(q)
    p_lse = torch.empty((PREFILL.B, PREFILL.Hq, PREFILL.Lq), dtype=torch.float32, device=dev)
    d_out = torch.empty_like(dq)
    d_lse = torch.empty((dshape.B, dshape.Hq), dtype=torch.float32, device=dev)
    ws_bytes = (attn.decode_kv8_workspace_size(dshape.B, dshape.Hq, dshape.Hkv, 1, dshape.Lmax, dshape.D) if kv8
                else attn.decode_workspace_size(dshape.B, dshape.Hq, dshape.Hkv, dshape.Lmax, dshape.D))
    ws = torch.empty(ws_bytes, dtype=torch.uint8, device=dev)
    p_ws = torch.empty(max(1, attn.prefill_workspace_size(PREFILL.B, PREFILL.Hq, PREFILL.Hkv, PREFILL.Lq, PREFILL.Lk,
                                                          PREFILL.D, PREFILL.is_causal)), dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)

    do_pre = args.only in (None, "prefill")
    do_dec = args.only in (None, "decode")

    def call_prefill():
        if do_pre:
            attn.prefill(q, k, v, scale=PREFILL.scale, is_causal=PREFILL.is_causal, out=p_out, lse=p_lse,
                         workspace=p_ws, stream=stream)

    def call_decode():
        if do_dec and kv8:
            attn.decode_kv8(dq, dk, dv, dks, dvs, dsl, out=d_out, lse=d_lse, workspace=ws, stream=stream)
        elif do_dec:
            attn.decode(dq, dk, dv, dsl, out=d_out, lse=d_lse, workspace=ws, stream=stream)

    def step():
        call_prefill()
        call_decode()

    def barrier():
        if dist is not None:
            dist.barrier()

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    assert attn.device_error(reset=True) == 0, "device error word set during warm-up"

    # ---- timed region: K steps, events around each call on the launching stream ----
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(args.steps)]
    sampler = ClockSampler(local_rank)
    barrier()
    torch.cuda.synchronize()
    sampler.start()
    time.sleep(0.3)
    t_start = torch.cuda.Event(enable_timing=True)
    t_end = torch.cuda.Event(enable_timing=True)
    t_start.record(stream)
    for i in range(args.steps):
        ev[i][0].record(stream)
        call_prefill()
        ev[i][1].record(stream)
        call_decode()
        ev[i][2].record(stream)
    t_end.record(stream)
    torch.cuda.synchronize()
    barrier()
    clocks = sampler.stop()
    total_ms = t_start.elapsed_time(t_end)
    pre_ms = [e[0].elapsed_time(e[1]) for e in ev]
    dec_ms = [e[1].elapsed_time(e[2]) for e in ev]
    derr = attn.device_error(reset=True)
    assert derr == 0, f"device error word {derr:#x} after the timed region"

    def max_over_ranks(x):
        return _max_over_ranks(x, device=dev)

    total_ms = max_over_ranks(total_ms)
    pre_avg = max_over_ranks(sum(pre_ms) / len(pre_ms))
    dec_avg = max_over_ranks(sum(dec_ms) / len(dec_ms))

    # ---- end to end through the public API with host buffers ----
    pin = lambda t: t.cpu().pin_memory()
    hq, hk, hv, hdq, hsl = pin(q_h), pin(k_h), pin(v_h), pin(dq), pin(dsl)
    ho, hl = torch.empty_like(hq).pin_memory(), torch.empty(p_lse.shape, dtype=torch.float32).pin_memory()
    hdo, hdl = torch.empty_like(hdq).pin_memory(), torch.empty(d_lse.shape, dtype=torch.float32).pin_memory()
    e2e_pre, e2e_dec = [], []
    ws_host = None if args.only is not None else torch.empty(
        attn.decode_host_workspace_size(dshape.B, dshape.Hq, dshape.Hkv, dshape.Lmax, dshape.D), dtype=torch.uint8,
        device=dev)
    # prefill end to end: the host-buffer call, which pipelines copies in, kernels and copies out
    scr = torch.empty(attn.prefill_host_scratch_size(PREFILL.B, PREFILL.Hq, PREFILL.Hkv, PREFILL.Lq, PREFILL.Lk,
                                                     PREFILL.D), dtype=torch.uint8, device=dev)
    for i in range(args.e2e_steps + 1 if args.only is None else 0):
        e = [torch.cuda.Event(enable_timing=True) for _ in range(3)]
        e[0].record(stream)
        attn.prefill_host(hq, hk, hv, is_causal=True, out=ho, lse=hl, scratch=scr, device=dev, stream=stream)
        e[1].record(stream)
        # the host-buffer call: q and seqlens in, decode, out and lse back (bf16 cache: 8-bit caches
        # only run with --only decode, which has no end-to-end leg)
        attn.decode_host(hdq, dk, dv, hsl, out=hdo, lse=hdl, workspace=ws_host, stream=stream)
        e[2].record(stream)
        torch.cuda.synchronize()
        if i > 0:   # the first is a warm-up of the copy path
            e2e_pre.append(e[0].elapsed_time(e[1]))
            e2e_dec.append(e[1].elapsed_time(e[2]))
    e2e_pre_ms = max_over_ranks(sum(e2e_pre) / max(1, len(e2e_pre)))
    e2e_dec_ms = max_over_ranks(sum(e2e_dec) / max(1, len(e2e_dec)))
    if args.only is not None:
        print(json.dumps({"only": args.only, "prefill_ms": pre_avg, "decode_ms": dec_avg,
                          "prefill_tflops": p_flops / (pre_avg * 1e-3) / 1e12 if do_pre else None,
                          "decode_gbs": d_bytes / (dec_avg * 1e-3) / 1e9 if do_dec else None}), flush=True)
        return None
    h2d = (hq.numel() + hk.numel() + hv.numel() + hdq.numel()) * 2 + hsl.numel() * 4
    d2h = (ho.numel() + hdo.numel()) * 2 + (hl.numel() + hdl.numel()) * 4

    kvp_line = None
    if args.only is None:
        kvp_line = run_kv_parallel(attn, dev, stream, rank, world, args.seed, max(3, args.steps // 4),
                                   max(3, args.warmup), max_over_ranks, barrier)

    cpu_line = None
    if rank == 0 and not args.no_cpu_baseline and args.only is None:
        cpu_line = cpu_baseline(args, q_h, k_h, v_h, dq.cpu(), dk, dv, seqlens_host)
    sweeps = None
    if not args.no_sweeps and args.only is None:
        del dk, dv   # make room: the group-size sweep holds up to 34 GB of cache at a time
        torch.cuda.empty_cache()
        sweeps = run_sweeps(attn, dev, stream, seed, max_over_ranks)
    if rank != 0:
        return None
    pre_tflops = world * p_flops / (pre_avg * 1e-3) / 1e12
    dec_gbs = world * d_bytes / (dec_avg * 1e-3) / 1e9
    peak_t = float(peaks["bf16_tflops"])
    peak_b = float(peaks["hbm_gbs"])
    traffic = RL.committed_traffic()
    line = {
        "metric": METRIC,
        "value": round(pre_tflops, 2),
        "unit": "TFLOP/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": round(total_ms / args.steps, 4),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "bf16",
        "data": "synthetic N(0,1) bf16, seeded; Qwen3-8B attention shapes, no weights",
        "config": {
            "workload": f"{PREFILL.name} + {DECODE.name}",
            "prefill": {"B": PREFILL.B, "Hq": PREFILL.Hq, "Hkv": PREFILL.Hkv, "Lq": PREFILL.Lq, "Lk": PREFILL.Lk,
                        "D": PREFILL.D, "is_causal": True, "flops_per_call": p_flops},
            "decode": {"B": DECODE.B, "Hq": DECODE.Hq, "Hkv": DECODE.Hkv, "Lmax": DECODE.Lmax, "D": DECODE.D,
                       "seqlens": "uniform [1024, 32768]", "bytes_per_call": d_bytes},
            "l2": "inputs larger than L2 (prefill q/k/v 403 MB, decode cache 8.6 GB); no flush",
            "parallelism": f"replicas x{world} (independent sequences per GPU)",
        },
        "decode": {"value": round(dec_gbs, 1), "unit": "GB/s", "ms_per_call": round(dec_avg, 4),
                   "frac_of_measured_hbm": round(dec_gbs / world / peak_b, 4),
                   "frac_of_8000": round(dec_gbs / world / 8000.0, 4)},
        "roofline": {"bound": "tensor", "kernel": "attn_prefill_sm100_kernel",
                     "achieved": round(pre_tflops / world, 2), "peak": peak_t, "unit": "TFLOP/s",
                     "frac": round(pre_tflops / world / peak_t, 4),
                     "peak_source": f"{peaks['source']} bf16_tflops (burst)",
                     "frac_of_sustained": round(pre_tflops / world / float(peaks.get("bf16_tflops_sustained", peak_t)), 4),
                     "traffic": traffic.get("attn_prefill_sm100_kernel"),
                     "ms_per_call": round(pre_avg, 4),
                     # the step's other kernel: the decode batch against its HBM roofline
                     "decode": {"bound": "hbm", "kernel": "attn_decode_split_kernel + attn_decode_combine_kernel",
                                "achieved": round(dec_gbs / world, 1), "peak": peak_b, "unit": "GB/s",
                                "frac": round(dec_gbs / world / peak_b, 4),
                                "peak_source": f"{peaks['source']} hbm_gbs",
                                "traffic": traffic.get("attn_decode_split_kernel"),
                                "ms_per_call": round(dec_avg, 4)}},
        "e2e": {"value": round(world * p_flops / (e2e_pre_ms * 1e-3) / 1e12, 2), "unit": "TFLOP/s",
                "decode_gbs": round(world * d_bytes / (e2e_dec_ms * 1e-3) / 1e9, 1),
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                "what": "prefill: attn_prefill_host on pinned host q/k/v/out/lse (copies in, kernels and copies "
                        "out pipelined by the library); decode: attn_decode_host on pinned host q/seqlens/out/lse "
                        "(one call: copies in, kernels, copies out), KV cache resident on the device"},
        "gpu_launches": 3 * args.steps,
        "kv_parallel": kvp_line,
        "sweeps": sweeps,
        "clocks": clocks,
    }
    if cpu_line is not None:
        line["cpu_baseline"] = cpu_line
    return line


def run_kv_parallel(attn, dev, stream, rank, world, seed, steps, warmup, max_over_ranks, barrier):
    """KV-parallel decode of the Qwen3-8B decode batch (the NVIDIA attention page,
    "Parameter four: parallelism"): every rank holds a 1/world share of each
    sequence's cached rows, so the batch is fixed as ranks are added (strong
    scaling).  A step is attn_decode_partial on the local rows, an all-gather of
    the fp32 partials over NCCL, and attn_decode_merge (multigpu.KVParallelDecode).
    At one GPU the step is the partial and the merge, with no exchange."""
    from exact_tiled_attention_gqa_b200.multigpu import KVParallelDecode, kv_shard_rows, shard_seqlens
    shape = DECODE
    gcpu = torch.Generator().manual_seed(seed + 4242)   # the same sequences and queries on every rank
    sl = torch.randint(shape.seqlen_lo, shape.seqlen_hi + 1, (shape.B,), generator=gcpu).to(torch.int32)
    q = torch.randn((shape.B, shape.Hq, shape.D), generator=gcpu).to(torch.bfloat16).to(dev)
    rows = kv_shard_rows(shape.Lmax, rank, world)
    g = torch.Generator(device=dev)
    g.manual_seed(seed + 77 + rank)
    k = torch.empty((shape.B, shape.Hkv, len(rows), shape.D), dtype=torch.bfloat16, device=dev)
    v = torch.empty_like(k)
    for cache in (k, v):
        for b in range(shape.B):
            cache[b].copy_(torch.randn(cache[b].shape, generator=g, device=dev).to(torch.bfloat16))
    ws = torch.empty(attn.decode_workspace_size(shape.B, shape.Hq, shape.Hkv, len(rows), shape.D), dtype=torch.uint8,
                     device=dev)
    kvp = KVParallelDecode(q, k, v, shard_seqlens(sl, rows).to(dev), scale=shape.scale, workspace=ws)
    for _ in range(warmup):
        kvp.step()
    torch.cuda.synchronize()
    barrier()
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
    for e0, e1 in ev:
        e0.record(stream)
        kvp.step()
        e1.record(stream)
    torch.cuda.synchronize()
    barrier()
    ms = max_over_ranks(sum(e0.elapsed_time(e1) for e0, e1 in ev) / steps)
    by = RL.decode_bytes(sl.tolist(), shape.B, shape.Hq, shape.Hkv, shape.D)
    peak_b = float(RL.measured_peaks()["hbm_gbs"])
    del kvp, k, v, ws
    torch.cuda.empty_cache()
    return {"workload": shape.name + f", cache rows split over {world} GPU(s)", "n_gpus": world,
            "scaling": "strong", "ms_per_step": round(ms, 4), "value": round(by / ms / 1e6, 1), "unit": "GB/s",
            "bytes_per_step": by, "frac_of_measured_hbm_per_gpu": round(by / ms / 1e6 / world / peak_b, 4),
            "exchange": (f"all-gather of fp32 partials over NCCL, {shape.B * shape.Hq * (shape.D + 1) * 4} bytes "
                         "per rank" if world > 1 else "none (one GPU)")}


_L2_FLUSH = None
_L2_FLUSH = None


def _time_calls(fn, stream, n_warm=2, n=10, flush=False):
    """Mean device time of fn() over n calls (CUDA events on `stream` around each
    call).  All n calls are enqueued before one synchronisation, so the host's
    launch work overlaps the device's and no event pair holds an idle gap.  With
    flush, a 256 MB write (twice the L2) precedes every call, outside its events."""
    global _L2_FLUSH
    for _ in range(n_warm):
        fn()
    if flush and _L2_FLUSH is None:
        _L2_FLUSH = torch.empty(256 << 20, dtype=torch.uint8, device=torch.cuda.current_device())
    evs = []
    torch.cuda.synchronize()
    for _ in range(n):
        if flush:
            with torch.cuda.stream(stream):
                _L2_FLUSH.fill_(1)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        fn()
        e1.record(stream)
        evs.append((e0, e1))
    torch.cuda.synchronize()
    return sum(e0.elapsed_time(e1) for e0, e1 in evs) / n


def run_sweeps(attn, dev, stream, seed, max_over_ranks):
    """The other workloads: Qwen3-8B prefill B1 L4096, the chunked prefills, head dim
    256 prefill and decode, the paged decode, and the group-size decode sweep
    (Hq=64, D=128, batch 8, 131072 keys, G = 1 .. 64)."""
    peaks = RL.measured_peaks()
    out = {"prefill": [], "decode_group_sweep": []}
    for shape in (W.QWEN_PREFILL_4K, W.CHUNKED_16K, W.CHUNKED_32K, W.HD256_PREFILL, W.HD64_PREFILL):
        q, k, v = (t.to(dev) for t in W.prefill_inputs_for(shape, seed=seed))
        o = torch.empty_like(q)
        l = torch.empty((shape.B, shape.Hq, shape.Lq), dtype=torch.float32, device=dev)
        small = (q.numel() + 2 * k.numel()) * 2 < 126e6
        ws = torch.empty(max(1, attn.prefill_workspace_size(shape.B, shape.Hq, shape.Hkv, shape.Lq, shape.Lk,
                                                            shape.D, True)), dtype=torch.uint8, device=dev)
        ms = max_over_ranks(_time_calls(lambda: attn.prefill(q, k, v, scale=shape.scale, is_causal=True, out=o,
                                                              lse=l, workspace=ws, stream=stream),
                                        stream, n=20, flush=small))
        fl = RL.prefill_flops(shape.B, shape.Hq, shape.Lq, shape.Lk, shape.D, True)
        out["prefill"].append({"workload": shape.name, "ms": round(ms, 4), "tflops": round(fl / ms / 1e9, 1),
                               "frac_of_measured_bf16": round(fl / ms / 1e9 / float(peaks["bf16_tflops"]), 4),
                               "l2": "L2 flushed (256 MB write) before each timed call" if small else
                                     "inputs larger than L2"})
        del q, k, v, o, l
    # the Qwen3-8B decode batch again, its cache in 128-row pages handed out in shuffled order
    shape = DECODE
    g = torch.Generator(device=dev)
    g.manual_seed(seed + 77)
    gcpu = torch.Generator().manual_seed(seed)
    sl = torch.randint(shape.seqlen_lo, shape.seqlen_hi + 1, (shape.B,), generator=gcpu).to(torch.int32)
    page = 128
    per = [-(-int(n) // page) for n in sl]
    n_pages = sum(per)
    kp = torch.randn((n_pages, shape.Hkv, page, shape.D), generator=g, device=dev).to(torch.bfloat16)
    vp = torch.randn((n_pages, shape.Hkv, page, shape.D), generator=g, device=dev).to(torch.bfloat16)
    perm = torch.randperm(n_pages, generator=gcpu).to(torch.int32)
    table = torch.zeros((shape.B, max(per)), dtype=torch.int32)
    o0 = 0
    for b_, n_ in enumerate(per):
        table[b_, :n_] = perm[o0:o0 + n_]
        o0 += n_
    table, sl_d = table.to(dev), sl.to(dev)
    dq = torch.randn((shape.B, shape.Hq, 1, shape.D), generator=g, device=dev).to(torch.bfloat16)
    o = torch.empty_like(dq)
    l = torch.empty((shape.B, shape.Hq, 1), dtype=torch.float32, device=dev)
    ws = torch.empty(attn.decode_workspace_size(shape.B, shape.Hq, shape.Hkv, page * table.shape[1], shape.D) + 4096,
                     dtype=torch.uint8, device=dev)
    ms = max_over_ranks(_time_calls(lambda: attn.decode_paged(dq, kp, vp, table, sl_d, scale=shape.scale, out=o, lse=l,
                                                               workspace=ws, stream=stream), stream, n=10))
    by = RL.decode_bytes(sl.tolist(), shape.B, shape.Hq, shape.Hkv, shape.D)
    out["decode_paged"] = {"workload": shape.name + ", 128-row pages in shuffled order", "ms": round(ms, 4),
                           "gbs": round(by / ms / 1e6, 1),
                           "frac_of_measured_hbm": round(by / ms / 1e6 / float(peaks["hbm_gbs"]), 4)}
    del kp, vp, dq, o, l, ws, table
    torch.cuda.empty_cache()
    out["decode_kv8"] = []
    for fmt, shape in ((W.KV_E4M3, W.QWEN_DECODE_E4M3), (W.KV_Q8_0, W.QWEN_DECODE_Q8_0)):
        dq, dk, dv, dks, dvs, dsl = W.decode_inputs_kv8(shape.B, shape.Hq, shape.Hkv, shape.Lmax, shape.D,
                                                        shape.seqlen_lo, shape.seqlen_hi, fmt, seed=seed,
                                                        device=dev)
        o = torch.empty_like(dq)
        l = torch.empty((shape.B, shape.Hq, 1), dtype=torch.float32, device=dev)
        ws = torch.empty(attn.decode_kv8_workspace_size(shape.B, shape.Hq, shape.Hkv, 1, shape.Lmax, shape.D),
                         dtype=torch.uint8, device=dev)
        ms = max_over_ranks(_time_calls(lambda: attn.decode_kv8(dq, dk, dv, dks, dvs, dsl, scale=shape.scale, out=o,
                                                                 lse=l, workspace=ws, stream=stream), stream, n=10))
        by = RL.decode_kv8_bytes(dsl.cpu().tolist(), shape.B, shape.Hq, shape.Hkv, shape.D, fmt == W.KV_Q8_0)
        out["decode_kv8"].append({"workload": shape.name, "ms": round(ms, 4), "bytes": by,
                                  "gbs": round(by / ms / 1e6, 1),
                                  "frac_of_measured_hbm": round(by / ms / 1e6 / float(peaks["hbm_gbs"]), 4)})
        del dq, dk, dv, dks, dvs, dsl, o, l, ws
        torch.cuda.empty_cache()
    shape = W.HD256_DECODE
    dq, dk, dv, dsl = W.decode_inputs_for(shape, seed=seed + 256, device=dev)
    o = torch.empty_like(dq)
    l = torch.empty((shape.B, shape.Hq), dtype=torch.float32, device=dev)
    ws = torch.empty(attn.decode_workspace_size(shape.B, shape.Hq, shape.Hkv, shape.Lmax, shape.D),
                     dtype=torch.uint8, device=dev)
    ms = max_over_ranks(_time_calls(lambda: attn.decode(dq, dk, dv, dsl, scale=shape.scale, out=o, lse=l,
                                                         workspace=ws, stream=stream), stream, n=10))
    by = RL.decode_bytes(dsl.cpu().tolist(), shape.B, shape.Hq, shape.Hkv, shape.D)
    out["decode_hd256"] = {"workload": shape.name, "ms": round(ms, 4), "gbs": round(by / ms / 1e6, 1),
                           "frac_of_measured_hbm": round(by / ms / 1e6 / float(peaks["hbm_gbs"]), 4)}
    del dq, dk, dv, dsl, o, l, ws
    torch.cuda.empty_cache()
    for G in W.GROUP_SWEEP:
        shape = W.group_sweep_decode(G)
        dq, dk, dv, dsl = W.decode_inputs_for(shape, seed=seed + G, device=dev)
        o = torch.empty_like(dq)
        l = torch.empty((shape.B, shape.Hq), dtype=torch.float32, device=dev)
        ws = torch.empty(attn.decode_workspace_size(shape.B, shape.Hq, shape.Hkv, shape.Lmax, shape.D),
                         dtype=torch.uint8, device=dev)
        ms = max_over_ranks(_time_calls(lambda: attn.decode(dq, dk, dv, dsl, scale=shape.scale, out=o, lse=l,
                                                             workspace=ws, stream=stream), stream, n=10))
        by = RL.decode_bytes(dsl.cpu().tolist(), shape.B, shape.Hq, shape.Hkv, shape.D)
        out["decode_group_sweep"].append({"G": G, "Hkv": shape.Hkv, "ms": round(ms, 4), "bytes": by,
                                          "gbs": round(by / ms / 1e6, 1),
                                          "frac_of_measured_hbm": round(by / ms / 1e6 / float(peaks["hbm_gbs"]), 4)})
        del dq, dk, dv, dsl, o, l, ws
        torch.cuda.empty_cache()
    return out


# --------------------------------------------------------------------------
# the oracle on this host's cores (bounded samples)
# --------------------------------------------------------------------------
def _prefill_sample_rows(n):
    return sorted(set(int(x) for x in np.linspace(0, PREFILL.Lq - 1, n)))


def oracle_prefill_rate(q_h, k_h, v_h, n_rows):
    import oracle
    rows = _prefill_sample_rows(n_rows)
    qb, kb, vb = q_h[:1], k_h[:1], v_h[:1]
    flops = sum(4 * PREFILL.D * min(PREFILL.Lk, r + PREFILL.Lk - PREFILL.Lq + 1) for r in rows) * PREFILL.Hq
    t0 = time.perf_counter()
    oracle.attention_prefill(qb, kb, vb, PREFILL.scale, True, rows=rows)
    dt = time.perf_counter() - t0
    return flops, dt, rows


def cpu_baseline(args, q_h, k_h, v_h, dq_h, dk, dv, seqlens_host):
    import oracle
    cores = oracle.num_threads(0)
    # calibrate, then size the sample to about args.cpu_seconds
    f0, t0, _ = oracle_prefill_rate(q_h, k_h, v_h, 8)
    n = int(max(8, min(PREFILL.Lq, 8 * args.cpu_seconds / max(t0, 1e-3))))
    flops, dt, rows = oracle_prefill_rate(q_h, k_h, v_h, n)
    pre = flops / dt / 1e12
    # decode: whole (b, h) rows of the Qwen3-8B decode batch, cache slices copied to the host
    G = DECODE.G
    sel = [(b, g) for b in range(DECODE.B) for g in range(DECODE.Hkv)]
    rng = np.random.default_rng(0)
    rng.shuffle(sel)
    done_bytes, dt_dec, used = 0, 0.0, 0
    for b, g in sel:
        n_b = int(seqlens_host[b])
        kb = dk[b:b + 1, g:g + 1, :n_b].cpu()
        vb = dv[b:b + 1, g:g + 1, :n_b].cpu()
        qb = dq_h[b:b + 1, g * G:(g + 1) * G]
        t0 = time.perf_counter()
        oracle.attention_decode(qb, kb, vb, np.array([n_b], np.int32), DECODE.scale)
        dt_dec += time.perf_counter() - t0
        done_bytes += n_b * DECODE.D * 2 * 2 + G * DECODE.D * 2 * 2 + G * 4
        used += 1
        if dt_dec > args.cpu_seconds / 2:
            break
    return {"value": round(pre, 6), "unit": "TFLOP/s", "cores": cores, "kind": "oracle",
            "sample": f"prefill: batch 0, all 32 heads, {len(rows)} query rows spread over 0..8191 "
                      f"({flops / 1e9:.1f} GFLOP in {dt:.1f} s); fp64 C eager attention, OpenMP",
            "decode": {"value": round(done_bytes / dt_dec / 1e9, 4), "unit": "GB/s",
                       "sample": f"{used} (batch, KV head) groups of the decode batch, {dt_dec:.1f} s"}}


def run_reference(args, rank, world):
    """The oracle as it stands, on this host's cores, each step a bounded sample."""
    if rank != 0:
        return None
    import oracle
    oracle.build()
    q_h, k_h, v_h = W.prefill_inputs_for(PREFILL, seed=args.seed, device="cpu")
    cores = oracle.num_threads(0)
    f0, t0, _ = oracle_prefill_rate(q_h, k_h, v_h, 8)
    budget = args.ref_seconds / max(1, args.steps + args.warmup)   # whole run within a few minutes
    n = int(max(8, min(PREFILL.Lq, 8 * budget / max(t0, 1e-3))))
    for _ in range(args.warmup):
        oracle_prefill_rate(q_h, k_h, v_h, 8)
    flops_t, dt_t = 0, 0.0
    for _ in range(args.steps):
        f, dt, rows = oracle_prefill_rate(q_h, k_h, v_h, n)
        flops_t += f
        dt_t += dt
    val = flops_t / dt_t / 1e12
    return {
        "metric": METRIC, "value": round(val, 6), "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(1e3 * dt_t / args.steps, 3), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic N(0,1) bf16, seeded",
        "impl": "reference",
        "config": {"workload": f"{PREFILL.name} (sampled query rows)", "rows_per_step": n},
        "cpu_baseline": {"value": round(val, 6), "unit": "TFLOP/s", "cores": cores, "kind": "oracle",
                         "sample": f"batch 0, all heads, {n} query rows per step"},
        "e2e": {"value": round(val, 6), "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }


def main():
    args = parse()
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        line = run_reference(args, rank, world)
        if line is not None:
            print(json.dumps(line), flush=True)
        return
    if world > 1:
        import datetime
        import torch.distributed as dist
        torch.cuda.set_device(local_rank)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local_rank))
    try:
        line = run_ours(args, rank, world, local_rank)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()
    if line is not None:
        print(json.dumps(line), flush=True)


if __name__ == "__main__":
    main()
