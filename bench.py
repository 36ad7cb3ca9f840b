"""Benchmark of the compressed-KV hot path: tq_quantize (prefill of the whole context) followed by
tq_decode_attn (one decode query per sequence).  Default workload: one Llama-3-8B-shaped layer at
128K context, batch 4 (32 query heads, 8 kv-heads, head_dim 128, turbo4: 4-bit keys + QJL m=128,
4-bit values); --workload selects any of the five recipes (e.g. moe_1m: 1M tokens, streamed in
8192-token chunks).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl reference]

Prints one JSON line.  value = compressed-KV bytes read by decode / decode time (GB/s, whole job);
quantize throughput is reported beside it.  Multi-GPU (torchrun): every rank runs its own
independent replica of the workload (the path has no exchange step), timing is the max over ranks.
"""
from __future__ import annotations

import argparse
import dataclasses
import json
import math
import os
import statistics
import subprocess
import sys
import time

import numpy as np
import torch

import workloads as W

ROOT = os.path.dirname(os.path.abspath(__file__))
DEFAULT_WORKLOAD = "llama3_8b_128k_b4"
SPEC_HBM_GBS = 8000.0  # B200 HBM3e nominal bandwidth (the method statement's "about 8 TB/s")
L2_FLUSH_BYTES = 256 << 20


TRAFFIC_FILE = os.path.join(ROOT, "profiles", "dram_traffic.json")


def source_digest(rel: str) -> str:
    """Digest of a kernel source with comments, blank lines and the debug-build blocks
    (``#ifdef TQ_DEBUG`` ... ``#endif``, compiled out of the library that is timed) removed, so that
    a change to those alone keeps a capture valid."""
    import hashlib
    import re
    with open(os.path.join(ROOT, rel), encoding="utf-8") as f:
        text = f.read()
    text = re.sub(r"^[ \t]*#ifdef TQ_DEBUG\b.*?^[ \t]*#endif[^\n]*\n", "", text, flags=re.S | re.M)
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    text = re.sub(r"//[^\n]*", "", text)
    code = "\n".join(line.rstrip() for line in text.splitlines() if line.strip())
    return hashlib.sha256(code.encode()).hexdigest()[:16]


def dram_traffic(kernel: str, workload: str, batch, context):
    """DRAM bytes per launch of `kernel` (dram__bytes_read.sum + dram__bytes_write.sum) from a
    committed ncu capture, scaled by batch to the launch timed here (traffic grows with the number
    of (sequence, kv-head) units).  None when the kernel source changed since the capture or no
    capture covers this workload."""
    if not os.path.exists(TRAFFIC_FILE):
        return None, "no capture"
    with open(TRAFFIC_FILE) as f:
        table = json.load(f)
    for e in table.get("captures", []):
        if e["api"] != kernel or e["workload"] != workload or context is not None:
            continue
        if source_digest(e["source"]) != e["source_sha256"]:
            return None, "kernel changed since the capture"
        full_b = W.CONFIGS[workload].B
        b = batch if batch is not None else full_b
        per_unit = e["bytes_per_launch"] / e["batch"]
        note = "ncu capture at batch %d" % e["batch"] + ("" if b == e["batch"] else ", scaled to batch %d" % b)
        return per_unit * b, note
    return None, "no capture of this workload"


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            p = json.load(f)
        return float(p["hbm_gbs"]), float(p.get("bf16_tflops", 1590.0)), "measured"
    return 6650.0, 1590.0, "fallback"


class ClockSampler:
    """SM clock and clock-event reasons sampled through NVML every millisecond while the timed
    region runs (the region can be a few milliseconds long); nvidia-smi polling if NVML is
    unavailable."""

    NAMES = {0x8: "hw_slowdown", 0x40: "hw_thermal_slowdown", 0x20: "sw_thermal_slowdown",
             0x4: "sw_power_cap", 0x80: "hw_power_brake_slowdown"}

    def __init__(self, device_index: int):
        self.device_index = device_index
        self.samples = []  # (sm_mhz, sm_max_mhz, reasons bitmask, power_w)
        self._stop = None
        self._thread = None
        self._smi = None

    def _nvml_handle(self):
        import pynvml
        pynvml.nvmlInit()
        props = torch.cuda.get_device_properties(self.device_index)
        bus = "%08x:%02x:%02x.0" % (props.pci_domain_id, props.pci_bus_id, props.pci_device_id)
        return pynvml, pynvml.nvmlDeviceGetHandleByPciBusId(bus)

    def __enter__(self):
        import threading
        try:
            nv, h = self._nvml_handle()
        except Exception:
            nv = None
        if nv is not None:
            self._stop = threading.Event()
            get_reasons = getattr(nv, "nvmlDeviceGetCurrentClocksEventReasons", None) or \
                nv.nvmlDeviceGetCurrentClocksThrottleReasons

            started = threading.Event()

            def run():
                smax = nv.nvmlDeviceGetMaxClockInfo(h, nv.NVML_CLOCK_SM)
                while True:
                    try:
                        self.samples.append((nv.nvmlDeviceGetClockInfo(h, nv.NVML_CLOCK_SM), smax,
                                             int(get_reasons(h)), nv.nvmlDeviceGetPowerUsage(h) / 1e3))
                    except Exception:
                        pass
                    started.set()
                    if self._stop.is_set():
                        break  # one last sample after the region ends
                    time.sleep(0.0005)  # releases the interpreter lock for the launching thread

            self._thread = threading.Thread(target=run, daemon=True)
            self._thread.start()
            started.wait(timeout=5)
        else:
            try:
                self._smi = subprocess.Popen(
                    ["nvidia-smi", "-i", str(self.device_index),
                     "--query-gpu=clocks.sm,clocks.max.sm,clocks_event_reasons.active,power.draw",
                     "--format=csv,noheader,nounits", "-lms", "100"],
                    stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            except OSError:
                self._smi = None
        return self

    def __exit__(self, *exc):
        if self._thread is not None:
            self._stop.set()
            self._thread.join(timeout=5)
        if self._smi is not None:
            self._smi.terminate()
            try:
                out, _ = self._smi.communicate(timeout=5)
            except subprocess.TimeoutExpired:
                self._smi.kill()
                out, _ = self._smi.communicate()
            for line in out.splitlines():
                parts = [p.strip() for p in line.split(",")]
                try:
                    self.samples.append((float(parts[0]), float(parts[1]), int(parts[2], 16), float(parts[3])))
                except (ValueError, IndexError):
                    continue

    def summary(self):
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
        sm = [x[0] for x in self.samples]
        reasons = set()
        for x in self.samples:
            for bit, name in self.NAMES.items():
                if x[2] & bit:
                    reasons.add(name)
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(x[1] for x in self.samples),
                "sm_mhz_min": min(sm), "power_w_max": max(x[3] for x in self.samples),
                "reasons": sorted(reasons), "samples": len(sm)}


def dist_env():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return world, rank, local


def max_over_ranks(x: float, world: int) -> float:
    if world == 1:
        return x
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64,
                     device="cuda" if dist.get_backend() == "nccl" else "cpu")
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


# --------------------------------------------------------------------------------------- CPU arm

def oracle_sample(w: W.Workload, tokens: int):
    """Oracle quantize + decode for one (batch, kv-head) unit over `tokens` tokens (CPU)."""
    from oracle import tq_oracle as O
    sw = w.scaled(T=tokens, B=1, Hkv=1, Hq=w.group)
    K = W.make_kv(sw, "k").double().numpy()
    V = W.make_kv(sw, "v").double().numpy()
    q = W.make_queries(sw).double().numpy()
    Pi, S = W.rotation_for(w), W.qjl_for(w)
    if w.layout == "mixed":
        oc, kb, vb = W.outlier_channels_for(w), (w.k_bits, w.k_bits - 1), (w.v_bits, w.v_bits - 1)
        t0 = time.perf_counter()
        cache = O.quantize_cache_mixed(K, V, Pi, oc, kb, vb, S)
        t1 = time.perf_counter()
        O.decode_attention_mixed(q, Pi, S, cache, kb, vb, tokens)
        t2 = time.perf_counter()
        return t1 - t0, t2 - t1, sw
    t0 = time.perf_counter()
    cache = O.quantize_cache(K, V, Pi, w.k_bits, w.v_bits, S)
    t1 = time.perf_counter()
    O.decode_attention(q, Pi, S, cache, w.k_bits, w.v_bits, tokens)
    t2 = time.perf_counter()
    return t1 - t0, t2 - t1, sw


def blas_threads() -> int:
    """Threads of numpy's BLAS pool: the oracle's matrix products run on up to this many; its
    other numpy work runs on one."""
    try:
        import numpy  # noqa: F401  (the pool is visible once numpy is loaded)
        from threadpoolctl import threadpool_info
        n = [d.get("num_threads", 1) for d in threadpool_info() if d.get("user_api") == "blas"]
        return max(n) if n else 1
    except ImportError:
        return os.cpu_count() or 1


def cpu_baseline(w: W.Workload, budget_s: float = 20.0, single_thread: bool = True):
    tokens = 2048
    qt, dt, sw = oracle_sample(w, tokens)
    # grow the sample toward the time budget
    while qt + dt < budget_s / 4 and tokens < w.T:
        tokens = min(w.T, tokens * 2)
        qt, dt, sw = oracle_sample(w, tokens)
    dec_bytes = sw.decode_bytes()
    threads = blas_threads()
    cb = {
        "value": dec_bytes / dt / 1e9, "unit": "GB/s", "cores": threads, "kind": "oracle",
        "sample": f"one (batch, kv-head) unit of {w.name}: {tokens} tokens, {w.group} query heads; "
                  f"numpy float64, matrix products on up to {threads} BLAS threads "
                  f"({os.cpu_count()} host CPUs)",
        "quantize_tokens_per_s": tokens / qt, "decode_s": dt, "quantize_s": qt,
    }
    if single_thread:
        # the same sample with the BLAS pool held to one thread
        try:
            from threadpoolctl import threadpool_limits
            with threadpool_limits(1):
                qt1, dt1, _ = oracle_sample(w, tokens)
            cb["single_thread"] = {"value": dec_bytes / dt1 / 1e9, "unit": "GB/s",
                                   "quantize_tokens_per_s": tokens / qt1}
        except ImportError:
            pass
    return cb


def run_reference(args, w):
    world, rank, _ = dist_env()
    if rank != 0:
        return
    cb = cpu_baseline(w, budget_s=20.0, single_thread=False)
    steps = []
    tokens = int(cb["sample"].split(": ")[1].split(" ")[0])
    for _ in range(args.warmup + args.steps):
        steps.append(oracle_sample(w, tokens))
    timed = steps[args.warmup:]
    dt = sum(s[1] for s in timed)
    qt = sum(s[0] for s in timed)
    dec_bytes = timed[0][2].decode_bytes() * len(timed)
    value = dec_bytes / dt / 1e9
    line = {
        "impl": "reference", "metric": "compressed-KV decode-attn GB/s (% HBM peak); tq_quantize tokens/s",
        "value": value, "unit": "GB/s", "n_gpus": args.gpus, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": 1e3 * (dt + qt) / len(timed),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic", "config": workload_config(w, sample_tokens=tokens),
        "quantize_tokens_per_s": tokens * len(timed) / qt,
        "cpu_baseline": {"value": value, "unit": "GB/s", "cores": cb["cores"], "kind": "oracle",
                         "sample": cb["sample"]},
        "e2e": {"value": value, "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def workload_config(w: W.Workload, **extra):
    c = {"workload": w.name, "batch": w.B, "q_heads": w.Hq, "kv_heads": w.Hkv, "head_dim": w.head_dim,
         "context": w.T, "k_bits": w.k_bits, "v_bits": w.v_bits, "qjl_m": w.qjl_m,
         "input_dtype": w.in_dtype, "quantize_chunk": w.chunk, "rotation": w.rotation,
         "layout": w.layout,
         "l2": f"flushed before every kernel call ({L2_FLUSH_BYTES >> 20} MiB write)"}
    c.update(extra)
    return c


# --------------------------------------------------------------------------------------- GPU arm

def run_gpu(args, w):
    import decode_attention_11_b200 as tq

    world, rank, local = dist_env()
    if world > 1:
        import torch.distributed as dist
        import datetime
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    dev = torch.device("cuda", local if world > 1 else 0)
    torch.cuda.set_device(dev)
    stream = torch.cuda.current_stream()

    mixed = w.layout == "mixed"
    params = tq.Params.create(W.rotation_for(w), W.qjl_for(w), w.k_bits, w.v_bits, device=dev,
                              outlier_channels=W.outlier_channels_for(w) if mixed else None)
    K = W.make_kv(w, "k", device=dev)
    V = W.make_kv(w, "v", device=dev)
    q = W.make_queries(w, device=dev)
    cache = tq.Cache.allocate(w.B, w.Hkv, w.T, w.k_bits, w.v_bits, w.qjl_m, device=dev,
                              layout=tq.TQ_LAYOUT_MIXED if mixed else tq.TQ_LAYOUT_PLAIN)
    out = torch.empty(w.B, w.Hq, 128, dtype=torch.float32, device=dev)
    ws = torch.empty(tq.decode_workspace_size(w.B, w.Hq, cache, w.T), dtype=torch.uint8, device=dev)
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
    n_chunks = math.ceil(w.T / w.chunk)

    def quantize_all():
        for s in range(0, w.T, w.chunk):
            tq.quantize(params, K[:, :, s:s + w.chunk], V[:, :, s:s + w.chunk], cache, t_offset=s)

    def decode():
        tq.decode_attn(params, q, cache, w.T, out=out, workspace=ws)

    # One direct pass first: the kernel's count of coordinates within 1e-6 of a threshold over the
    # whole workload (the cases the parity rule exempts; the fraction must stay <= 1e-5).
    ex_c0, ex_s0 = tq.quantize_exempt_codes(), tq.quantize_exempt_signs()
    quantize_all()
    torch.cuda.synchronize()
    exempt = {"codes": tq.quantize_exempt_codes() - ex_c0, "coords": w.B * w.Hkv * w.T * 2 * w.head_dim,
              "near_zero_signs": tq.quantize_exempt_signs() - ex_s0,
              "sign_bits": w.B * w.Hkv * w.T * (w.qjl_m or 0), "bound": 1e-5}
    exempt["fraction"] = exempt["codes"] / exempt["coords"]

    # Each op is captured once into a CUDA graph and replayed per step, so that host launch
    # latency (the moe workload makes 128 quantize calls per step) stays out of the device timing.
    run_q, run_d = quantize_all, decode
    if not args.no_graph:
        side = torch.cuda.Stream()
        side.wait_stream(stream)
        with torch.cuda.stream(side):  # warm-up outside capture (function attributes, tensor maps)
            quantize_all()
            decode()
        stream.wait_stream(side)
        torch.cuda.synchronize()
        gq, gd = torch.cuda.CUDAGraph(), torch.cuda.CUDAGraph()
        with torch.cuda.graph(gq):
            quantize_all()
        with torch.cuda.graph(gd):
            decode()
        run_q, run_d = gq.replay, gd.replay

    def step(ev):
        flush.zero_()
        ev[0].record(stream)
        run_q()
        ev[1].record(stream)
        flush.zero_()
        ev[2].record(stream)
        run_d()
        ev[3].record(stream)

    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(args.steps)]
    for _ in range(args.warmup):
        step([torch.cuda.Event(enable_timing=True) for _ in range(4)])
    torch.cuda.synchronize()
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    t_all0 = torch.cuda.Event(enable_timing=True)
    t_all1 = torch.cuda.Event(enable_timing=True)
    with ClockSampler(dev.index if dev.index is not None else 0) as clk:
        # a short device-side delay ahead of the timed region lets the host queue the first steps,
        # so that no host launch latency lands between a step's events
        torch.cuda._sleep(2_000_000)
        t_all0.record(stream)
        for i in range(args.steps):
            step(evs[i])
        t_all1.record(stream)
        torch.cuda.synchronize()
    if world > 1:
        torch.distributed.barrier()
    total_ms = t_all0.elapsed_time(t_all1)
    q_ms = [e[0].elapsed_time(e[1]) for e in evs]
    d_ms = [e[2].elapsed_time(e[3]) for e in evs]
    total_ms = max_over_ranks(total_ms, world)
    q_tot = max_over_ranks(sum(q_ms), world)
    d_tot = max_over_ranks(sum(d_ms), world)

    dec_bytes = w.decode_bytes()
    qnt_bytes = w.quantize_bytes()
    hbm, tflops, peak_kind = load_peaks()
    dec_gbs = world * dec_bytes * args.steps / (d_tot * 1e-3) / 1e9
    q_tok_s = world * w.B * w.T * args.steps / (q_tot * 1e-3)
    q_gbs = world * qnt_bytes * args.steps / (q_tot * 1e-3) / 1e9

    # end to end through the public API with host buffers (pinned), copies inside the timed region
    e2e = None
    if not args.no_e2e:
        Kh = K.cpu().pin_memory()
        Vh = V.cpu().pin_memory()
        qh = q.cpu().pin_memory()
        oh = torch.empty(out.shape, dtype=out.dtype).pin_memory()

        def e2e_step():
            K.copy_(Kh, non_blocking=True)
            V.copy_(Vh, non_blocking=True)
            q.copy_(qh, non_blocking=True)
            quantize_all()
            tq.decode_attn(params, q, cache, w.T, out=out, workspace=ws)
            oh.copy_(out, non_blocking=True)

        for _ in range(2):
            e2e_step()
        torch.cuda.synchronize()
        a0 = torch.cuda.Event(enable_timing=True)
        a1 = torch.cuda.Event(enable_timing=True)
        e_steps = max(3, args.steps // 2)
        a0.record(stream)
        for _ in range(e_steps):
            e2e_step()
        a1.record(stream)
        torch.cuda.synchronize()
        e_ms = max_over_ranks(a0.elapsed_time(a1), world)
        h2d = Kh.numel() * Kh.element_size() + Vh.numel() * Vh.element_size() + qh.numel() * qh.element_size()
        d2h = oh.numel() * oh.element_size()
        e2e = {"value": world * dec_bytes * e_steps / (e_ms * 1e-3) / 1e9, "unit": "GB/s",
               "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
               "ms_per_step": e_ms / e_steps}

    # one autoregressive step at the last row (tq_decode_step: row T-1 written again from the same
    # K/V, then attention over all T rows), replayed from a CUDA graph like the ops above, L2 flushed
    # before each replay; reported beside the metric, outside its timed region
    kn, vn = K[:, :, w.T - 1].contiguous(), V[:, :, w.T - 1].contiguous()

    def dstep():
        tq.decode_step(params, kn, vn, q, cache, w.T - 1, out=out, workspace=ws)

    run_s = dstep
    if not args.no_graph:
        with torch.cuda.stream(side):
            dstep()
        stream.wait_stream(side)
        torch.cuda.synchronize()
        gs = torch.cuda.CUDAGraph()
        with torch.cuda.graph(gs):
            dstep()
        run_s = gs.replay
    s_ms = []
    for i in range(args.warmup + max(3, args.steps)):
        flush.zero_()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        run_s()
        e1.record(stream)
        torch.cuda.synchronize()
        if i >= args.warmup:
            s_ms.append(e0.elapsed_time(e1))
    decode_step = {"ms": sorted(s_ms)[len(s_ms) // 2], "t": w.T - 1,
                   "fused": tq.decode_step_fused(cache, w.Hq, w.T - 1),
                   "what": "append row T-1 (quantize) + attend over T rows, one tq_decode_step call"}

    if world > 1:
        torch.distributed.barrier()
    if rank != 0:
        if world > 1:
            torch.distributed.destroy_process_group()
        return

    dec_frac = (dec_bytes / (sum(d_ms) / len(d_ms) * 1e-3) / 1e9) / hbm
    q_frac = (qnt_bytes / (sum(q_ms) / len(q_ms) * 1e-3) / 1e9) / hbm
    dominant = "tq_quantize" if sum(q_ms) >= sum(d_ms) else "tq_decode_attn"

    def roof(name, bytes_per_launch, ms):
        achieved = bytes_per_launch / (ms * 1e-3) / 1e9
        traffic, note = dram_traffic(name, args.workload, args.batch, args.context)
        return {"kernel": name, "bound": "hbm", "achieved": achieved, "peak": hbm, "unit": "GB/s",
                "frac": achieved / hbm, "traffic": traffic, "traffic_note": note,
                "algorithmic_bytes": bytes_per_launch, "peak_kind": peak_kind,
                "spec_peak": SPEC_HBM_GBS, "frac_of_spec": achieved / SPEC_HBM_GBS}

    per_launch_q = qnt_bytes / n_chunks
    roof_q = roof("tq_quantize", per_launch_q, (sum(q_ms) / len(q_ms)) / n_chunks)
    roof_d = roof("tq_decode_attn", dec_bytes, sum(d_ms) / len(d_ms))
    cb = cpu_baseline(w) if (world == 1 and not args.no_cpu_baseline) else None
    line = {
        "metric": "compressed-KV decode-attn GB/s (% HBM peak); tq_quantize tokens/s",
        "value": dec_gbs, "unit": "GB/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": total_ms / args.steps, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f16 mma / f32 accumulate (decode); f32+f64 (quantize)",
        "data": "synthetic", "config": workload_config(w, parallelism=f"replicas x{world}",
                                                      launch="direct" if args.no_graph else "cuda graph per op"),
        "decode_hbm_frac": dec_frac, "decode_spec_frac": dec_frac * hbm / SPEC_HBM_GBS,
        "decode_ms": sum(d_ms) / len(d_ms),
        "quantize_tokens_per_s": q_tok_s, "quantize_GBps": q_gbs, "quantize_hbm_frac": q_frac,
        "quantize_spec_frac": q_frac * hbm / SPEC_HBM_GBS, "quantize_ms": sum(q_ms) / len(q_ms),
        "exempt": exempt,
        "roofline": roof_q if dominant == "tq_quantize" else roof_d,
        "roofline_decode": roof_d, "roofline_quantize": roof_q,
        "cpu_baseline": cb, "e2e": e2e,
        "gpu_launches": args.steps * (n_chunks + 2),
        "decode_step": decode_step,
        "quantize_fp64_fixups": {"coords": tq.quantize_code_fixups(), "key_vectors": tq.quantize_vector_fixups(),
                                 "calls": (args.warmup + args.steps) * n_chunks},
        "clocks": clk.summary(),
    }
    print(json.dumps(line), flush=True)
    if world > 1:
        torch.distributed.destroy_process_group()


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="tq", choices=["tq", "reference"])
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD, choices=W.CONFIG_ORDER)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-graph", action="store_true", help="launch every op directly in the timed steps")
    ap.add_argument("--rotation", default="haar", choices=["haar", "hadamard"],
                    help="Pi: dense Haar-random (default) or the structured D1 H D2 H D3 / 128")
    ap.add_argument("--layout", default="plain", choices=["plain", "mixed"],
                    help="cache layout: plain, or outlier-aware mixed precision (3.5 bits: the outlier "
                         "half of the channels at 4 bits, the rest at 3; needs 4-bit keys and values)")
    ap.add_argument("--batch", type=int, default=None, help="override the workload's batch")
    ap.add_argument("--context", type=int, default=None, help="override the workload's context")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3
    w = W.CONFIGS[args.workload]
    if args.batch is not None or args.context is not None:
        w = w.scaled(B=args.batch, T=args.context, name=w.name + "(resized)")
    if args.rotation != w.rotation:
        w = dataclasses.replace(w, rotation=args.rotation)
    if args.layout != w.layout:
        if w.k_bits != 4 or w.v_bits != 4:
            ap.error("--layout mixed needs a workload with 4-bit keys and values")
        w = dataclasses.replace(w, layout=args.layout)
    if args.impl == "reference":
        run_reference(args, w)
    else:
        run_gpu(args, w)


if __name__ == "__main__":
    main()
