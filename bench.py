#!/usr/bin/env python
"""Benchmark of the exact-attention hot path on B200.

One step is one pass of the whole hot path over one batch of synthetic input:
  prefill  causal GQA attention with RoPE, B=2, Hq=32, Hkv=8, N=8192, D=128 (attn_fwd: the
           query/key rotation pass plus the attention kernel), and
  decode   one paged-KV decode token for 64 sequences with lengths uniform in [512, 16384],
           Hq=32, Hkv=8, D=128, 16-token pages (attn_decode_paged: split kernel plus merge).
The headline value is prefill TFLOP/s (algorithmic FLOPs = 4*D per unmasked (query, key) pair per
query head) over the device time of the prefill calls; the decode line reports KV-cache GB/s
(algorithmic bytes = every cached K/V byte of every sequence once, plus q, o, lse, block table and
lengths) over the decode calls' device time.

Usage: python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
With N > 1 it runs under torchrun, one process per GPU; every rank runs its own copy of the
workload (weak scaling, no data-path collective) and rank 0 prints one JSON line.
--impl reference times the fp64 CPU oracle (the reference arm of this benchmark) on a bounded
sample of the same workload.
"""
import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from exact_attention_161_b200 import synth  # noqa: E402

PREFILL = synth.GQA_CAUSAL_N8192
DECODE = synth.PAGED_DECODE_64
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
DATASHEET_BF16_TFLOPS = 2250.0
DATASHEET_HBM_GBS = 8000.0
KERNEL_SOURCES = ["exact_attention_161_b200/csrc/fwd_sm100.cuh", "exact_attention_161_b200/csrc/decode.cuh",
                  "exact_attention_161_b200/csrc/bwd_sm100.cuh", "exact_attention_161_b200/csrc/ptx.cuh",
                  "exact_attention_161_b200/csrc/rope.cuh", "exact_attention_161_b200/csrc/common.cuh",
                  "exact_attention_161_b200/csrc/attn_api.cu"]


# ------------------------------------------------------------------------------ workload arithmetic
def visible_pairs(N, causal, window):
    """Unmasked (query, key) pairs of one head: N^2, N(N+1)/2, or sum_i min(i+1, w)."""
    if not causal:
        return N * N
    if window <= 0 or window >= N:
        return N * (N + 1) // 2
    w = window
    return w * (w + 1) // 2 + (N - w) * w


def prefill_flops(cfg=None):
    cfg = cfg or PREFILL
    return 4 * cfg.D * visible_pairs(cfg.N, cfg.causal, cfg.window) * cfg.B * cfg.Hq


def prefill_label():
    """Metric label of the timed prefill workload (the default is the causal GQA N=8192 one)."""
    c = PREFILL
    if c is synth.GQA_CAUSAL_N8192:
        return "causal GQA prefill B2 Hq32 Hkv8 N8192 D128, RoPE 5e5"
    mask = ("causal, window %d" % c.window) if c.window else ("causal" if c.causal else "no mask")
    rope = (", RoPE %g" % c.rope_base) if c.rope_base > 0 else ""
    return "prefill B%d Hq%d Hkv%d N%d D%d, %s%s" % (c.B, c.Hq, c.Hkv, c.N, c.D, mask, rope)


def decode_bytes(cache):
    kv = int(cache.seq_lens.to(torch.int64).sum()) * 2 * cache.Hkv * cache.D * 2
    io = cache.q.numel() * 2 * 2 + cache.num_seqs * cache.Hq * 4
    tables = cache.num_seqs * 4 + sum(((int(n) + cache.page_size - 1) // cache.page_size)
                                      for n in cache.seq_lens) * 4
    return kv + io + tables


def step_bytes(cache, T):
    """Algorithmic bytes of a decode step with T new tokens per sequence: the cache read once, the
    new keys and values read and written into their slots, T query rows in and out, LSE, tables."""
    S, Hq, Hkv, D = cache.num_seqs, cache.Hq, cache.Hkv, cache.D
    kv = int(cache.seq_lens.to(torch.int64).sum()) * 2 * Hkv * D * 2
    append = S * T * Hkv * D * 2 * 2 * 2
    io = S * T * Hq * D * 2 * 2 + S * T * Hq * 4
    tables = S * 4 + sum(((int(n) + cache.page_size - 1) // cache.page_size) for n in cache.seq_lens) * 4
    return kv + append + io + tables


# ------------------------------------------------------------------------------ ranks
def dist_env():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return rank, world, local


def init_dist(world, backend):
    if world > 1 and not torch.distributed.is_initialized():
        import datetime
        torch.distributed.init_process_group(backend=backend, timeout=datetime.timedelta(seconds=120))


def barrier(world):
    if world > 1:
        torch.distributed.barrier()


def reduce_max(value, world, device=None):
    """Max of a float over ranks (every rank takes the same collective steps)."""
    if world == 1:
        return float(value)
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def job_throughput(units_per_rank, world, seconds):
    """Whole-job throughput: units processed by all ranks over the slowest rank's time."""
    return units_per_rank * world / seconds


# ------------------------------------------------------------------------------ clocks, peaks
class ClockSampler:
    """nvidia-smi sampling of SM clock and throttle reasons during the timed region."""
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index):
        self.device_index = device_index
        self.proc = None
        self.path = None

    def start(self):
        try:
            uuid = "GPU-" + str(torch.cuda.get_device_properties(self.device_index).uuid)
            fd, self.path = tempfile.mkstemp(suffix=".csv")
            os.close(fd)
            self.proc = subprocess.Popen(["nvidia-smi", "-i", uuid, "--query-gpu=" + self.FIELDS,
                                          "--format=csv,noheader,nounits", "-lms", "200"],
                                         stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        rows = []
        for line in open(self.path):
            parts = [x.strip() for x in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                rows.append((float(parts[1]), float(parts[2]), parts[5:9]))
            except ValueError:
                continue
        os.unlink(self.path)
        if not rows:
            return None
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for _, _, flags in rows for i, f in enumerate(flags) if f.lower() == "active"})
        return {"sm_mhz": statistics.median(r[0] for r in rows), "sm_max_mhz": max(r[1] for r in rows),
                "reasons": reasons, "samples": len(rows)}


class NvmlSampler:
    """SM clock and clock-event (throttle) reasons from NVML every millisecond in a thread, for
    timed regions that are too short for nvidia-smi's interval."""

    REASONS = (("nvmlClocksEventReasonSwPowerCap", "sw_power_cap"),
               ("nvmlClocksEventReasonHwSlowdown", "hw_slowdown"),
               ("nvmlClocksEventReasonHwThermalSlowdown", "hw_thermal_slowdown"),
               ("nvmlClocksEventReasonSwThermalSlowdown", "sw_thermal_slowdown"),
               ("nvmlClocksEventReasonHwPowerBrakeSlowdown", "hw_power_brake_slowdown"))

    def __init__(self, device_index, interval_s=0.001):
        self.device_index, self.interval_s = device_index, interval_s
        self.samples, self.reason_bits, self.thread, self.stop_flag = [], 0, None, False

    def start(self):
        try:
            import threading
            import pynvml
            pynvml.nvmlInit()
            handle = pynvml.nvmlDeviceGetHandleByIndex(self.device_index)
        except Exception:
            return

        def run():
            import pynvml
            # the reasons query has two names across NVML versions; a driver may support neither
            reason_fns = [getattr(pynvml, f) for f in ("nvmlDeviceGetCurrentClocksEventReasons",
                                                        "nvmlDeviceGetCurrentClocksThrottleReasons")
                          if hasattr(pynvml, f)]
            while not self.stop_flag:
                try:
                    self.samples.append(pynvml.nvmlDeviceGetClockInfo(handle, pynvml.NVML_CLOCK_SM))
                except Exception:
                    return
                while reason_fns:
                    try:
                        self.reason_bits |= int(reason_fns[0](handle))
                        break
                    except Exception:
                        reason_fns.pop(0)
                time.sleep(self.interval_s)

        self.thread = threading.Thread(target=run, daemon=True)
        self.thread.start()

    def reasons(self):
        import pynvml
        return sorted(label for attr, label in self.REASONS
                      if hasattr(pynvml, attr) and self.reason_bits & int(getattr(pynvml, attr)))

    def stop(self):
        if self.thread is None:
            return None
        self.stop_flag = True
        self.thread.join(timeout=1.0)
        if not self.samples:
            return None
        return {"sm_mhz_median": statistics.median(self.samples), "sm_mhz_min": min(self.samples),
                "samples": len(self.samples), "interval_ms": self.interval_s * 1e3, "reasons": self.reasons()}


def tensor_peak_for(peaks, peaks_kind, timed_s):
    """The bf16 GEMM peak that applies to a leg: the burst figure for a timed region under a second
    (clocks have not settled under the power cap yet), the sustained one for longer regions."""
    if timed_s < 1.0 or "bf16_tflops_sustained" not in peaks:
        return peaks["bf16_tflops"], "%s bf16 GEMM, burst (timed region %.3f s)" % (peaks_kind, timed_s)
    return peaks["bf16_tflops_sustained"], "%s bf16 GEMM, sustained (timed region %.1f s)" % (peaks_kind, timed_s)


def measured_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def kernel_source_hash():
    h = hashlib.sha256()
    for rel in KERNEL_SOURCES:
        with open(os.path.join(ROOT, rel), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def profiled_traffic(kind):
    """DRAM bytes per launch from the committed ncu summary, or None when the kernels changed
    after the counters were taken."""
    path = os.path.join(ROOT, "profiles", "traffic.txt")
    if not os.path.exists(path):
        return None
    with open(path) as f:
        d = json.load(f)
    if d.get("kernel_source_hash") != kernel_source_hash():
        return None
    return d.get(kind, {}).get("dram_bytes_per_launch")


# ------------------------------------------------------------------------------ CPU baseline (oracle)
def oracle_prefill_sample(q, k, v, budget_s):
    """Time the fp64 oracle on a bounded sample of prefill rows; returns (TFLOP/s, rows, seconds,
    threads). The rows are evenly spaced over every (batch, head, position) of the workload, so
    the mix of causal lengths matches it."""
    import oracle
    qb, kb, vb = synth.bits(q), synth.bits(k), synth.bits(v)
    N, D = PREFILL.N, PREFILL.D
    total = PREFILL.B * PREFILL.Hq * N

    def run(n_rows):
        rows = np.linspace(0, total - 1, n_rows).astype(np.int64)
        flops = int((4 * D * ((rows % N) + 1)).sum())
        t0 = time.perf_counter()
        oracle.attention(qb, kb, vb, causal=PREFILL.causal, window=PREFILL.window, rope_base=PREFILL.rope_base, scale=PREFILL.scale, rows=rows)
        return flops, time.perf_counter() - t0

    f, t = run(256)  # calibration (includes the one-off key rotation of every KV head)
    n = int(min(total, max(256, 256 * budget_s / max(t, 1e-3))))
    f, t = run(n)
    return f / t / 1e12, n, t, oracle.max_threads()


def oracle_decode_sample(cache, budget_s):
    import oracle
    S = cache.num_seqs

    def run(n_seq):
        sub = slice(0, n_seq)
        c = synth.PagedCache(cache.q[sub], cache.k_pages, cache.v_pages, cache.block_table[sub],
                             cache.seq_lens[sub], cache.page_size, cache.Hq, cache.Hkv, cache.D)
        t0 = time.perf_counter()
        oracle.decode_paged(synth.bits(c.q), synth.bits(c.k_pages), synth.bits(c.v_pages), c.block_table.numpy(),
                            c.seq_lens.numpy())
        return decode_bytes(c), time.perf_counter() - t0

    b, t = run(1)
    n = int(min(S, max(1, budget_s / max(t, 1e-3))))
    b, t = run(n)
    return b / t / 1e9, n, t


# ------------------------------------------------------------------------------ our arm
def time_loop(fn, calls, stream, world, dev):
    """Mean ms per call of `calls` back-to-back calls on `stream` (events on that stream), after
    the caller's warm-up; the max over ranks."""
    barrier(world)
    torch.cuda.synchronize()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record(stream)
    for _ in range(calls):
        fn()
    b.record(stream)
    torch.cuda.synchronize()
    return reduce_max(a.elapsed_time(b), world, dev) / calls


def e2e_pipeline(steps, h2d, compute, d2h, dev):
    """End-to-end rate through the public API: step i's host->device copies (pinned host buffers),
    its compute and its device->host copies run on three streams, so step i+1's upload, step i's
    compute and step i-1's download overlap. Two device buffer sets alternate; events order each
    reuse. h2d(i, stream), compute(i, stream), d2h(i, stream) enqueue step i's work for buffer set
    i % 2. Returns ms for `steps` steps, from the first upload to the last download (one untimed
    pass first)."""
    s_up, s_run, s_down = (torch.cuda.Stream(device=dev) for _ in range(3))
    ev = lambda: torch.cuda.Event(enable_timing=True)

    def run(n):
        up, ran, down = [ev() for _ in range(n)], [ev() for _ in range(n)], [ev() for _ in range(n)]
        t0, t1 = ev(), ev()
        t0.record(s_up)
        for i in range(n):
            if i >= 2:
                s_up.wait_event(ran[i - 2])     # buffer set i % 2 is free once step i-2 computed
            h2d(i, s_up)
            up[i].record(s_up)
            s_run.wait_event(up[i])
            if i >= 2:
                s_run.wait_event(down[i - 2])   # its outputs were read back
            compute(i, s_run)
            ran[i].record(s_run)
            s_down.wait_event(ran[i])
            d2h(i, s_down)
            down[i].record(s_down)
        t1.record(s_down)
        torch.cuda.synchronize()
        return t0.elapsed_time(t1)

    run(2)
    return run(steps)


def run_ours(args, rank, world, local):
    from exact_attention_161_b200 import api
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    init_dist(world, "nccl")
    stream = torch.cuda.current_stream()

    do_prefill = args.only in ("all", "prefill")
    do_decode = args.only in ("all", "decode")
    if do_prefill:
        q_h, k_h, v_h = synth.prefill_inputs_for(PREFILL)
        q, k, v = q_h.to(dev), k_h.to(dev), v_h.to(dev)
        o = torch.empty_like(q)
        lse = torch.empty((PREFILL.B, PREFILL.Hq, PREFILL.N), dtype=torch.float32, device=dev)
    if do_decode:
        cache_h = synth.paged_decode_inputs_for(DECODE)
        dq, kp, vp = cache_h.q.to(dev), cache_h.k_pages.to(dev), cache_h.v_pages.to(dev)
        bt, sl = cache_h.block_table.to(dev), cache_h.seq_lens.to(dev)
        do = torch.empty_like(dq)
        dlse = torch.empty((DECODE.num_seqs, DECODE.Hq), dtype=torch.float32, device=dev)
        ws = torch.empty(api.decode_workspace_size(DECODE.num_seqs, cache_h.max_blocks, DECODE.page_size,
                                                   DECODE.Hq, DECODE.D), dtype=torch.uint8, device=dev)

    def prefill():
        api.attn_fwd(q, k, v, causal=PREFILL.causal, window=PREFILL.window, rope_base=PREFILL.rope_base,
                     o=o, lse=lse, stream=stream)

    def decode():
        api.attn_decode_paged(dq, kp, vp, bt, sl, o=do, lse=dlse, workspace=ws, stream=stream)

    for _ in range(args.warmup):
        if do_prefill:
            prefill()
        if do_decode:
            decode()
    torch.cuda.synchronize()
    if api.device_status() != 0:
        raise RuntimeError("device status raised during warm-up")

    K = args.steps
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(K)]
    clocks = ClockSampler(local)
    nvml = NvmlSampler(local)
    barrier(world)
    torch.cuda.synchronize()
    clocks.start()
    time.sleep(0.3)  # let the sampler take its first reading
    nvml.start()
    t_start = torch.cuda.Event(enable_timing=True)
    t_end = torch.cuda.Event(enable_timing=True)
    t_start.record(stream)
    for s in range(K):
        ev[s][0].record(stream)
        if do_prefill:
            prefill()
        ev[s][1].record(stream)
        if do_decode:
            decode()
        ev[s][2].record(stream)
    t_end.record(stream)
    torch.cuda.synchronize()
    nvml_clk = nvml.stop()
    barrier(world)
    clk = clocks.stop()
    if clk is not None and nvml_clk is not None:
        clk["nvml"] = nvml_clk
        # the reasons either sampler saw during the timed region
        clk["reasons"] = sorted(set(clk.get("reasons", [])) | set(nvml_clk.get("reasons", [])))
    total_ms = t_start.elapsed_time(t_end)
    prefill_ms = [ev[s][0].elapsed_time(ev[s][1]) for s in range(K)]
    decode_ms = [ev[s][1].elapsed_time(ev[s][2]) for s in range(K)]
    status = api.device_status()

    total_ms_max = reduce_max(total_ms, world, dev)
    prefill_sum_max = reduce_max(sum(prefill_ms), world, dev)
    decode_sum_max = reduce_max(sum(decode_ms), world, dev)
    flops = prefill_flops()
    dbytes = decode_bytes(cache_h) if do_decode else 0
    value = job_throughput(flops * K, world, prefill_sum_max / 1e3) / 1e12 if do_prefill else None
    decode_value = job_throughput(dbytes * K, world, decode_sum_max / 1e3) / 1e9 if do_decode else None

    # ---- the attention kernel alone: the same call without RoPE launches only attn_fwd_kernel (the
    # same instance; the rotation pass is skipped), so its event time is that kernel's launch time
    kern = None
    if do_prefill and args.kernel_calls > 0:
        def kernel_only():
            api.attn_fwd(q, k, v, causal=PREFILL.causal, window=PREFILL.window, rope_base=0.0, o=o, lse=lse,
                         stream=stream)

        for _ in range(args.warmup):
            kernel_only()
        kern_ms = time_loop(kernel_only, args.kernel_calls, stream, world, dev)
        kern = {"ms_per_launch": round(kern_ms, 4), "launches": args.kernel_calls,
                "timed_s": kern_ms * args.kernel_calls / 1e3}

    # ---- the other prefill workloads through the same call (own loops; not part of the step)
    configs_out = None
    if do_prefill and args.config_calls > 0:
        configs_out = {}
        for cfg in synth.PREFILL_CONFIGS:
            if cfg is PREFILL:
                continue
            cq, ck, cv = (t.to(dev) for t in synth.prefill_inputs_for(cfg))
            co = torch.empty_like(cq)
            cl = torch.empty((cfg.B, cfg.Hq, cfg.N), dtype=torch.float32, device=dev)

            def cfg_call():
                api.attn_fwd(cq, ck, cv, causal=cfg.causal, window=cfg.window, rope_base=cfg.rope_base, o=co,
                             lse=cl, stream=stream)

            for _ in range(args.warmup):
                cfg_call()
            n_calls = args.config_calls * (20 if cfg.N <= 128 else 1)
            cms = time_loop(cfg_call, n_calls, stream, world, dev)
            if api.device_status() != 0:
                raise RuntimeError("device status raised during the %s loop" % cfg.name)
            cf = prefill_flops(cfg)
            configs_out[cfg.name] = {
                "value": round(job_throughput(cf, world, cms / 1e3) / 1e12, 3), "unit": "TFLOP/s",
                "ms_per_call": round(cms, 5), "calls": n_calls, "flops_per_call": cf,
                "timed_s": cms * n_calls / 1e3,
                "config": {"B": cfg.B, "Hq": cfg.Hq, "Hkv": cfg.Hkv, "N": cfg.N, "D": cfg.D, "causal": cfg.causal,
                           "window": cfg.window, "rope_base": cfg.rope_base}}
            del cq, ck, cv, co, cl

    # ---- backward of the prefill workload (its own loop; not part of the step)
    bwd = None
    if do_prefill and args.bwd_steps > 0:
        dout = synth.randn_bf16(tuple(q.shape), torch.Generator().manual_seed(PREFILL.seed + 1)).to(dev)
        gq, gk, gv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
        bws = torch.empty(api.bwd_workspace_size(PREFILL.B, PREFILL.Hq, PREFILL.Hkv, PREFILL.N, PREFILL.D,
                                                 PREFILL.rope_base), dtype=torch.uint8, device=dev)

        def backward():
            api.attn_bwd(q, k, v, o, lse, dout, causal=PREFILL.causal, window=PREFILL.window,
                         rope_base=PREFILL.rope_base, dq=gq, dk=gk, dv=gv, workspace=bws, stream=stream)

        prefill()
        for _ in range(args.warmup):
            backward()
        bwd_ms = time_loop(backward, args.bwd_steps, stream, world, dev)
        if api.device_status() != 0:
            raise RuntimeError("device status raised during the backward loop")
        bwd_flops = flops * 5 // 2  # five products per unmasked pair (S, dP, dV, dK, dQ) vs two forward
        bwd = {"metric": "attn bwd TFLOP/s (same workload; algorithmic FLOPs = 2.5 x forward)",
               "value": round(job_throughput(bwd_flops, world, bwd_ms / 1e3) / 1e12, 2), "unit": "TFLOP/s",
               "ms_per_call": round(bwd_ms, 4), "calls": args.bwd_steps, "timed_s": bwd_ms * args.bwd_steps / 1e3,
               "roofline": {"bound": "tensor", "achieved": round(bwd_flops / (bwd_ms / 1e3) / 1e12, 2),
                            "unit": "TFLOP/s", "note": "the whole call: rotation pass, prep (which also zeroes the dq sums), the gradient kernel, the dq store"}}
        del dout, gq, gk, gv, bws

    # ---- position variants of the prefill workload (own loops; not part of the step)
    variants = None
    if do_prefill and args.variant_calls > 0:
        variants = {}
        slopes = synth.alibi_slopes(PREFILL.Hq).to(dev)
        for name, kw in (("alibi", dict(alibi_slopes=slopes)),
                         ("half_split_rope_ntk4", dict(rope_half_split=True, rope_ntk_factor=4.0))):
            def variant_call():
                api.attn_fwd_pos(q, k, v, causal=PREFILL.causal, window=PREFILL.window, rope_base=PREFILL.rope_base,
                                 o=o, lse=lse, stream=stream, **kw)

            for _ in range(args.warmup):
                variant_call()
            vms = time_loop(variant_call, args.variant_calls, stream, world, dev)
            if api.device_status() != 0:
                raise RuntimeError("device status raised during the %s loop" % name)
            variants[name] = {"value": round(job_throughput(flops, world, vms / 1e3) / 1e12, 2), "unit": "TFLOP/s",
                              "ms_per_call": round(vms, 4), "calls": args.variant_calls,
                              "timed_s": vms * args.variant_calls / 1e3,
                              "roofline": {"bound": "tensor", "achieved": round(flops / (vms / 1e3) / 1e12, 2),
                                           "unit": "TFLOP/s"}}

    # ---- FP8 e4m3 prefill of the same shape (inputs quantised per tensor; no RoPE on this path)
    fp8 = None
    if do_prefill and args.fp8_calls > 0:
        f8 = synth.fp8_inputs_for(PREFILL)
        q8, k8, v8 = f8.q8.to(dev), f8.k8.to(dev), f8.v8.to(dev)

        def fp8_call():
            api.attn_fwd_fp8(q8, k8, v8, f8.descale_q, f8.descale_k, f8.descale_v, causal=PREFILL.causal,
                             window=PREFILL.window, o=o, lse=lse, stream=stream)

        for _ in range(args.warmup):
            fp8_call()
        fms = time_loop(fp8_call, args.fp8_calls, stream, world, dev)
        if api.device_status() != 0:
            raise RuntimeError("device status raised during the FP8 loop")
        fp8 = {"metric": "attn fwd TFLOP/s, e4m3 Q/K/V (per-tensor scales), same shape and mask, no RoPE",
               "value": round(job_throughput(flops, world, fms / 1e3) / 1e12, 2), "unit": "TFLOP/s", "dtype": "e4m3",
               "ms_per_call": round(fms, 4), "calls": args.fp8_calls, "timed_s": fms * args.fp8_calls / 1e3,
               "roofline": {"bound": "tensor", "achieved": round(flops / (fms / 1e3) / 1e12, 2), "unit": "TFLOP/s"}}
        del q8, k8, v8

    # ---- end to end through the public API: pinned host buffers, uploads, compute and downloads of
    # successive steps overlapped on three streams (prefill and decode timed as separate pipelines)
    E = min(args.e2e_steps, K) if (args.e2e_steps > 0 and args.only == "all") else 0
    e2e_value = e2e_decode = None
    if E:
        q_p, k_p, v_p = q_h.pin_memory(), k_h.pin_memory(), v_h.pin_memory()
        bufs = [(q, k, v, o, lse), tuple(torch.empty_like(t) for t in (q, k, v, o, lse))]
        outs_p = [(torch.empty(o.shape, dtype=o.dtype).pin_memory(), torch.empty(lse.shape, dtype=lse.dtype).pin_memory())
                  for _ in range(2)]

        def p_up(i, st):
            with torch.cuda.stream(st):
                for dst, src in zip(bufs[i % 2][:3], (q_p, k_p, v_p)):
                    dst.copy_(src, non_blocking=True)

        def p_run(i, st):
            bq, bk, bv, bo, bl = bufs[i % 2]
            api.attn_fwd(bq, bk, bv, causal=PREFILL.causal, window=PREFILL.window, rope_base=PREFILL.rope_base,
                         o=bo, lse=bl, stream=st)

        def p_down(i, st):
            with torch.cuda.stream(st):
                outs_p[i % 2][0].copy_(bufs[i % 2][3], non_blocking=True)
                outs_p[i % 2][1].copy_(bufs[i % 2][4], non_blocking=True)

        e_pre = reduce_max(e2e_pipeline(E, p_up, p_run, p_down, dev), world, dev)
        e2e_value = job_throughput(flops * E, world, e_pre / 1e3) / 1e12
        del bufs, outs_p
        dq_p, bt_p, sl_p = cache_h.q.pin_memory(), cache_h.block_table.pin_memory(), cache_h.seq_lens.pin_memory()
        dbufs = [(dq, bt, sl, do, dlse, ws),
                 tuple(torch.empty_like(t) for t in (dq, bt, sl, do, dlse, ws))]
        douts_p = [(torch.empty(do.shape, dtype=do.dtype).pin_memory(),
                    torch.empty(dlse.shape, dtype=dlse.dtype).pin_memory()) for _ in range(2)]

        def d_up(i, st):
            with torch.cuda.stream(st):
                for dst, src in zip(dbufs[i % 2][:3], (dq_p, bt_p, sl_p)):
                    dst.copy_(src, non_blocking=True)

        def d_run(i, st):
            bq, bbt, bsl, bo, bl, bws = dbufs[i % 2]
            api.attn_decode_paged(bq, kp, vp, bbt, bsl, o=bo, lse=bl, workspace=bws, stream=st)

        def d_down(i, st):
            with torch.cuda.stream(st):
                douts_p[i % 2][0].copy_(dbufs[i % 2][3], non_blocking=True)
                douts_p[i % 2][1].copy_(dbufs[i % 2][4], non_blocking=True)

        e_dec = reduce_max(e2e_pipeline(E, d_up, d_run, d_down, dev), world, dev)
        e2e_decode = job_throughput(dbytes * E, world, e_dec / 1e3) / 1e9
        del dbufs, douts_p
        if api.device_status() != 0:
            raise RuntimeError("device status raised during the end-to-end legs")
    h2d = sum(t.numel() * t.element_size() for t in (q_h, k_h, v_h)) if do_prefill else 0
    d2h = o.numel() * 2 + lse.numel() * 4 if do_prefill else 0
    dh2d = sum(t.numel() * t.element_size() for t in (cache_h.q, cache_h.block_table, cache_h.seq_lens)) if do_decode else 0
    dd2h = do.numel() * 2 + dlse.numel() * 4 if do_decode else 0

    # ---- decode step: append one or four new tokens per sequence (keys rotated, RoPE 1e4) and attend
    # with their rotated queries, on the same cache (runs after the legs above: it writes the cache)
    steps_out = None
    if do_decode and args.step_calls > 0:
        steps_out = {}
        S, Hq, Hkv, D = DECODE.num_seqs, DECODE.Hq, DECODE.Hkv, DECODE.D
        gen = torch.Generator().manual_seed(DECODE.seed + 7919)
        for T in (1, 4):
            sq = synth.randn_bf16((S, T, Hq, D), gen).to(dev)
            kn = synth.randn_bf16((S, T, Hkv, D), gen).to(dev)
            vn = synth.randn_bf16((S, T, Hkv, D), gen).to(dev)
            so = torch.empty_like(sq)
            slse = torch.empty((S, T, Hq), dtype=torch.float32, device=dev)
            sws = torch.empty(api.decode_step_workspace_size(S, T, cache_h.max_blocks, DECODE.page_size, Hq, D),
                              dtype=torch.uint8, device=dev)

            def step_call():
                api.attn_decode_step(sq, kp, vp, bt, sl, k_new=kn, v_new=vn, rope_base=10000.0, o=so, lse=slse,
                                     workspace=sws, stream=stream)

            for _ in range(args.warmup):
                step_call()
            ms = time_loop(step_call, args.step_calls, stream, world, dev)
            if api.device_status() != 0:
                raise RuntimeError("device status raised during the decode-step loop")
            sbytes = step_bytes(cache_h, T)
            steps_out["q_len=%d" % T] = {
                "value": round(job_throughput(sbytes, world, ms / 1e3) / 1e9, 1), "unit": "GB/s",
                "ms_per_call": round(ms, 4), "calls": args.step_calls, "bytes_per_call": sbytes,
                "roofline": {"bound": "hbm", "achieved": round(sbytes / (ms / 1e3) / 1e9, 1), "unit": "GB/s"}}

    if rank != 0:
        return None
    peaks, peaks_kind = measured_peaks()
    hbm = peaks["hbm_gbs"]
    if steps_out is not None:
        for key, v in steps_out.items():
            v["roofline"].update({"peak": hbm, "frac": round(v["roofline"]["achieved"] / hbm, 4),
                                  "peak_kind": "%s HBM copy" % peaks_kind,
                                  "traffic": profiled_traffic("decode_split" if key == "q_len=1" else "decode_step_split_q4")})
    pre_launch_ms = statistics.mean(prefill_ms)
    dec_launch_ms = statistics.mean(decode_ms)
    tflops_call = flops / (pre_launch_ms / 1e3) / 1e12 if do_prefill else float("nan")
    gbs_launch = dbytes / (dec_launch_ms / 1e3) / 1e9 if do_decode else float("nan")
    step_peak, step_peak_kind = tensor_peak_for(peaks, peaks_kind, prefill_sum_max / 1e3)
    if kern is not None:
        k_peak, k_kind = tensor_peak_for(peaks, peaks_kind, kern["timed_s"])
        k_tf = flops / (kern["ms_per_launch"] / 1e3) / 1e12
        roof = {"bound": "tensor", "achieved": round(k_tf, 2), "peak": k_peak, "unit": "TFLOP/s",
                "frac": round(k_tf / k_peak, 4), "peak_kind": k_kind, "frac_of_2250": round(k_tf / DATASHEET_BF16_TFLOPS, 4),
                "traffic": profiled_traffic("attn_fwd"),
                "kernel": "attn_fwd_kernel<128, 0, 0>, its own launches (%d, %.4f ms each) timed in a loop of the "
                          "same call without RoPE (the rotation pass is the only launch RoPE adds)"
                          % (kern["launches"], kern["ms_per_launch"]),
                "call": {"achieved": round(tflops_call, 2), "frac": round(tflops_call / step_peak, 4),
                         "peak_kind": step_peak_kind,
                         "note": "the whole attn_fwd call with RoPE in the timed step (rotation pass + attention kernel)",
                         "rotation_pass_traffic": profiled_traffic("rope_rows")}}
    else:
        roof = {"bound": "tensor", "achieved": round(tflops_call, 2), "peak": step_peak, "unit": "TFLOP/s",
                "frac": round(tflops_call / step_peak, 4), "peak_kind": step_peak_kind,
                "traffic": profiled_traffic("attn_fwd"), "kernel": "attn_fwd call (rotation pass + attention kernel)"}
    if configs_out is not None:
        for cname, cv in configs_out.items():
            cp, ck = tensor_peak_for(peaks, peaks_kind, cv["timed_s"])
            if cv["config"]["N"] <= 128:
                cv["latency_us"] = round(cv["ms_per_call"] * 1e3, 2)
                cv["roofline"] = {"bound": "latency", "note": "one CTA; no roofline claim"}
            else:
                cv["roofline"] = {"bound": "tensor", "achieved": cv["value"], "peak": cp, "unit": "TFLOP/s",
                                  "frac": round(cv["value"] / cp, 4), "peak_kind": ck}
    if bwd is not None:
        bp, bk = tensor_peak_for(peaks, peaks_kind, bwd["timed_s"])
        bwd["roofline"].update({"peak": bp, "frac": round(bwd["roofline"]["achieved"] / bp, 4), "peak_kind": bk,
                                "traffic": profiled_traffic("attn_bwd"),
                                "traffic_kernel": "attn_bwd_kernel<128> (dQ, dK and dV; five products per tile pair)"})
    if fp8 is not None:
        fp, fk = tensor_peak_for(peaks, peaks_kind, fp8["timed_s"])
        fp8["roofline"].update({"peak": 2.0 * fp, "frac": round(fp8["roofline"]["achieved"] / (2.0 * fp), 4),
                                "peak_kind": "2 x (%s) (nominal fp8:bf16 ratio 4.5:2.25)" % fk,
                                "traffic": profiled_traffic("attn_fwd_fp8")})
    if variants is not None:
        for vv in variants.values():
            vp_, vk = tensor_peak_for(peaks, peaks_kind, vv["timed_s"])
            vv["roofline"].update({"peak": vp_, "frac": round(vv["roofline"]["achieved"] / vp_, 4), "peak_kind": vk})
    line = {
        "metric": "attn fwd TFLOP/s (%s) & paged-decode KV GB/s" % prefill_label(),
        "value": round(value, 2) if do_prefill else None,
        "unit": "TFLOP/s",
        "n_gpus": world,
        "steps": K,
        "warmup": args.warmup,
        "ms_per_step": round(total_ms_max / K, 4),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "bf16",
        "data": "synthetic (seeded N(0,1) bf16; paged cache from a seeded permutation)",
        "config": {
            "workload": "prefill %s + decode %s" % (PREFILL.name, DECODE.name),
            "prefill": {"B": PREFILL.B, "Hq": PREFILL.Hq, "Hkv": PREFILL.Hkv, "N": PREFILL.N, "D": PREFILL.D,
                        "causal": PREFILL.causal, "window": PREFILL.window, "rope_base": PREFILL.rope_base,
                        "flops_per_step": flops},
            "decode": {"num_seqs": DECODE.num_seqs, "Hq": DECODE.Hq, "Hkv": DECODE.Hkv, "D": DECODE.D,
                       "page_size": DECODE.page_size, "total_tokens": cache_h.total_tokens if do_decode else None,
                       "bytes_per_step": dbytes},
            "l2": "inputs larger than L2 (prefill Q/K/V 201 MB, decode KV 2.2 GB); no flush",
            "parallelism": "replica per GPU" if world > 1 else "single GPU",
        },
        "decode": {"metric": "paged-decode KV GB/s", "value": round(decode_value, 1) if do_decode else None, "unit": "GB/s",
                   "ms_per_step": round(decode_sum_max / K, 4),
                   "roofline": {"bound": "hbm", "achieved": round(gbs_launch, 1), "peak": hbm,
                                "unit": "GB/s", "frac": round(gbs_launch / hbm, 4),
                                "peak_kind": "%s HBM copy" % peaks_kind, "frac_of_8TBs": round(gbs_launch / DATASHEET_HBM_GBS, 4),
                                "traffic": profiled_traffic("decode_split")},
                   "e2e": {"value": round(e2e_decode, 2) if E else None, "unit": "GB/s", "h2d_bytes_per_step": dh2d,
                           "d2h_bytes_per_step": dd2h, "overlap": "upload, compute and download on three streams"}},
        "roofline": roof,
        "e2e": {"value": round(e2e_value, 2) if E else None, "unit": "TFLOP/s", "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h, "steps": E,
                "overlap": "step i+1's upload, step i's compute and step i-1's download on three streams"},
        "gpu_launches": (2 * do_prefill + 2 * do_decode) * K,
        "prefill_configs": configs_out,
        "backward": bwd,
        "fp8": fp8,
        "position_variants": None if variants is None else dict(
            {"metric": "attn fwd TFLOP/s of the same prefill workload with ALiBi (slopes 2^(-8h/H)), and with "
                       "half-split RoPE pairing plus NTK-aware base scaling x4"}, **variants),
        "decode_step": None if steps_out is None else dict(
            {"metric": "decode step KV GB/s: append q_len new tokens per sequence (keys rotated, RoPE 1e4) into "
                       "the 64-sequence paged cache, then attend with their rotated queries"}, **steps_out),
        "device_status": status,
        "clocks": clk,
    }
    return line


def add_cpu_baseline(line, args):
    if args.no_cpu_baseline:
        line["cpu_baseline"] = None
        return
    q, k, v = synth.prefill_inputs_for(PREFILL)
    tf, n, t, threads = oracle_prefill_sample(q, k, v, args.cpu_budget)
    cache = synth.paged_decode_inputs_for(DECODE)
    gbs, ns, td = oracle_decode_sample(cache, args.cpu_budget / 2)
    line["cpu_baseline"] = {"value": round(tf, 6), "unit": "TFLOP/s", "cores": threads, "kind": "oracle",
                            "sample": "%d query rows evenly spaced over all (batch, head, position) of the "
                                      "prefill workload (causal, RoPE), %.1f s" % (n, t),
                            "decode": {"value": round(gbs, 4), "unit": "GB/s",
                                       "sample": "%d of 64 sequences, %.1f s" % (ns, td)}}


# ------------------------------------------------------------------------------ reference arm
def run_reference(args, rank, world):
    if rank != 0:
        return None
    import oracle
    q, k, v = synth.prefill_inputs_for(PREFILL)
    qb, kb, vb = synth.bits(q), synth.bits(k), synth.bits(v)
    # per-step budget so that warm-up + steps end within a few minutes
    per_step = max(0.05, min(5.0, 150.0 / (args.steps + args.warmup)))
    N, D = PREFILL.N, PREFILL.D
    rows_probe = np.linspace(0, N - 1, 16).astype(np.int64)
    t0 = time.perf_counter()
    oracle.attention(qb, kb, vb, causal=PREFILL.causal, window=PREFILL.window, rope_base=PREFILL.rope_base, scale=PREFILL.scale, rows=rows_probe)
    t_probe = time.perf_counter() - t0
    n_rows = int(max(4, min(N, 16 * per_step / max(t_probe, 1e-4))))
    rng = np.random.default_rng(0)
    flops_total, secs_total = 0, 0.0
    for s in range(args.warmup + args.steps):
        rows = np.sort(rng.choice(N, size=n_rows, replace=False)).astype(np.int64)
        t0 = time.perf_counter()
        oracle.attention(qb, kb, vb, causal=PREFILL.causal, window=PREFILL.window, rope_base=PREFILL.rope_base, scale=PREFILL.scale, rows=rows)
        dt = time.perf_counter() - t0
        if s >= args.warmup:
            flops_total += sum(4 * D * (int(i) + 1) for i in rows)
            secs_total += dt
    value = flops_total / secs_total / 1e12
    sample = ("%d random query rows of one head of the prefill workload per step (causal, RoPE); "
              "the oracle rotates that head's keys each step" % n_rows)
    return {
        "impl": "reference",
        "metric": "attn fwd TFLOP/s (%s) & paged-decode KV GB/s" % prefill_label(),
        "value": round(value, 6),
        "unit": "TFLOP/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": round(secs_total / args.steps * 1e3, 3),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "f64",
        "data": "synthetic",
        "config": {"workload": "prefill %s (bounded row sample on the host CPU)" % PREFILL.name},
        "cpu_baseline": {"value": round(value, 6), "unit": "TFLOP/s", "cores": oracle.max_threads(),
                         "kind": "oracle", "sample": sample},
        "e2e": {"value": round(value, 6), "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }


def parse_args(argv=None):
    ap = argparse.ArgumentParser(description=__doc__.splitlines()[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=400)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--e2e-steps", type=int, default=10, help="0 skips the end-to-end leg")
    ap.add_argument("--kernel-calls", type=int, default=20,
                    help="attention-kernel-only launches timed for the roofline; 0 skips")
    ap.add_argument("--config-calls", type=int, default=20,
                    help="calls timed per other prefill workload (x20 for the N=128 one); 0 skips")
    ap.add_argument("--bwd-steps", type=int, default=20, help="backward calls timed after the step loop; 0 skips")
    ap.add_argument("--step-calls", type=int, default=50, help="decode-step calls timed per q_len; 0 skips")
    ap.add_argument("--variant-calls", type=int, default=20, help="position-variant prefill calls timed each; 0 skips")
    ap.add_argument("--fp8-calls", type=int, default=20, help="FP8 prefill calls timed; 0 skips")
    ap.add_argument("--prefill-workload", choices=[c.name for c in synth.PREFILL_CONFIGS],
                    default=synth.GQA_CAUSAL_N8192.name,
                    help="prefill workload to time (default: the causal GQA N=8192 one)")
    ap.add_argument("--only", choices=["all", "prefill", "decode"], default="all",
                    help="time one half of the step only (profiling runs); the JSON line is then partial")
    ap.add_argument("--cpu-budget", type=float, default=15.0, help="seconds of oracle time for the CPU baseline")
    ap.add_argument("--no-cpu-baseline", action="store_true", help="skip the oracle timing (profiling runs)")
    args = ap.parse_args(argv)
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    return args


def main(argv=None):
    global PREFILL
    args = parse_args(argv)
    PREFILL = next(c for c in synth.PREFILL_CONFIGS if c.name == args.prefill_workload)
    rank, world, local = dist_env()
    if world != args.gpus:
        print("warning: --gpus %d but WORLD_SIZE %d; using WORLD_SIZE" % (args.gpus, world), file=sys.stderr)
    if args.impl == "reference":
        line = run_reference(args, rank, world)
    else:
        line = run_ours(args, rank, world, local)
        if line is not None and world == 1 and args.only == "all":
            add_cpu_baseline(line, args)
        elif line is not None:
            line["cpu_baseline"] = None
    if line is not None:
        print(json.dumps(line), flush=True)
    if world > 1 and torch.distributed.is_initialized():
        torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
