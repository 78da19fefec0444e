"""Benchmark of the SAS gated block-sparse attention library on B200.

One step = one pass of the training hot path over one synthetic batch of the
Qwen3-4B-shaped layer (B=1, 32 q heads / 8 KV heads, d=128, T=16384, b=64,
K=16): gate softmax + Top-K (sas_gate_topk), the gated sparse forward and
its backward into q, k, v and the selector scores, as the pair that carries
the forward's output residual (sas_attn_fwd_res / sas_attn_bwd_res: the same
results, the backward's row sums from o and the residual). `value` is the algorithmic fwd+bwd TFLOP/s of the whole job
(14*d FLOPs per attended (query, key) pair per query head; dense and skipped
work never counted). Beside it the line reports the decode hot path (one token
per sequence over 64K and 512K caches, gates off and on) in GB/s of selected
K/V bytes, the same library's dense kernels, the roofline of the dominant
kernel, an end-to-end figure through host buffers and the float64 oracle's
CPU throughput.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

With N > 1 every rank runs its own batch (weak scaling, no collective on the
data path); the step time is the max over ranks. Started without a torchrun
environment, `--gpus N` re-launches itself under torch.distributed.run with N
ranks on 127.0.0.1.
"""
from __future__ import annotations

import argparse
import json
import os
import socket
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from block_sparse_attention_sas_b200 import dist as D  # noqa: E402
from block_sparse_attention_sas_b200 import workloads as W  # noqa: E402

TRAIN = W.QWEN3_4B_TRAIN
DECODES = [(W.QWEN3_4B_DECODE, 0), (W.QWEN3_4B_DECODE, 1), (W.QWEN3_14B_DECODE, 0)]
METRIC = "gated sparse attn fwd+bwd TFLOP/s & decode GB/s; % of B200 roofline"
L2_FLUSH_BYTES = 256 << 20
# GPU-side sleep after each flush (about 1 ms at 1.9 GHz): the host enqueues
# the whole timed step behind it, so the events bracket back-to-back kernels
# and not host launch latency.
HEAD_START_CYCLES = 2_000_000


# DRAM bytes (read + write) per call from ncu (dram__bytes_read.sum +
# dram__bytes_write.sum summed over the call's kernels, one --set full capture
# each of `bench.py --profile-train 8192`), for the kernels as they stand:
# the backward with the residual D pass is D-from-o 206.1 MB, dK/dV 1229.5 MB
# and dq 608.6 MB per call at T = 8192. The capture ran the same layer at
# T = 8192; the figure is scaled to T = 16384 by the attended pairs
# (536.1 M / 259.1 M), which every kernel's work follows.
MEASURED_TRAFFIC = {
    ("qwen3-4b-train B1 Hq32/Hkv8 T16384 d128 b64 K16", "sas_attn_bwd_res"):
        (206.1e6 + 1229.5e6 + 608.6e6) * 536084480 / 259129344,
}


def attended_pairs(B, Hq, T, b, K):
    """Sum over query rows of the keys each row attends (selected blocks + causal current)."""
    N = (T + b - 1) // b
    tot = 0
    for j in range(N):
        rows = min(T, (j + 1) * b) - j * b
        tot += rows * b * min(K, j) + rows * (rows + 1) // 2
    return tot * B * Hq


def train_flops(cfg):
    pairs = attended_pairs(cfg.B, cfg.Hq, cfg.T, cfg.b, cfg.K)
    return 4 * cfg.d * pairs, 10 * cfg.d * pairs


def decode_bytes(cfg, dense=False):
    """Algorithmic bytes of one decode call: the attended K and V rows
    (selected history blocks + the current block) plus q, o, idx and gates."""
    e = 2 if cfg.dtype == "bf16" else 4
    n_blocks = (cfg.C + 1) if dense else (min(cfg.K, cfg.C) + 1)
    cur = cfg.L - cfg.C * cfg.b
    rows = (n_blocks - 1) * cfg.b + cur
    kv = 2 * rows * cfg.d * e * cfg.B * cfg.Hkv
    small = 2 * cfg.B * cfg.Hq * cfg.d * e + (0 if dense else cfg.B * cfg.Hkv * cfg.K * 4)
    return kv + small


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        d = json.load(open(p))
        return {"hbm_gbs": float(d["hbm_gbs"]), "bf16_tflops": float(d["bf16_tflops"]),
                "bf16_tflops_sustained": float(d.get("bf16_tflops_sustained", d["bf16_tflops"])),
                "source": "measured"}
    except Exception:
        return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0,
                "source": "fallback"}


# ---------------------------------------------------------------------- clocks

class ClockSampler:
    """SM clocks and throttle reasons sampled while the timed region runs: an
    NVML polling thread (every 5 ms, read-only queries), else nvidia-smi
    every 50 ms. Samples taken before mark() (the idle lead-in) are dropped."""
    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
    NAMES = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")

    def __init__(self, gpu_id: str | None):
        self.proc = None
        self.path = None
        self.gpu_id = gpu_id
        self.skip = 0
        self.samples = []  # (sm_mhz, sm_max_mhz, reasons) from NVML
        self.thread = None
        self.stop = False

    def _nvml_loop(self, nv, h):
        bits = {"hw_slowdown": nv.nvmlClocksEventReasonHwSlowdown,
                "hw_thermal_slowdown": nv.nvmlClocksEventReasonHwThermalSlowdown,
                "sw_thermal_slowdown": nv.nvmlClocksEventReasonSwThermalSlowdown,
                "sw_power_cap": nv.nvmlClocksEventReasonSwPowerCap}
        smax = nv.nvmlDeviceGetMaxClockInfo(h, nv.NVML_CLOCK_SM)
        while not self.stop:
            try:
                sm = nv.nvmlDeviceGetClockInfo(h, nv.NVML_CLOCK_SM)
                r = nv.nvmlDeviceGetCurrentClocksEventReasons(h)
                self.samples.append((sm, smax, [n for n, b in bits.items() if r & b]))
            except Exception:
                pass
            time.sleep(0.005)

    def __enter__(self):
        try:
            import threading

            import pynvml as nv
            nv.nvmlInit()
            h = nv.nvmlDeviceGetHandleByPciBusId(self.gpu_id) if self.gpu_id else \
                nv.nvmlDeviceGetHandleByIndex(0)
            self.thread = threading.Thread(target=self._nvml_loop, args=(nv, h), daemon=True)
            self.thread.start()
            t0 = time.time()
            while not self.samples and time.time() - t0 < 2.0:
                time.sleep(0.005)
            if self.samples:
                return self
            self.stop = True
        except Exception:
            self.thread = None
        try:
            fd, self.path = tempfile.mkstemp(suffix=".csv")
            os.close(fd)
            cmd = ["nvidia-smi", f"--query-gpu={self.Q}", "--format=csv,noheader,nounits",
                   "-lms", "50"]
            if self.gpu_id:
                cmd += ["-i", self.gpu_id]
            self.proc = subprocess.Popen(cmd, stdout=open(self.path, "w"),
                                         stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None
        # nvidia-smi takes a moment to start: wait (up to 5 s) for its first
        # sample so the timed region that follows is covered.
        t0 = time.time()
        while self.proc is not None and time.time() - t0 < 5.0:
            if os.path.getsize(self.path) > 0:
                break
            time.sleep(0.02)
        return self

    def mark(self):
        """Samples taken before this call (the idle lead-in) are left out."""
        if self.thread is not None and not self.stop:
            self.skip = len(self.samples)
            return
        try:
            with open(self.path) as f:
                self.skip = sum(1 for _ in f)
        except (OSError, TypeError):
            self.skip = 0

    def __exit__(self, *a):
        self.stop = True
        if self.thread is not None:
            self.thread.join(timeout=1.0)
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()

    def summary(self):
        if self.samples and self.proc is None:
            got = self.samples[self.skip:] or self.samples[-1:]
            reasons = sorted({r for _, _, rs in got for r in rs})
            return {"sm_mhz": statistics.median(x for x, _, _ in got),
                    "sm_max_mhz": max(y for _, y, _ in got), "reasons": reasons,
                    "samples": len(got), "source": "nvml 5 ms"}
        if not self.path or not os.path.exists(self.path):
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"], "samples": 0}
        sm, smax, reasons = [], [], set()
        for n_line, line in enumerate(open(self.path)):
            if n_line < self.skip:
                continue
            f = [x.strip() for x in line.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                smax.append(float(f[2]))
            except ValueError:
                continue
            for n, v in zip(self.NAMES, f[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        os.unlink(self.path)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"], "samples": 0}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(smax),
                "reasons": sorted(reasons), "samples": len(sm), "source": "nvidia-smi 50 ms"}


def gpu_pci_id(torch, dev):
    try:
        p = torch.cuda.get_device_properties(dev)
        return "%08X:%02X:%02X.0" % (p.pci_domain_id, p.pci_bus_id, p.pci_device_id)
    except Exception:
        vis = os.environ.get("CUDA_VISIBLE_DEVICES")
        return vis.split(",")[dev.index or 0] if vis else str(dev.index or 0)


# ------------------------------------------------------------------ CPU side

def cpu_model():
    try:
        for line in open("/proc/cpuinfo"):
            if line.startswith("model name"):
                return line.split(":", 1)[1].strip()
    except OSError:
        pass
    return "unknown"


def blas_threads():
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads") for i in threadpool_info() if i.get("user_api") == "blas"]
        return int(max(n)) if n else os.cpu_count()
    except Exception:
        return os.cpu_count()


def oracle_sample(cfg, kv_heads=(0,), x=None):
    """The float64 oracle on a bounded sample of the training layer: every query
    block of the given KV heads (gates, Top-K, forward, backward). Returns
    (seconds, algorithmic FLOPs of the sample)."""
    from oracle import sas_oracle as O
    if x is None:
        x = W.make_train_inputs(cfg)
    t0 = time.perf_counter()
    for kvh in kv_heads:
        sl = slice(kvh, kvh + 1)
        g, lg, ix = O.gate_topk(x.scores[:, sl], cfg.K)
        q = x.q[:, kvh * cfg.G:(kvh + 1) * cfg.G]
        k, v = x.k[:, sl], x.v[:, sl]
        dO = x.dO[:, kvh * cfg.G:(kvh + 1) * cfg.G]
        O.attn_fwd(q, k, v, ix, lg, cfg.b)
        O.attn_bwd(q, k, v, dO, ix, g, lg, cfg.b)
    dt = time.perf_counter() - t0
    f, b = train_flops(cfg)
    return dt, (f + b) * len(kv_heads) / (cfg.B * cfg.Hkv)


# ------------------------------------------------------------------ our arm

def run_ours(args):
    import torch
    from block_sparse_attention_sas_b200 import _lib as S

    rank, local_rank, world = D.env_rank()
    if not torch.cuda.is_available():
        raise SystemExit("bench.py needs a CUDA device")
    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    D.init("nccl", timeout_s=300)
    peaks = load_peaks()
    cfg = TRAIN
    seed = D.rank_seed(cfg.seed, rank)

    # ---- inputs: host (pinned) and device copies
    x = W.make_train_inputs(cfg, seed=seed)
    bf = torch.bfloat16

    def pin(a, dt):
        t = torch.from_numpy(a)
        if dt is not None:
            t = t.to(dt)
        return t.pin_memory()

    h = dict(q=pin(x.q, bf), k=pin(x.k, bf), v=pin(x.v, bf), dO=pin(x.dO, bf),
             scores=pin(x.scores, None))
    d = {n: t.to(dev, non_blocking=False) for n, t in h.items()}
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)
    f_fwd, f_bwd = train_flops(cfg)

    def step(inp, ev=None):
        if ev:
            ev[0].record(stream)
        gates, idx = S.gate_topk(inp["scores"], cfg.K, causal=True)
        if ev:
            ev[1].record(stream)
        o, o_res, lse = S.attn_fwd_res(inp["q"], inp["k"], inp["v"], idx, gates, cfg.b)
        if ev:
            ev[2].record(stream)
        dq, dk, dv, ds = S.attn_bwd_res(inp["q"], inp["k"], inp["v"], o, o_res, lse, inp["dO"],
                                        idx, gates,
                                    cfg.b)
        if ev:
            ev[3].record(stream)
        return o, dq, dk, dv, ds

    for _ in range(args.warmup):
        step(d)
    torch.cuda.synchronize(dev)
    st, raw = S.device_error()
    if st != 0:
        raise SystemExit(f"device error during warm-up: {raw:#x}")

    # ---- timed region: K steps, L2 flushed before each, CUDA events per step
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(args.steps)]
    n_launch0 = S.launch_count()
    with ClockSampler(gpu_pci_id(torch, dev)) as clk:
        D.barrier(dev)
        torch.cuda.synchronize(dev)
        clk.mark()
        t_wall = time.perf_counter()
        for i in range(args.steps):
            flush.zero_()
            torch.cuda._sleep(HEAD_START_CYCLES)
            step(d, evs[i])
        torch.cuda.synchronize(dev)
        t_wall = time.perf_counter() - t_wall
        D.barrier(dev)
    launches = S.launch_count() - n_launch0
    clocks = clk.summary()
    per = [[e[a].elapsed_time(e[a + 1]) for a in range(3)] for e in evs]  # ms
    step_ms = sum(sum(p) for p in per) / args.steps
    k_ms = {n: sum(p[i] for p in per) / args.steps for i, n in
            enumerate(("sas_gate_topk", "sas_attn_fwd_res", "sas_attn_bwd_res"))}
    step_ms_max = D.max_over_ranks(step_ms, dev)
    value = world * (f_fwd + f_bwd) / (step_ms_max * 1e-3) / 1e12

    # ---- e2e: host buffers in, every result out, through the same calls.
    # Three streams (host-to-device copies, compute, device-to-host copies)
    # and two device buffer sets, so step i's inputs cross PCIe while step
    # i - 1 computes and its results come back; the value is K steps over the
    # time from the first copy to the last result on the host side.
    e2e = run_e2e(S, torch, dev, h, d, step, args, world, f_fwd + f_bwd)

    # ---- decode lines (one call per timing, L2 flushed before each)
    decode_lines = []
    if not args.no_decode:
        decode_lines = bench_decode(S, torch, dev, stream, flush, peaks, args, rank)

    # ---- the Qwen3-8B training layer (device-timed; median of its steps)
    other_train = []
    if not args.no_8b:
        other_train.append(run_train_line(S, torch, dev, W.QWEN3_8B_TRAIN, flush, peaks,
                                          max(3, min(args.steps, 10)), 2, rank))

    # ---- the dense causal comparison on the same layer (speedup denominator)
    dense_line = None
    if not args.no_dense:
        dense_line = run_dense_line(S, torch, dev, cfg, d, flush, peaks, step_ms)

    # ---- the gate variants on the same layer
    variant_lines = None
    if not args.no_variants:
        variant_lines = run_variant_lines(S, torch, dev, cfg, d, flush, peaks)

    # ---- roofline of the dominant call of the training step
    dom = max(k_ms, key=k_ms.get)
    dom_flops = {"sas_attn_fwd_res": f_fwd, "sas_attn_bwd_res": f_bwd}.get(dom, 0.0)
    achieved = dom_flops / (k_ms[dom] * 1e-3) / 1e12 if dom_flops else None
    roof = {"kernel": dom, "bound": "tensor", "achieved": achieved,
            "peak": peaks["bf16_tflops"], "unit": "TFLOP/s",
            "frac": (achieved / peaks["bf16_tflops"]) if achieved else None,
            "traffic": MEASURED_TRAFFIC.get((cfg.name, dom)),
            "traffic_unit": "bytes per call",
            "peak_source": peaks["source"] + " (burst bf16 dense)"}

    line = {
        "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": step_ms_max,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic (seeded numpy PCG64; shapes and distributions of the Qwen3-4B layer)",
        "config": {"workload": cfg.name, "model": "qwen3-4b attention layer (synthetic)",
                   "global_batch": cfg.B * world, "seq_len": cfg.T, "parallelism": f"dp{world}",
                   "heads": f"{cfg.Hq}/{cfg.Hkv}", "head_dim": cfg.d, "block": cfg.b,
                   "K": cfg.K, "l2": "flushed (256 MB write) before every timed step",
                   "algorithmic_tflop_per_step": (f_fwd + f_bwd) / 1e12},
        "kernels_ms": k_ms,
        "roofline": roof,
        "e2e": e2e,
        "gpu_launches": launches,
        "clocks": clocks,
        "decode": decode_lines,
        "train_other": other_train,
        "dense_train": dense_line,
        "train_variants": variant_lines,
        "wall_s_timed": t_wall,
    }
    if rank == 0 and world == 1 and not args.no_cpu:
        line["cpu_baseline"] = cpu_baseline(cfg, x, args.cpu_heads)
    if rank == 0:
        print(json.dumps(line), flush=True)
    D.shutdown()


def cpu_baseline(cfg, x, heads):
    """The float64 oracle on the host: `heads` KV heads with every BLAS thread,
    and one KV head on one thread."""
    kvh = tuple(range(heads))
    secs, fl = oracle_sample(cfg, kvh, x)
    out = {"value": fl / secs / 1e12, "unit": "TFLOP/s", "cores": blas_threads(),
           "kind": "oracle", "cpu_model": cpu_model(), "host_cpus": os.cpu_count(),
           "sample": f"float64 oracle, gates+top-k+fwd+bwd of {len(kvh)} of "
                     f"{cfg.Hkv} KV heads of {cfg.name} ({secs:.1f} s)"}
    try:
        from threadpoolctl import threadpool_limits
        with threadpool_limits(limits=1):
            s1, f1 = oracle_sample(cfg, (0,), x)
        out["single_thread"] = {"value": f1 / s1 / 1e12, "unit": "TFLOP/s", "cores": 1,
                                "sample": f"one KV head on one BLAS thread ({s1:.1f} s)"}
    except Exception as e:  # threadpoolctl missing: report the all-thread figure only
        out["single_thread"] = {"unavailable": str(e)}
    return out


def run_e2e(S, torch, dev, h, d, step, args, world, flops):
    """End-to-end training steps from pinned host buffers: inputs copied in,
    gate + Top-K, forward and backward through the library, and every result
    (o, dq, dk, dv, dscores) copied back to pinned host memory."""
    s_in = torch.cuda.Stream(dev)
    s_comp = torch.cuda.current_stream(dev)
    s_out = torch.cuda.Stream(dev)
    bufs = [d, {n: torch.empty_like(t) for n, t in d.items()}]
    outs = None
    in_ev = [torch.cuda.Event() for _ in range(2)]
    done_ev = [torch.cuda.Event() for _ in range(2)]
    back_ev = [torch.cuda.Event() for _ in range(2)]
    names = ("o", "dq", "dk", "dv", "dscores")
    K = args.steps
    h2d = sum(t.numel() * t.element_size() for t in h.values())

    def one(i, t0=None):
        nonlocal outs
        b = i % 2
        with torch.cuda.stream(s_in):
            if i >= 2:
                s_in.wait_event(done_ev[b])  # step i - 2 has finished with this buffer set
            if t0 is not None:
                t0.record(s_in)
            for n in bufs[b]:
                bufs[b][n].copy_(h[n], non_blocking=True)
            in_ev[b].record(s_in)
        s_comp.wait_event(in_ev[b])
        res = step(bufs[b])
        done_ev[b].record(s_comp)
        with torch.cuda.stream(s_out):
            s_out.wait_event(done_ev[b])
            if outs is None:
                outs = [[torch.empty(t.shape, dtype=t.dtype).pin_memory() for t in res]
                        for _ in range(2)]
            if i >= 2:
                # The host has the results of step i - 2. This also paces the
                # host: run ahead, it keeps allocating outputs faster than the
                # copy-outs release them (measured: 7.9 ms a step with the
                # wait, 7.9 to 9.5 ms and growing without it).
                back_ev[b].synchronize()
            for dst, src in zip(outs[b], res):
                dst.copy_(src, non_blocking=True)
                src.record_stream(s_out)
            back_ev[b].record(s_out)

    for i in range(2):
        one(i)
    torch.cuda.synchronize(dev)
    D.barrier(dev)
    torch.cuda.synchronize(dev)
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    for i in range(K):
        one(i, t0 if i == 0 else None)
    t1.record(s_out)
    torch.cuda.synchronize(dev)
    ms = D.max_over_ranks(t0.elapsed_time(t1) / K, dev)
    d2h = sum(t.numel() * t.element_size() for t in outs[0])
    return {"value": world * flops / (ms * 1e-3) / 1e12, "unit": "TFLOP/s", "ms_per_step": ms,
            "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "results_copied": list(names),
            "overlap": "copy-in, compute and copy-out on three streams, two buffer sets"}


def run_train_line(S, torch, dev, cfg, flush, peaks, steps, warmup, rank):
    """Device-timed training steps of another layer shape (L2 flushed before each)."""
    x = W.make_train_inputs(cfg, seed=D.rank_seed(cfg.seed, rank))
    bf = torch.bfloat16
    t = {n: torch.from_numpy(getattr(x, n)).to(bf).to(dev) for n in ("q", "k", "v", "dO")}
    t["scores"] = torch.from_numpy(x.scores).to(dev)
    del x
    stream = torch.cuda.current_stream(dev)

    def step(ev=None):
        if ev:
            ev[0].record(stream)
        gates, idx = S.gate_topk(t["scores"], cfg.K, causal=True)
        o, o_res, lse = S.attn_fwd_res(t["q"], t["k"], t["v"], idx, gates, cfg.b)
        if ev:
            ev[1].record(stream)
        S.attn_bwd_res(t["q"], t["k"], t["v"], o, o_res, lse, t["dO"], idx, gates, cfg.b)
        if ev:
            ev[2].record(stream)

    for _ in range(warmup):
        step()
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(steps)]
    for i in range(steps):
        flush.zero_()
        torch.cuda._sleep(HEAD_START_CYCLES)
        step(evs[i])
    torch.cuda.synchronize(dev)
    f_fwd, f_bwd = train_flops(cfg)
    fwd_ms = statistics.median(e[0].elapsed_time(e[1]) for e in evs)
    bwd_ms = statistics.median(e[1].elapsed_time(e[2]) for e in evs)
    ms = fwd_ms + bwd_ms
    tf = (f_fwd + f_bwd) / (ms * 1e-3) / 1e12
    del t
    torch.cuda.empty_cache()
    return {"workload": cfg.name, "ms_per_step": ms, "gate_fwd_ms": fwd_ms, "bwd_ms": bwd_ms,
            "TFLOP/s": tf, "frac": tf / peaks["bf16_tflops"],
            "algorithmic_tflop_per_step": (f_fwd + f_bwd) / 1e12}


def run_variant_lines(S, torch, dev, cfg, d, flush, peaks):
    """The training step of the same layer with the ablation variants' gates
    (phi: sigmoid or raw logits; outer gating), through sas_gate_topk_phi,
    sas_attn_fwd_gated and sas_attn_bwd_gated, device-timed (L2 flushed
    before each step); the plain softmax / inner pair (sas_attn_fwd +
    sas_attn_bwd) beside them on the same box."""
    stream = torch.cuda.current_stream(dev)
    f_fwd, f_bwd = train_flops(cfg)
    out = []
    for phi, gating in (("softmax", "inner"), ("sigmoid", "inner"), ("raw", "inner"),
                        ("softmax", "outer")):
        def one(ev=None):
            if ev:
                ev[0].record(stream)
            gates, idx = S.gate_topk(d["scores"], cfg.K, causal=True, phi=phi)
            o, lse = S.attn_fwd(d["q"], d["k"], d["v"], idx, gates, cfg.b, gating=gating)
            S.attn_bwd(d["q"], d["k"], d["v"], o, lse, d["dO"], idx, gates, cfg.b, phi=phi,
                       gating=gating)
            if ev:
                ev[1].record(stream)

        one()
        evs = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(3)]
        for e in evs:
            flush.zero_()
            torch.cuda._sleep(HEAD_START_CYCLES)
            one(e)
        torch.cuda.synchronize(dev)
        ms = statistics.median(a.elapsed_time(b) for a, b in evs)
        out.append({"phi": phi, "gating": gating, "ms_per_step": ms,
                    "TFLOP/s": (f_fwd + f_bwd) / (ms * 1e-3) / 1e12})
    return {"workload": cfg.name, "pair": "sas_attn_fwd(_gated) + sas_attn_bwd(_gated), D "
            "recomputed (the residual pair takes softmax / inner gating only)", "lines": out}


def run_dense_line(S, torch, dev, cfg, d, flush, peaks, sparse_ms):
    """Dense causal attention (every block, no gates) forward + backward on
    the same inputs through sas_dense_fwd / sas_dense_bwd, device-timed (L2
    flushed before each step); the sparse step's speedup over it."""
    stream = torch.cuda.current_stream(dev)
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(3)]

    def one(ev=None):
        if ev:
            ev[0].record(stream)
        o, lse = S.dense_fwd(d["q"], d["k"], d["v"], b=cfg.b)
        if ev:
            ev[1].record(stream)
        S.dense_bwd(d["q"], d["k"], d["v"], o, lse, d["dO"], b=cfg.b)
        if ev:
            ev[2].record(stream)

    one()
    for e in evs:
        flush.zero_()
        torch.cuda._sleep(HEAD_START_CYCLES)
        one(e)
    torch.cuda.synchronize(dev)
    fwd_ms = statistics.median(e[0].elapsed_time(e[1]) for e in evs)
    bwd_ms = statistics.median(e[1].elapsed_time(e[2]) for e in evs)
    pairs = attended_pairs(cfg.B, cfg.Hq, cfg.T, cfg.b, cfg.N)
    flops = 14 * cfg.d * pairs
    tf = flops / ((fwd_ms + bwd_ms) * 1e-3) / 1e12
    return {"workload": cfg.name + " dense causal", "fwd_ms": fwd_ms, "bwd_ms": bwd_ms,
            "ms_per_step": fwd_ms + bwd_ms, "algorithmic_tflop_per_step": flops / 1e12,
            "TFLOP/s": tf, "frac": tf / peaks["bf16_tflops"],
            "speedup_sparse_step": (fwd_ms + bwd_ms) / sparse_ms}


def bench_decode(S, torch, dev, stream, flush, peaks, args, rank):
    out = []
    cache = {}
    for cfg, use_gates in DECODES:
        if cfg.name not in cache:
            cache.clear()
            torch.cuda.empty_cache()
            x = W.make_decode_inputs(cfg, seed=D.rank_seed(cfg.seed, rank))
            bf = torch.bfloat16
            cache[cfg.name] = dict(
                q=torch.from_numpy(x.q).to(bf).to(dev),
                kc=torch.from_numpy(x.kcache).to(bf).to(dev),
                vc=torch.from_numpy(x.vcache).to(bf).to(dev),
                s=torch.from_numpy(x.scores[:, :, None, :].copy()).to(dev))
            del x
        t = cache[cfg.name]

        def one(ev=None):
            if ev:
                ev[0].record(stream)
            gates, idx = S.gate_topk(t["s"], cfg.K, causal=False)
            if ev:
                ev[1].record(stream)
            o = S.decode(t["q"], t["kc"], t["vc"], idx[:, :, 0], gates[:, :, 0], use_gates, cfg.b,
                         L=cfg.L)
            if ev:
                ev[2].record(stream)
            return o

        def two(ev):  # gate_topk then decode, no event between them
            ev[0].record(stream)
            gates, idx = S.gate_topk(t["s"], cfg.K, causal=False)
            S.decode(t["q"], t["kc"], t["vc"], idx[:, :, 0], gates[:, :, 0], use_gates, cfg.b,
                     L=cfg.L)
            ev[1].record(stream)

        s3 = t["s"][:, :, 0]

        def fused(ev):  # the one call: selection inside the decode's launch
            ev[0].record(stream)
            S.decode_select(t["q"], t["kc"], t["vc"], s3, cfg.K, use_gates, cfg.b, L=cfg.L)
            ev[1].record(stream)

        for _ in range(max(3, args.warmup)):
            one()
        reps = max(10, args.steps)

        def timed(fn, nev):
            evs = [[torch.cuda.Event(enable_timing=True) for _ in range(nev)] for _ in range(reps)]
            for i in range(reps):
                flush.zero_()
                torch.cuda._sleep(HEAD_START_CYCLES)
                fn(evs[i])
            torch.cuda.synchronize(dev)
            return evs

        evs = timed(one, 3)
        topk_us = 1e3 * statistics.median(e[0].elapsed_time(e[1]) for e in evs)
        dec_us = 1e3 * statistics.median(e[1].elapsed_time(e[2]) for e in evs)
        evs = timed(two, 2)
        two_us = 1e3 * statistics.median(e[0].elapsed_time(e[1]) for e in evs)
        for _ in range(3):
            fused([torch.cuda.Event(enable_timing=True) for _ in range(2)])
        evs = timed(fused, 2)
        step_us = 1e3 * statistics.median(e[0].elapsed_time(e[1]) for e in evs)
        nbytes = decode_bytes(cfg)
        gbs = nbytes / (dec_us * 1e-6) / 1e9
        line = {"workload": cfg.name, "use_gates": use_gates,
                "step_us": step_us, "step": "sas_decode_select (gates, Top-K and decode, one call)",
                "decode_us": dec_us, "gate_topk_us": topk_us, "two_launch_step_us": two_us,
                "selected_bytes": nbytes, "GB/s": gbs, "step_GB/s": nbytes / (step_us * 1e-6) / 1e9,
                "roofline": {"kernel": "decode_tc_kernel (sas_decode)", "bound": "hbm",
                             "achieved": gbs, "peak": peaks["hbm_gbs"],
                             "unit": "GB/s", "frac": gbs / peaks["hbm_gbs"],
                             "peak_source": peaks["source"] + " (copy bandwidth)"}}
        if use_gates == 0:
            dev_ev = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(5)]
            for i in range(5):
                flush.zero_()
                torch.cuda._sleep(HEAD_START_CYCLES)
                dev_ev[i][0].record(stream)
                S.dense_decode(t["q"], t["kc"], t["vc"], L=cfg.L)
                dev_ev[i][1].record(stream)
            torch.cuda.synchronize(dev)
            dense_us = 1e3 * statistics.median(a.elapsed_time(b) for a, b in dev_ev)
            dbytes = decode_bytes(cfg, dense=True)
            line["dense"] = {"decode_us": dense_us, "bytes": dbytes,
                             "GB/s": dbytes / (dense_us * 1e-6) / 1e9,
                             "speedup_sparse_step": dense_us / step_us}
            line["paged"] = bench_paged(S, torch, dev, stream, flush, t, cfg, use_gates, reps)
            line["with_selector"] = bench_selector_step(S, torch, dev, stream, flush, t, cfg,
                                                        use_gates, reps)
        out.append(line)
    return out


def paged_copy(torch, dev, kc, vc, cfg, P=16):
    """A paged copy of contiguous caches [B, Hkv, L, d]: P-token pages placed
    in a seeded random order, with their page table and lengths."""
    B, Hkv, L, d = kc.shape
    npp = L // P
    perm = torch.randperm(B * npp, generator=torch.Generator().manual_seed(cfg.seed + 17))
    kp = torch.empty((B * npp, Hkv, P, d), dtype=kc.dtype, device=dev)
    vp = torch.empty_like(kp)
    pd = perm.to(dev)
    kp[pd] = kc.view(B, Hkv, npp, P, d).permute(0, 2, 1, 3, 4).reshape(B * npp, Hkv, P, d)
    vp[pd] = vc.view(B, Hkv, npp, P, d).permute(0, 2, 1, 3, 4).reshape(B * npp, Hkv, P, d)
    indptr = torch.arange(0, B * npp + 1, npp, dtype=torch.int32, device=dev)
    indices = pd.to(torch.int32)
    lens = torch.full((B,), cfg.L, dtype=torch.int32, device=dev)
    return kp, vp, indptr, indices, lens


def bench_paged(S, torch, dev, stream, flush, t, cfg, use_gates, reps, P=16):
    """The same decode over a paged copy of the caches (P-token pages placed
    in a seeded random order): sas_decode_paged with the same selection,
    timed like the contiguous decode; its output must equal the contiguous
    one."""
    B, Hkv, L, d = t["kc"].shape
    npp = L // P
    kp, vp, indptr, indices, lens = paged_copy(torch, dev, t["kc"], t["vc"], cfg, P)
    gates, idx = S.gate_topk(t["s"], cfg.K, causal=False)
    ix, g = idx[:, :, 0].contiguous(), gates[:, :, 0].contiguous()

    def call():
        return S.decode_paged(t["q"], kp, vp, indptr, indices, lens, ix, g, use_gates, cfg.b,
                              max_len=cfg.L)

    o_ref = S.decode(t["q"], t["kc"], t["vc"], ix, g, use_gates, cfg.b, L=cfg.L)
    o_pg = call()
    torch.cuda.synchronize(dev)
    same = bool(torch.equal(o_ref, o_pg))
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(reps)]
    for i in range(reps):
        flush.zero_()
        torch.cuda._sleep(HEAD_START_CYCLES)
        evs[i][0].record(stream)
        call()
        evs[i][1].record(stream)
    torch.cuda.synchronize(dev)
    us = 1e3 * statistics.median(a.elapsed_time(b) for a, b in evs)
    nbytes = decode_bytes(cfg)
    del kp, vp
    torch.cuda.empty_cache()
    return {"page_tokens": P, "pages": B * npp, "order": "seeded random permutation",
            "decode_us": us, "GB/s": nbytes / (us * 1e-6) / 1e9,
            "equals_contiguous_decode": same}


def _time_us(torch, stream, flush, reps, fn):
    """Median device time (µs) of fn() on `stream`: 3 untimed calls, then
    `reps` calls, each after an L2 flush and a head start of the stream."""
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(reps)]
    for i in range(reps + 3):
        flush.zero_()
        torch.cuda._sleep(HEAD_START_CYCLES)
        ev = evs[i - 3] if i >= 3 else None
        if ev:
            ev[0].record(stream)
        fn()
        if ev:
            ev[1].record(stream)
    torch.cuda.synchronize()
    return 1e3 * statistics.median(a.elapsed_time(b) for a, b in evs)


def bench_selector_step(S, torch, dev, stream, flush, t, cfg, use_gates, reps):
    """The decode step with the weight-free block selector in front: the
    scores of q against the history blocks' mean keys (kept per block, so
    computed once here, as a serving loop would keep them), then the fused
    selection and decode; and the same step as one call that forms the
    scores itself (sas_decode_select_pooled)."""
    kbar = S.block_summaries(t["kc"], cfg.b, L=cfg.L)
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(reps)]
    for i in range(reps + 3):
        flush.zero_()
        torch.cuda._sleep(HEAD_START_CYCLES)
        ev = evs[i - 3] if i >= 3 else None
        if ev:
            ev[0].record(stream)
        sc = S.selector_scores_decode(t["q"], kbar)
        if ev:
            ev[1].record(stream)
        S.decode_select(t["q"], t["kc"], t["vc"], sc, cfg.K, use_gates, cfg.b, L=cfg.L)
        if ev:
            ev[2].record(stream)
    torch.cuda.synchronize(dev)
    sel = 1e3 * statistics.median(e[0].elapsed_time(e[1]) for e in evs)
    step = 1e3 * statistics.median(e[0].elapsed_time(e[2]) for e in evs)
    pooled = _time_us(torch, stream, flush, reps, lambda: S.decode_select_pooled(
        t["q"], t["kc"], t["vc"], kbar, cfg.K, use_gates, cfg.b, L=cfg.L))
    del kbar
    return {"selector_scores_us": sel, "two_call_step_us": step, "step_us": pooled,
            "step": "sas_decode_select_pooled (scores, selection and decode in one call)",
            "two_call_step": "sas_selector_scores_decode + sas_decode_select",
            "block_summaries": "computed once (a serving loop adds one per filled block)"}


def run_decode_only(args):
    """Only the decode lines of one preset (both gate modes it lists)."""
    import torch
    from block_sparse_attention_sas_b200 import _lib as S
    global DECODES
    cfg = W.PRESETS[args.decode_only]
    DECODES = [(cfg, g) for g in cfg.gate_modes]
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
    lines = bench_decode(S, torch, dev, torch.cuda.current_stream(dev), flush, load_peaks(), args,
                         0)
    print(json.dumps({"decode": lines}), flush=True)


def run_profile_train(args):
    """The training step (gate_topk, forward, backward) of the Qwen3-4B layer
    shape at a shorter sequence length, for kernel captures: warm-up steps,
    then `steps` more, with no timing and no decode."""
    import torch
    from block_sparse_attention_sas_b200 import _lib as S
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    cfg = W.small_train_config(B=1, Hq=32, Hkv=8, T=args.profile_train, d=128, b=64, K=16,
                               dtype="bf16", hot_key_frac=0.05, hot_key_scale=3.0)
    x = W.make_train_inputs(cfg)
    t = {n: torch.from_numpy(getattr(x, n)).to(dev).to(torch.bfloat16)
         for n in ("q", "k", "v", "dO")}
    scores = torch.from_numpy(x.scores).to(dev)
    for _ in range(args.warmup + args.steps):
        gates, idx = S.gate_topk(scores, cfg.K)
        o, o_res, lse = S.attn_fwd_res(t["q"], t["k"], t["v"], idx, gates, cfg.b)
        S.attn_bwd_res(t["q"], t["k"], t["v"], o, o_res, lse, t["dO"], idx, gates, cfg.b)
    torch.cuda.synchronize(dev)
    st, raw = S.device_error()
    print(json.dumps({"profile_train": cfg.name, "steps": args.warmup + args.steps,
                      "device_error": st}), flush=True)
    if st != 0:
        raise SystemExit(1)


def run_profile_decode(args):
    """The decode step of one preset, gates on, warm-up plus `steps` calls
    with the L2 flushed before each, untimed, for kernel captures: the fused
    step (sas_decode_select) by default, or the pooled call, the two-call
    step with the standalone selector, or the paged decode."""
    import torch
    from block_sparse_attention_sas_b200 import _lib as S
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    cfg = W.PRESETS[args.profile_decode]
    x = W.make_decode_inputs(cfg)
    bf = torch.bfloat16
    q = torch.from_numpy(x.q).to(bf).to(dev)
    kc = torch.from_numpy(x.kcache).to(bf).to(dev)
    vc = torch.from_numpy(x.vcache).to(bf).to(dev)
    sc = torch.from_numpy(x.scores).to(dev)
    del x
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
    kbar = S.block_summaries(kc, cfg.b, L=cfg.L) if (args.pooled or args.two_call) else None
    if args.paged:
        kp, vp, indptr, indices, lens = paged_copy(torch, dev, kc, vc, cfg)
        gates, idx = S.gate_topk(sc[:, :, None, :].contiguous(), cfg.K, causal=False)
        ix, g = idx[:, :, 0].contiguous(), gates[:, :, 0].contiguous()
    for _ in range(args.warmup + args.steps):
        flush.zero_()
        if args.paged:
            S.decode_paged(q, kp, vp, indptr, indices, lens, ix, g, True, cfg.b, max_len=cfg.L)
        elif args.pooled:
            S.decode_select_pooled(q, kc, vc, kbar, cfg.K, True, cfg.b, L=cfg.L)
        elif args.two_call:
            s2 = S.selector_scores_decode(q, kbar)
            S.decode_select(q, kc, vc, s2, cfg.K, True, cfg.b, L=cfg.L)
        else:
            S.decode_select(q, kc, vc, sc, cfg.K, True, cfg.b, L=cfg.L)
    torch.cuda.synchronize(dev)
    st, raw = S.device_error()
    mode = ("paged" if args.paged else "pooled" if args.pooled else
            "two_call" if args.two_call else "fused")
    print(json.dumps({"profile_decode": cfg.name, "mode": mode,
                      "steps": args.warmup + args.steps, "device_error": st}), flush=True)
    if st != 0:
        raise SystemExit(1)


# ----------------------------------------------------------- reference arm

def run_reference(args):
    """The float64 oracle as it stands, on the host cores: each step is a
    bounded sample (one KV head of the Qwen3-4B layer: gates, Top-K, forward,
    backward), reported in the same metric and unit."""
    rank, _, world = D.env_rank()
    if rank != 0:
        return
    cfg = TRAIN
    x = W.make_train_inputs(cfg)
    for _ in range(args.warmup if args.warmup < 2 else 1):
        oracle_sample(cfg, (0,), x)
    secs, fl = 0.0, 0.0
    for i in range(args.steps):
        s, f = oracle_sample(cfg, (i % cfg.Hkv,), x)
        secs += s
        fl += f
    val = fl / secs / 1e12
    line = {"impl": "reference", "metric": METRIC, "value": val, "unit": "TFLOP/s",
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": 1e3 * secs / args.steps, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": cfg.name, "sample_per_step": "1 of 8 KV heads"},
            "cpu_baseline": {"value": val, "unit": "TFLOP/s", "cores": blas_threads(),
                             "kind": "oracle",
                             "sample": "one KV head of the Qwen3-4B layer per step"},
            "e2e": {"value": val, "unit": "TFLOP/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def _free_port() -> int:
    with socket.socket() as sk:
        sk.bind(("127.0.0.1", 0))
        return sk.getsockname()[1]


def relaunch(n: int) -> int:
    """Runs this script again under torch.distributed.run with n ranks (one
    per GPU) on 127.0.0.1 and returns its exit code."""
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", f"--nproc-per-node={n}",
           "--master-addr", "127.0.0.1", "--master-port", str(_free_port()),
           os.path.abspath(__file__), *sys.argv[1:]]
    return subprocess.call(cmd)


def run_dry(args):
    """The launch and timing plumbing without a GPU: gloo ranks time a small
    host-side step, reduce the max over ranks, and rank 0 prints a JSON line."""
    rank, _, world = D.env_rank()
    D.init("gloo", timeout_s=60)
    a = np.random.default_rng(D.rank_seed(0, rank)).standard_normal((256, 256))
    for _ in range(args.warmup):
        a @ a
    D.barrier()
    t = time.perf_counter()
    for _ in range(args.steps):
        a @ a
    ms = D.max_over_ranks(1e3 * (time.perf_counter() - t) / max(1, args.steps))
    if rank == 0:
        print(json.dumps({"dry_run": True, "n_gpus": world, "steps": args.steps,
                          "warmup": args.warmup, "ms_per_step": ms, "scaling": "weak"}),
              flush=True)
    D.shutdown()


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--no-decode", action="store_true")
    ap.add_argument("--no-cpu", action="store_true")
    ap.add_argument("--cpu-heads", type=int, default=2)
    ap.add_argument("--decode-only", default=None, metavar="PRESET",
                    help="time only the decode path of one preset (for profiling)")
    ap.add_argument("--profile-train", type=int, default=0, metavar="T",
                    help="run only the training step at sequence length T (for profiling)")
    ap.add_argument("--profile-decode", default=None, metavar="PRESET",
                    help="only run the decode step (sas_decode_select) warmup + steps times, "
                         "untimed, for kernel captures")
    ap.add_argument("--pooled", action="store_true",
                    help="with --profile-decode: sas_decode_select_pooled (the selector's "
                         "scores formed in the launch from the block means)")
    ap.add_argument("--two-call", action="store_true",
                    help="with --profile-decode: sas_selector_scores_decode, then "
                         "sas_decode_select")
    ap.add_argument("--paged", action="store_true",
                    help="with --profile-decode: sas_decode_paged over a paged copy of the "
                         "caches (16-token pages in a seeded random order)")
    ap.add_argument("--no-8b", action="store_true", help="skip the Qwen3-8B training line")
    ap.add_argument("--no-variants", action="store_true",
                    help="skip the gate-variant training lines")
    ap.add_argument("--no-dense", action="store_true", help="skip the dense training line")
    ap.add_argument("--dry-run", action="store_true",
                    help="CPU only: exercise the rank launch and timing reduction on gloo")
    args = ap.parse_args()
    if args.gpus > 1 and "WORLD_SIZE" not in os.environ:
        raise SystemExit(relaunch(args.gpus))
    if args.warmup < 3 and args.impl == "ours":
        args.warmup = 3
    if args.dry_run:
        run_dry(args)
    elif args.impl == "reference":
        run_reference(args)
    elif args.decode_only:
        run_decode_only(args)
    elif args.profile_train:
        run_profile_train(args)
    elif args.profile_decode:
        run_profile_decode(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
