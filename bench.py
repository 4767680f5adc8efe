#!/usr/bin/env python
"""Benchmark of the differential-attention hot path on B200.

One step = one pass of the hot path over one batch: lambda from its four
per-head vectors, then V1 causal prefill with the per-head RMS norm and the
(1 - lambda_init) scale (batch 4, 16 heads, 4096 tokens, 64-wide branches,
128-wide values, layer 12).  Metric: DiffAttn forward TFLOP/s, counting
2 QK^T + 2 PV contractions per visible (query, key) pair (768 flop per pair
for this shape, masked pairs excluded).

Usage:  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
For N > 1 launch one process per GPU with torch.distributed.run; each rank
runs the same per-GPU workload (weak scaling, no collective on the data
path), timing is taken as the max over ranks, and rank 0 prints one JSON line.
"""
from __future__ import annotations

import argparse
import hashlib
import re
import json
import os
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "DiffAttn fwd TFLOP/s (prefill), decode HBM GB/s; % of B200 roofline"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
# The decode target (70 % of HBM bandwidth) is stated against about 8 TB/s of
# nominal HBM3e bandwidth; the measured peak is a read+write copy, which a
# pure read stream can exceed, so decode lines report both fractions.
NOMINAL_HBM_GBS = 8000.0


# ---------------------------------------------------------------------------
# algorithmic work
# ---------------------------------------------------------------------------
def prefill_pairs(B, N, H, causal=True):
    """Visible (query, key) pairs of one prefill call."""
    return B * H * (N * (N + 1) // 2 if causal else N * N)


def v1_flops_per_pair(d, dv):
    return 2 * (2 * d) + 2 * (2 * dv)          # two QK^T branches + two P.V


def v1_bwd_flops_per_pair(d, dv):
    """Backward work per visible pair, both branches: recomputed scores (2d),
    dP = dO V^T (2dv), dQ (2d), dK (2d) and dV (2dv) per branch (V2: d = dv)."""
    return 2 * (6 * d + 4 * dv)


def v2_flops_per_pair(d):
    return 2 * (2 * d) + 2 * (2 * d)


def v2_decode_bytes(B, L, Hkv, d, Hq):
    return B * L * Hkv * d * 2 * 2 + B * Hq * d * 2 + B * (Hq // 2) * d * 2


def window_pairs(B, N, H, W):
    """Visible (query, key) pairs of causal prefill with a sliding window W:
    row i sees min(i + 1, W) keys."""
    full = min(N, W)
    return B * H * (full * (full + 1) // 2 + (N - full) * W)


def v1_decode_bytes(B, L, H, d, dv):
    return B * L * H * (2 * d + dv) * 2 + B * H * 2 * d * 2 + B * H * dv * 2


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(p) as f:
            d = json.load(f)
        return {k: float(d[k]) for k in FALLBACK_PEAKS}, "measured (MEASURED_PEAKS.json)"
    except Exception:
        return dict(FALLBACK_PEAKS), "fallback (no MEASURED_PEAKS.json)"


def code_without_comments(text: str) -> str:
    """Source text with // comments, /* */ comments and blank lines removed
    (string literals in these files hold no comment markers)."""
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    lines = [re.sub(r"//.*$", "", ln).rstrip() for ln in text.splitlines()]
    return "\n".join(ln for ln in lines if ln.strip())


def kernel_source_hash():
    """Hash of the prefill kernel's code (comments excluded: they do not change
    the kernel), which a recorded traffic figure must match to be reported."""
    h = hashlib.sha256()
    for rel in ("prefill_tc.cu", "ptx.cuh"):
        with open(os.path.join(ROOT, "differential_attention_sm_b200", "csrc", rel)) as f:
            h.update(code_without_comments(f.read()).encode())
    return h.hexdigest()[:16]


def recorded_traffic(kernel: str, workload: str):
    """DRAM bytes per launch from a committed ncu summary, valid only while
    the kernel source is unchanged since the capture (else None)."""
    p = os.path.join(ROOT, "profiles", "dram_traffic.txt")
    if not os.path.exists(p):
        return None
    cur = kernel_source_hash()
    for line in open(p):
        parts = line.split()
        if len(parts) >= 4 and parts[0] == kernel and parts[1] == workload and parts[3] == cur:
            return float(parts[2])
    return None


# ---------------------------------------------------------------------------
# clocks during the timed region (NVML, read only)
# ---------------------------------------------------------------------------
_REASONS = {0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap",
            0x8: "hw_slowdown", 0x10: "sync_boost", 0x20: "sw_thermal_slowdown",
            0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown",
            0x100: "display_clock_setting"}


class ClockSampler:
    def __init__(self, device_index: int, period_s: float = 0.02):
        self.samples = []
        self.reasons = 0
        self.ok = False
        self.max_mhz = None
        self._stop = threading.Event()
        try:
            import pynvml
            pynvml.nvmlInit()
            uuid = None
            try:
                import torch
                uuid = str(torch.cuda.get_device_properties(device_index).uuid)
            except Exception:
                pass
            self.h = None
            if uuid:
                for i in range(pynvml.nvmlDeviceGetCount()):
                    hh = pynvml.nvmlDeviceGetHandleByIndex(i)
                    u = pynvml.nvmlDeviceGetUUID(hh)
                    u = u.decode() if isinstance(u, bytes) else u
                    if u.replace("GPU-", "") == uuid.replace("GPU-", ""):
                        self.h = hh
            if self.h is None:
                self.h = pynvml.nvmlDeviceGetHandleByIndex(device_index)
            self.nv = pynvml
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
            self.ok = True
        except Exception:
            self.ok = False
        self.period = period_s

    def _run(self):
        nv = self.nv
        while not self._stop.is_set():
            try:
                self.samples.append(nv.nvmlDeviceGetClockInfo(self.h, nv.NVML_CLOCK_SM))
                self.reasons |= int(nv.nvmlDeviceGetCurrentClocksEventReasons(self.h))
            except Exception:
                pass
            time.sleep(self.period)

    def __enter__(self):
        if self.ok:
            self.t = threading.Thread(target=self._run, daemon=True)
            self.t.start()
        return self

    def __exit__(self, *a):
        if self.ok:
            self._stop.set()
            self.t.join()

    def summary(self):
        if not self.ok:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvml unavailable"]}
        names = [n for bit, n in _REASONS.items() if self.reasons & bit and n != "gpu_idle"]
        return {"sm_mhz": float(np.median(self.samples)) if self.samples else None,
                "sm_max_mhz": self.max_mhz, "reasons": names, "samples": len(self.samples)}


# ---------------------------------------------------------------------------
# distributed plumbing (one process per GPU)
# ---------------------------------------------------------------------------
def dist_env():
    return (int(os.environ.get("RANK", "0")), int(os.environ.get("WORLD_SIZE", "1")),
            int(os.environ.get("LOCAL_RANK", "0")))


def max_over_ranks(x: float, world: int, device=None) -> float:
    if world == 1:
        return x
    import torch
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def barrier(world: int):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


# ---------------------------------------------------------------------------
# our arm
# ---------------------------------------------------------------------------
def timed_loop(fn, steps, warmup, world, stream, side_streams=()):
    """W untimed steps, then exactly K steps bracketed by barrier+sync;
    returns (device ms for the K steps, max over ranks).  Work the steps put
    on `side_streams` is inside the timed region: those streams start after
    the opening event and the closing event waits for them."""
    import torch
    for _ in range(warmup):
        fn()
    torch.cuda.synchronize()
    barrier(world)
    torch.cuda.synchronize()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for s_ in side_streams:
        s_.wait_stream(stream)
    for _ in range(steps):
        fn()
    for s_ in side_streams:
        stream.wait_stream(s_)
    e1.record(stream)
    torch.cuda.synchronize()
    barrier(world)
    ms = e0.elapsed_time(e1)
    return max_over_ranks(ms, world, torch.device("cuda"))


def run_headline(args, rank, world, local_rank, peaks, peak_src):
    import torch
    from differential_attention_sm_b200 import binding as Bd
    from differential_attention_sm_b200 import inputs as I

    w = I.WORKLOADS["v1_prefill_bf16"]
    dev = torch.device("cuda", local_rank)
    x = I.v1_inputs(w.B, w.N, w.H, w.d, w.dv, w.seed + 1000 * rank)
    q, k, v = (x[n].to(dev) for n in ("q", "k", "v"))
    lv = [x[n].to(dev) for n in ("lq1", "lk1", "lq2", "lk2")]
    lam = torch.empty(w.H, dtype=torch.float32, device=dev)
    out = torch.empty(w.B, w.N, w.H, w.dv, dtype=torch.bfloat16, device=dev)
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    li = Bd.diffattn_lambda_init(w.layer)
    stream = torch.cuda.current_stream(dev)
    flops = prefill_pairs(w.B, w.N, w.H) * v1_flops_per_pair(w.d, w.dv)

    def step():
        Bd.lambda_from_params(*lv, w.layer, out=lam)
        Bd.diffattn_v1_fwd(q, k, v, lam, causal=True, apply_norm=True, norm_eps=w.eps,
                           lambda_init=li, out=out, dev_status=status)

    # The dominant kernel alone, as a short burst before the long loop (the
    # measured bf16 peak it is compared with is a burst figure too), timed
    # with events on the stream it is launched on.
    for _ in range(3):
        step()
    torch.cuda.synchronize()
    kms = []
    for _ in range(max(5, min(args.steps, 50))):
        Bd.lambda_from_params(*lv, w.layer, out=lam)
        a = torch.cuda.Event(enable_timing=True)
        b = torch.cuda.Event(enable_timing=True)
        a.record(stream)
        Bd.diffattn_v1_fwd(q, k, v, lam, causal=True, apply_norm=True, norm_eps=w.eps,
                           lambda_init=li, out=out, dev_status=status)
        b.record(stream)
        kms.append((a, b))
    torch.cuda.synchronize()
    kernel_ms = float(np.mean([a.elapsed_time(b) for a, b in kms]))
    with ClockSampler(local_rank) as clk:
        ms = timed_loop(step, args.steps, args.warmup, world, stream)
    if int(status.item()) != 0:
        raise RuntimeError("device status %d during the benchmark" % int(status.item()))

    # End to end through the public API with pinned host buffers: every step
    # uploads its inputs, runs lambda_from_params and the prefill, and reads
    # its output back.  Steps are pipelined as a serving loop would run them:
    # two device buffer sets, uploads on one copy stream and read-backs on
    # another, so step i+1's upload (host to device) overlaps step i's kernels
    # and its read-back (device to host, the other direction of the link).
    hq, hk, hv = (x[n].pin_memory() for n in ("q", "k", "v"))
    hl = [x[n].pin_memory() for n in ("lq1", "lk1", "lq2", "lk2")]
    hout = [torch.empty(out.shape, dtype=out.dtype).pin_memory() for _ in range(2)]
    sets = []
    for _ in range(2):
        sets.append({"in": [torch.empty_like(q), torch.empty_like(k), torch.empty_like(v),
                            *[torch.empty_like(t) for t in lv]],
                     "lam": torch.empty_like(lam), "out": torch.empty_like(out)})
    up_stream, down_stream = torch.cuda.Stream(), torch.cuda.Stream()
    ev = {n_: [torch.cuda.Event() for _ in range(2)] for n_ in ("up", "comp", "down")}
    used = [False, False]
    e2e_i = [0]

    def e2e_step():
        b = e2e_i[0] % 2
        S = sets[b]
        if used[b]:  # the set's previous step must have read its inputs
            up_stream.wait_event(ev["comp"][b])
        with torch.cuda.stream(up_stream):
            for d_, h_ in zip(S["in"], (hq, hk, hv, *hl)):
                d_.copy_(h_, non_blocking=True)
        ev["up"][b].record(up_stream)
        stream.wait_event(ev["up"][b])
        if used[b]:  # ... and its output must have been read back
            stream.wait_event(ev["down"][b])
        Bd.lambda_from_params(*S["in"][3:], w.layer, out=S["lam"])
        Bd.diffattn_v1_fwd(*S["in"][:3], S["lam"], causal=True, apply_norm=True,
                           norm_eps=w.eps, lambda_init=li, out=S["out"], dev_status=status)
        ev["comp"][b].record(stream)
        down_stream.wait_event(ev["comp"][b])
        with torch.cuda.stream(down_stream):
            hout[b].copy_(S["out"], non_blocking=True)
        ev["down"][b].record(down_stream)
        used[b] = True
        e2e_i[0] += 1

    e2e_steps = max(3, min(args.steps, 20))
    e2e_ms = timed_loop(e2e_step, e2e_steps, max(3, min(args.warmup, 5)), world, stream,
                        side_streams=(up_stream, down_stream))
    h2d = sum(t.numel() * t.element_size() for t in (hq, hk, hv, *hl))
    d2h = hout[0].numel() * hout[0].element_size()
    # the pipelined path computes what the device path computed (same inputs)
    last = hout[(e2e_i[0] - 1) % 2]
    if not torch.equal(last.view(torch.int16), out.cpu().view(torch.int16)):
        raise RuntimeError("end-to-end output differs from the device-resident run")

    achieved = flops / (kernel_ms * 1e-3) / 1e12
    peak = peaks["bf16_tflops"]
    in_loop = flops * args.steps / (ms * 1e-3) / 1e12  # per GPU, under the power cap
    peak_sus = peaks.get("bf16_tflops_sustained")
    traffic = recorded_traffic("diffattn_prefill_tc_kernel", "v1_prefill_bf16")
    res = {
        "value": world * flops * args.steps / (ms * 1e-3) / 1e12,
        "ms_per_step": ms / args.steps,
        "roofline": {"bound": "tensor", "achieved": round(achieved, 2), "peak": peak,
                     "unit": "TFLOP/s", "frac": round(achieved / peak, 4), "traffic": traffic,
                     "kernel": "diffattn_prefill_tc_kernel", "kernel_ms": round(kernel_ms, 4),
                     "kernel_timing": "%d launches alone, before the timed loop" % len(kms),
                     "peak_source": "%s dense bf16 burst" % peak_src,
                     "in_timed_loop": {"achieved": round(in_loop, 2), "peak": peak_sus,
                                       "frac": round(in_loop / peak_sus, 4) if peak_sus else None,
                                       "peak_source": "%s dense bf16 sustained" % peak_src},
                     "work_per_launch": "%.4e flop (768 flop x %d causal pairs)" % (
                         flops, prefill_pairs(w.B, w.N, w.H))},
        "e2e": {"value": world * flops * e2e_steps / (e2e_ms * 1e-3) / 1e12, "unit": "TFLOP/s",
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                "ms_per_step": e2e_ms / e2e_steps,
                "pipelining": "two device buffer sets; each step's upload and read-back are "
                              "timed, and step i+1's upload overlaps step i's kernels and "
                              "read-back"},
        "gpu_launches": 2 * args.steps,
        "clocks": clk.summary(),
        "config": {"workload": "v1_prefill_bf16: V1 causal prefill, batch 4, 16 heads, "
                               "seq 4096, QK 64 per branch, V 128, lambda from params "
                               "(layer 12), per-head RMSNorm eps 1e-5, x(1-lambda_init)",
                   "batch_per_gpu": w.B, "global_batch": w.B * world, "seq_len": w.N,
                   "heads": w.H, "d_qk": w.d, "d_v": w.dv, "causal": True,
                   "parallelism": "dp%d (independent batches)" % world,
                   "l2": "inputs 192 MiB per step > 126 MB L2 (no flush needed)"},
    }
    del q, k, v, out, sets
    torch.cuda.empty_cache()
    return res, x


def time_call(fn, iters, warmup, stream):
    import torch
    for _ in range(warmup):
        fn()
    torch.cuda.synchronize()
    a = torch.cuda.Event(enable_timing=True)
    b = torch.cuda.Event(enable_timing=True)
    a.record(stream)
    for _ in range(iters):
        fn()
    b.record(stream)
    torch.cuda.synchronize()
    return a.elapsed_time(b) / iters


def oracle_rate(run_once, target_s: float, unit_scale: float, what: str):
    """Bounded CPU-baseline sample: calls ``run_once(n)`` (runs the oracle on
    n units of the workload and returns the algorithmic work it covered)
    with n doubling until about ``target_s`` seconds of host time are spent.
    Returns the ``cpu_baseline`` object for one workload."""
    import oracle as O
    n, work, secs, units = 1, 0.0, 0.0, 0
    while secs < target_s:
        t0 = time.perf_counter()
        work += run_once(n)
        dt = time.perf_counter() - t0
        secs += dt
        units += n
        if dt < target_s / 4:
            n *= 2
    return {"value": work / secs / unit_scale, "cores": O.n_threads(), "kind": "oracle",
            "sample": "%d %s (%.1f s)" % (units, what, secs)}


def _rows_sampler(fn, total_rows, per_row_work, seed):
    """run_once(n) for row-wise oracle calls: n random output rows."""
    rng = np.random.default_rng(seed)

    def run_once(n):
        rows = rng.integers(0, total_rows, n)
        fn(rows)
        return float(sum(per_row_work(int(r)) for r in rows))
    return run_once


def _decode_sampler(ref_entry, caches, B, per_entry_bytes, seed):
    """run_once(n) for decode: n random batch entries, each entry's cache
    slices copied to the host, all of its outputs by the oracle."""
    rng = np.random.default_rng(seed)

    def run_once(n):
        for b in rng.integers(0, B, n):
            k, v = caches[0][int(b)].cpu(), caches[1][int(b)].cpu()
            ref_entry(int(b), k, v)
        return float(n * per_entry_bytes)
    return run_once


def run_extras(local_rank, peaks, peak_src, only=None, decode_batch=None, cpu_s=2.0):
    """The other workloads, one GPU: V2 prefill, V1 long-context prefill,
    V2 decode and V1 decode (same kernels the parity tests check).
    `only` restricts the run to one of them and `decode_batch` shrinks the
    decode batch (used for small profiling runs).  Each entry carries the
    oracle timed on a bounded sample of its workload (``cpu_baseline``,
    about ``cpu_s`` seconds of host work; 0 skips it)."""
    import dataclasses

    import oracle as O
    import torch
    from differential_attention_sm_b200 import binding as Bd
    from differential_attention_sm_b200 import inputs as I
    dev = torch.device("cuda", local_rank)
    stream = torch.cuda.current_stream(dev)
    out = {}

    def want(name):
        return only is None or only == name

    def wl(name):
        w = I.WORKLOADS[name]
        if decode_batch and w.kind.endswith("decode"):
            w = dataclasses.replace(w, B=decode_batch)
        return w

    if want("v2_prefill_bf16"):  # B2 Hq32 Hkv8 d128 N8192
        w = wl("v2_prefill_bf16")
        x = I.v2_inputs(w.B, w.N, w.Hq, w.Hkv, w.d, w.seed)
        q, k, v, lam = (x[n].to(dev) for n in ("q", "k", "v", "lam"))
        o = torch.empty(w.B, w.N, w.Hq // 2, w.d, dtype=torch.bfloat16, device=dev)
        ms = time_call(lambda: Bd.diffattn_v2_prefill(q, k, v, lam, causal=True, out=o), 20, 3,
                       stream)
        fl = prefill_pairs(w.B, w.N, w.Hq // 2) * v2_flops_per_pair(w.d)
        t = fl / (ms * 1e-3) / 1e12
        out["v2_prefill_bf16"] = {"value": round(t, 2), "unit": "TFLOP/s", "ms": round(ms, 4),
                                  "frac": round(t / peaks["bf16_tflops"], 4),
                                  "peak": peaks["bf16_tflops"], "flop": fl}
        if cpu_s > 0:
            P_ = w.Hq // 2
            out["v2_prefill_bf16"]["cpu_baseline"] = dict(oracle_rate(_rows_sampler(
                lambda r: O.v2_rows(x["q"], x["k"], x["v"], x["lam"], r, causal=True),
                w.B * w.N * P_, lambda r: ((r // P_) % w.N + 1) * v2_flops_per_pair(w.d), 11),
                cpu_s, 1e12, "random output rows"), unit="TFLOP/s")
        del q, k, v, o, x

    if want("v1_long_bf16"):  # B1 H16 N32768, layer 24, planted signal
        w = wl("v1_long_bf16")
        x = I.v1_inputs(w.B, w.N, w.H, w.d, w.dv, w.seed, planted=w.planted)
        q, k, v = (x[n].to(dev) for n in ("q", "k", "v"))
        lamt = Bd.lambda_from_params(*(x[n].to(dev) for n in ("lq1", "lk1", "lq2", "lk2")),
                                     w.layer)
        li = Bd.diffattn_lambda_init(w.layer)
        o = torch.empty(w.B, w.N, w.H, w.dv, dtype=torch.bfloat16, device=dev)
        ms = time_call(lambda: Bd.diffattn_v1_fwd(q, k, v, lamt, causal=True, apply_norm=True,
                                                  lambda_init=li, out=o), 5, 2, stream)
        fl = prefill_pairs(w.B, w.N, w.H) * v1_flops_per_pair(w.d, w.dv)
        t = fl / (ms * 1e-3) / 1e12
        out["v1_long_bf16"] = {"value": round(t, 2), "unit": "TFLOP/s", "ms": round(ms, 4),
                               "frac": round(t / peaks["bf16_tflops"], 4), "flop": fl}
        if cpu_s > 0:
            lam_h = O.lambda_from_params(x["lq1"], x["lk1"], x["lq2"], x["lk2"], w.layer)
            out["v1_long_bf16"]["cpu_baseline"] = dict(oracle_rate(_rows_sampler(
                lambda r: O.v1_rows(x["q"], x["k"], x["v"], lam_h, r, causal=True,
                                    apply_norm=True, eps=w.eps, lambda_init_value=li),
                w.B * w.N * w.H, lambda r: ((r // w.H) % w.N + 1) * v1_flops_per_pair(w.d, w.dv),
                12), cpu_s, 1e12, "random output rows"), unit="TFLOP/s")
        del q, k, v, o, x

    if want("v2_decode_bf16"):  # B64 L32768 Hq64 Hkv8 d128
        w = wl("v2_decode_bf16")
        x = I.v2_decode_inputs(w.B, w.L, w.Hq, w.Hkv, w.d, w.seed, fill_caches=False)
        kc = I.fill_normal_on_device(torch.empty(w.B, w.L, w.Hkv, w.d, dtype=torch.bfloat16,
                                                 device=dev), 1)
        vc = I.fill_normal_on_device(torch.empty_like(kc), 2)
        q, lam = x["q"].to(dev), x["lam"].to(dev)
        ws = torch.empty(Bd.diffattn_v2_decode_workspace_size(w.B, w.Hq, w.Hkv, w.d, w.L),
                         dtype=torch.uint8, device=dev)
        o = torch.empty(w.B, w.Hq // 2, w.d, dtype=torch.bfloat16, device=dev)
        ms = time_call(lambda: Bd.diffattn_v2_decode(q, kc, vc, lam, workspace=ws, out=o), 20, 3,
                       stream)
        by = v2_decode_bytes(w.B, w.L, w.Hkv, w.d, w.Hq)
        gbs = by / (ms * 1e-3) / 1e9
        out["v2_decode_bf16"] = {"value": round(gbs, 1), "unit": "GB/s", "ms": round(ms, 4),
                                 "frac": round(gbs / peaks["hbm_gbs"], 4),
                                 "peak": peaks["hbm_gbs"], "bytes": by, "batch": w.B,
                                 "frac_of_nominal": round(gbs / NOMINAL_HBM_GBS, 4),
                                 "target": ">= 0.70 of the nominal %.0f GB/s" % NOMINAL_HBM_GBS}
        if cpu_s > 0:
            P_ = w.Hq // 2
            out["v2_decode_bf16"]["cpu_baseline"] = dict(oracle_rate(_decode_sampler(
                lambda b, k_, v_: O.v2_decode_rows(x["q"][b:b + 1], k_[None], v_[None], x["lam"],
                                                   np.arange(P_)),
                (kc, vc), w.B, v2_decode_bytes(1, w.L, w.Hkv, w.d, w.Hq), 13),
                cpu_s, 1e9, "batch entries, every output"), unit="GB/s")
        del kc, vc, ws
        torch.cuda.empty_cache()

    if want("v1_decode_bf16"):  # B64 L32768 H32 d64 dv128 (comparison)
        w = wl("v1_decode_bf16")
        x = I.v1_decode_inputs(w.B, w.L, w.H, w.d, w.dv, w.seed, fill_caches=False)
        kc = I.fill_normal_on_device(torch.empty(w.B, w.L, w.H, 2 * w.d, dtype=torch.bfloat16,
                                                 device=dev), 3)
        vc = I.fill_normal_on_device(torch.empty(w.B, w.L, w.H, w.dv, dtype=torch.bfloat16,
                                                 device=dev), 4)
        q = x["q"].to(dev)
        lamt = Bd.lambda_from_params(*(x[n].to(dev) for n in ("lq1", "lk1", "lq2", "lk2")),
                                     w.layer)
        li = Bd.diffattn_lambda_init(w.layer)
        ws = torch.empty(Bd.diffattn_v1_decode_workspace_size(w.B, w.H, w.d, w.dv, w.L),
                         dtype=torch.uint8, device=dev)
        o = torch.empty(w.B, w.H, w.dv, dtype=torch.bfloat16, device=dev)
        ms = time_call(lambda: Bd.diffattn_v1_decode(q, kc, vc, lamt, apply_norm=True,
                                                     lambda_init=li, workspace=ws, out=o), 5, 2,
                       stream)
        by = v1_decode_bytes(w.B, w.L, w.H, w.d, w.dv)
        gbs = by / (ms * 1e-3) / 1e9
        out["v1_decode_bf16"] = {"value": round(gbs, 1), "unit": "GB/s", "ms": round(ms, 4),
                                 "frac": round(gbs / peaks["hbm_gbs"], 4), "bytes": by,
                                 "batch": w.B,
                                 "frac_of_nominal": round(gbs / NOMINAL_HBM_GBS, 4)}
        if cpu_s > 0:
            lam_h = O.lambda_from_params(x["lq1"], x["lk1"], x["lq2"], x["lk2"], w.layer)
            out["v1_decode_bf16"]["cpu_baseline"] = dict(oracle_rate(_decode_sampler(
                lambda b, k_, v_: O.v1_decode_rows(x["q"][b:b + 1], k_[None], v_[None], lam_h,
                                                   np.arange(w.H), apply_norm=True, eps=w.eps,
                                                   lambda_init_value=li),
                (kc, vc), w.B, v1_decode_bytes(1, w.L, w.H, w.d, w.dv), 14),
                cpu_s, 1e9, "batch entries, every output"), unit="GB/s")
        del kc, vc, ws
        torch.cuda.empty_cache()

    if want("v2_prefill_window_bf16"):  # V2 prefill with a 1024-key sliding window
        w = wl("v2_prefill_window_bf16")
        W = w.extra["window"]
        x = I.v2_inputs(w.B, w.N, w.Hq, w.Hkv, w.d, w.seed)
        q, k, v, lamt = (x[n].to(dev) for n in ("q", "k", "v", "lam"))
        o = torch.empty(w.B, w.N, w.Hq // 2, w.d, dtype=torch.bfloat16, device=dev)
        ms = time_call(lambda: Bd.diffattn_v2_prefill_window(q, k, v, lamt, W, out=o), 20, 3,
                       stream)
        pairs = window_pairs(w.B, w.N, w.Hq // 2, W)
        flop = pairs * v2_flops_per_pair(w.d)
        t = flop / (ms * 1e-3) / 1e12
        out["v2_prefill_window_bf16"] = {"value": round(t, 2), "unit": "TFLOP/s",
                                         "ms": round(ms, 4),
                                         "frac": round(t / peaks["bf16_tflops"], 4),
                                         "flop": flop, "window": W}
        if cpu_s > 0:
            P_ = w.Hq // 2
            out["v2_prefill_window_bf16"]["cpu_baseline"] = dict(oracle_rate(_rows_sampler(
                lambda r: O.v2_rows(x["q"], x["k"], x["v"], x["lam"], r, causal=True, window=W),
                w.B * w.N * P_,
                lambda r: min((r // P_) % w.N + 1, W) * v2_flops_per_pair(w.d), 15),
                cpu_s, 1e12, "random output rows"), unit="TFLOP/s")
        del q, k, v, o
        torch.cuda.empty_cache()

    if want("v2_decode_window_bf16"):  # V2 decode reading the last 4096 of 32768 entries
        w = wl("v2_decode_window_bf16")
        W = w.extra["window"]
        x = I.v2_decode_inputs(w.B, w.L, w.Hq, w.Hkv, w.d, w.seed, fill_caches=False)
        kc = I.fill_normal_on_device(torch.empty(w.B, w.L, w.Hkv, w.d, dtype=torch.bfloat16,
                                                 device=dev), 5)
        vc = I.fill_normal_on_device(torch.empty(w.B, w.L, w.Hkv, w.d, dtype=torch.bfloat16,
                                                 device=dev), 6)
        q, lamt = x["q"].to(dev), x["lam"].to(dev)
        span = min(W, w.L)
        ws = torch.empty(Bd.diffattn_v2_decode_workspace_size(w.B, w.Hq, w.Hkv, w.d, span),
                         dtype=torch.uint8, device=dev)
        o = torch.empty(w.B, w.Hq // 2, w.d, dtype=torch.bfloat16, device=dev)
        ms = time_call(lambda: Bd.diffattn_v2_decode_window(q, kc, vc, lamt, W, workspace=ws,
                                                            out=o), 20, 3, stream)
        by = v2_decode_bytes(w.B, span, w.Hkv, w.d, w.Hq)
        gbs = by / (ms * 1e-3) / 1e9
        out["v2_decode_window_bf16"] = {"value": round(gbs, 1), "unit": "GB/s",
                                        "ms": round(ms, 4),
                                        "frac": round(gbs / peaks["hbm_gbs"], 4), "bytes": by,
                                        "batch": w.B, "window": W,
                                        "frac_of_nominal": round(gbs / NOMINAL_HBM_GBS, 4)}
        if cpu_s > 0:  # the oracle reads the window's entries only: copy just those
            P_ = w.Hq // 2
            out["v2_decode_window_bf16"]["cpu_baseline"] = dict(oracle_rate(_decode_sampler(
                lambda b, k_, v_: O.v2_decode_rows(x["q"][b:b + 1], k_[None], v_[None], x["lam"],
                                                   np.arange(P_)),
                (kc[:, w.L - span:], vc[:, w.L - span:]), w.B,
                v2_decode_bytes(1, span, w.Hkv, w.d, w.Hq), 16),
                cpu_s, 1e9, "batch entries, every output"), unit="GB/s")
        del kc, vc, ws
        torch.cuda.empty_cache()

    if want("v1_backward_bf16"):  # gradients at the V1 headline shape (B4 H16 N4096, norm)
        w = wl("v1_prefill_bf16")
        x = I.v1_inputs(w.B, w.N, w.H, w.d, w.dv, w.seed)
        q, k, v = (x[n].to(dev) for n in ("q", "k", "v"))
        dout = torch.randn(w.B, w.N, w.H, w.dv, device=dev).to(torch.bfloat16)
        lamt = Bd.lambda_from_params(*(x[n].to(dev) for n in ("lq1", "lk1", "lq2", "lk2")),
                                     w.layer)
        li = Bd.diffattn_lambda_init(w.layer)
        ws = torch.empty(Bd.diffattn_v1_bwd_workspace_size(w.B, w.N, w.H, w.d, w.dv),
                         dtype=torch.uint8, device=dev)
        ms = time_call(lambda: Bd.diffattn_v1_bwd(q, k, v, dout, lamt, causal=True,
                                                  apply_norm=True, norm_eps=w.eps,
                                                  lambda_init=li, workspace=ws), 5, 2, stream)
        flop = prefill_pairs(w.B, w.N, w.H) * v1_bwd_flops_per_pair(w.d, w.dv)
        t = flop / (ms * 1e-3) / 1e12
        out["v1_backward_bf16"] = {"value": round(t, 2), "unit": "TFLOP/s", "ms": round(ms, 4),
                                   "frac": round(t / peaks["bf16_tflops"], 4), "flop": flop,
                                   "workspace_bytes": ws.numel()}
        if cpu_s > 0:  # the oracle's backward on (batch, head) slices of the first 512 tokens
            lam_h = O.lambda_from_params(x["lq1"], x["lk1"], x["lq2"], x["lk2"], w.layer)
            g_h = dout.cpu()
            rng = np.random.default_rng(17)
            n_p = 512

            def bwd_once(n):
                for _ in range(n):
                    b, h = int(rng.integers(w.B)), int(rng.integers(w.H))
                    sl = (slice(b, b + 1), slice(0, n_p), slice(h, h + 1))
                    O.v1_bwd(x["q"][sl], x["k"][sl], x["v"][sl], g_h[sl], lam_h[h:h + 1],
                             causal=True, apply_norm=True, eps=w.eps, lambda_init_value=li)
                return float(n * prefill_pairs(1, n_p, 1) * v1_bwd_flops_per_pair(w.d, w.dv))
            out["v1_backward_bf16"]["cpu_baseline"] = dict(oracle_rate(
                bwd_once, cpu_s, 1e12, "(batch, head) slices of the first 512 tokens"),
                unit="TFLOP/s", cores=1)
        del q, k, v, dout, ws
        torch.cuda.empty_cache()

    if want("v1_backward_saved_bf16"):  # V1 headline shape: training forward + backward from saves
        w = wl("v1_prefill_bf16")
        x = I.v1_inputs(w.B, w.N, w.H, w.d, w.dv, w.seed)
        q, k, v = (x[n].to(dev) for n in ("q", "k", "v"))
        dout = torch.randn(w.B, w.N, w.H, w.dv, device=dev).to(torch.bfloat16)
        lamt = Bd.lambda_from_params(*(x[n].to(dev) for n in ("lq1", "lk1", "lq2", "lk2")),
                                     w.layer)
        li = Bd.diffattn_lambda_init(w.layer)
        kw = dict(causal=True, apply_norm=True, norm_eps=w.eps, lambda_init=li)
        o = torch.empty(w.B, w.N, w.H, w.dv, dtype=torch.bfloat16, device=dev)
        _, saves = Bd.diffattn_v1_fwd_train(q, k, v, lamt, out=o, **kw)
        ws = torch.empty(Bd.load().diffattn_v1_bwd_saved_workspace_size(w.B, w.N, w.H),
                         dtype=torch.uint8, device=dev)
        f32 = dict(dtype=torch.float32, device=dev)
        grads = {"dq": torch.empty(q.shape, **f32), "dk": torch.empty(k.shape, **f32),
                 "dv": torch.empty(v.shape, **f32), "dlambda": torch.empty(w.H, **f32),
                 "dnorm_weight": torch.empty(w.dv, **f32)}
        ms_b = time_call(lambda: Bd.diffattn_v1_bwd_saved(q, k, v, dout, lamt, saves, workspace=ws,
                                                          out=grads, **kw), 5, 2, stream)

        def train_step():
            Bd.diffattn_v1_fwd_train(q, k, v, lamt, out=o, saves=saves, **kw)
            Bd.diffattn_v1_bwd_saved(q, k, v, dout, lamt, saves, workspace=ws, out=grads, **kw)
        ms_t = time_call(train_step, 5, 2, stream)
        pairs = prefill_pairs(w.B, w.N, w.H)
        fb = pairs * v1_bwd_flops_per_pair(w.d, w.dv)
        ft = pairs * (v1_flops_per_pair(w.d, w.dv) + v1_bwd_flops_per_pair(w.d, w.dv))
        tb, tt = fb / (ms_b * 1e-3) / 1e12, ft / (ms_t * 1e-3) / 1e12
        out["v1_backward_saved_bf16"] = {
            "value": round(tb, 2), "unit": "TFLOP/s", "ms": round(ms_b, 4),
            "frac": round(tb / peaks["bf16_tflops"], 4), "flop": fb,
            "what": "backward from the training forward's saves (row kernel, dQ, dK/dV)"}
        out["v1_train_step_bf16"] = {
            "value": round(tt, 2), "unit": "TFLOP/s", "ms": round(ms_t, 4),
            "frac": round(tt / peaks["bf16_tflops"], 4), "flop": ft,
            "what": "training forward with saves + backward from the saves "
                    "(768 + 1792 flop per visible pair)"}
        if cpu_s > 0:  # the oracle's backward (it runs the forward too) on head slices
            lam_h = O.lambda_from_params(x["lq1"], x["lk1"], x["lq2"], x["lk2"], w.layer)
            g_h = dout.cpu()
            rng = np.random.default_rng(20)
            n_p = 512

            def slices_once(n):
                for _ in range(n):
                    b, h = int(rng.integers(w.B)), int(rng.integers(w.H))
                    sl = (slice(b, b + 1), slice(0, n_p), slice(h, h + 1))
                    O.v1_bwd(x["q"][sl], x["k"][sl], x["v"][sl], g_h[sl], lam_h[h:h + 1],
                             causal=True, apply_norm=True, eps=w.eps, lambda_init_value=li)
                return float(n * prefill_pairs(1, n_p, 1) * v1_bwd_flops_per_pair(w.d, w.dv))
            cb = dict(oracle_rate(slices_once, cpu_s, 1e12,
                                  "(batch, head) slices of the first 512 tokens"),
                      unit="TFLOP/s", cores=1)
            out["v1_backward_saved_bf16"]["cpu_baseline"] = cb
            # the same oracle calls, counted with the forward's flops as well
            ct = dict(cb)
            ct["value"] = cb["value"] * (v1_flops_per_pair(w.d, w.dv) + v1_bwd_flops_per_pair(
                w.d, w.dv)) / v1_bwd_flops_per_pair(w.d, w.dv)
            out["v1_train_step_bf16"]["cpu_baseline"] = ct
        del q, k, v, dout, ws, saves, grads, o
        torch.cuda.empty_cache()

    if want("v2_backward_bf16"):  # gradients at the V2 prefill shape (B2 Hq32 Hkv8 N8192)
        w = wl("v2_prefill_bf16")
        x = I.v2_inputs(w.B, w.N, w.Hq, w.Hkv, w.d, w.seed)
        q, k, v, lamt = (x[n].to(dev) for n in ("q", "k", "v", "lam"))
        dout = torch.randn(w.B, w.N, w.Hq // 2, w.d, device=dev).to(torch.bfloat16)
        ws = torch.empty(Bd.diffattn_v2_bwd_workspace_size(w.B, w.N, w.Hq, w.Hkv, w.d),
                         dtype=torch.uint8, device=dev)
        ms = time_call(lambda: Bd.diffattn_v2_bwd(q, k, v, dout, lamt, causal=True,
                                                  workspace=ws), 5, 2, stream)
        flop = prefill_pairs(w.B, w.N, w.Hq // 2) * v1_bwd_flops_per_pair(w.d, w.d)
        t = flop / (ms * 1e-3) / 1e12
        out["v2_backward_bf16"] = {"value": round(t, 2), "unit": "TFLOP/s", "ms": round(ms, 4),
                                   "frac": round(t / peaks["bf16_tflops"], 4), "flop": flop,
                                   "workspace_bytes": ws.numel()}
        if cpu_s > 0:  # the oracle's backward on (batch, KV head) slices of 512 tokens
            g_h = dout.cpu()
            rng = np.random.default_rng(18)
            n_p, grp = 512, w.Hq // w.Hkv

            def bwd_once(n):
                for _ in range(n):
                    b, g = int(rng.integers(w.B)), int(rng.integers(w.Hkv))
                    tq = (slice(b, b + 1), slice(0, n_p), slice(g * grp, (g + 1) * grp))
                    tk = (slice(b, b + 1), slice(0, n_p), slice(g, g + 1))
                    to = (slice(b, b + 1), slice(0, n_p), slice(g * grp // 2, (g + 1) * grp // 2))
                    O.v2_bwd(x["q"][tq], x["k"][tk], x["v"][tk], g_h[to],
                             x["lam"][g * grp // 2:(g + 1) * grp // 2], causal=True)
                return float(n * prefill_pairs(1, n_p, grp // 2) * v1_bwd_flops_per_pair(w.d, w.d))
            out["v2_backward_bf16"]["cpu_baseline"] = dict(oracle_rate(
                bwd_once, cpu_s, 1e12, "(batch, KV head) slices of the first 512 tokens"),
                unit="TFLOP/s", cores=1)
        del q, k, v, dout, ws
        torch.cuda.empty_cache()

    if want("v2_prefill_oproj_bf16"):  # V2 prefill + output projection to d_model 2048
        w = wl("v2_prefill_bf16")
        dm = 2048
        x = I.v2_inputs(w.B, w.N, w.Hq, w.Hkv, w.d, w.seed)
        q, k, v, lamt = (x[n].to(dev) for n in ("q", "k", "v", "lam"))
        W = (torch.randn(w.Hq // 2 * w.d, dm, device=dev) / (w.Hq // 2 * w.d) ** 0.5).to(
            torch.bfloat16)
        ws = torch.empty(Bd.diffattn_v2_prefill_oproj_workspace_size(w.B, w.N, w.Hq, w.d),
                         dtype=torch.uint8, device=dev)
        o = torch.empty(w.B, w.N, dm, dtype=torch.bfloat16, device=dev)
        ms = time_call(lambda: Bd.diffattn_v2_prefill_oproj(q, k, v, lamt, W, workspace=ws,
                                                            out=o), 20, 3, stream)
        flop_att = prefill_pairs(w.B, w.N, w.Hq // 2) * v2_flops_per_pair(w.d)
        flop_gemm = 2 * w.B * w.N * (w.Hq // 2 * w.d) * dm
        t = (flop_att + flop_gemm) / (ms * 1e-3) / 1e12
        out["v2_prefill_oproj_bf16"] = {"value": round(t, 2), "unit": "TFLOP/s",
                                        "ms": round(ms, 4),
                                        "frac": round(t / peaks["bf16_tflops"], 4),
                                        "flop": flop_att + flop_gemm, "d_model": dm}
        if cpu_s > 0:  # every pair of random tokens, then the projection, in float64
            P_ = w.Hq // 2
            W_h = W.double().cpu().numpy()
            rng = np.random.default_rng(19)

            def proj_once(n):
                toks = rng.integers(0, w.B * w.N, n)
                rows = (toks[:, None] * P_ + np.arange(P_)[None, :]).reshape(-1)
                o_h = O.v2_rows(x["q"], x["k"], x["v"], x["lam"], rows, causal=True)
                _ = o_h.reshape(n, P_ * w.d) @ W_h
                return float(sum((int(t) % w.N + 1) * P_ * v2_flops_per_pair(w.d) for t in toks)
                             + n * 2 * P_ * w.d * dm)
            out["v2_prefill_oproj_bf16"]["cpu_baseline"] = dict(oracle_rate(
                proj_once, cpu_s, 1e12, "random tokens, every pair and the projection"),
                unit="TFLOP/s")
        del q, k, v, W, ws, o
        torch.cuda.empty_cache()

    if want("snr_v1_decode"):  # noise-cancellation sweep, 6 configs x 11 lambdas, L 1024
        from differential_attention_sm_b200 import snr as S
        w = wl("snr_v1_decode")
        x = I.snr_inputs(w.seed, w.L, w.d, w.dv, **{k: w.extra[k] for k in
                                                     ("sigmas", "rhos", "alpha", "pos")})
        res = S.run_sweep(x, device=str(dev))
        q, kc, vc, lamt = (x[n].to(dev) for n in ("q", "k_cache", "v_cache", "lam"))
        B_, H_ = q.shape[0], q.shape[1]
        ws = torch.empty(Bd.diffattn_v1_decode_workspace_size(B_, H_, w.d, w.dv, w.L),
                         dtype=torch.uint8, device=dev)
        o = torch.empty(B_, H_, w.dv, dtype=torch.bfloat16, device=dev)
        ms = time_call(lambda: Bd.diffattn_v1_decode(q, kc, vc, lamt, workspace=ws, out=o),
                       20, 3, stream)
        by = v1_decode_bytes(B_, w.L, H_, w.d, w.dv)
        gbs = by / (ms * 1e-3) / 1e9
        summary = []
        for c, (sigma, rho) in enumerate(res["configs"]):
            r = res["snr"][c]
            i = int(np.nanargmax(r))
            summary.append({"sigma": sigma, "rho": rho, "snr_softmax": round(float(r[0]), 3),
                            "snr_best": round(float(r[i]), 3),
                            "best_lambda": round(float(res["lam"][i]), 2)})
        out["snr_v1_decode"] = {"value": round(gbs, 1), "unit": "GB/s", "ms": round(ms, 4),
                                "frac": round(gbs / peaks["hbm_gbs"], 4), "bytes": by,
                                "batch": B_, "sweep": summary}
        del kc, vc, ws
        torch.cuda.empty_cache()
    out["peak_source"] = peak_src
    return out


# ---------------------------------------------------------------------------
# CPU baseline / reference arm: the fp64 oracle on host cores
# ---------------------------------------------------------------------------
def oracle_sample(x, w, target_s: float, seed: int):
    """Runs the oracle on random rows of the workload until about target_s
    seconds of work; returns (algorithmic flop done, seconds, rows)."""
    import oracle as O
    lam = O.lambda_from_params(x["lq1"], x["lk1"], x["lq2"], x["lk2"], w.layer)
    li = O.lambda_init(w.layer)
    rng = np.random.default_rng(seed)
    fpp = v1_flops_per_pair(w.d, w.dv)
    total_rows = w.B * w.N * w.H
    n, done_fl, done_s, rows_done = 8, 0.0, 0.0, 0
    while done_s < target_s:
        rows = rng.integers(0, total_rows, n)
        i = (rows // w.H) % w.N
        t0 = time.perf_counter()
        O.v1_rows(x["q"], x["k"], x["v"], lam, rows, causal=True, apply_norm=True,
                  eps=w.eps, lambda_init_value=li)
        dt = time.perf_counter() - t0
        done_fl += float(((i + 1) * fpp).sum())
        done_s += dt
        rows_done += n
        if dt < target_s / 4:
            n *= 2
    return done_fl, done_s, rows_done


def run_reference(args, rank, world):
    if rank != 0:
        return 0
    import oracle as O
    from differential_attention_sm_b200 import inputs as I
    O.build()
    w = I.WORKLOADS["v1_prefill_bf16"]
    x = I.v1_inputs(w.B, w.N, w.H, w.d, w.dv, w.seed)
    # bounded host work: the whole run stays near 90 s whatever K and W are
    per_step = max(0.01, min(2.0, 90.0 / max(1, args.steps + args.warmup)))
    for s in range(args.warmup):
        oracle_sample(x, w, per_step, seed=s)
    fl, secs, rows = 0.0, 0.0, 0
    for s in range(args.steps):
        f, t, r = oracle_sample(x, w, per_step, seed=1000 + s)
        fl += f
        secs += t
        rows += r
    val = fl / secs / 1e12
    line = {
        "impl": "reference", "metric": METRIC, "value": val, "unit": "TFLOP/s",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": 1e3 * secs / args.steps, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": "v1_prefill_bf16: V1 causal prefill, batch 4, 16 heads, seq 4096, "
                               "QK 64 per branch, V 128, layer 12, RMSNorm",
                   "note": "reference arm = the fp64 CPU oracle; each step is a bounded random "
                           "sample of output rows (%.2f s of host work)" % per_step},
        "cpu_baseline": {"value": val, "unit": "TFLOP/s", "cores": O.n_threads(),
                         "kind": "oracle",
                         "sample": "%d random output rows of the workload over %d steps" % (
                             rows, args.steps)},
        "e2e": {"value": val, "unit": "TFLOP/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=1000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--no-extras", action="store_true",
                    help="skip the secondary workloads (V2 prefill, long V1, decode, SNR sweep)")
    ap.add_argument("--cpu-seconds", type=float, default=12.0,
                    help="bounded host time for the oracle CPU baseline")
    ap.add_argument("--extras-cpu-seconds", type=float, default=2.0,
                    help="bounded host time of each secondary workload's oracle sample "
                         "(0 skips them)")
    ap.add_argument("--only", default=None,
                    choices=["v2_prefill_bf16", "v1_long_bf16", "v2_decode_bf16",
                             "v1_decode_bf16", "snr_v1_decode", "v2_prefill_window_bf16",
                             "v2_decode_window_bf16", "v1_backward_bf16",
                             "v1_backward_saved_bf16",
                             "v2_backward_bf16", "v2_prefill_oproj_bf16"],
                    help="run just this secondary workload (one GPU) and print its numbers")
    ap.add_argument("--decode-batch", type=int, default=None,
                    help="with --only: smaller decode batch (profiling runs)")
    args = ap.parse_args()
    rank, world, local_rank = dist_env()
    if args.impl == "reference":
        return run_reference(args, rank, world)
    if args.only:
        import torch
        torch.cuda.set_device(local_rank)
        peaks, peak_src = load_peaks()
        print(json.dumps(run_extras(local_rank, peaks, peak_src, args.only, args.decode_batch,
                                    cpu_s=args.extras_cpu_seconds)), flush=True)
        return 0

    import torch
    torch.cuda.set_device(local_rank)
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local_rank))
    from differential_attention_sm_b200 import binding as Bd
    Bd.load()
    peaks, peak_src = load_peaks()
    res, x = run_headline(args, rank, world, local_rank, peaks, peak_src)
    extras = None
    if world == 1 and not args.no_extras:
        extras = run_extras(local_rank, peaks, peak_src, cpu_s=args.extras_cpu_seconds)
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
        dist.destroy_process_group()
    if rank != 0:
        return 0
    import oracle as O
    from differential_attention_sm_b200 import inputs as I
    cpu = None
    if world == 1:
        O.build()
        w = I.WORKLOADS["v1_prefill_bf16"]
        fl, secs, rows = oracle_sample(x, w, args.cpu_seconds, seed=7)
        cpu = {"value": fl / secs / 1e12, "unit": "TFLOP/s", "cores": O.n_threads(),
               "kind": "oracle",
               "sample": "%d random output rows of the V1 prefill workload (%.1f s)" % (
                   rows, secs)}
    line = {
        "metric": METRIC, "value": res["value"], "unit": "TFLOP/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": res["ms_per_step"],
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic (seeded N(0,1), bf16-rounded)", "config": res["config"],
        "roofline": res["roofline"], "cpu_baseline": cpu, "e2e": res["e2e"],
        "gpu_launches": res["gpu_launches"], "clocks": res["clocks"],
    }
    if extras is not None:
        line["also"] = extras
    print(json.dumps(line), flush=True)
    return 0


if __name__ == "__main__":
    sys.exit(main())
