"""Throughput of the Flash-Cache step on B200: query-tokens/s per fused step.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl ours|reference]

A step is one fc_step (QKV projection + RoPE + KV-cache write, bidirectional
attention with importance, importance finalisation) plus one fc_topk_tracked
on the headline workload: B=32 sequences, cache 1536 each, 128 query rows
(64 tracked + 64 masked window) per sequence, hidden 4096, 32 heads x 128,
bf16 (LLaDA-8B-shaped, random weights, synthetic data).

Timing: W untimed warm-up steps, then K steps timed with CUDA events on the
launching stream; an L2 flush (a 256 MiB write) runs between steps outside the
events.  Under torchrun every rank runs its own batch (sequences are
independent, no collective on the data path): value = all ranks' query tokens
/ the slowest rank's time.  ``--impl reference`` times the fp64 CPU oracle on
the host cores instead (the deliberately slow baseline arm).
"""
from __future__ import annotations

import argparse
import ctypes
import json
import os
import statistics
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "query-tokens/s per fused Flash-Cache step (B=32, L=1536); % of roofline"
UNIT = "query-tokens/s"


# Sources whose SHA-256 (concatenated, first 16 hex digits) keys a committed
# ncu traffic figure for each kernel.
_KERNEL_SOURCES = {
    "qkv_rope_scatter": ["qkv_tc.cu", "ptx.cuh", "fc_internal.h", "fc_api.cu"],
    "attention": ["attn_tc.cu", "ptx.cuh", "fc_internal.h", "fc_api.cu"],
}


# Nominal B200 figures (dense bf16 tensor rate, HBM3e bandwidth), context only.
SPEC_BF16_TFLOPS, SPEC_HBM_GBS = 2250.0, 7700.0


def _tensor_peaks(peaks, sm_mhz):
    """The bf16 peaks a tensor-bound figure is set against: the measured
    sustained GEMM rate as measured, the same rate scaled to the SM clock the
    timed window ran at (a GEMM's rate follows the SM clock; the sustained
    figure was taken at the median clock recorded beside it), the measured
    burst rate, and the nominal dense rate."""
    out = {"sustained": peaks["bf16_tflops_sustained"], "burst": peaks["bf16_tflops"],
           "spec": SPEC_BF16_TFLOPS}
    ref_mhz = peaks.get("sustained_mhz")
    if sm_mhz and ref_mhz:
        out["sustained_clock_scaled"] = peaks["bf16_tflops_sustained"] * sm_mhz / ref_mhz
    return out


def _kernel_roofline(name, bound, work, timing, peaks, traffic, sm_mhz=None):
    """Achieved rate of one kernel (algorithmic work / mean launch time).  The
    kernels are timed in the steady state of a sustained load, so a contraction
    is set against the sustained bf16 GEMM rate (`frac`); `frac_vs` gives the
    same rate against every peak variant."""
    ms, n = timing
    avg_s = ms / max(n, 1) / 1e3
    if bound == "tensor":
        achieved, peak, unit = work / avg_s / 1e12, peaks["bf16_tflops_sustained"], "TFLOP/s"
        frac_vs = {k: achieved / v for k, v in _tensor_peaks(peaks, sm_mhz).items()}
    else:
        achieved, peak, unit = work / avg_s / 1e9, peaks["hbm_gbs"], "GB/s"
        frac_vs = {"measured_copy": achieved / peaks["hbm_gbs"], "spec": achieved / SPEC_HBM_GBS}
    return {"bound": bound, "achieved": achieved, "peak": peak, "unit": unit, "frac": achieved / peak,
            "frac_vs": frac_vs, "us_per_launch": avg_s * 1e6, "traffic": traffic}


def _step_roofline(wk, t_step_s, peaks, sm_mhz):
    """The whole step against max(FLOPs / bf16 peak, bytes / HBM bandwidth),
    for every peak variant; `frac` uses the measured sustained rate, and the
    clock-scaled variant is the one the step target is judged on."""
    tp = _tensor_peaks(peaks, sm_mhz)
    var = {}
    for k, tf in tp.items():
        bw = SPEC_HBM_GBS if k == "spec" else peaks["hbm_gbs"]
        t_c, t_b = wk["flops"] / (tf * 1e12), wk["bytes"] / (bw * 1e9)
        var[k] = {"bf16_tflops": tf, "hbm_gbs": bw, "t_roof_us": max(t_c, t_b) * 1e6,
                  "bound": "tensor" if t_c >= t_b else "hbm", "frac": max(t_c, t_b) / t_step_s}
    s = var["sustained"]
    return {"t_roof_us": s["t_roof_us"], "t_step_us": t_step_s * 1e6, "frac": s["frac"],
            "bound": s["bound"], "flops": wk["flops"], "bytes": wk["bytes"], "variants": var,
            "judged_on": "sustained_clock_scaled" if "sustained_clock_scaled" in var else "sustained",
            "sm_mhz": sm_mhz, "sustained_peak_mhz": peaks.get("sustained_mhz")}


def _dram_traffic(workload):
    """DRAM bytes per launch from the committed ncu summary, for kernels whose
    sources are unchanged since the capture (else absent -> null)."""
    import hashlib
    path = os.path.join(ROOT, "profiles", f"dram_traffic_{workload}.txt")
    out = {}
    if not os.path.exists(path):
        return out
    csrc = os.path.join(ROOT, "kv_cache_attention_qkv_b200", "csrc")
    for line in open(path):
        f = line.split()
        if not f or f[0].startswith("#") or len(f) < 5 or f[0] not in _KERNEL_SOURCES:
            continue
        h = hashlib.sha256()
        for name in _KERNEL_SOURCES[f[0]]:
            with open(os.path.join(csrc, name), "rb") as fh:
                h.update(fh.read())
        if f[1] == workload and h.hexdigest()[:16] == f[2]:
            out[f[0]] = int(f[3]) + int(f[4])
    return out


def _peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            j = json.load(f)
        return {"hbm_gbs": j["hbm_gbs"], "bf16_tflops": j["bf16_tflops"],
                "bf16_tflops_sustained": j.get("bf16_tflops_sustained"),
                "sustained_mhz": (j.get("clocks_under_load") or {}).get("sm_mhz_median"),
                "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0,
            "sustained_mhz": 1300.0, "source": "fallback"}


def _work(inp):
    """Algorithmic FLOPs and bytes of one step (what the method must compute/move)."""
    T, S, D, H, d = inp.total_q, inp.total_k, inp.hidden, inp.n_heads, inp.head_dim
    es = 2 if inp.dtype == "bf16" else 4
    n = np.diff(inp.cu_seqlens_q).astype(np.int64)
    L = np.diff(inp.cu_seqlens_k).astype(np.int64)
    qkv_flops = 2.0 * T * D * 3 * H * d
    attn_flops = 4.0 * H * d * float((n * L).sum())
    qkv_bytes = es * (T * D + 3 * H * d * D) + es * 2 * T * H * d  # X, W read; K/V rows written
    attn_bytes = es * 2 * S * H * d + es * T * H * d  # whole cache read, O written
    return {"qkv_flops": qkv_flops, "attn_flops": attn_flops, "qkv_bytes": qkv_bytes,
            "attn_bytes": attn_bytes, "flops": qkv_flops + attn_flops,
            "bytes": qkv_bytes + attn_bytes}


class ClockSampler:
    """nvidia-smi clocks and throttle reasons, sampled every 100 ms; the summary
    keeps the samples taken between window_start() and window_end() (the load
    window around the timed steps)."""

    Q = ("timestamp,index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.idx = gpu_index
        self.proc = None
        self.path = None
        self.t0 = self.t1 = None

    def __enter__(self):
        import tempfile

        fd, self.path = tempfile.mkstemp(prefix="clocks_", suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.idx}", f"--query-gpu={self.Q}", "--format=csv,noheader,nounits",
                 "-lms", "100"], stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None
        time.sleep(0.3)
        return self

    def window_start(self):
        self.t0 = time.time()

    def window_end(self):
        self.t1 = time.time()

    def __exit__(self, *exc):
        if self.proc is not None:
            time.sleep(0.2)
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()

    def summary(self):
        import datetime

        if self.proc is None or not self.path or not os.path.exists(self.path):
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        rows = []
        for line in open(self.path):
            parts = [p.strip() for p in line.split(",")]
            if len(parts) >= 10:
                try:
                    ts = datetime.datetime.strptime(parts[0], "%Y/%m/%d %H:%M:%S.%f").timestamp()
                except ValueError:
                    ts = None
                rows.append((ts, parts[1:]))
        os.unlink(self.path)
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}
        inside = rows
        if self.t0 is not None and self.t1 is not None:
            inside = [r for r in rows if r[0] is not None and self.t0 <= r[0] <= self.t1]
        window = [r for _, r in (inside or rows)]

        def num(v):
            try:
                return float(v)
            except ValueError:
                return None

        sm = [num(r[1]) for r in window if num(r[1]) is not None]
        mx = [num(r[2]) for r in window if num(r[2]) is not None]
        pw = [num(r[3]) for r in window if num(r[3]) is not None]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in window for i in range(4) if r[5 + i].lower() == "active"})
        out = {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(mx) if mx else None,
               "power_w_max": max(pw) if pw else None, "samples": len(window), "reasons": reasons}
        if self.t0 is not None and self.t1 is not None:
            out["window_s"] = round(self.t1 - self.t0, 3)
            if not inside:
                out["note"] = "no sample inside the load window; all samples summarised"
        return out


def _dist_env():
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return ws, rank, local


def _work_balance(inp, num_ctas, qtile=128, ktile=128):
    """Balance of the attention kernels' static schedule: the work list holds
    one item per (sequence, head, 128-row query tile), longest caches first;
    in round r CTA c takes item r * num_ctas + c (even r) or
    r * num_ctas + num_ctas - 1 - c (odd r); an item's cost is taken as its
    number of 128-key tiles."""
    n = np.diff(inp.cu_seqlens_q).astype(np.int64)
    L = np.diff(inp.cu_seqlens_k).astype(np.int64)
    order = sorted(range(inp.batch), key=lambda b: (-int(L[b]), b))
    cost = []
    for b in order:
        if n[b] > 0 and L[b] > 0:
            cost += [int((L[b] + ktile - 1) // ktile)] * (inp.n_heads * int((n[b] + qtile - 1) // qtile))
    per = np.zeros(num_ctas, np.int64)
    for i, c in enumerate(cost):
        r, k = divmod(i, num_ctas)
        per[num_ctas - 1 - k if r % 2 else k] += c
    return {"items": len(cost), "ctas": num_ctas, "tiles_max_per_cta": int(per.max()),
            "tiles_mean_per_cta": float(per.mean()),
            "max_over_mean": float(per.max() / per.mean()) if per.mean() else None,
            "note": "static alternating-direction schedule over the longest-first work "
                    "list; cost = key tiles per item"}


def _step_result(args, inp, ws, *, total_ms, burst_ms, per_kernel, launches, err, e2e_ms, h2d,
                 d2h, clocks, noimp=None, num_sms=148, e2e_host_ms=None):
    """The JSON line of a step run from its measurements (no GPU needed).

    per_kernel: {name: (total ms, launches)} of the per-kernel pass; total_ms,
    burst_ms, e2e_ms: max over ranks of the K steps' device time."""
    peaks = _peaks()
    wk = _work(inp)
    T = inp.total_q
    # a step with importance runs the two-pass attention kernel alone; a step
    # without runs the one-pass kernel and the two-pass kernel for the items it
    # hands over (usually none): its attention is the sum of the two.  A small
    # batch split over the SMs runs two launches (row statistics, then pass 2
    # and the combine): its attention is their sum too.
    per_kernel = dict(per_kernel)
    if getattr(args, "no_importance", False) and per_kernel.get("attention_one_pass", (0, 0))[1]:
        (ma, na), (mb, _) = per_kernel["attention_one_pass"], per_kernel["attention"]
        per_kernel["attention"] = (ma + mb, na)
    if per_kernel.get("attention_split_pass1", (0, 0))[1]:
        (ma, _), (mb, nb) = per_kernel["attention_split_pass1"], per_kernel["attention"]
        per_kernel["attention"] = (ma + mb, nb)
    ms_per_step = total_ms / args.steps
    tokens = T * ws * args.steps
    value = tokens / (total_ms / 1e3)
    # dominant kernel by measured share
    names = {"qkv_rope_scatter": ("tensor", wk["qkv_flops"]), "attention": ("hbm", wk["attn_bytes"])}
    dom = max(names, key=lambda k: per_kernel[k][0])
    traffic = _dram_traffic(args.workload)
    sm_mhz = (clocks or {}).get("sm_mhz")
    rl = _kernel_roofline(dom, *names[dom], per_kernel[dom], peaks, traffic.get(dom), sm_mhz)
    extra = {}
    if noimp is not None:
        nms, npk = noimp
        one = npk.get("attention_one_pass", (0.0, 0))
        extra["no_importance"] = {
            "ms_per_step": nms / args.steps, "value": T * ws * args.steps / (nms / 1e3),
            "kernels_ms_per_step": {k: v[0] / max(v[1], 1) for k, v in npk.items() if v[1]},
            "attention_one_pass": (_kernel_roofline("attention_one_pass", "hbm", wk["attn_bytes"],
                                                    one, peaks, None, sm_mhz) if one[1] else None),
            "note": "context: the same step without importance or reselection; its attention "
                    "runs in the one-pass kernel"}
    return {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": ws, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": inp.dtype, "data": "synthetic",
        "config": _step_config(args.workload, inp, ws, not getattr(args, "no_importance", False)),
        "roofline": {"kernel": dom, "bound": rl["bound"], "achieved": rl["achieved"],
                     "peak": rl["peak"], "unit": rl["unit"], "frac": rl["frac"],
                     "traffic": rl["traffic"], "frac_vs": rl["frac_vs"],
                     "peak_source": f"{peaks['source']} (MEASURED_PEAKS.json: sustained bf16 for "
                                    "tensor-bound kernels, copy bandwidth for HBM-bound ones)"},
        "kernel_rooflines": {k: _kernel_roofline(k, b, w, per_kernel[k], peaks, traffic.get(k), sm_mhz)
                             for k, (b, w) in names.items()},
        "step_roofline": _step_roofline(wk, ms_per_step / 1e3, peaks, sm_mhz),
        "kernels_ms_per_step": {k: v[0] / max(v[1], 1) for k, v in per_kernel.items()},
        "gpu_launches": launches,
        "device_error_word": err,
        "burst": {"value": tokens / (burst_ms / 1e3), "ms_per_step": burst_ms / args.steps,
                  "note": "the same K steps right after the warm-up, before the power "
                          "controller reacts; value and rooflines above are the steady state"},
        "e2e": {"value": tokens / (e2e_ms / 1e3), "unit": UNIT,
                "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h),
                **({"ms_per_step": e2e_ms / args.steps,
                    "host_enqueue_ms_per_step": e2e_host_ms / args.steps}
                   if e2e_host_ms is not None else {})},
        "clocks": clocks,
        "work_balance": _work_balance(inp, num_sms),
        **extra,
    }


def run_ours(args):
    import torch
    import torch.distributed as dist

    from kv_cache_attention_qkv_b200 import FlashCache, shard, workloads

    ws, rank, local = _dist_env()
    if ws > 1:
        os.environ.setdefault("MASTER_ADDR", "127.0.0.1")
        torch.cuda.set_device(local)
        from datetime import timedelta

        dist.init_process_group("nccl", timeout=timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    else:
        torch.cuda.set_device(0)
    dev = torch.device("cuda", torch.cuda.current_device())

    # every rank draws its own batch of the same recipe
    base_seed = workloads.WORKLOADS.index(args.workload) if args.workload in workloads.WORKLOADS else 100
    inp = workloads.generate(args.workload, seed=base_seed + 1000 * rank)
    dt = torch.bfloat16 if inp.dtype == "bf16" else torch.float32
    f = lambda a: torch.from_numpy(np.ascontiguousarray(a)).to(dev, dtype=dt)
    i = lambda a: torch.from_numpy(np.ascontiguousarray(a, dtype=np.int32)).to(dev)
    x, w, kc, vc = f(inp.x), f(inp.w_qkv), f(inp.k_cache), f(inp.v_cache)
    qp, cq, ck = i(inp.q_pos), i(inp.cu_seqlens_q), i(inp.cu_seqlens_k)
    lo, hi, kps = i(inp.cand_lo), i(inp.cand_hi), i(inp.topk)
    T, S, H, d, B = inp.total_q, inp.total_k, inp.n_heads, inp.head_dim, inp.batch
    K = int(inp.topk.max())
    layer = FlashCache(w, hidden=inp.hidden, n_heads=H, head_dim=d, rope_theta=inp.rope_theta,
                       max_batch=B, max_total_q=T, max_total_k=S,
                       max_seqlen_q=int(np.diff(inp.cu_seqlens_q).max()),
                       max_pos=int(np.diff(inp.cu_seqlens_k).max()), max_topk=K)
    layer.set_qkv_kernel(args.qkv_kernel, args.qkv_split)
    layer.set_attn_split({"auto": True, "never": False, "always": "always"}[args.attn_split])
    out = torch.empty((T, H, d), device=dev, dtype=dt)
    imp = torch.empty((S,), device=dev, dtype=torch.float32)
    tracked = torch.empty((B, K), device=dev, dtype=torch.int32)
    flush = torch.empty(256 * 1024 * 1024 // 4, device=dev, dtype=torch.float32)
    stream = torch.cuda.current_stream()

    def step():
        if args.no_importance:  # attention only (the one-pass kernel), no reselection
            layer.step(x, qp, cq, ck, kc, vc, out, None)
            return layer.last_launch_count
        layer.step(x, qp, cq, ck, kc, vc, out, imp)
        n = layer.last_launch_count
        layer.topk_tracked(imp, ck, lo, hi, K, tracked, k_per_seq=kps)
        return n + layer.last_launch_count

    def step_noimp():
        layer.step(x, qp, cq, ck, kc, vc, out, None)

    for _ in range(args.warmup):
        flush.fill_(1.0)
        step()
    torch.cuda.synchronize()
    if layer.get_error() != 0:
        raise RuntimeError("device error word set during warm-up")

    def timed_steps(n):
        """n steps with an event pair around each, an L2 flush before each."""
        evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
               for _ in range(n)]
        nl = 0
        for k in range(n):
            flush.fill_(float(k))
            evs[k][0].record(stream)
            nl += step()
            evs[k][1].record(stream)
        torch.cuda.synchronize()
        return [a.elapsed_time(b) for a, b in evs], nl

    if ws > 1:
        dist.barrier()
    torch.cuda.synchronize()
    # burst (context only): the same K steps right after the warm-up, before the
    # power controller has reacted to the load
    burst_ms = float(sum(timed_steps(args.steps)[0]))
    with ClockSampler(torch.cuda.current_device()) as clk:
        # The K timed steps last milliseconds, less than the sampler's period, so
        # they are taken in the steady state of the load: after about a second
        # of the same untimed steps.  The sampler's window covers that second,
        # the timed steps and the per-kernel pass.
        clk.window_start()
        soak_t0, soak = time.perf_counter(), 0
        while time.perf_counter() - soak_t0 < 1.0:
            flush.fill_(float(soak))
            step()
            soak += 1
            if soak % 32 == 0:
                torch.cuda.synchronize()
        torch.cuda.synchronize()
        if ws > 1:
            dist.barrier()
        torch.cuda.synchronize()
        step_ms, launches = timed_steps(args.steps)
        if ws > 1:
            dist.barrier()
        # Per-kernel durations: the same K steps again with a CUDA event pair
        # around every kernel on its launching stream (events between kernels
        # stop the programmatic overlap of neighbouring kernels, so this pass is
        # not the step-time pass above).
        layer.profile(True)
        layer.profile_read()
        torch.cuda.synchronize()
        for k in range(args.steps):
            flush.fill_(float(k))
            step()
        torch.cuda.synchronize()
        per_kernel = layer.profile_read()
        # context: the same step without importance (its attention runs in the
        # one-pass kernel), step time and per-kernel times
        noimp = None
        if not args.no_importance:
            layer.profile(False)
            torch.cuda.synchronize()
            ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
                  for _ in range(args.steps)]
            for k in range(args.steps):
                flush.fill_(float(k))
                ev[k][0].record(stream)
                step_noimp()
                ev[k][1].record(stream)
            torch.cuda.synchronize()
            noimp_ms = sum(a.elapsed_time(b) for a, b in ev)
            layer.profile(True)
            layer.profile_read()
            for k in range(args.steps):
                flush.fill_(float(k))
                step_noimp()
            torch.cuda.synchronize()
            noimp = (noimp_ms, layer.profile_read())
        layer.profile(False)
        clk.window_end()
    total_ms = float(sum(step_ms))
    err = layer.get_error()
    if ws > 1:  # the slowest rank sets the time
        total_ms, burst_ms = shard.max_over_ranks([total_ms, burst_ms], device=dev)

    # ---- end to end through the public API with host buffers
    x_h = torch.from_numpy(np.ascontiguousarray(inp.x)).to(dt).pin_memory()
    small_h = {n: torch.from_numpy(np.ascontiguousarray(a, dtype=np.int32)).pin_memory()
               for n, a in (("q_pos", inp.q_pos), ("cu_q", inp.cu_seqlens_q), ("cu_k", inp.cu_seqlens_k),
                            ("lo", inp.cand_lo), ("hi", inp.cand_hi), ("kps", inp.topk))}
    out_h = torch.empty((T, H, d), dtype=dt).pin_memory()
    tr_h = torch.empty((B, K), dtype=torch.int32).pin_memory()
    h2d = x_h.numel() * x_h.element_size() + sum(t.numel() * 4 for t in small_h.values())
    d2h = out_h.numel() * out_h.element_size() + tr_h.numel() * 4

    def e2e_step():
        # fc_step_host: inputs copied in and outputs copied out every step on the
        # handle's copy streams, double-buffered against the kernels
        layer.step_host(x_h, small_h["q_pos"], small_h["cu_q"], small_h["cu_k"], kc, vc,
                        small_h["lo"], small_h["hi"], K, out_h, tr_h, k_per_seq=small_h["kps"])

    for _ in range(max(3, args.warmup)):
        e2e_step()
    layer.host_sync()
    torch.cuda.synchronize()
    if ws > 1:
        dist.barrier()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    t_host = time.perf_counter()
    for _ in range(args.steps):
        e2e_step()
    t_host = time.perf_counter() - t_host  # host time to enqueue the K steps
    layer.host_sync()  # the stream waits for the last output copies
    e1.record(stream)
    torch.cuda.synchronize()
    e2e_ms = e0.elapsed_time(e1)
    if ws > 1:
        e2e_ms = shard.max_over_ranks(e2e_ms, device=dev)

    result = None
    if rank == 0:
        result = _step_result(args, inp, ws, total_ms=total_ms, burst_ms=burst_ms,
                              e2e_host_ms=t_host * 1e3,
                              per_kernel=per_kernel, launches=launches, err=err, e2e_ms=e2e_ms,
                              h2d=h2d, d2h=d2h, clocks=clk.summary(), noimp=noimp,
                              num_sms=torch.cuda.get_device_properties(dev).multi_processor_count)
        result["qkv_plan"] = layer.qkv_plan(T)
        # the oracle's timing is a single-GPU line's context: rank 0 at N = 1 only
        result["cpu_baseline"] = (cpu_baseline(inp, budget_s=args.cpu_budget)
                                  if args.cpu_budget > 0 and ws == 1 else None)
    layer.close()
    if ws > 1:
        dist.barrier()
        dist.destroy_process_group()
    return result


def _oracle_threads():
    try:
        from threadpoolctl import threadpool_info

        n = [p.get("num_threads") for p in threadpool_info() if p.get("user_api") == "blas"]
        return int(max(n)) if n else os.cpu_count()
    except Exception:
        return os.cpu_count()


def _step_config(workload, inp, ws, importance=True):
    """The workload description both arms print (the same keys at every N)."""
    extra = {} if importance else {"importance": False}
    return {**extra, "workload": workload, "batch": inp.batch, "seq_len": int(np.diff(inp.cu_seqlens_k).max()),
            "query_rows_per_seq": int(np.diff(inp.cu_seqlens_q).max()), "hidden": inp.hidden,
            "heads": inp.n_heads, "head_dim": inp.head_dim, "topk": int(inp.topk.max()),
            "total_q": inp.total_q, "total_k": inp.total_k,
            "l2": "flushed between steps (256 MiB write)", "parallelism": f"sequence-sharded x{ws}"}


def cpu_baseline(inp, budget_s: float = 12.0):
    """Time the fp64 oracle, as it stands, on a bounded sample of sequences."""
    sys.path.insert(0, ROOT)
    import oracle

    done, tokens, t0 = 0, 0, time.perf_counter()
    while True:
        b = done % inp.batch
        qs, ks = inp.seq_slice_q(b), inp.seq_slice_k(b)
        r = oracle.step_sequence(inp.x[qs], inp.w_qkv, inp.q_pos[qs], inp.k_cache[ks], inp.v_cache[ks],
                                 inp.n_heads, inp.head_dim, inp.rope_theta, inp.dtype)
        imp = np.zeros(inp.total_k)
        imp[ks] = r["importance"]
        oracle.topk_tracked(imp, inp.cu_seqlens_k, inp.cand_lo, inp.cand_hi, inp.topk, int(inp.topk.max()))
        done += 1
        tokens += qs.stop - qs.start
        if time.perf_counter() - t0 >= budget_s:
            break
    el = time.perf_counter() - t0
    return {"value": tokens / el, "unit": UNIT, "cores": _oracle_threads(), "kind": "oracle",
            "sample": f"{done} sequence(s) of workload {inp.name} ({tokens} query rows), "
                      f"fp64 NumPy, {el:.1f} s wall"}


def run_reference(args):
    ws, rank, _ = _dist_env()
    if rank != 0:
        return None
    from kv_cache_attention_qkv_b200 import workloads
    import oracle

    inp = workloads.generate(args.workload)
    per_step = []
    tokens_total = 0

    def one(bidx):
        qs, ks = inp.seq_slice_q(bidx), inp.seq_slice_k(bidx)
        r = oracle.step_sequence(inp.x[qs], inp.w_qkv, inp.q_pos[qs], inp.k_cache[ks], inp.v_cache[ks],
                                 inp.n_heads, inp.head_dim, inp.rope_theta, inp.dtype)
        imp = np.zeros(inp.total_k)
        imp[ks] = r["importance"]
        oracle.topk_tracked(imp, inp.cu_seqlens_k, inp.cand_lo, inp.cand_hi, inp.topk, int(inp.topk.max()))
        return qs.stop - qs.start

    for k in range(args.warmup):
        one(k % inp.batch)
    for k in range(args.steps):
        t0 = time.perf_counter()
        tokens_total += one(k % inp.batch)
        per_step.append(time.perf_counter() - t0)
    el = sum(per_step)
    value = tokens_total / el
    return {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": ws,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": el / args.steps * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic",
        "config": _step_config(args.workload, inp, ws),
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": _oracle_threads(), "kind": "oracle",
                         "sample": f"{args.steps} sequence(s) of workload {args.workload}, one per step "
                                   "(each step times one sequence's query rows)"},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }


def run_model(args):
    """The LLaDA-8B-shaped model step (32 decoder layers around the Flash-Cache
    layer, LM head over the window rows, Flash-Verify confidence), both views
    (the [MASK] view, then the draft view) per step, then the reselection of
    the tracked positions from the draft view's importance summed over layers."""
    import torch

    from kv_cache_attention_qkv_b200 import FlashCacheModel, workloads
    from kv_cache_attention_qkv_b200.binding import load_library

    torch.cuda.set_device(0)
    dev = torch.device("cuda", 0)
    mi = workloads.generate_model("model_llada8b", device=dev)
    n = np.diff(mi.cu_seqlens_q)
    L = np.diff(mi.cu_seqlens_k)
    R, T, S, B = len(mi.head_rows), mi.total_q, mi.total_k, mi.batch
    K = int(mi.topk.max())
    model = FlashCacheModel(mi.layers, mi.final_norm, mi.lm_head, hidden=mi.hidden,
                            n_heads=mi.n_heads, head_dim=mi.head_dim, rope_theta=mi.rope_theta,
                            intermediate=mi.intermediate, max_batch=B, max_total_q=T,
                            max_total_k=S, max_seqlen_q=int(n.max()), max_pos=int(L.max()),
                            max_topk=K, max_head_rows=R)
    lib = load_library()
    i32 = lambda a: torch.from_numpy(np.ascontiguousarray(a, dtype=np.int32)).to(dev)
    qp, cq, ck, hr = i32(mi.q_pos), i32(mi.cu_seqlens_q), i32(mi.cu_seqlens_k), i32(mi.head_rows)
    lo, hi, kps = i32(mi.cand_lo), i32(mi.cand_hi), i32(mi.topk)
    imp = torch.empty((S,), device=dev)
    outs = {v: (torch.empty((R,), dtype=torch.int32, device=dev), torch.empty((R,), device=dev),
                torch.empty((R,), dtype=torch.uint8, device=dev)) for v in ("mask", "draft")}
    tracked = torch.empty((B, K), dtype=torch.int32, device=dev)
    layer_h = lib.fc_model_layer_handle(model._m)
    stream = torch.cuda.current_stream()

    def step():
        model.step(mi.x_mask, qp, cq, ck, mi.k_caches, mi.v_caches, head_rows=hr,
                   token=outs["mask"][0], confidence=outs["mask"][1], accept=outs["mask"][2])
        n1 = model.last_launch_count
        model.step(mi.x_draft, qp, cq, ck, mi.k_caches, mi.v_caches, head_rows=hr, importance=imp,
                   token=outs["draft"][0], confidence=outs["draft"][1], accept=outs["draft"][2])
        n2 = model.last_launch_count
        st = lib.fc_topk_tracked(layer_h, ctypes.c_void_p(stream.cuda_stream), B, S,
                                 ctypes.c_void_p(imp.data_ptr()), ctypes.c_void_p(ck.data_ptr()),
                                 ctypes.c_void_p(lo.data_ptr()), ctypes.c_void_p(hi.data_ptr()),
                                 ctypes.c_void_p(kps.data_ptr()), K,
                                 ctypes.c_void_p(tracked.data_ptr()))
        if st != 0:
            raise RuntimeError(f"fc_topk_tracked: {st}")
        return n1 + n2 + lib.fc_last_launch_count(layer_h)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    if model.get_error() != 0:
        raise RuntimeError("device error word set during warm-up")
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    launches = 0
    with ClockSampler(0) as clk:
        clk.window_start()
        e0.record(stream)
        for _ in range(args.steps):
            launches += step()
        e1.record(stream)
        torch.cuda.synchronize()
        clk.window_end()
    if model.get_error() != 0:
        raise RuntimeError("device error word set during the timed steps")
    ms = e0.elapsed_time(e1) / args.steps
    D, H, d, I, V, NL = mi.hidden, mi.n_heads, mi.head_dim, mi.intermediate, mi.vocab, mi.n_layers
    per_layer = (2.0 * T * D * 3 * H * d + 4.0 * H * d * float((n * L).sum()) + 2.0 * T * H * d * D
                 + 2.0 * T * D * 2 * I + 2.0 * T * I * D)
    flops = 2 * (NL * per_layer + 2.0 * R * D * V)  # two views
    peaks = _peaks()
    achieved = flops / (ms / 1e3) / 1e12
    model.close()
    return {
        "metric": "query-tokens/s per model step (32 layers, two Flash-Verify views)",
        "value": T / (ms / 1e3), "unit": UNIT, "n_gpus": 1, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic (random-init weights)",
        "config": {"workload": "model_llada8b", "layers": NL, "hidden": D, "heads": H,
                   "head_dim": d, "intermediate": I, "vocab": V, "batch": B, "seq_len": int(L.max()),
                   "query_rows_per_seq": int(n.max()), "head_rows": R, "views": 2,
                   "l2": "working set (weights 9 GB, caches 26 GB) far above L2"},
        "roofline": {"bound": "tensor", "achieved": achieved, "peak": peaks["bf16_tflops_sustained"],
                     "unit": "TFLOP/s", "frac": achieved / peaks["bf16_tflops_sustained"],
                     "flops_per_step": flops, "traffic": None,
                     "peak_source": f"{peaks['source']} (MEASURED_PEAKS.json sustained)"},
        "gpu_launches": launches,
        "clocks": clk.summary(),
    }


def run_decode(args):
    """Draft-and-verify decode iterations of the LLaDA-8B-shaped model: per
    iteration both views of the 32-layer model step, acceptance, window
    advance and reselection, all on the device.  Random weights never reach
    the 0.9 threshold, so each iteration decodes one token per sequence."""
    import torch

    from kv_cache_attention_qkv_b200 import FlashCacheModel, workloads

    torch.cuda.set_device(0)
    dev = torch.device("cuda", 0)
    mi = workloads.generate_model("model_llada8b", device=dev)
    B, K, W = mi.batch, 64, 64
    L = np.diff(mi.cu_seqlens_k)
    model = FlashCacheModel(mi.layers, mi.final_norm, mi.lm_head, hidden=mi.hidden,
                            n_heads=mi.n_heads, head_dim=mi.head_dim, rope_theta=mi.rope_theta,
                            intermediate=mi.intermediate, max_batch=B, max_total_q=B * (K + W),
                            max_total_k=mi.total_k, max_seqlen_q=K + W, max_pos=int(L.max()),
                            max_topk=K, max_head_rows=B * W)
    rng = np.random.default_rng(11)
    prompt = np.full(B, 1024, np.int64)  # 1024 prompt rows, 512 generated
    tokens = np.full(mi.total_k, -1, np.int32)
    tracked = np.zeros((B, K), np.int32)
    for b in range(B):
        k0 = mi.cu_seqlens_k[b]
        tokens[k0:k0 + prompt[b]] = rng.integers(0, mi.vocab - 1, size=prompt[b])
        tracked[b] = np.sort(rng.choice(prompt[b], size=K, replace=False))
    i32 = lambda a: torch.from_numpy(np.ascontiguousarray(a, dtype=np.int32)).to(dev)
    st = [i32(tokens), i32(np.full(mi.total_k, -1)), i32(tracked), i32(prompt), i32(np.zeros(B))]
    gen_end, cu_k = i32(L), i32(mi.cu_seqlens_k)
    stream = torch.cuda.current_stream()

    def iteration():
        model.decode_iteration(cu_k, mi.k_caches, mi.v_caches, mi.embed, mi.vocab - 1, st[2],
                               st[3], gen_end, st[0], st[1], st[4], W)
        return model.last_launch_count

    for _ in range(args.warmup):
        iteration()
    torch.cuda.synchronize()
    if model.get_error() != 0:
        raise RuntimeError("device error word set during warm-up")
    decided0 = int((st[0] >= 0).sum().item())
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    launches = 0
    with ClockSampler(0) as clk:
        clk.window_start()
        e0.record(stream)
        for _ in range(args.steps):
            launches += iteration()
        e1.record(stream)
        torch.cuda.synchronize()
        clk.window_end()
    if model.get_error() != 0:
        raise RuntimeError("device error word set during the timed iterations")
    decoded = int((st[0] >= 0).sum().item()) - decided0
    ms = e0.elapsed_time(e1) / args.steps
    model.close()
    return {
        "metric": "decoded tokens/s (draft-and-verify iterations, 32-layer model, both views)",
        "value": decoded / (ms * args.steps / 1e3), "unit": "tokens/s", "n_gpus": 1,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic (random-init weights: one token per sequence per iteration)",
        "config": {"workload": "model_llada8b", "batch": B, "tracked": K, "window": W,
                   "prompt": 1024, "seq_len": int(L.max()), "threshold": 0.9,
                   "decoded_tokens": decoded, "iterations": args.steps},
        "gpu_launches": launches, "clocks": clk.summary(),
    }


def _copy_rates(torch, nbytes, dev, reps=10):
    """GB/s of pinned host<->device copies of nbytes: each direction alone on
    its own stream, then both at once on two streams (CUDA events)."""
    h_in = torch.empty(nbytes, dtype=torch.uint8).pin_memory()
    h_out = torch.empty(nbytes, dtype=torch.uint8).pin_memory()
    d_in = torch.empty(nbytes, dtype=torch.uint8, device=dev)
    d_out = torch.empty(nbytes, dtype=torch.uint8, device=dev)
    s1, s2 = torch.cuda.Stream(), torch.cuda.Stream()
    res = {}
    for name, legs in (("h2d", [(s1, d_in, h_in)]), ("d2h", [(s2, h_out, d_out)]),
                       ("both", [(s1, d_in, h_in), (s2, h_out, d_out)])):
        for _ in range(2):
            for st, dst, src in legs:
                with torch.cuda.stream(st):
                    dst.copy_(src, non_blocking=True)
        torch.cuda.synchronize()
        evs = []
        for st, dst, src in legs:
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(st)
            with torch.cuda.stream(st):
                for _ in range(reps):
                    dst.copy_(src, non_blocking=True)
            b.record(st)
            evs.append((a, b))
        torch.cuda.synchronize()
        res[name] = [nbytes * reps / (a.elapsed_time(b) / 1e3) / 1e9 for a, b in evs]
    return {"h2d_gbs": res["h2d"][0], "d2h_gbs": res["d2h"][0],
            "both_h2d_gbs": res["both"][0], "both_d2h_gbs": res["both"][1], "bytes": nbytes}


def run_e2e_timeline(args):
    """Per-stage timeline of the end-to-end step (fc_step_host): the input
    copies and output copies on the handle's copy streams and the kernels on
    the compute stream, recorded with CUDA events for K steps after W warm-up
    steps, plus the bare copy rates of the same sizes."""
    import torch

    from kv_cache_attention_qkv_b200 import FlashCache, workloads

    torch.cuda.set_device(0)
    dev = torch.device("cuda", 0)
    inp = workloads.generate(args.workload)
    dt = torch.bfloat16 if inp.dtype == "bf16" else torch.float32
    f = lambda a: torch.from_numpy(np.ascontiguousarray(a)).to(dev, dtype=dt)
    w, kc, vc = f(inp.w_qkv), f(inp.k_cache), f(inp.v_cache)
    T, S, H, d, B = inp.total_q, inp.total_k, inp.n_heads, inp.head_dim, inp.batch
    K = int(inp.topk.max())
    layer = FlashCache(w, hidden=inp.hidden, n_heads=H, head_dim=d, rope_theta=inp.rope_theta,
                       max_batch=B, max_total_q=T, max_total_k=S,
                       max_seqlen_q=int(np.diff(inp.cu_seqlens_q).max()),
                       max_pos=int(np.diff(inp.cu_seqlens_k).max()), max_topk=K)
    x_h = torch.from_numpy(np.ascontiguousarray(inp.x)).to(dt).pin_memory()
    small_h = {n: torch.from_numpy(np.ascontiguousarray(a, dtype=np.int32)).pin_memory()
               for n, a in (("q_pos", inp.q_pos), ("cu_q", inp.cu_seqlens_q), ("cu_k", inp.cu_seqlens_k),
                            ("lo", inp.cand_lo), ("hi", inp.cand_hi), ("kps", inp.topk))}
    out_h = torch.empty((T, H, d), dtype=dt).pin_memory()
    tr_h = torch.empty((B, K), dtype=torch.int32).pin_memory()

    def e2e_step():
        layer.step_host(x_h, small_h["q_pos"], small_h["cu_q"], small_h["cu_k"], kc, vc,
                        small_h["lo"], small_h["hi"], K, out_h, tr_h, k_per_seq=small_h["kps"])

    for _ in range(args.warmup):
        e2e_step()
    layer.host_sync()
    torch.cuda.synchronize()
    if args.soak > 0:  # the steady state of a sustained load, as the main bench times it
        t0, n_ = time.perf_counter(), 0
        while time.perf_counter() - t0 < args.soak:
            e2e_step()
            n_ += 1
            if n_ % 16 == 0:
                layer.host_sync()
                torch.cuda.synchronize()
        layer.host_sync()
        torch.cuda.synchronize()
    # the same K steps timed as the main bench times them (no per-stage events)
    stream = torch.cuda.current_stream()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(args.steps):
        e2e_step()
    layer.host_sync()
    e1.record(stream)
    torch.cuda.synchronize()
    plain_ms = e0.elapsed_time(e1) / args.steps
    layer.profile(True)
    layer.profile_read()
    e0.record(stream)
    for _ in range(args.steps):
        e2e_step()
    layer.host_sync()
    e1.record(stream)
    torch.cuda.synchronize()
    profiled_ms = e0.elapsed_time(e1) / args.steps
    tl_ = layer.profile_timeline()
    layer.profile_read()
    layer.profile(False)
    layer.close()
    # group the records by step: every step has one h2d_copy record
    steps, cur = [], None
    for name, a, b in tl_:
        if name == "h2d_copy":
            cur = {"h2d": (a, b), "kernels": [], "d2h": None}
            steps.append(cur)
        elif name == "d2h_copy":
            cur["d2h"] = (a, b)
        else:
            cur["kernels"].append((a, b))
    mid = steps[2:-2] if len(steps) > 6 else steps
    mean = lambda xs: float(np.mean(xs)) if xs else None
    h2d = [s_["h2d"][1] - s_["h2d"][0] for s_ in mid]
    d2h = [s_["d2h"][1] - s_["d2h"][0] for s_ in mid]
    comp = [s_["kernels"][-1][1] - s_["kernels"][0][0] for s_ in mid]
    period = [b_["h2d"][0] - a_["h2d"][0] for a_, b_ in zip(mid, mid[1:])]
    # time each copy of step n overlaps the other direction's copies
    def overlap(a, others):
        return sum(max(0.0, min(a[1], o[1]) - max(a[0], o[0])) for o in others)
    ov = [overlap(s_["h2d"], [t_["d2h"] for t_ in steps]) / (s_["h2d"][1] - s_["h2d"][0]) for s_ in mid]
    h2d_bytes = x_h.numel() * x_h.element_size() + sum(t.numel() * 4 for t in small_h.values())
    d2h_bytes = out_h.numel() * out_h.element_size() + tr_h.numel() * 4
    rates = _copy_rates(torch, int(x_h.numel() * x_h.element_size()), dev)
    return {
        "metric": "end-to-end step timeline (fc_step_host)", "workload": args.workload,
        "steps": args.steps, "warmup": args.warmup, "soak_s": args.soak, "steps_analysed": len(mid),
        "ms_per_step_without_events": plain_ms, "ms_per_step_with_events": profiled_ms,
        "period_ms": mean(period), "h2d_copy_ms": mean(h2d), "d2h_copy_ms": mean(d2h),
        "kernels_ms": mean(comp), "h2d_bytes": int(h2d_bytes), "d2h_bytes": int(d2h_bytes),
        "h2d_gbs_in_step": h2d_bytes / (mean(h2d) / 1e3) / 1e9,
        "d2h_gbs_in_step": d2h_bytes / (mean(d2h) / 1e3) / 1e9,
        "h2d_overlapped_by_d2h": mean(ov), "bare_copy_rates": rates,
        "note": "per-kernel events on the compute stream stop the programmatic overlap of its "
                "kernels, so kernels_ms is a little above the step's device time",
    }


# Sweep axes (the pages' measured axes, throughput side): batch size at the
# headline query and cache, query size beta_m at batch 32, cache length at
# batch 32 and beta_m 128, and cache length at batch 1-4.
SWEEPS = {
    "batch": [f"sweep_b{b}_m128_L1536" for b in (1, 2, 4, 8, 16, 32, 64)],
    "beta": [f"sweep_b32_m{m}_L1536" for m in (64, 128, 192, 256)],
    "cache": [f"sweep_b32_m128_L{L}" for L in (768, 1536, 3072, 4096, 8192)],
    # small batches with long caches: the attention split over the SMs (B = 1, 2 from 1280 rows
    # on average; B = 4 has too many items to split)
    "small_batch_long_cache": [f"sweep_b{b}_m128_L{L}" for b, L in
                               ((1, 1536), (1, 2048), (1, 4096), (1, 8192), (2, 8192), (4, 8192))],
}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default="batch32_uniform")
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--cpu-budget", type=float, default=12.0,
                    help="seconds of oracle time for cpu_baseline (0 = skip)")
    ap.add_argument("--decode", action="store_true",
                    help="time draft-and-verify decode iterations of the model (one JSON line)")
    ap.add_argument("--model", action="store_true",
                    help="time the 32-layer model step around the layer (one JSON line)")
    ap.add_argument("--e2e-timeline", action="store_true",
                    help="per-stage timeline of the end-to-end (host-buffer) step (one JSON line)")
    ap.add_argument("--soak", type=float, default=0.0,
                    help="with --e2e-timeline: seconds of the same end-to-end steps first")
    ap.add_argument("--no-importance", action="store_true",
                    help="time fc_step without importance or reselection (the one-pass attention "
                         "kernel); for profiling, not the headline")
    ap.add_argument("--qkv-kernel", choices=["auto", "pair", "splitk"], default="auto",
                    help="projection kernel of the tensor-core path (default: the CTA-pair kernel)")
    ap.add_argument("--qkv-split", type=int, default=0,
                    help="cluster size of the split-K projection (default: the largest that fits at once)")
    ap.add_argument("--attn-split", choices=["auto", "never", "always"], default="auto",
                    help="small-batch attention split over the SMs (default: small batches "
                         "without importance or with caches of 1280 rows or more)")
    ap.add_argument("--sweep", choices=sorted(SWEEPS) + ["all"], default=None,
                    help="time every point of a sweep axis (one JSON line per point, no cpu_baseline)")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    if args.model:
        print(json.dumps(run_model(args)), flush=True)
        return
    if args.e2e_timeline:
        print(json.dumps(run_e2e_timeline(args)), flush=True)
        return
    if args.decode:
        print(json.dumps(run_decode(args)), flush=True)
        return
    if args.sweep is not None:
        if args.impl != "ours":
            ap.error("--sweep times this implementation only")
        axes = sorted(SWEEPS) if args.sweep == "all" else [args.sweep]
        for axis in axes:
            for point in SWEEPS[axis]:
                args.workload, args.cpu_budget = point, 0.0
                res = run_ours(args)
                if res is not None:
                    res["sweep"] = axis
                    print(json.dumps(res), flush=True)
        return
    res = run_reference(args) if args.impl == "reference" else run_ours(args)
    if res is not None:
        print(json.dumps(res), flush=True)


if __name__ == "__main__":
    main()
