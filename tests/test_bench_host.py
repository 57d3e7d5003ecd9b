"""Host logic of bench.py that needs no GPU: the clock record's load window,
the workload description shared by both arms, and the reference arm's JSON
line under torchrun (rank 0 prints it, the other ranks exit quietly)."""
import datetime
import json
import os
import socket
import subprocess
import sys
import time

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
import bench  # noqa: E402


def _write_samples(path, t_first, rows):
    with open(path, "w") as f:
        for i, (mhz, watts, cap) in enumerate(rows):
            ts = datetime.datetime.fromtimestamp(t_first + 0.1 * i).strftime("%Y/%m/%d %H:%M:%S.%f")[:-3]
            state = "Active" if cap else "Not Active"
            f.write(f"{ts}, 0, {mhz}, 1965, {watts}, 0x0, Not Active, Not Active, Not Active, {state}\n")


def _sampler(tmp_path, rows, window=None):
    c = bench.ClockSampler(0)
    c.proc = object()  # stands for a running nvidia-smi
    c.path = str(tmp_path / "clocks.csv")
    t_first = time.time()
    _write_samples(c.path, t_first, rows)
    if window is not None:
        c.t0, c.t1 = t_first + window[0], t_first + window[1]
    return c


def test_clock_summary_keeps_only_the_load_window(tmp_path):
    # idle at 1965 MHz, then 10 samples of load at 1600 MHz under the power cap, then idle
    rows = [(1965, 120.0, False)] * 5 + [(1600, 960.0, True)] * 10 + [(1965, 150.0, False)] * 5
    s = _sampler(tmp_path, rows, window=(0.45, 1.45)).summary()
    assert s["samples"] == 10 and s["sm_mhz"] == 1600.0 and s["reasons"] == ["sw_power_cap"]
    assert s["sm_max_mhz"] == 1965.0 and s["power_w_max"] == 960.0 and s["window_s"] == 1.0


def test_clock_summary_without_a_window_or_samples(tmp_path):
    rows = [(1965, 120.0, False)] * 3
    s = _sampler(tmp_path, rows).summary()
    assert s["samples"] == 3 and s["sm_mhz"] == 1965.0 and s["reasons"] == []
    # a window that no sample falls in: everything is summarised, and said so
    s = _sampler(tmp_path, rows, window=(100.0, 101.0)).summary()
    assert s["samples"] == 3 and "note" in s
    c = bench.ClockSampler(0)
    assert c.summary()["reasons"] == ["nvidia-smi unavailable"]


def test_both_arms_describe_the_workload_alike():
    from kv_cache_attention_qkv_b200 import workloads

    inp = workloads.generate("tiny_fp32")
    cfg = bench._step_config("tiny_fp32", inp, 2)
    assert cfg["workload"] == "tiny_fp32" and cfg["parallelism"] == "sequence-sharded x2"
    assert (cfg["batch"], cfg["total_q"], cfg["total_k"]) == (inp.batch, inp.total_q, inp.total_k)


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


@pytest.mark.timeout(300)
def test_reference_arm_under_torchrun_prints_one_line():
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node", "2",
           "--master-addr", "127.0.0.1", "--master-port", str(_free_port()), "bench.py",
           "--impl", "reference", "--gpus", "2", "--steps", "1", "--warmup", "3",
           "--workload", "tiny_fp32"]
    p = subprocess.run(cmd, cwd=ROOT, capture_output=True, text=True, timeout=280)
    assert p.returncode == 0, p.stderr[-2000:]
    lines = [json.loads(l) for l in p.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1
    line = lines[0]
    assert line["impl"] == "reference" and line["n_gpus"] == 2 and line["steps"] == 1
    assert line["config"] == bench._step_config("tiny_fp32", _tiny(), 2)
    assert line["cpu_baseline"]["kind"] == "oracle" and line["value"] > 0
    assert line["e2e"]["h2d_bytes_per_step"] == 0 and line["e2e"]["value"] == line["value"]


def _tiny():
    from kv_cache_attention_qkv_b200 import workloads

    return workloads.generate("tiny_fp32")


def test_step_result_line_follows_the_contract():
    """The JSON line a step run prints, from made-up measurements: every key of
    the contract, and the numbers derived from the timings as stated."""
    import argparse

    from kv_cache_attention_qkv_b200 import workloads

    inp = workloads.generate("tiny_fp32")
    args = argparse.Namespace(steps=10, warmup=3, workload="tiny_fp32")
    per_kernel = {"prep": (0.1, 10), "qkv_rope_scatter": (3.0, 10), "attention": (2.0, 10),
                  "importance_finalize": (0.05, 10), "topk": (0.1, 10)}
    clocks = {"sm_mhz": 1600.0, "sm_max_mhz": 1965.0, "reasons": ["sw_power_cap"]}
    r = bench._step_result(args, inp, 2, total_ms=5.0, burst_ms=4.0, per_kernel=per_kernel,
                           launches=50, err=0, e2e_ms=8.0, h2d=1000, d2h=2000, clocks=clocks)
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step",
                "higher_is_better", "scaling", "vs_baseline", "dtype", "data", "config", "roofline",
                "e2e", "gpu_launches", "clocks"):
        assert key in r, key
    T = inp.total_q
    assert r["value"] == pytest.approx(T * 2 * 10 / 5e-3)        # all ranks' tokens / max time
    assert r["ms_per_step"] == pytest.approx(0.5) and r["n_gpus"] == 2
    assert r["burst"]["value"] == pytest.approx(T * 2 * 10 / 4e-3)
    assert r["e2e"] == {"value": pytest.approx(T * 2 * 10 / 8e-3), "unit": r["unit"],
                        "h2d_bytes_per_step": 1000, "d2h_bytes_per_step": 2000}
    rl = r["roofline"]
    assert rl["kernel"] == "qkv_rope_scatter" and rl["bound"] == "tensor"  # the larger share
    wk = bench._work(inp)
    assert rl["achieved"] == pytest.approx(wk["qkv_flops"] / 0.3e-3 / 1e12)  # 0.3 ms per launch
    assert rl["frac"] == pytest.approx(rl["achieved"] / rl["peak"])
    assert rl["peak"] == bench._peaks()["bf16_tflops_sustained"]
    att = r["kernel_rooflines"]["attention"]
    assert att["unit"] == "GB/s" and att["achieved"] == pytest.approx(wk["attn_bytes"] / 0.2e-3 / 1e9)
    assert r["clocks"] is clocks and r["gpu_launches"] == 50 and r["higher_is_better"] is True
    # the step against every peak variant, reproducible from the peaks file and
    # the sampled clock
    pk = bench._peaks()
    st = r["step_roofline"]
    scaled = pk["bf16_tflops_sustained"] * 1600.0 / pk["sustained_mhz"]
    want = {"sustained": pk["bf16_tflops_sustained"], "burst": pk["bf16_tflops"],
            "spec": bench.SPEC_BF16_TFLOPS, "sustained_clock_scaled": scaled}
    for k, tf in want.items():
        bw = bench.SPEC_HBM_GBS if k == "spec" else pk["hbm_gbs"]
        t = max(wk["flops"] / (tf * 1e12), wk["bytes"] / (bw * 1e9))
        assert st["variants"][k]["frac"] == pytest.approx(t / 0.5e-3), k
    assert st["frac"] == st["variants"]["sustained"]["frac"]
    assert st["judged_on"] == "sustained_clock_scaled"
    assert rl["frac_vs"]["sustained_clock_scaled"] == pytest.approx(rl["achieved"] / scaled)
    assert rl["frac_vs"]["spec"] == pytest.approx(rl["achieved"] / bench.SPEC_BF16_TFLOPS)
    wb = r["work_balance"]
    assert wb["items"] == 2 and wb["tiles_max_per_cta"] == 1  # 2 heads x 1 query tile, 64 keys
    # the no-importance context line, from made-up per-kernel times
    noimp = (3.0, {"prep": (0.1, 10), "qkv_rope_scatter": (2.5, 10), "attention": (0.01, 10),
                   "attention_one_pass": (0.4, 10)})
    r2 = bench._step_result(args, inp, 2, total_ms=5.0, burst_ms=4.0, per_kernel=per_kernel,
                            launches=50, err=0, e2e_ms=8.0, h2d=1000, d2h=2000, clocks=clocks,
                            noimp=noimp, num_sms=148)
    ni = r2["no_importance"]
    assert ni["ms_per_step"] == pytest.approx(0.3)
    assert ni["attention_one_pass"]["achieved"] == pytest.approx(wk["attn_bytes"] / 0.04e-3 / 1e9)
    # a split small batch: its attention is the sum of its two launches
    pk3 = dict(per_kernel)
    pk3["attention_split_pass1"] = (0.5, 10)
    r3 = bench._step_result(args, inp, 2, total_ms=5.0, burst_ms=4.0, per_kernel=pk3,
                            launches=50, err=0, e2e_ms=8.0, h2d=1000, d2h=2000, clocks=clocks,
                            num_sms=148)
    att3 = r3["kernel_rooflines"]["attention"]
    assert att3["achieved"] == pytest.approx(wk["attn_bytes"] / ((2.0 + 0.5) / 10 * 1e-3) / 1e9)
