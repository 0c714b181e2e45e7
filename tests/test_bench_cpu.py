"""bench.py's reference arm (the oracle on the host cores) and its JSON contract, on CPU."""
import json
import os
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _lines(out: str):
    return [json.loads(line) for line in out.splitlines() if line.startswith("{")]


def test_reference_arm_json_line():
    r = subprocess.run([sys.executable, "bench.py", "--impl", "reference", "--workload", "c1", "--steps", "1",
                        "--warmup", "0", "--cpu-tokens", "8"], cwd=ROOT, capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = _lines(r.stdout)
    assert len(lines) == 1
    d = lines[0]
    assert d["impl"] == "reference" and d["unit"] == "TFLOP/s" and d["higher_is_better"] is True
    assert d["value"] > 0 and d["n_gpus"] == 1 and d["steps"] == 1
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["value"] == d["value"]
    assert d["e2e"] == {"value": d["value"], "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}
    assert "workload" in d["config"]


def test_reference_arm_prints_on_rank_zero_only():
    env = dict(os.environ, MASTER_ADDR="127.0.0.1")
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node", "2",
           "--master-addr", "127.0.0.1", "--master-port", "29611", "bench.py", "--impl", "reference", "--workload",
           "c1", "--gpus", "2", "--steps", "1", "--warmup", "0", "--cpu-tokens", "8"]
    r = subprocess.run(cmd, cwd=ROOT, capture_output=True, text=True, timeout=600, env=env)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = _lines(r.stdout)
    assert len(lines) == 1 and lines[0]["n_gpus"] == 2


def _bench():
    import importlib.util
    spec = importlib.util.spec_from_file_location("bench_mod", os.path.join(ROOT, "bench.py"))
    m = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(m)
    return m


def test_roofline_frac_is_against_burst_peak():
    b = _bench()
    from synth import CONFIGS
    cases = CONFIGS["c2"]
    peaks = {"bf16_tflops": 1600.0, "bf16_tflops_sustained": 1400.0}
    clk = {"sm_mhz": 1500.0, "sm_max_mhz": 1965.0, "reasons": ["sw_power_cap"]}
    fl = sum(sum(b.gemm_flops(c)) for c in cases)  # one step's GEMM flops
    g_ms = fl / 1.2e15 * 1e3  # GEMMs at 1200 TFLOP/s, split over fwd and bwd
    r = b.gemm_roofline(cases, False, 1, g_ms / 2, g_ms / 2, 6, 10.0, peaks, clk)
    assert abs(r["achieved"] - 1200.0) < 1e-6
    assert r["peak"] == 1600.0 and abs(r["frac"] - 0.75) < 1e-12  # power cap seen: still the burst peak
    assert abs(r["frac_of_sustained"] - 1200.0 / 1400.0) < 1e-12
    assert "achieved_at_max_clock" not in r
    assert abs(r["gemm_share_of_step"] - g_ms / 10.0) < 1e-12


def test_clock_summary_window_opens_to_warmup_when_short():
    b = _bench()
    s = b.ClockSampler("GPU-x")
    s.source = "nvml"
    s.marks = {"t_warm": 0.0, "t_start": 1.0, "t_end": 1.05}
    # 100 samples over the warm-up, 5 inside the timed region (too few on their own)
    s.samples = [(0.009 * i, 1900.0, 1965.0, 700.0, set()) for i in range(100)]
    s.samples += [(1.0 + 0.01 * i, 1500.0, 1965.0, 990.0, {"sw_power_cap"}) for i in range(5)]
    d = s.summary("t_start", "t_end", "t_warm")
    assert d["samples"] == 105 and d["samples"] >= b.MIN_CLOCK_SAMPLES
    assert "warm-up" in d["window"] and d["reasons"] == ["sw_power_cap"] and d["samples_power_capped"] == 5
    assert d["sm_mhz"] == 1900.0 and d["sm_min_mhz"] == 1500.0
    # enough samples in the timed region: that region alone
    s.samples += [(1.001 + 0.004 * i, 1700.0, 1965.0, 990.0, set()) for i in range(12)]
    d = s.summary("t_start", "t_end", "t_warm")
    assert d["window"] == "timed region" and d["samples"] == 17


def test_clock_summary_leaves_idle_gaps_out():
    b = _bench()
    s = b.ClockSampler("GPU-x")
    s.source = "nvml"
    s.marks = {"t_start": 0.0, "t_end": 3.0}
    # loaded samples at 1500 MHz, idle ones (between sweep cases) at the top clock
    s.samples = [(0.01 * i, 1500.0, 1965.0, 950.0, {"sw_power_cap"}) for i in range(100)]
    s.samples += [(1.0 + 0.01 * i, 1965.0, 1965.0, 120.0, set()) for i in range(150)]
    s.samples += [(2.5 + 0.01 * i, 1400.0, 1965.0, 990.0, {"sw_power_cap"}) for i in range(50)]
    s.idle_spans = [(0.995, 2.495)]
    d = s.summary("t_start", "t_end")
    assert d["samples"] == 150 and d["samples_power_capped"] == 150
    assert d["sm_mhz"] == 1500.0 and d["power_w_max"] == 990.0


def test_select_cases_filters_the_rank_sweep():
    b = _bench()
    from synth import CONFIGS
    c4 = CONFIGS["c4"]
    assert len(c4) == 48
    sel = b.select_cases(c4, "M=512,r=16,fmt=block4")
    assert {(c.K, c.N) for c in sel} == {(8192, 8192), (8192, 28672)} and len(sel) == 2
    assert len(b.select_cases(c4, "M=512,M=4096")) == 32
    assert len(b.select_cases(c4, "r=128,N=28672")) == 6
