"""Benchmark: fused LoRA-linear forward + hand-derived backward on B200.

One step = forward and backward of every projection of the workload (default: the
Llama-8B MLP projections gate, up and down at M = 16384 tokens, r = 16, bf16 weight),
with inputs resident in device memory.  Prints one JSON line (rank 0).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload c2|c1|c3|c4|c4s|qkv|mlp|ce] [--impl ours|reference]
    python bench.py --workload c4 [--select M=512,r=16,fmt=block4,N=28672]   (rank sweep, one line for the set)

Multi-GPU (one process per GPU under torch.distributed.run): data parallel over tokens,
every rank runs the full per-rank workload (weak scaling) and the adapter gradients dA
and dB, written in fp32, are summed across ranks with one NCCL all-reduce per step (the
layer's one exchange step) and rounded to bf16 once.
"""
from __future__ import annotations

import argparse
import datetime
import json
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "LoRA linear fwd+bwd TFLOP/s & tokens/s; % of B200 BF16 tensor peak"
FALLBACK_PEAKS = {"bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "hbm_gbs": 6650.0}
NOMINAL_BF16_TFLOPS = 2250.0  # B200 dense bf16 tensor peak, datasheet figure


def workload(name: str):
    from synth import CONFIGS, MlpCase
    if name == "mlp":
        blk = MlpCase("mlp_llama8b", 16384, 4096, 14336, 16, 32.0, "bf16", 7000)
        cases = [blk.gate_up_case(), blk.down_case()]
    elif name == "c4s":
        cases = [c for c in CONFIGS["c4"] if c.M == 512 and c.r == 16 and c.fmt == "bf16"]
    elif name == "c4":
        cases = list(CONFIGS["c4"])
    elif name == "ce":
        # the LM head as a projection: M tokens, K = D, N = V (no adapter; r only sizes nothing)
        from synth import LoraCase
        cases = [LoraCase("ce_llama3_head", 16384, 128256, 4096, 8, 16.0, "bf16", 7100)]
    else:
        cases = CONFIGS[name]
    desc = {
        "c1": "Llama-8B attention projection, M=8192, K=N=4096, r=16, alpha=32, bf16 weight",
        "c2": "Llama-8B MLP projections gate+up (K=4096,N=14336) and down (K=14336,N=4096), "
              "M=16384, r=16, alpha=32, bf16 weight",
        "c3": "QLoRA 4-bit blockwise weight K=4096 N=14336 (16-level codebook, fp16 absmax per 64), "
              "M=8192, r=16, alpha=32",
        "c4": "wide-model rank sweep: K=N=8192 and K=8192 N=28672, M in {512, 4096, 16384}, r in {8, 16, 64, 128}, "
              "alpha=2r, bf16 and 4-bit blockwise weights (each case timed on its own, L2 flushed before every step)",
        "c4s": "rank-sweep shapes at the smallest batch: M=512, K=N=8192 and K=8192 N=28672, r=16, alpha=32, "
               "bf16 weight (the most weight-heavy cases; L2 flushed before every step)",
        "ce": "cross-entropy over the Llama-3 LM head (V=128256, D=4096), M=16384 tokens, backward in "
              "16384-column vocabulary slices, bf16 head, no [M, V] logits",
        "mlp": "Llama-8B feed-forward block (D=4096, I=14336) with LoRA on gate, up and down and SwiGLU, "
               "M=16384, r=16, alpha=32, bf16 weights",
        "qkv": "Llama-8B attention q/k/v as one grouped layer (q 4096, k 1024, v 1024 rows, K=4096), "
               "M=8192, r=16 per projection, alpha=32, bf16 weight",
    }[name]
    return cases, desc


def select_cases(cases, spec: str):
    """Cases whose fields match every key of `spec` ("M=512,r=16,fmt=block4"); a key
    given more than once matches any of its values."""
    want: dict[str, set] = {}
    for item in spec.split(","):
        if not item.strip():
            continue
        k, _, v = item.partition("=")
        k, v = k.strip(), v.strip()
        if k not in ("M", "N", "K", "r", "fmt"):
            raise SystemExit(f"--select: unknown key {k!r} (M, N, K, r, fmt)")
        want.setdefault(k, set()).add(v if k == "fmt" else int(v))
    return [c for c in cases if all(getattr(c, k) in vs for k, vs in want.items())]


def ce_flops(c) -> float:
    """Cross-entropy step: logits in the forward and again in the backward, and dX:
    three M×V×D products, 6MVD."""
    return 6.0 * c.M * c.N * c.K


def case_flops(c) -> float:
    """Algorithmic FLOPs of one forward + backward: 4MNK + 6Mr(N+K) per projection
    (a grouped case sums this over its projections: 4MNK + 6Mr(N + G·K))."""
    return 4.0 * c.M * c.N * c.K + 6.0 * c.M * c.r * (c.N + c.G * c.K)


def case_bytes(c) -> float:
    """HBM floor of one forward + backward: the frozen weight read twice (bf16 2·NK·2,
    4-bit 2·(NK/2 + NK/32), 8-bit 2·(NK + 4N)) plus X, dY and XA read and Y, dX, dA, dB
    written once, 2·(3MK + 2MN) + 4Mr."""
    w = {"bf16": 2 * c.N * c.K, "block4": c.N * c.K / 2 + c.N * c.K / 32}.get(c.fmt, c.N * c.K + 4 * c.N)
    return 2.0 * w + 2.0 * (3 * c.M * c.K + 2 * c.M * c.N) + 4.0 * c.M * c.r


def gemm_flops(c) -> tuple[float, float]:
    """Algorithmic FLOPs of the Y GEMM (2MNK + 2MNr) and of the dX GEMM (2MNK + 2MK·Gr)."""
    return 2.0 * c.M * c.N * c.K + 2.0 * c.M * c.N * c.r, 2.0 * c.M * c.N * c.K + 2.0 * c.M * c.K * c.G * c.r


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def cpu_threads() -> int:
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads", 0) for i in threadpool_info() if i.get("user_api") == "blas"]
        if n:
            return int(max(n))
    except Exception:
        pass
    return os.cpu_count() or 1


# ---------------------------------------------------------------------------- clocks
REASON_NAMES = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")
MIN_CLOCK_SAMPLES = 10
CASE_GAP_S = 1.0  # idle time before each case of the rank sweep


class ClockSampler:
    """Samples the SM clock, its maximum, board power and the active clock-event
    (throttle) reasons while the benchmark runs: through NVML every 10 ms (read-only
    queries), else through `nvidia-smi -lms 100`.  Each sample is a tuple
    (time, sm_mhz, sm_max_mhz, power_w, set of reason names)."""

    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_id: str, index: int = 0, period_s: float = 0.01):
        self.gpu_id = gpu_id
        self.index = index
        self.period_s = period_s
        self.proc = None
        self.samples = []
        self.thread = None
        self.stop_ev = threading.Event()
        self.source = None
        self.marks = {}
        self.idle_spans = []

    def start(self):
        try:
            import pynvml
            pynvml.nvmlInit()
            try:
                h = pynvml.nvmlDeviceGetHandleByUUID(self.gpu_id)
            except Exception:
                h = pynvml.nvmlDeviceGetHandleByIndex(self.index)
            bits = {"hw_slowdown": pynvml.nvmlClocksEventReasonHwSlowdown,
                    "hw_thermal_slowdown": pynvml.nvmlClocksEventReasonHwThermalSlowdown,
                    "sw_thermal_slowdown": pynvml.nvmlClocksEventReasonSwThermalSlowdown,
                    "sw_power_cap": pynvml.nvmlClocksEventReasonSwPowerCap}
            self.source = "nvml"
            self.thread = threading.Thread(target=self._poll_nvml, args=(pynvml, h, bits), daemon=True)
            self.thread.start()
            return
        except Exception:
            pass
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", self.gpu_id, f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "100"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None
            return
        self.source = "nvidia-smi"
        self.thread = threading.Thread(target=self._read_smi, daemon=True)
        self.thread.start()

    def _poll_nvml(self, nv, h, bits):
        smax = float(nv.nvmlDeviceGetMaxClockInfo(h, nv.NVML_CLOCK_SM))
        while not self.stop_ev.is_set():
            try:
                sm = float(nv.nvmlDeviceGetClockInfo(h, nv.NVML_CLOCK_SM))
                pw = nv.nvmlDeviceGetPowerUsage(h) / 1000.0
                rb = nv.nvmlDeviceGetCurrentClocksEventReasons(h)
                self.samples.append((time.time(), sm, smax, pw, {n for n, b in bits.items() if rb & b}))
            except Exception:
                pass
            self.stop_ev.wait(self.period_s)

    def _read_smi(self):
        for line in self.proc.stdout:
            parts = [p.strip() for p in line.strip().split(",")]
            if len(parts) < 8:
                continue
            try:
                sm, smax = float(parts[0]), float(parts[1])
                pw = float(parts[2]) if parts[2] not in ("", "[N/A]") else 0.0
            except ValueError:
                continue
            reasons = {nm for nm, v in zip(REASON_NAMES, parts[4:8]) if v.lower() == "active"}
            self.samples.append((time.time(), sm, smax, pw, reasons))

    def mark(self, which: str):
        self.marks[which] = time.time()

    def idle(self, seconds: float):
        """Sleeps with the GPU idle; the summaries leave the samples of that time out."""
        t0 = time.time()
        time.sleep(seconds)
        self.idle_spans.append((t0, time.time()))

    def count_since(self, which: str) -> int:
        t0 = self.marks.get(which, 0.0)
        return sum(1 for s in list(self.samples) if s[0] >= t0)

    def stop(self):
        self.stop_ev.set()
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()
        if self.thread:
            self.thread.join(timeout=2)

    def summary(self, t0_mark: str, t1_mark: str, wide_mark: str | None = None):
        """Clock record of the region between two marks.  When that region holds fewer
        than MIN_CLOCK_SAMPLES samples, the window opens back to `wide_mark` (the start
        of the warm-up steps, which run the same work) and says so."""
        if not self.samples:
            return None
        t0, t1 = self.marks.get(t0_mark, 0.0), self.marks.get(t1_mark, float("inf"))

        def busy(s):
            return not any(a <= s[0] <= b for a, b in self.idle_spans)

        win = [s for s in self.samples if t0 <= s[0] <= t1 and busy(s)]
        window = "timed region"
        if len(win) < MIN_CLOCK_SAMPLES and wide_mark is not None:
            tw = self.marks.get(wide_mark, t0)
            win = [s for s in self.samples if tw <= s[0] <= t1 and busy(s)]
            window = "warm-up and timed region (the timed region alone held fewer than " \
                     f"{MIN_CLOCK_SAMPLES} samples)"
        if not win:
            win = self.samples[-MIN_CLOCK_SAMPLES:]
            window = "last samples before the end of the timed region"
        reasons = set().union(*(s[4] for s in win))
        capped = sum(1 for s in win if "sw_power_cap" in s[4])
        return {"sm_mhz": statistics.median(s[1] for s in win), "sm_max_mhz": max(s[2] for s in win),
                "sm_min_mhz": min(s[1] for s in win), "power_w_max": max(s[3] for s in win),
                "reasons": sorted(reasons), "samples": len(win), "samples_power_capped": capped,
                "window": window, "source": self.source,
                "period_ms": self.period_s * 1e3 if self.source == "nvml" else 100.0}


def gpu_uuid(dev) -> str:
    import torch
    try:
        return "GPU-" + str(torch.cuda.get_device_properties(dev).uuid)
    except Exception:
        return str(dev.index if hasattr(dev, "index") else 0)


# ---------------------------------------------------------------------------- oracle leg
def oracle_sample(cases, tokens: int, mlp: bool = False, ce: bool = False):
    """Runs the fp64 oracle (as it stands) on the first `tokens` tokens of every
    projection (of the feed-forward block when `mlp`, of the LM-head cross-entropy when
    `ce`); returns (seconds, algorithmic flops of the sample)."""
    import oracle as O
    from synth import make_case
    if ce:
        from synth import CeCase, make_ce_case
        c = cases[0].with_M(tokens)
        inp = make_ce_case(CeCase(c.name, tokens, c.K, c.N, c.seed))
        t0 = time.perf_counter()
        O.cross_entropy_rows_bits(inp["X"], inp["W"], inp["labels"], -100, inp["dloss"])
        return time.perf_counter() - t0, ce_flops(c)
    if mlp:
        gu_c, dn_c = (c.with_M(tokens) for c in cases)
        gu = make_case(gu_c, want=("X", "W", "A", "B"))
        dn = make_case(dn_c, want=("W", "A", "B", "dY"))
        t0 = time.perf_counter()
        args = (O.bf16_to_f64(gu["X"]), O.weight_f64(gu), O.bf16_to_f64(gu["A"]), O.bf16_to_f64(gu["B"]),
                O.weight_f64(dn), O.bf16_to_f64(dn["A"]), O.bf16_to_f64(dn["B"]))
        O.lora_mlp_backward(O.bf16_to_f64(dn["dY"]), *args, gu_c.s)  # runs the forward too
        return time.perf_counter() - t0, case_flops(gu_c) + case_flops(dn_c)
    inputs = [make_case(c.with_M(tokens)) for c in cases]
    t0 = time.perf_counter()
    flops = 0.0
    for inp in inputs:
        c = inp["case"]
        W = O.weight_f64(inp)
        X, A, B, dY = (O.bf16_to_f64(inp[k]) for k in ("X", "A", "B", "dY"))
        if c.rows is None:
            O.lora_forward(X, W, A, B, c.s)
            O.lora_backward(dY, X, W, A, B, c.s)
        else:
            offs = [0]
            for n in c.rows:
                offs.append(offs[-1] + n)
            Ws = [W[offs[g]:offs[g + 1]] for g in range(c.G)]
            As = [A[g * c.r:(g + 1) * c.r] for g in range(c.G)]
            Bs = [B[offs[g]:offs[g + 1]] for g in range(c.G)]
            O.lora_grouped_forward(X, Ws, As, Bs, c.s)
            O.lora_grouped_backward(dY, X, Ws, As, Bs, c.s)
        flops += case_flops(c)
    return time.perf_counter() - t0, flops


def run_reference(args, cases, desc, rank, world):
    if rank != 0:
        return 0
    tokens = args.cpu_tokens
    for _ in range(args.warmup):
        oracle_sample(cases, tokens, mlp=args.workload == "mlp", ce=args.workload == "ce")
    times, flops = [], 0.0
    for _ in range(args.steps):
        t, flops = oracle_sample(cases, tokens, mlp=args.workload == "mlp", ce=args.workload == "ce")
        times.append(t)
    total = sum(times)
    val = args.steps * flops / total / 1e12
    sample = f"first {tokens} tokens of each projection per step (full K and N), fp64 numpy oracle"
    line = {
        "impl": "reference", "metric": METRIC, "value": val, "unit": "TFLOP/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * total / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": desc, "tokens_per_step": tokens, "projections": [c.name for c in cases]},
        "tokens_per_s": args.steps * tokens / total,
        "cpu_baseline": {"value": val, "unit": "TFLOP/s", "cores": cpu_threads(), "kind": "oracle", "sample": sample},
        "e2e": {"value": val, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


# ---------------------------------------------------------------------------- our leg
def traffic_record():
    p = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(p):
        return None
    try:
        with open(p) as f:
            return json.load(f)
    except Exception:
        return None


def source_hash() -> str:
    """Hash of the sources the bf16 GEMM (the kernel of the traffic record) and its launch
    are built from; the record counts only while they are unchanged."""
    import hashlib
    h = hashlib.sha256()
    for f in ("gemm_common.cuh", "gemm_pair.cuh", "ptx.cuh", "lora_api.cu"):
        with open(os.path.join(ROOT, "qlora_linear_b200", "csrc", f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def make_weight_dev(q, c, d):
    """LoraWeight over the device-drawn arrays of case c."""
    if c.fmt == "bf16":
        return q.LoraWeight(c.N, c.K, d["W"])
    if c.fmt == "block4":
        return q.LoraWeight(c.N, c.K, d["codes"], d["absmax"], d["codebook"])
    fmt = q.LORA_W_INT8 if c.fmt == "int8" else q.LORA_W_FP8_E4M3
    return q.LoraWeight(c.N, c.K, d["codes"], d["row_scale"], None, fmt)


class LinearSet:
    """The projections of a layer workload with their resident inputs and outputs."""

    def __init__(self, cases, dev, rank, world):
        import torch

        import qlora_linear_b200 as q
        from synth.device import make_case_device

        self.cases, self.world = cases, world
        self.layers, self.data = [], []
        x_cache = {}
        for c in cases:
            want = ["W", "A", "B", "dY"]
            xkey = c.x_seed if c.x_seed is not None else (c.data_seed if c.data_seed is not None else c.seed)
            xkey = (xkey, c.M, c.K)
            if xkey not in x_cache:
                want.append("X")
            d = make_case_device(c, dev, rank=rank, want=tuple(want))
            if "X" in d:
                x_cache[xkey] = d["X"]
            d["X"] = x_cache[xkey]
            W = make_weight_dev(q, c, d)
            if c.rows is None:
                layer = q.LoraLinear(W, d["A"], d["B"], c.alpha)
            else:
                layer = q.LoraGroupedLinear(W, c.rows, d["A"], d["B"], c.alpha)
            layer.workspace(c.M)
            out = {
                "Y": torch.empty((c.M, c.N), dtype=torch.bfloat16, device=dev),
                "XA": torch.empty((c.M, c.G * c.r), dtype=torch.bfloat16, device=dev),
                "dX": torch.empty((c.M, c.K), dtype=torch.bfloat16, device=dev),
                "dA": torch.empty((c.G * c.r, c.K), dtype=torch.bfloat16, device=dev),
                "dB": torch.empty((c.N, c.r), dtype=torch.bfloat16, device=dev),
            }
            self.layers.append(layer)
            self.data.append((d, out))
        # data parallel: every projection's fp32 adapter gradients in one exchange buffer,
        # summed over ranks by one all-reduce per step and rounded to bf16 once
        self.exchange = None
        if world > 1:
            shapes = [s for _, o in self.data for s in (o["dA"].shape, o["dB"].shape)]
            self.exchange = q.AdapterGradExchange(shapes, dev)

    def step(self, inputs=None):
        for i, (layer, (d, o)) in enumerate(zip(self.layers, self.data)):
            X = d["X"] if inputs is None else inputs[i]["X"]
            dY = d["dY"] if inputs is None else inputs[i]["dY"]
            layer.forward(X, Y=o["Y"], XA=o["XA"])
            if self.exchange is None:
                layer.backward(dY, X, o["XA"], out=(o["dX"], o["dA"], o["dB"]))
            else:
                v = self.exchange.views
                layer.backward(dY, X, o["XA"], out=(o["dX"], v[2 * i], v[2 * i + 1]), grads_f32=True)
        if self.exchange is not None:
            self.exchange.allreduce()
            self.exchange.round_into([t for _, o in self.data for t in (o["dA"], o["dB"])])

    def statuses(self):
        import qlora_linear_b200 as q
        return [q.lora_device_status(layer.workspace(c.M)) for layer, c in zip(self.layers, self.cases)]


class MlpSet:
    """The feed-forward block workload: one LoraMLP (cases = its gate/up and down
    projections, for the FLOP count) with resident inputs, saved tensors and outputs."""

    def __init__(self, cases, dev, rank, world):
        import torch

        import qlora_linear_b200 as q
        from synth.device import make_case_device

        gu_c, dn_c = cases
        self.cases, self.world, self.dev = cases, world, dev
        self.M, self.D, self.I, self.r = gu_c.M, gu_c.K, dn_c.K, gu_c.r
        gu = make_case_device(gu_c, dev, rank=rank, want=("X", "W", "A", "B"))
        dn = make_case_device(dn_c, dev, rank=rank, want=("W", "A", "B", "dY"))

        self.mlp = q.LoraMLP(make_weight_dev(q, gu_c, gu), make_weight_dev(q, dn_c, dn), gu["A"], gu["B"], dn["A"], dn["B"], gu_c.alpha)
        self.inputs = {"X": gu["X"], "dZ": dn["dY"], "gu": gu, "dn": dn}
        self.mlp.workspace(self.M)
        bf = torch.bfloat16
        self.saved = self.mlp.alloc_saved(self.M, dev)
        self.Z = torch.empty((self.M, self.D), dtype=bf, device=dev)
        self.grads = (torch.empty((self.M, self.D), dtype=bf, device=dev),
                      torch.empty((2 * self.r, self.D), dtype=bf, device=dev),
                      torch.empty((2 * self.I, self.r), dtype=bf, device=dev),
                      torch.empty((self.r, self.I), dtype=bf, device=dev),
                      torch.empty((self.D, self.r), dtype=bf, device=dev))
        self.layers = [self.mlp]
        self.data = []
        self.exchange = q.AdapterGradExchange([g.shape for g in self.grads[1:]], dev) if world > 1 else None

    def step(self, inputs=None):
        X = self.inputs["X"] if inputs is None else inputs["X"]
        dZ = self.inputs["dZ"] if inputs is None else inputs["dZ"]
        self.mlp.forward(X, Z=self.Z, saved=self.saved)
        if self.exchange is None:
            self.mlp.backward(dZ, X, self.saved, out=self.grads)
        else:
            self.mlp.backward(dZ, X, self.saved, out=(self.grads[0], *self.exchange.views), grads_f32=True)
            self.exchange.allreduce()
            self.exchange.round_into(list(self.grads[1:]))

    def statuses(self):
        import qlora_linear_b200 as q
        return [q.lora_device_status(self.mlp.workspace(self.M))]

    def e2e(self, args, step):
        """End to end with host buffers: X, dZ and the four adapters in and the step's result,
        the four adapter gradients, out every step (Z and dX are activations a model keeps on
        the device); the frozen weights stay resident."""
        import torch
        import torch.distributed as dist

        stream = torch.cuda.current_stream()
        m = self.mlp
        h_in = {k: t.cpu().pin_memory() for k, t in (("X", self.inputs["X"]), ("dZ", self.inputs["dZ"]),
                                                       ("A_gate_up", m.A_gate_up), ("B_gate_up", m.B_gate_up),
                                                       ("A_down", m.A_down), ("B_down", m.B_down))}
        d_in = {"X": torch.empty_like(self.inputs["X"]), "dZ": torch.empty_like(self.inputs["dZ"])}
        outs = tuple(self.grads[1:])  # dA_gate_up, dB_gate_up, dA_down, dB_down (not dX)
        h_out = [torch.empty(t.shape, dtype=t.dtype).pin_memory() for t in outs]
        h2d = sum(t.numel() * 2 for t in h_in.values())
        d2h = sum(t.numel() * 2 for t in h_out)

        def e2e_step():
            d_in["X"].copy_(h_in["X"], non_blocking=True)
            d_in["dZ"].copy_(h_in["dZ"], non_blocking=True)
            for k in ("A_gate_up", "B_gate_up", "A_down", "B_down"):
                getattr(m, k).copy_(h_in[k], non_blocking=True)
            step(inputs=d_in)
            for h, t in zip(h_out, outs):
                h.copy_(t, non_blocking=True)

        for _ in range(2):
            e2e_step()
        torch.cuda.synchronize()
        steps = max(3, args.steps // 2)
        if self.world > 1:
            dist.barrier()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(steps):
            e2e_step()
        e1.record(stream)
        torch.cuda.synchronize()
        ms = e0.elapsed_time(e1) / steps
        if self.world > 1:
            t = torch.tensor([ms], device=self.dev, dtype=torch.float64)
            dist.all_reduce(t, op=dist.ReduceOp.MAX)
            ms = float(t.item())
        flops_step = sum(case_flops(c) for c in self.cases)
        return {"value": self.world * flops_step / (ms * 1e-3) / 1e12, "unit": "TFLOP/s", "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h, "ms_per_step": ms, "steps": steps,
                "note": "X, dZ and the four adapters copied from pinned host memory and the four adapter gradients "
                        "read back every step; the frozen weights stay resident"}


class CeSet:
    """The cross-entropy workload: hidden states, head, labels and dloss resident."""

    def __init__(self, cases, dev, rank, world):
        import torch

        import qlora_linear_b200 as q

        c = cases[0]
        self.cases, self.world, self.dev = cases, world, dev
        self.M, self.D, self.V = c.M, c.K, c.N
        g = torch.Generator(device=dev)
        g.manual_seed(c.seed * 1_000_003 + rank)
        self.X = torch.randn((self.M, self.D), generator=g, device=dev).to(torch.bfloat16)
        self.Wt = (torch.randn((self.V, self.D), generator=g, device=dev) * (2.0 / self.D ** 0.5)).to(torch.bfloat16)
        self.labels = torch.randint(0, self.V, (self.M,), generator=g, device=dev, dtype=torch.int32)
        self.labels[torch.rand(self.M, generator=g, device=dev) < 0.05] = -100
        self.dloss = torch.full((self.M,), 1.0 / self.M, device=dev)
        self.ce = q.LoraCrossEntropy(q.LoraWeight(self.V, self.D, self.Wt), -100, 16384)
        self.ce.workspace(self.M)
        self.dX = torch.empty((self.M, self.D), dtype=torch.bfloat16, device=dev)
        self.layers, self.data = [self.ce], []

    def step(self, inputs=None):
        X = self.X if inputs is None else inputs["X"]
        loss, lse = self.ce.forward(X, self.labels)
        self.loss = loss
        self.ce.backward(X, self.labels, lse, self.dloss, dX=self.dX)

    def statuses(self):
        import qlora_linear_b200 as q
        return [q.lora_device_status(self.ce.workspace(self.M))]

    def e2e(self, args, step):
        """X in from pinned host memory and the per-row losses (the step's result) out, every step."""
        import torch

        stream = torch.cuda.current_stream()
        hX = self.X.cpu().pin_memory()
        dXin = torch.empty_like(self.X)
        hloss = torch.empty(self.M, dtype=torch.float32).pin_memory()

        def e2e_step():
            dXin.copy_(hX, non_blocking=True)
            step(inputs={"X": dXin})
            hloss.copy_(self.loss, non_blocking=True)

        for _ in range(2):
            e2e_step()
        torch.cuda.synchronize()
        steps = max(3, args.steps // 2)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(steps):
            e2e_step()
        e1.record(stream)
        torch.cuda.synchronize()
        ms = e0.elapsed_time(e1) / steps
        return {"value": self.world * ce_flops(self.cases[0]) / (ms * 1e-3) / 1e12, "unit": "TFLOP/s",
                "h2d_bytes_per_step": hX.numel() * 2, "d2h_bytes_per_step": hloss.numel() * 4,
                "ms_per_step": ms, "steps": steps,
                "note": "X copied from pinned host memory and the step's result, the per-row losses, read back "
                        "every step (dX stays on the device for the layers below); head, labels and dloss resident"}


def time_separate_ce(args, cases, ws, dev):
    """The same loss the plain way: full [M, V] logits by torch.matmul, torch's
    cross_entropy in fp32 and autograd for dX; reports its time and peak memory."""
    import torch

    stream = torch.cuda.current_stream()
    X = ws.X.clone().requires_grad_(True)
    labels = ws.labels.long()

    def step():
        X.grad = None
        logits = X @ ws.Wt.T
        loss = torch.nn.functional.cross_entropy(logits.float(), labels, ignore_index=-100, reduction="none")
        (loss * ws.dloss).sum().backward()

    for _ in range(max(1, args.warmup)):
        step()
    torch.cuda.synchronize()
    torch.cuda.reset_peak_memory_stats(dev)
    base = torch.cuda.memory_allocated(dev)
    steps = max(3, args.steps // 4)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(steps):
        step()
    e1.record(stream)
    torch.cuda.synchronize()
    ms = e0.elapsed_time(e1) / steps
    peak = torch.cuda.max_memory_allocated(dev) - base
    return {"ms_per_step": ms, "value": ce_flops(cases[0]) / (ms * 1e-3) / 1e12, "unit": "TFLOP/s",
            "extra_peak_bytes": int(peak),
            "note": "full logits (torch.matmul, bf16), fp32 cross_entropy and autograd; extra_peak_bytes is the "
                    "memory above the resident inputs"}


def time_separate_mlp(args, cases, ws, dev):
    """The same block unfused: gate, up and down as three separate layers, SwiGLU and its
    derivative as torch elementwise ops between them (what a model without the fused
    block runs)."""
    import torch

    import qlora_linear_b200 as q

    stream = torch.cuda.current_stream()
    m, M, D, I, r = ws.mlp, ws.M, ws.D, ws.I, ws.r
    gu = ws.inputs["gu"]
    bf = torch.bfloat16
    Wg = q.LoraWeight(I, D, m.gate_up.data[:I]) if m.gate_up.fmt == q.LORA_W_BF16 else None
    if Wg is None:
        return None
    Wu = q.LoraWeight(I, D, m.gate_up.data[I:])
    gate = q.LoraLinear(Wg, m.A_gate_up[:r], m.B_gate_up[:I], r * m.s)
    up = q.LoraLinear(Wu, m.A_gate_up[r:], m.B_gate_up[I:], r * m.s)
    down = q.LoraLinear(m.down, m.A_down, m.B_down, r * m.s)
    for L in (gate, up, down):
        L.workspace(M)
    X, dZ = gu["X"], ws.inputs["dZ"]
    G, U, H = (torch.empty((M, I), dtype=bf, device=dev) for _ in range(3))
    XAg, XAu, XAd = (torch.empty((M, r), dtype=bf, device=dev) for _ in range(3))
    Z = torch.empty((M, D), dtype=bf, device=dev)
    dH = torch.empty((M, I), dtype=bf, device=dev)
    gbufs = [(torch.empty((M, D), dtype=bf, device=dev), torch.empty((r, D), dtype=bf, device=dev),
              torch.empty((I, r), dtype=bf, device=dev)) for _ in range(2)]
    dgd = (dH, torch.empty((r, I), dtype=bf, device=dev), torch.empty((D, r), dtype=bf, device=dev))

    def step():
        gate.forward(X, Y=G, XA=XAg)
        up.forward(X, Y=U, XA=XAu)
        g32 = G.float()
        H.copy_(g32 * torch.sigmoid(g32) * U.float())
        down.forward(H, Y=Z, XA=XAd)
        down.backward(dZ, H, XAd, out=dgd)
        g32, u32, dh32 = G.float(), U.float(), dH.float()
        sg = torch.sigmoid(g32)
        dG = (dh32 * u32 * sg * (1 + g32 * (1 - sg))).to(bf)
        dU = (dh32 * g32 * sg).to(bf)
        gate.backward(dG, X, XAg, out=gbufs[0])
        up.backward(dU, X, XAu, out=gbufs[1])
        gbufs[0][0].add_(gbufs[1][0])

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(args.steps):
        step()
    e1.record(stream)
    torch.cuda.synchronize()
    ms = e0.elapsed_time(e1) / args.steps
    flops_step = sum(case_flops(c) for c in cases)
    return {"ms_per_step": ms, "value": flops_step / (ms * 1e-3) / 1e12, "unit": "TFLOP/s",
            "note": "gate, up, down as three separate layers of this library, SwiGLU forward and backward as "
                    "torch elementwise ops in fp32, dX of gate and up summed by torch"}


def gemm_roofline(cases, ce, steps, fwd_ms, bwd_ms, g_launches, step_ms, peaks, clk):
    """Roofline of the dominant kernel, the tcgen05 GEMM (its Y and dX launches):
    algorithmic FLOPs of those launches over their summed CUDA-event time, against the
    measured dense bf16 peak.  `frac` is always against the burst peak (the GEMM is timed
    inside a region of well under a minute); the fraction of the sustained peak is reported
    beside it.  (No clock-scaled figure: the median of sampled SM clocks misses the power
    limiter's short slowdowns, and scaling by it overstates the rate at the top clock.)"""
    gflops = (ce_flops(cases[0]) if ce else sum(sum(gemm_flops(c)) for c in cases)) * steps
    g_ms = fwd_ms + bwd_ms
    achieved = gflops / (g_ms * 1e-3) / 1e12 if g_ms > 0 else None
    peak_burst = peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"])
    peak_sust = peaks.get("bf16_tflops_sustained", FALLBACK_PEAKS["bf16_tflops_sustained"])
    return {
        "bound": "tensor", "achieved": achieved, "peak": peak_burst, "unit": "TFLOP/s",
        "frac": achieved / peak_burst if achieved else None,
        "peak_source": "bf16_tflops (burst) of MEASURED_PEAKS.json" if "bf16_tflops" in peaks
                       else "fallback burst figure",
        "frac_of_sustained": achieved / peak_sust if achieved else None,
        "launches": g_launches, "avg_launch_ms": g_ms / g_launches if g_launches else None,
        "gemm_share_of_step": g_ms / (step_ms * steps) if step_ms > 0 else None,
    }


def time_steps(q, torch, step, steps, stream, flush_buf=None):
    """Runs `steps` steps between two CUDA events on `stream` and returns (ms per step,
    GEMM fwd ms, GEMM bwd ms, GEMM launches, library launches).  With `flush_buf`, a
    buffer larger than L2 is rewritten before every step, outside that step's events."""
    q.lora_timing_enable(True)
    q.lora_timing_read(q.LORA_KERNEL_FWD_GEMM)
    q.lora_timing_read(q.LORA_KERNEL_BWD_GEMM)
    launches0 = q.lora_launch_count()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
    e0.record(stream)
    for i in range(steps):
        if flush_buf is not None:
            flush_buf.fill_(i & 0xFF)
            ev[i][0].record(stream)
        step()
        if flush_buf is not None:
            ev[i][1].record(stream)
    e1.record(stream)
    torch.cuda.synchronize()
    launches = q.lora_launch_count() - launches0
    q.lora_timing_enable(False)
    fwd_ms, fwd_n = q.lora_timing_read(q.LORA_KERNEL_FWD_GEMM)
    bwd_ms, bwd_n = q.lora_timing_read(q.LORA_KERNEL_BWD_GEMM)
    ms = (sum(a.elapsed_time(b) for a, b in ev) if flush_buf is not None else e0.elapsed_time(e1)) / steps
    return ms, fwd_ms, bwd_ms, fwd_n + bwd_n, launches


def run_sweep(args, cases, desc, rank, world, local_rank):
    """The rank sweep (one projection per case): each case is built, warmed up and timed
    on its own (forward + backward per step, L2 flushed before every step, outside the
    step's events), then freed.  Each case starts after the GPU has been idle for
    CASE_GAP_S, so a small case does not inherit the clock the power limiter holds after a
    large one (measured: the 512-token 4-bit cases ran at half speed right after the
    16384-token cases, and at full speed on their own).  The line's value is the
    algorithmic FLOPs of one pass over every selected case divided by the sum of their
    per-step times; `sweep` lists each case."""
    import torch
    import torch.distributed as dist

    import qlora_linear_b200 as q

    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    stream = torch.cuda.current_stream()
    peaks, peak_src = load_peaks()
    hbm = peaks.get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"])
    flush_buf = torch.empty(512 << 20, dtype=torch.uint8, device=dev)
    clocks = ClockSampler(gpu_uuid(dev), local_rank)
    clocks.start()
    rows, tot_ms, tot_flops, tot_launches = [], 0.0, 0.0, 0
    g_ms_all, g_fl_all = 0.0, 0.0
    clocks.mark("t_warm")
    clocks.mark("t_start")
    for c in cases:
        torch.cuda.synchronize()
        clocks.idle(CASE_GAP_S)
        ws = LinearSet([c], dev, rank, world)
        for _ in range(args.warmup):
            ws.step()
        torch.cuda.synchronize()
        if world > 1:
            dist.barrier()
        ms, fwd_ms, bwd_ms, g_n, launches = time_steps(q, torch, ws.step, args.steps, stream, flush_buf)
        if world > 1:
            t = torch.tensor([ms], device=dev, dtype=torch.float64)
            dist.all_reduce(t, op=dist.ReduceOp.MAX)
            ms = float(t.item())
        for st in ws.statuses():
            if st != q.LORA_OK:
                raise RuntimeError(f"device status after {c.name}: " + q.status_string(st))
        fl = case_flops(c)
        gfl = sum(gemm_flops(c)) * args.steps
        g_ms = fwd_ms + bwd_ms
        rows.append({
            "case": c.name, "M": c.M, "N": c.N, "K": c.K, "r": c.r, "fmt": c.fmt, "ms_per_step": ms,
            "tflops": fl / (ms * 1e-3) / 1e12, "frac_of_burst": fl / (ms * 1e-3) / 1e12 / peaks.get(
                "bf16_tflops", FALLBACK_PEAKS["bf16_tflops"]),
            "tokens_per_s": c.M / (ms * 1e-3),
            "gemm_tflops": gfl / (g_ms * 1e-3) / 1e12 if g_ms > 0 else None,
            "gemm_share": g_ms / (ms * args.steps) if ms > 0 else None,
            "rank_r_passes_share": 1.0 - g_ms / (ms * args.steps) if ms > 0 else None,
            "hbm_floor_gbs": case_bytes(c) / (ms * 1e-3) / 1e9,
            "hbm_floor_frac": case_bytes(c) / (ms * 1e-3) / 1e9 / hbm,
            "launches_per_step": launches / args.steps,
        })
        tot_ms += ms
        tot_flops += fl
        tot_launches += launches
        g_ms_all += g_ms
        g_fl_all += gfl
        del ws
        torch.cuda.empty_cache()
    clocks.mark("t_end")
    clocks.stop()
    clk = clocks.summary("t_start", "t_end", "t_warm")
    achieved = g_fl_all / (g_ms_all * 1e-3) / 1e12 if g_ms_all > 0 else None
    peak_burst = peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"])
    if rank == 0:
        line = {
            "metric": METRIC, "value": world * tot_flops / (tot_ms * 1e-3) / 1e12, "unit": "TFLOP/s",
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup, "ms_per_step": tot_ms,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic (seeded, drawn on device)",
            "config": {"workload": desc, "cases": len(cases), "parallelism": f"dp{world}",
                       "l2": "L2 flushed (512 MB written) before every timed step, outside its events",
                       "step": "one forward + backward of every selected case, each timed on its own"},
            "tokens_per_s": world * sum(c.M for c in cases) / (tot_ms * 1e-3),
            "roofline": {"bound": "tensor", "achieved": achieved, "peak": peak_burst, "unit": "TFLOP/s",
                         "frac": achieved / peak_burst if achieved else None, "traffic": None,
                         "peak_source": f"{peak_src} bf16 dense, burst"},
            "cpu_baseline": None, "e2e": None, "gpu_launches": tot_launches, "clocks": clk,
            "sweep": rows,
        }
        print(json.dumps(line), flush=True)


def run_ours(args, cases, desc, rank, world, local_rank):
    import torch
    import torch.distributed as dist

    import qlora_linear_b200 as q

    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    stream = torch.cuda.current_stream()

    # ---- inputs resident in HBM (drawn on the device)
    if args.workload == "mlp":
        ws = MlpSet(cases, dev, rank, world)
    elif args.workload == "ce":
        ws = CeSet(cases, dev, rank, world)
    else:
        ws = LinearSet(cases, dev, rank, world)
    layers, data, step = ws.layers, ws.data, ws.step
    torch.cuda.synchronize()

    def barrier():
        if world > 1:
            dist.barrier()

    # the clock record covers the warm-up steps too (the same work), so a short timed
    # region still has enough samples
    clocks = ClockSampler(gpu_uuid(dev), local_rank)
    clocks.start()
    time.sleep(0.05)
    clocks.mark("t_warm")
    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    # short steps on one GPU: keep warming up (same work) until the clock record holds
    # enough samples (with several ranks every rank must run the same steps, each with its
    # collective, so the count is not decided per rank)
    t_w = time.time()
    while world == 1 and clocks.source and clocks.count_since("t_warm") < MIN_CLOCK_SAMPLES \
            and time.time() - t_w < 2.0:
        step()
        torch.cuda.synchronize()
    for st in ws.statuses():
        if st != q.LORA_OK:
            raise RuntimeError("device status after warm-up: " + q.status_string(st))

    # ---- timed region: K steps, device time (CUDA events), max over ranks
    flush = args.workload == "c4s"  # working set near the L2 size: flush it before every step
    flush_buf = torch.empty(512 << 20, dtype=torch.uint8, device=dev) if flush else None
    barrier()
    torch.cuda.synchronize()
    clocks.mark("t_start")
    ms, fwd_ms, bwd_ms, g_launches, launches = time_steps(q, torch, step, args.steps, stream, flush_buf)
    clocks.mark("t_end")
    barrier()
    clocks.stop()
    clk = clocks.summary("t_start", "t_end", "t_warm")
    if world > 1:
        t = torch.tensor([ms], device=dev, dtype=torch.float64)
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        ms = float(t.item())
    for st in ws.statuses():
        if st != q.LORA_OK:
            raise RuntimeError("device status after timing: " + q.status_string(st))

    ce = args.workload == "ce"
    flops_step = ce_flops(cases[0]) if ce else sum(case_flops(c) for c in cases)
    tokens_step = cases[0].M
    value = world * flops_step / (ms * 1e-3) / 1e12
    peaks, peak_src = load_peaks()
    peak_sust = peaks.get("bf16_tflops_sustained", FALLBACK_PEAKS["bf16_tflops_sustained"])

    # ---- roofline of the dominant kernel (the tcgen05 GEMM: Y and dX launches)
    roofline = gemm_roofline(cases, ce, args.steps, fwd_ms, bwd_ms, g_launches, ms, peaks, clk)
    roofline["kernel"] = ("lora_gemm_pair_kernel" if all(c.fmt == "bf16" for c in cases) else
                          "lora_gemm_q_kernel" if all(c.fmt != "bf16" for c in cases) else
                          "lora_gemm_pair_kernel / lora_gemm_q_kernel") + " (Y and dX GEMMs)"
    tr = traffic_record()
    roofline["traffic"] = None
    if tr and tr.get("source_hash") == source_hash() and tr.get("workload") == args.workload and \
            args.weight in (None, "bf16") and not args.rank and not args.only:
        roofline["traffic"] = tr.get("bytes_per_launch")

    # ---- grouped workloads: the same projections as separate layers, for comparison
    separate = None
    if args.no_separate:
        pass
    elif world == 1 and args.workload == "mlp":
        separate = time_separate_mlp(args, cases, ws, dev)
    elif world == 1 and args.workload == "ce":
        separate = time_separate_ce(args, cases, ws, dev)
    elif world == 1 and any(c.rows is not None for c in cases):
        separate = time_separate(args, cases, data, dev)

    # ---- forward and backward timed on their own (single-projection workloads)
    split = None
    if isinstance(ws, LinearSet):
        split = time_split(args, ws, stream)

    # ---- end to end through the public API with host buffers
    e2e = None
    if not args.no_e2e:
        if args.workload in ("mlp", "ce"):
            e2e = ws.e2e(args, step)
        else:
            e2e = run_e2e(args, cases, layers, data, step, world, dev)
            # the same with every output (Y and dX too) read back each step
            e2e["all_outputs"] = run_e2e(args, cases, layers, data, step, world, dev, outs=("Y", "dX", "dA", "dB"))

    # ---- oracle on the host cores (rank 0, N = 1 only)
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        t, fl = oracle_sample(cases, args.cpu_tokens, mlp=args.workload == "mlp", ce=args.workload == "ce")
        cpu = {"value": fl / t / 1e12, "unit": "TFLOP/s", "cores": cpu_threads(), "kind": "oracle",
               "sample": f"first {args.cpu_tokens} tokens of each projection (full K and N), fp64 numpy oracle, "
                         f"{t:.1f} s", "tokens_per_s": args.cpu_tokens / t}

    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "bf16", "data": "synthetic (seeded, drawn on device)",
            "config": {"workload": desc, "tokens_per_rank_per_step": tokens_step,
                       "global_batch_tokens": tokens_step * world, "r": cases[0].r,
                       "projections": [c.name for c in cases], "parallelism": f"dp{world}",
                       "l2": ("L2 flushed (512 MB written) before every timed step, outside its events" if flush
                              else "inputs larger than L2 (step working set several GB >> 126 MB)")},
            "tokens_per_s": world * tokens_step / (ms * 1e-3),
            "pct_peak_burst": value / world / peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"]),
            "pct_peak_sustained": value / world / peak_sust,
            "pct_peak_nominal": value / world / NOMINAL_BF16_TFLOPS,
            "peak_source": peak_src,
            "roofline": roofline, "cpu_baseline": cpu, "e2e": e2e, "gpu_launches": launches,
            "clocks": clk,
        }
        if separate is not None:
            line["separate_layers"] = separate
        if split is not None:
            line["split"] = split
        if isinstance(ws, LinearSet):
            line["algorithmic_gbs"] = world * sum(case_bytes(c) for c in cases) / (ms * 1e-3) / 1e9
            line["algorithmic_gbs_note"] = ("HBM floor of the step (weights read twice, activations and outputs once) "
                                            "over its time, against the measured copy bandwidth "
                                            f"{peaks.get('hbm_gbs', FALLBACK_PEAKS['hbm_gbs'])} GB/s")
        print(json.dumps(line), flush=True)


def time_separate(args, cases, data, dev):
    """Device time per step of a grouped workload run as G separate single-projection
    layers (each with its own dY and outputs, as an unfused model would hold them)."""
    import torch

    import qlora_linear_b200 as q

    stream = torch.cuda.current_stream()
    parts = []
    for c, (d, _) in zip(cases, data):
        off = 0
        for g, n in enumerate(c.rows):
            W = q.LoraWeight(n, c.K, d["W"][off:off + n])
            layer = q.LoraLinear(W, d["A"][g * c.r:(g + 1) * c.r], d["B"][off:off + n], c.alpha)
            layer.workspace(c.M)
            dY = d["dY"][:, off:off + n].contiguous()
            o = (torch.empty((c.M, n), dtype=torch.bfloat16, device=dev),
                 torch.empty((c.M, c.r), dtype=torch.bfloat16, device=dev),
                 torch.empty((c.M, c.K), dtype=torch.bfloat16, device=dev),
                 torch.empty((c.r, c.K), dtype=torch.bfloat16, device=dev),
                 torch.empty((n, c.r), dtype=torch.bfloat16, device=dev))
            parts.append((layer, d["X"], dY, o))
            off += n

    def step():
        for layer, X, dY, (Y, XA, dX, dA, dB) in parts:
            layer.forward(X, Y=Y, XA=XA)
            layer.backward(dY, X, XA, out=(dX, dA, dB))

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(args.steps):
        step()
    e1.record(stream)
    torch.cuda.synchronize()
    ms = e0.elapsed_time(e1) / args.steps
    flops_step = sum(case_flops(c) for c in cases)
    return {"ms_per_step": ms, "value": flops_step / (ms * 1e-3) / 1e12, "unit": "TFLOP/s",
            "note": "the same projections as separate layers (dX of each written separately, not summed)"}


def time_split(args, ws, stream):
    """Forward alone and backward alone over the step's projections (CUDA events)."""
    import torch

    res = {}
    for name in ("fwd", "bwd"):
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        n = max(3, args.steps // 2)
        e0.record(stream)
        for _ in range(n):
            for layer, (d, o) in zip(ws.layers, ws.data):
                if name == "fwd":
                    layer.forward(d["X"], Y=o["Y"], XA=o["XA"])
                else:
                    layer.backward(d["dY"], d["X"], o["XA"], out=(o["dX"], o["dA"], o["dB"]))
        e1.record(stream)
        torch.cuda.synchronize()
        res[name + "_ms"] = e0.elapsed_time(e1) / n
    return res


def run_e2e(args, cases, layers, data, step, world, dev, outs=("dA", "dB")):
    """Same metric through the public API with host buffers: each step copies that
    step's inputs (X, dY and the adapter A, B) from pinned host memory and reads the
    step's result back: by default the adapter gradients dA, dB, the trainable outputs
    of a LoRA training step (Y and dX are activations that a model keeps on the device);
    outs=("Y", "dX", "dA", "dB") reads every output back.  The frozen weight stays
    resident.  Uploads, compute and read-backs run on three streams over two sets of
    device buffers, so one step's copies overlap the neighbouring steps' compute."""
    import torch
    import torch.distributed as dist

    import qlora_linear_b200 as q

    s_comp = torch.cuda.current_stream()
    s_h2d = torch.cuda.Stream(device=dev)
    s_d2h = torch.cuda.Stream(device=dev)
    NB = 2
    bf = torch.bfloat16
    host_in, host_out = [], []
    h2d = d2h = 0
    x_of = []  # index of the unique X each projection reads
    xs_host = []
    for (d, o) in data:
        k = next((u for u, hx in enumerate(xs_host) if hx[0] is d["X"]), None)
        if k is None:
            xs_host.append((d["X"], d["X"].cpu().pin_memory()))
            k = len(xs_host) - 1
            h2d += d["X"].numel() * 2
        x_of.append(k)
        hi = {"dY": d["dY"].cpu().pin_memory(), "A": d["A"].cpu().pin_memory(), "B": d["B"].cpu().pin_memory()}
        h2d += (hi["dY"].numel() + hi["A"].numel() + hi["B"].numel()) * 2
        host_in.append(hi)
        ho = {k2: torch.empty(o[k2].shape, dtype=o[k2].dtype).pin_memory() for k2 in outs}
        d2h += sum(v.numel() * 2 for v in ho.values())
        host_out.append(ho)
    dev_x = [[torch.empty_like(x) for x, _ in xs_host] for _ in range(NB)]
    dev_dy = [[torch.empty_like(d["dY"]) for d, _ in data] for _ in range(NB)]
    # each buffer set has its own adapter tensors, uploaded on the upload stream with X and
    # dY (an upload on the compute stream would queue behind the next step's large copies);
    # the layer copies share the weight and the workspace (their calls are stream-ordered)
    import copy
    lay_b = []
    for _ in range(NB):
        row = []
        for layer in layers:
            lb = copy.copy(layer)
            lb.A, lb.B = torch.empty_like(layer.A), torch.empty_like(layer.B)
            row.append(lb)
        lay_b.append(row)
    dev_out = [[{k2: torch.empty_like(o[k2]) for k2 in ("Y", "XA", "dX", "dA", "dB")} for _, o in data]
               for _ in range(NB)]
    ex = [[q.AdapterGradExchange([o["dA"].shape, o["dB"].shape], dev) for _, o in data] for _ in range(NB)] \
        if world > 1 else None
    ev_in = [[torch.cuda.Event() for _ in data] for _ in range(NB)]
    ev_comp = [torch.cuda.Event() for _ in range(NB)]
    ev_out = [[torch.cuda.Event() for _ in data] for _ in range(NB)]

    def e2e_step(s):
        b = s % NB
        # the uploads into buffer set b wait until the step that last read it is computed
        s_h2d.wait_event(ev_comp[b])
        with torch.cuda.stream(s_h2d):
            done = set()
            for i in range(len(data)):
                if x_of[i] not in done:
                    dev_x[b][x_of[i]].copy_(xs_host[x_of[i]][1], non_blocking=True)
                    done.add(x_of[i])
                dev_dy[b][i].copy_(host_in[i]["dY"], non_blocking=True)
                lay_b[b][i].A.copy_(host_in[i]["A"], non_blocking=True)
                lay_b[b][i].B.copy_(host_in[i]["B"], non_blocking=True)
                ev_in[b][i].record(s_h2d)
        for i, layer in enumerate(lay_b[b]):
            o = dev_out[b][i]
            s_comp.wait_event(ev_in[b][i])
            s_comp.wait_event(ev_out[b][i])  # this buffer's previous outputs have been read back
            X = dev_x[b][x_of[i]]
            layer.forward(X, Y=o["Y"], XA=o["XA"], stream=s_comp)
            if world == 1:
                layer.backward(dev_dy[b][i], X, o["XA"], out=(o["dX"], o["dA"], o["dB"]), stream=s_comp)
            else:
                v = ex[b][i].views
                layer.backward(dev_dy[b][i], X, o["XA"], out=(o["dX"], v[0], v[1]), stream=s_comp, grads_f32=True)
                with torch.cuda.stream(s_comp):
                    ex[b][i].allreduce()
                    ex[b][i].round_into([o["dA"], o["dB"]])
            ev = torch.cuda.Event()
            ev.record(s_comp)
            s_d2h.wait_event(ev)
            with torch.cuda.stream(s_d2h):
                for k2 in outs:
                    host_out[i][k2].copy_(o[k2], non_blocking=True)
                ev_out[b][i].record(s_d2h)
        ev_comp[b].record(s_comp)

    for s in range(2):
        e2e_step(s)
    torch.cuda.synchronize()
    steps = max(4, args.steps // 2)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(s_comp)
    s_h2d.wait_event(e0)
    s_d2h.wait_event(e0)
    for s in range(steps):
        e2e_step(s)
    s_comp.wait_stream(s_d2h)
    s_comp.wait_stream(s_h2d)
    e1.record(s_comp)
    torch.cuda.synchronize()
    ms = e0.elapsed_time(e1) / steps
    if world > 1:
        t = torch.tensor([ms], device=dev, dtype=torch.float64)
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        ms = float(t.item())
    flops_step = sum(case_flops(c) for c in cases)
    return {"value": world * flops_step / (ms * 1e-3) / 1e12, "unit": "TFLOP/s", "h2d_bytes_per_step": h2d,
            "d2h_bytes_per_step": d2h, "ms_per_step": ms, "steps": steps,
            "note": "inputs X, dY, A, B copied from pinned host memory and " + ", ".join(outs) +
                    " read back every step; the frozen weight stays resident; uploads, compute and read-backs on "
                    "three streams over two buffer sets"}


def main(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default="c2", choices=["c1", "c2", "c3", "c4", "c4s", "qkv", "mlp", "ce"])
    ap.add_argument("--select", default=None,
                    help="rank sweep only: comma-separated key=value filters on M, N, K, r and fmt "
                         "(a key may repeat: M=512,M=4096)")
    ap.add_argument("--only", default=None, help="run a single projection of the workload (e.g. c2_gate)")
    ap.add_argument("--cpu-tokens", type=int, default=256)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-separate", action="store_true", help="skip the unfused comparison of qkv / mlp")
    ap.add_argument("--weight", default=None, choices=["bf16", "block4", "int8", "fp8"],
                    help="store every frozen weight of the workload in this format")
    ap.add_argument("--rank", type=int, default=None,
                    help="run every projection at this LoRA rank (alpha = 2·rank) instead of the workload's")
    args = ap.parse_args(argv)
    if args.warmup < 3 and args.impl == "ours":
        args.warmup = 3

    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    cases, desc = workload(args.workload)
    if args.weight:
        import dataclasses
        cases = [dataclasses.replace(c, fmt=args.weight) for c in cases]
        desc = f"{desc}; frozen weights stored as {args.weight}"
    if args.rank:
        import dataclasses
        cases = [dataclasses.replace(c, r=args.rank, alpha=2.0 * args.rank) for c in cases]
        desc = f"{desc}; LoRA rank {args.rank}, alpha {2 * args.rank}"
    if args.select:
        cases = select_cases(cases, args.select)
        if not cases:
            raise SystemExit(f"no case of {args.workload} matches {args.select}")
        desc = f"{desc}; selected {args.select}"
    if args.only:
        cases = [c for c in cases if c.name == args.only]
        if not cases:
            raise SystemExit(f"no projection named {args.only} in {args.workload}")
        desc = f"{desc}; only {args.only}"

    if args.impl == "reference":
        return run_reference(args, cases, desc, rank, world)

    import torch
    import torch.distributed as dist
    if world > 1:
        torch.cuda.set_device(local_rank)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local_rank))
    try:
        if args.workload == "c4":
            run_sweep(args, cases, desc, rank, world, local_rank)
        else:
            run_ours(args, cases, desc, rank, world, local_rank)
    finally:
        if world > 1 and dist.is_initialized():
            dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
