"""Seeded synthetic inputs for the LoRA-adapted linear layer.

Shapes follow the PyTorch ``Linear`` convention used throughout this project:
``X:[M,K]``, ``W:[N,K]``, ``A:[r,K]``, ``B:[N,r]``, ``dY:[M,N]``.  Every tensor is
stored the way the library takes it: bf16 tensors as ``uint16`` bit patterns, the
4-bit weight as packed codes (``uint8 [N, K/2]``, element ``2j`` in the low nibble),
one fp16 absmax per 64 contiguous elements (``uint16`` bit patterns) and a 16-entry
float32 codebook.

Value recipe (one seed per case, one independent stream per tensor and per 2^20-element
chunk, so the result does not depend on the number of worker threads):

* ``X ~ N(0, 1)``, ``dY ~ N(0, 1)``
* ``W ~ N(0, 1/K)`` (variance ``1/K``)
* ``A ~ U(-1/sqrt(K), 1/sqrt(K))``
* ``B ~ N(0, 0.01)`` read as variance 0.01, i.e. standard deviation 0.1
* 4-bit weight: codes uniform on ``{0..15}``; scale of block ``b`` is
  ``fp16_rn((1.2 + 0.8 u_b)/sqrt(K))`` with ``u_b ~ U(0,1)``; codebook levels
  ``(2i - 15)/15`` for ``i = 0..15`` rounded to float32 (16 symmetric levels in
  ``[-1, 1]``).  With these, the 4-bit weight has rms close to ``1/sqrt(K)``, the
  same as the bf16 weight.

Every draw is rounded to the storage type (round to nearest even) and nothing else
happens to it here.
"""
from __future__ import annotations

import dataclasses
import os
from concurrent.futures import ThreadPoolExecutor

import numpy as np

BASE_SEED = 20261202
_CHUNK = 1 << 20

# tensor ids for the per-tensor random streams
_TID = {"X": 1, "W": 2, "A": 3, "B": 4, "dY": 5, "codes": 6, "absmax": 7}


def bf16_bits_from_f32(x: np.ndarray) -> np.ndarray:
    """Round float32 values to bfloat16, nearest-even; returns the uint16 bit patterns."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    lsb = (u >> np.uint32(16)) & np.uint32(1)
    r = ((u + np.uint32(0x7FFF) + lsb) >> np.uint32(16)).astype(np.uint16)
    nan = np.isnan(np.ascontiguousarray(x, dtype=np.float32))
    if nan.any():
        r[nan] = np.uint16(0x7FC0)
    return r


def f32_from_bf16_bits(b: np.ndarray) -> np.ndarray:
    """Widen bf16 bit patterns to float32 (exact)."""
    return (np.ascontiguousarray(b, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


@dataclasses.dataclass(frozen=True)
class LoraCase:
    """One LoRA-linear problem: sizes, format and seed."""

    name: str
    M: int
    N: int
    K: int
    r: int
    alpha: float
    fmt: str  # "bf16", "block4", "int8" or "fp8"
    seed: int                  # stream of A and B (and of X, W, dY unless set below)
    x_seed: int | None = None  # X stream: lets two projections share one activation tensor
    data_seed: int | None = None  # W and dY stream (and X if x_seed is None)
    rows: tuple | None = None  # several projections sharing X, stacked along N (rows sum to N)

    @property
    def s(self) -> float:
        return float(self.alpha) / float(self.r)

    @property
    def G(self) -> int:
        """Number of projections (1 unless ``rows`` is set); A is ``[G·r, K]``."""
        return 1 if self.rows is None else len(self.rows)

    def with_M(self, M: int) -> "LoraCase":
        return dataclasses.replace(self, M=M, name=f"{self.name}_M{M}")


def _cases() -> dict[str, list[LoraCase]]:
    b = BASE_SEED
    c = {}
    c["c0"] = [LoraCase("c0_tiny", 256, 512, 512, 8, 16.0, "bf16", b + 0)]
    c["c1"] = [LoraCase("c1_attn", 8192, 4096, 4096, 16, 32.0, "bf16", b + 1)]
    c["c2"] = [
        LoraCase("c2_gate", 16384, 14336, 4096, 16, 32.0, "bf16", b + 2, x_seed=b + 2),
        LoraCase("c2_up", 16384, 14336, 4096, 16, 32.0, "bf16", b + 2 + 100, x_seed=b + 2),
        LoraCase("c2_down", 16384, 4096, 14336, 16, 32.0, "bf16", b + 2 + 200),
    ]
    c["c3"] = [LoraCase("c3_qlora", 8192, 14336, 4096, 16, 32.0, "block4", b + 3)]
    sweep = []
    g = 0
    for fmt in ("bf16", "block4"):
        for (K, N) in ((8192, 8192), (8192, 28672)):
            for M in (512, 4096, 16384):
                g += 1
                for r in (8, 16, 64, 128):
                    # X, W and dY are shared by the four ranks of one shape and format
                    sweep.append(LoraCase(f"c4_{fmt}_K{K}_N{N}_M{M}_r{r}", M, N, K, r, 2.0 * r, fmt,
                                          b + 4 + 1000 * g + r, data_seed=b + 4 + 1000 * g))
    c["c4"] = sweep
    # Llama-8B attention q/k/v (grouped-query: 32 query heads, 8 key/value heads of 128)
    c["qkv"] = [LoraCase("qkv_llama8b", 8192, 6144, 4096, 16, 32.0, "bf16", b + 5, rows=(4096, 1024, 1024))]
    return c


CONFIGS: dict[str, list[LoraCase]] = _cases()


def config_cases(name: str) -> list[LoraCase]:
    return list(CONFIGS[name])


def _threads() -> int:
    return max(1, min(32, os.cpu_count() or 1))


def _fill(shape, seed: int, tid: int, draw) -> np.ndarray:
    """Fill an array chunk by chunk; chunk i uses stream SeedSequence([seed, tid, i])."""
    n = int(np.prod(shape)) if len(shape) else 1
    out = np.empty(n, dtype=np.uint16)
    nchunks = (n + _CHUNK - 1) // _CHUNK

    def work(i):
        lo, hi = i * _CHUNK, min(n, (i + 1) * _CHUNK)
        g = np.random.Generator(np.random.PCG64(np.random.SeedSequence([seed, tid, i])))
        out[lo:hi] = draw(g, hi - lo)

    if nchunks <= 1:
        for i in range(nchunks):
            work(i)
    else:
        with ThreadPoolExecutor(_threads()) as ex:
            list(ex.map(work, range(nchunks)))
    return out.reshape(shape)


def _normal_bf16(std: float):
    def draw(g, n):
        v = g.standard_normal(n, dtype=np.float32)
        if std != 1.0:
            v *= np.float32(std)
        return bf16_bits_from_f32(v)
    return draw


def _uniform_bf16(lo: float, hi: float):
    def draw(g, n):
        v = g.random(n, dtype=np.float32) * np.float32(hi - lo) + np.float32(lo)
        return bf16_bits_from_f32(v)
    return draw


def codebook_levels() -> np.ndarray:
    """The 16 symmetric levels (2i-15)/15, i = 0..15, rounded to float32."""
    return np.array([(2 * i - 15) / 15.0 for i in range(16)], dtype=np.float64).astype(np.float32)


def make_case(case: LoraCase, want=("X", "W", "A", "B", "dY")) -> dict:
    """Draw the inputs of ``case``.  ``want`` limits which tensors are drawn."""
    M, N, K, r = case.M, case.N, case.K, case.r
    out: dict = {"case": case}
    ds = case.data_seed if case.data_seed is not None else case.seed
    xs = case.x_seed if case.x_seed is not None else ds
    if "X" in want:
        out["X"] = _fill((M, K), xs, _TID["X"], _normal_bf16(1.0))
    if "W" in want:
        if case.fmt == "bf16":
            out["W"] = _fill((N, K), ds, _TID["W"], _normal_bf16(1.0 / np.sqrt(K)))
        elif case.fmt == "block4":
            assert K % 64 == 0
            g = np.random.Generator(np.random.PCG64(np.random.SeedSequence([ds, _TID["codes"]])))
            out["codes"] = g.integers(0, 256, size=(N, K // 2), dtype=np.uint8)
            g = np.random.Generator(np.random.PCG64(np.random.SeedSequence([ds, _TID["absmax"]])))
            u = g.random(N * K // 64)
            out["absmax"] = ((1.2 + 0.8 * u) / np.sqrt(K)).astype(np.float16).view(np.uint16)
            out["codebook"] = codebook_levels()
        if case.fmt in ("int8", "fp8"):
            out.update(_codes8(case, ds))
    if "A" in want:
        a = 1.0 / np.sqrt(K)
        out["A"] = _fill((case.G * r, K), case.seed, _TID["A"], _uniform_bf16(-a, a))
    if "B" in want:
        out["B"] = _fill((N, r), case.seed, _TID["B"], _normal_bf16(0.1))
    if case.rows is not None:
        out["rows"] = [int(n) for n in case.rows]
    if "dY" in want:
        out["dY"] = _fill((M, N), ds, _TID["dY"], _normal_bf16(1.0))
    return out


# rms of the decoded codes drawn below: int8 uniform on [-127, 127] has mean square
# 127·128/3; fp8 with exponent field uniform on 1..14 and mantissa uniform on 0..7 has
# mean square (4^14 - 1)/(3·4^6)/14 · 2.1484375
RMS_INT8 = float(np.sqrt(127 * 128 / 3))
RMS_FP8 = float(np.sqrt((4 ** 14 - 1) / (3 * 4 ** 6) / 14 * 2.1484375))


def _codes8(case: LoraCase, ds: int) -> dict:
    """8-bit weight codes [N, K] and fp32 row scales [N]: int8 codes uniform on
    [-127, 127]; fp8 e4m3 codes with sign uniform, exponent field uniform on 1..14 and
    mantissa uniform on 0..7 (never NaN); scale of row n ``(0.8 + 0.4 u_n)/(rms·sqrt(K))``
    so that the weight's rms is about 1/sqrt(K), as for the bf16 weights."""
    N, K = case.N, case.K
    g = np.random.Generator(np.random.PCG64(np.random.SeedSequence([ds, _TID["codes"]])))
    if case.fmt == "int8":
        codes = g.integers(-127, 128, size=(N, K), dtype=np.int16).astype(np.int8).view(np.uint8)
        rms = RMS_INT8
    else:
        sign = g.integers(0, 2, size=(N, K), dtype=np.uint8)
        expo = g.integers(1, 15, size=(N, K), dtype=np.uint8)
        mant = g.integers(0, 8, size=(N, K), dtype=np.uint8)
        codes = ((sign << 7) | (expo << 3) | mant).astype(np.uint8)
        rms = RMS_FP8
    g = np.random.Generator(np.random.PCG64(np.random.SeedSequence([ds, _TID["absmax"]])))
    u = g.random(N)
    return {"codes": codes, "row_scale": ((0.8 + 0.4 * u) / (rms * np.sqrt(K))).astype(np.float32)}


def make_grouped_case(case: LoraCase, rows, want=("X", "W", "A", "B", "dY")) -> dict:
    """Inputs of G projections sharing X (``rows`` sum to ``case.N``): W, B and dY are
    drawn for the stacked ``[ΣN_g, ...]`` shapes and A for ``[G·r, K]``."""
    assert sum(int(n) for n in rows) == case.N
    return make_case(dataclasses.replace(case, rows=tuple(int(n) for n in rows)), want=want)


@dataclasses.dataclass(frozen=True)
class MlpCase:
    """One feed-forward block: tokens M, model width D, hidden width I, rank r."""

    name: str
    M: int
    D: int
    I: int  # noqa: E741
    r: int
    alpha: float
    fmt: str
    seed: int

    @property
    def s(self) -> float:
        return float(self.alpha) / float(self.r)

    def gate_up_case(self) -> LoraCase:
        """The gate and up projections as two projections of X stacked along rows."""
        return LoraCase(self.name + "_gate_up", self.M, 2 * self.I, self.D, self.r, self.alpha, self.fmt, self.seed,
                        rows=(self.I, self.I))

    def down_case(self) -> LoraCase:
        return LoraCase(self.name + "_down", self.M, self.D, self.I, self.r, self.alpha, self.fmt, self.seed + 7919)


def make_mlp_case(case: MlpCase) -> dict:
    """Inputs of a feed-forward block: X and the gate/up weight and adapters from the
    gate/up case (W ~ N(0, 1/D)), the down weight and adapters and dZ (the down case's dY)
    from the down case (W ~ N(0, 1/I)); same distributions as :func:`make_case`."""
    gu = make_case(case.gate_up_case(), want=("X", "W", "A", "B"))
    dn = make_case(case.down_case(), want=("W", "A", "B", "dY"))
    return {"case": case, "X": gu["X"], "A_gu": gu["A"], "B_gu": gu["B"], "A_d": dn["A"], "B_d": dn["B"],
            "dZ": dn["dY"], "gate_up": gu, "down": dn}


@dataclasses.dataclass(frozen=True)
class CeCase:
    """Cross-entropy over an LM head: M rows of hidden states of width D, vocabulary V."""

    name: str
    M: int
    D: int
    V: int
    seed: int
    ignore_index: int = -100
    ignore_frac: float = 0.05


def make_ce_case(case: CeCase) -> dict:
    """X ~ N(0, 1) [M, D] and head W ~ N(0, 4/D) [V, D] in bf16 (logits of std about 2);
    labels uniform on [0, V) with a fraction set to ignore_index; dloss uniform on
    [0.5, 1.5) as fp32."""
    M, D, V = case.M, case.D, case.V
    X = _fill((M, D), case.seed, _TID["X"], _normal_bf16(1.0))
    W = _fill((V, D), case.seed, _TID["W"], _normal_bf16(2.0 / np.sqrt(D)))
    g = np.random.Generator(np.random.PCG64(np.random.SeedSequence([case.seed, 8])))
    labels = g.integers(0, V, M).astype(np.int32)
    labels[g.random(M) < case.ignore_frac] = case.ignore_index
    dloss = (0.5 + g.random(M)).astype(np.float32)
    return {"case": case, "X": X, "W": W, "labels": labels, "dloss": dloss}
