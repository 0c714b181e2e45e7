"""ctypes binding of liblora_linear.so (include/lora_linear.h).

Argument marshalling only: every step of the layer runs in the library's CUDA
kernels.  Tensors are torch CUDA tensors (plumbing for device memory and streams);
their ``data_ptr()`` is passed straight through.  There is no CPU fallback: if the
library is missing this module raises on import.
"""
from __future__ import annotations

import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
# LORA_LIB_PATH selects another build of the library (e.g. one compiled with different flags).
LIB_PATH = os.environ.get("LORA_LIB_PATH") or os.path.join(_HERE, "liblora_linear.so")

LORA_OK = 0
LORA_ERR_INVALID_ARG = 1
LORA_ERR_ALIGNMENT = 2
LORA_ERR_UNSUPPORTED = 3
LORA_ERR_WORKSPACE = 4
LORA_ERR_CUDA = 5
LORA_ERR_DEVICE_TIMEOUT = 6
LORA_ERR_SCRATCH_LIMIT = 7
LORA_ERR_DEVICE_BOUNDS = 8
LORA_NOALLOC_SCRATCH_BYTES = 16 * 1024 * 1024

LORA_GRADS_F32 = 1  # flags of the *_bwd_ex calls: adapter gradients as fp32

LORA_W_BF16 = 0
LORA_W_BLOCK4 = 1
LORA_W_INT8 = 2
LORA_W_FP8_E4M3 = 3

EXPORTED = (
    "lora_workspace_bytes", "lora_linear_fwd", "lora_linear_bwd", "dequant_blockwise4",
    "lora_merge", "lora_device_status", "lora_status_string", "lora_version",
    "lora_testing_bounded_wait", "lora_testing_gemm_streamk", "lora_testing_xpass_tma", "lora_testing_dual_blocking", "lora_timing_enable", "lora_timing_read",
    "lora_launch_count",
    "lora_linear_fwd_noalloc", "lora_grouped_workspace_bytes", "lora_grouped_fwd", "lora_grouped_bwd",
    "lora_mlp_workspace_bytes", "lora_mlp_fwd", "lora_mlp_bwd", "lora_dequant",
    "lora_ce_workspace_bytes", "lora_ce_fwd", "lora_ce_bwd",
    "lora_linear_bwd_ex", "lora_grouped_bwd_ex", "lora_mlp_bwd_ex", "lora_round_bf16",
    "lora_testing_tcproj_extra_tile", "lora_testing_tcproj_splits",
)

LORA_MAX_SEGMENTS = 8


class LoraError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: status {status}: {status_string(status)}")


class lora_weight_t(ctypes.Structure):
    _fields_ = [
        ("fmt", ctypes.c_int32),
        ("reserved", ctypes.c_int32),
        ("N", ctypes.c_int64),
        ("K", ctypes.c_int64),
        ("data", ctypes.c_void_p),
        ("absmax", ctypes.c_void_p),
        ("codebook", ctypes.c_void_p),
    ]


class lora_segments_t(ctypes.Structure):
    _fields_ = [
        ("count", ctypes.c_int32),
        ("reserved", ctypes.c_int32),
        ("rows", ctypes.c_int64 * 8),
    ]


class lora_mlp_t(ctypes.Structure):
    _fields_ = [
        ("gate_up", lora_weight_t),
        ("down", lora_weight_t),
        ("A_gate_up", ctypes.c_void_p),
        ("B_gate_up", ctypes.c_void_p),
        ("A_down", ctypes.c_void_p),
        ("B_down", ctypes.c_void_p),
    ]


def segments(rows) -> lora_segments_t:
    rows = [int(x) for x in rows]
    if not 1 <= len(rows) <= LORA_MAX_SEGMENTS:
        raise ValueError("between 1 and 8 projections")
    seg = lora_segments_t()
    seg.count = len(rows)
    seg.reserved = 0
    for i, n in enumerate(rows):
        seg.rows[i] = n
    return seg


def _load() -> ctypes.CDLL:
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"{LIB_PATH} is missing: build it with `python qlora_linear_b200/build.py`")
    lib = ctypes.CDLL(LIB_PATH)
    vp, i32, i64, sz, f32 = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_size_t, ctypes.c_float
    W = ctypes.POINTER(lora_weight_t)
    lib.lora_workspace_bytes.argtypes = [i64, i64, i64, i32, i32]
    lib.lora_workspace_bytes.restype = sz
    lib.lora_linear_fwd.argtypes = [vp, i64, W, vp, vp, i32, f32, vp, vp, vp, sz, vp]
    lib.lora_linear_fwd.restype = i32
    lib.lora_linear_bwd.argtypes = [vp, vp, vp, i64, W, vp, vp, i32, f32, vp, vp, vp, vp, sz, vp]
    lib.lora_linear_bwd.restype = i32
    u32 = ctypes.c_uint32
    lib.lora_linear_bwd_ex.argtypes = [vp, vp, vp, i64, W, vp, vp, i32, f32, vp, vp, vp, u32, vp, sz, vp]
    lib.lora_linear_bwd_ex.restype = i32
    lib.lora_round_bf16.argtypes = [vp, vp, i64, vp]
    lib.lora_round_bf16.restype = i32
    lib.dequant_blockwise4.argtypes = [W, vp, vp]
    lib.dequant_blockwise4.restype = i32
    lib.lora_dequant.argtypes = [W, vp, vp]
    lib.lora_dequant.restype = i32
    lib.lora_ce_workspace_bytes.argtypes = [i64, i64, i64, i64]
    lib.lora_ce_workspace_bytes.restype = sz
    lib.lora_ce_fwd.argtypes = [vp, i64, W, vp, i32, vp, vp, vp, sz, vp]
    lib.lora_ce_fwd.restype = i32
    lib.lora_ce_bwd.argtypes = [vp, i64, W, vp, i32, vp, vp, vp, vp, sz, vp]
    lib.lora_ce_bwd.restype = i32
    lib.lora_merge.argtypes = [W, vp, vp, i32, f32, vp, vp]
    lib.lora_merge.restype = i32
    lib.lora_device_status.argtypes = [vp, vp]
    lib.lora_device_status.restype = i32
    lib.lora_status_string.argtypes = [i32]
    lib.lora_status_string.restype = ctypes.c_char_p
    lib.lora_version.argtypes = []
    lib.lora_version.restype = i32
    lib.lora_testing_bounded_wait.argtypes = [vp, ctypes.c_uint64, vp]
    lib.lora_testing_bounded_wait.restype = i32
    lib.lora_testing_gemm_streamk.argtypes = [i64, i64, i64, i32, i32]
    lib.lora_testing_gemm_streamk.restype = i32
    lib.lora_testing_xpass_tma.argtypes = [i64, i64, i32]
    lib.lora_testing_xpass_tma.restype = i32
    lib.lora_testing_dual_blocking.argtypes = [i64, i64, i32, i32, ctypes.POINTER(i32)]
    lib.lora_testing_dual_blocking.restype = i32
    lib.lora_testing_tcproj_extra_tile.argtypes = [vp, vp, i64, i64, i32, vp, sz, vp, vp]
    lib.lora_testing_tcproj_extra_tile.restype = i32
    lib.lora_testing_tcproj_splits.argtypes = [i64, i64, i32]
    lib.lora_testing_tcproj_splits.restype = i32
    lib.lora_timing_enable.argtypes = [i32]
    lib.lora_timing_enable.restype = i32
    lib.lora_timing_read.argtypes = [i32, ctypes.POINTER(ctypes.c_double), ctypes.POINTER(ctypes.c_int64)]
    lib.lora_timing_read.restype = i32
    lib.lora_launch_count.argtypes = []
    lib.lora_launch_count.restype = i64
    lib.lora_linear_fwd_noalloc.argtypes = [vp, i64, W, vp, vp, i32, f32, vp, vp, vp]
    lib.lora_linear_fwd_noalloc.restype = i32
    S = ctypes.POINTER(lora_segments_t)
    lib.lora_grouped_workspace_bytes.argtypes = [i64, i64, i64, i32, i32, i32]
    lib.lora_grouped_workspace_bytes.restype = sz
    lib.lora_grouped_fwd.argtypes = [vp, i64, W, S, vp, vp, i32, f32, vp, vp, vp, sz, vp]
    lib.lora_grouped_fwd.restype = i32
    lib.lora_grouped_bwd.argtypes = [vp, vp, vp, i64, W, S, vp, vp, i32, f32, vp, vp, vp, vp, sz, vp]
    lib.lora_grouped_bwd.restype = i32
    lib.lora_grouped_bwd_ex.argtypes = [vp, vp, vp, i64, W, S, vp, vp, i32, f32, vp, vp, vp, u32, vp, sz, vp]
    lib.lora_grouped_bwd_ex.restype = i32
    P = ctypes.POINTER(lora_mlp_t)
    lib.lora_mlp_workspace_bytes.argtypes = [i64, i64, i64, i32, i32]
    lib.lora_mlp_workspace_bytes.restype = sz
    lib.lora_mlp_fwd.argtypes = [vp, i64, P, i32, f32, vp, vp, vp, vp, vp, vp, sz, vp]
    lib.lora_mlp_fwd.restype = i32
    lib.lora_mlp_bwd.argtypes = [vp, vp, vp, vp, vp, vp, i64, P, i32, f32, vp, vp, vp, vp, vp, vp, sz, vp]
    lib.lora_mlp_bwd.restype = i32
    lib.lora_mlp_bwd_ex.argtypes = [vp, vp, vp, vp, vp, vp, i64, P, i32, f32, vp, vp, vp, vp, vp, u32, vp, sz, vp]
    lib.lora_mlp_bwd_ex.restype = i32
    return lib


_lib = _load()


def lib() -> ctypes.CDLL:
    return _lib


def status_string(status: int) -> str:
    return _lib.lora_status_string(int(status)).decode()


def _ptr(t) -> int | None:
    if t is None:
        return None
    if isinstance(t, int):
        return t
    return t.data_ptr()


def _stream(stream) -> int | None:
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def _check(st: int, where: str):
    if st != LORA_OK:
        raise LoraError(st, where)


class LoraWeight:
    """A frozen weight [N, K]: bf16 tensor, the 4-bit blockwise triple (codes uint8
    [N, K/2], absmax fp16 [N*K/64], codebook float32 [16]), or 8-bit codes [N, K]
    (int8 or fp8 e4m3, one byte each) with float32 row scales [N] (``fmt`` given)."""

    def __init__(self, N: int, K: int, data, absmax=None, codebook=None, fmt=None):
        self.N, self.K = int(N), int(K)
        self.data, self.absmax, self.codebook = data, absmax, codebook
        if fmt is None:
            fmt = LORA_W_BF16 if absmax is None else LORA_W_BLOCK4
        self.fmt = int(fmt)

    @classmethod
    def int8(cls, codes: torch.Tensor, row_scale: torch.Tensor) -> "LoraWeight":
        return cls(codes.shape[0], codes.shape[1], codes, row_scale, None, LORA_W_INT8)

    @classmethod
    def fp8(cls, codes: torch.Tensor, row_scale: torch.Tensor) -> "LoraWeight":
        return cls(codes.shape[0], codes.shape[1], codes, row_scale, None, LORA_W_FP8_E4M3)

    @classmethod
    def bf16(cls, w: torch.Tensor) -> "LoraWeight":
        return cls(w.shape[0], w.shape[1], w)

    @classmethod
    def block4(cls, codes: torch.Tensor, absmax: torch.Tensor, codebook: torch.Tensor, K: int) -> "LoraWeight":
        return cls(codes.shape[0], K, codes, absmax, codebook)

    def c_struct(self) -> lora_weight_t:
        return lora_weight_t(self.fmt, 0, self.N, self.K, _ptr(self.data), _ptr(self.absmax), _ptr(self.codebook))


def workspace_bytes(M: int, N: int, K: int, r: int, fmt: int = LORA_W_BF16) -> int:
    return int(_lib.lora_workspace_bytes(int(M), int(N), int(K), int(r), int(fmt)))


def alloc_workspace(M: int, N: int, K: int, r: int, fmt: int = LORA_W_BF16, device=None) -> torch.Tensor:
    """Zero-filled workspace (the status word at its head must start at zero)."""
    n = workspace_bytes(M, N, K, r, fmt)
    if n == 0:
        raise LoraError(LORA_ERR_UNSUPPORTED, "workspace_bytes")
    return torch.zeros(n, dtype=torch.uint8, device=device or "cuda")


def lora_linear_fwd(X, M: int, W: LoraWeight, A, B, r: int, s: float, Y, XA, workspace, ws_bytes=None,
                    stream=None) -> None:
    w = W.c_struct()
    nb = workspace.numel() * workspace.element_size() if ws_bytes is None else ws_bytes
    _check(_lib.lora_linear_fwd(_ptr(X), int(M), ctypes.byref(w), _ptr(A), _ptr(B), int(r), float(s), _ptr(Y),
                                _ptr(XA), _ptr(workspace), int(nb), _stream(stream)), "lora_linear_fwd")


def lora_linear_bwd(dY, X, XA, M: int, W: LoraWeight, A, B, r: int, s: float, dX, dA, dB, workspace, ws_bytes=None,
                    stream=None) -> None:
    w = W.c_struct()
    nb = workspace.numel() * workspace.element_size() if ws_bytes is None else ws_bytes
    _check(_lib.lora_linear_bwd(_ptr(dY), _ptr(X), _ptr(XA), int(M), ctypes.byref(w), _ptr(A), _ptr(B), int(r),
                                float(s), _ptr(dX), _ptr(dA), _ptr(dB), _ptr(workspace), int(nb), _stream(stream)),
           "lora_linear_bwd")


def lora_linear_bwd_ex(dY, X, XA, M: int, W: LoraWeight, A, B, r: int, s: float, dX, dA, dB, flags: int, workspace,
                       ws_bytes=None, stream=None) -> None:
    """lora_linear_bwd with flags; LORA_GRADS_F32 writes dA and dB as fp32 tensors."""
    w = W.c_struct()
    nb = workspace.numel() * workspace.element_size() if ws_bytes is None else ws_bytes
    _check(_lib.lora_linear_bwd_ex(_ptr(dY), _ptr(X), _ptr(XA), int(M), ctypes.byref(w), _ptr(A), _ptr(B), int(r),
                                   float(s), _ptr(dX), _ptr(dA), _ptr(dB), int(flags), _ptr(workspace), int(nb),
                                   _stream(stream)), "lora_linear_bwd_ex")


def lora_round_bf16(src, dst, n: int | None = None, stream=None) -> None:
    """dst (bf16) = round-to-nearest-even of src (fp32), n elements (default: all of src)."""
    n = src.numel() if n is None else int(n)
    _check(_lib.lora_round_bf16(_ptr(src), _ptr(dst), n, _stream(stream)), "lora_round_bf16")


def lora_dequant(W: LoraWeight, W_out, stream=None) -> None:
    """bf16 [N, K] copy of a weight of any format (bit-exact)."""
    w = W.c_struct()
    _check(_lib.lora_dequant(ctypes.byref(w), _ptr(W_out), _stream(stream)), "lora_dequant")


def dequant_blockwise4(Wq: LoraWeight, W_out, stream=None) -> None:
    w = Wq.c_struct()
    _check(_lib.dequant_blockwise4(ctypes.byref(w), _ptr(W_out), _stream(stream)), "dequant_blockwise4")


def lora_merge(W: LoraWeight, A, B, r: int, s: float, W_out, stream=None) -> None:
    w = W.c_struct()
    _check(_lib.lora_merge(ctypes.byref(w), _ptr(A), _ptr(B), int(r), float(s), _ptr(W_out), _stream(stream)),
           "lora_merge")


def lora_device_status(workspace, stream=None) -> int:
    return int(_lib.lora_device_status(_ptr(workspace), _stream(stream)))


def lora_testing_bounded_wait(workspace, limit_ns: int, stream=None) -> int:
    return int(_lib.lora_testing_bounded_wait(_ptr(workspace), int(limit_ns), _stream(stream)))


def lora_testing_dual_blocking(M: int, C: int, r: int, mode: int = 0):
    """(used, (a, b, row_tiles, col_tiles)) of the one-pass kernel over [M, C] at rank r."""
    out = (ctypes.c_int32 * 4)()
    used = int(_lib.lora_testing_dual_blocking(int(M), int(C), int(r), int(mode), out))
    return used, tuple(int(v) for v in out)


def lora_testing_xpass_tma(M: int, K: int, r: int) -> int:
    """Bit 0: the forward's X·Aᵀ, bit 1: the backward's pass for dA run on the TMA stream."""
    return int(_lib.lora_testing_xpass_tma(int(M), int(K), int(r)))


def lora_testing_tcproj_splits(rows: int, red: int, r: int) -> int:
    return int(_lib.lora_testing_tcproj_splits(int(rows), int(red), int(r)))


def lora_testing_tcproj_extra_tile(P, A, rows: int, red: int, r: int, part, workspace, stream=None) -> int:
    """Rank-r row projection with one output tile past the last row (see lora_linear_testing.h)."""
    return int(_lib.lora_testing_tcproj_extra_tile(_ptr(P), _ptr(A), int(rows), int(red), int(r), _ptr(part),
                                                   int(part.numel() * part.element_size()), _ptr(workspace),
                                                   _stream(stream)))


def lora_testing_gemm_streamk(M: int, Nout: int, Kred: int, r: int, fmt: int = LORA_W_BF16) -> int:
    """Output tiles the Y / dX GEMM shares out as stream-K pieces (0: all tiles whole)."""
    return int(_lib.lora_testing_gemm_streamk(int(M), int(Nout), int(Kred), int(r), int(fmt)))




LORA_KERNEL_FWD_GEMM = 0
LORA_KERNEL_BWD_GEMM = 1


def lora_timing_enable(on: bool) -> None:
    _check(_lib.lora_timing_enable(1 if on else 0), "lora_timing_enable")


def lora_timing_read(kernel: int) -> tuple[float, int]:
    """(summed device milliseconds, launches) of one GEMM kind since the last read."""
    ms = ctypes.c_double(0.0)
    n = ctypes.c_int64(0)
    _check(_lib.lora_timing_read(int(kernel), ctypes.byref(ms), ctypes.byref(n)), "lora_timing_read")
    return ms.value, n.value


def lora_launch_count() -> int:
    return int(_lib.lora_launch_count())


def lora_linear_fwd_noalloc(X, M: int, W: LoraWeight, A, B, r: int, s: float, Y, XA, stream=None) -> None:
    """Forward that allocates nothing and takes no workspace: for callers that are given
    only their input and output buffers and may not obtain other device memory.  Its
    scratch is a fixed 16 MiB array inside the library, shared by every call on a
    device, so calls must not overlap on the GPU (keep them on one stream)."""
    w = W.c_struct()
    _check(_lib.lora_linear_fwd_noalloc(_ptr(X), int(M), ctypes.byref(w), _ptr(A), _ptr(B), int(r), float(s),
                                        _ptr(Y), _ptr(XA), _stream(stream)), "lora_linear_fwd_noalloc")


def grouped_workspace_bytes(M: int, N: int, K: int, r: int, nseg: int, fmt: int = LORA_W_BF16) -> int:
    return int(_lib.lora_grouped_workspace_bytes(int(M), int(N), int(K), int(r), int(nseg), int(fmt)))


def lora_grouped_fwd(X, M: int, W: LoraWeight, rows, A, B, r: int, s: float, Y, XA, workspace, ws_bytes=None,
                     stream=None) -> None:
    """Forward of G projections sharing X (weights stacked along rows, see lora_linear.h)."""
    w = W.c_struct()
    seg = segments(rows)
    nb = workspace.numel() * workspace.element_size() if ws_bytes is None else ws_bytes
    _check(_lib.lora_grouped_fwd(_ptr(X), int(M), ctypes.byref(w), ctypes.byref(seg), _ptr(A), _ptr(B), int(r),
                                 float(s), _ptr(Y), _ptr(XA), _ptr(workspace), int(nb), _stream(stream)),
           "lora_grouped_fwd")


def lora_grouped_bwd(dY, X, XA, M: int, W: LoraWeight, rows, A, B, r: int, s: float, dX, dA, dB, workspace,
                     ws_bytes=None, stream=None) -> None:
    w = W.c_struct()
    seg = segments(rows)
    nb = workspace.numel() * workspace.element_size() if ws_bytes is None else ws_bytes
    _check(_lib.lora_grouped_bwd(_ptr(dY), _ptr(X), _ptr(XA), int(M), ctypes.byref(w), ctypes.byref(seg), _ptr(A),
                                 _ptr(B), int(r), float(s), _ptr(dX), _ptr(dA), _ptr(dB), _ptr(workspace), int(nb),
                                 _stream(stream)), "lora_grouped_bwd")


def lora_grouped_bwd_ex(dY, X, XA, M: int, W: LoraWeight, rows, A, B, r: int, s: float, dX, dA, dB, flags: int,
                        workspace, ws_bytes=None, stream=None) -> None:
    w = W.c_struct()
    seg = segments(rows)
    nb = workspace.numel() * workspace.element_size() if ws_bytes is None else ws_bytes
    _check(_lib.lora_grouped_bwd_ex(_ptr(dY), _ptr(X), _ptr(XA), int(M), ctypes.byref(w), ctypes.byref(seg),
                                    _ptr(A), _ptr(B), int(r), float(s), _ptr(dX), _ptr(dA), _ptr(dB), int(flags),
                                    _ptr(workspace), int(nb), _stream(stream)), "lora_grouped_bwd_ex")


def mlp_workspace_bytes(M: int, D: int, I: int, r: int, fmt: int = LORA_W_BF16) -> int:
    return int(_lib.lora_mlp_workspace_bytes(int(M), int(D), int(I), int(r), int(fmt)))


def mlp_struct(gate_up: LoraWeight, down: LoraWeight, A_gate_up, B_gate_up, A_down, B_down) -> lora_mlp_t:
    return lora_mlp_t(gate_up.c_struct(), down.c_struct(), _ptr(A_gate_up), _ptr(B_gate_up), _ptr(A_down),
                      _ptr(B_down))


def lora_mlp_fwd(X, M: int, mlp: lora_mlp_t, r: int, s: float, Z, GU, H, XA_gate_up, XA_down, workspace,
                 ws_bytes=None, stream=None) -> None:
    """Forward of the SwiGLU feed-forward block with LoRA on gate, up and down (see lora_linear.h)."""
    nb = workspace.numel() * workspace.element_size() if ws_bytes is None else ws_bytes
    _check(_lib.lora_mlp_fwd(_ptr(X), int(M), ctypes.byref(mlp), int(r), float(s), _ptr(Z), _ptr(GU), _ptr(H),
                             _ptr(XA_gate_up), _ptr(XA_down), _ptr(workspace), int(nb), _stream(stream)),
           "lora_mlp_fwd")


def lora_mlp_bwd(dZ, X, GU, H, XA_gate_up, XA_down, M: int, mlp: lora_mlp_t, r: int, s: float, dX, dA_gate_up,
                 dB_gate_up, dA_down, dB_down, workspace, ws_bytes=None, stream=None) -> None:
    """Backward of the block; GU (the forward's G | U) is overwritten with dG | dU."""
    nb = workspace.numel() * workspace.element_size() if ws_bytes is None else ws_bytes
    _check(_lib.lora_mlp_bwd(_ptr(dZ), _ptr(X), _ptr(GU), _ptr(H), _ptr(XA_gate_up), _ptr(XA_down), int(M),
                             ctypes.byref(mlp), int(r), float(s), _ptr(dX), _ptr(dA_gate_up), _ptr(dB_gate_up),
                             _ptr(dA_down), _ptr(dB_down), _ptr(workspace), int(nb), _stream(stream)),
           "lora_mlp_bwd")


def lora_mlp_bwd_ex(dZ, X, GU, H, XA_gate_up, XA_down, M: int, mlp: lora_mlp_t, r: int, s: float, dX, dA_gate_up,
                    dB_gate_up, dA_down, dB_down, flags: int, workspace, ws_bytes=None, stream=None) -> None:
    nb = workspace.numel() * workspace.element_size() if ws_bytes is None else ws_bytes
    _check(_lib.lora_mlp_bwd_ex(_ptr(dZ), _ptr(X), _ptr(GU), _ptr(H), _ptr(XA_gate_up), _ptr(XA_down), int(M),
                                ctypes.byref(mlp), int(r), float(s), _ptr(dX), _ptr(dA_gate_up), _ptr(dB_gate_up),
                                _ptr(dA_down), _ptr(dB_down), int(flags), _ptr(workspace), int(nb), _stream(stream)),
           "lora_mlp_bwd_ex")


def ce_workspace_bytes(M: int, D: int, V: int, slice_: int = 0) -> int:
    return int(_lib.lora_ce_workspace_bytes(int(M), int(D), int(V), int(slice_)))


def lora_ce_fwd(X, M: int, W: LoraWeight, labels, ignore_index: int, loss, lse, workspace, ws_bytes=None,
                stream=None) -> None:
    """Per-row cross-entropy of X·Wᵀ against labels, without the logits (see lora_linear.h)."""
    w = W.c_struct()
    nb = workspace.numel() * workspace.element_size() if ws_bytes is None else ws_bytes
    _check(_lib.lora_ce_fwd(_ptr(X), int(M), ctypes.byref(w), _ptr(labels), int(ignore_index), _ptr(loss),
                            _ptr(lse), _ptr(workspace), int(nb), _stream(stream)), "lora_ce_fwd")


def lora_ce_bwd(X, M: int, W: LoraWeight, labels, ignore_index: int, lse, dloss, dX, workspace, ws_bytes=None,
                stream=None) -> None:
    """Gradient of Σ dloss·loss in X, vocabulary slice by slice (slice size from the workspace)."""
    w = W.c_struct()
    nb = workspace.numel() * workspace.element_size() if ws_bytes is None else ws_bytes
    _check(_lib.lora_ce_bwd(_ptr(X), int(M), ctypes.byref(w), _ptr(labels), int(ignore_index), _ptr(lse),
                            _ptr(dloss), _ptr(dX), _ptr(workspace), int(nb), _stream(stream)), "lora_ce_bwd")
