"""The C-ABI library loads, exports every symbol the headers declare, and validates
arguments on the host before touching the GPU (no device needed for these)."""
import ctypes
import glob
import os
import re

import pytest

import qlora_linear_b200 as q
from qlora_linear_b200.binding import lora_weight_t

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

# fake, never dereferenced device addresses (validation runs before any CUDA call)
P = 0x10000
P2 = 0x20000


def _declared_functions():
    names = set()
    for h in glob.glob(os.path.join(ROOT, "include", "*.h")):
        src = open(h).read()
        src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
        for m in re.finditer(r"^[A-Za-z_][\w\s\*]*?\b(\w+)\s*\(", src, flags=re.M):
            if m.group(1) not in ("if", "defined"):
                names.add(m.group(1))
    return names


def test_library_exports_every_declared_symbol():
    declared = _declared_functions()
    assert {"lora_linear_fwd", "lora_linear_bwd", "dequant_blockwise4", "lora_merge",
            "lora_workspace_bytes", "lora_device_status", "lora_status_string"} <= declared
    lib = ctypes.CDLL(q.LIB_PATH)
    for name in sorted(declared):
        assert hasattr(lib, name), name
    assert set(q.EXPORTED) == declared


def test_status_strings_and_version():
    for code in range(7):
        assert q.status_string(code)
    assert q.status_string(99) == "unknown status"
    assert q.lib().lora_version() >= 100


def _w(fmt=0, N=512, K=512, data=P, absmax=P, cb=P):
    return lora_weight_t(fmt, 0, N, K, data, absmax, cb)


def fwd(W, M=256, r=8, s=2.0, X=P, A=P, B=P, Y=P, XA=P, ws=P2, nb=1 << 30):
    return q.lib().lora_linear_fwd(X, M, ctypes.byref(W) if W is not None else None, A, B, r, s, Y, XA, ws, nb, None)


def bwd(W, M=256, r=8, s=2.0, dY=P, X=P, XA=P, A=P, B=P, dX=P, dA=P, dB=P, ws=P2, nb=1 << 30):
    return q.lib().lora_linear_bwd(dY, X, XA, M, ctypes.byref(W) if W is not None else None, A, B, r, s, dX, dA, dB,
                                   ws, nb, None)


@pytest.mark.parametrize("call", [fwd, bwd])
def test_host_validation_errors(call):
    assert call(None) == q.LORA_ERR_INVALID_ARG
    assert call(_w(fmt=7)) == q.LORA_ERR_INVALID_ARG
    assert call(_w(N=0)) == q.LORA_ERR_INVALID_ARG
    assert call(_w(K=-8)) == q.LORA_ERR_INVALID_ARG
    assert call(_w(data=0)) == q.LORA_ERR_INVALID_ARG
    assert call(_w(data=P + 8)) == q.LORA_ERR_ALIGNMENT
    assert call(_w(N=513)) == q.LORA_ERR_UNSUPPORTED
    assert call(_w(K=516)) == q.LORA_ERR_UNSUPPORTED
    assert call(_w(fmt=1, K=520)) == q.LORA_ERR_UNSUPPORTED       # 4-bit needs K % 64
    assert call(_w(fmt=1, absmax=0)) == q.LORA_ERR_INVALID_ARG
    assert call(_w(fmt=1, cb=P + 4)) == q.LORA_ERR_ALIGNMENT
    for f8 in (2, 3):                                               # 8-bit: K % 16, fp32 row scales
        assert call(_w(fmt=f8, K=520)) == q.LORA_ERR_UNSUPPORTED
        assert call(_w(fmt=f8, absmax=0)) == q.LORA_ERR_INVALID_ARG
        assert call(_w(fmt=f8, absmax=P + 4)) == q.LORA_ERR_ALIGNMENT
    assert call(_w(fmt=4)) == q.LORA_ERR_INVALID_ARG
    for r in (0, 4, 12, 136, 256):
        assert call(_w(), r=r) == q.LORA_ERR_UNSUPPORTED, r
    assert call(_w(), s=float("nan")) == q.LORA_ERR_INVALID_ARG
    assert call(_w(), s=float("inf")) == q.LORA_ERR_INVALID_ARG
    assert call(_w(), M=-1) == q.LORA_ERR_INVALID_ARG
    assert call(_w(), A=0) == q.LORA_ERR_INVALID_ARG
    assert call(_w(), B=P + 2) == q.LORA_ERR_ALIGNMENT
    assert call(_w(), ws=0) == q.LORA_ERR_WORKSPACE
    assert call(_w(), ws=P2 + 4) == q.LORA_ERR_ALIGNMENT
    assert call(_w(), nb=q.workspace_bytes(256, 512, 512, 8) - 1) == q.LORA_ERR_WORKSPACE


def test_forward_specific_validation():
    assert fwd(_w(), X=0) == q.LORA_ERR_INVALID_ARG
    assert fwd(_w(), Y=P + 6) == q.LORA_ERR_ALIGNMENT
    assert fwd(_w(), XA=0) == q.LORA_ERR_INVALID_ARG
    # an empty batch is valid and enqueues nothing
    assert fwd(_w(), M=0, X=0, Y=0, XA=0, ws=0, nb=0) == q.LORA_OK


def test_backward_specific_validation():
    assert bwd(_w(), dY=0) == q.LORA_ERR_INVALID_ARG
    assert bwd(_w(), dA=0) == q.LORA_ERR_INVALID_ARG
    assert bwd(_w(), dB=P + 2) == q.LORA_ERR_ALIGNMENT
    assert bwd(_w(), dX=P + 2) == q.LORA_ERR_ALIGNMENT


def test_dequant_and_merge_validation():
    lib = q.lib()
    assert lib.dequant_blockwise4(ctypes.byref(_w(fmt=0)), P, None) == q.LORA_ERR_INVALID_ARG
    assert lib.dequant_blockwise4(ctypes.byref(_w(fmt=1)), 0, None) == q.LORA_ERR_INVALID_ARG
    assert lib.dequant_blockwise4(ctypes.byref(_w(fmt=1)), P + 2, None) == q.LORA_ERR_ALIGNMENT
    assert lib.lora_merge(ctypes.byref(_w()), P, P, 12, 2.0, P, None) == q.LORA_ERR_UNSUPPORTED
    assert lib.lora_merge(ctypes.byref(_w()), P, P, 8, float("nan"), P, None) == q.LORA_ERR_INVALID_ARG
    # a 4-bit merge whose output overlaps the packed codes is rejected
    assert lib.lora_merge(ctypes.byref(_w(fmt=1, data=P)), P2, P2, 8, 2.0, P, None) == q.LORA_ERR_INVALID_ARG


def test_workspace_bytes_is_a_pure_function_of_sizes():
    a = q.workspace_bytes(16384, 14336, 4096, 16)
    assert a == q.workspace_bytes(16384, 14336, 4096, 16, q.LORA_W_BLOCK4)
    assert a >= 256 + 16384 * 16 * 2
    assert q.workspace_bytes(0, 512, 512, 8) >= 256
    assert q.workspace_bytes(256, 512, 512, 7) == 0
    assert q.workspace_bytes(256, 0, 512, 8) == 0
    assert q.workspace_bytes(256, 512, 512, 8, 5) == 0
    # grows with M; holds the rank-r operand s·XA (the fp32 partials of the passes at r <= 16,
    # which run on the TMA stream with a blocking of their own, can outweigh it)
    assert q.workspace_bytes(512, 4096, 4096, 16) < q.workspace_bytes(4096, 4096, 4096, 16)
    assert q.workspace_bytes(4096, 4096, 4096, 128) >= 256 + 4096 * 128 * 2
    assert q.workspace_bytes(4096, 4096, 4096, 16) >= 256 + 4096 * 16 * 2


def test_gemm_streamk_only_where_the_last_wave_leaves_pairs_idle():
    k = q.lora_testing_gemm_streamk
    B4, I8 = q.LORA_W_BLOCK4, q.LORA_W_INT8
    # the rank sweep's 512-token shapes with quantized weights: 32 tiles of 512 x 256 for
    # 74 CTA pairs, all shared out as pieces; 112 tiles: one wave whole, 38 as pieces
    assert k(512, 8192, 8192, 16, B4) == 32 and k(512, 28672, 8192, 16, B4) == 112 - 74
    assert k(512, 8192, 28672, 16, B4) == 32 and k(512, 8192, 8192, 16, I8) == 32
    # the QLoRA dX GEMM: 256 tiles = 3.46 waves; three waves whole, the last 34 tiles as
    # pieces (fewer fp32 slots than cutting the third wave too)
    assert k(8192, 4096, 14336, 16, B4) == 256 - 222
    # the QLoRA Y GEMM: 896 tiles = 12.1 waves; the 8 tiles of the partial wave as pieces
    assert k(8192, 14336, 4096, 16, B4) == 8
    # bf16 at 512 tokens and N = 28672: 224 tiles, 76 as pieces; N = 8192: 64 tiles, whole
    assert k(512, 28672, 8192, 16) == 76 and k(512, 8192, 8192, 16) == 0
    # many waves, or too little work per pair: whole tiles
    assert k(16384, 14336, 4096, 16) == 0 and k(16384, 4096, 14336, 16) == 0 and k(8192, 4096, 4096, 16) == 0
    assert k(256, 512, 512, 8) == 0
    assert k(512, 8192, 8192, 16, 9) == -1 and k(512, 8192, 8192, 129, 0) == -1
    # the workspace holds the schedule's fp32 slots: two tiles of 512 x 256 per pair
    assert q.workspace_bytes(512, 8192, 8192, 16, B4) >= 256 + 2 * 74 * 512 * 256 * 4
    assert q.workspace_bytes(512, 8192, 8192, 16) < 512 * 8192 * 4


def test_grouped_validation():
    from qlora_linear_b200.binding import segments
    lib = q.lib()
    W = _w(N=6144, K=512)

    def gf(rows, r=16, nseg_ptr=True):
        seg = segments(rows) if nseg_ptr else None
        return lib.lora_grouped_fwd(P, 256, ctypes.byref(W), ctypes.byref(seg) if seg else None, P, P, r, 2.0, P, P,
                                    P2, 1 << 30, None)

    assert gf([4096, 1024, 1024], nseg_ptr=False) == q.LORA_ERR_INVALID_ARG
    assert gf([4096, 1024, 1000]) == q.LORA_ERR_INVALID_ARG          # rows do not add up to N
    assert gf([4000, 1024, 1120]) == q.LORA_ERR_UNSUPPORTED          # boundary not on 256 rows
    assert gf([4096, 1024, 1024], r=48) == q.LORA_ERR_UNSUPPORTED    # G·r > 128
    assert gf([6144, 0]) == q.LORA_ERR_INVALID_ARG
    seg = segments([4096, 1024, 1024])
    seg.reserved = 1
    assert lib.lora_grouped_fwd(P, 256, ctypes.byref(W), ctypes.byref(seg), P, P, 16, 2.0, P, P, P2, 1 << 30,
                                None) == q.LORA_ERR_INVALID_ARG
    # the workspace grows with the number of projections and is zero when G·r > 128
    assert q.grouped_workspace_bytes(4096, 6144, 4096, 16, 3) > q.workspace_bytes(4096, 6144, 4096, 16)
    assert q.grouped_workspace_bytes(4096, 6144, 4096, 16, 1) == q.workspace_bytes(4096, 6144, 4096, 16)
    assert q.grouped_workspace_bytes(4096, 6144, 4096, 48, 3) == 0


def test_mlp_validation():
    lib = q.lib()
    D, I, r = 512, 1024, 16

    def mlp(**kw):
        gu = _w(N=2 * I, K=D)
        dn = _w(N=D, K=I)
        m = q.lora_mlp_t(gu, dn, P, P, P, P)
        for k, v in kw.items():
            setattr(m, k, v)
        return m

    def fwd(m, r=r, M=256, X=P):
        return lib.lora_mlp_fwd(X, M, ctypes.byref(m), r, 2.0, P, P, P, P, P, P2, 1 << 30, None)

    assert lib.lora_mlp_fwd(P, 256, None, r, 2.0, P, P, P, P, P, P2, 1 << 30, None) == q.LORA_ERR_INVALID_ARG
    assert fwd(mlp(down=_w(N=D + 8, K=I))) == q.LORA_ERR_INVALID_ARG      # down rows != D
    assert fwd(mlp(down=_w(N=D, K=I - 8))) == q.LORA_ERR_INVALID_ARG      # gate_up rows != 2I
    assert fwd(mlp(), r=72) == q.LORA_ERR_UNSUPPORTED                     # 2r > 128
    assert fwd(mlp(), r=12) == q.LORA_ERR_UNSUPPORTED
    assert fwd(mlp(A_down=None)) == q.LORA_ERR_INVALID_ARG
    assert fwd(mlp(B_gate_up=P + 2)) == q.LORA_ERR_ALIGNMENT
    assert fwd(mlp(), M=0, X=None) == q.LORA_OK                            # empty batch: nothing to do
    assert fwd(mlp(), X=None) == q.LORA_ERR_INVALID_ARG
    assert lib.lora_mlp_fwd(P, 256, ctypes.byref(mlp()), r, 2.0, P, P, P, P, P, P2, 1000, None) == \
        q.LORA_ERR_WORKSPACE
    assert q.mlp_workspace_bytes(4096, D, I, r) > 0
    assert q.mlp_workspace_bytes(4096, D, I, 72) == 0


def test_dequant_validation():
    lib = q.lib()
    assert lib.lora_dequant(None, P2, None) == q.LORA_ERR_INVALID_ARG
    assert lib.lora_dequant(ctypes.byref(_w(fmt=2)), 0, None) == q.LORA_ERR_INVALID_ARG
    assert lib.lora_dequant(ctypes.byref(_w(fmt=3)), P2 + 2, None) == q.LORA_ERR_ALIGNMENT
    # the output may not overlap the stored codes
    assert lib.lora_dequant(ctypes.byref(_w(fmt=2, data=P)), P + 256, None) == q.LORA_ERR_INVALID_ARG
    assert lib.lora_dequant(ctypes.byref(_w(fmt=0, data=P)), P, None) == q.LORA_ERR_INVALID_ARG
    assert q.workspace_bytes(4096, 4096, 4096, 16, q.LORA_W_INT8) == q.workspace_bytes(4096, 4096, 4096, 16)
    assert q.workspace_bytes(4096, 4096, 4096, 16, 4) == 0


def test_ce_validation():
    lib = q.lib()
    W = _w(N=1000, K=256)

    def fwd(W=W, M=64, X=P, labels=P, loss=P, lse=P, ws=P2, nb=1 << 30):
        return lib.lora_ce_fwd(X, M, ctypes.byref(W) if W is not None else None, labels, -100, loss, lse, ws, nb, None)

    def bwd(W=W, M=64, nb=1 << 30, dX=P):
        return lib.lora_ce_bwd(P, M, ctypes.byref(W), P, -100, P, P, dX, P2, nb, None)

    assert fwd(W=None) == q.LORA_ERR_INVALID_ARG
    assert fwd(W=_w(fmt=1, N=1000, K=256)) == q.LORA_ERR_UNSUPPORTED   # the head is bf16
    assert fwd(labels=0) == q.LORA_ERR_INVALID_ARG
    assert fwd(loss=P + 4) == q.LORA_ERR_ALIGNMENT
    assert fwd(M=-1) == q.LORA_ERR_INVALID_ARG
    assert fwd(M=0, X=0, labels=0) == q.LORA_OK
    assert fwd(nb=100) == q.LORA_ERR_WORKSPACE
    assert bwd(dX=0) == q.LORA_ERR_INVALID_ARG
    # room for fewer than 256 vocabulary columns of dlogits beside the fp32 dX sum
    fixed = q.ce_workspace_bytes(64, 256, 1000, 256) - 64 * 256 * 2
    assert bwd(nb=fixed + 64 * 255 * 2) == q.LORA_ERR_WORKSPACE
    assert q.ce_workspace_bytes(64, 256, 1000, 512) > q.ce_workspace_bytes(64, 256, 1000, 256)
    assert q.ce_workspace_bytes(64, 256, 1000, 0) == q.ce_workspace_bytes(64, 256, 1000, 1024)


def bwd_ex(W, flags=1, M=256, r=8, s=2.0, dY=P, X=P, XA=P, A=P, B=P, dX=P, dA=P, dB=P, ws=P2, nb=1 << 30):
    return q.lib().lora_linear_bwd_ex(dY, X, XA, M, ctypes.byref(W) if W is not None else None, A, B, r, s, dX, dA,
                                      dB, flags, ws, nb, None)


def test_fp32_gradient_entries_validate_like_the_plain_ones():
    # the same host checks as lora_linear_bwd, with fp32 or bf16 gradients
    for flags in (0, q.LORA_GRADS_F32):
        assert bwd_ex(None, flags) == q.LORA_ERR_INVALID_ARG
        assert bwd_ex(_w(N=513), flags) == q.LORA_ERR_UNSUPPORTED
        assert bwd_ex(_w(), flags, dA=0) == q.LORA_ERR_INVALID_ARG
        assert bwd_ex(_w(), flags, dB=P + 4) == q.LORA_ERR_ALIGNMENT
        assert bwd_ex(_w(), flags, ws=0) == q.LORA_ERR_WORKSPACE
    # unknown flag bits are rejected before anything else
    for bad in (2, 4, 0x80000000, 3):
        assert bwd_ex(_w(), bad) == q.LORA_ERR_INVALID_ARG, bad
    lib = q.lib()
    seg = q.segments([256, 256])
    assert lib.lora_grouped_bwd_ex(P, P, P, 256, ctypes.byref(_w()), ctypes.byref(seg), P, P, 8, 2.0, P, P, P, 2,
                                   P2, 1 << 30, None) == q.LORA_ERR_INVALID_ARG
    assert lib.lora_grouped_bwd_ex(P, P, P, 256, ctypes.byref(_w()), None, P, P, 8, 2.0, P, P, P, 1,
                                   P2, 1 << 30, None) == q.LORA_ERR_INVALID_ARG
    m = q.mlp_struct(q.LoraWeight(1024, 512, P), q.LoraWeight(512, 512, P), P, P, P, P)
    assert lib.lora_mlp_bwd_ex(P, P, P, P, P, P, 256, ctypes.byref(m), 8, 2.0, P, P, P, P, P, 8, P2, 1 << 30,
                               None) == q.LORA_ERR_INVALID_ARG


def test_round_bf16_validation():
    lib = q.lib()
    assert lib.lora_round_bf16(P, P2, -1, None) == q.LORA_ERR_INVALID_ARG
    assert lib.lora_round_bf16(0, P2, 16, None) == q.LORA_ERR_INVALID_ARG
    assert lib.lora_round_bf16(P + 4, P2, 16, None) == q.LORA_ERR_ALIGNMENT
    assert lib.lora_round_bf16(P, P2 + 8, 16, None) == q.LORA_ERR_ALIGNMENT
    assert lib.lora_round_bf16(P, P + 16, 16, None) == q.LORA_ERR_INVALID_ARG  # output overlaps the input
    assert lib.lora_round_bf16(0, 0, 0, None) == q.LORA_OK  # nothing to do, nothing enqueued
