"""Pins of the fp64 oracle against things other than itself (CPU only).

Each test checks an oracle function against brute force on tiny inputs, a closed
form, an invariant of the mathematics, or an independent library routine, chosen so
that a dropped term, a wrong sign or index, a transposed operand or a wrong scale
fails at least one of them.
"""
from fractions import Fraction

import numpy as np
import pytest
import torch

import oracle as O
from synth import bf16_bits_from_f32, f32_from_bf16_bits
from synth.inputs import codebook_levels


# ---------------------------------------------------------------------------
# brute force on tiny integer inputs (exact rational arithmetic, pure Python)
# ---------------------------------------------------------------------------

def _bf_matmul(a, b):
    return [[sum(a[i][t] * b[t][j] for t in range(len(b))) for j in range(len(b[0]))]
            for i in range(len(a))]


def _bf_T(a):
    return [list(r) for r in zip(*a)]


def _bf_layer(X, W, A, B, dY, s):
    """Forward and backward by the definition, with Python Fractions, one loop nest
    per product, no numpy."""
    M, K, N, r = len(X), len(X[0]), len(W), len(A)
    # Y[m][n] = sum_k X[m][k] W[n][k] + s * sum_j (sum_k X[m][k] A[j][k]) B[n][j]
    XA = [[sum(X[m][k] * A[j][k] for k in range(K)) for j in range(r)] for m in range(M)]
    Y = [[sum(X[m][k] * W[n][k] for k in range(K)) + s * sum(XA[m][j] * B[n][j] for j in range(r))
          for n in range(N)] for m in range(M)]
    # L = sum_{m,n} dY[m][n] Y[m][n]; gradients of L by the chain rule written per element
    dX = [[sum(dY[m][n] * (W[n][k] + s * sum(B[n][j] * A[j][k] for j in range(r)))
               for n in range(N)) for k in range(K)] for m in range(M)]
    dA = [[sum(dY[m][n] * s * B[n][j] * X[m][k] for m in range(M) for n in range(N))
           for k in range(K)] for j in range(r)]
    dB = [[sum(dY[m][n] * s * XA[m][j] for m in range(M)) for j in range(r)] for n in range(N)]
    return Y, XA, dX, dA, dB


def _ints(rng, shape, lo=-4, hi=5):
    return rng.integers(lo, hi, size=shape).astype(np.int64)


@pytest.mark.parametrize("alpha", [3, 16])
def test_layer_matches_brute_force_exactly(alpha):
    rng = np.random.default_rng(11)
    M, K, N, r = 3, 5, 4, 2
    X, W, A, B, dY = (_ints(rng, s) for s in [(M, K), (N, K), (r, K), (N, r), (M, N)])
    s = Fraction(alpha, r)
    Yb, XAb, dXb, dAb, dBb = _bf_layer(*(t.tolist() for t in (X, W, A, B, dY)), s)
    Y, XA = O.lora_forward(X, W, A, B, float(s))
    g = O.lora_backward(dY, X, W, A, B, float(s))
    # small integers and s = alpha/2: every value is exact in fp64
    assert np.array_equal(Y, np.array(Yb, dtype=np.float64))
    assert np.array_equal(XA, np.array(XAb, dtype=np.float64))
    assert np.array_equal(g["dX"], np.array(dXb, dtype=np.float64))
    assert np.array_equal(g["dA"], np.array(dAb, dtype=np.float64))
    assert np.array_equal(g["dB"], np.array(dBb, dtype=np.float64))
    assert np.array_equal(g["XA"], XA)


def test_brute_force_helper_is_a_plain_matmul():
    # the brute-force forward reduces to a plain product when the adapter is zero
    rng = np.random.default_rng(3)
    X, W = _ints(rng, (2, 3)), _ints(rng, (4, 3))
    Z = [[0, 0]] * 4
    Yb = _bf_layer(X.tolist(), W.tolist(), [[0, 0, 0]] * 2, Z, [[0] * 4] * 2, 1)[0]
    assert Yb == _bf_matmul(X.tolist(), _bf_T(W.tolist()))


# ---------------------------------------------------------------------------
# invariants on random fp64 inputs
# ---------------------------------------------------------------------------

def _rand(rng, M=37, K=48, N=29, r=6):
    X = rng.standard_normal((M, K))
    W = rng.standard_normal((N, K)) / np.sqrt(K)
    A = rng.uniform(-1, 1, (r, K)) / np.sqrt(K)
    B = rng.standard_normal((N, r)) * 0.1
    dY = rng.standard_normal((M, N))
    return X, W, A, B, dY


def _rel(a, b):
    return np.linalg.norm(a - b) / max(np.linalg.norm(b), 1e-300)


def test_associativity_and_merge_invariant():
    """Bracketed forward equals the unbracketed X·(W + s·B·A)ᵀ, which is also X
    times the merged weight."""
    rng = np.random.default_rng(5)
    X, W, A, B, dY = _rand(rng)
    s = 2.5
    Y, _ = O.lora_forward(X, W, A, B, s)
    naive = X @ (W + s * (B @ A)).T
    assert _rel(Y, naive) <= 1e-12
    assert _rel(X @ O.lora_merge(W, A, B, s).T, naive) <= 1e-12
    # the merged weight against its definition element by element
    Wm = O.lora_merge(W, A, B, s)
    n, k = 7, 11
    assert abs(Wm[n, k] - (W[n, k] + s * sum(B[n, j] * A[j, k] for j in range(A.shape[0])))) < 1e-13


def test_b_zero_reduces_to_plain_linear():
    rng = np.random.default_rng(6)
    X, W, A, B, dY = _rand(rng)
    B0 = np.zeros_like(B)
    s = 2.0
    Y, XA = O.lora_forward(X, W, A, B0, s)
    g = O.lora_backward(dY, X, W, A, B0, s)
    assert np.array_equal(Y, X @ W.T)
    assert np.array_equal(g["dX"], dY @ W)
    assert np.array_equal(g["dA"], np.zeros_like(A))
    # dB does not vanish: it is s·dYᵀ·XA
    assert np.linalg.norm(g["dB"]) > 0
    assert _rel(g["dB"], s * np.einsum("mn,mj->nj", dY, X @ A.T)) <= 1e-12
    # merge with B = 0 gives W back exactly
    assert np.array_equal(O.lora_merge(W, A, B0, s), W)


def test_w_zero_leaves_the_low_rank_path():
    rng = np.random.default_rng(7)
    X, W, A, B, dY = _rand(rng)
    s = 0.75
    Y, _ = O.lora_forward(X, np.zeros_like(W), A, B, s)
    assert _rel(Y, X @ (s * B @ A).T) <= 1e-12
    g = O.lora_backward(dY, X, np.zeros_like(W), A, B, s)
    assert _rel(g["dX"], dY @ (s * B @ A)) <= 1e-12


def test_finite_differences():
    """L = Σ dY ⊙ Y is linear in X, in A and in B separately, so central
    differences are exact up to fp64 round-off."""
    rng = np.random.default_rng(8)
    M, K, N, r = 3, 5, 4, 2
    X, W, A, B, dY = _rand(rng, M, K, N, r)
    s = 1.7
    g = O.lora_backward(dY, X, W, A, B, s)

    def L(X_, A_, B_):
        return float(np.sum(dY * O.lora_forward(X_, W, A_, B_, s)[0]))

    h = 1e-3
    for name, T, grad in (("X", X, g["dX"]), ("A", A, g["dA"]), ("B", B, g["dB"])):
        fd = np.zeros_like(T)
        for idx in np.ndindex(T.shape):
            Tp, Tm = T.copy(), T.copy()
            Tp[idx] += h
            Tm[idx] -= h
            args_p = {"X": X, "A": A, "B": B}
            args_m = dict(args_p)
            args_p[name], args_m[name] = Tp, Tm
            fd[idx] = (L(args_p["X"], args_p["A"], args_p["B"]) - L(args_m["X"], args_m["A"], args_m["B"])) / (2 * h)
        assert _rel(fd, grad) <= 1e-9, name


def test_row_sampled_versions_match_full():
    rng = np.random.default_rng(9)
    X, W, A, B, dY = _rand(rng)
    s = 2.0
    Y, XA = O.lora_forward(X, W, A, B, s)
    g = O.lora_backward(dY, X, W, A, B, s)
    rows = np.array([0, 5, 17, 36])
    Yr, XAr = O.lora_forward_rows(X[rows], W, A, B, s)
    assert _rel(Yr, Y[rows]) <= 1e-14 and _rel(XAr, XA[rows]) <= 1e-14
    assert _rel(O.lora_backward_rows(dY[rows], W, A, B, s), g["dX"][rows]) <= 1e-13


# ---------------------------------------------------------------------------
# storage types and the 4-bit format
# ---------------------------------------------------------------------------

def _bf16_nearest_even_fraction(x: float) -> float:
    """Nearest bf16 to x (a normal float32) by exact rational comparison of the two
    neighbouring 8-significant-bit values; ties go to the even significand."""
    f = Fraction(x)
    sign = -1 if f < 0 else 1
    f = abs(f)
    e = 0
    while f >= 2:
        f /= 2
        e += 1
    while f < 1:
        f *= 2
        e -= 1
    lo = Fraction(int(f * 128), 128)
    hi = lo + Fraction(1, 128)
    dlo, dhi = f - lo, hi - f
    if dlo < dhi or (dlo == dhi and int(lo * 128) % 2 == 0):
        q = lo
    else:
        q = hi
    return float(sign * q * Fraction(2) ** e)


def test_bf16_rounding_against_exact_rationals_and_torch():
    rng = np.random.default_rng(10)
    x = (rng.standard_normal(4000) * np.exp(rng.uniform(-20, 20, 4000))).astype(np.float32)
    # exact ties: 1 + 2^-8 -> 1 (even), 1 + 3·2^-8 -> 1 + 2^-6 (even), negatives too
    ties = np.array([1 + 2 ** -8, 1 + 3 * 2 ** -8, -(1 + 2 ** -8), 3 * (1 + 2 ** -8), 0.0],
                    dtype=np.float32)
    x = np.concatenate([x, ties])
    bits = O.bf16_round_bits(x)
    got = f32_from_bf16_bits(bits).astype(np.float64)
    want = np.array([_bf16_nearest_even_fraction(float(v)) if v != 0 else 0.0 for v in x])
    assert np.array_equal(got, want)
    # an independent library path: torch's float32 -> bfloat16 conversion
    tb = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(bits, tb)
    # the input generator's rounding agrees as well
    assert np.array_equal(bits, bf16_bits_from_f32(x))


def test_codebook_levels_are_correctly_rounded():
    cb = codebook_levels()
    assert cb.dtype == np.float32 and cb.shape == (16,)
    for i, v in enumerate(cb):
        exact = Fraction(2 * i - 15, 15)
        # float32 neighbours of the exact level bracket it and v is the nearer one
        below = np.nextafter(v, np.float32(-np.inf))
        above = np.nextafter(v, np.float32(np.inf))
        assert abs(Fraction(float(v)) - exact) <= abs(Fraction(float(below)) - exact)
        assert abs(Fraction(float(v)) - exact) <= abs(Fraction(float(above)) - exact)
    assert cb[0] == -1 and cb[15] == 1 and np.array_equal(cb, -cb[::-1])


def test_dequant_hand_example_nibble_order_and_blocks():
    """Two rows of 128 elements: byte j holds element 2j in its low nibble; each row
    has two 64-element blocks with their own scale."""
    N, K = 2, 128
    cb = codebook_levels()
    codes = np.zeros((N, K // 2), dtype=np.uint8)
    codes[0, 0] = 0x2F  # element 0 -> code 15 (+1.0), element 1 -> code 2 (-11/15)
    codes[1, 40] = 0x70  # row 1, element 80 -> code 0 (-1.0), element 81 -> code 7 (-1/15)
    scales = np.array([2.0, 4.0, 0.5, 8.0], dtype=np.float16)
    bits = O.dequant_blockwise4(codes, scales.view(np.uint16), cb, N, K)
    v = f32_from_bf16_bits(bits)
    assert v[0, 0] == np.float32(2.0) * cb[15] == 2.0
    want01 = f32_from_bf16_bits(bf16_bits_from_f32(np.float32(cb[2]) * np.float32(2.0)))
    assert v[0, 1] == want01
    assert v[0, 64] == f32_from_bf16_bits(bf16_bits_from_f32(np.float32(cb[0]) * np.float32(4.0)))
    assert v[1, 80] == -8.0  # block 3 (row 1, second half), scale 8, level -1
    assert v[1, 81] == f32_from_bf16_bits(bf16_bits_from_f32(cb[7] * np.float32(8.0)))
    assert v[1, 0] == f32_from_bf16_bits(bf16_bits_from_f32(cb[0] * np.float32(0.5)))


def test_dequant_against_torch_float32_product():
    """Library cross-check: torch multiplies the fp32 level by the fp32 scale and
    converts to bf16; the oracle's fp64 path must land on the same bits."""
    rng = np.random.default_rng(12)
    N, K = 64, 256
    codes = rng.integers(0, 256, (N, K // 2), dtype=np.uint8)
    scales = rng.uniform(1e-3, 30.0, N * K // 64).astype(np.float16)
    cb = codebook_levels()
    bits = O.dequant_blockwise4(codes, scales.view(np.uint16), cb, N, K)
    c = np.empty((N, K), dtype=np.int64)
    c[:, 0::2] = codes & 15
    c[:, 1::2] = codes >> 4
    lv = torch.from_numpy(cb)[torch.from_numpy(c)]
    sc = torch.from_numpy(scales.astype(np.float32)).repeat_interleave(64).reshape(N, K)
    tb = (lv * sc).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(bits, tb)


def test_codebook_round_trip_exhaustive():
    """For every code and every positive normal fp16 scale, dequantizing and taking
    the nearest level under the same scale gives the code back."""
    cb = codebook_levels()
    e = np.arange(1, 31, dtype=np.uint16)
    m = np.arange(0, 1024, dtype=np.uint16)
    sbits = ((e[:, None] << np.uint16(10)) | m[None, :]).reshape(-1)  # all positive normals
    nS = sbits.size
    for c in range(16):
        # one block of 64 per scale, every element carrying code c
        byte = np.uint8(c | (c << 4))
        codes = np.full((nS, 32), byte, dtype=np.uint8)
        bits = O.dequant_blockwise4(codes, sbits, cb, nS, 64)
        vals = O.bf16_to_f64(bits)
        back = O.nearest_codes(vals, O.fp16_to_f64(sbits), cb)
        assert np.all(back == c), c


def test_requantize_is_idempotent():
    rng = np.random.default_rng(13)
    N, K = 32, 192
    W = rng.standard_normal((N, K)) / np.sqrt(K)
    cb = codebook_levels()
    q1, s1 = O.quantize_blockwise4(W, cb)
    W1 = O.bf16_to_f64(O.dequant_blockwise4(q1, s1, cb, N, K))
    q2, s2 = O.quantize_blockwise4(W1, cb)
    W2 = O.bf16_to_f64(O.dequant_blockwise4(q2, s2, cb, N, K))
    q3, s3 = O.quantize_blockwise4(W2, cb)
    assert np.array_equal(q2, q3) and np.array_equal(s2, s3)
    assert np.array_equal(W2, O.bf16_to_f64(O.dequant_blockwise4(q3, s3, cb, N, K)))
    # quantization error is bounded by half a level spacing times the scale plus rounding
    err = np.abs(W1 - W).reshape(-1, 64).max(axis=1)
    assert np.all(err <= (1 / 15 + 2 ** -7) * O.fp16_to_f64(s1) + 1e-12)


def test_zero_block_takes_code_seven():
    cb = codebook_levels()
    W = np.zeros((1, 64))
    q, s = O.quantize_blockwise4(W, cb)
    assert np.all(q == 0x77) and s[0] == 0
    # level -1/15 times a zero scale is IEEE negative zero
    d = O.dequant_blockwise4(q, s, cb, 1, 64)
    assert np.all(O.bf16_to_f64(d) == 0.0) and np.all(d == 0x8000)


def test_sampled_adapter_grads_match_full_backward():
    """The chunked, sampled dA/dB helper agrees with the full backward (chunk size
    smaller than M and not dividing it)."""
    rng = np.random.default_rng(14)
    M, K, N, r = 50, 40, 24, 8
    X = bf16_bits_from_f32(rng.standard_normal((M, K)).astype(np.float32))
    dY = bf16_bits_from_f32(rng.standard_normal((M, N)).astype(np.float32))
    W = rng.standard_normal((N, K))
    A = rng.uniform(-0.2, 0.2, (r, K))
    B = rng.standard_normal((N, r)) * 0.1
    s = 3.0
    g = O.lora_backward(O.bf16_to_f64(dY), O.bf16_to_f64(X), W, A, B, s)
    n_idx = np.array([0, 3, 23])
    k_idx = np.array([1, 39, 7])
    dB_s, dA_s = O.lora_adapter_grads_sampled(dY, X, A, B, s, n_idx, k_idx, chunk_rows=7)
    assert _rel(dB_s, g["dB"][n_idx]) <= 1e-13
    assert _rel(dA_s, g["dA"][:, k_idx]) <= 1e-13


# ---------------------------------------------------------------------------
# grouped projections sharing X (fused q/k/v)
# ---------------------------------------------------------------------------

def _grouped(rng, M=9, K=12, Ns=(8, 4, 4), r=3):
    X = rng.standard_normal((M, K))
    Ws = [rng.standard_normal((n, K)) / np.sqrt(K) for n in Ns]
    As = [rng.uniform(-1, 1, (r, K)) / np.sqrt(K) for _ in Ns]
    Bs = [rng.standard_normal((n, r)) * 0.1 for n in Ns]
    dY = rng.standard_normal((M, sum(Ns)))
    return X, Ws, As, Bs, dY


def test_grouped_equals_one_layer_with_block_diagonal_adapter():
    """Stacking the weights and the A's and putting the B's on the diagonal of one
    [ΣN, G·r] matrix turns the G projections into one LoRA linear of rank G·r: same Y,
    same dX, and the diagonal blocks of its dB / the stacked dA are the per-projection
    gradients."""
    rng = np.random.default_rng(21)
    X, Ws, As, Bs, dY = _grouped(rng)
    s = 1.5
    Wall, Aall = np.concatenate(Ws), np.concatenate(As)
    r, Ns = As[0].shape[0], [W.shape[0] for W in Ws]
    Bbd = np.zeros((sum(Ns), r * len(Ns)))
    o = 0
    for g, B in enumerate(Bs):
        Bbd[o:o + Ns[g], g * r:(g + 1) * r] = B
        o += Ns[g]
    Y, XA = O.lora_grouped_forward(X, Ws, As, Bs, s)
    Y1, XA1 = O.lora_forward(X, Wall, Aall, Bbd, s)
    assert _rel(Y, Y1) <= 1e-13 and _rel(XA, XA1) <= 1e-13
    g = O.lora_grouped_backward(dY, X, Ws, As, Bs, s)
    g1 = O.lora_backward(dY, X, Wall, Aall, Bbd, s)
    assert _rel(g["dX"], g1["dX"]) <= 1e-13
    assert _rel(g["dA"], g1["dA"]) <= 1e-13
    o = 0
    for q in range(len(Ns)):
        assert _rel(g["dB"][o:o + Ns[q]], g1["dB"][o:o + Ns[q], q * r:(q + 1) * r]) <= 1e-13
        o += Ns[q]


def test_grouped_finite_differences():
    rng = np.random.default_rng(22)
    X, Ws, As, Bs, dY = _grouped(rng, M=3, K=4, Ns=(2, 3), r=2)
    s = 0.7
    g = O.lora_grouped_backward(dY, X, Ws, As, Bs, s)

    def L(X_, As_, Bs_):
        return float(np.sum(dY * O.lora_grouped_forward(X_, Ws, As_, Bs_, s)[0]))

    h = 1e-3
    fd = np.zeros_like(X)
    for idx in np.ndindex(X.shape):
        Xp, Xm = X.copy(), X.copy()
        Xp[idx] += h
        Xm[idx] -= h
        fd[idx] = (L(Xp, As, Bs) - L(Xm, As, Bs)) / (2 * h)
    assert _rel(fd, g["dX"]) <= 1e-9
    for q in range(2):
        for name, T in (("A", As[q]), ("B", Bs[q])):
            fdT = np.zeros_like(T)
            for idx in np.ndindex(T.shape):
                Tp, Tm = T.copy(), T.copy()
                Tp[idx] += h
                Tm[idx] -= h
                Ap, Am = list(As), list(As)
                Bp, Bm = list(Bs), list(Bs)
                if name == "A":
                    Ap[q], Am[q] = Tp, Tm
                else:
                    Bp[q], Bm[q] = Tp, Tm
                fdT[idx] = (L(X, Ap, Bp) - L(X, Am, Bm)) / (2 * h)
            r = As[0].shape[0]
            want = g["dA"][q * r:(q + 1) * r] if name == "A" else g["dB"][sum(W.shape[0] for W in Ws[:q]):][:Ws[q].shape[0]]
            assert _rel(fdT, want) <= 1e-9, (name, q)


# ---------------------------------------------------------------- feed-forward block


def test_sigmoid_closed_forms_and_symmetry():
    """sigmoid(0) = 1/2, sigmoid(±ln 3) = 3/4 and 1/4 exactly (1/(1+1/3)); no overflow at
    ±800; sigmoid(x) + sigmoid(-x) = 1; silu(g) = g·sigmoid(g) follows."""
    ln3 = np.log(3.0)
    got = O.sigmoid(np.array([0.0, ln3, -ln3, 800.0, -800.0]))
    assert got[0] == 0.5
    assert abs(got[1] - 0.75) <= 2e-16 and abs(got[2] - 0.25) <= 2e-16
    assert got[3] == 1.0 and 0.0 <= got[4] < 1e-300
    x = np.linspace(-30, 30, 1001)
    assert np.max(np.abs(O.sigmoid(x) + O.sigmoid(-x) - 1.0)) <= np.finfo(np.float64).eps  # one ulp of 1
    H = O.swiglu_forward(np.array([ln3, 0.0, -ln3]), np.array([2.0, 5.0, 4.0]))
    assert np.allclose(H, [0.75 * ln3 * 2.0, 0.0, -0.25 * ln3 * 4.0], rtol=0, atol=1e-15)


def test_swiglu_backward_against_torch_autograd():
    """The hand-derived dG, dU equal torch's autograd of F.silu(G)·U in float64."""
    rng = np.random.default_rng(31)
    G = rng.standard_normal((7, 11)) * 3
    U = rng.standard_normal((7, 11))
    dH = rng.standard_normal((7, 11))
    tg = torch.tensor(G, requires_grad=True)
    tu = torch.tensor(U, requires_grad=True)
    th = torch.nn.functional.silu(tg) * tu
    th.backward(torch.tensor(dH))
    assert _rel(O.swiglu_forward(G, U), th.detach().numpy()) <= 1e-15
    dG, dU = O.swiglu_backward(dH, G, U)
    assert _rel(dG, tg.grad.numpy()) <= 1e-14
    assert _rel(dU, tu.grad.numpy()) <= 1e-14


def _mlp(rng, M=6, D=10, I=7, r=3):
    X = rng.standard_normal((M, D))
    W_gu = rng.standard_normal((2 * I, D)) / np.sqrt(D)
    A_gu = rng.uniform(-1, 1, (2 * r, D)) / np.sqrt(D)
    B_gu = rng.standard_normal((2 * I, r)) * 0.3
    W_d = rng.standard_normal((D, I)) / np.sqrt(I)
    A_d = rng.uniform(-1, 1, (r, I)) / np.sqrt(I)
    B_d = rng.standard_normal((D, r)) * 0.3
    dZ = rng.standard_normal((M, D))
    return X, W_gu, A_gu, B_gu, W_d, A_d, B_d, dZ


def test_mlp_block_against_torch_autograd():
    """Forward against the block written with torch's own linear and silu; every gradient
    against torch's autograd of it (float64), so the chain rule is checked by a
    derivation other than the oracle's."""
    rng = np.random.default_rng(32)
    X, W_gu, A_gu, B_gu, W_d, A_d, B_d, dZ = _mlp(rng)
    s = 1.25
    I, r = W_d.shape[1], A_d.shape[0]
    t = {k: torch.tensor(v, requires_grad=True) for k, v in
         dict(X=X, A_gu=A_gu, B_gu=B_gu, A_d=A_d, B_d=B_d).items()}
    F = torch.nn.functional

    def lin(x, W, A, B):
        return F.linear(x, torch.tensor(W)) + s * F.linear(F.linear(x, A), B)

    G = lin(t["X"], W_gu[:I], t["A_gu"][:r], t["B_gu"][:I])
    U = lin(t["X"], W_gu[I:], t["A_gu"][r:], t["B_gu"][I:])
    Z = lin(F.silu(G) * U, W_d, t["A_d"], t["B_d"])
    Z.backward(torch.tensor(dZ))
    f = O.lora_mlp_forward(X, W_gu, A_gu, B_gu, W_d, A_d, B_d, s)
    assert _rel(f["Z"], Z.detach().numpy()) <= 1e-14
    g = O.lora_mlp_backward(dZ, X, W_gu, A_gu, B_gu, W_d, A_d, B_d, s)
    for k in ("X", "A_gu", "B_gu", "A_d", "B_d"):
        assert _rel(g["d" + k], t[k].grad.numpy()) <= 1e-13, k


def test_mlp_finite_differences():
    rng = np.random.default_rng(33)
    X, W_gu, A_gu, B_gu, W_d, A_d, B_d, dZ = _mlp(rng, M=3, D=4, I=3, r=2)
    s = 0.8
    g = O.lora_mlp_backward(dZ, X, W_gu, A_gu, B_gu, W_d, A_d, B_d, s)
    args = dict(X=X, A_gu=A_gu, B_gu=B_gu, A_d=A_d, B_d=B_d)

    def L(**kw):
        a = dict(args, **kw)
        return float(np.sum(dZ * O.lora_mlp_forward(a["X"], W_gu, a["A_gu"], a["B_gu"], W_d, a["A_d"], a["B_d"],
                                                      s)["Z"]))

    h = 1e-4
    for name, T in args.items():
        fd = np.zeros_like(T)
        for idx in np.ndindex(T.shape):
            Tp, Tm = T.copy(), T.copy()
            Tp[idx] += h
            Tm[idx] -= h
            fd[idx] = (L(**{name: Tp}) - L(**{name: Tm})) / (2 * h)
        assert _rel(fd, g["d" + name]) <= 1e-7, name


def test_mlp_zero_adapters_give_the_plain_block():
    """With every B zero (the adapter's initial state) the block is the plain SwiGLU
    feed-forward, silu from torch; the A gradients are exactly zero."""
    rng = np.random.default_rng(34)
    X, W_gu, A_gu, B_gu, W_d, A_d, B_d, dZ = _mlp(rng)
    B_gu, B_d = np.zeros_like(B_gu), np.zeros_like(B_d)
    I = W_d.shape[1]
    f = O.lora_mlp_forward(X, W_gu, A_gu, B_gu, W_d, A_d, B_d, 2.0)
    G, U = X @ W_gu[:I].T, X @ W_gu[I:].T
    H = torch.nn.functional.silu(torch.tensor(G)).numpy() * U
    assert _rel(f["Z"], H @ W_d.T) <= 1e-14
    g = O.lora_mlp_backward(dZ, X, W_gu, A_gu, B_gu, W_d, A_d, B_d, 2.0)
    assert np.all(g["dA_gu"] == 0) and np.all(g["dA_d"] == 0)
    assert np.any(g["dB_gu"] != 0) and np.any(g["dB_d"] != 0)


# ---------------------------------------------------------------- 8-bit formats


def test_e4m3_decode_against_torch_and_closed_forms():
    c = np.arange(256, dtype=np.uint8)
    v = O.e4m3_value(c)
    t = torch.from_numpy(c.copy()).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    assert np.array_equal(np.isnan(v), np.isnan(t))
    assert np.array_equal(v[~np.isnan(v)], t[~np.isnan(t)])
    assert v[0x38] == 1.0 and v[0x7E] == 448.0 and v[0x01] == 2.0 ** -9 and v[0x08] == 2.0 ** -6
    assert v[0x80] == 0.0 and np.signbit(v[0x80]) and v[0xB8] == -1.0
    assert np.isnan(v[0x7F]) and np.isnan(v[0xFF]) and np.sum(np.isnan(v)) == 2


def test_int8_decode_closed_forms():
    v = O.int8_value(np.array([0x00, 0x01, 0x7F, 0x80, 0xFF, 0xFE], dtype=np.uint8))
    assert list(v) == [0.0, 1.0, 127.0, -128.0, -1.0, -2.0]


def test_dequant_rowwise8_hand_example():
    """int8 codes [[1, -2], [127, 0]] with row scales [0.5, 3]: 0.5, -1, 381 -> 380 (a tie
    between the bf16 neighbours 380 and 382 goes to the even mantissa), 0."""
    codes = np.array([[1, 0xFE], [127, 0]], dtype=np.uint8)
    got = O.bf16_to_f64(O.dequant_rowwise8(codes, np.array([0.5, 3.0], dtype=np.float32), "int8"))
    assert got.tolist() == [[0.5, -1.0], [380.0, 0.0]]
    # fp8: 0x38 = 1.0 and 0xC4 = -(1 + 4/8)·2^1 = -3.0 at scale 0.25
    got = O.bf16_to_f64(O.dequant_rowwise8(np.array([[0x38, 0xC4]], dtype=np.uint8),
                                           np.array([0.25], dtype=np.float32), "fp8"))
    assert got.tolist() == [[0.25, -0.75]]


@pytest.mark.parametrize("fmt", ["int8", "fp8"])
def test_dequant_rowwise8_against_torch(fmt):
    """Bit-exact against torch: decode (int8 / float8_e4m3fn dtype), float32 multiply by
    the row scale, bf16 cast."""
    rng = np.random.default_rng(41)
    N, K = 37, 96
    codes = rng.integers(0, 256, (N, K), dtype=np.uint8)
    if fmt == "fp8":
        codes[(codes & 0x7F) == 0x7F] = 0x10  # no NaN codes
    scale = (rng.random(N) * 0.01 + 1e-4).astype(np.float32)
    tc = torch.from_numpy(codes.copy())
    val = (tc.view(torch.int8) if fmt == "int8" else tc.view(torch.float8_e4m3fn)).to(torch.float32)
    ref = (val * torch.from_numpy(scale)[:, None]).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(O.dequant_rowwise8(codes, scale, fmt), ref)


def test_e4m3_nearest_round_trip_ties_and_torch():
    finite = [c for c in range(256) if c not in (0x7F, 0xFF)]
    v = O.e4m3_value(np.array(finite, dtype=np.uint8))
    assert np.array_equal(O.e4m3_nearest(v), np.array(finite, dtype=np.uint8))  # every code back, -0 included
    # midpoints go to the even mantissa
    assert O.e4m3_nearest(np.array([1.0625, 1.1875, -1.0625]))[:].tolist() == [0x38, 0x3A, 0xB8]
    x = np.linspace(-448, 448, 20001)
    t = torch.from_numpy(x).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(O.e4m3_nearest(x), t)


@pytest.mark.parametrize("fmt", ["int8", "fp8"])
def test_quantize_rowwise8_round_trip_and_bound(fmt):
    """Rows that hold the extreme code (127 or 448) quantize back to the same codes and
    scales exactly; a random weight dequantizes within half a step of the format."""
    rng = np.random.default_rng(42)
    N, K = 16, 64
    if fmt == "int8":
        codes = rng.integers(-127, 128, (N, K)).astype(np.int8).view(np.uint8)
        codes[:, 3] = 127
    else:
        codes = rng.integers(0, 256, (N, K), dtype=np.uint8)
        codes[(codes & 0x7F) == 0x7F] = 0x33
        codes[:, 3] = 0x7E
    scale = (rng.random(N) + 0.5).astype(np.float32)
    from oracle.lora_oracle import code8_value
    W = code8_value(codes, fmt) * scale.astype(np.float64)[:, None]
    c2, s2 = O.quantize_rowwise8(W, fmt)
    assert np.array_equal(s2, scale)
    assert np.array_equal(code8_value(c2, fmt), code8_value(codes, fmt))
    Wr = rng.standard_normal((N, K))
    c3, s3 = O.quantize_rowwise8(Wr, fmt)
    err = np.abs(code8_value(c3, fmt) * s3.astype(np.float64)[:, None] - Wr)
    if fmt == "int8":
        assert np.all(err <= 0.5 * s3[:, None] * (1 + 1e-6))
    else:  # half a spacing of e4m3 at the value's binade, 2^-4 relative, plus the subnormal step
        assert np.all(err <= np.abs(Wr) * 2.0 ** -4 + s3[:, None] * 2.0 ** -10)


# ---------------------------------------------------------------- cross-entropy over an LM head


def _ce_inputs(rng, M=9, D=12, V=37):
    X = rng.standard_normal((M, D))
    W = rng.standard_normal((V, D)) / np.sqrt(D) * 2
    y = rng.integers(0, V, M)
    y[[1, min(5, M - 1)]] = -100
    dloss = rng.random(M) + 0.5
    return X, W, y, dloss


def test_cross_entropy_against_torch():
    """Loss against torch's cross_entropy (float64, no reduction, ignore_index) and dX
    against torch's autograd of the dloss-weighted sum of the losses."""
    rng = np.random.default_rng(51)
    X, W, y, dloss = _ce_inputs(rng)
    loss, lse, dX = O.cross_entropy(X, W, y, -100, dloss)
    tX = torch.tensor(X, requires_grad=True)
    tl = torch.nn.functional.cross_entropy(tX @ torch.tensor(W).T, torch.tensor(y), ignore_index=-100,
                                           reduction="none")
    assert _rel(loss, tl.detach().numpy()) <= 1e-14
    (tl * torch.tensor(dloss)).sum().backward()
    assert _rel(dX, tX.grad.numpy()) <= 1e-13
    assert _rel(lse, torch.logsumexp(torch.tensor(X @ W.T), dim=1).numpy()) <= 1e-15
    assert np.all(loss[[1, 5]] == 0) and np.all(dX[[1, 5]] == 0)


def test_cross_entropy_uniform_logits_and_finite_differences():
    rng = np.random.default_rng(52)
    X, W, y, dloss = _ce_inputs(rng)
    loss, lse, dX = O.cross_entropy(X, np.zeros_like(W), y, -100, dloss)
    V = W.shape[0]
    assert np.allclose(lse, np.log(V), rtol=0, atol=1e-15)
    assert np.allclose(loss[y != -100], np.log(V), rtol=0, atol=1e-15)
    assert np.all(dX == 0)
    X, W, y, dloss = _ce_inputs(rng, M=4, D=5, V=7)
    _, _, dX = O.cross_entropy(X, W, y, -100, dloss)
    h = 1e-5
    fd = np.zeros_like(X)
    for idx in np.ndindex(X.shape):
        Xp, Xm = X.copy(), X.copy()
        Xp[idx] += h
        Xm[idx] -= h
        fd[idx] = (np.sum(dloss * O.cross_entropy(Xp, W, y, -100)[0]) -
                   np.sum(dloss * O.cross_entropy(Xm, W, y, -100)[0])) / (2 * h)
    assert _rel(fd, dX) <= 1e-8


def test_cross_entropy_rows_helper_matches_full():
    rng = np.random.default_rng(53)
    M, D, V = 6, 16, 1000
    Xb = bf16_bits_from_f32(rng.standard_normal((M, D)).astype(np.float32))
    Wb = bf16_bits_from_f32((rng.standard_normal((V, D)) / 4).astype(np.float32))
    y = rng.integers(0, V, M)
    y[2] = -1
    dloss = rng.random(M)
    full = O.cross_entropy(O.bf16_to_f64(Xb), O.bf16_to_f64(Wb), y, -1, dloss)
    rows = O.cross_entropy_rows_bits(Xb, Wb, y, -1, dloss, chunk=97)
    for a, b in zip(full, rows):
        assert _rel(a, b) <= 1e-13
