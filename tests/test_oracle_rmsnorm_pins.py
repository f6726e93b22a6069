"""Pins for the oracle's input RMSNorm and residual (CPU, independent of the oracle).

Source: comfy-kitchen 0.2.40 (PyPI page), "Huawei Ascend backend": int8_linear
accepts the input RMSNorm and residual arguments and applies them with shared
device-side helpers apart from the GEMM. The page prints no formula; the
reading (the oracle's input RMSNorm section) is the add-then-normalise form:
h = bf16(x + r) as a bf16 tensor addition stores it, and y = the bf16 value
nearest to the exact h g / sqrt(mean(h^2) + eps). Elements whose exact value
lies within 2^-34 (relative) of a rounding midpoint accept either neighbour
(the oracle reports the other one in Yalt).

What pins it here: PyTorch's bf16 addition (an independent implementation
of the residual add); an exact evaluation of y (rational sum of squares,
60-digit decimal square root, exact rational rounding to bf16) on rows of
several scales; the honesty of the Yalt flags (an exact midpoint and a value
2^-41 below one are flagged, values far from midpoints are not); closed
forms on constant and two-valued rows; exact power-of-two invariance; the
unit weight; zero rows.
"""
from decimal import Decimal, localcontext
from fractions import Fraction
import struct

import numpy as np
import pytest
import torch

import oracle
import workloads


def _bits(t):
    return workloads.bf16_bits(t)


def _val(bits):
    return workloads.from_bf16_bits(bits).double()


def _f(b: int) -> float:
    return struct.unpack("<f", struct.pack("<I", (int(b) & 0xFFFF) << 16))[0]


def _to_bits(f: float) -> int:
    return struct.unpack("<I", struct.pack("<f", f))[0] >> 16


def _rows(M, K, seed, scale=1.0):
    g = torch.Generator().manual_seed(seed)
    X = (torch.randn(M, K, generator=g) * scale).to(torch.bfloat16)
    R = (torch.randn(M, K, generator=g) * scale).to(torch.bfloat16)
    w = (1.0 + 0.25 * torch.randn(K, generator=g)).to(torch.bfloat16)
    return X, R, w


def _round_exact(v: Fraction):
    """bf16 rounding of an exact rational (ties to even), and the distance of
    v from the nearest midpoint relative to |v|."""
    neg = v < 0
    a = -v if neg else v
    if a == 0:
        return 0, Fraction(1)
    e = a.numerator.bit_length() - a.denominator.bit_length()
    while Fraction(2) ** e <= a:
        e += 1
    while Fraction(2) ** (e - 1) > a:
        e -= 1
    q = Fraction(2) ** max(e - 8, -133)
    n = a / q
    lo = n.numerator // n.denominator
    rem = n - lo
    mid_dist = abs(rem - Fraction(1, 2)) * q / a
    if rem > Fraction(1, 2) or (rem == Fraction(1, 2) and lo % 2 == 1):
        lo += 1
    r = float(lo * q)
    return (0x8000 if neg else 0) | _to_bits(r), mid_dist


def _exact_rows(H_bits, g_bits, eps):
    """y of every element from its definition: the sum of squares as an exact
    rational, the square root at 60 digits, the rounding exact."""
    M, K = H_bits.shape
    out = np.zeros((M, K), np.uint16)
    dist = np.zeros((M, K), np.float64)
    with localcontext() as ctx:
        ctx.prec = 60
        for m in range(M):
            h = [Fraction(_f(b)) for b in H_bits[m].tolist()]
            ss = sum(v * v for v in h)
            t = ss / K + Fraction(float(eps))
            root = (Decimal(t.numerator) / Decimal(t.denominator)).sqrt()
            inv = Fraction(1) / Fraction(root)
            for k in range(K):
                gk = Fraction(_f(g_bits[k])) if g_bits is not None else Fraction(1)
                out[m, k], d = _round_exact(h[k] * gk * inv)
                dist[m, k] = float(d)
    return out, dist


@pytest.mark.parametrize("M,K,seed", [(5, 256, 1), (7, 768, 2), (3, 5376, 3)])
def test_residual_add_is_torch_bf16_add(M, K, seed):
    X, R, w = _rows(M, K, seed)
    _, H = oracle.rmsnorm_rows(_bits(X), _bits(R), _bits(w), 1e-6)
    assert np.array_equal(H, _bits(X + R))  # torch adds bf16 in fp32 and rounds once
    _, H0 = oracle.rmsnorm_rows(_bits(X), None, _bits(w), 1e-6)
    assert np.array_equal(H0, _bits(X))


@pytest.mark.parametrize("M,K,seed,eps,scale,with_g", [
    (3, 512, 4, 1e-6, 1.0, True), (2, 5376, 5, 1e-5, 30.0, True), (3, 1024, 6, 1.0, 0.5, False),
    (2, 256, 7, 1e-6, 1e-3, True), (2, 768, 8, 1e-6, 2.0 ** -70, True)])
def test_matches_exact_evaluation(M, K, seed, eps, scale, with_g):
    X, R, w = _rows(M, K, seed, scale)
    gb = _bits(w) if with_g else None
    Y, H, Ya = oracle.rmsnorm_rows(_bits(X), _bits(R), gb, eps, with_alt=True)
    want, dist = _exact_rows(H, gb, np.float32(eps))
    flagged = Ya != Y
    # the exact value's rounding wherever the oracle raises no flag
    assert np.array_equal(Y[~flagged], want[~flagged])
    # flags only near midpoints, and both neighbours offered there
    assert np.all(dist[flagged] <= 2.0 ** -33)
    assert np.all((want[flagged] == Y[flagged]) | (want[flagged] == Ya[flagged]))
    assert np.all(dist[~flagged] >= 2.0 ** -35)


def test_midpoint_values_are_flagged():
    # a row whose mean of squares is exactly 1: h0 = 1.5, 63 values 2, one 1,
    # three 0.5, the rest 0 (2.25 + 252 + 1 + 0.75 = 256 = K). With
    # g0 = 1 + 2^-7, h0 g0 = 1.51171875 is the midpoint of bf16 1.5078125 and
    # 1.515625: exactly on it (eps = 0), and 2^-41 below it (eps = 2^-40)
    K = 256
    h = np.zeros(K, np.float32)
    h[0] = 1.5
    h[1:64] = 2.0
    h[64] = 1.0
    h[65:68] = 0.5
    X = torch.from_numpy(h[None, :]).to(torch.bfloat16)
    g = torch.ones(K, dtype=torch.bfloat16)
    g[0] = 1.0 + 2.0 ** -7
    lo, hi = _to_bits(1.5078125), _to_bits(1.515625)
    Y, _, Ya = oracle.rmsnorm_rows(_bits(X), None, _bits(g), 0.0, with_alt=True)
    assert (Y[0, 0], Ya[0, 0]) == (hi, lo)  # a tie: even first, the other offered
    Y, _, Ya = oracle.rmsnorm_rows(_bits(X), None, _bits(g), 2.0 ** -40, with_alt=True)
    assert {int(Y[0, 0]), int(Ya[0, 0])} == {lo, hi} and Y[0, 0] == lo  # just below it
    assert np.array_equal(Y[0, 1:], Ya[0, 1:])


def test_constant_rows_closed_form():
    K = 512
    X = torch.full((2, K), 2.0, dtype=torch.bfloat16)
    X[1] = -0.5
    Y, _ = oracle.rmsnorm_rows(_bits(X), None, None, 0.0)
    # mean of squares = c^2, so y = c / |c| = sign(c) exactly
    assert np.all(_val(Y)[0].numpy() == 1.0) and np.all(_val(Y)[1].numpy() == -1.0)
    w = (torch.arange(K) % 7 - 3).to(torch.bfloat16)
    Yw, _ = oracle.rmsnorm_rows(_bits(X), None, _bits(w), 0.0)
    assert np.array_equal(Yw[0], _bits(w)) and np.array_equal(Yw[1], _bits(-w))


def test_two_valued_rows_closed_form():
    # half the row 3, half 4: mean of squares 12.5, y = v / sqrt(12.5) =
    # 0.8485281... and 1.1313708..., rounded: 0.84765625 and 1.1328125
    K = 1024
    X = torch.full((1, K), 3.0, dtype=torch.bfloat16)
    X[0, 1::2] = 4.0
    Y, _ = oracle.rmsnorm_rows(_bits(X), None, None, 0.0)
    assert np.all(Y[0, 0::2] == _to_bits(0.84765625))
    assert np.all(Y[0, 1::2] == _to_bits(1.1328125))


@pytest.mark.parametrize("k", [-20, -3, 5, 40])
def test_power_of_two_invariance(k):
    X, R, w = _rows(4, 768, 11)
    Y, _ = oracle.rmsnorm_rows(_bits(X), _bits(R), _bits(w), 0.0)
    Ys, Hs = oracle.rmsnorm_rows(_bits(X * 2.0 ** k), _bits(R * 2.0 ** k), _bits(w), 0.0)
    assert np.array_equal(Y, Ys)
    assert np.array_equal(Hs, _bits((X + R) * 2.0 ** k))


def test_close_to_float64_formula():
    X, R, w = _rows(6, 512, 4)
    Y, _ = oracle.rmsnorm_rows(_bits(X), _bits(R), _bits(w), 1e-6)
    h = (X + R).double()
    ref = h / torch.sqrt((h * h).mean(-1, keepdim=True) + np.float32(1e-6)) * w.double()
    assert torch.all((_val(Y) - ref).abs() <= ref.abs() * 2.0 ** -8 + 1e-30)


def test_unit_weight_equals_no_weight():
    X, R, _ = _rows(3, 512, 12)
    ones = torch.ones(512, dtype=torch.bfloat16)
    a, _ = oracle.rmsnorm_rows(_bits(X), _bits(R), _bits(ones), 1e-6)
    b, _ = oracle.rmsnorm_rows(_bits(X), _bits(R), None, 1e-6)
    assert np.array_equal(a, b)


def test_zero_row_with_eps_is_zero():
    Z = torch.zeros((2, 256), dtype=torch.bfloat16)
    Y, H = oracle.rmsnorm_rows(_bits(Z), None, None, 1e-6)
    assert not Y.any() and not H.any()
