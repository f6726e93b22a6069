"""Pins for the oracle's input activations (int8_linear(input_act=...),
comfy-kitchen 0.2.40 "HIP backend": the activation is folded into the fused
ConvRot quantiser's load). The pages do not list the activations; the ones
built are relu, silu x / (1 + e^-x) and the tanh form of gelu, each as the
bf16 value nearest to the exact act(x) of the bf16 input, then rotated.

What pins the oracle here, independently of it:
  * its float64 -> bf16 rounding against exact rational arithmetic
    (``fractions``), ties and subnormals included;
  * its activation of every finite bf16 input (all 65,280 of them) against a
    90-digit ``decimal`` evaluation of the formulas (pi from Machin's
    formula), rounded to bf16 with exact rationals; that evaluation also
    shows every input's exact value lies far from a rounding midpoint, so the
    bf16 result is unique;
  * relu against torch's, silu and gelu against torch's fp32-based bf16
    implementations (within one bf16 ulp), and the quantiser's wiring.
"""
from decimal import Decimal, localcontext
from fractions import Fraction
import struct

import numpy as np
import pytest
import torch

import oracle
import workloads

PREC = 90
GELU_C = Decimal("0.044715")


def _bits_to_float(b: int) -> float:
    return struct.unpack("<f", struct.pack("<I", (int(b) & 0xFFFF) << 16))[0]


def _float_to_bits(f: float) -> int:
    return struct.unpack("<I", struct.pack("<f", f))[0] >> 16


def _exact_bf16(v: Fraction) -> tuple[int, Fraction]:
    """Round an exact rational to bf16 (ties to even). Returns the bits and
    the distance of v from the nearest rounding midpoint, in units of the
    local spacing (0.5 means v sits on a representable value)."""
    neg = v < 0
    a = -v if neg else v
    sign = 0x8000 if neg else 0
    if a == 0:
        return sign, Fraction(1, 2)
    e = a.numerator.bit_length() - a.denominator.bit_length()
    # 2^(e-1) <= a < 2^e after the adjustment below
    while Fraction(2) ** e <= a:
        e += 1
    while Fraction(2) ** (e - 1) > a:
        e -= 1
    qe = max(e - 8, -133)
    n = a / Fraction(2) ** qe
    lo = n.numerator // n.denominator
    rem = n - lo
    if rem > Fraction(1, 2) or (rem == Fraction(1, 2) and lo % 2 == 1):
        lo += 1
    r = Fraction(lo) * Fraction(2) ** qe
    if r >= Fraction(2) ** 128:
        return sign | 0x7F80, abs(rem - Fraction(1, 2))
    return sign | _float_to_bits(float(r)), abs(rem - Fraction(1, 2))


# -------------------------------------------------------- float64 -> bf16


def _some_doubles():
    rng = np.random.default_rng(17)
    vals = list(rng.standard_normal(300) * np.exp2(rng.integers(-140, 130, 300)))
    for b in list(rng.integers(1, 0x7F7F, 200)) + [1, 2, 3, 0x7F, 0x80, 0x81, 0x7F7D, 0x7F7E]:
        x, y = _bits_to_float(b), _bits_to_float(b + 1)
        mid = (x + y) / 2  # exact in double
        ulp = np.spacing(mid)
        vals += [mid, mid + ulp, mid - ulp, x, -mid, -(mid + ulp)]
    vals += [0.0, -0.0, 2.0 ** -150, 2.0 ** -134, 3 * 2.0 ** -134, 2.0 ** -134 + 2.0 ** -200,
             3.3961775292304e38, 3.3961775292305e38, 3.40e38, 1e300, -1e300, 5e-324]
    return vals


def test_f64_to_bf16_is_exact_rounding():
    vals = _some_doubles()
    got = oracle.f64_to_bf16(np.array(vals, np.float64))
    for v, g in zip(vals, got):
        want, _ = _exact_bf16(Fraction(v))
        if v == 0.0 and np.signbit(v):
            want = 0x8000
        assert int(g) == want, (v, hex(int(g)), hex(want))


def test_f64_to_bf16_does_not_round_twice():
    # 1 + 2^-9 + 2^-30: fp32 would first round it to 1 + 2^-9 (a bf16 tie,
    # which goes to even: 1.0); the value itself lies above the midpoint
    v = 1.0 + 2.0 ** -9 + 2.0 ** -30
    assert int(oracle.f64_to_bf16(np.array([v]))[0]) == _float_to_bits(1.0 + 2.0 ** -8)


# -------------------------------------------------------- exact activations


def _pi() -> Decimal:
    """pi from Machin's formula 16 atan(1/5) - 4 atan(1/239)."""
    def atan_inv(n):
        x = Decimal(1) / n
        x2 = x * x
        term, total, k = x, x, 1
        while True:
            term *= -x2
            t = term / (2 * k + 1)
            if t == 0 or abs(t) < Decimal(10) ** (-PREC - 5):
                break
            total += t
            k += 1
        return total

    return 16 * atan_inv(5) - 4 * atan_inv(239)


def _exact_act(name: str, x: Decimal, sqrt2pi: Decimal) -> Decimal:
    if name == "silu":
        arg = -x
    else:
        u = sqrt2pi * (x + GELU_C * x * x * x)
        arg = -2 * u
    if arg > 100000:  # e^arg beyond any bf16 ratio: |act| < |x| e^-1e5
        return Decimal(0) * x.copy_sign(1) if x != 0 else Decimal(0)
    if arg < -100000:  # e^arg < e^-1e5: act(x) = x (1 - tiny)
        return x * (1 - Decimal(10) ** -40000)
    return x / (1 + arg.exp())


def _all_finite_bf16():
    b = np.arange(0x10000, dtype=np.uint32)
    finite = (b & 0x7F80) != 0x7F80
    return b[finite].astype(np.uint16)


@pytest.mark.parametrize("name", ["silu", "gelu_tanh"])
def test_every_bf16_input_matches_high_precision_evaluation(name):
    xs = _all_finite_bf16()
    got = oracle.act_bf16(name, xs)
    worst = Fraction(1, 2)
    with localcontext() as ctx:
        ctx.prec = PREC
        ctx.Emax = 10 ** 9
        ctx.Emin = -10 ** 9
        sqrt2pi = (Decimal(2) / _pi()).sqrt()
        for xb, g in zip(xs.tolist(), got.tolist()):
            x = Decimal(_bits_to_float(xb))
            v = _exact_act(name, x, sqrt2pi)
            want, dist = _exact_bf16(Fraction(v))
            if v == 0:
                want = 0x8000 if (xb & 0x8000) else 0
            assert g == want or (g & 0x7FFF) == (want & 0x7FFF) == 0, (hex(xb), hex(g), hex(want))
            worst = min(worst, dist)
    # every exact value lies far (relative to the 90-digit evaluation error)
    # from a rounding midpoint: the bf16 result is unique for every input
    assert worst > Fraction(1, 10 ** 60), float(worst)


def test_relu_every_input_equals_torch():
    xs = _all_finite_bf16()
    got = oracle.act_bf16("relu", xs)
    ref = workloads.bf16_bits(torch.relu(workloads.from_bf16_bits(xs)))
    same = (got == ref) | (((got & 0x7FFF) == 0) & ((ref & 0x7FFF) == 0))  # -0 vs +0
    assert same.all()


def test_tiny_inputs_round_up_from_half():
    # act(x) - x/2 > 0 for x != 0 and far below the subnormal spacing, so an
    # x/2 that is a midpoint rounds up: +min subnormal -> +min subnormal,
    # -min subnormal -> -0, 3 * min -> 2 * min, -3 * min -> -1 * min
    xs = np.array([0x0001, 0x8001, 0x0003, 0x8003, 0x0002, 0x8002], np.uint16)
    want = np.array([0x0001, 0x8000, 0x0002, 0x8001, 0x0001, 0x8001], np.uint16)
    for name in ("silu", "gelu_tanh"):
        assert np.array_equal(oracle.act_bf16(name, xs), want), name


def test_large_inputs_limits():
    big = np.array([_float_to_bits(200.0), _float_to_bits(-200.0), 0x7F7F, 0xFF7F], np.uint16)
    for name in ("silu", "gelu_tanh"):
        got = oracle.act_bf16(name, big)
        assert got[0] == big[0] and got[2] == big[2]  # act(x) = x (1 - tiny) -> x
        assert got[1] in (0x8000,) and got[3] == 0x8000  # |act| far below the smallest subnormal
    # silu(-90) = -90 e^-90 / (1 + e^-90) is a normal bf16 number, not 0
    s = oracle.act_bf16("silu", np.array([_float_to_bits(-90.0)], np.uint16))[0]
    assert abs(_bits_to_float(s) - (-90.0 * np.exp(-90.0))) <= 2.0 ** -8 * 90.0 * np.exp(-90.0)


@pytest.mark.parametrize("name", ["silu", "gelu_tanh"])
def test_closed_forms_far_from_and_near_zero(name):
    """Properties of the definitions over every bf16 input, which the
    quantiser's activation table relies on outside |x| in [2^-9, 2^7):
    act(x) = x (1 - e^-x / (1 + e^-x)) rounds to x for x >= 2^7 and to -0
    for x <= -2^7 (the exact value is below 2^-134 in magnitude there);
    act(x) = x / 2 + c x^2 + O(x^3), c = 1/4 (silu) or sqrt(2/pi)/2 (gelu),
    rounds to x / 2 for 2^-125 <= |x| < 2^-9, and act(+-0) = +-0."""
    h = np.arange(65536, dtype=np.uint32)
    got = oracle.act_bf16(name, h.astype(np.uint16)).astype(np.uint32)
    mag = h & 0x7FFF
    neg = (h & 0x8000) != 0
    big = (mag >= 0x4300) & (mag < 0x7F80)
    assert np.array_equal(got[big & ~neg], h[big & ~neg])
    assert (got[big & neg] == 0x8000).all()
    small = (mag >= 0x0100) & (mag < 0x3B00)
    assert np.array_equal(got[small], h[small] - 0x80)  # one less in the exponent field
    assert got[0] == 0x0000 and got[0x8000] == 0x8000
    # and they do not hold one binade further in: silu's large-|x| form
    # fails for some |x| in [2^6, 2^7), gelu's x / 2 for some |x| in
    # [2^-9, 2^-8)
    if name == "silu":
        far = (mag >= 0x4280) & (mag < 0x4300)
        assert (got[far] != np.where(neg[far], 0x8000, h[far])).any()
    else:
        near = (mag >= 0x3B00) & (mag < 0x3B80)
        assert (got[near] != h[near] - 0x80).any()


@pytest.mark.parametrize("name,fn", [
    ("silu", lambda t: torch.nn.functional.silu(t)),
    ("gelu_tanh", lambda t: torch.nn.functional.gelu(t, approximate="tanh")),
])
def test_bf16_activation_close_to_torch(name, fn):
    # torch evaluates in fp32 and rounds; its tanh-form gelu cancels to 0
    # below about x = -5, so compare where both are accurate
    rng = np.random.default_rng(3)
    xs = rng.standard_normal(20000).astype(np.float32) * 3
    x = torch.from_numpy(xs[xs > -4.0]).to(torch.bfloat16)
    mine = oracle.act_bf16(name, workloads.bf16_bits(x))
    theirs = workloads.bf16_bits(fn(x.float()).to(torch.bfloat16))
    d = np.abs(mine.astype(np.int32) - theirs.astype(np.int32))
    assert (d <= 1).all()
    assert (d != 0).mean() < 0.01


def test_act_f64_is_the_tanh_form():
    x = np.linspace(-3.0, 6.0, 2001)
    u = np.sqrt(2.0 / np.pi) * (x + 0.044715 * x ** 3)
    assert np.allclose(oracle.act_f64("gelu_tanh", x), 0.5 * x * (1.0 + np.tanh(u)),
                       rtol=1e-13, atol=1e-300)
    assert np.allclose(oracle.act_f64("silu", x), x / (1.0 + np.exp(-x)), rtol=1e-15, atol=0)


def test_quantize_with_relu_equals_quantize_of_torch_relu():
    cfg = workloads.custom(6, 768, 8, seed=9)
    X, _, _ = workloads.make_inputs(cfg)
    a = oracle.quantize_rows_bf16(workloads.bf16_bits(X), act="relu")
    b = oracle.quantize_rows_bf16(workloads.bf16_bits(torch.relu(X)))
    assert np.array_equal(a[0], b[0]) and np.array_equal(a[1], b[1])


@pytest.mark.parametrize("name", ["silu", "gelu_tanh"])
def test_quantize_with_act_equals_quantize_of_rounded_act(name):
    cfg = workloads.custom(5, 512, 8, seed=10)
    X, _, _ = workloads.make_inputs(cfg)
    a_bits = oracle.act_bf16(name, workloads.bf16_bits(X))
    a = oracle.quantize_rows_bf16(workloads.bf16_bits(X), act=name)
    b = oracle.quantize_rows_bf16(a_bits)
    assert np.array_equal(a[0], b[0]) and np.array_equal(a[1], b[1])
