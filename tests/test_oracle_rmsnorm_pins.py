"""Pins for the oracle's input RMSNorm and residual (CPU, independent of the oracle).

Source: comfy-kitchen 0.2.40 (PyPI page), "Huawei Ascend backend": int8_linear
accepts the input RMSNorm and residual arguments and applies them with shared
device-side helpers apart from the GEMM. The page prints no formula; the
reading (the oracle's input RMSNorm section) is the add-then-normalise form
h = bf16(x + r), y = bf16((h / sqrt(mean(h^2) + eps)) * g). What pins it here:
PyTorch's bf16 addition (an independent implementation of the residual add),
the float64 formula on the rounded h within half a bf16 ulp plus the fp32
error, closed forms on constant and two-valued rows, exact power-of-two
invariance, and the unit weight.
"""
import numpy as np
import pytest
import torch

import oracle
import workloads


def _bits(t):
    return workloads.bf16_bits(t)


def _val(bits):
    return workloads.from_bf16_bits(bits).double()


def _rows(M, K, seed, scale=1.0):
    g = torch.Generator().manual_seed(seed)
    X = (torch.randn(M, K, generator=g) * scale).to(torch.bfloat16)
    R = (torch.randn(M, K, generator=g) * scale).to(torch.bfloat16)
    w = (1.0 + 0.25 * torch.randn(K, generator=g)).to(torch.bfloat16)
    return X, R, w


@pytest.mark.parametrize("M,K,seed", [(5, 256, 1), (7, 768, 2), (3, 5376, 3)])
def test_residual_add_is_torch_bf16_add(M, K, seed):
    X, R, w = _rows(M, K, seed)
    _, H = oracle.rmsnorm_rows(_bits(X), _bits(R), _bits(w), 1e-6)
    assert np.array_equal(H, _bits(X + R))  # torch adds bf16 in fp32 and rounds once
    _, H0 = oracle.rmsnorm_rows(_bits(X), None, _bits(w), 1e-6)
    assert np.array_equal(H0, _bits(X))


@pytest.mark.parametrize("M,K,seed,eps,scale", [(6, 512, 4, 1e-6, 1.0), (4, 5376, 5, 1e-5, 30.0),
                                                (5, 1024, 6, 1.0, 0.5), (3, 256, 7, 1e-6, 1e-3)])
def test_matches_float64_formula_on_the_rounded_sum(M, K, seed, eps, scale):
    X, R, w = _rows(M, K, seed, scale)
    Y, _ = oracle.rmsnorm_rows(_bits(X), _bits(R), _bits(w), eps)
    h = (X + R).double()
    ref = h / torch.sqrt((h * h).mean(-1, keepdim=True) + eps) * w.double()
    y = _val(Y)
    # half a bf16 ulp of the fp32 value (at most 2^-8 of it: 8 significant
    # bits), plus the fp32 steps (K terms of the sum, the division, sqrt and
    # two products), relative
    tol = ref.abs() * (2.0 ** -8 * (1 + 2.0 ** -7) + (K + 8) * 2.0 ** -24) + 1e-30
    assert torch.all((y - ref).abs() <= tol)


def test_constant_rows_closed_form():
    K = 512
    X = torch.full((2, K), 2.0, dtype=torch.bfloat16)
    X[1] = -0.5
    Y, _ = oracle.rmsnorm_rows(_bits(X), None, None, 0.0)
    # ss = K c^2 exactly, mean = c^2, inv = 1/|c| exactly: y = sign(c)
    assert np.all(_val(Y)[0].numpy() == 1.0) and np.all(_val(Y)[1].numpy() == -1.0)
    w = (torch.arange(K) % 7 - 3).to(torch.bfloat16)
    Yw, _ = oracle.rmsnorm_rows(_bits(X), None, _bits(w), 0.0)
    assert np.array_equal(Yw[0], _bits(w)) and np.array_equal(Yw[1], _bits(-w))


def test_two_valued_rows_closed_form():
    # half the row 3, half 4 (interleaved by blocks of 8): mean of squares
    # 12.5, inv = 1/sqrt(12.5) (IEEE), y = bf16(v * inv)
    K = 1024
    X = torch.full((1, K), 3.0, dtype=torch.bfloat16)
    X[0, 8::16] = 4.0
    for j in range(1, 8):
        X[0, 8 + j::16] = 4.0
    Y, _ = oracle.rmsnorm_rows(_bits(X), None, None, 0.0)
    inv = np.float32(1.0) / np.sqrt(np.float32(12.5))
    want3 = _bits(torch.tensor([float(np.float32(3.0) * inv)]).to(torch.bfloat16))[0]
    want4 = _bits(torch.tensor([float(np.float32(4.0) * inv)]).to(torch.bfloat16))[0]
    assert np.all(Y[0][X[0].float().numpy() == 3.0] == want3)
    assert np.all(Y[0][X[0].float().numpy() == 4.0] == want4)


@pytest.mark.parametrize("k", [-20, -3, 5, 40])
def test_power_of_two_invariance(k):
    X, R, w = _rows(4, 768, 11)
    Y, _ = oracle.rmsnorm_rows(_bits(X), _bits(R), _bits(w), 0.0)
    Ys, Hs = oracle.rmsnorm_rows(_bits(X * 2.0 ** k), _bits(R * 2.0 ** k), _bits(w), 0.0)
    assert np.array_equal(Y, Ys)
    assert np.array_equal(Hs, _bits((X + R) * 2.0 ** k))


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
