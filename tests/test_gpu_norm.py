"""Input RMSNorm with a residual on the GPU against the CPU oracle (through the C ABI).

The normalised rows, the residual output, the codes and the row scales are
compared bit for bit; linear outputs within 1 bf16 ulp (0 expected).
Source: comfy-kitchen 0.2.40, "Huawei Ascend backend" (int8_linear's input
RMSNorm and residual arguments); the reading is stated in include/ck.h.
"""
import numpy as np
import pytest
import torch

import oracle
import workloads

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def ck():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import int8_quantized_linear_convrot256_b200 as m

    m.clear_device_error()
    yield m
    assert m.device_error() == m.CK_OK


def _bits(t):
    return workloads.bf16_bits(t.cpu())


def _inputs(M, K, seed, scale=1.0):
    cfg = workloads.custom(M, K, 8, seed=seed)
    X, _, _ = workloads.make_inputs(cfg)
    g = torch.Generator().manual_seed(seed + 1)
    R = (torch.randn(M, K, generator=g) * scale).to(torch.bfloat16)
    w = (1.0 + 0.25 * torch.randn(K, generator=g)).to(torch.bfloat16)
    return X, R, w


def _ordered(bits):
    b = bits.astype(np.int32)
    return np.where(b & 0x8000, 0x8000 - b, b)


@pytest.mark.parametrize("M,K", [(1, 256), (37, 768), (130, 5376), (9, 28672), (2, 132864)])
@pytest.mark.parametrize("with_residual,with_g", [(True, True), (False, True), (True, False),
                                                  (False, False)])
def test_rmsnorm_bit_exact(ck, M, K, with_residual, with_g):
    X, R, w = _inputs(M, K, M + K)
    eps = 1e-5
    R = R if with_residual else None
    w = w if with_g else None
    Yr, Hr = oracle.rmsnorm_rows(_bits(X), None if R is None else _bits(R),
                                 None if w is None else _bits(w), eps)
    Ro = torch.empty((M, K), dtype=torch.bfloat16, device="cuda")
    Y = ck.rmsnorm_residual(X.cuda(), None if R is None else R.cuda(),
                            None if w is None else w.cuda(), eps, residual_out=Ro)
    assert np.array_equal(_bits(Y), Yr)
    assert np.array_equal(_bits(Ro), Hr)


def test_rmsnorm_in_place_residual_and_strides(ck):
    M, K = 45, 1024
    X, R, w = _inputs(M, K, 5)
    Yr, Hr = oracle.rmsnorm_rows(_bits(X), _bits(R), _bits(w), 1e-6)
    wideX = torch.zeros((M, K + 256), dtype=torch.bfloat16, device="cuda")
    wideX[:, :K] = X.cuda()
    wideR = torch.zeros((M, K + 512), dtype=torch.bfloat16, device="cuda")
    wideR[:, :K] = R.cuda()
    r = wideR[:, :K]
    Y = ck.rmsnorm_residual(wideX[:, :K], r, w.cuda(), 1e-6, residual_out=r)  # in place
    assert np.array_equal(_bits(Y), Yr)
    assert np.array_equal(_bits(r), Hr)
    assert not wideR[:, K:].any()


def test_rmsnorm_extreme_rows(ck):
    """Zero rows, tiny and huge rows (power-of-two scaled), eps dominating."""
    M, K = 8, 512
    X, R, w = _inputs(M, K, 9)
    x = X.float()
    x[0] = 0.0
    x[1] *= 2.0 ** -60
    x[2] *= 2.0 ** 60
    x[3] = 1e-3
    X = x.to(torch.bfloat16)
    for eps in (1e-6, 1.0):
        Yr, _ = oracle.rmsnorm_rows(_bits(X), None, _bits(w), eps)
        Y = ck.rmsnorm_residual(X.cuda(), None, w.cuda(), eps)
        assert np.array_equal(_bits(Y), Yr)


@pytest.mark.parametrize("M,K,N", [(1, 256, 8), (130, 5376, 264), (300, 1024, 520)])
def test_int8_linear_norm_matches_oracle(ck, M, K, N):
    X, R, w = _inputs(M, K, 3 * M + K)
    cfg = workloads.custom(M, K, N, seed=M + N)
    _, W, bias = workloads.make_inputs(cfg)
    Qw, s_w = ck.rotate_quant_weight(W.cuda())
    Qw_r, s_w_r = oracle.rotate_quant_weight(W.numpy())
    Yr, Hr, Qx_r, s_x_r = oracle.int8_linear_norm(_bits(X), Qw_r, s_w_r, _bits(bias), _bits(R),
                                                  _bits(w), 1e-6)
    ws = torch.empty((ck.norm_workspace_bytes(M, K),), dtype=torch.uint8, device="cuda")
    Ro = torch.empty((M, K), dtype=torch.bfloat16, device="cuda")
    Y = ck.int8_linear_norm(X.cuda(), Qw, s_w, bias.cuda(), R.cuda(), w.cuda(), 1e-6,
                            residual_out=Ro, workspace=ws)
    torch.cuda.synchronize()
    off_q = (M * K * 2 + 255) // 256 * 256
    Qx = ws[off_q: off_q + M * K].view(M, K).view(torch.int8)
    off_s = off_q + (M * K + 255) // 256 * 256
    s_x = ws[off_s: off_s + 4 * M].view(torch.float32)
    assert np.array_equal(_bits(Ro), Hr)
    assert np.array_equal(s_x.cpu().numpy().view(np.uint32), s_x_r.view(np.uint32))
    assert np.array_equal(Qx.cpu().numpy(), Qx_r)
    d = np.abs(_ordered(_bits(Y)) - _ordered(Yr))
    assert d.max(initial=0) <= 1


@pytest.mark.slow
def test_rmsnorm_full_size_headline(ck):
    """M32700/K5376 (the benchmarked activation shape) with a residual and a
    weight: every normalised value and residual output bit-exact."""
    cfg = workloads.HEADLINE
    X, _, _ = workloads.make_inputs(cfg)
    g = torch.Generator().manual_seed(123)
    R = torch.randn(cfg.M, cfg.K, generator=g).to(torch.bfloat16)
    w = (1.0 + 0.25 * torch.randn(cfg.K, generator=g)).to(torch.bfloat16)
    Yr, Hr = oracle.rmsnorm_rows(_bits(X), _bits(R), _bits(w), 1e-6)
    Ro = torch.empty((cfg.M, cfg.K), dtype=torch.bfloat16, device="cuda")
    Y = ck.rmsnorm_residual(X.cuda(), R.cuda(), w.cuda(), 1e-6, residual_out=Ro)
    assert np.array_equal(_bits(Y), Yr)
    assert np.array_equal(_bits(Ro), Hr)
