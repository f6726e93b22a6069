"""Input RMSNorm with a residual on the GPU against the CPU oracle (through the C ABI).

Bar: the residual output bit for bit; each normalised value equal to the
oracle's bf16 rounding of the exact value, or, where that value lies within
2^-34 (relative) of a rounding midpoint, to either neighbour (the oracle's
Yalt); the codes and row scales of the normalised rows equal the oracle's
for some admissible choice there (the rest: bit for bit); linear outputs
within 1 bf16 ulp.
Source: comfy-kitchen 0.2.40, "Huawei Ascend backend" (int8_linear's input
RMSNorm and residual arguments); the reading is stated in include/ck.h.
"""
import numpy as np
import pytest
import torch

import oracle
import workloads
from parity_helpers import assert_bf16_close, assert_codes_admissible, tile_rows

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


def _assert_y(got, Yr, Ya):
    ok = (got == Yr) | (got == Ya)
    assert ok.all(), f"{(~ok).sum()} normalised values differ from both admissible roundings"


@pytest.mark.parametrize("M,K", [(1, 256), (37, 768), (130, 5376), (9, 28672), (2, 132864)])
@pytest.mark.parametrize("with_residual,with_g", [(True, True), (False, True), (True, False),
                                                  (False, False)])
def test_rmsnorm_matches_oracle(ck, M, K, with_residual, with_g):
    X, R, w = _inputs(M, K, M + K)
    eps = 1e-5
    R = R if with_residual else None
    w = w if with_g else None
    Yr, Hr, Ya = oracle.rmsnorm_rows(_bits(X), None if R is None else _bits(R),
                                     None if w is None else _bits(w), eps, with_alt=True)
    Ro = torch.empty((M, K), dtype=torch.bfloat16, device="cuda")
    Y = ck.rmsnorm_residual(X.cuda(), None if R is None else R.cuda(),
                            None if w is None else w.cuda(), eps, residual_out=Ro)
    _assert_y(_bits(Y), Yr, Ya)
    assert np.array_equal(_bits(Ro), Hr)


def test_rmsnorm_in_place_residual_and_strides(ck):
    M, K = 45, 1024
    X, R, w = _inputs(M, K, 5)
    Yr, Hr, Ya = oracle.rmsnorm_rows(_bits(X), _bits(R), _bits(w), 1e-6, with_alt=True)
    wideX = torch.zeros((M, K + 256), dtype=torch.bfloat16, device="cuda")
    wideX[:, :K] = X.cuda()
    wideR = torch.zeros((M, K + 512), dtype=torch.bfloat16, device="cuda")
    wideR[:, :K] = R.cuda()
    r = wideR[:, :K]
    Y = ck.rmsnorm_residual(wideX[:, :K], r, w.cuda(), 1e-6, residual_out=r)  # in place
    _assert_y(_bits(Y), Yr, Ya)
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
        Yr, _, Ya = oracle.rmsnorm_rows(_bits(X), None, _bits(w), eps, with_alt=True)
        Y = ck.rmsnorm_residual(X.cuda(), None, w.cuda(), eps)
        _assert_y(_bits(Y), Yr, Ya)


def _norm_linear_check(ck, X, R, w, W, bias, eps, rows=None, in_place=False):
    """ck_int8_linear_norm against the oracle: residual output bit for bit,
    codes and row scales admissible (the normalised rows, when the workspace
    holds them, too), output rows (those whose normalised values are
    unambiguous) within 1 bf16 ulp."""
    M, K = X.shape
    Qw, s_w = ck.rotate_quant_weight(W.cuda())
    Qw_r, s_w_r = oracle.rotate_quant_weight(W.numpy())
    Yn, Hr, Ya = oracle.rmsnorm_rows(_bits(X), _bits(R), _bits(w), eps, with_alt=True)
    need = ck.norm_workspace_bytes(M, K)
    fused = need == ck.workspace_bytes(M, K)
    assert fused == (K <= ck.NORM_FUSED_MAX_K)
    ws = torch.empty((need,), dtype=torch.uint8, device="cuda")
    Rd = R.cuda()
    Ro = Rd if in_place else torch.empty((M, K), dtype=torch.bfloat16, device="cuda")
    Y = ck.int8_linear_norm(X.cuda(), Qw, s_w, bias.cuda(), Rd, w.cuda(), eps,
                            residual_out=Ro, workspace=ws)
    torch.cuda.synchronize()
    off_q = 0 if fused else (M * K * 2 + 255) // 256 * 256
    Qx = ws[off_q: off_q + M * K].view(M, K).view(torch.int8).cpu().numpy()
    off_s = off_q + (M * K + 255) // 256 * 256
    s_x = ws[off_s: off_s + 4 * M].view(torch.float32).cpu().numpy()
    assert np.array_equal(_bits(Ro), Hr)
    if not fused:
        _assert_y(_bits(ws[: M * K * 2].view(torch.bfloat16).view(M, K)), Yn, Ya)
    assert_codes_admissible(Qx, s_x, Yn, Ya)
    Qx_r, s_x_r = oracle.quantize_rows_bf16(Yn, rotate=True)
    rows = np.arange(M) if rows is None else rows
    rows = rows[~(Yn[rows] != Ya[rows]).any(axis=1)]
    Yr = oracle.linear_rows(Qx_r, s_x_r, Qw_r, s_w_r, _bits(bias), rows)
    assert_bf16_close(_bits(Y[torch.from_numpy(rows).cuda()]), Yr)


@pytest.mark.parametrize("M,K,N", [(1, 256, 8), (130, 5376, 264), (300, 1024, 520),
                                   (37, 14336, 264), (9, 14592, 256), (5, 28672, 8)])
def test_int8_linear_norm_matches_oracle(ck, M, K, N):
    """K up to 14336 normalises inside the quantiser; above that the
    RMSNorm runs first into the workspace."""
    X, R, w = _inputs(M, K, 3 * M + K)
    cfg = workloads.custom(M, K, N, seed=M + N)
    _, W, bias = workloads.make_inputs(cfg)
    _norm_linear_check(ck, X, R, w, W, bias, 1e-6)


def test_int8_linear_norm_residual_updated_in_place(ck):
    X, R, w = _inputs(260, 768, 17)
    _, W, bias = workloads.make_inputs(workloads.custom(260, 768, 264, seed=18))
    _norm_linear_check(ck, X, R, w, W, bias, 1e-5, in_place=True)


def _norm_quant_check(ck, X, R, w, eps):
    M, K = X.shape
    Yn, Hr, Ya = oracle.rmsnorm_rows(_bits(X), None if R is None else _bits(R),
                                     None if w is None else _bits(w), eps, with_alt=True)
    Ro = torch.empty((M, K), dtype=torch.bfloat16, device="cuda")
    Qx, s_x = ck.quantize_rotate_rowwise_norm(X.cuda(), None if R is None else R.cuda(),
                                              None if w is None else w.cuda(), eps,
                                              residual_out=Ro)
    torch.cuda.synchronize()
    assert np.array_equal(_bits(Ro), Hr)
    assert_codes_admissible(Qx.cpu().numpy(), s_x.cpu().numpy(), Yn, Ya)


@pytest.mark.parametrize("with_residual,with_g", [(True, True), (False, True), (True, False),
                                                  (False, False)])
@pytest.mark.parametrize("M,K", [(1, 256), (131, 5376), (7, 14336)])
def test_quantize_rotate_rowwise_norm(ck, M, K, with_residual, with_g):
    X, R, w = _inputs(M, K, 5 * M + K)
    _norm_quant_check(ck, X, R if with_residual else None, w if with_g else None, 1e-6)


def test_quantize_rotate_rowwise_norm_special_rows(ck):
    """Zero rows, rows of subnormal and huge values, a residual that cancels
    x exactly, eps dominating, weights far above 1 (the fast path's tiny-value
    bound grows with them) and weights of 2^16 and more (every value then
    takes the double-precision path)."""
    M, K = 9, 768
    X, R, w = _inputs(M, K, 23)
    x, r = X.float(), R.float()
    x[0] = 0.0
    r[0] = 0.0
    x[1] *= 2.0 ** -130  # subnormal bf16 inputs
    r[1] *= 2.0 ** -130
    x[2] *= 2.0 ** 100
    r[2] = -x[2]         # h = 0 exactly
    x[3] *= 2.0 ** 60
    x[4] = 1e-20
    X, R = x.to(torch.bfloat16), r.to(torch.bfloat16)
    for eps in (1e-6, 1.0):
        _norm_quant_check(ck, X, R, w, eps)
    for scale in (3.0, 2.0 ** 12, 2.0 ** 17):
        _norm_quant_check(ck, X, R, (w.float() * scale).to(torch.bfloat16), 1e-6)
    tiny_g = (w.float() * 2.0 ** -100).to(torch.bfloat16)  # outputs in the subnormal range
    _norm_quant_check(ck, X, R, tiny_g, 1e-6)


@pytest.mark.slow
def test_int8_linear_norm_full_size_ragged(ck):
    """The ragged M8193/K5376/N16128 workload with a residual and a weight:
    every code and row scale, every residual and normalised value, and all
    outputs of one row per 256-row M-tile."""
    cfg = workloads.CONFIGS[1]
    X, W, bias = workloads.make_inputs(cfg)
    g = torch.Generator().manual_seed(321)
    R = torch.randn(cfg.M, cfg.K, generator=g).to(torch.bfloat16)
    w = (1.0 + 0.25 * torch.randn(cfg.K, generator=g)).to(torch.bfloat16)
    _norm_linear_check(ck, X, R, w, W, bias, 1e-6, rows=tile_rows(cfg.M))


@pytest.mark.slow
def test_rmsnorm_full_size_headline(ck):
    """M32700/K5376 (the benchmarked activation shape) with a residual and a
    weight: every normalised value admissible, every residual output exact."""
    cfg = workloads.HEADLINE
    X, _, _ = workloads.make_inputs(cfg)
    g = torch.Generator().manual_seed(123)
    R = torch.randn(cfg.M, cfg.K, generator=g).to(torch.bfloat16)
    w = (1.0 + 0.25 * torch.randn(cfg.K, generator=g)).to(torch.bfloat16)
    Yr, Hr, Ya = oracle.rmsnorm_rows(_bits(X), _bits(R), _bits(w), 1e-6, with_alt=True)
    Ro = torch.empty((cfg.M, cfg.K), dtype=torch.bfloat16, device="cuda")
    Y = ck.rmsnorm_residual(X.cuda(), R.cuda(), w.cuda(), 1e-6, residual_out=Ro)
    _assert_y(_bits(Y), Yr, Ya)
    assert np.array_equal(_bits(Ro), Hr)
