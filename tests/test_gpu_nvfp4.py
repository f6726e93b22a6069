"""ConvRot NVFP4 on the GPU against the CPU oracle (through the C ABI).

Codes, block scales, the per-tensor scale and decoded values are compared bit
for bit. The block-scaled GEMM accumulates the exact products in the tensor
cores' fp32 (their summation order), so its outputs are compared with the
oracle's (double-precision sum, then the same fp32 epilogue) within one bf16
ulp plus the float accumulation bound K * 2^-24 * sum|products| * alpha.
Source: ComfyUI-HSWQ-Loader-and-Tools, "NVFP4 torch.compile Fix", section 5-1.
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


def _np(t):
    return t.cpu().numpy()


@pytest.mark.parametrize("M,K", [(1, 256), (37, 768), (130, 5376), (5, 28672), (300, 512),
                                 (2, 32768)])
def test_quantize_rotate_nvfp4_bit_exact(ck, M, K):
    cfg = workloads.custom(M, K, 8, seed=M * 7 + K)
    X, _, _ = workloads.make_inputs(cfg)
    Qr, Sr, sr = oracle.quantize_rotate_nvfp4(workloads.bf16_bits(X))
    Q, S, s_t = ck.quantize_rotate_nvfp4(X.cuda())
    assert np.float32(_np(s_t)[0]) == np.float32(sr)
    assert np.array_equal(_np(S)[: Sr.size], Sr)
    assert np.array_equal(_np(Q), Qr)


@pytest.mark.parametrize("N,K", [(264, 768), (520, 5376), (8, 256)])
def test_rotate_quant_weight_nvfp4_bit_exact(ck, N, K):
    cfg = workloads.custom(4, K, N, seed=N + K)
    _, W, _ = workloads.make_inputs(cfg)
    Qr, Sr, sr = oracle.rotate_quant_weight_nvfp4(W.numpy())
    Q, S, s_t = ck.rotate_quant_weight_nvfp4(W.cuda())
    assert np.float32(_np(s_t)[0]) == np.float32(sr)
    assert np.array_equal(_np(S)[: Sr.size], Sr)
    assert np.array_equal(_np(Q), Qr)


def test_quantize_nvfp4_row_stride(ck):
    """X with a row stride larger than K (a column slice of a wider tensor)."""
    cfg = workloads.custom(45, 1024, 8, seed=44)
    X, _, _ = workloads.make_inputs(cfg)
    wide = torch.zeros((45, 1024 + 512), dtype=torch.bfloat16)
    wide[:, :1024] = X
    Qr, Sr, sr = oracle.quantize_rotate_nvfp4(workloads.bf16_bits(X))
    Q, S, s_t = ck.quantize_rotate_nvfp4(wide.cuda()[:, :1024])
    assert np.float32(_np(s_t)[0]) == np.float32(sr)
    assert np.array_equal(_np(S)[: Sr.size], Sr) and np.array_equal(_np(Q), Qr)


def test_quantize_nvfp4_zero_and_scaled_tensors(ck):
    Z = torch.zeros((3, 512), dtype=torch.bfloat16, device="cuda")
    Q, S, s_t = ck.quantize_rotate_nvfp4(Z)
    assert float(s_t[0]) == 0.0 and not Q.any() and not S.any()
    cfg = workloads.custom(6, 512, 8, seed=3)
    X, _, _ = workloads.make_inputs(cfg)
    a = ck.quantize_rotate_nvfp4(X.cuda())
    b = ck.quantize_rotate_nvfp4((X * 4).cuda())
    assert torch.equal(a[0], b[0]) and torch.equal(a[1], b[1]) and float(b[2][0]) == 4 * float(a[2][0])


def test_quantize_nvfp4_rounding_ties(ck):
    """Inputs whose rotated values hit the E4M3 and E2M1 rounding ties exactly.

    Row 0 holds A = 258048 in column 0: every rotated value is A / 16, so the
    tensor's absmax is 16128 and s_t = 16128 / 2688 = 6. A row with one value
    a has the block absmax m = a / 16 and the block-scale quotient m / 36:
    a = 612 gives 1.0625, half-way between the E4M3 values 1 and 1.125 (ties
    to 1.0, byte 0x38); a = 8 and a = 1 fall in E4M3's subnormal range. A row
    a e_0 + b e_1 rotates to (a + b) / 16 and (a - b) / 16 in alternate
    places; with a + b = 576 the block scale is exactly 1 (d = 6), and
    a - b = 24, 72, 240, 480 puts (a - b) / 96 on the E2M1 ties 0.25, 0.75,
    2.5 and 5. Every tie must round to even, as the oracle does."""
    rows = [[(0, 258048.0)], [(0, 612.0)], [(0, 8.0)], [(0, 1.0)],
            [(0, 300.0), (1, 276.0)], [(0, 324.0), (1, 252.0)], [(0, 408.0), (1, 168.0)],
            [(0, 528.0), (1, 48.0)], [(0, -612.0)], [(3, 612.0), (200, -300.0)]]
    X = torch.zeros((len(rows), 256), dtype=torch.float32)
    for r, entries in enumerate(rows):
        for c, v in entries:
            X[r, c] = v
    X = X.to(torch.bfloat16)
    assert torch.equal(X.float(), X.to(torch.float32))
    Qr, Sr, sr = oracle.quantize_rotate_nvfp4(workloads.bf16_bits(X))
    assert np.float32(sr) == np.float32(6.0)
    # the a = 612 row: every block's scale ties to E4M3 1.0
    assert all(Sr[oracle.nvfp4_sf_offset(1, c, 16)] == 0x38 for c in range(16))
    Q, S, s_t = ck.quantize_rotate_nvfp4(X.cuda())
    assert np.float32(_np(s_t)[0]) == np.float32(sr)
    assert np.array_equal(_np(S)[: Sr.size], Sr)
    assert np.array_equal(_np(Q), Qr)


@pytest.mark.parametrize("hi_first", [False, True])
def test_dequantize_nvfp4_bit_exact(ck, hi_first):
    cfg = workloads.custom(33, 768, 8, seed=21)
    X, _, _ = workloads.make_inputs(cfg)
    Q, S, s_t = ck.quantize_rotate_nvfp4(X.cuda())
    got = _np(ck.dequantize_nvfp4(Q, S, s_t, hi_first=hi_first))
    want = oracle.dequantize_nvfp4(_np(Q), _np(S), float(_np(s_t)[0]), hi_first=hi_first)
    assert np.array_equal(got.view(np.uint32), want.view(np.uint32))


def test_dequantize_nvfp4_every_scale_byte(ck):
    """Every non-NaN positive E4M3 byte (subnormals included) as a block scale
    with E2M1 code 2 (= 1.0) and s_t = 1: the decoded values are the scales
    themselves, compared with the oracle and with PyTorch's float8_e4m3fn."""
    rows, K = 128, 2048
    C = K // 16
    S = np.zeros(ck.nvfp4_scale_bytes(rows, K), np.uint8)
    byte_of = np.zeros((rows, C), np.uint8)
    for r in range(rows):
        for c in range(C):
            b = (r * C + c) % 127
            byte_of[r, c] = b
            S[oracle.nvfp4_sf_offset(r, c, C)] = b
    Q = np.full((rows, K // 2), 0x22, np.uint8)
    s_t = np.ones(1, np.float32)
    got = _np(ck.dequantize_nvfp4(torch.from_numpy(Q).cuda(), torch.from_numpy(S).cuda(),
                                  torch.from_numpy(s_t).cuda()))
    want = oracle.dequantize_nvfp4(Q, S, 1.0)
    assert np.array_equal(got.view(np.uint32), want.view(np.uint32))
    e4m3 = torch.from_numpy(byte_of).view(torch.float8_e4m3fn).float().numpy()
    assert np.array_equal(got.reshape(rows, C, 16), np.repeat(e4m3[:, :, None], 16, axis=2))


def _bf16_val(bits):
    return workloads.from_bf16_bits(bits).double().numpy()


def _assert_gemm_close(Y_bits, Yr_bits, mag, K):
    y, r = _bf16_val(Y_bits), _bf16_val(Yr_bits)
    ulp = np.maximum(np.abs(r), np.abs(y)) * 2.0 ** -7  # one bf16 ulp, generously
    tol = ulp + K * 2.0 ** -24 * mag + 1e-30
    bad = np.abs(y - r) > tol
    assert not bad.any(), f"{bad.sum()} outputs off, first at {np.argwhere(bad)[0]}: {y[bad][0]} vs {r[bad][0]}"


@pytest.mark.parametrize("M,K,N", [(128, 256, 128), (1, 256, 8), (129, 768, 264), (300, 5376, 520),
                                   (257, 1024, 136),
                                   # the 2-SM kernel's raster walks groups of 32 N-tiles: a
                                   # full group and a second, ragged one of 2, ragged M
                                   (300, 256, 33 * 256 + 40)])
def test_nvfp4_gemm_matches_oracle(ck, M, K, N):
    cfg = workloads.custom(M, K, N, seed=M + 3 * N + K)
    X, W, bias = workloads.make_inputs(cfg)
    Qa, Sa, sa = ck.quantize_rotate_nvfp4(X.cuda())
    Qw, Sw, sw = ck.rotate_quant_weight_nvfp4(W.cuda())
    Y = ck.nvfp4_gemm(Qa, Sa, sa, Qw, Sw, sw, bias.cuda())
    Yr, mag = oracle.nvfp4_linear_rows(_np(Qa), _np(Sa), float(_np(sa)[0]), _np(Qw), _np(Sw),
                                       float(_np(sw)[0]), workloads.bf16_bits(bias))
    _assert_gemm_close(workloads.bf16_bits(Y.cpu()), Yr, mag, K)


def test_convrot_nvfp4_linear_matches_oracle_and_fp64(ck):
    M, K, N = 200, 1024, 264
    cfg = workloads.custom(M, K, N, seed=31)
    X, W, bias = workloads.make_inputs(cfg)
    Qw, Sw, sw = ck.rotate_quant_weight_nvfp4(W.cuda())
    Y = ck.convrot_nvfp4_linear(X.cuda(), Qw, Sw, sw, bias.cuda())
    Qa, Sa, sa = oracle.quantize_rotate_nvfp4(workloads.bf16_bits(X))
    Yr, mag = oracle.nvfp4_linear_rows(Qa, Sa, sa, _np(Qw), _np(Sw), float(_np(sw)[0]),
                                       workloads.bf16_bits(bias))
    _assert_gemm_close(workloads.bf16_bits(Y.cpu()), Yr, mag, K)
    # and the quantised linear is close to the unquantised one (FP4: a few per cent)
    ref = X.double().numpy() @ W.double().numpy().T + _bf16_val(workloads.bf16_bits(bias))[None, :]
    rel = np.linalg.norm(_bf16_val(workloads.bf16_bits(Y.cpu())) - ref) / np.linalg.norm(ref)
    assert rel < 0.2, rel


@pytest.mark.slow
@pytest.mark.parametrize("name", ["ragged_m8193_k5376_n16128", "qkv_m32700_k5376_n16128"])
def test_full_size_nvfp4_codes_and_sampled_rows(ck, name):
    """The benchmark's shapes: every code and scale bit-exact, and sampled
    output rows (first, last, tile edges, random) within the GEMM bound."""
    cfg = workloads.BY_NAME[name]
    X, W, bias = workloads.make_inputs(cfg)
    Qr, Sr, sr = oracle.quantize_rotate_nvfp4(workloads.bf16_bits(X))
    Xd = X.cuda()
    Qw, Sw, sw = ck.rotate_quant_weight_nvfp4(W.cuda())
    Qa, Sa, sa = ck.quantize_rotate_nvfp4(Xd)
    assert np.float32(_np(sa)[0]) == np.float32(sr)
    assert np.array_equal(_np(Sa)[: Sr.size], Sr)
    assert np.array_equal(_np(Qa), Qr)
    Y = ck.convrot_nvfp4_linear(Xd, Qw, Sw, sw, bias.cuda())
    M = cfg.M
    rng = np.random.default_rng(0)
    rows = np.unique(np.concatenate([[0, 127, 128, M // 2, M - 1], rng.integers(0, M, 8)]))
    Yr, mag = oracle.nvfp4_linear_rows(Qr, Sr, sr, _np(Qw), _np(Sw), float(_np(sw)[0]),
                                       workloads.bf16_bits(bias), rows=rows)
    got = workloads.bf16_bits(Y[torch.from_numpy(rows).cuda()].cpu())
    _assert_gemm_close(got, Yr, mag, cfg.K)
