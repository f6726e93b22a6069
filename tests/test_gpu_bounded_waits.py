"""Failure detection without a GPU fault: every wait inside the GEMM kernels is
bounded. The test makes one wait run out on purpose (the TMA producer is told
to issue nothing, so the MMA warp's wait for the first stage can never be
satisfied); the kernel must record CK_ERR_DEVICE_TIMEOUT, free its TMEM and
return, and the context must stay usable for the next, correct call. Both GEMM
variants are covered (M <= 128: one SM per tile; M > 128: CTA pairs)."""
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
    m.clear_device_error()


@pytest.mark.parametrize("M", [64, 384])
def test_stalled_producer_times_out_and_context_survives(ck, M):
    K, N = 512, 264
    rng = np.random.default_rng(M)
    a = rng.integers(-127, 128, size=(M, K)).astype(np.int8)
    b = rng.integers(-127, 128, size=(N, K)).astype(np.int8)
    Qx = torch.from_numpy(a).cuda()
    Qw = torch.from_numpy(b).cuda()
    ck.clear_device_error()
    ck.inject_producer_stall(1, 20_000_000)  # 20 ms bound for this one launch
    ck.test_int8_gemm_i32(Qx, Qw)
    assert ck.device_error() == ck.CK_ERR_DEVICE_TIMEOUT
    ck.clear_device_error()
    assert ck.device_error() == ck.CK_OK
    acc = ck.test_int8_gemm_i32(Qx, Qw)  # the next call is unaffected
    assert np.array_equal(acc.cpu().numpy(), oracle.gemm_i32(a, b))
    assert ck.device_error() == ck.CK_OK


@pytest.mark.parametrize("M", [64, 384])
def test_stalled_producer_times_out_in_the_nvfp4_gemm(ck, M):
    """The same for the block-scaled FP4 GEMM (M <= 128: 1-SM kernel; M > 128:
    CTA pairs): the stalled launch reports the timeout, the next is correct."""
    K, N = 512, 264
    cfg = workloads.custom(M, K, N, seed=M + 1)
    X, W, bias = workloads.make_inputs(cfg)
    Qa, Sa, sa = ck.quantize_rotate_nvfp4(X.cuda())
    Qw, Sw, sw = ck.rotate_quant_weight_nvfp4(W.cuda())
    torch.cuda.synchronize()
    ck.clear_device_error()
    ck.inject_producer_stall(1, 20_000_000)
    ck.nvfp4_gemm(Qa, Sa, sa, Qw, Sw, sw)
    assert ck.device_error() == ck.CK_ERR_DEVICE_TIMEOUT
    ck.clear_device_error()
    Y = ck.nvfp4_gemm(Qa, Sa, sa, Qw, Sw, sw)
    Yr, mag = oracle.nvfp4_linear_rows(Qa.cpu().numpy(), Sa.cpu().numpy(), float(sa.cpu()[0]),
                                       Qw.cpu().numpy(), Sw.cpu().numpy(), float(sw.cpu()[0]))
    y = workloads.from_bf16_bits(workloads.bf16_bits(Y.cpu())).double().numpy()
    r = workloads.from_bf16_bits(Yr).double().numpy()
    assert np.all(np.abs(y - r) <= np.abs(r) * 2.0 ** -7 + K * 2.0 ** -24 * mag + 1e-30)
    assert ck.device_error() == ck.CK_OK

