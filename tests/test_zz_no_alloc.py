"""ck_int8_linear_noalloc: the linear for callers that cannot allocate device
memory (a plugin inside an engine that owns all device memory, code with a
memory budget fixed at start-up, code that must not risk the device-wide
synchronisation cudaFree can cause). It keeps the activation codes and row
scales in the library's fixed device array instead of a caller workspace, so
it must give the same output as ck_int8_linear with a workspace, and the
oracle's.

This file is named to be collected last: if it fails in a run that stops at
the first failure, every other test has already run. It passes on its own in
a fresh process as well as after the other tests.
"""
import ctypes

import numpy as np
import pytest
import torch

import oracle
import workloads

BF16_ULP_TOL = 1
FAKE = 0x10000  # 64 KiB: aligned, never dereferenced (host-side checks only)
MIS = FAKE + 4


def _ulp_distance(a_bits: np.ndarray, b_bits: np.ndarray) -> int:
    def ordered(bits):
        b = bits.astype(np.int32)
        return np.where(b & 0x8000, 0x8000 - b, b)

    return int(np.abs(ordered(a_bits) - ordered(b_bits)).max(initial=0))


@pytest.mark.gpu
def test_noalloc_matches_workspace_entry_point_on_two_calls_in_a_row():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import int8_quantized_linear_convrot256_b200 as ck

    ck.clear_device_error()
    stream = torch.cuda.current_stream()
    # a larger problem first, then a smaller one that reuses the same array
    for (M, K, N, seed) in [(3000, 7168, 264, 101), (517, 1024, 520, 102)]:
        cfg = workloads.custom(M, K, N, seed=seed)
        assert ck.workspace_bytes(M, K) <= ck.NOALLOC_SCRATCH_BYTES
        X, W, bias = workloads.make_inputs(cfg)
        Xd, bd = X.cuda(), bias.cuda()
        Qw, s_w = ck.rotate_quant_weight(W.cuda())
        ref = ck.int8_linear(Xd, Qw, s_w, bd)
        out = torch.full((M, N), float("nan"), dtype=torch.bfloat16, device="cuda")
        status = ck.lib.ck_int8_linear_noalloc(
            ctypes.c_void_p(Xd.data_ptr()), Xd.stride(0), ctypes.c_void_p(Qw.data_ptr()),
            ctypes.c_void_p(s_w.data_ptr()), ctypes.c_void_p(bd.data_ptr()),
            ctypes.c_void_p(out.data_ptr()), M, N, K, ctypes.c_void_p(stream.cuda_stream))
        assert status == ck.CK_OK, ck.status_string(status)
        torch.cuda.synchronize()
        got = workloads.bf16_bits(out.cpu())
        d = _ulp_distance(got, workloads.bf16_bits(ref.cpu()))
        assert d <= BF16_ULP_TOL, (M, K, N, d)
        # and the oracle's output, computed from the same inputs on the CPU
        rqw, rsw = oracle.rotate_quant_weight(W.numpy())
        Yr = oracle.int8_linear(workloads.bf16_bits(X), rqw, rsw, workloads.bf16_bits(bias))[0]
        assert _ulp_distance(got, Yr) <= BF16_ULP_TOL
    assert ck.device_error() == ck.CK_OK


@pytest.mark.gpu
def test_noalloc_python_wrapper():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import int8_quantized_linear_convrot256_b200 as ck

    cfg = workloads.custom(300, 768, 264, seed=103)
    X, W, bias = workloads.make_inputs(cfg)
    Qw, s_w = ck.rotate_quant_weight(W.cuda())
    out = torch.empty((300, 264), dtype=torch.bfloat16, device="cuda")
    Y = ck.int8_linear_noalloc(X.cuda(), Qw, s_w, bias.cuda(), out=out)
    torch.cuda.synchronize()
    assert Y.data_ptr() == out.data_ptr()
    rqw, rsw = oracle.rotate_quant_weight(W.numpy())
    Yr = oracle.int8_linear(workloads.bf16_bits(X), rqw, rsw, workloads.bf16_bits(bias))[0]
    assert _ulp_distance(workloads.bf16_bits(Y.cpu()), Yr) <= BF16_ULP_TOL


def test_noalloc_wrapper_rejects_a_column_slice_of_weights():
    """Qw must be row-contiguous: the library reads it with row stride K."""
    from torch._subclasses.fake_tensor import FakeTensorMode

    import int8_quantized_linear_convrot256_b200 as ck

    with FakeTensorMode():  # CUDA-typed tensors without a device: checks only
        X = torch.empty((4, 256), dtype=torch.bfloat16, device="cuda")
        wide = torch.empty((8, 512), dtype=torch.int8, device="cuda")
        s_w = torch.empty(8, dtype=torch.float32, device="cuda")
        with pytest.raises(ValueError, match="Qw must be contiguous"):
            ck.int8_linear_noalloc(X, wide[:, :256], s_w)


def test_noalloc_rejects_problems_larger_than_its_array():
    import int8_quantized_linear_convrot256_b200 as ck

    M, K = 8192, 5376  # 44 MB of codes > 32 MiB
    assert ck.workspace_bytes(M, K) > ck.NOALLOC_SCRATCH_BYTES
    st = ck.lib.ck_int8_linear_noalloc(FAKE, K, FAKE, FAKE, None, FAKE, M, 256, K, None)
    assert st == ck.CK_ERR_WORKSPACE
    assert ck.lib.ck_int8_linear_noalloc(FAKE, K, FAKE, FAKE, None, FAKE, 0, 256, K, None) == ck.CK_OK


@pytest.mark.parametrize("args,status", [
    (dict(X=None), "CK_ERR_INVALID_VALUE"),
    (dict(ldx=4096), "CK_ERR_INVALID_VALUE"),
    (dict(K=300, ldx=5376), "CK_ERR_UNSUPPORTED_SHAPE"),
    (dict(N=12), "CK_ERR_UNSUPPORTED_SHAPE"),
    (dict(X=MIS), "CK_ERR_MISALIGNED"),
    (dict(Y=MIS), "CK_ERR_MISALIGNED"),
])
def test_noalloc_checks_come_in_ck_int8_linear_order(args, status):
    """Argument errors are reported before the size check, as ck_int8_linear
    reports them before its workspace check (a too-large M here)."""
    import int8_quantized_linear_convrot256_b200 as ck

    a = dict(X=FAKE, ldx=5376, Qw=FAKE, s_w=FAKE, bias=None, Y=FAKE, M=8192, N=256, K=5376)
    a.update(args)
    st = ck.lib.ck_int8_linear_noalloc(a["X"], a["ldx"], a["Qw"], a["s_w"], a["bias"], a["Y"],
                                       a["M"], a["N"], a["K"], None)
    assert st == getattr(ck, status)
