"""ck_int8_linear_noalloc: the linear for callers that cannot allocate device
memory (a plugin inside an engine that owns all device memory, code with a
memory budget fixed at start-up, code that must not risk the device-wide
synchronisation cudaFree can cause). It keeps the activation codes and row
scales in the library's fixed device array instead of a caller workspace, so
it must give the same output as ck_int8_linear with a workspace.

This file is named to be collected last: if it fails in a run that stops at
the first failure, every other test has already run. It passes on its own in
a fresh process as well as after the other tests.
"""
import ctypes

import numpy as np
import pytest
import torch

import workloads

BF16_ULP_TOL = 1


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
        d = _ulp_distance(workloads.bf16_bits(out.cpu()), workloads.bf16_bits(ref.cpu()))
        assert d <= BF16_ULP_TOL, (M, K, N, d)
    assert ck.device_error() == ck.CK_OK


def test_noalloc_rejects_problems_larger_than_its_array():
    import int8_quantized_linear_convrot256_b200 as ck

    fake = 0x10000  # never dereferenced: the size check comes first
    M, K = 8192, 5376  # 44 MB of codes > 32 MiB
    assert ck.workspace_bytes(M, K) > ck.NOALLOC_SCRATCH_BYTES
    st = ck.lib.ck_int8_linear_noalloc(fake, K, fake, fake, None, fake, M, 256, K, None)
    assert st == ck.CK_ERR_WORKSPACE
    assert ck.lib.ck_int8_linear_noalloc(fake, K, fake, fake, None, fake, 0, 256, K, None) == ck.CK_OK
