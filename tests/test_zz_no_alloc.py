"""The allocation-free forward (mmf_bitlinear_forward_noalloc), for callers that cannot call
cudaMalloc: its output must match the workspace-taking mmf_bitlinear_forward on the same
inputs, on two calls in a row (the second call reuses the shared scratch left by the first).
Collected last on purpose, so a run that stops at the first failure has run everything else.
"""
import ctypes

import numpy as np
import pytest
import torch

import synth
import ternary_weight_lm_b200 as mmf
from gpu_helpers import DEV, assert_out_close, to_dev

SCRATCH_BYTES = 4 << 20


def _noalloc(x, Wp, beta, N, y):
    T, K = x.shape
    return mmf.lib().mmf_bitlinear_forward_noalloc(
        x.data_ptr(), mmf.MMF_F16, T, K, None, ctypes.c_float(1e-8), Wp.data_ptr(),
        beta.data_ptr(), N, y.data_ptr(), mmf.MMF_F16, torch.cuda.current_stream().cuda_stream)


@pytest.mark.gpu
def test_noalloc_matches_forward_on_two_calls():
    cases = [(64, 1024, 1024, "first"), (17, 2816, 1024, "second")]
    for T, K, N, label in cases:
        x = to_dev(synth.activations(11, f"noalloc/{label}", T, K))
        W = to_dev(synth.weights(11, f"noalloc/{label}", N, K))
        Wp, beta = mmf.quantize_weights(W)
        y_ref = mmf.bitlinear_forward(x, Wp, beta)            # the existing entry point
        y = torch.full((T, N), float("nan"), dtype=torch.float16, device=DEV)
        assert _noalloc(x, Wp, beta, N, y) == 0
        torch.cuda.synchronize()
        assert torch.isfinite(y).all()
        assert_out_close(y.double().cpu().numpy(), y_ref.double().cpu().numpy())
    assert mmf.mmf_get_device_status() == 0


@pytest.mark.gpu
def test_noalloc_rejects_oversized_calls():
    # T x K codes + gamma + sums beyond the 4 MiB array: rejected before any launch
    T, K, N = 512, 8192, 128
    x = torch.zeros((T, K), dtype=torch.float16, device=DEV)
    Wp = torch.zeros((N, K // 4), dtype=torch.uint8, device=DEV)
    beta = torch.ones(1, dtype=torch.float32, device=DEV)
    y = torch.zeros((T, N), dtype=torch.float16, device=DEV)
    assert T * K + 2 * 2048 > SCRATCH_BYTES
    assert _noalloc(x, Wp, beta, N, y) == 6          # MMF_ERR_WORKSPACE
    assert not y.any()
