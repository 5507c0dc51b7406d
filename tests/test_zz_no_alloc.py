"""The allocation-free forward (mmf_bitlinear_forward_noalloc), for callers that cannot call
cudaMalloc: its output must equal, bit for bit, that of the workspace-taking
mmf_bitlinear_forward on the same inputs, on two calls in a row (the second call reuses the
shared scratch left by the first).
Collected last on purpose, so a run that stops at the first failure has run everything else.
"""
import ctypes

import numpy as np
import pytest
import torch

import synth
import ternary_weight_lm_b200 as mmf
from gpu_helpers import DEV, assert_out_close, oracle_forward_from_parts, to_dev

SCRATCH_BYTES = 4 << 20


def _noalloc(x, Wp, beta, N, y, norm_w=None):
    T, K = x.shape
    dt = {torch.float16: mmf.MMF_F16, torch.float32: mmf.MMF_F32}
    return mmf.lib().mmf_bitlinear_forward_noalloc(
        x.data_ptr(), dt[x.dtype], T, K, None if norm_w is None else norm_w.data_ptr(),
        ctypes.c_float(1e-8), Wp.data_ptr(), beta.data_ptr(), N, y.data_ptr(), dt[y.dtype],
        torch.cuda.current_stream().cuda_stream)


@pytest.mark.gpu
def test_noalloc_matches_forward_on_two_calls():
    # The allocation-free call runs the same two kernels on the same inputs as
    # mmf_bitlinear_forward, only with its scratch elsewhere, so the outputs must agree bit for
    # bit.  Two calls in a row: the second one finds the first one's codes in the shared array.
    # The second call also covers fp32 in, fp32 out and a non-trivial norm weight.
    cases = [(64, 1024, 1024, "first", torch.float16, False),
             (17, 2816, 1024, "second", torch.float32, True)]
    for T, K, N, label, dt, with_g in cases:
        xnp = synth.activations(11, f"noalloc/{label}", T, K,
                                dtype=np.float32 if dt == torch.float32 else np.float16)
        x = to_dev(xnp)
        W = to_dev(synth.weights(11, f"noalloc/{label}", N, K))
        g = to_dev(synth.norm_weight(11, f"noalloc/{label}", K, ones=False)) if with_g else None
        Wp, beta = mmf.quantize_weights(W)
        y_ref = mmf.bitlinear_forward(x, Wp, beta, norm_w=g, out_dtype=dt)   # existing entry
        y = torch.full((T, N), float("nan"), dtype=dt, device=DEV)
        assert _noalloc(x, Wp, beta, N, y, norm_w=g) == 0
        torch.cuda.synchronize()
        assert torch.isfinite(y).all()
        assert torch.equal(y, y_ref), f"{label}: differs from mmf_bitlinear_forward"
        # and within the parity tolerance of the oracle
        y_orc = oracle_forward_from_parts(xnp, Wp.cpu().numpy(), float(beta.item()), K,
                                          g=None if g is None else g.cpu().numpy())
        assert_out_close(y.double().cpu().numpy(), y_orc)
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
