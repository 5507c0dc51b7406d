"""GPU parity: the CUDA path through the C ABI against the oracle, element by element.

Bit-exact: beta, ternary codes and packed bytes, int32 accumulators given the same int8 codes.
Tolerance: int8 activation codes (<= 0.1 % off by 1), fp16/fp32 outputs (max error <= 1e-2 of
each row's largest magnitude).  Sizes span several tiles along every dimension with ragged
token tails, every token-tile width of the contraction kernel (16, 32, 64, 128, 256) and the
shapes of the model zoo's projections.
"""
import numpy as np
import pytest
import torch

import oracle
import synth
import ternary_weight_lm_b200 as mmf
from gpu_helpers import (DEV, assert_codes_close, assert_out_close, gpu_accumulate,
                         gpu_act_quant, gpu_forward, gpu_quantize_weights,
                         oracle_forward_from_parts, to_dev)

pytestmark = pytest.mark.gpu


# ---------------------------------------------------------------------------- weights
@pytest.mark.parametrize("N,K", [(128, 128), (512, 256), (384, 1152), (1024, 2816),
                                 (5632, 1024)])
@pytest.mark.parametrize("dt", [np.float32, np.float16])
def test_quantize_weights_bit_exact(N, K, dt):
    W = synth.weights(N + K, f"qw{N}x{K}", N, K, dtype=dt)
    Wp, beta = gpu_quantize_weights(W)
    beta_ref = oracle.absmean_beta(W)
    assert beta == beta_ref, (beta, beta_ref)
    Wp_ref, _, _ = oracle.quantize_weights(W)
    np.testing.assert_array_equal(Wp, Wp_ref)


def test_quantize_weights_special_values():
    rng = np.random.default_rng(0)
    W = (rng.standard_normal((256, 256)) * 0.02).astype(np.float32)
    W.reshape(-1)[:64] = np.array([1e-40, 3e38, -1e30, 2.5, -0.0, 7e-39, 1.4e-45, 65504.0] * 8,
                                  np.float32)
    Wp, beta = gpu_quantize_weights(W)
    assert beta == oracle.absmean_beta(W)
    np.testing.assert_array_equal(Wp, oracle.quantize_weights(W)[0])
    # all zeros: beta floors at 1e-5, every code 0 (packed byte 0x55)
    Z = np.zeros((128, 128), np.float32)
    Wp, beta = gpu_quantize_weights(Z)
    assert beta == np.float32(1e-5)
    assert np.all(Wp == 0x55)
    # W = a * S: beta = a, codes = S
    a = np.float32(0.0173)
    S = np.where(synth.ternary(5, "sgn", 256, 384, p_zero=0.0) > 0, 1, -1).astype(np.float32)
    Wp, beta = gpu_quantize_weights(a * S)
    assert beta == a
    np.testing.assert_array_equal(oracle.unpack_codes(Wp, 384), S.astype(np.int8))


def test_ternary_encode_given_beta():
    W = synth.weights(3, "enc", 640, 512)
    beta = np.float32(0.0123)
    Wp = torch.empty((640, 128), dtype=torch.uint8, device=DEV)
    mmf.mmf_ternary_encode(to_dev(W), torch.tensor([beta], device=DEV), Wp)
    torch.cuda.synchronize()
    np.testing.assert_array_equal(Wp.cpu().numpy(),
                                  oracle.pack_codes(oracle.ternary_codes(W, beta)))


# ---------------------------------------------------------------------------- activations
@pytest.mark.parametrize("T,K,dt,outliers,gw", [
    (1, 128, np.float16, 0.0, False), (37, 1024, np.float16, 0.0, True),
    (64, 2816, np.float16, 0.0, False), (300, 2048, np.float16, 0.01, False),
    (16, 256, np.float32, 0.0, False), (9, 7040, np.float16, 0.01, True),
    (5, 8192, np.float32, 0.0, True), (3, 8192, np.float16, 0.0, False),
    # T >= 256: one warp per row, 8 / 16 / 24 vectors per lane, with and without a norm weight
    (300, 2048, np.float16, 0.01, True), (264, 4096, np.float16, 0.0, False),
    (260, 5632, np.float16, 0.01, True), (257, 5632, np.float16, 0.0, False),
    (300, 1024, np.float32, 0.01, True), (256, 2816, np.float32, 0.0, False),
    (259, 2816, np.float32, 0.0, True),
])
def test_quantize_activations(T, K, dt, outliers, gw):
    x = synth.activations(T * 7 + K, f"aq{T}x{K}", T, K, dtype=dt, outlier_frac=outliers)
    g = synth.norm_weight(T, f"aq{K}", K, ones=not gw)
    A, gamma, rs = gpu_act_quant(x, g=g if gw else None)
    q_ref, gamma_ref, rs_ref = oracle.rmsnorm_actquant(x, g=g if gw else None)
    assert_codes_close(A, q_ref)
    np.testing.assert_array_equal(rs, A.astype(np.int64).sum(axis=1))
    # gamma: within one float ulp of the oracle's (exact unless a sum of squares rounds
    # differently in its last double bit)
    ulp = np.spacing(gamma_ref)
    assert np.all(np.abs(gamma - gamma_ref) <= ulp)


def test_quantize_activations_zero_and_constant_rows():
    x = np.zeros((4, 512), np.float16)
    x[1, :] = 0.75
    x[2, 100] = -2.0
    A, gamma, rs = gpu_act_quant(x)
    assert not A[0].any() and gamma[0] == np.float32(1e-5) and rs[0] == 0
    assert np.all(A[1] == 127) and rs[1] == 127 * 512
    assert A[2, 100] == -127 and np.count_nonzero(A[2]) == 1


# ---------------------------------------------------------------------------- accumulator
@pytest.mark.parametrize("T", [1, 7, 16, 17, 33, 64, 65, 100, 128, 129, 300, 517, 1111])
@pytest.mark.parametrize("N,K", [(128, 128), (384, 1152), (512, 640)])
def test_accumulate_i32_bit_exact(T, N, K):
    q = synth.int8_codes(T, f"acc{T}", T, K)
    c = synth.ternary(N, f"acc{N}x{K}", N, K)
    Wp = oracle.pack_codes(c)
    acc = gpu_accumulate(q, Wp)
    np.testing.assert_array_equal(acc, oracle.ternary_accumulate(q, c))


def test_accumulate_i32_extremes():
    # every activation code at -128 or 127 against all +1 / all -1 rows: largest magnitudes
    T, N, K = 16, 256, 8192
    q = np.full((T, K), 127, np.int8)
    q[1::2] = -128
    c = np.ones((N, K), np.int8)
    c[1::2] = -1
    acc = gpu_accumulate(q, oracle.pack_codes(c))
    np.testing.assert_array_equal(acc, oracle.ternary_accumulate(q, c))
    assert acc.max() == 128 * K and acc.min() == -128 * K   # (-128) * (-1) * K at the top


# ---------------------------------------------------------------------------- forward
@pytest.mark.parametrize("T,K,N,dt,odt", [
    (16, 256, 512, np.float32, torch.float32),          # the tiny single-projection workload
    (1, 1024, 1024, np.float16, torch.float16),
    (8, 2048, 2048, np.float16, torch.float16),
    (64, 2816, 1024, np.float16, torch.float16),
    (77, 640, 384, np.float16, torch.float32),
    (300, 1024, 256, np.float16, torch.float16),
    # the 2.7B-shaped down_proj (K = 7040, a partial last 512-wide k stage) at decode and
    # above the 256-token tile
    (8, 7040, 2560, np.float16, torch.float16),
    (300, 7040, 2560, np.float16, torch.float16),
    # the persistent prefill kernel (T > 128): fp32 output, ragged last token tile, more
    # tiles than SMs
    (200, 640, 384, np.float16, torch.float32),
    (1000, 1024, 1024, np.float16, torch.float16),
    (1500, 512, 1280, np.float32, torch.float16),
])
def test_forward_parity(T, K, N, dt, odt):
    x = synth.activations(T + N, f"fw{T}", T, K, dtype=dt)
    W = synth.weights(K + N, f"fw{N}x{K}", N, K)
    Wp, beta = gpu_quantize_weights(W)
    y = gpu_forward(x, Wp, beta, out_dtype=odt)
    y_ref, beta_ref = oracle.bitlinear_forward(x, W)
    assert beta == beta_ref
    assert_out_close(y, y_ref)


@pytest.mark.parametrize("T,K,I,odt", [(1, 1024, 2816, torch.float16),
                                       (64, 1024, 2816, torch.float16),
                                       (8, 2048, 5632, torch.float16),
                                       (130, 512, 192, torch.float16),
                                       (16, 2560, 7040, torch.float16),
                                       (300, 768, 320, torch.float32),
                                       (777, 512, 640, torch.float16)])
def test_glu_forward_parity(T, K, I, odt):
    x = synth.activations(T + I, f"glu{T}", T, K)
    W = synth.weights(K + I, f"glu{I}x{K}", 2 * I, K)
    Wp, beta = gpu_quantize_weights(W)
    h = gpu_forward(x, Wp, beta, glu=True, out_dtype=odt)
    h_ref, beta_ref = oracle.bitlinear_forward(x, W, glu=True)
    assert beta == beta_ref
    assert_out_close(h, h_ref)


@pytest.mark.parametrize("T,K,N,glu,odt", [(300, 1024, 512, False, torch.float16),
                                            (257, 640, 768, True, torch.float16),
                                            (1000, 512, 1024, False, torch.float32),
                                            (513, 768, 512, True, torch.float32)])
def test_quantized_forward_both_contractions_agree(T, K, N, glu, odt):
    """From the same activation codes, the prefill contraction that expands the weights into a
    workspace and the one that needs none give the same bits, and match the oracle."""
    x = synth.activations(T + K, f"qf{T}", T, K)
    W = synth.weights(N + K, f"qf{N}x{K}", N, K)
    Wp, beta = gpu_quantize_weights(W)
    A, gamma, rs = (to_dev(v) for v in gpu_act_quant(x))
    Wpd, bd = to_dev(Wp), torch.tensor([beta], dtype=torch.float32, device=DEV)
    n_out = N // 2 if glu else N
    outs = []
    for use_ws in (True, False):
        y = torch.full((T, n_out), float("nan"), dtype=odt, device=DEV)
        ws = mmf.workspace(mmf.mmf_quantized_workspace_bytes(T, K, N), DEV) if use_ws else None
        mmf.mmf_bitlinear_forward_quantized(A, gamma, rs, Wpd, bd, N, glu, y, ws)
        torch.cuda.synchronize()
        outs.append(y.cpu())
    assert torch.isfinite(outs[0]).all()
    assert torch.equal(outs[0], outs[1])
    y_ref = oracle_forward_from_parts(x, Wp, beta, K, glu=glu)
    assert_out_close(outs[0].double().numpy(), y_ref)


def test_forward_norm_weight_and_zero_rows():
    T, K, N = 20, 768, 256
    x = synth.activations(1, "nz", T, K)
    x[3] = 0
    g = synth.norm_weight(1, "nz", K, ones=False)
    W = synth.weights(1, "nz", N, K)
    Wp, beta = gpu_quantize_weights(W)
    y = gpu_forward(x, Wp, beta, g=g)
    y_ref = oracle_forward_from_parts(x, Wp, beta, K, g=g)
    assert_out_close(y, y_ref)
    assert not y[3].any()


def test_block_projections_370m_t64():
    """All six FusedBitLinear projections of a 370M-shaped block at 64 tokens, with down_proj
    fed by the GLU output of gate_proj as in the MLP."""
    wl = synth.WORKLOADS["hgrn370m_block_t64"]
    T = wl.T
    xs = {src: synth.activations(0, src, T, 1024) for src in ("x_attn", "x_o", "x_mlp")}
    h_gpu = h_ref = None
    for p in wl.projections:
        W = synth.weights(0, p.name, p.N, p.K)
        Wp, beta = gpu_quantize_weights(W)
        if p.src == "h":
            x_gpu = h_gpu.astype(np.float16)
            x_ref = h_gpu.astype(np.float16)   # same fp16 input on both sides
        else:
            x_gpu = x_ref = xs[p.src]
        y = gpu_forward(x_gpu, Wp, beta, glu=p.glu)
        y_ref = oracle_forward_from_parts(x_ref, Wp, beta, p.K, glu=p.glu)
        assert_out_close(y, y_ref)
        if p.glu:
            h_gpu, h_ref = y, y_ref


def _sampled_rows(T, n, seed):
    rows = np.random.default_rng(seed).choice(T, n, replace=False)
    rows[0], rows[-1] = 0, T - 1
    return rows


def test_prefill_sampled_rows_1p3b_gate():
    """The 1.3B prefill gate_proj at full size (32768 tokens, 1 % outliers x20): every
    activation code, and every output of 24 sampled token rows, against the oracle."""
    T, K, I = 32768, 2048, 5632
    x = synth.activations(0, "prefill", T, K, outlier_frac=0.01)
    W = synth.weights(0, "prefill_gate", 2 * I, K)
    Wp, beta = gpu_quantize_weights(W)
    assert beta == oracle.absmean_beta(W)
    A, gamma, _ = gpu_act_quant(x)
    q_ref, gamma_ref, _ = oracle.rmsnorm_actquant(x)
    assert_codes_close(A, q_ref)
    h = gpu_forward(x, Wp, beta, glu=True)
    rows = _sampled_rows(T, 24, 1)
    h_ref = oracle_forward_from_parts(x[rows], Wp, beta, K, glu=True)
    assert_out_close(h[rows], h_ref)


def test_prefill_sampled_rows_2p7b_gate_and_down():
    """The 2.7B prefill shapes at full size: gate_proj 2560 -> 14080 with the GLU at 8192
    tokens, then down_proj 7040 -> 2560 fed by its fp16 GLU output.  Every activation code of
    both inputs, and 16 sampled token rows of both outputs, against the oracle."""
    T, H, I = 8192, 2560, 7040
    x = synth.activations(0, "prefill27", T, H)
    Wg = synth.weights(0, "prefill27_gate", 2 * I, H)
    Wd = synth.weights(0, "prefill27_down", H, I)
    Wpg, bg = gpu_quantize_weights(Wg)
    Wpd, bd = gpu_quantize_weights(Wd)
    assert bg == oracle.absmean_beta(Wg) and bd == oracle.absmean_beta(Wd)
    rows = _sampled_rows(T, 16, 2)
    A, _, _ = gpu_act_quant(x)
    assert_codes_close(A, oracle.rmsnorm_actquant(x)[0])
    h = gpu_forward(x, Wpg, bg, glu=True)
    assert_out_close(h[rows], oracle_forward_from_parts(x[rows], Wpg, bg, H, glu=True))
    h16 = h.astype(np.float16)                  # down_proj reads the fp16 GLU output
    A, _, _ = gpu_act_quant(h16)
    assert_codes_close(A, oracle.rmsnorm_actquant(h16)[0])
    y = gpu_forward(h16, Wpd, bd)
    assert_out_close(y[rows], oracle_forward_from_parts(h16[rows], Wpd, bd, I))


# ---------------------------------------------------------------------------- status
def test_wait_timeout_probe_reports_and_context_survives():
    assert mmf.mmf_get_device_status() == 0
    mmf.mmf_debug_wait_timeout_probe(5_000_000)     # 5 ms
    torch.cuda.synchronize()
    assert mmf.mmf_get_device_status() == 5         # MMF_ERR_TIMEOUT
    assert mmf.mmf_get_device_status() == 0         # reading cleared it
    # the context is still usable
    q = synth.int8_codes(0, "after", 4, 256)
    c = synth.ternary(0, "after", 128, 256)
    np.testing.assert_array_equal(gpu_accumulate(q, oracle.pack_codes(c)),
                                  oracle.ternary_accumulate(q, c))
