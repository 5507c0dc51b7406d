"""GPU parity of the straight-through backward against the double-precision oracle, through the
C ABI binding.  Both sides get the same activation codes and scales (the oracle's) and the same
packed weights, so the comparison isolates the backward's arithmetic.

Tolerances, derived from the arithmetic the library states:
  - dW = sum_t fp16(dy_tn * gamma_t/127) * q_tk with fp32 accumulation: every term's factor is
    rounded once to fp16 (relative error <= 2^-11, or <= 2^-25 absolute below fp16's normal
    range), so |dW - dW_ref| <= 2^-11 (|dy a| @ |q|) + T * 127 * 2^-25, plus fp32 accumulation
    (a further 1e-5 of the row's rms);
  - dxh = beta * sum_n dy_tn c_nk with exact fp16 operands and fp32 accumulation:
    |dxh error| <= E = beta * N * 2^-23 * (|dy| @ |c|); through the norm,
    |dx error| <= g E / r + |x| (sum g E |x|) / (K r^3), plus the float norm step (2e-5 of the
    row's rms and of |dx|), plus fp16 output rounding when dx is fp16;
  - dg = sum_t dxh x / r: |error| <= sum_t E |x| / r plus 2e-5 of its rms.
"""
import numpy as np
import pytest
import torch

import oracle
import synth
import ternary_weight_lm_b200 as mmf
from gpu_helpers import DEV, to_dev

pytestmark = pytest.mark.gpu


def _problem(T, K, N, seed, xdt=np.float16, with_g=False, eps=1e-8):
    x = synth.activations(seed, f"bwd{T}_{K}", T, K, dtype=xdt)
    W = synth.weights(seed, f"bwd{K}_{N}", N, K)
    Wp, beta, c = oracle.quantize_weights(W)
    g = (0.5 + np.abs(synth.normal(seed, "bwd_g", (K,), dtype=np.float32))) if with_g else None
    q, gamma, _ = oracle.rmsnorm_actquant(x.astype(np.float32), g, eps)
    dy = synth.normal(seed, f"bwd_dy{T}_{N}", (T, N), dtype=np.float16)
    return x, g, Wp, beta, c, q, gamma, dy


def _gpu(x, g, Wp, beta, q, gamma, dy, eps=1e-8, dx_dtype=torch.float32, want_dx=True,
         want_dW=True, want_dg=False, codes=True):
    dx, dW, dg = mmf.bitlinear_backward(
        to_dev(x), to_dev(Wp), torch.tensor([beta], dtype=torch.float32, device=DEV), to_dev(dy),
        norm_w=None if g is None else to_dev(g), eps=eps,
        A=to_dev(q) if codes else None, gamma=to_dev(gamma) if codes else None,
        dx_dtype=dx_dtype, want_dx=want_dx, want_dW=want_dW, want_dnorm_w=want_dg)
    torch.cuda.synchronize()
    assert mmf.mmf_get_device_status() == 0
    f = (lambda t: None if t is None else t.float().cpu().numpy().astype(np.float64))
    return f(dx), f(dW), f(dg)


def _dW_tol(dy, gamma, q):
    a = np.abs(dy.astype(np.float64)) * (gamma.astype(np.float64) / 127.0)[:, None]
    bound = 2.0 ** -11 * (a.T @ np.abs(q.astype(np.float64)))
    return bound + q.shape[0] * 127 * 2.0 ** -25


def _dxh_bound(dy, c, beta):
    N = dy.shape[1]
    return float(beta) * N * 2.0 ** -23 * (np.abs(dy.astype(np.float64)) @ np.abs(c.astype(np.float64)))


def _check_dW(dW, dW_ref, dy, gamma, q):
    rms = np.sqrt((dW_ref ** 2).mean(axis=1, keepdims=True))
    tol = _dW_tol(dy, gamma, q) + 1e-5 * rms
    bad = np.abs(dW - dW_ref) > tol
    assert not bad.any(), (np.argwhere(bad)[:5], np.abs(dW - dW_ref).max())


def _check_dx(dx, dx_ref, x, g, dy, c, beta, eps, fp16=False):
    x = x.astype(np.float64)
    K = x.shape[1]
    gg = np.ones(K) if g is None else g.astype(np.float64)
    r = np.sqrt((x * x).mean(axis=1, keepdims=True) + eps)
    E = _dxh_bound(dy, c, beta)
    bound = gg * E / r + np.abs(x) * ((gg * E * np.abs(x)).sum(axis=1, keepdims=True) / (K * r ** 3))
    rms = np.sqrt((dx_ref ** 2).mean(axis=1, keepdims=True))
    tol = bound + 2e-5 * (np.abs(dx_ref) + rms)
    if fp16:
        tol = tol + 2.0 ** -11 * np.abs(dx_ref) + 2.0 ** -24
    bad = np.abs(dx - dx_ref) > tol
    assert not bad.any(), (np.argwhere(bad)[:5], np.abs(dx - dx_ref).max())


def _check_dg(dg, dg_ref, x, dy, c, beta, eps):
    x = x.astype(np.float64)
    r = np.sqrt((x * x).mean(axis=1, keepdims=True) + eps)
    E = _dxh_bound(dy, c, beta)
    bound = (E * np.abs(x) / r).sum(axis=0)
    rms = np.sqrt((dg_ref ** 2).mean())
    bad = np.abs(dg - dg_ref) > bound + 2e-5 * (np.abs(dg_ref) + rms)
    assert not bad.any(), (np.argwhere(bad)[:5], np.abs(dg - dg_ref).max())


# T from one token to several 256-token tiles with a ragged tail; N and K with an odd number of
# 128-row halves (the second CTA of a pair reads rows past the end: zeros); K = 7040, the 2.7B
# down projection's input (27.5 tiles of 256 rows for dxh and dW); the 2.7B gate projection
# (2560 -> 14080), whose dxh contraction over N is split eight ways.
@pytest.mark.parametrize("T,K,N", [(1, 128, 128), (17, 256, 384), (300, 1024, 2048),
                                   (257, 2816, 1024), (130, 7040, 2560), (64, 2048, 5632),
                                   (33, 2560, 14080)])
def test_backward_matches_oracle(T, K, N):
    x, g, Wp, beta, c, q, gamma, dy = _problem(T, K, N, seed=T + K + N)
    dx, dW, _ = _gpu(x, g, Wp, beta, q, gamma, dy)
    dx_ref, dW_ref, _ = oracle.bitlinear_backward(x, q, gamma, c, beta, dy, want_dg=False)
    _check_dW(dW, dW_ref, dy, gamma, q)
    _check_dx(dx, dx_ref, x, g, dy, c, beta, 1e-8)


def test_backward_norm_weight_eps_fp16_out_and_dnorm_w():
    T, K, N, eps = 190, 1024, 1536, 1e-3
    x, g, Wp, beta, c, q, gamma, dy = _problem(T, K, N, seed=5, with_g=True, eps=eps)
    dx, dW, dg = _gpu(x, g, Wp, beta, q, gamma, dy, eps=eps, dx_dtype=torch.float16, want_dg=True)
    dx_ref, dW_ref, dg_ref = oracle.bitlinear_backward(x, q, gamma, c, beta, dy, g=g, eps=eps)
    _check_dW(dW, dW_ref, dy, gamma, q)
    _check_dx(dx, dx_ref, x, g, dy, c, beta, eps, fp16=True)
    _check_dg(dg, dg_ref, x, dy, c, beta, eps)


def test_backward_fp32_input():
    T, K, N = 77, 512, 640
    x, g, Wp, beta, c, q, gamma, dy = _problem(T, K, N, seed=7, xdt=np.float32)
    dx, dW, _ = _gpu(x, g, Wp, beta, q, gamma, dy)
    dx_ref, dW_ref, _ = oracle.bitlinear_backward(x, q, gamma, c, beta, dy, want_dg=False)
    _check_dW(dW, dW_ref, dy, gamma, q)
    _check_dx(dx, dx_ref, x, g, dy, c, beta, 1e-8)


def test_backward_split_contraction_over_tokens():
    # 2000 tokens and 16 output tiles: the weight gradient's token contraction is split three
    # ways (the workspace size test pins that choice on the host) and the partials summed; the
    # 300-token case above splits dxh's contraction four ways
    T, K, N = 2000, 1024, 1024
    x, g, Wp, beta, c, q, gamma, dy = _problem(T, K, N, seed=11)
    _, dW, _ = _gpu(x, g, Wp, beta, q, gamma, dy, want_dx=False)
    _, dW_ref, _ = oracle.bitlinear_backward(x, q, gamma, c, beta, dy, want_dg=False)
    _check_dW(dW, dW_ref, dy, gamma, q)


def test_backward_recomputed_codes_equal_given_codes():
    # A/gamma NULL: the call quantises x itself, with the forward's kernel; the result equals the
    # call given that kernel's codes, bit for bit
    T, K, N = 333, 768, 1280
    x, g, Wp, beta, c, _, _, dy = _problem(T, K, N, seed=13, with_g=True)
    xd = to_dev(x)
    A = torch.empty((T, K), dtype=torch.int8, device=DEV)
    gam = torch.empty(T, dtype=torch.float32, device=DEV)
    mmf.mmf_quantize_activations(xd, to_dev(g), 1e-8, A, gam)
    torch.cuda.synchronize()
    q_gpu, g_gpu = A.cpu().numpy(), gam.cpu().numpy()
    a = _gpu(x, g, Wp, beta, q_gpu, g_gpu, dy, want_dg=True)
    b = _gpu(x, g, Wp, beta, None, None, dy, want_dg=True, codes=False)
    for u, v in zip(a, b):
        np.testing.assert_array_equal(u, v)


def test_backward_outputs_are_independent():
    # asking for one output gives the same values as asking for all of them
    T, K, N = 150, 512, 512
    x, g, Wp, beta, c, q, gamma, dy = _problem(T, K, N, seed=17, with_g=True)
    dx, dW, dg = _gpu(x, g, Wp, beta, q, gamma, dy, want_dg=True)
    dx1, _, _ = _gpu(x, g, Wp, beta, q, gamma, dy, want_dW=False)
    _, dW1, _ = _gpu(x, g, Wp, beta, q, gamma, dy, want_dx=False)
    _, _, dg1 = _gpu(x, g, Wp, beta, q, gamma, dy, want_dx=False, want_dW=False, want_dg=True)
    np.testing.assert_array_equal(dx, dx1)
    np.testing.assert_array_equal(dW, dW1)
    np.testing.assert_array_equal(dg, dg1)


def test_backward_full_size_sampled():
    # the 1.3B i_proj shape at the prefill length bench.py times (32768 tokens, K = N = 2048):
    # dx of sampled tokens (a token's dx depends on that token only) and dW of sampled weight
    # rows (a row of dW depends on that column of dy only), each from the oracle
    T, K, N = 32768, 2048, 2048
    x = synth.activations(3, "bwd_full", T, K, dtype=np.float16, outlier_frac=0.01)
    W = synth.weights(3, "bwd_full", N, K)
    Wp, beta, c = oracle.quantize_weights(W)
    q, gamma, _ = oracle.rmsnorm_actquant(x.astype(np.float32), None, 1e-8)
    dy = synth.normal(3, "bwd_full_dy", (T, N), dtype=np.float16)
    dx, dW, _ = _gpu(x, None, Wp, beta, q, gamma, dy)
    ts = np.array([0, 1, 255, 256, 12345, T - 1])
    dx_ref, _, _ = oracle.bitlinear_backward(x[ts], q[ts], gamma[ts], c, beta, dy[ts],
                                             want_dg=False)
    _check_dx(dx[ts], dx_ref, x[ts], None, dy[ts], c, beta, 1e-8)
    ns = np.array([0, 127, 128, 1000, N - 1])
    _, dW_ref, _ = oracle.bitlinear_backward(x, q, gamma, c[ns], beta, dy[:, ns], want_dg=False)
    _check_dW(dW[ns], dW_ref, dy[:, ns], gamma, q)
    assert np.isfinite(dx).all() and np.isfinite(dW).all()
