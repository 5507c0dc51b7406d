"""GPU parity of the MLGRU recurrence + swish gate norm (and its fusion with o_proj's activation
pre-pass) against the double-precision oracle, through the C ABI binding.

Tolerances, from the arithmetic: the kernel runs the recurrence and the norm in float with the
fast exponential and reciprocal (relative error a few 1e-6 per step, damped by the gates) and
composes chunk maps in another order than the sequential oracle, so its float result is within
~1e-5 of the oracle's, far below the fp16 output's own rounding (2^-11).  Hence:
  - o (fp16): |o - o_ref| <= 2^-10 |o_ref| + 1e-4 rms(o_ref[t, :]) element-wise;
  - o (fp32) and the final state: |d| <= 1e-4 (|ref| + rms(ref));
  - fused o_proj codes against the oracle's pre-pass of o_ref rounded to fp16: at most 1 % of
    codes off by one (an fp16 rounding of o that moved by one ulp), none by more; gamma within
    2^-9 relative; against the library's own separate pre-pass of the fp16 o: identical.
"""
import numpy as np
import pytest
import torch

import oracle
import synth
import ternary_weight_lm_b200 as mmf
from gpu_helpers import DEV, to_dev

pytestmark = pytest.mark.gpu


def _inputs(T, H, seed=0, dtype=np.float16, scale=1.0):
    I = synth.normal(seed, "mlgru_I", (T, H), std=1.5 * scale, dtype=dtype)
    F = synth.normal(seed, "mlgru_F", (T, H), std=1.5 * scale, dtype=dtype)
    G = synth.normal(seed, "mlgru_G", (T, H), std=1.5 * scale, dtype=dtype)
    return I, F, G


def _run(I, F, G, h0=None, w=None, eps=1e-8, out_dtype=torch.float16):
    T, H = I.shape
    hT = torch.empty(H, dtype=torch.float32, device=DEV)
    o = mmf.mlgru_forward(to_dev(I), to_dev(F), to_dev(G),
                          h0=None if h0 is None else to_dev(h0.astype(np.float32)),
                          norm_w=None if w is None else to_dev(w.astype(np.float32)),
                          eps=eps, out_dtype=out_dtype, hT=hT)
    torch.cuda.synchronize()
    assert mmf.mmf_get_device_status() == 0
    return o.float().cpu().numpy(), hT.cpu().numpy()


def _check_o(o, o_ref, fp16=True):
    rms = np.sqrt((o_ref ** 2).mean(axis=1, keepdims=True))
    if fp16:
        tol = 2.0 ** -10 * np.abs(o_ref) + 1e-4 * rms
    else:
        tol = 1e-4 * (np.abs(o_ref) + rms)
    bad = np.abs(o - o_ref) > tol
    assert not bad.any(), (np.argwhere(bad)[:5], np.abs(o - o_ref).max())


def _check_state(hT, hT_ref):
    rms = np.sqrt((hT_ref ** 2).mean())
    assert np.all(np.abs(hT - hT_ref) <= 1e-4 * (np.abs(hT_ref) + rms))


# T around the 32-token chunk (one chunk, a boundary, a ragged second chunk), several chunks,
# more than 32 chunks (the carry scan's second round of shuffles) and more than 256 (its second
# batch of prefetched rounds); H from two to twenty warps of channel quads.
@pytest.mark.parametrize("T,H", [(1, 256), (17, 512), (32, 2048), (33, 256), (200, 2560),
                                 (2577, 1024), (8230, 256)])
def test_mlgru_matches_oracle(T, H):
    I, F, G = _inputs(T, H, seed=T + H)
    o, hT = _run(I, F, G)
    o_ref, hT_ref = oracle.mlgru_forward(I.astype(np.float64), F.astype(np.float64),
                                         G.astype(np.float64))
    _check_o(o, o_ref)
    _check_state(hT, hT_ref)


@pytest.mark.parametrize("T", [5, 300])
def test_mlgru_initial_state_norm_weight_and_eps(T):
    H = 768
    I, F, G = _inputs(T, H, seed=7)
    h0 = synth.normal(7, "mlgru_h0", (H,), std=2.0, dtype=np.float32)
    w = 0.5 + np.abs(synth.normal(7, "mlgru_w", (H,), dtype=np.float32))
    o, hT = _run(I, F, G, h0=h0, w=w, eps=1e-3)
    o_ref, hT_ref = oracle.mlgru_forward(I.astype(np.float64), F.astype(np.float64),
                                         G.astype(np.float64), h0=h0.astype(np.float64),
                                         w=w.astype(np.float64), eps=1e-3)
    _check_o(o, o_ref)
    _check_state(hT, hT_ref)


def test_mlgru_fp32_in_and_out():
    T, H = 130, 512
    I, F, G = _inputs(T, H, seed=11, dtype=np.float32)
    o, hT = _run(I, F, G, out_dtype=torch.float32)
    o_ref, hT_ref = oracle.mlgru_forward(I, F, G)
    _check_o(o, o_ref, fp16=False)
    _check_state(hT, hT_ref)


def test_mlgru_saturated_gates():
    # gates far in their tails (|F|, |I| up to ~40 and beyond the exp cap): closed gates take
    # the candidate, open ones keep the state, and nothing overflows
    T, H = 150, 256
    I, F, G = _inputs(T, H, seed=13, scale=20.0)
    F[:, :64] = 60.0
    F[:, 64:128] = -60.0
    I[:, 128:192] = -90.0
    h0 = synth.normal(13, "mlgru_h0", (H,), dtype=np.float32)
    o, hT = _run(I, F, G, h0=h0)
    assert np.isfinite(o).all() and np.isfinite(hT).all()
    o_ref, hT_ref = oracle.mlgru_forward(I.astype(np.float64), F.astype(np.float64),
                                         G.astype(np.float64), h0=h0.astype(np.float64))
    _check_o(o, o_ref)
    _check_state(hT, hT_ref)


def test_mlgru_split_sequence_carries_the_state():
    # two calls, the second starting from the first's final state, give one call's outputs
    T, H, t0 = 1000, 1024, 333
    I, F, G = _inputs(T, H, seed=17)
    o, hT = _run(I, F, G)
    o1, h1 = _run(I[:t0], F[:t0], G[:t0])
    o2, h2 = _run(I[t0:], F[t0:], G[t0:], h0=h1)
    both = np.concatenate([o1, o2])
    rms = np.sqrt((o ** 2).mean(axis=1, keepdims=True))
    assert np.all(np.abs(both - o) <= 2.0 ** -10 * np.abs(o) + 1e-4 * rms)
    _check_state(h2, hT.astype(np.float64))


def _fused(I, F, G, h0=None, w=None, eps=1e-8, qw=None, qeps=1e-8):
    T, H = I.shape
    A = torch.empty((T, H), dtype=torch.int8, device=DEV)
    gamma = torch.empty(T, dtype=torch.float32, device=DEV)
    rs = torch.empty(T, dtype=torch.int32, device=DEV)
    hT = torch.empty(H, dtype=torch.float32, device=DEV)
    need = mmf.mmf_mlgru_workspace_bytes(T, H)
    ws = mmf.workspace(need, DEV) if need else None
    mmf.mmf_mlgru_forward_quantized(
        to_dev(I), to_dev(F), to_dev(G), None if h0 is None else to_dev(h0), None if w is None
        else to_dev(w), eps, None if qw is None else to_dev(qw), qeps, A, gamma, rs, hT, ws)
    torch.cuda.synchronize()
    assert mmf.mmf_get_device_status() == 0
    return A.cpu().numpy(), gamma.cpu().numpy(), rs.cpu().numpy(), hT.cpu().numpy()


@pytest.mark.parametrize("T,H,with_qw", [(3, 512, False), (190, 2048, True), (700, 2560, False)])
def test_mlgru_fused_oproj_quantisation(T, H, with_qw):
    I, F, G = _inputs(T, H, seed=19 + T)
    qw = (0.5 + np.abs(synth.normal(19, "oproj_w", (H,), dtype=np.float32))) if with_qw else None
    A, gamma, rs, hT = _fused(I, F, G, qw=qw)
    # against the oracle: the oracle's o rounded to fp16, then the oracle's pre-pass
    o_ref, hT_ref = oracle.mlgru_forward(I.astype(np.float64), F.astype(np.float64),
                                         G.astype(np.float64))
    o16 = o_ref.astype(np.float16).astype(np.float32)
    q_ref, g_ref, rs_ref = oracle.rmsnorm_actquant(o16, qw, 1e-8)
    d = A.astype(np.int32) - q_ref.astype(np.int32)
    assert np.abs(d).max() <= 1
    assert (d != 0).mean() <= 1e-2
    assert np.all(np.abs(gamma - g_ref) <= 2.0 ** -9 * g_ref)
    assert np.all(np.abs(rs - rs_ref) <= np.abs(d).sum(axis=1))
    _check_state(hT, hT_ref)
    # against the library's own two steps: fp16 o, then the separate pre-pass
    o16_gpu = mmf.mlgru_forward(to_dev(I), to_dev(F), to_dev(G), out_dtype=torch.float16)
    A2 = torch.empty((T, H), dtype=torch.int8, device=DEV)
    g2 = torch.empty(T, dtype=torch.float32, device=DEV)
    rs2 = torch.empty(T, dtype=torch.int32, device=DEV)
    mmf.mmf_quantize_activations(o16_gpu, None if qw is None else to_dev(qw), 1e-8, A2, g2, rs2)
    torch.cuda.synchronize()
    np.testing.assert_array_equal(A, A2.cpu().numpy())
    np.testing.assert_array_equal(gamma, g2.cpu().numpy())
    np.testing.assert_array_equal(rs, rs2.cpu().numpy())


def test_mlgru_fused_feeds_oproj():
    # the fused codes go straight into the quantised contraction (o_proj, K = H)
    T, H, N = 40, 1024, 1024
    I, F, G = _inputs(T, H, seed=23)
    A, gamma, rs, _ = _fused(I, F, G)
    W = synth.weights(23, "oproj", N, H)
    Wp, beta, c = oracle.quantize_weights(W)
    y = torch.empty((T, N), dtype=torch.float16, device=DEV)
    mmf.mmf_bitlinear_forward_quantized(to_dev(A), to_dev(gamma), to_dev(rs), to_dev(Wp),
                                        torch.tensor([beta], device=DEV), N, False, y)
    torch.cuda.synchronize()
    acc = oracle.ternary_accumulate(A, c)
    y_ref = oracle.dequant(acc, gamma, beta)
    tol = 1e-2 * np.abs(y_ref).max(axis=1, keepdims=True)
    assert np.all(np.abs(y.float().cpu().numpy() - y_ref) <= tol)


def test_mlgru_full_size_first_rows():
    # the 1.3B prefill shape, as bench.py times it: every output row depends only on the tokens
    # up to it, so the first 2048 rows are checked against the oracle over those tokens
    T, H, Tc = 32768, 2048, 2048
    I, F, G = _inputs(T, H, seed=29)
    o, hT = _run(I, F, G)
    o_ref, _ = oracle.mlgru_forward(I[:Tc].astype(np.float64), F[:Tc].astype(np.float64),
                                    G[:Tc].astype(np.float64))
    _check_o(o[:Tc], o_ref)
    assert np.isfinite(o).all() and np.isfinite(hT).all()
    # and the last rows from the first run's state after token T - 512 (a second call)
    o_tail, h_tail = _run(I[-512:], F[-512:], G[-512:],
                          h0=_run(I[:-512], F[:-512], G[:-512])[1])
    rms = np.sqrt((o[-512:] ** 2).mean(axis=1, keepdims=True))
    assert np.all(np.abs(o_tail - o[-512:]) <= 2.0 ** -10 * np.abs(o[-512:]) + 1e-4 * rms)
    _check_state(h_tail, hT.astype(np.float64))
