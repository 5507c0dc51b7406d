"""Shared helpers for the GPU parity tests: move seeded numpy inputs to the device, call the
library through its C ABI binding, and compare with the oracle."""
import numpy as np
import torch

import oracle
import ternary_weight_lm_b200 as mmf

DEV = "cuda:0"

# Tolerances (the projection's parity criteria):
#  - activation codes: at most 0.1 % of codes off by exactly 1, none by more;
#  - outputs: |y_gpu - y_oracle| <= 1e-2 * max_n |y_oracle[t, :]| for every token row t.
CODE_MISMATCH_FRAC = 1e-3
OUT_REL_TOL = 1e-2


def to_dev(a, dtype=None):
    t = torch.from_numpy(np.ascontiguousarray(a))
    if dtype is not None:
        t = t.to(dtype)
    return t.to(DEV)


def gpu_quantize_weights(W):
    Wd = to_dev(W)
    Wp, beta = mmf.quantize_weights(Wd)
    torch.cuda.synchronize()
    return Wp.cpu().numpy(), np.float32(beta.cpu().numpy()[0])


def gpu_act_quant(x, g=None, eps=1e-8):
    xd = to_dev(x)
    T, K = x.shape
    A = torch.empty((T, K), dtype=torch.int8, device=DEV)
    gamma = torch.empty(T, dtype=torch.float32, device=DEV)
    rs = torch.empty(T, dtype=torch.int32, device=DEV)
    gd = None if g is None else to_dev(g.astype(np.float32))
    mmf.mmf_quantize_activations(xd, gd, eps, A, gamma, rs)
    torch.cuda.synchronize()
    return A.cpu().numpy(), gamma.cpu().numpy(), rs.cpu().numpy()


def gpu_accumulate(q, Wp):
    T, K = q.shape
    N = Wp.shape[0]
    acc = torch.empty((T, N), dtype=torch.int32, device=DEV)
    ws = mmf.workspace(mmf.mmf_forward_workspace_bytes(T, K, N), DEV)
    mmf.mmf_ternary_accumulate_i32(to_dev(q), to_dev(Wp), N, acc, ws)
    torch.cuda.synchronize()
    return acc.cpu().numpy()


def gpu_forward(x, Wp, beta, g=None, eps=1e-8, glu=False, out_dtype=torch.float16):
    xd = to_dev(x)
    Wpd = to_dev(Wp)
    bd = torch.tensor([beta], dtype=torch.float32, device=DEV)
    gd = None if g is None else to_dev(g.astype(np.float32))
    f = mmf.bitlinear_glu_forward if glu else mmf.bitlinear_forward
    y = f(xd, Wpd, bd, norm_w=gd, eps=eps, out_dtype=out_dtype)
    torch.cuda.synchronize()
    return y.float().cpu().numpy().astype(np.float64)


def assert_codes_close(A_gpu, A_ref):
    d = A_gpu.astype(np.int32) - A_ref.astype(np.int32)
    assert np.abs(d).max(initial=0) <= 1, "an activation code differs by more than 1"
    frac = np.count_nonzero(d) / d.size
    assert frac <= CODE_MISMATCH_FRAC, f"{frac:.2e} of activation codes differ by 1"
    return frac


def assert_out_close(y_gpu, y_ref):
    scale = np.abs(y_ref).max(axis=1, keepdims=True)
    scale = np.where(scale > 0, scale, 1.0)
    err = np.abs(y_gpu - y_ref) / scale
    worst = float(err.max(initial=0.0))
    assert worst <= OUT_REL_TOL, f"max relative error {worst:.3e}"
    return worst


def oracle_forward_from_parts(x, Wp, beta, K, g=None, eps=1e-8, glu=False):
    """The oracle's projection given the already packed weights and beta."""
    q, gamma, _ = oracle.rmsnorm_actquant(x, g=g, eps=eps)
    c = oracle.unpack_codes(Wp, K)
    acc = oracle.ternary_accumulate(q, c)
    y = oracle.dequant(acc, gamma, beta)
    return oracle.silu_glu(y) if glu else y
