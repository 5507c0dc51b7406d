"""Host-side checks of the C ABI: the library loads without a GPU, exports every entry point
that include/mmf.h declares, and rejects bad arguments on the host before any launch."""
import ctypes
import os
import re
import subprocess

import pytest

import ternary_weight_lm_b200 as mmf

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "mmf.h")

OK, INVALID, SHAPE, ALIGN, CUDA, TIMEOUT, WS = 0, 1, 2, 3, 4, 5, 6


def declared_functions():
    text = open(HEADER, encoding="utf-8").read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    names = re.findall(r"^\s*(?:const\s+)?[A-Za-z_][A-Za-z0-9_]*\s*\*?\s*(mmf_[a-z0-9_]+)\s*\(",
                       text, flags=re.M)
    return sorted(set(names))


def test_library_builds_and_loads():
    from ternary_weight_lm_b200 import build
    build.build()
    assert mmf.mmf_version() == 100


def test_every_declared_symbol_is_exported():
    names = declared_functions()
    assert len(names) >= 12, names
    L = ctypes.CDLL(mmf.lib_path)
    for n in names:
        assert hasattr(L, n), n
    out = subprocess.run(["nm", "-D", "--defined-only", mmf.lib_path], capture_output=True,
                         text=True, check=True).stdout
    exported = sorted({ln.split()[-1] for ln in out.splitlines() if " T " in ln})
    assert exported == names


def test_status_strings():
    for code, name in mmf.STATUS.items():
        assert mmf.mmf_status_string(code) == name


def test_workspace_sizes():
    L = mmf.lib()
    assert L.mmf_quantize_weights_workspace_bytes(2048, 2048) == 4096
    # A [T x K] + gamma [T] + rowsum [T], each rounded up to 256 bytes
    assert L.mmf_forward_workspace_bytes(64, 1024, 1024) == 64 * 1024 + 256 + 256
    assert L.mmf_forward_workspace_bytes(3, 128, 128) == 512 + 256 + 256
    assert L.mmf_forward_workspace_bytes(0, 128, 128) == 0
    # more than 128 tokens: also the weight codes expanded to int8, N x K
    assert L.mmf_forward_workspace_bytes(300, 256, 512) == 300 * 256 + 2 * 1280 + 512 * 256
    assert L.mmf_quantized_workspace_bytes(300, 256, 512) == 512 * 256
    assert L.mmf_quantized_workspace_bytes(128, 256, 512) == 0


A16 = 0x10000   # fake, aligned "device" addresses: never dereferenced by rejected calls


def fwd(**kw):
    a = dict(x=A16, xdt=1, T=4, K=256, g=None, eps=1e-8, Wp=A16, beta=A16, N=256, y=A16, ydt=1,
             ws=A16, wsb=1 << 20, stream=None)
    a.update(kw)
    return mmf.lib().mmf_bitlinear_forward(a["x"], a["xdt"], a["T"], a["K"], a["g"], a["eps"],
                                           a["Wp"], a["beta"], a["N"], a["y"], a["ydt"], a["ws"],
                                           a["wsb"], a["stream"])


@pytest.mark.parametrize("kw,code", [
    (dict(x=None), INVALID), (dict(Wp=None), INVALID), (dict(beta=None), INVALID),
    (dict(y=None), INVALID), (dict(xdt=2), INVALID), (dict(ydt=-1), INVALID),
    (dict(eps=0.0), INVALID), (dict(eps=-1e-8), INVALID), (dict(eps=float("nan")), INVALID),
    (dict(T=0), SHAPE), (dict(T=-3), SHAPE), (dict(K=100), SHAPE), (dict(K=64), SHAPE),
    (dict(K=8320), SHAPE), (dict(N=192), SHAPE), (dict(N=0), SHAPE),
    (dict(x=A16 + 8), ALIGN), (dict(y=A16 + 2), ALIGN), (dict(Wp=A16 + 4), ALIGN),
    (dict(g=A16 + 4), ALIGN), (dict(ws=A16 + 16), ALIGN),
    (dict(ws=None), WS), (dict(wsb=100), WS),
])
def test_forward_rejects_on_host(kw, code):
    assert fwd(**kw) == code


def test_glu_and_other_entry_points_reject_on_host():
    L = mmf.lib()
    # N2 must be a multiple of 128 (so that I is a multiple of 64)
    assert L.mmf_bitlinear_glu_forward(A16, 1, 4, 256, None, 1e-8, A16, A16, 192, A16, 1, A16,
                                       1 << 20, None) == SHAPE
    assert L.mmf_quantize_weights(None, 0, 128, 128, A16, A16, A16, 4096, None) == INVALID
    assert L.mmf_quantize_weights(A16, 0, 128, 120, A16, A16, A16, 4096, None) == SHAPE
    assert L.mmf_quantize_weights(A16, 0, 128, 128, A16, A16, A16, 100, None) == WS
    assert L.mmf_quantize_weights(A16 + 4, 0, 128, 128, A16, A16, A16, 4096, None) == ALIGN
    assert L.mmf_ternary_encode(A16, 5, 128, 128, A16, A16, None) == INVALID
    assert L.mmf_quantize_activations(A16, 1, 4, 256, None, 0.0, A16, A16, None, None) == INVALID
    assert L.mmf_quantize_activations(A16, 1, 4, 200, None, 1e-8, A16, A16, None, None) == SHAPE
    assert L.mmf_ternary_accumulate_i32(A16, 4, 256, A16, 256, A16 + 4, A16, 1 << 20,
                                        None) == ALIGN
    assert L.mmf_ternary_accumulate_i32(A16, 4, 256, A16, 256, A16, A16, 10, None) == WS
    # a non-null workspace smaller than the query, or a size without a workspace
    assert L.mmf_bitlinear_forward_quantized(A16, A16, A16, 300, 256, A16, A16, 512, 0, A16, 1,
                                             A16, 1024, None) == WS
    assert L.mmf_bitlinear_forward_quantized(A16, A16, A16, 300, 256, A16, A16, 512, 0, A16, 1,
                                             None, 1024, None) == WS
    assert L.mmf_debug_wait_timeout_probe(10, None) == INVALID
    assert L.mmf_debug_wait_timeout_probe(10 ** 10, None) == INVALID


def test_valid_call_without_gpu_reports_cuda_error():
    # With no CUDA device the call must fail loudly (no host fallback exists).
    import torch
    if torch.cuda.is_available():
        pytest.skip("a GPU is present")
    assert fwd() == CUDA
    with pytest.raises(mmf.MMFError):
        mmf._check("mmf_bitlinear_forward", fwd())


def test_program_run_refuses_a_workspace_without_a_plan():
    # A workspace that no successful mmf_program_init planned is refused on the host, before
    # any launch (the run could not know the plan's token tile or grid).
    L = mmf.lib()
    assert L.mmf_program_run(A16, None) == INVALID
    assert L.mmf_program_run(None, None) == INVALID


def test_program_init_rejects_on_host():
    L = mmf.lib()
    p = mmf.Projection(A16, 1, None, A16, A16, 256, 256, 0, 0, A16, 1)
    arr = (mmf.Projection * 1)(p)
    assert L.mmf_program_init(arr, 1, 65, 1e-8, A16, 1 << 30, None) == SHAPE   # T > 64
    assert L.mmf_program_init(arr, 1, 8, 0.0, A16, 1 << 30, None) == INVALID   # eps
    assert L.mmf_program_init(arr, 0, 8, 1e-8, A16, 1 << 30, None) == INVALID  # no projection
    assert L.mmf_program_init(arr, 1, 8, 1e-8, None, 1 << 30, None) == WS
    assert L.mmf_program_init(arr, 1, 8, 1e-8, A16 + 16, 1 << 30, None) == ALIGN
    bad = (mmf.Projection * 1)(mmf.Projection(A16, 1, None, A16, A16, 200, 256, 0, 0, A16, 1))
    assert L.mmf_program_init(bad, 1, 8, 1e-8, A16, 1 << 30, None) == SHAPE      # K % 128
    assert L.mmf_program_workspace_bytes(bad, 1, 8) == 0


# ---------------------------------------------------------------------------------- MLGRU
def test_mlgru_workspace_sizes():
    L = mmf.lib()
    # chunk maps a, b and the carries: three [chunks x H] fp32 arrays, 256-byte rounded
    assert L.mmf_mlgru_workspace_bytes(32768, 2048) == 3 * 1024 * 2048 * 4
    assert L.mmf_mlgru_workspace_bytes(65, 256) == 3 * 3 * 256 * 4
    assert L.mmf_mlgru_workspace_bytes(32, 2048) == 0      # one chunk: no scan across chunks
    assert L.mmf_mlgru_workspace_bytes(1, 4096) == 0
    assert L.mmf_mlgru_workspace_bytes(100, 200) == 0      # unsupported H
    assert L.mmf_mlgru_workspace_bytes(0, 256) == 0


def mlgru(**kw):
    a = dict(I=A16, F=A16, G=A16, xdt=1, T=200, H=512, h0=None, w=None, eps=1e-8, o=A16, odt=1,
             hT=None, ws=A16, wsb=1 << 20, stream=None)
    a.update(kw)
    return mmf.lib().mmf_mlgru_forward(a["I"], a["F"], a["G"], a["xdt"], a["T"], a["H"],
                                       a["h0"], a["w"], a["eps"], a["o"], a["odt"], a["hT"],
                                       a["ws"], a["wsb"], a["stream"])


@pytest.mark.parametrize("kw,code", [
    (dict(I=None), INVALID), (dict(F=None), INVALID), (dict(G=None), INVALID),
    (dict(o=None), INVALID), (dict(xdt=3), INVALID), (dict(odt=2), INVALID),
    (dict(eps=0.0), INVALID), (dict(eps=float("nan")), INVALID), (dict(eps=2.0), INVALID),
    (dict(T=0), SHAPE), (dict(H=128), SHAPE), (dict(H=768 + 128), SHAPE), (dict(H=4352), SHAPE),
    (dict(I=A16 + 8), ALIGN), (dict(o=A16 + 2), ALIGN), (dict(h0=A16 + 4), ALIGN),
    (dict(hT=A16 + 4), ALIGN), (dict(w=A16 + 4), ALIGN), (dict(ws=A16 + 16), ALIGN),
    (dict(ws=None, wsb=0), WS), (dict(wsb=100), WS), (dict(T=32, ws=None, wsb=8), WS),
])
def test_mlgru_rejects_on_host(kw, code):
    assert mlgru(**kw) == code


@pytest.mark.parametrize("kw,code", [
    (dict(A=None), INVALID), (dict(gamma=None), INVALID), (dict(qeps=0.0), INVALID),
    (dict(A=A16 + 8), ALIGN), (dict(gamma=A16 + 2), ALIGN), (dict(rowsum=A16 + 2), ALIGN),
    (dict(qw=A16 + 4), ALIGN), (dict(H=100), SHAPE), (dict(wsb=16), WS),
])
def test_mlgru_quantized_rejects_on_host(kw, code):
    a = dict(I=A16, F=A16, G=A16, xdt=1, T=200, H=512, h0=None, w=None, eps=1e-8, qw=None,
             qeps=1e-8, A=A16, gamma=A16, rowsum=A16, hT=None, ws=A16, wsb=1 << 20, stream=None)
    a.update(kw)
    assert mmf.lib().mmf_mlgru_forward_quantized(
        a["I"], a["F"], a["G"], a["xdt"], a["T"], a["H"], a["h0"], a["w"], a["eps"], a["qw"],
        a["qeps"], a["A"], a["gamma"], a["rowsum"], a["hT"], a["ws"], a["wsb"],
        a["stream"]) == code


# ------------------------------------------------------------------------------- backward
def _bwd_base(T, K, N):
    # codes [T x K], gamma [T], cT [K x N] fp16, dyT [N x T64] fp16, qT [K x T64] fp16,
    # dxh [T x K] fp32, 1/r [T], norm-weight partials [64 x K], each rounded up to 256 bytes
    up = lambda v: (v + 255) // 256 * 256
    t64 = (T + 63) // 64 * 64
    return (up(T * K) + up(4 * T) + up(2 * K * N) + up(2 * N * t64) + up(2 * K * t64) +
            up(4 * T * K) + up(4 * T) + up(4 * 64 * K))


def test_backward_workspace_sizes():
    L = mmf.lib()
    # no split: one partial-free contraction each
    assert L.mmf_backward_workspace_bytes(17, 256, 384) == _bwd_base(17, 256, 384)
    assert L.mmf_backward_workspace_bytes(32768, 2048, 2048) == _bwd_base(32768, 2048, 2048)
    # 2000 tokens, 16 output tiles of dW: its token contraction is split three ways
    # (3 partial [1024 x 1024] fp32 tiles)
    assert L.mmf_backward_workspace_bytes(2000, 1024, 1024) == \
        _bwd_base(2000, 1024, 1024) + 3 * 1024 * 1024 * 4
    # 300 tokens, 8 output tiles of dxh: its contraction over N = 2048 is split four ways
    # (4 partial [512 x 1024] tiles, 512 = 300 rounded up to the 256-token tile)
    assert L.mmf_backward_workspace_bytes(300, 1024, 2048) == \
        _bwd_base(300, 1024, 2048) + 4 * 512 * 1024 * 4
    assert L.mmf_backward_workspace_bytes(0, 256, 256) == 0
    assert L.mmf_backward_workspace_bytes(4, 200, 256) == 0
    assert L.mmf_backward_workspace_bytes(4, 256, 200) == 0


def bwd(**kw):
    a = dict(x=A16, xdt=1, T=4, K=256, g=None, eps=1e-8, A=None, gamma=None, Wp=A16, beta=A16,
             N=256, dy=A16, dx=A16, dxdt=0, dW=A16, dg=None, ws=A16, wsb=1 << 24, stream=None)
    a.update(kw)
    return mmf.lib().mmf_bitlinear_backward(
        a["x"], a["xdt"], a["T"], a["K"], a["g"], a["eps"], a["A"], a["gamma"], a["Wp"],
        a["beta"], a["N"], a["dy"], a["dx"], a["dxdt"], a["dW"], a["dg"], a["ws"], a["wsb"],
        a["stream"])


@pytest.mark.parametrize("kw,code", [
    (dict(x=None), INVALID), (dict(Wp=None), INVALID), (dict(beta=None), INVALID),
    (dict(dy=None), INVALID), (dict(dx=None, dW=None, dg=None), INVALID),
    (dict(A=A16), INVALID), (dict(gamma=A16), INVALID), (dict(xdt=2), INVALID),
    (dict(dxdt=7), INVALID), (dict(eps=0.0), INVALID), (dict(eps=float("nan")), INVALID),
    (dict(T=0), SHAPE), (dict(K=192), SHAPE), (dict(N=64), SHAPE), (dict(K=8320), SHAPE),
    (dict(x=A16 + 8), ALIGN), (dict(dy=A16 + 2), ALIGN), (dict(dx=A16 + 4), ALIGN),
    (dict(dW=A16 + 8), ALIGN), (dict(dg=A16 + 4), ALIGN), (dict(A=A16 + 1, gamma=A16), ALIGN),
    (dict(g=A16 + 4), ALIGN), (dict(ws=A16 + 16), ALIGN),
    (dict(ws=None), WS), (dict(wsb=1000), WS),
])
def test_backward_rejects_on_host(kw, code):
    assert bwd(**kw) == code


def test_backward_valid_call_without_gpu_reports_cuda_error():
    import torch
    if torch.cuda.is_available():
        pytest.skip("a GPU is present")
    assert bwd() == CUDA
