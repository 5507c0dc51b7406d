"""Oracle for the FusedBitLinear projection: ctypes wrapper over the scalar C code.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline
leg of ``bench.py`` may import this package.  It shares no code with the CUDA path in
``ternary_weight_lm_b200``; the two meet only through the seeded inputs of ``synth``.

Each function states the page passage it follows in ``mmf_oracle.c``.  All arrays are numpy;
fp16 inputs are widened to fp32 exactly before the C code sees them.  Every function here is
pinned by ``tests/test_oracle_pins.py`` (no function is "parity unpinned").
"""
import ctypes
import numpy as np

from . import build as _build

_lib = None


def _L():
    global _lib
    if _lib is None:
        path = _build.build()
        lib = ctypes.CDLL(path)
        P = ctypes.c_void_p
        I64 = ctypes.c_int64
        F = ctypes.c_float
        lib.orc_dense_matmul_i64.argtypes = [P, P, I64, I64, I64, P]
        lib.orc_rmsnorm_actquant.argtypes = [P, I64, I64, P, F, P, P, P]
        lib.orc_abs_sum_exact.argtypes = [P, I64]
        lib.orc_abs_sum_exact.restype = ctypes.c_double
        lib.orc_absmean_beta.argtypes = [P, I64]
        lib.orc_absmean_beta.restype = F
        lib.orc_ternary_codes.argtypes = [P, I64, F, P]
        lib.orc_pack_codes.argtypes = [P, I64, I64, P]
        lib.orc_unpack_codes.argtypes = [P, I64, I64, P]
        lib.orc_ternary_accumulate.argtypes = [P, I64, I64, P, I64, P]
        lib.orc_dequant.argtypes = [P, I64, I64, P, F, P]
        lib.orc_silu_glu.argtypes = [P, I64, I64, P]
        lib.orc_bitlinear_forward.argtypes = [P, I64, I64, P, F, P, I64, ctypes.c_int, P]
        lib.orc_bitlinear_forward.restype = F
        D = ctypes.c_double
        lib.orc_mlgru_scan.argtypes = [P, P, I64, I64, P, P, P]
        lib.orc_swish_gate_norm.argtypes = [P, P, I64, I64, P, D, P]
        lib.orc_bitlinear_backward.argtypes = [P, I64, I64, P, D, P, P, P, F, I64, P, P, P, P]
        _lib = lib
    return _lib


def _p(a):
    return a.ctypes.data_as(ctypes.c_void_p)


def _f32(a):
    return np.ascontiguousarray(np.asarray(a), dtype=np.float32)


def dense_matmul_i64(A, B):
    """C = A @ B over int64, the textbook definition (integer worked example)."""
    A = np.ascontiguousarray(A, dtype=np.int64)
    B = np.ascontiguousarray(B, dtype=np.int64)
    m, k = A.shape
    k2, n = B.shape
    assert k == k2
    C = np.empty((m, n), dtype=np.int64)
    _L().orc_dense_matmul_i64(_p(A), _p(B), m, k, n, _p(C))
    return C


def rmsnorm_actquant(x, g=None, eps=1e-8):
    """RMSNorm (eps inside the root) then per-token absmax int8 codes.

    Returns ``(q int8 [T,K], gamma f32 [T], rowsum int32 [T])``.
    """
    x = _f32(x)
    T, K = x.shape
    gg = None if g is None else _f32(g)
    q = np.empty((T, K), dtype=np.int8)
    gamma = np.empty(T, dtype=np.float32)
    rs = np.empty(T, dtype=np.int32)
    _L().orc_rmsnorm_actquant(_p(x), T, K, None if gg is None else _p(gg), eps, _p(q),
                              _p(gamma), _p(rs))
    return q, gamma, rs


def abs_sum_exact(W):
    """Exact sum of |W| rounded once to double (NaN if W holds a non-finite value)."""
    W = _f32(W).reshape(-1)
    return float(_L().orc_abs_sum_exact(_p(W), W.size))


def absmean_beta(W):
    """beta = float(double(exact sum |W|) / count), floored at 1e-5."""
    W = _f32(W).reshape(-1)
    return np.float32(_L().orc_absmean_beta(_p(W), W.size))


def ternary_codes(W, beta):
    """c = clamp(round_half_even(W / beta), -1, 1), division in float."""
    W = _f32(W)
    c = np.empty(W.shape, dtype=np.int8)
    _L().orc_ternary_codes(_p(W), W.size, float(np.float32(beta)), _p(c))
    return c


def pack_codes(c):
    """Pack int8 codes [N,K] in {-1,0,1} into the library's 2-bit layout, uint8 [N, K/4]."""
    c = np.ascontiguousarray(c, dtype=np.int8)
    N, K = c.shape
    assert K % 16 == 0
    Wp = np.empty((N, K // 4), dtype=np.uint8)
    _L().orc_pack_codes(_p(c), N, K, _p(Wp))
    return Wp


def unpack_codes(Wp, K):
    Wp = np.ascontiguousarray(Wp, dtype=np.uint8)
    N = Wp.shape[0]
    c = np.empty((N, K), dtype=np.int8)
    _L().orc_unpack_codes(_p(Wp), N, K, _p(c))
    return c


def ternary_accumulate(q, c):
    """acc[t,n] = sum_{c=+1} q - sum_{c=-1} q, int32 [T,N]."""
    q = np.ascontiguousarray(q, dtype=np.int8)
    c = np.ascontiguousarray(c, dtype=np.int8)
    T, K = q.shape
    N, K2 = c.shape
    assert K == K2
    acc = np.empty((T, N), dtype=np.int32)
    _L().orc_ternary_accumulate(_p(q), T, K, _p(c), N, _p(acc))
    return acc


def dequant(acc, gamma, beta):
    acc = np.ascontiguousarray(acc, dtype=np.int32)
    gamma = _f32(gamma)
    T, N = acc.shape
    y = np.empty((T, N), dtype=np.float64)
    _L().orc_dequant(_p(acc), T, N, _p(gamma), float(np.float32(beta)), _p(y))
    return y


def silu_glu(y):
    """h = silu(y[:, :I]) * y[:, I:], double."""
    y = np.ascontiguousarray(y, dtype=np.float64)
    T, N2 = y.shape
    assert N2 % 2 == 0
    h = np.empty((T, N2 // 2), dtype=np.float64)
    _L().orc_silu_glu(_p(y), T, N2 // 2, _p(h))
    return h


def quantize_weights(W):
    """Return ``(Wp uint8 [N, K/4], beta f32, codes int8 [N,K])``."""
    beta = absmean_beta(W)
    c = ternary_codes(W, beta)
    return pack_codes(c), beta, c


def bitlinear_forward(x, W, g=None, eps=1e-8, glu=False):
    """Whole projection in double: returns ``(out float64 [T, N or N/2], beta)``."""
    x = _f32(x)
    W = _f32(W)
    T, K = x.shape
    N, K2 = W.shape
    assert K == K2
    gg = None if g is None else _f32(g)
    out = np.empty((T, N // 2 if glu else N), dtype=np.float64)
    beta = _L().orc_bitlinear_forward(_p(x), T, K, None if gg is None else _p(gg), eps, _p(W),
                                      N, 1 if glu else 0, _p(out))
    return out, np.float32(beta)


def _f64(a):
    return np.ascontiguousarray(np.asarray(a), dtype=np.float64)


def mlgru_scan(I, F, h0=None):
    """MLGRU recurrence h_t = sigmoid(F_t) h_{t-1} + (1 - sigmoid(F_t)) silu(I_t), in double.

    ``I``, ``F``: [T, H]; ``h0``: [H] or None (zero).  Returns ``(h [T, H], hT [H])``.
    """
    I = _f64(I)
    F = _f64(F)
    T, H = I.shape
    assert F.shape == (T, H)
    hh = None if h0 is None else _f64(h0)
    h = np.empty((T, H), dtype=np.float64)
    hT = np.empty(H, dtype=np.float64)
    _L().orc_mlgru_scan(_p(I), _p(F), T, H, None if hh is None else _p(hh), _p(h), _p(hT))
    return h, hT


def swish_gate_norm(h, G, w=None, eps=1e-8):
    """FusedRMSNormSwishGate: h / sqrt(mean(h^2) + eps) * w * silu(G) per token, in double."""
    h = _f64(h)
    G = _f64(G)
    T, H = h.shape
    assert G.shape == (T, H)
    ww = None if w is None else _f64(w)
    o = np.empty((T, H), dtype=np.float64)
    _L().orc_swish_gate_norm(_p(h), _p(G), T, H, None if ww is None else _p(ww), float(eps), _p(o))
    return o


def mlgru_forward(I, F, G, h0=None, w=None, eps=1e-8):
    """Recurrence then the swish gate norm.  Returns ``(o [T, H] double, hT [H] double)``."""
    h, hT = mlgru_scan(I, F, h0)
    return swish_gate_norm(h, G, w, eps), hT


def bitlinear_backward(x, q, gamma, c, beta, dy, g=None, eps=1e-8, want_dg=True):
    """Straight-through backward of the projection, in double.

    ``x`` [T, K] (the forward input), ``q`` [T, K] int8 and ``gamma`` [T] (the forward's
    activation codes and scales), ``c`` [N, K] int8 and ``beta`` (the weight codes and scale),
    ``dy`` [T, N].  Returns ``(dx [T, K], dW [N, K], dg [K] or None)``.
    """
    x = _f64(x)
    dy = _f64(dy)
    T, K = x.shape
    N = dy.shape[1]
    assert dy.shape[0] == T
    q = np.ascontiguousarray(q, dtype=np.int8)
    c = np.ascontiguousarray(c, dtype=np.int8)
    assert q.shape == (T, K) and c.shape == (N, K)
    gamma = _f32(gamma)
    gg = None if g is None else _f64(g)
    dx = np.empty((T, K), dtype=np.float64)
    dW = np.empty((N, K), dtype=np.float64)
    dg = np.empty(K, dtype=np.float64) if want_dg else None
    _L().orc_bitlinear_backward(_p(x), T, K, None if gg is None else _p(gg), float(eps), _p(q),
                                _p(gamma), _p(c), float(np.float32(beta)), N, _p(dy), _p(dx),
                                _p(dW), None if dg is None else _p(dg))
    return dx, dW, dg
