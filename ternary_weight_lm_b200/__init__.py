"""Python binding of libmmf.so, the B200 FusedBitLinear library.

Argument marshalling only: every step of the projection runs in the library's CUDA kernels.
PyTorch supplies device memory (``tensor.data_ptr()``) and streams
(``torch.cuda.current_stream().cuda_stream``).  There is no CPU path: if the library or a GPU
is missing, calls raise.

The functions named ``mmf_*`` mirror the C ABI in ``include/mmf.h`` one to one and take
tensors that the caller owns.  ``quantize_weights``, ``bitlinear_forward``,
``bitlinear_glu_forward``, ``mlgru_forward`` and ``bitlinear_backward`` are conveniences that
allocate the outputs and the workspace with torch and then call the same entry points.
"""
import ctypes
import os

__all__ = [
    "MMFError", "lib", "lib_path",
    "mmf_quantize_weights_workspace_bytes", "mmf_quantize_weights", "mmf_ternary_encode",
    "mmf_forward_workspace_bytes", "mmf_bitlinear_forward", "mmf_bitlinear_glu_forward",
    "mmf_quantize_activations", "mmf_quantized_workspace_bytes",
    "mmf_bitlinear_forward_quantized",
    "mmf_ternary_accumulate_i32", "mmf_bitlinear_forward_noalloc", "mmf_get_device_status",
    "mmf_debug_wait_timeout_probe", "mmf_status_string", "mmf_version",
    "mmf_program_workspace_bytes", "mmf_program_init", "mmf_program_run", "Projection",
    "Program", "quantize_weights", "bitlinear_forward", "bitlinear_glu_forward", "workspace",
    "mmf_mlgru_workspace_bytes", "mmf_mlgru_forward", "mmf_mlgru_forward_quantized",
    "mlgru_forward", "mmf_backward_workspace_bytes", "mmf_bitlinear_backward",
    "bitlinear_backward",
    "MMF_F32", "MMF_F16", "STATUS",
]

_HERE = os.path.dirname(os.path.abspath(__file__))
lib_path = os.path.join(_HERE, "libmmf.so")

MMF_F32 = 0
MMF_F16 = 1
STATUS = {
    0: "MMF_OK", 1: "MMF_ERR_INVALID_ARG", 2: "MMF_ERR_UNSUPPORTED_SHAPE",
    3: "MMF_ERR_ALIGNMENT", 4: "MMF_ERR_CUDA", 5: "MMF_ERR_TIMEOUT", 6: "MMF_ERR_WORKSPACE",
    7: "MMF_ERR_RESOURCES", 8: "MMF_ERR_PLAN",
}


class MMFError(RuntimeError):
    def __init__(self, fn, code):
        super().__init__(f"{fn} failed: {STATUS.get(code, code)}")
        self.code = code


class Projection(ctypes.Structure):
    """Mirror of the C struct mmf_projection (one FusedBitLinear of a program)."""
    _fields_ = [("x", ctypes.c_void_p), ("xdt", ctypes.c_int), ("norm_w", ctypes.c_void_p),
                ("Wp", ctypes.c_void_p), ("beta", ctypes.c_void_p), ("K", ctypes.c_int64),
                ("N", ctypes.c_int64), ("glu", ctypes.c_int32), ("level", ctypes.c_int32),
                ("y", ctypes.c_void_p), ("ydt", ctypes.c_int)]


_lib = None


def lib():
    """Load libmmf.so (raises OSError if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(lib_path):
            raise OSError(f"{lib_path} is missing: run ternary_weight_lm_b200/build.py")
        L = ctypes.CDLL(lib_path)
        P, I64, F, SZ, I = (ctypes.c_void_p, ctypes.c_int64, ctypes.c_float, ctypes.c_size_t,
                            ctypes.c_int)
        sigs = {
            "mmf_quantize_weights_workspace_bytes": ([I64, I64], SZ),
            "mmf_quantize_weights": ([P, I, I64, I64, P, P, P, SZ, P], I),
            "mmf_ternary_encode": ([P, I, I64, I64, P, P, P], I),
            "mmf_forward_workspace_bytes": ([I64, I64, I64], SZ),
            "mmf_bitlinear_forward": ([P, I, I64, I64, P, F, P, P, I64, P, I, P, SZ, P], I),
            "mmf_bitlinear_glu_forward": ([P, I, I64, I64, P, F, P, P, I64, P, I, P, SZ, P], I),
            "mmf_quantize_activations": ([P, I, I64, I64, P, F, P, P, P, P], I),
            "mmf_quantized_workspace_bytes": ([I64, I64, I64], SZ),
            "mmf_bitlinear_forward_quantized": ([P, P, P, I64, I64, P, P, I64, I, P, I, P, SZ, P],
                                                I),
            "mmf_ternary_accumulate_i32": ([P, I64, I64, P, I64, P, P, SZ, P], I),
            "mmf_bitlinear_forward_noalloc": ([P, I, I64, I64, P, F, P, P, I64, P, I, P], I),
            "mmf_backward_workspace_bytes": ([I64, I64, I64], SZ),
            "mmf_bitlinear_backward": ([P, I, I64, I64, P, F, P, P, P, P, I64, P, P, I, P, P, P,
                                        SZ, P], I),
            "mmf_mlgru_workspace_bytes": ([I64, I64], SZ),
            "mmf_mlgru_forward": ([P, P, P, I, I64, I64, P, P, F, P, I, P, P, SZ, P], I),
            "mmf_mlgru_forward_quantized": ([P, P, P, I, I64, I64, P, P, F, P, F, P, P, P, P, P,
                                             SZ, P], I),
            "mmf_program_workspace_bytes": ([P, I, I64], SZ),
            "mmf_program_init": ([P, I, I64, F, P, SZ, P], I),
            "mmf_program_run": ([P, P], I),
            "mmf_get_device_status": ([], I),
            "mmf_debug_wait_timeout_probe": ([ctypes.c_uint64, P], I),
            "mmf_status_string": ([I], ctypes.c_char_p),
            "mmf_version": ([], I),
        }
        for name, (args, res) in sigs.items():
            f = getattr(L, name)
            f.argtypes = args
            f.restype = res
        _lib = L
    return _lib


# ------------------------------------------------------------------------------ marshalling
def _ptr(t):
    if t is None:
        return None
    if isinstance(t, int):
        return t
    return t.data_ptr()


def _dt(t):
    import torch
    if t.dtype == torch.float32:
        return MMF_F32
    if t.dtype == torch.float16:
        return MMF_F16
    raise TypeError(f"unsupported dtype {t.dtype}")


def _stream(stream):
    if stream is None:
        import torch
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def _check(fn, code):
    if code != 0:
        raise MMFError(fn, code)


def _nbytes(t):
    return t.numel() * t.element_size()


# ------------------------------------------------------------------------------ C ABI mirror
def mmf_quantize_weights_workspace_bytes(N, K):
    return lib().mmf_quantize_weights_workspace_bytes(N, K)


def mmf_quantize_weights(W, Wp, beta, ws, stream=None):
    N, K = W.shape
    _check("mmf_quantize_weights", lib().mmf_quantize_weights(
        _ptr(W), _dt(W), N, K, _ptr(Wp), _ptr(beta), _ptr(ws), _nbytes(ws), _stream(stream)))


def mmf_ternary_encode(W, beta, Wp, stream=None):
    N, K = W.shape
    _check("mmf_ternary_encode", lib().mmf_ternary_encode(
        _ptr(W), _dt(W), N, K, _ptr(beta), _ptr(Wp), _stream(stream)))


def mmf_forward_workspace_bytes(T, K, N):
    return lib().mmf_forward_workspace_bytes(T, K, N)


def mmf_bitlinear_forward(x, norm_w, eps, Wp, beta, N, y, ws, stream=None):
    T, K = x.shape
    _check("mmf_bitlinear_forward", lib().mmf_bitlinear_forward(
        _ptr(x), _dt(x), T, K, _ptr(norm_w), float(eps), _ptr(Wp), _ptr(beta), N, _ptr(y),
        _dt(y), _ptr(ws), _nbytes(ws), _stream(stream)))


def mmf_bitlinear_glu_forward(x, norm_w, eps, Wp, beta, N2, h, ws, stream=None):
    T, K = x.shape
    _check("mmf_bitlinear_glu_forward", lib().mmf_bitlinear_glu_forward(
        _ptr(x), _dt(x), T, K, _ptr(norm_w), float(eps), _ptr(Wp), _ptr(beta), N2, _ptr(h),
        _dt(h), _ptr(ws), _nbytes(ws), _stream(stream)))


def mmf_quantize_activations(x, norm_w, eps, A, gamma, rowsum=None, stream=None):
    T, K = x.shape
    _check("mmf_quantize_activations", lib().mmf_quantize_activations(
        _ptr(x), _dt(x), T, K, _ptr(norm_w), float(eps), _ptr(A), _ptr(gamma), _ptr(rowsum),
        _stream(stream)))


def mmf_quantized_workspace_bytes(T, K, N):
    return lib().mmf_quantized_workspace_bytes(T, K, N)


def mmf_bitlinear_forward_quantized(A, gamma, rowsum, Wp, beta, N, glu, y, ws=None,
                                    stream=None):
    """ws: None (the contraction that needs no workspace) or a tensor of at least
    mmf_quantized_workspace_bytes(T, K, N) bytes."""
    T, K = A.shape
    _check("mmf_bitlinear_forward_quantized", lib().mmf_bitlinear_forward_quantized(
        _ptr(A), _ptr(gamma), _ptr(rowsum), T, K, _ptr(Wp), _ptr(beta), N, 1 if glu else 0,
        _ptr(y), _dt(y), _ptr(ws), 0 if ws is None else _nbytes(ws), _stream(stream)))


def mmf_ternary_accumulate_i32(A, Wp, N, acc, ws, stream=None):
    T, K = A.shape
    _check("mmf_ternary_accumulate_i32", lib().mmf_ternary_accumulate_i32(
        _ptr(A), T, K, _ptr(Wp), N, _ptr(acc), _ptr(ws), _nbytes(ws), _stream(stream)))


def mmf_bitlinear_forward_noalloc(x, norm_w, eps, Wp, beta, N, y, stream=None):
    """Forward without a workspace argument: for callers that cannot allocate device memory.
    Scratch is a fixed 4 MiB device array shared by all calls (see include/mmf.h)."""
    T, K = x.shape
    _check("mmf_bitlinear_forward_noalloc", lib().mmf_bitlinear_forward_noalloc(
        _ptr(x), _dt(x), T, K, _ptr(norm_w), float(eps), _ptr(Wp), _ptr(beta), N, _ptr(y),
        _dt(y), _stream(stream)))


def mmf_backward_workspace_bytes(T, K, N):
    return lib().mmf_backward_workspace_bytes(T, K, N)


def mmf_bitlinear_backward(x, norm_w, eps, A, gamma, Wp, beta, N, dy, dx, dW, dnorm_w, ws,
                           stream=None):
    """Straight-through backward (include/mmf.h).  A/gamma: the forward's codes and scales or
    both None; dx, dW, dnorm_w: outputs or None (dx's dtype selects dxdt)."""
    T, K = x.shape
    _check("mmf_bitlinear_backward", lib().mmf_bitlinear_backward(
        _ptr(x), _dt(x), T, K, _ptr(norm_w), float(eps), _ptr(A), _ptr(gamma), _ptr(Wp),
        _ptr(beta), N, _ptr(dy), _ptr(dx), MMF_F32 if dx is None else _dt(dx), _ptr(dW),
        _ptr(dnorm_w), _ptr(ws), _nbytes(ws), _stream(stream)))


def mmf_mlgru_workspace_bytes(T, H):
    return lib().mmf_mlgru_workspace_bytes(T, H)


def _ws(ws):
    return (None, 0) if ws is None else (_ptr(ws), _nbytes(ws))


def mmf_mlgru_forward(I, F, G, h0, norm_w, eps, o, hT=None, ws=None, stream=None):
    """MLGRU recurrence + swish gate norm (include/mmf.h): o [T, H] from I, F, G [T, H]."""
    T, H = I.shape
    wp, wn = _ws(ws)
    _check("mmf_mlgru_forward", lib().mmf_mlgru_forward(
        _ptr(I), _ptr(F), _ptr(G), _dt(I), T, H, _ptr(h0), _ptr(norm_w), float(eps), _ptr(o),
        _dt(o), _ptr(hT), wp, wn, _stream(stream)))


def mmf_mlgru_forward_quantized(I, F, G, h0, norm_w, eps, oproj_norm_w, oproj_eps, A, gamma,
                                rowsum=None, hT=None, ws=None, stream=None):
    """The same, writing o_proj's int8 codes, gamma and code sums instead of o."""
    T, H = I.shape
    wp, wn = _ws(ws)
    _check("mmf_mlgru_forward_quantized", lib().mmf_mlgru_forward_quantized(
        _ptr(I), _ptr(F), _ptr(G), _dt(I), T, H, _ptr(h0), _ptr(norm_w), float(eps),
        _ptr(oproj_norm_w), float(oproj_eps), _ptr(A), _ptr(gamma), _ptr(rowsum), _ptr(hT), wp,
        wn, _stream(stream)))


def _proj_array(projs):
    arr = (Projection * len(projs))()
    for i, p in enumerate(projs):
        x, norm_w, Wp, beta, y, glu, level = (p["x"], p.get("norm_w"), p["Wp"], p["beta"], p["y"],
                                              p.get("glu", False), p.get("level", 0))
        arr[i] = Projection(_ptr(x), _dt(x), _ptr(norm_w), _ptr(Wp), _ptr(beta), x.shape[1],
                            Wp.shape[0], 1 if glu else 0, level, _ptr(y), _dt(y))
    return arr


def mmf_program_workspace_bytes(projs, T):
    arr = _proj_array(projs)
    return lib().mmf_program_workspace_bytes(arr, len(projs), T)


def mmf_program_init(projs, T, eps, ws, stream=None):
    arr = _proj_array(projs)
    _check("mmf_program_init", lib().mmf_program_init(arr, len(projs), T, float(eps), _ptr(ws),
                                                      _nbytes(ws), _stream(stream)))


def mmf_program_run(ws, stream=None):
    _check("mmf_program_run", lib().mmf_program_run(_ptr(ws), _stream(stream)))


class Program:
    """A planned list of projections run as one launch (see mmf_program_init).

    ``projs`` is a list of dicts with keys x, Wp, beta, y and optionally norm_w, glu, level;
    the tensors must stay alive and in place for as long as the program is run."""

    def __init__(self, projs, T, eps=1e-8, stream=None):
        n = mmf_program_workspace_bytes(projs, T)
        if n == 0:
            raise MMFError("mmf_program_workspace_bytes", 2)
        self.projs = list(projs)
        self.ws = workspace(n, projs[0]["x"].device)
        mmf_program_init(self.projs, T, eps, self.ws, stream)

    def run(self, stream=None):
        mmf_program_run(self.ws, stream)


def mmf_get_device_status():
    """Status code (int) of the device status word; reading clears it."""
    return lib().mmf_get_device_status()


def mmf_debug_wait_timeout_probe(limit_ns, stream=None):
    _check("mmf_debug_wait_timeout_probe",
           lib().mmf_debug_wait_timeout_probe(int(limit_ns), _stream(stream)))


def mmf_status_string(code):
    return lib().mmf_status_string(code).decode()


def mmf_version():
    return lib().mmf_version()


# ------------------------------------------------------------------------------ conveniences
def workspace(nbytes, device="cuda"):
    import torch
    return torch.empty(max(int(nbytes), 256), dtype=torch.uint8, device=device)


def quantize_weights(W, stream=None):
    """W [N,K] (fp32/fp16, CUDA) -> (Wp uint8 [N, K/4], beta float32 [1])."""
    import torch
    N, K = W.shape
    Wp = torch.empty((N, K // 4), dtype=torch.uint8, device=W.device)
    beta = torch.empty(1, dtype=torch.float32, device=W.device)
    ws = workspace(mmf_quantize_weights_workspace_bytes(N, K), W.device)
    mmf_quantize_weights(W, Wp, beta, ws, stream)
    return Wp, beta


def bitlinear_forward(x, Wp, beta, norm_w=None, eps=1e-8, out_dtype=None, ws=None,
                      stream=None):
    import torch
    T, K = x.shape
    N = Wp.shape[0]
    y = torch.empty((T, N), dtype=out_dtype or x.dtype, device=x.device)
    if ws is None:
        ws = workspace(mmf_forward_workspace_bytes(T, K, N), x.device)
    mmf_bitlinear_forward(x, norm_w, eps, Wp, beta, N, y, ws, stream)
    return y


def mlgru_forward(I, F, G, h0=None, norm_w=None, eps=1e-8, out_dtype=None, hT=None, ws=None,
                  stream=None):
    """o [T, H] of the MLGRU recurrence and swish gate norm; hT (optional [H] fp32) receives
    the state after the last token."""
    import torch
    T, H = I.shape
    o = torch.empty((T, H), dtype=out_dtype or I.dtype, device=I.device)
    need = mmf_mlgru_workspace_bytes(T, H)
    if ws is None and need > 0:
        ws = workspace(need, I.device)
    mmf_mlgru_forward(I, F, G, h0, norm_w, eps, o, hT, ws, stream)
    return o


def bitlinear_glu_forward(x, Wp, beta, norm_w=None, eps=1e-8, out_dtype=None, ws=None,
                          stream=None):
    import torch
    T, K = x.shape
    N2 = Wp.shape[0]
    h = torch.empty((T, N2 // 2), dtype=out_dtype or x.dtype, device=x.device)
    if ws is None:
        ws = workspace(mmf_forward_workspace_bytes(T, K, N2), x.device)
    mmf_bitlinear_glu_forward(x, norm_w, eps, Wp, beta, N2, h, ws, stream)
    return h


def bitlinear_backward(x, Wp, beta, dy, norm_w=None, eps=1e-8, A=None, gamma=None,
                       dx_dtype=None, want_dx=True, want_dW=True, want_dnorm_w=False, ws=None,
                       stream=None):
    """Straight-through backward of bitlinear_forward: returns ``(dx, dW, dnorm_w)`` (None for
    what was not asked).  dy: fp16 [T, N]; dW and dnorm_w are fp32."""
    import torch
    T, K = x.shape
    N = Wp.shape[0]
    dev = x.device
    dx = torch.empty((T, K), dtype=dx_dtype or x.dtype, device=dev) if want_dx else None
    dW = torch.empty((N, K), dtype=torch.float32, device=dev) if want_dW else None
    dg = torch.empty(K, dtype=torch.float32, device=dev) if want_dnorm_w else None
    if ws is None:
        ws = workspace(mmf_backward_workspace_bytes(T, K, N), dev)
    mmf_bitlinear_backward(x, norm_w, eps, A, gamma, Wp, beta, N, dy, dx, dW, dg, ws, stream)
    return dx, dW, dg
