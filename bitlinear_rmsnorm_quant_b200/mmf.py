"""ctypes binding of libmmf.so (the C ABI in include/mmf.h).

Argument marshalling only: every step of the layer runs in the library's CUDA
kernels.  PyTorch supplies device memory and streams.  If the library has not
been built this module raises on first use; there is no fallback path.

Raw entry points (``lib()``) take integer device pointers; the tensor helpers
below check dtypes/devices, allocate outputs with torch when none are given,
and pass the current torch stream.
"""
from __future__ import annotations

import ctypes as C
import os
import threading

import torch

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libmmf.so")

MMF_OK = 0
STATUS = {
    0: "MMF_OK", 1: "MMF_ERR_INVALID_ARG", 2: "MMF_ERR_UNSUPPORTED_SHAPE", 3: "MMF_ERR_MISALIGNED",
    4: "MMF_ERR_WORKSPACE", 5: "MMF_ERR_CUDA", 6: "MMF_ERR_TIMEOUT", 7: "MMF_ERR_NO_DEVICE",
}

_lock = threading.Lock()
_lib = None

_P, _I64, _F, _SZ, _INT = C.c_void_p, C.c_int64, C.c_float, C.c_size_t, C.c_int

# name -> (restype, argtypes); mirrors include/mmf.h
SIGNATURES = {
    "mmf_status_string": (C.c_char_p, [_INT]),
    "mmf_version": (C.c_char_p, []),
    "mmf_packed_bytes": (_SZ, [_I64, _I64]),
    "mmf_workspace_bytes": (_SZ, [_I64, _I64, _I64]),
    "mmf_fwd_launches": (_INT, [_I64, _I64, _I64, _INT]),
    "mmf_pack_ternary": (_INT, [_P, _I64, _I64, _F, _P, _P, _P]),
    "mmf_quantize_act": (_INT, [_P, _P, _F, _I64, _I64, _P, _P, _P]),
    "mmf_ternary_acc": (_INT, [_P, _P, _I64, _I64, _I64, _P, _P, _SZ, _P]),
    "mmf_bitlinear_fwd": (_INT, [_P, _P, _F, _P, _P, _I64, _I64, _I64, _P, _P, _SZ, _P]),
    "mmf_bitlinear_fwd_glu": (_INT, [_P, _P, _P, _F, _P, _P, _I64, _I64, _I64, _P, _P, _SZ, C.c_uint, _P]),
    "mmf_mlgru_scan": (_INT, [_P, _P, _P, _P, _I64, _I64, _I64, _P, _P, _P]),
    "mmf_bwd_workspace_bytes": (_SZ, [_I64, _I64, _I64]),
    "mmf_bitlinear_bwd": (_INT, [_P, _P, _P, _F, _P, _P, _I64, _I64, _I64, _P, _P, _P, _P, _SZ, _P]),
    "mmf_bitlinear_fwd_group": (_INT, [_P, _P, _F, _I64, _I64, _P, _INT, _P, _SZ, C.c_uint, _P]),
    "mmf_bitlinear_fwd_noalloc": (_INT, [_P, _P, _F, _P, _P, _I64, _I64, _I64, _P, _P]),
    "mmf_hbm_copy": (_INT, [_P, _P, _SZ, _P]),
    "mmf_selftest_timeout": (_INT, [C.c_uint64, _P, _P]),
    "mmf_check_async": (_INT, [_P]),
}


FWD_PDL = 1
NOALLOC_SCRATCH_BYTES = 64 << 20   # MMF_NOALLOC_SCRATCH_BYTES
MAX_GROUP = 8


class Projection(C.Structure):
    """mirror of mmf_projection"""
    _fields_ = [("packed", _P), ("scale", _P), ("y", _P), ("N", _I64)]


class MMFError(RuntimeError):
    def __init__(self, what: str, status: int):
        super().__init__(f"{what}: {STATUS.get(status, status)}")
        self.status = status


def lib() -> C.CDLL:
    """Loads libmmf.so (once); raises if it is missing."""
    global _lib
    with _lock:
        if _lib is None:
            if not os.path.exists(LIB_PATH):
                raise RuntimeError(
                    f"{LIB_PATH} is missing: build it with `python -m bitlinear_rmsnorm_quant_b200.build`")
            L = C.CDLL(LIB_PATH)
            for name, (res, args) in SIGNATURES.items():
                f = getattr(L, name)
                f.restype = res
                f.argtypes = args
            _lib = L
    return _lib


def check(status: int, what: str) -> None:
    if status != MMF_OK:
        raise MMFError(what, status)


def _stream(stream) -> int:
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, torch.cuda.Stream):
        return stream.cuda_stream
    return int(stream)


def _dev(t: torch.Tensor, dtype, name: str):
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")


# -- sizes ----------------------------------------------------------------------

def packed_bytes(N: int, K: int) -> int:
    return int(lib().mmf_packed_bytes(N, K))


def workspace_bytes(M: int, K: int, N: int) -> int:
    return int(lib().mmf_workspace_bytes(M, K, N))


def fwd_launches(M: int, K: int, N: int, count: int = 1) -> int:
    return int(lib().mmf_fwd_launches(M, K, N, count))


def version() -> str:
    return lib().mmf_version().decode()


# -- entry points ---------------------------------------------------------------

def pack_ternary(W: torch.Tensor, eps_w: float = 1e-5, packed: torch.Tensor | None = None,
                 scale: torch.Tensor | None = None, stream=None):
    """fp32 W[N, K] -> (packed int32[N, K/16] holding uint32 words, scale fp32[1])."""
    _dev(W, torch.float32, "W")
    N, K = W.shape
    if packed is None:
        packed = torch.empty((N, K // 16), dtype=torch.int32, device=W.device)
    if scale is None:
        scale = torch.empty(4, dtype=torch.float32, device=W.device)[:1]
    check(lib().mmf_pack_ternary(W.data_ptr(), N, K, eps_w, packed.data_ptr(), scale.data_ptr(), _stream(stream)),
          "mmf_pack_ternary")
    return packed, scale


def quantize_act(x: torch.Tensor, gamma: torch.Tensor, eps: float = 1e-6, stream=None):
    """bf16 x[M, K] -> (q int8[M, K], absmax fp32[M])."""
    _dev(x, torch.bfloat16, "x")
    _dev(gamma, torch.float32, "gamma")
    M, K = x.shape
    q = torch.empty((M, K), dtype=torch.int8, device=x.device)
    a = torch.empty(max(M, 4), dtype=torch.float32, device=x.device)[:M]
    check(lib().mmf_quantize_act(x.data_ptr(), gamma.data_ptr(), eps, M, K, q.data_ptr(), a.data_ptr(),
                                 _stream(stream)), "mmf_quantize_act")
    return q, a


def _workspace(M, K, N, device, workspace):
    need = workspace_bytes(M, K, N)
    if need == 0:
        return None, 0
    if workspace is None:
        workspace = torch.empty(need, dtype=torch.uint8, device=device)
    if workspace.numel() < need:
        raise ValueError(f"workspace needs {need} bytes")
    return workspace, workspace.numel()


def ternary_acc(q: torch.Tensor, packed: torch.Tensor, N: int, workspace=None, out=None, stream=None):
    """int8 q[M, K] x packed[N, K/16] -> int32 acc[M, N]."""
    _dev(q, torch.int8, "q")
    M, K = q.shape
    acc = out if out is not None else torch.empty((M, N), dtype=torch.int32, device=q.device)
    ws, ws_n = _workspace(M, K, N, q.device, workspace)
    check(lib().mmf_ternary_acc(q.data_ptr(), packed.data_ptr(), M, K, N, acc.data_ptr(),
                                ws.data_ptr() if ws is not None else None, ws_n, _stream(stream)),
          "mmf_ternary_acc")
    return acc


def bitlinear_fwd(x: torch.Tensor, gamma: torch.Tensor, packed: torch.Tensor, scale: torch.Tensor, N: int,
                  eps: float = 1e-6, workspace=None, out=None, stream=None):
    """bf16 x[M, K] -> bf16 y[M, N]."""
    _dev(x, torch.bfloat16, "x")
    M, K = x.shape
    y = out if out is not None else torch.empty((M, N), dtype=torch.bfloat16, device=x.device)
    ws, ws_n = _workspace(M, K, N, x.device, workspace)
    check(lib().mmf_bitlinear_fwd(x.data_ptr(), gamma.data_ptr(), eps, packed.data_ptr(), scale.data_ptr(), M, K, N,
                                  y.data_ptr(), ws.data_ptr() if ws is not None else None, ws_n, _stream(stream)),
          "mmf_bitlinear_fwd")
    return y


def projection_array(items):
    """[(packed, scale, y, N), ...] -> ctypes array of mmf_projection (keep it alive while used)."""
    arr = (Projection * len(items))()
    for i, (packed, scale, y, N) in enumerate(items):
        arr[i] = Projection(packed.data_ptr(), scale.data_ptr(), y.data_ptr() if y is not None else None, N)
    return arr


def bitlinear_fwd_glu(g: torch.Tensor, u: torch.Tensor, gamma: torch.Tensor, packed: torch.Tensor,
                      scale: torch.Tensor, N: int, eps: float = 1e-6, workspace=None, out=None, flags: int = 0,
                      stream=None):
    """GLU down projection: bf16 g[M, K], u[M, K] -> bf16 y[M, N] of BitLinear(bf16(SiLU(g) * u))."""
    _dev(g, torch.bfloat16, "g")
    _dev(u, torch.bfloat16, "u")
    M, K = g.shape
    assert u.shape == g.shape
    y = out if out is not None else torch.empty((M, N), dtype=torch.bfloat16, device=g.device)
    ws, ws_n = _workspace(M, K, N, g.device, workspace)
    check(lib().mmf_bitlinear_fwd_glu(g.data_ptr(), u.data_ptr(), gamma.data_ptr(), eps, packed.data_ptr(),
                                      scale.data_ptr(), M, K, N, y.data_ptr(),
                                      ws.data_ptr() if ws is not None else None, ws_n, flags, _stream(stream)),
          "mmf_bitlinear_fwd_glu")
    return y


def mlgru_scan(f_pre: torch.Tensor, c_pre: torch.Tensor, g_pre: torch.Tensor, h0: torch.Tensor | None = None,
               out=None, h_last=None, stream=None):
    """MLGRU recurrence: bf16 [B, T, D] pre-activations -> (bf16 o [B, T, D], fp32 h_last [B, D])."""
    for name, t in (("f_pre", f_pre), ("c_pre", c_pre), ("g_pre", g_pre)):
        _dev(t, torch.bfloat16, name)
    B, T, D = f_pre.shape
    o = out if out is not None else torch.empty((B, T, D), dtype=torch.bfloat16, device=f_pre.device)
    hl = h_last if h_last is not None else torch.empty((B, D), dtype=torch.float32, device=f_pre.device)
    check(lib().mmf_mlgru_scan(f_pre.data_ptr(), c_pre.data_ptr(), g_pre.data_ptr(),
                               h0.data_ptr() if h0 is not None else None, B, T, D, o.data_ptr(), hl.data_ptr(),
                               _stream(stream)), "mmf_mlgru_scan")
    return o, hl


def bitlinear_bwd(dy: torch.Tensor, x: torch.Tensor, gamma: torch.Tensor, packed: torch.Tensor,
                  scale: torch.Tensor, eps: float = 1e-6, stream=None):
    """Straight-through backward: bf16 dy[M, N], x[M, K] -> (bf16 dx[M, K], fp32 dgamma[K], fp32 dW[N, K])."""
    _dev(dy, torch.bfloat16, "dy")
    _dev(x, torch.bfloat16, "x")
    M, K = x.shape
    N = dy.shape[1]
    dx = torch.empty((M, K), dtype=torch.bfloat16, device=x.device)
    dg = torch.empty(K, dtype=torch.float32, device=x.device)
    dW = torch.empty((N, K), dtype=torch.float32, device=x.device)
    n = int(lib().mmf_bwd_workspace_bytes(M, K, N))
    ws = torch.empty(max(n, 256), dtype=torch.uint8, device=x.device)
    check(lib().mmf_bitlinear_bwd(dy.data_ptr(), x.data_ptr(), gamma.data_ptr(), eps, packed.data_ptr(),
                                  scale.data_ptr(), M, K, N, dx.data_ptr(), dg.data_ptr(), dW.data_ptr(),
                                  ws.data_ptr(), ws.numel(), _stream(stream)), "mmf_bitlinear_bwd")
    return dx, dg, dW


def bitlinear_fwd_group(x: torch.Tensor, gamma: torch.Tensor, weights, eps: float = 1e-6, workspace=None,
                        outs=None, flags: int = 0, stream=None):
    """bf16 x[M, K] and [(packed, scale, N), ...] sharing x -> [bf16 y_i[M, N_i], ...]."""
    _dev(x, torch.bfloat16, "x")
    M, K = x.shape
    ys = outs if outs is not None else [torch.empty((M, N), dtype=torch.bfloat16, device=x.device)
                                        for (_, _, N) in weights]
    arr = projection_array([(pk, sc, y, N) for (pk, sc, N), y in zip(weights, ys)])
    ws, ws_n = _workspace(M, K, sum(N for _, _, N in weights), x.device, workspace)
    check(lib().mmf_bitlinear_fwd_group(x.data_ptr(), gamma.data_ptr(), eps, M, K, arr, len(weights),
                                        ws.data_ptr() if ws is not None else None, ws_n, flags, _stream(stream)),
          "mmf_bitlinear_fwd_group")
    return ys


def bitlinear_fwd_noalloc(x: torch.Tensor, gamma: torch.Tensor, packed: torch.Tensor, scale: torch.Tensor, N: int,
                          eps: float = 1e-6, out: torch.Tensor | None = None, stream=None):
    """As bitlinear_fwd, but the library's static scratch replaces the workspace
    (for callers that cannot allocate device memory; pass `out` to allocate
    nothing here either)."""
    _dev(x, torch.bfloat16, "x")
    M, K = x.shape
    y = out if out is not None else torch.empty((M, N), dtype=torch.bfloat16, device=x.device)
    check(lib().mmf_bitlinear_fwd_noalloc(x.data_ptr(), gamma.data_ptr(), eps, packed.data_ptr(), scale.data_ptr(),
                                          M, K, N, y.data_ptr(), _stream(stream)), "mmf_bitlinear_fwd_noalloc")
    return y


def hbm_copy(src: torch.Tensor, dst: torch.Tensor, stream=None):
    nbytes = src.numel() * src.element_size()
    check(lib().mmf_hbm_copy(src.data_ptr(), dst.data_ptr(), nbytes, _stream(stream)), "mmf_hbm_copy")


def selftest_timeout(limit_ns: int, waited_out: torch.Tensor | None = None, stream=None):
    check(lib().mmf_selftest_timeout(limit_ns, waited_out.data_ptr() if waited_out is not None else None,
                                     _stream(stream)), "mmf_selftest_timeout")


def check_async(stream=None):
    check(lib().mmf_check_async(_stream(stream)), "mmf_check_async")
