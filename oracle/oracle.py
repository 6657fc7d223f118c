"""ctypes wrapper around the C oracle (test infrastructure only).

Arrays are numpy; bf16 tensors travel as uint16 bit patterns.  Each method is a
thin call into the C function of the same name in ``mmf_oracle.c``, which holds
all of the arithmetic and cites the passage it follows.
"""
from __future__ import annotations

import ctypes as C
import os

import numpy as np

from .build import LIB, build

_P = C.c_void_p
_I64 = C.c_int64
_F = C.c_float


def _ptr(a: np.ndarray) -> int:
    assert a.flags["C_CONTIGUOUS"]
    return a.ctypes.data


class Oracle:
    def __init__(self, path: str):
        self.path = path
        lib = C.CDLL(path)
        lib.orc_bf16_to_f32.argtypes = [C.c_uint16]
        lib.orc_bf16_to_f32.restype = C.c_float
        lib.orc_f64_to_bf16.argtypes = [C.c_double]
        lib.orc_f64_to_bf16.restype = C.c_uint16
        lib.orc_absmean_ternary.argtypes = [_P, _I64, _I64, _F, _P, _P]
        lib.orc_absmean_ternary.restype = None
        lib.orc_encode_packed.argtypes = [_P, _I64, _I64, _P]
        lib.orc_encode_packed.restype = None
        lib.orc_decode_packed.argtypes = [_P, _I64, _I64, _P]
        lib.orc_decode_packed.restype = C.c_int64
        lib.orc_rmsnorm_quant.argtypes = [_P, _P, _F, _I64, _I64, _P, _P]
        lib.orc_rmsnorm_quant.restype = None
        lib.orc_ternary_acc.argtypes = [_P, _P, _I64, _I64, _I64, _P]
        lib.orc_ternary_acc.restype = None
        lib.orc_rescale.argtypes = [_P, _P, _F, _I64, _I64, _P]
        lib.orc_rescale.restype = None
        lib.orc_bitlinear.argtypes = [_P, _P, _F, _P, _F, _I64, _I64, _I64, _P, _P]
        lib.orc_bitlinear.restype = C.c_int
        lib.orc_glu_gate.argtypes = [_P, _P, _I64, _P]
        lib.orc_glu_gate.restype = None
        lib.orc_mlgru_scan.argtypes = [_P, _P, _P, _P, _I64, _I64, _I64, _P, _P]
        lib.orc_mlgru_scan.restype = None
        lib.orc_bitlinear_bwd.argtypes = [_P, _P, _P, _F, _P, _F, _I64, _I64, _I64, _P, _P, _P]
        lib.orc_bitlinear_bwd.restype = C.c_int
        lib.orc_num_threads.argtypes = []
        lib.orc_num_threads.restype = C.c_int
        self.lib = lib

    # -- scalars ---------------------------------------------------------------
    def bf16_to_f32(self, b: int) -> float:
        return float(self.lib.orc_bf16_to_f32(int(b)))

    def f64_to_bf16(self, v: float) -> int:
        return int(self.lib.orc_f64_to_bf16(float(v)))

    def f64_to_bf16_array(self, v: np.ndarray) -> np.ndarray:
        flat = np.asarray(v, dtype=np.float64).ravel()
        out = np.empty(flat.shape, dtype=np.uint16)
        f = self.lib.orc_f64_to_bf16
        for i, e in enumerate(flat):
            out[i] = f(float(e))
        return out.reshape(np.shape(v))

    # -- steps -----------------------------------------------------------------
    def absmean_ternary(self, W: np.ndarray, eps_w: float):
        W = np.ascontiguousarray(W, dtype=np.float32)
        N, K = W.shape
        wt = np.empty((N, K), dtype=np.int8)
        beta = np.zeros(1, dtype=np.float32)
        self.lib.orc_absmean_ternary(_ptr(W), N, K, eps_w, _ptr(wt), _ptr(beta))
        return wt, np.float32(beta[0])

    def encode_packed(self, wt: np.ndarray) -> np.ndarray:
        wt = np.ascontiguousarray(wt, dtype=np.int8)
        N, K = wt.shape
        assert K % 16 == 0
        out = np.empty((N, K // 16), dtype=np.uint32)
        self.lib.orc_encode_packed(_ptr(wt), N, K, _ptr(out))
        return out

    def decode_packed(self, packed: np.ndarray, K: int):
        packed = np.ascontiguousarray(packed, dtype=np.uint32)
        N = packed.shape[0]
        wt = np.empty((N, K), dtype=np.int8)
        bad = self.lib.orc_decode_packed(_ptr(packed), N, K, _ptr(wt))
        return wt, int(bad)

    def rmsnorm_quant(self, x_bits: np.ndarray, gamma: np.ndarray, eps: float):
        x_bits = np.ascontiguousarray(x_bits, dtype=np.uint16)
        gamma = np.ascontiguousarray(gamma, dtype=np.float32)
        M, K = x_bits.shape
        q = np.empty((M, K), dtype=np.int8)
        a = np.empty(M, dtype=np.float32)
        self.lib.orc_rmsnorm_quant(_ptr(x_bits), _ptr(gamma), eps, M, K, _ptr(q), _ptr(a))
        return q, a

    def ternary_acc(self, q: np.ndarray, wt: np.ndarray) -> np.ndarray:
        q = np.ascontiguousarray(q, dtype=np.int8)
        wt = np.ascontiguousarray(wt, dtype=np.int8)
        M, K = q.shape
        N = wt.shape[0]
        assert wt.shape[1] == K
        acc = np.empty((M, N), dtype=np.int32)
        self.lib.orc_ternary_acc(_ptr(q), _ptr(wt), M, K, N, _ptr(acc))
        return acc

    def rescale(self, acc: np.ndarray, absmax: np.ndarray, beta: float) -> np.ndarray:
        acc = np.ascontiguousarray(acc, dtype=np.int32)
        absmax = np.ascontiguousarray(absmax, dtype=np.float32)
        M, N = acc.shape
        y = np.empty((M, N), dtype=np.uint16)
        self.lib.orc_rescale(_ptr(acc), _ptr(absmax), float(beta), M, N, _ptr(y))
        return y

    def glu_gate(self, g_bits: np.ndarray, u_bits: np.ndarray) -> np.ndarray:
        g_bits = np.ascontiguousarray(g_bits, dtype=np.uint16)
        u_bits = np.ascontiguousarray(u_bits, dtype=np.uint16)
        assert g_bits.shape == u_bits.shape
        p = np.empty(g_bits.shape, dtype=np.uint16)
        self.lib.orc_glu_gate(_ptr(g_bits), _ptr(u_bits), g_bits.size, _ptr(p))
        return p

    def mlgru_scan(self, f_bits, c_bits, g_bits, h0=None):
        """bf16 [B, T, D] pre-activations -> (o bf16 bits [B, T, D], h_last fp32 [B, D])."""
        f_bits = np.ascontiguousarray(f_bits, dtype=np.uint16)
        c_bits = np.ascontiguousarray(c_bits, dtype=np.uint16)
        g_bits = np.ascontiguousarray(g_bits, dtype=np.uint16)
        B, T, D = f_bits.shape
        o = np.empty((B, T, D), dtype=np.uint16)
        h_last = np.empty((B, D), dtype=np.float32)
        h0p = None
        if h0 is not None:
            h0 = np.ascontiguousarray(h0, dtype=np.float32)
            h0p = _ptr(h0)
        self.lib.orc_mlgru_scan(_ptr(f_bits), _ptr(c_bits), _ptr(g_bits), h0p, B, T, D, _ptr(o), _ptr(h_last))
        return o, h_last

    def bitlinear_bwd(self, dy_bits, x_bits, gamma, eps, wt, beta):
        """-> (dx bf16 bits [M, K], dgamma fp32 [K], dW fp32 [N, K]) under the straight-through estimator."""
        dy_bits = np.ascontiguousarray(dy_bits, dtype=np.uint16)
        x_bits = np.ascontiguousarray(x_bits, dtype=np.uint16)
        gamma = np.ascontiguousarray(gamma, dtype=np.float32)
        wt = np.ascontiguousarray(wt, dtype=np.int8)
        M, K = x_bits.shape
        N = wt.shape[0]
        dx = np.empty((M, K), dtype=np.uint16)
        dg = np.empty(K, dtype=np.float32)
        dW = np.empty((N, K), dtype=np.float32)
        if self.lib.orc_bitlinear_bwd(_ptr(dy_bits), _ptr(x_bits), _ptr(gamma), eps, _ptr(wt), float(beta),
                                      M, K, N, _ptr(dx), _ptr(dg), _ptr(dW)) != 0:
            raise MemoryError("oracle allocation failed")
        return dx, dg, dW

    def bitlinear(self, x_bits, gamma, eps, W, eps_w):
        x_bits = np.ascontiguousarray(x_bits, dtype=np.uint16)
        gamma = np.ascontiguousarray(gamma, dtype=np.float32)
        W = np.ascontiguousarray(W, dtype=np.float32)
        M, K = x_bits.shape
        N = W.shape[0]
        y = np.empty((M, N), dtype=np.uint16)
        beta = np.zeros(1, dtype=np.float32)
        rc = self.lib.orc_bitlinear(_ptr(x_bits), _ptr(gamma), eps, _ptr(W), eps_w,
                                    M, K, N, _ptr(y), _ptr(beta))
        if rc != 0:
            raise MemoryError("oracle allocation failed")
        return y, np.float32(beta[0])

    def num_threads(self) -> int:
        return int(self.lib.orc_num_threads())


_CACHE: dict[str, Oracle] = {}


def load(path: str | None = None) -> Oracle:
    """Builds (if stale) and loads the oracle library."""
    if path is None:
        path = build()
    path = os.path.abspath(path)
    if path not in _CACHE:
        _CACHE[path] = Oracle(path)
    return _CACHE[path]
