"""Window-attention oracle: plain fp64 CPU reference (ctypes over winattn_oracle.c).

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` may import this package.  It shares no code with
the CUDA path and the CUDA path never calls it.

What it computes is the plain definition of exact windowed softmax attention
from "FLASHSWIN: Unlocking Large Windows and Dense Tokens in Swin Vision
Transformers with Memory Efficient Attention" (section "어떻게 동작하나": window
partition, cyclic shift with an additive wrap mask, window-local 2D RoPE) and
the feature concatenation of "Rank-Factorized Implicit Neural Bias" (section
2.1).  Steps are written out in ``winattn_oracle.c``.

Inputs are numpy arrays in storage form: ``uint16`` arrays holding bf16 bits,
or ``float32`` arrays.  ``theta`` is float32 ``[heads][d/4]``; ``bias`` is
``[heads][2][M*M][rank]`` in the same storage dtype as q/k/v.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "winattn_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")

_lib = None


def build(src: str = _SRC, out: str = _LIB, extra_flags: tuple = ()) -> str:
    """Compile the oracle with gcc into a shared library; returns its path."""
    cmd = ["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-o", out, src,
           "-lm", "-lpthread", *extra_flags]
    subprocess.run(cmd, check=True)
    return out


def load(path: str | None = None):
    """Load (building if missing or stale) the oracle library."""
    global _lib
    if path is not None:
        return _bind(ctypes.CDLL(path))
    if _lib is None:
        if (not os.path.exists(_LIB)) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
            build()
        _lib = _bind(ctypes.CDLL(_LIB))
    return _lib


def _bind(lib):
    vp, i32, i64, f64 = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_double
    lib.oracle_fwd.argtypes = [vp, vp, vp, i32, vp, vp] + [i32] * 8 + [vp, i32, f64]
    lib.oracle_fwd.restype = i32
    lib.oracle_fwd_lse.argtypes = [vp, vp, vp, i32, vp, vp] + [i32] * 8 + [vp, vp, i32, f64]
    lib.oracle_fwd_lse.restype = i32
    lib.oracle_fwd_sparse.argtypes = [vp, vp, vp, i32, vp, vp] + [i32] * 8 + [vp, i64, vp]
    lib.oracle_fwd_sparse.restype = i32
    lib.oracle_rib_features.argtypes = [vp, vp, i32, i32, i32, vp]
    lib.oracle_rib_features.restype = i32
    lib.oracle_cla_gate.argtypes = [vp, vp, i32, vp, vp, vp, vp, i32, i32, i32, i32, vp]
    lib.oracle_cla_gate.restype = i32
    lib.oracle_fwd_units.argtypes = [vp, vp, vp, i32, vp, vp] + [i32] * 8 + [vp, i64, vp, i32, f64]
    lib.oracle_fwd_units.restype = i32
    lib.oracle_rope.argtypes = [vp, i32, f64, f64, vp, vp]
    lib.oracle_rope.restype = i32
    lib.oracle_token_origin.argtypes = [i32] * 7 + [vp, vp]
    lib.oracle_token_origin.restype = i32
    lib.oracle_bwd.argtypes = [vp, vp, vp, i32, vp, vp] + [i32] * 8 + [vp] * 6 + [i32]
    lib.oracle_bwd.restype = i32
    return lib


def _dtype_code(a: np.ndarray) -> int:
    if a.dtype == np.uint16:
        return 0
    if a.dtype == np.float32:
        return 1
    raise TypeError(f"oracle inputs must be uint16 (bf16 bits) or float32, got {a.dtype}")


def _ptr(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


class Oracle:
    """A bound oracle library (the real one, or a test-built variant)."""

    def __init__(self, lib=None):
        self.lib = lib if lib is not None else load()

    def _prep(self, q, k, v, theta, bias, M):
        q, k, v = (np.ascontiguousarray(x) for x in (q, k, v))
        if not (q.shape == k.shape == v.shape) or q.ndim != 5:
            raise ValueError("q, k, v must share one [B, H, W, heads, d] shape")
        code = _dtype_code(q)
        if _dtype_code(k) != code or _dtype_code(v) != code:
            raise TypeError("q, k, v must share one storage dtype")
        B, H, W, heads, d = q.shape
        if theta is not None:
            theta = np.ascontiguousarray(theta, dtype=np.float32)
            if theta.shape != (heads, d // 4):
                raise ValueError(f"theta must be [heads, d/4] = {(heads, d // 4)}")
        rank = 0
        if bias is not None:
            bias = np.ascontiguousarray(bias)
            if _dtype_code(bias) != code:
                raise TypeError("bias must share the q/k/v storage dtype")
            if bias.ndim != 4 or bias.shape[:3] != (heads, 2, M * M):
                raise ValueError("bias must be [heads, 2, M*M, rank]")
            rank = bias.shape[3]
        return q, k, v, theta, bias, code, (B, H, W, heads, d, rank)

    def fwd(self, q, k, v, *, M, shift=0, theta=None, bias=None, nthreads=0,
            mem_budget=8e9) -> np.ndarray:
        """Whole output map [B, H, W, heads, d] in fp64."""
        q, k, v, theta, bias, code, (B, H, W, heads, d, rank) = self._prep(q, k, v, theta, bias, M)
        out = np.zeros((B, H, W, heads, d), dtype=np.float64)
        rc = self.lib.oracle_fwd(_ptr(q), _ptr(k), _ptr(v), code, _ptr(theta), _ptr(bias),
                                 B, H, W, M, shift, heads, d, rank, _ptr(out), nthreads,
                                 float(mem_budget))
        if rc < 0:
            raise ValueError(f"oracle rejected the problem (code {rc})")
        return out

    def fwd_lse(self, q, k, v, *, M, shift=0, theta=None, bias=None, nthreads=0, mem_budget=8e9):
        """(O [B, H, W, heads, d], lse [B, H, W, heads]) in fp64: lse is each
        row's log-sum-exp of its masked scores (natural log)."""
        q, k, v, theta, bias, code, (B, H, W, heads, d, rank) = self._prep(q, k, v, theta, bias, M)
        out = np.zeros((B, H, W, heads, d), dtype=np.float64)
        lse = np.zeros((B, H, W, heads), dtype=np.float64)
        rc = self.lib.oracle_fwd_lse(_ptr(q), _ptr(k), _ptr(v), code, _ptr(theta), _ptr(bias),
                                     B, H, W, M, shift, heads, d, rank, _ptr(out), _ptr(lse), nthreads,
                                     float(mem_budget))
        if rc < 0:
            raise ValueError(f"oracle rejected the problem (code {rc})")
        return out, lse

    def fwd_sparse(self, q, k, v, o_lin, windows, *, M, shift=0, theta=None, bias=None) -> np.ndarray:
        """The gated residual of HSMLA's two-path kernel: a copy of o_lin
        [B, H, W, heads, d] where every token of the listed windows
        (w = (b*nWy + wy)*nWx + wx, all heads) gets O_local - O_lin-local
        added; fp64."""
        q, k, v, theta, bias, code, (B, H, W, heads, d, rank) = self._prep(q, k, v, theta, bias, M)
        out = np.array(o_lin, dtype=np.float64, copy=True, order="C")
        if out.shape != q.shape:
            raise ValueError("o_lin must have the shape of q")
        windows = np.ascontiguousarray(windows, dtype=np.int32)
        rc = self.lib.oracle_fwd_sparse(_ptr(q), _ptr(k), _ptr(v), code, _ptr(theta), _ptr(bias),
                                        B, H, W, M, shift, heads, d, rank, _ptr(windows), len(windows), _ptr(out))
        if rc < 0:
            raise ValueError(f"oracle rejected the problem (code {rc})")
        return out

    def fwd_units(self, q, k, v, units, *, M, shift=0, theta=None, bias=None,
                  nthreads=0, mem_budget=8e9) -> np.ndarray:
        """Selected units u = ((b*nWy + wy)*nWx + wx)*heads + h -> [n, M*M, d] fp64,
        each in window order p = i*M + j (nWy, nWx count the windows of the
        grid padded to multiples of M; rows at pad positions are NaN)."""
        q, k, v, theta, bias, code, (B, H, W, heads, d, rank) = self._prep(q, k, v, theta, bias, M)
        units = np.ascontiguousarray(units, dtype=np.int64)
        out = np.zeros((len(units), M * M, d), dtype=np.float64)
        rc = self.lib.oracle_fwd_units(_ptr(q), _ptr(k), _ptr(v), code, _ptr(theta), _ptr(bias),
                                       B, H, W, M, shift, heads, d, rank, _ptr(units),
                                       len(units), _ptr(out), nthreads, float(mem_budget))
        if rc < 0:
            raise ValueError(f"oracle rejected the problem (code {rc})")
        return out

    def bwd(self, q, k, v, dout, *, M, shift=0, theta=None, bias=None, nthreads=0):
        """Gradients of a scalar loss given dout = dL/dO [B, H, W, heads, d]:
        (dq, dk, dv, dtheta, dbias) in fp64; dtheta [heads, d/4] (None without
        theta), dbias [heads, 2, M*M, rank] (None without bias)."""
        q, k, v, theta, bias, code, (B, H, W, heads, d, rank) = self._prep(q, k, v, theta, bias, M)
        dout = np.ascontiguousarray(dout, dtype=np.float64)
        if dout.shape != q.shape:
            raise ValueError("dout must have the shape of q")
        dq, dk, dv = (np.zeros(q.shape, dtype=np.float64) for _ in range(3))
        dtheta = None if theta is None else np.zeros((heads, d // 4), dtype=np.float64)
        dbias = None if bias is None else np.zeros(bias.shape, dtype=np.float64)
        rc = self.lib.oracle_bwd(_ptr(q), _ptr(k), _ptr(v), code, _ptr(theta), _ptr(bias),
                                 B, H, W, M, shift, heads, d, rank, _ptr(dout), _ptr(dq), _ptr(dk), _ptr(dv),
                                 _ptr(dtheta), _ptr(dbias), nthreads)
        if rc < 0:
            raise ValueError(f"oracle rejected the problem (code {rc})")
        return dq, dk, dv, dtheta, dbias

    def rib_features(self, w1, w2, M) -> np.ndarray:
        """Rank-r factor table [heads, 2, M*M, rank] fp64 from the MLP weights
        w1 [heads, 2, 32, 64] and w2 [heads, 2, 64, rank] (fp32)."""
        w1 = np.ascontiguousarray(w1, dtype=np.float32)
        w2 = np.ascontiguousarray(w2, dtype=np.float32)
        heads, rank = w1.shape[0], w2.shape[3]
        if w1.shape != (heads, 2, 32, 64) or w2.shape != (heads, 2, 64, rank):
            raise ValueError("w1 must be [heads, 2, 32, 64] and w2 [heads, 2, 64, rank]")
        out = np.zeros((heads, 2, M * M, rank), dtype=np.float64)
        if self.lib.oracle_rib_features(_ptr(w1), _ptr(w2), M, heads, rank, _ptr(out)):
            raise ValueError("bad feature arguments")
        return out

    def cla_gate(self, x, o, dw, dw_b, pw, pw_b) -> np.ndarray:
        """O * sigmoid(PW(DW3x3(x))) [B, H, W, C] fp64; x, o in storage form."""
        x, o = np.ascontiguousarray(x), np.ascontiguousarray(o)
        code = _dtype_code(x)
        if _dtype_code(o) != code or x.shape != o.shape or x.ndim != 4:
            raise ValueError("x and o must share one [B, H, W, C] shape and storage dtype")
        B, H, W, C = x.shape
        dw, dw_b, pw, pw_b = (np.ascontiguousarray(a, dtype=np.float32) for a in (dw, dw_b, pw, pw_b))
        if dw.shape != (C, 3, 3) or dw_b.shape != (C,) or pw.shape != (C, C) or pw_b.shape != (C,):
            raise ValueError("dw [C, 3, 3], dw_b [C], pw [C, C], pw_b [C]")
        out = np.zeros((B, H, W, C), dtype=np.float64)
        if self.lib.oracle_cla_gate(_ptr(x), _ptr(o), code, _ptr(dw), _ptr(dw_b), _ptr(pw), _ptr(pw_b), B, H, W, C,
                                    _ptr(out)):
            raise ValueError("bad gate arguments")
        return out

    def rope(self, vec, i, j, theta_h) -> np.ndarray:
        """R(i, j) vec for one d-vector (window-local row i, column j)."""
        vec = np.ascontiguousarray(vec, dtype=np.float64)
        theta_h = np.ascontiguousarray(theta_h, dtype=np.float32)
        out = np.empty_like(vec)
        if self.lib.oracle_rope(_ptr(vec), vec.shape[0], float(i), float(j), _ptr(theta_h), _ptr(out)):
            raise ValueError("bad rope arguments")
        return out

    def token_origin(self, H, W, M, shift, wy, wx, p):
        """Original (row, col) of token p of rolled window (wy, wx) in the grid
        padded to multiples of M (row >= H or col >= W: a pad position)."""
        y, x = ctypes.c_int(), ctypes.c_int()
        if self.lib.oracle_token_origin(H, W, M, shift, wy, wx, p, ctypes.byref(y), ctypes.byref(x)) < 0:
            raise ValueError("bad token arguments")
        return y.value, x.value


def oracle() -> Oracle:
    return Oracle()
