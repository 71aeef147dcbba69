"""ctypes binding of the C ABI in include/winattn.h (argument marshalling only).

Every step of the attention runs inside the CUDA library; this module only
passes pointers, sizes and the stream.  It raises ``WinattnError`` when the
library is missing or a call fails: there is no fallback.
"""
from __future__ import annotations

import ctypes
import os

HERE = os.path.dirname(os.path.abspath(__file__))
# WINATTN_LIB selects another build of the library, e.g. the bounds-checking
# debug build (libwinattn_debug.so, made by build.build(debug=True))
LIB_PATH = os.environ.get("WINATTN_LIB") or os.path.join(HERE, "libwinattn.so")
DEBUG_LIB_PATH = os.path.join(HERE, "libwinattn_debug.so")

OK = 0
ERR_ARG, ERR_RANK, ERR_ALIGN, ERR_DTYPE, ERR_ARCH = -1, -2, -3, -4, -5
ERR_CUDA, ERR_DEVICE_TIMEOUT, ERR_ALIAS, ERR_SIZE, ERR_DEVICE_BOUNDS = -6, -7, -8, -9, -10
BF16, FP32 = 0, 1

EXPORTS = ("winattn_fwd", "winattn_fwd_lse", "winattn_check_args", "winattn_fwd_host", "winattn_host_workspace_bytes",
           "winattn_strerror", "winattn_last_device_status", "winattn_launch_info", "winattn_fwd_host_static",
           "winattn_selftest_wait_timeout", "winattn_set_kernel_enabled", "winattn_bwd",
           "winattn_bwd_workspace_bytes", "winattn_fwd_sparse", "winattn_rib_features", "winattn_fwd_rib",
           "winattn_cla_gate")
STATIC_WORKSPACE_BYTES = 32 << 20


class WinattnError(RuntimeError):
    def __init__(self, code: int, what: str = ""):
        self.code = code
        msg = strerror(code) if _lib is not None else f"code {code}"
        super().__init__(f"{what}: {msg} ({code})" if what else f"{msg} ({code})")


_lib = None
loaded_path = None  # the library file this process loaded


def load(path: str = LIB_PATH):
    """Load the in-tree CUDA library (built by ``build.build()``)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(path):
        raise WinattnError(ERR_CUDA, f"CUDA library {path} is missing; run __graft_entry__.build()")
    lib = ctypes.CDLL(path)
    global loaded_path
    loaded_path = path
    vp, i32, i64, sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_size_t
    lib.winattn_fwd.argtypes = [vp, vp, vp, vp, vp] + [i32] * 9 + [vp, vp]
    lib.winattn_fwd.restype = i32
    lib.winattn_fwd_lse.argtypes = [vp, vp, vp, vp, vp] + [i32] * 9 + [vp, vp, vp]
    lib.winattn_fwd_lse.restype = i32
    lib.winattn_check_args.argtypes = [vp, vp, vp, vp, vp] + [i32] * 9 + [vp]
    lib.winattn_check_args.restype = i32
    lib.winattn_fwd_host.argtypes = [vp, vp, vp, vp, vp] + [i32] * 9 + [vp, vp, sz, vp]
    lib.winattn_fwd_host.restype = i32
    lib.winattn_fwd_host_static.argtypes = [vp, vp, vp, vp, vp] + [i32] * 9 + [vp, vp]
    lib.winattn_fwd_host_static.restype = i32
    lib.winattn_host_workspace_bytes.argtypes = [i32] * 6
    lib.winattn_host_workspace_bytes.restype = sz
    lib.winattn_strerror.argtypes = [i32]
    lib.winattn_strerror.restype = ctypes.c_char_p
    lib.winattn_last_device_status.argtypes = [vp]
    lib.winattn_last_device_status.restype = i32
    lib.winattn_launch_info.argtypes = [i32] * 9 + [ctypes.POINTER(i64)] + [ctypes.POINTER(i32)] * 5
    lib.winattn_launch_info.restype = i32
    lib.winattn_selftest_wait_timeout.argtypes = [vp]
    lib.winattn_selftest_wait_timeout.restype = i32
    lib.winattn_bwd.argtypes = [vp] * 8 + [i32] * 9 + [vp] * 6 + [sz, vp]
    lib.winattn_bwd.restype = i32
    lib.winattn_bwd_workspace_bytes.argtypes = [i32] * 6
    lib.winattn_bwd_workspace_bytes.restype = sz
    lib.winattn_fwd_sparse.argtypes = [vp] * 5 + [i32] * 9 + [vp, i32, vp, vp]
    lib.winattn_fwd_sparse.restype = i32
    lib.winattn_rib_features.argtypes = [vp, vp, i32, i32, i32, vp, vp]
    lib.winattn_rib_features.restype = i32
    lib.winattn_fwd_rib.argtypes = [vp] * 6 + [i32] * 9 + [vp, vp, vp]
    lib.winattn_fwd_rib.restype = i32
    lib.winattn_cla_gate.argtypes = [vp] * 6 + [i32] * 5 + [vp, vp]
    lib.winattn_cla_gate.restype = i32
    lib.winattn_set_kernel_enabled.argtypes = [i32, i32]
    lib.winattn_set_kernel_enabled.restype = i32
    _lib = lib
    return lib


def strerror(code: int) -> str:
    return load().winattn_strerror(code).decode()


def fwd(q_ptr, k_ptr, v_ptr, theta_ptr, bias_ptr, B, H, W, M, shift, heads, d, rank, dtype, out_ptr,
        stream) -> int:
    return load().winattn_fwd(q_ptr, k_ptr, v_ptr, theta_ptr, bias_ptr, B, H, W, M, shift, heads, d, rank,
                              dtype, out_ptr, stream)


def fwd_lse(q_ptr, k_ptr, v_ptr, theta_ptr, bias_ptr, B, H, W, M, shift, heads, d, rank, dtype, out_ptr, lse_ptr,
            stream) -> int:
    return load().winattn_fwd_lse(q_ptr, k_ptr, v_ptr, theta_ptr, bias_ptr, B, H, W, M, shift, heads, d, rank,
                                  dtype, out_ptr, lse_ptr, stream)


def bwd(q_ptr, k_ptr, v_ptr, theta_ptr, bias_ptr, out_ptr, dout_ptr, lse_ptr, B, H, W, M, shift, heads, d, rank,
        dtype, dq_ptr, dk_ptr, dv_ptr, dtheta_ptr, dbias_ptr, ws_ptr, ws_bytes, stream) -> int:
    return load().winattn_bwd(q_ptr, k_ptr, v_ptr, theta_ptr, bias_ptr, out_ptr, dout_ptr, lse_ptr, B, H, W, M, shift,
                              heads, d, rank, dtype, dq_ptr, dk_ptr, dv_ptr, dtheta_ptr, dbias_ptr, ws_ptr, ws_bytes,
                              stream)


def bwd_workspace_bytes(B, H, W, M, heads, d) -> int:
    return load().winattn_bwd_workspace_bytes(B, H, W, M, heads, d)


def fwd_sparse(q_ptr, k_ptr, v_ptr, theta_ptr, bias_ptr, B, H, W, M, shift, heads, d, rank, dtype, win_ptr, n_win,
               out_ptr, stream) -> int:
    return load().winattn_fwd_sparse(q_ptr, k_ptr, v_ptr, theta_ptr, bias_ptr, B, H, W, M, shift, heads, d, rank,
                                     dtype, win_ptr, n_win, out_ptr, stream)


def rib_features(w1_ptr, w2_ptr, M, heads, rank, table_ptr, stream) -> int:
    return load().winattn_rib_features(w1_ptr, w2_ptr, M, heads, rank, table_ptr, stream)


def fwd_rib(q_ptr, k_ptr, v_ptr, theta_ptr, w1_ptr, w2_ptr, B, H, W, M, shift, heads, d, rank, dtype, table_ptr,
            out_ptr, stream) -> int:
    return load().winattn_fwd_rib(q_ptr, k_ptr, v_ptr, theta_ptr, w1_ptr, w2_ptr, B, H, W, M, shift, heads, d, rank,
                                  dtype, table_ptr, out_ptr, stream)


def cla_gate(x_ptr, o_ptr, dw_ptr, dwb_ptr, pw_ptr, pwb_ptr, B, H, W, C, dtype, out_ptr, stream) -> int:
    return load().winattn_cla_gate(x_ptr, o_ptr, dw_ptr, dwb_ptr, pw_ptr, pwb_ptr, B, H, W, C, dtype, out_ptr,
                                   stream)


def check_args(q_ptr, k_ptr, v_ptr, theta_ptr, bias_ptr, B, H, W, M, shift, heads, d, rank, dtype,
               out_ptr) -> int:
    return load().winattn_check_args(q_ptr, k_ptr, v_ptr, theta_ptr, bias_ptr, B, H, W, M, shift, heads, d,
                                     rank, dtype, out_ptr)


def fwd_host(q_ptr, k_ptr, v_ptr, theta_ptr, bias_ptr, B, H, W, M, shift, heads, d, rank, dtype, out_ptr,
             ws_ptr, ws_bytes, stream) -> int:
    return load().winattn_fwd_host(q_ptr, k_ptr, v_ptr, theta_ptr, bias_ptr, B, H, W, M, shift, heads, d,
                                   rank, dtype, out_ptr, ws_ptr, ws_bytes, stream)


def fwd_host_static(q_ptr, k_ptr, v_ptr, theta_ptr, bias_ptr, B, H, W, M, shift, heads, d, rank, dtype, out_ptr,
                    stream) -> int:
    return load().winattn_fwd_host_static(q_ptr, k_ptr, v_ptr, theta_ptr, bias_ptr, B, H, W, M, shift, heads, d,
                                          rank, dtype, out_ptr, stream)


def host_workspace_bytes(B, H, W, heads, d, dtype) -> int:
    return load().winattn_host_workspace_bytes(B, H, W, heads, d, dtype)


def last_device_status(stream) -> int:
    return load().winattn_last_device_status(stream)


def selftest_wait_timeout(stream) -> int:
    return load().winattn_selftest_wait_timeout(stream)


KERNEL_GENERIC, KERNEL_SMALL, KERNEL_LARGE, KERNEL_SIMT, KERNEL_PIPE, KERNEL_PIPE16 = 0, 1, 2, 3, 4, 5


def set_kernel_enabled(kernel: int, enabled: bool) -> int:
    """Switch a specialised kernel off (its problems go to the next kernel that
    serves them) or back on; returns the previous state or ERR_ARG."""
    return load().winattn_set_kernel_enabled(kernel, 1 if enabled else 0)


def launch_info(B, H, W, M, shift, heads, d, rank, dtype):
    """(rc, dict) with work_items, grid, threads, smem_bytes, windows_per_tile, kernel."""
    i64, i32 = ctypes.c_int64, ctypes.c_int
    items, grid, threads, smem, wpt, kern = i64(), i32(), i32(), i32(), i32(), i32()
    rc = load().winattn_launch_info(B, H, W, M, shift, heads, d, rank, dtype, ctypes.byref(items),
                                    ctypes.byref(grid), ctypes.byref(threads), ctypes.byref(smem),
                                    ctypes.byref(wpt), ctypes.byref(kern))
    return rc, dict(work_items=items.value, grid=grid.value, threads=threads.value, smem_bytes=smem.value,
                    windows_per_tile=wpt.value, kernel=kern.value)
