"""The C ABI without a GPU: the library loads, exports every declared entry
point, and its host-side checks and launch plan behave as documented."""
import math
import os
import re

import pytest

from windowed_attention_vision_b200 import _lib, build

HEADER = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "include", "winattn.h")


@pytest.fixture(scope="module")
def lib():
    build.build()
    return _lib.load()


def declared_functions():
    text = open(HEADER).read()
    return sorted(set(re.findall(r"^\s*(?:const\s+)?[A-Za-z_][A-Za-z0-9_ ]*?\*?\s*\b(winattn_[a-z_]+)\s*\(",
                                 text, re.M)))


def test_exports_every_declared_symbol(lib):
    names = declared_functions()
    assert len(names) >= 7, names
    for n in names:
        assert hasattr(lib, n), f"{n} declared in winattn.h but not exported"
    assert set(names) == set(_lib.EXPORTS)


A = 1 << 20  # fake, 16-byte aligned addresses: only compared, never dereferenced


def chk(**kw):
    a = dict(q=A, k=2 * A, v=3 * A, theta=None, bias=None, B=2, H=16, W=16, M=8, shift=4, heads=2, d=32,
             rank=0, dtype=_lib.BF16, out=4 * A)
    a.update(kw)
    return _lib.check_args(a["q"], a["k"], a["v"], a["theta"], a["bias"], a["B"], a["H"], a["W"], a["M"],
                           a["shift"], a["heads"], a["d"], a["rank"], a["dtype"], a["out"])


def test_check_args_accepts_valid(lib):
    assert chk() == _lib.OK
    assert chk(theta=5 * A) == _lib.OK
    assert chk(rank=16, bias=6 * A) == _lib.OK
    assert chk(dtype=_lib.FP32, d=16) == _lib.OK
    assert chk(M=1, shift=0) == _lib.OK
    assert chk(M=3, shift=1) == _lib.OK   # 16 % 3 != 0: the grid is padded to 18 x 18


@pytest.mark.parametrize("kw,code", [
    (dict(q=None), _lib.ERR_ARG),
    (dict(out=None), _lib.ERR_ARG),
    (dict(B=0), _lib.ERR_ARG),
    (dict(heads=-1), _lib.ERR_ARG),
    (dict(M=0), _lib.ERR_ARG),
    (dict(shift=8), _lib.ERR_ARG),        # shift must be < M
    (dict(shift=-1), _lib.ERR_ARG),
    (dict(d=48), _lib.ERR_ARG),           # bf16 head dims are 32 or 64
    (dict(d=8, dtype=_lib.FP32), _lib.ERR_ARG),
    (dict(M=512, H=512, W=512), _lib.ERR_ARG),
    (dict(rank=16), _lib.ERR_RANK),       # rank without bias_feats
    (dict(bias=6 * A), _lib.ERR_RANK),    # bias_feats without rank
    (dict(rank=8, bias=6 * A), _lib.ERR_RANK),
    (dict(q=A + 8), _lib.ERR_ALIGN),
    (dict(out=4 * A + 2), _lib.ERR_ALIGN),
    (dict(theta=5 * A + 2), _lib.ERR_ALIGN),
    (dict(rank=16, bias=6 * A + 4), _lib.ERR_ALIGN),
    (dict(dtype=7), _lib.ERR_DTYPE),
    (dict(out=A + 4096), _lib.ERR_ALIAS),  # overlaps q
])
def test_check_args_rejects(lib, kw, code):
    assert chk(**kw) == code


def test_strerror_covers_codes(lib):
    for code in range(-10, 1):
        s = _lib.strerror(code)
        assert s and s != "unknown error code"
    assert _lib.strerror(-100) == "unknown error code"


def test_host_workspace_bytes(lib):
    n = 2 * 16 * 16 * 2 * 32 * 2
    assert _lib.host_workspace_bytes(2, 16, 16, 2, 32, _lib.BF16) == 4 * ((n + 255) // 256 * 256)
    assert _lib.host_workspace_bytes(0, 16, 16, 2, 32, _lib.BF16) == 0


GENERIC, SMALL, LARGE, SIMT, PIPE, PIPE16 = 0, 1, 2, 3, 4, 5


@pytest.mark.parametrize("B,H,W,M,shift,heads,d,rank,U,tiles,kernel", [
    (64, 56, 56, 8, 4, 3, 32, 0, 2, 1, PIPE),        # Swin stage 1: two 64-token windows per tile
    (64, 56, 56, 8, 0, 3, 32, 0, 2, 1, PIPE),
    (4, 32, 32, 8, 4, 4, 64, 0, 2, 1, PIPE),
    (4, 32, 32, 8, 3, 4, 32, 0, 2, 1, SMALL),        # shift 3: boxes are not whole swizzle atoms
    (4, 32, 32, 8, 4, 4, 32, 16, 2, 1, SMALL),       # rank-r factors
    (4, 64, 64, 16, 8, 4, 32, 0, 1, 2, PIPE16),      # 256-token windows: two query tiles against one S
    (2, 32, 48, 16, 0, 3, 64, 0, 1, 2, PIPE16),
    (2, 32, 48, 16, 0, 16, 64, 0, 1, 2, LARGE),      # RoPE table of 16 heads: the 16 x 16 kernel has no room
    (2, 32, 32, 16, 8, 2, 64, 16, 1, 2, GENERIC),    # rank-r factors at d = 64
    (2, 32, 32, 16, 4, 2, 32, 0, 1, 2, GENERIC),     # shift 4: a query tile would straddle the row seam
    (16, 128, 128, 32, 0, 3, 32, 0, 1, 8, LARGE),    # 1024-token windows: 8 query tiles each
    (4, 192, 192, 96, 0, 6, 32, 16, 1, 72, LARGE),   # 9216-token windows
    (1, 48, 48, 24, 0, 1, 32, 0, 1, 5, GENERIC),     # 576 tokens: no whole-row key tiles
    (1, 24, 24, 12, 0, 1, 32, 0, 1, 2, GENERIC),     # 144 tokens: a ragged second tile
    (1, 9, 9, 3, 0, 2, 64, 0, 14, 1, SMALL),         # 9-token windows: 14 per tile
    (2, 5, 5, 1, 0, 1, 32, 0, 128, 1, SMALL),        # one-token windows
    (1, 10, 10, 10, 0, 1, 32, 0, 1, 1, SMALL),       # 100 tokens: one ragged tile
    (1, 8, 8, 8, 0, 80, 32, 0, 2, 1, GENERIC),       # too many heads for a shared-memory RoPE table
    (64, 56, 56, 32, 16, 3, 32, 0, 1, 8, LARGE),     # FlashSwin-T at M = 32: 56 padded to 64, pad keys masked
    (64, 56, 56, 16, 8, 3, 32, 0, 1, 2, PIPE16),     # FlashSwin-T at M = 16: padded by half a window
    (2, 40, 24, 16, 0, 2, 32, 0, 1, 2, PIPE16),      # the same without shift
    (1, 36, 32, 16, 8, 2, 32, 0, 1, 2, LARGE),       # padded by 12 rows: pads split key granules
    (2, 10, 13, 4, 2, 2, 32, 0, 8, 1, GENERIC),      # padded 12 x 16 grid of 16-token windows
])
def test_launch_plan(lib, B, H, W, M, shift, heads, d, rank, U, tiles, kernel):
    rc, info = _lib.launch_info(B, H, W, M, shift, heads, d, rank, _lib.BF16)
    assert rc == _lib.OK
    windows = B * (-(-H // M)) * (-(-W // M))   # windows of the grid padded to multiples of M
    assert info["windows_per_tile"] == U
    assert info["kernel"] == kernel
    if kernel in (LARGE, PIPE16):  # items are pairs of query tiles
        assert info["work_items"] == heads * windows * tiles // 2
        threads = 512 if kernel == LARGE else 1024  # the 16 x 16 kernel: RoPE x2, softmax x4, epilogue, 4 warps
        assert info["threads"] == threads and info["grid"] == min(148, info["work_items"])
    else:
        assert info["work_items"] == heads * math.ceil(windows / U) * tiles
    if kernel == SMALL:
        groups = 4 if d == 32 else 3  # compute warpgroups, plus a loader warp
        assert info["threads"] == (4 * groups + 1) * 32 and info["grid"] == min(148, info["work_items"])
    elif kernel == PIPE:  # RoPE x2, softmax x2, epilogue warpgroups, two loader and two MMA warps
        assert info["threads"] == 24 * 32 and info["grid"] == min(148, info["work_items"])
    elif kernel == GENERIC:
        assert info["threads"] == 128 and info["grid"] == info["work_items"]
    assert 0 < info["smem_bytes"] <= 227 * 1024


def test_launch_plan_fp32(lib):
    rc, info = _lib.launch_info(1, 16, 16, 8, 0, 2, 32, 0, _lib.FP32)
    assert rc == _lib.OK and info["kernel"] == SIMT


def test_kernel_switch_routes_to_fallbacks(lib):
    """Disabling a specialised kernel sends its problems to the next kernel
    that serves them (in the end the generic tensor-core kernel); the switch
    is process-wide and returns its previous state."""
    dense = (16, 128, 128, 32, 16, 3, 32, 0, _lib.BF16)
    swin = (64, 56, 56, 8, 4, 3, 32, 0, _lib.BF16)
    m16 = (4, 64, 64, 16, 8, 4, 32, 0, _lib.BF16)
    assert _lib.launch_info(*dense)[1]["kernel"] == _lib.KERNEL_LARGE
    assert _lib.launch_info(*swin)[1]["kernel"] == _lib.KERNEL_PIPE
    assert _lib.launch_info(*m16)[1]["kernel"] == _lib.KERNEL_PIPE16
    try:
        assert _lib.set_kernel_enabled(_lib.KERNEL_PIPE16, False) == 1
        assert _lib.launch_info(*m16)[1]["kernel"] == _lib.KERNEL_LARGE
        assert _lib.set_kernel_enabled(_lib.KERNEL_LARGE, False) == 1
        assert _lib.launch_info(*dense)[1]["kernel"] == _lib.KERNEL_GENERIC
        assert _lib.set_kernel_enabled(_lib.KERNEL_PIPE, False) == 1
        assert _lib.launch_info(*swin)[1]["kernel"] == _lib.KERNEL_SMALL
        assert _lib.set_kernel_enabled(_lib.KERNEL_SMALL, False) == 1
        assert _lib.launch_info(*swin)[1]["kernel"] == _lib.KERNEL_GENERIC
        assert _lib.set_kernel_enabled(_lib.KERNEL_SMALL, False) == 0
    finally:
        for k in (_lib.KERNEL_LARGE, _lib.KERNEL_PIPE, _lib.KERNEL_SMALL, _lib.KERNEL_PIPE16):
            _lib.set_kernel_enabled(k, True)
    assert _lib.launch_info(*m16)[1]["kernel"] == _lib.KERNEL_PIPE16
    assert _lib.launch_info(*dense)[1]["kernel"] == _lib.KERNEL_LARGE
    assert _lib.launch_info(*swin)[1]["kernel"] == _lib.KERNEL_PIPE
    # the generic and fp32 kernels have no switch
    assert _lib.set_kernel_enabled(_lib.KERNEL_GENERIC, False) == _lib.ERR_ARG
    assert _lib.set_kernel_enabled(_lib.KERNEL_SIMT, False) == _lib.ERR_ARG


def test_bwd_workspace_bytes(lib):
    # windows of at most one 128-row tile need none; larger ones an fp32 map
    assert _lib.bwd_workspace_bytes(64, 56, 56, 8, 3, 32) == 0
    assert _lib.bwd_workspace_bytes(1, 20, 20, 10, 2, 32) == 0
    n = 16 * 128 * 128 * 3 * 32 * 4
    assert _lib.bwd_workspace_bytes(16, 128, 128, 32, 3, 32) == (n + 255) // 256 * 256
    assert _lib.bwd_workspace_bytes(1, 56, 56, 32, 3, 64) == (56 * 56 * 3 * 64 * 4 + 255) // 256 * 256
    assert _lib.bwd_workspace_bytes(0, 8, 8, 4, 1, 32) == 0
    assert _lib.bwd_workspace_bytes(1, 8, 8, 4, 1, 48) == 0
