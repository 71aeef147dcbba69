"""GPU parity: the CUDA path through the C ABI against the fp64 oracle, element
by element on the same seeded inputs.

Small shapes are compared over the whole output; the full-size workloads (the
shapes the benchmark times) are compared on sampled windows that always include
every wrap case (corner, edge and interior windows), with a finiteness scan of
the whole output.  Tolerances: fp32 rel-L2 <= 1e-5; bf16 max-abs <= 2e-2 and
rel-L2 <= 5e-3."""
import numpy as np
import pytest
import torch

import windowed_attention_vision_b200 as wa
from windowed_attention_vision_b200 import _lib
from windowed_attention_vision_b200 import inputs as I
from tests import gpu_helpers as G

pytestmark = pytest.mark.gpu

SMALL = [
    # name, B, H, W, M, shift, heads, d, dtype, rope, rank
    ("m8_s4_d32", 2, 16, 16, 8, 4, 2, 32, "bf16", "learned", 0),
    ("m8_s0_d64", 2, 16, 24, 8, 0, 2, 64, "bf16", "standard", 0),
    ("m8_odd_pack", 1, 24, 8, 8, 3, 1, 32, "bf16", "learned", 0),   # 3 windows: a half-empty pack
    ("m8_odd_pack_tma", 1, 24, 8, 8, 4, 2, 32, "bf16", "learned", 0),  # TMA quadrants + empty slot
    ("m8_s4_d64_tma", 3, 16, 16, 8, 4, 2, 64, "bf16", "learned", 0),
    ("m8_s0_d64_nope", 1, 16, 16, 8, 0, 3, 64, "bf16", None, 0),
    ("m8_s4_d32_nope_odd", 5, 24, 40, 8, 4, 3, 32, "bf16", None, 0),  # 75 windows per head: odd packs
    ("m8_s4_d32_deep", 8, 64, 64, 8, 4, 4, 32, "bf16", "learned", 0),  # many tiles per CTA
    ("m4_s0_tma", 2, 8, 12, 4, 0, 2, 32, "bf16", "learned", 0),      # 8 windows per tile via TMA
    ("m7_s3", 2, 14, 21, 7, 3, 2, 32, "bf16", "learned", 0),        # 49-token windows, 2 per tile
    ("m4_s2", 1, 12, 8, 4, 2, 3, 32, "bf16", "learned", 0),         # 16-token windows, 8 per tile
    ("m3_s1", 1, 9, 6, 3, 1, 2, 64, "bf16", "learned", 0),          # 9-token windows, 14 per tile
    ("m1", 2, 5, 7, 1, 0, 2, 32, "bf16", "learned", 0),             # one-token windows
    ("m2_s1", 1, 4, 6, 2, 1, 1, 32, "bf16", None, 0),
    ("m10_s5", 1, 20, 20, 10, 5, 2, 32, "bf16", "learned", 0),      # 100 tokens: ragged single tile
    ("m12_s6", 1, 24, 24, 12, 6, 2, 32, "bf16", "learned", 0),      # 144 tokens: ragged second tile
    ("m16_s8_d64", 1, 32, 32, 16, 8, 2, 64, "bf16", "learned", 0),
    ("m32_s16", 1, 64, 64, 32, 16, 2, 32, "bf16", "standard", 0),
    ("m8_s4_many_heads", 1, 16, 16, 8, 4, 80, 32, "bf16", "learned", 0),  # generic kernel at N = 64
    ("m11_s5_d64_r16", 1, 22, 22, 11, 5, 2, 64, "bf16", "learned", 16),   # 121 tokens, small kernel
    ("m9_s4_r32", 2, 18, 9, 9, 4, 3, 32, "bf16", None, 32),
    ("m24_s0_r16", 1, 48, 48, 24, 0, 2, 32, "bf16", None, 16),      # bias factors, no RoPE
    ("m16_s0_d32", 2, 32, 48, 16, 0, 2, 32, "bf16", "learned", 0),  # pipelined 16 x 16 kernel
    # several items per CTA: both O buffers of a query tile in turn, and the
    # epilogue of each item trailing the next item's first step
    ("m16_s8_d32_items", 8, 64, 64, 16, 8, 4, 32, "bf16", "learned", 0),
    ("m32_s16_d32_items", 8, 64, 64, 32, 16, 3, 32, "bf16", "learned", 0),
    ("m32_s0_d32_items", 8, 64, 64, 32, 0, 3, 32, "bf16", "standard", 0),
    ("m16_s8_d64_items", 8, 64, 64, 16, 8, 2, 64, "bf16", "learned", 0),  # one O buffer
    ("m16_s8_d32_nope", 1, 32, 32, 16, 8, 3, 32, "bf16", None, 0),
    ("m32_s0_d64", 1, 64, 96, 32, 0, 2, 64, "bf16", "standard", 0),
    ("m32_s0_r16", 1, 64, 64, 32, 0, 2, 32, "bf16", None, 16),
    ("m32_s0_r32_rope", 1, 64, 64, 32, 0, 1, 64, "bf16", "learned", 32),
    ("m64_s32", 1, 128, 128, 64, 32, 1, 32, "bf16", "learned", 0),
    ("m96_s48_d64", 1, 192, 96, 96, 48, 1, 64, "bf16", "learned", 0),
    ("m96_s0_r16", 1, 96, 96, 96, 0, 2, 32, "bf16", None, 16),
    ("m8_s4_r32_rope", 2, 16, 16, 8, 4, 2, 32, "bf16", "learned", 32),
    ("m16_s8_d64_r16", 1, 32, 32, 16, 8, 1, 64, "bf16", "learned", 16),
    # grids that are not multiples of M: padded, pad positions masked and never written
    ("m32_s16_pad56", 1, 56, 56, 32, 16, 2, 32, "bf16", "learned", 0),
    ("m32_s0_pad56", 1, 56, 56, 32, 0, 2, 32, "bf16", "standard", 0),
    ("m16_s8_pad_d64", 1, 56, 40, 16, 8, 2, 64, "bf16", "learned", 0),   # half-window pads: 16 x 16 kernel
    ("m16_s0_pad_d32", 2, 40, 24, 16, 0, 2, 32, "bf16", "learned", 0),   # the same without shift
    ("m16_s8_padw", 1, 32, 56, 16, 8, 3, 32, "bf16", "standard", 0),     # pad columns only
    ("m16_s8_pad12", 1, 36, 32, 16, 8, 2, 32, "bf16", "learned", 0),     # 12 pad rows: large-window kernel
    ("m4_s2_pad", 2, 10, 13, 4, 2, 2, 32, "bf16", "learned", 0),
    ("m8_s4_pad20", 1, 20, 20, 8, 4, 2, 32, "bf16", "learned", 0),
    ("m7_s3_pad_r16", 1, 10, 9, 7, 3, 2, 32, "bf16", None, 16),
    ("fp32_m5_pad", 1, 12, 7, 5, 2, 2, 32, "fp32", "learned", 0),
    ("fp32_m8_d16", 1, 16, 16, 8, 4, 2, 16, "fp32", "learned", 0),
    ("fp32_m12_d64_r16", 1, 24, 24, 12, 6, 1, 64, "fp32", "learned", 16),
    ("fp32_m4_d32_r32", 2, 8, 8, 4, 2, 2, 32, "fp32", None, 32),
]


@pytest.mark.parametrize("case", SMALL, ids=[c[0] for c in SMALL])
def test_small_full(case):
    name, B, H, W, M, s, heads, d, dt, rope, r = case
    w = I.Workload(name, B, H, W, M, (s,), heads, d, dt, rope, r)
    G.full_compare(w, s)


def test_tiny_fp32_full():
    w = I.WORKLOADS["tiny"]
    G.full_compare(w, w.shifts[0])


def test_swin_full():
    """Swin-T stage-1 shape, whole output (9408 windows-heads)."""
    w = I.WORKLOADS["swin"]
    G.full_compare(w, w.shifts[0])


@pytest.mark.parametrize("shift", [0, 16])
def test_dense_sampled(shift):
    w = I.WORKLOADS["dense"]
    G.sampled_compare(w, shift, images=[0, w.B - 1], extra_windows=3)


def test_sr_rib_sampled():
    w = I.WORKLOADS["sr"]
    G.sampled_compare(w, 0, images=[w.B - 1], heads=[0, 5], extra_windows=0, max_units=6)


@pytest.mark.parametrize("name", ["flashswin_M16", "flashswin_M32"])
def test_flashswin_padded_sampled(name):
    """FlashSwin-T's 56 x 56 map at M = 16 and 32 (padded to 64 x 64), full
    size, sampled windows: every corner and seam window, which hold the pad
    positions."""
    w = I.WORKLOADS[name]
    G.sampled_compare(w, w.shifts[0], images=[0, w.B - 1], extra_windows=2, max_units=12)


SWEEP = [n for n in I.WORKLOADS if n.startswith("sweep_")]


@pytest.mark.parametrize("name", SWEEP)
def test_sweep_sampled(name):
    w = I.WORKLOADS[name]
    units = 16 if w.M <= 32 else 4
    G.sampled_compare(w, w.shifts[0], images=[w.B - 1], heads=[0, w.heads - 1], extra_windows=1,
                      max_units=units)


def test_largest_window_properties():
    """M = 256 (65536-token windows, too large for the oracle): properties that
    hold at any size.  Constant V gives that constant; Q = 0 without bias gives
    the plain mean of V over the allowed set (here the whole window, no shift)."""
    torch.manual_seed(0)
    B, H, W, heads, d, M = 1, 256, 256, 1, 32, 256
    k = torch.randn(B, H, W, heads, d, device="cuda").to(torch.bfloat16)
    q = torch.randn_like(k)
    c = torch.linspace(-1, 1, d, device="cuda").to(torch.bfloat16)
    v = c.expand(B, H, W, heads, d).contiguous()
    theta = I.make_theta(heads, d, "learned", 1).cuda()
    out = G.run_gpu(q, k, v, M, 0, theta)
    np.testing.assert_allclose(G.as_f64(out), np.broadcast_to(G.as_f64(c), out.shape), atol=2e-2)
    v = torch.randn_like(k)
    out = G.run_gpu(torch.zeros_like(q), k, v, M, 0, theta)
    mean = v.double().mean(dim=(1, 2), keepdim=True)
    G.check(G.as_f64(out), np.broadcast_to(mean.cpu().numpy(), out.shape), "bf16", "zero-Q mean, M=256")


def test_host_path_matches_device_path():
    w = I.Workload("host", 2, 16, 16, 8, (4,), 2, 32, "bf16", "learned")
    (qkv,), theta, _ = I.make_inputs(w)
    dev = [t.cuda() for t in qkv]
    ref = G.run_gpu(*dev, w.M, 4, theta.cuda())
    pinned = [t.pin_memory() for t in qkv]
    out = wa.window_attention_host(*pinned, w.M, 4, theta=theta.cuda())
    assert torch.equal(out, ref.cpu())


def test_host_path_chunks_odd_windows_per_image():
    """The host-buffer path cuts the batch into chunks of whole images; with
    49 windows per image (Swin's map) the window pairs of a chunk differ from
    those of the whole batch, and the result still matches the oracle."""
    w = I.WORKLOADS["swin"]
    (qkv,), theta, _ = I.make_inputs(w)
    pinned = [t.pin_memory() for t in qkv]
    out = wa.window_attention_host(*pinned, w.M, 4, theta=theta.cuda())
    ref = G.orc().fwd(*(I.to_storage_numpy(t) for t in qkv), M=w.M, shift=4, theta=theta.numpy())
    G.check(G.as_f64(out), ref, "bf16", "host path, swin")


def test_deterministic():
    w = I.WORKLOADS["swin"]
    (qkv,), theta, _ = I.make_inputs(w, "cuda")
    a = G.run_gpu(*qkv, w.M, 4, theta)
    b = G.run_gpu(*qkv, w.M, 4, theta)
    assert torch.equal(a, b)


def test_errors_leave_out_untouched():
    q = torch.randn(1, 16, 16, 2, 32, device="cuda").to(torch.bfloat16)
    out = torch.full_like(q, 7.0)
    with pytest.raises(wa.WinattnError) as e:
        wa.window_attention(q, q, q, 8, shift=8, out=out)   # shift must be < M
    assert e.value.code == -1
    with pytest.raises(wa.WinattnError) as e:
        wa.window_attention(q, q, q, 8, out=q)              # out aliases q
    assert e.value.code == -8
    torch.cuda.synchronize()
    assert bool((out == 7.0).all())
    assert wa.device_status() == 0


FALLBACKS = [
    # switched off, workload, shift, kernel that serves it then
    ((_lib.KERNEL_LARGE,), "dense", 16, _lib.KERNEL_GENERIC),
    ((_lib.KERNEL_PIPE,), "swin", 4, _lib.KERNEL_SMALL),
    ((_lib.KERNEL_PIPE, _lib.KERNEL_SMALL), "swin", 4, _lib.KERNEL_GENERIC),
    ((_lib.KERNEL_PIPE16,), "sweep_M16_d32_s8", 8, _lib.KERNEL_LARGE),
    ((_lib.KERNEL_PIPE16,), "sweep_M16_d64_s8", 0, _lib.KERNEL_LARGE),
    ((_lib.KERNEL_PIPE16,), "flashswin_M16", 8, _lib.KERNEL_LARGE),
]


@pytest.mark.parametrize("off,name,shift,serves", FALLBACKS, ids=["large-off", "pipe-off", "pipe-small-off", "pipe16-off-s8", "pipe16-off-d64-s0",
                              "pipe16-off-flashswin"])
def test_fallback_kernels(off, name, shift, serves):
    """With specialised kernels switched off, their problems run on the next
    kernel that serves them (the path a build with an unexpected register
    count takes for the large-window kernel) and still match the oracle."""
    w = I.WORKLOADS[name]
    try:
        for k in off:
            assert _lib.set_kernel_enabled(k, False) == 1
        rc, info = _lib.launch_info(w.B, w.H, w.W, w.M, shift, w.heads, w.d, w.rank, _lib.BF16)
        assert rc == 0 and info["kernel"] == serves
        if w.name == "dense":
            G.sampled_compare(w, shift, images=[0, w.B - 1], extra_windows=2)
        elif w.name.startswith("flashswin"):
            G.sampled_compare(w, shift, images=[0, w.B - 1], extra_windows=2, max_units=12)
        elif w.name.startswith("sweep_"):
            G.sampled_compare(w, shift, images=[w.B - 1], heads=[0, w.heads - 1], extra_windows=1, max_units=16)
        else:
            G.full_compare(w, shift)
    finally:
        for k in off:
            _lib.set_kernel_enabled(k, True)


LSE_CASES = [
    # name, B, H, W, M, shift, heads, d, dtype, rope, rank   (kernel that serves it)
    ("swin", 64, 56, 56, 8, 4, 3, 32, "bf16", "learned", 0),            # pipelined 8 x 8
    ("m8_s0_d64_lse", 2, 16, 24, 8, 0, 2, 64, "bf16", "standard", 0),   # pipelined, d = 64
    ("m4_s2_lse", 2, 8, 12, 4, 2, 2, 32, "bf16", "learned", 0),         # generic (small kernel has no lse)
    ("m12_s6_r16_lse", 1, 24, 24, 12, 6, 2, 32, "bf16", "learned", 16), # generic, ragged tiles, factors
    ("m16_s8_lse", 2, 32, 48, 16, 8, 2, 32, "bf16", "learned", 0),     # pipelined 16 x 16
    ("m16_s8_pad_d64_lse", 1, 56, 40, 16, 8, 2, 64, "bf16", "learned", 0),  # 16 x 16, half-window pads
    ("m32_s16_lse", 2, 64, 64, 32, 16, 2, 32, "bf16", "learned", 0),    # large-window
    ("m16_s0_d64_r16_lse", 1, 32, 48, 16, 0, 2, 64, "bf16", "learned", 16),
    ("m32_s16_pad56_lse", 1, 56, 56, 32, 16, 2, 32, "bf16", "learned", 0),  # large-window, padded
    ("fp32_lse", 1, 16, 16, 8, 4, 2, 32, "fp32", "learned", 0),         # fp32
]


@pytest.mark.parametrize("case", LSE_CASES, ids=[c[0] for c in LSE_CASES])
def test_forward_saves_lse(case):
    name, B, H, W, M, s, heads, d, dt, rope, r = case
    w = I.Workload(name, B, H, W, M, (s,), heads, d, dt, rope, r)
    G.lse_compare(w, s)
