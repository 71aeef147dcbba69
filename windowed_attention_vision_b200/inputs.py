"""Seeded synthetic inputs and the named workloads.

This module only draws and shapes input data; it holds none of the attention
arithmetic.  Both the oracle tests and the CUDA path take their inputs from
here.

Workload shapes follow the pages' settings (no dataset is used; only shapes):
  - "FLASHSWIN: Unlocking Large Windows and Dense Tokens in Swin Vision
    Transformers with Memory Efficient Attention", section "무엇과 다른가":
    224 px at patch 4 (56 x 56 tokens) and patch 2 (dense grid), windows
    M = 8 ... 32; section "어떻게 동작하나": RoPE frequencies initialised from
    the standard geometric schedule, theta_i = exp(omega_i).
  - "Rank-Factorized Implicit Neural Bias: Scaling Super-Resolution
    Transformer with FlashAttention", sections 2.1 (Fourier features of 2D
    coordinates through a light MLP give the low-rank position factors) and 3
    (windows up to 96 x 96).

Every tensor is drawn from its own ``torch.Generator`` seeded with
``base + crc32("<workload>:<tensor>")``.
"""
from __future__ import annotations

import dataclasses
import math
import zlib
from typing import Optional

import numpy as np
import torch


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    B: int
    H: int
    W: int
    M: int
    shifts: tuple          # one call per entry; several entries alternate per step
    heads: int
    d: int
    dtype: str             # "bf16" or "fp32"
    rope: Optional[str]    # None, "standard" or "learned" (omega + N(0, 0.1))
    rank: int = 0          # rank-r bias features appended to Q/K (0 = none)

    @property
    def tokens(self) -> int:
        return self.B * self.H * self.W

    @property
    def N(self) -> int:
        return self.M * self.M

    @property
    def elt(self) -> int:
        return 2 if self.dtype == "bf16" else 4

    def flops(self) -> float:
        """Algorithmic FLOPs of one call: QK^T over d (+ rank) and PV over d,
        every pair of each window counted (masked pairs included; on a padded
        grid, the pairs of real query tokens with every position of their
        window, as the method computes whole windows)."""
        per_pair = 2 * (self.d + self.rank) + 2 * self.d
        return float(self.tokens) * self.heads * self.N * per_pair

    def bytes(self) -> float:
        """Algorithmic HBM bytes of one call: Q, K, V read once, O written once,
        plus the bias-feature table when present."""
        b = 4.0 * self.tokens * self.heads * self.d * self.elt
        if self.rank:
            b += self.heads * 2 * self.N * self.rank * self.elt
        return b


def _sweep(M: int, d: int, shift: int) -> Workload:
    if M == 96:
        B, side = 114, 192      # 2^22 is not a multiple of 96^2; 114 * 192^2 = 2^22 + 8192
    else:
        B, side = 64, 256       # 64 * 256^2 = 2^22
    return Workload(f"sweep_M{M}_d{d}_s{shift}", B, side, side, M, (shift,), 4, d, "bf16", "standard")


WORKLOADS = {
    "tiny": Workload("tiny", 1, 16, 16, 8, (0,), 2, 32, "fp32", "standard"),
    "swin": Workload("swin", 64, 56, 56, 8, (4,), 3, 32, "bf16", "learned"),
    "dense": Workload("dense", 16, 128, 128, 32, (0, 16), 3, 32, "bf16", "standard"),
    "sr": Workload("sr", 4, 192, 192, 96, (0,), 6, 32, "bf16", None, rank=16),
    # FlashSwin-T's stage 1 with its larger windows (FLASHSWIN page, section
    # "무엇과 다른가": M = 16 and 32 at patch 4 on the 56 x 56 map, which is
    # not a multiple of either, so the grid is padded to 64 x 64)
    "flashswin_M16": Workload("flashswin_M16", 64, 56, 56, 16, (8,), 3, 32, "bf16", "learned"),
    "flashswin_M32": Workload("flashswin_M32", 64, 56, 56, 32, (16,), 3, 32, "bf16", "learned"),
}
for _M in (8, 16, 32, 64, 96):
    for _d in (32, 64):
        for _s in (0, _M // 2):
            _w = _sweep(_M, _d, _s)
            WORKLOADS[_w.name] = _w


def seed_for(workload: str, tensor: str, base: int = 0) -> int:
    return base + zlib.crc32(f"{workload}:{tensor}".encode())


def _gen(seed: int, device) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    return g


def torch_dtype(name: str):
    return {"bf16": torch.bfloat16, "fp32": torch.float32}[name]


def make_map(shape, dtype: str, seed: int, device="cpu") -> torch.Tensor:
    """N(0, 1) drawn in fp32, then cast to the storage dtype."""
    x = torch.randn(shape, generator=_gen(seed, device), device=device, dtype=torch.float32)
    return x.to(torch_dtype(dtype))


def make_theta(heads: int, d: int, mode: Optional[str], seed: int) -> Optional[torch.Tensor]:
    """Per-head frequencies theta_k = exp(omega_k), k < d/4, fp32 [heads, d/4].

    omega_k = log(10000^(-2k/(d/2))), the standard geometric schedule; "learned"
    adds N(0, 0.1) to every omega, standing in for trained values."""
    if mode is None:
        return None
    k = torch.arange(d // 4, dtype=torch.float64)
    omega = (-2.0 * k / (d / 2)) * math.log(10000.0)
    omega = omega.expand(heads, d // 4).clone()
    if mode == "learned":
        omega += 0.1 * torch.randn((heads, d // 4), generator=_gen(seed, "cpu"), dtype=torch.float64)
    elif mode != "standard":
        raise ValueError(f"unknown rope mode {mode!r}")
    return torch.exp(omega).to(torch.float32)


def make_bias_feats(heads: int, M: int, rank: int, dtype: str, seed: int) -> torch.Tensor:
    """Rank-r position factors u(p), w(p) for window-local p = i*M + j:
    [heads, 2, M*M, rank] (index 0 = u for queries, 1 = w for keys).

    Each is tanh(F(p) W1) W2 with F(p) = sin/cos of the normalised window
    coordinates c = 2*i/(M-1) - 1 at 8 octave frequencies 2^k * pi (32
    features), W1: 32 x 64 ~ N(0, 1/32), W2: 64 x rank ~ N(0, 1/64), drawn
    separately per head and per side."""
    g = _gen(seed, "cpu")
    idx = torch.arange(M, dtype=torch.float64)
    c = 2.0 * idx / (M - 1) - 1.0 if M > 1 else torch.zeros(1, dtype=torch.float64)
    cy = c.repeat_interleave(M)       # row coordinate of p = i*M + j
    cx = c.repeat(M)                  # column coordinate
    freqs = (2.0 ** torch.arange(8, dtype=torch.float64)) * math.pi
    F = torch.cat([torch.sin(cy[:, None] * freqs), torch.cos(cy[:, None] * freqs),
                   torch.sin(cx[:, None] * freqs), torch.cos(cx[:, None] * freqs)], dim=1)
    out = torch.empty((heads, 2, M * M, rank), dtype=torch.float64)
    for h in range(heads):
        for side in range(2):
            W1 = torch.randn((32, 64), generator=g, dtype=torch.float64) / math.sqrt(32)
            W2 = torch.randn((64, rank), generator=g, dtype=torch.float64) / math.sqrt(64)
            out[h, side] = torch.tanh(F @ W1) @ W2
    return out.to(torch_dtype(dtype))


def make_inputs(w: Workload, device="cpu", base: int = 0, copies: int = 1):
    """q, k, v ([B, H, W, heads, d]), theta ([heads, d/4] fp32 or None) and
    bias ([heads, 2, M*M, rank] or None).  ``copies`` > 1 returns that many
    independent (q, k, v) sets (differently seeded) for L2 rotation."""
    shape = (w.B, w.H, w.W, w.heads, w.d)
    sets = []
    for c in range(copies):
        tag = w.name if c == 0 else f"{w.name}#{c}"
        sets.append(tuple(make_map(shape, w.dtype, seed_for(tag, t, base), device) for t in "qkv"))
    theta = make_theta(w.heads, w.d, w.rope, seed_for(w.name, "omega", base))
    bias = None
    if w.rank:
        bias = make_bias_feats(w.heads, w.M, w.rank, w.dtype, seed_for(w.name, "rib", base))
    if theta is not None:
        theta = theta.to(device)
    if bias is not None:
        bias = bias.to(device)
    return sets, theta, bias


def to_storage_numpy(t: Optional[torch.Tensor]):
    """A torch tensor in the numpy storage form the oracle reads:
    bf16 -> uint16 bits, fp32 -> float32."""
    if t is None:
        return None
    t = t.detach().to("cpu").contiguous()
    if t.dtype == torch.bfloat16:
        return t.view(torch.int16).numpy().view(np.uint16)
    if t.dtype == torch.float32:
        return t.numpy()
    raise TypeError(f"unsupported dtype {t.dtype}")
