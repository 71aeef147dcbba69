"""The large-window kernel's lazy rescale: the running row max moves (and O is
rescaled in TMEM) only when a key tile's max exceeds it by more than 2^8.
Inputs drawn N(0, 1) never get there, so these cases build rows whose scores
grow by far more than that from the first key tiles to the later ones: keys
of the first window rows shrunk, later ones enlarged (by powers of two, so
the bf16 values stay exact), no RoPE (the stored values enter the MMA
unrounded), and the oracle compared element by element."""
import numpy as np
import pytest
import torch

from windowed_attention_vision_b200 import inputs as I
from tests import gpu_helpers as G

pytestmark = pytest.mark.gpu

CASES = [
    # name, B, H, W, M, shift, heads, d
    ("m32_s0", 1, 64, 64, 32, 0, 2, 32),
    ("m16_s8", 2, 32, 32, 16, 8, 2, 32),
    ("m32_s16_d64", 1, 64, 64, 32, 16, 2, 64),
]


def grown_scores(B, H, W, M, s, heads, d, seed):
    g = torch.Generator().manual_seed(seed)
    q, k, v = (torch.randn(B, H, W, heads, d, generator=g) for _ in range(3))
    # keys of every window's first key tile (its first 128 / M rows, in the
    # rolled frame, where rolled row yr holds original row yr + s) shrunk,
    # the others enlarged
    row_in_window = (((torch.arange(H) - s) % H) % M).view(1, H, 1, 1, 1)
    kscale = torch.where(row_in_window < 128 // M, torch.tensor(0.25), torch.tensor(4.0))
    return [t.to(torch.bfloat16) for t in (q * 2.0, k * kscale, v)]


def max_growth_log2(q, k, M, s, d, first_keys):
    """Per query row of the first window (head 0): how far, in log2 units, the
    row's max over all keys exceeds its max over the first key tile."""
    qw, kw = (torch.roll(t.double(), shifts=(-s, -s), dims=(1, 2))[0, :M, :M, 0].reshape(M * M, d) for t in (q, k))
    sc = qw @ kw.T / d ** 0.5
    return (sc.max(dim=1).values - sc[:, :first_keys].max(dim=1).values) * np.log2(np.e)


@pytest.mark.parametrize("case", CASES, ids=[c[0] for c in CASES])
def test_lazy_rescale_against_oracle(case):
    name, B, H, W, M, s, heads, d = case
    q, k, v = grown_scores(B, H, W, M, s, heads, d, seed=len(name))
    # precondition: most rows' maxima grow past the 2^8 threshold after the
    # first key tile (128 keys), so the rescale path runs
    growth = max_growth_log2(q, k, M, s, d, first_keys=128)
    assert float((growth > 8.0).double().mean()) > 0.5
    out = G.run_gpu(q.cuda(), k.cuda(), v.cuda(), M, s)
    ref = G.orc().fwd(*(I.to_storage_numpy(t) for t in (q, k, v)), M=M, shift=s)
    G.check(G.as_f64(out), ref, "bf16", f"rescale {name}")
