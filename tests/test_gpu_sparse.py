"""GPU parity of the gated-window residual (winattn_fwd_sparse) against the
fp64 oracle (oracle_fwd_sparse, pinned by an independent global formulation):
the tokens of the listed windows match within the forward's bf16 tolerance,
every other token keeps O_lin bit for bit.  Lists hold about 30% of the
windows, the share of blocks the HSMLA page's gate routes to the softmax
path (section 2, Hierarchical Block-Level Gating)."""
import numpy as np
import pytest
import torch

import windowed_attention_vision_b200 as wa
from windowed_attention_vision_b200 import _lib
from windowed_attention_vision_b200 import inputs as I
from tests import gpu_helpers as G

pytestmark = pytest.mark.gpu

CASES = [
    # name, B, H, W, M, shift, heads, d, rope, rank
    ("m8_s4", 4, 16, 24, 8, 4, 3, 32, "learned", 0),          # packed windows: list packs of two
    ("m8_s0_d64", 2, 16, 24, 8, 0, 2, 64, "standard", 0),
    ("m7_s3_r16", 2, 14, 21, 7, 3, 2, 32, "learned", 16),      # 49-token windows, bias factors
    ("m12_s6", 2, 24, 36, 12, 6, 2, 32, "learned", 0),         # two ragged query tiles per window
    ("m32_s16", 2, 64, 96, 32, 16, 2, 32, "learned", 0),
    ("m32_s16_pad56", 1, 56, 56, 32, 16, 2, 32, "learned", 0),  # padded grid
]


def gated_list(n_windows, frac, seed):
    rng = np.random.default_rng(seed)
    n = max(1, int(round(frac * n_windows)))
    return np.sort(rng.choice(n_windows, n, replace=False)).astype(np.int32)


def run_case(w, shift, frac=0.3, seed=0):
    (qkv,), theta, bias = I.make_inputs(w, "cpu")
    o_lin = I.make_map(qkv[0].shape, "bf16", I.seed_for(w.name, "o_lin"))
    nwin = w.B * (-(-w.H // w.M)) * (-(-w.W // w.M))
    wins = gated_list(nwin, frac, seed)
    q, k, v = (t.cuda() for t in qkv)
    out = o_lin.cuda().clone()
    wa.window_attention_gated_residual(q, k, v, out, torch.from_numpy(wins).cuda(), w.M, shift,
                                       theta=None if theta is None else theta.cuda(),
                                       bias_feats=None if bias is None else bias.cuda())
    torch.cuda.synchronize()
    assert wa.device_status() == 0
    ref = G.orc().fwd_sparse(*(I.to_storage_numpy(t) for t in qkv), G.as_f64(o_lin), wins, M=w.M, shift=shift,
                             theta=None if theta is None else theta.numpy(), bias=I.to_storage_numpy(bias))
    got = G.as_f64(out)
    base = G.as_f64(o_lin)
    touched = ref != base
    assert np.array_equal(got[~touched], base[~touched]), "tokens outside the listed windows changed"
    G.check(got[touched], ref[touched], "bf16", f"{w.name} gated windows")


@pytest.mark.parametrize("case", CASES, ids=[c[0] for c in CASES])
def test_gated_residual_matches_oracle(case):
    name, B, H, W, M, s, heads, d, rope, r = case
    w = I.Workload(name, B, H, W, M, (s,), heads, d, "bf16", rope, r)
    run_case(w, s)


def test_all_windows_listed():
    w = I.Workload("all", 2, 16, 16, 8, (4,), 2, 32, "bf16", "learned")
    run_case(w, 4, frac=1.0)


def test_empty_list_touches_nothing():
    q = torch.randn(1, 16, 16, 2, 32, device="cuda").to(torch.bfloat16)
    out = torch.randn_like(q)
    before = out.clone()
    wa.window_attention_gated_residual(q, q, q, out, torch.zeros(0, dtype=torch.int32, device="cuda"), 8, 4)
    torch.cuda.synchronize()
    assert torch.equal(out, before)
    # fp32 storage has no gated path; too many ids cannot all be distinct
    f = torch.randn(1, 16, 16, 2, 32, device="cuda")
    ids = torch.arange(5, dtype=torch.int32, device="cuda")
    s = torch.cuda.current_stream().cuda_stream
    assert _lib.fwd_sparse(f.data_ptr(), f.data_ptr(), f.data_ptr(), None, None, 1, 16, 16, 8, 4, 2, 32, 0,
                           _lib.FP32, ids.data_ptr(), 4, torch.empty_like(f).data_ptr(), s) == _lib.ERR_DTYPE
    assert _lib.fwd_sparse(q.data_ptr(), q.data_ptr(), q.data_ptr(), None, None, 1, 16, 16, 8, 4, 2, 32, 0,
                           _lib.BF16, ids.data_ptr(), 5, out.data_ptr(), s) == _lib.ERR_ARG
