"""GPU parity of the two pieces around the attention on the RIB page ("Rank-
Factorized Implicit Neural Bias: Scaling Super-Resolution Transformer with
FlashAttention"): the factor table of section 2.1 (winattn_rib_features and
the combined winattn_fwd_rib) and the CLA gate of section 2.2
(winattn_cla_gate), against the fp64 oracle (pinned by closed forms,
symmetries and library routines, tests/pins.py).

Tolerances: the table is stored in bf16 (relative rounding 2^-9) after an
fp32 evaluation: rel-L2 <= 5e-3.  The attention with the generated table and
the gate use the forward's bf16 bound (max-abs <= 2e-2, rel-L2 <= 5e-3): the
gate rounds the depth-wise output and the point-wise weights to bf16 once
each (2^-9 relative) before an fp32 contraction, and the sigmoid's slope is
at most 1/4."""
import math

import numpy as np
import pytest
import torch

import windowed_attention_vision_b200 as wa
from windowed_attention_vision_b200 import inputs as I
from tests import gpu_helpers as G

pytestmark = pytest.mark.gpu


def rib_weights(heads, rank, seed):
    g = torch.Generator().manual_seed(seed)
    w1 = torch.randn((heads, 2, 32, 64), generator=g) / math.sqrt(32)
    w2 = torch.randn((heads, 2, 64, rank), generator=g) / math.sqrt(64)
    return w1.float(), w2.float()


@pytest.mark.parametrize("M,heads,rank", [(1, 2, 16), (2, 1, 16), (7, 2, 32), (16, 3, 16), (96, 6, 16)])
def test_rib_features_match_oracle(M, heads, rank):
    w1, w2 = rib_weights(heads, rank, M)
    got = wa.rib_features(w1.cuda(), w2.cuda(), M)
    torch.cuda.synchronize()
    ref = G.orc().rib_features(w1.numpy(), w2.numpy(), M)
    g = G.as_f64(got)
    rel = np.linalg.norm(g - ref) / np.linalg.norm(ref)
    assert np.all(np.isfinite(g)) and rel <= 5e-3, f"rel-L2 {rel:.3e}"


def _oracle_table_bf16(w1, w2, M):
    """The oracle's fp64 table rounded to the bf16 storage the attention reads."""
    t = torch.from_numpy(G.orc().rib_features(w1.numpy(), w2.numpy(), M))
    return I.to_storage_numpy(t.to(torch.bfloat16))


@pytest.mark.parametrize("case", [(2, 32, 32, 16, 0, 2, 32, 16, "learned"), (1, 24, 24, 12, 6, 2, 64, 32, None),
                                  (2, 16, 16, 8, 0, 3, 32, 16, "learned")], ids=["m16", "m12_s6_r32", "m8"])
def test_fwd_rib_matches_oracle(case):
    B, H, W, M, s, heads, d, rank, rope = case
    w = I.Workload("rib", B, H, W, M, (s,), heads, d, "bf16", rope)
    (qkv,), theta, _ = I.make_inputs(w)
    w1, w2 = rib_weights(heads, rank, 7)
    q, k, v = (t.cuda() for t in qkv)
    out, table = wa.window_attention_rib(q, k, v, M, s, w1.cuda(), w2.cuda(),
                                         theta=None if theta is None else theta.cuda())
    torch.cuda.synchronize()
    assert wa.device_status() == 0
    ref = G.orc().fwd(*(I.to_storage_numpy(t) for t in qkv), M=M, shift=s,
                      theta=None if theta is None else theta.numpy(), bias=_oracle_table_bf16(w1, w2, M))
    G.check(G.as_f64(out), ref, "bf16", "attention with generated RIB features")


def test_fwd_rib_sr_sampled():
    """The SR workload's shape (B4, 192^2, M = 96, 6 heads, d = 32, rank 16)
    with its factors generated on the GPU; sampled corner windows."""
    w = I.WORKLOADS["sr"]
    (qkv,), _, _ = I.make_inputs(w, "cuda")
    w1, w2 = rib_weights(w.heads, w.rank, 11)
    out, _ = wa.window_attention_rib(*qkv, w.M, 0, w1.cuda(), w2.cuda())
    torch.cuda.synchronize()
    table = _oracle_table_bf16(w1, w2, w.M)
    b = w.B - 1
    sub = [I.to_storage_numpy(t[b:b + 1]) for t in qkv]
    nWx = w.W // w.M
    locs = [(0, 0, 0), (1, 1, 5), (0, 1, 2)]
    units = [(wy * nWx + wx) * w.heads + h for (wy, wx, h) in locs]
    ref = G.orc().fwd_units(*sub, units, M=w.M, shift=0, bias=table)
    got_img = G.as_f64(out[b])
    got = np.stack([got_img[G.window_positions(w.H, w.W, w.M, 0, wy, wx)[:2] + (h,)] for (wy, wx, h) in locs])
    G.check(got, ref, "bf16", "SR with generated factors")


def gate_inputs(B, H, W, C, seed):
    g = torch.Generator().manual_seed(seed)
    x = torch.randn((B, H, W, C), generator=g).to(torch.bfloat16)
    o = torch.randn((B, H, W, C), generator=g).to(torch.bfloat16)
    dw = torch.randn((C, 3, 3), generator=g) / 3.0
    dw_b = 0.1 * torch.randn(C, generator=g)
    pw = torch.randn((C, C), generator=g) / math.sqrt(C)
    pw_b = 0.1 * torch.randn(C, generator=g)
    return x, o, dw, dw_b, pw, pw_b


@pytest.mark.parametrize("B,H,W,C", [(2, 16, 16, 96), (1, 56, 56, 96), (1, 32, 32, 192), (2, 7, 9, 32),
                                     (1, 12, 20, 256), (3, 5, 5, 16)])
def test_cla_gate_matches_oracle(B, H, W, C):
    x, o, dw, dw_b, pw, pw_b = gate_inputs(B, H, W, C, C + H)
    out = wa.cla_gate(x.cuda(), o.cuda(), dw.cuda(), dw_b.cuda(), pw.cuda(), pw_b.cuda())
    torch.cuda.synchronize()
    assert wa.device_status() == 0
    ref = G.orc().cla_gate(I.to_storage_numpy(x), I.to_storage_numpy(o), dw.numpy(), dw_b.numpy(), pw.numpy(),
                           pw_b.numpy())
    G.check(G.as_f64(out), ref, "bf16", f"CLA gate {B}x{H}x{W}x{C}")


def test_cla_gate_in_place():
    x, o, dw, dw_b, pw, pw_b = gate_inputs(2, 24, 24, 96, 3)
    od = o.cuda()
    expect = wa.cla_gate(x.cuda(), od, dw.cuda(), dw_b.cuda(), pw.cuda(), pw_b.cuda())
    wa.cla_gate(x.cuda(), od, dw.cuda(), dw_b.cuda(), pw.cuda(), pw_b.cuda(), out=od)
    torch.cuda.synchronize()
    assert torch.equal(od, expect)
