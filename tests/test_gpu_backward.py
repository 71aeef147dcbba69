"""GPU parity of the backward pass (winattn_bwd) against the fp64 backward
oracle (itself pinned by central finite differences of the pinned forward,
tests/test_oracle_bwd.py), on the same seeded inputs, element by element over
whole maps.

Tolerances (relative L2 error over each gradient, and max-abs relative to the
gradient's largest magnitude).  The forward's bound for O (rel-L2 <= 5e-3)
comes from bf16 rounding of the rotated q, k (scores off by up to about
2^-8 |q||k| d^-1/2) and of P.  dv = P^T dO has the same structure, plus the
saved log-sum-exp (fp32, from the same bf16 scores): rel-L2 <= 1e-2.  dq, dk,
the theta and bias-table gradients go through dS = P o (dP - dO.O), a
difference of nearly equal terms for the rows that P concentrates on, rounded
to bf16 once more before the last contraction: rel-L2 <= 2e-2.  Max-abs of
every gradient <= 0.1 of its largest magnitude."""
import numpy as np
import pytest
import torch

import windowed_attention_vision_b200 as wa
from windowed_attention_vision_b200 import _lib
from windowed_attention_vision_b200 import inputs as I
from tests import gpu_helpers as G

pytestmark = pytest.mark.gpu

BWD_TOL = {"dq": 2e-2, "dk": 2e-2, "dv": 1e-2, "dtheta": 2e-2, "dbias": 2e-2}
MAX_ABS_FRAC = 0.1

CASES = [
    # name, B, H, W, M, shift, heads, d, rope, rank
    ("swin", 64, 56, 56, 8, 4, 3, 32, "learned", 0),          # two 8 x 8 windows per tile (Swin-T stage 1)
    ("m8_s0_d64", 2, 16, 24, 8, 0, 2, 64, "standard", 0),
    ("m8_s4_nope", 2, 16, 16, 8, 4, 2, 32, None, 0),
    ("m4_s2", 2, 8, 12, 4, 2, 2, 32, "learned", 0),            # eight windows per tile
    ("m10_s5", 1, 20, 20, 10, 5, 2, 32, "learned", 0),         # one ragged tile per window
    ("m12_s6_r16", 1, 24, 24, 12, 6, 2, 32, "learned", 16),    # two tiles, ragged; bias factors
    ("m16_s8_d64", 1, 32, 32, 16, 8, 2, 64, "learned", 0),
    ("m32_s16", 2, 64, 64, 32, 16, 2, 32, "learned", 0),       # eight key tiles per window
    ("m32_s0_d64_r32", 1, 64, 64, 32, 0, 1, 64, "learned", 32),
    ("m16_s0_r16_nope", 1, 32, 48, 16, 0, 2, 32, None, 16),
    ("m32_s16_pad56", 1, 56, 56, 32, 16, 2, 32, "learned", 0),  # padded grid
    ("m8_s4_pad20", 1, 20, 20, 8, 4, 2, 32, "learned", 0),
]


def rel_check(got, ref, tol, what):
    got = np.asarray(got, dtype=np.float64)
    assert np.all(np.isfinite(got)), f"{what}: non-finite values"
    diff = got - ref
    rel = float(np.linalg.norm(diff) / max(np.linalg.norm(ref), 1e-300))
    mx = float(np.max(np.abs(diff)) / max(np.max(np.abs(ref)), 1e-300))
    assert rel <= tol, f"{what}: rel-L2 {rel:.3e} > {tol:.0e}"
    assert mx <= MAX_ABS_FRAC, f"{what}: max-abs {mx:.3e} of the largest magnitude"
    return rel


def run_case(w, shift, base=0):
    (qkv,), theta, bias = I.make_inputs(w, "cpu", base)
    dout = I.make_map(qkv[0].shape, "bf16", I.seed_for(w.name, "dout", base))
    q, k, v, do = (t.cuda() for t in (*qkv, dout))
    th = None if theta is None else theta.cuda()
    bs = None if bias is None else bias.cuda()
    lse = torch.empty((w.B, w.H, w.W, w.heads), dtype=torch.float32, device="cuda")
    out = wa.window_attention(q, k, v, w.M, shift, theta=th, bias_feats=bs, lse=lse)
    dq, dk, dv, dth, dbi = wa.window_attention_backward(q, k, v, out, do, lse, w.M, shift, theta=th,
                                                        bias_feats=bs)
    torch.cuda.synchronize()
    assert wa.device_status() == 0, "a bounded wait timed out"
    ref = G.orc().bwd(*(I.to_storage_numpy(t) for t in qkv), G.as_f64(dout), M=w.M, shift=shift,
                      theta=None if theta is None else theta.numpy(), bias=I.to_storage_numpy(bias))
    got = {"dq": dq, "dk": dk, "dv": dv, "dtheta": dth, "dbias": dbi}
    errs = {}
    for name, r in zip(("dq", "dk", "dv", "dtheta", "dbias"), ref):
        if r is None:
            assert got[name] is None
            continue
        errs[name] = rel_check(G.as_f64(got[name]), r, BWD_TOL[name], f"{w.name} {name}")
    return errs


@pytest.mark.parametrize("case", CASES, ids=[c[0] for c in CASES])
def test_backward_matches_oracle(case):
    name, B, H, W, M, s, heads, d, rope, r = case
    w = I.Workload(name, B, H, W, M, (s,), heads, d, "bf16", rope, r)
    run_case(w, s)


def test_backward_single_tile_is_deterministic():
    """Windows of at most 128 tokens write dq, dk, dv directly: two runs give
    the same bits."""
    w = I.Workload("det", 4, 16, 16, 8, (4,), 2, 32, "bf16", "learned")
    (qkv,), theta, _ = I.make_inputs(w, "cuda")
    do = I.make_map(qkv[0].shape, "bf16", 5, "cuda")
    lse = torch.empty((w.B, w.H, w.W, w.heads), dtype=torch.float32, device="cuda")
    out = wa.window_attention(*qkv, w.M, 4, theta=theta, lse=lse)
    a = wa.window_attention_backward(*qkv, out, do, lse, w.M, 4, theta=theta)
    b = wa.window_attention_backward(*qkv, out, do, lse, w.M, 4, theta=theta)
    for x, y in zip(a[:3], b[:3]):
        assert torch.equal(x, y)


def test_backward_rejects_bad_arguments():
    q = torch.randn(1, 16, 16, 2, 32, device="cuda").to(torch.bfloat16)
    lse = torch.zeros(1, 16, 16, 2, device="cuda")
    f = torch.randn(1, 16, 16, 2, 32, device="cuda")
    stream = torch.cuda.current_stream().cuda_stream
    p = q.data_ptr()
    # fp32 storage has no backward
    rc = _lib.bwd(f.data_ptr(), f.data_ptr(), f.data_ptr(), None, None, f.data_ptr(), f.data_ptr(), lse.data_ptr(),
                  1, 16, 16, 8, 4, 2, 32, 0, _lib.FP32, f.data_ptr(), f.data_ptr(), f.data_ptr(), None, None, None, 0,
                  stream)
    assert rc == _lib.ERR_DTYPE
    # gradients may not overlap the inputs
    dq = torch.empty_like(q)
    rc = _lib.bwd(p, p, p, None, None, p, p, lse.data_ptr(), 1, 16, 16, 8, 4, 2, 32, 0, _lib.BF16, dq.data_ptr(),
                  p, dq.data_ptr() + 0, None, None, None, 0, stream)
    assert rc == _lib.ERR_ALIAS
    # a window of more than 128 tokens needs the workspace
    big = torch.randn(1, 32, 32, 2, 32, device="cuda").to(torch.bfloat16)
    lb = torch.zeros(1, 32, 32, 2, device="cuda")
    g3 = [torch.empty_like(big) for _ in range(3)]
    bp = big.data_ptr()
    assert _lib.bwd_workspace_bytes(1, 32, 32, 16, 2, 32) > 0
    rc = _lib.bwd(bp, bp, bp, None, None, bp, bp, lb.data_ptr(), 1, 32, 32, 16, 8, 2, 32, 0, _lib.BF16,
                  *(t.data_ptr() for t in g3), None, None, None, 0, stream)
    assert rc == _lib.ERR_SIZE
