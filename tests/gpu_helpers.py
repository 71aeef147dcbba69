"""Shared helpers of the GPU parity tests: run the CUDA path, run the oracle on
the same inputs (whole map or sampled windows), compare with the stated
tolerances."""
from __future__ import annotations

import numpy as np
import torch

import oracle
import windowed_attention_vision_b200 as wa
from windowed_attention_vision_b200 import inputs as I

# Tolerances of the forward pass: fp32 storage -> rel-L2 <= 1e-5; bf16 storage
# -> max-abs <= 2e-2 and rel-L2 <= 5e-3 (bf16 rounding of the rotated Q/K and
# of P, fp32 accumulation).
TOL = {"fp32": dict(rel_l2=1e-5, max_abs=None), "bf16": dict(rel_l2=5e-3, max_abs=2e-2)}

_ORC = None


def orc():
    global _ORC
    if _ORC is None:
        _ORC = oracle.oracle()
    return _ORC


def as_f64(t: torch.Tensor) -> np.ndarray:
    return t.detach().float().cpu().numpy().astype(np.float64)


def check(got: np.ndarray, ref: np.ndarray, dtype: str, what: str = ""):
    assert np.all(np.isfinite(got)), f"{what}: non-finite output"
    diff = got - ref
    rel_l2 = float(np.linalg.norm(diff) / max(np.linalg.norm(ref), 1e-300))
    max_abs = float(np.max(np.abs(diff))) if diff.size else 0.0
    tol = TOL[dtype]
    assert rel_l2 <= tol["rel_l2"], f"{what}: rel-L2 {rel_l2:.3e} > {tol['rel_l2']:.0e} (max-abs {max_abs:.3e})"
    if tol["max_abs"] is not None:
        assert max_abs <= tol["max_abs"], f"{what}: max-abs {max_abs:.3e} > {tol['max_abs']:.0e}"
    return rel_l2, max_abs


def run_gpu(q, k, v, M, shift, theta=None, bias=None):
    out = wa.window_attention(q, k, v, M, shift, theta=theta, bias_feats=bias)
    torch.cuda.synchronize()
    assert wa.device_status() == 0, "a bounded wait timed out"
    return out


def full_compare(w: I.Workload, shift: int, device="cuda", base: int = 0):
    """Whole-map parity on a workload small enough for the oracle."""
    (qkv,), theta, bias = I.make_inputs(w, "cpu", base)
    dq, dk, dv = (t.to(device) for t in qkv)
    out = run_gpu(dq, dk, dv, w.M, shift, None if theta is None else theta.to(device),
                  None if bias is None else bias.to(device))
    ref = orc().fwd(*(I.to_storage_numpy(t) for t in qkv), M=w.M, shift=shift,
                    theta=None if theta is None else theta.numpy(), bias=I.to_storage_numpy(bias))
    return check(as_f64(out), ref, w.dtype, f"{w.name} s{shift}")


def window_positions(H, W, M, shift, wy, wx):
    """Original (y, x) of the window's tokens in window order, on the grid
    padded to multiples of M, and which of them are real (not padding)."""
    Hp, Wp = -(-H // M) * M, -(-W // M) * M
    p = np.arange(M * M)
    y = (wy * M + p // M + shift) % Hp
    x = (wx * M + p % M + shift) % Wp
    return y, x, (y < H) & (x < W)


def sample_windows(nWy, nWx, rng, extra=2):
    """Corner, edge and interior windows: every wrap case when shifted."""
    wins = {(0, 0), (nWy - 1, nWx - 1), (0, nWx - 1), (nWy - 1, 0)}
    for _ in range(extra):
        wins.add((int(rng.integers(nWy)), int(rng.integers(nWx))))
    return sorted(wins)


def sampled_compare(w: I.Workload, shift: int, images, heads=None, extra_windows=2, device="cuda",
                    max_units=None, seed=0):
    """Full-size GPU call; oracle on sampled windows of a few images."""
    (qkv,), theta, bias = I.make_inputs(w, device)
    out = run_gpu(*qkv, w.M, shift, theta, bias)
    assert torch.isfinite(out.float()).all().item(), "non-finite values in the output"
    rng = np.random.default_rng(seed)
    nWy, nWx = -(-w.H // w.M), -(-w.W // w.M)
    heads = list(range(w.heads)) if heads is None else heads
    th = None if theta is None else theta.cpu().numpy()
    bs = I.to_storage_numpy(bias)
    results = []
    for b in images:
        sub = [I.to_storage_numpy(t[b:b + 1]) for t in qkv]
        wins = sample_windows(nWy, nWx, rng, extra_windows)
        units, locs = [], []
        for (wy, wx) in wins:
            for h in heads:
                units.append((wy * nWx + wx) * w.heads + h)
                locs.append((wy, wx, h))
        if max_units is not None:
            # always the four corner windows (every wrap case of a shifted map,
            # heads taken in turn) and an edge window of each seam; then random
            # units up to max_units
            must = {}
            corners = [(0, 0), (0, nWx - 1), (nWy - 1, 0), (nWy - 1, nWx - 1)]
            edges = [(nWy - 1, nWx // 2), (nWy // 2, nWx - 1)]
            for n_, (wy, wx) in enumerate(corners + edges):
                if (wy, wx) in [(a, b) for (a, b, _) in must.values()]:
                    continue
                h = heads[n_ % len(heads)]
                must[(wy * nWx + wx) * w.heads + h] = (wy, wx, h)
            rest = [i for i in rng.permutation(len(units)) if units[i] not in must]
            extra = max(0, max_units - len(must))
            units = list(must) + [units[i] for i in rest[:extra]]
            locs = list(must.values()) + [locs[i] for i in rest[:extra]]
        ref = orc().fwd_units(*sub, units, M=w.M, shift=shift, theta=th, bias=bs)
        got_img = out[b].float().cpu().numpy().astype(np.float64)
        got, keep = [], []
        for (wy, wx, h) in locs:
            y, x, real = window_positions(w.H, w.W, w.M, shift, wy, wx)
            got.append(got_img[y[real], x[real], h])
            keep.append(real)
        # pad positions hold no token: compared rows are the real ones
        got = np.concatenate(got)
        ref = np.concatenate([r[k] for r, k in zip(ref, keep)])
        results.append(check(got, ref, w.dtype, f"{w.name} s{shift} image {b}"))
    return results


# Tolerance of the saved log-sum-exp: it moves by at most the largest error of
# the row's scores (log-sum-exp is 1-Lipschitz in the max norm), and the bf16
# scores carry the rounding of the rotated q and k (2^-9 relative each), at
# most about 2^-8 |q||k| d^-1/2 ~ 2e-2 for N(0, 1) inputs at d = 32.
LSE_TOL = {"fp32": dict(max_abs=1e-4), "bf16": dict(max_abs=3e-2, mean_abs=3e-3)}


def lse_compare(w: I.Workload, shift: int, device="cuda", base: int = 0):
    """Whole-map parity of O and of the saved log-sum-exp (winattn_fwd_lse)."""
    (qkv,), theta, bias = I.make_inputs(w, "cpu", base)
    dq, dk, dv = (t.to(device) for t in qkv)
    lse = torch.full((w.B, w.H, w.W, w.heads), float("nan"), device=device)
    out = wa.window_attention(dq, dk, dv, w.M, shift, theta=None if theta is None else theta.to(device),
                              bias_feats=None if bias is None else bias.to(device), lse=lse)
    torch.cuda.synchronize()
    assert wa.device_status() == 0, "a bounded wait timed out"
    ref, ref_lse = orc().fwd_lse(*(I.to_storage_numpy(t) for t in qkv), M=w.M, shift=shift,
                                 theta=None if theta is None else theta.numpy(), bias=I.to_storage_numpy(bias))
    check(as_f64(out), ref, w.dtype, f"{w.name} s{shift} (with lse)")
    got = lse.double().cpu().numpy()
    assert np.all(np.isfinite(got)), f"{w.name}: lse not written everywhere"
    err = np.abs(got - ref_lse)
    tol = LSE_TOL[w.dtype]
    assert err.max() <= tol["max_abs"], f"{w.name} s{shift}: lse max-abs {err.max():.3e}"
    if "mean_abs" in tol:
        assert err.mean() <= tol["mean_abs"], f"{w.name} s{shift}: lse mean-abs {err.mean():.3e}"
    return float(err.max())
