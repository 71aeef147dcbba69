"""Checks that pin the oracle to facts other than itself.

Each ``pin_*`` function takes an ``oracle.Oracle`` and raises AssertionError
when the oracle disagrees with:
  - the mathematics the FlashSwin page fixes (section "어떻게 동작하나"): the
    rotation composes as R(p)^T R(p') = R(p' - p), so scores depend only on
    the displacement; attention is the exact softmax restricted to windows;
  - closed forms (one-token windows, constant V, zero Q, a hand-worked case);
  - a brute-force *global* attention over the whole image written here from
    a different formulation: original (not window-local) coordinates for the
    rotation, done as complex multiplication, and Swin's slice-based region
    labels of the rolled map for the shifted-window mask;
  - the concatenation identity of the RIB page (section 2.1),
    [Qc, Qp][Kc, Kp]^T = Qc Kc^T + Qp Kp^T, by folding the bias factors into
    wider content vectors of a bias-free problem.

The same functions run against deliberately broken builds of the oracle
(``test_oracle_mutants.py``) to show that each planted mistake fails a pin.
"""
from __future__ import annotations

import math

import numpy as np
import torch

from windowed_attention_vision_b200 import inputs as I

TOL = 1e-10


def storage_to_f64(a: np.ndarray) -> np.ndarray:
    if a.dtype == np.uint16:
        return (a.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    return a.astype(np.float64)


def _maps(shape, dtype, tag, seed=0):
    return [I.to_storage_numpy(I.make_map(shape, dtype, I.seed_for(tag, t, seed))) for t in "qkv"]


def swin_region_labels(H, W, M, s):
    """Region ids of the rolled map built the way Swin builds its attention
    mask: per axis the slices [0, -M), [-M, -s), [-s, end)."""
    img = np.zeros((H, W), dtype=np.int64)
    if s == 0:
        return img
    cnt = 0
    for hs in (slice(0, -M), slice(-M, -s), slice(-s, None)):
        for ws in (slice(0, -M), slice(-M, -s), slice(-s, None)):
            img[hs, ws] = cnt
            cnt += 1
    return img


def rotate_complex(x: np.ndarray, ycoord: np.ndarray, xcoord: np.ndarray, theta_h: np.ndarray):
    """2D RoPE as complex multiplication: pair k of the first half is the
    complex number x[2k] + i x[2k+1] multiplied by exp(i y theta_k), pair k of
    the second half likewise with the column x.  x: [T, d]."""
    T, d = x.shape
    half = d // 2
    th = theta_h.astype(np.float64)
    zy = x[:, 0:half:2] + 1j * x[:, 1:half:2]
    zx = x[:, half::2] + 1j * x[:, half + 1::2]
    zy = zy * np.exp(1j * ycoord[:, None] * th[None, :])
    zx = zx * np.exp(1j * xcoord[:, None] * th[None, :])
    out = np.empty_like(x)
    out[:, 0:half:2], out[:, 1:half:2] = zy.real, zy.imag
    out[:, half::2], out[:, half + 1::2] = zx.real, zx.imag
    return out


def brute_global(q, k, v, M, s, theta=None, bias=None, with_lse=False):
    """Masked global attention over all H*W tokens of each image and head.

    The map's grid is padded to Hp x Wp, the multiples of M at or above H and
    W (Swin pads before it rolls); only the H*W real tokens exist here.
    Token (y, x) of the original map sits at rolled position ((y - s) mod Hp,
    (x - s) mod Wp).  Two tokens may attend iff they fall in the same window
    of the rolled grid and carry the same Swin region id of that grid.  RoPE
    uses original coordinates; the bias factors use the window-local
    position."""
    q, k, v = (storage_to_f64(a) for a in (q, k, v))
    B, H, W, heads, d = q.shape
    Hp, Wp = -(-H // M) * M, -(-W // M) * M
    ys, xs = np.meshgrid(np.arange(H), np.arange(W), indexing="ij")
    yr, xr = (ys - s) % Hp, (xs - s) % Wp
    win = ((yr // M) * (Wp // M) + (xr // M)).ravel()
    region = swin_region_labels(Hp, Wp, M, s)[yr, xr].ravel()
    allowed = (win[:, None] == win[None, :]) & (region[:, None] == region[None, :])
    plocal = ((yr % M) * M + (xr % M)).ravel()
    out = np.zeros_like(q)
    lse = np.zeros(q.shape[:4])
    for b in range(B):
        for h in range(heads):
            Q = q[b, :, :, h, :].reshape(H * W, d)
            K = k[b, :, :, h, :].reshape(H * W, d)
            V = v[b, :, :, h, :].reshape(H * W, d)
            if theta is not None:
                Q = rotate_complex(Q, ys.ravel().astype(float), xs.ravel().astype(float), theta[h])
                K = rotate_complex(K, ys.ravel().astype(float), xs.ravel().astype(float), theta[h])
            S = (Q @ K.T) / math.sqrt(d)
            if bias is not None:
                bf = storage_to_f64(bias)
                S = S + bf[h, 0][plocal] @ bf[h, 1][plocal].T
            S = np.where(allowed, S, -np.inf)
            mx = S.max(axis=1, keepdims=True)
            P = np.exp(S - mx)
            tot = P.sum(axis=1, keepdims=True)
            P /= tot
            out[b, :, :, h, :] = (P @ V).reshape(H, W, d)
            lse[b, :, :, h] = (mx + np.log(tot)).reshape(H, W)
    return (out, lse) if with_lse else out


def _close(a, b, tol=TOL, what=""):
    err = np.max(np.abs(a - b)) / max(1.0, np.max(np.abs(b)))
    assert err <= tol, f"{what}: max rel err {err:.3e} > {tol:.1e}"


# --------------------------------------------------------------------------- pins

def pin_rope_displacement(o):
    """R(p)^T R(p') = R(p' - p): <R(p) q, R(p') k> = <q, R(p' - p) k>, and the
    rotation equals complex multiplication by exp(i * angle) (counter-clockwise,
    adjacent pairs, first half by row)."""
    rng = np.random.default_rng(1)
    for d in (4, 8, 32, 64):
        th = np.exp(rng.uniform(-6, 0.3, size=d // 4)).astype(np.float32)
        for _ in range(20):
            qv, kv = rng.standard_normal(d), rng.standard_normal(d)
            i, j, i2, j2 = (int(x) for x in rng.integers(0, 96, size=4))
            lhs = o.rope(qv, i, j, th) @ o.rope(kv, i2, j2, th)
            rhs = qv @ o.rope(kv, i2 - i, j2 - j, th)
            assert abs(lhs - rhs) <= 1e-9 * max(1.0, abs(lhs)), "displacement identity"
            ref = rotate_complex(qv[None, :], np.array([float(i)]), np.array([float(j)]), th)[0]
            _close(o.rope(qv, i, j, th), ref, 1e-12, "rotation as complex multiply")


def pin_theta_zero(o):
    """theta = 0 turns every rotation into the identity: same output as no RoPE."""
    q, k, v = _maps((2, 8, 8, 2, 8), "bf16", "pin-theta0")
    zero = np.zeros((2, 2), np.float32)
    a = o.fwd(q, k, v, M=4, shift=2, theta=zero)
    b = o.fwd(q, k, v, M=4, shift=2, theta=None)
    assert np.array_equal(a, b), "theta = 0 must equal no RoPE"


def pin_one_token_windows(o):
    """M = 1: each window holds one token, its softmax weight is 1, O = V."""
    q, k, v = _maps((2, 3, 5, 2, 8), "fp32", "pin-m1")
    th = I.make_theta(2, 8, "learned", 5).numpy()
    out = o.fwd(q, k, v, M=1, shift=0, theta=th)
    assert np.array_equal(out, storage_to_f64(v)), "M = 1 must give O = V"


def pin_constant_v(o):
    """Every token carries the same V row c: any convex combination is c."""
    q, k, _ = _maps((1, 8, 8, 2, 8), "fp32", "pin-constv")
    c = np.linspace(-2, 3, 8).astype(np.float32)
    v = np.broadcast_to(c, (1, 8, 8, 2, 8)).copy()
    th = I.make_theta(2, 8, "learned", 3).numpy()
    bias = I.to_storage_numpy(I.make_bias_feats(2, 4, 4, "fp32", 9))
    out = o.fwd(q, k, v, M=4, shift=2, theta=th, bias=bias)
    _close(out, np.broadcast_to(c.astype(np.float64), out.shape), 1e-12, "constant V")


def pin_zero_q_mean(o):
    """Q = 0 and no bias make all allowed scores equal: O is the plain mean of V
    over the allowed set, here enumerated from Swin's region construction."""
    B, H, W, heads, d, M, s = 1, 8, 12, 2, 4, 4, 1
    _, k, v = _maps((B, H, W, heads, d), "fp32", "pin-q0")
    q = np.zeros_like(k)
    out = o.fwd(q, k, v, M=M, shift=s, theta=None)
    vv = storage_to_f64(v)
    reg = swin_region_labels(H, W, M, s)
    for y in range(H):
        for x in range(W):
            yr, xr = (y - s) % H, (x - s) % W
            members = [((y2 + s) % H, (x2 + s) % W)
                       for y2 in range((yr // M) * M, (yr // M) * M + M)
                       for x2 in range((xr // M) * M, (xr // M) * M + M)
                       if reg[y2, x2] == reg[yr, xr]]
            mean = np.mean([vv[0, a, b] for a, b in members], axis=0)
            _close(out[0, y, x], mean, 1e-12, f"zero-Q mean at ({y},{x})")


def pin_hand_worked(o):
    """Hand-worked single window (H = W = M = 2, d = 4, fp32, no RoPE): every
    query is (2, 0, 0, 0) and key t is (t, 0, 0, 0), so with scale 1/2 the
    score of key t is t and every output row is sum_t e^t v_t / sum_t e^t.
    Then the corner window of a 4x4 map shifted by 1 with M = 2: its four
    tokens come from four different regions, each attends only to itself."""
    q = np.zeros((1, 2, 2, 1, 4), np.float32)
    k = np.zeros_like(q)
    v = np.zeros_like(q)
    q[..., 0] = 2.0
    for t in range(4):
        y, x = divmod(t, 2)
        k[0, y, x, 0, 0] = t
        v[0, y, x, 0] = (t, 10 * t, -1.0, 0.5)
    w = np.array([math.exp(t) for t in range(4)])
    expect = (w[:, None] * np.array([(t, 10 * t, -1.0, 0.5) for t in range(4)])).sum(0) / w.sum()
    out = o.fwd(q, k, v, M=2, shift=0)
    for y in range(2):
        for x in range(2):
            _close(out[0, y, x, 0], expect, 1e-13, "hand-worked window")

    rng = np.random.default_rng(7)
    q = rng.standard_normal((1, 4, 4, 1, 4)).astype(np.float32)
    k = rng.standard_normal((1, 4, 4, 1, 4)).astype(np.float32)
    v = rng.standard_normal((1, 4, 4, 1, 4)).astype(np.float32)
    out = o.fwd(q, k, v, M=2, shift=1)
    # rolled rows/cols 2..3 are original rows/cols 3 and 0: the corner window.
    for y in (3, 0):
        for x in (3, 0):
            _close(out[0, y, x, 0], v[0, y, x, 0].astype(np.float64), 1e-13, "corner window")
    # rolled window (0, 0) covers original rows 1..2 and cols 1..2, no wrap:
    # with Q = 0 each output there is the mean of those four V rows.
    qz = np.zeros_like(q)
    out = o.fwd(qz, k, v, M=2, shift=1)
    mean = v[0, 1:3, 1:3, 0].astype(np.float64).reshape(4, 4).mean(0)
    for y in (1, 2):
        for x in (1, 2):
            _close(out[0, y, x, 0], mean, 1e-13, "unwrapped window mean")


def pin_brute_global(o):
    """Oracle == brute-force masked global attention on several shapes."""
    cases = [
        # B, H, W, heads, d, M, s, dtype, rope, rank
        (2, 8, 8, 2, 8, 4, 0, "fp32", "learned", 0),
        (1, 8, 12, 2, 8, 4, 2, "bf16", "learned", 0),
        (1, 12, 8, 1, 16, 4, 3, "bf16", "standard", 0),
        (2, 6, 6, 2, 4, 3, 1, "fp32", None, 4),
        (1, 8, 8, 2, 8, 4, 1, "bf16", "learned", 4),
        (1, 9, 6, 1, 8, 3, 2, "fp32", "learned", 0),
        # maps that are not multiples of M: padded grid, pad positions hold no token
        (1, 10, 7, 2, 8, 4, 2, "bf16", "learned", 0),
        (2, 9, 13, 1, 8, 4, 0, "fp32", "learned", 0),
        (1, 7, 5, 2, 4, 3, 1, "fp32", None, 4),
        (1, 6, 14, 1, 8, 4, 3, "bf16", "standard", 0),
        (1, 5, 5, 1, 8, 8, 4, "fp32", "learned", 0),
    ]
    for n, (B, H, W, heads, d, M, s, dt, rope, r) in enumerate(cases):
        q, k, v = _maps((B, H, W, heads, d), dt, f"pin-brute-{n}")
        th = I.make_theta(heads, d, rope, 11 + n)
        th = None if th is None else th.numpy()
        bias = I.to_storage_numpy(I.make_bias_feats(heads, M, r, dt, 13 + n)) if r else None
        got = o.fwd(q, k, v, M=M, shift=s, theta=th, bias=bias)
        ref = brute_global(q, k, v, M, s, th, bias)
        _close(got, ref, 1e-10, f"brute-force global case {n}")


def pin_lse(o):
    """The log-sum-exp the forward saves for the backward: equal to the
    brute-force global one (masked scores over all real tokens, padded and
    shifted grids included), and log(n) for Q = 0 without bias, where all n
    allowed scores of a row are zero."""
    cases = [(1, 8, 12, 2, 8, 4, 2, "bf16", "learned", 0), (1, 7, 5, 2, 4, 3, 1, "fp32", None, 4),
             (2, 6, 9, 1, 8, 4, 0, "fp32", "learned", 0)]
    for n, (B, H, W, heads, d, M, s, dt, rope, r) in enumerate(cases):
        q, k, v = _maps((B, H, W, heads, d), dt, f"pin-lse-{n}")
        th = I.make_theta(heads, d, rope, 31 + n)
        th = None if th is None else th.numpy()
        bias = I.to_storage_numpy(I.make_bias_feats(heads, M, r, dt, 37 + n)) if r else None
        out, lse = o.fwd_lse(q, k, v, M=M, shift=s, theta=th, bias=bias)
        ref_out, ref_lse = brute_global(q, k, v, M, s, th, bias, with_lse=True)
        _close(out, ref_out, 1e-10, f"lse case {n}: output")
        _close(lse, ref_lse, 1e-10, f"lse case {n}: log-sum-exp")
    # zero queries: lse = log(size of the row's allowed set)
    B, H, W, heads, d, M, s = 1, 8, 12, 1, 4, 4, 1
    _, k, v = _maps((B, H, W, heads, d), "fp32", "pin-lse-q0")
    _, lse = o.fwd_lse(np.zeros_like(k), k, v, M=M, shift=s)
    reg = swin_region_labels(H, W, M, s)
    for y in range(H):
        for x in range(W):
            yr, xr = (y - s) % H, (x - s) % W
            n_allowed = sum(1 for y2 in range((yr // M) * M, (yr // M) * M + M)
                            for x2 in range((xr // M) * M, (xr // M) * M + M) if reg[y2, x2] == reg[yr, xr])
            assert abs(lse[0, y, x, 0] - math.log(n_allowed)) < 1e-13, f"zero-Q lse at ({y},{x})"


def brute_sparse(q, k, v, o_lin, windows, M, s, theta=None, bias=None):
    """HSMLA's gated residual written from the global formulation: softmax
    part from brute_global, the local linear part as a masked matrix product
    relu(Q) relu(K)^T over the same allowed pairs, added only to the tokens
    of the listed windows of the rolled (padded) grid."""
    B, H, W, heads, d = q.shape
    Hp, Wp = -(-H // M) * M, -(-W // M) * M
    soft = brute_global(q, k, v, M, s, theta, bias)
    qf, kf, vf = (storage_to_f64(a) for a in (q, k, v))
    ys, xs = np.meshgrid(np.arange(H), np.arange(W), indexing="ij")
    yr, xr = (ys - s) % Hp, (xs - s) % Wp
    win = ((yr // M) * (Wp // M) + (xr // M)).ravel()
    region = swin_region_labels(Hp, Wp, M, s)[yr, xr].ravel()
    allowed = (win[:, None] == win[None, :]) & (region[:, None] == region[None, :])
    out = np.array(o_lin, dtype=np.float64, copy=True)
    per_img = (Hp // M) * (Wp // M)
    for b in range(B):
        sel = np.isin(win, [w - b * per_img for w in windows if b * per_img <= w < (b + 1) * per_img])
        for h in range(heads):
            Q = np.maximum(qf[b, :, :, h].reshape(H * W, d), 0)
            K = np.maximum(kf[b, :, :, h].reshape(H * W, d), 0)
            V = vf[b, :, :, h].reshape(H * W, d)
            L = np.where(allowed, Q @ K.T, 0.0)
            den = L.sum(axis=1, keepdims=True)
            lin = np.where(den > 0, (L @ V) / np.where(den > 0, den, 1.0), 0.0)
            res = soft[b, :, :, h].reshape(H * W, d) - lin
            o = out[b, :, :, h].reshape(H * W, d)
            o[sel] += res[sel]
            out[b, :, :, h] = o.reshape(H, W, d)
    return out


def pin_sparse_residual(o):
    """The gated residual equals its global formulation on several shapes
    (shifted, padded, with bias factors); windows that are not listed keep
    O_lin bit for bit; with every window listed and the same constant
    positive q and k everywhere, softmax and linear weights are both uniform,
    so the residual vanishes and the output is O_lin."""
    cases = [(2, 8, 12, 2, 8, 4, 2, "bf16", "learned", 0, [0, 3, 7, 9]),
             (1, 10, 7, 1, 8, 4, 3, "fp32", None, 0, [1, 2, 5]),
             (1, 8, 8, 2, 4, 4, 0, "bf16", None, 4, [0, 2, 3])]
    for n, (B, H, W, heads, d, M, s, dt, rope, r, wins) in enumerate(cases):
        q, k, v = _maps((B, H, W, heads, d), dt, f"pin-sparse-{n}")
        th = I.make_theta(heads, d, rope, 41 + n)
        th = None if th is None else th.numpy()
        bias = I.to_storage_numpy(I.make_bias_feats(heads, M, r, dt, 43 + n)) if r else None
        o_lin = np.random.default_rng(n).standard_normal((B, H, W, heads, d))
        got = o.fwd_sparse(q, k, v, o_lin, wins, M=M, shift=s, theta=th, bias=bias)
        ref = brute_sparse(q, k, v, o_lin, wins, M, s, th, bias)
        _close(got, ref, 1e-10, f"sparse case {n}")
        untouched = np.isclose(ref, o_lin, rtol=0, atol=0)
        assert np.array_equal(got[untouched], o_lin[untouched]), "unlisted windows keep O_lin"
    B, H, W, heads, d, M = 1, 8, 8, 1, 4, 4
    c = np.full((B, H, W, heads, d), 0.5, np.float32)
    _, _, v = _maps((B, H, W, heads, d), "fp32", "pin-sparse-const")
    o_lin = np.random.default_rng(9).standard_normal((B, H, W, heads, d))
    got = o.fwd_sparse(c, c, v, o_lin, [0, 1, 2, 3], M=M, shift=2)
    _close(got, o_lin, 1e-12, "uniform weights: zero residual")


def _rib_weights(heads, rank, seed, scale=1.0):
    rng = np.random.default_rng(seed)
    w1 = (scale * rng.standard_normal((heads, 2, 32, 64)) / math.sqrt(32)).astype(np.float32)
    w2 = (rng.standard_normal((heads, 2, 64, rank)) / math.sqrt(64)).astype(np.float32)
    return w1, w2


def pin_rib_features(o):
    """The RIB factor MLP (RIB page, section 2.1) by closed forms and
    symmetries of its Fourier features: at M = 1 every coordinate is 0 (sin 0,
    cos 1); at M = 2 the coordinates are -1 and 1, where sin(2^k pi c) = 0 and
    cos(2^k pi c) = -1 for k = 0, 1 after; with only cosine rows the table is
    mirror-symmetric in each axis (cos is even), with only sine rows it is odd
    under the point reflection (sin and tanh are odd); with only the row-axis
    rows it does not depend on the column."""
    heads, rank = 2, 16
    w1, w2 = _rib_weights(heads, rank, 3)
    f0 = np.concatenate([np.zeros(8), np.ones(8), np.zeros(8), np.ones(8)])
    got = o.rib_features(w1, w2, 1)
    for h in range(heads):
        for s in range(2):
            ref = np.tanh(f0 @ w1[h, s].astype(np.float64)) @ w2[h, s].astype(np.float64)
            _close(got[h, s, 0], ref, 1e-12, "M = 1 closed form")
    got = o.rib_features(w1, w2, 2)
    cosv = np.array([-1.0] + [1.0] * 7)
    for p in range(4):
        f = np.concatenate([np.zeros(8), cosv, np.zeros(8), cosv])
        for h in range(heads):
            for s in range(2):
                ref = np.tanh(f @ w1[h, s].astype(np.float64)) @ w2[h, s].astype(np.float64)
                _close(got[h, s, p], ref, 1e-12, "M = 2 closed form")
    M = 7
    cos_only, sin_only, y_only = w1.copy(), w1.copy(), w1.copy()
    cos_only[:, :, 0:8] = 0
    cos_only[:, :, 16:24] = 0
    sin_only[:, :, 8:16] = 0
    sin_only[:, :, 24:32] = 0
    y_only[:, :, 16:32] = 0
    t = o.rib_features(cos_only, w2, M).reshape(heads, 2, M, M, rank)
    _close(t, t[:, :, ::-1, :, :], 1e-12, "cosine rows: mirror in rows")
    _close(t, t[:, :, :, ::-1, :], 1e-12, "cosine rows: mirror in columns")
    t = o.rib_features(sin_only, w2, M).reshape(heads, 2, M, M, rank)
    _close(t, -t[:, :, ::-1, ::-1, :], 1e-12, "sine rows: odd under point reflection")
    t = o.rib_features(y_only, w2, M).reshape(heads, 2, M, M, rank)
    _close(t, np.broadcast_to(t[:, :, :, :1, :], t.shape), 1e-12, "row-axis rows: no column dependence")


def pin_cla_gate(o):
    """The CLA gate (RIB page, section 2.2) against library routines: a
    per-channel 2-D correlation with zero fill (scipy.signal.correlate2d),
    a matrix product and the logistic function (scipy.special.expit); and
    the closed form O * sigmoid(b) when the point-wise weights are zero."""
    from scipy.signal import correlate2d
    from scipy.special import expit
    rng = np.random.default_rng(5)
    B, H, W, C = 2, 5, 7, 8
    x = I.to_storage_numpy(I.make_map((B, H, W, C), "bf16", 61))
    ob = I.to_storage_numpy(I.make_map((B, H, W, C), "bf16", 62))
    dw = rng.standard_normal((C, 3, 3)).astype(np.float32)
    dw_b = rng.standard_normal(C).astype(np.float32)
    pw = (rng.standard_normal((C, C)) / math.sqrt(C)).astype(np.float32)
    pw_b = rng.standard_normal(C).astype(np.float32)
    got = o.cla_gate(x, ob, dw, dw_b, pw, pw_b)
    xf, of = storage_to_f64(x), storage_to_f64(ob)
    y = np.zeros((B, H, W, C))
    for b in range(B):
        for c in range(C):
            y[b, :, :, c] = correlate2d(xf[b, :, :, c], dw[c].astype(np.float64), mode="same",
                                        boundary="fill") + dw_b[c]
    ref = of * expit(y @ pw.T.astype(np.float64) + pw_b)
    _close(got, ref, 1e-12, "gate against library routines")
    got = o.cla_gate(x, ob, dw, dw_b, np.zeros_like(pw), pw_b)
    _close(got, of * expit(pw_b.astype(np.float64)), 1e-12, "zero point-wise weights")


def pin_bias_concat(o):
    """[Qc, Qp][Kc, Kp]^T = Qc Kc^T + Qp Kp^T: a problem with rank-r bias
    factors equals a bias-free problem of head dim d + r whose query rows are
    [q * sqrt((d+r)/d), u(p) * sqrt(d+r)] and key rows [k, w(p)] (the wider
    problem's own scale (d+r)^-1/2 is undone by the factors)."""
    B, H, W, heads, d, r, M, s = 1, 8, 8, 2, 8, 4, 4, 2
    q, k, v = _maps((B, H, W, heads, d), "fp32", "pin-concat")
    bias = I.to_storage_numpy(I.make_bias_feats(heads, M, r, "fp32", 21))
    got = o.fwd(q, k, v, M=M, shift=s, bias=bias)
    D = d + r
    qq = np.zeros((B, H, W, heads, D))
    kk = np.zeros((B, H, W, heads, D))
    vv = np.zeros((B, H, W, heads, D))
    qq[..., :d] = q.astype(np.float64) * math.sqrt(D / d)
    kk[..., :d] = k
    vv[..., :d] = v
    for y in range(H):
        for x in range(W):
            p = ((y - s) % H % M) * M + ((x - s) % W % M)
            qq[:, y, x, :, d:] = bias[:, 0, p, :].astype(np.float64) * math.sqrt(D)
            kk[:, y, x, :, d:] = bias[:, 1, p, :]
    ref = brute_global(qq, kk, vv, M, s)[..., :d]
    _close(got, ref, 1e-10, "concatenation identity")


def pin_distinct_offsets(o, M=32, expected=3969):
    """The relative-position table the rotation replaces has (2M - 1)^2 entries
    (3969 at M = 32 on the FlashSwin page): count distinct displacements of
    token pairs of one window through the oracle's own token coordinates."""
    coords = [o.token_origin(M, M, M, 0, 0, 0, p) for p in range(M * M)]
    ys = np.array([c[0] for c in coords])
    xs = np.array([c[1] for c in coords])
    dy = (ys[:, None] - ys[None, :]).ravel()
    dx = (xs[:, None] - xs[None, :]).ravel()
    n = len(set(zip(dy.tolist(), dx.tolist())))
    assert n == expected, f"{n} distinct offsets, expected {expected}"


def pin_padding_closed_forms(o):
    """Padding, by closed forms.  A 5 x 6 map at M = 4 pads to 8 x 8: rolled
    window row 1 (no shift) holds only original row 4, so with Q = 0 each of
    its outputs is the mean of V over that row's tokens of the same window
    (the pad keys take no weight); constant V still gives the constant; and
    the units' output marks pad positions NaN, real ones finite."""
    B, H, W, heads, d, M = 1, 5, 6, 1, 4, 4
    _, k, v = _maps((B, H, W, heads, d), "fp32", "pin-pad")
    q = np.zeros_like(k)
    out = o.fwd(q, k, v, M=M, shift=0)
    vv = storage_to_f64(v)
    _close(out[0, 4, 0:4, 0], np.broadcast_to(vv[0, 4, 0:4, 0].mean(0), (4, d)), 1e-13, "row-4 window mean")
    _close(out[0, 4, 4:6, 0], np.broadcast_to(vv[0, 4, 4:6, 0].mean(0), (2, d)), 1e-13, "row-4 corner mean")
    _close(out[0, 0:4, 4:6, 0], np.broadcast_to(vv[0, 0:4, 4:6, 0].reshape(8, d).mean(0), (4, 2, d)), 1e-13,
           "right-edge window mean")
    c = np.linspace(-1, 2, d).astype(np.float32)
    cv = np.broadcast_to(c, v.shape).copy()
    th = I.make_theta(heads, d, "learned", 4).numpy()
    out = o.fwd(q + 1, k, cv, M=M, shift=3, theta=th)
    _close(out, np.broadcast_to(c.astype(np.float64), out.shape), 1e-12, "constant V, padded")
    units = o.fwd_units(q, k, v, [1 * 2 + 1], M=M, shift=0)   # window (1, 1): rows 4..7, cols 4..7
    pad = np.array([(4 + p // M) >= H or (4 + p % M) >= W for p in range(M * M)])
    assert np.all(np.isnan(units[0][pad])) and np.all(np.isfinite(units[0][~pad])), "pad rows NaN, real finite"


ALL_PINS = [pin_rope_displacement, pin_theta_zero, pin_one_token_windows, pin_constant_v,
            pin_zero_q_mean, pin_hand_worked, pin_brute_global, pin_bias_concat, pin_padding_closed_forms,
            pin_lse, pin_sparse_residual, pin_rib_features, pin_cla_gate]
