"""Pins of the oracle's backward (the gradients of the window attention with
respect to q, k, v, the RoPE frequencies theta and the bias table), by central
finite differences of the forward oracle, which its own pins fix, and by the
closed-form invariant that every row of P sums to one.

The FLASHSWIN page ("FLASHSWIN: Unlocking Large Windows and Dense Tokens in
Swin Vision Transformers with Memory Efficient Attention") trains the model
with learned frequencies theta = exp(omega) (section "어떻게 동작하나"); these
gradients are what a training step needs from the fused operator."""
import os

import numpy as np
import pytest

import oracle

H_STEP = np.float32(2.0 ** -10)  # exactly representable perturbation of fp32 storage


def problem(seed, shift, with_theta, with_bias, B=1, H=8, W=8, M=4, heads=2, d=8, rank=4):
    rng = np.random.default_rng(seed)
    q, k, v = (rng.standard_normal((B, H, W, heads, d)).astype(np.float32) for _ in range(3))
    theta = (0.3 + 0.5 * rng.random((heads, d // 4))).astype(np.float32) if with_theta else None
    bias = (0.5 * rng.standard_normal((heads, 2, M * M, rank))).astype(np.float32) if with_bias else None
    dout = rng.standard_normal((B, H, W, heads, d))
    return dict(q=q, k=k, v=v, theta=theta, bias=bias, dout=dout, M=M, shift=shift)


def loss(o, pr, **over):
    args = dict(q=pr["q"], k=pr["k"], v=pr["v"], theta=pr["theta"], bias=pr["bias"])
    args.update(over)
    out = o.fwd(args["q"], args["k"], args["v"], M=pr["M"], shift=pr["shift"], theta=args["theta"],
                bias=args["bias"])
    return float(np.sum(out * pr["dout"]))


def fd_check(o, pr, name, grad, n_samples, seed):
    base = pr[name]
    rng = np.random.default_rng(seed)
    flat_idx = rng.choice(base.size, size=min(n_samples, base.size), replace=False)
    scale = max(1.0, float(np.max(np.abs(grad))))
    for fi in flat_idx:
        idx = np.unravel_index(fi, base.shape)
        plus, minus = base.copy(), base.copy()
        plus[idx] += H_STEP
        minus[idx] -= H_STEP
        fd = (loss(o, pr, **{name: plus}) - loss(o, pr, **{name: minus})) / (2.0 * float(H_STEP))
        an = float(grad[idx])
        assert abs(fd - an) <= 2e-5 * scale, f"d{name}{idx}: finite difference {fd:.8f}, backward {an:.8f}"


@pytest.mark.parametrize("shift,with_theta,with_bias,H,W", [(2, True, False, 8, 8), (0, True, True, 8, 8),
                                                            (2, False, True, 8, 8), (1, True, True, 8, 8),
                                                            (3, True, True, 7, 6), (0, True, False, 5, 9)])
def test_gradients_match_finite_differences(shift, with_theta, with_bias, H, W):
    """(the last two maps are not multiples of M = 4: the padded grid)"""
    o = oracle.oracle()
    pr = problem(7 + shift, shift, with_theta, with_bias, H=H, W=W)
    dq, dk, dv, dtheta, dbias = o.bwd(pr["q"], pr["k"], pr["v"], pr["dout"], M=pr["M"], shift=shift,
                                      theta=pr["theta"], bias=pr["bias"])
    fd_check(o, pr, "q", dq, 48, 1)
    fd_check(o, pr, "k", dk, 48, 2)
    fd_check(o, pr, "v", dv, 48, 3)
    if with_theta:
        fd_check(o, pr, "theta", dtheta, dtheta.size, 4)
    else:
        assert dtheta is None
    if with_bias:
        fd_check(o, pr, "bias", dbias, 48, 5)
    else:
        assert dbias is None


def test_value_gradient_sums_to_output_gradient():
    # every row of P sums to one, so within a window sum_c dV[c] = sum_a dO[a];
    # the windows partition the map, so the sums agree per (image, head)
    o = oracle.oracle()
    pr = problem(3, 2, True, False, B=2, H=8, W=12, M=4, heads=3, d=16)
    _, _, dv, _, _ = o.bwd(pr["q"], pr["k"], pr["v"], pr["dout"], M=pr["M"], shift=2, theta=pr["theta"])
    np.testing.assert_allclose(dv.sum(axis=(1, 2)), pr["dout"].sum(axis=(1, 2)), rtol=1e-12, atol=1e-10)


def test_zero_output_gradient_gives_zero_gradients():
    o = oracle.oracle()
    pr = problem(5, 2, True, True)
    zeros = np.zeros_like(pr["dout"])
    grads = o.bwd(pr["q"], pr["k"], pr["v"], zeros, M=pr["M"], shift=2, theta=pr["theta"], bias=pr["bias"])
    for g in grads:
        assert np.all(g == 0.0)


def test_constant_values_leave_no_score_gradient():
    # with every value vector equal, O = v whatever P is: dq, dk, dtheta and
    # dbias vanish, and dv collects dO of every row of its window
    o = oracle.oracle()
    pr = problem(9, 2, True, True)
    v = np.broadcast_to(pr["v"][:1, :1, :1], pr["v"].shape).copy()
    dq, dk, dv, dtheta, dbias = o.bwd(pr["q"], pr["k"], v, pr["dout"], M=pr["M"], shift=2, theta=pr["theta"],
                                      bias=pr["bias"])
    for g in (dq, dk, dtheta, dbias):
        assert np.max(np.abs(g)) < 1e-12


SRC = os.path.join(os.path.dirname(oracle.__file__), "winattn_oracle.c")

# Planted mistakes in the backward; each must fail a finite-difference pin.
MUTANTS = {
    "softmax_jacobian_row_term_dropped": [(
        "g_s[(size_t)a * N + c] = w->s[(size_t)a * N + c] * (g_s[(size_t)a * N + c] - rowdot);",
        "g_s[(size_t)a * N + c] = w->s[(size_t)a * N + c] * g_s[(size_t)a * N + c];")],
    "value_gradient_transposed": [(
        "acc += w->s[(size_t)a * N + c] * g_o[(size_t)a * d + e];",
        "acc += w->s[(size_t)c * N + a] * g_o[(size_t)a * d + e];")],
    "query_gradient_not_rotated_back": [("rope_rotate(gq, d, -i, -j, th);", "(void)th;")],
    "theta_gradient_sign": [(
        "dtheta_h[k] += i * (gq[a1] * xq[a0] - gq[a0] * xq[a1])",
        "dtheta_h[k] += i * (gq[a0] * xq[a1] - gq[a1] * xq[a0])")],
    "key_gradient_unscaled": [("g_k[(size_t)c * d + e] = scale * acc;", "g_k[(size_t)c * d + e] = acc;")],
    "bias_gradient_sides_swapped": [("dbias_h[(size_t)a * r + e] += acc;", "dbias_h[((size_t)N + a) * r + e] += acc;")],
}


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_planted_backward_mistake_fails_a_pin(name, tmp_path):
    with open(SRC) as f:
        src = f.read()
    for old, new in MUTANTS[name]:
        assert src.count(old) == 1, f"mutation site for {name!r} not found exactly once"
        src = src.replace(old, new)
    path = tmp_path / "mutant.c"
    path.write_text(src)
    orc = oracle.Oracle(oracle.load(oracle.build(str(path), str(tmp_path / "libmutant.so"))))
    caught = False
    for shift, with_theta, with_bias in [(2, True, True), (0, True, True)]:
        pr = problem(11, shift, with_theta, with_bias)
        grads = orc.bwd(pr["q"], pr["k"], pr["v"], pr["dout"], M=pr["M"], shift=shift, theta=pr["theta"],
                        bias=pr["bias"])
        for name_t, g in zip(("q", "k", "v", "theta", "bias"), grads):
            try:
                fd_check(orc, pr, name_t, g, 24, 6)
            except AssertionError:
                caught = True
        if caught:
            break
    assert caught, f"backward mutant {name!r} passed every finite-difference pin"
