"""The differentiable op (window_attention_autograd: winattn_fwd_lse +
winattn_bwd) in a torch training step: gradients of q, k, v, the learned
log-frequencies omega (theta = exp(omega), FLASHSWIN page, section "어떻게
동작하나") and the bias features against the fp64 backward oracle, with the
backward's tolerances; and the same step captured in a CUDA graph and
replayed gives the same bits."""
import numpy as np
import pytest
import torch

import windowed_attention_vision_b200 as wa
from windowed_attention_vision_b200 import inputs as I
from tests import gpu_helpers as G
from tests.test_gpu_backward import BWD_TOL, rel_check

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("case", [(2, 16, 16, 8, 4, 2, 32, 0), (1, 32, 32, 16, 8, 2, 32, 16)], ids=["m8", "m16_r16"])
def test_autograd_gradients_match_oracle(case):
    B, H, W, M, s, heads, d, r = case
    w = I.Workload("ag", B, H, W, M, (s,), heads, d, "bf16", "learned", r)
    (qkv,), theta, bias = I.make_inputs(w)
    dout = I.make_map(qkv[0].shape, "bf16", 17)
    q, k, v = (t.cuda().requires_grad_() for t in qkv)
    omega = theta.log().cuda().requires_grad_()
    bs = None if bias is None else bias.cuda().requires_grad_()
    out = wa.window_attention_autograd(q, k, v, M, s, theta=omega.exp(), bias_feats=bs)
    (out.float() * dout.cuda().float()).sum().backward()
    torch.cuda.synchronize()
    assert wa.device_status() == 0
    th32 = omega.detach().exp().cpu()
    dq, dk, dv, dth, dbi = G.orc().bwd(*(I.to_storage_numpy(t) for t in qkv), G.as_f64(dout), M=M, shift=s,
                                       theta=th32.numpy(), bias=I.to_storage_numpy(bias))
    rel_check(G.as_f64(q.grad), dq, BWD_TOL["dq"], "q.grad")
    rel_check(G.as_f64(k.grad), dk, BWD_TOL["dk"], "k.grad")
    rel_check(G.as_f64(v.grad), dv, BWD_TOL["dv"], "v.grad")
    # d/domega = theta * d/dtheta
    rel_check(G.as_f64(omega.grad), th32.double().numpy() * dth, BWD_TOL["dtheta"], "omega.grad")
    if bs is not None:
        rel_check(G.as_f64(bs.grad), dbi, BWD_TOL["dbias"], "bias_feats.grad")


def test_training_step_in_a_cuda_graph():
    w = I.Workload("graph", 4, 16, 16, 8, (4,), 2, 32, "bf16", "learned")
    (qkv,), theta, _ = I.make_inputs(w, "cuda")
    q, k, v = qkv
    dout = I.make_map(q.shape, "bf16", 3, "cuda")
    lse = torch.empty((w.B, w.H, w.W, w.heads), dtype=torch.float32, device="cuda")
    out = torch.empty_like(q)

    def step():
        wa.window_attention(q, k, v, w.M, 4, theta=theta, out=out, lse=lse)
        return wa.window_attention_backward(q, k, v, out, dout, lse, w.M, 4, theta=theta)

    eager = [t.clone() for t in step()[:3]]
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        step()  # warm-up on a side stream before capture
    torch.cuda.current_stream().wait_stream(side)
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        grads = step()
    g.replay()
    torch.cuda.synchronize()
    assert wa.device_status() == 0
    for a, b in zip(eager, grads[:3]):
        assert torch.equal(a, b)
