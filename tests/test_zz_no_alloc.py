"""The no-allocation host entry point, winattn_fwd_host_static.

Some callers cannot allocate device memory (the process's device memory
belongs to someone else, or no allocator is reachable from the calling
code), so they can pass neither device buffers nor a workspace.  For them
the library keeps one static device buffer and does the host-buffer call
with it.  Here it must give the result winattn_fwd gives on device copies of
the same inputs, bit for bit, on two calls in a row with different inputs
(the buffer keeps the previous call's contents), match the fp64 oracle, leave
the device's free memory unchanged, and refuse problems that do not fit its
fixed size.  This file is collected last on purpose.
"""
import pytest
import torch

import windowed_attention_vision_b200 as wa
from windowed_attention_vision_b200 import _lib
from windowed_attention_vision_b200 import inputs as I
from tests import gpu_helpers as G

pytestmark = pytest.mark.gpu


def _static_call(q, k, v, theta, M, shift):
    B, H, W, heads, d = q.shape
    out = torch.empty_like(q).pin_memory()
    stream = torch.cuda.current_stream().cuda_stream
    rc = _lib.fwd_host_static(q.data_ptr(), k.data_ptr(), v.data_ptr(), theta.data_ptr(), None, B, H, W, M,
                              shift, heads, d, 0, _lib.BF16, out.data_ptr(), stream)
    assert rc == _lib.OK, _lib.strerror(rc)
    torch.cuda.current_stream().synchronize()
    return out


def test_static_workspace_matches_device_entry_point_on_two_calls():
    """Two calls in a row with different inputs (the buffer keeps the previous
    call's contents): each equals winattn_fwd on device copies of the same
    inputs bit for bit (the same kernel on the same problem), matches the fp64
    oracle within the bf16 tolerance, and leaves the device's free memory
    unchanged (the call allocates nothing)."""
    w = I.Workload("no-alloc", 2, 16, 24, 8, (4,), 3, 32, "bf16", "learned")
    cases = []
    for base in (0, 1):
        (qkv,), theta, _ = I.make_inputs(w, base=base)
        pinned = [t.pin_memory() for t in qkv]
        dev = G.run_gpu(*(t.cuda() for t in qkv), w.M, 4, theta.cuda())
        ref = G.orc().fwd(*(I.to_storage_numpy(t) for t in qkv), M=w.M, shift=4, theta=theta.numpy())
        cases.append((pinned, theta.cuda(), dev.cpu(), ref))
    # the first call on the device looks up the buffer's address (and may load
    # the library's module, which holds the buffer): not part of the check
    _static_call(*cases[0][0], cases[0][1], w.M, 4)
    torch.cuda.synchronize()
    free_before = torch.cuda.mem_get_info()[0]
    for n, (pinned, theta, dev, ref) in enumerate(cases):
        got = _static_call(*pinned, theta, w.M, 4)
        assert torch.equal(got, dev), f"call {n + 1}: static-workspace result differs from winattn_fwd"
        G.check(G.as_f64(got), ref, "bf16", f"static workspace, call {n + 1}")
    torch.cuda.synchronize()
    assert torch.cuda.mem_get_info()[0] >= free_before, "free device memory dropped during the calls"
    assert wa.device_status() == 0


def test_static_workspace_refuses_problems_that_do_not_fit():
    # four bf16 maps of 2 x 256 x 256 x 4 x 32 elements (16 MiB each) exceed
    # the static buffer; nothing is touched before the size check
    B, H, W, heads, d = 2, 256, 256, 4, 32
    assert _lib.host_workspace_bytes(B, H, W, heads, d, _lib.BF16) > _lib.STATIC_WORKSPACE_BYTES
    fake = 1 << 20
    rc = _lib.fwd_host_static(fake, 2 * fake, 3 * fake, None, None, B, H, W, 8, 4, heads, d, 0, _lib.BF16,
                              4 * fake, None)
    assert rc == _lib.ERR_SIZE
