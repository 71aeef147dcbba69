"""Failure detection on the GPU without a fault: the bounded wait the
attention kernels use runs out on an mbarrier that nothing arrives at (a
self-test entry point of the library), the host reads
WINATTN_ERR_DEVICE_TIMEOUT from the status word, and the device stays usable
for the next call."""
import time

import pytest
import torch

import windowed_attention_vision_b200 as wa
from windowed_attention_vision_b200 import _lib
from windowed_attention_vision_b200 import inputs as I
from tests import gpu_helpers as G

pytestmark = pytest.mark.gpu


def test_bounded_wait_gives_up_and_device_stays_usable():
    assert wa.device_status() == _lib.OK
    stream = torch.cuda.current_stream().cuda_stream
    t0 = time.monotonic()
    assert _lib.selftest_wait_timeout(stream) == _lib.OK
    assert wa.device_status() == _lib.ERR_DEVICE_TIMEOUT
    elapsed = time.monotonic() - t0
    assert 1.5 < elapsed < 60, elapsed  # the 2 s wall-clock limit of a wait
    assert wa.device_status() == _lib.OK  # read and cleared
    w = I.Workload("after_timeout", 1, 16, 16, 8, (4,), 2, 32, "bf16", "learned", 0)
    G.full_compare(w, 4)
