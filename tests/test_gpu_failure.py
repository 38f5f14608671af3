"""GPU: the device-side timeout path, made to run out on purpose without a fault.

Every wait of the library's kernels on an mbarrier or a flag is bounded; on
expiry the kernel records a timeout in a device word and returns.  The
self-test kernel waits on an mbarrier nobody arrives at with a short limit;
the host must then read RQ_ERR_TIMEOUT, the word must be cleared by the read,
and the context must stay usable (a rotation afterwards is still exact).
"""

import numpy as np
import pytest
import torch

import parity
from oracle import hadamard
from rotation_w4a4_quantization_b200 import synthetic as syn

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def rq():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    from rotation_w4a4_quantization_b200 import rq as m
    m.init(0)
    return m


def test_bounded_wait_reports_timeout_and_context_survives(rq):
    rq.get_device_error()                       # start clean
    rq.selftest_wait_timeout(1_000_000)         # ~0.5 ms of spinning, then give up
    with pytest.raises(rq.RQError) as e:
        rq.get_device_error()
    assert e.value.status == 6                  # RQ_ERR_TIMEOUT
    rq.get_device_error()                       # the read cleared the word
    x = syn.activations("tiny_int4")
    s = syn.workload_signs("tiny_int4")
    got = rq.rotate_f32(x.cuda(), s.cuda(), 128)
    torch.cuda.synchronize()
    parity.check_rotation(parity.to_np(got), hadamard.rotate(parity.bf16_to_f64(x), s.numpy(), 128))
    rq.get_device_error()


def test_selftest_rejects_bad_limits(rq):
    for lim in (0, -5, 3_000_000_000):
        with pytest.raises(rq.RQError) as e:
            rq.selftest_wait_timeout(lim)
        assert e.value.status == 1
