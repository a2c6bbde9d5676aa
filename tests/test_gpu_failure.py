"""Failure detection without a GPU fault: a wait that runs out is reported in
the device status word, and the context stays usable.

The self-test kernel waits on a barrier nothing arrives on (20 ms limit);
nothing is faulted, trapped or hung.
"""
import numpy as np
import pytest
import torch

import synthetic
from gpu_util import f64, to_device
from parity import compare_codes, reference

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def kq():
    if not torch.cuda.is_available():
        pytest.fail("CUDA device required for -m gpu tests")
    from w4a4_dit_post_b200 import build
    build.build()
    import w4a4_dit_post_b200 as k
    k.kq_device_status(clear=True)
    yield k
    assert k.kq_device_status(clear=True) == 0


def test_timed_out_wait_is_reported_and_context_survives(kq):
    assert kq.kq_device_status(clear=True) == 0
    kq.kq_selftest_bounded_wait(20000)          # 20 ms, nothing ever arrives
    flags = kq.kq_device_status(clear=True)
    assert flags & 0x1, "the timed-out wait must set KQ_DEVSTAT_WAIT_TIMEOUT"
    assert kq.kq_device_status() == 0           # cleared
    # the context is intact: a real quantization still matches the oracle
    w = synthetic.Workload("after", 64, 256, "bf16", "normal", 0.02, None, 20.0, 1.0, 7)
    raw = synthetic.make_activations(w)
    p = synthetic.make_params(w.nb, 7)
    codes, scales = kq.kq_quantize(to_device(raw, "bf16"), torch.from_numpy(p).cuda())
    y_ref, tol = reference(f64(raw, "bf16"), params=p)
    assert compare_codes(codes.cpu().numpy(), scales.cpu().numpy(), y_ref, tol).ok
    assert kq.kq_device_status() == 0


def test_selftest_argument_check(kq):
    with pytest.raises(RuntimeError):
        kq.kq_selftest_bounded_wait(0)
