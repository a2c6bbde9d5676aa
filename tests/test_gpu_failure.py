"""Failure detection without a GPU fault: a wait that runs out, or LU
parameters that define no factor (u = 0, a non-finite value), are reported in
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


def _bad_params(nb, where, value):
    p = synthetic.make_params(nb, 3).copy()
    p[where] = value
    return torch.from_numpy(p).cuda()


@pytest.mark.parametrize("where,value", [((1, 8), 0.0), ((0, 0), float("nan")), ((2, 4), float("inf"))],
                         ids=["u_zero", "a_nan", "b_inf"])
def test_bad_parameters_are_reported(kq, where, value):
    """Every call that reads the LU parameters flags them; outputs are
    unspecified, nothing faults, and good parameters afterwards are clean."""
    M, d = 64, 96
    nb = d // 32
    pd = _bad_params(nb, where, value)
    w = synthetic.Workload("badp", M, d, "bf16", "normal", 0.02, None, 20.0, 1.0, 8)
    x = to_device(synthetic.make_activations(w), "bf16")
    W = torch.from_numpy(synthetic.make_weights(16, d, 8)).cuda()
    calls = [
        lambda: kq.kq_quantize(x, pd),
        lambda: kq.kq_quantize(x.float(), pd),
        lambda: kq.kq_quantize_tc(x, pd),
        lambda: kq.kq_transform(x, pd),
        lambda: kq.kq_expand_params(pd),
        lambda: kq.kq_fold_weights(W, pd),
        lambda: kq.kq_quantize_weights(W, pd),
    ]
    assert kq.kq_device_status(clear=True) == 0
    for call in calls:
        call()
        assert kq.kq_device_status(clear=True) == 0x2
    good = torch.from_numpy(synthetic.make_params(nb, 3)).cuda()
    for call in [lambda: kq.kq_quantize(x, good), lambda: kq.kq_quantize_weights(W, good)]:
        call()
        assert kq.kq_device_status() == 0
