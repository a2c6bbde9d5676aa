"""The library's launches (programmatic dependent launch on the caller's
stream) captured into a CUDA graph and replayed: one W4A4 layer step
(activation quantizer, scale tiling, GEMM) gives the same bits replayed as
run eagerly.  Needs a B200.
"""
import numpy as np
import pytest
import torch

import synthetic
from gpu_util import device_activations

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
    assert k.kq_device_status() == 0, "a bounded device wait ran out"


def test_layer_step_in_a_cuda_graph(kq):
    w = synthetic.CONFIGS["flux"][0]                      # 4608 x 3072 bf16
    x = device_activations(w)
    p = torch.from_numpy(synthetic.make_params(w.nb, w.seed)).cuda()
    W = torch.from_numpy(synthetic.make_weights(512, w.d, 12)).cuda()
    cw, sw = kq.kq_quantize_weights(W, p)
    tw = kq.kq_sf_tile(sw)

    codes = torch.empty((w.M, w.d // 2), dtype=torch.uint8, device="cuda")
    scales = torch.empty((w.M, w.d // 32), dtype=torch.uint8, device="cuda")
    tiled = torch.empty(((w.M + 127) // 128, w.d // 128, 512), dtype=torch.uint8, device="cuda")
    Y = torch.empty((w.M, 512), dtype=torch.float32, device="cuda")

    def step():
        kq.kq_quantize(x, p, codes, scales)
        kq.kq_sf_tile(scales, tiled)
        kq.kq_gemm_mxfp4(codes, tiled, cw, tw, Y)

    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        step()                                  # eager, on the capture stream
    torch.cuda.current_stream().wait_stream(s)
    torch.cuda.synchronize()
    ref = (codes.clone(), scales.clone(), Y.clone())

    codes.zero_()
    scales.zero_()
    Y.zero_()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        step()
    for _ in range(3):
        g.replay()
    torch.cuda.synchronize()
    assert torch.equal(codes, ref[0]) and torch.equal(scales, ref[1])
    assert torch.equal(Y, ref[2])
    assert np.isfinite(Y.cpu().numpy()).all()
