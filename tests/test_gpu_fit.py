"""Offline fitting of the LU parameters (w4a4_dit_post_b200.fit) on synthetic
FLUX-shaped calibration tokens, judged on held-out tokens of the same
workload.  Needs a B200."""
import numpy as np
import pytest
import torch

import synthetic

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


def _tokens(w, rows):
    raw = synthetic.make_activations(w, rows)
    return torch.from_numpy(raw.view(np.int16)).view(torch.bfloat16).cuda()


def test_fitted_parameters_beat_plain_mxfp4_on_held_out_tokens(kq):
    from w4a4_dit_post_b200 import fit
    w = synthetic.CONFIGS["flux"][0]                          # d = 3072, outliers x100
    x_cal = _tokens(w, np.arange(512))
    x_test = _tokens(w, np.arange(2048, 2560))
    W = torch.from_numpy(synthetic.make_weights(256, w.d, 10)).cuda()
    P, hist = fit.fit_params(x_cal, W, sweeps=1, n_perturb=2, seed=1)
    assert all(b <= a for a, b in zip(hist, hist[1:]))       # coordinate descent never worsens
    ident = torch.from_numpy(np.tile(fit.identity_block(), (w.nb, 1))).cuda()
    hada = torch.from_numpy(np.tile(fit.hadamard_block(), (w.nb, 1))).cuda()
    e_plain = fit.layer_error(x_test, W, ident)
    e_hada = fit.layer_error(x_test, W, hada)
    e_fit = fit.layer_error(x_test, W, P)
    e_rand = fit.layer_error(x_test, W, torch.from_numpy(synthetic.make_params(w.nb, w.seed)).cuda())
    e_sq = _smoothquant_error(kq, w, x_cal, x_test, W, ident)
    print(f"held-out layer error: plain MXFP4 {e_plain:.4f}, SmoothQuant {e_sq:.4f}, "
          f"Hadamard {e_hada:.4f}, fitted {e_fit:.4f}, random {e_rand:.4f}; "
          f"calibration {hist[0]:.4f} -> {hist[-1]:.4f}")
    assert e_fit < 0.9 * e_plain
    assert e_fit < e_sq


def _smoothquant_error(kq, w, x_cal, x_test, W, ident):
    """The same layer with SmoothQuant (alpha = 0.5, scales from the
    calibration tokens): activations x / s through sq_quantize, weights W s
    quantised plainly (identity parameters), FP4 GEMM."""
    inv_s = torch.from_numpy(synthetic.smoothquant_inv_scales(x_cal.float().cpu().numpy())).cuda()
    c, sc = kq.sq_quantize(x_test, inv_s)
    cw, sw = kq.kq_quantize_weights((W / inv_s[None, :]).contiguous(), ident)
    Y = kq.kq_gemm_mxfp4(c, kq.kq_sf_tile(sc), cw, kq.kq_sf_tile(sw))
    ref = x_test.float() @ W.t()
    return float(torch.linalg.norm(Y - ref) / torch.linalg.norm(ref))


def test_layer_error_matches_oracle(kq):
    """fit.layer_error (GPU quantizers, FP4 GEMM and torch's norm) against the
    oracle's fp64 layer error on a 64 x 256 case.  Two checks: given the
    GPU's own codes, the oracle's fp64 evaluation of the same error agrees
    to fp32 accumulation accuracy; and against the oracle's end-to-end value
    (its own quantisation) the difference stays within what the few exempt
    rounding decisions can move it."""
    import oracle.kq_oracle as o
    from w4a4_dit_post_b200 import fit
    w = synthetic.Workload("fit", 64, 256, "bf16", "normal", 0.02, None, 50.0, 2.0, 81)
    raw = synthetic.make_activations(w)
    x = torch.from_numpy(raw.view(np.int16)).view(torch.bfloat16).cuda()
    X = synthetic.f32_from_bf16_bits(raw).astype(np.float64)
    W = synthetic.make_weights(48, w.d, 82)
    Wd = torch.from_numpy(W).cuda()
    for p in (np.tile(fit.identity_block(), (w.nb, 1)), np.tile(fit.hadamard_block(), (w.nb, 1)),
              synthetic.make_params(w.nb, 83)):
        pd = torch.from_numpy(np.ascontiguousarray(p, dtype=np.float32)).cuda()
        e_gpu = fit.layer_error(x, Wd, pd)
        ca, sa = kq.kq_quantize(x, pd)
        cb, sb = kq.kq_quantize_weights(Wd, pd)
        ca, sa, cb, sb = (t.cpu().numpy() for t in (ca, sa, cb, sb))
        ref = X @ W.astype(np.float64).T
        e_same_codes = np.linalg.norm(o.gemm_mxfp4(ca, sa, cb, sb) - ref) / np.linalg.norm(ref)
        e_oracle = o.layer_error(X, W, p)
        print(f"layer error: gpu {e_gpu:.6f}, oracle on gpu codes {e_same_codes:.6f}, oracle {e_oracle:.6f}")
        assert abs(e_gpu - e_same_codes) <= 1e-4 * e_same_codes
        assert abs(e_gpu - e_oracle) <= 2e-3 * e_oracle
