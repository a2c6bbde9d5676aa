"""The centring variant: per-token offsets out before the transform
(kq_row_sum, kq_quantize_centered) and back in the GEMM's epilogue
(kq_gemm_mxfp4_rank1), against the oracle; and its effect on the error of
a FLUX-shaped layer whose tokens carry a per-token mean.  Needs a B200."""
import numpy as np
import pytest
import torch

import oracle.kq_oracle as o
import synthetic
from gpu_util import f64
from parity import TOL_REL, compare_codes

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


def _bf16(raw):
    return torch.from_numpy(raw.view(np.int16)).view(torch.bfloat16).cuda()


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
@pytest.mark.parametrize("M,d", [(1, 32), (257, 1152), (4608, 3072)])
def test_row_sum(kq, M, d, dtype):
    w = synthetic.Workload("rs", M, d, dtype, "normal", 0.01, None, 100.0, 4.0, 61)
    raw = synthetic.make_activations(w)
    x = _bf16(raw) if dtype == "bf16" else torch.from_numpy(raw).cuda()
    xs = f64(raw, dtype)
    got = kq.kq_row_sum(x, 1.0 / d).cpu().numpy().astype(np.float64)
    ref = o.row_sum(xs, 1.0 / d)
    tol = d * 2.0 ** -23 * o.row_sum(np.abs(xs), 1.0 / d)
    assert np.all(np.abs(got - ref) <= tol)


@pytest.mark.parametrize("M,d", [(3, 64), (257, 1152), (1031, 3072)])
def test_quantize_centered_matches_oracle(kq, M, d):
    w = synthetic.Workload("cq", M, d, "bf16", "normal", 0.01, None, 100.0, 4.0, 62)
    raw = synthetic.make_activations(w)
    x = f64(raw, "bf16")
    p = synthetic.make_params(w.nb, 62)
    mu = o.row_sum(x, 1.0 / d).astype(np.float32)             # the same offsets for both sides
    codes, scales = kq.kq_quantize_centered(_bf16(raw), torch.from_numpy(p).cuda(), torch.from_numpy(mu).cuda())
    # the oracle's centred quantizer gives the expected codes and scales; the
    # exemptions come from its transformed values and their fp32 tolerance
    c_ref, s_ref = o.quantize_centered(x, p, mu)
    xc = x - mu.astype(np.float64)[:, None]
    y_ref = o.transform(xc, p)
    tol = TOL_REL * o.error_scale(xc, p)
    rep = compare_codes(codes.cpu().numpy(), scales.cpu().numpy(), y_ref, tol, ref=(c_ref, s_ref))
    print(f"centred {M}x{d}: {rep.counts()}")
    rep.assert_ok(f"centred {M}x{d}")


def test_gemm_rank1_matches_oracle(kq):
    rng = np.random.default_rng(63)
    M, N, K = 200, 136, 384
    ca = rng.integers(0, 256, size=(M, K // 2), dtype=np.uint8)
    cb = rng.integers(0, 256, size=(N, K // 2), dtype=np.uint8)
    sa = rng.integers(120, 134, size=(M, K // 32), dtype=np.uint8)
    sb = rng.integers(120, 134, size=(N, K // 32), dtype=np.uint8)
    mu = rng.normal(0, 4, size=M).astype(np.float32)
    wsum = rng.normal(0, 1, size=N).astype(np.float32)
    t = lambda a: torch.from_numpy(np.ascontiguousarray(a)).cuda()
    Y = kq.kq_gemm_mxfp4_rank1(t(ca), kq.kq_sf_tile(t(sa)), t(cb), kq.kq_sf_tile(t(sb)), t(mu), t(wsum))
    ref = o.gemm_mxfp4_rank1(ca, sa, cb, sb, mu, wsum)
    tol = (K / 64 + 64) * 2.0 ** -23 * o.gemm_error_scale(ca, sa, cb, sb) + \
        2.0 ** -22 * (np.abs(np.outer(mu, wsum)) + np.abs(ref))
    assert np.all(np.abs(Y.cpu().numpy().astype(np.float64) - ref) <= tol)


def test_centring_lowers_the_layer_error(kq):
    """FLUX-shaped tokens carry a per-token mean N(0, 4) on top of N(0, 1):
    with the offset out of the quantised operand the layer error drops."""
    w = synthetic.CONFIGS["flux"][0]
    raw = synthetic.make_activations(w, np.arange(512))
    x = _bf16(raw)
    X = f64(raw, w.dtype)
    W = torch.from_numpy(synthetic.make_weights(256, w.d, 10)).cuda()
    Y = X @ W.cpu().numpy().astype(np.float64).T
    errs = {}
    for name, p in (("identity", synthetic.identity_params(w.nb)),
                    ("hadamard", np.tile(np.array([-1.0, 0.5 ** 0.5, 0.5 ** 0.5] * 5, dtype=np.float32),
                                         (w.nb, 1)))):
        pd = torch.from_numpy(p).cuda()
        cw, sw = kq.kq_quantize_weights(W, pd)
        tw = kq.kq_sf_tile(sw)
        c, s = kq.kq_quantize(x, pd)
        Yp = kq.kq_gemm_mxfp4(c, kq.kq_sf_tile(s), cw, tw).cpu().numpy().astype(np.float64)
        mu = kq.kq_row_sum(x, 1.0 / w.d)
        wsum = kq.kq_row_sum(W, 1.0)
        cc, sc = kq.kq_quantize_centered(x, pd, mu)
        Yc = kq.kq_gemm_mxfp4_rank1(cc, kq.kq_sf_tile(sc), cw, tw, mu, wsum).cpu().numpy().astype(np.float64)
        errs[name] = (np.linalg.norm(Yp - Y) / np.linalg.norm(Y), np.linalg.norm(Yc - Y) / np.linalg.norm(Y))
    print("layer error (plain, centred):", {k: tuple(round(v, 4) for v in e) for k, e in errs.items()})
    for plain, centred in errs.values():
        assert centred < plain
