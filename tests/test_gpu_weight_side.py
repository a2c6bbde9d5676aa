"""The weight side of the W4A4 layer on the GPU, and one whole linear layer.

kq_quantize_weights (the folded weights W blockdiag(T_j)^{-1} quantised to
MXFP4) is compared with the oracle like the activation quantizer; then a
layer Y = X W^T is run through both quantizers and the dequantised product is
checked against the fp64 product within the error bound that the MXFP4
rounding rules give.  Needs a B200.
"""
import numpy as np
import pytest
import torch

import oracle.kq_oracle as o
import synthetic
from gpu_util import device_activations, f64, guards_intact, padded_u8, sample_rows
from parity import TOL_REL, compare_codes, reference

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


def check(rep, label):
    print(f"{label}: {rep.counts()}")
    rep.assert_ok(label)


# (N, d): tiny and ragged shapes, then the FLUX.1-schnell layer shapes
# (d x d attention projection, MLP in 3072 -> 12288, MLP out 12288 -> 3072)
SHAPES = [(1, 32), (37, 224), (129, 1152), (3072, 3072), (12288, 3072), (3072, 12288)]


@pytest.mark.parametrize("N,d", SHAPES)
def test_quantize_weights_matches_oracle(kq, N, d):
    p = synthetic.make_params(d // 32, 43)
    W = synthetic.make_weights(N, d, 6)
    codes, cw = padded_u8((N, d // 2))
    scales, sw = padded_u8((N, d // 32))
    kq.kq_quantize_weights(torch.from_numpy(W).cuda(), torch.from_numpy(p).cuda(), codes, scales)
    torch.cuda.synchronize()
    assert guards_intact(cw, N * d // 2) and guards_intact(sw, N * d // 32)
    rows = sample_rows(N, 256, 4)
    ref = o.fold_weights(W[rows].astype(np.float64), p)
    tol = TOL_REL * o.fold_error_scale(W[rows], p)
    check(compare_codes(codes[rows].cpu().numpy(), scales[rows].cpu().numpy(), ref, tol),
          f"weights {N}x{d}")


@pytest.mark.parametrize("N,d", [(300, 1152), (300, 3072), (7, 1024)])
def test_quantize_weights_equals_quantized_fold(kq, N, d):
    """The fused kernel encodes exactly what kq_fold_weights writes: the same
    fp32 evaluation, then the activation encoder on it (sq_quantize with unit
    scales multiplies by 1, exactly).  d = 1152 takes the per-block kernel,
    d = 3072 and 1024 (d / 32 a multiple of 32) the column-stationary one."""
    p = torch.from_numpy(synthetic.make_params(d // 32, 44)).cuda()
    W = torch.from_numpy(synthetic.make_weights(N, d, 8)).cuda()
    c1, s1 = kq.kq_quantize_weights(W, p)
    Wf = kq.kq_fold_weights(W, p)
    c2, s2 = kq.sq_quantize(Wf, torch.ones(d, device="cuda"))
    assert torch.equal(c1, c2) and torch.equal(s1, s2)


@pytest.mark.parametrize("N,d", [(64, 512), (64, 2048)])
def test_quantize_weights_identity_is_plain_mxfp4(kq, N, d):
    W = synthetic.make_weights(N, d, 9)
    p = synthetic.identity_params(d // 32)
    c, s = kq.kq_quantize_weights(torch.from_numpy(W).cuda(), torch.from_numpy(p).cuda())
    c_ref, s_ref = o.quantize_mxfp4(W.astype(np.float64))
    assert np.array_equal(c.cpu().numpy(), c_ref) and np.array_equal(s.cpu().numpy(), s_ref)


def _mxfp4_bound(v, scales):
    """Largest |dequant(quant(v)) - v| the MXFP4 rules allow for values v
    encoded with these scale bytes: half a grid step at r = |v| / 2^e (0.25,
    0.5, 1 in the binades [0, 2), [2, 4), [4, 6]), or |r| - 6 when saturated."""
    e = (scales.astype(np.int64) - 127).repeat(32, axis=1)
    r = np.abs(v) / 2.0 ** e
    half = np.where(r < 2, 0.25, np.where(r < 4, 0.5, 1.0))
    return np.where(r > 6, r - 6, half) * 2.0 ** e


def _layer(kq, p):
    """X (512 tokens of the FLUX d = 3072 workload), W (256 x 3072) and both
    operands through the CUDA quantizers with parameters p."""
    w = synthetic.CONFIGS["flux"][0]
    X = f64(synthetic.make_activations(w, np.arange(512)), w.dtype)
    W = synthetic.make_weights(256, w.d, 10).astype(np.float64)   # fp32 values, exact
    pd = torch.from_numpy(p).cuda()
    xd = device_activations(w)[:512].contiguous()
    cx, sx = kq.kq_quantize(xd, pd)
    cw, sw = kq.kq_quantize_weights(torch.from_numpy(W.astype(np.float32)).cuda(), pd)
    Xq = kq.kq_dequant(cx, sx).cpu().numpy().astype(np.float64)
    Wq = kq.kq_dequant(cw, sw).cpu().numpy().astype(np.float64)
    return X, W, Xq, Wq, sx.cpu().numpy(), sw.cpu().numpy()


def test_linear_layer_error_bound(kq):
    """Y = X W^T with both operands through the CUDA quantizers.  The fold
    makes X' W'^T = X W^T (X' = T x per token, W' = W T^{-1}), so the
    dequantised product differs from the fp64 product only by the two
    quantisation errors: |Y_q - Y| <= |dX| |W'|^T + |X'| |dW|^T + |dX| |dW|^T
    elementwise, with |dX| and |dW| bounded by the rounding rules at the
    scales the kernels chose, plus the fp32 evaluation error of the transforms."""
    w = synthetic.CONFIGS["flux"][0]
    p = synthetic.make_params(w.nb, w.seed)
    X, W, Xq, Wq, sx, sw = _layer(kq, p)
    Xt, tol_x = reference(X, params=p)
    Wt = o.fold_weights(W, p)
    tol_w = TOL_REL * o.fold_error_scale(W, p)
    dX = _mxfp4_bound(np.abs(Xt) + tol_x, sx) + tol_x
    dW = _mxfp4_bound(np.abs(Wt) + tol_w, sw) + tol_w
    Y = X @ W.T
    Yq = Xq @ Wq.T
    bound = dX @ np.abs(Wt).T + np.abs(Xt) @ dW.T + dX @ dW.T
    assert np.all(np.abs(Yq - Y) <= bound * (1 + 1e-9) + 1e-9 * np.abs(Y).max())


def test_linear_layer_fold_matters(kq):
    """With moderate parameters (the synthetic draw with a, b scaled by 0.3
    and u -> u^0.3) the quantised layer's error is the quantisation error of
    a 4-bit format, and half or less of what the same activation codes give
    against weights that were not folded.  (With the full synthetic draw the
    transforms are poorly conditioned and the layer error is about 1.06
    against 0.20 for plain MXFP4: random parameters are not fitted ones.)"""
    w = synthetic.CONFIGS["flux"][0]
    p = synthetic.make_params(w.nb, w.seed).reshape(w.nb, 5, 3).copy()
    p[:, :, 0] *= 0.3
    p[:, :, 1] *= 0.3
    p[:, :, 2] = p[:, :, 2] ** 0.3
    p = np.ascontiguousarray(p.reshape(w.nb, 15), dtype=np.float32)
    X, W, Xq, Wq, _, _ = _layer(kq, p)
    Y = X @ W.T
    rel = np.linalg.norm(Xq @ Wq.T - Y) / np.linalg.norm(Y)
    cu, su = kq.kq_quantize_weights(torch.from_numpy(W.astype(np.float32)).cuda(),
                                    torch.from_numpy(synthetic.identity_params(w.nb)).cuda())
    Wu = kq.kq_dequant(cu, su).cpu().numpy().astype(np.float64)
    rel_unfolded = np.linalg.norm(Xq @ Wu.T - Y) / np.linalg.norm(Y)
    print(f"linear layer 512x3072 @ 3072x256: rel error {rel:.4f}, weights not folded {rel_unfolded:.4f}")
    assert rel < 0.3 and rel_unfolded > 1.5 * rel
