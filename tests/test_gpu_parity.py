"""Parity of the CUDA path with the CPU oracle (needs a B200).

Every call goes through the C ABI (via the thin binding).  Small cases are
compared element by element; the full-size workloads run in the same launch
configuration the bench times and are compared on sampled rows.
"""
import numpy as np
import pytest
import torch

import oracle.kq_oracle as o
import synthetic
from golden_cases import hand_blocks
from gpu_util import device_activations, f64, guards_intact, padded_u8, sample_rows, to_device
from parity import compare_codes, compare_transform, reference

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


def params_dev(nb, seed):
    p = synthetic.make_params(nb, seed)
    return p, torch.from_numpy(p).cuda()


def check(rep, label):
    """No mismatch outside the exempt decisions, exemptions within budget;
    the counts are printed and carried by the failure message."""
    print(f"{label}: {rep.counts()}")
    rep.assert_ok(label)


# ---------------------------------------------------------------------------
# small shapes, every element
# ---------------------------------------------------------------------------
# (13, 3072) and (1031, 1024) run the kernel compiled for 32-block column groups
# on a row count that ends inside a tile (8 rows per tile)
SMALL = [(1, 32), (3, 64), (7, 96), (129, 96), (256, 1152), (300, 160), (1031, 224), (13, 3072),
         (1031, 1024)]


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
@pytest.mark.parametrize("M,d", SMALL)
def test_quantize_small(kq, M, d, dtype):
    w = synthetic.Workload("small", M, d, dtype, "normal", 0.05, None, 40.0, 2.0, 17)
    raw = synthetic.make_activations(w)
    x = f64(raw, dtype)
    p, pd = params_dev(w.nb, 5)
    xd = to_device(raw, dtype)
    codes, cw = padded_u8((M, d // 2))
    scales, sw = padded_u8((M, d // 32))
    kq.kq_quantize(xd, pd, codes, scales)
    torch.cuda.synchronize()
    assert guards_intact(cw, M * d // 2) and guards_intact(sw, M * d // 32)
    y_ref, tol = reference(x, params=p)
    check(compare_codes(codes.cpu().numpy(), scales.cpu().numpy(), y_ref, tol),
          f"kq {M}x{d} {dtype}")
    y = kq.kq_transform(xd, pd)
    check(compare_transform(y.cpu().numpy(), y_ref, tol), f"transform {M}x{d} {dtype}")


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
@pytest.mark.parametrize("M,d", [(1, 32), (129, 96), (256, 1152)])
def test_smoothquant_small(kq, M, d, dtype):
    w = synthetic.Workload("small", M, d, dtype, "normal", 0.05, None, 40.0, 2.0, 18)
    raw = synthetic.make_activations(w)
    x = f64(raw, dtype)
    inv_s = synthetic.smoothquant_inv_scales(x.astype(np.float32))
    codes, scales = kq.sq_quantize(to_device(raw, dtype), torch.from_numpy(inv_s).cuda())
    y_ref, tol = reference(x, inv_s=inv_s)
    check(compare_codes(codes.cpu().numpy(), scales.cpu().numpy(), y_ref, tol), f"sq {M}x{d}")


# ---------------------------------------------------------------------------
# the pages' workload shapes at full size (sampled rows)
# ---------------------------------------------------------------------------
FULL = synthetic.workloads(["tiny", "pixart", "sana", "flux"])


@pytest.mark.parametrize("w", FULL, ids=lambda w: w.key)
def test_quantize_workloads(kq, w):
    xd = device_activations(w)
    p, pd = params_dev(w.nb, w.seed)
    codes, scales = kq.kq_quantize(xd, pd)
    torch.cuda.synchronize()
    rows = sample_rows(w.M, 512, w.seed)
    x = f64(synthetic.make_activations(w, rows), w.dtype)
    y_ref, tol = reference(x, params=p)
    check(compare_codes(codes[rows].cpu().numpy(), scales[rows].cpu().numpy(), y_ref, tol),
          f"kq {w.key} rows={rows.size}")
    yd = kq.kq_transform(xd[torch.from_numpy(rows).cuda()].contiguous(), pd)
    check(compare_transform(yd.cpu().numpy(), y_ref, tol), f"transform {w.key}")
    inv_s = synthetic.smoothquant_inv_scales(x.astype(np.float32))
    sc, ss = kq.sq_quantize(xd, torch.from_numpy(inv_s).cuda())
    y_sq, tol_sq = reference(x, inv_s=inv_s)
    check(compare_codes(sc[rows].cpu().numpy(), ss[rows].cpu().numpy(), y_sq, tol_sq),
          f"sq {w.key}")


SWEEP = synthetic.workloads(["sweep"])


@pytest.mark.parametrize("w", SWEEP, ids=lambda w: w.key)
def test_quantize_sweep(kq, w):
    xd = device_activations(w)
    p, pd = params_dev(w.nb, w.seed)
    codes, scales = kq.kq_quantize(xd, pd)
    torch.cuda.synchronize()
    rows = sample_rows(w.M, 256, w.seed)
    x = f64(synthetic.make_activations(w, rows), w.dtype)
    y_ref, tol = reference(x, params=p)
    check(compare_codes(codes[rows].cpu().numpy(), scales[rows].cpu().numpy(), y_ref, tol),
          f"kq {w.key}")
    del xd, codes, scales
    torch.cuda.empty_cache()


# ---------------------------------------------------------------------------
# hand-worked blocks (tests/golden/kq_hand_blocks.txt), bit for bit: every
# decision there is an exact tie or far from a rounding or scale boundary
# ---------------------------------------------------------------------------
def _golden_input(hb, dtype):
    x = torch.from_numpy(hb.x.astype(np.float32)).cuda()
    return x.to(torch.bfloat16) if dtype == "bf16" else x


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_golden_hand_blocks(kq, dtype):
    for hb in hand_blocks():
        codes, scales = kq.kq_quantize(_golden_input(hb, dtype), torch.from_numpy(hb.params).cuda())
        assert int(scales.cpu()[0, 0]) == hb.scale, hb.name
        assert np.array_equal(codes.cpu().numpy(), hb.codes), hb.name


def test_golden_hand_blocks_tensor_core(kq):
    for hb in hand_blocks():
        codes, scales = kq.kq_quantize_tc(_golden_input(hb, "bf16"), torch.from_numpy(hb.params).cuda())
        assert int(scales.cpu()[0, 0]) == hb.scale, hb.name
        assert np.array_equal(codes.cpu().numpy(), hb.codes), hb.name


def test_golden_hand_blocks_smoothquant_identity(kq):
    """With unit scales SmoothQuant is plain MXFP4: the identity-transform blocks."""
    ones = torch.ones(32, device="cuda")
    for hb in hand_blocks():
        if not np.array_equal(hb.params, np.tile(np.array([0, 0, 1], np.float32), 5).reshape(1, 15)):
            continue
        codes, scales = kq.sq_quantize(_golden_input(hb, "f32"), ones)
        assert int(scales.cpu()[0, 0]) == hb.scale, hb.name
        assert np.array_equal(codes.cpu().numpy(), hb.codes), hb.name


# ---------------------------------------------------------------------------
# exact paths: the transform is exact, so every decision must match
# ---------------------------------------------------------------------------
def edge_block_values():
    mids = [0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0]
    vals = [6.0, -7.9, 7.0, 6.5, -6.0, 0.0, -0.0, -0.1, 0.1, 1e-30, -1e-30]
    for m in mids:
        vals += [m, -m, m * (1 + 2 ** -20), m * (1 - 2 ** -20)]
    return np.array(vals, dtype=np.float32)


@pytest.mark.parametrize("scale_pow", [0, -20, 40, -126, 100])
def test_exact_encoding_identity(kq, scale_pow):
    """Identity parameters make y = x exactly, so kq_quantize is MXFP4 of the
    input: checks rounding (ties, saturation, sign of zero) and the scale."""
    v = edge_block_values()
    d = 32 * int(np.ceil(v.size / 32))
    x = np.zeros((3, d), dtype=np.float32)
    x[0, :v.size] = v
    x[1, :v.size] = v[::-1]
    x[2] = np.random.default_rng(1).uniform(-8, 8, d).astype(np.float32)
    x = np.ldexp(x, scale_pow).astype(np.float32)
    p = synthetic.identity_params(d // 32)
    codes, scales = kq.kq_quantize(torch.from_numpy(x).cuda(), torch.from_numpy(p).cuda())
    rep = compare_codes(codes.cpu().numpy(), scales.cpu().numpy(), x.astype(np.float64),
                        np.zeros_like(x, dtype=np.float64), exact=True)
    check(rep, f"identity 2^{scale_pow}")


@pytest.mark.parametrize("w", synthetic.workloads(["tiny", "pixart", "sana", "flux"]), ids=lambda w: w.key)
def test_smoothquant_bit_exact_fp32(kq, w):
    """SmoothQuant's transform is one multiplication, so the oracle can take
    every decision in the kernel's precision: y = fl32(x * inv_s) (an IEEE
    single product in NumPy), then the oracle's MXFP4 encoding.  Codes and
    scales must match bit for bit, with no exemptions."""
    xd = device_activations(w)
    rows = sample_rows(w.M, 512, w.seed)
    x32 = f64(synthetic.make_activations(w, rows), w.dtype).astype(np.float32)
    inv_s = synthetic.smoothquant_inv_scales(x32)
    codes, scales = kq.sq_quantize(xd, torch.from_numpy(inv_s).cuda())
    y32 = (x32 * inv_s[None, :]).astype(np.float64)
    c_ref, s_ref = o.quantize_mxfp4(y32)
    assert np.array_equal(scales[rows].cpu().numpy(), s_ref)
    assert np.array_equal(codes[rows].cpu().numpy(), c_ref)


def test_exact_encoding_smoothquant_unit(kq):
    w = synthetic.Workload("u", 512, 1024, "bf16", "normal", 0.01, None, 100.0, 3.0, 23)
    raw = synthetic.make_activations(w)
    x = f64(raw, "bf16")
    ones = np.ones(w.d, dtype=np.float32)
    codes, scales = kq.sq_quantize(to_device(raw, "bf16"), torch.from_numpy(ones).cuda())
    c_ref, s_ref = o.quantize_mxfp4(x)
    assert np.array_equal(scales.cpu().numpy(), s_ref)
    assert np.array_equal(codes.cpu().numpy(), c_ref)


def test_exact_power_of_two_diagonal(kq):
    """u = 2^k, a = b = 0: T is a diagonal of powers of two, exact in fp32."""
    nb = 12
    rng = np.random.default_rng(8)
    p = np.zeros((nb, 5, 3), dtype=np.float32)
    p[:, :, 2] = np.ldexp(1.0, rng.integers(-3, 4, size=(nb, 5)))
    p = p.reshape(nb, 15)
    w = synthetic.Workload("p2", 333, 32 * nb, "bf16", "normal", 0.02, None, 50.0, 1.0, 24)
    raw = synthetic.make_activations(w)
    x = f64(raw, "bf16")
    codes, scales = kq.kq_quantize(to_device(raw, "bf16"), torch.from_numpy(p).cuda())
    c_ref, s_ref = o.kq_quantize(x, p)
    assert np.array_equal(scales.cpu().numpy(), s_ref)
    assert np.array_equal(codes.cpu().numpy(), c_ref)


def test_zero_nan_inf_blocks(kq):
    d = 128
    x = np.random.default_rng(2).normal(size=(4, d)).astype(np.float32)
    x[0, :32] = 0.0                 # block (0,0): amax 0 -> byte 0, codes 0
    x[1, 40] = np.nan               # block (1,1): NaN -> 0xFF
    x[2, 70] = np.inf               # block (2,2): Inf -> 0xFF
    x[3, 100] = -np.inf
    for use_kq in (True, False):
        xd = torch.from_numpy(x).cuda()
        if use_kq:
            p = synthetic.make_params(d // 32, 3)
            codes, scales = kq.kq_quantize(xd, torch.from_numpy(p).cuda())
        else:
            codes, scales = kq.sq_quantize(xd, torch.ones(d, device="cuda"))
        s = scales.cpu().numpy()
        assert s[0, 0] == 0 and not codes.cpu().numpy()[0, :16].any()
        assert s[1, 1] == 255 and s[2, 2] == 255 and s[3, 3] == 255
        assert s[1, 0] != 255 and s[2, 0] != 255


# ---------------------------------------------------------------------------
# support kernels
# ---------------------------------------------------------------------------
def test_expand_params(kq):
    nb = 40
    p, pd = params_dev(nb, 31)
    T = kq.kq_expand_params(pd).cpu().numpy().astype(np.float64)
    T_ref = o.expand_params(p)
    mag = o.expand_magnitude(p)
    assert np.all(np.abs(T - T_ref) <= 1e-6 * mag)


@pytest.mark.parametrize("N,d", [(1, 32), (24, 128), (384, 1152), (5, 3072), (7, 12288), (3072, 3072)])
def test_fold_weights(kq, N, d):
    p, pd = params_dev(d // 32, 41)
    W = synthetic.make_weights(N, d, 5)
    Wd = torch.from_numpy(W).cuda()
    out = kq.kq_fold_weights(Wd, pd).cpu().numpy().astype(np.float64)
    rows = sample_rows(N, 256, 3)
    ref = o.fold_weights(W[rows].astype(np.float64), p)
    tol = 1e-5 * o.fold_error_scale(W[rows], p)
    assert np.all(np.abs(out[rows] - ref) <= tol)
    # in place gives the same bits
    kq.kq_fold_weights(Wd, pd, Wd)
    assert np.array_equal(Wd.cpu().numpy(), out.astype(np.float32))


def test_dequant_exact(kq):
    rng = np.random.default_rng(12)
    M, d = 77, 256
    codes = rng.integers(0, 256, size=(M, d // 2), dtype=np.uint8)
    scales = rng.integers(0, 253, size=(M, d // 32), dtype=np.uint8)
    scales[0, 0] = 0
    scales[1, 1] = 255
    scales[2, 2] = 252
    out = kq.kq_dequant(torch.from_numpy(codes).cuda(), torch.from_numpy(scales).cuda()).cpu().numpy()
    ref = o.dequant(codes, scales)
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(out), nan)
    assert np.array_equal(out[~nan].astype(np.float64), ref[~nan])


def test_dequant_roundtrip_flux_rows(kq):
    w = synthetic.CONFIGS["flux"][0]
    rows = np.arange(64)
    raw = synthetic.make_activations(w, rows)
    p, pd = params_dev(w.nb, w.seed)
    codes, scales = kq.kq_quantize(to_device(raw, "bf16"), pd)
    deq = kq.kq_dequant(codes, scales).cpu().numpy()
    assert np.array_equal(deq.astype(np.float64), o.dequant(codes.cpu().numpy(), scales.cpu().numpy()))


# ---------------------------------------------------------------------------
# launch behaviour
# ---------------------------------------------------------------------------
def test_side_stream_and_determinism(kq):
    w = synthetic.CONFIGS["flux"][0]
    xd = device_activations(w)
    p, pd = params_dev(w.nb, w.seed)
    c1, s1 = kq.kq_quantize(xd, pd)
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        c2, s2 = kq.kq_quantize(xd, pd)
    torch.cuda.synchronize()
    assert torch.equal(c1, c2) and torch.equal(s1, s2)


def test_max_width(kq):
    M, d = 64, 32768
    w = synthetic.Workload("wide", M, d, "bf16", "normal", 0.01, None, 50.0, 0.0, 29)
    raw = synthetic.make_activations(w)
    p, pd = params_dev(w.nb, 2)
    codes, scales = kq.kq_quantize(to_device(raw, "bf16"), pd)
    rows = np.arange(0, M, 9)
    y_ref, tol = reference(f64(raw[rows], "bf16"), params=p)
    check(compare_codes(codes[rows].cpu().numpy(), scales[rows].cpu().numpy(), y_ref, tol), "d=32768")
    inv_s = np.full(d, 0.5, dtype=np.float32)
    sc, ss = kq.sq_quantize(to_device(raw, "bf16"), torch.from_numpy(inv_s).cuda())
    c_ref, s_ref = o.sq_quantize(f64(raw, "bf16"), inv_s)
    assert np.array_equal(ss.cpu().numpy(), s_ref) and np.array_equal(sc.cpu().numpy(), c_ref)


def test_empty_input(kq):
    x = torch.empty((0, 64), dtype=torch.bfloat16, device="cuda")
    p = torch.zeros((2, 15), device="cuda")
    codes, scales = kq.kq_quantize(x, p)
    assert codes.shape == (0, 32) and scales.shape == (0, 2)


# ---------------------------------------------------------------------------
# the tensor-core formulation (kq_quantize_tc): same contract
# ---------------------------------------------------------------------------
@pytest.mark.parametrize("M,d", [(1, 32), (129, 96), (200, 1152), (1031, 224), (333, 5600)])
def test_tensor_core_small(kq, M, d):
    w = synthetic.Workload("tcs", M, d, "bf16", "normal", 0.05, None, 40.0, 2.0, 19)
    raw = synthetic.make_activations(w)
    p, pd = params_dev(w.nb, 6)
    codes, cw = padded_u8((M, d // 2))
    scales, sw = padded_u8((M, d // 32))
    kq.kq_quantize_tc(to_device(raw, "bf16"), pd, codes, scales)
    torch.cuda.synchronize()
    assert guards_intact(cw, M * d // 2) and guards_intact(sw, M * d // 32)
    y_ref, tol = reference(f64(raw, "bf16"), params=p)
    check(compare_codes(codes.cpu().numpy(), scales.cpu().numpy(), y_ref, tol), f"tc {M}x{d}")


@pytest.mark.parametrize("w", synthetic.workloads(["pixart", "sana", "flux"]), ids=lambda w: w.key)
def test_tensor_core_workloads(kq, w):
    xd = device_activations(w)
    p, pd = params_dev(w.nb, w.seed)
    codes, scales = kq.kq_quantize_tc(xd, pd)
    torch.cuda.synchronize()
    rows = sample_rows(w.M, 384, w.seed)
    y_ref, tol = reference(f64(synthetic.make_activations(w, rows), w.dtype), params=p)
    check(compare_codes(codes[rows].cpu().numpy(), scales[rows].cpu().numpy(), y_ref, tol), f"tc {w.key}")


def test_tensor_core_exact_identity(kq):
    w = synthetic.Workload("tci", 300, 1024, "bf16", "normal", 0.02, None, 50.0, 1.0, 26)
    raw = synthetic.make_activations(w)
    p = synthetic.identity_params(w.nb)
    codes, scales = kq.kq_quantize_tc(to_device(raw, "bf16"), torch.from_numpy(p).cuda())
    c_ref, s_ref = o.quantize_mxfp4(f64(raw, "bf16"))
    assert np.array_equal(scales.cpu().numpy(), s_ref)
    assert np.array_equal(codes.cpu().numpy(), c_ref)
