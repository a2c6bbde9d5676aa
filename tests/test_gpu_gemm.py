"""The W4A4 GEMM on the quantised operands (kq_sf_tile + kq_gemm_mxfp4, and
kq_gemm_mxfp4_bf16)
against the oracle.  Operand codes and scales are seeded or come from the
oracle's own quantizers; the GPU computes Y from them.  Needs a B200.
"""
import numpy as np
import pytest
import torch

import oracle.kq_oracle as o
import synthetic
from gpu_util import f64

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


def _cuda(a):
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


def _operands(rng, rows, K, scale_lo, scale_hi):
    codes = rng.integers(0, 256, size=(rows, K // 2), dtype=np.uint8)
    scales = rng.integers(scale_lo, scale_hi + 1, size=(rows, K // 32), dtype=np.uint8)
    return codes, scales


def _gemm(kq, ca, sa, cb, sb):
    ta = kq.kq_sf_tile(_cuda(sa))
    tb = kq.kq_sf_tile(_cuda(sb))
    Y = kq.kq_gemm_mxfp4(_cuda(ca), ta, _cuda(cb), tb)
    torch.cuda.synchronize()
    return Y.cpu().numpy().astype(np.float64)


@pytest.mark.parametrize("R,K", [(1, 128), (130, 256), (4608, 3072)])
def test_sf_tile_matches_oracle(kq, R, K):
    rng = np.random.default_rng(R + K)
    s = rng.integers(0, 256, size=(R, K // 32), dtype=np.uint8)
    t = kq.kq_sf_tile(_cuda(s)).cpu().numpy()
    assert np.array_equal(t, o.sf_tile(s))


@pytest.mark.parametrize("M,N,K", [(128, 128, 128), (200, 72, 384), (256, 384, 1024), (1, 1, 128), (300, 1029, 256)])
def test_gemm_unit_scales_is_exact(kq, M, N, K):
    """Unit scales: every product is a multiple of 1/4 below 36 and every sum
    fits fp32 exactly, so any accumulation order gives the oracle's bits.  A
    misplaced code, scale or row shows up as a wrong value."""
    rng = np.random.default_rng(M * 7 + N * 3 + K)
    ca, sa = _operands(rng, M, K, 127, 127)
    cb, sb = _operands(rng, N, K, 127, 127)
    Y = _gemm(kq, ca, sa, cb, sb)
    assert np.array_equal(Y, o.gemm_mxfp4(ca, sa, cb, sb))


@pytest.mark.parametrize("M,N,K", [(128, 128, 256), (200, 72, 384), (384, 256, 3072)])
def test_gemm_scaled_operands(kq, M, N, K):
    """Scales 2^-10 .. 2^10 per 32-element block (each block of each row its
    own): within fp32 accumulation error of the fp64 product."""
    rng = np.random.default_rng(M + 11 * N + K)
    ca, sa = _operands(rng, M, K, 117, 137)
    cb, sb = _operands(rng, N, K, 117, 137)
    Y = _gemm(kq, ca, sa, cb, sb)
    ref = o.gemm_mxfp4(ca, sa, cb, sb)
    tol = (K / 64 + 64) * 2.0 ** -23 * o.gemm_error_scale(ca, sa, cb, sb)
    assert np.all(np.abs(Y - ref) <= tol)


def test_gemm_on_quantized_layer(kq):
    """A FLUX.1-schnell-shaped layer: 512 tokens x 3072 channels through the
    oracle's KroQuant quantizer, 256 x 3072 weights through the oracle's
    weight quantizer (folded), then the GPU GEMM on those codes."""
    w = synthetic.CONFIGS["flux"][0]
    X = f64(synthetic.make_activations(w, np.arange(512)), w.dtype)
    W = synthetic.make_weights(256, w.d, 10).astype(np.float64)
    p = synthetic.make_params(w.nb, w.seed)
    ca, sa = o.kq_quantize(X, p)
    cb, sb = o.quantize_weights(W, p)
    Y = _gemm(kq, ca, sa, cb, sb)
    ref = o.gemm_mxfp4(ca, sa, cb, sb)
    tol = (w.d / 64 + 64) * 2.0 ** -23 * o.gemm_error_scale(ca, sa, cb, sb)
    assert np.all(np.abs(Y - ref) <= tol)


# ---------------------------------------------------------------------------
# bf16 output (kq_gemm_mxfp4_bf16): the same fp32 sums, rounded to nearest even
# ---------------------------------------------------------------------------
def _gemm_bf16(kq, ca, sa, cb, sb):
    ta = kq.kq_sf_tile(_cuda(sa))
    tb = kq.kq_sf_tile(_cuda(sb))
    Y = kq.kq_gemm_mxfp4_bf16(_cuda(ca), ta, _cuda(cb), tb)
    torch.cuda.synchronize()
    return Y.cpu()


def _bf16_bits(t):
    return t.contiguous().view(torch.int16).numpy()


@pytest.mark.parametrize("M,N,K", [(128, 128, 128), (200, 72, 384), (256, 384, 1024), (1, 1, 128), (300, 1029, 256)])
def test_gemm_bf16_unit_scales_is_exact(kq, M, N, K):
    """Unit scales: the fp32 sum is the oracle's exact value, so Y is that value
    rounded to bf16 (torch's round-to-nearest-even conversion), bit for bit.
    N = 72 and 1029 take the row-store path (N not a multiple of 8)."""
    rng = np.random.default_rng(M * 7 + N * 3 + K)
    ca, sa = _operands(rng, M, K, 127, 127)
    cb, sb = _operands(rng, N, K, 127, 127)
    Y = _gemm_bf16(kq, ca, sa, cb, sb)
    ref = torch.from_numpy(o.gemm_mxfp4(ca, sa, cb, sb).astype(np.float32)).to(torch.bfloat16)
    assert np.array_equal(_bf16_bits(Y), _bf16_bits(ref))


@pytest.mark.parametrize("M,N,K", [(128, 128, 256), (200, 72, 384), (384, 256, 3072), (4608, 3072, 3072)])
def test_gemm_bf16_matches_fp32_gemm(kq, M, N, K):
    """Scales 2^-10 .. 2^10: the bf16 output is the fp32 GEMM's output rounded
    to bf16, bit for bit (same MMAs, same accumulation), and within the fp32
    accumulation bound plus half a bf16 unit of the fp64 product."""
    rng = np.random.default_rng(M + 11 * N + K)
    ca, sa = _operands(rng, M, K, 117, 137)
    cb, sb = _operands(rng, N, K, 117, 137)
    Y16 = _gemm_bf16(kq, ca, sa, cb, sb)
    Y32 = torch.from_numpy(_gemm(kq, ca, sa, cb, sb).astype(np.float32))
    assert np.array_equal(_bf16_bits(Y16), _bf16_bits(Y32.to(torch.bfloat16)))
    if M * N <= 1 << 20:
        ref = o.gemm_mxfp4(ca, sa, cb, sb)
        tol = (K / 64 + 64) * 2.0 ** -23 * o.gemm_error_scale(ca, sa, cb, sb)
        err = np.abs(Y16.to(torch.float64).numpy() - ref)
        assert np.all(err <= tol + 2.0 ** -8 * (np.abs(ref) + tol))


@pytest.mark.parametrize("M,d", [(1, 128), (200, 1152), (1031, 3072), (4608, 3072)])
def test_quantize_with_tiled_scales(kq, M, d):
    """kq_quantize_sf_tiled writes the codes of kq_quantize and the scale
    blocks kq_sf_tile makes from kq_quantize's scales (rows past M untouched)."""
    w = synthetic.Workload("sft", M, d, "bf16", "normal", 0.01, None, 50.0, 2.0, 23)
    raw = synthetic.make_activations(w)
    x = torch.from_numpy(raw.view(np.int16)).view(torch.bfloat16).cuda()
    p = torch.from_numpy(synthetic.make_params(w.nb, 23)).cuda()
    c1, s1 = kq.kq_quantize(x, p)
    t1 = kq.kq_sf_tile(s1)
    c2 = torch.empty_like(c1)
    t2 = torch.zeros_like(t1)
    kq.kq_quantize_sf_tiled(x, p, c2, t2)
    torch.cuda.synchronize()
    assert torch.equal(c1, c2) and torch.equal(t1, t2)


# ---------------------------------------------------------------------------
# the persistent schedule: more output tiles than CTAs or CTA pairs, so they
# walk two or more tiles and the stage ring and the accumulator hand-back
# carry over from one tile to the next.  2176 x 2304: the single-CTA kernel,
# 306 tiles of 128 x 128 over 296 CTAs; 2048 x 2560 and 4608 x 3072: the pair
# kernel, 80 and 216 tiles of 256 x 256 over 74 pairs; 4608 x 2880: 270
# tiles of 256 x 192 (two accumulators)
# ---------------------------------------------------------------------------
MULTI_TILE = [(2048, 2560, 1024), (2176, 2304, 512), (4608, 3072, 3072), (4608, 2880, 1024)]


def _sampled_rows(M, n, seed):
    if M <= n:
        return np.arange(M)
    rng = np.random.default_rng([seed, M])
    return np.unique(np.concatenate([[0, M - 1], rng.choice(M, n, replace=False)]))


@pytest.mark.parametrize("M,N,K", MULTI_TILE)
def test_gemm_persistent_unit_scales_exact(kq, M, N, K):
    """Unit scales keep every sum exact in fp32 (|sum| <= 36 K, a multiple of
    1/4: at most 19 significant bits here), so each sampled row must equal
    the oracle bit for bit, whichever CTA and tile produced it."""
    rng = np.random.default_rng(M + N + K)
    ca, sa = _operands(rng, M, K, 127, 127)
    cb, sb = _operands(rng, N, K, 127, 127)
    Y = _gemm(kq, ca, sa, cb, sb)
    rows = _sampled_rows(M, 256, K)
    assert np.array_equal(Y[rows], o.gemm_mxfp4(ca[rows], sa[rows], cb, sb))


@pytest.mark.parametrize("M,N,K", MULTI_TILE)
def test_gemm_persistent_scaled_matches_oracle(kq, M, N, K):
    """Scales 2^-10 .. 2^10, fp32 and bf16 outputs and the rank-1 epilogue,
    on sampled rows x all columns (every tile column), within the fp32
    accumulation bound of the fp64 oracle."""
    rng = np.random.default_rng(3 * M + N + K)
    ca, sa = _operands(rng, M, K, 117, 137)
    cb, sb = _operands(rng, N, K, 117, 137)
    ta, tb = kq.kq_sf_tile(_cuda(sa)), kq.kq_sf_tile(_cuda(sb))
    da, db = _cuda(ca), _cuda(cb)
    mu = rng.normal(0, 4, size=M).astype(np.float32)
    wsum = rng.normal(0, 1, size=N).astype(np.float32)
    Y = kq.kq_gemm_mxfp4(da, ta, db, tb).cpu().numpy().astype(np.float64)
    Y16 = kq.kq_gemm_mxfp4_bf16(da, ta, db, tb).cpu().to(torch.float64).numpy()
    Y1 = kq.kq_gemm_mxfp4_rank1(da, ta, db, tb, _cuda(mu), _cuda(wsum)).cpu().numpy().astype(np.float64)
    rows = _sampled_rows(M, 256, K + 1)
    ref = o.gemm_mxfp4(ca[rows], sa[rows], cb, sb)
    tol = (K / 64 + 64) * 2.0 ** -23 * o.gemm_error_scale(ca[rows], sa[rows], cb, sb)
    assert np.all(np.abs(Y[rows] - ref) <= tol)
    assert np.all(np.abs(Y16[rows] - ref) <= tol + 2.0 ** -8 * (np.abs(ref) + tol))
    ref1 = o.gemm_mxfp4_rank1(ca[rows], sa[rows], cb, sb, mu[rows], wsum)
    tol1 = tol + 2.0 ** -22 * (np.abs(np.outer(mu[rows], wsum)) + np.abs(ref1))
    assert np.all(np.abs(Y1[rows] - ref1) <= tol1)


# ---------------------------------------------------------------------------
# the CTA-pair kernel (M and K multiples of 256; N a multiple of 256: 256 x 256
# tiles and one accumulator, else of 192: 256 x 192 tiles and two) on small
# shapes, and an independent cross-check against cuBLAS's block-scaled FP4
# GEMM.  192-wide tiles with odd indices read B scales from the middle of a
# 128-row scale block.  2560 x 3840 has 150 tiles and 2560 x 2880 has 150
# (192-wide), so some pairs run three tiles: the accumulator barriers turn
# over.
# ---------------------------------------------------------------------------
PAIR = [(256, 256, 256), (256, 512, 512), (768, 256, 1024), (512, 768, 2048), (2560, 3840, 512),  # 256 wide
        (256, 192, 256), (512, 576, 512), (768, 1344, 1024), (2560, 2880, 512)]                   # 192 wide


@pytest.mark.parametrize("M,N,K", PAIR)
def test_gemm_pair_kernel_matches_oracle(kq, M, N, K):
    rng = np.random.default_rng(5 * M + N + K)
    ca, sa = _operands(rng, M, K, 127, 127)
    cb, sb = _operands(rng, N, K, 127, 127)
    assert np.array_equal(_gemm(kq, ca, sa, cb, sb), o.gemm_mxfp4(ca, sa, cb, sb))
    ca, sa = _operands(rng, M, K, 117, 137)
    cb, sb = _operands(rng, N, K, 117, 137)
    Y = _gemm(kq, ca, sa, cb, sb)
    ref = o.gemm_mxfp4(ca, sa, cb, sb)
    tol = (K / 64 + 64) * 2.0 ** -23 * o.gemm_error_scale(ca, sa, cb, sb)
    assert np.all(np.abs(Y - ref) <= tol)
    Y16 = _gemm_bf16(kq, ca, sa, cb, sb)
    assert np.array_equal(_bf16_bits(Y16), _bf16_bits(torch.from_numpy(Y.astype(np.float32)).to(torch.bfloat16)))


def test_gemm_matches_cublas_mxfp4(kq):
    """cuBLAS's block-scaled FP4 GEMM (torch.nn.functional.scaled_mm with
    E8M0 scales in the same 128 x 4 swizzled blocks) on the FLUX attention
    projection: the same products in fp32, rounded to bf16, must give the
    same bits (the pair kernel with 192- and 256-column tiles and, at
    N = 3072 - 128, the single-CTA one)."""
    F = pytest.importorskip("torch.nn.functional")
    if not hasattr(F, "scaled_mm"):
        pytest.skip("torch.nn.functional.scaled_mm not available")
    g = torch.Generator(device="cuda")
    g.manual_seed(11)
    for M, N, K in ((4608, 3072, 3072), (4608, 2880, 3072), (4608, 2944, 3072)):
        ca = torch.randint(0, 256, (M, K // 2), dtype=torch.uint8, device="cuda", generator=g)
        cb = torch.randint(0, 256, (N, K // 2), dtype=torch.uint8, device="cuda", generator=g)
        ta = kq.kq_sf_tile(torch.randint(120, 134, (M, K // 32), dtype=torch.uint8, device="cuda", generator=g))
        tb = kq.kq_sf_tile(torch.randint(120, 134, (N, K // 32), dtype=torch.uint8, device="cuda", generator=g))
        ours = kq.kq_gemm_mxfp4_bf16(ca, ta, cb, tb)
        ref = F.scaled_mm(ca.view(torch.float4_e2m1fn_x2), cb.view(torch.float4_e2m1fn_x2).t(),
                          ta.view(torch.float8_e8m0fnu).reshape(-1, K // 32), F.ScalingType.BlockWise1x32,
                          tb.view(torch.float8_e8m0fnu).reshape(-1, K // 32), F.ScalingType.BlockWise1x32,
                          swizzle_a=F.SwizzleType.SWIZZLE_32_4_4, swizzle_b=F.SwizzleType.SWIZZLE_32_4_4,
                          output_dtype=torch.bfloat16)
        torch.cuda.synchronize()
        assert torch.equal(ours.view(torch.int16), ref.view(torch.int16)), (M, N, K)
