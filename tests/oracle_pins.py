"""Checks that pin the CPU oracle to facts fixed outside it.

Each ``pin_*`` takes the oracle module and raises AssertionError when the
oracle disagrees with what the pages, the MX format or plain mathematics
fix.  ``tests/test_oracle_pins.py`` runs them on the real oracle;
``tests/test_oracle_mutants.py`` plants typical mistakes in copies of the
oracle and checks that some pin fails for every one of them.

Nothing here calls the oracle to produce its own expected values: the
expected side is a closed form, a library routine (numpy.linalg, scipy,
ml_dtypes, torch dtypes), a brute-force search written here, a value
worked out by hand in a comment, or a hand-worked block in
tests/golden/kq_hand_blocks.txt (each derived there from the definitions).
"""
from __future__ import annotations

import math

import ml_dtypes
import numpy as np
import scipy.linalg
import torch

import synthetic
from golden_cases import hand_blocks

RNG_SEED = 1234


def _rand_params(nb, seed=RNG_SEED):
    return synthetic.make_params(nb, seed)


# --------------------------------------------------------------------------
# transform
# --------------------------------------------------------------------------
def pin_factor_unit_determinant(o):
    """Each factor has determinant 1 (unit-determinant LU factors)."""
    rng = np.random.default_rng(1)
    for _ in range(200):
        a, b = rng.normal(0, 2, 2)
        u = math.exp(rng.normal(0, 1))
        A = o.lu_factor(a, b, u)
        assert abs(np.linalg.det(A) - 1.0) < 1e-12, (a, b, u, np.linalg.det(A))


def pin_factor_lu_entries(o):
    """A = L U with L = [[1,0],[a,1]], U = [[u,b],[0,1/u]]: worked by hand,
    A = [[u, b], [a u, a b + 1/u]]."""
    a, b, u = 0.75, -1.25, 2.0
    A = o.lu_factor(a, b, u)
    want = np.array([[2.0, -1.25], [1.5, 0.75 * -1.25 + 0.5]])
    assert np.array_equal(A, want), A


def pin_block_unit_determinant(o):
    T = o.expand_params(_rand_params(8))
    for Tj in T:
        sign, logdet = np.linalg.slogdet(Tj)
        assert sign == 1.0 and abs(logdet) < 1e-10, (sign, logdet)


def pin_inverse(o):
    p = _rand_params(6)
    T = o.expand_params(p)
    Ti = o.expand_inverse(p)
    for Tj, Tij in zip(T, Ti):
        assert np.allclose(Tij @ Tj, np.eye(32), atol=1e-11)
        ref = np.linalg.inv(Tj)
        assert np.allclose(Tij, ref, rtol=1e-9, atol=1e-11)


def _kron_by_index_bits(p):
    """T[i][k] = prod_m A_m[bit(i, 4-m)][bit(k, 4-m)], the Kronecker index map
    written out with the factor built from its definition (not the oracle's)."""
    p = np.asarray(p, dtype=np.float64).reshape(5, 3)
    A = []
    for a, b, u in p:
        A.append([[u, b], [a * u, a * b + 1.0 / u]])
    T = np.empty((32, 32))
    for i in range(32):
        for k in range(32):
            v = 1.0
            for m in range(5):
                s = 4 - m
                v *= A[m][(i >> s) & 1][(k >> s) & 1]
            T[i, k] = v
    return T


def pin_kronecker_index_map(o):
    p = _rand_params(4, seed=5)
    T = o.expand_params(p)
    for j in range(4):
        ref = _kron_by_index_bits(p[j])
        assert np.allclose(T[j], ref, rtol=1e-14, atol=0), np.abs(T[j] - ref).max()


def pin_param_count(o):
    """15 parameters per 32-channel block, fewer than half of per-channel
    scaling's 32 (abstract: 'less than half the parameters')."""
    assert o.PARAMS_PER_BLOCK == 15
    assert o.PARAMS_PER_BLOCK * 2 < o.BLOCK
    assert o.expand_params(np.zeros((1, 15), np.float32) + np.tile([0, 0, 1], 5)).shape == (1, 32, 32)


def pin_factor_order(o):
    """Factor 1 on the most significant index bit: with factor 1 = diag(2, 1/2)
    and the others identity, T = diag(2 x16, 1/2 x16); factor 5 the same
    gives diag(2, 1/2, 2, 1/2, ...)."""
    for m, want in ((0, [2.0] * 16 + [0.5] * 16), (4, [2.0, 0.5] * 16),
                    (1, ([2.0] * 8 + [0.5] * 8) * 2)):
        p = np.tile(np.array([0.0, 0.0, 1.0]), 5)
        p[3 * m + 2] = 2.0
        T = o.expand_params(p[None])[0]
        assert np.array_equal(T, np.diag(want)), (m, np.diag(T))


def pin_lower_factor_position(o):
    """Shear a in factor 1 only: T = [[I, 0], [a I, I]] (16x16 blocks); a lower
    (not upper) triangular L puts a below the diagonal."""
    p = np.tile(np.array([0.0, 0.0, 1.0]), 5)
    p[0] = 3.0
    T = o.expand_params(p[None])[0]
    want = np.eye(32)
    want[16:, :16] = 3.0 * np.eye(16)
    assert np.array_equal(T, want)
    p = np.tile(np.array([0.0, 0.0, 1.0]), 5)
    p[3 * 4 + 1] = -2.0     # b of factor 5: upper entry, pairs (2i, 2i+1)
    T = o.expand_params(p[None])[0]
    want = np.eye(32)
    for i in range(0, 32, 2):
        want[i, i + 1] = -2.0
    assert np.array_equal(T, want)


def pin_rotation_is_hadamard(o):
    """Five 45-degree rotations R = [[c, -s], [s, c]] (u = c, b = -s, a = s/c = 1)
    give T = H_32 diag((-1)^popcount(k)) / sqrt(32), H_32 Sylvester's Hadamard
    matrix (scipy), because R = H_2 diag(1, -1) / sqrt(2)."""
    c = 1.0 / math.sqrt(2.0)
    p = np.tile(np.array([1.0, -c, c]), 5)
    T = o.expand_params(p[None])[0]
    H = scipy.linalg.hadamard(32).astype(np.float64)
    D = np.diag([(-1.0) ** bin(k).count("1") for k in range(32)])
    assert np.allclose(T, H @ D / math.sqrt(32), atol=1e-14)
    x = np.random.default_rng(3).normal(size=(5, 64))
    y = o.transform(x, np.stack([p, p]))
    # FWHT of the sign-flipped input, by the textbook in-place butterfly
    for r in range(5):
        for j in range(2):
            v = x[r, 32 * j:32 * j + 32] * np.diag(D)
            h = 1
            v = v.copy()
            while h < 32:
                for i in range(0, 32, 2 * h):
                    for k in range(i, i + h):
                        v[k], v[k + h] = v[k] + v[k + h], v[k] - v[k + h]
                h *= 2
            assert np.allclose(y[r, 32 * j:32 * j + 32], v / math.sqrt(32), atol=1e-12)


def pin_identity_params(o):
    nb = 3
    p = synthetic.identity_params(nb)
    assert np.array_equal(o.expand_params(p), np.stack([np.eye(32)] * nb))
    x = np.random.default_rng(4).normal(size=(7, 32 * nb)) * 3
    assert np.array_equal(o.transform(x, p), x)


def pin_transform_column_convention(o):
    """y = T x per token (x a column vector): with only b of factor 1 set,
    y[i] = x[i] + b x[i + 16] for i < 16 and y[i] = x[i] above."""
    p = np.tile(np.array([0.0, 0.0, 1.0]), 5)
    p[1] = 0.5
    x = np.arange(32, dtype=np.float64)[None]
    y = o.transform(x, p[None])[0]
    want = x[0].copy()
    want[:16] += 0.5 * x[0, 16:]
    assert np.array_equal(y, want), y


# --------------------------------------------------------------------------
# MXFP4
# --------------------------------------------------------------------------
def _ml_code(v):
    q = np.asarray(v, dtype=np.float32).astype(ml_dtypes.float4_e2m1fn)
    return q.view(np.uint8) & 0xF


def pin_e2m1_grid(o):
    codes = np.arange(16, dtype=np.uint8)
    ml = codes.view(ml_dtypes.float4_e2m1fn).astype(np.float64)
    assert np.array_equal(o.e2m1_decode(codes), ml)
    assert set(np.abs(o.e2m1_decode(codes))) == {0, 0.5, 1, 1.5, 2, 3, 4, 6}


def _brute_e2m1(r):
    """Nearest of the 16 codes; ties to the code with mantissa bit 0; beyond 6
    saturate; the sign bit copies r's sign (so -0.1 gives 0x8)."""
    mags = [0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0]
    m = abs(r)
    best, bestd = None, None
    for c in range(8):
        dd = abs(mags[c] - m)
        if best is None or dd < bestd - 1e-300 or (dd == bestd and (c & 1) == 0):
            best, bestd = c, dd
    sign = 1 if math.copysign(1.0, r) < 0 else 0
    return sign << 3 | best


def _edge_values():
    mids = [0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0]
    grid = [0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0]
    vals = []
    for m in mids + grid + [6.5, 7.0, 7.5, 7.999, 8.0, 100.0, 1e-30]:
        for eps in (0.0, 1e-6, -1e-6, 2.0 ** -20, -(2.0 ** -20)):
            v = m + eps
            if v >= 0:
                vals += [v, -v]
    return np.array(vals + [-0.0, 0.0])


def pin_e2m1_rounding(o):
    vals = np.concatenate([_edge_values(),
                           np.random.default_rng(6).uniform(-9, 9, 4000)]).astype(np.float32)
    got = o.e2m1_code(vals.astype(np.float64))
    assert np.array_equal(got, _ml_code(vals)), vals[got != _ml_code(vals)]
    brute = np.array([_brute_e2m1(float(v)) for v in vals], dtype=np.uint8)
    assert np.array_equal(got, brute), vals[got != brute]


def pin_e8m0(o):
    bytes_ = np.arange(256, dtype=np.uint8)
    ref = torch.from_numpy(bytes_).view(torch.float8_e8m0fnu).to(torch.float64).numpy()
    got = o.e8m0_decode(bytes_)
    assert np.array_equal(np.isnan(got), np.isnan(ref))
    ok = ~np.isnan(ref)
    assert np.array_equal(got[ok], ref[ok])


def pin_shared_exponent(o):
    """floor(log2(amax)) - 2, clamped to [-127, 127]; worked by hand."""
    cases = {1.0: -2, 6.0: 0, 7.99: 0, 8.0: 1, 4.0: 0, 3.999: -1, 0.5: -3,
             2.0 ** 100: 98, 2.0 ** 200: 127, 0.0: -127, 2.0 ** -126: -127,
             2.0 ** -124: -126, 2.0 ** -125: -127, 5e-324: -127}
    for amax, e in cases.items():
        got = int(o.shared_exponent(np.array([amax]))[0])
        assert got == e, (amax, got, e)


def pin_hand_block(o):
    """One block worked by hand.  Values (then padded with zeros):
      x = [6, -7.5, 0.3, -0.2, 1.25, 2.5, 3.5, 5, -0.75, 0.74, ...]
    amax = 7.5 -> floor(log2 7.5) = 2 -> e = 0, scale byte 127, r = x.
      6 -> 6 (0x7); -7.5 -> saturates -6 (0xF); 0.3 -> 0.5 (0x1);
      -0.2 -> -0 (0x8); 1.25 tie -> 1.0 (0x2); 2.5 tie -> 2 (0x4);
      3.5 tie -> 4 (0x6); 5 tie -> 4 (0x6); -0.75 tie -> -1.0 (0xA);
      0.74 -> 0.5 (0x1); zeros -> 0x0.
    Bytes pack (even element low nibble): 0xF7, 0x81, 0x42, 0x66, 0x1A, 0, ..."""
    x = np.zeros((1, 32))
    x[0, :10] = [6, -7.5, 0.3, -0.2, 1.25, 2.5, 3.5, 5, -0.75, 0.74]
    codes, scales = o.quantize_mxfp4(x)
    assert scales.tolist() == [[127]]
    assert codes[0, :5].tolist() == [0xF7, 0x81, 0x42, 0x66, 0x1A]
    assert not codes[0, 5:].any()
    # scaled copy: x * 2**-10 only moves the scale byte by -10
    codes2, scales2 = o.quantize_mxfp4(x * 2.0 ** -10)
    assert scales2.tolist() == [[117]] and np.array_equal(codes2, codes)
    # all-zero block: byte 0 (2**-127), codes 0
    codes3, scales3 = o.quantize_mxfp4(np.zeros((1, 32)))
    assert scales3.tolist() == [[0]] and not codes3.any()
    # NaN anywhere: byte 0xFF
    xn = x.copy()
    xn[0, 31] = np.nan
    assert o.quantize_mxfp4(xn)[1].tolist() == [[255]]
    xi = x.copy()
    xi[0, 3] = -np.inf
    assert o.quantize_mxfp4(xi)[1].tolist() == [[255]]


def pin_brute_pipeline(o):
    """A few blocks of the tiny workload, every step by plain loops in fp64:
    T from the index-bit product, y from explicit sums, amax, frexp exponent,
    brute-force code search, nibble packing."""
    w = synthetic.CONFIGS["tiny"][0]
    raw = synthetic.make_activations(w, rows=[0, 77, 255])
    x = raw.astype(np.float64)
    p = synthetic.make_params(w.nb, w.seed)
    codes, scales = o.kq_quantize(x, p)
    for j in (0, 7, 35):
        T = _kron_by_index_bits(p[j])
        for r in range(3):
            xb = x[r, 32 * j:32 * j + 32]
            y = [math.fsum(T[i, k] * xb[k] for k in range(32)) for i in range(32)]
            amax = max(abs(v) for v in y)
            e = max(-127, min(127, math.frexp(amax)[1] - 1 - 2)) if amax > 0 else -127
            assert scales[r, j] == e + 127
            nib = [_brute_e2m1(v / 2.0 ** e) for v in y]
            packed = [nib[2 * i] | nib[2 * i + 1] << 4 for i in range(16)]
            assert codes[r, 16 * j:16 * j + 16].tolist() == packed, (r, j)


def pin_roundtrip_bound(o):
    """dequant(quant(y)) differs from y by at most half a grid step at r
    (0.25, 0.5, 1 in binades [0,2), [2,4), [4,6]) or by |r| - 6 when
    saturated, times 2**e; undoing T then bounds the error in x."""
    w = synthetic.CONFIGS["tiny"][0]
    x = synthetic.make_activations(w, rows=np.arange(64)).astype(np.float64)
    p = synthetic.make_params(w.nb, w.seed)
    y = o.transform(x, p)
    codes, scales = o.quantize_mxfp4(y)
    deq = o.dequant(codes, scales)
    M, d = y.shape
    e = (scales.astype(np.int64) - 127).repeat(32, axis=1)
    r = np.abs(y) / 2.0 ** e
    half = np.where(r < 2, 0.25, np.where(r < 4, 0.5, 1.0))
    bound = np.where(r > 6, r - 6, half) * 2.0 ** e
    assert np.all(np.abs(deq - y) <= bound * (1 + 1e-12))
    Tinv = o.expand_inverse(p)
    xr = o.apply_blockdiag(deq, Tinv)
    xb = o.apply_blockdiag(bound, np.abs(Tinv))
    assert np.all(np.abs(xr - x) <= xb * (1 + 1e-9) + 1e-12)


def pin_fold_invariance(o):
    """W' (T x) = W x for W' = fold(W)."""
    nb = 4
    p = _rand_params(nb, seed=11)
    W = synthetic.make_weights(24, 32 * nb, 3).astype(np.float64)
    x = np.random.default_rng(12).normal(size=(32 * nb, 5))
    Wf = o.fold_weights(W, p)
    Tx = o.transform(x.T, p).T
    lhs = Wf @ Tx
    rhs = W @ x
    assert np.allclose(lhs, rhs, rtol=1e-10, atol=1e-10 * np.abs(rhs).max())


def pin_weight_quantizer_direction(o):
    """With a = b = 0 the transform is the diagonal D = diag(T), so the folded
    weights are W D^{-1}: the weight codes equal plain MXFP4 of W divided
    column-wise by diag(T), computed here without the oracle's fold; with
    identity parameters they are plain MXFP4 of W."""
    nb = 3
    p = _rand_params(nb, seed=31).reshape(nb, 5, 3).copy()
    p[:, :, 0] = 0
    p[:, :, 1] = 0
    p = p.reshape(nb, 15)
    diag = np.empty(32 * nb)
    for j in range(nb):
        for i in range(32):
            v = 1.0
            for m in range(5):
                u = p[j, 3 * m + 2]
                v *= (1.0 / u) if (i >> (4 - m)) & 1 else u
            diag[32 * j + i] = v
    W = synthetic.make_weights(7, 32 * nb, 5).astype(np.float64)
    c1, s1 = o.quantize_weights(W, p)
    c2, s2 = o.quantize_mxfp4(W / diag[None, :])
    assert np.array_equal(c1, c2) and np.array_equal(s1, s2)
    ci, si = o.quantize_weights(W, synthetic.identity_params(nb))
    c3, s3 = o.quantize_mxfp4(W)
    assert np.array_equal(ci, c3) and np.array_equal(si, s3)


def pin_gemm_mxfp4_by_hand(o):
    """The quantised GEMM against a plain triple loop over decoded values,
    each decoded by hand from the E2M1 grid and 2**(byte - 127); and the
    blocked scale layout against its defining formula on a small case."""
    rng = np.random.default_rng(41)
    M, N, K = 3, 2, 64
    ca = rng.integers(0, 256, size=(M, K // 2), dtype=np.uint8)
    cb = rng.integers(0, 256, size=(N, K // 2), dtype=np.uint8)
    sa = rng.integers(120, 135, size=(M, K // 32), dtype=np.uint8)
    sb = rng.integers(120, 135, size=(N, K // 32), dtype=np.uint8)
    grid = [0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0]

    def val(codes, scales, r, k):
        byte = int(codes[r, k // 2])
        nib = (byte >> 4) if k % 2 else (byte & 15)
        mag = grid[nib & 7] * 2.0 ** (int(scales[r, k // 32]) - 127)
        return -mag if nib & 8 else mag
    Y = o.gemm_mxfp4(ca, sa, cb, sb)
    for m in range(M):
        for n in range(N):
            ref = math.fsum(val(ca, sa, m, k) * val(cb, sb, n, k) for k in range(K))
            assert Y[m, n] == ref
    sc = np.arange(130 * 8, dtype=np.uint32).reshape(130, 8).astype(np.uint8)
    t = o.sf_tile(sc)
    assert t.shape == (2, 2, 512)
    assert t[0, 0, 0] == sc[0, 0] and t[0, 0, 1] == sc[0, 1] and t[0, 0, 4] == sc[32, 0]
    assert t[0, 1, 16 * 5 + 4 * 3 + 2] == sc[101, 6]
    assert t[1, 1, 16 * 1 + 3] == sc[129, 7] and t[1, 0, 16 * 2] == 0


def pin_centering(o):
    """Shifting every token by its own constant changes nothing after
    centring (the shift is exact in fp64 here: dyadic values); the rank-1
    term restores the layer exactly without quantisation: with the
    quantised operands replaced by their exact values, (x - mu 1) W'^T-side
    plus mu (W 1) is x W^T."""
    rng = np.random.default_rng(51)
    M, d, N = 6, 96, 5
    x = np.round(rng.normal(size=(M, d)) * 64) / 64
    p = _rand_params(d // 32, seed=52)
    mu = o.row_sum(x, 1.0 / d)
    assert np.allclose(mu, x.mean(axis=1), rtol=0, atol=1e-15)
    shift = np.round(rng.normal(size=M) * 8) / 8
    c1, s1 = o.quantize_centered(x, p, mu)
    c2, s2 = o.quantize_centered(x + shift[:, None], p, mu + shift)
    assert np.array_equal(c1, c2) and np.array_equal(s1, s2)
    W = rng.normal(size=(N, d))
    wsum = o.row_sum(W)
    xt = o.transform(x - mu[:, None], p)                   # exact transformed, centred tokens
    Wt = o.fold_weights(W, p)
    lhs = xt @ Wt.T + np.outer(mu, wsum)
    assert np.allclose(lhs, x @ W.T, rtol=1e-10, atol=1e-10 * np.abs(x @ W.T).max())


def pin_smoothquant_is_diagonal_case(o):
    """a = b = 0 makes T diagonal; SmoothQuant with 1/s = diag(T) then gives
    the same codes and scales."""
    nb = 3
    p = _rand_params(nb, seed=21).reshape(nb, 5, 3).copy()
    p[:, :, 0] = 0
    p[:, :, 1] = 0
    p = p.reshape(nb, 15)
    T = o.expand_params(p)
    diag = np.concatenate([np.diag(t) for t in T])
    x = synthetic.f32_from_bf16_bits(
        synthetic.bf16_bits_from_f32(np.random.default_rng(2).normal(size=(9, 96)).astype(np.float32))
    ).astype(np.float64)
    c1, s1 = o.kq_quantize(x, p)
    c2, s2 = o.sq_quantize(x, diag)
    assert np.array_equal(c1, c2) and np.array_equal(s1, s2)


def pin_undecided_flags(o):
    y = np.zeros((1, 32))
    y[0, 0] = 4.0 * 1.25          # amax 5 -> e = 0; r = 5 is a midpoint
    y[0, 1] = 1.3                 # far from any midpoint
    y[0, 2] = 0.25 * (1 + 5e-5)   # within 1e-4 relative of 0.25
    tol = np.full((1, 32), 1e-9)
    elem, blk = o.undecided(y, tol)
    assert elem[0, 0] and not elem[0, 1] and elem[0, 2]
    assert not blk[0, 0]
    y2 = y.copy()
    y2[0, 0] = 4.0 * (1 + 1e-6)   # amax next to a power of two
    elem2, blk2 = o.undecided(y2, tol)
    assert blk2[0, 0] and elem2.all()



# --------------------------------------------------------------------------
# the tolerance functions (they set every parity tolerance and exemption)
# --------------------------------------------------------------------------
def _mag_factor_by_hand(a, b, u):
    """|L| |U| written out: |L| = [[1, 0], [|a|, 1]], |U| = [[|u|, |b|], [0, 1/|u|]],
    so |L||U| = [[|u|, |b|], [|a||u|, |a||b| + 1/|u|]]."""
    a, b, u = abs(float(a)), abs(float(b)), abs(float(u))
    return [[u, b], [a * u, a * b + 1.0 / u]]


def _inv_mag_factor_by_hand(a, b, u):
    """|U^-1| |L^-1| written out: U^-1 = [[1/u, -b], [0, u]], L^-1 = [[1, 0], [-a, 1]],
    so |U^-1||L^-1| = [[1/|u| + |b||a|, |b|], [|u||a|, |u|]]."""
    a, b, u = abs(float(a)), abs(float(b)), abs(float(u))
    return [[1.0 / u + b * a, b], [u * a, u]]


def _kron_entry(F, i, k):
    """Entry (i, k) of F[0] (x) ... (x) F[4] by the index-bit product."""
    v = 1.0
    for m in range(5):
        s = 4 - m
        v *= F[m][(i >> s) & 1][(k >> s) & 1]
    return v


def pin_error_scale_by_hand(o):
    """One block worked by hand.  Factor 1 (the most significant index bit)
    has a = 2, b = -3, u = 0.5; the others are the identity.  Then
    |L||U| = [[0.5, 3], [1, 2*3 + 2]] = [[0.5, 3], [1, 8]] on bit 4, so for
    x with x_0 = 1, x_16 = -2, x_5 = 4 and zeros elsewhere:
      element 0:  0.5 |x_0| + 3 |x_16| = 0.5 + 6 = 6.5
      element 16: 1 |x_0| + 8 |x_16| = 1 + 16 = 17
      element 5:  0.5 |x_5| + 3 |x_21| = 2
      element 21: 1 |x_5| + 8 |x_21| = 4
    and 0 elsewhere.  Note |T| has 4 (= |2*(-3) + 2|) where |L||U| has 8: the
    scale is the size of the summed terms, not of their (cancelling) sum."""
    p = np.tile(np.array([0.0, 0.0, 1.0]), 5)
    p[0:3] = [2.0, -3.0, 0.5]
    x = np.zeros((1, 32))
    x[0, 0], x[0, 16], x[0, 5] = 1.0, -2.0, 4.0
    es = o.error_scale(x, p[None])
    want = np.zeros((1, 32))
    want[0, 0], want[0, 16], want[0, 5], want[0, 21] = 6.5, 17.0, 2.0, 4.0
    assert np.array_equal(es, want), es
    assert np.array_equal(o.lu_factor_magnitude(2.0, -3.0, 0.5), np.array([[0.5, 3.0], [1.0, 8.0]]))


def pin_error_scale_definition(o):
    """error_scale[m, 32 j + i] = sum_k ((x)_m |L_m||U_m|)[i, k] |x[m, 32 j + k]|,
    rebuilt with plain loops (math.fsum) from the factor magnitudes written out
    by hand; expand_magnitude against the same index-bit product."""
    p = _rand_params(3, seed=71)
    x = np.random.default_rng(72).normal(size=(4, 96)) * 3
    es = o.error_scale(x, p)
    em = o.expand_magnitude(p)
    for j in range(3):
        F = [_mag_factor_by_hand(*p[j, 3 * m:3 * m + 3]) for m in range(5)]
        Tm = np.array([[_kron_entry(F, i, k) for k in range(32)] for i in range(32)])
        assert np.allclose(em[j], Tm, rtol=1e-14, atol=0), j
        for r in range(4):
            for i in range(32):
                ref = math.fsum(Tm[i, k] * abs(x[r, 32 * j + k]) for k in range(32))
                assert abs(es[r, 32 * j + i] - ref) <= 1e-13 * ref, (r, j, i, es[r, 32 * j + i], ref)


def pin_fold_error_scale(o):
    """fold_error_scale[n, 32 j + i] = sum_k |W[n, 32 j + k]| ((x)_m |U_m^-1||L_m^-1|)[k, i]
    (the folded weight is W T^-1, so the sum runs over the row index of T^-1),
    by plain loops; and one entry by hand: factor 5 (least significant bit)
    with a = 1, b = 2, u = 4, the rest identity, gives
    |U^-1||L^-1| = [[1/4 + 2, 2], [4, 4]] on bit 0; for a row with w_0 = 1,
    w_1 = -1: entry 0 = 1 * 2.25 + 1 * 4 = 6.25, entry 1 = 1 * 2 + 1 * 4 = 6."""
    p = np.tile(np.array([0.0, 0.0, 1.0]), 5)
    p[12:15] = [1.0, 2.0, 4.0]
    W = np.zeros((1, 32))
    W[0, 0], W[0, 1] = 1.0, -1.0
    fe = o.fold_error_scale(W, p[None])
    assert fe[0, 0] == 6.25 and fe[0, 1] == 6.0 and not fe[0, 2:].any(), fe
    p = _rand_params(2, seed=73)
    W = np.random.default_rng(74).normal(size=(3, 64))
    fe = o.fold_error_scale(W, p)
    for j in range(2):
        F = [_inv_mag_factor_by_hand(*p[j, 3 * m:3 * m + 3]) for m in range(5)]
        for n in range(3):
            for i in range(32):
                ref = math.fsum(abs(W[n, 32 * j + k]) * _kron_entry(F, k, i) for k in range(32))
                assert abs(fe[n, 32 * j + i] - ref) <= 1e-13 * ref, (n, j, i)


def pin_gemm_error_scale(o):
    """gemm_error_scale[m, n] = sum_k |a_mk| |b_nk| over the decoded MXFP4
    values, each decoded by hand from the E2M1 grid and 2^(byte - 127); and
    one entry by hand: a row of codes 0x7 (6) and 0xF (-6) with scale 2^1
    against codes 0x2 (1) with scale 2^-1 gives K * 12 * 0.5 = 6 K."""
    rng = np.random.default_rng(75)
    M, N, K = 3, 2, 96
    ca = rng.integers(0, 256, size=(M, K // 2), dtype=np.uint8)
    cb = rng.integers(0, 256, size=(N, K // 2), dtype=np.uint8)
    sa = rng.integers(120, 135, size=(M, K // 32), dtype=np.uint8)
    sb = rng.integers(120, 135, size=(N, K // 32), dtype=np.uint8)
    grid = [0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0]

    def mag(codes, scales, r, k):
        byte = int(codes[r, k // 2])
        nib = (byte >> 4) if k % 2 else (byte & 15)
        return grid[nib & 7] * 2.0 ** (int(scales[r, k // 32]) - 127)
    G = o.gemm_error_scale(ca, sa, cb, sb)
    for m in range(M):
        for n in range(N):
            assert G[m, n] == math.fsum(mag(ca, sa, m, k) * mag(cb, sb, n, k) for k in range(K))
    ca1 = np.full((1, K // 2), 0xF7, dtype=np.uint8)
    sa1 = np.full((1, K // 32), 128, dtype=np.uint8)
    cb1 = np.full((1, K // 2), 0x22, dtype=np.uint8)
    sb1 = np.full((1, K // 32), 126, dtype=np.uint8)
    assert o.gemm_error_scale(ca1, sa1, cb1, sb1)[0, 0] == 6.0 * K


def pin_undecided_tolerance_branches(o):
    """The tolerance terms of the exemption rule, worked by hand.

    Block A: amax = 22 (in [16, 32): floor(log2) = 4, e = 2, r = y / 4;
      r = 5.5 and 0.65 for y = 22 and 2.6, far from every boundary).
      y_1 = 4 * 1.251 = 5.004: r = 1.251 is 0.001 from the midpoint 1.25,
      outside the relative window 1.25e-4.  The tolerance window is tol / 2^e:
      tol = 0.003 gives 0.00075 (not flagged), tol = 0.005 gives 0.00125
      (flagged).  (tol * 2^e or tol alone would flag both.)
      y_2 = -0.001 lies 0.249 from the nearest midpoint in r; it is flagged
      only through |y| <= tol: flagged for tol = 0.003, not for tol = 0.0005.
    Block B: amax = 16.016, 0.016 above 2^4, outside the relative window
      16e-4: the block is open for tol = 0.02, decided for tol = 0.01."""
    y = np.zeros((1, 64))
    y[0, 0] = 22.0
    y[0, 1] = 4 * 1.251
    y[0, 2] = -0.001
    y[0, 3] = 2.6
    y[0, 32] = 16.016
    y[0, 33] = 1.3

    def flags(tol_a, tol_b):
        tol = np.zeros((1, 64))
        tol[0, :32] = tol_a
        tol[0, 32:] = tol_b
        return o.undecided(y, tol)
    e, b = flags(0.003, 0.01)
    assert not e[0, 1] and e[0, 2] and not e[0, 0] and not e[0, 3]
    assert not b[0, 0] and not b[0, 1] and not e[0, 33]
    e, b = flags(0.005, 0.02)
    assert e[0, 1] and b[0, 1] and e[0, 32:].all()
    e, b = flags(0.0005, 0.0)
    assert not e[0, 1] and not e[0, 2] and not b[0, 1]
    # with a zero tolerance only the relative windows and exact zeros remain
    e, b = o.undecided(y, np.zeros_like(y))
    assert e[0, 4] and not e[0, 2] and not e[0, 1]


def pin_layer_error_by_hand(o):
    """The quantised layer's relative error, worked by hand on one 32-channel
    block.  x = [7, 3, 0, ...], W = [[1, 0, ...], [0, 1, 0, ...]], identity
    parameters: amax 7 gives e = 0, 7 saturates to 6 and 3 is on the grid, so
    Q(x) = [6, 3, 0, ...]; W is exact.  x W^T = [7, 3], the quantised layer
    gives [6, 3]: error 1 / sqrt(49 + 9) = 1 / sqrt(58).
    With u = 2 on factor 1 (T = diag(2 x16, 1/2 x16)) the token becomes
    [14, 6, ...]: e = 1, r = [7, 3] -> [6, 3], Q(T x) = [12, 6]; W T^-1 =
    [[1/2, 0, ...], [0, 1/2, 0, ...]] is exact, so the layer gives [6, 3]
    again: the same error.  u = 6/7 on factor 1 moves the outlier onto the
    grid (T x = [6, 18/7]; amax 6, e = 0; 18/7 ~ 2.571 -> 3), but the folded
    weights W T^-1 = [[7/6, 0, ...], [0, 7/6, 0, ...]] are quantised too:
    amax 7/6 gives e = -2, r = 14/3 ~ 4.67 -> 4, i.e. 1.  The layer gives
    [6 * 1, 3 * 1] = [6, 3] once more: error 1 / sqrt(58) (the weight side
    takes back what the activation side gained)."""
    x = np.zeros((1, 32))
    x[0, 0], x[0, 1] = 7.0, 3.0
    W = np.zeros((2, 32))
    W[0, 0] = W[1, 1] = 1.0
    ident = np.tile(np.array([0.0, 0.0, 1.0]), 5)[None]
    assert abs(o.layer_error(x, W, ident) - 1.0 / math.sqrt(58.0)) < 1e-15
    p = ident.copy()
    p[0, 2] = 2.0
    assert abs(o.layer_error(x, W, p) - 1.0 / math.sqrt(58.0)) < 1e-15
    p[0, 2] = 6.0 / 7.0
    assert abs(o.layer_error(x, W, p) - 1.0 / math.sqrt(58.0)) < 1e-15


def pin_golden_hand_blocks(o):
    """The hand-worked blocks of tests/golden/kq_hand_blocks.txt: ties and
    saturation, the Kronecker factor order (a diagonal factor on the most and on
    the least significant index bit), five rotations on a unit vector, a power-
    of-two amax, an all-zero block and a tiny amax.  Inputs as the kernels see
    them (rounded to fp32)."""
    for hb in hand_blocks():
        x = hb.x.astype(np.float32).astype(np.float64)
        codes, scales = o.kq_quantize(x, hb.params)
        assert int(scales[0, 0]) == hb.scale, (hb.name, int(scales[0, 0]), hb.scale)
        assert np.array_equal(codes, hb.codes), (hb.name, codes, hb.codes)

ALL_PINS = [v for k, v in sorted(globals().items()) if k.startswith("pin_")]
