"""CPU oracle for the KroQuant online activation quantizer (fp64, NumPy).

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
CPU-baseline / reference legs of ``bench.py`` import this module.  The CUDA
library never calls it and it never calls the CUDA library; the two share no
code.  It is written to be read against the pages, not to be fast.

Sources (cited by page title and section):

* [ABS]  "KroQuant: Kronecker-Structured Block Transforms for Efficient
  Post-Training Quantization of Diffusion Transformers", Abstract: an
  invertible linear transform is applied to the activations and its inverse to
  the weights before both are quantized; the transform is learned,
  Kronecker-structured and acts on each 32-element block of the activation;
  it stores fewer than half the parameters of per-channel scaling; W4A4 uses
  MXFP4.
* [POD]  The same title, research-summary page, method paragraph: each
  32x32 block is a Kronecker product of five 2x2 unit-determinant
  LU-decomposed matrices.
* [MX]   OCP Microscaling Formats (MX) v1.0 (public format specification, not
  among the pages): MXFP4 = blocks of 32 E2M1 elements sharing one E8M0
  scale; the shared exponent is floor(log2(amax)) minus the element format's
  largest exponent (2 for E2M1); elements are rounded to nearest-even and
  saturated to the largest finite magnitude (6).

Readings taken where the pages are silent:

* factor form: A = L U with L = [[1, 0], [a, 1]] and U = [[u, b], [0, 1/u]],
  three parameters (a, b, u) per factor, fifteen per block;
* Kronecker order: factor 1 acts on the most significant bit of the index
  inside the block (standard Kronecker index map), factor 5 on the least;
* column-vector convention: y_j = T_j x_j per token; the folded weight is
  W' = W T^{-1} for W laid out [out, in];
* a negative value that rounds to zero keeps its sign (code 0x8);
* NaN or infinity anywhere in a block gives the NaN scale byte 0xFF and
  leaves the block's codes unspecified.

Pins (tests/test_oracle_pins.py): det(A) = det(T) = 1; T^{-1} T = I;
Kronecker product against an explicit index-bit product; the factor-order
special cases; the 45-degree-rotation case against a textbook Hadamard
matrix; the E2M1 grid and RNE against ml_dtypes and against brute-force
nearest-code search; E8M0 decode against torch's float8_e8m0fnu; fold
invariance W' (T x) = W x; round-trip error bound.
"""
from __future__ import annotations

import numpy as np

BLOCK = 32          # [ABS]: 32-element blocks; [MX]: 32 elements per scale
N_FACTORS = 5       # [POD]: 2**5 = 32
PARAMS_PER_BLOCK = 3 * N_FACTORS   # 15 (a, b, u per factor)
E2M1_EMAX = 2       # [MX]: largest exponent of E2M1 (6 = 1.5 * 2**2)
E2M1_MAX = 6.0
E8M0_BIAS = 127
E8M0_NAN = 0xFF

# E2M1 magnitudes indexed by the 3-bit code (exponent 2 bits, mantissa 1 bit):
# code 0 is zero, code 1 the subnormal 0.5, then 1.0 * 2**(E-1) * (1 + m/2).
E2M1_MAGNITUDES = np.array([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0])


# ---------------------------------------------------------------------------
# transform: parameters -> factors -> Kronecker block
# ---------------------------------------------------------------------------
def lu_factor(a: float, b: float, u: float) -> np.ndarray:
    """[POD] one unit-determinant factor A = L U (fp64)."""
    L = np.array([[1.0, 0.0], [float(a), 1.0]])
    U = np.array([[float(u), float(b)], [0.0, 1.0 / float(u)]])
    return L @ U


def lu_factor_inverse(a: float, b: float, u: float) -> np.ndarray:
    """A^{-1} = U^{-1} L^{-1}, each triangular factor inverted in closed form."""
    Linv = np.array([[1.0, 0.0], [-float(a), 1.0]])
    Uinv = np.array([[1.0 / float(u), -float(b)], [0.0, float(u)]])
    return Uinv @ Linv


def lu_factor_magnitude(a: float, b: float, u: float) -> np.ndarray:
    """|L| |U| (entrywise absolute values, then the product): the size of the
    terms an evaluation of L U sums, used as the scale of rounding error."""
    L = np.abs(np.array([[1.0, 0.0], [float(a), 1.0]]))
    U = np.abs(np.array([[float(u), float(b)], [0.0, 1.0 / float(u)]]))
    return L @ U


def _factors(params_block: np.ndarray, fn) -> list[np.ndarray]:
    p = np.asarray(params_block, dtype=np.float64).reshape(N_FACTORS, 3)
    return [fn(p[m, 0], p[m, 1], p[m, 2]) for m in range(N_FACTORS)]


def _kron_all(mats: list[np.ndarray]) -> np.ndarray:
    out = mats[0]
    for A in mats[1:]:
        out = np.kron(out, A)
    return out


def expand_block(params_block: np.ndarray) -> np.ndarray:
    """[POD] T_j = A_j1 (x) A_j2 (x) A_j3 (x) A_j4 (x) A_j5, a 32x32 fp64 matrix."""
    return _kron_all(_factors(params_block, lu_factor))


def expand_params(params: np.ndarray) -> np.ndarray:
    """[nb, 15] -> [nb, 32, 32] fp64."""
    params = np.asarray(params).reshape(-1, PARAMS_PER_BLOCK)
    return np.stack([expand_block(p) for p in params])


def expand_inverse(params: np.ndarray) -> np.ndarray:
    """T_j^{-1} = (x)_m A_jm^{-1} (mixed-product property), [nb, 32, 32]."""
    params = np.asarray(params).reshape(-1, PARAMS_PER_BLOCK)
    return np.stack([_kron_all(_factors(p, lu_factor_inverse)) for p in params])


def expand_magnitude(params: np.ndarray) -> np.ndarray:
    """(x)_m |L_jm| |U_jm|, [nb, 32, 32]; equals |T_j| when no factor's
    bottom-right entry a b + 1/u cancels."""
    params = np.asarray(params).reshape(-1, PARAMS_PER_BLOCK)
    return np.stack([_kron_all(_factors(p, lu_factor_magnitude)) for p in params])


def _blocks(x: np.ndarray) -> np.ndarray:
    x = np.asarray(x, dtype=np.float64)
    M, d = x.shape
    if d % BLOCK:
        raise ValueError("d must be a multiple of 32")
    return x.reshape(M, d // BLOCK, BLOCK)


def apply_blockdiag(x: np.ndarray, T: np.ndarray) -> np.ndarray:
    """y[m, 32j + i] = sum_k T[j, i, k] x[m, 32j + k]  (column-vector form)."""
    xb = _blocks(x)
    M, nb, _ = xb.shape
    y = np.matmul(T[None, :, :, :], xb[:, :, :, None])[..., 0]
    return y.reshape(M, nb * BLOCK)


def transform(x: np.ndarray, params: np.ndarray) -> np.ndarray:
    """[ABS] the online block-diagonal transform y = blockdiag(T_j) x, fp64."""
    return apply_blockdiag(x, expand_params(params))


def error_scale(x: np.ndarray, params: np.ndarray) -> np.ndarray:
    """sum_k ((x)_m |L||U|)[i, k] |x_k| per element: the magnitude against
    which a floating-point evaluation of the transform is judged."""
    return apply_blockdiag(np.abs(np.asarray(x, dtype=np.float64)), expand_magnitude(params))


# ---------------------------------------------------------------------------
# MXFP4 encoding [MX]
# ---------------------------------------------------------------------------
def shared_exponent(amax: np.ndarray) -> np.ndarray:
    """Unbiased E8M0 exponent per block: floor(log2(amax)) - emax(E2M1),
    clamped to the E8M0 range [-127, 127]; amax = 0 gives -127.  floor(log2)
    is read exactly from frexp (amax = f * 2**k, f in [0.5, 1))."""
    amax = np.asarray(amax, dtype=np.float64)
    f, k = np.frexp(amax)
    fl = np.where(amax > 0, k - 1, -(2 ** 20))
    return np.clip(fl - E2M1_EMAX, -E8M0_BIAS, E8M0_BIAS).astype(np.int64)


def e2m1_round_magnitude(mag: np.ndarray) -> np.ndarray:
    """Round |r| onto the E2M1 grid, nearest with ties to even mantissa,
    saturating at 6.  Below 1 the grid is the subnormal step 0.5; in binade
    [2**E, 2**(E+1)) (E = 0, 1, 2) the step is 2**(E-1)."""
    mag = np.asarray(mag, dtype=np.float64)
    E = np.floor(np.log2(np.where(mag > 0, mag, 1.0)))
    E = np.clip(E, 0, E2M1_EMAX)
    # exact check of the binade: log2 may be off by one ulp at powers of two
    E = np.where(mag < 2.0 ** E, E - 1, E)
    E = np.where(mag >= 2.0 ** (E + 1), E + 1, E)
    E = np.clip(E, 0, E2M1_EMAX)
    step = np.where(mag < 1.0, 0.5, 2.0 ** (E - 1))
    q = np.rint(mag / step) * step        # np.rint: round half to even
    return np.minimum(q, E2M1_MAX)


def e2m1_code(r: np.ndarray) -> np.ndarray:
    """4-bit E2M1 code of r: sign bit 3, magnitude code in bits 0..2.  The sign
    is taken from r itself, so a negative value that rounds to 0 gives 0x8."""
    r = np.asarray(r, dtype=np.float64)
    q = e2m1_round_magnitude(np.abs(r))
    mag_code = np.searchsorted(E2M1_MAGNITUDES, q)
    assert np.all(E2M1_MAGNITUDES[mag_code] == q)
    sign = np.signbit(r).astype(np.int64)
    return (sign << 3 | mag_code).astype(np.uint8)


def e2m1_decode(code: np.ndarray) -> np.ndarray:
    code = np.asarray(code, dtype=np.int64)
    v = E2M1_MAGNITUDES[code & 7]
    return np.where(code & 8, -v, v)


def e8m0_decode(byte: np.ndarray) -> np.ndarray:
    byte = np.asarray(byte, dtype=np.int64)
    v = np.ldexp(1.0, byte - E8M0_BIAS)
    return np.where(byte == E8M0_NAN, np.nan, v)


def quantize_mxfp4(y: np.ndarray):
    """MXFP4-encode y [M, d] block by block along d.

    Returns (codes uint8 [M, d/2], scales uint8 [M, d/32]).  Element 2i of a
    row goes to the low nibble of byte i, element 2i+1 to the high nibble.
    """
    yb = _blocks(y)
    M, nb, _ = yb.shape
    finite = np.all(np.isfinite(yb), axis=2)
    with np.errstate(invalid="ignore"):
        amax = np.max(np.abs(np.where(np.isfinite(yb), yb, 0.0)), axis=2)
    e = shared_exponent(amax)
    scales = np.where(finite, e + E8M0_BIAS, E8M0_NAN).astype(np.uint8)
    # r = y / 2**e is exact (a power-of-two scaling of an fp64 value)
    r = np.ldexp(np.where(np.isfinite(yb), yb, 0.0), -e[:, :, None])
    nib = e2m1_code(r).reshape(M, nb * BLOCK)
    codes = (nib[:, 0::2] | (nib[:, 1::2] << 4)).astype(np.uint8)
    return codes, scales


def unpack_nibbles(codes: np.ndarray) -> np.ndarray:
    codes = np.asarray(codes, dtype=np.uint8)
    M, half = codes.shape
    out = np.empty((M, 2 * half), dtype=np.uint8)
    out[:, 0::2] = codes & 0xF
    out[:, 1::2] = codes >> 4
    return out


def dequant(codes: np.ndarray, scales: np.ndarray) -> np.ndarray:
    """[MX] element value = E2M1(code) * 2**(scale - 127); scale 0xFF is NaN."""
    nib = unpack_nibbles(codes)
    M, d = nib.shape
    v = e2m1_decode(nib).reshape(M, d // BLOCK, BLOCK)
    s = e8m0_decode(scales)[:, :, None]
    return (v * s).reshape(M, d)


# ---------------------------------------------------------------------------
# the quantizers and the weight fold
# ---------------------------------------------------------------------------
def kq_quantize(x: np.ndarray, params: np.ndarray):
    """[ABS]+[POD]+[MX] KroQuant activation quantizer: transform, then MXFP4."""
    return quantize_mxfp4(transform(x, params))


def sq_transform(x: np.ndarray, inv_s: np.ndarray) -> np.ndarray:
    """[ABS] per-channel scaling (SmoothQuant): y_c = x_c / s_c, given 1/s_c."""
    return np.asarray(x, dtype=np.float64) * np.asarray(inv_s, dtype=np.float64)[None, :]


def sq_quantize(x: np.ndarray, inv_s: np.ndarray):
    return quantize_mxfp4(sq_transform(x, inv_s))


def fold_weights(W: np.ndarray, params: np.ndarray) -> np.ndarray:
    """[ABS] the inverse goes to the weights: W' = W blockdiag(T_j)^{-1} for
    W [n_out, d], so that W' (T x) = W x."""
    W = np.asarray(W, dtype=np.float64)
    Tinv = expand_inverse(params)
    n, d = W.shape
    Wb = W.reshape(n, d // BLOCK, BLOCK)
    out = np.einsum("njk,jki->nji", Wb, Tinv)
    return out.reshape(n, d)


def quantize_weights(W: np.ndarray, params: np.ndarray):
    """[ABS] the weight side of the W4A4 layer: the folded weights
    W' = W blockdiag(T_j)^{-1}, quantised to MXFP4 in 32-element blocks along
    the input dimension d (the dimension the GEMM sums over, blocked like the
    transformed activations).  Returns (codes [n, d/2], scales [n, d/32])."""
    return quantize_mxfp4(fold_weights(W, params))


def row_sum(x: np.ndarray, scale: float = 1.0) -> np.ndarray:
    """scale * sum over the row of x (fp64): the per-token mean with
    scale = 1/d, the weight row sums W 1 with scale = 1."""
    return scale * np.sum(np.asarray(x, dtype=np.float64), axis=1)


def quantize_centered(x: np.ndarray, params: np.ndarray, mu: np.ndarray):
    """[centering variant] the quantizer applied to the centred tokens:
    MXFP4(T (x - mu 1)) for each token row with its own offset mu (the
    per-token mean in the variant; any per-token constant restores exactly)."""
    x = np.asarray(x, dtype=np.float64)
    return quantize_mxfp4(transform(x - np.asarray(mu, dtype=np.float64)[:, None], params))


def gemm_mxfp4_rank1(codes_a, scales_a, codes_b, scales_b, mu, wsum) -> np.ndarray:
    """The layer on centred activations with the removed mean restored in
    full precision: Y = MXFP4(A) MXFP4(B)^T + mu wsum^T, where mu [M] are the
    per-token offsets and wsum [N] = W 1 the row sums of the unfolded weights:
    (x - mu 1) W^T + mu (W 1)^T = x W^T."""
    return gemm_mxfp4(codes_a, scales_a, codes_b, scales_b) + np.outer(
        np.asarray(mu, dtype=np.float64), np.asarray(wsum, dtype=np.float64))


def gemm_mxfp4(codes_a, scales_a, codes_b, scales_b) -> np.ndarray:
    """[ABS] the W4A4 linear layer on the quantised operands: every MXFP4
    value decoded (E2M1 code times its block's E8M0 scale), then
    Y = A B^T summed over the input dimension in fp64, where A [M, K] are the
    activation codes and B [N, K] the weight codes."""
    return dequant(codes_a, scales_a) @ dequant(codes_b, scales_b).T


def layer_error(x: np.ndarray, W: np.ndarray, params: np.ndarray) -> float:
    """[ABS] the quantised W4A4 layer against the unquantised one, as one
    number: ||Q(T x) Q(W T^-1)^T - x W^T||_F / ||x W^T||_F over the token rows
    of x [M, d] and the weight rows of W [N, d], where Q is MXFP4 in
    32-element blocks along d.  The pages learn the transform but state no
    objective; this is the plain reading of "closer to the full-precision
    output" (the quantity an offline fit of the parameters minimises)."""
    x = np.asarray(x, dtype=np.float64)
    W = np.asarray(W, dtype=np.float64)
    ca, sa = kq_quantize(x, params)
    cb, sb = quantize_weights(W, params)
    ref = x @ W.T
    return float(np.linalg.norm(gemm_mxfp4(ca, sa, cb, sb) - ref) / np.linalg.norm(ref))


def gemm_error_scale(codes_a, scales_a, codes_b, scales_b) -> np.ndarray:
    """sum_k |a_k| |b_k| per output: the size of the terms an fp32
    accumulation adds up."""
    return np.abs(dequant(codes_a, scales_a)) @ np.abs(dequant(codes_b, scales_b)).T


def sf_tile(scales: np.ndarray) -> np.ndarray:
    """Scale bytes [R, K/32] (row-major) in the blocked layout the tensor
    cores read scale factors from: for each 128-row tile and each group of 4
    scale columns (128 input channels), 512 bytes in which row r of the tile
    and scale column j of the group sit at byte (r % 32) * 16 + (r // 32) * 4 + j.
    Rows beyond R are padded to a multiple of 128 with zero bytes.  Returns a
    flat uint8 array [ceil(R/128), (K/32)/4, 512]."""
    scales = np.asarray(scales, dtype=np.uint8)
    R, ns = scales.shape
    assert ns % 4 == 0
    rt = (R + 127) // 128
    out = np.zeros((rt, ns // 4, 512), dtype=np.uint8)
    for r in range(R):
        for s in range(ns):
            out[r // 128, s // 4, (r % 32) * 16 + ((r % 128) // 32) * 4 + (s % 4)] = scales[r, s]
    return out


def fold_error_scale(W: np.ndarray, params: np.ndarray) -> np.ndarray:
    """|W| times the magnitude of the inverse factors U^{-1} L^{-1}."""
    params = np.asarray(params).reshape(-1, PARAMS_PER_BLOCK)

    def mag_inv(a, b, u):
        Linv = np.abs(np.array([[1.0, 0.0], [-float(a), 1.0]]))
        Uinv = np.abs(np.array([[1.0 / float(u), -float(b)], [0.0, float(u)]]))
        return Uinv @ Linv

    Tm = np.stack([_kron_all(_factors(p, mag_inv)) for p in params])
    W = np.abs(np.asarray(W, dtype=np.float64))
    n, d = W.shape
    return np.einsum("njk,jki->nji", W.reshape(n, d // BLOCK, BLOCK), Tm).reshape(n, d)


# ---------------------------------------------------------------------------
# which decisions a correct fp32 evaluation may take differently
# ---------------------------------------------------------------------------
E2M1_MIDPOINTS = np.array([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0])


def undecided(y: np.ndarray, tol: np.ndarray, rel: float = 1e-4):
    """Flags for outputs whose encoding an evaluation of y within +-tol may
    legitimately change.

    An element is flagged when its pre-rounding value r = y / 2**e lies within
    max(rel * b, tol / 2**e) of a rounding boundary b (an E2M1 midpoint), or
    when |y| <= tol (its sign, hence the sign bit of a zero code, is open).
    A block is flagged when its amax lies within max(rel * 2**k, tol_amax) of
    a power of two 2**k (its shared exponent is open); every element of a
    flagged block is flagged.  Returns (elem_flags [M, d], block_flags [M, nb]).
    """
    yb = _blocks(y)
    tb = _blocks(tol)
    M, nb, _ = yb.shape
    amax = np.max(np.abs(yb), axis=2)
    arg = np.argmax(np.abs(yb), axis=2)
    tol_amax = np.take_along_axis(tb, arg[:, :, None], axis=2)[..., 0]
    tol_amax = np.maximum(tol_amax, tb.max(axis=2))
    with np.errstate(divide="ignore"):
        k = np.floor(np.log2(np.where(amax > 0, amax, 1.0)))
    near = np.zeros_like(amax, dtype=bool)
    for kk in (k - 1, k, k + 1):
        p = 2.0 ** kk
        near |= np.abs(amax - p) <= np.maximum(rel * p, tol_amax)
    near &= amax > 0
    e = shared_exponent(amax)
    r = np.ldexp(yb, -e[:, :, None])
    tr = np.ldexp(tb, -e[:, :, None])
    mag = np.abs(r)[..., None]
    win = np.maximum(rel * E2M1_MIDPOINTS[None, None, None, :], tr[..., None])
    elem = np.any(np.abs(mag - E2M1_MIDPOINTS) <= win, axis=-1)
    elem |= np.abs(yb) <= tb
    elem |= near[:, :, None]
    return elem.reshape(M, nb * BLOCK), near
