"""Plant typical mistakes in copies of the CPU oracle and check that at least
one pin catches each of them.  The mistakes are planted in the oracle, on the
CPU; nothing here touches the CUDA library."""
import importlib.util
import os

import numpy as np
import pytest

from oracle_pins import ALL_PINS

ORACLE_PATH = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))),
                           "oracle", "kq_oracle.py")


def fresh_oracle():
    spec = importlib.util.spec_from_file_location("kq_oracle_mutant", ORACLE_PATH)
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


def m_transposed_factor(o):
    f = o.lu_factor
    o.lu_factor = lambda a, b, u: f(a, b, u).T


def m_upper_times_lower(o):
    def uL(a, b, u):
        L = np.array([[1.0, 0.0], [float(a), 1.0]])
        U = np.array([[float(u), float(b)], [0.0, 1.0 / float(u)]])
        return U @ L
    o.lu_factor = uL


def m_dropped_ab_term(o):
    o.lu_factor = lambda a, b, u: np.array([[u, b], [a * u, 1.0 / u]], dtype=np.float64)


def m_reversed_kron_order(o):
    k = o._kron_all
    o._kron_all = lambda mats: k(list(reversed(mats)))


def m_row_vector_convention(o):
    f = o.apply_blockdiag
    o.apply_blockdiag = lambda x, T: f(x, np.transpose(T, (0, 2, 1)))


def m_inverse_sign(o):
    def inv(a, b, u):
        Linv = np.array([[1.0, 0.0], [-float(a), 1.0]])
        Uinv = np.array([[1.0 / float(u), float(b)], [0.0, float(u)]])
        return Uinv @ Linv
    o.lu_factor_inverse = inv


def m_inverse_wrong_order(o):
    def inv(a, b, u):
        Linv = np.array([[1.0, 0.0], [-float(a), 1.0]])
        Uinv = np.array([[1.0 / float(u), -float(b)], [0.0, float(u)]])
        return Linv @ Uinv
    o.lu_factor_inverse = inv


def m_ceil_scale(o):
    def se(amax):
        amax = np.asarray(amax, dtype=np.float64)
        c = np.ceil(np.log2(np.where(amax > 0, amax, 2.0 ** -200)))
        return np.clip(c - o.E2M1_EMAX, -127, 127).astype(np.int64)
    o.shared_exponent = se


def m_emax_three(o):
    o.E2M1_EMAX = 3


def m_ties_away(o):
    f = o.e2m1_round_magnitude

    def r(mag):
        mag = np.asarray(mag, dtype=np.float64)
        E = np.clip(np.floor(np.log2(np.where(mag > 0, mag, 1.0))), 0, 2)
        step = np.where(mag < 1.0, 0.5, 2.0 ** (E - 1))
        return np.minimum(np.floor(mag / step + 0.5) * step, 6.0)
    o.e2m1_round_magnitude = r


def m_truncate(o):
    def r(mag):
        mag = np.asarray(mag, dtype=np.float64)
        E = np.clip(np.floor(np.log2(np.where(mag > 0, mag, 1.0))), 0, 2)
        step = np.where(mag < 1.0, 0.5, 2.0 ** (E - 1))
        return np.minimum(np.floor(mag / step) * step, 6.0)
    o.e2m1_round_magnitude = r


def m_swapped_nibbles(o):
    f = o.quantize_mxfp4

    def q(y):
        c, s = f(y)
        return ((c >> 4) | ((c & 0xF) << 4)).astype(np.uint8), s
    o.quantize_mxfp4 = q


def m_unsigned_zero(o):
    f = o.e2m1_code

    def c(r):
        out = f(r)
        return np.where((out & 7) == 0, 0, out).astype(np.uint8)
    o.e2m1_code = c


def m_bias_128(o):
    o.E8M0_BIAS = 128


def m_fold_uses_forward(o):
    o.expand_inverse = o.expand_params


def m_nan_not_flagged(o):
    f = o.quantize_mxfp4

    def q(y):
        y = np.nan_to_num(np.asarray(y, dtype=np.float64), nan=0.0, posinf=0.0, neginf=0.0)
        return f(y)
    o.quantize_mxfp4 = q


def m_wrong_grid(o):
    o.E2M1_MAGNITUDES = np.array([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 5.0])


def m_weights_not_folded(o):
    o.quantize_weights = lambda W, params: o.quantize_mxfp4(W)


def m_weights_folded_with_forward(o):
    def qw(W, params):
        T = o.expand_params(params)
        n, d = np.asarray(W).shape
        Wb = np.asarray(W, dtype=np.float64).reshape(n, d // 32, 32)
        return o.quantize_mxfp4(np.einsum("njk,jki->nji", Wb, T).reshape(n, d))
    o.quantize_weights = qw


def m_centering_after_transform(o):
    o.quantize_centered = lambda x, params, mu: o.quantize_mxfp4(
        o.transform(np.asarray(x, dtype=np.float64), params) - np.asarray(mu, dtype=np.float64)[:, None])


# the tolerance functions: each scaled by 10, or a term dropped or misplaced
def m_error_scale_x10(o):
    f = o.error_scale
    o.error_scale = lambda x, params: 10.0 * f(x, params)


def m_expand_magnitude_x10(o):
    f = o.expand_magnitude
    o.expand_magnitude = lambda params: 10.0 * f(params)


def m_lu_factor_magnitude_x10(o):
    f = o.lu_factor_magnitude
    o.lu_factor_magnitude = lambda a, b, u: 10.0 * f(a, b, u)


def m_error_scale_uses_abs_T(o):
    o.expand_magnitude = lambda params: np.abs(o.expand_params(params))


def m_fold_error_scale_x10(o):
    f = o.fold_error_scale
    o.fold_error_scale = lambda W, params: 10.0 * f(W, params)


def m_gemm_error_scale_x10(o):
    f = o.gemm_error_scale
    o.gemm_error_scale = lambda *a: 10.0 * f(*a)


def m_undecided_tol_x10(o):
    f = o.undecided
    o.undecided = lambda y, tol, rel=1e-4: f(y, 10.0 * np.asarray(tol), rel)


def m_undecided_rel_x10(o):
    f = o.undecided
    o.undecided = lambda y, tol, rel=1e-4: f(y, tol, 10.0 * rel)


def m_undecided_tol_times_scale(o):
    """tol * 2^e instead of tol / 2^e in the element window."""
    src = open(ORACLE_PATH).read()
    assert "tr = np.ldexp(tb, -e[:, :, None])" in src
    ns = {}
    exec(compile(src.replace("tr = np.ldexp(tb, -e[:, :, None])", "tr = np.ldexp(tb, e[:, :, None])"),
                 ORACLE_PATH, "exec"), ns)
    o.undecided = ns["undecided"]


def m_undecided_no_sign_branch(o):
    src = open(ORACLE_PATH).read()
    assert "elem |= np.abs(yb) <= tb" in src
    ns = {}
    exec(compile(src.replace("elem |= np.abs(yb) <= tb", "pass"), ORACLE_PATH, "exec"), ns)
    o.undecided = ns["undecided"]



def m_layer_error_unfolded_weights(o):
    def le(x, W, params):
        ca, sa = o.kq_quantize(np.asarray(x, dtype=np.float64), params)
        cb, sb = o.quantize_mxfp4(np.asarray(W, dtype=np.float64))
        ref = np.asarray(x, dtype=np.float64) @ np.asarray(W, dtype=np.float64).T
        return float(np.linalg.norm(o.gemm_mxfp4(ca, sa, cb, sb) - ref) / np.linalg.norm(ref))
    o.layer_error = le


MUTANTS = [v for k, v in sorted(globals().items()) if k.startswith("m_")]


@pytest.mark.parametrize("mutate", MUTANTS, ids=lambda f: f.__name__)
def test_some_pin_catches(mutate):
    o = fresh_oracle()
    mutate(o)
    caught = []
    for pin in ALL_PINS:
        try:
            pin(o)
        except Exception as e:     # an assertion or a crash both count
            caught.append(pin.__name__)
    assert caught, f"no pin caught mutant {mutate.__name__}"
