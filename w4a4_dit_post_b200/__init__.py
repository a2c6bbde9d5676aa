"""Python binding of the KroQuant C ABI (``include/kq.h``, ``libkroquant.so``).

Argument marshalling only: every function checks that it was handed CUDA
tensors of the right dtype and shape, that every array the kernels read
through a raw pointer (parameters, inverse scales, offsets, row sums) holds
exactly the number of elements the call reads and sits on the same device as
the activations, allocates missing outputs with torch (device memory is
PyTorch's job here), and passes raw device pointers and the current torch
stream to the C function of the same name.  Sizes and devices are checked
before the CUDA check, so the checks also run on tensors of any device.  All arithmetic runs
in the library's sm_100a kernels; there is no CPU path.  If the library has
not been built, the first call raises ``RuntimeError`` (build it with
``python -m w4a4_dit_post_b200.build``).
"""
from __future__ import annotations

import ctypes
import os
import threading

import torch

from .build import LIB_PATH

__all__ = [
    "abi", "kq_quantize", "kq_quantize_sf_tiled", "kq_quantize_centered", "kq_row_sum",
    "kq_quantize_tc", "kq_transform", "sq_quantize", "kq_expand_params",
    "kq_fold_weights", "kq_quantize_weights", "kq_sf_tile", "kq_gemm_mxfp4", "kq_gemm_mxfp4_bf16", "kq_gemm_mxfp4_rank1",
    "kq_dequant",
    "kq_device_status",
    "kq_selftest_bounded_wait",
    "KroQuantError",
    "KQ_DTYPE_BF16", "KQ_DTYPE_F32", "KQ_MAX_D", "KQ_DEVSTAT_WAIT_TIMEOUT", "KQ_DEVSTAT_BAD_PARAMS",
    "EXPORTED_FUNCTIONS",
]

KQ_OK = 0
KQ_DTYPE_BF16 = 0
KQ_DTYPE_F32 = 1
KQ_MAX_D = 32768
KQ_DEVSTAT_WAIT_TIMEOUT = 0x1
KQ_DEVSTAT_BAD_PARAMS = 0x2

_c_void_p = ctypes.c_void_p
_i64 = ctypes.c_int64
_int = ctypes.c_int

# name -> (restype, argtypes), mirroring include/kq.h
_SIGNATURES = {
    "kq_quantize": (_int, [_c_void_p, _int, _i64, _i64, _c_void_p, _c_void_p, _c_void_p, _c_void_p]),
    "kq_quantize_tc": (_int, [_c_void_p, _int, _i64, _i64, _c_void_p, _c_void_p, _c_void_p, _c_void_p]),
    "kq_quantize_sf_tiled": (_int, [_c_void_p, _int, _i64, _i64, _c_void_p, _c_void_p, _c_void_p,
                                    _c_void_p]),
    "kq_transform": (_int, [_c_void_p, _int, _i64, _i64, _c_void_p, _c_void_p, _c_void_p]),
    "sq_quantize": (_int, [_c_void_p, _int, _i64, _i64, _c_void_p, _c_void_p, _c_void_p, _c_void_p]),
    "kq_expand_params": (_int, [_c_void_p, _i64, _c_void_p, _c_void_p]),
    "kq_fold_weights": (_int, [_c_void_p, _i64, _i64, _c_void_p, _c_void_p, _c_void_p]),
    "kq_quantize_weights": (_int, [_c_void_p, _i64, _i64, _c_void_p, _c_void_p, _c_void_p, _c_void_p]),
    "kq_sf_tile": (_int, [_c_void_p, _i64, _i64, _c_void_p, _c_void_p]),
    "kq_quantize_centered": (_int, [_c_void_p, _int, _i64, _i64, _c_void_p, _c_void_p, _c_void_p,
                                    _c_void_p, _c_void_p]),
    "kq_row_sum": (_int, [_c_void_p, _int, _i64, _i64, ctypes.c_float, _c_void_p, _c_void_p]),
    "kq_gemm_mxfp4_rank1": (_int, [_c_void_p, _c_void_p, _c_void_p, _c_void_p, _i64, _i64, _i64,
                                   _c_void_p, _c_void_p, _c_void_p, _c_void_p]),
    "kq_gemm_mxfp4": (_int, [_c_void_p, _c_void_p, _c_void_p, _c_void_p, _i64, _i64, _i64, _c_void_p,
                             _c_void_p]),
    "kq_gemm_mxfp4_bf16": (_int, [_c_void_p, _c_void_p, _c_void_p, _c_void_p, _i64, _i64, _i64, _c_void_p,
                                  _c_void_p]),
    "kq_dequant": (_int, [_c_void_p, _c_void_p, _i64, _i64, _c_void_p, _c_void_p]),
    "kq_device_status": (_int, [ctypes.POINTER(ctypes.c_uint32), _int]),
    "kq_selftest_bounded_wait": (_int, [ctypes.c_uint32, _c_void_p]),
    "kq_status_string": (ctypes.c_char_p, [_int]),
    "kq_last_error": (ctypes.c_char_p, []),
    "kq_version": (_int, []),
}
EXPORTED_FUNCTIONS = tuple(_SIGNATURES)

_lib = None
_lock = threading.Lock()


class KroQuantError(RuntimeError):
    def __init__(self, fn: str, status: int, detail: str, text: str):
        super().__init__(f"{fn}: {text} -- {detail}")
        self.status = status


def abi() -> ctypes.CDLL:
    """The loaded library with argument types set (raises if not built)."""
    global _lib
    if _lib is None:
        with _lock:
            if _lib is None:
                if not os.path.exists(LIB_PATH):
                    raise RuntimeError(
                        f"KroQuant CUDA library not found at {LIB_PATH}; build it with "
                        "`python -m w4a4_dit_post_b200.build` (there is no CPU fallback)")
                lib = ctypes.CDLL(LIB_PATH)
                for name, (res, args) in _SIGNATURES.items():
                    f = getattr(lib, name)
                    f.restype = res
                    f.argtypes = args
                _lib = lib
    return _lib


def _check(fn: str, status: int) -> None:
    if status != KQ_OK:
        lib = abi()
        raise KroQuantError(fn, status, lib.kq_last_error().decode(),
                            lib.kq_status_string(status).decode())


def _stream(t: torch.Tensor) -> int:
    return torch.cuda.current_stream(t.device).cuda_stream


def _need(name: str, t: torch.Tensor, dtypes, ndim: int | None = None) -> None:
    """Type, dtype, rank and contiguity of a tensor argument (any device)."""
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if t.dtype not in dtypes:
        raise TypeError(f"{name} has dtype {t.dtype}, expected one of {dtypes}")
    if ndim is not None and t.dim() != ndim:
        raise ValueError(f"{name} must be {ndim}-D, got shape {tuple(t.shape)}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")


def _need_cuda(name: str, t: torch.Tensor) -> None:
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor (the library takes device pointers)")


def _same_device(name: str, t: torch.Tensor, like: torch.Tensor, like_name: str) -> None:
    if t.device != like.device:
        raise ValueError(f"{name} is on {t.device}, {like_name} on {like.device}")


def _need_numel(name: str, t: torch.Tensor, n: int, what: str) -> None:
    # the kernels read exactly n elements through the raw pointer: a shorter
    # tensor would be read out of bounds
    if t.numel() != n:
        raise ValueError(f"{name} has {t.numel()} elements, expected {n} ({what})")


def _need_params(params: torch.Tensor, d: int, like: torch.Tensor, like_name: str = "x") -> None:
    """LU parameters: fp32, exactly 15 per 32-channel block of d, on like's device."""
    _need("params", params, (torch.float32,))
    _need_numel("params", params, 15 * (d // 32), f"15 LU parameters per 32-channel block of d = {d}")
    _same_device("params", params, like, like_name)


def _x_dtype(x: torch.Tensor) -> int:
    return KQ_DTYPE_BF16 if x.dtype == torch.bfloat16 else KQ_DTYPE_F32


def _out(t, shape, dtype, like, name):
    if t is None:
        return torch.empty(shape, dtype=dtype, device=like.device)
    _need(name, t, (dtype,))
    if tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} has shape {tuple(t.shape)}, expected {tuple(shape)}")
    _same_device(name, t, like, "the inputs")
    return t


_ACT = (torch.bfloat16, torch.float32)


def _activation(x, dtypes=_ACT):
    """x [M, d]: dtype, rank, contiguity; returns (M, d).  d is checked by
    the library (a positive multiple of 32)."""
    _need("x", x, dtypes, 2)
    return x.shape


def kq_quantize(x, params, codes=None, scales=None):
    """KroQuant quantizer: x [M, d] bf16/fp32, params [d/32, 15] fp32 ->
    (codes uint8 [M, d/2], scales uint8 [M, d/32])."""
    M, d = _activation(x)
    _need_params(params, d, x)
    _need_cuda("x", x)
    codes = _out(codes, (M, d // 2), torch.uint8, x, "codes")
    scales = _out(scales, (M, d // 32), torch.uint8, x, "scales")
    with torch.cuda.device(x.device):
        _check("kq_quantize", abi().kq_quantize(
            x.data_ptr(), _x_dtype(x), M, d, params.data_ptr(), codes.data_ptr(),
            scales.data_ptr(), _stream(x)))
    return codes, scales


def kq_quantize_sf_tiled(x, params, codes=None, scales_tiled=None):
    """kq_quantize with the scales in the blocked layout kq_gemm_mxfp4 reads:
    (codes uint8 [M, d/2], scales_tiled uint8 [ceil(M/128), d/128, 512])."""
    M, d = _activation(x)
    _need_params(params, d, x)
    _need_cuda("x", x)
    codes = _out(codes, (M, d // 2), torch.uint8, x, "codes")
    scales_tiled = _out(scales_tiled, ((M + 127) // 128, d // 128 if d % 128 == 0 else 0, 512),
                        torch.uint8, x, "scales_tiled")
    with torch.cuda.device(x.device):
        _check("kq_quantize_sf_tiled", abi().kq_quantize_sf_tiled(
            x.data_ptr(), _x_dtype(x), M, d, params.data_ptr(), codes.data_ptr(),
            scales_tiled.data_ptr(), _stream(x)))
    return codes, scales_tiled


def kq_quantize_tc(x, params, codes=None, scales=None):
    """Same result contract as kq_quantize, computed on the tensor cores
    (bf16 input only); kept for comparison with the SIMT path."""
    M, d = _activation(x, (torch.bfloat16,))
    _need_params(params, d, x)
    _need_cuda("x", x)
    codes = _out(codes, (M, d // 2), torch.uint8, x, "codes")
    scales = _out(scales, (M, d // 32), torch.uint8, x, "scales")
    with torch.cuda.device(x.device):
        _check("kq_quantize_tc", abi().kq_quantize_tc(
            x.data_ptr(), KQ_DTYPE_BF16, M, d, params.data_ptr(), codes.data_ptr(),
            scales.data_ptr(), _stream(x)))
    return codes, scales


def kq_transform(x, params, y=None):
    """Transform stage alone: y = blockdiag(T_j) x, fp32 [M, d]."""
    M, d = _activation(x)
    _need_params(params, d, x)
    _need_cuda("x", x)
    y = _out(y, (M, d), torch.float32, x, "y")
    with torch.cuda.device(x.device):
        _check("kq_transform", abi().kq_transform(
            x.data_ptr(), _x_dtype(x), M, d, params.data_ptr(), y.data_ptr(), _stream(x)))
    return y


def sq_quantize(x, inv_s, codes=None, scales=None):
    """SmoothQuant comparison quantizer: y_c = x_c * inv_s[c], then MXFP4."""
    M, d = _activation(x)
    _need("inv_s", inv_s, (torch.float32,), 1)
    _need_numel("inv_s", inv_s, d, "one inverse scale per channel")
    _same_device("inv_s", inv_s, x, "x")
    _need_cuda("x", x)
    codes = _out(codes, (M, d // 2), torch.uint8, x, "codes")
    scales = _out(scales, (M, d // 32), torch.uint8, x, "scales")
    with torch.cuda.device(x.device):
        _check("sq_quantize", abi().sq_quantize(
            x.data_ptr(), _x_dtype(x), M, d, inv_s.data_ptr(), codes.data_ptr(),
            scales.data_ptr(), _stream(x)))
    return codes, scales


def kq_expand_params(params, T=None):
    """params [nb, 15] -> T [nb, 32, 32] fp32."""
    _need("params", params, (torch.float32,))
    if params.numel() == 0 or params.numel() % 15:
        raise ValueError(f"params has {params.numel()} elements, expected a positive multiple of 15")
    _need_cuda("params", params)
    nb = params.numel() // 15
    T = _out(T, (nb, 32, 32), torch.float32, params, "T")
    with torch.cuda.device(params.device):
        _check("kq_expand_params", abi().kq_expand_params(
            params.data_ptr(), 32 * nb, T.data_ptr(), _stream(params)))
    return T


def kq_fold_weights(W, params, W_out=None):
    """W [N, d] fp32 -> W blockdiag(T_j)^{-1}.  Pass W_out=W for in place."""
    _need("W", W, (torch.float32,), 2)
    N, d = W.shape
    _need_params(params, d, W, "W")
    _need_cuda("W", W)
    W_out = _out(W_out, (N, d), torch.float32, W, "W_out")
    with torch.cuda.device(W.device):
        _check("kq_fold_weights", abi().kq_fold_weights(
            W.data_ptr(), N, d, params.data_ptr(), W_out.data_ptr(), _stream(W)))
    return W_out


def kq_quantize_weights(W, params, codes=None, scales=None):
    """Weight side: W [N, d] fp32 -> MXFP4 (codes uint8 [N, d/2], scales
    uint8 [N, d/32]) of the folded weights W blockdiag(T_j)^{-1}."""
    _need("W", W, (torch.float32,), 2)
    N, d = W.shape
    _need_params(params, d, W, "W")
    _need_cuda("W", W)
    codes = _out(codes, (N, d // 2), torch.uint8, W, "codes")
    scales = _out(scales, (N, d // 32), torch.uint8, W, "scales")
    with torch.cuda.device(W.device):
        _check("kq_quantize_weights", abi().kq_quantize_weights(
            W.data_ptr(), N, d, params.data_ptr(), codes.data_ptr(), scales.data_ptr(), _stream(W)))
    return codes, scales


def kq_sf_tile(scales, out=None):
    """Scale bytes [R, K/32] -> the blocked layout [ceil(R/128), K/128, 512]
    that kq_gemm_mxfp4 reads."""
    _need("scales", scales, (torch.uint8,), 2)
    _need_cuda("scales", scales)
    R, ns = scales.shape
    K = 32 * ns
    out = _out(out, ((R + 127) // 128, K // 128 if K % 128 == 0 else 0, 512), torch.uint8, scales, "out")
    with torch.cuda.device(scales.device):
        _check("kq_sf_tile", abi().kq_sf_tile(scales.data_ptr(), R, K, out.data_ptr(), _stream(scales)))
    return out


def _gemm_shapes(a_codes, a_sf_tiled, b_codes, b_sf_tiled):
    for name, t in (("a_codes", a_codes), ("b_codes", b_codes)):
        _need(name, t, (torch.uint8,), 2)
    for name, t in (("a_sf_tiled", a_sf_tiled), ("b_sf_tiled", b_sf_tiled)):
        _need(name, t, (torch.uint8,), 3)
    M, half = a_codes.shape
    N = b_codes.shape[0]
    K = 2 * half
    if b_codes.shape[1] != half:
        raise ValueError("a_codes and b_codes disagree on K")
    for name, t, rows in (("a_sf_tiled", a_sf_tiled, M), ("b_sf_tiled", b_sf_tiled, N)):
        if tuple(t.shape) != ((rows + 127) // 128, K // 128, 512):
            raise ValueError(f"{name} has shape {tuple(t.shape)}, expected "
                             f"{((rows + 127) // 128, K // 128, 512)}")
    for name, t in (("a_sf_tiled", a_sf_tiled), ("b_codes", b_codes), ("b_sf_tiled", b_sf_tiled)):
        _same_device(name, t, a_codes, "a_codes")
    return M, N, K


def kq_gemm_mxfp4(a_codes, a_sf_tiled, b_codes, b_sf_tiled, Y=None):
    """Y [M, N] fp32 = MXFP4(A) MXFP4(B)^T from codes [M, K/2] / [N, K/2] and
    scales tiled by kq_sf_tile."""
    M, N, K = _gemm_shapes(a_codes, a_sf_tiled, b_codes, b_sf_tiled)
    _need_cuda("a_codes", a_codes)
    Y = _out(Y, (M, N), torch.float32, a_codes, "Y")
    with torch.cuda.device(a_codes.device):
        _check("kq_gemm_mxfp4", abi().kq_gemm_mxfp4(
            a_codes.data_ptr(), a_sf_tiled.data_ptr(), b_codes.data_ptr(), b_sf_tiled.data_ptr(),
            M, N, K, Y.data_ptr(), _stream(a_codes)))
    return Y


def kq_gemm_mxfp4_bf16(a_codes, a_sf_tiled, b_codes, b_sf_tiled, Y=None):
    """kq_gemm_mxfp4 with Y [M, N] bf16 (each fp32 sum rounded to nearest even)."""
    M, N, K = _gemm_shapes(a_codes, a_sf_tiled, b_codes, b_sf_tiled)
    _need_cuda("a_codes", a_codes)
    Y = _out(Y, (M, N), torch.bfloat16, a_codes, "Y")
    with torch.cuda.device(a_codes.device):
        _check("kq_gemm_mxfp4_bf16", abi().kq_gemm_mxfp4_bf16(
            a_codes.data_ptr(), a_sf_tiled.data_ptr(), b_codes.data_ptr(), b_sf_tiled.data_ptr(),
            M, N, K, Y.data_ptr(), _stream(a_codes)))
    return Y


def kq_row_sum(x, scale=1.0, out=None):
    """out [M] fp32 = scale * row sums of x [M, d] (bf16 or fp32)."""
    M, d = _activation(x)
    _need_cuda("x", x)
    out = _out(out, (M,), torch.float32, x, "out")
    with torch.cuda.device(x.device):
        _check("kq_row_sum", abi().kq_row_sum(x.data_ptr(), _x_dtype(x), M, d, float(scale),
                                              out.data_ptr(), _stream(x)))
    return out


def kq_quantize_centered(x, params, mu, codes=None, scales=None):
    """Centring variant: MXFP4(T (x - mu 1)) with mu [M] fp32 per-token offsets."""
    M, d = _activation(x)
    _need_params(params, d, x)
    _need("mu", mu, (torch.float32,), 1)
    _need_numel("mu", mu, M, "one offset per row of x")
    _same_device("mu", mu, x, "x")
    _need_cuda("x", x)
    codes = _out(codes, (M, d // 2), torch.uint8, x, "codes")
    scales = _out(scales, (M, d // 32), torch.uint8, x, "scales")
    with torch.cuda.device(x.device):
        _check("kq_quantize_centered", abi().kq_quantize_centered(
            x.data_ptr(), _x_dtype(x), M, d, params.data_ptr(), mu.data_ptr(), codes.data_ptr(),
            scales.data_ptr(), _stream(x)))
    return codes, scales


def kq_gemm_mxfp4_rank1(a_codes, a_sf_tiled, b_codes, b_sf_tiled, mu, wsum, Y=None):
    """kq_gemm_mxfp4 plus mu wsum^T (mu [M], wsum [N] fp32)."""
    M, N, K = _gemm_shapes(a_codes, a_sf_tiled, b_codes, b_sf_tiled)
    _need("mu", mu, (torch.float32,), 1)
    _need("wsum", wsum, (torch.float32,), 1)
    _need_numel("mu", mu, M, "one offset per activation row")
    _need_numel("wsum", wsum, N, "one row sum per weight row")
    _same_device("mu", mu, a_codes, "a_codes")
    _same_device("wsum", wsum, a_codes, "a_codes")
    _need_cuda("a_codes", a_codes)
    Y = _out(Y, (M, N), torch.float32, a_codes, "Y")
    with torch.cuda.device(a_codes.device):
        _check("kq_gemm_mxfp4_rank1", abi().kq_gemm_mxfp4_rank1(
            a_codes.data_ptr(), a_sf_tiled.data_ptr(), b_codes.data_ptr(), b_sf_tiled.data_ptr(),
            M, N, K, mu.data_ptr(), wsum.data_ptr(), Y.data_ptr(), _stream(a_codes)))
    return Y


def kq_dequant(codes, scales, out=None):
    """MXFP4 -> fp32 [M, d]."""
    _need("codes", codes, (torch.uint8,), 2)
    _need("scales", scales, (torch.uint8,), 2)
    M, half = codes.shape
    d = 2 * half
    if tuple(scales.shape) != (M, d // 32):
        raise ValueError("scales shape does not match codes")
    _same_device("scales", scales, codes, "codes")
    _need_cuda("codes", codes)
    out = _out(out, (M, d), torch.float32, codes, "out")
    with torch.cuda.device(codes.device):
        _check("kq_dequant", abi().kq_dequant(
            codes.data_ptr(), scales.data_ptr(), M, d, out.data_ptr(), _stream(codes)))
    return out


def kq_device_status(device=None, clear: bool = False) -> int:
    """KQ_DEVSTAT_* bits of a device (synchronises the device)."""
    dev = torch.device("cuda", torch.cuda.current_device()) if device is None else torch.device(device)
    flags = ctypes.c_uint32(0)
    with torch.cuda.device(dev):
        _check("kq_device_status", abi().kq_device_status(ctypes.byref(flags), int(bool(clear))))
    return flags.value


def kq_selftest_bounded_wait(limit_us: int, device=None) -> None:
    """Enqueue the bounded-wait self-test on the current stream of `device`."""
    dev = torch.device("cuda", torch.cuda.current_device()) if device is None else torch.device(device)
    with torch.cuda.device(dev):
        _check("kq_selftest_bounded_wait", abi().kq_selftest_bounded_wait(
            int(limit_us), torch.cuda.current_stream(dev).cuda_stream))
