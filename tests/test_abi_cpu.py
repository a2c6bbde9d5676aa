"""The C-ABI library without a GPU: it builds for sm_100a, loads, exports
every function include/kq.h declares, and rejects bad arguments on the host
with the documented status before touching the device.  No compute call is
made here (arguments that pass the checks are only used with M == 0)."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "kq.h")


@pytest.fixture(scope="module")
def lib():
    from w4a4_dit_post_b200 import build
    build.build()
    import w4a4_dit_post_b200 as k
    return k.abi()


def header_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"^\s*(?:const\s+)?\w+\**\s+\**((?:kq|sq)_\w+)\s*\(", text, re.M)))


def test_header_declares_the_abi():
    names = header_functions()
    for want in ("kq_quantize", "kq_quantize_sf_tiled", "kq_quantize_centered", "kq_row_sum",
                 "kq_gemm_mxfp4_rank1", "kq_quantize_tc", "kq_transform", "sq_quantize", "kq_expand_params",
                 "kq_fold_weights", "kq_quantize_weights", "kq_sf_tile", "kq_gemm_mxfp4", "kq_gemm_mxfp4_bf16",
                 "kq_dequant", "kq_status_string",
                 "kq_device_status"):
        assert want in names


def test_every_declared_symbol_is_exported(lib):
    import w4a4_dit_post_b200 as k
    names = header_functions()
    assert sorted(k.EXPORTED_FUNCTIONS) == names
    for n in names:
        assert hasattr(lib, n), n


def test_library_is_sm100a(lib):
    from w4a4_dit_post_b200 import build
    assert "arch=compute_100a,code=sm_100a" in " ".join(build.ARCH_FLAGS)
    assert build.is_current()


def test_status_strings(lib):
    for code in range(6):
        s = lib.kq_status_string(code).decode()
        assert s.startswith("KQ_")
    assert lib.kq_status_string(99).decode()
    assert lib.kq_version() == 10000


# fake, suitably aligned device addresses: never dereferenced by these calls
A16 = 0x7F0000000000
A16b = 0x7F0000100000
A16c = 0x7F0000200000
A16d = 0x7F0000300000


def test_quantize_argument_checks(lib):
    q = lib.kq_quantize
    assert q(None, 0, 4, 64, A16b, A16c, A16d, None) == 1          # NULL x
    assert q(A16, 0, 4, 64, None, A16c, A16d, None) == 1           # NULL params
    assert q(A16, 0, 4, 64, A16b, None, A16d, None) == 1           # NULL codes
    assert q(A16, 0, 4, 64, A16b, A16c, None, None) == 1           # NULL scales
    assert q(A16, 0, -1, 64, A16b, A16c, A16d, None) == 1          # M < 0
    assert q(A16, 0, 4, 48, A16b, A16c, A16d, None) == 1           # d % 32
    assert q(A16, 0, 4, 0, A16b, A16c, A16d, None) == 1            # d == 0
    assert q(A16, 7, 4, 64, A16b, A16c, A16d, None) == 3           # dtype
    assert q(A16 + 8, 0, 4, 64, A16b, A16c, A16d, None) == 2       # x alignment
    assert q(A16, 0, 4, 64, A16b + 2, A16c, A16d, None) == 2       # params alignment
    assert q(A16, 0, 4, 64, A16b, A16c + 4, A16d, None) == 2       # codes alignment
    assert q(A16, 0, 4, 32768 + 32, A16b, A16c, A16d, None) == 4   # d limit
    assert q(A16, 0, 2 ** 40, 1024, A16b, A16c, A16d, None) == 4   # block count
    assert q(A16, 0, 2 ** 30, 32, A16b, A16c, A16d, None) == 4     # row count (M < 2^30)
    assert lib.sq_quantize(A16, 0, 2 ** 30, 32, A16b, A16c, A16d, None) == 4
    assert q(A16, 0, 0, 64, A16b, A16c, A16d + 1, None) == 0       # M == 0: no-op
    assert q(None, 0, 0, 64, None, None, None, None) == 0          # ... pointers unused
    assert q(None, 0, 0, 48, None, None, None, None) == 1          # shape still checked
    assert b"kq_quantize" in lib.kq_last_error()


def test_tensor_core_variant_checks(lib):
    t = lib.kq_quantize_tc
    assert t(A16, 1, 4, 64, A16b, A16c, A16d, None) == 3          # fp32 input refused
    assert t(A16, 0, 4, 48, A16b, A16c, A16d, None) == 1
    assert t(A16 + 8, 0, 4, 64, A16b, A16c, A16d, None) == 2
    assert t(None, 0, 0, 64, None, None, None, None) == 0          # M == 0


def test_other_argument_checks(lib):
    assert lib.kq_transform(A16, 0, 4, 64, A16b, A16c + 4, None) == 2
    assert lib.kq_transform(A16, 1, 0, 64, A16b, A16c, None) == 0
    assert lib.sq_quantize(A16, 0, 4, 33, A16b, A16c, A16d, None) == 1
    assert lib.sq_quantize(A16, 1, 0, 64, A16b, A16c, A16d, None) == 0
    assert lib.kq_expand_params(None, 64, A16, None) == 1
    assert lib.kq_expand_params(A16, 40, A16b, None) == 1
    assert lib.kq_fold_weights(A16, 4, 64, A16b, A16 + 8, None) == 2
    assert lib.kq_fold_weights(A16, 4, 64, A16b, A16 + 64, None) == 1   # partial overlap
    assert lib.kq_fold_weights(A16, 0, 64, A16b, A16c, None) == 0
    assert lib.kq_fold_weights(None, 0, 64, None, None, None) == 0
    assert lib.kq_quantize_weights(A16, 4, 64, A16b, A16c + 8, A16d, None) == 2
    assert lib.kq_quantize_weights(A16 + 4, 4, 64, A16b, A16c, A16d, None) == 2
    assert lib.kq_quantize_weights(A16, 4, 48, A16b, A16c, A16d, None) == 1
    assert lib.kq_quantize_weights(A16, 4, 64, None, A16c, A16d, None) == 1
    assert lib.kq_quantize_weights(None, 0, 64, None, None, None, None) == 0
    assert lib.kq_sf_tile(A16, 4, 96, A16b, None) == 1                  # K % 128
    assert lib.kq_quantize_centered(A16, 0, 4, 64, A16b, None, A16c, A16d, None) == 1   # NULL mu
    assert lib.kq_quantize_centered(A16, 0, 4, 64, A16b, A16 + 2, A16c, A16d, None) == 2
    assert lib.kq_row_sum(A16, 2, 4, 64, 1.0, A16b, None) == 3
    assert lib.kq_row_sum(A16 + 8, 0, 4, 64, 1.0, A16b, None) == 2
    assert lib.kq_gemm_mxfp4_rank1(A16, A16b, A16c, A16d, 128, 128, 256, None, A16, A16, None) == 1
    assert lib.kq_quantize_sf_tiled(A16, 0, 4, 96, A16b, A16c, A16d, None) == 1   # d % 128
    assert lib.kq_quantize_sf_tiled(None, 0, 0, 128, None, None, None, None) == 0
    assert lib.kq_sf_tile(None, 0, 128, None, None) == 0
    g = lib.kq_gemm_mxfp4
    assert g(A16, A16b, A16c, A16d, 128, 128, 192, A16, None) == 1        # K % 128
    assert g(A16 + 8, A16b, A16c, A16d, 128, 128, 256, A16, None) == 2
    assert g(A16, A16b, A16c, A16d, 0, 128, 256, None, None) == 0
    assert g(A16, A16b, None, A16d, 128, 128, 256, A16, None) == 1
    assert g(A16, A16b, A16c, A16d, 2 ** 31, 128, 256, A16, None) == 4
    assert lib.kq_dequant(A16, A16b, 4, 64, A16c + 4, None) == 2
    assert lib.kq_dequant(A16, A16b, 0, 64, A16c, None) == 0
    assert lib.kq_device_status(None, 0) == 1
    assert lib.kq_selftest_bounded_wait(0, None) == 1
    assert lib.kq_selftest_bounded_wait(2000000, None) == 1


def test_binding_refuses_host_tensors(lib):
    import torch
    import w4a4_dit_post_b200 as k
    x = torch.zeros(4, 64, dtype=torch.bfloat16)
    p = torch.zeros(2, 15)
    with pytest.raises(ValueError, match="CUDA tensor"):
        k.kq_quantize(x, p)
    with pytest.raises(ValueError, match="CUDA tensor"):
        k.kq_dequant(torch.zeros(4, 32, dtype=torch.uint8), torch.zeros(4, 2, dtype=torch.uint8))


def test_binding_checks_array_sizes_and_devices(lib):
    """The kernels read 15 parameters per 32-channel block (d inverse scales,
    M offsets) through a raw pointer; an undersized array or one on another
    device must be refused before anything is launched.  Sizes and devices
    are checked before the CUDA check, so CPU tensors exercise them here."""
    import torch
    import w4a4_dit_post_b200 as k
    x = torch.zeros(4, 64, dtype=torch.bfloat16)
    good = torch.zeros(2, 15)
    for bad in (torch.zeros(1, 15), torch.zeros(2, 14), torch.zeros(45)):
        for fn in (k.kq_quantize, k.kq_quantize_sf_tiled, k.kq_transform):
            with pytest.raises(ValueError, match="params has"):
                fn(x, bad)
        with pytest.raises(ValueError, match="params has"):
            k.kq_quantize_tc(x, bad)
        with pytest.raises(ValueError, match="params has"):
            k.kq_quantize_centered(x, bad, torch.zeros(4))
        with pytest.raises(ValueError, match="params has"):
            k.kq_fold_weights(torch.zeros(3, 64), bad)
        with pytest.raises(ValueError, match="params has"):
            k.kq_quantize_weights(torch.zeros(3, 64), bad)
    meta = torch.zeros(2, 15, device="meta")
    with pytest.raises(ValueError, match="params is on meta"):
        k.kq_quantize(x, meta)
    with pytest.raises(ValueError, match="params is on meta"):
        k.kq_quantize_weights(torch.zeros(3, 64), meta)
    with pytest.raises(ValueError, match="inv_s has 63"):
        k.sq_quantize(x, torch.zeros(63))
    with pytest.raises(ValueError, match="inv_s is on meta"):
        k.sq_quantize(x, torch.zeros(64, device="meta"))
    with pytest.raises(ValueError, match="mu has 3"):
        k.kq_quantize_centered(x, good, torch.zeros(3))
    with pytest.raises(ValueError, match="mu is on meta"):
        k.kq_quantize_centered(x, good, torch.zeros(4, device="meta"))
    with pytest.raises(ValueError, match="positive multiple of 15"):
        k.kq_expand_params(torch.zeros(16))
    ca = torch.zeros(128, 64, dtype=torch.uint8)
    ta = torch.zeros(1, 1, 512, dtype=torch.uint8)
    with pytest.raises(ValueError, match="wsum has 3"):
        k.kq_gemm_mxfp4_rank1(ca, ta, ca, ta, torch.zeros(128), torch.zeros(3))
    with pytest.raises(ValueError, match="b_codes is on meta"):
        k.kq_gemm_mxfp4(ca, ta, ca.to("meta"), ta)
    # well-formed CPU tensors get as far as the device check
    with pytest.raises(ValueError, match="CUDA tensor"):
        k.kq_quantize(x, good)
    with pytest.raises(ValueError, match="CUDA tensor"):
        k.sq_quantize(x, torch.zeros(64))
