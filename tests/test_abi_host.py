"""Host-side checks of the C ABI that need no GPU: the library loads, exports
every entry point include/fftconv.h declares, and rejects bad arguments before
touching the device."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared():
    with open(os.path.join(ROOT, "include", "fftconv.h")) as f:
        text = f.read()
    return sorted(set(re.findall(r"FFTCONV_API\s+[\w\s\*]+?\b(fftconv_\w+)\s*\(", text)))


def test_header_declares_the_entry_points():
    names = _declared()
    for n in ("fftconv_plan_create", "fftconv_filter_precompute", "fftconv_forward", "fftconv_plan_destroy"):
        assert n in names
    assert len(names) >= 15


def test_library_exports_every_declared_symbol():
    import long_sequence_fft_b200 as lsf
    lib = ctypes.CDLL(lsf.LIB_PATH)
    for n in _declared():
        assert hasattr(lib, n), n
    assert lsf.version().startswith("fftconv-b200")


def test_status_strings_and_null_handles():
    import long_sequence_fft_b200 as lsf
    lib = lsf.library()
    for code in (0, -1, -2, -3, -4, -5, -6):
        assert lib.fftconv_status_string(code)
    assert lib.fftconv_filter_bytes(None) == 0
    assert lib.fftconv_workspace_bytes(None) == 0
    assert lib.fftconv_plan_destroy(None) == 0
    assert lib.fftconv_plan_path(None) == lsf.ERR_INVALID_ARG
    assert lib.fftconv_forward(None, None, None, None, 1, 1, 1, None, None, None, 0, None) == lsf.ERR_INVALID_ARG
    assert b"plan" in lib.fftconv_last_error()
    assert lib.fftconv_selftest_bounded_wait(None, 16, 0, None) == lsf.ERR_INVALID_ARG


@pytest.mark.parametrize("N,H,dtype,order,L,status", [
    (1000, 2, 0, 0, 1000, -2),     # not a power of two
    (128, 2, 0, 0, 128, -2),       # below the minimum length
    (1 << 23, 2, 0, 0, 1 << 23, -2),
    (1024, 0, 0, 0, 1024, -1),     # no channels
    (1024, 2, 7, 0, 1024, -1),     # unknown dtype
    (1024, 2, 0, 9, 1024, -2),     # unknown order
    (1024, 2, 0, 6, 1024, -2),
    (32768, 2, 0, 5, 32768, -2),   # tensor-core staged rows: fp16/bf16 only,
    (8192, 2, 1, 5, 8192, -2),     # N >= 16384,
    (32768, 2, 2, 5, 2049, -2),    # and filters longer than the windows take
    (1024, 2, 0, 0, 2048, -1),     # filter longer than the sequence
    (1024, 2, 0, 0, 0, -1),
])
def test_plan_create_rejects_bad_arguments(N, H, dtype, order, L, status):
    import long_sequence_fft_b200 as lsf
    h = ctypes.c_void_p(1)
    rc = lsf.library().fftconv_plan_create_ex(ctypes.byref(h), N, H, dtype, order, L)
    assert rc == status
    assert not h.value
    assert lsf.library().fftconv_last_error()


def test_fftconv_refuses_a_mask_with_grad_before_any_device_work():
    # the backward pass takes no block mask: the refusal comes first, so it
    # holds on tensors that never reach a plan
    import torch
    import long_sequence_fft_b200 as lsf
    u = torch.zeros((2, 3, 256), requires_grad=True)
    k = torch.zeros((3, 256))
    with pytest.raises(NotImplementedError):
        lsf.fftconv(u, k, mask=torch.ones((1, 8), dtype=torch.uint8))
