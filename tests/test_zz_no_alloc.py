"""fftconv_forward_noalloc: the convolution for callers that may not allocate
device memory (a host framework whose memory pool owns all device memory, or
a latency-critical path that cannot pay for cudaMalloc's synchronisation).

It runs the staged passes with their scratch in the library's static device
arrays instead of a plan workspace.  These tests call it through the C ABI
and compare it with fftconv_forward on an order-4 plan (the existing entry
point with the same passes) on two calls in a row with different inputs, so
the second call also shows that nothing the first call left in the shared
scratch leaks into its result.  This file is collected last on purpose."""
import ctypes

import numpy as np
import pytest

import workloads as W
from parity_util import assert_close, to_dev


def _lib():
    import long_sequence_fft_b200 as lsf
    lib = lsf.library()
    f = lib.fftconv_forward_noalloc
    f.restype = ctypes.c_int
    f.argtypes = [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int64, ctypes.c_int64,
                  ctypes.c_int64, ctypes.c_int, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p,
                  ctypes.c_int64, ctypes.c_void_p]
    return lsf, f


def test_noalloc_rejects_sizes_beyond_its_scratch():
    lsf, f = _lib()
    rc = f(None, None, None, 1, 1, 1 << 21, lsf.BF16, None, None, None, 0, None)
    assert rc == lsf.ERR_UNSUPPORTED
    assert b"static scratch" in lsf.library().fftconv_last_error()


@pytest.mark.gpu
@pytest.mark.parametrize("dtype,N,gated,masked", [("bf16", 4096, True, False), ("f32", 1024, False, True),
                                                  ("f16", 32768, False, False)])
def test_noalloc_matches_plan_entry_point_twice(dtype, N, gated, masked):
    import torch
    lsf, f = _lib()
    B, H = 3, 2
    plan = lsf.Plan(N, H, dtype, order=4)
    codes = {"f32": lsf.F32, "f16": lsf.F16, "bf16": lsf.BF16}
    rng = np.random.default_rng(N + B)
    k = W.round_to(rng.standard_normal((H, N), dtype=np.float32) / np.float32(np.sqrt(N)), dtype)
    Kf = plan.precompute(to_dev(k, dtype))
    mask = None
    if masked:
        mask = torch.from_numpy((rng.random((H, N // 32)) < 0.5).astype(np.uint8)).cuda()
    stream = torch.cuda.current_stream().cuda_stream
    for call in range(2):
        u = to_dev(W.round_to(rng.standard_normal((B, H, N), dtype=np.float32), dtype), dtype)
        w = to_dev(W.round_to(rng.standard_normal((B, H, N), dtype=np.float32), dtype), dtype) if gated else None
        v = to_dev(W.round_to(rng.standard_normal((B, H, N), dtype=np.float32), dtype), dtype) if gated else None
        ref = plan.forward(u, Kf, w=w, v=v, mask=mask)
        y = torch.full_like(u, float("nan"))
        rc = f(u.data_ptr(), Kf.data_ptr(), y.data_ptr(), B, H, N, codes[dtype],
               None if w is None else w.data_ptr(), None if v is None else v.data_ptr(),
               None if mask is None else mask.data_ptr(), 0 if mask is None else mask.shape[0], stream)
        assert rc == 0, lsf.library().fftconv_last_error()
        torch.cuda.synchronize()
        got = y.float().cpu().numpy().astype(np.float64)
        want = ref.float().cpu().numpy().astype(np.float64)
        assert np.isfinite(got).all()
        assert_close(got, want, dtype, f"noalloc call {call} ({dtype}, N={N})")
