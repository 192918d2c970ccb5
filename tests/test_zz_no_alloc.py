"""fftconv_forward_noalloc: the convolution for callers that may not allocate
device memory (a host framework whose memory pool owns all device memory, or
a latency-critical path that cannot pay for cudaMalloc's synchronisation).

It runs the staged passes with their scratch in the library's static device
arrays instead of a plan workspace.  These tests call it through the C ABI on
two calls in a row with different inputs and compare each result with the
fp64 oracle (an independent check) and with fftconv_forward on an order-4
plan (the existing entry point), so the second call also shows that nothing
the first call left in the shared scratch leaks into its result.  The largest
case, N = 2^20, fills the scratch exactly (one sequence pair per chunk).
This file is collected last on purpose."""
import ctypes

import numpy as np
import pytest

import oracle
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
@pytest.mark.parametrize("dtype,N,B,H,gated,masked", [("bf16", 4096, 3, 2, True, False),
                                                      ("f32", 1024, 3, 2, False, True),
                                                      ("f16", 32768, 3, 2, False, False),
                                                      ("bf16", 1 << 20, 2, 1, True, False)])
def test_noalloc_matches_oracle_and_plan_entry_point_twice(dtype, N, B, H, gated, masked):
    import torch
    lsf, f = _lib()
    plan = lsf.Plan(N, H, dtype, order=4)
    codes = {"f32": lsf.F32, "f16": lsf.F16, "bf16": lsf.BF16}
    rng = np.random.default_rng(N + B)
    k = W.round_to(rng.standard_normal((H, N), dtype=np.float32) / np.float32(np.sqrt(N)), dtype)
    Kf = plan.precompute(to_dev(k, dtype))
    mask = mask_np = None
    if masked:
        mask_np = (rng.random((H, N // 32)) < 0.5).astype(np.uint8)
        mask = torch.from_numpy(mask_np).cuda()
    stream = torch.cuda.current_stream().cuda_stream
    for call in range(2):
        u_np = W.round_to(rng.standard_normal((B, H, N), dtype=np.float32), dtype)
        w_np = W.round_to(rng.standard_normal((B, H, N), dtype=np.float32), dtype) if gated else None
        v_np = W.round_to(rng.standard_normal((B, H, N), dtype=np.float32), dtype) if gated else None
        u, w, v = to_dev(u_np, dtype), to_dev(w_np, dtype), to_dev(v_np, dtype)
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
        exact = oracle.fftconv(u_np, k, w=w_np, v=v_np, mask=mask_np)
        assert_close(got, exact, dtype, f"noalloc call {call} vs oracle ({dtype}, N={N})")
        assert_close(got, want, dtype, f"noalloc call {call} vs fftconv_forward ({dtype}, N={N})")


@pytest.mark.gpu
def test_noalloc_rejects_y_overlapping_the_filter():
    import torch
    lsf, f = _lib()
    N, H, B = 1024, 1, 2
    plan = lsf.Plan(N, H, "f32", order=4)
    Kf = plan.precompute(torch.zeros((H, N), dtype=torch.float32, device="cuda"))
    u = torch.zeros((B, H, N), dtype=torch.float32, device="cuda")
    rc = f(u.data_ptr(), Kf.data_ptr(), Kf.data_ptr(), B, H, N, lsf.F32, None, None, None, 0,
           torch.cuda.current_stream().cuda_stream)
    assert rc == lsf.ERR_INVALID_ARG
    assert b"overlaps" in lsf.library().fftconv_last_error()
