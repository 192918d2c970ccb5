"""Shared helpers for the GPU parity tests: run the CUDA path through the
Python binding of the C ABI and compare with the fp64 oracle."""
import json
import os

import numpy as np

# Tolerances for the CUDA path against the fp64 oracle on identical
# (dtype-rounded) inputs: fp32 plans must reach relative L2 <= 1e-5; fp16/bf16
# plans relative L2 <= 5e-3 and max |error| <= 2e-2 * rms(y).  The max-abs
# bound is applied to the error beyond the unavoidable rounding of y to the
# output dtype: storing y in bf16 alone can be off by half an ulp (1/64 at
# |y| in [4, 8)), more than 2e-2 * rms(y) whenever |y| exceeds ~4.6 rms, so
# each element is allowed 2e-2 * rms(y) + ulp_dtype(y_ref) / 2.
TOL = {"f32": dict(rel_l2=1e-5, max_abs_rms=None, mant_bits=23),
       "f16": dict(rel_l2=5e-3, max_abs_rms=2e-2, mant_bits=10),
       "bf16": dict(rel_l2=5e-3, max_abs_rms=2e-2, mant_bits=7)}


def half_ulp(x, mant_bits):
    """Half a unit in the last place of |x| in a format with `mant_bits`
    stored mantissa bits (normal range)."""
    ax = np.maximum(np.abs(np.asarray(x, np.float64)), 1e-30)
    return 0.5 * np.exp2(np.floor(np.log2(ax)) - mant_bits)


def rel_l2(got, ref):
    got = np.asarray(got, np.float64)
    ref = np.asarray(ref, np.float64)
    den = np.sqrt(np.sum(ref ** 2))
    return float(np.sqrt(np.sum((got - ref) ** 2)) / (den if den > 0 else 1.0))


def assert_close(got, ref, dtype, what=""):
    got = np.asarray(got, np.float64)
    ref = np.asarray(ref, np.float64)
    tol = TOL[dtype]
    e = rel_l2(got, ref)
    assert e <= tol["rel_l2"], f"{what}: relative L2 {e:.3e} > {tol['rel_l2']:.0e}"
    if tol["max_abs_rms"] is not None and ref.size:
        rms = float(np.sqrt(np.mean(ref ** 2)))
        excess = np.abs(got - ref) - half_ulp(ref, tol["mant_bits"])
        m = float(np.max(excess))
        assert m <= tol["max_abs_rms"] * rms, \
            f"{what}: max abs error beyond output rounding {m:.3e} > {tol['max_abs_rms']}*rms ({rms:.3e})"
    log = os.environ.get("PARITY_LOG")
    if log:
        with open(log, "a") as f:
            f.write(json.dumps({"case": what, "dtype": dtype, "rel_l2": e}) + "\n")
    return e


def to_dev(a, dtype):
    import torch
    import workloads as W
    if a is None:
        return None
    return torch.from_numpy(np.ascontiguousarray(a)).to(W.torch_dtype(dtype)).cuda()


def run_cuda(inputs, dtype, order=0, L=None, mask_dev=True):
    """Plan + precompute + forward through the binding; returns (y as float64
    numpy, plan)."""
    import torch
    import long_sequence_fft_b200 as lsf
    u = to_dev(inputs["u"], dtype)
    k = to_dev(inputs["k"], dtype)
    w = to_dev(inputs.get("w"), dtype)
    v = to_dev(inputs.get("v"), dtype)
    m = inputs.get("mask")
    mask = torch.from_numpy(np.ascontiguousarray(m)).cuda() if m is not None else None
    B, H, N = inputs["u"].shape
    plan = lsf.Plan(N, H, dtype, order=order, L=k.shape[1])
    Kf = plan.precompute(k)
    y = plan.forward(u, Kf, w=w, v=v, mask=mask)
    torch.cuda.synchronize()
    assert plan.device_status() == 0
    return y.float().cpu().numpy().astype(np.float64), plan
