"""GPU parity of the backward pass (fftconv_backward) against the fp64
oracle's adjoints on the same seeded, dtype-rounded inputs.

du, dw and dv come from the tensor-core kernels (correlation launch with the
product by conj(K_f) and two gated outputs; the forward kernel with dy as the
output gate) and are held to the fp16/bf16 tolerances; dk is computed on fp32
lanes from the exactly representable inputs and summed over the batch in
fp32, and is held to the fp32 tolerance.  Sizes include several tiles per CTA
packed short sequences and the two-block mode of N = 8192."""
import numpy as np
import pytest

import oracle
import workloads as W
from parity_util import assert_close, rel_l2, to_dev

pytestmark = pytest.mark.gpu


def _inputs(B, H, N, L, dtype, gated, seed):
    rng = np.random.default_rng(seed)
    r = lambda shape: W.round_to(rng.standard_normal(shape, dtype=np.float32), dtype)
    u, dy = r((B, H, N)), r((B, H, N))
    k = W.round_to(rng.standard_normal((H, L), dtype=np.float32) / np.float32(np.sqrt(L)), dtype)
    w = r((B, H, N)) if gated else None
    v = r((B, H, N)) if gated else None
    return u, k, dy, w, v


def _run(u, k, dy, w, v, dtype):
    import torch
    import long_sequence_fft_b200 as lsf
    B, H, N = u.shape
    plan = lsf.Plan(N, H, dtype, L=k.shape[1])
    assert plan.path_name == "tc_fused"
    Kf = plan.precompute(to_dev(k, dtype))
    g = plan.backward(to_dev(u, dtype), Kf, to_dev(dy, dtype), w=to_dev(w, dtype), v=to_dev(v, dtype))
    torch.cuda.synchronize()
    assert plan.device_status() == 0
    return {n: (None if t is None else t.float().cpu().numpy().astype(np.float64)) for n, t in g.items()}


@pytest.mark.parametrize("B,H,N,L,gated,dtype", [
    (3, 2, 4096, 4096, True, "bf16"),
    (2, 3, 4096, 1000, False, "f16"),
    (5, 2, 1024, 1024, True, "bf16"),
    (4, 3, 256, 200, True, "f16"),
    (16, 256, 4096, 4096, True, "bf16"),      # 512 tiles: several per CTA
    (3, 2, 8192, 8192, True, "bf16"),         # two blocks: block 0 takes block 1's spectrum
    (2, 3, 8192, 3000, False, "f16"),         # k1 = 0: G_1 = (-1)^f G_0
    (5, 2, 8192, 6000, True, "f16"),
    (16, 112, 8192, 8192, True, "bf16"),      # 448 tiles
])
def test_backward_matches_oracle_adjoints(B, H, N, L, gated, dtype):
    u, k, dy, w, v = _inputs(B, H, N, L, dtype, gated, seed=N + L + B)
    got = _run(u, k, dy, w, v, dtype)
    ref = oracle.conv_backward(u, k, dy, w=w, v=v, route="fft")
    for name in ("du", "dw", "dv"):
        if ref[name] is None:
            assert got[name] is None
            continue
        assert_close(got[name], ref[name], dtype, f"{name} B={B} H={H} N={N} L={L}")
    e = rel_l2(got["dk"], ref["dk"])
    assert e <= 1e-5, f"dk relative L2 {e:.2e}"


def test_backward_finite_difference_of_the_gpu_forward():
    """The GPU gradient of <y, dy> matches a central difference of the GPU
    forward pass itself, along a random direction of u (fp16 inputs, so the
    difference is taken in fp32 on exactly representable perturbations)."""
    import torch
    import long_sequence_fft_b200 as lsf
    B, H, N = 2, 2, 1024
    u, k, dy, w, v = _inputs(B, H, N, N, "f16", True, seed=77)
    plan = lsf.Plan(N, H, "f16")
    Kf = plan.precompute(to_dev(k, "f16"))
    g = plan.backward(to_dev(u, "f16"), Kf, to_dev(dy, "f16"), w=to_dev(w, "f16"), v=to_dev(v, "f16"))
    du = g["du"].float().cpu().numpy().astype(np.float64)
    rng = np.random.default_rng(5)
    d = W.round_to(rng.choice([-1.0, 1.0], size=u.shape).astype(np.float32) * np.float32(0.125), "f16")

    def loss(uu):
        y = plan.forward(to_dev(uu, "f16"), Kf, w=to_dev(w, "f16"), v=to_dev(v, "f16"))
        torch.cuda.synchronize()
        return float(np.sum(y.float().cpu().numpy().astype(np.float64) * dy))

    fd = (loss(u + d) - loss(u - d)) / 2.0
    an = float(np.sum(du * d))
    assert abs(fd - an) <= 1e-2 * max(1.0, abs(an)), (fd, an)


def test_backward_arguments():
    import torch
    import long_sequence_fft_b200 as lsf
    N, H = 1024, 2
    plan1 = lsf.Plan(N, H, "f32", order=1)
    Kf1 = plan1.precompute(torch.zeros((H, N), device="cuda"))
    z = torch.zeros((2, H, N), device="cuda")
    with pytest.raises(lsf.FFTConvError) as ei:
        plan1.backward(z, Kf1, z.clone())
    assert ei.value.status == lsf.ERR_UNSUPPORTED
    plan = lsf.Plan(N, H, "bf16")
    Kf = plan.precompute(torch.zeros((H, N), dtype=torch.bfloat16, device="cuda"))
    zb = torch.zeros((2, H, N), dtype=torch.bfloat16, device="cuda")
    du = torch.empty_like(zb)
    rc = lsf.library().fftconv_backward(plan.handle, zb.data_ptr(), Kf.data_ptr(), zb.data_ptr(), 2, H, N, None,
                                        None, du.data_ptr(), du.data_ptr() + 2, None, None, None)
    assert rc == lsf.ERR_INVALID_ARG                     # dw without w
    # an empty batch still clears dk
    dk = torch.full((H, N), 7.0, device="cuda")
    e = zb[:0]
    rc = lsf.library().fftconv_backward(plan.handle, e.data_ptr(), Kf.data_ptr(), e.data_ptr(), 0, H, N, None,
                                        None, e.data_ptr(), None, None, dk.data_ptr(), None)
    torch.cuda.synchronize()
    assert rc == 0 and float(dk.abs().max()) == 0.0


@pytest.mark.parametrize("B,H,N,L", [(1, 1, 8192, 8192), (1, 2, 4096, 100)])
def test_backward_single_row(B, H, N, L):
    u, k, dy, w, v = _inputs(B, H, N, L, "bf16", True, seed=B + H + N + L)
    got = _run(u, k, dy, w, v, "bf16")
    ref = oracle.conv_backward(u, k, dy, w=w, v=v, route="fft")
    for name in ("du", "dw", "dv"):
        assert_close(got[name], ref[name], "bf16", f"{name} single row N={N}")
    assert rel_l2(got["dk"], ref["dk"]) <= 1e-5


def test_backward_into_preallocated_gradients():
    """Plan.backward(out=...) writes into an earlier call's tensors: du, dw, dv
    bit for bit as the allocating call (dk up to the order of its atomic fp32
    sums over CTAs); a missing or extra gradient tensor is rejected."""
    import torch
    import long_sequence_fft_b200 as lsf
    B, H, N, L, dtype = 4, 3, 4096, 4096, "bf16"
    u, k, dy, w, v = _inputs(B, H, N, L, dtype, True, seed=21)
    plan = lsf.Plan(N, H, dtype, L=L)
    Kf = plan.precompute(to_dev(k, dtype))
    ud, dyd, wd, vd = (to_dev(a, dtype) for a in (u, dy, w, v))
    first = plan.backward(ud, Kf, dyd, w=wd, v=vd)
    out = {n: torch.full_like(t, float("nan")) for n, t in first.items()}
    second = plan.backward(ud, Kf, dyd, w=wd, v=vd, out=out)
    torch.cuda.synchronize()
    assert plan.device_status() == 0
    for n in ("du", "dw", "dv", "dk"):
        assert second[n] is out[n]
    for n in ("du", "dw", "dv"):
        assert torch.equal(first[n], out[n]), n
    assert rel_l2(out["dk"].cpu().numpy().astype(np.float64), first["dk"].cpu().numpy().astype(np.float64)) <= 1e-6
    with pytest.raises(ValueError):
        plan.backward(ud, Kf, dyd, w=wd, v=vd, out=dict(out, dw=None))
    with pytest.raises(ValueError):
        plan.backward(ud, Kf, dyd, v=vd, out=out)                       # dw given without w


def test_autograd_through_fftconv():
    """lsf.fftconv under autograd: backward of y with incoming gradient dy
    gives the oracle's adjoints for u, w, v and k (dk in k's dtype, so held to
    the 16-bit tolerance); the forward value equals the call without grad; a
    block mask with grad is refused."""
    import torch
    import long_sequence_fft_b200 as lsf
    B, H, N, L, dtype = 3, 2, 4096, 4096, "bf16"
    u, k, dy, w, v = _inputs(B, H, N, L, dtype, True, seed=31)
    dev = lambda a: torch.from_numpy(a).to(torch.bfloat16).cuda().requires_grad_()
    ut, kt, wt, vt = dev(u), dev(k), dev(w), dev(v)
    y = lsf.fftconv(ut, kt, w=wt, v=vt)
    y.backward(torch.from_numpy(dy).to(torch.bfloat16).cuda())
    ref = oracle.conv_backward(u, k, dy, w=w, v=v, route="fft")
    host = lambda t: t.float().cpu().numpy().astype(np.float64)
    for name, t in (("du", ut), ("dw", wt), ("dv", vt), ("dk", kt)):
        assert t.grad is not None and t.grad.dtype == torch.bfloat16, name
        assert_close(host(t.grad), ref[name], dtype, f"autograd {name}")
    with torch.no_grad():
        y2 = lsf.fftconv(ut, kt, w=wt, v=vt)
    assert torch.equal(y.detach(), y2)
    mask = torch.ones((1, N // 32), dtype=torch.uint8, device="cuda")
    with pytest.raises(NotImplementedError):
        lsf.fftconv(ut, kt, w=wt, v=vt, mask=mask)
