"""Pins of the oracle's backward pass (the gradients of the gated causal
convolution) against things other than itself: finite differences of the
pinned forward oracle, the bilinear identity <z, g> = <x, dx> = <k, dk>, the
direct-sum route, and closed forms.  Planted mistakes in a compiled copy must
fail at least one pin.

The gradients are the plain adjoints of the forward definition ("FlashFFTConv:
Efficient Convolutions for Long Sequences with Tensor Cores", "Key results":
the convolution is used in trained models; the page gives no backward).
"""
import numpy as np
import pytest

import oracle


def _case(B, H, N, L, gated, seed):
    rng = np.random.default_rng(seed)
    u = rng.standard_normal((B, H, N))
    k = rng.standard_normal((H, L)) / np.sqrt(L)
    dy = rng.standard_normal((B, H, N))
    w = rng.standard_normal((B, H, N)) if gated else None
    v = rng.standard_normal((B, H, N)) if gated else None
    return u, k, dy, w, v


def _loss(u, k, dy, w, v):
    return float(np.sum(oracle.fftconv(u, k, w=w, v=v) * dy))


@pytest.mark.parametrize("B,H,N,L,gated", [(2, 2, 64, 64, True), (3, 1, 128, 37, True), (1, 3, 32, 1, False)])
def test_fft_route_equals_direct_sums(B, H, N, L, gated):
    u, k, dy, w, v = _case(B, H, N, L, gated, seed=N + L)
    a = oracle.conv_backward(u, k, dy, w=w, v=v, route="fft")
    b = oracle.conv_backward(u, k, dy, w=w, v=v, route="direct")
    for name in ("du", "dw", "dv", "dk"):
        if a[name] is None:
            assert b[name] is None
            continue
        assert np.allclose(a[name], b[name], rtol=1e-10, atol=1e-10), name


def test_finite_differences_of_the_forward_oracle():
    B, H, N, L = 2, 2, 32, 20
    u, k, dy, w, v = _case(B, H, N, L, True, seed=5)
    g = oracle.conv_backward(u, k, dy, w=w, v=v, route="direct")
    rng = np.random.default_rng(6)
    eps = 1e-6
    for name, arr, grad in (("u", u, g["du"]), ("w", w, g["dw"]), ("v", v, g["dv"]), ("k", k, g["dk"])):
        for _ in range(6):
            idx = tuple(int(rng.integers(0, n)) for n in arr.shape)
            old = arr[idx]
            arr[idx] = old + eps
            lp = _loss(u, k, dy, w, v)
            arr[idx] = old - eps
            lm = _loss(u, k, dy, w, v)
            arr[idx] = old
            fd = (lp - lm) / (2 * eps)
            assert abs(fd - grad[idx]) <= 1e-6 * max(1.0, abs(fd)), (name, idx, fd, grad[idx])


def test_bilinear_identity():
    """With z = conv(x, k) and any g: <z, g> = <x, corr(g, k)> = <k, dk>
    (dk summed over the batch); here x = u (no gates) and g = dy."""
    B, H, N, L = 3, 2, 256, 100
    u, k, dy, _, _ = _case(B, H, N, L, False, seed=11)
    z = oracle.fftconv(u, k)
    g = oracle.conv_backward(u, k, dy, route="fft")
    lhs = np.sum(z * dy)
    assert abs(lhs - np.sum(u * g["du"])) <= 1e-9 * np.sum(np.abs(z * dy))
    assert abs(lhs - np.sum(k * g["dk"])) <= 1e-9 * np.sum(np.abs(z * dy))


def test_closed_forms():
    B, H, N = 2, 2, 64
    rng = np.random.default_rng(3)
    dy = rng.standard_normal((B, H, N))
    u = rng.standard_normal((B, H, N))
    # shifted delta filter d: dx[t] = dy[t + d] for t + d < N, else 0
    for d in (0, 5, N - 1):
        k = np.zeros((H, N))
        k[:, d] = 1.0
        du = oracle.conv_backward(u, k, dy, route="direct")["du"]
        ref = np.zeros_like(dy)
        ref[:, :, :N - d] = dy[:, :, d:]
        assert np.allclose(du, ref, atol=1e-12), d
    # x = 1, g = 1: dk[s] = sum_b (N - s) = B (N - s)
    ones = np.ones((B, H, N))
    for route in ("direct", "fft"):
        dk = oracle.conv_backward(ones, np.ones((H, N)), ones, route=route)["dk"]
        assert np.allclose(dk, B * (N - np.arange(N))[None, :], atol=1e-9), route


MUTANTS = {
    # convolution instead of correlation in the direct du sum
    "corr_as_conv": ("for (int64_t q = 0; q <= smax; ++q) acc += g[t + q] * kh[q];",
                     "for (int64_t q = 0; q <= smax && q <= t; ++q) acc += g[t - q] * kh[q];"),
    # dk over one tap too few positions
    "dk_range": ("for (int64_t t = q; t < N; ++t) acc += g[t] * x[t - q];",
                 "for (int64_t t = q + 1; t < N; ++t) acc += g[t] * x[t - q];"),
    # FFT route: K not conjugated (convolution)
    "fft_no_conj": ("a[f].im = G[f].im * K[f].re - G[f].re * K[f].im;",
                    "a[f].im = G[f].im * K[f].re + G[f].re * K[f].im;"),
    # dw multiplied by w instead of u
    "dw_wrong_gate": ("if (dw) dw[s * N + t] = acc * u[s * N + t];",
                      "if (dw) dw[s * N + t] = acc * w[s * N + t];"),
    # dv without the incoming gradient
    "dv_no_dy": ("dv[s * N + t] = dy[s * N + t] * z;", "dv[s * N + t] = z;"),
}


def _pins():
    yield lambda: test_fft_route_equals_direct_sums(2, 2, 64, 64, True)
    yield test_finite_differences_of_the_forward_oracle
    yield test_bilinear_identity
    yield test_closed_forms


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_pins_catch_planted_backward_mistake(name, tmp_path):
    old, new = MUTANTS[name]
    src = oracle.source_text()
    assert src.count(old) == 1, f"mutation anchor for {name} not unique"
    lib = oracle.compile_variant(src.replace(old, new), str(tmp_path / f"liboracle_{name}.so"))
    caught = False
    with oracle.using_library(lib):
        for pin in _pins():
            try:
                pin()
            except (AssertionError, ValueError):
                caught = True
                break
    assert caught, f"no pin caught mutant {name}"
