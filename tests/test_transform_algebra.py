"""The index algebra the kernels are built on, checked on the CPU (FlashFFTConv:
Efficient Convolutions for Long Sequences with Tensor Cores, "Approach": the
order-p Monarch decomposition of the FFT, read as mixed-radix Cooley-Tukey).

Each identity is checked against numpy's FFT or the oracle, which share
nothing with the CUDA code: the staged column/row split M = R x C, the
three-digit split of the 8192-point transform, the parity split of the
16384-point spectrum, and the two-for-one packing of two real rows."""
import numpy as np
import pytest

import oracle


def _w(n, e):
    return np.exp(-2j * np.pi * np.asarray(e, dtype=np.float64) / n)


@pytest.mark.parametrize("R,C", [(4, 8), (8, 16), (16, 4), (2, 32)])
def test_staged_split_is_the_dft(R, C):
    """Column pass: A[c, r] = sum_j x[j C + r] w_R^(j c) * w_M^(c r); row pass:
    X[c + R e] = sum_r A[c, r] w_C^(r e)."""
    M = R * C
    rng = np.random.default_rng(M + R)
    x = rng.standard_normal(M) + 1j * rng.standard_normal(M)
    X0 = x.reshape(R, C)                                   # [j, r]
    j = np.arange(R)
    c = np.arange(R)
    r = np.arange(C)
    A = (_w(R, np.outer(c, j)) @ X0) * _w(M, np.outer(c, r))   # [c, r]
    e = np.arange(C)
    Y = A @ _w(C, np.outer(r, e))                          # [c, e] = X[c + R e]
    X = np.empty(M, dtype=complex)
    X[(c[:, None] + R * e[None, :]).ravel()] = Y.ravel()
    np.testing.assert_allclose(X, np.fft.fft(x), rtol=0, atol=1e-9 * np.abs(X).max())


def test_three_digit_split_of_8192_exponents():
    """t = 256 j1 + 8 l + j3, f = c1 + 32 c2 + 1024 c3: f t = 256 c1 j1 + 8 c1 l
    + c1 j3 + 256 c2 l + 32 c2 j3 + 1024 c3 j3 (mod 8192), i.e. w8192^(f t) is
    w32^(c1 j1) w1024^(c1 l) w8192^(c1 j3) w32^(c2 l) w256^(c2 j3) w8^(c3 j3),
    for every (f, t)."""
    t = np.arange(8192, dtype=np.int64)
    j1, l, j3 = t // 256, (t // 8) % 32, t % 8
    for f0 in range(0, 8192, 512):
        f = np.arange(f0, f0 + 512, dtype=np.int64)[:, None]
        c1, c2, c3 = f % 32, (f // 32) % 32, f // 1024
        lhs = (f * t[None, :]) % 8192
        rhs = (256 * c1 * j1 + 8 * c1 * l + c1 * j3 + 256 * c2 * l + 32 * c2 * j3 + 1024 * c3 * j3) % 8192
        assert np.array_equal(lhs, rhs)


@pytest.mark.parametrize("n", [16, 64])
def test_parity_split_of_the_doubled_spectrum(n):
    """Sequences of n with a full-length filter: with M = 2n, X(2f) is the
    n-point transform of x and X(2f+1) that of x[t] w_M^t; the output is
    y[t] = (z_even[t] + w_M^(-t) z_odd[t]) / 2."""
    rng = np.random.default_rng(n)
    u = rng.standard_normal((1, 1, n))
    k = rng.standard_normal((1, n))
    t = np.arange(n)
    Km = np.fft.fft(np.pad(k[0], (0, n)))                  # 2n-point spectrum of k
    x = u[0, 0]
    ze = np.fft.ifft(np.fft.fft(x) * Km[0::2])
    zo = np.fft.ifft(np.fft.fft(x * _w(2 * n, t)) * Km[1::2])
    y = ((ze + np.conj(_w(2 * n, t)) * zo) / 2).real
    np.testing.assert_allclose(y, oracle.fftconv(u, k)[0, 0], rtol=0, atol=1e-10)


def test_two_for_one_packing():
    """Two real rows of one channel as one complex sequence: the real filter
    keeps them apart, so one complex convolution returns both exactly."""
    rng = np.random.default_rng(3)
    n = 128
    u = rng.standard_normal((2, 1, n))
    k = rng.standard_normal((1, n))
    z = np.fft.ifft(np.fft.fft(u[0, 0] + 1j * u[1, 0], 2 * n) * np.fft.fft(k[0], 2 * n))[:n]
    ref = oracle.fftconv(u, k)
    np.testing.assert_allclose(z.real, ref[0, 0], rtol=0, atol=1e-10)
    np.testing.assert_allclose(z.imag, ref[1, 0], rtol=0, atol=1e-10)
