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


def _stage_values(x, K):
    """The intermediate values of the fused kernel's 8192-point pipeline,
    written from the three-digit split (t = 256 j1 + 8 l + j3, f = c1 + 32 c2 +
    1024 c3, unitary factors 1/sqrt(32), 1/sqrt(32), 1/sqrt(8)): forward S1
    (over j1, then the twiddle w8192^(c1 (8 l + j3))), S2 (over l), S3 (over j3
    with w256^(c2 j3)), the filter product, then S3' (over c3), S2' (over c2,
    then the conjugate twiddle) and S1' (over c1).  Returns the stages that
    are stored as fp16 in the kernel and the output."""
    r32, r8 = 1 / np.sqrt(32), 1 / np.sqrt(8)
    a32 = np.arange(32)
    a8 = np.arange(8)
    W32 = _w(32, np.outer(a32, a32))
    tw = _w(8192, a32[:, None, None] * (8 * a32[None, :, None] + a8[None, None, :]))    # [c1, l, j3]
    G = _w(8, np.outer(a8, a8))[None] * _w(256, a32[:, None, None] * a8[None, None, :])  # [c2, c3, j3]
    A1 = r32 * np.einsum("cj,jlk->clk", W32, x.reshape(32, 32, 8)) * tw
    A2 = r32 * np.einsum("dl,clk->cdk", W32, A1)
    X = r8 * np.einsum("dek,cdk->cde", G, A2)
    Y = X * K.reshape(8, 32, 32).transpose(2, 1, 0)
    P = r8 * np.einsum("dek,cde->cdk", np.conj(G), Y)
    Q = r32 * np.einsum("dl,cdk->clk", np.conj(W32), P) * np.conj(tw)
    z = r32 * np.einsum("cj,clk->jlk", np.conj(W32), Q).reshape(-1)
    return {"forward": (A1, A2, X, Y), "P": P, "Q": Q, "z": z}


def test_stage_model_is_the_circular_convolution():
    rng = np.random.default_rng(5)
    u, k = rng.standard_normal(8192), rng.standard_normal(8192)
    K = np.fft.fft(k)
    z = _stage_values(u.astype(complex), K)["z"]
    np.testing.assert_allclose(z, np.fft.ifft(np.fft.fft(u) * K), rtol=0, atol=1e-9 * np.abs(z).max())


@pytest.mark.parametrize("T", [4093, 1021])
def test_matched_chirp_overflows_only_one_inverse_residue(T):
    """The input of the GPU test of an inverse-stage fp16 overflow: a linear
    chirp of T samples and its reversal as the filter (the kernel stores the
    filter spectrum over s_h = max |Re|, |Im|).  Per unit amplitude the
    largest forward value is 2.45 (T = 4093) or 0.67 (T = 1021), the S3' values
    stay near those, and the S2' output reaches 5.93 or 2.97 at one residue
    (l, j3) = (31, 4) while every other (l, j3) stays below 0.12: scaled by
    2e4 (4e4 for T = 1021) only that S2' value passes fp16's 65504."""
    t = np.arange(T)
    chirp = np.cos(np.pi * t.astype(np.float64) ** 2 / (2 * T))
    u = np.zeros(8192)
    u[:T] = chirp
    k = np.zeros(8192)
    k[:T] = chirp[::-1]
    K = np.fft.fft(k)
    K = K / max(np.abs(K.real).max(), np.abs(K.imag).max())
    S = _stage_values(u.astype(complex), K)
    comp = lambda a: np.maximum(np.abs(a.real), np.abs(a.imag))
    fwd = max(comp(a).max() for a in S["forward"])
    q = comp(S["Q"]).max(axis=0)                    # [l, j3]
    amp = 2.0e4 if T == 4093 else 4.0e4
    assert fwd * amp < 0.8 * 65504
    assert comp(S["P"]).max() * amp < 0.5 * 65504
    assert q[31, 4] * amp > 1.5 * 65504
    others = q.copy()
    others[31, 4] = 0
    assert others.max() * amp < 0.1 * 65504
    assert (T - 1) % 256 == 8 * 31 + 4                # the compressed sample's (l, j3)


def test_masked_8192_in_blocks_of_4096():
    """A masked N = 8192 call in blocks of 4096: with k_M = IFFT_16384(K M) and
    G'_d the 8192-point spectrum of k_M's taps at lags 4096 d + m, m in
    (-4096, 4096) (m < 0 stored at 8192 + m), y_0 = IFFT(X_0 G'_0 + X_1 G'_-1)
    and y_1 = IFFT(X_1 G'_0 + X_0 G'_1) (first 4096 outputs each) equal
    IFFT_16384(X K M)[:8192] for any Hermitian mask M."""
    rng = np.random.default_rng(8)
    N, M = 8192, 16384
    x, k = rng.standard_normal(N), rng.standard_normal(N)
    K = np.fft.fft(k, M)
    mask = (rng.random(M // 32) > 0.75).repeat(32).astype(float)
    mask = np.maximum(mask, mask[(-np.arange(M)) % M])
    y = np.fft.ifft(np.fft.fft(x, M) * K * mask)[:N]
    kM = np.fft.ifft(K * mask)
    m = np.arange(4096)
    mn = np.arange(4097, 8192)

    def G(d):
        g = np.zeros(8192, dtype=complex)
        g[m] = kM[(4096 * d + m) % M]
        g[mn] = kM[(4096 * d + mn - 8192) % M]
        return np.fft.fft(g)

    X0 = np.fft.fft(x[:4096], 8192)
    X1 = np.fft.fft(x[4096:], 8192)
    y0 = np.fft.ifft(X0 * G(0) + X1 * G(-1))[:4096]
    y1 = np.fft.ifft(X1 * G(0) + X0 * G(1))[:4096]
    np.testing.assert_allclose(np.r_[y0, y1], y, rtol=0, atol=1e-9 * np.abs(y).max())
