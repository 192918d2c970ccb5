"""Pins for the fp64 oracle against facts that do not come from the oracle itself:
the textbook DFT sum, closed forms, Parseval, shift/linearity invariants, a
direct causal sum and hand-computed fixtures.  A planted mistake (see
test_oracle_mutants.py) must fail at least one of them.

What is pinned (FlashFFTConv: Efficient Convolutions for Long Sequences with
Tensor Cores, summary paragraph, "Approach" and "Key results"): the exact
causal convolution y = v * irfft(rfft(u*w, 2N) * rfft(k, 2N))[:N], with the
partial (L < N) and frequency-sparse (block-masked rfft(k)) variants.
"""
import json
import math
import os

import numpy as np
import pytest

import oracle

HERE = os.path.dirname(os.path.abspath(__file__))
RNG = np.random.default_rng(12345)


def crand(M):
    return RNG.standard_normal(M) + 1j * RNG.standard_normal(M)


# ----------------------------------------------------------------- FFT ---

@pytest.mark.parametrize("M", [1, 2, 4, 8, 16, 64, 256, 1024])
def test_fft_matches_textbook_dft(M):
    x = crand(M)
    for inv in (False, True):
        X = oracle.fft(x, inverse=inv)
        D = oracle.dft_direct(x, inverse=inv)
        assert np.max(np.abs(X - D)) <= 1e-9 * max(1.0, np.max(np.abs(D)))


@pytest.mark.parametrize("M", [2, 32, 4096])
def test_fft_closed_forms(M):
    # constant c -> M*c at f=0, zero elsewhere
    c = 0.75 - 0.5j
    X = oracle.fft(np.full(M, c))
    ref = np.zeros(M, complex)
    ref[0] = M * c
    assert np.max(np.abs(X - ref)) <= 1e-10 * M
    # delta at 0 -> all ones
    d = np.zeros(M, complex)
    d[0] = 1
    assert np.max(np.abs(oracle.fft(d) - 1)) <= 1e-12
    # delta at t0 -> exp(-2 pi i f t0 / M)
    t0 = M // 2 + (1 if M > 2 else 0)
    t0 %= M
    d = np.zeros(M, complex)
    d[t0] = 1
    f = np.arange(M)
    ref = np.exp(-2j * np.pi * f * t0 / M)
    assert np.max(np.abs(oracle.fft(d) - ref)) <= 1e-11
    # single tone exp(+2 pi i f0 n / M) -> M at f0
    f0 = 3 % M
    n = np.arange(M)
    X = oracle.fft(np.exp(2j * np.pi * f0 * n / M))
    ref = np.zeros(M, complex)
    ref[f0] = M
    assert np.max(np.abs(X - ref)) <= 1e-9 * M


@pytest.mark.parametrize("M", [16, 2048, 1 << 15])
def test_fft_parseval_roundtrip_and_numpy(M):
    x = crand(M)
    X = oracle.fft(x)
    assert abs(np.sum(np.abs(x) ** 2) - np.sum(np.abs(X) ** 2) / M) <= 1e-10 * np.sum(np.abs(x) ** 2)
    back = oracle.fft(X, inverse=True) / M
    assert np.max(np.abs(back - x)) <= 1e-12 * math.log2(M) * 10
    # a library FFT used as an independent check (not as the oracle)
    ref = np.fft.fft(x)
    assert np.max(np.abs(X - ref)) <= 1e-12 * np.max(np.abs(ref)) * math.log2(M)


def test_fft_rejects_non_power_of_two():
    with pytest.raises(ValueError):
        oracle.fft(np.ones(12))


# ---------------------------------------------------------- convolution ---

def test_hand_computed_fixtures():
    with open(os.path.join(HERE, "golden", "hand_cases.json")) as f:
        cases = json.load(f)["cases"]
    for c in cases:
        u = np.array(c["u"], float)
        k = np.array(c["k"], float)
        w = np.array(c["w"], float) if "w" in c else None
        v = np.array(c["v"], float) if "v" in c else None
        ref = np.array(c["y"], float)
        got = oracle.fftconv(u, k, w=w, v=v)
        assert np.max(np.abs(got - ref)) <= 1e-12, c["name"]
        got_d = oracle.direct_conv(u, k, w=w, v=v)
        assert np.max(np.abs(got_d - ref)) <= 1e-12, c["name"]


@pytest.mark.parametrize("B,H,N,L,gated", [(1, 1, 1, 1, False), (2, 3, 16, 16, True),
                                           (1, 2, 64, 17, True), (3, 1, 256, 256, False),
                                           (2, 2, 512, 100, True)])
def test_fft_route_equals_direct_sum(B, H, N, L, gated):
    u = RNG.standard_normal((B, H, N))
    k = RNG.standard_normal((H, L))
    w = RNG.standard_normal((B, H, N)) if gated else None
    v = RNG.standard_normal((B, H, N)) if gated else None
    y, ratio = oracle.fftconv(u, k, w=w, v=v, return_imag_ratio=True)
    ref = oracle.direct_conv(u, k, w=w, v=v)
    assert np.max(np.abs(y - ref)) <= 1e-11 * max(1.0, np.max(np.abs(ref)))
    assert ratio <= 1e-9
    # sampled direct sums agree with the full direct sum
    seq = RNG.integers(0, B * H, size=20)
    ts = RNG.integers(0, N, size=20)
    ys = oracle.direct_conv(u, k, w=w, v=v, seq=seq, ts=ts)
    flat = ref.reshape(B * H, N)
    assert np.max(np.abs(ys - flat[seq, ts])) <= 1e-12 * max(1.0, np.max(np.abs(flat)))


def test_delta_filters_and_shift():
    N = 128
    u = RNG.standard_normal((2, 1, N))
    w = RNG.standard_normal((2, 1, N))
    v = RNG.standard_normal((2, 1, N))
    k = np.zeros((1, N))
    k[0, 0] = 1.0
    y = oracle.fftconv(u, k, w=w, v=v)
    assert np.max(np.abs(y - u * w * v)) <= 1e-12
    for d in (1, 5, N - 1):
        k = np.zeros((1, N))
        k[0, d] = 1.0
        y = oracle.fftconv(u, k)
        ref = np.zeros_like(u)
        ref[..., d:] = u[..., :N - d]
        assert np.max(np.abs(y - ref)) <= 1e-12


def test_shift_equivariance():
    N, d = 256, 37
    u = RNG.standard_normal((1, 2, N))
    k = RNG.standard_normal((2, N))
    us = np.zeros_like(u)
    us[..., d:] = u[..., :N - d]
    y = oracle.fftconv(u, k)
    ys = oracle.fftconv(us, k)
    assert np.max(np.abs(ys[..., :d])) <= 1e-11
    assert np.max(np.abs(ys[..., d:] - y[..., :N - d])) <= 1e-10


def test_linearity():
    N = 256
    u1, u2 = RNG.standard_normal((2, 1, 2, N))
    k1, k2 = RNG.standard_normal((2, 2, N))
    a, b = 0.7, -1.3
    lhs = oracle.fftconv(a * u1 + b * u2, k1)
    rhs = a * oracle.fftconv(u1, k1) + b * oracle.fftconv(u2, k1)
    assert np.max(np.abs(lhs - rhs)) <= 1e-10
    lhs = oracle.fftconv(u1, a * k1 + b * k2)
    rhs = a * oracle.fftconv(u1, k1) + b * oracle.fftconv(u1, k2)
    assert np.max(np.abs(lhs - rhs)) <= 1e-10


def test_closed_forms():
    N = 1024
    t = np.arange(N)
    # u = k = 1  ->  y[t] = t + 1
    y = oracle.fftconv(np.ones((1, 1, N)), np.ones((1, N)))
    assert np.max(np.abs(y[0, 0] - (t + 1))) <= 1e-9
    # u = 1, k[s] = r^s  ->  y[t] = (1 - r^(t+1)) / (1 - r)
    r = 0.99
    y = oracle.fftconv(np.ones((1, 1, N)), r ** t[None, :].astype(float))
    assert np.max(np.abs(y[0, 0] - (1 - r ** (t + 1)) / (1 - r))) <= 1e-10
    # u = delta_0  ->  y = k
    u = np.zeros((1, 1, N))
    u[0, 0, 0] = 1
    k = RNG.standard_normal((1, N))
    assert np.max(np.abs(oracle.fftconv(u, k)[0, 0] - k[0])) <= 1e-12
    # partial filter of length L: u = 1  ->  y[t] = sum_{s<=min(t,L-1)} k[s]
    L = 100
    kp = RNG.standard_normal((1, L))
    y = oracle.fftconv(np.ones((1, 1, N)), kp)
    cs = np.cumsum(kp[0])
    ref = np.where(t < L, cs[np.minimum(t, L - 1)], cs[-1])
    assert np.max(np.abs(y[0, 0] - ref)) <= 1e-10


def test_partial_filter_equals_zero_padded_full_filter():
    N, L = 512, 64
    u = RNG.standard_normal((2, 3, N))
    k = RNG.standard_normal((3, L))
    kpad = np.zeros((3, N))
    kpad[:, :L] = k
    assert np.max(np.abs(oracle.fftconv(u, k) - oracle.fftconv(u, kpad))) <= 1e-11


# ------------------------------------------------------- frequency mask ---

def test_filter_rfft_against_library_and_textbook():
    N, L = 64, 40
    k = RNG.standard_normal((2, L))
    K = oracle.filter_rfft(k, N)
    kp = np.zeros((2, 2 * N))
    kp[:, :L] = k
    assert np.max(np.abs(K - np.fft.rfft(kp, axis=1))) <= 1e-11
    D = oracle.dft_direct(kp[1])
    assert np.max(np.abs(K[1] - D[:N + 1])) <= 1e-10


def test_mask_dirichlet_closed_form():
    # k = delta_0 so K = 1 everywhere; keep block 0 (bins 0..31) of N=64 and drop
    # block 1 (bins 32..64, Nyquist included).  With the mirrors dropped too the
    # effective filter is the Dirichlet kernel sin(63 pi t/128) / (128 sin(pi t/128)),
    # and u = delta_0 returns it on t < N.
    N = 64
    M = 2 * N
    k = np.zeros((1, N))
    k[0, 0] = 1
    u = np.zeros((1, 1, N))
    u[0, 0, 0] = 1
    mask = np.array([[1, 0]], np.uint8)
    y = oracle.fftconv(u, k, mask=mask)[0, 0]
    t = np.arange(1, N)
    ref = np.empty(N)
    ref[0] = 63 / M
    ref[1:] = np.sin(63 * np.pi * t / M) / (M * np.sin(np.pi * t / M))
    assert np.max(np.abs(y - ref)) <= 1e-12
    # the direct-IDFT and FFT routes to the effective filter agree with it too
    ke_d = oracle.masked_filter(k, N, mask, direct=True)[0]
    ke_f = oracle.masked_filter(k, N, mask, direct=False)[0]
    assert np.max(np.abs(ke_d[:N] - ref)) <= 1e-12
    assert np.max(np.abs(ke_f - ke_d)) <= 1e-12
    # only block 1 kept: the complement, i.e. delta minus the Dirichlet kernel
    y2 = oracle.fftconv(u, k, mask=np.array([[0, 1]], np.uint8))[0, 0]
    delta = np.zeros(N)
    delta[0] = 1
    assert np.max(np.abs(y2 - (delta - ref))) <= 1e-12


def test_masked_fft_route_equals_circular_sum():
    B, H, N = 2, 3, 128
    u = RNG.standard_normal((B, H, N))
    w = RNG.standard_normal((B, H, N))
    v = RNG.standard_normal((B, H, N))
    k = RNG.standard_normal((H, N))
    mask = (RNG.random((H, N // 32)) < 0.5).astype(np.uint8)
    y = oracle.fftconv(u, k, w=w, v=v, mask=mask)
    keff = oracle.masked_filter(k, N, mask, direct=True)
    seq = np.repeat(np.arange(B * H), N)
    ts = np.tile(np.arange(N), B * H)
    ref = oracle.circular_conv_samples(u, keff, seq, ts, w=w, v=v).reshape(B, H, N)
    assert np.max(np.abs(y - ref)) <= 1e-10
    # an all-ones mask is the dense convolution, bit for bit
    dense = oracle.fftconv(u, k, w=w, v=v)
    ones = oracle.fftconv(u, k, w=w, v=v, mask=np.ones((1, N // 32), np.uint8))
    assert np.array_equal(dense, ones)
    # one shared mask row == that row repeated per channel
    shared = oracle.fftconv(u, k, mask=mask[:1])
    per = oracle.fftconv(u, k, mask=np.repeat(mask[:1], H, axis=0))
    assert np.array_equal(shared, per)


def test_masked_filter_is_real_and_zero_mask_kills_output():
    N = 64
    k = RNG.standard_normal((1, N))
    u = RNG.standard_normal((1, 1, N))
    y = oracle.fftconv(u, k, mask=np.zeros((1, 2), np.uint8))
    assert np.max(np.abs(y)) <= 1e-14
    _, ratio = oracle.fftconv(u, k, mask=np.array([[0, 1]], np.uint8), return_imag_ratio=True)
    assert ratio <= 1e-9


def test_threads_do_not_change_results():
    u = RNG.standard_normal((3, 5, 256))
    k = RNG.standard_normal((5, 256))
    a = oracle.fftconv(u, k, nthreads=1)
    b = oracle.fftconv(u, k, nthreads=4)
    assert np.array_equal(a, b)


def test_empty_batch():
    y = oracle.fftconv(np.zeros((0, 2, 64)), np.ones((2, 64)))
    assert y.shape == (0, 2, 64)
