"""The overlap-save identities the windowed paths rely on, checked on the CPU
against the oracle (FlashFFTConv: Efficient Convolutions for Long Sequences
with Tensor Cores, "Approach": partial convolutions; the result is defined as
the convolution with the filter zero-padded to N).

Both windowed paths cut a sequence into windows of 2 x hop inputs starting
at (w - 1) x hop (zeros before position 0), take one circular convolution of
window length per window, and keep its second half as outputs
[w x hop, (w + 1) x hop).  That is exact when the filter has at most hop + 1
taps (the tensor-core kernel's windows: hop 2048, filters up to 2049 taps)
and in particular when it has at most hop taps (the staged windows: hop the
power of two >= max(L, 16384)).  Here the windows are assembled with numpy's
FFT, which shares nothing with either side, and compared with the oracle."""
import numpy as np
import pytest

import oracle


def _windows(u, k, hop):
    """y[b, h] from circular convolutions of the 2*hop-input windows."""
    B, H, N = u.shape
    L = k.shape[1]
    n = 2 * hop
    y = np.zeros((B, H, N))
    K = np.fft.fft(np.pad(k.astype(np.float64), ((0, 0), (0, n - L))), axis=-1)
    up = np.concatenate([np.zeros((B, H, hop)), u.astype(np.float64)], axis=-1)
    for w in range(N // hop):
        x = up[:, :, w * hop:w * hop + n]          # inputs [(w-1) hop, (w+1) hop)
        z = np.fft.ifft(np.fft.fft(x, axis=-1) * K[None], axis=-1).real
        y[:, :, w * hop:(w + 1) * hop] = z[:, :, hop:]
    return y


@pytest.mark.parametrize("N,L,hop", [
    (1 << 13, 2049, 2048),      # the tensor-core kernel's windows, longest filter
    (1 << 13, 1, 2048),
    (1 << 14, 4096, 4096),      # staged windows, L equal to the hop
    (1 << 14, 3000, 4096),
])
def test_overlap_save_windows_equal_the_convolution(N, L, hop):
    rng = np.random.default_rng(N + L)
    u = rng.standard_normal((2, 2, N))
    k = rng.standard_normal((2, L)) / np.sqrt(L)
    ref = oracle.fftconv(u, k)
    got = _windows(u, k, hop)
    assert np.max(np.abs(got - ref)) <= 1e-10 * max(1.0, np.max(np.abs(ref)))


def test_one_tap_too_many_breaks_the_windows():
    """With hop + 2 taps the first kept position of each window wraps around:
    the bound on the filter length is tight."""
    N, hop = 1 << 12, 1024
    L = hop + 2
    rng = np.random.default_rng(7)
    u = rng.standard_normal((1, 1, N))
    k = rng.standard_normal((1, L))
    err = np.max(np.abs(_windows(u, k, hop) - oracle.fftconv(u, k)))
    assert err > 1e-3


# ------------------------------------------- two-block partitioned form ---
# Sequences of 8192 on the tensor-core kernel run as two blocks of 4096:
# with X_b the 8192-point transform of block b (zero-padded), G_0 that of
# [k0; 0] and G_1 that of [k1; k0] (k0, k1 the taps [0, 4096), [4096, 8192)),
# block 0's outputs are the first 4096 of IFFT(X_0 G_0) and block 1's those
# of IFFT(X_1 G_0 + X_0 G_1).  The filter rows come from one transform of
# k0 + i k1: G_0 = (Z[f] + conj Z[-f]) / 2, G_1 = (Z[f] - conj Z[-f]) / 2i
# + (-1)^f G_0, and for L <= 4096, G_1 = (-1)^f G_0.

def _two_block(u, k):
    B, H, N = u.shape
    assert N == 8192
    kk = np.zeros((H, 8192))
    kk[:, :k.shape[1]] = k
    Z = np.fft.fft(np.pad(kk[:, :4096] + 1j * kk[:, 4096:], ((0, 0), (0, 4096))), axis=-1)
    Zm = np.conj(Z[:, (-np.arange(8192)) % 8192])
    G0 = (Z + Zm) / 2
    sg = np.where(np.arange(8192) % 2 == 1, -1.0, 1.0)
    G1 = (Z - Zm) / 2j + sg * G0
    pad = lambda x: np.pad(x.astype(np.float64), ((0, 0), (0, 0), (0, 4096)))
    X0 = np.fft.fft(pad(u[:, :, :4096]), axis=-1)
    X1 = np.fft.fft(pad(u[:, :, 4096:]), axis=-1)
    y0 = np.fft.ifft(X0 * G0[None], axis=-1).real[:, :, :4096]
    y1 = np.fft.ifft(X1 * G0[None] + X0 * G1[None], axis=-1).real[:, :, :4096]
    return np.concatenate([y0, y1], axis=-1), G0, G1


@pytest.mark.parametrize("L", [1, 2048, 4096, 4097, 6000, 8192])
def test_two_block_form_equals_the_convolution(L):
    rng = np.random.default_rng(L)
    u = rng.standard_normal((2, 2, 8192))
    k = rng.standard_normal((2, L)) / np.sqrt(L)
    y, G0, G1 = _two_block(u, k)
    ref = oracle.fftconv(u, k)
    assert np.max(np.abs(y - ref)) <= 1e-9 * max(1.0, np.max(np.abs(ref)))
    if L <= 4096:
        assert np.allclose(G1, np.where(np.arange(8192) % 2 == 1, -1.0, 1.0) * G0, atol=1e-9)
