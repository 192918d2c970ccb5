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
