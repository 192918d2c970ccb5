"""Pins of the oracle's per-bin masked route (oracle.fftconv_bins): a mask
over the individual bins of the 2N-point filter spectrum, the form a
Monarch-aligned sparsity pattern takes ("FlashFFTConv: Efficient Convolutions
for Long Sequences with Tensor Cores", "Approach": frequency-sparse
convolutions skip blocks of the Monarch matrix products; "Key results": 79%
frequency sparsity).  Pinned against the block-mask route (itself pinned by
the Dirichlet closed form), closed forms for masks that keep one or three
bins (direct sums, no FFT), the real-output self-check, and planted
mistakes."""
import numpy as np
import pytest

import oracle


def _case(B, H, N, L, seed):
    rng = np.random.default_rng(seed)
    return rng.standard_normal((B, H, N)), rng.standard_normal((H, L)) / np.sqrt(L)


def test_all_ones_equals_unmasked():
    u, k = _case(2, 3, 256, 200, 1)
    assert np.array_equal(oracle.fftconv_bins(u, k, np.ones((1, 512), np.uint8)), oracle.fftconv(u, k))


def test_block_mask_expanded_per_bin_equals_block_route():
    """Reading of the block mask: rfft bin g of [0, N] in block g // 32 (the
    Nyquist bin in the last block), a zero block zeroes the bin and its mirror."""
    B, H, N = 2, 3, 512
    u, k = _case(B, H, N, N, 2)
    rng = np.random.default_rng(3)
    blocks = (rng.random((H, N // 32)) < 0.5).astype(np.uint8)
    M = 2 * N
    bins = np.ones((H, M), np.uint8)
    for h in range(H):
        for g in range(N + 1):
            if not blocks[h, min(g // 32, N // 32 - 1)]:
                bins[h, g] = 0
                bins[h, (M - g) % M] = 0
    assert np.allclose(oracle.fftconv_bins(u, k, bins), oracle.fftconv(u, k, mask=blocks), atol=1e-12)


def test_dc_only_is_the_product_of_sums():
    """Only bin 0 kept: y[t] = (sum_s x[s]) (sum_s k[s]) / 2N for every t."""
    B, H, N, L = 2, 2, 128, 50
    u, k = _case(B, H, N, L, 4)
    w = np.random.default_rng(5).standard_normal((B, H, N))
    m = np.zeros((1, 2 * N), np.uint8)
    m[0, 0] = 1
    y = oracle.fftconv_bins(u, k, m, w=w)
    ref = ((u * w).sum(-1) * k.sum(-1)[None, :])[:, :, None] / (2 * N)
    assert np.allclose(y, np.broadcast_to(ref, y.shape), atol=1e-12)


def test_three_bins_closed_form():
    """Bins 0, 1 and 2N - 1 kept: y[t] = (X0 K0 + 2 Re(X1 K1 e^{2 pi i t / 2N})) / 2N
    with X1, K1 the direct sums at frequency 1."""
    B, H, N, L = 1, 2, 64, 64
    u, k = _case(B, H, N, L, 6)
    M = 2 * N
    m = np.zeros((1, M), np.uint8)
    m[0, [0, 1, M - 1]] = 1
    y = oracle.fftconv_bins(u, k, m)
    e = np.exp(-2j * np.pi * np.arange(N) / M)
    X0, X1 = u.sum(-1), (u * e).sum(-1)
    K0, K1 = k.sum(-1), (k * e[:L]).sum(-1)
    t = np.arange(N)
    ref = (X0[..., None] * K0[None, :, None]
           + 2 * np.real((X1 * K1[None])[..., None] * np.exp(2j * np.pi * t / M))) / M
    assert np.allclose(y, ref, atol=1e-12)


def test_non_hermitian_mask_is_reported():
    u, k = _case(1, 1, 128, 128, 7)
    m = np.ones((1, 256), np.uint8)
    m[0, 5] = 0                                      # its mirror 251 stays
    _, ratio = oracle.fftconv_bins(u, k, m, return_imag_ratio=True)
    assert ratio > 1e-6
    m[0, 251] = 0
    _, ratio = oracle.fftconv_bins(u, k, m, return_imag_ratio=True)
    assert ratio < 1e-12


def test_per_channel_rows():
    B, H, N = 2, 3, 128
    u, k = _case(B, H, N, N, 8)
    rng = np.random.default_rng(9)
    rows = np.ones((H, 2 * N), np.uint8)
    for h in range(H):
        for f in rng.choice(np.arange(1, N), 20, replace=False):
            rows[h, f] = rows[h, 2 * N - f] = 0
    y = oracle.fftconv_bins(u, k, rows)
    for h in range(H):
        yh = oracle.fftconv_bins(u[:, h:h + 1], k[h:h + 1], rows[h:h + 1])
        assert np.allclose(y[:, h:h + 1], yh, atol=1e-14)
    assert not np.allclose(y[:, 0], oracle.fftconv_bins(u[:, :1], k[:1], rows[1:2])[:, 0])


MUTANTS = {
    # the mask ignored
    "ignored": ("if (!brow[f]) K[f].re = K[f].im = 0.0;", "(void)brow;"),
    # off by one bin
    "shifted": ("if (!brow[f]) K[f].re = K[f].im = 0.0;", "if (!brow[(f + 1) % M]) K[f].re = K[f].im = 0.0;"),
    # every channel reads row 0
    "row0": ("(J->binmask_h == 1 ? 0 : h) * M", "0 * M"),
}


def _pins():
    yield test_dc_only_is_the_product_of_sums
    yield test_three_bins_closed_form
    yield test_per_channel_rows


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_pins_catch_planted_binmask_mistake(name, tmp_path):
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
