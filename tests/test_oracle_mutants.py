"""Plant plausible mistakes in a copy of the oracle (on the CPU) and check that
the pins of test_oracle_pins.py catch each one.  The copy is compiled into a
temporary directory; the real oracle is untouched."""
import os

import numpy as np
import pytest

import oracle
import test_oracle_pins as pins

MUTANTS = {
    # wrong twiddle sign inside the butterfly
    "twiddle_sign": ("cplx t = { w.re * o.re - w.im * o.im, w.re * o.im + w.im * o.re };",
                     "cplx t = { w.re * o.re + w.im * o.im, w.re * o.im + w.im * o.re };"),
    # wrong twiddle index in the butterfly
    "twiddle_index": ("cplx w = tw[k * twstride];", "cplx w = tw[(k + 1) % h * twstride];"),
    # dropped mirror zeroing of masked bins
    "mask_no_mirror": ("K[(M - g) % M].re = K[(M - g) % M].im = 0.0;", "(void)0;"),
    # Nyquist bin assigned to no block (off by one in the clamp)
    "mask_nyquist": ("if (blk >= nblk) blk = nblk - 1;", "if (blk >= nblk) return 1;"),
    # gate w dropped
    "drop_w_gate": ("x[t].re = (t < N) ? us[t] * (ws ? ws[t] : 1.0) : 0.0;",
                    "x[t].re = (t < N) ? us[t] : 0.0;"),
    # v and w applied to the wrong side (v before the conv)
    "gate_swap": ("J->y[s * N + t] = vs ? vs[t] * z : z;", "J->y[s * N + t] = ws ? ws[t] * z : z;"),
    # missing 1/M normalisation
    "no_normalise": ("double z = X[t].re / (double)M;", "double z = X[t].re;"),
    # filter not truncated to its length (reads past L)
    "filter_len": ("kap[t].re = (t < L) ? J->k[h * L + t] : 0.0;",
                   "kap[t].re = (t < L - 1) ? J->k[h * L + t] : 0.0;"),
    # direct sum off by one tap
    "direct_taps": ("int64_t smax = t < L - 1 ? t : L - 1;",
                    "int64_t smax = t < L - 1 ? t : L - 2;"),
}

PIN_TESTS = [
    lambda: pins.test_fft_matches_textbook_dft(64),
    lambda: pins.test_fft_closed_forms(32),
    pins.test_hand_computed_fixtures,
    lambda: pins.test_fft_route_equals_direct_sum(2, 3, 16, 16, True),
    lambda: pins.test_fft_route_equals_direct_sum(2, 2, 512, 100, True),
    pins.test_delta_filters_and_shift,
    pins.test_closed_forms,
    pins.test_mask_dirichlet_closed_form,
    pins.test_masked_fft_route_equals_circular_sum,
]


def _fails_some_pin():
    for t in PIN_TESTS:
        try:
            t()
        except (AssertionError, ValueError):
            return True
    return False


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_pins_catch_planted_mistake(name, tmp_path):
    old, new = MUTANTS[name]
    src = oracle.source_text()
    assert src.count(old) >= 1, f"mutation anchor for {name} not found"
    mutated = src.replace(old, new, 1)
    lib = oracle.compile_variant(mutated, str(tmp_path / f"liboracle_{name}.so"))
    np.random.seed(0)
    with oracle.using_library(lib):
        assert _fails_some_pin(), f"no pin caught mutant {name}"


def test_unmutated_copy_passes_all_pins(tmp_path):
    lib = oracle.compile_variant(oracle.source_text(), str(tmp_path / "liboracle_copy.so"))
    with oracle.using_library(lib):
        assert not _fails_some_pin()
