"""fp64 CPU oracle for the exact causal long convolution (test infrastructure).

Only the tests, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline /
reference leg may import this package.  The product path (the CUDA library and
its Python binding) never does, and shares no code with it.

The arithmetic lives in ``fftconv_oracle.c`` (plain C, fp64, own recursive
radix-2 FFT and direct sums); this module only compiles it and marshals numpy
arrays.  What it computes follows "FlashFFTConv: Efficient Convolutions for
Long Sequences with Tensor Cores" (summary paragraph, "Approach", "Key
results"): y = v * irfft(rfft(u*w, 2N) * rfft(k, 2N))[:N], optionally with a
filter shorter than N (partial convolution) or a block mask on the filter's
rfft bins (frequency-sparse convolution).
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "fftconv_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")
_lock = threading.Lock()
_lib = None

BLOCK = 32  # bins per frequency-mask block


def build(force: bool = False) -> str:
    """Compile the oracle with gcc into oracle/liboracle.so (idempotent)."""
    if (not force and os.path.exists(_LIB)
            and os.path.getmtime(_LIB) >= os.path.getmtime(_SRC)):
        return _LIB
    tmp = _LIB + ".tmp%d" % os.getpid()
    cmd = ["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-Wall", "-Wextra",
           "-o", tmp, _SRC, "-lm", "-lpthread"]
    subprocess.check_call(cmd)
    os.replace(tmp, _LIB)
    return _LIB


def _bind(lib):
    dp = ctypes.POINTER(ctypes.c_double)
    i64 = ctypes.c_int64
    u8p = ctypes.POINTER(ctypes.c_uint8)
    i64p = ctypes.POINTER(ctypes.c_int64)
    lib.oracle_fft.argtypes = [dp, dp, i64, ctypes.c_int]
    lib.oracle_dft_direct.argtypes = [dp, dp, dp, dp, i64, ctypes.c_int]
    lib.oracle_fftconv.argtypes = [dp, dp, dp, i64, i64, i64, i64, dp, dp,
                                   u8p, i64, ctypes.c_int, dp]
    lib.oracle_fftconv_bins.argtypes = [dp, dp, dp, i64, i64, i64, i64, dp, dp,
                                        u8p, i64, ctypes.c_int, dp]
    lib.oracle_filter_rfft.argtypes = [dp, dp, i64, i64, i64, u8p, i64]
    lib.oracle_direct_conv.argtypes = [dp, dp, dp, i64, i64, i64, i64, dp, dp,
                                       i64p, i64p, i64]
    lib.oracle_masked_filter_direct.argtypes = [dp, dp, i64, i64, i64, u8p, i64]
    lib.oracle_masked_filter_fft.argtypes = [dp, dp, i64, i64, i64, u8p, i64]
    lib.oracle_circular_conv_samples.argtypes = [dp, dp, dp, i64, i64, i64, dp, dp,
                                                 i64p, i64p, i64]
    lib.oracle_conv_backward_direct.argtypes = [dp, dp, dp, dp, dp, i64, i64, i64, i64, dp, dp, dp, dp]
    lib.oracle_conv_backward_fft.argtypes = [dp, dp, dp, dp, dp, i64, i64, i64, i64, dp, dp, dp, dp]
    for f in ("oracle_fft", "oracle_dft_direct", "oracle_fftconv", "oracle_fftconv_bins",
              "oracle_filter_rfft", "oracle_direct_conv",
              "oracle_masked_filter_direct", "oracle_masked_filter_fft",
              "oracle_circular_conv_samples", "oracle_conv_backward_direct",
              "oracle_conv_backward_fft"):
        getattr(lib, f).restype = ctypes.c_int
    return lib


def _load():
    global _lib
    with _lock:
        if _lib is None:
            build()
            _lib = _bind(ctypes.CDLL(_LIB))
    return _lib


def _f64(a):
    if a is None:
        return None
    return np.ascontiguousarray(np.asarray(a, dtype=np.float64))


def _ptr(a, ctype=ctypes.c_double):
    if a is None:
        return None
    return a.ctypes.data_as(ctypes.POINTER(ctype))


def _mask(mask):
    if mask is None:
        return None, 0
    m = np.ascontiguousarray(np.asarray(mask, dtype=np.uint8))
    if m.ndim == 1:
        m = m[None, :]
    return m, m.shape[0]


def _check(rc, what):
    if rc != 0:
        raise ValueError(f"oracle {what} failed with code {rc}")


def fft(x, inverse=False):
    """Unnormalised length-M DFT (M a power of two) of a complex vector."""
    x = np.asarray(x, dtype=np.complex128)
    re = np.ascontiguousarray(x.real.copy())
    im = np.ascontiguousarray(x.imag.copy())
    _check(_load().oracle_fft(_ptr(re), _ptr(im), x.shape[0], int(bool(inverse))), "fft")
    return re + 1j * im


def dft_direct(x, inverse=False):
    """Textbook O(M^2) DFT (any M), unnormalised."""
    x = np.asarray(x, dtype=np.complex128)
    re = np.ascontiguousarray(x.real.copy())
    im = np.ascontiguousarray(x.imag.copy())
    ore = np.empty_like(re)
    oim = np.empty_like(im)
    _load().oracle_dft_direct(_ptr(re), _ptr(im), _ptr(ore), _ptr(oim), x.shape[0],
                              int(bool(inverse)))
    return ore + 1j * oim


def fftconv(u, k, w=None, v=None, mask=None, nthreads=None, return_imag_ratio=False):
    """FFT route.  u, w, v: [B, H, N]; k: [H, L]; mask: [mask_h, N/32] or None."""
    u = _f64(u)
    k = _f64(k)
    w = _f64(w)
    v = _f64(v)
    B, H, N = u.shape
    L = k.shape[1]
    assert k.shape[0] == H
    m, mh = _mask(mask)
    y = np.empty((B, H, N), dtype=np.float64)
    ratio = ctypes.c_double(0.0)
    if nthreads is None:
        nthreads = os.cpu_count() or 1
    rc = _load().oracle_fftconv(_ptr(u), _ptr(k), _ptr(y), B, H, N, L, _ptr(w), _ptr(v),
                                _ptr(m, ctypes.c_uint8), mh, int(nthreads),
                                ctypes.byref(ratio))
    _check(rc, "fftconv")
    if return_imag_ratio:
        return y, ratio.value
    return y


def fftconv_bins(u, k, binmask, w=None, v=None, nthreads=None, return_imag_ratio=False):
    """FFT route with a per-bin mask of the full 2N-point filter spectrum:
    binmask [binmask_h, 2N] (or [2N]), a zero entry zeroes that bin; keep it
    Hermitian-symmetric (entry f == entry (2N - f) mod 2N) for a real result."""
    u = _f64(u)
    k = _f64(k)
    w = _f64(w)
    v = _f64(v)
    B, H, N = u.shape
    L = k.shape[1]
    m, mh = _mask(binmask)
    assert m.shape[1] == 2 * N
    y = np.empty((B, H, N), dtype=np.float64)
    ratio = ctypes.c_double(0.0)
    if nthreads is None:
        nthreads = os.cpu_count() or 1
    rc = _load().oracle_fftconv_bins(_ptr(u), _ptr(k), _ptr(y), B, H, N, L, _ptr(w), _ptr(v),
                                     _ptr(m, ctypes.c_uint8), mh, int(nthreads), ctypes.byref(ratio))
    _check(rc, "fftconv_bins")
    if return_imag_ratio:
        return y, ratio.value
    return y


def filter_rfft(k, N, mask=None):
    """K[h, f] = rfft(pad(k[h], 2N))[f] for f in [0, N], masked bins zeroed."""
    k = _f64(k)
    H, L = k.shape
    m, mh = _mask(mask)
    out = np.empty((H, N + 1, 2), dtype=np.float64)
    _check(_load().oracle_filter_rfft(_ptr(k), _ptr(out), H, N, L,
                                      _ptr(m, ctypes.c_uint8), mh), "filter_rfft")
    return out[..., 0] + 1j * out[..., 1]


def direct_conv(u, k, w=None, v=None, seq=None, ts=None):
    """Direct causal sum, everywhere (seq/ts None) or at samples (seq[i], ts[i])."""
    u = _f64(u)
    k = _f64(k)
    w = _f64(w)
    v = _f64(v)
    B, H, N = u.shape
    L = k.shape[1]
    lib = _load()
    if seq is None:
        y = np.empty((B, H, N), dtype=np.float64)
        _check(lib.oracle_direct_conv(_ptr(u), _ptr(k), _ptr(y), B, H, N, L, _ptr(w), _ptr(v),
                                      None, None, -1), "direct_conv")
        return y
    seq = np.ascontiguousarray(np.asarray(seq, dtype=np.int64))
    ts = np.ascontiguousarray(np.asarray(ts, dtype=np.int64))
    y = np.empty(seq.shape[0], dtype=np.float64)
    _check(lib.oracle_direct_conv(_ptr(u), _ptr(k), _ptr(y), B, H, N, L, _ptr(w), _ptr(v),
                                  _ptr(seq, ctypes.c_int64), _ptr(ts, ctypes.c_int64),
                                  seq.shape[0]), "direct_conv")
    return y


def masked_filter(k, N, mask, direct=False):
    """Effective length-2N time-domain filter of the masked spectrum, [H, 2N]."""
    k = _f64(k)
    H, L = k.shape
    m, mh = _mask(mask)
    out = np.empty((H, 2 * N), dtype=np.float64)
    fn = _load().oracle_masked_filter_direct if direct else _load().oracle_masked_filter_fft
    _check(fn(_ptr(k), _ptr(out), H, N, L, _ptr(m, ctypes.c_uint8), mh), "masked_filter")
    return out


def circular_conv_samples(u, keff, seq, ts, w=None, v=None):
    """v[t] * sum_s keff[h, s] * x[(t - s) mod 2N] at the samples (x zero-padded)."""
    u = _f64(u)
    keff = _f64(keff)
    w = _f64(w)
    v = _f64(v)
    B, H, N = u.shape
    seq = np.ascontiguousarray(np.asarray(seq, dtype=np.int64))
    ts = np.ascontiguousarray(np.asarray(ts, dtype=np.int64))
    y = np.empty(seq.shape[0], dtype=np.float64)
    _check(_load().oracle_circular_conv_samples(_ptr(u), _ptr(keff), _ptr(y), B, H, N,
                                                _ptr(w), _ptr(v), _ptr(seq, ctypes.c_int64),
                                                _ptr(ts, ctypes.c_int64), seq.shape[0]),
           "circular_conv_samples")
    return y


def conv_backward(u, k, dy, w=None, v=None, route="fft"):
    """Gradients of y = v * conv(u * w, k) for the incoming gradient dy:
    dict(du, dw, dv, dk) (dw only with w, dv only with v); dk is [H, L] summed
    over the batch.  route "fft" (own FFT, any size) or "direct" (O(N*L)
    sums)."""
    u = _f64(u)
    k = _f64(k)
    dy = _f64(dy)
    w = _f64(w)
    v = _f64(v)
    B, H, N = u.shape
    L = k.shape[1]
    du = np.empty((B, H, N))
    dw = np.empty((B, H, N)) if w is not None else None
    dv = np.empty((B, H, N)) if v is not None else None
    dk = np.empty((H, L))
    fn = _load().oracle_conv_backward_fft if route == "fft" else _load().oracle_conv_backward_direct
    _check(fn(_ptr(u), _ptr(k), _ptr(w), _ptr(v), _ptr(dy), B, H, N, L, _ptr(du), _ptr(dw), _ptr(dv),
              _ptr(dk)), "conv_backward")
    return {"du": du, "dw": dw, "dv": dv, "dk": dk}


def compile_variant(src_text: str, out_path: str) -> str:
    """Compile C source text (e.g. a deliberately mutated copy of the oracle,
    used by the tests to show that the pins catch planted mistakes)."""
    src = out_path + ".c"
    with open(src, "w") as f:
        f.write(src_text)
    subprocess.check_call(["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-o", out_path,
                           src, "-lm", "-lpthread"])
    return out_path


def source_text() -> str:
    with open(_SRC) as f:
        return f.read()


class using_library:
    """Context manager: route every oracle call through another compiled copy."""

    def __init__(self, path: str):
        self.path = path
        self.old = None

    def __enter__(self):
        global _lib
        _load()
        self.old = _lib
        _lib = _bind(ctypes.CDLL(self.path))
        return self

    def __exit__(self, *exc):
        global _lib
        _lib = self.old
        return False
