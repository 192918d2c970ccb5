"""Python binding of the B200 causal long-convolution library (libfftconv.so).

Argument marshalling only: every step of the convolution runs in the library's
CUDA kernels.  PyTorch provides device memory and streams.  There is no CPU or
PyTorch fallback: if the compiled library is missing, importing this package
fails with an ImportError that says how to build it.

Operation (FlashFFTConv: Efficient Convolutions for Long Sequences with Tensor
Cores, summary paragraph, "Approach", "Key results"):

    y[b,h,t] = v[b,h,t] * sum_{s <= min(t, L-1)} k[h,s] * u[b,h,t-s] * w[b,h,t-s]

computed as irfft(rfft(u*w, 2N) * rfft(k, 2N))[:N].
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libfftconv.so")

if not os.path.exists(LIB_PATH):
    raise ImportError(
        f"{LIB_PATH} is missing: build it with `python long_sequence_fft_b200/build.py` "
        "(nvcc, sm_100a). There is no CPU fallback.")

_lib = ctypes.CDLL(LIB_PATH)

F32, F16, BF16 = 0, 1, 2
OK, ERR_INVALID_ARG, ERR_UNSUPPORTED, ERR_ALIGNMENT, ERR_CUDA, ERR_OOM, ERR_TIMEOUT, ERR_RANGE = 0, -1, -2, -3, -4, -5, -6, -7
PATH_SIMT_FUSED, PATH_SIMT_STAGED, PATH_TC_FUSED, PATH_TC_STAGED = 1, 2, 3, 4
PATH_NAMES = {PATH_SIMT_FUSED: "simt_fused", PATH_SIMT_STAGED: "simt_staged", PATH_TC_FUSED: "tc_fused",
              PATH_TC_STAGED: "tc_staged"}

_vp = ctypes.c_void_p
_i64 = ctypes.c_int64
_sz = ctypes.c_size_t

_SIGNATURES = {
    "fftconv_plan_create": (ctypes.c_int, [ctypes.POINTER(_vp), _i64, _i64, ctypes.c_int, ctypes.c_int]),
    "fftconv_plan_create_ex": (ctypes.c_int, [ctypes.POINTER(_vp), _i64, _i64, ctypes.c_int, ctypes.c_int, _i64]),
    "fftconv_plan_destroy": (ctypes.c_int, [_vp]),
    "fftconv_filter_bytes": (_sz, [_vp]),
    "fftconv_workspace_bytes": (_sz, [_vp]),
    "fftconv_plan_path": (ctypes.c_int, [_vp]),
    "fftconv_filter_precompute": (ctypes.c_int, [_vp, _vp, _vp, _vp]),
    "fftconv_forward": (ctypes.c_int, [_vp, _vp, _vp, _vp, _i64, _i64, _i64, _vp, _vp, _vp, _i64, _vp]),
    "fftconv_forward_monarch": (ctypes.c_int, [_vp, _vp, _vp, _vp, _i64, _i64, _i64, _vp, _vp, ctypes.c_uint32,
                                               _vp]),
    "fftconv_forward_host_staging_bytes": (_sz, [_vp, _i64, ctypes.c_int, ctypes.c_int, ctypes.c_int, _i64]),
    "fftconv_forward_host": (ctypes.c_int, [_vp, _vp, _vp, _vp, _i64, _i64, _i64, _vp, _vp, _vp, _i64, _vp,
                                            _sz, _vp]),
    "fftconv_backward": (ctypes.c_int, [_vp, _vp, _vp, _vp, _i64, _i64, _i64, _vp, _vp, _vp, _vp, _vp, _vp,
                                        _vp]),
    "fftconv_filter_to_rfft": (ctypes.c_int, [_vp, _vp, _vp, _vp]),
    "fftconv_device_status": (ctypes.c_int, [_vp, _vp]),
    "fftconv_selftest_bounded_wait": (ctypes.c_int, [_vp, _i64, ctypes.c_int, _vp]),
    "fftconv_status_string": (ctypes.c_char_p, [ctypes.c_int]),
    "fftconv_last_error": (ctypes.c_char_p, []),
    "fftconv_version": (ctypes.c_char_p, []),
}
for _name, (_res, _args) in _SIGNATURES.items():
    _f = getattr(_lib, _name)
    _f.restype = _res
    _f.argtypes = _args


class FFTConvError(RuntimeError):
    def __init__(self, status: int, detail: str):
        self.status = status
        super().__init__(f"{_lib.fftconv_status_string(status).decode()} ({status}): {detail}")


def _check(rc: int):
    if rc != OK:
        raise FFTConvError(rc, _lib.fftconv_last_error().decode())


def version() -> str:
    return _lib.fftconv_version().decode()


def library():
    """The loaded ctypes library (tests use it to call the C ABI directly)."""
    return _lib


def _dtype_code(dtype) -> int:
    import torch
    if dtype in (torch.float32, "f32", "float32", F32):
        return F32
    if dtype in (torch.float16, "f16", "float16", F16):
        return F16
    if dtype in (torch.bfloat16, "bf16", "bfloat16", BF16):
        return BF16
    raise ValueError(f"unsupported dtype {dtype}")


def _torch_dtype(code: int):
    import torch
    return {F32: torch.float32, F16: torch.float16, BF16: torch.bfloat16}[code]


def _ptr(t) -> Optional[int]:
    return None if t is None else t.data_ptr()


def _stream_handle(stream) -> Optional[int]:
    import torch
    if stream is None:
        stream = torch.cuda.current_stream()
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


class Plan:
    """A convolution plan for sequences of length N, H channels, one dtype.

    order: the Monarch order requested (include/fftconv.h): 0 automatic,
    2 or 3 fused on chip (one kernel; tensor cores where available), 4 staged
    through a device-memory workspace on fp32 lanes (any N); and two engine
    choices: 1 fused on fp32 lanes (N <= 8192), 5 staged with the row pass on
    the tensor cores (fp16/bf16, 16384 <= N <= 2^22, L > 2049).  L < N gives
    the partial convolution."""

    def __init__(self, N: int, H: int, dtype="bf16", order: int = 0, L: Optional[int] = None):
        self.N, self.H = int(N), int(H)
        self.L = int(L) if L is not None else self.N
        self.dtype_code = _dtype_code(dtype)
        self.order = int(order)
        h = _vp()
        _check(_lib.fftconv_plan_create_ex(ctypes.byref(h), self.N, self.H, self.dtype_code, self.order, self.L))
        self._h = h

    # -- properties
    @property
    def handle(self):
        return self._h

    @property
    def dtype(self):
        return _torch_dtype(self.dtype_code)

    @property
    def filter_bytes(self) -> int:
        return int(_lib.fftconv_filter_bytes(self._h))

    @property
    def workspace_bytes(self) -> int:
        return int(_lib.fftconv_workspace_bytes(self._h))

    @property
    def path(self) -> int:
        p = _lib.fftconv_plan_path(self._h)
        if p < 0:
            _check(p)
        return p

    @property
    def path_name(self) -> str:
        return PATH_NAMES.get(self.path, "?")

    def close(self):
        if getattr(self, "_h", None) is not None and self._h.value:
            _lib.fftconv_plan_destroy(self._h)
            self._h = _vp()

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    # -- calls
    def _check_tensor(self, t, shape, name):
        import torch
        if t is None:
            return
        if not t.is_cuda:
            raise ValueError(f"{name} must be a CUDA tensor")
        if t.dtype != self.dtype:
            raise ValueError(f"{name} has dtype {t.dtype}, plan expects {self.dtype}")
        if tuple(t.shape) != tuple(shape):
            raise ValueError(f"{name} has shape {tuple(t.shape)}, expected {tuple(shape)}")
        if not t.is_contiguous():
            raise ValueError(f"{name} must be contiguous")

    def new_filter(self):
        import torch
        return torch.empty(self.filter_bytes, dtype=torch.uint8, device="cuda")

    def precompute(self, k, out=None, stream=None):
        """K_f for filter k [H, L] (plan dtype, CUDA): an opaque uint8 tensor."""
        self._check_tensor(k, (self.H, self.L), "k")
        if out is None:
            out = self.new_filter()
        _check(_lib.fftconv_filter_precompute(self._h, _ptr(k), _ptr(out), _stream_handle(stream)))
        return out

    def forward(self, u, Kf, w=None, v=None, mask=None, out=None, stream=None):
        """y = v * conv(u * w, k) for u [B, H, N]; mask [mask_h, N/32] uint8 or None."""
        import torch
        B = u.shape[0]
        shape = (B, self.H, self.N)
        self._check_tensor(u, shape, "u")
        self._check_tensor(w, shape, "w")
        self._check_tensor(v, shape, "v")
        if out is None:
            out = torch.empty(shape, dtype=self.dtype, device=u.device)
        self._check_tensor(out, shape, "out")
        mask_h = 0
        if mask is not None:
            if mask.dtype != torch.uint8 or not mask.is_cuda or mask.dim() != 2:
                raise ValueError("mask must be a 2-D CUDA uint8 tensor [mask_h, N/32]")
            mask_h = mask.shape[0]
        _check(_lib.fftconv_forward(self._h, _ptr(u), _ptr(Kf), _ptr(out), B, self.H, self.N, _ptr(w), _ptr(v),
                                    _ptr(mask), mask_h, _stream_handle(stream)))
        return out

    def forward_monarch(self, u, Kf, keep_c2, w=None, v=None, out=None, stream=None):
        """forward with a Monarch-aligned frequency mask (N = 4096 tensor-core
        plans): bit c2 of keep_c2 keeps the 8192-point spectrum bins whose
        middle digit (f >> 5) & 31 is c2 (and whose mirror's is kept too)."""
        import torch
        B = u.shape[0]
        shape = (B, self.H, self.N)
        self._check_tensor(u, shape, "u")
        self._check_tensor(w, shape, "w")
        self._check_tensor(v, shape, "v")
        if out is None:
            out = torch.empty(shape, dtype=self.dtype, device=u.device)
        self._check_tensor(out, shape, "out")
        _check(_lib.fftconv_forward_monarch(self._h, _ptr(u), _ptr(Kf), _ptr(out), B, self.H, self.N, _ptr(w),
                                            _ptr(v), int(keep_c2) & 0xffffffff, _stream_handle(stream)))
        return out

    def backward(self, u, Kf, dy, w=None, v=None, want_dk=True, stream=None, out=None):
        """Gradients of y = v * conv(u * w, k) for dy: dict(du, dw, dv, dk) with
        dw only when w is given, dv only when v is given, dk an fp32 [H, L]
        tensor (summed over the batch) when want_dk.  `out`: an earlier
        call's dict to write into instead of allocating."""
        import torch
        B = u.shape[0]
        shape = (B, self.H, self.N)
        for t, name in ((u, "u"), (w, "w"), (v, "v"), (dy, "dy")):
            self._check_tensor(t, shape, name)
        if out is not None:
            du, dw, dv, dk = out.get("du"), out.get("dw"), out.get("dv"), out.get("dk")
            for t, name, need in ((du, "du", True), (dw, "dw", w is not None), (dv, "dv", v is not None)):
                if need and t is None:
                    raise ValueError(f"out[{name!r}] is missing")
                if not need and t is not None:
                    raise ValueError(f"out[{name!r}] given without its gate")
                self._check_tensor(t, shape, name)
            if want_dk and (dk is None or dk.dtype != torch.float32 or tuple(dk.shape) != (self.H, self.L)
                            or not dk.is_contiguous()):
                raise ValueError("out['dk'] must be a contiguous float32 [H, L] tensor")
            if not want_dk:
                dk = None
            return self._backward_into(u, Kf, dy, w, v, du, dw, dv, dk, B, stream)
        du = torch.empty(shape, dtype=self.dtype, device=u.device)
        dw = torch.empty_like(du) if w is not None else None
        dv = torch.empty_like(du) if v is not None else None
        dk = torch.empty((self.H, self.L), dtype=torch.float32, device=u.device) if want_dk else None
        return self._backward_into(u, Kf, dy, w, v, du, dw, dv, dk, B, stream)

    def _backward_into(self, u, Kf, dy, w, v, du, dw, dv, dk, B, stream):
        _check(_lib.fftconv_backward(self._h, _ptr(u), _ptr(Kf), _ptr(dy), B, self.H, self.N, _ptr(w), _ptr(v),
                                     _ptr(du), _ptr(dw), _ptr(dv), _ptr(dk), _stream_handle(stream)))
        return {"du": du, "dw": dw, "dv": dv, "dk": dk}

    def staging_bytes(self, B: int, has_w: bool, has_v: bool, mask_h: int = 0) -> int:
        return int(_lib.fftconv_forward_host_staging_bytes(self._h, B, int(has_w), int(has_v), int(mask_h > 0),
                                                           mask_h))

    def forward_host(self, u_host, Kf, y_host, staging, w_host=None, v_host=None, mask_host=None, stream=None):
        """fftconv_forward_host on (pinned) CPU tensors; K_f and staging on the device."""
        B = u_host.shape[0]
        mask_h = 0 if mask_host is None else mask_host.shape[0]
        _check(_lib.fftconv_forward_host(self._h, _ptr(u_host), _ptr(Kf), _ptr(y_host), B, self.H, self.N,
                                         _ptr(w_host), _ptr(v_host), _ptr(mask_host), mask_h, _ptr(staging),
                                         staging.numel() * staging.element_size(), _stream_handle(stream)))
        return y_host

    def export_rfft(self, Kf, stream=None):
        """rfft(k)[h, 0..N] from K_f as a complex64 [H, N+1] tensor (test hook)."""
        import torch
        out = torch.empty((self.H, self.N + 1, 2), dtype=torch.float32, device="cuda")
        _check(_lib.fftconv_filter_to_rfft(self._h, _ptr(Kf), _ptr(out), _stream_handle(stream)))
        return torch.view_as_complex(out)

    def device_status(self, stream=None) -> int:
        return int(_lib.fftconv_device_status(self._h, _stream_handle(stream)))


_PLAN_CACHE = {}


def cached_plan(N: int, H: int, dtype, L: int, order: int = 0) -> "Plan":
    """A plan per (device, N, H, dtype, L, order), created on first use and
    kept for the process (plans own device tables; creating one per call
    would repeat their uploads)."""
    import torch
    key = (torch.cuda.current_device(), int(N), int(H), str(dtype), int(L), int(order))
    plan = _PLAN_CACHE.get(key)
    if plan is None:
        plan = _PLAN_CACHE[key] = Plan(N, H, dtype, order=order, L=L)
    return plan


_AUTOGRAD_FN = None


def _autograd_function():
    """torch.autograd.Function over fftconv_forward / fftconv_backward, built
    on first use so that importing the package does not import torch."""
    global _AUTOGRAD_FN
    if _AUTOGRAD_FN is not None:
        return _AUTOGRAD_FN
    import torch

    class FFTConvFunction(torch.autograd.Function):
        @staticmethod
        def forward(ctx, u, k, w, v, plan):
            Kf = plan.precompute(k)
            ctx.plan = plan
            ctx.k_dtype = k.dtype
            ctx.save_for_backward(u, w, v, Kf)
            return plan.forward(u, Kf, w=w, v=v)

        @staticmethod
        def backward(ctx, dy):
            u, w, v, Kf = ctx.saved_tensors
            need_u, need_k, need_w, need_v = ctx.needs_input_grad[:4]
            g = ctx.plan.backward(u, Kf, dy.contiguous(), w=w, v=v, want_dk=need_k)
            dk = g["dk"].to(ctx.k_dtype) if need_k else None
            return (g["du"] if need_u else None, dk, g["dw"] if need_w else None,
                    g["dv"] if need_v else None, None)

    _AUTOGRAD_FN = FFTConvFunction
    return _AUTOGRAD_FN


def fftconv(u, k, w=None, v=None, mask=None, order: int = 0):
    """One-shot convenience: y = v * conv(u * w, k) through a cached plan.

    Differentiable when autograd is on and an input requires grad: the
    backward pass runs fftconv_backward (fp16/bf16 tensor-core plans with
    N <= 8192; other plans raise FFTConvError from the backward pass) and
    returns du, dk (cast to k's dtype), dw, dv.  Block masks are forward
    only."""
    import torch
    H, L = k.shape
    needs_grad = torch.is_grad_enabled() and any(t is not None and t.requires_grad for t in (u, k, w, v))
    if needs_grad and mask is not None:
        raise NotImplementedError("fftconv: the backward pass takes no block mask")
    plan = cached_plan(u.shape[2], H, u.dtype, L, order)
    if needs_grad:
        return _autograd_function().apply(u, k, w, v, plan)
    Kf = plan.precompute(k)
    return plan.forward(u, Kf, w=w, v=v, mask=mask)
