// common.cuh -- shared device helpers: complex arithmetic on float2, I/O type
// conversion, compile-time DFT twiddles and register-resident small DFTs.
//
// The small DFTs are the "DFT factors" of the Monarch decomposition of the FFT
// (FlashFFTConv: Efficient Convolutions for Long Sequences with Tensor Cores,
// "Approach"): a length-L transform is a product of length-R_i DFTs applied
// along one digit of the index, with twiddle scalings in between.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <type_traits>
#include <utility>

namespace fftconv {

// ------------------------------------------------------------ complex ---

__device__ __forceinline__ float2 cadd(float2 a, float2 b) { return make_float2(a.x + b.x, a.y + b.y); }
__device__ __forceinline__ float2 csub(float2 a, float2 b) { return make_float2(a.x - b.x, a.y - b.y); }
__device__ __forceinline__ float2 cmul(float2 a, float2 b) {
    return make_float2(fmaf(a.x, b.x, -a.y * b.y), fmaf(a.x, b.y, a.y * b.x));
}
// a * conj(b)
__device__ __forceinline__ float2 cmulc(float2 a, float2 b) {
    return make_float2(fmaf(a.x, b.x, a.y * b.y), fmaf(a.y, b.x, -a.x * b.y));
}
__device__ __forceinline__ float2 cscale(float2 a, float s) { return make_float2(a.x * s, a.y * s); }

// ------------------------------------------------------- I/O dtypes ---

template <typename T> __device__ __forceinline__ float to_f32(T v);
template <> __device__ __forceinline__ float to_f32<float>(float v) { return v; }
template <> __device__ __forceinline__ float to_f32<__half>(__half v) { return __half2float(v); }
template <> __device__ __forceinline__ float to_f32<__nv_bfloat16>(__nv_bfloat16 v) { return __bfloat162float(v); }

template <typename T> __device__ __forceinline__ T from_f32(float v);
template <> __device__ __forceinline__ float from_f32<float>(float v) { return v; }
template <> __device__ __forceinline__ __half from_f32<__half>(float v) { return __float2half_rn(v); }
template <> __device__ __forceinline__ __nv_bfloat16 from_f32<__nv_bfloat16>(float v) { return __float2bfloat16_rn(v); }

// ----------------------------------------------- compile-time twiddles ---
// cos(2*pi*k/n), sin(2*pi*k/n) as constant expressions: the angle is reduced
// exactly (integer arithmetic) to the nearest quarter turn plus a residual in
// [-pi/4, pi/4], where a Taylor series converges to double precision.

constexpr double kPi = 3.14159265358979323846264338327950288;

__host__ __device__ constexpr double taylor_cos(double x) {
    double term = 1.0, sum = 1.0;
    for (int i = 1; i < 24; ++i) { term *= -x * x / ((2.0 * i - 1.0) * (2.0 * i)); sum += term; }
    return sum;
}
__host__ __device__ constexpr double taylor_sin(double x) {
    double term = x, sum = x;
    for (int i = 1; i < 24; ++i) { term *= -x * x / ((2.0 * i) * (2.0 * i + 1.0)); sum += term; }
    return sum;
}
// quarter-turn index q and residual angle x with 2*pi*k/n = q*pi/2 + x
__host__ __device__ constexpr long long quarter_index(long long k, long long n) {
    return (4 * k + n / 2) / n;                      // k in [0, n)
}
__host__ __device__ constexpr double quarter_residual(long long k, long long n) {
    return (2.0 * kPi / (4.0 * (double)n)) * (double)(4 * k - quarter_index(k, n) * n);
}
__host__ __device__ constexpr double cos2pi(long long k, long long n) {
    k %= n; if (k < 0) k += n;
    long long q = quarter_index(k, n) & 3;
    double x = quarter_residual(k, n);
    return q == 0 ? taylor_cos(x) : q == 1 ? -taylor_sin(x) : q == 2 ? -taylor_cos(x) : taylor_sin(x);
}
__host__ __device__ constexpr double sin2pi(long long k, long long n) {
    k %= n; if (k < 0) k += n;
    long long q = quarter_index(k, n) & 3;
    double x = quarter_residual(k, n);
    return q == 0 ? taylor_sin(x) : q == 1 ? taylor_cos(x) : q == 2 ? -taylor_sin(x) : -taylor_cos(x);
}

template <int I, int N, typename F>
__device__ __forceinline__ void static_for(F&& f) {
    if constexpr (I < N) {
        f(std::integral_constant<int, I>{});
        static_for<I + 1, N>(f);
    }
}

// x * exp(DIR * 2*pi*i * J / R) with J, R compile-time constants.
template <int DIR, int J, int R>
__device__ __forceinline__ float2 twiddle_const(float2 x) {
    constexpr int j = ((J % R) + R) % R;
    if constexpr (j == 0) {
        return x;
    } else if constexpr (4 * j == R) {              // DIR * i
        return DIR > 0 ? make_float2(-x.y, x.x) : make_float2(x.y, -x.x);
    } else if constexpr (2 * j == R) {              // -1
        return make_float2(-x.x, -x.y);
    } else if constexpr (4 * j == 3 * R) {          // -DIR * i
        return DIR > 0 ? make_float2(x.y, -x.x) : make_float2(-x.y, x.x);
    } else {
        constexpr float c = (float)cos2pi(j, R);
        constexpr float s = (float)(DIR * sin2pi(j, R));
        if constexpr (8 * j == R || 8 * j == 3 * R || 8 * j == 5 * R || 8 * j == 7 * R) {
            // |c| == |s| == 1/sqrt(2): two adds and two multiplies
            constexpr float a = c > 0.f ? c : -c;
            constexpr float sc = (c > 0.f) ? 1.f : -1.f;
            constexpr float ss = (s > 0.f) ? 1.f : -1.f;
            float re = sc * x.x - ss * x.y;
            float im = sc * x.y + ss * x.x;
            return make_float2(a * re, a * im);
        } else {
            return make_float2(fmaf(c, x.x, -s * x.y), fmaf(c, x.y, s * x.x));
        }
    }
}

// In-register DFT of length R (power of two), natural order in and out:
//   X[c] = sum_j x[j] * exp(DIR * 2*pi*i * c*j / R)
// by radix-2 decimation in frequency with compile-time twiddles.
template <int R, int DIR>
struct Dft {
    static __device__ __forceinline__ void run(float2 (&x)[R]) {
        float2 e[R / 2], o[R / 2];
        static_for<0, R / 2>([&](auto jc) {
            constexpr int j = decltype(jc)::value;
            float2 a = x[j], b = x[j + R / 2];
            e[j] = cadd(a, b);
            o[j] = twiddle_const<DIR, j, R>(csub(a, b));
        });
        Dft<R / 2, DIR>::run(e);
        Dft<R / 2, DIR>::run(o);
#pragma unroll
        for (int c = 0; c < R / 2; ++c) { x[2 * c] = e[c]; x[2 * c + 1] = o[c]; }
    }
    // Same transform when x[j] == 0 for j >= R/2 (zero-padded input): the
    // first butterfly level reduces to a copy and a twiddle.
    static __device__ __forceinline__ void run_half_input(float2 (&x)[R]) {
        float2 e[R / 2], o[R / 2];
        static_for<0, R / 2>([&](auto jc) {
            constexpr int j = decltype(jc)::value;
            e[j] = x[j];
            o[j] = twiddle_const<DIR, j, R>(x[j]);
        });
        Dft<R / 2, DIR>::run(e);
        Dft<R / 2, DIR>::run(o);
#pragma unroll
        for (int c = 0; c < R / 2; ++c) { x[2 * c] = e[c]; x[2 * c + 1] = o[c]; }
    }
};
template <int DIR>
struct Dft<1, DIR> {
    static __device__ __forceinline__ void run(float2 (&)[1]) {}
    static __device__ __forceinline__ void run_half_input(float2 (&)[1]) {}
};

// ------------------------------------------------------- status word ---

enum : int { kStatusOk = 0, kStatusTimeout = -6, kStatusRange = -7 };

// Non-finite detector for the 16-bit tensor-core paths, whose intermediates
// are fp16: acc stays 0 while every value folded in is finite and becomes NaN
// once one is inf or NaN (0 * inf and 0 * NaN are NaN).  Inline PTX keeps the
// compiler from folding x * 0 away.
__device__ __forceinline__ void nonfinite_fold(float& acc, float x) {
    asm("fma.rn.f32 %0, %1, 0f00000000, %0;" : "+f"(acc) : "f"(x));
}
// Record FFTCONV_ERR_RANGE in the status word if acc saw a non-finite value
// (an earlier timeout is not overwritten).
__device__ __forceinline__ void nonfinite_report(float acc, int* status) {
    if (acc != acc) atomicCAS(status, 0, kStatusRange);
}

}  // namespace fftconv
