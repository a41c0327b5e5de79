// fft_reg.cuh -- in-register complex FFT building blocks for sm_100a.
//
// Every array index below is a compile-time constant after unrolling, so the
// arrays live in registers and the twiddles omega_R^e (read from the constant
// bank c_w128) become constant-bank operands of the FP32 instructions.
//
// Convention: forward transforms use omega_R = exp(-2*pi*i/R); inverse
// transforms use its conjugate and are unnormalised (the caller scales once).
#pragma once

#include <cuda_runtime.h>

namespace ccv {

// exp(-2*pi*i*k/128), k = 0..127; filled once per device from host fp64 values.
__constant__ float2 c_w128[128];

constexpr int ilog2(int n) { return n <= 1 ? 0 : 1 + ilog2(n >> 1); }

constexpr int bitrev(int x, int bits) {
    int r = 0;
    for (int i = 0; i < bits; ++i) r = (r << 1) | ((x >> i) & 1);
    return r;
}

// omega_R^e for compile-time e, R (R divides 128).
__device__ __forceinline__ float2 tw_const(int e, int R) { return c_w128[(e * (128 / R)) & 127]; }

__device__ __forceinline__ float2 cmul(float2 a, float2 w) {
    return make_float2(fmaf(a.x, w.x, -a.y * w.y), fmaf(a.x, w.y, a.y * w.x));
}
// a * conj(w)
__device__ __forceinline__ float2 cmul_conj(float2 a, float2 w) {
    return make_float2(fmaf(a.x, w.x, a.y * w.y), fmaf(a.y, w.x, -a.x * w.y));
}
__device__ __forceinline__ float2 cadd(float2 a, float2 b) { return make_float2(a.x + b.x, a.y + b.y); }
__device__ __forceinline__ float2 csub(float2 a, float2 b) { return make_float2(a.x - b.x, a.y - b.y); }
__device__ __forceinline__ float2 cconj(float2 a) { return make_float2(a.x, -a.y); }

// Radix-2 DIT butterfly (a, b) <- (a + w b, a - w b); the difference is
// formed as 2a - (a + w b) so the whole butterfly is six FMAs.
// INV selects w -> conj(w).
template <bool INV>
__device__ __forceinline__ void bfly_tw(float2 &a, float2 &b, float2 w) {
    const float wy = INV ? -w.y : w.y;
    const float sx = fmaf(w.x, b.x, fmaf(-wy, b.y, a.x));
    const float sy = fmaf(w.x, b.y, fmaf(wy, b.x, a.y));
    b.x = fmaf(2.f, a.x, -sx);
    b.y = fmaf(2.f, a.y, -sy);
    a.x = sx;
    a.y = sy;
}

// w = 1
__device__ __forceinline__ void bfly_one(float2 &a, float2 &b) {
    const float2 s = cadd(a, b);
    b = csub(a, b);
    a = s;
}

// w = -i (forward) or +i (inverse)
template <bool INV>
__device__ __forceinline__ void bfly_quarter(float2 &a, float2 &b) {
    // forward: w b = (b.y, -b.x);  inverse: w b = (-b.y, b.x)
    float2 s, d;
    if (!INV) {
        s = make_float2(a.x + b.y, a.y - b.x);
        d = make_float2(a.x - b.y, a.y + b.x);
    } else {
        s = make_float2(a.x - b.y, a.y + b.x);
        d = make_float2(a.x + b.y, a.y - b.x);
    }
    a = s;
    b = d;
}

// In-place radix-2 decimation-in-time FFT of length R on x[], whose entries
// must hold the input in bit-reversed order; the output is in natural order.
// ZERO_ODD: the odd slots hold zeros (the upper half of a zero-padded input),
//           so the first stage is a copy.
// KEEP_LOW: only outputs [0, R/2) are formed in the last stage (truncation).
template <int R, bool INV, bool ZERO_ODD = false, bool KEEP_LOW = false>
__device__ __forceinline__ void fft_dit(float2 (&x)[R]) {
#pragma unroll
    for (int half = 1; half < R; half <<= 1) {
#pragma unroll
        for (int base = 0; base < R; base += 2 * half) {
#pragma unroll
            for (int k = 0; k < half; ++k) {
                const int e = k * (R / (2 * half));  // twiddle exponent in units of omega_R
                float2 &a = x[base + k];
                float2 &b = x[base + k + half];
                if (ZERO_ODD && half == 1) {
                    b = a;
                } else if (KEEP_LOW && 2 * half == R) {
                    if (e == 0) {
                        a = cadd(a, b);
                    } else if (4 * e == R) {
                        a = INV ? make_float2(a.x - b.y, a.y + b.x) : make_float2(a.x + b.y, a.y - b.x);
                    } else {
                        const float2 w = tw_const(e, R);
                        const float wy = INV ? -w.y : w.y;
                        a = make_float2(fmaf(w.x, b.x, fmaf(-wy, b.y, a.x)), fmaf(w.x, b.y, fmaf(wy, b.x, a.y)));
                    }
                } else if (e == 0) {
                    bfly_one(a, b);
                } else if (4 * e == R) {
                    bfly_quarter<INV>(a, b);
                } else {
                    bfly_tw<INV>(a, b, tw_const(e, R));
                }
            }
        }
    }
}

// Power-of-two scale alpha ~ sqrt(sv / sg) that balances a row's value and
// gate streams before they share one complex transform (z = v + i alpha g).
// The spectra are separated as V = (Z_k + conj Z_m)/2, G = (Z_k - conj Z_m)/2i,
// so a stream much smaller than the other inherits the other's absolute
// rounding error; equal norms remove that amplification.  A power of two
// makes the scaling (and the undoing of it on the output) exact.
__device__ __forceinline__ float balance_scale(float sv, float sg) {
    if (!(sv > 0.f) || !(sg > 0.f)) return 1.f;
    int e = __float2int_rn(0.5f * log2f(sv / sg));
    e = max(-60, min(60, e));
    return ldexpf(1.f, e);
}

}  // namespace ccv
