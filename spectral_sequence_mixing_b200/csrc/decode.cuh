// decode.cuh -- one autoregressive step of the causal convolution.
//
// Caracal (Causal Architecture via Spectral Mixing) predicts the next token
// ("next-token prediction" in its framework figure); at generation time the
// new position t needs only
//
//     r[b, t, d] = sum_{j=0..t} v[b, j, d] * g[b, t-j, d]
//
// from the cached value and gate streams: an O(t) dot product per channel,
// which reads 2 (t+1) values per channel once and is bound by HBM bandwidth,
// not by a transform.
//
// Layout: caches [B, Lcap, D] channel-last; output [B, D].  Work is split
// over j into `splits` ranges so the whole GPU streams the caches: kernel 1
// writes fp64 partial sums part[split][b][d] (caller's workspace), kernel 2
// adds them in a fixed order and rounds once.  Accumulating in fp64 keeps the
// result within one fp32 rounding of the exact sum and makes it
// deterministic.
#pragma once

#include <stdint.h>

#include "fftconv_fused.cuh"  // IO_t

namespace ccv {

constexpr int kDecodeThreads = 256;
constexpr int kDecodeUnroll = 4;

// Number of j-ranges for a decode call: aim at ~1024 CTAs of 256 channels,
// at least 64 positions per range, at most 64 ranges.  Depends only on the
// problem (so the workspace size is host-computable).
static inline int decode_splits(int64_t B, int64_t D, int64_t t) {
    const int64_t ctas = B * ((D + kDecodeThreads - 1) / kDecodeThreads);
    int64_t s = (1024 + ctas - 1) / ctas;
    const int64_t max_by_len = (t + 1 + 63) / 64;
    if (s > max_by_len) s = max_by_len;
    if (s > 64) s = 64;
    if (s < 1) s = 1;
    return (int)s;
}

template <typename IO>
__global__ void __launch_bounds__(kDecodeThreads)
    decode_partial_kernel(const IO *__restrict__ v, const IO *__restrict__ g, double *__restrict__ part, int B,
                          int Lcap, int D, int t, int chunk) {
    const int d = blockIdx.x * kDecodeThreads + threadIdx.x;
    const int sp = blockIdx.y, b = blockIdx.z;
    if (d >= D) return;
    const int j0 = sp * chunk;
    const int j1 = min(t + 1, j0 + chunk);
    const int64_t row = (int64_t)b * Lcap;
    const IO *vb = v + row * D + d;
    const IO *gb = g + row * D + d;
    double acc[kDecodeUnroll] = {0.0, 0.0, 0.0, 0.0};
    int j = j0;
    for (; j + kDecodeUnroll <= j1; j += kDecodeUnroll) {
#pragma unroll
        for (int u = 0; u < kDecodeUnroll; ++u) {
            const float a = IO_t<IO>::cvt(IO_t<IO>::ld(vb + (int64_t)(j + u) * D));
            const float c = IO_t<IO>::cvt(IO_t<IO>::ld(gb + (int64_t)(t - j - u) * D));
            acc[u] = fma((double)a, (double)c, acc[u]);
        }
    }
    for (; j < j1; ++j) {
        const float a = IO_t<IO>::cvt(IO_t<IO>::ld(vb + (int64_t)j * D));
        const float c = IO_t<IO>::cvt(IO_t<IO>::ld(gb + (int64_t)(t - j) * D));
        acc[0] = fma((double)a, (double)c, acc[0]);
    }
    part[((int64_t)sp * B + b) * D + d] = (acc[0] + acc[1]) + (acc[2] + acc[3]);
}

template <typename IO>
__global__ void __launch_bounds__(kDecodeThreads)
    decode_reduce_kernel(const double *__restrict__ part, IO *__restrict__ r, int64_t BD, int splits) {
    const int64_t i = (int64_t)blockIdx.x * kDecodeThreads + threadIdx.x;
    if (i >= BD) return;
    double s = 0.0;
    for (int k = 0; k < splits; ++k) s += part[(int64_t)k * BD + i];
    IO_t<IO>::st(r + i, (float)s);
}

template <typename IO>
static int decode_launch(const IO *v, const IO *g, IO *r, int64_t B, int64_t Lcap, int64_t D, int64_t t,
                         double *part, cudaStream_t s) {
    const int splits = decode_splits(B, D, t);
    const int chunk = (int)((t + 1 + splits - 1) / splits);
    const dim3 grid((unsigned)((D + kDecodeThreads - 1) / kDecodeThreads), (unsigned)splits, (unsigned)B);
    decode_partial_kernel<IO><<<grid, kDecodeThreads, 0, s>>>(v, g, part, (int)B, (int)Lcap, (int)D, (int)t, chunk);
    if (cudaGetLastError() != cudaSuccess) return 5;  // CC_ERR_CUDA
    const int64_t BD = B * D;
    decode_reduce_kernel<IO><<<(unsigned)((BD + kDecodeThreads - 1) / kDecodeThreads), kDecodeThreads, 0, s>>>(
        part, r, BD, splits);
    return cudaGetLastError() == cudaSuccess ? 0 : 5;
}

}  // namespace ccv
