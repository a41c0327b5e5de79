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
// (each thread four adjacent channels, one 16-byte fp32 or 8-byte bf16
// access per cache row) writes fp64 partial sums part[split][b][d] (caller's
// workspace), kernel 2 adds them in a fixed order and rounds once (launched
// as a programmatic dependent of kernel 1, so its launch latency overlaps
// kernel 1's tail).  Accumulating in fp64 keeps the
// result within one fp32 rounding of the exact sum and makes it
// deterministic.
#pragma once

#include <stdint.h>

#include "fftconv_fused.cuh"  // IO_t

namespace ccv {

constexpr int kDecodeThreads = 64;   // partial kernel: 64 threads x 4 channels per CTA
constexpr int kDecodeVec = 4;        // channels per thread (one 16-byte fp32 / 8-byte bf16 access)
constexpr int kReduceThreads = 256;
constexpr int kDecodeUnroll = 8;

// Number of j-ranges for a decode call: aim at ~2368 CTAs (16 per SM of a
// 148-SM part) of 256 channels, at least 16 positions per range, at most 128
// ranges.  Depends only on the problem (so the workspace size is
// host-computable).
static inline int decode_splits(int64_t B, int64_t D, int64_t t) {
    const int64_t ctas = B * ((D + kDecodeThreads * kDecodeVec - 1) / (kDecodeThreads * kDecodeVec));
    int64_t s = (2368 + ctas - 1) / ctas;
    const int64_t max_by_len = (t + 1 + 15) / 16;
    if (s > max_by_len) s = max_by_len;
    if (s > 128) s = 128;
    if (s < 1) s = 1;
    return (int)s;
}

// kDecodeVec consecutive channels starting at p (aligned for one access).
__device__ __forceinline__ void decode_ld4(const float *p, float (&o)[kDecodeVec]) {
    const float4 x = __ldg(reinterpret_cast<const float4 *>(p));
    o[0] = x.x;
    o[1] = x.y;
    o[2] = x.z;
    o[3] = x.w;
}
__device__ __forceinline__ void decode_ld4(const __nv_bfloat16 *p, float (&o)[kDecodeVec]) {
    const uint2 x = __ldg(reinterpret_cast<const uint2 *>(p));
    o[0] = __uint_as_float(x.x << 16);
    o[1] = __uint_as_float(x.x & 0xffff0000u);
    o[2] = __uint_as_float(x.y << 16);
    o[3] = __uint_as_float(x.y & 0xffff0000u);
}

// part[split][b][d] = sum over the split's j of v[b, j, d] g[b, t-j, d], in
// fp64, j ascending.  vec: D is a multiple of kDecodeVec and the caches are
// aligned for one access per kDecodeVec channels.
template <typename IO>
__global__ void __launch_bounds__(kDecodeThreads)
    decode_partial_kernel(const IO *__restrict__ v, const IO *__restrict__ g, double *__restrict__ part, int B,
                          int Lcap, int D, int t, int chunk, int vec) {
    const int d0 = (blockIdx.x * kDecodeThreads + threadIdx.x) * kDecodeVec;
    const int sp = blockIdx.y, b = blockIdx.z;
    if (d0 >= D) return;
    const int j0 = sp * chunk;
    const int j1 = min(t + 1, j0 + chunk);
    const int64_t row = (int64_t)b * Lcap;
    const IO *vb = v + row * D + d0;
    const IO *gb = g + row * D + d0;
    double acc[kDecodeVec] = {0.0, 0.0, 0.0, 0.0};
    if (vec) {
#pragma unroll kDecodeUnroll
        for (int j = j0; j < j1; ++j) {
            float a[kDecodeVec], c[kDecodeVec];
            decode_ld4(vb + (int64_t)j * D, a);
            decode_ld4(gb + (int64_t)(t - j) * D, c);
#pragma unroll
            for (int q = 0; q < kDecodeVec; ++q) acc[q] = fma((double)a[q], (double)c[q], acc[q]);
        }
    } else {
        const int nc = min(kDecodeVec, D - d0);
        for (int j = j0; j < j1; ++j) {
#pragma unroll
            for (int q = 0; q < kDecodeVec; ++q)
                if (q < nc) {
                    const float a = IO_t<IO>::cvt(IO_t<IO>::ld(vb + (int64_t)j * D + q));
                    const float c = IO_t<IO>::cvt(IO_t<IO>::ld(gb + (int64_t)(t - j) * D + q));
                    acc[q] = fma((double)a, (double)c, acc[q]);
                }
        }
    }
    double *pp = part + ((int64_t)sp * B + b) * D + d0;
#pragma unroll
    for (int q = 0; q < kDecodeVec; ++q)
        if (d0 + q < D) pp[q] = acc[q];
    // the reduction kernel may be scheduled now; it waits for this grid's
    // completion (griddepcontrol.wait) before it reads the partial sums
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

template <typename IO>
__global__ void __launch_bounds__(kReduceThreads)
    decode_reduce_kernel(const double *__restrict__ part, IO *__restrict__ r, int64_t BD, int splits) {
    // launched as a programmatic dependent of the partial kernel: wait until
    // that grid has completed and its partial sums are visible
    asm volatile("griddepcontrol.wait;" ::: "memory");
    const int64_t i = (int64_t)blockIdx.x * kReduceThreads + threadIdx.x;
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
    const int per_cta = kDecodeThreads * kDecodeVec;
    const dim3 grid((unsigned)((D + per_cta - 1) / per_cta), (unsigned)splits, (unsigned)B);
    const size_t align = kDecodeVec * sizeof(IO);
    const int vec = (D % kDecodeVec) == 0 && ((uintptr_t)v % align) == 0 && ((uintptr_t)g % align) == 0;
    decode_partial_kernel<IO><<<grid, kDecodeThreads, 0, s>>>(v, g, part, (int)B, (int)Lcap, (int)D, (int)t, chunk,
                                                              vec);
    if (cudaGetLastError() != cudaSuccess) return 5;  // CC_ERR_CUDA
    const int64_t BD = B * D;
    // programmatic dependent launch: the reduction's launch overlaps the
    // partial kernel's tail instead of waiting for it on the stream
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)((BD + kReduceThreads - 1) / kReduceThreads));
    cfg.blockDim = dim3(kReduceThreads);
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if (cudaLaunchKernelEx(&cfg, decode_reduce_kernel<IO>, (const double *)part, r, BD, splits) != cudaSuccess) {
        cudaGetLastError();
        return 5;
    }
    return 0;
}

}  // namespace ccv
