// dwconv.cuh -- causal depthwise convolution of the Multi-Head Fourier block.
//
// Caracal: Causal Architecture via Spectral Mixing, "Key design 1": the
// block's first step is a causal depthwise 1-D convolution (kernel size 3)
// that restores local patterns.  For channel-last [B, L, D] arrays and K taps
// per channel:
//
//   y[b, t, d] = bias[d] + sum_{k<K} w[d][k] * x[b, t-(K-1)+k, d],   x[t < 0] = 0
//
// Purely memory-bound (2K flops per 8 bytes at fp32): one thread owns 4
// adjacent channels over a run of kDwRun time steps, consecutive threads take
// consecutive channel quads (a warp reads 512 contiguous bytes per time step
// at fp32), the run's kDwRun vector loads are issued together, and the K-1
// steps before the run are re-read as a halo (K-1 of kDwRun + K-1 rows).
#pragma once

#include <cuda_bf16.h>
#include <stdint.h>

#include <algorithm>
#include <atomic>

namespace ccv {

constexpr int kDwRun = 8;        // time steps per thread (8: 75% of HBM, 16: 72%, 32: 56% on B200)
constexpr int kDwThreads = 256;
constexpr int kDwMaxTaps = 8;

template <typename IO>
struct DwVec;
template <>
struct DwVec<float> {
    __device__ __forceinline__ static float4 load(const float *p) { return __ldg(reinterpret_cast<const float4 *>(p)); }
    __device__ __forceinline__ static void store(float *p, float4 v) { *reinterpret_cast<float4 *>(p) = v; }
    __device__ __forceinline__ static float load1(const float *p) { return __ldg(p); }
    __device__ __forceinline__ static void store1(float *p, float v) { *p = v; }
};
template <>
struct DwVec<__nv_bfloat16> {
    __device__ __forceinline__ static float4 load(const __nv_bfloat16 *p) {
        const uint2 u = __ldg(reinterpret_cast<const uint2 *>(p));
        return make_float4(__uint_as_float(u.x << 16), __uint_as_float(u.x & 0xFFFF0000u),
                           __uint_as_float(u.y << 16), __uint_as_float(u.y & 0xFFFF0000u));
    }
    __device__ __forceinline__ static void store(__nv_bfloat16 *p, float4 v) {
        const __nv_bfloat162 a = __floats2bfloat162_rn(v.x, v.y), b = __floats2bfloat162_rn(v.z, v.w);
        *reinterpret_cast<uint2 *>(p) =
            make_uint2(*reinterpret_cast<const unsigned *>(&a), *reinterpret_cast<const unsigned *>(&b));
    }
    __device__ __forceinline__ static float load1(const __nv_bfloat16 *p) { return __bfloat162float(*p); }
    __device__ __forceinline__ static void store1(__nv_bfloat16 *p, float v) { *p = __float2bfloat16_rn(v); }
};

// Vector path: D % 4 == 0 and 4-channel-aligned rows.  Work item i: channel
// quad i % D4, run (i / D4) % runs, batch i / (D4 runs); the grid (as many
// CTAs as are resident at once) strides over the items, so no partial last
// wave idles part of the machine.
template <int K, typename IO>
__global__ void __launch_bounds__(kDwThreads) dwconv_vec_kernel(const IO *__restrict__ x, const float *__restrict__ w,
                                                                const float *__restrict__ bias, IO *__restrict__ y,
                                                                int L, int D, int runs, int64_t nitems) {
    for (int64_t i = (int64_t)blockIdx.x * kDwThreads + threadIdx.x; i < nitems;
         i += (int64_t)gridDim.x * kDwThreads) {
        const int D4 = D >> 2;
        const int q = (int)(i % D4);
        const int64_t rest = i / D4;
        const int run = (int)(rest % runs);
        const int64_t b = rest / runs;
        const int d = 4 * q, t0 = run * kDwRun;
        float4 wk[K];
#pragma unroll
        for (int k = 0; k < K; ++k)
            wk[k] = make_float4(__ldg(w + (int64_t)(d + 0) * K + k), __ldg(w + (int64_t)(d + 1) * K + k),
                                __ldg(w + (int64_t)(d + 2) * K + k), __ldg(w + (int64_t)(d + 3) * K + k));
        const float4 bs = bias ? make_float4(__ldg(bias + d), __ldg(bias + d + 1), __ldg(bias + d + 2),
                                             __ldg(bias + d + 3))
                               : make_float4(0.f, 0.f, 0.f, 0.f);
        const IO *xb = x + b * (int64_t)L * D + d;
        IO *yb = y + b * (int64_t)L * D + d;
        // window[j] = x[t0 - (K-1) + j], j < K-1+kDwRun; zero before t = 0 and past L
        float4 win[K - 1 + kDwRun];
#pragma unroll
        for (int j = 0; j < K - 1 + kDwRun; ++j) {
            const int t = t0 - (K - 1) + j;
            win[j] = (t >= 0 && t < L) ? DwVec<IO>::load(xb + (int64_t)t * D) : make_float4(0.f, 0.f, 0.f, 0.f);
        }
#pragma unroll
        for (int s = 0; s < kDwRun; ++s) {
            const int t = t0 + s;
            if (t >= L) break;
            float4 acc = bs;
#pragma unroll
            for (int k = 0; k < K; ++k) {
                const float4 xv = win[s + k];
                acc.x = fmaf(wk[k].x, xv.x, acc.x);
                acc.y = fmaf(wk[k].y, xv.y, acc.y);
                acc.z = fmaf(wk[k].z, xv.z, acc.z);
                acc.w = fmaf(wk[k].w, xv.w, acc.w);
            }
            DwVec<IO>::store(yb + (int64_t)t * D, acc);
        }
    }
}

// Scalar path (any D, any alignment): one channel per thread, same runs.
template <int K, typename IO>
__global__ void __launch_bounds__(kDwThreads) dwconv_scalar_kernel(const IO *__restrict__ x, const float *__restrict__ w,
                                                                   const float *__restrict__ bias, IO *__restrict__ y,
                                                                   int L, int D, int runs, int64_t nitems) {
    for (int64_t i = (int64_t)blockIdx.x * kDwThreads + threadIdx.x; i < nitems;
         i += (int64_t)gridDim.x * kDwThreads) {
        const int d = (int)(i % D);
        const int64_t rest = i / D;
        const int run = (int)(rest % runs);
        const int64_t b = rest / runs;
        const int t0 = run * kDwRun;
        float wk[K];
#pragma unroll
        for (int k = 0; k < K; ++k) wk[k] = __ldg(w + (int64_t)d * K + k);
        const float bs = bias ? __ldg(bias + d) : 0.f;
        const IO *xb = x + b * (int64_t)L * D + d;
        IO *yb = y + b * (int64_t)L * D + d;
        float win[K - 1 + kDwRun];
#pragma unroll
        for (int j = 0; j < K - 1 + kDwRun; ++j) {
            const int t = t0 - (K - 1) + j;
            win[j] = (t >= 0 && t < L) ? DwVec<IO>::load1(xb + (int64_t)t * D) : 0.f;
        }
#pragma unroll
        for (int s = 0; s < kDwRun; ++s) {
            const int t = t0 + s;
            if (t >= L) break;
            float acc = bs;
#pragma unroll
            for (int k = 0; k < K; ++k) acc = fmaf(wk[k], win[s + k], acc);
            DwVec<IO>::store1(yb + (int64_t)t * D, acc);
        }
    }
}

// CTAs of `kern` resident on the device at once (cached per device and kernel).
template <typename Kern>
static int64_t dw_resident_ctas(Kern kern, int dev, std::atomic<int> *cache) {
    int n = cache[dev].load(std::memory_order_relaxed);
    if (n == 0) {
        int per_sm = 0, sms = 0;
        if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, kDwThreads, 0) != cudaSuccess ||
            cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
            return -1;
        n = std::max(1, per_sm) * std::max(1, sms);
        cache[dev].store(n, std::memory_order_relaxed);
    }
    return n;
}

template <int K, typename IO>
static int launch_dwconv_k(const IO *x, const float *w, const float *bias, IO *y, int64_t B, int64_t L, int64_t D,
                           cudaStream_t s, int dev) {
    static std::atomic<int> resident_vec[128], resident_scalar[128];
    const int64_t runs = (L + kDwRun - 1) / kDwRun;
    const bool vec = D % 4 == 0 && (uintptr_t)x % (4 * sizeof(IO)) == 0 && (uintptr_t)y % (4 * sizeof(IO)) == 0;
    const int64_t nitems = B * runs * (vec ? D / 4 : D);
    const int64_t cap = vec ? dw_resident_ctas(dwconv_vec_kernel<K, IO>, dev, resident_vec)
                            : dw_resident_ctas(dwconv_scalar_kernel<K, IO>, dev, resident_scalar);
    if (cap < 0) return 5;  // CC_ERR_CUDA
    const int64_t blocks = std::max<int64_t>(1, std::min<int64_t>((nitems + kDwThreads - 1) / kDwThreads, cap));
    if (vec)
        dwconv_vec_kernel<K, IO><<<(unsigned)blocks, kDwThreads, 0, s>>>(x, w, bias, y, (int)L, (int)D, (int)runs,
                                                                          nitems);
    else
        dwconv_scalar_kernel<K, IO><<<(unsigned)blocks, kDwThreads, 0, s>>>(x, w, bias, y, (int)L, (int)D, (int)runs,
                                                                             nitems);
    return cudaGetLastError() == cudaSuccess ? 0 : 5;  // CC_OK / CC_ERR_CUDA
}

template <typename IO>
static int launch_dwconv(const IO *x, const float *w, const float *bias, IO *y, int64_t B, int64_t L, int64_t D,
                         int64_t K, cudaStream_t s, int dev) {
    switch (K) {
        case 1: return launch_dwconv_k<1, IO>(x, w, bias, y, B, L, D, s, dev);
        case 2: return launch_dwconv_k<2, IO>(x, w, bias, y, B, L, D, s, dev);
        case 3: return launch_dwconv_k<3, IO>(x, w, bias, y, B, L, D, s, dev);
        case 4: return launch_dwconv_k<4, IO>(x, w, bias, y, B, L, D, s, dev);
        case 5: return launch_dwconv_k<5, IO>(x, w, bias, y, B, L, D, s, dev);
        case 6: return launch_dwconv_k<6, IO>(x, w, bias, y, B, L, D, s, dev);
        case 7: return launch_dwconv_k<7, IO>(x, w, bias, y, B, L, D, s, dev);
        case 8: return launch_dwconv_k<8, IO>(x, w, bias, y, B, L, D, s, dev);
        default: return 2;  // CC_ERR_UNSUPPORTED
    }
}

}  // namespace ccv
