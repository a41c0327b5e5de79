// api.cu -- C ABI of the causal sequence convolution (see include/causalconv.h).
//
// Host side: argument checks, one-time per-device constant/twiddle setup,
// and dispatch to the sm_100a kernels.  The library allocates no device
// memory: its tables are static __device__ arrays filled on first use.
#include <cuda_runtime.h>
#include <math.h>
#include <stdint.h>
#include <string.h>

#include <mutex>
#include <vector>

#include "causalconv.h"
#include "fftconv_fused.cuh"
#include "ntt.cuh"

namespace ccv {

// ------------------------------------------------------------------ tables
using CfgS = FusedCfg<16, 8>;  // N = 512,  L <= 256
using CfgM = FusedCfg<32, 4>;  // N = 2048, L <= 1024

__device__ float2 g_tw_s[CfgS::TW_SIZE];
__device__ float2 g_tw_m[CfgM::TW_SIZE];

static double kTwoPi = 6.283185307179586476925286766559;

// omega_n^e = exp(-2 pi i e / n), evaluated in double after exact reduction of e.
static float2 omega(int64_t e, int64_t n) {
    e %= n;
    if (e < 0) e += n;
    const double a = kTwoPi * (double)e / (double)n;
    return make_float2((float)cos(a), (float)-sin(a));
}

template <class Cfg>
static std::vector<float2> fused_twiddles() {
    constexpr int N = Cfg::N, N1 = Cfg::N1, N2 = Cfg::N2, M2 = Cfg::M2, M = N / 2;
    std::vector<float2> t(Cfg::TW_SIZE);
    for (int k1 = 0; k1 < N1; ++k1)
        for (int n2 = 0; n2 < N2; ++n2) t[k1 * N2 + n2] = omega((int64_t)n2 * k1, N);
    for (int k2 = 0; k2 < M2; ++k2)
        for (int k1 = 0; k1 < N1; ++k1) t[Cfg::TW_P + k2 * N1 + k1] = omega(-(int64_t)(k1 + N1 * k2), N);
    for (int m2 = 0; m2 < M2; ++m2)
        for (int k1 = 0; k1 < N1; ++k1) t[Cfg::TW_Q + m2 * N1 + k1] = omega(-(int64_t)k1 * m2, M);
    return t;
}

static std::mutex g_init_mu;
static bool g_init_done[128];

template <class Cfg, typename IO, int MINB>
static cudaError_t set_smem_attr() {
    return cudaFuncSetAttribute(fftconv_fused_kernel<Cfg::N2, Cfg::ROWS, MINB, IO>,
                                cudaFuncAttributeMaxDynamicSharedMemorySize, (int)Cfg::SMEM_BYTES);
}

constexpr int kMinbS = 3;
constexpr int kMinbM = 3;

static cudaError_t ensure_init(int dev) {
    if (dev < 0 || dev >= 128) return cudaErrorInvalidDevice;
    std::lock_guard<std::mutex> lk(g_init_mu);
    if (g_init_done[dev]) return cudaSuccess;
    cudaError_t e;
    float2 w64[64];
    for (int k = 0; k < 64; ++k) w64[k] = omega(k, 64);
    if ((e = cudaMemcpyToSymbol(c_w64, w64, sizeof(w64))) != cudaSuccess) return e;
    {
        auto t = fused_twiddles<CfgS>();
        if ((e = cudaMemcpyToSymbol(g_tw_s, t.data(), t.size() * sizeof(float2))) != cudaSuccess) return e;
    }
    {
        auto t = fused_twiddles<CfgM>();
        if ((e = cudaMemcpyToSymbol(g_tw_m, t.data(), t.size() * sizeof(float2))) != cudaSuccess) return e;
    }
    if ((e = ntt_init_device()) != cudaSuccess) return e;
    if ((e = set_smem_attr<CfgS, float, kMinbS>()) != cudaSuccess) return e;
    if ((e = set_smem_attr<CfgS, __nv_bfloat16, kMinbS>()) != cudaSuccess) return e;
    if ((e = set_smem_attr<CfgM, float, kMinbM>()) != cudaSuccess) return e;
    if ((e = set_smem_attr<CfgM, __nv_bfloat16, kMinbM>()) != cudaSuccess) return e;
    g_init_done[dev] = true;
    return cudaSuccess;
}

// ------------------------------------------------------------------ checks
static size_t dtype_size(int dtype) {
    switch (dtype) {
        case CC_DTYPE_F32: return 4;
        case CC_DTYPE_BF16: return 2;
        case CC_DTYPE_I32: return 4;
        default: return 0;
    }
}

static int64_t max_len(int dtype) {
    switch (dtype) {
        case CC_DTYPE_F32:
        case CC_DTYPE_BF16: return 1024;
        case CC_DTYPE_I32: return kNttMaxL;
        default: return 0;
    }
}

static bool ranges_overlap(const void *a, const void *b, size_t bytes) {
    const uintptr_t x = (uintptr_t)a, y = (uintptr_t)b;
    return x < y + bytes && y < x + bytes;
}

static int check_shape(int dtype, int64_t B, int64_t L, int64_t D, size_t *bytes) {
    const size_t es = dtype_size(dtype);
    if (es == 0) return CC_ERR_INVALID_ARG;
    if (B < 1 || L < 1 || D < 1) return CC_ERR_INVALID_ARG;
    if (L > INT32_MAX || D > INT32_MAX || B > INT32_MAX) return CC_ERR_INVALID_ARG;
    // B*L*D*es must fit in int64 / size_t
    const int64_t lim = INT64_MAX / (int64_t)es;
    if (L > lim / D || B > lim / (L * D)) return CC_ERR_INVALID_ARG;
    if (L > max_len(dtype)) return CC_ERR_UNSUPPORTED;
    *bytes = (size_t)(B * L * D) * es;
    return CC_OK;
}

static int check_device_ptr(const void *p, int dev) {
    cudaPointerAttributes a;
    if (cudaPointerGetAttributes(&a, p) != cudaSuccess) {
        cudaGetLastError();
        return CC_ERR_NOT_DEVICE;
    }
    if (a.type == cudaMemoryTypeManaged) return CC_OK;
    if (a.type != cudaMemoryTypeDevice || a.device != dev) return CC_ERR_NOT_DEVICE;
    return CC_OK;
}

static int check_common(int dtype, const void *v, const void *g, const void *r, int64_t B, int64_t L, int64_t D,
                        size_t ws_bytes, int *dev_out) {
    if (!v || !g || !r) return CC_ERR_INVALID_ARG;
    size_t bytes = 0;
    int st = check_shape(dtype, B, L, D, &bytes);
    if (st != CC_OK) return st;
    if (ranges_overlap(r, v, bytes) || ranges_overlap(r, g, bytes)) return CC_ERR_ALIAS;
    if (ws_bytes < causal_conv_workspace_bytes(dtype, B, L, D)) return CC_ERR_WORKSPACE;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) {
        cudaGetLastError();
        return CC_ERR_CUDA;
    }
    if ((st = check_device_ptr(v, dev)) != CC_OK) return st;
    if ((st = check_device_ptr(g, dev)) != CC_OK) return st;
    if ((st = check_device_ptr(r, dev)) != CC_OK) return st;
    *dev_out = dev;
    return CC_OK;
}

// ------------------------------------------------------------------ launch
template <class Cfg, int MINB, typename IO>
static int launch_fused(const IO *v, const IO *g, IO *r, int64_t B, int64_t L, int64_t D, const float2 *tw,
                        cudaStream_t s) {
    const int64_t groups = (D + Cfg::ROWS - 1) / Cfg::ROWS;
    const int64_t blocks = B * groups;
    if (blocks > INT32_MAX) return CC_ERR_UNSUPPORTED;
    fftconv_fused_kernel<Cfg::N2, Cfg::ROWS, MINB, IO>
        <<<(unsigned)blocks, Cfg::THREADS, Cfg::SMEM_BYTES, s>>>(v, g, r, (int)L, (int)D, (int)groups, tw);
    return cudaGetLastError() == cudaSuccess ? CC_OK : CC_ERR_CUDA;
}

template <typename IO>
static int fftconv_dispatch(const IO *v, const IO *g, IO *r, int64_t B, int64_t L, int64_t D, cudaStream_t s) {
    void *tw = nullptr;
    if (L <= CfgS::N / 2) {
        if (cudaGetSymbolAddress(&tw, g_tw_s) != cudaSuccess) return CC_ERR_CUDA;
        return launch_fused<CfgS, kMinbS>(v, g, r, B, L, D, (const float2 *)tw, s);
    }
    if (L <= CfgM::N / 2) {
        if (cudaGetSymbolAddress(&tw, g_tw_m) != cudaSuccess) return CC_ERR_CUDA;
        return launch_fused<CfgM, kMinbM>(v, g, r, B, L, D, (const float2 *)tw, s);
    }
    return CC_ERR_UNSUPPORTED;
}

}  // namespace ccv

using namespace ccv;

extern "C" {

size_t causal_conv_workspace_bytes(int dtype, int64_t B, int64_t L, int64_t D) {
    size_t bytes;
    const int st = check_shape(dtype, B, L, D, &bytes);
    if (st == CC_ERR_INVALID_ARG) return (size_t)-1;
    return 0;
}

int64_t causal_conv_max_len(int dtype) { return max_len(dtype); }

const char *causal_conv_strerror(int status) {
    switch (status) {
        case CC_OK: return "success";
        case CC_ERR_INVALID_ARG: return "invalid argument (null pointer, non-positive or overflowing size, bad dtype)";
        case CC_ERR_UNSUPPORTED: return "sequence length beyond the supported range for this dtype";
        case CC_ERR_ALIAS: return "output overlaps an input";
        case CC_ERR_WORKSPACE: return "workspace smaller than causal_conv_workspace_bytes()";
        case CC_ERR_CUDA: return "CUDA runtime error or kernel launch failure";
        case CC_ERR_NOT_DEVICE: return "pointer is not device memory of the current device";
        default: return "unknown status";
    }
}

int causal_fftconv_f32(const float *v, const float *g, float *r, int64_t B, int64_t L, int64_t D, void *workspace,
                       size_t workspace_bytes, void *stream) {
    (void)workspace;
    int dev;
    int st = check_common(CC_DTYPE_F32, v, g, r, B, L, D, workspace_bytes, &dev);
    if (st != CC_OK) return st;
    if (ensure_init(dev) != cudaSuccess) return CC_ERR_CUDA;
    return fftconv_dispatch<float>(v, g, r, B, L, D, (cudaStream_t)stream);
}

int causal_fftconv_bf16(const uint16_t *v, const uint16_t *g, uint16_t *r, int64_t B, int64_t L, int64_t D,
                        void *workspace, size_t workspace_bytes, void *stream) {
    (void)workspace;
    int dev;
    int st = check_common(CC_DTYPE_BF16, v, g, r, B, L, D, workspace_bytes, &dev);
    if (st != CC_OK) return st;
    if (ensure_init(dev) != cudaSuccess) return CC_ERR_CUDA;
    return fftconv_dispatch<__nv_bfloat16>((const __nv_bfloat16 *)v, (const __nv_bfloat16 *)g, (__nv_bfloat16 *)r, B,
                                           L, D, (cudaStream_t)stream);
}

int causal_ntt_conv_i32(const int32_t *v, const int32_t *g, int32_t *r, int64_t B, int64_t L, int64_t D,
                        void *workspace, size_t workspace_bytes, void *stream) {
    (void)workspace;
    int dev;
    int st = check_common(CC_DTYPE_I32, v, g, r, B, L, D, workspace_bytes, &dev);
    if (st != CC_OK) return st;
    if (ensure_init(dev) != cudaSuccess) return CC_ERR_CUDA;
    return ntt_dispatch(v, g, r, B, L, D, (cudaStream_t)stream);
}

int causal_conv_from_host(int dtype, const void *v_host, const void *g_host, void *r_host, void *v_dev, void *g_dev,
                          void *r_dev, int64_t B, int64_t L, int64_t D, void *workspace, size_t workspace_bytes,
                          void *stream) {
    if (!v_host || !g_host || !r_host) return CC_ERR_INVALID_ARG;
    int dev;
    int st = check_common(dtype, v_dev, g_dev, r_dev, B, L, D, workspace_bytes, &dev);
    if (st != CC_OK) return st;
    const size_t bytes = (size_t)(B * L * D) * dtype_size(dtype);
    if (ranges_overlap(v_dev, g_dev, bytes)) return CC_ERR_ALIAS;
    cudaStream_t s = (cudaStream_t)stream;
    if (cudaMemcpyAsync(v_dev, v_host, bytes, cudaMemcpyHostToDevice, s) != cudaSuccess ||
        cudaMemcpyAsync(g_dev, g_host, bytes, cudaMemcpyHostToDevice, s) != cudaSuccess) {
        cudaGetLastError();
        return CC_ERR_CUDA;
    }
    switch (dtype) {
        case CC_DTYPE_F32:
            st = causal_fftconv_f32((const float *)v_dev, (const float *)g_dev, (float *)r_dev, B, L, D, workspace,
                                    workspace_bytes, stream);
            break;
        case CC_DTYPE_BF16:
            st = causal_fftconv_bf16((const uint16_t *)v_dev, (const uint16_t *)g_dev, (uint16_t *)r_dev, B, L, D,
                                     workspace, workspace_bytes, stream);
            break;
        default:
            st = causal_ntt_conv_i32((const int32_t *)v_dev, (const int32_t *)g_dev, (int32_t *)r_dev, B, L, D,
                                     workspace, workspace_bytes, stream);
            break;
    }
    if (st != CC_OK) return st;
    if (cudaMemcpyAsync(r_host, r_dev, bytes, cudaMemcpyDeviceToHost, s) != cudaSuccess) {
        cudaGetLastError();
        return CC_ERR_CUDA;
    }
    return CC_OK;
}

int causal_ntt_params(int64_t N, uint32_t out[6]) {
    if (!out) return CC_ERR_INVALID_ARG;
    NttParams p;
    if (!ntt_params_host(N, &p)) return CC_ERR_INVALID_ARG;
    out[0] = p.p;
    out[1] = p.w;
    out[2] = p.winv;
    out[3] = p.ninv;
    out[4] = p.pinv;
    out[5] = p.r2;
    return CC_OK;
}

}  // extern "C"
