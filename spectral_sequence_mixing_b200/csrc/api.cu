// api.cu -- C ABI of the causal sequence convolution (see include/causalconv.h).
//
// Host side: argument checks, one-time per-device constant/twiddle setup,
// and dispatch to the sm_100a kernels.  The library allocates no device
// memory: its tables are static __device__ arrays filled on first use.
#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>
#include <math.h>
#include <stdint.h>
#include <string.h>

#include <algorithm>
#include <atomic>
#include <initializer_list>
#include <mutex>
#include <type_traits>
#include <vector>

#include "causalconv.h"
#include "fftconv_fused.cuh"
#include "bigconv.cuh"
#include "ntt.cuh"
#include "decode.cuh"
#include "hbmrows.cuh"
#include "mhf_gate.cuh"
#include "dwconv.cuh"
#include "tcconv.cuh"
#include "configs.cuh"

namespace ccv {

// ------------------------------------------------------------------ tables
// Twiddle tables per size class (configs.cuh; they depend only on the geometry).
__device__ float2 g_tw_s[CfgS<float>::TW_SIZE];
__device__ float2 g_tw_m[CfgM<float>::TW_SIZE];

__device__ float2 g_tw_bm[BigM<float>::TW_SIZE];
__device__ float2 g_tw_bl[BigL<float>::TW_SIZE];
__device__ float2 g_tw_bx[BigX<float>::TW_SIZE];
__device__ __align__(16) float2 g_tw_hr[kHrTwSize];

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
    // theta = omega_2N; see the table layout in FusedCfg
    constexpr int N = Cfg::N, N1 = Cfg::N1, N2 = Cfg::N2, M2 = Cfg::M2;
    const int64_t N2x = 2 * (int64_t)N;
    std::vector<float2> t(Cfg::TW_SIZE);
    for (int k1 = 0; k1 < N1; ++k1)
        for (int n2 = 0; n2 < N2; ++n2) t[k1 * N2 + n2] = omega((int64_t)n2 * (2 * k1 + 1), N2x);
    for (int k2 = 0; k2 < M2; ++k2)
        for (int k1 = 0; k1 < N1; ++k1)
            t[Cfg::TW_P + k2 * N1 + k1] = omega(-(2 * (int64_t)(k1 + N1 * k2) + 1), N2x);
    for (int m2 = 0; m2 < M2; ++m2)
        for (int k1 = 0; k1 < N1; ++k1) t[Cfg::TW_Q + m2 * N1 + k1] = omega(-2 * (int64_t)m2 * (2 * k1 + 1), N2x);
    return t;
}

template <class Cfg>
static std::vector<float2> big_twiddles() {
    // factor tables, see BigCfg
    constexpr int S = Cfg::S, SL = Cfg::SL, R0 = Cfg::R0, RA = Cfg::RA, RB = Cfg::RB, RC = Cfg::RC;
    constexpr int Q0 = Cfg::Q0, QA = Cfg::QA, STA = Cfg::STA;
    std::vector<float2> t(Cfg::TW_SIZE);
    const int64_t S2 = 2 * (int64_t)S;
    for (int k0 = 0; k0 < R0; ++k0) {
        for (int nl = 0; nl < Q0; ++nl) t[Cfg::T0A + k0 * Q0 + nl] = omega((int64_t)nl * (2 * k0 + 1), S2);
        for (int nh = 0; nh < SL / Q0; ++nh)
            t[Cfg::T0B + k0 * (SL / Q0) + nh] = omega((int64_t)Q0 * nh * (2 * k0 + 1), S2);
    }
    for (int k = 0; k < RA; ++k) {
        for (int ll = 0; ll < QA; ++ll) t[Cfg::TAA + k * QA + ll] = omega((int64_t)ll * k, SL);
        for (int lh = 0; lh < STA / QA; ++lh) t[Cfg::TAB + k * (STA / QA) + lh] = omega((int64_t)QA * lh * k, SL);
    }
    for (int k = 0; k < RB; ++k)
        for (int lo = 0; lo < RC; ++lo) t[Cfg::TB + k * RC + lo] = omega((int64_t)lo * k, RB * RC);
    if constexpr (Cfg::MIRROR) {
        // half-length real-output inverse, see BigCfg
        constexpr int RCH = Cfg::RCH, STAH = Cfg::STAH;
        for (int ka = 0; ka < RA; ++ka) t[Cfg::TPA + ka] = omega(ka, SL);
        for (int j = 0; j < STAH; ++j) t[Cfg::TPB + j] = omega(j, SL / RA);
        for (int k = 0; k < RB; ++k)
            for (int lo = 0; lo < RCH; ++lo) t[Cfg::TBH + k * RCH + lo] = omega((int64_t)lo * k, RB * RCH);
        for (int k = 0; k < RA; ++k) {
            for (int ll = 0; ll < QA; ++ll) t[Cfg::TAHA + k * QA + ll] = omega((int64_t)ll * k, SL / 2);
            for (int lh = 0; lh < STAH / QA; ++lh)
                t[Cfg::TAHB + k * (STAH / QA) + lh] = omega((int64_t)QA * lh * k, SL / 2);
        }
    }
    return t;
}

// Four-step long-row tables (hbmrows.cuh); theta = omega_2N, phi = theta^2.
static std::vector<float2> hr_twiddles() {
    std::vector<float2> t(kHrTwSize);
    const int64_t N2 = 2 * (int64_t)kHrN;
    for (int n2 = 0; n2 < 128; ++n2) t[kHrTW1 + n2] = omega(n2, 512);
    for (int a = 0; a < 16; ++a)
        for (int c = 0; c < 16; ++c) t[kHrTA + a * 16 + c] = omega(a * c, 256);
    for (int n1 = 0; n1 < kHrA; ++n1)
        for (int k2 = 0; k2 < kHrB; ++k2) t[kHrTO + n1 * kHrB + k2] = omega((int64_t)n1 * (2 * k2 + 1), N2);
    for (int p = 0; p < 16; ++p)
        for (int u = 0; u < 32; ++u) t[kHrT512 + p * 32 + u] = omega(p * u, 512);
    for (int k2 = 0; k2 < kHrB; ++k2) t[kHrPK1 + k2] = omega(-(2 * (int64_t)k2 + 1), N2);
    for (int u = 0; u < 32; ++u)
        for (int q = 0; q < 8; ++q) {
            t[kHrPK2 + u * 8 + q] = omega(-(512 * (int64_t)u + 16384 * (int64_t)q), N2);
            t[kHrTI + u * 8 + q] = omega(-(int64_t)u * q, 256);
        }
    for (int k2 = 0; k2 < kHrB; ++k2) {
        for (int al = 0; al < 8; ++al) t[kHrTWa + k2 * 8 + al] = omega(-2 * (int64_t)al * (2 * k2 + 1), N2);
        for (int be = 0; be < 32; ++be) t[kHrTWb + k2 * 32 + be] = omega(-16 * (int64_t)be * (2 * k2 + 1), N2);
    }
    for (int m2 = 0; m2 < 128; ++m2) t[kHrTU + m2] = omega(-m2, 512);
    return t;
}

// ---- tensor-core transform (tcconv.cuh): stage matrices and twiddle pairs
static uint16_t h_half(double x) { return __half_as_ushort(__float2half_rn((float)x)); }

// byte offset of fp16 element (row, k) in a K-major no-swizzle operand of 128 rows
static size_t tc_kmajor(int row, int k) { return (size_t)(k / 8) * kTcChunkPitch + (size_t)row * 16 + (size_t)(k % 8) * 2; }

static std::vector<uint16_t> tc_const_table() {
    // A1 (F1 / 4, rows = lanes (k1, re/im), K = 2 n1 + re/im), B2 (F64 / 8,
    // rows 2 q + re/im, K = 2 m + re/im), A4 (conj F1 / 4, real part only:
    // rows n1 < 32, K = 2 k1 + re/im), each in its shared-memory layout; then
    // the twiddle table F0[k1][m] = theta^(m (2 k1 + 1)) / 2, w[m] = omega_128^m
    // and c64[k1] = theta^(64 (2 k1 + 1)) as float2 (theta = omega_2N)
    std::vector<uint16_t> t(kTcConstBytes / 2, 0);
    auto put = [&](unsigned off, int row, int k, double x) { t[(off + tc_kmajor(row, k)) / 2] = h_half(x); };
    auto putf2 = [&](unsigned off, int i, double re, double im) {
        const float f[2] = {(float)re, (float)im};
        memcpy(&t[(off + 8u * (unsigned)i) / 2], f, 8);
    };
    const double pi = kTwoPi / 2;
    for (int l = 0; l < 128; ++l) {
        const int k1 = tc_kappa(l);
        for (int n1 = 0; n1 < 32; ++n1) {
            const double a = -pi * n1 * (2 * k1 + 1) / 64.0, fr = 0.25 * cos(a), fi = 0.25 * sin(a);
            if ((l & 1) == 0) {
                put(kTcOffA1, l, 2 * n1, fr);
                put(kTcOffA1, l, 2 * n1 + 1, -fi);
            } else {
                put(kTcOffA1, l, 2 * n1, fi);
                put(kTcOffA1, l, 2 * n1 + 1, fr);
            }
        }
    }
    for (int q = 0; q < 64; ++q)
        for (int m = 0; m < 64; ++m) {
            const double a = -kTwoPi * (double)((m * q) % 64) / 64.0, fr = 0.125 * cos(a), fi = 0.125 * sin(a);
            put(kTcOffB2, 2 * q, 2 * m, fr);
            put(kTcOffB2, 2 * q, 2 * m + 1, -fi);
            put(kTcOffB2, 2 * q + 1, 2 * m, fi);
            put(kTcOffB2, 2 * q + 1, 2 * m + 1, fr);
        }
    for (int n1 = 0; n1 < 32; ++n1)
        for (int k1 = 0; k1 < 64; ++k1) {
            const double a = pi * n1 * (2 * k1 + 1) / 64.0, gr = 0.25 * cos(a), gi = 0.25 * sin(a);
            put(kTcOffA4, n1, 2 * k1, gr);
            put(kTcOffA4, n1, 2 * k1 + 1, -gi);
        }
    const int64_t N2 = 2 * (int64_t)kTcN;  // theta = omega_2N
    auto ang = [&](int64_t e) { return -kTwoPi * (double)(e % N2) / (double)N2; };
    for (int k1 = 0; k1 < 64; ++k1) {
        for (int m = 0; m < 64; ++m) {
            const double a = ang((int64_t)m * (2 * k1 + 1));
            putf2(kTcOffTw, k1 * kTcTwPitch + m, 0.5 * cos(a), 0.5 * sin(a));
        }
        const double a = ang((int64_t)64 * (2 * k1 + 1));
        putf2(kTcOffW, 64 + k1, cos(a), sin(a));
    }
    for (int m = 0; m < 64; ++m) putf2(kTcOffW, m, cos(kTwoPi * m / 128.0), -sin(kTwoPi * m / 128.0));
    return t;
}

template <class Cfg, typename IO, int MINB>
static cudaError_t set_big_attr() {
    if constexpr (Cfg::CL == 1)
        return cudaFuncSetAttribute(bigrow_group_kernel<Cfg::R0, Cfg::RA, Cfg::RB, Cfg::RC, Cfg::T, MINB, IO>,
                                    cudaFuncAttributeMaxDynamicSharedMemorySize, (int)Cfg::SMEM_BYTES);
    else
        return cudaFuncSetAttribute(bigconv_kernel<Cfg::R0, Cfg::RA, Cfg::RB, Cfg::RC, Cfg::CL, Cfg::T, MINB, IO>,
                                    cudaFuncAttributeMaxDynamicSharedMemorySize, (int)Cfg::SMEM_BYTES);
}

static std::mutex g_init_mu;
static bool g_init_done[128];
// Context the per-device state was built in (0: none yet).
static unsigned long long g_init_ctx[128];

// Identifier of the calling thread's current CUDA context (cuCtxGetId through
// the runtime's driver entry points; 0 when there is none or it cannot be
// read).  Per-device state -- the tables' contents, kernel attributes, the
// no-allocation scratch address -- belongs to one context; a cudaDeviceReset
// destroys it, so the state is rebuilt when the identifier changes.
static unsigned long long current_ctx_id() {
    typedef CUresult (*CtxGetCurrent)(CUcontext *);
    typedef CUresult (*CtxGetId)(CUcontext, unsigned long long *);
    static CtxGetCurrent get_cur = nullptr;
    static CtxGetId get_id = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            get_cur = reinterpret_cast<CtxGetCurrent>(p);
        if (cudaGetDriverEntryPoint("cuCtxGetId", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            get_id = reinterpret_cast<CtxGetId>(p);
        cudaGetLastError();
    });
    CUcontext c = nullptr;
    unsigned long long id = 0;
    if (!get_cur || !get_id || get_cur(&c) != CUDA_SUCCESS || !c || get_id(c, &id) != CUDA_SUCCESS) return 0;
    return id;
}


// Per device: SM count and, per kernel instantiation, resident CTAs per SM.
static int g_num_sms[128];
// Per device: device addresses of the twiddle tables (fused N = 512, 2048; one-CTA
// rows N = 8192; cluster rows; one-CTA rows N = 4096; four-step long rows).
static void *g_tw_addr[128][6];

template <class Cfg, typename IO, int MINB>
static cudaError_t set_smem_attr() {
    const cudaError_t e = cudaFuncSetAttribute(fftconv_fused_kernel<Cfg::N2, Cfg::ROWS, MINB, IO, false>,
                                               cudaFuncAttributeMaxDynamicSharedMemorySize, (int)Cfg::SMEM_BYTES);
    if (e != cudaSuccess) return e;
    return cudaFuncSetAttribute(fftconv_fused_kernel<Cfg::N2, Cfg::ROWS, MINB, IO, true>,
                                cudaFuncAttributeMaxDynamicSharedMemorySize, (int)Cfg::SMEM_BYTES);
}

static cudaError_t ensure_init(int dev) {
    if (dev < 0 || dev >= 128) return cudaErrorInvalidDevice;
    std::lock_guard<std::mutex> lk(g_init_mu);
    if (g_init_done[dev] && g_init_ctx[dev] == current_ctx_id()) return cudaSuccess;
    g_init_done[dev] = false;
    cudaError_t e;
    float2 w128[128];
    for (int k = 0; k < 128; ++k) w128[k] = omega(k, 128);
    if ((e = cudaMemcpyToSymbol(c_w128, w128, sizeof(w128))) != cudaSuccess) return e;
    {
        float2 tw1[2][2][32];
        for (int sz = 0; sz < 2; ++sz) {
            const int n2s = sz ? 32 : 16, two_n1 = 4 * n2s;
            for (int ee = 0; ee < 2; ++ee)
                for (int n1 = 0; n1 < 32; ++n1) tw1[sz][ee][n1] = omega((int64_t)(2 * ee + 1) * n1, two_n1);
        }
        if ((e = cudaMemcpyToSymbol(c_f1_twist, tw1, sizeof(tw1))) != cudaSuccess) return e;
    }
    {
        auto t = fused_twiddles<CfgS<float>>();
        if ((e = cudaMemcpyToSymbol(g_tw_s, t.data(), t.size() * sizeof(float2))) != cudaSuccess) return e;
    }
    {
        auto t = fused_twiddles<CfgM<float>>();
        if ((e = cudaMemcpyToSymbol(g_tw_m, t.data(), t.size() * sizeof(float2))) != cudaSuccess) return e;
    }
    {
        auto t = big_twiddles<BigM<float>>();
        if ((e = cudaMemcpyToSymbol(g_tw_bm, t.data(), t.size() * sizeof(float2))) != cudaSuccess) return e;
    }
    {
        auto t = big_twiddles<BigL<float>>();
        if ((e = cudaMemcpyToSymbol(g_tw_bl, t.data(), t.size() * sizeof(float2))) != cudaSuccess) return e;
    }
    {
        auto t = big_twiddles<BigX<float>>();
        if ((e = cudaMemcpyToSymbol(g_tw_bx, t.data(), t.size() * sizeof(float2))) != cudaSuccess) return e;
    }
    {
        auto t = hr_twiddles();
        if ((e = cudaMemcpyToSymbol(g_tw_hr, t.data(), t.size() * sizeof(float2))) != cudaSuccess) return e;
        if ((e = cudaFuncSetAttribute(hr_fwd_kernel<float>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                      (int)kHrFwdSmem)) != cudaSuccess ||
            (e = cudaFuncSetAttribute(hr_fwd_kernel<__nv_bfloat16>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                      (int)kHrFwdSmem)) != cudaSuccess ||
            (e = cudaFuncSetAttribute(hr_inv_kernel<float>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                      (int)kHrFwdSmem)) != cudaSuccess ||
            (e = cudaFuncSetAttribute(hr_inv_kernel<__nv_bfloat16>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                      (int)kHrFwdSmem)) != cudaSuccess ||
            (e = cudaFuncSetAttribute(hr_fwd_tma_kernel<float, false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                      (int)hr_fwd_tma_smem<float>())) != cudaSuccess ||
            (e = cudaFuncSetAttribute(hr_fwd_tma_kernel<float, true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                      (int)hr_fwd_tma_smem<float>())) != cudaSuccess ||
            (e = cudaFuncSetAttribute(hr_fwd_tma_kernel<__nv_bfloat16, false>,
                                      cudaFuncAttributeMaxDynamicSharedMemorySize,
                                      (int)hr_fwd_tma_smem<__nv_bfloat16>())) != cudaSuccess ||
            (e = cudaFuncSetAttribute(hr_fwd_tma_kernel<__nv_bfloat16, true>,
                                      cudaFuncAttributeMaxDynamicSharedMemorySize,
                                      (int)hr_fwd_tma_smem<__nv_bfloat16>())) != cudaSuccess ||
            (e = cudaFuncSetAttribute(hr_mid_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                      (int)kHrMidSmem)) != cudaSuccess)
            return e;
    }
    if ((e = set_big_attr<BigM<float>, float, kMinbBigM>()) != cudaSuccess) return e;
    if ((e = set_big_attr<BigM<__nv_bfloat16>, __nv_bfloat16, kMinbBigM>()) != cudaSuccess) return e;
    if ((e = set_big_attr<BigL<float>, float, kMinbBigL>()) != cudaSuccess) return e;
    if ((e = set_big_attr<BigL<__nv_bfloat16>, __nv_bfloat16, kMinbBigL>()) != cudaSuccess) return e;
    if ((e = set_big_attr<BigX<float>, float, kMinbBigX>()) != cudaSuccess) return e;
    if ((e = set_big_attr<BigX<__nv_bfloat16>, __nv_bfloat16, kMinbBigX>()) != cudaSuccess) return e;
    if ((e = ntt_init_device()) != cudaSuccess) return e;
    {
        auto t = tc_const_table();
        if ((e = cudaMemcpyToSymbol(g_tc_consts, t.data(), t.size() * sizeof(uint16_t))) != cudaSuccess) return e;
        if ((e = cudaFuncSetAttribute(tcconv_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                      (int)kTcSmemBytes)) != cudaSuccess)
            return e;
    }
    if ((e = set_smem_attr<CfgS<float>, float, kMinbS>()) != cudaSuccess) return e;
    if ((e = set_smem_attr<CfgS<__nv_bfloat16>, __nv_bfloat16, kMinbS>()) != cudaSuccess) return e;
    if ((e = set_smem_attr<CfgM<float>, float, kMinbM>()) != cudaSuccess) return e;
    if ((e = set_smem_attr<CfgM<__nv_bfloat16>, __nv_bfloat16, kMinbM>()) != cudaSuccess) return e;
    if ((e = cudaDeviceGetAttribute(&g_num_sms[dev], cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess) return e;
    if ((e = cudaGetSymbolAddress(&g_tw_addr[dev][0], g_tw_s)) != cudaSuccess) return e;
    if ((e = cudaGetSymbolAddress(&g_tw_addr[dev][1], g_tw_m)) != cudaSuccess) return e;
    if ((e = cudaGetSymbolAddress(&g_tw_addr[dev][2], g_tw_bl)) != cudaSuccess) return e;
    if ((e = cudaGetSymbolAddress(&g_tw_addr[dev][3], g_tw_bx)) != cudaSuccess) return e;
    if ((e = cudaGetSymbolAddress(&g_tw_addr[dev][4], g_tw_bm)) != cudaSuccess) return e;
    if ((e = cudaGetSymbolAddress(&g_tw_addr[dev][5], g_tw_hr)) != cudaSuccess) return e;
    g_init_ctx[dev] = current_ctx_id();
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
        case CC_DTYPE_BF16: return BigX<float>::LMAX;
        case CC_DTYPE_I32: return kNttMaxL;
        default: return 0;
    }
}

static bool ranges_overlap(const void *a, size_t a_bytes, const void *b, size_t b_bytes) {
    const uintptr_t x = (uintptr_t)a, y = (uintptr_t)b;
    return x < y + b_bytes && y < x + a_bytes;
}
static bool ranges_overlap(const void *a, const void *b, size_t bytes) { return ranges_overlap(a, bytes, b, bytes); }

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

// Checks that need no CUDA call: null pointers, sizes, aliasing, workspace.
static int check_host(int dtype, const void *v, const void *g, const void *r, int64_t B, int64_t L, int64_t D,
                      size_t ws_bytes) {
    if (!v || !g || !r) return CC_ERR_INVALID_ARG;
    size_t bytes = 0;
    int st = check_shape(dtype, B, L, D, &bytes);
    if (st != CC_OK) return st;
    if (ranges_overlap(r, v, bytes) || ranges_overlap(r, g, bytes)) return CC_ERR_ALIAS;
    if (ws_bytes < causal_conv_workspace_bytes(dtype, B, L, D)) return CC_ERR_WORKSPACE;
    return CC_OK;
}

// Every pointer is device memory of the current device (cudaPointerGetAttributes).
static int check_device(std::initializer_list<const void *> ptrs, int *dev_out) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) {
        cudaGetLastError();
        return CC_ERR_CUDA;
    }
    for (const void *p : ptrs) {
        const int st = check_device_ptr(p, dev);
        if (st != CC_OK) return st;
    }
    *dev_out = dev;
    return CC_OK;
}

static int check_common(int dtype, const void *v, const void *g, const void *r, int64_t B, int64_t L, int64_t D,
                        size_t ws_bytes, int *dev_out) {
    const int st = check_host(dtype, v, g, r, B, L, D, ws_bytes);
    if (st != CC_OK) return st;
    return check_device({v, g, r}, dev_out);
}

// ------------------------------------------------------------------ tensor maps
// cuTensorMapEncodeTiled from the driver, looked up once (no link against libcuda).
static PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
        cudaGetLastError();
    });
    return fn;
}

// 3-D map over a channel-last [B, L, D] tensor (dims innermost first: D, L, B)
// with boxes of [box_t][box_d]; elements outside the tensor read as zero.
// False when the layout cannot be described (strides or base not 16-byte aligned).
template <typename IO>
static bool encode_btd_map(CUtensorMap *m, const IO *base, int64_t B, int64_t L, int64_t D, int box_d, int box_t) {
    const size_t es = sizeof(IO);
    if (((uintptr_t)base & 15) != 0 || (D * (int64_t)es) % 16 != 0) return false;
    if (D > (int64_t)UINT32_MAX || L > (int64_t)UINT32_MAX || B > (int64_t)UINT32_MAX) return false;
    if ((int64_t)es * D * L >= ((int64_t)1 << 40)) return false;
    auto enc = tensor_map_encoder();
    if (!enc) return false;
    const cuuint64_t dims[3] = {(cuuint64_t)D, (cuuint64_t)L, (cuuint64_t)B};
    const cuuint64_t strides[2] = {(cuuint64_t)(D * es), (cuuint64_t)(D * L * es)};
    const cuuint32_t box[3] = {(cuuint32_t)box_d, (cuuint32_t)box_t, 1};
    const cuuint32_t estr[3] = {1, 1, 1};
    const CUtensorMapDataType dt = sizeof(IO) == 4 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
    return enc(m, dt, 3, const_cast<IO *>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
               CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_128B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// 4-D map {d, n1, n2, b} of a [B, L, D] tensor for the four-step forward
// pass: time t = n1 + 512 n2 for the whole 512-step rows n2 < L / 512; box
// [128 n2][1 n1][16 d].  False when the layout allows no map.
template <typename IO>
static bool encode_hr_map(CUtensorMap *m, const IO *base, int64_t B, int64_t L, int64_t D) {
    const int64_t es = sizeof(IO), nb2 = L / kHrA;
    if (((uintptr_t)base & 15) != 0 || (D * es) % 16 != 0 || nb2 < 1) return false;
    if (D > (int64_t)UINT32_MAX || B > (int64_t)UINT32_MAX || es * D * L >= ((int64_t)1 << 40)) return false;
    auto enc = tensor_map_encoder();
    if (!enc) return false;
    const cuuint64_t dims[4] = {(cuuint64_t)D, (cuuint64_t)kHrA, (cuuint64_t)nb2, (cuuint64_t)B};
    const cuuint64_t strides[3] = {(cuuint64_t)(D * es), (cuuint64_t)(kHrA * D * es), (cuuint64_t)(L * D * es)};
    const cuuint32_t box[4] = {(cuuint32_t)kHrFwdCG, 1, 128, 1};
    const cuuint32_t estr[4] = {1, 1, 1, 1};
    const CUtensorMapDataType dt = sizeof(IO) == 4 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
    return enc(m, dt, 4, const_cast<IO *>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
               CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_128B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// ------------------------------------------------------------------ launch
template <class Cfg, int MINB, typename IO>
static int launch_fused(const IO *v, const IO *g, IO *r, int64_t B, int64_t L, int64_t D, const float2 *tw,
                        cudaStream_t s, int dev, int rev) {
    const int64_t groups = (D + Cfg::ROWS - 1) / Cfg::ROWS;
    const int64_t tiles = B * groups;
    if (tiles > INT32_MAX) return CC_ERR_UNSUPPORTED;
    // v read reversed in time (backward pass): the kernel instance that reverses on its shared-memory reads
    auto kern = (rev & 1) ? fftconv_fused_kernel<Cfg::N2, Cfg::ROWS, MINB, IO, true>
                          : fftconv_fused_kernel<Cfg::N2, Cfg::ROWS, MINB, IO, false>;
    // resident CTAs per SM, queried once per device and kernel instance
    static std::atomic<int> resident[2][128];
    int per_sm = resident[rev & 1][dev].load(std::memory_order_relaxed);
    if (per_sm == 0) {
        if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, Cfg::THREADS, Cfg::SMEM_BYTES) !=
                cudaSuccess ||
            per_sm < 1) {
            cudaGetLastError();
            return CC_ERR_CUDA;
        }
        resident[rev & 1][dev].store(per_sm, std::memory_order_relaxed);
    }
    const int64_t grid = std::min<int64_t>(tiles, (int64_t)per_sm * g_num_sms[dev]);
    // whole-chunk async copies need full, aligned channel groups
    const bool vec = (D % Cfg::ROWS) == 0 && ((uintptr_t)v % Cfg::CHUNK) == 0 && ((uintptr_t)g % Cfg::CHUNK) == 0;
    // TMA boxes when a tile row is whole 16-byte units
    CUtensorMap tmv, tmg;
    memset(&tmv, 0, sizeof(tmv));
    memset(&tmg, 0, sizeof(tmg));
    const bool tma = Cfg::TMA_OK &&
                     encode_btd_map<IO>(&tmv, v, B, L, D, Cfg::SW, Cfg::BOXT) &&
                     encode_btd_map<IO>(&tmg, g, B, L, D, Cfg::SW, Cfg::BOXT);
    kern<<<(unsigned)grid, Cfg::THREADS, Cfg::SMEM_BYTES, s>>>(v, g, r, (int)L, (int)D, (int)groups, (int)tiles,
                                                              vec ? 1 : 0, rev, tw, tmv, tmg, tma ? 1 : 0);
    return cudaGetLastError() == cudaSuccess ? CC_OK : CC_ERR_CUDA;
}

template <class Cfg, int MINB, typename IO>
static int launch_big(const IO *v, const IO *g, IO *r, int64_t B, int64_t L, int64_t D, const float2 *tw,
                      cudaStream_t s, int rev, int row_major) {
    const int64_t rows = B * D;
    if (rows * Cfg::CL > INT32_MAX) return CC_ERR_UNSUPPORTED;
    auto kern = bigconv_kernel<Cfg::R0, Cfg::RA, Cfg::RB, Cfg::RC, Cfg::CL, Cfg::T, MINB, IO>;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)(rows * Cfg::CL));
    cfg.blockDim = dim3(Cfg::T);
    cfg.dynamicSmemBytes = Cfg::SMEM_BYTES;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = Cfg::CL;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    const cudaError_t e = cudaLaunchKernelEx(&cfg, kern, v, g, r, (int)L, (int)D, rev, row_major, tw);
    if (e != cudaSuccess) {
        cudaGetLastError();
        return CC_ERR_CUDA;
    }
    return CC_OK;
}

// Workspace that enables the four-step path of rows longer than one CTA
// holds (hbmrows.cuh: the partial transforms of every row, norm partials and
// per-row scales); 0 when that path does not apply.
static size_t fast_ws_bytes(int dtype, int64_t B, int64_t L, int64_t D) {
    if (dtype != CC_DTYPE_F32 && dtype != CC_DTYPE_BF16) return 0;
    if (B < 1 || D < 1 || L <= BigL<float>::LMAX || L > BigX<float>::LMAX) return 0;
    if (D > INT32_MAX / B) return 0;  // rows and channel tiles are int
    return hr_ws_bytes(B * D);
}

// A workspace large enough for the four-step path is used by it: it must be
// device memory of the current device and overlap none of the tensors.
static int check_fast_ws(int dtype, int64_t B, int64_t L, int64_t D, const void *ws, size_t ws_bytes,
                         std::initializer_list<const void *> tensors) {
    const size_t fast = fast_ws_bytes(dtype, B, L, D);
    if (!ws || fast == 0 || ws_bytes < fast) return CC_OK;
    const size_t bytes = (size_t)(B * L * D) * dtype_size(dtype);
    for (const void *t : tensors)
        if (ranges_overlap(ws, fast, t, bytes)) return CC_ERR_ALIAS;
    int dev;
    return check_device({ws}, &dev);
}

// Rows that fit one CTA, kGroup adjacent channels per cluster.
template <class Cfg, int MINB, typename IO>
static int launch_group(const IO *v, const IO *g, IO *r, int64_t B, int64_t L, int64_t D, const float2 *tw,
                        cudaStream_t s, int rev) {
    static_assert(Cfg::CL == 1, "one row per CTA");
    const int64_t gpb = (D + kGroup - 1) / kGroup;
    if (B * gpb * kGroup > INT32_MAX) return CC_ERR_UNSUPPORTED;
    auto kern = bigrow_group_kernel<Cfg::R0, Cfg::RA, Cfg::RB, Cfg::RC, Cfg::T, MINB, IO>;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)(B * gpb * kGroup));
    cfg.blockDim = dim3(Cfg::T);
    cfg.dynamicSmemBytes = Cfg::SMEM_BYTES;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = kGroup;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    // 16-byte group accesses: every (b, t) row of D elements and the bases 16-byte aligned
    const bool vec = (D * (int64_t)sizeof(IO)) % 16 == 0 && ((uintptr_t)v % 16) == 0 && ((uintptr_t)g % 16) == 0 &&
                     ((uintptr_t)r % 16) == 0;
    const cudaError_t e =
        cudaLaunchKernelEx(&cfg, kern, v, g, r, (int)L, (int)D, (int)gpb, rev, vec ? 1 : 0, tw);
    if (e != cudaSuccess) {
        cudaGetLastError();
        return CC_ERR_CUDA;
    }
    return CC_OK;
}

// bf16 rows with 2048 < L <= 4096 on the tensor cores: clusters of 4 CTAs
// (8 adjacent channels, two per CTA), persistent over the channel groups.
static int launch_tcconv(const __nv_bfloat16 *v, const __nv_bfloat16 *g, __nv_bfloat16 *r, int64_t B, int64_t L,
                         int64_t D, cudaStream_t s, int dev, int rev) {
    const int64_t gpb = (D + kTcGroup - 1) / kTcGroup;
    const int64_t groups = B * gpb;
    if (groups > INT32_MAX / kTcCluster) return CC_ERR_UNSUPPORTED;
    static std::atomic<int> max_clusters[128];
    int mc = max_clusters[dev].load(std::memory_order_relaxed);
    if (mc == 0) {
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3(kTcCluster * 64);
        cfg.blockDim = dim3(kTcThreads);
        cfg.dynamicSmemBytes = kTcSmemBytes;
        if (cudaOccupancyMaxActiveClusters(&mc, tcconv_kernel, &cfg) != cudaSuccess || mc < 1) {
            cudaGetLastError();
            return CC_ERR_CUDA;
        }
        max_clusters[dev].store(mc, std::memory_order_relaxed);
    }
    const int64_t clusters = std::min<int64_t>(groups, mc);
    const bool vec = (D * 2) % 16 == 0 && ((uintptr_t)v % 16) == 0 && ((uintptr_t)g % 16) == 0 &&
                     ((uintptr_t)r % 16) == 0;
    // inputs staged by TMA boxes [256 t][8 d] when the layout allows a tensor map
    CUtensorMap tmv, tmg;
    memset(&tmv, 0, sizeof(tmv));
    memset(&tmg, 0, sizeof(tmg));
    const bool tma = encode_btd_map<__nv_bfloat16>(&tmv, v, B, L, D, kTcGroup, kTcBoxT) &&
                     encode_btd_map<__nv_bfloat16>(&tmg, g, B, L, D, kTcGroup, kTcBoxT);
    tcconv_kernel<<<(unsigned)(clusters * kTcCluster), kTcThreads, kTcSmemBytes, s>>>(
        v, g, r, (int)L, (int)D, (int)gpb, (int)groups, rev, vec ? 1 : 0, tmv, tmg, tma ? 1 : 0);
    return cudaGetLastError() == cudaSuccess ? CC_OK : CC_ERR_CUDA;
}

// Four-step long rows through the workspace (hbmrows.cuh): norms, alpha,
// forward over n2, the middle pass (forward over n1, product, packing, inner
// inverse) in place, inverse over k2 with the stores.
template <typename IO>
static int launch_hbm_rows(const IO *v, const IO *g, IO *r, int64_t B, int64_t L, int64_t D, void *ws,
                           const float2 *tw, cudaStream_t s, int dev, int rev) {
    const int64_t rows = B * D, tpb = (D + kHrCG - 1) / kHrCG, tiles = B * tpb;
    float2 *Y = reinterpret_cast<float2 *>(ws);
    float2 *part = reinterpret_cast<float2 *>(reinterpret_cast<char *>(ws) + hr_ws_part_off(rows));
    float2 *as = reinterpret_cast<float2 *>(reinterpret_cast<char *>(ws) + hr_ws_as_off(rows));
    constexpr uintptr_t vb = 4 * sizeof(IO);  // bytes of four channels
    if (D % 4 == 0 && (reinterpret_cast<uintptr_t>(v) % vb) == 0 && (reinterpret_cast<uintptr_t>(g) % vb) == 0) {
        const int64_t tpb4 = (D + 127) / 128;
        hr_norms4_kernel<IO><<<dim3((unsigned)(B * tpb4), kHrSlices), 256, 0, s>>>(v, g, part, (int)L, (int)D,
                                                                                  (int)rows, (int)tpb4);
    } else {
        hr_norms_kernel<IO><<<dim3((unsigned)tiles, kHrSlices), kHrNormThreads, 0, s>>>(v, g, part, (int)L, (int)D,
                                                                                         (int)rows, (int)tpb);
    }
    hr_alpha_kernel<<<(unsigned)((rows + 255) / 256), 256, 0, s>>>(part, as, (int)rows);
    // inputs staged by TMA where a map describes the tensors (v read reversed
    // in time for the backward pass)
    CUtensorMap tmv, tmg;
    memset(&tmv, 0, sizeof(tmv));
    memset(&tmg, 0, sizeof(tmg));
    const int64_t tpb16 = (D + kHrFwdCG - 1) / kHrFwdCG, tiles16 = B * tpb16, items = tiles16 * kHrA;
    // (item indices of the persistent loop stay below INT32_MAX, lookahead included)
    if (items <= INT32_MAX - 8 * (int64_t)g_num_sms[dev] && encode_hr_map<IO>(&tmv, v, B, L, D) &&
        encode_hr_map<IO>(&tmg, g, B, L, D)) {
        const int64_t grid = std::min<int64_t>(items, 2 * (int64_t)g_num_sms[dev]);
        auto kern = (rev & 1) ? hr_fwd_tma_kernel<IO, true> : hr_fwd_tma_kernel<IO, false>;
        kern<<<(unsigned)grid, kHrFwdTmaThreads, hr_fwd_tma_smem<IO>(), s>>>(
            v, g, Y, as, tw, (int)L, (int)D, (int)rows, (int)tpb16, (int)tiles16, (int)items, tmv, tmg);
    } else {
        hr_fwd_kernel<IO><<<dim3((unsigned)tiles, kHrA), kHrFwdThreads, kHrFwdSmem, s>>>(v, g, Y, as, tw, (int)L,
                                                                                          (int)D, (int)rows,
                                                                                          (int)tpb, rev);
    }
    hr_mid_kernel<<<dim3((unsigned)((rows + kHrRows2 - 1) / kHrRows2), kHrB / 2), kHrMidThreads, kHrMidSmem, s>>>(
        Y, tw, (int)rows);
    hr_inv_kernel<IO><<<dim3((unsigned)tiles, kHrB), kHrInvThreads, kHrFwdSmem, s>>>(Y, r, as, v, g, tw, (int)L,
                                                                                      (int)D, (int)rows, (int)tpb, rev);
    return cudaGetLastError() == cudaSuccess ? CC_OK : CC_ERR_CUDA;
}

template <typename IO>
static int fftconv_dispatch(const IO *v, const IO *g, IO *r, int64_t B, int64_t L, int64_t D, void *ws,
                            size_t ws_bytes, cudaStream_t s, int dev, int rev = 0) {
    void *const *tws = g_tw_addr[dev];  // filled by ensure_init
    if (L <= CfgS<IO>::LMAX)
        return launch_fused<CfgS<IO>, kMinbS>(v, g, r, B, L, D, (const float2 *)tws[0], s, dev, rev);
    if (L <= CfgM<IO>::LMAX)
        return launch_fused<CfgM<IO>, kMinbM>(v, g, r, B, L, D, (const float2 *)tws[1], s, dev, rev);
    if (L <= BigM<IO>::LMAX)
        return launch_group<BigM<IO>, kMinbBigM>(v, g, r, B, L, D, (const float2 *)tws[4], s, rev);
    if (L <= BigL<IO>::LMAX) {
        if constexpr (sizeof(IO) == 2)
            return launch_tcconv((const __nv_bfloat16 *)v, (const __nv_bfloat16 *)g, (__nv_bfloat16 *)r, B, L, D, s,
                                 dev, rev);
        return launch_group<BigL<IO>, kMinbBigL>(v, g, r, B, L, D, (const float2 *)tws[2], s, rev);
    }
    if (L <= BigX<IO>::LMAX) {
        // rows of 8-CTA clusters read straight from the tensors, or the
        // four-step path through a workspace that holds it
        const size_t fast = fast_ws_bytes(sizeof(IO) == 4 ? CC_DTYPE_F32 : CC_DTYPE_BF16, B, L, D);
        if (ws == nullptr || fast == 0 || ws_bytes < fast || (reinterpret_cast<uintptr_t>(ws) & 15) != 0)
            return launch_big<BigX<IO>, kMinbBigX>(v, g, r, B, L, D, (const float2 *)tws[3], s, rev, 0);
        return launch_hbm_rows<IO>(v, g, r, B, L, D, ws, (const float2 *)tws[5], s, dev, rev);
    }
    return CC_ERR_UNSUPPORTED;
}

// A library-owned stream per device for work that may run beside the
// caller's stream, with the events that fork it from and join it back to
// that stream.
struct SidePipe {
    cudaStream_t s2 = nullptr;
    cudaEvent_t fork = nullptr, join = nullptr;
    std::mutex mu;
};

static SidePipe *side_pipe(int dev) {
    static SidePipe pipes[128];
    static std::once_flag once[128];
    static bool ok[128];
    std::call_once(once[dev], [dev] {
        SidePipe &p = pipes[dev];
        ok[dev] = cudaStreamCreateWithFlags(&p.s2, cudaStreamNonBlocking) == cudaSuccess &&
                  cudaEventCreateWithFlags(&p.fork, cudaEventDisableTiming) == cudaSuccess &&
                  cudaEventCreateWithFlags(&p.join, cudaEventDisableTiming) == cudaSuccess;
        cudaGetLastError();
    });
    return ok[dev] ? &pipes[dev] : nullptr;
}

// Backward: dv = rev(conv(rev(dr), g)), dg = rev(conv(rev(dr), v)).
template <typename IO>
static int fftconv_bwd(const IO *dr, const IO *v, const IO *g, IO *dv, IO *dg, int64_t B, int64_t L, int64_t D,
                       void *ws, size_t ws_bytes, cudaStream_t s, int dev) {
    // Rows of the fused kernel (no workspace involved): dg goes on a library
    // stream forked from the caller's, so its CTAs take the SMs that dv's last,
    // partial wave leaves idle; the caller's stream then waits for both.
    SidePipe *sp = L <= CfgM<IO>::LMAX ? side_pipe(dev) : nullptr;
    if (sp) {
        std::lock_guard<std::mutex> lk(sp->mu);
        if (cudaEventRecord(sp->fork, s) != cudaSuccess || cudaStreamWaitEvent(sp->s2, sp->fork, 0) != cudaSuccess) {
            cudaGetLastError();
            return CC_ERR_CUDA;
        }
        const int st1 = fftconv_dispatch<IO>(dr, g, dv, B, L, D, ws, ws_bytes, s, dev, 3);
        const int st2 = fftconv_dispatch<IO>(dr, v, dg, B, L, D, ws, ws_bytes, sp->s2, dev, 3);
        // join whatever was enqueued, also after an error
        if (cudaEventRecord(sp->join, sp->s2) != cudaSuccess || cudaStreamWaitEvent(s, sp->join, 0) != cudaSuccess) {
            cudaGetLastError();
            return CC_ERR_CUDA;
        }
        return st1 != CC_OK ? st1 : st2;
    }
    int st = fftconv_dispatch<IO>(dr, g, dv, B, L, D, ws, ws_bytes, s, dev, 3);
    if (st != CC_OK) return st;
    return fftconv_dispatch<IO>(dr, v, dg, B, L, D, ws, ws_bytes, s, dev, 3);
}

static int check_bwd(int dtype, const void *dr, const void *v, const void *g, const void *dv, const void *dg,
                     int64_t B, int64_t L, int64_t D, size_t ws_bytes, int *dev) {
    if (!dv || !dg) return CC_ERR_INVALID_ARG;
    int st = check_host(dtype, dr, g, dv, B, L, D, ws_bytes);
    if (st != CC_OK) return st;
    if ((st = check_host(dtype, dr, v, dg, B, L, D, ws_bytes)) != CC_OK) return st;
    const size_t bytes = (size_t)(B * L * D) * dtype_size(dtype);
    if (ranges_overlap(dv, dg, bytes) || ranges_overlap(dv, v, bytes) || ranges_overlap(dg, g, bytes)) return CC_ERR_ALIAS;
    return check_device({dr, v, g, dv, dg}, dev);
}

// ---------------------------------------------------------------- decode
static int check_decode(int dtype, const void *v, const void *g, const void *r, int64_t B, int64_t Lcap, int64_t D,
                        int64_t t, const void *ws, size_t ws_bytes) {
    const size_t es = dtype_size(dtype);
    if (es == 0 || !v || !g || !r) return CC_ERR_INVALID_ARG;
    if (B < 1 || Lcap < 1 || D < 1 || t < 0 || t >= Lcap) return CC_ERR_INVALID_ARG;
    if (B > 65535 || Lcap > INT32_MAX || D > INT32_MAX) return CC_ERR_INVALID_ARG;
    const int64_t lim = INT64_MAX / (int64_t)es;
    if (Lcap > lim / D || B > lim / (Lcap * D)) return CC_ERR_INVALID_ARG;
    if (dtype == CC_DTYPE_I32) return CC_ERR_UNSUPPORTED;
    const size_t cache_bytes = (size_t)(B * Lcap * D) * es, out_bytes = (size_t)(B * D) * es;
    if (ranges_overlap(r, out_bytes, v, cache_bytes) || ranges_overlap(r, out_bytes, g, cache_bytes))
        return CC_ERR_ALIAS;
    const size_t need = (size_t)decode_splits(B, D, t) * (size_t)(B * D) * sizeof(double);
    if (!ws || ws_bytes < need) return CC_ERR_WORKSPACE;
    return CC_OK;
}

template <typename IO>
static int decode_entry(int dtype, const IO *v, const IO *g, IO *r, int64_t B, int64_t Lcap, int64_t D, int64_t t,
                        void *workspace, size_t workspace_bytes, void *stream) {
    int st = check_decode(dtype, v, g, r, B, Lcap, D, t, workspace, workspace_bytes);
    if (st != CC_OK) return st;
    int dev;
    if ((st = check_device({v, g, r, workspace}, &dev)) != CC_OK) return st;
    return decode_launch<IO>(v, g, r, B, Lcap, D, t, (double *)workspace, (cudaStream_t)stream);
}

// ------------------------------------------------- decode without allocation
// Fixed scratch for causal_conv_decode_f32_noalloc: the fp64 partial sums of
// the split reduction live here instead of in a caller workspace.  Every GPU
// that loads this library holds these 8 MiB until the process exits.
constexpr size_t kNoAllocScratchBytes = (size_t)8 << 20;
static __device__ __align__(256) double g_noalloc_scratch[kNoAllocScratchBytes / sizeof(double)];

// Device address of g_noalloc_scratch per device.  In host code the symbol
// only names a host-side stand-in, so the address is looked up with the
// device current on first use and cached together with the context it
// belongs to (looked up again if a device reset replaced that context).
static std::mutex g_noalloc_mu;
static double *g_noalloc_ptr[128];
static unsigned long long g_noalloc_ctx[128];

static int noalloc_scratch(int dev, double **out) {
    if (dev < 0 || dev >= 128) return CC_ERR_CUDA;
    std::lock_guard<std::mutex> lk(g_noalloc_mu);
    const unsigned long long ctx = current_ctx_id();
    if (!g_noalloc_ptr[dev] || ctx == 0 || g_noalloc_ctx[dev] != ctx) {
        void *p = nullptr;
        if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || !p) {
            cudaGetLastError();
            return CC_ERR_CUDA;
        }
        g_noalloc_ptr[dev] = (double *)p;
        g_noalloc_ctx[dev] = ctx;
    }
    *out = g_noalloc_ptr[dev];
    return CC_OK;
}

}  // namespace ccv

using namespace ccv;

// ------------------------------------------------------------------ host buffers
constexpr int64_t kHostChunks = 4;

// Per device: the two streams and events of the pipelined host-buffer path.
struct HostPipe {
    cudaStream_t up = nullptr, down = nullptr;
    cudaEvent_t start = nullptr, handoff = nullptr, done = nullptr;
    std::mutex mu;
};

static HostPipe *host_pipe(int dev) {
    static HostPipe pipes[128];
    static std::once_flag once[128];
    static bool ok[128];
    std::call_once(once[dev], [dev] {
        HostPipe &p = pipes[dev];
        ok[dev] = cudaStreamCreateWithFlags(&p.up, cudaStreamNonBlocking) == cudaSuccess &&
                  cudaStreamCreateWithFlags(&p.down, cudaStreamNonBlocking) == cudaSuccess &&
                  cudaEventCreateWithFlags(&p.start, cudaEventDisableTiming) == cudaSuccess &&
                  cudaEventCreateWithFlags(&p.handoff, cudaEventDisableTiming) == cudaSuccess &&
                  cudaEventCreateWithFlags(&p.done, cudaEventDisableTiming) == cudaSuccess;
        cudaGetLastError();
    });
    return ok[dev] ? &pipes[dev] : nullptr;
}

// Batches [b0, b0 + nb) of a host-buffer call: upload v, g on `up`, transform
// on `up`, download r on `down` after `up` (through `handoff` when the streams differ).
static int from_host_chunk(int dtype, const void *v_host, const void *g_host, void *r_host, void *v_dev, void *g_dev,
                           void *r_dev, int64_t b0, int64_t nb, int64_t L, int64_t D, void *ws, size_t ws_bytes,
                           cudaStream_t up, cudaStream_t down, cudaEvent_t handoff = nullptr) {
    const size_t es = dtype_size(dtype);
    const size_t off = (size_t)(b0 * L * D) * es, bytes = (size_t)(nb * L * D) * es;
    const char *hv = (const char *)v_host + off, *hg = (const char *)g_host + off;
    char *hr = (char *)r_host + off, *dv = (char *)v_dev + off, *dg = (char *)g_dev + off, *dr = (char *)r_dev + off;
    if (cudaMemcpyAsync(dv, hv, bytes, cudaMemcpyHostToDevice, up) != cudaSuccess ||
        cudaMemcpyAsync(dg, hg, bytes, cudaMemcpyHostToDevice, up) != cudaSuccess) {
        cudaGetLastError();
        return CC_ERR_CUDA;
    }
    int st;
    switch (dtype) {
        case CC_DTYPE_F32:
            st = causal_fftconv_f32((const float *)dv, (const float *)dg, (float *)dr, nb, L, D, ws, ws_bytes, up);
            break;
        case CC_DTYPE_BF16:
            st = causal_fftconv_bf16((const uint16_t *)dv, (const uint16_t *)dg, (uint16_t *)dr, nb, L, D, ws, ws_bytes,
                                     up);
            break;
        default:
            st = causal_ntt_conv_i32((const int32_t *)dv, (const int32_t *)dg, (int32_t *)dr, nb, L, D, ws, ws_bytes,
                                     up);
            break;
    }
    if (st != CC_OK) return st;
    if (up != down && (cudaEventRecord(handoff, up) != cudaSuccess || cudaStreamWaitEvent(down, handoff, 0) != cudaSuccess)) {
        cudaGetLastError();
        return CC_ERR_CUDA;
    }
    if (cudaMemcpyAsync(hr, dr, bytes, cudaMemcpyDeviceToHost, down) != cudaSuccess) {
        cudaGetLastError();
        return CC_ERR_CUDA;
    }
    return CC_OK;
}

// ------------------------------------------------------------------ MHF gate
template <int C, int KT, typename IO>
static int launch_gate_ck(const IO *a, const float *w, const float *bias, IO *g, int64_t B, int64_t L, int64_t D,
                          int64_t H, cudaStream_t s, int dev) {
    using Cfg = GateCfg<C, KT>;
    // the attribute belongs to the context it was set in (see current_ctx_id)
    static std::atomic<unsigned long long> attr_ctx[128];
    const unsigned long long ctx = current_ctx_id();
    if (ctx == 0 || attr_ctx[dev].load(std::memory_order_acquire) != ctx) {
        if (cudaFuncSetAttribute(mhf_gate_kernel<C, KT, IO>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 (int)Cfg::SMEM_BYTES) != cudaSuccess)
            return CC_ERR_CUDA;
        attr_ctx[dev].store(ctx, std::memory_order_release);
    }
    const int64_t per_row = (L + kGateM - 1) / kGateM;
    const int64_t tiles = B * per_row;  // tiles of one head
    if (tiles > INT32_MAX || H > INT32_MAX / 2) return CC_ERR_UNSUPPORTED;
    // persistent CTAs: as many as fit on the SMs at once, split evenly over the heads
    static std::atomic<int> resident[128];
    int cps = resident[dev].load(std::memory_order_relaxed);
    if (cps == 0) {
        if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&cps, mhf_gate_kernel<C, KT, IO>, kGateThreads,
                                                          Cfg::SMEM_BYTES) != cudaSuccess)
            return CC_ERR_CUDA;
        cps = std::max(1, cps);
        resident[dev].store(cps, std::memory_order_relaxed);
    }
    const int64_t groups = std::max<int64_t>(1, std::min<int64_t>(tiles, (int64_t)g_num_sms[dev] * cps / H));
    const int64_t grid = H * groups;
    if (grid > INT32_MAX) return CC_ERR_UNSUPPORTED;
    const int vec_in = ((uintptr_t)a % (sizeof(IO) == 4 ? 16 : 8)) == 0;
    const int vec_out = ((uintptr_t)g % 16) == 0;
    // fp32 input tiles [ROWS t][C ch] staged by TMA when the layout allows a tensor map
    CUtensorMap tma_a;
    memset(&tma_a, 0, sizeof(tma_a));
    const bool tma = sizeof(IO) == 4 && encode_btd_map<IO>(&tma_a, a, B, L, D, C, Cfg::ROWS);
    mhf_gate_kernel<C, KT, IO><<<(unsigned)grid, kGateThreads, Cfg::SMEM_BYTES, s>>>(
        a, w, bias, g, (int)L, (int)D, (int)H, (int)groups, (int)per_row, (int)tiles, vec_in, vec_out, tma_a,
        tma ? 1 : 0);
    return cudaGetLastError() == cudaSuccess ? CC_OK : CC_ERR_CUDA;
}

template <int C, typename IO>
static int launch_gate_c(const IO *a, const float *w, const float *bias, IO *g, int64_t B, int64_t L, int64_t D,
                         int64_t H, int64_t K, cudaStream_t s, int dev) {
    switch (K) {
        case 1: return launch_gate_ck<C, 1, IO>(a, w, bias, g, B, L, D, H, s, dev);
        case 2: return launch_gate_ck<C, 2, IO>(a, w, bias, g, B, L, D, H, s, dev);
        case 3: return launch_gate_ck<C, 3, IO>(a, w, bias, g, B, L, D, H, s, dev);
        case 4: return launch_gate_ck<C, 4, IO>(a, w, bias, g, B, L, D, H, s, dev);
        default: return CC_ERR_UNSUPPORTED;
    }
}

template <typename IO>
static int launch_gate(const IO *a, const float *w, const float *bias, IO *g, int64_t B, int64_t L, int64_t D,
                       int64_t H, int64_t K, cudaStream_t s, int dev) {
    switch (D / H) {
        case 16: return launch_gate_c<16, IO>(a, w, bias, g, B, L, D, H, K, s, dev);
        case 32: return launch_gate_c<32, IO>(a, w, bias, g, B, L, D, H, K, s, dev);
        case 64: return launch_gate_c<64, IO>(a, w, bias, g, B, L, D, H, K, s, dev);
        default: return CC_ERR_UNSUPPORTED;
    }
}

// Shapes, head width, taps and aliasing of a gate call (no CUDA call).
static int check_gate_host(int dtype, const void *a, const float *w, const float *bias, const void *g, int64_t B,
                           int64_t L, int64_t D, int64_t H, int64_t K, size_t *bytes) {
    if (dtype != CC_DTYPE_F32 && dtype != CC_DTYPE_BF16) return CC_ERR_INVALID_ARG;
    if (!a || !w || !g) return CC_ERR_INVALID_ARG;
    int st = check_shape(dtype, B, L, D, bytes);
    if (st != CC_OK) return st;
    if (H < 1 || K < 1 || D % H != 0) return CC_ERR_INVALID_ARG;
    const int64_t C = D / H;
    if ((C != 16 && C != 32 && C != 64) || K > kGateMaxTaps) return CC_ERR_UNSUPPORTED;
    const size_t wb = (size_t)D * (size_t)C * (size_t)K * sizeof(float);
    if (ranges_overlap(g, *bytes, a, *bytes) || ranges_overlap(g, *bytes, w, wb) ||
        (bias && ranges_overlap(g, *bytes, bias, (size_t)D * sizeof(float))))
        return CC_ERR_ALIAS;
    return CC_OK;
}

template <typename IO>
static int gate_entry(int dtype, const IO *a, const float *w, const float *bias, IO *g, int64_t B, int64_t L,
                      int64_t D, int64_t H, int64_t K, cudaStream_t s) {
    size_t bytes = 0;
    int st = check_gate_host(dtype, a, w, bias, g, B, L, D, H, K, &bytes);
    if (st != CC_OK) return st;
    int dev;
    if ((st = check_device({a, w, g}, &dev)) != CC_OK) return st;
    if (bias && (st = check_device_ptr(bias, dev)) != CC_OK) return st;
    if (ensure_init(dev) != cudaSuccess) return CC_ERR_CUDA;
    return launch_gate<IO>(a, w, bias, g, B, L, D, H, K, s, dev);
}

template <typename IO>
static int gated_conv_entry(int dtype, const IO *v, const IO *a, const float *w, const float *bias, IO *r, int64_t B,
                            int64_t L, int64_t D, int64_t H, int64_t K, void *ws, size_t ws_bytes, cudaStream_t s) {
    if (!v || !r || !ws) return CC_ERR_INVALID_ARG;
    size_t bytes = 0;
    int st = check_gate_host(dtype, a, w, bias, ws, B, L, D, H, K, &bytes);
    if (st != CC_OK) return st;
    if (ws_bytes < bytes) return CC_ERR_WORKSPACE;
    const int64_t C = D / H;
    const size_t wb = (size_t)D * (size_t)C * (size_t)K * sizeof(float);
    if (ranges_overlap(r, bytes, v, bytes) || ranges_overlap(r, bytes, a, bytes) || ranges_overlap(r, bytes, w, wb) ||
        ranges_overlap(r, bytes, ws, bytes) || ranges_overlap(ws, bytes, v, bytes) ||
        (bias && ranges_overlap(r, bytes, bias, (size_t)D * sizeof(float))))
        return CC_ERR_ALIAS;
    int dev;
    if ((st = check_device({v, a, w, r, ws}, &dev)) != CC_OK) return st;
    if (bias && (st = check_device_ptr(bias, dev)) != CC_OK) return st;
    if (ensure_init(dev) != cudaSuccess) return CC_ERR_CUDA;
    IO *gbuf = reinterpret_cast<IO *>(ws);
    if ((st = launch_gate<IO>(a, w, bias, gbuf, B, L, D, H, K, s, dev)) != CC_OK) return st;
    return fftconv_dispatch<IO>(v, gbuf, r, B, L, D, nullptr, 0, s, dev);
}

// ------------------------------------------------------------------ depthwise conv
template <typename IO>
static int dwconv_entry(int dtype, const IO *x, const float *w, const float *bias, IO *y, int64_t B, int64_t L,
                        int64_t D, int64_t K, cudaStream_t s) {
    if (!x || !w || !y) return CC_ERR_INVALID_ARG;
    const size_t es = dtype_size(dtype);
    if (B < 1 || L < 1 || D < 1 || K < 1) return CC_ERR_INVALID_ARG;
    if (L > INT32_MAX || D > INT32_MAX || B > INT32_MAX) return CC_ERR_INVALID_ARG;
    const int64_t lim = INT64_MAX / (int64_t)es;
    if (L > lim / D || B > lim / (L * D)) return CC_ERR_INVALID_ARG;
    if (K > kDwMaxTaps) return CC_ERR_UNSUPPORTED;
    const size_t bytes = (size_t)(B * L * D) * es;
    if (ranges_overlap(y, bytes, x, bytes) || ranges_overlap(y, bytes, w, (size_t)(D * K) * sizeof(float)) ||
        (bias && ranges_overlap(y, bytes, bias, (size_t)D * sizeof(float))))
        return CC_ERR_ALIAS;
    int dev, st;
    if ((st = check_device({x, w, y}, &dev)) != CC_OK) return st;
    if (bias && (st = check_device_ptr(bias, dev)) != CC_OK) return st;
    return launch_dwconv<IO>(x, w, bias, y, B, L, D, K, s, dev);
}

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
        case CC_ERR_SCRATCH_LIMIT: return "problem needs more scratch than the fixed 8 MiB buffer of the no-allocation entry point";
        default: return "unknown status";
    }
}

int causal_fftconv_f32(const float *v, const float *g, float *r, int64_t B, int64_t L, int64_t D, void *workspace,
                       size_t workspace_bytes, void *stream) {
    int dev;
    int st = check_common(CC_DTYPE_F32, v, g, r, B, L, D, workspace_bytes, &dev);
    if (st != CC_OK) return st;
    if ((st = check_fast_ws(CC_DTYPE_F32, B, L, D, workspace, workspace_bytes, {v, g, r})) != CC_OK) return st;
    if (ensure_init(dev) != cudaSuccess) return CC_ERR_CUDA;
    return fftconv_dispatch<float>(v, g, r, B, L, D, workspace, workspace_bytes, (cudaStream_t)stream, dev);
}

int causal_fftconv_bf16(const uint16_t *v, const uint16_t *g, uint16_t *r, int64_t B, int64_t L, int64_t D,
                        void *workspace, size_t workspace_bytes, void *stream) {
    int dev;
    int st = check_common(CC_DTYPE_BF16, v, g, r, B, L, D, workspace_bytes, &dev);
    if (st != CC_OK) return st;
    if ((st = check_fast_ws(CC_DTYPE_BF16, B, L, D, workspace, workspace_bytes, {v, g, r})) != CC_OK) return st;
    if (ensure_init(dev) != cudaSuccess) return CC_ERR_CUDA;
    return fftconv_dispatch<__nv_bfloat16>((const __nv_bfloat16 *)v, (const __nv_bfloat16 *)g, (__nv_bfloat16 *)r, B,
                                           L, D, workspace, workspace_bytes, (cudaStream_t)stream, dev);
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

int causal_fftconv_bwd_f32(const float *dr, const float *v, const float *g, float *dv, float *dg, int64_t B,
                           int64_t L, int64_t D, void *workspace, size_t workspace_bytes, void *stream) {
    int dev;
    int st = check_bwd(CC_DTYPE_F32, dr, v, g, dv, dg, B, L, D, workspace_bytes, &dev);
    if (st != CC_OK) return st;
    if ((st = check_fast_ws(CC_DTYPE_F32, B, L, D, workspace, workspace_bytes, {dr, v, g, dv, dg})) != CC_OK)
        return st;
    if (ensure_init(dev) != cudaSuccess) return CC_ERR_CUDA;
    return fftconv_bwd<float>(dr, v, g, dv, dg, B, L, D, workspace, workspace_bytes, (cudaStream_t)stream, dev);
}

int causal_fftconv_bwd_bf16(const uint16_t *dr, const uint16_t *v, const uint16_t *g, uint16_t *dv, uint16_t *dg,
                            int64_t B, int64_t L, int64_t D, void *workspace, size_t workspace_bytes, void *stream) {
    int dev;
    int st = check_bwd(CC_DTYPE_BF16, dr, v, g, dv, dg, B, L, D, workspace_bytes, &dev);
    if (st != CC_OK) return st;
    if ((st = check_fast_ws(CC_DTYPE_BF16, B, L, D, workspace, workspace_bytes, {dr, v, g, dv, dg})) != CC_OK)
        return st;
    if (ensure_init(dev) != cudaSuccess) return CC_ERR_CUDA;
    typedef __nv_bfloat16 bf;
    return fftconv_bwd<bf>((const bf *)dr, (const bf *)v, (const bf *)g, (bf *)dv, (bf *)dg, B, L, D, workspace,
                           workspace_bytes, (cudaStream_t)stream, dev);
}

size_t causal_conv_fast_workspace_bytes(int dtype, int64_t B, int64_t L, int64_t D) {
    return fast_ws_bytes(dtype, B, L, D);
}

size_t causal_conv_decode_workspace_bytes(int dtype, int64_t B, int64_t D, int64_t t) {
    if (dtype_size(dtype) == 0 || B < 1 || D < 1 || t < 0 || B > 65535 || D > INT32_MAX || t >= INT32_MAX)
        return (size_t)-1;
    return (size_t)decode_splits(B, D, t) * (size_t)(B * D) * sizeof(double);
}

int causal_conv_decode_f32(const float *v, const float *g, float *r, int64_t B, int64_t Lcap, int64_t D, int64_t t,
                           void *workspace, size_t workspace_bytes, void *stream) {
    return decode_entry<float>(CC_DTYPE_F32, v, g, r, B, Lcap, D, t, workspace, workspace_bytes, stream);
}

int causal_conv_decode_bf16(const uint16_t *v, const uint16_t *g, uint16_t *r, int64_t B, int64_t Lcap, int64_t D,
                            int64_t t, void *workspace, size_t workspace_bytes, void *stream) {
    typedef __nv_bfloat16 bf;
    return decode_entry<bf>(CC_DTYPE_BF16, (const bf *)v, (const bf *)g, (bf *)r, B, Lcap, D, t, workspace,
                            workspace_bytes, stream);
}

int causal_conv_decode_f32_noalloc(const float *v, const float *g, float *r, int64_t B, int64_t Lcap, int64_t D,
                                   int64_t t, void *stream) {
    // Same checks as causal_conv_decode_f32 with the library's own scratch
    // standing in for the workspace; a problem whose partial sums exceed the
    // fixed scratch is refused before anything is enqueued.
    if (!v || !g || !r) return CC_ERR_INVALID_ARG;
    if (B < 1 || D < 1 || t < 0 || B > 65535 || D > INT32_MAX || t >= INT32_MAX) return CC_ERR_INVALID_ARG;
    const size_t need = (size_t)decode_splits(B, D, t) * (size_t)(B * D) * sizeof(double);
    if (need > kNoAllocScratchBytes) return CC_ERR_SCRATCH_LIMIT;
    // the fixed scratch stands in for the workspace argument (non-null, large enough)
    int st = check_decode(CC_DTYPE_F32, v, g, r, B, Lcap, D, t, &need, kNoAllocScratchBytes);
    if (st != CC_OK) return st;
    int dev;
    if ((st = check_device({v, g, r}, &dev)) != CC_OK) return st;
    double *scratch = nullptr;
    if ((st = noalloc_scratch(dev, &scratch)) != CC_OK) return st;
    return decode_launch<float>(v, g, r, B, Lcap, D, t, scratch, (cudaStream_t)stream);
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
    if (ensure_init(dev) != cudaSuccess) return CC_ERR_CUDA;
    cudaStream_t s = (cudaStream_t)stream;
    const int64_t chunks = std::min<int64_t>(B, kHostChunks);
    HostPipe *pipe = chunks > 1 ? host_pipe(dev) : nullptr;
    if (!pipe) return from_host_chunk(dtype, v_host, g_host, r_host, v_dev, g_dev, r_dev, 0, B, L, D, workspace,
                                      workspace_bytes, s, s);
    // batches in kHostChunks pieces: the upload and transform of piece c+1 (stream
    // up) overlap the download of piece c (stream down); the caller's stream
    // waits for the last download
    std::lock_guard<std::mutex> lk(pipe->mu);
    if (cudaEventRecord(pipe->start, s) != cudaSuccess || cudaStreamWaitEvent(pipe->up, pipe->start, 0) != cudaSuccess ||
        cudaStreamWaitEvent(pipe->down, pipe->start, 0) != cudaSuccess) {
        cudaGetLastError();
        return CC_ERR_CUDA;
    }
    for (int64_t c = 0; c < chunks; ++c) {
        const int64_t b0 = c * B / chunks, b1 = (c + 1) * B / chunks;
        st = from_host_chunk(dtype, v_host, g_host, r_host, v_dev, g_dev, r_dev, b0, b1 - b0, L, D, workspace,
                             workspace_bytes, pipe->up, pipe->down, pipe->handoff);
        if (st != CC_OK) return st;
    }
    if (cudaEventRecord(pipe->done, pipe->down) != cudaSuccess || cudaStreamWaitEvent(s, pipe->done, 0) != cudaSuccess) {
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

int causal_mhf_gate_f32(const float *a, const float *w, const float *bias, float *g, int64_t B, int64_t L,
                        int64_t D, int64_t H, int64_t K, void *stream) {
    return gate_entry<float>(CC_DTYPE_F32, a, w, bias, g, B, L, D, H, K, (cudaStream_t)stream);
}

int causal_mhf_gate_bf16(const uint16_t *a, const float *w, const float *bias, uint16_t *g, int64_t B, int64_t L,
                         int64_t D, int64_t H, int64_t K, void *stream) {
    return gate_entry<__nv_bfloat16>(CC_DTYPE_BF16, (const __nv_bfloat16 *)a, w, bias, (__nv_bfloat16 *)g, B, L, D, H,
                                     K, (cudaStream_t)stream);
}

size_t causal_mhf_gated_conv_workspace_bytes(int dtype, int64_t B, int64_t L, int64_t D) {
    size_t bytes = 0;
    if ((dtype != CC_DTYPE_F32 && dtype != CC_DTYPE_BF16) || check_shape(dtype, B, L, D, &bytes) != CC_OK)
        return (size_t)-1;
    return bytes;
}

int causal_mhf_gated_conv_f32(const float *v, const float *a, const float *w, const float *bias, float *r, int64_t B,
                              int64_t L, int64_t D, int64_t H, int64_t K, void *workspace, size_t workspace_bytes,
                              void *stream) {
    return gated_conv_entry<float>(CC_DTYPE_F32, v, a, w, bias, r, B, L, D, H, K, workspace, workspace_bytes,
                                   (cudaStream_t)stream);
}

int causal_mhf_gated_conv_bf16(const uint16_t *v, const uint16_t *a, const float *w, const float *bias, uint16_t *r,
                               int64_t B, int64_t L, int64_t D, int64_t H, int64_t K, void *workspace,
                               size_t workspace_bytes, void *stream) {
    return gated_conv_entry<__nv_bfloat16>(CC_DTYPE_BF16, (const __nv_bfloat16 *)v, (const __nv_bfloat16 *)a, w, bias,
                                           (__nv_bfloat16 *)r, B, L, D, H, K, workspace, workspace_bytes,
                                           (cudaStream_t)stream);
}

int causal_dwconv_f32(const float *x, const float *w, const float *bias, float *y, int64_t B, int64_t L, int64_t D,
                      int64_t K, void *stream) {
    return dwconv_entry<float>(CC_DTYPE_F32, x, w, bias, y, B, L, D, K, (cudaStream_t)stream);
}

int causal_dwconv_bf16(const uint16_t *x, const float *w, const float *bias, uint16_t *y, int64_t B, int64_t L,
                       int64_t D, int64_t K, void *stream) {
    return dwconv_entry<__nv_bfloat16>(CC_DTYPE_BF16, (const __nv_bfloat16 *)x, w, bias, (__nv_bfloat16 *)y, B, L, D,
                                       K, (cudaStream_t)stream);
}

int causal_conv_fault_flags(int device, unsigned int *flags, int clear) {
    if (!flags) return CC_ERR_INVALID_ARG;
    int n = 0;
    if (cudaGetDeviceCount(&n) != cudaSuccess || device < 0 || device >= n) {
        cudaGetLastError();
        return CC_ERR_INVALID_ARG;
    }
    int prev = 0;
    if (cudaGetDevice(&prev) != cudaSuccess || cudaSetDevice(device) != cudaSuccess) {
        cudaGetLastError();
        return CC_ERR_CUDA;
    }
    cudaError_t e = cudaDeviceSynchronize();
    if (e == cudaSuccess) e = cudaMemcpyFromSymbol(flags, g_cc_fault, sizeof(unsigned int));
    if (e == cudaSuccess && clear) {
        const unsigned int zero = 0;
        e = cudaMemcpyToSymbol(g_cc_fault, &zero, sizeof(zero));
    }
    cudaSetDevice(prev);
    if (e != cudaSuccess) {
        cudaGetLastError();
        return CC_ERR_CUDA;
    }
    return CC_OK;
}

}  // extern "C"
