// ntt.cuh -- exact causal convolution by a number-theoretic transform mod
// p = 2013265921 = 15 * 2^27 + 1 (primitive root 31).
//
// "Catastrophic Token Leakage in Convolutional Sequence Modeling and How to
// Mitigate It" (TL;DR and abstract) replaces the float FFT by a transform over
// the integers mod a prime, which has no rounding and so cannot leak future
// tokens.  Here each (b, d) row is zero-padded to N = 16384, transformed
// (v and g separately: Z_p has no conjugation to pack two real rows into
// one), multiplied pointwise, inverse-transformed, scaled by N^-1 and lifted
// to the centered residue; only t < L is computed and stored.
//
// Arithmetic: residues in [0, p).  Twiddle products use Shoup's method with
// a precomputed companion w' = floor(w 2^32 / p) (one mul.hi, two mul.lo);
// the data-by-data product uses Montgomery reduction with R = 2^32.
//
// Layout: one CTA per row, both transforms resident in shared memory (two
// arrays of N words, one pad word per 32 so every pass is conflict-free).
// The CTAs of a cluster take kNttGroup adjacent channels of one batch: CTA q
// reads time steps [q LMAX/kNttGroup, (q+1) LMAX/kNttGroup) of all of them
// with one 16-byte access per time step and array, and writes each
// channel's residues into the owning CTA's arrays (distributed shared
// memory), at the slots the first pass reads; the last pass leaves the
// outputs in place and CTA q stores its time steps of the whole group.
// N = 16 x 32 x 32, index n = nA*1024 + nB*32 + nC; three in-place passes
// (16-point over nA, 32-point over nB, 32-point over nC) with the inter-pass
// twiddles of the four-step decomposition.  The forward passes are
// decimation-in-frequency (natural in, digit-reversed out); the inverse
// passes undo them in reverse order with decimation in time, so no
// reordering pass exists.  The last forward pass of g, the pointwise
// product and the first inverse pass run back to back in registers.
#pragma once

#include <cooperative_groups.h>
#include <stdint.h>

namespace ccv {

constexpr uint32_t kNttP = 2013265921u;
constexpr int kNttN = 16384;
constexpr int64_t kNttMaxL = kNttN / 2;
constexpr int kNttThreads = 512;
constexpr int kNttWordsPerArray = kNttN + kNttN / 32;
constexpr int kNttGroup = 4;  // channels per cluster (4 x 4 bytes per time step)
constexpr size_t kNttSmemBytes = 2u * kNttWordsPerArray * 4u + 2u * 32 * 32 * 8;

struct NttParams {
    uint32_t p, w, winv, ninv, pinv, r2;
};

// ---- host-side number theory (exact, 64-bit) ----
static inline uint64_t h_mulmod(uint64_t a, uint64_t b, uint64_t m) { return (uint64_t)((__uint128_t)a * b % m); }
static inline uint64_t h_powmod(uint64_t a, uint64_t e, uint64_t m) {
    uint64_t r = 1 % m;
    a %= m;
    while (e) {
        if (e & 1) r = h_mulmod(r, a, m);
        a = h_mulmod(a, a, m);
        e >>= 1;
    }
    return r;
}
// Shoup companion floor(w * 2^32 / p)
static inline uint32_t h_shoup(uint32_t w) { return (uint32_t)(((uint64_t)w << 32) / kNttP); }

static inline bool ntt_params_host(int64_t N, NttParams *out) {
    if (N < 2 || N > (int64_t)1 << 27 || (N & (N - 1))) return false;
    const uint64_t p = kNttP;
    NttParams r;
    r.p = (uint32_t)p;
    r.w = (uint32_t)h_powmod(31, (p - 1) / (uint64_t)N, p);
    r.winv = (uint32_t)h_powmod(r.w, p - 2, p);
    r.ninv = (uint32_t)h_powmod((uint64_t)N, p - 2, p);
    // p^-1 mod 2^32 by Newton iteration (p odd)
    uint32_t x = (uint32_t)p;  // correct to 3 bits
    for (int i = 0; i < 5; ++i) x *= 2u - (uint32_t)p * x;
    r.pinv = x;
    r.r2 = (uint32_t)h_powmod(2, 64, p);
    *out = r;
    return true;
}

// ---- device constants and tables ----
// omega_32^k and omega_32^-k (k < 16) with Shoup companions.
__constant__ uint32_t c_nw32[16], c_nw32s[16], c_niw32[16], c_niw32s[16];
__constant__ uint32_t c_npinv, c_nscale, c_nscale_s;  // p^-1 mod 2^32; N^-1 * 2^32 mod p and its companion

// Inter-pass twiddles, indexed by storage slot (see ntt_init_device):
//   TF1[i*1024 + n2] = omega_N^(n2 * bitrev4(i))      TI1 = its inverse
//   TF2[i*32 + nC]   = omega_1024^(nC * bitrev5(i))   TI2 = its inverse
__device__ uint2 g_ntf1[16 * 1024], g_nti1[16 * 1024], g_ntf2[32 * 32], g_nti2[32 * 32];

__device__ __forceinline__ uint32_t n_red(uint32_t x) { return min(x, x - kNttP); }  // [0,2p) -> [0,p)
__device__ __forceinline__ uint32_t n_add(uint32_t a, uint32_t b) { return n_red(a + b); }
__device__ __forceinline__ uint32_t n_sub(uint32_t a, uint32_t b) { return n_red(a + kNttP - b); }
// a * w mod p (a < 2^32, result in [0, p))
__device__ __forceinline__ uint32_t n_mul_shoup(uint32_t a, uint32_t w, uint32_t ws) {
    const uint32_t q = __umulhi(a, ws);
    return n_red(a * w - q * kNttP);
}
// a * b * 2^-32 mod p (a, b < p)
__device__ __forceinline__ uint32_t n_mont(uint32_t a, uint32_t b) {
    const uint32_t lo = a * b, hi = __umulhi(a, b);
    const uint32_t m = lo * c_npinv;
    const uint32_t t = __umulhi(m, kNttP);
    const uint32_t r = hi - t;
    return hi < t ? r + kNttP : r;
}
__device__ __forceinline__ uint32_t n_from_int(int32_t x) {
    const uint32_t u = x < 0 ? (uint32_t)((int64_t)x + 2 * (int64_t)kNttP) : (uint32_t)x;  // < 2p
    return n_red(u);
}
__device__ __forceinline__ int32_t n_centered(uint32_t x) {
    return x > (kNttP - 1) / 2 ? (int32_t)((int64_t)x - (int64_t)kNttP) : (int32_t)x;
}

// Forward radix-2 DIF on R points (natural in, bit-reversed out).  Inputs
// x[ZERO_FROM..R) are known zero (only the first stage uses that).
template <int R, int ZERO_FROM>
__device__ __forceinline__ void ntt_dif(uint32_t (&x)[R]) {
#pragma unroll
    for (int half = R / 2; half >= 1; half >>= 1) {
#pragma unroll
        for (int base = 0; base < R; base += 2 * half) {
#pragma unroll
            for (int k = 0; k < half; ++k) {
                const int e = k * (32 / (2 * half));  // omega_{2 half}^k = omega_32^e
                const uint32_t a = x[base + k], b = x[base + k + half];
                if (half == R / 2 && base + k + half >= ZERO_FROM) {
                    x[base + k] = a;
                    x[base + k + half] = e == 0 ? a : n_mul_shoup(a, c_nw32[e], c_nw32s[e]);
                } else {
                    x[base + k] = n_add(a, b);
                    const uint32_t d = a + kNttP - b;  // < 2p
                    x[base + k + half] = e == 0 ? n_red(d) : n_mul_shoup(d, c_nw32[e], c_nw32s[e]);
                }
            }
        }
    }
}

// Inverse radix-2 DIT on R points (bit-reversed in, natural out), with
// conjugate twiddles, unnormalised.  Only outputs [0, KEEP) are formed in the
// last stage.
template <int R, int KEEP>
__device__ __forceinline__ void ntt_dit_inv(uint32_t (&x)[R]) {
#pragma unroll
    for (int half = 1; half < R; half <<= 1) {
#pragma unroll
        for (int base = 0; base < R; base += 2 * half) {
#pragma unroll
            for (int k = 0; k < half; ++k) {
                const int e = k * (32 / (2 * half));
                const uint32_t a = x[base + k];
                const uint32_t t = e == 0 ? x[base + k + half] : n_mul_shoup(x[base + k + half], c_niw32[e], c_niw32s[e]);
                x[base + k] = n_add(a, t);
                if (!(2 * half == R && base + k + half >= KEEP)) x[base + k + half] = n_sub(a, t);
            }
        }
    }
}

__device__ __forceinline__ int pad_idx(int s) { return s + (s >> 5); }

__device__ __forceinline__ void st_cluster_u32(uint32_t addr, uint32_t x) {
    asm volatile("st.shared::cluster.u32 [%0], %1;\n" ::"r"(addr), "r"(x) : "memory");
}
__device__ __forceinline__ uint32_t ld_cluster_u32(uint32_t addr) {
    uint32_t x;
    asm volatile("ld.shared::cluster.u32 %0, [%1];\n" : "=r"(x) : "r"(addr) : "memory");
    return x;
}

// One CTA per (b, d) row, kNttGroup rows per cluster.  smem: V[N + N/32],
// G[N + N/32] (padded words).  vec_ok: 16-byte group accesses are aligned.
__global__ void __launch_bounds__(kNttThreads, 1)
    ntt_conv_kernel(const int32_t *__restrict__ v, const int32_t *__restrict__ g, int32_t *__restrict__ r, int L,
                    int D, int groups_per_batch, int vec_ok) {
    extern __shared__ uint32_t nsm[];
    uint32_t *sv = nsm;
    uint32_t *sg = nsm + kNttWordsPerArray;
    uint2 *stf2 = reinterpret_cast<uint2 *>(nsm + 2 * kNttWordsPerArray);  // pass-2 twiddles, forward
    uint2 *sti2 = stf2 + 32 * 32;                                            // and inverse
    const int tid = threadIdx.x;
    for (int i = tid; i < 32 * 32; i += kNttThreads) {
        stf2[i] = g_ntf2[i];
        sti2[i] = g_nti2[i];
    }
    cooperative_groups::cluster_group cluster = cooperative_groups::this_cluster();
    const int rank = (int)cluster.block_rank();
    const int grp = blockIdx.x / kNttGroup;
    const int b = grp / groups_per_batch, d0 = (grp - b * groups_per_batch) * kNttGroup;
    const int nch = min(kNttGroup, D - d0);
    const bool vec = vec_ok && nch == kNttGroup;
    const int64_t gbase = (int64_t)b * L * D + d0;  // element (b, 0, d0)
    const uint32_t sv_addr = (uint32_t)__cvta_generic_to_shared(sv);
    const uint32_t sg_addr = (uint32_t)__cvta_generic_to_shared(sg);
    cluster.sync();  // every CTA of the cluster runs before the first remote store

    // Load: residues of time steps [t0, t0 + TC) of the group, zeros past L,
    // into slot t of each channel's CTA
    {
        constexpr int TC = (int)kNttMaxL / kNttGroup;
        const int t0 = rank * TC;
        uint32_t dv[kNttGroup], dg[kNttGroup];
#pragma unroll
        for (int c = 0; c < kNttGroup; ++c) {
            asm volatile("mapa.shared::cluster.u32 %0, %1, %2;\n" : "=r"(dv[c]) : "r"(sv_addr), "r"(c));
            asm volatile("mapa.shared::cluster.u32 %0, %1, %2;\n" : "=r"(dg[c]) : "r"(sg_addr), "r"(c));
        }
#pragma unroll 2
        for (int t = t0 + tid; t < t0 + TC; t += kNttThreads) {
            int32_t a[kNttGroup] = {0, 0, 0, 0}, q[kNttGroup] = {0, 0, 0, 0};
            if (t < L) {
                const int32_t *pv = v + gbase + (int64_t)t * D;
                const int32_t *pg = g + gbase + (int64_t)t * D;
                if (vec) {
                    const int4 x = __ldg(reinterpret_cast<const int4 *>(pv));
                    const int4 y = __ldg(reinterpret_cast<const int4 *>(pg));
                    a[0] = x.x; a[1] = x.y; a[2] = x.z; a[3] = x.w;
                    q[0] = y.x; q[1] = y.y; q[2] = y.z; q[3] = y.w;
                } else {
#pragma unroll
                    for (int c = 0; c < kNttGroup; ++c)
                        if (c < nch) {
                            a[c] = __ldg(pv + c);
                            q[c] = __ldg(pg + c);
                        }
                }
            }
            const uint32_t off = 4u * (uint32_t)pad_idx(t);
#pragma unroll
            for (int c = 0; c < kNttGroup; ++c) {
                st_cluster_u32(dv[c] + off, n_from_int(a[c]));
                st_cluster_u32(dg[c] + off, n_from_int(q[c]));
            }
        }
    }
    cluster.sync();

    // F1: 16-point DIF over nA for each n2 (inputs with nA >= 8 are padding
    // zeros); column n2 is read (slots of t = nA 1024 + n2) and rewritten in place
#pragma unroll 1
    for (int rep = 0; rep < 2; ++rep) {
        const int n2 = tid + rep * kNttThreads;
        uint32_t xv[16], xg[16];
#pragma unroll
        for (int nA = 0; nA < 16; ++nA) {
            const int s = pad_idx(nA * 1024 + n2);
            xv[nA] = nA < 8 ? sv[s] : 0u;
            xg[nA] = nA < 8 ? sg[s] : 0u;
        }
        ntt_dif<16, 8>(xv);
        ntt_dif<16, 8>(xg);
#pragma unroll
        for (int i = 0; i < 16; ++i) {
            const uint2 w = g_ntf1[i * 1024 + n2];
            const int s = pad_idx(i * 1024 + n2);
            sv[s] = i == 0 ? xv[i] : n_mul_shoup(xv[i], w.x, w.y);
            sg[s] = i == 0 ? xg[i] : n_mul_shoup(xg[i], w.x, w.y);
        }
    }
    __syncthreads();

    // F2: 32-point DIF over nB for each (slot a, nC)
    {
        const int a = tid >> 5, nC = tid & 31;
#pragma unroll 1
        for (int arr = 0; arr < 2; ++arr) {
            uint32_t *s = arr ? sg : sv;
            uint32_t x[32];
#pragma unroll
            for (int nB = 0; nB < 32; ++nB) x[nB] = s[pad_idx(a * 1024 + nB * 32 + nC)];
            ntt_dif<32, 32>(x);
#pragma unroll
            for (int i = 0; i < 32; ++i) {
                const uint2 w = stf2[i * 32 + nC];
                s[pad_idx(a * 1024 + i * 32 + nC)] = i == 0 ? x[i] : n_mul_shoup(x[i], w.x, w.y);
            }
        }
    }
    __syncthreads();

    // F3 of v and g, pointwise product, then I3 (inverse 32-point DIT over the same slots)
    {
        const int a = tid >> 5, bb = tid & 31;
        const int s0 = a * 1024 + bb * 32;
        uint32_t x[32], y[32];
#pragma unroll
        for (int i = 0; i < 32; ++i) {
            x[i] = sv[pad_idx(s0 + i)];
            y[i] = sg[pad_idx(s0 + i)];
        }
        ntt_dif<32, 32>(x);
        ntt_dif<32, 32>(y);
#pragma unroll
        for (int i = 0; i < 32; ++i) x[i] = n_mont(x[i], y[i]);
        ntt_dit_inv<32, 32>(x);
#pragma unroll
        for (int i = 0; i < 32; ++i) sv[pad_idx(s0 + i)] = x[i];
    }
    __syncthreads();

    // I2: twiddle then inverse 32-point DIT over the nB slots
    {
        const int a = tid >> 5, nC = tid & 31;
        uint32_t x[32];
#pragma unroll
        for (int i = 0; i < 32; ++i) {
            const uint32_t val = sv[pad_idx(a * 1024 + i * 32 + nC)];
            const uint2 w = sti2[i * 32 + nC];
            x[i] = i == 0 ? val : n_mul_shoup(val, w.x, w.y);
        }
        ntt_dit_inv<32, 32>(x);
#pragma unroll
        for (int nB = 0; nB < 32; ++nB) sv[pad_idx(a * 1024 + nB * 32 + nC)] = x[nB];
    }
    __syncthreads();

    // I1: twiddle, inverse 16-point DIT over the nA slots keeping nA < 8,
    // scale, lift; r_t is left in slot t of the same column
    const uint32_t sc = c_nscale, scs = c_nscale_s;
#pragma unroll 1
    for (int rep = 0; rep < 2; ++rep) {
        const int n2 = tid + rep * kNttThreads;
        uint32_t x[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) {
            const uint32_t val = sv[pad_idx(i * 1024 + n2)];
            const uint2 w = g_nti1[i * 1024 + n2];
            x[i] = i == 0 ? val : n_mul_shoup(val, w.x, w.y);
        }
        ntt_dit_inv<16, 8>(x);
#pragma unroll
        for (int nA = 0; nA < 8; ++nA)
            sv[pad_idx(nA * 1024 + n2)] = (uint32_t)n_centered(n_mul_shoup(x[nA], sc, scs));
    }
    cluster.sync();

    // Store: time steps [t0, t1) of the group, gathered from the channels' CTAs
    {
        const int TS = (L + kNttGroup - 1) / kNttGroup;
        const int t0 = rank * TS, t1 = min(L, t0 + TS);
        uint32_t src[kNttGroup];
#pragma unroll
        for (int c = 0; c < kNttGroup; ++c)
            asm volatile("mapa.shared::cluster.u32 %0, %1, %2;\n" : "=r"(src[c]) : "r"(sv_addr), "r"(c));
#pragma unroll 2
        for (int t = t0 + tid; t < t1; t += kNttThreads) {
            const uint32_t off = 4u * (uint32_t)pad_idx(t);
            uint32_t o[kNttGroup];
#pragma unroll
            for (int c = 0; c < kNttGroup; ++c) o[c] = ld_cluster_u32(src[c] + off);
            int32_t *pr = r + gbase + (int64_t)t * D;
            if (vec) {
                *reinterpret_cast<int4 *>(pr) = make_int4((int)o[0], (int)o[1], (int)o[2], (int)o[3]);
            } else {
#pragma unroll
                for (int c = 0; c < kNttGroup; ++c)
                    if (c < nch) pr[c] = (int32_t)o[c];
            }
        }
    }
    cluster.sync();  // remote reads of this CTA's slots are done before it exits
}

static inline uint32_t h_bitrev(uint32_t x, int bits) {
    uint32_t r = 0;
    for (int i = 0; i < bits; ++i) r = (r << 1) | ((x >> i) & 1u);
    return r;
}

static cudaError_t ntt_init_device() {
    NttParams P16, P32, P1024;
    ntt_params_host(kNttN, &P16);
    ntt_params_host(32, &P32);
    ntt_params_host(1024, &P1024);
    uint32_t w[16], ws[16], iw[16], iws[16];
    for (int k = 0; k < 16; ++k) {
        w[k] = (uint32_t)h_powmod(P32.w, k, kNttP);
        iw[k] = (uint32_t)h_powmod(P32.winv, k, kNttP);
        ws[k] = h_shoup(w[k]);
        iws[k] = h_shoup(iw[k]);
    }
    cudaError_t e;
    if ((e = cudaMemcpyToSymbol(c_nw32, w, sizeof(w))) != cudaSuccess) return e;
    if ((e = cudaMemcpyToSymbol(c_nw32s, ws, sizeof(ws))) != cudaSuccess) return e;
    if ((e = cudaMemcpyToSymbol(c_niw32, iw, sizeof(iw))) != cudaSuccess) return e;
    if ((e = cudaMemcpyToSymbol(c_niw32s, iws, sizeof(iws))) != cudaSuccess) return e;
    const uint32_t pinv = P16.pinv;
    const uint32_t scale = (uint32_t)h_mulmod(P16.ninv, h_powmod(2, 32, kNttP), kNttP);
    const uint32_t scale_s = h_shoup(scale);
    if ((e = cudaMemcpyToSymbol(c_npinv, &pinv, 4)) != cudaSuccess) return e;
    if ((e = cudaMemcpyToSymbol(c_nscale, &scale, 4)) != cudaSuccess) return e;
    if ((e = cudaMemcpyToSymbol(c_nscale_s, &scale_s, 4)) != cudaSuccess) return e;
    static uint2 t1[16 * 1024], ti1[16 * 1024], t2[32 * 32], ti2[32 * 32];
    for (uint32_t i = 0; i < 16; ++i)
        for (uint32_t n2 = 0; n2 < 1024; ++n2) {
            const uint64_t ex = (uint64_t)n2 * h_bitrev(i, 4);
            const uint32_t a = (uint32_t)h_powmod(P16.w, ex, kNttP), ai = (uint32_t)h_powmod(P16.winv, ex, kNttP);
            t1[i * 1024 + n2] = make_uint2(a, h_shoup(a));
            ti1[i * 1024 + n2] = make_uint2(ai, h_shoup(ai));
        }
    for (uint32_t i = 0; i < 32; ++i)
        for (uint32_t nC = 0; nC < 32; ++nC) {
            const uint64_t ex = (uint64_t)nC * h_bitrev(i, 5);
            const uint32_t a = (uint32_t)h_powmod(P1024.w, ex, kNttP), ai = (uint32_t)h_powmod(P1024.winv, ex, kNttP);
            t2[i * 32 + nC] = make_uint2(a, h_shoup(a));
            ti2[i * 32 + nC] = make_uint2(ai, h_shoup(ai));
        }
    if ((e = cudaMemcpyToSymbol(g_ntf1, t1, sizeof(t1))) != cudaSuccess) return e;
    if ((e = cudaMemcpyToSymbol(g_nti1, ti1, sizeof(ti1))) != cudaSuccess) return e;
    if ((e = cudaMemcpyToSymbol(g_ntf2, t2, sizeof(t2))) != cudaSuccess) return e;
    if ((e = cudaMemcpyToSymbol(g_nti2, ti2, sizeof(ti2))) != cudaSuccess) return e;
    return cudaFuncSetAttribute(ntt_conv_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kNttSmemBytes);
}

static int ntt_dispatch(const int32_t *v, const int32_t *g, int32_t *r, int64_t B, int64_t L, int64_t D,
                        cudaStream_t s) {
    if (L > kNttMaxL) return 2;  // CC_ERR_UNSUPPORTED
    const int64_t gpb = (D + kNttGroup - 1) / kNttGroup;
    if (B * gpb * kNttGroup > INT32_MAX) return 2;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)(B * gpb * kNttGroup));
    cfg.blockDim = dim3(kNttThreads);
    cfg.dynamicSmemBytes = kNttSmemBytes;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = kNttGroup;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    const int vec = (D % 4) == 0 && ((uintptr_t)v % 16) == 0 && ((uintptr_t)g % 16) == 0 && ((uintptr_t)r % 16) == 0;
    if (cudaLaunchKernelEx(&cfg, ntt_conv_kernel, v, g, r, (int)L, (int)D, (int)gpb, vec) != cudaSuccess) {
        cudaGetLastError();
        return 5;  // CC_ERR_CUDA
    }
    return 0;  // CC_OK
}

}  // namespace ccv
