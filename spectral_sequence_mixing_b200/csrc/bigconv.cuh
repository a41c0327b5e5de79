// bigconv.cuh -- causal convolution for transform lengths beyond one tile of
// the fused kernel: one (b, d) row per CTA, or per thread-block cluster whose
// CTAs pool their shared memory (distributed shared memory) when the row's
// spectrum exceeds one SM.
//
// Same method as the fused kernel (Caracal: Causal Architecture via Spectral
// Mixing, key designs 1 and 2: pad to N >= 2L, transform, multiply, inverse
// transform, truncate), for long contexts (the limitations section singles
// out 100k+ tokens).  Per row:
//   * z = v + i g, odd-frequency forward transform of length S:
//     Z_k = sum_n z_n theta^(n(2k+1)), theta = exp(-i pi / S);
//   * X_k = V_k G_k from Z_k and its mirror Z_{S-1-k};
//   * inverse transform of X and untwist: r_n = Re(theta^-n IDFT(X)_n) for
//     n < L, the imaginary part being zero up to rounding;
//   * outputs t < 32 by direct summation.
//
// Transform structure: S = R0 * RA * RB * RC (RC may be 1).  The array of S
// complex values lives in shared memory in "digit order": bin
// k = k0 + R0 (kA + RA (kB + RB kC)) sits at slot
// k0 * SL + kA * (RB RC) + kB * RC + kC with SL = S / R0, each digit in natural
// order.  The mirror bin S-1-k complements every digit, so it sits at slot
// S-1-s.  Forward passes run over digits from the most significant (pass 0
// reads the zero-padded input from global memory), each a radix-R DFT of
// R strided elements followed by the four-step twiddle; the inverse passes
// undo them in reverse order (twiddle, then inverse DFT), the last one
// writing only t < L to global memory.
//
// With CL > 1 (CL == R0) the CTA with cluster rank q holds the slots of
// k0 == q; only pass 0, the mirror read and the inverse pass 0 cross CTAs.
#pragma once

#include <cooperative_groups.h>

#include "fft_reg.cuh"
#include "fftconv_fused.cuh"  // IO_t, spectral_product, kHeadT0

namespace ccv {

namespace cg = cooperative_groups;

template <int R0_, int RA_, int RB_, int RC_, int CL_, int T_, typename IO>
struct BigCfg {
    static constexpr int R0 = R0_, RA = RA_, RB = RB_, RC = RC_, CL = CL_, T = T_;
    static constexpr int SL = RA * RB * RC;  // sub-transform size after pass 0
    static constexpr int S = R0 * SL;
    static constexpr int LMAX = S / 2;
    static constexpr int SC = S / CL;        // slots per CTA
    static constexpr int K0C = R0 / CL;      // values of k0 per CTA
    static constexpr int COLS0 = SL / CL;    // pass-0 columns per CTA
    static constexpr int HEAD = kHeadT0;
    static constexpr int WORDS = SC + SC / 16;  // padded float2 words
    static constexpr int PER0 = COLS0 / T;  // pass-0 columns per thread
    static constexpr size_t SMEM_BYTES = (size_t)WORDS * 8 + (size_t)HEAD * 8 + (size_t)(T / 32 + 1) * 8;
    // Twiddle tables (float2), each factored into two small tables that stay
    // in L1 (value = product of two correctly rounded unit numbers):
    //   pass 0:  theta^(n (2 k0 + 1)), n = nh Q0 + nl
    //            = T0A[k0][nl] * T0B[k0][nh],  T0A = theta^(nl (2k0+1)), T0B = theta^(Q0 nh (2k0+1))
    //   pass A:  omega_SL^(lo k), lo = lh QA + ll
    //            = TAa[k][ll] * TAb[k][lh]
    //   pass B:  omega_(RB RC)^(lo k) = TB[k][lo]   (only when RC > 1)
    static constexpr int STA = RB * RC;  // slot stride of pass A
    static constexpr int Q0 = SL < 64 ? SL : 64;
    static constexpr int QA = STA < 32 ? STA : 32;
    static constexpr int T0A = 0;
    static constexpr int T0B = T0A + R0 * Q0;
    static constexpr int TAA = T0B + R0 * (SL / Q0);
    static constexpr int TAB = TAA + RA * QA;
    static constexpr int TB = TAB + RA * (STA / QA);
    static constexpr int TW_SIZE = TB + RB * RC;
    static constexpr int LAST_R = RC > 1 ? RC : RB;
    static_assert(CL == 1 || CL == R0, "a cluster splits the most significant digit");
    static_assert(LAST_R == 16, "innermost radix must be 16 (conflict-free padded layout)");
    static_assert(R0 <= 64 && RA <= 32 && RB <= 32 && RC <= 32, "register DFT sizes");
    static_assert(SC % T == 0 && COLS0 % T == 0, "pass work split");
};

__device__ __forceinline__ int bc_pad(int p) { return p + (p >> 4); }

// Distributed shared memory: 32-bit shared-window addresses of the same
// offset in another CTA of the cluster, and 8-byte loads / stores there.
__device__ __forceinline__ uint32_t smem_addr(const void *p) { return (uint32_t)__cvta_generic_to_shared(p); }
__device__ __forceinline__ uint32_t cluster_map(uint32_t addr, int rank) {
    uint32_t r;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;\n" : "=r"(r) : "r"(addr), "r"(rank));
    return r;
}
__device__ __forceinline__ void st_cluster(uint32_t addr, float2 v) {
    asm volatile("st.shared::cluster.v2.f32 [%0], {%1, %2};\n" ::"r"(addr), "f"(v.x), "f"(v.y) : "memory");
}
__device__ __forceinline__ float2 ld_cluster(uint32_t addr) {
    float2 v;
    asm volatile("ld.shared::cluster.v2.f32 {%0, %1}, [%2];\n" : "=f"(v.x), "=f"(v.y) : "r"(addr) : "memory");
    return v;
}

// One local forward (INV=false) or inverse (INV=true) pass over a digit of
// radix R and slot stride ST inside sub-arrays of SL slots.  The twiddle
// omega_(R ST)^(lo k) is Wa[k][lo % Q] * Wb[k][lo / Q] (Wb unused when
// ST <= Q; no twiddle when ST == 1).  With ST a multiple of 16 (or 1 and
// R == 16) the padded address of element j is pad(base) + j * PST, a
// compile-time offset.
template <int R, int ST, int Q, int SL, int SC, int T, bool INV>
__device__ __forceinline__ void bc_local_pass(float2 *xs, const float2 *__restrict__ Wa,
                                              const float2 *__restrict__ Wb) {
    constexpr int NDFT = SC / R;
    constexpr int LOG_R = ilog2(R);
    constexpr int PST = ST == 1 ? 1 : ST + ST / 16;
    static_assert(ST == 1 ? R == 16 : ST % 16 == 0, "linear padded addressing");
#pragma unroll 1
    for (int q = threadIdx.x; q < NDFT; q += T) {
        const int sub = q / (SL / R), w = q - sub * (SL / R);
        const int hi = w / ST, lo = w - hi * ST;
        float2 *xp = xs + bc_pad(sub * SL + hi * R * ST + lo);
        const float2 *wa = Wa + (lo % Q);
        const float2 *wb = Wb + (lo / Q);
        float2 x[R];
        if (!INV) {
#pragma unroll
            for (int j = 0; j < R; ++j) x[bitrev(j, LOG_R)] = xp[j * PST];
            fft_dit<R, false>(x);
            if (ST > 1) {
#pragma unroll
                for (int k = 1; k < R; ++k) {
                    float2 w2 = __ldg(wa + k * Q);
                    if (ST > Q) w2 = cmul(w2, __ldg(wb + k * (ST / Q)));
                    x[k] = cmul(x[k], w2);
                }
            }
#pragma unroll
            for (int k = 0; k < R; ++k) xp[k * PST] = x[k];
        } else {
#pragma unroll
            for (int k = 0; k < R; ++k) {
                float2 y = xp[k * PST];
                if (ST > 1 && k > 0) {
                    float2 w2 = __ldg(wa + k * Q);
                    if (ST > Q) w2 = cmul(w2, __ldg(wb + k * (ST / Q)));
                    y = cmul_conj(y, w2);
                }
                x[bitrev(k, LOG_R)] = y;
            }
            fft_dit<R, true>(x);
#pragma unroll
            for (int j = 0; j < R; ++j) xp[j * PST] = x[j];
        }
    }
}

template <int R0, int RA, int RB, int RC, int CL, int T, int MINB, typename IO>
__global__ void __launch_bounds__(T, MINB)
    bigconv_kernel(const IO *__restrict__ v, const IO *__restrict__ g, IO *__restrict__ r, int L, int D, int rev,
                   const float2 *__restrict__ tw) {
    // rev bit 0: read v reversed in time; bit 1: write r reversed
    using C = BigCfg<R0, RA, RB, RC, CL, T, IO>;
    constexpr int S = C::S, SL = C::SL, SC = C::SC, HEAD = C::HEAD;
    constexpr int LOG_R0 = ilog2(R0);
    extern __shared__ float4 bsm_raw[];
    float2 *xs = reinterpret_cast<float2 *>(bsm_raw);
    float2 *head = xs + C::WORDS;
    const int tid = threadIdx.x;
    int rank = 0;
    if constexpr (CL > 1) rank = (int)cg::this_cluster().block_rank();
    const int row = blockIdx.x / CL;
    const int b = row / D, d = row - b * D;
    const int64_t base = (int64_t)b * L * D + d;

    auto cluster_sync = [&]() {
        if constexpr (CL > 1)
            cg::this_cluster().sync();
        else
            __syncthreads();
    };
    if constexpr (CL > 1) cluster_sync();  // all CTAs of the cluster resident before any remote store
    // Slot (k0, n) of the row lives in CTA k0 / K0C at local offset
    // (k0 % K0C) SL + n; with a cluster it is reached through the shared
    // window address of that CTA (same layout in every CTA).
    const uint32_t xs_addr = smem_addr(xs);
    auto slot_addr = [&](int k0, int n) -> uint32_t {
        const int owner = k0 / C::K0C;
        const uint32_t local = xs_addr + 8u * (uint32_t)bc_pad((k0 - owner * C::K0C) * SL + n);
        if constexpr (CL > 1) return cluster_map(local, owner);
        return local;
    };
    auto slot_st = [&](uint32_t a, float2 val) {
        if constexpr (CL > 1)
            st_cluster(a, val);
        else
            asm volatile("st.shared.v2.f32 [%0], {%1, %2};\n" ::"r"(a), "f"(val.x), "f"(val.y) : "memory");
    };
    auto slot_ld = [&](uint32_t a) -> float2 {
        float2 val;
        if constexpr (CL > 1)
            val = ld_cluster(a);
        else
            asm volatile("ld.shared.v2.f32 {%0, %1}, [%2];\n" : "=f"(val.x), "=f"(val.y) : "r"(a) : "memory");
        return val;
    };
    // theta^(n (2 k0 + 1)) from the two factor tables
    auto tw0 = [&](int k0, int n) -> float2 {
        const float2 a = __ldg(tw + C::T0A + k0 * C::Q0 + (n % C::Q0));
        if constexpr (SL > C::Q0) return cmul(a, __ldg(tw + C::T0B + k0 * (SL / C::Q0) + (n / C::Q0)));
        return a;
    };

    // ---- load the padded input of this CTA's pass-0 columns; stream norms for balancing
    float2 zin[C::PER0][R0 / 2];
    float nv = 0.f, ng = 0.f;
#pragma unroll
    for (int p = 0; p < C::PER0; ++p) {
        const int n = rank * C::COLS0 + tid + p * T;  // column n_low in [0, SL)
#pragma unroll
        for (int n0 = 0; n0 < R0 / 2; ++n0) {
            const int t = n0 * SL + n;
            float2 z = make_float2(0.f, 0.f);
            if (t < L) z = make_float2(IO_t<IO>::cvt(IO_t<IO>::ld(v + base + (int64_t)((rev & 1) ? L - 1 - t : t) * D)),
                                       IO_t<IO>::cvt(IO_t<IO>::ld(g + base + (int64_t)t * D)));
            if (t < HEAD) head[t] = z;
            zin[p][n0] = z;
            nv = fmaf(z.x, z.x, nv);
            ng = fmaf(z.y, z.y, ng);
        }
    }
    float alpha;
    {
        float2 *red = head + HEAD;  // [T/32] warp partials, then [T/32] = CTA total
#pragma unroll
        for (int m = 1; m < 32; m <<= 1) {
            nv += __shfl_xor_sync(0xffffffffu, nv, m);
            ng += __shfl_xor_sync(0xffffffffu, ng, m);
        }
        if ((tid & 31) == 0) red[tid >> 5] = make_float2(nv, ng);
        __syncthreads();
        if (tid == 0) {
            float2 tot = make_float2(0.f, 0.f);
            for (int w = 0; w < T / 32; ++w) {
                tot.x += red[w].x;
                tot.y += red[w].y;
            }
            red[T / 32] = tot;
        }
        cluster_sync();
        float2 tot = red[T / 32];
        if constexpr (CL > 1) {
            tot = make_float2(0.f, 0.f);
            for (int q = 0; q < CL; ++q) {
                const float2 part = *cg::this_cluster().map_shared_rank(red + T / 32, q);
                tot.x += part.x;
                tot.y += part.y;
            }
        }
        alpha = balance_scale(tot.x, tot.y);
    }

    // ---- forward pass 0: odd-frequency R0-point DFT over n0 of z = v + i alpha g
#pragma unroll
    for (int p = 0; p < C::PER0; ++p) {
        const int n = rank * C::COLS0 + tid + p * T;
        float2 x[R0];
#pragma unroll
        for (int n0 = 0; n0 < R0 / 2; ++n0) {
            const float2 z = make_float2(zin[p][n0].x, alpha * zin[p][n0].y);
            x[bitrev(n0, LOG_R0)] = n0 == 0 ? z : cmul(z, tw_const(n0, 2 * R0));
        }
        fft_dit<R0, false, true>(x);
#pragma unroll
        for (int k0 = 0; k0 < R0; ++k0) slot_st(slot_addr(k0, n), cmul(x[k0], tw0(k0, n)));
    }
    cluster_sync();

    // ---- forward local passes
    bc_local_pass<RA, C::STA, C::QA, SL, SC, T, false>(xs, tw + C::TAA, tw + C::TAB);
    __syncthreads();
    if constexpr (RC > 1) {
        bc_local_pass<RB, RC, RC, SL, SC, T, false>(xs, tw + C::TB, tw + C::TB);
        __syncthreads();
        bc_local_pass<RC, 1, 1, SL, SC, T, false>(xs, tw, tw);
    } else {
        bc_local_pass<RB, 1, 1, SL, SC, T, false>(xs, tw, tw);
    }
    cluster_sync();

    // ---- spectral product X' = 4 V G at every own slot, from Z_s and Z_{S-1-s}
    {
        constexpr int PER = SC / T;
        float2 xv[PER];
#pragma unroll
        for (int i = 0; i < PER; ++i) {
            const int o = tid + i * T;               // own offset
            const int s = rank * SC + o;             // global slot (k0-major within the cluster)
            const float2 zk = xs[bc_pad(o)];
            const int sm = S - 1 - s;
            const float2 zm = slot_ld(slot_addr(sm / SL, sm % SL));
            xv[i] = spectral_product(zk, zm);
        }
        cluster_sync();  // every mirror read done before any slot is overwritten
#pragma unroll
        for (int i = 0; i < PER; ++i) xs[bc_pad(tid + i * T)] = xv[i];
    }
    __syncthreads();

    // ---- inverse local passes
    if constexpr (RC > 1) {
        bc_local_pass<RC, 1, 1, SL, SC, T, true>(xs, tw, tw);
        __syncthreads();
        bc_local_pass<RB, RC, RC, SL, SC, T, true>(xs, tw + C::TB, tw + C::TB);
    } else {
        bc_local_pass<RB, 1, 1, SL, SC, T, true>(xs, tw, tw);
    }
    __syncthreads();
    bc_local_pass<RA, C::STA, C::QA, SL, SC, T, true>(xs, tw + C::TAA, tw + C::TAB);
    cluster_sync();

    // ---- inverse pass 0: twiddle, inverse R0-point DFT (outputs n0 < R0/2), untwist, store t < L
    {
        const float s = 1.f / (4.f * (float)S * alpha);
#pragma unroll 1
        for (int c = tid; c < C::COLS0; c += T) {
            const int n = rank * C::COLS0 + c;
            float2 x[R0];
#pragma unroll
            for (int k0 = 0; k0 < R0; ++k0) {
                x[bitrev(k0, LOG_R0)] = cmul_conj(slot_ld(slot_addr(k0, n)), tw0(k0, n));
            }
            fft_dit<R0, true, false, true>(x);
#pragma unroll
            for (int n0 = 0; n0 < R0 / 2; ++n0) {
                const int t = n0 * SL + n;
                if (t >= L) continue;
                // untwist omega_2R0^-n0; only the real part is the output
                const float2 w = tw_const(n0, 2 * R0);
                float out = (n0 == 0 ? x[0].x : fmaf(x[n0].x, w.x, x[n0].y * w.y)) * s;
                if (t < HEAD) {
                    float a = 0.f;
                    for (int j = 0; j <= t; ++j) a = fmaf(head[j].x, head[t - j].y, a);
                    out = a;
                }
                IO_t<IO>::st(r + base + (int64_t)((rev & 2) ? L - 1 - t : t) * D, out);
            }
        }
    }
    cluster_sync();  // keep this CTA's shared memory alive until the cluster is done with it
}

}  // namespace ccv
