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
    // twiddle tables (float2): TW0[k0*SL + n] = theta^(n (2 k0 + 1)),
    // TWA[k*(RB RC) + lo] = omega_SL^(lo k), TWB[k*RC + lo] = omega_(RB RC)^(lo k)
    static constexpr int TW0 = 0;
    static constexpr int TWA = S;
    static constexpr int TWB = S + SL;
    static constexpr int TW_SIZE = S + SL + RB * RC;
    static constexpr int LAST_R = RC > 1 ? RC : RB;
    static_assert(CL == 1 || CL == R0, "a cluster splits the most significant digit");
    static_assert(LAST_R == 16, "innermost radix must be 16 (conflict-free padded layout)");
    static_assert(R0 <= 64 && RA <= 32 && RB <= 32 && RC <= 32, "register DFT sizes");
    static_assert(SC % T == 0 && COLS0 % T == 0, "pass work split");
};

__device__ __forceinline__ int bc_pad(int p) { return p + (p >> 4); }

// One local forward (INV=false) or inverse (INV=true) pass over a digit of
// radix R and slot stride ST inside sub-arrays of SL slots; W = twiddle table
// omega_(R*ST)^(lo*k) laid out [k][lo] (nullptr when ST == 1).
template <int R, int ST, int SL, int SC, int T, bool INV>
__device__ __forceinline__ void bc_local_pass(float2 *xs, const float2 *__restrict__ W) {
    constexpr int NDFT = SC / R;
    constexpr int LOG_R = ilog2(R);
#pragma unroll 1
    for (int q = threadIdx.x; q < NDFT; q += T) {
        const int sub = q / (SL / R), w = q - sub * (SL / R);
        const int hi = w / ST, lo = w - hi * ST;
        const int base = sub * SL + hi * R * ST + lo;
        float2 x[R];
        if (!INV) {
#pragma unroll
            for (int j = 0; j < R; ++j) x[bitrev(j, LOG_R)] = xs[bc_pad(base + j * ST)];
            fft_dit<R, false>(x);
            if (ST > 1) {
#pragma unroll
                for (int k = 1; k < R; ++k) x[k] = cmul(x[k], __ldg(W + k * ST + lo));
            }
#pragma unroll
            for (int k = 0; k < R; ++k) xs[bc_pad(base + k * ST)] = x[k];
        } else {
#pragma unroll
            for (int k = 0; k < R; ++k) {
                float2 y = xs[bc_pad(base + k * ST)];
                if (ST > 1 && k > 0) y = cmul_conj(y, __ldg(W + k * ST + lo));
                x[bitrev(k, LOG_R)] = y;
            }
            fft_dit<R, true>(x);
#pragma unroll
            for (int j = 0; j < R; ++j) xs[bc_pad(base + j * ST)] = x[j];
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
    // generic pointer to slot s of the row (any CTA of the cluster)
    auto slot_ptr = [&](int s) -> float2 * {
        const int k0 = s / SL;
        const int owner = k0 / C::K0C;
        float2 *p = xs + bc_pad((k0 - owner * C::K0C) * SL + (s - k0 * SL));
        if constexpr (CL > 1) return cg::this_cluster().map_shared_rank(p, owner);
        return p;
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
        for (int k0 = 0; k0 < R0; ++k0) {
            const float2 y = cmul(x[k0], __ldg(tw + C::TW0 + k0 * SL + n));
            *slot_ptr(k0 * SL + n) = y;
        }
    }
    cluster_sync();

    // ---- forward local passes
    bc_local_pass<RA, RB * RC, SL, SC, T, false>(xs, tw + C::TWA);
    __syncthreads();
    if constexpr (RC > 1) {
        bc_local_pass<RB, RC, SL, SC, T, false>(xs, tw + C::TWB);
        __syncthreads();
        bc_local_pass<RC, 1, SL, SC, T, false>(xs, nullptr);
    } else {
        bc_local_pass<RB, 1, SL, SC, T, false>(xs, nullptr);
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
            const float2 zm = *slot_ptr(S - 1 - s);
            xv[i] = spectral_product(zk, zm);
        }
        cluster_sync();  // every mirror read done before any slot is overwritten
#pragma unroll
        for (int i = 0; i < PER; ++i) xs[bc_pad(tid + i * T)] = xv[i];
    }
    __syncthreads();

    // ---- inverse local passes
    if constexpr (RC > 1) {
        bc_local_pass<RC, 1, SL, SC, T, true>(xs, nullptr);
        __syncthreads();
        bc_local_pass<RB, RC, SL, SC, T, true>(xs, tw + C::TWB);
    } else {
        bc_local_pass<RB, 1, SL, SC, T, true>(xs, nullptr);
    }
    __syncthreads();
    bc_local_pass<RA, RB * RC, SL, SC, T, true>(xs, tw + C::TWA);
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
                const float2 y = *slot_ptr(k0 * SL + n);
                x[bitrev(k0, LOG_R0)] = cmul_conj(y, __ldg(tw + C::TW0 + k0 * SL + n));
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
