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
// With CL == R0 / 2 ("mirror pairs") CTA q holds k0 == q at local offsets
// [0, SL) and k0 == R0-1-q at [SL, 2 SL): a bin and its mirror then share a
// CTA (local offsets o and 2 SL-1-o), so the spectral product stays in the
// CTA and only pass 0 and the inverse pass 0 exchange data between CTAs.
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
    static constexpr bool MIRROR = CL > 1 && 2 * CL == R0;  // k0 pairs (q, R0-1-q) per CTA
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
    // Real-output inverse (mirror pairs only; see bigconv_kernel): a transform
    // of half the length, M = S / 2, whose innermost digit has RC / 2 values.
    //   packing: theta^(2 R0 k'') = omega_SL^k'', k'' = kA + RA j (j < RB RC / 2)
    //            = TPA[kA] * TPB[j]          (omega_SL^kA, omega_(SL / RA)^j)
    //   pass B:  omega_(RB RC/2)^(lo k) = TBH[k][lo], lo < RC / 2
    //   pass A:  omega_(SL/2)^(lo k), lo = lh QA + ll < RB RC / 2
    //            = TAHA[k][ll] * TAHB[k][lh]
    static constexpr int RCH = RC / 2;
    static constexpr int STAH = RB * RCH;  // logical stride of the half-length pass A
    static constexpr int TPA = TB + RB * RC;
    static constexpr int TPB = TPA + RA;
    static constexpr int TBH = TPB + STAH;
    static constexpr int TAHA = TBH + RB * RCH;
    static constexpr int TAHB = TAHA + RA * QA;
    static constexpr int TW_SIZE = MIRROR ? TAHB + RA * (STAH / QA) : TB + RB * RC;
    static constexpr int LAST_R = RC > 1 ? RC : RB;
    static_assert(CL == 1 || CL == R0 || 2 * CL == R0, "a cluster splits the most significant digit");
    static_assert(LAST_R == 16, "innermost radix must be 16 (conflict-free padded layout)");
    static_assert(R0 <= 64 && RA <= 32 && RB <= 32 && RC <= 32, "register DFT sizes");
    static_assert(SC % (2 * T) == 0 && COLS0 % T == 0, "pass work split");
    static_assert(!MIRROR || (R0 == 16 && RA == 32 && RB == 16 && RC == 16 && CL == 8 && T == 512),
                  "the real-output inverse is written for the 16 x 32 x 16 x 16 cluster rows");
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
                   int row_major, const float2 *__restrict__ tw) {
    // rev bit 0: read v reversed in time; bit 1: write r reversed.
    // row_major: v, g, r are [B, D, L] (each row contiguous) instead of
    // channel-last [B, L, D].
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
    // element (row, t) sits at base + t * tstep
    const int64_t base = row_major ? (int64_t)row * L : (int64_t)b * L * D + d;
    const int64_t tstep = row_major ? 1 : D;

    auto cluster_sync = [&]() {
        if constexpr (CL > 1)
            cg::this_cluster().sync();
        else
            __syncthreads();
    };
    if constexpr (CL > 1) cluster_sync();  // all CTAs of the cluster resident before any remote store
    // Slot (k0, n) of the row lives in CTA k0 / K0C at local offset
    // (k0 % K0C) SL + n (mirror pairs: CTA min(k0, R0-1-k0), offset SL + n for
    // the upper k0); with a cluster it is reached through the shared window
    // address of that CTA (same layout in every CTA).
    const uint32_t xs_addr = smem_addr(xs);
    auto slot_addr = [&](int k0, int n) -> uint32_t {
        int owner, lk;
        if constexpr (C::MIRROR) {
            const bool up = k0 >= R0 / 2;
            owner = up ? R0 - 1 - k0 : k0;
            lk = up ? 1 : 0;
        } else {
            owner = k0 / C::K0C;
            lk = k0 - owner * C::K0C;
        }
        const uint32_t local = xs_addr + 8u * (uint32_t)bc_pad(lk * SL + n);
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
            if (t < L) z = make_float2(IO_t<IO>::cvt(IO_t<IO>::ld(v + base + (int64_t)((rev & 1) ? L - 1 - t : t) * tstep)),
                                       IO_t<IO>::cvt(IO_t<IO>::ld(g + base + (int64_t)t * tstep)));
            if (t < HEAD) head[t] = z;
            zin[p][n0] = z;
            nv = fmaf(z.x, z.x, nv);
            ng = fmaf(z.y, z.y, ng);
        }
    }
    float alpha;
    bool live;  // false: v or g is all zero, the row is exactly zero
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
        live = tot.x > 0.f && tot.y > 0.f;
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
    if constexpr (C::MIRROR)
        __syncthreads();
    else
        cluster_sync();

    // ---- real-output inverse (mirror pairs).  r is real, so the S-point
    // inverse y_n = sum_k X_k theta^(-n (2k+1)) is taken as one M = S/2-point
    // odd-frequency inverse whose outputs are w_m = y_2m + i y_2m+1:
    //   C_k = E_k + i O_k,  E_k = X_k + X_(k+M),  O_k = (X_k - X_(k+M)) theta^-(2k+1),
    //   w_m = sum_(k<M) C_k phi^(m (2k+1)),  phi = theta^-2
    // (bin k + M is the same slot with the innermost digit kC + RC/2, so the
    // packing stays in the CTA; it runs with the spectral product, below, and
    // leaves C_k in the slots with kC < RC/2).  With k = k0 + R0 k'' and m = m0 (SL/2) + m',
    // the M-point inverse splits like the S-point one: for each k0 an
    // (SL/2)-point inverse DFT over k'' (passes over kC < RC/2, kB, kA in
    // the slots' lower halves), then across the cluster the twiddle
    // conj(theta^(2m' (2 k0 + 1))), the inverse R0-point DFT over k0
    // (outputs m0 < R0/2) and the untwist.  Half the work and half the
    // distributed-shared-memory reads of the S-point inverse.
    auto inverse_real_output = [&]() {
        constexpr int RCH = C::RCH, STAH = C::STAH;
        constexpr int PSTB = RC + RC / 16, PSTA = RB * RC + (RB * RC) / 16;
        // innermost digit kC < RCH (slot stride 1): inverse RCH-point DFT, no twiddle
#pragma unroll 1
        for (int q = tid; q < SC / RC; q += T) {
            float2 *xp = xs + bc_pad(q * RC);
            float2 x[RCH];
#pragma unroll
            for (int k = 0; k < RCH; ++k) x[bitrev(k, ilog2(RCH))] = xp[k];
            fft_dit<RCH, true>(x);
#pragma unroll
            for (int j = 0; j < RCH; ++j) xp[j] = x[j];
        }
        __syncthreads();
        // digit kB (slot stride RC), lo = the kC digit's output (< RCH):
        // twiddle conj(omega_(RB RCH)^(lo kB)), inverse RB-point DFT
#pragma unroll 1
        for (int q = tid; q < 2 * RA * RCH; q += T) {
            const int lk = q / (RA * RCH), w = q - lk * (RA * RCH), ka = w / RCH, lo = w - ka * RCH;
            float2 *xp = xs + bc_pad(lk * SL + ka * (RB * RC) + lo);
            float2 x[RB];
#pragma unroll
            for (int k = 0; k < RB; ++k) {
                float2 y = xp[k * PSTB];
                if (k > 0) y = cmul_conj(y, __ldg(tw + C::TBH + k * RCH + lo));
                x[bitrev(k, ilog2(RB))] = y;
            }
            fft_dit<RB, true>(x);
#pragma unroll
            for (int j = 0; j < RB; ++j) xp[j * PSTB] = x[j];
        }
        __syncthreads();
        // digit kA (slot stride RB RC), logical lo = (kB output) RCH + (kC output) < STAH:
        // twiddle conj(omega_(SL/2)^(lo kA)), inverse RA-point DFT
#pragma unroll 1
        for (int q = tid; q < 2 * STAH; q += T) {
            const int lk = q / STAH, lol = q - lk * STAH;
            float2 *xp = xs + bc_pad(lk * SL + (lol / RCH) * RC + lol % RCH);
            float2 x[RA];
#pragma unroll
            for (int k = 0; k < RA; ++k) {
                float2 y = xp[k * PSTA];
                if (k > 0)
                    y = cmul_conj(y, cmul(__ldg(tw + C::TAHA + k * C::QA + lol % C::QA),
                                          __ldg(tw + C::TAHB + k * (STAH / C::QA) + lol / C::QA)));
                x[bitrev(k, ilog2(RA))] = y;
            }
            fft_dit<RA, true>(x);
#pragma unroll
            for (int j = 0; j < RA; ++j) xp[j * PSTA] = x[j];
        }
        // the direct sums r_t, t < HEAD (time steps of CTA 0's first columns),
        // into the norm-partials area, which is free by now
        float *hsum = reinterpret_cast<float *>(head + HEAD);
        static_assert(2 * (T / 32 + 1) >= HEAD, "head sums fit the norm-partials area");
        if (rank == 0 && tid < HEAD) {
            float a = 0.f;
            for (int j = 0; j <= tid; ++j) a = fmaf(head[j].x, head[tid - j].y, a);
            hsum[tid] = a;
        }
        cluster_sync();
        // across the cluster: column m' of both k0 halves of every CTA, twiddle,
        // inverse R0-point DFT over k0 (outputs m0 < R0/2), untwist; w_m gives
        // r_(2m) and r_(2m+1), m = m0 (SL/2) + m'
        {
            const float s = live ? 1.f / (4.f * (float)S * alpha) : 0.f;
            constexpr int COLSH = SL / 2 / CL;  // columns m' per CTA
#pragma unroll 1
            for (int c = tid; c < COLSH; c += T) {
                const int mp = rank * COLSH + c;
                // m' = a (RB RCH) + b RCH + e sits at slot a (RB RC) + b RC + e
                const int phys = (mp / (RB * RCH)) * (RB * RC) + ((mp / RCH) % RB) * RC + mp % RCH;
                float2 x[R0];
#pragma unroll
                for (int k0 = 0; k0 < R0; ++k0)
                    x[bitrev(k0, LOG_R0)] = cmul_conj(slot_ld(slot_addr(k0, phys)), tw0(k0, 2 * mp));
                fft_dit<R0, true, false, true>(x);
#pragma unroll
                for (int m0 = 0; m0 < R0 / 2; ++m0) {
                    const int t = 2 * (m0 * (SL / 2) + mp);
                    if (t >= L) continue;
                    // untwist conj(omega_2R0^m0)
                    const float2 z = m0 == 0 ? x[0] : cmul_conj(x[m0], tw_const(m0, 2 * R0));
                    float o0 = z.x * s, o1 = z.y * s;
                    if (t < HEAD) {  // HEAD is even, so t + 1 < HEAD too
                        o0 = hsum[t];
                        o1 = hsum[t + 1];
                    }
                    IO_t<IO>::st(r + base + (int64_t)((rev & 2) ? L - 1 - t : t) * tstep, o0);
                    if (t + 1 < L) IO_t<IO>::st(r + base + (int64_t)((rev & 2) ? L - 2 - t : t + 1) * tstep, o1);
                }
            }
        }
    };

    // ---- spectral product X' = 4 V G.  The pair (s, S-1-s) is handled by the
    // thread that owns s at local offset o < SC/2 (the mirror then sits at a
    // local offset >= SC/2: SC-1-o in this CTA with mirror pairs, else in CTA
    // R0-1-rank): it reads both bins and writes X'_s and X'_{S-1-s} =
    // conj(X'_s), so every slot is read and written by one thread only.
    {
        constexpr int PER2 = SC / (2 * T);
        if constexpr (C::MIRROR) {
            // With the real-output packing: a thread takes o (k0 = rank, kC < RC/2),
            // o + RC/2 (bin k + M), and their mirrors SC-1-o and p = SC-1-o-RC/2
            // (k0 = R0-1-rank; p's innermost digit is RC/2-1-kC, and p + RC/2 is
            // SC-1-o): two spectral products give all four X', then
            // C_o = pack(X'_o, X'_(o+RC/2)) and C_p = pack(X'_p, X'_(p+RC/2)).
            constexpr int RCH = C::RCH;
            // theta^(2 k0 + 1) for this CTA's two k0 (rank, R0-1-rank)
            const float2 tk0 = __ldg(tw + C::T0A + rank * C::Q0 + 1);
            const float2 tk1 = __ldg(tw + C::T0A + (R0 - 1 - rank) * C::Q0 + 1);
            // C = E + i O, E = a + b, O = (a - b) conj(w), w = theta^(2k+1)
            auto pack = [](float2 a, float2 b, float2 w) -> float2 {
                const float2 ov = cmul_conj(csub(a, b), w), ev = cadd(a, b);
                return make_float2(ev.x - ov.y, ev.y + ov.x);
            };
#pragma unroll 2
            for (int i = tid; i < SC / 4; i += T) {
                const int kc = i % RCH, kb = (i / RCH) % RB, ka = i / (RCH * RB);
                const int o = ka * (RB * RC) + kb * RC + kc, p = SC - 1 - o - RCH;
                const float2 xo = spectral_product(xs[bc_pad(o)], xs[bc_pad(SC - 1 - o)]);
                const float2 xo8 = spectral_product(xs[bc_pad(o + RCH)], xs[bc_pad(p)]);
                // theta^(2k+1) = theta^(2 k0 + 1) omega_SL^k'', k'' = kA + RA (kB + RB kC)
                const float2 wo = cmul(cmul(tk0, __ldg(tw + C::TPA + ka)), __ldg(tw + C::TPB + kb + RB * kc));
                const float2 wp = cmul(cmul(tk1, __ldg(tw + C::TPA + RA - 1 - ka)),
                                       __ldg(tw + C::TPB + (RB - 1 - kb) + RB * (RCH - 1 - kc)));
                xs[bc_pad(o)] = pack(xo, xo8, wo);
                xs[bc_pad(p)] = pack(cconj(xo8), cconj(xo), wp);
            }
        } else {
#pragma unroll 4
            for (int i = 0; i < PER2; ++i) {
                const int o = tid + i * T;
                const int sm = S - 1 - (rank * SC + o);
                const uint32_t am = slot_addr(sm / SL, sm % SL);
                const float2 xk = spectral_product(xs[bc_pad(o)], slot_ld(am));
                xs[bc_pad(o)] = xk;
                slot_st(am, cconj(xk));
            }
        }
    }
    if constexpr (C::MIRROR)
        __syncthreads();
    else
        cluster_sync();

    if constexpr (C::MIRROR) {
        inverse_real_output();
    } else {
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
            const float s = live ? 1.f / (4.f * (float)S * alpha) : 0.f;
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
                    IO_t<IO>::st(r + base + (int64_t)((rev & 2) ? L - 1 - t : t) * tstep, out);
                }
            }
        }
    }
    cluster_sync();  // keep this CTA's shared memory alive until the cluster is done with it
}

// ---------------------------------------------------------------------------
// Channel groups: rows that fit one CTA, kGroup adjacent channels of one
// batch per cluster (one channel per CTA).  Reading one channel of a
// channel-last tensor touches a separate 2..4-byte piece of memory per time
// step; a group reads all kGroup channels of a time step in one 16..32-byte
// piece instead.  CTA q of the cluster loads time steps
// [q LMAX/kGroup, (q+1) LMAX/kGroup) of the whole group and writes
// (v_t, g_t) of channel c straight into slot t of CTA c (distributed shared
// memory), which is where the row's pass 0 reads its input (t = n0 SL + n is
// slot (n0, n), the column pass 0 rewrites in place).  The last inverse pass
// leaves r_t in slot t the same way, and CTA q gathers its time steps of all
// kGroup channels for the stores.
constexpr int kGroup = 8;

__device__ __forceinline__ float ld_cluster_f32(uint32_t addr) {
    float x;
    asm volatile("ld.shared::cluster.f32 %0, [%1];\n" : "=f"(x) : "r"(addr) : "memory");
    return x;
}

// kGroup consecutive channels at p[0..nch) (zeros beyond nch, or everywhere when !inb).
template <typename IO>
__device__ __forceinline__ void load_group(const IO *__restrict__ p, int nch, bool vec, bool inb, float (&o)[kGroup]) {
#pragma unroll
    for (int c = 0; c < kGroup; ++c) o[c] = 0.f;
    if (!inb) return;
    if (vec) {
        if constexpr (sizeof(IO) == 2) {
            const uint4 w = __ldg(reinterpret_cast<const uint4 *>(p));
            const uint32_t u[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
            for (int c = 0; c < kGroup; ++c) o[c] = __uint_as_float(((u[c / 2] >> (16 * (c & 1))) & 0xffffu) << 16);
        } else {
            const float4 a = __ldg(reinterpret_cast<const float4 *>(p));
            const float4 bq = __ldg(reinterpret_cast<const float4 *>(p) + 1);
            o[0] = a.x; o[1] = a.y; o[2] = a.z; o[3] = a.w;
            o[4] = bq.x; o[5] = bq.y; o[6] = bq.z; o[7] = bq.w;
        }
    } else {
#pragma unroll
        for (int c = 0; c < kGroup; ++c)
            if (c < nch) o[c] = IO_t<IO>::cvt(IO_t<IO>::ld(p + c));
    }
}

template <typename IO>
__device__ __forceinline__ void store_group(IO *__restrict__ p, int nch, bool vec, const float (&o)[kGroup]) {
    if (vec) {
        if constexpr (sizeof(IO) == 2) {
            uint32_t u[4];
#pragma unroll
            for (int i = 0; i < 4; ++i)
                u[i] = (uint32_t)__bfloat16_as_ushort(__float2bfloat16_rn(o[2 * i])) |
                       ((uint32_t)__bfloat16_as_ushort(__float2bfloat16_rn(o[2 * i + 1])) << 16);
            *reinterpret_cast<uint4 *>(p) = make_uint4(u[0], u[1], u[2], u[3]);
        } else {
            reinterpret_cast<float4 *>(p)[0] = make_float4(o[0], o[1], o[2], o[3]);
            reinterpret_cast<float4 *>(p)[1] = make_float4(o[4], o[5], o[6], o[7]);
        }
    } else {
#pragma unroll
        for (int c = 0; c < kGroup; ++c)
            if (c < nch) IO_t<IO>::st(p + c, o[c]);
    }
}

template <int R0, int RA, int RB, int RC, int T, int MINB, typename IO>
__global__ void __launch_bounds__(T, MINB)
    bigrow_group_kernel(const IO *__restrict__ v, const IO *__restrict__ g, IO *__restrict__ r, int L, int D,
                        int groups_per_batch, int rev, int vec_ok, const float2 *__restrict__ tw) {
    // rev bit 0: read v reversed in time; bit 1: write r reversed.  vec_ok:
    // whole groups may use 16-byte accesses (D and the base pointers allow it).
    using C = BigCfg<R0, RA, RB, RC, 1, T, IO>;
    constexpr int S = C::S, SL = C::SL, HEAD = C::HEAD, LMAX = C::LMAX;
    constexpr int LOG_R0 = ilog2(R0);
    static_assert(LMAX % kGroup == 0, "time steps split evenly over the group");
    extern __shared__ float4 bsm_raw[];
    float2 *xs = reinterpret_cast<float2 *>(bsm_raw);
    float2 *head = xs + C::WORDS;
    const int tid = threadIdx.x;
    cg::cluster_group cluster = cg::this_cluster();
    const int rank = (int)cluster.block_rank();
    const int grp = blockIdx.x / kGroup;
    const int b = grp / groups_per_batch, d0 = (grp - b * groups_per_batch) * kGroup;
    const int nch = min(kGroup, D - d0);
    const bool vec = vec_ok && nch == kGroup;
    const int64_t gbase = (int64_t)b * L * D + d0;  // element (b, 0, d0)
    const uint32_t xs_addr = smem_addr(xs);
    cluster.sync();  // every CTA of the cluster runs before the first remote store

    // ---- cooperative load of time steps [t0, t0 + LMAX/kGroup), zeros past L
    {
        constexpr int TC = LMAX / kGroup;
        const int t0 = rank * TC;
        uint32_t dst[kGroup];
#pragma unroll
        for (int c = 0; c < kGroup; ++c) dst[c] = cluster_map(xs_addr, c);
#pragma unroll 2
        for (int t = t0 + tid; t < t0 + TC; t += T) {
            float vv[kGroup], gg[kGroup];
            const bool inb = t < L;
            load_group<IO>(v + gbase + (int64_t)((rev & 1) ? L - 1 - t : t) * D, nch, vec, inb, vv);
            load_group<IO>(g + gbase + (int64_t)t * D, nch, vec, inb, gg);
            const uint32_t off = 8u * (uint32_t)bc_pad(t);
#pragma unroll
            for (int c = 0; c < kGroup; ++c) st_cluster(dst[c] + off, make_float2(vv[c], gg[c]));
        }
    }
    cluster.sync();

    // ---- this CTA's row: input of the pass-0 columns, norms for balancing
    float2 zin[C::PER0][R0 / 2];
    float nv = 0.f, ng = 0.f;
#pragma unroll
    for (int p = 0; p < C::PER0; ++p) {
        const int n = tid + p * T;
#pragma unroll
        for (int n0 = 0; n0 < R0 / 2; ++n0) {
            const int t = n0 * SL + n;
            const float2 z = xs[bc_pad(t)];
            if (t < HEAD) head[t] = z;
            zin[p][n0] = z;
            nv = fmaf(z.x, z.x, nv);
            ng = fmaf(z.y, z.y, ng);
        }
    }
    float alpha;
    bool live;  // false: v or g is all zero, the row is exactly zero
    {
        float2 *red = head + HEAD;
#pragma unroll
        for (int m = 1; m < 32; m <<= 1) {
            nv += __shfl_xor_sync(0xffffffffu, nv, m);
            ng += __shfl_xor_sync(0xffffffffu, ng, m);
        }
        if ((tid & 31) == 0) red[tid >> 5] = make_float2(nv, ng);
        __syncthreads();
        float2 tot = make_float2(0.f, 0.f);
#pragma unroll
        for (int w = 0; w < T / 32; ++w) {
            tot.x += red[w].x;
            tot.y += red[w].y;
        }
        alpha = balance_scale(tot.x, tot.y);
        live = tot.x > 0.f && tot.y > 0.f;
    }
    auto tw0 = [&](int k0, int n) -> float2 {
        const float2 a = __ldg(tw + C::T0A + k0 * C::Q0 + (n % C::Q0));
        if constexpr (SL > C::Q0) return cmul(a, __ldg(tw + C::T0B + k0 * (SL / C::Q0) + (n / C::Q0)));
        return a;
    };

    // ---- forward pass 0 (in place per column n: reads slots (n0, n), writes (k0, n))
#pragma unroll
    for (int p = 0; p < C::PER0; ++p) {
        const int n = tid + p * T;
        float2 x[R0];
#pragma unroll
        for (int n0 = 0; n0 < R0 / 2; ++n0) {
            const float2 z = make_float2(zin[p][n0].x, alpha * zin[p][n0].y);
            x[bitrev(n0, LOG_R0)] = n0 == 0 ? z : cmul(z, tw_const(n0, 2 * R0));
        }
        fft_dit<R0, false, true>(x);
#pragma unroll
        for (int k0 = 0; k0 < R0; ++k0) xs[bc_pad(k0 * SL + n)] = cmul(x[k0], tw0(k0, n));
    }
    __syncthreads();

    // ---- forward local passes, spectral product, inverse local passes
    bc_local_pass<RA, C::STA, C::QA, SL, S, T, false>(xs, tw + C::TAA, tw + C::TAB);
    __syncthreads();
    if constexpr (RC > 1) {
        bc_local_pass<RB, RC, RC, SL, S, T, false>(xs, tw + C::TB, tw + C::TB);
        __syncthreads();
        bc_local_pass<RC, 1, 1, SL, S, T, false>(xs, tw, tw);
    } else {
        bc_local_pass<RB, 1, 1, SL, S, T, false>(xs, tw, tw);
    }
    __syncthreads();
#pragma unroll 4
    for (int i = 0; i < S / (2 * T); ++i) {  // pair (o, S-1-o), o < S/2
        const int o = tid + i * T;
        const float2 xk = spectral_product(xs[bc_pad(o)], xs[bc_pad(S - 1 - o)]);
        xs[bc_pad(o)] = xk;
        xs[bc_pad(S - 1 - o)] = cconj(xk);
    }
    __syncthreads();
    if constexpr (RC > 1) {
        bc_local_pass<RC, 1, 1, SL, S, T, true>(xs, tw, tw);
        __syncthreads();
        bc_local_pass<RB, RC, RC, SL, S, T, true>(xs, tw + C::TB, tw + C::TB);
    } else {
        bc_local_pass<RB, 1, 1, SL, S, T, true>(xs, tw, tw);
    }
    __syncthreads();
    bc_local_pass<RA, C::STA, C::QA, SL, S, T, true>(xs, tw + C::TAA, tw + C::TAB);
    __syncthreads();

    // ---- inverse pass 0: twiddle, inverse R0-point DFT (outputs n0 < R0/2),
    // untwist; r_t (t < L) is left in slot t of the same column
    {
        const float sc = live ? 1.f / (4.f * (float)S * alpha) : 0.f;
#pragma unroll 1
        for (int n = tid; n < SL; n += T) {
            float2 x[R0];
#pragma unroll
            for (int k0 = 0; k0 < R0; ++k0) x[bitrev(k0, LOG_R0)] = cmul_conj(xs[bc_pad(k0 * SL + n)], tw0(k0, n));
            fft_dit<R0, true, false, true>(x);
#pragma unroll
            for (int n0 = 0; n0 < R0 / 2; ++n0) {
                const int t = n0 * SL + n;
                if (t >= L) continue;
                const float2 w = tw_const(n0, 2 * R0);
                float out = (n0 == 0 ? x[0].x : fmaf(x[n0].x, w.x, x[n0].y * w.y)) * sc;
                if (t < HEAD) {
                    float a = 0.f;
                    for (int j = 0; j <= t; ++j) a = fmaf(head[j].x, head[t - j].y, a);
                    out = a;
                }
                xs[bc_pad(t)].x = out;
            }
        }
    }
    cluster.sync();

    // ---- cooperative store of time steps [t0, t1) of the group
    {
        const int TS = (L + kGroup - 1) / kGroup;
        const int t0 = rank * TS, t1 = min(L, t0 + TS);
        uint32_t src[kGroup];
#pragma unroll
        for (int c = 0; c < kGroup; ++c) src[c] = cluster_map(xs_addr, c);
#pragma unroll 2
        for (int t = t0 + tid; t < t1; t += T) {
            float o[kGroup];
            const uint32_t off = 8u * (uint32_t)bc_pad(t);
#pragma unroll
            for (int c = 0; c < kGroup; ++c) o[c] = ld_cluster_f32(src[c] + off);
            store_group<IO>(r + gbase + (int64_t)((rev & 2) ? L - 1 - t : t) * D, nch, vec, o);
        }
    }
    cluster.sync();  // remote reads of this CTA's slots are done before it exits
}

}  // namespace ccv
