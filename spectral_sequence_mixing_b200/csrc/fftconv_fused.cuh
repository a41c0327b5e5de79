// fftconv_fused.cuh -- fused pad -> FFT -> multiply -> inverse FFT -> truncate
// kernel for one tile of ROWS channels of one batch, whole rows on chip.
//
// Method (Caracal: Causal Architecture via Spectral Mixing, "Key design 1"
// and "Key design 2"): each (b, d) row of v (value stream) and g (gate
// stream) is zero-padded to N = 2L, transformed, multiplied pointwise,
// inverse-transformed and truncated to L, which equals
// r_t = sum_{j<=t} v_j g_{t-j}.  The real-FFT halving suggested in the
// limitations section ("use RFFT to halve compute") is realised twice:
//   * forward: one complex FFT of z = v + i g per row; V and G are separated
//     from the k and N-k bins of Z;
//   * inverse: the real length-N output is obtained from one complex FFT of
//     length M = N/2 whose output is r[2m] + i r[2m+1].
//
// Decomposition (N = N1 * N2, N1 = 2 * N2, one shared-memory exchange per
// transform):
//   F1  thread (c, n2): N1-point DFT over n1 of z[n2 + N2 n1]; half of the
//       inputs are padding zeros, so it is two N2-point DFTs (of z and of
//       z * omega_N1^n); times omega_N^(n2 k1); to shared memory.
//   F3  thread (c, j) owns columns k1 = j and N1 - j (j = 0: 0 and N1/2), so
//       every bin k = k1 + N1 k2 meets its mirror N - k and its half-length
//       partner M - k in registers: N2-point DFTs over n2, spectral product,
//       real-inverse packing, then the first inverse step (M2 = N2/2-point
//       DFTs over k2) and its twiddle; to shared memory.
//   I3  thread (c, m2, h): the last inverse step, an N1-point DFT over k1
//       split by parity of k1 between two lanes; only the outputs t < L are
//       formed (the truncation), exchanged by one shuffle round and stored.
// Outputs with t < kHeadT0 are replaced by the direct sum over the first
// kHeadT0 inputs, which the F1 threads stage in shared memory.
#pragma once

#include <cuda_bf16.h>
#include <stdint.h>

#include "fft_reg.cuh"

namespace ccv {

constexpr int kHeadT0 = 32;

template <typename IO>
struct IO_t;
template <>
struct IO_t<float> {
    static __device__ __forceinline__ float ld(const float *p) { return __ldg(p); }
    static __device__ __forceinline__ void st(float *p, float x) { *p = x; }
};
template <>
struct IO_t<__nv_bfloat16> {
    static __device__ __forceinline__ float ld(const __nv_bfloat16 *p) { return __bfloat162float(__ldg(p)); }
    static __device__ __forceinline__ void st(__nv_bfloat16 *p, float x) { *p = __float2bfloat16_rn(x); }
};

template <int N2_, int ROWS_>
struct FusedCfg {
    static constexpr int N2 = N2_;
    static constexpr int ROWS = ROWS_;
    static constexpr int N1 = 2 * N2;
    static constexpr int N = N1 * N2;
    static constexpr int M2 = N2 / 2;
    static constexpr int LOG_N2 = ilog2(N2);
    static constexpr int LOG_M2 = ilog2(M2);
    static constexpr int THREADS = ROWS * N2;
    // Shared-memory strides in float2 units.  With 8-byte accesses a
    // half-warp is conflict-free when its 16 lanes hit distinct (word mod 16):
    // SF_N = 1 (mod 16) serves the F1 stores / F3 loads, SI_M = 2 (mod 16) and
    // SC = 16/ROWS (mod 16) serve the F3 stores / I3 loads.
    static constexpr int SF_N = N1 + 1;
    static constexpr int SI_M = N1 + 2;
    static constexpr int SC = N + N2 + 16 / ROWS;
    static constexpr int HEAD = kHeadT0;
    static constexpr size_t SMEM_BYTES = (size_t)ROWS * SC * 8 + (size_t)ROWS * HEAD * 8;
    // Twiddle table layout (float2, built on the host in fp64):
    //   T1[k1*N2 + n2]        = omega_N^(n2 k1)          k1 < N1, n2 < N2
    //   P [N + k2*N1 + k1]    = omega_N^-(k1 + N1 k2)    k2 < M2
    //   Q [N + N/2 + m2*N1 + k1] = omega_M^-(k1 m2)      m2 < M2   (M = N/2)
    static constexpr int TW_P = N;
    static constexpr int TW_Q = N + N / 2;
    static constexpr int TW_SIZE = 2 * N;
    static_assert(N2 % 16 == 0 && N1 <= 64, "register DFT sizes 16..32 supported");
    static_assert(SC >= N2 * SF_N && SC >= M2 * SI_M, "exchange buffers must fit the row stride");
    static_assert(16 % ROWS == 0 && (32 / ROWS) % 2 == 0, "ROWS must divide 16");
    static_assert(HEAD % 2 == 0 && HEAD <= 2 * N2 * N2, "head must fit in a row");
};

// X' = -i (Zk + conj Zn)(Zk - conj Zn) = 4 * V_k * G_k for z = v + i g.
__device__ __forceinline__ float2 spectral_product(float2 zk, float2 zn) {
    const float px = zk.x + zn.x, py = zk.y - zn.y;  // Zk + conj(Zn)
    const float qx = zk.x - zn.x, qy = zk.y + zn.y;  // Zk - conj(Zn)
    const float re = fmaf(px, qx, -py * qy);
    const float im = fmaf(px, qy, py * qx);
    return make_float2(im, -re);
}

// Real-inverse packing for a bin k and its partner M - k:
//   E = X_k + conj X_{M-k},  O = X_k - conj X_{M-k},  C = E + i w O,
// with w = omega_N^-k.  Returns C for k; the partner's C is
//   conj(E) - i w_p conj(O)   (written by pack_partner).
__device__ __forceinline__ void pack_pair(float2 xk, float2 xp, float2 wk, float2 wp, float2 &ck, float2 &cp) {
    const float ex = xk.x + xp.x, ey = xk.y - xp.y;
    const float ox = xk.x - xp.x, oy = xk.y + xp.y;
    // C_k = E + i (wk * O):  i*(a+ib) = -b + ia
    ck.x = ex - fmaf(wk.x, oy, wk.y * ox);
    ck.y = ey + fmaf(wk.x, ox, -wk.y * oy);
    // partner: E' = conj(E) = (ex, -ey), O' = -conj(O) = (-ox, oy)
    cp.x = ex - fmaf(wp.x, oy, -wp.y * ox);
    cp.y = -ey + fmaf(-wp.x, ox, -wp.y * oy);
}
// Self-paired bin (partner == k): only C_k.
__device__ __forceinline__ float2 pack_self(float2 xk, float2 xp, float2 wk) {
    const float ex = xk.x + xp.x, ey = xk.y - xp.y;
    const float ox = xk.x - xp.x, oy = xk.y + xp.y;
    return make_float2(ex - fmaf(wk.x, oy, wk.y * ox), ey + fmaf(wk.x, ox, -wk.y * oy));
}

template <int N2, int ROWS, int MINB, typename IO>
__global__ void __launch_bounds__(ROWS *N2, MINB)
    fftconv_fused_kernel(const IO *__restrict__ v, const IO *__restrict__ g, IO *__restrict__ r, int L, int D,
                         int groups_per_batch, const float2 *__restrict__ tw) {
    using C = FusedCfg<N2, ROWS>;
    constexpr int N1 = C::N1, N = C::N, M2 = C::M2, SC = C::SC, SF_N = C::SF_N, SI_M = C::SI_M;
    constexpr int HEAD = C::HEAD;
    extern __shared__ float4 smem_raw[];
    float2 *xs = reinterpret_cast<float2 *>(smem_raw);
    float2 *head = xs + ROWS * SC;

    const int tid = threadIdx.x;
    const int b = blockIdx.x / groups_per_batch;
    const int d0 = (blockIdx.x - b * groups_per_batch) * ROWS;
    const int64_t boff = (int64_t)b * L * D;

    // ---------------------------------------------------------------- F1
    {
        const int c = tid % ROWS, n2 = tid / ROWS;
        const int d = d0 + c;
        const bool dok = d < D;
        const IO *vp = v + boff + d;
        const IO *gp = g + boff + d;
        float2 z[N2];
#pragma unroll
        for (int n1 = 0; n1 < N2; ++n1) {
            const int t = n2 + N2 * n1;
            float a = 0.f, q = 0.f;
            if (dok && t < L) {
                a = IO_t<IO>::ld(vp + (int64_t)t * D);
                q = IO_t<IO>::ld(gp + (int64_t)t * D);
            }
            z[bitrev(n1, C::LOG_N2)] = make_float2(a, q);
        }
#pragma unroll
        for (int n1 = 0; n1 * N2 < HEAD; ++n1) head[c * HEAD + n2 + N2 * n1] = z[bitrev(n1, C::LOG_N2)];

        float2 y[N2];
#pragma unroll
        for (int n = 0; n < N2; ++n) {
            const int p = bitrev(n, C::LOG_N2);
            y[p] = (n == 0) ? z[p] : cmul(z[p], tw_const(n, N1));
        }
        float2 *xrow = xs + c * SC + n2 * SF_N;
        const float2 *t1 = tw + n2;
        fft_dit<N2, false>(y);  // odd k1 = 2k'+1
#pragma unroll
        for (int kp = 0; kp < N2; ++kp) xrow[2 * kp + 1] = cmul(y[kp], __ldg(t1 + (2 * kp + 1) * N2));
        fft_dit<N2, false>(z);  // even k1 = 2k'
        xrow[0] = z[0];
#pragma unroll
        for (int kp = 1; kp < N2; ++kp) xrow[2 * kp] = cmul(z[kp], __ldg(t1 + (2 * kp) * N2));
    }
    __syncthreads();

    // ---------------------------------------------------------------- F3
    {
        const int c = tid / N2, j = tid % N2;
        float2 *xrow = xs + c * SC;
        const int ka = j;
        const int kb = (j == 0) ? N1 / 2 : N1 - j;
        float2 A[N2], Bc[N2];
#pragma unroll
        for (int n2 = 0; n2 < N2; ++n2) {
            A[bitrev(n2, C::LOG_N2)] = xrow[n2 * SF_N + ka];
            Bc[bitrev(n2, C::LOG_N2)] = xrow[n2 * SF_N + kb];
        }
        fft_dit<N2, false>(A);  // A[k2]  = Z[ka + N1 k2]
        fft_dit<N2, false>(Bc);  // Bc[k2] = Z[kb + N1 k2]

        const float2 *ptab = tw + C::TW_P;
        if (j != 0) {
            // mirror of (ka, k2) is (kb, N2-1-k2)
#pragma unroll
            for (int k2 = 0; k2 < N2; ++k2) {
                const float2 x = spectral_product(A[k2], Bc[N2 - 1 - k2]);
                A[k2] = x;
                Bc[N2 - 1 - k2] = cconj(x);
            }
            // half-length partner of (ka, k2) is (kb, M2-1-k2)
#pragma unroll
            for (int k2 = 0; k2 < M2; ++k2) {
                float2 ca, cb;
                pack_pair(A[k2], Bc[M2 - 1 - k2], __ldg(ptab + k2 * N1 + ka), __ldg(ptab + (M2 - 1 - k2) * N1 + kb),
                          ca, cb);
                A[k2] = ca;
                Bc[M2 - 1 - k2] = cb;
            }
        } else {
            // column 0: mirror of row k2 is row (N2-k2) mod N2; column N1/2: N2-1-k2
#pragma unroll
            for (int k2 = 0; k2 <= N2 / 2; ++k2) {
                const int p = (N2 - k2) % N2;
                const float2 x = spectral_product(A[k2], A[p]);
                A[k2] = x;
                if (p != k2) A[p] = cconj(x);
            }
#pragma unroll
            for (int k2 = 0; k2 < N2 / 2; ++k2) {
                const float2 x = spectral_product(Bc[k2], Bc[N2 - 1 - k2]);
                Bc[k2] = x;
                Bc[N2 - 1 - k2] = cconj(x);
            }
            // column 0: partner of row k2 is row M2-k2 (row M2 holds X_M)
            {
                const float2 c0 = pack_self(A[0], A[M2], make_float2(1.f, 0.f));
#pragma unroll
                for (int k2 = 1; k2 <= M2 / 2; ++k2) {
                    const int p = M2 - k2;
                    if (p == k2) {
                        A[k2] = pack_self(A[k2], A[k2], __ldg(ptab + k2 * N1));
                    } else {
                        float2 ca, cp;
                        pack_pair(A[k2], A[p], __ldg(ptab + k2 * N1), __ldg(ptab + p * N1), ca, cp);
                        A[k2] = ca;
                        A[p] = cp;
                    }
                }
                A[0] = c0;
            }
            // column N1/2: partner of row k2 is row M2-1-k2
#pragma unroll
            for (int k2 = 0; k2 < M2 / 2; ++k2) {
                float2 ca, cp;
                pack_pair(Bc[k2], Bc[M2 - 1 - k2], __ldg(ptab + k2 * N1 + N1 / 2),
                          __ldg(ptab + (M2 - 1 - k2) * N1 + N1 / 2), ca, cp);
                Bc[k2] = ca;
                Bc[M2 - 1 - k2] = cp;
            }
        }

        // first inverse step: M2-point DFT over k2 for both columns
        float2 ya[M2], yb[M2];
#pragma unroll
        for (int k2 = 0; k2 < M2; ++k2) {
            ya[bitrev(k2, C::LOG_M2)] = A[k2];
            yb[bitrev(k2, C::LOG_M2)] = Bc[k2];
        }
        fft_dit<M2, true>(ya);
        fft_dit<M2, true>(yb);
        const float2 *qtab = tw + C::TW_Q;
        __syncwarp();  // the inverse buffer aliases this row's forward buffer
        xrow[ka] = ya[0];
        xrow[kb] = yb[0];
#pragma unroll
        for (int m2 = 1; m2 < M2; ++m2) {
            xrow[m2 * SI_M + ka] = cmul(ya[m2], __ldg(qtab + m2 * N1 + ka));
            xrow[m2 * SI_M + kb] = cmul(yb[m2], __ldg(qtab + m2 * N1 + kb));
        }
    }
    __syncthreads();

    // ---------------------------------------------------------------- I3
    {
        const int c = tid % ROWS, u = tid / ROWS;
        const int m2 = u >> 1, h = u & 1;
        const float2 *xi = xs + c * SC + m2 * SI_M + h;
        float2 x[N2];
#pragma unroll
        for (int i = 0; i < N2; ++i) x[bitrev(i, C::LOG_N2)] = xi[2 * i];
        fft_dit<N2, true>(x);
        if (h) {
#pragma unroll
            for (int m1 = 1; m1 < N2; ++m1) x[m1] = cmul_conj(x[m1], tw_const(m1, N1));
        }
        const int d = d0 + c;
        const bool dok = d < D;
        IO *rp = r + boff + d;
        const float s = 1.f / (4.f * (float)N);
        const float2 *hrow = head + c * HEAD;
#pragma unroll
        for (int i = 0; i < N2 / 2; ++i) {
            const float2 send = h ? x[i] : x[N2 / 2 + i];
            const float2 own = h ? x[N2 / 2 + i] : x[i];
            float2 o;
            o.x = own.x + __shfl_xor_sync(0xffffffffu, send.x, ROWS);
            o.y = own.y + __shfl_xor_sync(0xffffffffu, send.y, ROWS);
            const int m1 = i + h * (N2 / 2);
            const int t = 2 * m2 + N2 * m1;
            float r0 = o.x * s, r1 = o.y * s;
            if (i * N2 < HEAD && t < HEAD) {
                // direct sums for the first outputs
                float a0 = 0.f, a1 = 0.f;
                for (int jj = 0; jj <= t; ++jj) {
                    const float vj = hrow[jj].x;
                    a0 = fmaf(vj, hrow[t - jj].y, a0);
                    a1 = fmaf(vj, hrow[t + 1 - jj].y, a1);
                }
                a1 = fmaf(hrow[t + 1].x, hrow[0].y, a1);
                r0 = a0;
                r1 = a1;
            }
            if (dok && t < L) IO_t<IO>::st(rp + (int64_t)t * D, r0);
            if (dok && t + 1 < L) IO_t<IO>::st(rp + (int64_t)(t + 1) * D, r1);
        }
    }
}

}  // namespace ccv
