// fftconv_fused.cuh -- fused pad -> FFT -> multiply -> inverse FFT -> truncate
// kernel, persistent over tiles of ROWS channels of one batch, whole rows on
// chip.
//
// Method (Caracal: Causal Architecture via Spectral Mixing, "Key design 1"
// and "Key design 2"): each (b, d) row of v (value stream) and g (gate
// stream) is zero-padded to N >= 2L, transformed, multiplied pointwise,
// inverse-transformed and truncated to L, which equals
// r_t = sum_{j<=t} v_j g_{t-j}.  The real-FFT halving suggested in the
// limitations section ("use RFFT to halve compute") is realised twice:
//   * forward: one complex transform of z = v + i g per row; V and G are
//     separated from mirrored bins of Z;
//   * inverse: the real length-N output comes from one complex transform of
//     length M = N/2 whose output is r[2m] + i r[2m+1].
//
// Odd-frequency transform.  The kernel evaluates the spectrum at the odd
// frequencies (k + 1/2): Z_k = sum_n z_n theta^(n(2k+1)), theta = exp(-i pi/N),
// i.e. the DFT of z_n theta^n.  Pointwise products of such spectra give the
// negacyclic convolution of length N, which equals the linear one here because
// the padding leaves at least L-1 trailing zeros.  The point of the shift is
// the mirror structure: for a real sequence the bin paired with k is N-1-k,
// never k itself, so every thread owns two mirror-image columns and no lane
// needs a special case.  The twist theta^n and the untwist fold into the
// twiddle tables, except for two constant per-element rotations.
//
// Decomposition (N = N1 * N2, N1 = 2 * N2, one shared-memory exchange per
// transform), n = n2 + N2 n1, k = k1 + N1 k2:
//   F1  thread (c, n2): sum over n1 of z[n2 + N2 n1] omega_2N1^(n1 (2 k1+1));
//       half the inputs are padding zeros, so it is two N2-point DFTs (even and
//       odd k1) of z times a constant rotation; times omega_2N^(n2 (2 k1+1)).
//   F3  thread (c, j) owns columns j and N1-1-j: N2-point DFTs over n2, the
//       spectral product (mirror of row k2 is row N2-1-k2 of the other
//       column), the real-inverse packing (partner of row k2 is row M2-1-k2 of
//       the other column), the first inverse step (M2 = N2/2-point DFTs over
//       k2) and its twiddle.
//   I3  thread (c, m2, h): the last inverse step, an N1-point DFT over k1
//       split by the parity h of k1 between two lanes; only outputs t < L are
//       formed (the truncation), exchanged by one shuffle round and stored.
// Outputs with t < kHeadT0 are replaced by the direct sum over the first
// kHeadT0 inputs.
//
// Pipeline: each CTA loops over tiles; the next tile's v and g are copied
// into a staging buffer with cp.async while the current tile runs F3 and I3.
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
    static __device__ __forceinline__ float cvt(float x) { return x; }
    static __device__ __forceinline__ void st(float *p, float x) { *p = x; }
};
template <>
struct IO_t<__nv_bfloat16> {
    static __device__ __forceinline__ __nv_bfloat16 ld(const __nv_bfloat16 *p) { return __ldg(p); }
    static __device__ __forceinline__ float cvt(__nv_bfloat16 x) { return __bfloat162float(x); }
    static __device__ __forceinline__ void st(__nv_bfloat16 *p, float x) { *p = __float2bfloat16_rn(x); }
};

template <int N2_, int ROWS_, typename IO>
struct FusedCfg {
    static constexpr int N2 = N2_;
    static constexpr int ROWS = ROWS_;
    static constexpr int N1 = 2 * N2;
    static constexpr int N = N1 * N2;
    static constexpr int LMAX = N / 2;
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
    // staging: [LMAX][ROWS] elements of IO for v, then for g
    static constexpr size_t XBYTES = (size_t)ROWS * SC * 8;
    static constexpr size_t HBYTES = (size_t)ROWS * HEAD * 8;
    static constexpr size_t SBYTES = (size_t)2 * LMAX * ROWS * sizeof(IO);
    static constexpr int NWARPS = THREADS / 32;
    static constexpr size_t RBYTES = (size_t)(NWARPS * ROWS + ROWS) * 8;  // norm partials, per-row scale
    static constexpr size_t SMEM_BYTES = XBYTES + HBYTES + SBYTES + RBYTES;
    // Twiddle table layout (float2, built on the host in fp64), theta = omega_2N:
    //   T1[k1*N2 + n2]           = theta^(n2 (2 k1 + 1))         k1 < N1, n2 < N2
    //   P [N + k2*N1 + k1]       = theta^-(2 (k1 + N1 k2) + 1)   k2 < M2
    //   Q [N + N/2 + m2*N1 + k1] = theta^-(2 m2 (2 k1 + 1))      m2 < M2
    static constexpr int TW_P = N;
    static constexpr int TW_Q = N + N / 2;
    static constexpr int TW_SIZE = 2 * N;
    static_assert(N2 % 16 == 0 && N1 <= 64, "register DFT sizes 16..32 supported");
    static_assert(SC >= N2 * SF_N && SC >= M2 * SI_M, "exchange buffers must fit the row stride");
    static_assert(16 % ROWS == 0 && (32 / ROWS) % 2 == 0, "ROWS must divide 16");
    static_assert(HEAD % N2 == 0 && HEAD <= LMAX, "head must be whole n1 blocks of a row");
    // bytes per t per array in staging, and the cp.async chunk covering them
    static constexpr int CH = ROWS * (int)sizeof(IO);
    static constexpr int CHUNK = CH < 16 ? CH : 16;
    static constexpr int NCHUNK = CH / CHUNK;
    static_assert(CH % CHUNK == 0 && (CHUNK == 4 || CHUNK == 8 || CHUNK == 16), "staging chunking");
    static_assert((XBYTES + HBYTES) % 16 == 0 && (LMAX * CH) % 16 == 0, "staging must be 16-byte aligned");
};

// X' = -i (Zk + conj Zm)(Zk - conj Zm) = 4 V_k G_k for z = v + i g, Zm = mirror bin.
__device__ __forceinline__ float2 spectral_product(float2 zk, float2 zm) {
    const float px = zk.x + zm.x, py = zk.y - zm.y;  // Zk + conj(Zm)
    const float qx = zk.x - zm.x, qy = zk.y + zm.y;  // Zk - conj(Zm)
    const float re = fmaf(px, qx, -py * qy);
    const float im = fmaf(px, qy, py * qx);
    return make_float2(im, -re);
}

// Real-inverse packing for a bin k and its partner p:
//   E = X_k + conj X_p,  O = X_k - conj X_p,  C_k = E + i w_k O,
// and for the partner (whose own partner is k): E_p = conj(E), O_p = -conj(O).
__device__ __forceinline__ void pack_pair(float2 xk, float2 xp, float2 wk, float2 wp, float2 &ck, float2 &cp) {
    const float ex = xk.x + xp.x, ey = xk.y - xp.y;
    const float ox = xk.x - xp.x, oy = xk.y + xp.y;
    ck.x = ex - fmaf(wk.x, oy, wk.y * ox);
    ck.y = ey + fmaf(wk.x, ox, -wk.y * oy);
    cp.x = ex - fmaf(wp.x, oy, -wp.y * ox);
    cp.y = -ey + fmaf(-wp.x, ox, -wp.y * oy);
}

__device__ __forceinline__ void cp_async16(void *smem, const void *gmem) {
    const unsigned s = (unsigned)__cvta_generic_to_shared(smem);
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;\n" ::"r"(s), "l"(gmem) : "memory");
}
__device__ __forceinline__ void cp_async8(void *smem, const void *gmem) {
    const unsigned s = (unsigned)__cvta_generic_to_shared(smem);
    asm volatile("cp.async.ca.shared.global [%0], [%1], 8;\n" ::"r"(s), "l"(gmem) : "memory");
}
__device__ __forceinline__ void cp_async4(void *smem, const void *gmem) {
    const unsigned s = (unsigned)__cvta_generic_to_shared(smem);
    asm volatile("cp.async.ca.shared.global [%0], [%1], 4;\n" ::"r"(s), "l"(gmem) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;\n" ::: "memory"); }
__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_all;\n" ::: "memory"); }

// Issue the copies of one tile's v and g (t < L, channels d0..d0+ROWS-1 that
// exist) into staging [t][c].  `vec` selects whole-row chunks (requires the
// chunk to be aligned, i.e. D*sizeof(IO) a multiple of ROWS*sizeof(IO) and a
// full channel group); otherwise element-wise copies (4-byte elements) or
// plain loads (2-byte elements) are used.
template <class C, typename IO>
__device__ __forceinline__ void stage_tile(const IO *__restrict__ v, const IO *__restrict__ g, IO *sv, IO *sg,
                                           int64_t boff, int d0, int L, int D, bool vec) {
    constexpr int ROWS = C::ROWS;
    const int tid = threadIdx.x;
    const IO *vb = v + boff + d0;
    const IO *gb = g + boff + d0;
    if (vec) {
        constexpr int EPC = C::CHUNK / (int)sizeof(IO);  // elements per chunk
        for (int e = tid; e < L * C::NCHUNK; e += C::THREADS) {
            const int t = e / C::NCHUNK, q = e - t * C::NCHUNK;
            const int64_t o = (int64_t)t * D + q * EPC;
            IO *dv = sv + t * ROWS + q * EPC;
            IO *dg = sg + t * ROWS + q * EPC;
            if (C::CHUNK == 16) {
                cp_async16(dv, vb + o);
                cp_async16(dg, gb + o);
            } else if (C::CHUNK == 8) {
                cp_async8(dv, vb + o);
                cp_async8(dg, gb + o);
            } else {
                cp_async4(dv, vb + o);
                cp_async4(dg, gb + o);
            }
        }
    } else {
        const int nc = min(ROWS, D - d0);
        for (int e = tid; e < L * ROWS; e += C::THREADS) {
            const int t = e / ROWS, c = e - t * ROWS;
            if (c < nc) {
                const int64_t o = (int64_t)t * D + c;
                if (sizeof(IO) == 4) {
                    cp_async4(sv + e, vb + o);
                    cp_async4(sg + e, gb + o);
                } else {
                    sv[e] = IO_t<IO>::ld(vb + o);
                    sg[e] = IO_t<IO>::ld(gb + o);
                }
            }
        }
    }
    cp_async_commit();
}

template <int N2, int ROWS, int MINB, typename IO>
__global__ void __launch_bounds__(ROWS *N2, MINB)
    fftconv_fused_kernel(const IO *__restrict__ v, const IO *__restrict__ g, IO *__restrict__ r, int L, int D,
                         int groups_per_batch, int num_tiles, int vec_ok, const float2 *__restrict__ tw) {
    using C = FusedCfg<N2, ROWS, IO>;
    constexpr int N1 = C::N1, N = C::N, M2 = C::M2, SC = C::SC, SF_N = C::SF_N, SI_M = C::SI_M;
    constexpr int HEAD = C::HEAD, LMAX = C::LMAX;
    extern __shared__ float4 smem_raw[];
    float2 *xs = reinterpret_cast<float2 *>(smem_raw);
    float2 *head = xs + ROWS * SC;
    IO *sv = reinterpret_cast<IO *>(head + ROWS * HEAD);
    IO *sg = sv + LMAX * ROWS;
    float2 *red = reinterpret_cast<float2 *>(sg + LMAX * ROWS);  // [NWARPS][ROWS] partial norms
    float *alpha_row = reinterpret_cast<float *>(red + C::NWARPS * ROWS);  // [ROWS] balance scale
    const int tid = threadIdx.x;

    int tile = blockIdx.x;
    if (tile >= num_tiles) return;
    {
        const int b = tile / groups_per_batch, d0 = (tile - b * groups_per_batch) * ROWS;
        stage_tile<C, IO>(v, g, sv, sg, (int64_t)b * L * D, d0, L, D, vec_ok && d0 + ROWS <= D);
    }

    for (; tile < num_tiles; tile += gridDim.x) {
        const int b = tile / groups_per_batch;
        const int d0 = (tile - b * groups_per_batch) * ROWS;
        const int64_t boff = (int64_t)b * L * D;
        cp_async_wait_all();
        __syncthreads();  // staging complete; previous tile's I3 done with xs / head

        // ------------------------------------------------------------ F1
        {
            const int c = tid % ROWS, n2 = tid / ROWS;
#pragma unroll
            for (int n1 = 0; n1 * N2 < HEAD; ++n1) {
                const int t = n2 + N2 * n1;
                const bool ok = t < L;
                head[c * HEAD + t] = make_float2(ok ? IO_t<IO>::cvt(sv[t * ROWS + c]) : 0.f,
                                                 ok ? IO_t<IO>::cvt(sg[t * ROWS + c]) : 0.f);
            }
            // this thread's inputs z[n2 + N2 n1] and the row's stream norms
            float2 zr[N2];
            float nv = 0.f, ng = 0.f;
#pragma unroll
            for (int n1 = 0; n1 < N2; ++n1) {
                const int t = n2 + N2 * n1;
                float2 zv = make_float2(0.f, 0.f);
                if (t < L) zv = make_float2(IO_t<IO>::cvt(sv[t * ROWS + c]), IO_t<IO>::cvt(sg[t * ROWS + c]));
                zr[n1] = zv;
                nv = fmaf(zv.x, zv.x, nv);
                ng = fmaf(zv.y, zv.y, ng);
            }
#pragma unroll
            for (int m = ROWS; m < 32; m <<= 1) {
                nv += __shfl_xor_sync(0xffffffffu, nv, m);
                ng += __shfl_xor_sync(0xffffffffu, ng, m);
            }
            if ((tid & 31) < ROWS) red[(tid >> 5) * ROWS + c] = make_float2(nv, ng);
            __syncthreads();
            float2 tot = make_float2(0.f, 0.f);
#pragma unroll
            for (int w = 0; w < C::NWARPS; ++w) {
                tot.x += red[w * ROWS + c].x;
                tot.y += red[w * ROWS + c].y;
            }
            const float alpha = balance_scale(tot.x, tot.y);
            if (n2 == 0) alpha_row[c] = alpha;
#pragma unroll
            for (int n1 = 0; n1 < N2; ++n1) zr[n1].y *= alpha;

            float2 *xrow = xs + c * SC + n2 * SF_N;
            const float2 *t1 = tw + n2;
#pragma unroll 1
            for (int e = 0; e < 2; ++e) {
                // x[n1] = z[n2 + N2 n1] * omega_2N1^((2e+1) n1), in bit-reversed slots
                float2 x[N2];
#pragma unroll
                for (int n1 = 0; n1 < N2; ++n1) {
                    const float2 zv = zr[n1];
                    const float2 w = e ? tw_const(3 * n1, 2 * N1) : tw_const(n1, 2 * N1);
                    x[bitrev(n1, C::LOG_N2)] = n1 == 0 ? zv : cmul(zv, w);
                }
                fft_dit<N2, false>(x);  // x[k'] -> k1 = 2k' + e
#pragma unroll
                for (int kp = 0; kp < N2; ++kp) {
                    const int k1 = 2 * kp + e;
                    xrow[k1] = cmul(x[kp], __ldg(t1 + k1 * N2));
                }
            }
        }
        __syncthreads();  // exchange complete; staging free

        // prefetch the next tile while this one finishes
        {
            const int nt = tile + gridDim.x;
            if (nt < num_tiles) {
                const int nb = nt / groups_per_batch, nd0 = (nt - nb * groups_per_batch) * ROWS;
                stage_tile<C, IO>(v, g, sv, sg, (int64_t)nb * L * D, nd0, L, D, vec_ok && nd0 + ROWS <= D);
            }
        }

        // ------------------------------------------------------------ F3
        {
            const int c = tid / N2, j = tid % N2;
            float2 *xrow = xs + c * SC;
            const int ka = j, kb = N1 - 1 - j;
            float2 A[N2], Bc[N2];
#pragma unroll
            for (int n2 = 0; n2 < N2; ++n2) {
                A[bitrev(n2, C::LOG_N2)] = xrow[n2 * SF_N + ka];
                Bc[bitrev(n2, C::LOG_N2)] = xrow[n2 * SF_N + kb];
            }
            fft_dit<N2, false>(A);   // A[k2]  = Z[ka + N1 k2]
            fft_dit<N2, false>(Bc);  // Bc[k2] = Z[kb + N1 k2]
            // mirror of (ka, k2) is (kb, N2-1-k2)
#pragma unroll
            for (int k2 = 0; k2 < N2; ++k2) {
                const float2 x = spectral_product(A[k2], Bc[N2 - 1 - k2]);
                A[k2] = x;
                Bc[N2 - 1 - k2] = cconj(x);
            }
            // half-length partner of (ka, k2) is (kb, M2-1-k2)
            const float2 *ptab = tw + C::TW_P;
#pragma unroll
            for (int k2 = 0; k2 < M2; ++k2) {
                float2 ca, cb;
                pack_pair(A[k2], Bc[M2 - 1 - k2], __ldg(ptab + k2 * N1 + ka), __ldg(ptab + (M2 - 1 - k2) * N1 + kb),
                          ca, cb);
                A[k2] = ca;
                Bc[M2 - 1 - k2] = cb;
            }
            // first inverse step: M2-point DFT over k2, then its twiddle
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
#pragma unroll
            for (int m2 = 0; m2 < M2; ++m2) {
                xrow[m2 * SI_M + ka] = cmul(ya[m2], __ldg(qtab + m2 * N1 + ka));
                xrow[m2 * SI_M + kb] = cmul(yb[m2], __ldg(qtab + m2 * N1 + kb));
            }
        }
        __syncthreads();

        // ------------------------------------------------------------ I3
        {
            const int c = tid % ROWS, u = tid / ROWS;
            const int m2 = u >> 1, h = u & 1;
            const float2 *xi = xs + c * SC + m2 * SI_M + h;
            float2 x[N2];
#pragma unroll
            for (int i = 0; i < N2; ++i) x[bitrev(i, C::LOG_N2)] = xi[2 * i];
            fft_dit<N2, true>(x);
            // untwist and odd-k1 rotation: times omega_2N1^-((2h+1) m1)
#pragma unroll
            for (int m1 = 1; m1 < N2; ++m1) {
                const float2 w = h ? tw_const(3 * m1, 2 * N1) : tw_const(m1, 2 * N1);
                x[m1] = cmul_conj(x[m1], w);
            }
            const int d = d0 + c;
            const bool dok = d < D;
            IO *rp = r + boff + d;
            const float s = 1.f / (4.f * (float)N * alpha_row[c]);
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
    cp_async_wait_all();
}

}  // namespace ccv
