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
// into a staging buffer while the current tile runs F3 and I3.  The copy is a
// handful of TMA boxes issued by one thread (completion counted on an
// mbarrier; the copy engine zero-fills t >= L and d >= D) whenever the tensors
// allow a tensor map (16-byte aligned base and row pitch); a staged row is
// widened to 16 bytes where the tile's is narrower (bf16 tiles of 4 channels
// stage 8 and read their half).  Otherwise the threads issue cp.async pieces.
// The backward pass reads v reversed in time: the staging keeps natural
// order and the reversal happens on the shared-memory reads.
#pragma once

#include <cuda_bf16.h>
#include <stdint.h>

#include "fft_reg.cuh"
#include "tma.cuh"

namespace ccv {

constexpr int kHeadT0 = 32;

// F1 input twist omega_2N1^((2e+1) n1) for N2 = 16 (N1 = 32) and N2 = 32
// (N1 = 64): c_f1_twist[N2 == 32][e][n1], n1 < N2; filled once per device.
__constant__ float2 c_f1_twist[2][2][32];

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
    static constexpr int H = N2 / 2;   // half column (first radix-2 split)
    static constexpr int MH = M2 / 2;  // half of the inverse column
    static constexpr int LOG_N2 = ilog2(N2);
    static constexpr int LOG_H = ilog2(H);
    static constexpr int LOG_MH = ilog2(MH);
    static constexpr int THREADS = ROWS * 2 * N2;  // two threads per (row, n2) / column pair / (m2, h)
    static constexpr int NWARPS = THREADS / 32;
    // Shared-memory strides in float2 units.  With 8-byte accesses a
    // half-warp is conflict-free when its 16 lanes hit distinct (word mod 16):
    // SF_N = 1 (mod 16) serves the F1 stores / F3 loads, SI_M = 2 (mod 16) and
    // SC = 16/ROWS (mod 16) serve the F3 stores / I3 loads.
    // With ROWS = 2 a half-warp of I3 also spans two m2 rows, which then
    // need SI_M = 4 (mod 16).
    static constexpr int SF_N = N1 + 1;
    static constexpr int SI_M = N1 + (ROWS == 2 ? 4 : 2);
    static constexpr int SC = N + N2 + 16 / ROWS;
    static constexpr int HEAD = kHeadT0;
    // the direct head of each row is split over HP warps by ranges of j
    static constexpr int HP = NWARPS / ROWS;
    static constexpr size_t XBYTES = (size_t)ROWS * SC * 8;
    static constexpr size_t HBYTES = ((size_t)ROWS * HP * HEAD * 4 + 15) / 16 * 16;  // [ROWS][HP][HEAD] partial sums
    // staging: [LMAX][ROWS] elements of IO for v, then for g
    // staged channels per time step: the tile's ROWS, widened to a whole
    // 16-byte TMA box row (bf16 tiles of 4 channels stage 8; the tile's
    // channels sit at offset d0 % SW of the row)
    static constexpr int SW = ROWS * (int)sizeof(IO) >= 16 ? ROWS : 16 / (int)sizeof(IO);
    static constexpr size_t SBYTES = (size_t)2 * LMAX * SW * sizeof(IO);
    // norm partials [NWARPS][ROWS] float2, per-row scale [ROWS] float (padded),
    // rotations [(2h+s)][H+1] float2 (padded so the four (h, s) lane groups hit distinct banks)
    static constexpr size_t RBYTES = (size_t)(NWARPS * ROWS) * 8 + (size_t)ROWS * 8 + (size_t)4 * (N2 / 2 + 1) * 8;
    // staging starts on a 128-byte boundary (TMA destination)
    static constexpr size_t SOFF = (XBYTES + HBYTES + 127) / 128 * 128;
    // + one mbarrier (8 bytes, padded)
    static constexpr size_t SMEM_BYTES = SOFF + SBYTES + RBYTES + 16;
    // TMA staging: boxes of [BOXT t][SW d]; a box row must be a multiple of 16 bytes
    static constexpr bool TMA_OK = (SW * sizeof(IO)) % 16 == 0;
    static constexpr int BOXT = LMAX < 256 ? LMAX : 256;
    static constexpr int NBOX = LMAX / BOXT;
    static constexpr unsigned STAGE_BYTES = (unsigned)SBYTES;
    // Twiddle table layout (float2, built on the host in fp64), theta = omega_2N:
    //   T1[k1*N2 + n2]           = theta^(n2 (2 k1 + 1))         k1 < N1, n2 < N2
    //   P [N + k2*N1 + k1]       = theta^-(2 (k1 + N1 k2) + 1)   k2 < M2
    //   Q [N + N/2 + m2*N1 + k1] = theta^-(2 m2 (2 k1 + 1))      m2 < M2
    static constexpr int TW_P = N;
    static constexpr int TW_Q = N + N / 2;
    static constexpr int TW_SIZE = 2 * N;
    static_assert(N2 == 16 || N2 == 32, "register DFT sizes 16..32 supported");
    static_assert(THREADS == 128 || THREADS == 256 || THREADS == 512, "lane maps assume 4, 8 or 16 warps per CTA");
    static_assert(NWARPS % ROWS == 0 && HEAD % HP == 0, "head split");
    static_assert(SC >= N2 * SF_N && SC >= M2 * SI_M, "exchange buffers must fit the row stride");
    static_assert(16 % ROWS == 0 && 4 * ROWS <= 32, "ROWS must divide 16 and leave room for (h, s) lane bits");
    static_assert(HEAD == 32 && HEAD <= LMAX && HEAD % N2 == 0, "the direct head spans one warp of t");
    // bytes per t per array in staging, and the cp.async chunk covering them
    static constexpr int CH = ROWS * (int)sizeof(IO);
    static constexpr int CHUNK = CH < 16 ? CH : 16;
    static constexpr int NCHUNK = CH / CHUNK;
    static_assert(CH % CHUNK == 0 && (CHUNK == 4 || CHUNK == 8 || CHUNK == 16), "staging chunking");
    static_assert(SW % ROWS == 0 && (LMAX * SW * sizeof(IO)) % 128 == 0 && LMAX % BOXT == 0,
                  "staging boxes must stay 128-byte aligned");
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
    constexpr int ROWS = C::ROWS, SW = C::SW;
    const int coff = d0 % SW;  // the tile's channels within a staged row
    const int tid = threadIdx.x;
    const IO *vb = v + boff + d0;
    const IO *gb = g + boff + d0;
    if (vec) {
        constexpr int EPC = C::CHUNK / (int)sizeof(IO);  // elements per chunk
        for (int e = tid; e < L * C::NCHUNK; e += C::THREADS) {
            const int t = e / C::NCHUNK, q = e - t * C::NCHUNK;
            const int64_t o = (int64_t)t * D + q * EPC;
            IO *dv = sv + t * SW + coff + q * EPC;
            IO *dg = sg + t * SW + coff + q * EPC;
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
                    cp_async4(sv + t * SW + coff + c, vb + o);
                    cp_async4(sg + t * SW + coff + c, gb + o);
                } else {
                    sv[t * SW + coff + c] = IO_t<IO>::ld(vb + o);
                    sg[t * SW + coff + c] = IO_t<IO>::ld(gb + o);
                }
            }
        }
    }
    cp_async_commit();
}

__device__ __forceinline__ float2 shfl_xor2(float2 a, int m) {
    return make_float2(__shfl_xor_sync(0xffffffffu, a.x, m), __shfl_xor_sync(0xffffffffu, a.y, m));
}


template <int N2, int ROWS, int MINB, typename IO, bool REVA>
__global__ void __launch_bounds__(ROWS * 2 * N2, MINB)
    fftconv_fused_kernel(const IO *__restrict__ v, const IO *__restrict__ g, IO *__restrict__ r, int L, int D,
                         int groups_per_batch, int num_tiles, int vec_ok, int rev, const float2 *__restrict__ tw,
                         const __grid_constant__ CUtensorMap tmv, const __grid_constant__ CUtensorMap tmg,
                         int use_tma) {
    // REVA: v is read reversed in time (v_t -> v_{L-1-t}); the staging keeps v
    // in natural order and the reversal happens on the shared-memory reads.
    // rev bit 1: write r reversed.
    // use_tma: stage tiles with TMA boxes from tmv / tmg (3-D maps over {D, L, B}),
    // otherwise with cp.async from the pointers
    using C = FusedCfg<N2, ROWS, IO>;
    constexpr int N1 = C::N1, N = C::N, M2 = C::M2, H = C::H, MH = C::MH;
    const bool rev_out = (rev >> 1) & 1;
    constexpr int SC = C::SC, SF_N = C::SF_N, SI_M = C::SI_M, HEAD = C::HEAD, LMAX = C::LMAX;
    constexpr int THREADS = C::THREADS;
    extern __shared__ float4 smem_raw[];
    float2 *xs = reinterpret_cast<float2 *>(smem_raw);
    float *hres = reinterpret_cast<float *>(xs + ROWS * SC);  // [ROWS][HP][HEAD]: partial direct sums, t < HEAD
    IO *sv = reinterpret_cast<IO *>(reinterpret_cast<char *>(smem_raw) + C::SOFF);
    constexpr int SW = C::SW;
    IO *sg = sv + LMAX * SW;
    float2 *red = reinterpret_cast<float2 *>(sg + LMAX * SW);  // [NWARPS][ROWS] partial norms
    // [ROWS] output scale 1/(4 N alpha), 0 for a row whose v or g is all zero; [ROWS] unused
    float *alpha_row = reinterpret_cast<float *>(red + C::NWARPS * ROWS);
    float2 *rot = reinterpret_cast<float2 *>(alpha_row + 2 * ROWS);       // [2h+s][H+1]
    uint64_t *bar = reinterpret_cast<uint64_t *>(rot + 4 * (H + 1));      // staging-complete barrier
    const int tid = threadIdx.x;
    // v at time t (0 <= t < LMAX) of staged channel cc (tile row + offset in
    // the staged row): v_t, or v_{L-1-t} (0 for t >= L)
    auto v_at = [&](int t, int cc) -> float {
        if constexpr (REVA) {
            const int tr = L - 1 - t;
            const float x = IO_t<IO>::cvt(sv[max(tr, 0) * SW + cc]);
            return tr >= 0 ? x : 0.f;
        } else {
            return IO_t<IO>::cvt(sv[t * SW + cc]);
        }
    };
    const bool tma = C::TMA_OK && use_tma && (smem_u32(sv) & 127) == 0;
    unsigned phase = 0;
    // stage tile `t` (v and g, t < LMAX, zero-filled past L and D) into sv / sg
    auto issue = [&](int t) {
        const int b = t / groups_per_batch, d0 = (t - b * groups_per_batch) * ROWS;
        if (tma) {
            if (tid == 0) {
                fence_proxy_async_smem();
                mbar_arrive_expect_tx(bar, C::STAGE_BYTES);
#pragma unroll
                for (int k = 0; k < C::NBOX; ++k) {
                    tma_load_3d(sv + k * C::BOXT * SW, &tmv, d0 - d0 % SW, k * C::BOXT, b, bar);
                    tma_load_3d(sg + k * C::BOXT * SW, &tmg, d0 - d0 % SW, k * C::BOXT, b, bar);
                }
            }
        } else {
            stage_tile<C, IO>(v, g, sv, sg, (int64_t)b * L * D, d0, L, D, vec_ok && d0 + ROWS <= D);
        }
    };

    // rot[2h+s][m] = omega_2N1^-((2h+1) m1), m1 = H s + m: untwist of the
    // odd-frequency grid times the parity rotation of the last inverse step
    for (int i = tid; i < 4 * H; i += THREADS) {
        const int hs = i / H, m = i - hs * H, hh = hs >> 1, m1 = H * (hs & 1) + m;
        rot[hs * (H + 1) + m] = cconj(c_w128[((2 * hh + 1) * m1 * (128 / (2 * N1))) & 127]);
    }
    if (tma) {
        if (tid == 0) mbar_init(bar, 1);
    } else {
        // staging beyond L is never written by the copies: zero it once so loads need no bounds test
        for (int i = L * SW + tid; i < LMAX * SW; i += THREADS) {
            sv[i] = IO(0.f);
            sg[i] = IO(0.f);
        }
    }
    __syncthreads();

    int tile = blockIdx.x;
    if (tile >= num_tiles) return;
    issue(tile);

    for (; tile < num_tiles; tile += gridDim.x) {
        const int b = tile / groups_per_batch;
        const int d0 = (tile - b * groups_per_batch) * ROWS;
        const int64_t boff = (int64_t)b * L * D;
        bool staged = true;
        if (tma) {
            staged = mbar_wait_bounded(bar, phase);
            phase ^= 1u;
        } else {
            cp_async_wait_all();
        }
        // staging complete; previous tile's I3 done with xs / head
        if (__syncthreads_or(!staged)) {
            // a copy did not complete in time: flag it, give the copies in
            // flight one more bounded wait, and stop
            if (tid == 0) {
                atomicOr(&g_cc_fault, kFaultTmaWait);
                mbar_wait_bounded(bar, phase ^ 1u);
            }
            return;
        }

        // ------------------------------------------------------------ F1
        // thread (e, n2, c): half-spectrum e (k1 = 2k'+e) of column n2 of row c
        {
            const int e = tid / (ROWS * N2);  // warp-uniform
            const int c = tid % ROWS, n2 = (tid / ROWS) % N2;
            const int coff = d0 % SW;  // the tile's channels within a staged row
            float2 zr[N2];
            float nv = 0.f, ng = 0.f;
#pragma unroll
            for (int n1 = 0; n1 < N2; ++n1) {
                const int t = n2 + N2 * n1;
                const float2 zv = make_float2(v_at(t, coff + c), IO_t<IO>::cvt(sg[t * SW + coff + c]));
                zr[n1] = zv;
                nv = fmaf(zv.x, zv.x, nv);
                ng = fmaf(zv.y, zv.y, ng);
            }
            // direct sums r_t = sum_{j<=t} v_j g_{t-j} for t < HEAD: warp w takes
            // row w % ROWS, lane t, and the j range of part w / ROWS
            {
                constexpr int HP = C::HP, JP = HEAD / HP;
                const int w = tid >> 5, hc = w % ROWS, hp = w / ROWS, lt = tid & 31;
                const float vt = v_at(lt, coff + hc);
                const float gt = IO_t<IO>::cvt(sg[lt * SW + coff + hc]);
                float acc = 0.f;
#pragma unroll
                for (int jj = 0; jj < JP; ++jj) {
                    const int j = hp * JP + jj;
                    const float vj = __shfl_sync(0xffffffffu, vt, j);
                    const float gtj = __shfl_up_sync(0xffffffffu, gt, j);
                    if (lt >= j) acc = fmaf(vj, gtj, acc);
                }
                hres[(hc * HP + hp) * HEAD + lt] = acc;
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
            for (int w = 0; w < C::NWARPS / 2; ++w) {  // the e == 0 warps cover each row once
                tot.x += red[w * ROWS + c].x;
                tot.y += red[w * ROWS + c].y;
            }
            const float alpha = balance_scale(tot.x, tot.y);
            // a stream that is all zero makes the row exactly zero (the transform
            // would otherwise spread the other stream's rounding over it)
            if (tid < ROWS) alpha_row[c] = (tot.x > 0.f && tot.y > 0.f) ? 1.f / (4.f * (float)N * alpha) : 0.f;

            // x[n1] = z[n2 + N2 n1] * omega_2N1^((2e+1) n1), in bit-reversed slots.
            // e is warp-uniform: the twist comes from a constant table at a
            // per-warp offset, so both halves share one copy of the code.
            const float2 *twist = c_f1_twist[N2 == 32 ? 1 : 0][e];
            float2 x[N2];
#pragma unroll
            for (int n1 = 0; n1 < N2; ++n1) {
                const float2 zv = make_float2(zr[n1].x, alpha * zr[n1].y);
                x[bitrev(n1, C::LOG_N2)] = n1 == 0 ? zv : cmul(zv, twist[n1]);
            }
            fft_dit<N2, false>(x);  // x[k'] -> k1 = 2k' + e
            float2 *xrow = xs + c * SC + n2 * SF_N + e;
            const float2 *t1 = tw + e * N2 + n2;
#pragma unroll
            for (int kp = 0; kp < N2; ++kp) xrow[2 * kp] = cmul(x[kp], __ldg(t1 + 2 * kp * N2));
        }
        __syncthreads();  // exchange complete; staging free

        // prefetch the next tile while this one finishes
        if (tile + (int)gridDim.x < num_tiles) issue(tile + gridDim.x);

        // ------------------------------------------------------------ F3
        // Column pair (j, N1-1-j) of row c is shared by two lanes s = 0, 1 (lane ^ 16).
        // Lane s keeps the even rows of its own column and receives the odd rows
        // of the other; that set is closed under both pairings (mirror: row k2 of
        // one column with row N2-1-k2 of the other; half-length partner: row k2
        // with row M2-1-k2), so both lanes run the same code.
        {
            const int c = tid / (2 * N2), rr = tid % (2 * N2);
            const int s = (rr >> 4) & 1, j = (rr >> 5) * 16 + (rr & 15);
            const int own_col = s ? N1 - 1 - j : j;
            const int rec_col = N1 - 1 - own_col;
            float2 *xrow = xs + c * SC;
            float2 own[H], rec[H];
            {
                float2 x[N2];
#pragma unroll
                for (int n2 = 0; n2 < N2; ++n2) x[n2] = xrow[n2 * SF_N + own_col];
                // first radix-2 DIF stage over n2: even rows <- x[n] + x[n+H], odd <- (x[n] - x[n+H]) w^n
#pragma unroll
                for (int n = 0; n < H; ++n) {
                    const float2 a = x[n], bq = x[n + H];
                    own[bitrev(n, C::LOG_H)] = cadd(a, bq);
                    const float2 d = csub(a, bq);
                    const float2 w = n == 0 ? d : (4 * n == N2 ? make_float2(d.y, -d.x) : cmul(d, tw_const(n, N2)));
                    rec[bitrev(n, C::LOG_H)] = shfl_xor2(w, 16);  // odd rows of the other column
                }
            }
            fft_dit<H, false>(own);  // own[k] = Z[own_col + N1 (2k)]
            fft_dit<H, false>(rec);  // rec[k] = Z[rec_col + N1 (2k+1)]
            // spectral product: mirror of (own_col, 2k) is (rec_col, N2-1-2k) = rec[H-1-k]
#pragma unroll
            for (int k = 0; k < H; ++k) {
                const float2 xv = spectral_product(own[k], rec[H - 1 - k]);
                own[k] = xv;
                rec[H - 1 - k] = cconj(xv);
            }
            // real-inverse packing: partner of (own_col, 2k) is (rec_col, M2-1-2k) = rec[MH-1-k]
            const float2 *ptab = tw + C::TW_P;
#pragma unroll
            for (int k = 0; k < MH; ++k) {
                float2 ca, cb;
                pack_pair(own[k], rec[MH - 1 - k], __ldg(ptab + (2 * k) * N1 + own_col),
                          __ldg(ptab + (M2 - 1 - 2 * k) * N1 + rec_col), ca, cb);
                own[k] = ca;
                rec[MH - 1 - k] = cb;
            }
            // first inverse step (M2-point DFT over k2) split by parity of k2:
            // E of own column here, O of own column at the partner
            float2 eo[MH], oo[MH];
#pragma unroll
            for (int k = 0; k < MH; ++k) {
                eo[bitrev(k, C::LOG_MH)] = own[k];
                oo[bitrev(k, C::LOG_MH)] = rec[k];
            }
            fft_dit<MH, true>(eo);  // E of own_col
            fft_dit<MH, true>(oo);  // O of rec_col
            float2 y[M2];
#pragma unroll
            for (int m = 0; m < MH; ++m) {
                const float2 op = shfl_xor2(oo[m], 16);  // O of own_col
                const float2 t = m == 0 ? op : cmul_conj(op, tw_const(m, M2));
                y[m] = cadd(eo[m], t);
                y[m + MH] = csub(eo[m], t);
            }
            const float2 *qtab = tw + C::TW_Q;
            if (N2 > 16)
                bar_sync(1 + c, 2 * N2);  // both warps of the row are done reading it
            else
                __syncwarp();
            xrow[own_col] = y[0];
#pragma unroll
            for (int m2 = 1; m2 < M2; ++m2) xrow[m2 * SI_M + own_col] = cmul(y[m2], __ldg(qtab + m2 * N1 + own_col));
        }
        __syncthreads();

        // ------------------------------------------------------------ I3
        // thread (m2, s, h, c): the N1-point inverse DFT over k1 = 2i + h of row
        // m2 of row c; lane s takes the even (s=0) or odd (s=1) i.
        {
            const int c = tid % ROWS, h = (tid / ROWS) & 1, s = (tid / (2 * ROWS)) & 1, m2 = tid / (4 * ROWS);
            const float2 *xi = xs + c * SC + m2 * SI_M + 2 * s + h;
            float2 x[H];
#pragma unroll
            for (int i = 0; i < H; ++i) x[bitrev(i, C::LOG_H)] = xi[4 * i];
            fft_dit<H, true>(x);  // E (s = 0) or O (s = 1), m in [0, H)
            // out[m] = E[m] + w^-m O[m] (m < H), out[m+H] = E[m] - w^-m O[m]; lane s keeps m1 = H s + m
            const float sg1 = s ? -1.f : 1.f;
            float2 out[H];
#pragma unroll
            for (int m = 0; m < H; ++m) {
                float2 mine = x[m];
                if (m > 0) {
                    const float2 w = tw_const(m, N2);
                    const float2 ws = s ? w : make_float2(1.f, 0.f);
                    mine = cmul_conj(mine, ws);
                }
                const float2 other = shfl_xor2(mine, 2 * ROWS);
                float2 o = make_float2(fmaf(sg1, mine.x, other.x), fmaf(sg1, mine.y, other.y));
                out[m] = cmul(o, rot[(2 * h + s) * (H + 1) + m]);
            }
            // combine the two parities h: lane h keeps m in [h H/2, (h+1) H/2)
            const int d = d0 + c;
            const bool dok = d < D;
            const float sc = alpha_row[c];
            const int t0 = 2 * m2 + N2 * (H * s + (H / 2) * h);
            const int64_t dir = rev_out ? -1 : 1;  // output time direction
            IO *rp = r + boff + d + (int64_t)(rev_out ? L - 1 - t0 : t0) * D;
            const int64_t step = dir * N2 * D;
#pragma unroll
            for (int i = 0; i < H / 2; ++i) {
                const float2 send = h ? out[i] : out[H / 2 + i];
                const float2 keep = h ? out[H / 2 + i] : out[i];
                const float2 o = cadd(keep, shfl_xor2(send, ROWS));
                const int t = t0 + N2 * i;
                float r0 = o.x * sc, r1 = o.y * sc;
                if (i * N2 < HEAD && t < HEAD) {
                    r0 = 0.f;
                    r1 = 0.f;
#pragma unroll
                    for (int p = 0; p < C::HP; ++p) {
                        r0 += hres[(c * C::HP + p) * HEAD + t];
                        r1 += hres[(c * C::HP + p) * HEAD + t + 1];
                    }
                }
                if (dok && t < L) IO_t<IO>::st(rp, r0);
                if (dok && t + 1 < L) IO_t<IO>::st(rp + dir * D, r1);
                rp += step;
            }
        }
    }
    if (!tma) cp_async_wait_all();
}

}  // namespace ccv
