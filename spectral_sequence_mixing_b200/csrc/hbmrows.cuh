// hbmrows.cuh -- long rows (4096 < L <= 65536, transform length N = 131072)
// as a four-step transform through a device workspace.
//
// Method (Caracal: Causal Architecture via Spectral Mixing, "Key design 1"
// and the limitations section on 100k+ contexts): each (b, d) row of v and
// g is zero-padded to N, transformed, multiplied and inverse-transformed,
// which equals r_t = sum_{j<=t} v_j g_{t-j} for t < L.  As in the fused
// kernel, one odd-frequency complex transform carries both streams
// (z = v + i alpha g, Z_k = sum_n z_n theta^(n(2k+1)), theta = exp(-i pi/N)),
// the product pairs bin k with its mirror N-1-k, and the real output comes
// from a complex inverse of half the length whose outputs are
// w_m = r_2m + i r_2m+1.
//
// A row does not fit on chip, so the transform is split into passes that
// each hold whole sub-transforms and exchange data through HBM (the
// "four-step" FFT), with n = n1 + A n2 (A = 512, n2 < 256), k = k2 + 256 k1:
//   norms   per row, the sums of squares of v and g (fixed-order partials per
//           time slice, then one thread per row): alpha and the output scale.
//   fwd     for each (row, n1): the 256-point odd-frequency DFT over n2
//           (only n2 < 128 carries data), times theta^(n1 (2 k2 + 1));
//           written as Y[k2][n1][row].
//   mid     for each (row, k2 pair {k2, 255 - k2}): the 512-point DFTs over
//           n1 (bin (k2, k1) has its mirror at (255 - k2, 511 - k1)), the
//           spectral product, the real-output packing
//           C_k = E_k + i O_k, E_k = X_k + X_(k+N/2),
//           O_k = (X_k - X_(k+N/2)) theta^-(2k+1)   (k < N/2),
//           and the inner 256-point inverse over k1 of the half-length
//           inverse, times phi^-(m1 (2 k2 + 1)), phi = theta^2; written in
//           place as W[k2][m1][row].
//   inv     for each (row, m1): the odd-frequency 256-point inverse over k2,
//           only the outputs m = m1 + 256 m2 with 2m < N/2 (the truncation),
//           scaled; r_t for t < kHeadT0 replaced by the direct sum.
// Rows are innermost in the workspace, so every pass reads and writes whole
// runs of adjacent channels (a channel-last tensor's rows are its channels):
// the fwd pass 16 channels per CTA with TMA-staged inputs (32, one per lane,
// in its direct-load variant), the inv pass 32, the mid pass kHrRows2 rows per
// CTA (one per warp), staged through shared memory.
//
// Each sub-transform is a two-level decomposition inside a CTA: register
// DFTs of 8, 16 or 32 points (fft_reg.cuh) with one shared-memory exchange.
#pragma once

#include <stdint.h>

#include "fft_reg.cuh"
#include "fftconv_fused.cuh"  // IO_t, spectral_product, kHeadT0
#include "tma.cuh"

namespace ccv {

constexpr int kHrN = 131072;          // transform length
constexpr int kHrA = 512;             // n = n1 + A n2; k = k2 + kHrB k1
constexpr int kHrB = 256;
constexpr int kHrLMAX = kHrN / 2;     // longest row
constexpr int kHrCG = 32;             // channels per fwd / inv CTA (one per lane)
constexpr int kHrRows2 = 4;           // rows per mid CTA (one per warp)
constexpr int kHrSlices = 64;         // time slices of the norm pass
constexpr int kHrSliceT = kHrLMAX / kHrSlices;
constexpr int kHrSP = 257;            // fwd / inv shared-memory column pitch (float2)
constexpr int kHrColM = 576;          // mid: one 512-point column (pitch-18 groups of 16 after the first step)
constexpr int kHrRowM = 2 * kHrColM + 4;  // mid: one row's two columns (pitch = 4 mod 16: conflict-free loads)
constexpr int kHrFwdThreads = 512, kHrMidThreads = 32 * kHrRows2, kHrInvThreads = 512, kHrNormThreads = 128;
constexpr size_t kHrFwdSmem = (size_t)kHrCG * kHrSP * 8;
constexpr int kHrMidSP = kHrRows2 + 1;  // mid output staging pitch: [sel][m1][rows + pad], over the row area
// one column's staging: m1 < 128, a gap of 8 float2 (so a lane pair's two
// halves m1 and m1 + 128 fall on different banks), then m1 >= 128
constexpr int kHrMidStageCol = kHrB * kHrMidSP + 8;
__device__ __forceinline__ int hr_stage_idx(int sel, int m1, int r) {
    return sel * kHrMidStageCol + m1 * kHrMidSP + (m1 >= kHrB / 2 ? 8 : 0) + r;
}
constexpr size_t kHrMidSmem = (size_t)kHrRows2 * kHrRowM * 8;
static_assert((size_t)2 * kHrMidStageCol <= (size_t)kHrRows2 * kHrRowM, "output staging fits the row area");

// Twiddle table (float2, built on the host in fp64); theta = exp(-i pi / N),
// omega_R = exp(-2 pi i / R), phi = theta^2.
constexpr int kHrTW1 = 0;                    // [n2 < 128]           omega_512^n2
constexpr int kHrTA = kHrTW1 + 128;          // [a * 16 + c]         omega_256^(a c)
constexpr int kHrTO = kHrTA + 256;           // [n1 * 256 + k2]      theta^(n1 (2 k2 + 1))
constexpr int kHrT512 = kHrTO + kHrA * kHrB; // [p * 32 + u]         omega_512^(p u)
constexpr int kHrPK1 = kHrT512 + 512;        // [k2]                 theta^-(2 k2 + 1)
constexpr int kHrPK2 = kHrPK1 + 256;         // [u * 8 + s]          theta^-(512 u + 16384 s)
constexpr int kHrTI = kHrPK2 + 256;          // [u * 8 + al]         exp(2 pi i u al / 256)
constexpr int kHrTWa = kHrTI + 256;          // [k2 * 8 + al]        phi^-(al (2 k2 + 1))
constexpr int kHrTWb = kHrTWa + 256 * 8;     // [k2 * 32 + be]       phi^-(8 be (2 k2 + 1))
constexpr int kHrTU = kHrTWb + 256 * 32;     // [m2 < 128]           exp(i pi m2 / 256)
constexpr int kHrTwSize = kHrTU + 128;

// Workspace (bytes from its base): Y / W [N][rows] float2, norm partials
// [kHrSlices][rows] float2, per-row (alpha, output scale) [rows] float2.
__host__ __device__ inline size_t hr_ws_part_off(int64_t rows) { return (size_t)kHrN * (size_t)rows * 8; }
__host__ __device__ inline size_t hr_ws_as_off(int64_t rows) {
    return hr_ws_part_off(rows) + (size_t)kHrSlices * (size_t)rows * 8;
}
__host__ __device__ inline size_t hr_ws_bytes(int64_t rows) { return hr_ws_as_off(rows) + (size_t)rows * 8; }

// ---------------------------------------------------------------- norms
// grid (channel tiles of 32, kHrSlices): lane = channel, warp w takes time
// steps slice * kHrSliceT + w + 4 i; the 4 warps' sums are added in order.
template <typename IO>
__global__ void __launch_bounds__(kHrNormThreads) hr_norms_kernel(const IO *__restrict__ v, const IO *__restrict__ g,
                                                                  float2 *__restrict__ part, int L, int D, int rows,
                                                                  int tiles_per_batch) {
    __shared__ float2 red[kHrNormThreads / 32][32];
    const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
    const int tile = blockIdx.x, b = tile / tiles_per_batch, d = (tile - b * tiles_per_batch) * kHrCG + lane;
    const bool ok = d < D;
    const int64_t base = (int64_t)b * L * D + d;
    const int t0 = blockIdx.y * kHrSliceT;
    float nv = 0.f, ng = 0.f;
    if (ok) {
#pragma unroll 8
        for (int i = 0; i < kHrSliceT / (kHrNormThreads / 32); ++i) {
            const int t = t0 + w + (kHrNormThreads / 32) * i;
            if (t < L) {
                const float a = IO_t<IO>::cvt(IO_t<IO>::ld(v + base + (int64_t)t * D));
                const float c = IO_t<IO>::cvt(IO_t<IO>::ld(g + base + (int64_t)t * D));
                nv = fmaf(a, a, nv);
                ng = fmaf(c, c, ng);
            }
        }
    }
    red[w][lane] = make_float2(nv, ng);
    __syncthreads();
    if (w == 0 && ok) {
        float2 s = red[0][lane];
#pragma unroll
        for (int k = 1; k < kHrNormThreads / 32; ++k) {
            s.x += red[k][lane].x;
            s.y += red[k][lane].y;
        }
        part[(int64_t)blockIdx.y * rows + (int64_t)b * D + d] = s;
    }
}

// The same partial sums with four adjacent channels per lane (one 16-byte
// fp32 or 8-byte bf16 access per time step and array; D a multiple of 4,
// aligned tensors): grid (channel tiles of 128, kHrSlices), 8 warps over t.
template <typename IO>
__device__ __forceinline__ void hr_ld4(const IO *p, float (&x)[4]) {
    if constexpr (sizeof(IO) == 4) {
        const float4 a = __ldg(reinterpret_cast<const float4 *>(p));
        x[0] = a.x; x[1] = a.y; x[2] = a.z; x[3] = a.w;
    } else {
        const uint2 a = __ldg(reinterpret_cast<const uint2 *>(p));
        x[0] = __uint_as_float(a.x << 16); x[1] = __uint_as_float(a.x & 0xffff0000u);
        x[2] = __uint_as_float(a.y << 16); x[3] = __uint_as_float(a.y & 0xffff0000u);
    }
}

template <typename IO>
__global__ void __launch_bounds__(256) hr_norms4_kernel(const IO *__restrict__ v, const IO *__restrict__ g,
                                                         float2 *__restrict__ part, int L, int D, int rows,
                                                         int tiles_per_batch) {
    __shared__ float2 red[8][128];
    const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
    const int tile = blockIdx.x, b = tile / tiles_per_batch, d = (tile - b * tiles_per_batch) * 128 + 4 * lane;
    const bool ok = d < D;  // D % 4 == 0: all four channels exist
    const int64_t base = (int64_t)b * L * D + d;
    const int t0 = blockIdx.y * kHrSliceT, t1 = min(t0 + kHrSliceT, L);
    float nv[4] = {0.f, 0.f, 0.f, 0.f}, ng[4] = {0.f, 0.f, 0.f, 0.f};
    if (ok) {
#pragma unroll 4
        for (int t = t0 + w; t < t1; t += 8) {
            float a[4], c[4];
            hr_ld4<IO>(v + base + (int64_t)t * D, a);
            hr_ld4<IO>(g + base + (int64_t)t * D, c);
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                nv[q] = fmaf(a[q], a[q], nv[q]);
                ng[q] = fmaf(c[q], c[q], ng[q]);
            }
        }
    }
#pragma unroll
    for (int q = 0; q < 4; ++q) red[w][4 * lane + q] = make_float2(nv[q], ng[q]);
    __syncthreads();
    if (threadIdx.x < 128) {
        const int dd = (tile - b * tiles_per_batch) * 128 + threadIdx.x;
        if (dd < D) {
            float2 s = red[0][threadIdx.x];
#pragma unroll
            for (int k = 1; k < 8; ++k) {
                s.x += red[k][threadIdx.x].x;
                s.y += red[k][threadIdx.x].y;
            }
            part[(int64_t)blockIdx.y * rows + (int64_t)b * D + dd] = s;
        }
    }
}

// One thread per row: the slices' partial sums in order, then the balance
// scale alpha and the output scale 1 / (4 N alpha) (0 when v or g is all zero).
__global__ void __launch_bounds__(256) hr_alpha_kernel(const float2 *__restrict__ part, float2 *__restrict__ as,
                                                       int rows) {
    const int row = blockIdx.x * 256 + threadIdx.x;
    if (row >= rows) return;
    float2 s = part[row];
    for (int k = 1; k < kHrSlices; ++k) {
        const float2 p = part[(int64_t)k * rows + row];
        s.x += p.x;
        s.y += p.y;
    }
    const float alpha = balance_scale(s.x, s.y);
    as[row] = make_float2(alpha, (s.x > 0.f && s.y > 0.f) ? 1.f / (4.f * (float)kHrN * alpha) : 0.f);
}

// ---------------------------------------------------------------- fwd
// grid (channel tiles of 32, n1 < 512).  Step A: warp a, lane = channel: the
// 16-point DFT over b of x[a + 16 b] (b < 8 carries data) -> c, twiddle
// omega_256^(a c); exchange; step B: warp c: 16-point DFT over a -> d, so
// k2 = c + 16 d; times theta^(n1 (2 k2 + 1)); stored at Y[k2][n1][row].
template <typename IO>
__global__ void __launch_bounds__(kHrFwdThreads, 2)
    hr_fwd_kernel(const IO *__restrict__ v, const IO *__restrict__ g, float2 *__restrict__ Y,
                  const float2 *__restrict__ as, const float2 *__restrict__ tw, int L, int D, int rows,
                  int tiles_per_batch, int rev) {
    extern __shared__ float2 hr_sm[];
    const int lane = threadIdx.x & 31, a = threadIdx.x >> 5;
    const int n1 = blockIdx.y;
    const int tile = blockIdx.x, b = tile / tiles_per_batch, d = (tile - b * tiles_per_batch) * kHrCG + lane;
    const bool ok = d < D;
    const int64_t row = (int64_t)b * D + d;
    const int64_t base = (int64_t)b * L * D + d;
    const float alpha = ok ? as[row].x : 1.f;
    float2 x[16];
#pragma unroll
    for (int bb = 0; bb < 8; ++bb) {
        const int n2 = a + 16 * bb;
        const int t = n1 + kHrA * n2;
        float2 z = make_float2(0.f, 0.f);
        if (ok && t < L) {
            const int tv = (rev & 1) ? L - 1 - t : t;
            z = make_float2(IO_t<IO>::cvt(IO_t<IO>::ld(v + base + (int64_t)tv * D)),
                            alpha * IO_t<IO>::cvt(IO_t<IO>::ld(g + base + (int64_t)t * D)));
        }
        x[bitrev(bb, 4)] = cmul(z, __ldg(tw + kHrTW1 + n2));
    }
    fft_dit<16, false, true>(x);  // x[c]; the odd slots (b >= 8) are padding zeros
    float2 *col = hr_sm + lane * kHrSP;
#pragma unroll
    for (int c = 0; c < 16; ++c) col[c * 16 + a] = cmul(x[c], __ldg(tw + kHrTA + a * 16 + c));
    __syncthreads();
    const int c = a;
    float2 y[16];
#pragma unroll
    for (int aa = 0; aa < 16; ++aa) y[bitrev(aa, 4)] = col[c * 16 + aa];
    fft_dit<16, false>(y);  // y[dd]: k2 = c + 16 dd
    if (ok) {
#pragma unroll
        for (int dd = 0; dd < 16; ++dd) {
            const int k2 = c + 16 * dd;
            Y[((int64_t)k2 * kHrA + n1) * rows + row] = cmul(y[dd], __ldg(tw + kHrTO + n1 * kHrB + k2));
        }
    }
}

// The forward pass with its inputs staged by TMA (D * element size a multiple
// of 16 bytes, aligned tensors; REVA: v read reversed in time, the backward): persistent CTAs, two per SM,
// walk the (n1, 16-channel tile) items (consecutive CTAs share n1, so
// together they read whole runs of adjacent time steps); one thread keeps the
// inputs of the next kHrFwdStages - 1 items in flight as TMA boxes
// [128 n2][1 n1][16 d] of the 4-D maps {d, n1, n2, b} of v and g (zero fill
// past D and past the last whole 512-step row; the ragged row of a length
// that is not a multiple of 512 is read directly), so the loads of later
// items overlap the transforms of the current one.
// 4-D tiled TMA load of one box into shared memory, completing on `bar`.
// x (innermost) * element size must be a multiple of 16 bytes.
__device__ __forceinline__ void tma_load_4d(void *dst, const CUtensorMap *map, int x, int y, int z, int w,
                                            uint64_t *bar) {
    asm volatile(
        "cp.async.bulk.tensor.4d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3, %4, "
        "%5}], [%6];" ::"r"(smem_u32(dst)),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(z), "r"(w), "r"(smem_u32(bar))
        : "memory");
}

constexpr int kHrFwdStages = 3;
constexpr int kHrFwdCG = 16;        // channels per CTA of the TMA forward pass (half a warp)
constexpr int kHrFwdTmaThreads = 256;
constexpr size_t kHrFwdXBytes = (size_t)kHrFwdCG * kHrSP * 8;  // exchange buffer, a multiple of 128 bytes
template <typename IO>
constexpr size_t hr_fwd_stage_elems() { return (size_t)2 * 128 * kHrFwdCG; }
template <typename IO>
constexpr size_t hr_fwd_tma_smem() {
    return kHrFwdXBytes + kHrFwdStages * hr_fwd_stage_elems<IO>() * sizeof(IO) + 8 * kHrFwdStages;
}

template <typename IO, bool REVA>
__global__ void __launch_bounds__(kHrFwdTmaThreads, 2)
    hr_fwd_tma_kernel(const IO *__restrict__ v, const IO *__restrict__ g, float2 *__restrict__ Y,
                      const float2 *__restrict__ as, const float2 *__restrict__ tw, int L, int D, int rows,
                      int tiles_per_batch, int ntiles, int items, const __grid_constant__ CUtensorMap tmv,
                      const __grid_constant__ CUtensorMap tmg) {
    extern __shared__ __align__(128) unsigned char hr_raw[];
    constexpr int S = kHrFwdStages, CG = kHrFwdCG;
    constexpr int SE = (int)hr_fwd_stage_elems<IO>();  // IO elements per stage: v then g, [n2][d]
    float2 *xs = reinterpret_cast<float2 *>(hr_raw);
    IO *stg = reinterpret_cast<IO *>(hr_raw + kHrFwdXBytes);
    uint64_t *full = reinterpret_cast<uint64_t *>(hr_raw + kHrFwdXBytes + (size_t)S * SE * sizeof(IO));
    // thread (a, channel): half-warp a = tid / 16 (step A: digit a; step B: digit c), channel tid % 16
    const int tid = threadIdx.x, ch = tid & (CG - 1), a = tid / CG;
    const int nb2 = L / kHrA;  // whole 512-step rows the maps cover
    if (tid == 0)
        for (int q = 0; q < S; ++q) mbar_init(full + q, 1);
    __syncthreads();
    auto item_at = [&](int j) { return (int)blockIdx.x + j * (int)gridDim.x; };
    auto issue = [&](int item, int q) {
        const int n1 = item / ntiles, tile = item - n1 * ntiles;
        const int b = tile / tiles_per_batch, d0 = (tile - b * tiles_per_batch) * CG;
        fence_proxy_async_smem();
        mbar_arrive_expect_tx(full + q, (unsigned)(SE * sizeof(IO)));
        if constexpr (REVA) {
            // v_(L-1-t) for t = n1 + 512 n2, n2 < 128: with L - 1 - n1 = c1 + 512 c2
            // these are rows c2 - n2 of column c1, a box of rows c2 - 127 .. c2
            // (row 127 - n2 of the box; rows below 0 arrive as zeros)
            const int c = L - 1 - n1;
            tma_load_4d(stg + q * SE, &tmv, d0, c & (kHrA - 1), (c >> 9) - 127, b, full + q);
        } else {
            tma_load_4d(stg + q * SE, &tmv, d0, n1, 0, b, full + q);
        }
        tma_load_4d(stg + q * SE + SE / 2, &tmg, d0, n1, 0, b, full + q);
    };
    if (tid == 0)
        for (int j = 0; j < S - 1; ++j)
            if (item_at(j) < items) issue(item_at(j), j);
    float2 *col = xs + ch * kHrSP;
    for (int j = 0; item_at(j) < items; ++j) {
        const int item = item_at(j), q = j % S;
        // the stage of item j + S - 1 was last read in iteration j - 1, before its barriers
        if (tid == 0 && item_at(j + S - 1) < items) issue(item_at(j + S - 1), (j + S - 1) % S);
        const bool got = mbar_wait_bounded(full + q, (unsigned)((j / S) & 1));
        if (!__syncthreads_and(got)) {
            // a copy did not arrive in time: flag it, give the copies in flight
            // one more bounded wait each, and stop
            if (tid == 0) {
                atomicOr(&g_cc_fault, kFaultTmaWait);
                for (int k = j; k < j + S && item_at(k) < items; ++k)
                    mbar_wait_bounded(full + k % S, (unsigned)((k / S) & 1));
            }
            return;
        }
        const int n1 = item / ntiles, tile = item - n1 * ntiles;
        const int b = tile / tiles_per_batch, d = (tile - b * tiles_per_batch) * CG + ch;
        const bool ok = d < D;
        const int64_t row = (int64_t)b * D + d;
        const int64_t base = (int64_t)b * L * D + d;
        const float alpha = ok ? as[row].x : 1.f;
        const IO *sv = stg + q * SE, *sg = sv + SE / 2;
        const int c2 = (L - 1 - n1) >> 9;  // reversed reads: v_(L-1-t) sits in row c2 - n2
        float2 x[16];
#pragma unroll
        for (int bb = 0; bb < 8; ++bb) {
            const int n2 = a + 16 * bb;
            const int t = n1 + kHrA * n2;
            float vv = 0.f, gg = 0.f;
            if constexpr (REVA) {
                const int n2v = c2 - n2;
                if (n2v >= 0 && n2v < nb2)
                    vv = IO_t<IO>::cvt(sv[(127 - n2) * CG + ch]);
                else if (n2v == nb2 && ok && t < L)  // the ragged last row, read directly
                    vv = IO_t<IO>::cvt(IO_t<IO>::ld(v + base + (int64_t)(L - 1 - t) * D));
            } else {
                if (n2 < nb2)
                    vv = IO_t<IO>::cvt(sv[n2 * CG + ch]);
                else if (ok && t < L)
                    vv = IO_t<IO>::cvt(IO_t<IO>::ld(v + base + (int64_t)t * D));
            }
            if (n2 < nb2)
                gg = IO_t<IO>::cvt(sg[n2 * CG + ch]);
            else if (ok && t < L)
                gg = IO_t<IO>::cvt(IO_t<IO>::ld(g + base + (int64_t)t * D));
            x[bitrev(bb, 4)] = cmul(make_float2(vv, alpha * gg), __ldg(tw + kHrTW1 + n2));
        }
        fft_dit<16, false, true>(x);  // x[c]
#pragma unroll
        for (int c = 0; c < 16; ++c) col[c * 16 + a] = cmul(x[c], __ldg(tw + kHrTA + a * 16 + c));
        __syncthreads();  // exchange written; stage q free
        const int c = a;
        float2 y[16];
#pragma unroll
        for (int aa = 0; aa < 16; ++aa) y[bitrev(aa, 4)] = col[c * 16 + aa];
        fft_dit<16, false>(y);  // y[dd]: k2 = c + 16 dd
        if (ok) {
#pragma unroll
            for (int dd = 0; dd < 16; ++dd) {
                const int k2 = c + 16 * dd;
                Y[((int64_t)k2 * kHrA + n1) * rows + row] = cmul(y[dd], __ldg(tw + kHrTO + n1 * kHrB + k2));
            }
        }
        __syncthreads();  // exchange read before the next item writes it
    }
}

// ---------------------------------------------------------------- mid
// grid (row groups of kHrRows2, k2 pairs kp < 128: k2a = kp, k2b = 255 - kp).
// Shared memory: per row (warp) two columns (sel = 0: k2a, 1: k2b) of
// kHrColM float2; at the end the output staging [sel][m1][rows (+1 pad)]
// over the same space.
// Within a warp (its row), n1 = p + 16 q and k1 = u + 32 s:
//   step A  lane (sel, p): 32-point DFT over q -> u, times omega_512^(p u);
//           stored at [u * 18 + p] (16-byte aligned pairs for step B);
//   step B  lane u: 16-point DFTs over p -> s of (k2a, u) and (k2b, 31 - u),
//           which hold each other's mirrors: X(k2a, u, s) pairs with
//           Z(k2b, 31 - u, 15 - s); the packing pairs s with s + 8; then the
//           8-point inverse over s -> al (k1' = u + 32 s, m1 = al + 8 be),
//           times exp(2 pi i u al / 256); stored at [al * 34 + u];
//   step C  lane (sel, al, h): 16-point inverse over u = 2 i + h, the
//           radix-2 combination with the partner lane (h ^ 1) -> be, times
//           phi^-(m1 (2 k2 + 1)); staged, then stored with rows innermost.
__global__ void __launch_bounds__(kHrMidThreads, 16 / kHrRows2) hr_mid_kernel(float2 *__restrict__ Y,
                                                                  const float2 *__restrict__ tw, int rows) {
    extern __shared__ float2 hr_sm[];
    float2 *stage = hr_sm;  // output staging, written once every warp is done with its row
    const int tid = threadIdx.x, lane = tid & 31, r8 = tid >> 5;
    const int64_t row0 = (int64_t)blockIdx.x * kHrRows2;
    const int kp = blockIdx.y, k2a = kp, k2b = kHrB - 1 - kp;
    // load Y[k2][n1][row0 + r] (r fastest; thread tid takes r = tid % kHrRows2
    // and n1 = tid / kHrRows2 + 32 j), each column's 16 loads issued before
    // their stores
    {
        constexpr int PER = kHrA * kHrRows2 / kHrMidThreads;  // loads per thread and column
        const int r = tid & (kHrRows2 - 1), nb = tid / kHrRows2;
        const bool rok = row0 + r < rows;
#pragma unroll
        for (int sel = 0; sel < 2; ++sel) {
            const float2 *src = Y + (int64_t)(sel ? k2b : k2a) * kHrA * rows + row0 + r;
            float2 buf[PER];
#pragma unroll
            for (int j = 0; j < PER; ++j)
                buf[j] = rok ? src[(int64_t)(nb + (kHrMidThreads / kHrRows2) * j) * rows] : make_float2(0.f, 0.f);
#pragma unroll
            for (int j = 0; j < PER; ++j)
                hr_sm[r * kHrRowM + sel * kHrColM + nb + (kHrMidThreads / kHrRows2) * j] = buf[j];
        }
    }
    __syncthreads();
    float2 *rowp = hr_sm + r8 * kHrRowM;
    // ---- step A: lane (sel, p)
    {
        const int sel = lane >> 4, p = lane & 15;
        float2 *colp = rowp + sel * kHrColM;
        float2 x[32];
#pragma unroll
        for (int q = 0; q < 32; ++q) x[bitrev(q, 5)] = colp[p + 16 * q];
        fft_dit<32, false>(x);  // x[u]
        __syncwarp();
        const float4 *t4 = reinterpret_cast<const float4 *>(tw + kHrT512 + p * 32);
#pragma unroll
        for (int u = 0; u < 32; u += 2) {
            const float4 w2 = __ldg(t4 + u / 2);
            colp[u * 18 + p] = cmul(x[u], make_float2(w2.x, w2.y));
            colp[(u + 1) * 18 + p] = cmul(x[u + 1], make_float2(w2.z, w2.w));
        }
    }
    __syncwarp();
    // ---- step B: lane u
    {
        const int u = lane, ub = 31 - u;
        float2 za[16], zb[16];
        {
            const float4 *pa = reinterpret_cast<const float4 *>(rowp + u * 18);
            const float4 *pb = reinterpret_cast<const float4 *>(rowp + kHrColM + ub * 18);
#pragma unroll
            for (int p = 0; p < 16; p += 2) {
                const float4 a4 = pa[p / 2], b4 = pb[p / 2];
                za[bitrev(p, 4)] = make_float2(a4.x, a4.y);
                za[bitrev(p + 1, 4)] = make_float2(a4.z, a4.w);
                zb[bitrev(p, 4)] = make_float2(b4.x, b4.y);
                zb[bitrev(p + 1, 4)] = make_float2(b4.z, b4.w);
            }
        }
        fft_dit<16, false>(za);  // Z(k2a, u + 32 s)
        fft_dit<16, false>(zb);  // Z(k2b, ub + 32 s)
        // spectral product: mirror of (k2a, u, s) is (k2b, ub, 15 - s)
#pragma unroll
        for (int s = 0; s < 16; ++s) {
            const float2 xa = spectral_product(za[s], zb[15 - s]);
            za[s] = xa;
            zb[15 - s] = cconj(xa);
        }
        // real-output packing: bin k + N/2 is (k2, u, s + 8)
        const float2 pka = __ldg(tw + kHrPK1 + k2a), pkb = __ldg(tw + kHrPK1 + k2b);
        float2 ca[8], cb[8];
        {
            const float4 *qa = reinterpret_cast<const float4 *>(tw + kHrPK2 + u * 8);
            const float4 *qb = reinterpret_cast<const float4 *>(tw + kHrPK2 + ub * 8);
#pragma unroll
            for (int s = 0; s < 8; ++s) {
                const float4 wa4 = __ldg(qa + s / 2), wb4 = __ldg(qb + s / 2);
                const float2 wa = (s & 1) ? make_float2(wa4.z, wa4.w) : make_float2(wa4.x, wa4.y);
                const float2 wb = (s & 1) ? make_float2(wb4.z, wb4.w) : make_float2(wb4.x, wb4.y);
                const float2 ea = cadd(za[s], za[s + 8]);
                const float2 oa = cmul(cmul(csub(za[s], za[s + 8]), pka), wa);
                ca[bitrev(s, 3)] = make_float2(ea.x - oa.y, ea.y + oa.x);
                const float2 eb = cadd(zb[s], zb[s + 8]);
                const float2 ob = cmul(cmul(csub(zb[s], zb[s + 8]), pkb), wb);
                cb[bitrev(s, 3)] = make_float2(eb.x - ob.y, eb.y + ob.x);
            }
        }
        fft_dit<8, true>(ca);  // ca[al]
        fft_dit<8, true>(cb);
        __syncwarp();
        const float4 *ia = reinterpret_cast<const float4 *>(tw + kHrTI + u * 8);
        const float4 *ib = reinterpret_cast<const float4 *>(tw + kHrTI + ub * 8);
#pragma unroll
        for (int al = 0; al < 8; al += 2) {
            const float4 wa4 = __ldg(ia + al / 2), wb4 = __ldg(ib + al / 2);
            rowp[al * 34 + u] = cmul(ca[al], make_float2(wa4.x, wa4.y));
            rowp[(al + 1) * 34 + u] = cmul(ca[al + 1], make_float2(wa4.z, wa4.w));
            rowp[kHrColM + al * 34 + ub] = cmul(cb[al], make_float2(wb4.x, wb4.y));
            rowp[kHrColM + (al + 1) * 34 + ub] = cmul(cb[al + 1], make_float2(wb4.z, wb4.w));
        }
    }
    __syncwarp();
    // ---- step C: lane (sel, al, h)
    float2 out[16];
    const int csel = lane >> 4, cal = (lane >> 1) & 7, ch = lane & 1;
    {
        const int sel = lane >> 4, al = (lane >> 1) & 7, h = lane & 1;
        const int k2 = sel ? k2b : k2a;
        const float2 *colp = rowp + sel * kHrColM + al * 34 + h;
        float2 x[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) x[bitrev(i, 4)] = colp[2 * i];
        fft_dit<16, true>(x);  // E (h = 0) or O (h = 1) at be' < 16
        const float sg1 = h ? -1.f : 1.f;
        const float2 twa = __ldg(tw + kHrTWa + k2 * 8 + al);
        const float4 *tb4 = reinterpret_cast<const float4 *>(tw + kHrTWb + k2 * 32 + 16 * h);
        float2 twb[16];
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            const float4 w4 = __ldg(tb4 + j);
            twb[2 * j] = make_float2(w4.x, w4.y);
            twb[2 * j + 1] = make_float2(w4.z, w4.w);
        }
#pragma unroll
        for (int bq = 0; bq < 16; ++bq) {
            float2 mine = x[bq];
            if (h && bq > 0) mine = cmul_conj(mine, tw_const(bq, 32));  // O times omega_32^-be'
            const float2 other = shfl_xor2(mine, 1);
            const float2 o = make_float2(fmaf(sg1, mine.x, other.x), fmaf(sg1, mine.y, other.y));
            out[bq] = cmul(cmul(o, twa), twb[bq]);
        }
    }
    __syncthreads();  // every warp is done with its row: the staging may overwrite them
    {
#pragma unroll
        for (int bq = 0; bq < 16; ++bq) stage[hr_stage_idx(csel, cal + 8 * (bq + 16 * ch), r8)] = out[bq];
    }
    __syncthreads();
    // W[k2][m1][row0 + r] over the first 256 slots of each k2 block of Y
    for (int e = tid; e < 2 * kHrB * kHrRows2; e += kHrMidThreads) {
        const int r = e & (kHrRows2 - 1), m1 = (e / kHrRows2) & (kHrB - 1), sel = e / (kHrRows2 * kHrB);
        const int k2 = sel ? k2b : k2a;
        if (row0 + r < rows)
            Y[((int64_t)k2 * kHrA + m1) * rows + row0 + r] = stage[hr_stage_idx(sel, m1, r)];
    }
}

// ---------------------------------------------------------------- inv
// grid (channel tiles of 32, m1 < 256).  Step 1: warp c, lane = channel:
// 16-point inverse DFT over d of W[c + 16 d][m1] -> mu, times
// exp(2 pi i c mu / 256); exchange; step 2: warp mu: 16-point inverse over
// c -> nu, only nu < 8 (m2 = mu + 16 nu < 128); times exp(i pi m2 / 256);
// m = m1 + 256 m2 gives r_2m and r_2m+1.
template <typename IO>
__global__ void __launch_bounds__(kHrInvThreads, 2)
    hr_inv_kernel(const float2 *__restrict__ W, IO *__restrict__ r, const float2 *__restrict__ as,
                  const IO *__restrict__ v, const IO *__restrict__ g, const float2 *__restrict__ tw, int L, int D,
                  int rows, int tiles_per_batch, int rev) {
    extern __shared__ float2 hr_sm[];
    const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
    const int m1 = blockIdx.y;
    const int tile = blockIdx.x, b = tile / tiles_per_batch, d = (tile - b * tiles_per_batch) * kHrCG + lane;
    const bool ok = d < D;
    const int64_t row = (int64_t)b * D + d;
    float2 *col = hr_sm + lane * kHrSP;
    {
        const int c = wid;
        float2 y[16];
#pragma unroll
        for (int dd = 0; dd < 16; ++dd)
            y[bitrev(dd, 4)] = ok ? W[((int64_t)(c + 16 * dd) * kHrA + m1) * rows + row] : make_float2(0.f, 0.f);
        fft_dit<16, true>(y);  // y[mu]
#pragma unroll
        for (int mu = 0; mu < 16; ++mu) col[mu * 16 + c] = cmul_conj(y[mu], __ldg(tw + kHrTA + c * 16 + mu));
    }
    __syncthreads();
    const int mu = wid;
    float2 y[16];
#pragma unroll
    for (int cc = 0; cc < 16; ++cc) y[bitrev(cc, 4)] = col[mu * 16 + cc];
    fft_dit<16, true, false, true>(y);  // y[nu], nu < 8
    if (!ok) return;
    const float sc = as[row].y;
    const int64_t base = (int64_t)b * L * D + d;
#pragma unroll
    for (int nu = 0; nu < 8; ++nu) {
        const int m2 = mu + 16 * nu;
        const float2 wv = cmul(y[nu], __ldg(tw + kHrTU + m2));
        const int t = 2 * (m1 + kHrB * m2);
        float r0 = wv.x * sc, r1 = wv.y * sc;
        if (t < kHeadT0) {
            // direct sums over the first kHeadT0 inputs (v reversed for rev bit 0)
            r0 = 0.f;
            r1 = 0.f;
            for (int j = 0; j <= t + 1 && j < L; ++j) {
                const float vj = IO_t<IO>::cvt(IO_t<IO>::ld(v + base + (int64_t)((rev & 1) ? L - 1 - j : j) * D));
                if (j <= t && t - j < L) r0 = fmaf(vj, IO_t<IO>::cvt(IO_t<IO>::ld(g + base + (int64_t)(t - j) * D)), r0);
                if (t + 1 - j < L) r1 = fmaf(vj, IO_t<IO>::cvt(IO_t<IO>::ld(g + base + (int64_t)(t + 1 - j) * D)), r1);
            }
        }
        if (t < L) IO_t<IO>::st(r + base + (int64_t)((rev & 2) ? L - 1 - t : t) * D, r0);
        if (t + 1 < L) IO_t<IO>::st(r + base + (int64_t)((rev & 2) ? L - 2 - t : t + 1) * D, r1);
    }
}

}  // namespace ccv
