// mhf_gate.cuh -- gate stream of the Multi-Head Fourier block on the tensor cores.
//
// Caracal: Causal Architecture via Spectral Mixing, "Key design 1": the gate
// stream is x_g = Conv1d_G2(sigma(Linear_G1(x_norm))), a 1-D convolution
// grouped by head.  Starting from a = Linear_G1(x_norm) ([B, L, D],
// channel-last, C = D / H channels a head, K taps, causal):
//
//   g[b, t, h C + n] = bias[h C + n]
//                    + sum_{k<K} sum_{c<C} w[h C + n][c][k] * sigmoid(a[b, t-(K-1)+k, h C + c])
//
// For one head and one batch this is a dense contraction over (k, c):
// [128 time steps x C] times [C x C] per tap, so it runs as tcgen05 MMAs:
// M = 128 time steps, N = C output channels, K = C input channels per tap,
// accumulated over the taps in TMEM.  The taps need no extra copies: the
// staged sigmoid tile holds time steps t0-(K-1) .. t0+127, and tap k's
// operand is the same tile started k rows later (16 bytes in the K-major
// no-swizzle layout).
//
// fp32 accuracy from tf32 tensor cores: every operand x is split into
// hi = x with its 13 low mantissa bits cleared (exact in tf32) and
// lo = x - hi (exact in fp32, |lo| <= 2^-10 |x|), and the product is
// hi*W_hi + hi*W_lo + lo*W_hi.  The dropped lo*W_lo term and the tf32 view of
// the lo parts are below 2^-20 of |x W|, so g carries fp32-level error.
//
// Schedule: a persistent CTA per (head, group of tiles); the head's weights
// are split and staged in shared memory once.  Per 128-step tile the CTA
// stores sigmoid(a) (hi, lo) to shared memory, warp 0 runs the loop of
// 3 K C/8 MMAs (one lane issues them, chosen by elect.sync) and commits them
// to an mbarrier, and the sixteen warps read the accumulator back (warp w:
// TMEM lanes 32 (w % 4) .. +31 = time steps, a quarter of the columns each),
// add the bias, stage the rows in shared memory and store g as whole rows
// (coalesced).  With two tile buffers and two accumulators (every head width
// and tap count whose tiles fit twice) the tensor core works on tile i+1
// while the warps drain tile i and stage tile i+2; a for the two tiles after
// that streams into two register sets meanwhile.  Every wait is bounded; no
// load uses cluster multicast.
#pragma once

#include <cuda_bf16.h>
#include <stdint.h>

#include "tcgen05.cuh"
#include "tma.cuh"

namespace ccv {

constexpr unsigned kFaultMmaWait = 2u;  // fault bit: an MMA completion wait ran out
constexpr int kGateM = 128;             // time steps per tile (MMA M)
constexpr int kGateThreads = 512;       // sixteen warps: four per TMEM lane quarter, a quarter of the columns each
constexpr int kGateMaxTaps = 4;

template <int C, int KT>
struct GateCfg {
    static_assert(C == 16 || C == 32 || C == 64, "head width");
    static_assert(KT >= 1 && KT <= kGateMaxTaps, "taps");
    static constexpr int ROWS = kGateM + KT - 1;          // staged time steps
    static constexpr int KC = C / 4;                       // 16-byte chunks along the contraction axis
    // Two sigmoid tiles (one being staged while the tensor core reads the
    // other) when they fit next to the weights; an odd row count keeps the
    // 16-byte stores conflict-free, an even one (2-way conflicts) is taken
    // when only that fits.
    static constexpr unsigned kMaxSmem = 232448;
    static constexpr unsigned FIXED = 2u * KT * C * C * 4u + C * 4u + 48u + 128u;
    static constexpr bool DB_ODD = 4u * KC * (ROWS | 1) * 16u + FIXED <= kMaxSmem;
    static constexpr bool DB_EVEN = (ROWS % 2 == 0) && 4u * KC * ROWS * 16u + FIXED <= kMaxSmem;
    static constexpr int NBUF = (DB_ODD || DB_EVEN) ? 2 : 1;
    static constexpr int R = DB_ODD ? (ROWS | 1) : (DB_EVEN ? ROWS : (ROWS | 1));
    static constexpr unsigned LBO_A = R * 16u;             // chunk pitch of the sigmoid tile
    static constexpr unsigned A_BYTES = KC * LBO_A;
    static constexpr unsigned LBO_W = C * 16u;             // chunk pitch of one tap's weights
    static constexpr unsigned W_TAP = KC * LBO_W;          // = C * C * 4
    static constexpr unsigned W_BYTES = KT * W_TAP;
    // buffer b: hi at OFF_A(b), lo at OFF_A(b) + A_BYTES
    static constexpr unsigned OFF_WHI = NBUF * 2 * A_BYTES, OFF_WLO = OFF_WHI + W_BYTES;
    static constexpr unsigned OFF_BIAS = OFF_WLO + W_BYTES;
    static constexpr unsigned OFF_BAR = (OFF_BIAS + C * 4u + 15u) & ~15u;  // NBUF mbarriers, then the TMEM slot
    static constexpr unsigned SMEM_BYTES = OFF_BAR + 32u + 128u;           // + alignment slack
    static_assert(SMEM_BYTES <= kMaxSmem, "shared memory");
    // one fp32 accumulator of C columns per buffer, in a power-of-two allocation >= 32
    static constexpr unsigned TMEM_COLS = NBUF * C <= 32 ? 32u : (NBUF * C <= 64 ? 64u : 128u);
    static constexpr int NLOAD = (ROWS * KC + kGateThreads - 1) / kGateThreads;  // 4-vectors per thread
    static constexpr int NMMA = 3 * KT * (C / 8);
    static constexpr int OPITCH = C + 4;  // row pitch (floats) of the output tile staged in a free tile buffer
    static_assert(kGateM * OPITCH * 4u <= 2u * A_BYTES, "output tile must fit in one tile buffer");
};

__device__ __forceinline__ void split_tf32(float x, float &hi, float &lo) {
    hi = __uint_as_float(__float_as_uint(x) & 0xFFFFE000u);
    lo = x - hi;
}

// Logistic function from the fast exponential and reciprocal (both within a
// few ulp; the bound on g is 1e-5 of |w| sigmoid(a)).  Saturates cleanly: a
// large negative x gives exp = inf and 1/inf = 0.
__device__ __forceinline__ float logistic(float x) { return __fdividef(1.0f, 1.0f + __expf(-x)); }

// Four consecutive channels of a, as loaded (fp32: one 16-byte load; bf16:
// 8 bytes).  The vector loads are volatile asm so that they issue where they
// are written -- a tile or two before their use -- and are not moved next
// to it.
template <typename IO>
struct Raw4;
template <>
struct Raw4<float> {
    float4 x;
    __device__ __forceinline__ void load(const float *p, bool vec) {
        if (vec)
            asm volatile("ld.global.nc.v4.f32 {%0, %1, %2, %3}, [%4];"
                         : "=f"(x.x), "=f"(x.y), "=f"(x.z), "=f"(x.w)
                         : "l"(p));
        else
            x = make_float4(p[0], p[1], p[2], p[3]);
    }
    __device__ __forceinline__ void zero() { x = make_float4(0.f, 0.f, 0.f, 0.f); }
    __device__ __forceinline__ float4 f32() const { return x; }
};
template <>
struct Raw4<__nv_bfloat16> {
    uint2 x;
    __device__ __forceinline__ void load(const __nv_bfloat16 *p, bool vec) {
        if (vec) {
            asm volatile("ld.global.nc.v2.u32 {%0, %1}, [%2];" : "=r"(x.x), "=r"(x.y) : "l"(p));
        } else {
            const uint16_t *q = reinterpret_cast<const uint16_t *>(p);
            x = make_uint2((unsigned)q[0] | ((unsigned)q[1] << 16), (unsigned)q[2] | ((unsigned)q[3] << 16));
        }
    }
    __device__ __forceinline__ void zero() { x = make_uint2(0u, 0u); }
    __device__ __forceinline__ float4 f32() const {
        return make_float4(__uint_as_float(x.x << 16), __uint_as_float(x.x & 0xFFFF0000u),
                           __uint_as_float(x.y << 16), __uint_as_float(x.y & 0xFFFF0000u));
    }
};

// Store 4 consecutive output channels of one time step.
__device__ __forceinline__ void store4(float *p, const float (&v)[4], bool vec) {
    if (vec) {
        *reinterpret_cast<float4 *>(p) = make_float4(v[0], v[1], v[2], v[3]);
    } else {
#pragma unroll
        for (int i = 0; i < 4; ++i) p[i] = v[i];
    }
}
__device__ __forceinline__ void store4(__nv_bfloat16 *p, const float (&v)[4], bool vec) {
    const __nv_bfloat162 h0 = __floats2bfloat162_rn(v[0], v[1]), h1 = __floats2bfloat162_rn(v[2], v[3]);
    const unsigned u0 = *reinterpret_cast<const unsigned *>(&h0), u1 = *reinterpret_cast<const unsigned *>(&h1);
    if (vec) {
        *reinterpret_cast<uint2 *>(p) = make_uint2(u0, u1);
    } else {
        uint16_t *q = reinterpret_cast<uint16_t *>(p);
        q[0] = (uint16_t)(u0 & 0xFFFFu);
        q[1] = (uint16_t)(u0 >> 16);
        q[2] = (uint16_t)(u1 & 0xFFFFu);
        q[3] = (uint16_t)(u1 >> 16);
    }
}

// grid = H * groups CTAs; CTA (h = blockIdx.x % H, j = blockIdx.x / H) takes
// the tiles j, j + groups, ... of head h, tile = b * tiles_per_row + t0 / 128.
// vec_in: a's rows allow 4-channel vector loads; vec_out: g allows 16-byte stores.
template <int C, int KT, typename IO>
__global__ void __launch_bounds__(kGateThreads, 1)
    mhf_gate_kernel(const IO *__restrict__ a, const float *__restrict__ w, const float *__restrict__ bias,
                    IO *__restrict__ g, int L, int D, int H, int groups, int tiles_per_row, int num_tiles,
                    int vec_in, int vec_out) {
    using Cfg = GateCfg<C, KT>;
    extern __shared__ unsigned char gate_smem_raw[];
    unsigned char *sm = reinterpret_cast<unsigned char *>(((uintptr_t)gate_smem_raw + 127) & ~(uintptr_t)127);
    const unsigned sb = smem_u32(sm);
    float *sbias = reinterpret_cast<float *>(sm + Cfg::OFF_BIAS);
    uint64_t *bar = reinterpret_cast<uint64_t *>(sm + Cfg::OFF_BAR);  // bar[0 .. NBUF-1]
    unsigned *tslot = reinterpret_cast<unsigned *>(sm + Cfg::OFF_BAR + 16);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int h = blockIdx.x % H;
    const int64_t col0 = (int64_t)h * C;

    if (warp == 0) tmem_alloc(tslot, Cfg::TMEM_COLS);
    if (tid == 0)
        for (int i = 0; i < Cfg::NBUF; ++i) mbar_init(bar + i, 1);

    // Two register sets of raw a: tile j of this CTA's sequence uses set j % 2,
    // so the loads of tiles j+2 and j+3 are in flight while j+1 is staged.
    Raw4<IO> raw0[Cfg::NLOAD], raw1[Cfg::NLOAD];
    auto load_tile = [&](Raw4<IO>(&raw)[Cfg::NLOAD], int tile) {
        const int b = tile / tiles_per_row;
        const int t0 = (tile % tiles_per_row) * kGateM;
        const IO *base = a + (int64_t)b * L * D + col0;
#pragma unroll
        for (int j = 0; j < Cfg::NLOAD; ++j) {
            const int i = tid + j * kGateThreads;
            const int r = i / Cfg::KC, kc = i % Cfg::KC;
            const int t = t0 - (KT - 1) + r;
            if (i < Cfg::ROWS * Cfg::KC && t >= 0 && t < L)
                raw[j].load(base + (int64_t)t * D + kc * 4, vec_in != 0);
            else
                raw[j].zero();
        }
    };
    auto stage_tile = [&](Raw4<IO>(&raw)[Cfg::NLOAD], int tile, int buf) {
        unsigned char *ahi = sm + buf * 2 * Cfg::A_BYTES, *alo = ahi + Cfg::A_BYTES;
        const int t0 = (tile % tiles_per_row) * kGateM;
#pragma unroll
        for (int j = 0; j < Cfg::NLOAD; ++j) {
            const int i = tid + j * kGateThreads;
            if (i >= Cfg::ROWS * Cfg::KC) break;
            const int r = i / Cfg::KC, kc = i % Cfg::KC;
            const int t = t0 - (KT - 1) + r;
            float4 s = make_float4(0.f, 0.f, 0.f, 0.f);  // the convolution's zero padding
            if (t >= 0 && t < L) {
                const float4 x = raw[j].f32();
                s = make_float4(logistic(x.x), logistic(x.y), logistic(x.z), logistic(x.w));
            }
            float4 hi, lo;
            split_tf32(s.x, hi.x, lo.x);
            split_tf32(s.y, hi.y, lo.y);
            split_tf32(s.z, hi.z, lo.z);
            split_tf32(s.w, hi.w, lo.w);
            const unsigned off = kc * Cfg::LBO_A + r * 16u;
            *reinterpret_cast<float4 *>(ahi + off) = hi;
            *reinterpret_cast<float4 *>(alo + off) = lo;
        }
    };

    // the first two tiles' a is in flight while the weights are staged
    int tile = blockIdx.x / H;
    if (tile < num_tiles) load_tile(raw0, tile);
    if (tile + groups < num_tiles) load_tile(raw1, tile + groups);

    // The head's weights, split into tf32 hi / lo, in the K-major layout:
    // tap k, chunk c/4, output channel n, element c%4.  One thread fills one
    // 16-byte slot (k, chunk, n) from four gathered loads of w ([D][C][K]);
    // consecutive threads take consecutive n, so the slot stores are
    // conflict-free.  (The head's block is read once per CTA, from L2 after
    // the first CTA of the head.)
    const float *wh = w + col0 * C * KT;
#pragma unroll 2
    for (int sl = tid; sl < KT * Cfg::KC * C; sl += kGateThreads) {
        const int n = sl % C, kc = (sl / C) % Cfg::KC, k = sl / (C * Cfg::KC);
        const float *src = wh + ((int64_t)n * C + kc * 4) * KT + k;
        float4 hi, lo;
        split_tf32(__ldg(src), hi.x, lo.x);
        split_tf32(__ldg(src + KT), hi.y, lo.y);
        split_tf32(__ldg(src + 2 * KT), hi.z, lo.z);
        split_tf32(__ldg(src + 3 * KT), hi.w, lo.w);
        const unsigned off = k * Cfg::W_TAP + kc * Cfg::LBO_W + n * 16u;
        *reinterpret_cast<float4 *>(sm + Cfg::OFF_WHI + off) = hi;
        *reinterpret_cast<float4 *>(sm + Cfg::OFF_WLO + off) = lo;
    }
    if (tid < C) sbias[tid] = bias ? __ldg(bias + col0 + tid) : 0.0f;

    tc_fence_before_sync();
    __syncthreads();
    tc_fence_after_sync();
    const unsigned tmem = *tslot;
    constexpr uint32_t idesc = umma_idesc_tf32(kGateM, C);

    // MMAs of one tile: 3 split products x K taps x C/8 steps of 8 channels,
    // into accumulator `buf`; committed to bar[buf].  Run by all of warp 0.  Descriptors advance by
    // (byte offset >> 4) in their address field.
    auto issue = [&](int buf) {
        const unsigned d = tmem + buf * C;
        const unsigned abase = sb + buf * 2 * Cfg::A_BYTES;
        int step = 0;
#pragma unroll 1
        for (int p = 0; p < 3; ++p) {  // hi*W_hi, hi*W_lo, lo*W_hi
            const uint64_t a0 = umma_smem_desc(abase + (p < 2 ? 0u : Cfg::A_BYTES), Cfg::LBO_A, 128u);
            const uint64_t b0 = umma_smem_desc(sb + (p == 1 ? Cfg::OFF_WLO : Cfg::OFF_WHI), Cfg::LBO_W, 128u);
#pragma unroll
            for (int k = 0; k < KT; ++k) {
#pragma unroll
                for (int s = 0; s < C / 8; ++s) {
                    umma_tf32_elect(d, a0 + ((k * 16u + 2u * s * Cfg::LBO_A) >> 4),
                              b0 + ((k * Cfg::W_TAP + 2u * s * Cfg::LBO_W) >> 4), idesc, step > 0);
                    ++step;
                }
            }
        }
        umma_commit_elect(bar + buf);
    };
    // the staged tile (generic-proxy stores) is made visible to the tensor
    // core, and every warp's earlier reads of the accumulator are ordered
    // before the MMAs that overwrite it
    auto publish = [&]() {
        fence_proxy_async_smem();
        tc_fence_before_sync();
        __syncthreads();
        tc_fence_after_sync();
    };

    // stage tile `stile` from register set s into tile buffer `buf`, start its
    // MMAs, then refill set s with tile `ltile` (the one two places later)
    auto stage_issue_load = [&](int s, int stile, int buf, int ltile) {
        if (s) stage_tile(raw1, stile, buf);
        else stage_tile(raw0, stile, buf);
        publish();
        if (warp == 0) issue(buf);  // the whole warp runs the loop, one lane issues
        if (ltile < num_tiles) {
            if (s) load_tile(raw1, ltile);
            else load_tile(raw0, ltile);
        }
    };

    unsigned parity = 0u, pending = 0u;  // bit i: phase parity awaited on / MMAs in flight on bar[i]
    bool ok = true;
    if (tile < num_tiles) {
        stage_issue_load(0, tile, 0, tile + 2 * groups);
        pending |= 1u;
    }
    for (int it = 0; tile < num_tiles; tile += groups, ++it) {
        const int cur = Cfg::NBUF == 2 ? (it & 1) : 0;
        const int next = tile + groups;
        if (Cfg::NBUF == 2 && next < num_tiles) {
            // the other buffer's MMAs completed in the previous iteration
            stage_issue_load((it + 1) & 1, next, cur ^ 1, next + 2 * groups);
            pending |= 1u << (cur ^ 1);
        }
        // one thread waits for this tile's MMAs; the barrier releases the rest
        bool done = true;
        if (tid == 0) done = mbar_wait_bounded(bar + cur, (parity >> cur) & 1u);
        if (!__syncthreads_and(done)) {
            ok = false;
            break;
        }
        parity ^= 1u << cur;
        pending &= ~(1u << cur);
        tc_fence_after_sync();

        // accumulator row m = 32 (warp % 4) + lane (time step t0 + m); warp w
        // takes the column quarter w / 4.  Rows are staged (with the bias) in
        // this tile's buffer, whose MMAs are done, then written out as whole
        // C-channel rows by consecutive threads.
        {
            const int q = warp & 3, cbase = (warp >> 2) * (C / 4);
            float *otile = reinterpret_cast<float *>(sm + cur * 2 * Cfg::A_BYTES);
            float *orow = otile + (q * 32 + lane) * Cfg::OPITCH + cbase;
            const unsigned trow = tmem + cur * C + ((unsigned)(q * 32) << 16) + cbase;
            if constexpr (C / 4 == 16) {
                float v[16];
                tmem_ld16(trow, v);
#pragma unroll
                for (int i = 0; i < 16; i += 4)
                    *reinterpret_cast<float4 *>(orow + i) = make_float4(
                        v[i] + sbias[cbase + i], v[i + 1] + sbias[cbase + i + 1], v[i + 2] + sbias[cbase + i + 2],
                        v[i + 3] + sbias[cbase + i + 3]);
            } else if constexpr (C / 4 == 8) {
                float v[8];
                tmem_ld8(trow, v);
#pragma unroll
                for (int i = 0; i < 8; i += 4)
                    *reinterpret_cast<float4 *>(orow + i) = make_float4(
                        v[i] + sbias[cbase + i], v[i + 1] + sbias[cbase + i + 1], v[i + 2] + sbias[cbase + i + 2],
                        v[i + 3] + sbias[cbase + i + 3]);
            } else {
                float v[4];
                tmem_ld4(trow, v);
                *reinterpret_cast<float4 *>(orow) =
                    make_float4(v[0] + sbias[cbase], v[1] + sbias[cbase + 1], v[2] + sbias[cbase + 2],
                                v[3] + sbias[cbase + 3]);
            }
            __syncthreads();
            const int b = tile / tiles_per_row, t0 = (tile % tiles_per_row) * kGateM;
            IO *gt = g + ((int64_t)b * L + t0) * D + col0;
#pragma unroll
            for (int i = tid; i < kGateM * (C / 4); i += kGateThreads) {
                const int m = i / (C / 4), c4 = i % (C / 4);
                if (t0 + m < L) {
                    const float4 x = *reinterpret_cast<const float4 *>(otile + m * Cfg::OPITCH + 4 * c4);
                    const float xv[4] = {x.x, x.y, x.z, x.w};
                    store4(gt + (int64_t)m * D + 4 * c4, xv, vec_out != 0);
                }
            }
            __syncthreads();  // the buffer is staged into again
        }
        if (Cfg::NBUF == 1 && next < num_tiles) {
            // single buffer: the next tile is staged once this one's MMAs are done
            stage_issue_load((it + 1) & 1, next, 0, next + 2 * groups);
            pending |= 1u;
        }
    }
    if (!ok && tid == 0) {
        atomicOr(&g_cc_fault, kFaultMmaWait);
        for (int i = 0; i < Cfg::NBUF; ++i)  // give the MMAs in flight a last chance to finish
            if ((pending >> i) & 1u) mbar_wait_bounded(bar + i, (parity >> i) & 1u);
    }
    tc_fence_before_sync();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after_sync();
        tmem_dealloc(tmem, Cfg::TMEM_COLS);
    }
}

}  // namespace ccv
