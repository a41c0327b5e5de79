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
// fp32 accuracy from fp16 tensor cores (kind::f16, fp32 accumulation):
// every operand x is split into hi = fp16(x) and lo = fp16(x - hi), and the
// product is hi*W_hi + hi*W_lo + lo*W_hi.  The dropped lo*W_lo term and the
// rounding of the lo parts are below 2^-21 of |x W| (sigmoid values lie in
// (0, 1) and the weights near 1/sqrt(C K), well inside fp16's range), so g
// carries fp32-level error.  fp16 operands take half the shared-memory bytes
// of tf32 per multiply-add: at M = 128, N = 64 the tensor core's operand
// reads are what bound it, so this halves the MMA time of a tile.
//
// Schedule: a persistent CTA per (head, group of tiles); the head's weights
// are split and staged in shared memory once.  Then the warps take roles:
// seven producer warps store sigmoid(a) (hi, lo) of 128-step tiles into a
// ring of tile buffers (the fp32 input tile arrives by TMA when the tensor
// allows a tensor map), one warp issues each tile's 3 K C/16 MMAs (one lane,
// elect.sync) into a ring of TMEM accumulators, and eight warps read each
// accumulator back (two per TMEM lane quarter: lanes 32 (w % 4) .. +31 =
// time steps, half of the C columns each), add the bias and store g.  Buffers and accumulators pass between
// the roles on mbarriers (tcgen05.commit frees a tile buffer and publishes
// its accumulator), so the tensor core, the sigmoid and the stores of
// different tiles overlap with no CTA-wide barrier.  Every wait is bounded;
// no load uses cluster multicast.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <stdint.h>

#include "tcgen05.cuh"
#include "tma.cuh"

namespace ccv {

constexpr unsigned kFaultMmaWait = 2u;  // fault bit: an MMA completion wait ran out
constexpr int kGateM = 128;             // time steps per tile (MMA M)
constexpr int kGateThreads = 640;       // twenty warps: eight epilogue, one MMA, eleven producer warps
constexpr int kGateMaxTaps = 4;

template <int C, int KT>
struct GateCfg {
    static_assert(C == 16 || C == 32 || C == 64, "head width");
    static_assert(KT >= 1 && KT <= kGateMaxTaps, "taps");
    static constexpr int ROWS = kGateM + KT - 1;          // staged time steps
    static constexpr int KC = C / 8;                       // 16-byte chunks (8 fp16) along the contraction axis
    static constexpr int C4 = C / 4;                       // 4-channel groups of a row
    static constexpr int NBUF = 2;                         // sigmoid tiles / accumulators in flight
    static constexpr int R = ROWS | 1;                     // rows of a tile chunk (odd: conflict-free stores)
    static constexpr unsigned LBO_A = R * 16u;             // chunk pitch of the sigmoid tile
    static constexpr unsigned A_BYTES = (KC * LBO_A + 127u) / 128u * 128u;  // one half (hi or lo)
    static constexpr unsigned RAW_BYTES = (ROWS * C * 4u + 127u) / 128u * 128u;  // fp32 input tile [ROWS][C]
    static constexpr unsigned LBO_W = C * 16u;             // chunk pitch of one tap's weights
    static constexpr unsigned W_TAP = KC * LBO_W;          // = C * C * 2
    static constexpr unsigned W_BYTES = KT * W_TAP;
    // buffer b: hi at b * 2 A_BYTES, lo A_BYTES later; then the input tiles, weights hi / lo, bias
    static constexpr unsigned OFF_RAW = NBUF * 2 * A_BYTES;
    static constexpr unsigned OFF_WHI = OFF_RAW + NBUF * RAW_BYTES, OFF_WLO = OFF_WHI + W_BYTES;
    static constexpr unsigned OFF_BIAS = OFF_WLO + W_BYTES;
    // output staging [kGateM t][OUT_PITCH] fp32 (rows 16 bytes longer than C channels,
    // so one thread per row writes and a warp per row pair reads without bank conflicts),
    // where it fits (not for four taps of 64 channels)
    static constexpr unsigned OUT_PITCH = C + 4;
    static constexpr unsigned OFF_OUT = (OFF_BIAS + C * 4u + 15u) & ~15u;
    static constexpr unsigned OUT_BYTES = kGateM * OUT_PITCH * 4u;
    static constexpr bool STAGE_OUT = OFF_OUT + OUT_BYTES + 96u + 128u <= 232448u;
    static constexpr unsigned OFF_BAR = STAGE_OUT ? OFF_OUT + OUT_BYTES : OFF_OUT;  // 5 NBUF mbarriers, then the TMEM slot
    static constexpr unsigned SMEM_BYTES = OFF_BAR + 96u + 128u;           // + alignment slack
    static_assert(SMEM_BYTES <= 232448, "shared memory");
    // one fp32 accumulator of C columns per buffer, in a power-of-two allocation >= 32
    static constexpr unsigned TMEM_COLS = NBUF * C <= 32 ? 32u : (NBUF * C <= 64 ? 64u : 128u);
};

// fp16 split of x: hi = x rounded to fp16, lo = the remainder rounded to fp16
// (|x - hi - lo| <= 2^-22 |x| while the parts are normal numbers).
__device__ __forceinline__ void split_f16(float x, __half &hi, __half &lo) {
    hi = __float2half_rn(x);
    lo = __float2half_rn(x - __half2float(hi));
}
// four consecutive channels split, packed as two 8-byte words (hi, lo);
// two channels per conversion (packed fp32 -> fp16x2 and back)
__device__ __forceinline__ void split4_f16(float4 x, uint2 &hi, uint2 &lo) {
    const __half2 h01 = __floats2half2_rn(x.x, x.y), h23 = __floats2half2_rn(x.z, x.w);
    const float2 b01 = __half22float2(h01), b23 = __half22float2(h23);
    const __half2 l01 = __floats2half2_rn(x.x - b01.x, x.y - b01.y), l23 = __floats2half2_rn(x.z - b23.x, x.w - b23.y);
    hi = make_uint2(*reinterpret_cast<const uint32_t *>(&h01), *reinterpret_cast<const uint32_t *>(&h23));
    lo = make_uint2(*reinterpret_cast<const uint32_t *>(&l01), *reinterpret_cast<const uint32_t *>(&l23));
}

// Instruction descriptor of a dense kind::f16 MMA with fp16 A and B, fp32
// accumulator, both operands K-major, M = 128, N = n.
__host__ __device__ constexpr uint32_t gate_idesc_f16(int n) {
    return (1u << 4) | ((uint32_t)(n >> 3) << 17) | ((128u >> 4) << 24);
}

__device__ __forceinline__ void umma_f16_elect(unsigned tmem_d, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                               bool accumulate) {
    asm volatile(
        "{\n .reg .pred p, e;\n setp.ne.b32 p, %4, 0;\n elect.sync _|e, 0xffffffff;\n"
        " @e tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n}\n" ::"r"(tmem_d),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"((unsigned)accumulate)
        : "memory");
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

// Warp roles (twenty warps): warps 0-7 drain the accumulators (warp w
// reads TMEM lanes 32 (w % 4) .. +31, i.e. time steps, and the column half
// w / 4, stages them with the bias, and the eight warps then store the tile
// in whole rows), warp 8 issues the MMAs (one lane, elect.sync), warps 9-19
// stage sigmoid tiles (the conversion is the slowest role, so it gets the
// most warps).  Tiles and accumulators (NBUF of each) are handed over on
// mbarriers -- full / empty for the sigmoid tiles, acc_full / acc_empty for
// the accumulators -- so no role waits at a CTA-wide barrier in the steady
// state.
constexpr int kGateEpiWarps = 8, kGateMmaWarp = 8, kGateProdWarp0 = 9;
constexpr int kGateProdThreads = kGateThreads - 32 * kGateProdWarp0;

// grid = H * groups CTAs; CTA (h = blockIdx.x % H, j = blockIdx.x / H) takes
// the tiles j, j + groups, ... of head h, tile = b * tiles_per_row + t0 / 128.
// vec_in: a's rows allow 4-channel vector loads; vec_out: g allows 16-byte stores.
template <int C, int KT, typename IO>
__global__ void __launch_bounds__(kGateThreads, 1)
    mhf_gate_kernel(const IO *__restrict__ a, const float *__restrict__ w, const float *__restrict__ bias,
                    IO *__restrict__ g, int L, int D, int H, int groups, int tiles_per_row, int num_tiles,
                    int vec_in, int vec_out, const __grid_constant__ CUtensorMap tma_a, int use_tma) {
    using Cfg = GateCfg<C, KT>;
    constexpr int NB = Cfg::NBUF;
    extern __shared__ unsigned char gate_smem_raw[];
    unsigned char *sm = reinterpret_cast<unsigned char *>(((uintptr_t)gate_smem_raw + 127) & ~(uintptr_t)127);
    const unsigned sb = smem_u32(sm);
    float *sbias = reinterpret_cast<float *>(sm + Cfg::OFF_BIAS);
    // full[NB], empty[NB], acc_full[NB], acc_empty[NB], loaded[NB], then the TMEM slot
    uint64_t *full = reinterpret_cast<uint64_t *>(sm + Cfg::OFF_BAR);
    uint64_t *empty = full + NB, *acc_full = full + 2 * NB, *acc_empty = full + 3 * NB, *loaded = full + 4 * NB;
    unsigned *tslot = reinterpret_cast<unsigned *>(loaded + NB);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int h = blockIdx.x % H;
    const int64_t col0 = (int64_t)h * C;
    const int first = blockIdx.x / H;

    if (tid == 0)
        for (int i = 0; i < NB; ++i) {
            mbar_init(full + i, kGateThreads / 32 - kGateProdWarp0);  // one arrival per producer warp
            mbar_init(empty + i, 1);                                  // tcgen05.commit
            mbar_init(acc_full + i, 1);                               // tcgen05.commit
            mbar_init(acc_empty + i, kGateEpiWarps);                  // one arrival per epilogue warp
            mbar_init(loaded + i, 1);                                 // TMA of a tile's input
        }
    __syncthreads();  // the barriers are initialised before any role uses them

    // The producers start on their first tiles at once; meanwhile the other
    // warps (MMA and epilogue) allocate TMEM and stage the head's weights and
    // bias, which only they use.
    constexpr int SET = 32 * kGateProdWarp0;  // threads of the MMA and epilogue roles
    unsigned tmem = 0;
    if (warp < kGateProdWarp0) {
        if (warp == 0) tmem_alloc(tslot, Cfg::TMEM_COLS);
        // The head's weights, split into fp16 hi / lo, in the K-major layout: tap
        // k, chunk c/8, output channel n, element c%8.  The head's block of w
        // ([D][C][K], C K contiguous floats per output channel n) is read with
        // coalesced 16-byte loads (vec_w: the block is 16-byte aligned) and each
        // element is split and placed by 2-byte stores.  (The block is read once
        // per CTA, from L2 after the first CTA of the head.)
        {
            const float *wh = w + col0 * C * KT;
            constexpr int NW = C * C * KT;  // the head's weights
            auto place = [&](int e, float x) {  // element e = (n C + c) KT + k
                const int k = e % KT, c = (e / KT) % C, n = e / (KT * C);
                const unsigned off = k * Cfg::W_TAP + (c >> 3) * Cfg::LBO_W + n * 16u + (c & 7) * 2u;
                const __half hi = __float2half_rn(x), lo = __float2half_rn(x - __half2float(hi));
                *reinterpret_cast<__half *>(sm + Cfg::OFF_WHI + off) = hi;
                *reinterpret_cast<__half *>(sm + Cfg::OFF_WLO + off) = lo;
            };
            if (((uintptr_t)wh & 15) == 0) {
#pragma unroll 2
                for (int q4 = tid; q4 < NW / 4; q4 += SET) {
                    const float4 x = __ldg(reinterpret_cast<const float4 *>(wh) + q4);
                    place(4 * q4, x.x);
                    place(4 * q4 + 1, x.y);
                    place(4 * q4 + 2, x.z);
                    place(4 * q4 + 3, x.w);
                }
            } else {
                for (int e = tid; e < NW; e += SET) place(e, __ldg(wh + e));
            }
        }
        static_assert(SET >= 64, "the bias is staged by the first 64 threads");
        if (tid < C) sbias[tid] = bias ? __ldg(bias + col0 + tid) : 0.0f;
        fence_proxy_async_smem();  // the weights are read by the tensor core
        tc_fence_before_sync();
        bar_sync(3, SET);
        tc_fence_after_sync();
        tmem = *tslot;
    }
    bool ok = true;    // every wait of this thread's role completed
    int last_it = -1;  // MMA warp: the last tile whose MMAs it committed

    if (warp >= kGateProdWarp0) {
        // ---- producers: sigmoid tiles, split into fp16 hi / lo, into buffer it % NB.
        // Item i of a tile is time step r = i / (C/4) (tile row, t = t0 - (KT-1) + r)
        // and channels 4 c4 .. 4 c4 + 3, c4 = i % (C/4): 8-byte halves of 16-byte chunks.
        const int pt = tid - 32 * kGateProdWarp0;
        constexpr int NITEM = Cfg::ROWS * Cfg::C4;
        constexpr int NU = (NITEM + kGateProdThreads - 1) / kGateProdThreads;
        // sigmoid of item j of this thread (zero outside [0, L): the convolution's padding),
        // split and stored into buffer buf
        auto put = [&](int buf, int t0, int j, float4 x) {
            const int i = pt + j * kGateProdThreads;
            const int r = i / Cfg::C4, c4 = i % Cfg::C4;
            const int t = t0 - (KT - 1) + r;
            float4 sg = make_float4(0.f, 0.f, 0.f, 0.f);
            if (t >= 0 && t < L) sg = make_float4(logistic(x.x), logistic(x.y), logistic(x.z), logistic(x.w));
            uint2 hi, lo;
            split4_f16(sg, hi, lo);
            unsigned char *ahi = sm + buf * 2 * Cfg::A_BYTES;
            const unsigned off = (c4 >> 1) * Cfg::LBO_A + r * 16u + (c4 & 1) * 8u;
            *reinterpret_cast<uint2 *>(ahi + off) = hi;
            *reinterpret_cast<uint2 *>(ahi + Cfg::A_BYTES + off) = lo;
        };
        auto publish = [&](int buf) {
            fence_proxy_async_smem();  // this thread's tile stores, before the tensor core reads them
            __syncwarp();
            if (lane == 0) mbar_arrive(full + buf);
        };
        int it = 0;
        constexpr bool kTmaIn = sizeof(IO) == 4;
        if (kTmaIn && use_tma) {
            // a tile's input [ROWS t][C ch] arrives by one TMA box in the buffer's input
            // tile (rows outside [0, L) read as zero and are masked in put)
            auto fetch = [&](int tile, int buf) {
                const int b = tile / tiles_per_row, t0 = (tile % tiles_per_row) * kGateM;
                fence_proxy_async_smem();
                mbar_arrive_expect_tx(loaded + buf, (unsigned)(Cfg::ROWS * C * 4));
                tma_load_3d(sm + Cfg::OFF_RAW + buf * Cfg::RAW_BYTES, &tma_a, (int)col0, t0 - (KT - 1), b,
                            loaded + buf);
            };
            int fetched = -1;  // thread pt == 0: the last tile iteration whose input it requested
            if (pt == 0 && first < num_tiles) {
                fetch(first, 0);
                fetched = 0;
            }
            for (int tile = first; tile < num_tiles; tile += groups, ++it) {
                const int buf = it % NB;
                // every producer agrees on whether the input arrived in time; past this
                // barrier no producer reads the previous tile's input tile any more
                if (!bar_and(1, kGateProdThreads, mbar_wait_bounded(loaded + buf, (it / NB) & 1u))) {
                    ok = false;
                    break;
                }
                // the next tile's input into the other input tile, while this one is converted
                const int nt = tile + groups;
                if (pt == 0 && nt < num_tiles) {
                    fetch(nt, (it + 1) % NB);
                    fetched = it + 1;
                }
                // the sigmoid buffer is free once the MMAs of the tile NB back are done
                if (it >= NB && !bar_and(1, kGateProdThreads, mbar_wait_bounded(empty + buf, (it / NB - 1) & 1u))) {
                    ok = false;
                    break;
                }
                const int t0 = (tile % tiles_per_row) * kGateM;
                const unsigned char *raw = sm + Cfg::OFF_RAW + buf * Cfg::RAW_BYTES;
#pragma unroll
                for (int j = 0; j < NU; ++j) {
                    const int i = pt + j * kGateProdThreads;
                    if (i >= NITEM) break;
                    put(buf, t0, j, *reinterpret_cast<const float4 *>(raw + (i / Cfg::C4) * (C * 4) + (i % Cfg::C4) * 16));
                }
                publish(buf);
            }
            // a request still in flight lands before the CTA's shared memory is released
            if (pt == 0 && fetched >= it && fetched >= 0) mbar_wait_bounded(loaded + fetched % NB, (fetched / NB) & 1u);
        } else {
            // loads from global memory, the next tile's into the other register set
            // before this tile's sigmoid is computed
            Raw4<IO> raw0[NU], raw1[NU];
            auto load = [&](Raw4<IO>(&rw)[NU], int tile) {
                const int b = tile / tiles_per_row;
                const int t0 = (tile % tiles_per_row) * kGateM;
                const IO *base = a + (int64_t)b * L * D + col0;
#pragma unroll
                for (int j = 0; j < NU; ++j) {
                    const int i = pt + j * kGateProdThreads;
                    const int r = i / Cfg::C4, c4 = i % Cfg::C4;
                    const int t = t0 - (KT - 1) + r;
                    if (i < NITEM && t >= 0 && t < L)
                        rw[j].load(base + (int64_t)t * D + c4 * 4, vec_in != 0);
                    else
                        rw[j].zero();
                }
            };
            auto produce = [&](Raw4<IO>(&rw)[NU], int tile, int itx) -> bool {
                const int buf = itx % NB;
                if (itx >= NB && !mbar_wait_bounded(empty + buf, ((itx / NB) - 1) & 1u)) return false;
                const int t0 = (tile % tiles_per_row) * kGateM;
#pragma unroll
                for (int j = 0; j < NU; ++j) {
                    if (pt + j * kGateProdThreads >= NITEM) break;
                    put(buf, t0, j, rw[j].f32());
                }
                publish(buf);
                return true;
            };
            if (first < num_tiles) load(raw0, first);
            for (int tile = first; tile < num_tiles && ok; tile += 2 * groups, it += 2) {
                const int t1 = tile + groups, t2 = tile + 2 * groups;
                if (t1 < num_tiles) load(raw1, t1);
                ok = produce(raw0, tile, it);
                if (!ok || t1 >= num_tiles) break;
                if (t2 < num_tiles) load(raw0, t2);
                ok = produce(raw1, t1, it + 1);
            }
        }
    } else if (warp == kGateMmaWarp) {
        // ---- MMA issue: 3 split products x K taps x C/16 steps of 16 channels per tile
        constexpr uint32_t idesc = gate_idesc_f16(C);
        int it = 0;
        last_it = -1;
        for (int tile = first; tile < num_tiles; tile += groups, ++it) {
            const int buf = it % NB;
            bool got = mbar_wait_bounded(full + buf, (it / NB) & 1u);
            if (got && it >= NB) got = mbar_wait_bounded(acc_empty + buf, ((it / NB) - 1) & 1u);
            if (!__all_sync(0xffffffffu, got)) {
                ok = false;
                break;
            }
            tc_fence_after_sync();
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
                    for (int s2 = 0; s2 < C / 16; ++s2) {
                        umma_f16_elect(d, a0 + ((k * 16u + 2u * s2 * Cfg::LBO_A) >> 4),
                                       b0 + ((k * Cfg::W_TAP + 2u * s2 * Cfg::LBO_W) >> 4), idesc, step > 0);
                        ++step;
                    }
                }
            }
            umma_commit_elect(empty + buf);     // the sigmoid tile may be restaged
            umma_commit_elect(acc_full + buf);  // the accumulator is ready
            last_it = it;
        }
    } else if (warp < kGateEpiWarps) {
        // ---- epilogue: accumulator rows 32 (warp % 4) + lane (time steps), column half warp / 4, + bias, store
        float *stg = reinterpret_cast<float *>(sm + Cfg::OFF_OUT);
        constexpr int EPT = 32 * kGateEpiWarps;  // epilogue threads
        int it = 0;
        for (int tile = first; tile < num_tiles; tile += groups, ++it) {
            const int buf = it % NB;
            // the epilogue warps agree on whether the accumulator arrived (with the
            // staging this is also their barrier: the previous tile's rows are read back)
            bool got = mbar_wait_bounded(acc_full + buf, (it / NB) & 1u);
            if constexpr (Cfg::STAGE_OUT)
                got = bar_and(2, EPT, got);
            else
                got = __all_sync(0xffffffffu, got);
            if (!got) {
                ok = false;
                break;
            }
            tc_fence_after_sync();
            constexpr int CH = C / 2;  // this warp's columns: [cb, cb + CH)
            const int cb = CH * (warp >> 2);
            float v[CH];
            const unsigned trow = tmem + buf * C + cb + ((unsigned)(32 * (warp & 3)) << 16);
            if constexpr (CH == 32) {
                float x0[16], x1[16];
                tmem_ld16x2(trow, trow + 16, x0, x1);
#pragma unroll
                for (int i = 0; i < 16; ++i) {
                    v[i] = x0[i];
                    v[16 + i] = x1[i];
                }
            } else if constexpr (CH == 16) {
                tmem_ld16(trow, v);
            } else {
                tmem_ld8(trow, v);
            }
            tc_fence_before_sync();
            __syncwarp();
            if (lane == 0) mbar_arrive(acc_empty + buf);  // the MMAs of tile it + NB may overwrite it
            const int b = tile / tiles_per_row, t0 = (tile % tiles_per_row) * kGateM, m = 32 * (warp & 3) + lane;
            if constexpr (Cfg::STAGE_OUT) {
                // this warp's half of row m into the staging, then the tile in whole rows:
                // C / 4 threads per time step
                float *srow = stg + m * Cfg::OUT_PITCH + cb;
#pragma unroll
                for (int c = 0; c < CH; c += 4)
                    *reinterpret_cast<float4 *>(srow + c) = make_float4(
                        v[c] + sbias[cb + c], v[c + 1] + sbias[cb + c + 1], v[c + 2] + sbias[cb + c + 2], v[c + 3] + sbias[cb + c + 3]);
                bar_sync(2, EPT);
#pragma unroll 4
                for (int q = tid; q < kGateM * Cfg::C4; q += EPT) {
                    const int row = q / Cfg::C4, c4 = q - row * Cfg::C4, t = t0 + row;
                    if (t < L) {
                        const float4 x = *reinterpret_cast<const float4 *>(stg + row * Cfg::OUT_PITCH + 4 * c4);
                        const float xv[4] = {x.x, x.y, x.z, x.w};
                        store4(g + ((int64_t)b * L + t) * D + col0 + 4 * c4, xv, vec_out != 0);
                    }
                }
            } else {
                const int t = t0 + m;
                if (t < L) {
                    IO *gt = g + ((int64_t)b * L + t) * D + col0 + cb;
#pragma unroll
                    for (int c = 0; c < CH; c += 4) {
                        const float xv[4] = {v[c] + sbias[cb + c], v[c + 1] + sbias[cb + c + 1],
                                             v[c + 2] + sbias[cb + c + 2], v[c + 3] + sbias[cb + c + 3]};
                        store4(gt + c, xv, vec_out != 0);
                    }
                }
            }
        }
    }
    if (!ok && lane == 0) atomicOr(&g_cc_fault, kFaultMmaWait);
    // every MMA this CTA issued has completed before the accumulators are
    // freed: the last commit tracks all of them (a phase the epilogue has
    // already seen completes the wait at once)
    if (warp == kGateMmaWarp && last_it >= 0) mbar_wait_bounded(acc_full + last_it % NB, (last_it / NB) & 1u);
    tc_fence_before_sync();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after_sync();
        tmem_dealloc(tmem, Cfg::TMEM_COLS);
    }
}

}  // namespace ccv
