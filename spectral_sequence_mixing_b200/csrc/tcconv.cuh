// tcconv.cuh -- the causal convolution of bf16 rows with N = 8192 (2048 < L <= 4096)
// on the fifth-generation tensor cores: the DFTs of the transform are dense
// matrix products (the Monarch / matrix-FFT route Caracal: Causal
// Architecture via Spectral Mixing names in its related work), run as
// tcgen05 kind::f16 MMAs with fp32 accumulators in tensor memory.
//
// Method (Caracal, "Key design 1" and "Key design 2"): per (b, d) row,
// z_t = v_t sv + i g_t sg (t < L, zero up to N/2 = 4096; sv, sg powers of two
// bringing each stream to unit mean square), odd-frequency spectrum
// Z_k = sum_t z_t theta^(t(2k+1)), theta = exp(-i pi / N), spectral product
// X_k = -i (Z_k + conj Z_m)(Z_k - conj Z_m) = 4 sv sg V_k G_k (m = N-1-k, the
// mirror bin), inverse transform, real part, truncation to t < L; outputs
// t < 64 are replaced by the direct sum.
//
// Factorisation.  t = n2 + 128 n1 (n1 < 32 carries data, n1 < 64 in the
// padded transform), k = k1 + 64 k2, k2 = 2 q + e, n2 = m + 64 h:
//   stage 1  Y[k1][n2]  = sum_n1 F1[k1][n1] z[n2 + 128 n1],
//                         F1 = omega_128^(n1 (2 k1 + 1))            (64 x 32)
//   twiddle  T1[k1][n2] = theta^(n2 (2 k1 + 1)) and the first radix-2 step
//            of the 128-point DFT over n2, on the CUDA cores:
//            U_e[k1][m] = w^(m e) (T1 Y[m] + (-1)^e T1 Y[m + 64]), w = omega_128
//   stage 2  Z[k1 + 64 (2q + e)] = sum_m omega_64^(m q) U_e[k1][m]  (64 x 64)
//   product  mirror of (k1, e, q) is (63 - k1, 1 - e, 63 - q)
//   stage 3  the inverse 64-point DFT over q (the same matrix applied to
//            conj X: an inverse DFT is conj(DFT(conj x)))
//   twiddle  the inverse radix-2 step and conj(T1)
//   stage 4  Re y[n2 + 128 n1] = Re sum_k1 conj(F1[k1][n1]) Y''[k1][n2], n1 < 32.
// Each stage is a real matrix product of the complex DFT's real form
// [[Re F, -Im F], [Im F, Re F]] (fp16 operands, exact in the MMA, fp32
// accumulation); the twiddles and the spectral product run in fp32.  The
// stage matrices carry power-of-two scales (1/4, 1/8) that keep every fp16
// operand near unit size; the output scale undoes them exactly.
//
// Operands (shared memory, no swizzle; "K-major": rows of 16-byte K chunks,
// chunk c of row r at c * 2048 + r * 16; "MN-major": 16-byte runs of 8
// consecutive rows, element (n, k) at (n / 8) 128 + (n % 8) 2 + (k % 8) 16 + (k / 8) 2048):
//   stage 1: A = F1 (rows: k1 and re/im, lane order below), B = data rows n2
//            (K = n1 < 32 and re/im), D[lane][n2];
//   stage 2: A = data rows (k1, e) (K = m and re/im), B = F64 (rows q and
//            re/im), D[lane][q, re/im];  stage 3: the same with conj X;
//   stage 4: A = conj F1 (rows n1 < 32, real part only; rows 32..127 zero),
//            B = data MN-major (N = n2, K = k1 and re/im), D[n1][n2].
// Lane l = 32 w + 2 j + b (w < 4, j < 16, b < 2) of stages 1..3 holds
// k1 = 8 w + j (j < 8) or 63 - 8 w - (j - 8) (j >= 8), and b = re/im in
// stage 1, b = e in stages 2 and 3: the lanes a thread needs -- the other
// half of its complex value (l ^ 1), the mirror bin's (l ^ 17), the other
// radix-2 branch (l ^ 1) -- are in its own warp, so warp shuffles exchange
// them.  The warps sharing a lane quarter split the columns.
//
// Channel groups: a cluster of 4 CTAs takes 8 adjacent channels of one
// batch (16-byte accesses per time step), two rows per CTA.  CTA q loads time
// steps [1024 q, 1024 q + 1024), which are exactly the K chunks 2q and 2q+1
// of every row's stage-1 operand, and stores them into the owning CTAs'
// operands over distributed shared memory; at the end every CTA sends its
// outputs to the CTA owning their time steps, which stores whole 16-byte
// groups.  Row norms for the scaling are reduced across the cluster the same
// way.  A CTA's two rows alternate on the tensor core: while it runs a stage
// of one row, the sixteen warps drain the other row's previous stage
// (separate operand buffers and accumulators).  The twiddles come from a
// 32 KiB table in shared memory.  Clusters are persistent over the channel
// groups.  Every MMA completion wait is bounded; no load uses cluster
// multicast.
#pragma once

#include <cooperative_groups.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <stdint.h>

#include "tcgen05.cuh"
#include "tma.cuh"

namespace ccv {

constexpr int kTcN = 8192;
constexpr int kTcLMax = kTcN / 2;
constexpr int kTcThreads = 512;
constexpr int kTcCluster = 4;                  // CTAs per cluster
constexpr int kTcRows = 2;                     // rows (channels) per CTA
constexpr int kTcGroup = kTcCluster * kTcRows; // channels per cluster
constexpr int kTcSpan = kTcLMax / kTcCluster;  // time steps each CTA loads and stores
constexpr int kTcHead = 64;                    // outputs t < kTcHead by direct summation
constexpr unsigned kTcChunkPitch = 2048;       // bytes between K chunks (128 rows x 16 B)
// shared-memory map (bytes from a 128-byte aligned base)
constexpr unsigned kTcOffA1 = 0;                     // F1 / 4, 128 x 64 fp16, K-major
constexpr unsigned kTcOffB2 = 16384;                 // F64 / 8, 128 x 128 fp16, K-major
constexpr unsigned kTcOffA4 = kTcOffB2 + 32768;      // conj F1 / 4, 128 x 128 fp16, K-major
// F0[k1][m] = theta^(m (2 k1 + 1)) / 2, float2, rows of kTcTwPitch entries: the
// 16 k1 rows a warp reads at one m then fall on 16 distinct bank pairs
constexpr int kTcTwPitch = 65;
constexpr unsigned kTcOffTw = kTcOffA4 + 32768;
constexpr unsigned kTcOffW = kTcOffTw + 64 * kTcTwPitch * 8;  // w[m] = omega_128^m, then c64[k1] = theta^(64 (2 k1 + 1))
constexpr unsigned kTcConstBytes = kTcOffW + 2 * 64 * 8;  // all of the above, staged from global once per CTA
constexpr unsigned kTcOffData = kTcConstBytes;            // two stage operands (rows 0, 1), 32 KiB each
constexpr unsigned kTcOffIn = kTcOffData + 2 * 32768;     // next group's input [v, g][1024 t][8 ch] bf16 (TMA)
constexpr unsigned kTcInBytes = 2u * kTcSpan * kTcGroup * 2u;
constexpr unsigned kTcOffOut = kTcOffIn + kTcInBytes;     // outputs of this CTA's time steps [8 ch][1024] bf16;
                                                          // before the outputs arrive: [16 warps][8] norm partials
constexpr unsigned kTcOffHead = kTcOffOut + kTcGroup * kTcSpan * 2;  // [2 rows][v, g][64] fp32
constexpr unsigned kTcOffRed = kTcOffHead + kTcRows * 2 * kTcHead * 4;  // [16] CTA sums, [16] scales
constexpr unsigned kTcOffBar = kTcOffRed + (16 + 16) * 4;
constexpr unsigned kTcSmemBytes = kTcOffBar + 40 + 128;  // + 3 barriers, TMEM slot, 2 counters, alignment slack
constexpr int kTcBoxT = 256;                             // TMA box: [kTcBoxT t][8 ch]
constexpr unsigned kTcTmemCols = 256;                    // one 128-column accumulator per row
constexpr float kTcOutScale = 8.0f;  // 1 / (4 N) times the inverse of the stage scales (1/64)^2 (1/64)
constexpr unsigned kFaultTcWait = 4u;
static_assert(kTcSmemBytes <= 232448, "shared memory");
static_assert(((kTcThreads / 32) & (kTcThreads / 32 - 1)) == 0, "the MMA issue counter counts warps in powers of two");

// Stage matrices and twiddle tables in their shared-memory byte layout;
// filled once per device from fp64 values.
__device__ __align__(16) uint4 g_tc_consts[kTcConstBytes / 16];

__host__ __device__ constexpr int tc_kappa(int l) {
    return ((l & 31) >> 1) < 8 ? 8 * (l >> 5) + ((l & 31) >> 1) : 63 - 8 * (l >> 5) - (((l & 31) >> 1) - 8);
}

// Instruction descriptor, kind::f16 with fp16 A and B, fp32 accumulator,
// M = 128, N = 128; b_mn: B is MN-major.
__host__ __device__ constexpr uint32_t tc_idesc(bool b_mn) {
    return (1u << 4) | (0u << 7) | (0u << 10) | ((b_mn ? 1u : 0u) << 16) | ((128u >> 3) << 17) | ((128u >> 4) << 24);
}

__device__ __forceinline__ void umma_f16(unsigned tmem_d, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                         bool accumulate) {
    asm volatile(
        "{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n"
        " tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n}\n" ::"r"(tmem_d),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"((unsigned)accumulate)
        : "memory");
}

__device__ __forceinline__ uint32_t pack_h2(float lo, float hi) {
    const __half2 h = __floats2half2_rn(lo, hi);
    return *reinterpret_cast<const uint32_t *>(&h);
}
__device__ __forceinline__ uint32_t pack_bf2(float lo, float hi) {
    const __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<const uint32_t *>(&h);
}

__device__ __forceinline__ uint32_t tc_mapa(uint32_t addr, int rank) {
    uint32_t r;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;\n" : "=r"(r) : "r"(addr), "r"(rank));
    return r;
}
__device__ __forceinline__ void st_cluster_v4(uint32_t addr, uint4 v) {
    asm volatile("st.shared::cluster.v4.b32 [%0], {%1, %2, %3, %4};\n" ::"r"(addr), "r"(v.x), "r"(v.y), "r"(v.z),
                 "r"(v.w)
                 : "memory");
}
__device__ __forceinline__ void st_cluster_b16(uint32_t addr, uint16_t v) {
    asm volatile("st.shared::cluster.b16 [%0], %1;\n" ::"r"(addr), "h"(v) : "memory");
}
__device__ __forceinline__ float ld_cluster_f(uint32_t addr) {
    float x;
    asm volatile("ld.shared::cluster.f32 %0, [%1];\n" : "=f"(x) : "r"(addr) : "memory");
    return x;
}
__device__ __forceinline__ void fence_proxy_async_all() { asm volatile("fence.proxy.async;" ::: "memory"); }

__device__ __forceinline__ float2 tc_cmul(float2 a, float2 b) {
    return make_float2(fmaf(a.x, b.x, -a.y * b.y), fmaf(a.x, b.y, a.y * b.x));
}
__device__ __forceinline__ float2 tc_cmulc(float2 a, float2 b) {  // a * conj(b)
    return make_float2(fmaf(a.x, b.x, a.y * b.y), fmaf(a.y, b.x, -a.x * b.y));
}

// 4 bf16 channels of one time step as fp32 (zeros when !ok); p 8-byte aligned when vec.
__device__ __forceinline__ void tc_load4(const __nv_bfloat16 *p, int nch, bool vec, bool ok, float (&o)[4]) {
#pragma unroll
    for (int c = 0; c < 4; ++c) o[c] = 0.f;
    if (!ok) return;
    if (vec) {
        const uint2 w = __ldg(reinterpret_cast<const uint2 *>(p));
        o[0] = __uint_as_float(w.x << 16);
        o[1] = __uint_as_float(w.x & 0xFFFF0000u);
        o[2] = __uint_as_float(w.y << 16);
        o[3] = __uint_as_float(w.y & 0xFFFF0000u);
    } else {
#pragma unroll
        for (int c = 0; c < 4; ++c)
            if (c < nch) o[c] = __bfloat162float(p[c]);
    }
}

// grid = clusters x 4 CTAs; cluster j takes the channel groups j, j + clusters, ...
// (group = b * groups_per_batch + d0 / 8).  rev bit 0: read v reversed in
// time; bit 1: write r reversed.  vec_ok: 16-byte group accesses allowed.
__global__ void __cluster_dims__(kTcCluster, 1, 1) __launch_bounds__(kTcThreads, 1)
    tcconv_kernel(const __nv_bfloat16 *__restrict__ v, const __nv_bfloat16 *__restrict__ g,
                  __nv_bfloat16 *__restrict__ r, int L, int D, int groups_per_batch, int num_groups, int rev,
                  int vec_ok, const __grid_constant__ CUtensorMap tmv, const __grid_constant__ CUtensorMap tmg,
                  int use_tma) {
    namespace cg = cooperative_groups;
    cg::cluster_group cluster = cg::this_cluster();
    extern __shared__ unsigned char tc_smem_raw[];
    unsigned char *sm = reinterpret_cast<unsigned char *>(((uintptr_t)tc_smem_raw + 127) & ~(uintptr_t)127);
    const unsigned sb = smem_u32(sm);
    const float2 *tw = reinterpret_cast<const float2 *>(sm + kTcOffTw);    // [64 k1][kTcTwPitch]
    const float2 *wtab = reinterpret_cast<const float2 *>(sm + kTcOffW);   // [64 m]
    const float2 *c64 = wtab + 64;                                          // [64 k1]
    float *red = reinterpret_cast<float *>(sm + kTcOffOut);  // [16 warps][8] (before the outputs arrive)
    float *tot = reinterpret_cast<float *>(sm + kTcOffRed);  // [16] this CTA's sums (v: 0..7, g: 8..15)
    float *scl = tot + 16;                                    // [16] scales (sv: 0..7, sg: 8..15)
    const uint16_t *sin_v = reinterpret_cast<const uint16_t *>(sm + kTcOffIn);  // [1024 t][8 ch]
    const uint16_t *sin_g = sin_v + kTcSpan * kTcGroup;
    float *head = reinterpret_cast<float *>(sm + kTcOffHead);  // [2 rows][v, g][64]
    uint16_t *outs = reinterpret_cast<uint16_t *>(sm + kTcOffOut);  // [8 channels][1024 slots]
    uint64_t *bar = reinterpret_cast<uint64_t *>(sm + kTcOffBar);   // one per row, then the input barrier
    unsigned *tslot = reinterpret_cast<unsigned *>(sm + kTcOffBar + 24);
    unsigned *icnt = reinterpret_cast<unsigned *>(sm + kTcOffBar + 32);  // per row: warps done with its operand

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int q = (int)cluster.block_rank();  // this CTA: channels 2q, 2q+1 of the group; time steps [1024 q, +1024)
    const int cid = blockIdx.x / kTcCluster, nclusters = gridDim.x / kTcCluster;

    if (warp == 0) tmem_alloc(tslot, kTcTmemCols);
    if (tid == 0) {
        mbar_init(bar, 1);
        mbar_init(bar + 1, 1);
        mbar_init(bar + 2, 1);
        icnt[0] = 0u;
        icnt[1] = 0u;
    }
    // TMA: this CTA's time steps of group gi (v reversed in time when rev & 1:
    // its staged rows then run backwards), completing on bar[2]
    auto prefetch = [&](int gi) {
        const int b = gi / groups_per_batch, dd = (gi - b * groups_per_batch) * kTcGroup;
        const int tv0 = (rev & 1) ? L - kTcSpan * (q + 1) : kTcSpan * q;
        fence_proxy_async_smem();
        mbar_arrive_expect_tx(bar + 2, kTcInBytes);
#pragma unroll
        for (int k = 0; k < kTcSpan / kTcBoxT; ++k) {
            tma_load_3d(sm + kTcOffIn + k * kTcBoxT * kTcGroup * 2, &tmv, dd, tv0 + k * kTcBoxT, b, bar + 2);
            tma_load_3d(sm + kTcOffIn + kTcSpan * kTcGroup * 2 + k * kTcBoxT * kTcGroup * 2, &tmg, dd,
                        kTcSpan * q + k * kTcBoxT, b, bar + 2);
        }
    };
    unsigned in_phase = 0;
    bool in_flight = false;  // a prefetch is outstanding on bar[2] (uniform over the CTA)
    for (unsigned i = tid; i < kTcConstBytes / 16; i += kTcThreads) reinterpret_cast<uint4 *>(sm)[i] = g_tc_consts[i];
    tc_fence_before_sync();
    __syncthreads();
    tc_fence_after_sync();
    const unsigned tmem = *tslot;
    unsigned phase = 0;    // bit x: parity awaited next on bar[x]
    unsigned pending = 0;  // bit x: a commit on bar[x] not yet waited for
    bool ok = true;        // every MMA wait so far completed

    const int l = 32 * (warp & 3) + lane;  // TMEM lane this thread reads
    const int cq = warp >> 2;              // column quarter
    const int k1 = tc_kappa(l), eb = l & 1;
    const float2 ck = c64[k1];
    if (use_tma && cid < num_groups) {
        if (tid == 0) prefetch(cid);
        in_flight = true;
    }
    // The direct head's inputs (thread tid < 256: row tid >> 7, v or g, time
    // step tid & 63) of group gi, loaded a group ahead so their latency hides
    // behind the previous group's stages.
    auto load_head = [&](int gi) -> float {
        if (tid >= 4 * kTcHead || gi >= num_groups) return 0.f;
        const int bb = gi / groups_per_batch, dd = (gi - bb * groups_per_batch) * kTcGroup;
        const int x = tid >> 7, arr = (tid >> 6) & 1, t = tid & 63, c = 2 * q + x;
        if (t >= L || c >= D - dd) return 0.f;
        const int ts = (arr == 0 && (rev & 1)) ? L - 1 - t : t;
        return __bfloat162float((arr ? g : v)[(int64_t)bb * L * D + dd + c + (int64_t)ts * D]);
    };
    float hreg = load_head(cid);
    // Row norms of group gi: the CTA's partial sums over its time steps (tot)
    // are published by a cluster barrier.  For every group after the first,
    // they are computed from the staged input at the end of the previous
    // group (before its last barrier), so that group needs no barrier of
    // its own for them.
    bool have_norms = false;
    // partial sums of the squares of this thread's (v, g) elements -> warp partials in red2 -> tot
    auto norms = [&](const float (&av)[4][4], const float (&ag)[4][4], float *red2) {
        float sq[8];
#pragma unroll
        for (int c = 0; c < 4; ++c) {
            sq[c] = 0.f;
            sq[4 + c] = 0.f;
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                sq[c] = fmaf(av[i][c], av[i][c], sq[c]);
                sq[4 + c] = fmaf(ag[i][c], ag[i][c], sq[4 + c]);
            }
        }
#pragma unroll
        for (int c = 0; c < 8; ++c) {
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) sq[c] += __shfl_xor_sync(0xffffffffu, sq[c], o);
        }
        if (lane == 0)
#pragma unroll
            for (int c = 0; c < 8; ++c) red2[warp * 8 + c] = sq[c];
        __syncthreads();
        if (tid < 16) {  // channel c = tid & 7 (half c / 4: warps 8 (c / 4) .. +8), stream tid >> 3
            const int c = tid & 7, st = tid >> 3, h = c >> 2;
            float acc = 0.f;
            for (int w2 = 8 * h; w2 < 8 * h + 8; ++w2) acc += red2[w2 * 8 + 4 * st + (c & 3)];
            tot[tid] = acc;
        }
    };
    // this thread's staged elements (time steps n2 + 128 (4 (2q + kl) + i), channels [4 hf, +4))
    auto read_staged = [&](int n2i, int kl, int hf, float (&av)[4][4], float (&ag)[4][4]) {
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const int tl = n2i + 128 * (4 * kl + i);
            const uint2 wv = *reinterpret_cast<const uint2 *>(sin_v + ((rev & 1) ? kTcSpan - 1 - tl : tl) * 8 + 4 * hf);
            const uint2 wg = *reinterpret_cast<const uint2 *>(sin_g + tl * 8 + 4 * hf);
            av[i][0] = __uint_as_float(wv.x << 16);
            av[i][1] = __uint_as_float(wv.x & 0xFFFF0000u);
            av[i][2] = __uint_as_float(wv.y << 16);
            av[i][3] = __uint_as_float(wv.y & 0xFFFF0000u);
            ag[i][0] = __uint_as_float(wg.x << 16);
            ag[i][1] = __uint_as_float(wg.x & 0xFFFF0000u);
            ag[i][2] = __uint_as_float(wg.y << 16);
            ag[i][3] = __uint_as_float(wg.y & 0xFFFF0000u);
        }
    };

    // stage s (1..4) of row x: 4 or 8 MMAs of K = 16 (two 16-byte chunks each).
    // No CTA barrier: each warp, once its part of the operand is written and
    // its accumulator reads are done, counts itself on icnt[x] (acquire-
    // release); the last of the 16 warps issues the MMAs and the commit, so
    // no thread waits here.  The counter only grows (a multiple of 16 marks
    // the last arrival), so it needs no reset.  If the issuing thread's
    // earlier waits ran out it completes bar[x] itself instead, so that no
    // thread waits for a commit that will not come; the failure reaches
    // every thread at the end of the group.
    auto issue = [&](int s, int x) {
        fence_proxy_async_smem();
        tc_fence_before_sync();
        pending |= 1u << x;
        __syncwarp();
        if (lane == 0) {
            unsigned n;
            asm volatile("atom.acq_rel.cta.shared::cta.add.u32 %0, [%1], 1;"
                         : "=r"(n)
                         : "r"(smem_u32(icnt + x))
                         : "memory");
            if (((n + 1u) & (kTcThreads / 32 - 1)) == 0u) {
                if (!ok) {
                    mbar_arrive(bar + x);
                    return;
                }
                tc_fence_after_sync();
                const unsigned data = kTcOffData + (unsigned)x * 32768u;
                const unsigned a_off = s == 1 ? kTcOffA1 : (s == 4 ? kTcOffA4 : data);
                const unsigned b_off = (s == 1 || s == 4) ? data : kTcOffB2;
                const int nk = s == 1 ? 4 : 8;
                const bool b_mn = s == 4;
                const uint32_t idesc = tc_idesc(b_mn);
                for (int k = 0; k < nk; ++k) {
                    const uint64_t ad = umma_smem_desc(sb + a_off + 2u * k * kTcChunkPitch, kTcChunkPitch, 128u);
                    const uint64_t bd = b_mn ? umma_smem_desc(sb + b_off + 2u * k * 2048u, 2048u, 128u)
                                             : umma_smem_desc(sb + b_off + 2u * k * kTcChunkPitch, kTcChunkPitch, 128u);
                    umma_f16(tmem + 128u * x, ad, bd, idesc, k > 0);
                }
                umma_commit(bar + x);
            }
        }
    };
    // Every thread observes the completion itself (no CTA barrier): the
    // next commit to the same barrier comes only after every warp has
    // counted itself in the next issue(), which each thread reaches after
    // this wait.
    auto wait = [&](int x) {
        if ((pending >> x) & 1u) {
            const bool done = mbar_wait_bounded(bar + x, (phase >> x) & 1u);
            if (done) {
                phase ^= 1u << x;
                pending &= ~(1u << x);
            }
            ok = ok && done;
        }
        tc_fence_after_sync();
    };

    for (int grp = cid; grp < num_groups; grp += nclusters) {
        const int b = grp / groups_per_batch;
        const int d0 = (grp - b * groups_per_batch) * kTcGroup;
        const int nch = min(kTcGroup, D - d0);
        const bool vec = vec_ok && nch == kTcGroup;
        const int64_t base = (int64_t)b * L * D + d0;

        // ---- input: item (n2, chunk 2q + kl) of channels [4 hf, 4 hf + 4): time steps n2 + 128 (4 kc + i)
        const int n2i = tid & 127, kl = (tid >> 7) & 1, hf = tid >> 8;
        const int kc = 2 * q + kl;
        const int nh = max(0, min(4, nch - 4 * hf));  // channels of this thread's half that exist
        float xv[4][4], xg[4][4];
        bool staged = true;
        if (use_tma && in_flight) {
            // the copy engine zero-filled t >= L (and t < 0 for a reversed v) and d >= D
            if (tid == 0) staged = mbar_wait_bounded(bar + 2, in_phase);
            staged = __syncthreads_and(staged);
            if (staged) {
                in_phase ^= 1u;
                in_flight = false;
            }
        } else {
            __syncthreads();  // the previous group's stores have read the output staging (reused below)
        }
        ok = ok && staged;
        if (use_tma) {
            read_staged(n2i, kl, hf, xv, xg);
        } else {
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const int t = n2i + 128 * (4 * kc + i);
                const bool in = t < L && nh > 0;
                const int tv = (rev & 1) ? L - 1 - t : t;
                tc_load4(v + base + 4 * hf + (int64_t)(in ? tv : 0) * D, nh, vec, in, xv[i]);
                tc_load4(g + base + 4 * hf + (int64_t)(in ? t : 0) * D, nh, vec, in, xg[i]);
            }
        }
        if (tid < 4 * kTcHead) head[((tid >> 7) * 2 + ((tid >> 6) & 1)) * kTcHead + (tid & 63)] = hreg;
        if (!have_norms) {
            norms(xv, xg, red);  // red aliases the output staging, which no peer writes before barrier #2
            cluster.sync();      // #1: partial sums visible
        }
        if (tid < 16) {
            float a = 0.f;
            const uint32_t ad = smem_u32(tot + tid);
            for (int p = 0; p < kTcCluster; ++p) a += ld_cluster_f(tc_mapa(ad, p));
            // power of two bringing the stream's mean square to about 1; 0 marks an all-zero
            // stream (the exponent is clamped so the scale stays a normal float)
            scl[tid] = (a > 0.f && a <= 3.0e38f)
                           ? ldexpf(1.f, -max(-100, min(100, __float2int_rn(0.5f * log2f(a / (float)L)))))
                           : 0.f;
        }
        __syncthreads();
        {
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const int c = 4 * hf + j;  // channel: CTA c / 2, row c % 2
                const float sv = scl[c], sg = scl[8 + c];
                uint4 w;
                w.x = pack_h2(xv[0][j] * sv, xg[0][j] * sg);
                w.y = pack_h2(xv[1][j] * sv, xg[1][j] * sg);
                w.z = pack_h2(xv[2][j] * sv, xg[2][j] * sg);
                w.w = pack_h2(xv[3][j] * sv, xg[3][j] * sg);
                const uint32_t dst =
                    sb + kTcOffData + (unsigned)(c & 1) * 32768u + (unsigned)kc * kTcChunkPitch + (unsigned)n2i * 16u;
                st_cluster_v4(tc_mapa(dst, c >> 1), w);
            }
        }
        fence_proxy_async_all();
        cluster.sync();  // #2: every CTA's stage-1 operands are complete
        if (use_tma && grp + nclusters < num_groups && ok) {
            if (tid == 0) prefetch(grp + nclusters);
            in_flight = true;
        }
        hreg = load_head(grp + nclusters);

        issue(1, 0);
        issue(1, 1);
        // ---- the direct head of this CTA's rows while the tensor core starts:
        // r_t = sum_{j<=t} v_j g_{t-j}, t < 64, four threads per (row, t)
        {
            const int x = tid >> 8, t = (tid >> 2) & 63, part = tid & 3;
            const float *hv = head + (x * 2) * kTcHead, *hg = hv + kTcHead;
            float a = 0.f;
            for (int j = part; j <= t; j += 4) a = fmaf(hv[j], hg[t - j], a);
            a += __shfl_xor_sync(0xffffffffu, a, 1);
            a += __shfl_xor_sync(0xffffffffu, a, 2);
            const int c = 2 * q + x;
            if (part == 0) {  // time step t < 64 lives in CTA 0, slot t
                const bool live = scl[c] > 0.f && scl[8 + c] > 0.f;
                st_cluster_b16(tc_mapa(smem_u32(outs + c * kTcSpan + t), 0),
                               __bfloat16_as_ushort(__float2bfloat16_rn(live ? a : 0.f)));
            }
        }

        for (int s = 1; s <= 4; ++s) {
            for (int x = 0; x < kTcRows; ++x) {
                wait(x);
                const unsigned tl = tmem + 128u * x + ((unsigned)(32 * (warp & 3)) << 16);
                unsigned char *dat = sm + kTcOffData + (unsigned)x * 32768u;
                if (s == 1) {
                    // twiddle and radix-2 step.  Lane l holds re (l even) or im (l odd) of
                    // Y[k1][n2]; thread l forms both branches e of its half of the m range,
                    // U_e = F0[k1][m] w^(m e) (Y[m] + (-1)^e c64[k1] Y[m + 64]), and writes
                    // them to operand rows l & ~1 (e = 0) and l | 1 (e = 1)
                    float ya[16], yb[16];
                    tmem_ld16x2(tl + 16 * cq, tl + 64 + 16 * cq, ya, yb);  // n2 = m and m + 64, m in [16 cq, +16)
                    uint32_t w0[8], w1[8];
#pragma unroll
                    for (int u = 0; u < 8; ++u) {
                        // send the partner the half it owns, receive the other part of mine
                        const float pa = __shfl_xor_sync(0xffffffffu, eb ? ya[u] : ya[8 + u], 1);
                        const float pb = __shfl_xor_sync(0xffffffffu, eb ? yb[u] : yb[8 + u], 1);
                        const float oa = eb ? ya[8 + u] : ya[u], ob = eb ? yb[8 + u] : yb[u];
                        const int m = 16 * cq + 8 * eb + u;
                        const float2 y0 = eb ? make_float2(pa, oa) : make_float2(oa, pa);
                        const float2 y1 = tc_cmul(eb ? make_float2(pb, ob) : make_float2(ob, pb), ck);
                        const float2 f = tw[k1 * kTcTwPitch + m];
                        const float2 u0 = tc_cmul(make_float2(y0.x + y1.x, y0.y + y1.y), f);
                        const float2 u1 = tc_cmul(tc_cmul(make_float2(y0.x - y1.x, y0.y - y1.y), wtab[m]), f);
                        w0[u] = pack_h2(u0.x, u0.y);
                        w1[u] = pack_h2(u1.x, u1.y);
                    }
                    // own row l gets branch e = eb, row l ^ 1 the other; K chunks (m / 4) 4 cq + 2 eb, +1
                    const unsigned c0 = (unsigned)(4 * cq + 2 * eb) * kTcChunkPitch;
                    const uint32_t *own = eb ? w1 : w0, *oth = eb ? w0 : w1;
                    unsigned char *ro = dat + (unsigned)l * 16u, *rx = dat + (unsigned)(l ^ 1) * 16u;
                    *reinterpret_cast<uint4 *>(ro + c0) = make_uint4(own[0], own[1], own[2], own[3]);
                    *reinterpret_cast<uint4 *>(ro + c0 + kTcChunkPitch) = make_uint4(own[4], own[5], own[6], own[7]);
                    *reinterpret_cast<uint4 *>(rx + c0) = make_uint4(oth[0], oth[1], oth[2], oth[3]);
                    *reinterpret_cast<uint4 *>(rx + c0 + kTcChunkPitch) = make_uint4(oth[4], oth[5], oth[6], oth[7]);
                } else if (s == 2) {
                    // spectral product with the mirror lane l ^ 17 at column 63 - q; operand = conj X
                    float za[16], zb[16];
                    tmem_ld16x2(tl + 16 * cq, tl + 112 - 16 * cq, za, zb);  // q = 8 cq + i; q = 56 - 8 cq + i
                    float pa[16], pb[16];
#pragma unroll
                    for (int i = 0; i < 16; ++i) {
                        pa[i] = __shfl_xor_sync(0xffffffffu, za[i], 17);
                        pb[i] = __shfl_xor_sync(0xffffffffu, zb[i], 17);
                    }
                    uint32_t wa[8], wb[8];
#pragma unroll
                    for (int i = 0; i < 8; ++i) {
                        // own q = 8 cq + i pairs with the partner's q = 56 - 8 cq + 7 - i, and vice versa;
                        // P = Zk + conj Zm, Q = Zk - conj Zm, conj X = conj(-i P Q) = (Im PQ, Re PQ)
                        {
                            const float zx = za[2 * i], zy = za[2 * i + 1];
                            const float mx = pb[2 * (7 - i)], my = pb[2 * (7 - i) + 1];
                            const float px = zx + mx, py = zy - my, qx = zx - mx, qy = zy + my;
                            wa[i] = pack_h2(fmaf(px, qy, py * qx), fmaf(px, qx, -py * qy));
                        }
                        {
                            const float zx = zb[2 * i], zy = zb[2 * i + 1];
                            const float mx = pa[2 * (7 - i)], my = pa[2 * (7 - i) + 1];
                            const float px = zx + mx, py = zy - my, qx = zx - mx, qy = zy + my;
                            wb[i] = pack_h2(fmaf(px, qy, py * qx), fmaf(px, qx, -py * qy));
                        }
                    }
                    // K chunk = q / 4
                    unsigned char *row = dat + (unsigned)l * 16u;
                    *reinterpret_cast<uint4 *>(row + (unsigned)(2 * cq) * kTcChunkPitch) = make_uint4(wa[0], wa[1], wa[2], wa[3]);
                    *reinterpret_cast<uint4 *>(row + (unsigned)(2 * cq + 1) * kTcChunkPitch) = make_uint4(wa[4], wa[5], wa[6], wa[7]);
                    *reinterpret_cast<uint4 *>(row + (unsigned)(14 - 2 * cq) * kTcChunkPitch) = make_uint4(wb[0], wb[1], wb[2], wb[3]);
                    *reinterpret_cast<uint4 *>(row + (unsigned)(15 - 2 * cq) * kTcChunkPitch) = make_uint4(wb[4], wb[5], wb[6], wb[7]);
                } else if (s == 3) {
                    // inverse radix-2 step and conj(T1).  Lane l holds conj(Uhat_e), e = l & 1, at
                    // m in [16 cq, +16); thread l forms both outputs of its half of the m range:
                    // Y''[m] = conj(F0) S0, Y''[m + 64] = conj(F0) conj(c64) S1,
                    // S0,1 = Uhat_0[m] +- conj(w^m) Uhat_1[m]
                    float da[16], db[16];
                    tmem_ld16x2(tl + 32 * cq, tl + 32 * cq + 16, da, db);  // (m, re/im), m in [16 cq, +8) and [+8, +16)
                    const int kk = 2 * k1;  // K index of the real part; +1 imaginary
                    float yr0[8], yi0[8], yr1[8], yi1[8];
#pragma unroll
                    for (int u = 0; u < 8; ++u) {
                        // my m = 16 cq + 8 eb + u sits in da (eb = 0) or db (eb = 1); the partner's copy likewise
                        const float sr = eb ? da[2 * u] : db[2 * u], si = eb ? da[2 * u + 1] : db[2 * u + 1];
                        const float pr = __shfl_xor_sync(0xffffffffu, sr, 1);
                        const float pi = __shfl_xor_sync(0xffffffffu, si, 1);
                        const float orr = eb ? db[2 * u] : da[2 * u], oi = eb ? db[2 * u + 1] : da[2 * u + 1];
                        const int m = 16 * cq + 8 * eb + u;
                        const float2 own = make_float2(orr, -oi), par = make_float2(pr, -pi);
                        const float2 u0 = eb ? par : own;
                        const float2 a = tc_cmulc(eb ? own : par, wtab[m]);
                        const float2 f = tw[k1 * kTcTwPitch + m];
                        const float2 y0 = tc_cmulc(make_float2(u0.x + a.x, u0.y + a.y), f);
                        const float2 y1 = tc_cmulc(tc_cmulc(make_float2(u0.x - a.x, u0.y - a.y), ck), f);
                        yr0[u] = y0.x;
                        yi0[u] = y0.y;
                        yr1[u] = y1.x;
                        yi1[u] = y1.y;
                    }
#pragma unroll
                    for (int h = 0; h < 2; ++h) {
                        const int n2 = 64 * h + 16 * cq + 8 * eb;  // 8 consecutive n2: one 16-byte MN run
                        unsigned char *p = dat + (unsigned)(n2 / 8) * 128u;
                        const float *yr = h ? yr1 : yr0, *yi = h ? yi1 : yi0;
                        *reinterpret_cast<uint4 *>(p + (unsigned)(kk % 8) * 16u + (unsigned)(kk / 8) * 2048u) =
                            make_uint4(pack_h2(yr[0], yr[1]), pack_h2(yr[2], yr[3]), pack_h2(yr[4], yr[5]),
                                       pack_h2(yr[6], yr[7]));
                        *reinterpret_cast<uint4 *>(p + (unsigned)((kk + 1) % 8) * 16u + (unsigned)((kk + 1) / 8) * 2048u) =
                            make_uint4(pack_h2(yi[0], yi[1]), pack_h2(yi[2], yi[3]), pack_h2(yi[4], yi[5]),
                                       pack_h2(yi[6], yi[7]));
                    }
                } else if ((warp & 3) == 0) {
                    // outputs t = n2 + 128 n1 (n1 = lane) of channel c = 2q + x -> the CTA owning
                    // t (n1 / 8), slots n2 + 128 (n1 % 8): 32 consecutive slots per thread, 4 stores;
                    // t < 64 (n1 = 0, n2 < 64) carries the direct head instead
                    const int c = 2 * q + x, n1 = lane;
                    const bool live = scl[c] > 0.f && scl[8 + c] > 0.f;
                    const float fs = live ? kTcOutScale / (scl[c] * scl[8 + c]) : 0.f;
                    // (the TMEM loads are warp-collective: every lane runs them, only the stores are skipped)
                    const bool keep = !(n1 == 0 && cq < 2);
                    const uint32_t dst = tc_mapa(smem_u32(outs + c * kTcSpan + 32 * cq + 128 * (n1 % 8)), n1 / 8);
                    float oo[2][16];
                    tmem_ld16x2(tl + 32 * cq, tl + 32 * cq + 16, oo[0], oo[1]);
#pragma unroll
                    for (int hh = 0; hh < 2; ++hh) {
                        const float *o = oo[hh];
                        if (keep) {
                            uint4 w0, w1;
                            w0.x = pack_bf2(o[0] * fs, o[1] * fs);
                            w0.y = pack_bf2(o[2] * fs, o[3] * fs);
                            w0.z = pack_bf2(o[4] * fs, o[5] * fs);
                            w0.w = pack_bf2(o[6] * fs, o[7] * fs);
                            w1.x = pack_bf2(o[8] * fs, o[9] * fs);
                            w1.y = pack_bf2(o[10] * fs, o[11] * fs);
                            w1.z = pack_bf2(o[12] * fs, o[13] * fs);
                            w1.w = pack_bf2(o[14] * fs, o[15] * fs);
                            st_cluster_v4(dst + 32u * hh, w0);
                            st_cluster_v4(dst + 32u * hh + 16u, w1);
                        }
                    }
                }
                if (s < 4) issue(s + 1, x);
            }
        }
        ok = __syncthreads_and(ok);  // the last two waits had no issue() after them
        // the next group's partial norms, from its staged input (the head buffer is free now)
        have_norms = false;
        if (use_tma && in_flight && ok) {
            bool got = true;
            if (tid == 0) got = mbar_wait_bounded(bar + 2, in_phase);
            got = __syncthreads_and(got);
            if (got) {
                in_phase ^= 1u;
                in_flight = false;
                float nv[4][4], ng[4][4];
                read_staged(n2i, kl, hf, nv, ng);
                norms(nv, ng, head);
                have_norms = true;
            } else {
                ok = false;
            }
        }
        cluster.sync();  // #3: every output of this CTA's time steps has arrived; norms published
        // ---- store time steps [1024 q, 1024 q + 1024) of the 8 channels
#pragma unroll
        for (int h2 = 0; h2 < 2; ++h2) {
            const int sl = tid + 512 * h2, t = kTcSpan * q + sl;
            if (t < L) {
                uint16_t hv[8];
#pragma unroll
                for (int c = 0; c < 8; ++c) hv[c] = outs[c * kTcSpan + sl];
                const int to = (rev & 2) ? L - 1 - t : t;
                __nv_bfloat16 *p = r + base + (int64_t)to * D;
                if (vec) {
                    *reinterpret_cast<uint4 *>(p) =
                        make_uint4((uint32_t)hv[0] | ((uint32_t)hv[1] << 16), (uint32_t)hv[2] | ((uint32_t)hv[3] << 16),
                                   (uint32_t)hv[4] | ((uint32_t)hv[5] << 16), (uint32_t)hv[6] | ((uint32_t)hv[7] << 16));
                } else {
                    for (int c = 0; c < nch; ++c) p[c] = __ushort_as_bfloat16(hv[c]);
                }
            }
        }
    }
    if (!ok && tid == 0) {
        atomicOr(&g_cc_fault, kFaultTcWait);
        for (int x = 0; x < kTcRows; ++x)
            if ((pending >> x) & 1u) mbar_wait_bounded(bar + x, (phase >> x) & 1u);
        if (in_flight) mbar_wait_bounded(bar + 2, in_phase);
    }
    tc_fence_before_sync();
    cluster.sync();  // no peer reads or writes this CTA's shared memory any more
    if (warp == 0) {
        tc_fence_after_sync();
        tmem_dealloc(tmem, kTcTmemCols);
    }
}

}  // namespace ccv
