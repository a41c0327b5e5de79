// probe.cu -- micro-kernels that measure the per-SM rates the kernels of this
// library are bound by: FP32 FMA (scalar and packed f32x2), 32-bit integer
// multiply-add (low and high half), shared-memory reads and distributed
// shared-memory stores across an 8-CTA cluster.  Built as its own library
// (libccprobe.so); the benchmark's probe mode times each kernel with CUDA
// events and divides by the SM clock sampled meanwhile.
//
// Every kernel runs a fixed number of iterations of independent dependency
// chains (enough per thread to cover the pipeline latency) and writes one
// value per thread, so no work can be removed; memory probes stay inside
// their own shared-memory buffers.
#include <cooperative_groups.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace cg = cooperative_groups;

namespace {

constexpr int kChains = 8;

__global__ void probe_ffma(float *out, int iters) {
    float a[kChains];
#pragma unroll
    for (int i = 0; i < kChains; ++i) a[i] = threadIdx.x * 1e-3f + i;
    const float m = 0.999f, c = 1e-3f;
    for (int it = 0; it < iters; ++it) {
#pragma unroll
        for (int i = 0; i < kChains; ++i) a[i] = fmaf(a[i], m, c);
    }
    float s = 0.f;
#pragma unroll
    for (int i = 0; i < kChains; ++i) s += a[i];
    out[blockIdx.x * blockDim.x + threadIdx.x] = s;
}

__global__ void probe_ffma2(float *out, int iters) {
    float2 a[kChains / 2];
#pragma unroll
    for (int i = 0; i < kChains / 2; ++i) a[i] = make_float2(threadIdx.x * 1e-3f + 2 * i, threadIdx.x * 1e-3f + 2 * i + 1);
    const float2 m = make_float2(0.999f, 0.999f), c = make_float2(1e-3f, 1e-3f);
    for (int it = 0; it < iters; ++it) {
#pragma unroll
        for (int i = 0; i < kChains / 2; ++i) a[i] = __ffma2_rn(a[i], m, c);
    }
    float s = 0.f;
#pragma unroll
    for (int i = 0; i < kChains / 2; ++i) s += a[i].x + a[i].y;
    out[blockIdx.x * blockDim.x + threadIdx.x] = s;
}

__global__ void probe_imad(float *out, int iters, unsigned seed) {
    unsigned a[kChains];
#pragma unroll
    for (int i = 0; i < kChains; ++i) a[i] = threadIdx.x + i * seed;
    const unsigned m = seed | 1u, c = seed >> 3;
    for (int it = 0; it < iters; ++it) {
#pragma unroll
        for (int i = 0; i < kChains; ++i) a[i] = a[i] * m + c;
    }
    unsigned s = 0;
#pragma unroll
    for (int i = 0; i < kChains; ++i) s ^= a[i];
    out[blockIdx.x * blockDim.x + threadIdx.x] = (float)s;
}

__global__ void probe_mulhi(float *out, int iters, unsigned seed) {
    unsigned a[kChains];
#pragma unroll
    for (int i = 0; i < kChains; ++i) a[i] = threadIdx.x + i * seed + 12345u;
    const unsigned m = seed | 0x80000001u;
    for (int it = 0; it < iters; ++it) {
#pragma unroll
        for (int i = 0; i < kChains; ++i) a[i] = __umulhi(a[i], m) + a[i];
    }
    unsigned s = 0;
#pragma unroll
    for (int i = 0; i < kChains; ++i) s ^= a[i];
    out[blockIdx.x * blockDim.x + threadIdx.x] = (float)s;
}

// 16-byte reads, each warp over 512 consecutive bytes (conflict-free), from a
// 32 KiB buffer per CTA.
constexpr int kSmemWords = 8192;  // 32 KiB of uint32
__global__ void probe_smem(float *out, int iters) {
    __shared__ uint4 buf[kSmemWords / 4];
    for (int i = threadIdx.x; i < kSmemWords / 4; i += blockDim.x) buf[i] = make_uint4(i, i + 1, i + 2, i + 3);
    __syncthreads();
    uint32_t x = 0;
    const int n = kSmemWords / 4;
    int p = threadIdx.x;
    for (int it = 0; it < iters; ++it) {
#pragma unroll
        for (int k = 0; k < 8; ++k) {
            const uint4 v = buf[(p + k * 32) & (n - 1)];
            x ^= v.x ^ v.y ^ v.z ^ v.w;
        }
        p += 256;
    }
    out[blockIdx.x * blockDim.x + threadIdx.x] = (float)x;
}

// All-to-all within an 8-CTA cluster: every CTA writes its 16 KiB slice of
// each CTA's 128 KiB buffer (8-byte stores, destinations visited in an
// order staggered by rank), then the cluster synchronises.
constexpr int kDsmCluster = 8, kDsmWords = 16384;  // float2 words per CTA
__global__ void __cluster_dims__(kDsmCluster, 1, 1) __launch_bounds__(512, 1) probe_dsmem(float *out, int iters) {
    extern __shared__ float2 xs[];
    const int tid = threadIdx.x;
    const int rank = (int)cg::this_cluster().block_rank();
    for (int i = tid; i < kDsmWords; i += blockDim.x) xs[i] = make_float2(i, rank);
    cg::this_cluster().sync();
    const uint32_t base = (uint32_t)__cvta_generic_to_shared(xs);
    constexpr int slice = kDsmWords / kDsmCluster;
    for (int it = 0; it < iters; ++it) {
        for (int j = 0; j < kDsmCluster; ++j) {
            const int d = (rank + j) & (kDsmCluster - 1);
            uint32_t rb;
            asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(rb) : "r"(base), "r"(d));
            rb += 8u * (uint32_t)(rank * slice);
            for (int i = tid; i < slice; i += blockDim.x)
                asm volatile("st.shared::cluster.v2.f32 [%0], {%1, %2};" ::"r"(rb + 8u * (uint32_t)i), "f"((float)i),
                             "f"((float)it)
                             : "memory");
        }
        cg::this_cluster().sync();
    }
    out[blockIdx.x * blockDim.x + tid] = xs[tid].x;
}

}  // namespace

extern "C" {

// Probe kinds: 0 FFMA, 1 FFMA2 (packed f32x2), 2 IMAD, 3 IMAD.HI (mul.hi.u32
// + add), 4 shared-memory reads, 5 distributed shared-memory stores (8-CTA
// clusters).  Runs the kernel once to warm up, then once timed; *ms is the
// timed launch's duration and *units the work it did: lane operations
// (0..3) or bytes (4, 5).  Returns 0, or a cudaError_t value.
__attribute__((visibility("default"))) int ccp_run(int kind, int blocks, int threads, int iters, float *ms,
                                                   double *units) {
    if (kind < 0 || kind > 5 || blocks < 1 || threads < 32 || threads > 1024 || iters < 1) return (int)cudaErrorInvalidValue;
    if (kind == 5) {
        blocks = (blocks / kDsmCluster) * kDsmCluster;
        threads = 512;
        if (blocks < kDsmCluster) return (int)cudaErrorInvalidValue;
    }
    float *out = nullptr;
    cudaError_t e = cudaMalloc(&out, (size_t)blocks * threads * sizeof(float));
    if (e != cudaSuccess) return (int)e;
    if (kind == 5) {
        e = cudaFuncSetAttribute(probe_dsmem, cudaFuncAttributeMaxDynamicSharedMemorySize, kDsmWords * 8);
        if (e != cudaSuccess) {
            cudaFree(out);
            return (int)e;
        }
    }
    auto launch = [&](int n) {
        switch (kind) {
            case 0: probe_ffma<<<blocks, threads>>>(out, n); break;
            case 1: probe_ffma2<<<blocks, threads>>>(out, n); break;
            case 2: probe_imad<<<blocks, threads>>>(out, n, 0x9E3779B9u); break;
            case 3: probe_mulhi<<<blocks, threads>>>(out, n, 0x9E3779B9u); break;
            case 4: probe_smem<<<blocks, threads>>>(out, n); break;
            default: probe_dsmem<<<blocks, 512, kDsmWords * 8>>>(out, n); break;
        }
    };
    launch(iters);
    cudaEvent_t e0, e1;
    cudaEventCreate(&e0);
    cudaEventCreate(&e1);
    cudaEventRecord(e0);
    launch(iters);
    cudaEventRecord(e1);
    e = cudaEventSynchronize(e1);
    if (e == cudaSuccess) e = cudaGetLastError();
    cudaEventElapsedTime(ms, e0, e1);
    cudaEventDestroy(e0);
    cudaEventDestroy(e1);
    cudaFree(out);
    const double thr = (double)blocks * threads * iters;
    switch (kind) {
        case 0: case 2: case 3: *units = thr * kChains; break;
        case 1: *units = thr * kChains; break;  // kChains / 2 packed chains of two lanes
        case 4: *units = thr * 8 * 16; break;
        default: *units = (double)blocks * kDsmWords * 8 * iters; break;
    }
    return (int)e;
}

}  // extern "C"
