// transpose.cuh -- [B, R, C] -> [B, C, R] layout change for the two-pass
// path of long rows.
//
// A row of the causal convolution is one channel d of a channel-last
// [B, L, D] tensor: its time steps are D elements apart, so a kernel that
// holds one row per cluster reads and writes one 2..4-byte piece of memory
// per time step.  With a caller workspace the long-row path instead
// transposes v and g to [B, D, L] (rows contiguous), runs the row kernel on
// contiguous rows and transposes r back; each transpose reads and writes
// whole 32 x 32 tiles, so both sides of it move full memory lines.
#pragma once

#include <stdint.h>

namespace ccv {

constexpr int kTrTile = 32;
constexpr int kTrThreads = 256;

// out[b][c][r] = in[b][r][c]; grid (ceil(C/32), ceil(R/32), B).  T is the
// element's storage type (uint16_t for bf16, uint32_t for fp32).
template <typename T>
__global__ void __launch_bounds__(kTrThreads) transpose_last2_kernel(const T *__restrict__ in, T *__restrict__ out,
                                                                     int R, int C) {
    __shared__ T tile[kTrTile][kTrTile + 1];
    const int64_t plane = (int64_t)R * C;
    const T *src = in + (int64_t)blockIdx.z * plane;
    T *dst = out + (int64_t)blockIdx.z * plane;
    const int r0 = blockIdx.y * kTrTile, c0 = blockIdx.x * kTrTile;
    const int tx = threadIdx.x % kTrTile, ty = threadIdx.x / kTrTile;
#pragma unroll
    for (int i = ty; i < kTrTile; i += kTrThreads / kTrTile) {
        const int r = r0 + i, c = c0 + tx;
        if (r < R && c < C) tile[i][tx] = src[(int64_t)r * C + c];
    }
    __syncthreads();
#pragma unroll
    for (int i = ty; i < kTrTile; i += kTrThreads / kTrTile) {
        const int c = c0 + i, r = r0 + tx;
        if (r < R && c < C) dst[(int64_t)c * R + r] = tile[tx][i];
    }
}

// Enqueue out = transpose of the last two dims of in ([B, R, C] -> [B, C, R]).
template <typename T>
static int transpose_last2(const T *in, T *out, int64_t B, int64_t R, int64_t C, cudaStream_t s) {
    const int64_t gx = (C + kTrTile - 1) / kTrTile, gy = (R + kTrTile - 1) / kTrTile;
    if (gx > INT32_MAX || gy > 65535 || B > 65535 || R > INT32_MAX || C > INT32_MAX) return 2;  // CC_ERR_UNSUPPORTED
    transpose_last2_kernel<T><<<dim3((unsigned)gx, (unsigned)gy, (unsigned)B), kTrThreads, 0, s>>>(in, out, (int)R,
                                                                                                   (int)C);
    return cudaGetLastError() == cudaSuccess ? 0 : 5;  // CC_OK / CC_ERR_CUDA
}

}  // namespace ccv
