/* C program against the library's C ABI (include/causalconv.h), used by the
 * tests: it shows the header is plain C and the entry points are callable
 * without Python.
 *
 *   abi_check host            host-only queries, printed one per line
 *   abi_check run B L D out   a float32 convolution of seeded inputs on
 *                             device 0 (inputs x_i = sin(0.37 i + k)), writing
 *                             v, g and r as raw float32 to out.{v,g,r}
 */
#include <math.h>
#include <stdio.h>
#include <stdlib.h>
#include <string.h>

#include "causalconv.h"

#ifdef ABI_CHECK_CUDA
#include <cuda_runtime.h>
#endif

static int host_queries(void) {
    uint32_t p[6];
    int st = causal_ntt_params(16384, p);
    printf("ntt_params %d %u %u %u %u %u %u\n", st, p[0], p[1], p[2], p[3], p[4], p[5]);
    printf("max_len %lld %lld %lld\n", (long long)causal_conv_max_len(CC_DTYPE_F32),
           (long long)causal_conv_max_len(CC_DTYPE_BF16), (long long)causal_conv_max_len(CC_DTYPE_I32));
    printf("workspace %zu\n", causal_conv_workspace_bytes(CC_DTYPE_F32, 2, 1000, 8));
    printf("fast_workspace %zu %zu\n", causal_conv_fast_workspace_bytes(CC_DTYPE_F32, 1, 4096, 8),
           causal_conv_fast_workspace_bytes(CC_DTYPE_F32, 1, 4097, 8));
    printf("strerror %s\n", causal_conv_strerror(CC_ERR_ALIAS));
    printf("null_args %d\n", causal_fftconv_f32(NULL, NULL, NULL, 1, 1, 1, NULL, 0, NULL));
    return 0;
}

#ifdef ABI_CHECK_CUDA
static int write_file(const char *base, const char *ext, const float *x, size_t n) {
    char name[4096];
    snprintf(name, sizeof name, "%s.%s", base, ext);
    FILE *f = fopen(name, "wb");
    if (!f) return 1;
    const size_t w = fwrite(x, sizeof(float), n, f);
    fclose(f);
    return w == n ? 0 : 1;
}

static int run(long long B, long long L, long long D, const char *out) {
    const size_t n = (size_t)(B * L * D), bytes = n * sizeof(float);
    float *hv = (float *)malloc(bytes), *hg = (float *)malloc(bytes), *hr = (float *)malloc(bytes);
    if (!hv || !hg || !hr) return 2;
    for (size_t i = 0; i < n; ++i) {
        hv[i] = (float)sin(0.37 * (double)i);
        hg[i] = (float)sin(0.37 * (double)i + 1.0);
    }
    float *dv, *dg, *dr;
    if (cudaMalloc((void **)&dv, bytes) || cudaMalloc((void **)&dg, bytes) || cudaMalloc((void **)&dr, bytes)) return 3;
    cudaMemcpy(dv, hv, bytes, cudaMemcpyHostToDevice);
    cudaMemcpy(dg, hg, bytes, cudaMemcpyHostToDevice);
    const int st = causal_fftconv_f32(dv, dg, dr, B, L, D, NULL, 0, NULL);
    if (st != CC_OK) {
        fprintf(stderr, "causal_fftconv_f32: %s\n", causal_conv_strerror(st));
        return 4;
    }
    if (cudaMemcpy(hr, dr, bytes, cudaMemcpyDeviceToHost) != cudaSuccess) return 5;
    int rc = write_file(out, "v", hv, n) | write_file(out, "g", hg, n) | write_file(out, "r", hr, n);
    cudaFree(dv);
    cudaFree(dg);
    cudaFree(dr);
    free(hv);
    free(hg);
    free(hr);
    return rc ? 6 : 0;
}
#endif

int main(int argc, char **argv) {
    if (argc >= 2 && strcmp(argv[1], "host") == 0) return host_queries();
#ifdef ABI_CHECK_CUDA
    if (argc >= 6 && strcmp(argv[1], "run") == 0)
        return run(atoll(argv[2]), atoll(argv[3]), atoll(argv[4]), argv[5]);
#endif
    fprintf(stderr, "usage: abi_check host | run B L D out\n");
    return 1;
}
