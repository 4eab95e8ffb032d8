/*
 * A plain C99 consumer of the libmx C ABI (include/mx.h): no C++, no PyTorch.
 * The caller owns every buffer, so this program allocates them with the CUDA
 * runtime and hands plain device pointers to the library.
 *
 * It reads A [M x K] and B [N x K] as raw bf16 bit patterns (little-endian
 * uint16 files), quantizes both to `fmt` with mx_quantize, multiplies them with
 * mx_gemm (C = A_dq * B_dq^T, bf16 [M x N]), checks the device error word, and
 * writes A's codes, A's scales, A's global scale (NVFP4) and C to
 * <prefix>.codes / .scales / .gscale / .c for the test that compares them with
 * the oracle.
 *
 * usage: mx_c_consumer fmt M N K a.bin b.bin out_prefix
 * exit status: 0 on success, 1 on bad arguments or I/O, 2 on a CUDA error,
 * 3 on a library error (its status string is printed).
 */
#include <stdint.h>
#include <stdio.h>
#include <stdlib.h>
#include <string.h>

#include <cuda_runtime_api.h>

#include "mx.h"

static int read_file(const char *path, void *buf, size_t bytes) {
    FILE *f = fopen(path, "rb");
    if (!f) return 0;
    const size_t n = fread(buf, 1, bytes, f);
    fclose(f);
    return n == bytes;
}

static int write_file(const char *prefix, const char *suffix, const void *buf, size_t bytes) {
    char path[4096];
    snprintf(path, sizeof path, "%s%s", prefix, suffix);
    FILE *f = fopen(path, "wb");
    if (!f) return 0;
    const size_t n = fwrite(buf, 1, bytes, f);
    fclose(f);
    return n == bytes;
}

#define CUDA_OK(call)                                                                 \
    do {                                                                              \
        cudaError_t e_ = (call);                                                      \
        if (e_ != cudaSuccess) {                                                      \
            fprintf(stderr, "%s: %s\n", #call, cudaGetErrorString(e_));               \
            return 2;                                                                 \
        }                                                                             \
    } while (0)

#define MX_OK_OR_FAIL(call)                                                           \
    do {                                                                              \
        mx_status s_ = (call);                                                        \
        if (s_ != MX_OK) {                                                            \
            fprintf(stderr, "%s: %s\n", #call, mx_status_string(s_));                 \
            return 3;                                                                 \
        }                                                                             \
    } while (0)

/* Device buffers of one quantized matrix, described by an mx_tensor. */
static int alloc_tensor(mx_tensor *t, int fmt, int64_t rows, int64_t cols) {
    memset(t, 0, sizeof *t);
    t->fmt = fmt;
    t->rows = rows;
    t->cols = cols;
    if (cudaMalloc(&t->codes, mx_codes_bytes(fmt, rows, cols)) != cudaSuccess) return 0;
    if (cudaMalloc((void **)&t->scales, mx_scales_bytes(fmt, rows, cols)) != cudaSuccess) return 0;
    if (fmt == MX_NVFP4 && cudaMalloc((void **)&t->gscale, sizeof(float)) != cudaSuccess) return 0;
    return 1;
}

int main(int argc, char **argv) {
    if (argc != 8) {
        fprintf(stderr, "usage: %s fmt M N K a.bin b.bin out_prefix\n", argv[0]);
        return 1;
    }
    const int fmt = atoi(argv[1]);
    const int64_t M = atoll(argv[2]), N = atoll(argv[3]), K = atoll(argv[4]);
    const size_t a_bytes = (size_t)(M * K) * 2, b_bytes = (size_t)(N * K) * 2, c_bytes = (size_t)(M * N) * 2;
    uint16_t *a_host = (uint16_t *)malloc(a_bytes), *b_host = (uint16_t *)malloc(b_bytes);
    if (!a_host || !b_host || !read_file(argv[5], a_host, a_bytes) || !read_file(argv[6], b_host, b_bytes)) {
        fprintf(stderr, "cannot read the inputs\n");
        return 1;
    }

    void *a_dev = NULL, *b_dev = NULL, *c_dev = NULL;
    CUDA_OK(cudaMalloc(&a_dev, a_bytes));
    CUDA_OK(cudaMalloc(&b_dev, b_bytes));
    CUDA_OK(cudaMalloc(&c_dev, c_bytes));
    CUDA_OK(cudaMemcpy(a_dev, a_host, a_bytes, cudaMemcpyHostToDevice));
    CUDA_OK(cudaMemcpy(b_dev, b_host, b_bytes, cudaMemcpyHostToDevice));
    mx_tensor qa, qb;
    if (!alloc_tensor(&qa, fmt, M, K) || !alloc_tensor(&qb, fmt, N, K)) {
        fprintf(stderr, "cudaMalloc of the quantized operands failed\n");
        return 2;
    }

    /* NULL stream: the legacy default stream; NULL gscale_in: NVFP4 computes g */
    MX_OK_OR_FAIL(mx_quantize(fmt, a_dev, M, K, K, &qa, NULL, NULL));
    MX_OK_OR_FAIL(mx_quantize(fmt, b_dev, N, K, K, &qb, NULL, NULL));
    MX_OK_OR_FAIL(mx_gemm(&qa, &qb, c_dev, N, NULL));
    uint32_t info[4];
    MX_OK_OR_FAIL(mx_check_device_error(NULL, info));
    CUDA_OK(cudaDeviceSynchronize());

    const size_t codes_bytes = mx_codes_bytes(fmt, M, K), scales_bytes = mx_scales_bytes(fmt, M, K);
    uint8_t *codes = (uint8_t *)malloc(codes_bytes), *scales = (uint8_t *)malloc(scales_bytes);
    uint16_t *c_host = (uint16_t *)malloc(c_bytes);
    float g = 1.0f;
    if (!codes || !scales || !c_host) return 1;
    CUDA_OK(cudaMemcpy(codes, qa.codes, codes_bytes, cudaMemcpyDeviceToHost));
    CUDA_OK(cudaMemcpy(scales, qa.scales, scales_bytes, cudaMemcpyDeviceToHost));
    if (fmt == MX_NVFP4) CUDA_OK(cudaMemcpy(&g, qa.gscale, sizeof g, cudaMemcpyDeviceToHost));
    CUDA_OK(cudaMemcpy(c_host, c_dev, c_bytes, cudaMemcpyDeviceToHost));
    if (!write_file(argv[7], ".codes", codes, codes_bytes) || !write_file(argv[7], ".scales", scales, scales_bytes) ||
        !write_file(argv[7], ".gscale", &g, sizeof g) || !write_file(argv[7], ".c", c_host, c_bytes)) {
        fprintf(stderr, "cannot write the outputs\n");
        return 1;
    }

    cudaFree(a_dev);
    cudaFree(b_dev);
    cudaFree(c_dev);
    cudaFree(qa.codes);
    cudaFree(qa.scales);
    cudaFree(qb.codes);
    cudaFree(qb.scales);
    if (fmt == MX_NVFP4) {
        cudaFree(qa.gscale);
        cudaFree(qb.gscale);
    }
    free(a_host);
    free(b_host);
    free(codes);
    free(scales);
    free(c_host);
    printf("ok fmt=%d M=%lld N=%lld K=%lld mx_version=%d\n", fmt, (long long)M, (long long)N, (long long)K,
           mx_version());
    return 0;
}
