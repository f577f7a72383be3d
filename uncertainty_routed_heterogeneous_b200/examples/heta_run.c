/* heta_run.c -- one step of the routed-attention path driven from plain C
 * through the library's C ABI alone (include/heta.h, libheta.so).  The CUDA
 * runtime is used only to allocate device memory, copy and create a stream;
 * every step of the path is a heta_* call.
 *
 * "Where Compute Matters: Heterogeneous Attention for Efficient Video
 * Diffusion": the previous step's uncertainty u routes the ceil(rho*N) most
 * uncertain tokens of each sample to dense attention (Eq. (11)-(12)), the
 * rest to windowed local attention (Eq. (2), (3), (13)), and the head
 * u = softplus(X.w) (Eq. (7)) gives the next step's u.
 *
 *   heta_run DIR
 *
 * Inputs (little-endian raw arrays):
 *   DIR/meta.txt   "B H d Tg Hg Wg wt wh ww C rho"
 *   DIR/q.bin, k.bin, v.bin   [B,H,N,d] bf16 bit patterns (uint16)
 *   DIR/u.bin      [B,N] float32, the previous step's uncertainty
 *   DIR/x.bin      [B,N,C] bf16 bit patterns, the head's input
 *   DIR/w.bin      [C] float32, the head's weights (bias 0)
 * Outputs:
 *   DIR/dense.bin  [B,k] int32     DIR/local.bin  [B,N-k] int32
 *   DIR/out.bin    [B,H,N,d] bf16  DIR/u_next.bin [B,N] float32
 *
 * Exit status: 0 done; 1 usage, file or allocation error; 2 a heta_* call
 * returned an error or the device reported one through status_dev.
 */
#include <math.h>
#include <stdint.h>
#include <stdio.h>
#include <stdlib.h>
#include <string.h>

#include <cuda_runtime_api.h>

#include "heta.h"

static void *read_file(const char *dir, const char *name, size_t bytes)
{
    char path[4096];
    snprintf(path, sizeof path, "%s/%s", dir, name);
    FILE *f = fopen(path, "rb");
    if (!f) {
        fprintf(stderr, "heta_run: cannot open %s\n", path);
        return NULL;
    }
    void *p = malloc(bytes ? bytes : 1);
    const size_t got = p ? fread(p, 1, bytes, f) : 0;
    fclose(f);
    if (!p || got != bytes) {
        fprintf(stderr, "heta_run: %s holds fewer than %zu bytes\n", path, bytes);
        free(p);
        return NULL;
    }
    return p;
}

static int write_file(const char *dir, const char *name, const void *p, size_t bytes)
{
    char path[4096];
    snprintf(path, sizeof path, "%s/%s", dir, name);
    FILE *f = fopen(path, "wb");
    if (!f || fwrite(p, 1, bytes, f) != bytes) {
        fprintf(stderr, "heta_run: cannot write %s\n", path);
        if (f) fclose(f);
        return 1;
    }
    return fclose(f) != 0;
}

/* device copy of a host array (NULL on failure) */
static void *to_device(const void *host, size_t bytes)
{
    void *d = NULL;
    if (cudaMalloc(&d, bytes ? bytes : 256) != cudaSuccess) return NULL;
    if (bytes && cudaMemcpy(d, host, bytes, cudaMemcpyHostToDevice) != cudaSuccess) {
        cudaFree(d);
        return NULL;
    }
    return d;
}

#define CHECK_HETA(call)                                                              \
    do {                                                                              \
        const heta_status st_ = (call);                                               \
        if (st_ != HETA_OK) {                                                         \
            fprintf(stderr, "heta_run: %s: %s\n", #call, heta_status_string(st_));    \
            rc = 2;                                                                   \
            goto done;                                                                \
        }                                                                             \
    } while (0)

int main(int argc, char **argv)
{
    if (argc != 2) {
        fprintf(stderr, "usage: heta_run DIR   (see the header of heta_run.c)\n");
        return 1;
    }
    const char *dir = argv[1];
    int B, H, d, Tg, Hg, Wg, wt, wh, ww, C;
    double rho;
    {
        char path[4096];
        snprintf(path, sizeof path, "%s/meta.txt", dir);
        FILE *f = fopen(path, "r");
        const int n = f ? fscanf(f, "%d %d %d %d %d %d %d %d %d %d %lf", &B, &H, &d, &Tg, &Hg,
                                 &Wg, &wt, &wh, &ww, &C, &rho)
                        : 0;
        if (f) fclose(f);
        if (n != 11 || B < 1 || H < 1 || d < 1 || Tg < 1 || Hg < 1 || Wg < 1 || C < 1) {
            fprintf(stderr, "heta_run: %s must hold B H d Tg Hg Wg wt wh ww C rho\n", path);
            return 1;
        }
    }
    if ((int64_t)Tg * Hg * Wg > INT32_MAX) {
        fprintf(stderr, "heta_run: the grid holds more than 2^31 - 1 tokens\n");
        return 1;
    }
    const int N = Tg * Hg * Wg;
    const size_t qkv_bytes = (size_t)B * H * N * d * 2;
    const size_t u_bytes = (size_t)B * N * 4;
    const size_t x_bytes = (size_t)B * N * C * 2;

    int rc = 1, k = 0;
    size_t dense_bytes = 0, local_bytes = 0, ws_bytes = 0;
    void *hq = NULL, *hk = NULL, *hv = NULL, *hu = NULL, *hx = NULL, *hw = NULL;
    void *dq = NULL, *dk = NULL, *dv = NULL, *du = NULL, *dx = NULL, *dw = NULL;
    void *ddense = NULL, *dlocal = NULL, *dout = NULL, *dunext = NULL, *dws = NULL;
    int32_t *dstatus = NULL;
    void *hdense = NULL, *hlocal = NULL, *hout = NULL, *hunext = NULL;
    cudaStream_t stream = NULL;

    hq = read_file(dir, "q.bin", qkv_bytes);
    hk = read_file(dir, "k.bin", qkv_bytes);
    hv = read_file(dir, "v.bin", qkv_bytes);
    hu = read_file(dir, "u.bin", u_bytes);
    hx = read_file(dir, "x.bin", x_bytes);
    hw = read_file(dir, "w.bin", (size_t)C * 4);
    if (!hq || !hk || !hv || !hu || !hx || !hw) goto done;

    CHECK_HETA(heta_dense_count(N, rho, &k));
    dense_bytes = (size_t)B * k * 4;
    local_bytes = (size_t)B * (N - k) * 4;
    CHECK_HETA(heta_attention_workspace_size(B, H, d, Tg, Hg, Wg, wt, wh, ww, k, &ws_bytes));

    dq = to_device(hq, qkv_bytes);
    dk = to_device(hk, qkv_bytes);
    dv = to_device(hv, qkv_bytes);
    du = to_device(hu, u_bytes);
    dx = to_device(hx, x_bytes);
    dw = to_device(hw, (size_t)C * 4);
    if (!dq || !dk || !dv || !du || !dx || !dw || cudaMalloc(&ddense, dense_bytes + 256) ||
        cudaMalloc(&dlocal, local_bytes + 256) || cudaMalloc(&dout, qkv_bytes) ||
        cudaMalloc(&dunext, u_bytes) || cudaMalloc(&dws, ws_bytes ? ws_bytes : 256) ||
        cudaMalloc((void **)&dstatus, sizeof(int32_t)) ||
        cudaMemset(dstatus, 0, sizeof(int32_t)) || cudaStreamCreate(&stream)) {
        fprintf(stderr, "heta_run: device allocation or copy failed\n");
        goto done;
    }

    /* the step: route by the previous u, attend, then the head for the next u */
    CHECK_HETA(heta_route((const float *)du, B, N, k, (int32_t *)ddense, (int32_t *)dlocal, NULL,
                          NULL, dstatus, stream));
    CHECK_HETA(heta_attention((const uint16_t *)dq, (const uint16_t *)dk, (const uint16_t *)dv, B,
                              H, d, Tg, Hg, Wg, wt, wh, ww, 1.0f / sqrtf((float)d),
                              (const int32_t *)ddense, k, (uint16_t *)dout, dws, ws_bytes, dstatus,
                              stream));
    CHECK_HETA(heta_uncertainty((const uint16_t *)dx, (const float *)dw, 0.0f, B, N, C,
                                (float *)dunext, dstatus, stream));
    if (cudaStreamSynchronize(stream) != cudaSuccess) {
        fprintf(stderr, "heta_run: the stream failed: %s\n",
                cudaGetErrorString(cudaGetLastError()));
        rc = 2;
        goto done;
    }
    {
        int32_t st = 0;
        if (cudaMemcpy(&st, dstatus, sizeof st, cudaMemcpyDeviceToHost) != cudaSuccess) goto done;
        if (st != HETA_OK) {
            fprintf(stderr, "heta_run: the device reported %s\n", heta_status_string(st));
            rc = 2;
            goto done;
        }
    }

    hdense = malloc(dense_bytes + 1);
    hlocal = malloc(local_bytes + 1);
    hout = malloc(qkv_bytes);
    hunext = malloc(u_bytes);
    if (!hdense || !hlocal || !hout || !hunext ||
        cudaMemcpy(hdense, ddense, dense_bytes, cudaMemcpyDeviceToHost) ||
        cudaMemcpy(hlocal, dlocal, local_bytes, cudaMemcpyDeviceToHost) ||
        cudaMemcpy(hout, dout, qkv_bytes, cudaMemcpyDeviceToHost) ||
        cudaMemcpy(hunext, dunext, u_bytes, cudaMemcpyDeviceToHost)) {
        fprintf(stderr, "heta_run: copying the results back failed\n");
        goto done;
    }
    rc = write_file(dir, "dense.bin", hdense, dense_bytes) |
         write_file(dir, "local.bin", hlocal, local_bytes) |
         write_file(dir, "out.bin", hout, qkv_bytes) |
         write_file(dir, "u_next.bin", hunext, u_bytes);
    if (rc == 0)
        printf("heta_run: B=%d H=%d N=%d d=%d k=%d: route, attention and head done\n", B, H, N, d,
               k);

done:
    if (stream) cudaStreamDestroy(stream);
    cudaFree(dq); cudaFree(dk); cudaFree(dv); cudaFree(du); cudaFree(dx); cudaFree(dw);
    cudaFree(ddense); cudaFree(dlocal); cudaFree(dout); cudaFree(dunext); cudaFree(dws);
    cudaFree(dstatus);
    free(hq); free(hk); free(hv); free(hu); free(hx); free(hw);
    free(hdense); free(hlocal); free(hout); free(hunext);
    return rc;
}
