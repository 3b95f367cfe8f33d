/* A plain C caller of the library's boundary: no Python, no PyTorch.
 *
 * It allocates the attention's buffers with the CUDA runtime, fills them
 * with seeded values, runs sr_chunk_attention_fwd through include/sr.h on
 * two ragged sessions of a two-segment window, and compares every output
 * row with the fp64 oracle's attention (oracle/sr_oracle.c, sro_attention)
 * over the same bf16 inputs: max-abs <= 2e-2 and mean-abs <= 2e-3 on o,
 * 1e-3 on lse.  Exit status: 0 pass, 1 mismatch, 2 library or CUDA error,
 * 77 no CUDA device. */
#include <math.h>
#include <stdint.h>
#include <stdio.h>
#include <stdlib.h>
#include <string.h>

#include <cuda_runtime.h>

#include "sr.h"

/* the oracle's plain attention (test infrastructure, linked by this test only) */
void sro_attention(const double *q, const double *k, const double *v, const long *rows, long nq, long nk, int D,
                   double scale, double *o, double *lse);

enum { B = 2, H = 2, D = 64, QCAP = 70, NSEG = 2 };
static const int32_t kCap[NSEG] = {128, 128};
static const int32_t kLen[B][NSEG] = {{100, 37}, {128, 1}};
static const int32_t kQLen[B] = {70, 33};

static uint64_t rng_state = 0x9E3779B97F4A7C15ull;
static double uniform(void) { /* xorshift64*, in [-1, 1) */
    rng_state ^= rng_state >> 12;
    rng_state ^= rng_state << 25;
    rng_state ^= rng_state >> 27;
    return (double)((rng_state * 0x2545F4914F6CDD1Dull) >> 11) / 4503599627370496.0 - 1.0;
}

/* bf16 bits of x, rounded to nearest even (finite inputs) */
static uint16_t to_bf16(float x) {
    uint32_t u;
    memcpy(&u, &x, 4);
    u += 0x7FFFu + ((u >> 16) & 1u);
    return (uint16_t)(u >> 16);
}
static double from_bf16(uint16_t h) {
    uint32_t u = (uint32_t)h << 16;
    float x;
    memcpy(&x, &u, 4);
    return (double)x;
}

#define CUDA_OK(call)                                                        \
    do {                                                                     \
        cudaError_t e_ = (call);                                             \
        if (e_ != cudaSuccess) {                                             \
            fprintf(stderr, "%s: %s\n", #call, cudaGetErrorString(e_));      \
            return 2;                                                        \
        }                                                                    \
    } while (0)

int main(void) {
    int n_dev = 0;
    if (cudaGetDeviceCount(&n_dev) != cudaSuccess || n_dev == 0) {
        printf("no CUDA device\n");
        return 77;
    }
    const long C = kCap[0] + kCap[1];
    const size_t nq = (size_t)B * H * QCAP * D, nkv = (size_t)B * H * C * D, no = (size_t)B * QCAP * H * D;
    uint16_t *hq = malloc(nq * 2), *hk = malloc(nkv * 2), *hv = malloc(nkv * 2), *ho = malloc(no * 2);
    float *hl = malloc((size_t)B * H * QCAP * 4);
    for (size_t i = 0; i < nq; ++i) hq[i] = to_bf16((float)uniform());
    for (size_t i = 0; i < nkv; ++i) hk[i] = to_bf16((float)(0.7 * uniform()));
    for (size_t i = 0; i < nkv; ++i) hv[i] = to_bf16((float)uniform());

    void *q, *k, *v, *o;
    float *lse;
    int32_t *kv_len, *q_len, *status;
    CUDA_OK(cudaMalloc(&q, nq * 2));
    CUDA_OK(cudaMalloc(&k, nkv * 2));
    CUDA_OK(cudaMalloc(&v, nkv * 2));
    CUDA_OK(cudaMalloc(&o, no * 2));
    CUDA_OK(cudaMalloc((void **)&lse, (size_t)B * H * QCAP * 4));
    CUDA_OK(cudaMalloc((void **)&kv_len, sizeof(kLen)));
    CUDA_OK(cudaMalloc((void **)&q_len, sizeof(kQLen)));
    CUDA_OK(cudaMalloc((void **)&status, 4));
    CUDA_OK(cudaMemcpy(q, hq, nq * 2, cudaMemcpyHostToDevice));
    CUDA_OK(cudaMemcpy(k, hk, nkv * 2, cudaMemcpyHostToDevice));
    CUDA_OK(cudaMemcpy(v, hv, nkv * 2, cudaMemcpyHostToDevice));
    CUDA_OK(cudaMemcpy(kv_len, kLen, sizeof(kLen), cudaMemcpyHostToDevice));
    CUDA_OK(cudaMemcpy(q_len, kQLen, sizeof(kQLen), cudaMemcpyHostToDevice));
    CUDA_OK(cudaMemset(o, 0, no * 2));
    CUDA_OK(cudaMemset(status, 0, 4));

    sr_kv_layout layout;
    memset(&layout, 0, sizeof(layout));
    layout.n_seg = NSEG;
    for (int s = 0; s < NSEG; ++s) layout.cap[s] = kCap[s];
    const double scale = 1.0 / sqrt((double)D);
    const size_t ws_bytes = sr_chunk_attention_workspace_bytes(B, H, D, QCAP);
    void *ws = NULL;
    if (ws_bytes) CUDA_OK(cudaMalloc(&ws, ws_bytes));
    int rc = sr_chunk_attention_fwd(q, k, v, o, lse, &layout, kv_len, q_len, B, H, D, QCAP, (float)scale, ws,
                                    ws_bytes, status, NULL);
    if (rc != SR_OK) {
        fprintf(stderr, "sr_chunk_attention_fwd: %d (%s)\n", rc, sr_get_last_error());
        return 2;
    }
    CUDA_OK(cudaDeviceSynchronize());
    int32_t st = -1;
    CUDA_OK(cudaMemcpy(&st, status, 4, cudaMemcpyDeviceToHost));
    if (st != 0) {
        fprintf(stderr, "status word %d\n", st);
        return 2;
    }
    CUDA_OK(cudaMemcpy(ho, o, no * 2, cudaMemcpyDeviceToHost));
    CUDA_OK(cudaMemcpy(hl, lse, (size_t)B * H * QCAP * 4, cudaMemcpyDeviceToHost));

    double max_err = 0.0, sum_err = 0.0, max_lse = 0.0;
    long n_err = 0;
    double *qq = malloc(sizeof(double) * QCAP * D), *kk = malloc(sizeof(double) * C * D),
           *vv = malloc(sizeof(double) * C * D), *ro = malloc(sizeof(double) * QCAP * D), *rl = malloc(sizeof(double) * QCAP);
    for (int b = 0; b < B; ++b)
        for (int h = 0; h < H; ++h) {
            const size_t qbase = (((size_t)b * H + h) * QCAP) * D, kbase = (((size_t)b * H + h) * C) * D;
            for (long i = 0; i < (long)QCAP * D; ++i) qq[i] = from_bf16(hq[qbase + i]);
            long nk = 0, off = 0;   /* the valid keys of every segment, in buffer order */
            for (int s = 0; s < NSEG; ++s) {
                for (int j = 0; j < kLen[b][s]; ++j, ++nk)
                    for (int d = 0; d < D; ++d) {
                        kk[nk * D + d] = from_bf16(hk[kbase + (size_t)(off + j) * D + d]);
                        vv[nk * D + d] = from_bf16(hv[kbase + (size_t)(off + j) * D + d]);
                    }
                off += kCap[s];
            }
            sro_attention(qq, kk, vv, NULL, kQLen[b], nk, D, scale, ro, rl);
            for (int i = 0; i < kQLen[b]; ++i) {
                for (int d = 0; d < D; ++d) {
                    const double got = from_bf16(ho[(((size_t)b * QCAP + i) * H + h) * D + d]);
                    const double err = fabs(got - ro[(long)i * D + d]);
                    max_err = err > max_err ? err : max_err;
                    sum_err += err;
                    ++n_err;
                }
                const double le = fabs((double)hl[((size_t)b * H + h) * QCAP + i] - rl[i]);
                max_lse = le > max_lse ? le : max_lse;
            }
        }
    const double mean_err = sum_err / (double)n_err;
    printf("C caller vs oracle: max-abs %.3e mean-abs %.3e lse %.3e\n", max_err, mean_err, max_lse);
    return (max_err <= 2e-2 && mean_err <= 2e-3 && max_lse <= 1e-3) ? 0 : 1;
}
