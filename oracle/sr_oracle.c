/*
 * sr_oracle.c -- plain, slow, fp64 CPU oracle for the chunk-streaming joint
 * video+audio self-attention step.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path may call, link or
 * load this file; only the test suite, the package smoke check and the CPU
 * baseline leg of the bench use it.  It shares no code, header or table with
 * the CUDA path.
 *
 * Every function is the plain definition written out: no tiling, no online
 * softmax, no fused or reordered arithmetic.  All arithmetic is IEEE double.
 *
 * Build: gcc -O2 -fopenmp -shared -fPIC sr_oracle.c -o libsr_oracle.so -lm
 */
#include <math.h>
#include <stddef.h>
#include <stdlib.h>
#ifdef _OPENMP
#include <omp.h>
#endif

/*
 * 3-D multimodal RoPE on (t, h, w).
 *
 * Source: "MiniMax-H3 deep dive" (fiv.co.kr), the H3-Omni-Transformer row of
 * the components table and the tensor-name paragraph: the single-stream DiT
 * applies 3D MM-RoPE to the shared attention.  The pages give no formula; the
 * reading used here: the head vector splits into contiguous sub-blocks
 * [t: d_t | h: d_h | w: d_w]; inside the sub-block of axis a (width d_a),
 * the interleaved pair (x[2j], x[2j+1]), j < d_a/2, turns by the angle
 *     phi = p_a * base^(-2j/d_a)
 * counter-clockwise:
 *     y[2j]   = x[2j] cos(phi) - x[2j+1] sin(phi)
 *     y[2j+1] = x[2j] sin(phi) + x[2j+1] cos(phi)
 *
 * x, y: [n][D] (row-major), pos: [n][3] = (t, h, w).  x and y must not alias.
 */
void sro_rope3d(const double *x, double *y, const double *pos, long n, int D,
                int d_t, int d_h, int d_w, double base)
{
    const int width[3] = {d_t, d_h, d_w};
    long i;
#pragma omp parallel for schedule(static)
    for (i = 0; i < n; ++i) {
        const double *xi = x + i * (long)D;
        double *yi = y + i * (long)D;
        int start = 0;
        for (int a = 0; a < 3; ++a) {
            const int da = width[a];
            for (int j = 0; j < da / 2; ++j) {
                const double theta = pow(base, -2.0 * (double)j / (double)da);
                const double phi = pos[i * 3 + a] * theta;
                const double c = cos(phi), s = sin(phi);
                const double x0 = xi[start + 2 * j], x1 = xi[start + 2 * j + 1];
                yi[start + 2 * j] = x0 * c - x1 * s;
                yi[start + 2 * j + 1] = x0 * s + x1 * c;
            }
            start += da;
        }
        (void)D;
    }
}

/*
 * QK normalisation: RMSNorm of every head vector before RoPE.
 *
 * Source: "MiniMax-H3 deep dive" (fiv.co.kr), tensor-name paragraph: the
 * attention carries norm_q / norm_k (QK normalisation) next to to_q / to_k.
 * Reading: per head vector of length D, with a learned gain g[D]:
 *     y[d] = x[d] / sqrt(mean_d(x[d]^2) + eps) * g[d]
 *
 * x, y: [n][D]; g: [D].
 */
void sro_rms_norm(const double *x, double *y, const double *g, long n, int D, double eps)
{
    long i;
#pragma omp parallel for schedule(static)
    for (i = 0; i < n; ++i) {
        const double *xi = x + i * (long)D;
        double *yi = y + i * (long)D;
        double ss = 0.0;
        for (int d = 0; d < D; ++d) ss += xi[d] * xi[d];
        const double inv = 1.0 / sqrt(ss / (double)D + eps);
        for (int d = 0; d < D; ++d) yi[d] = xi[d] * inv * g[d];
    }
}

/*
 * Spatial average pooling of one history tier.
 *
 * Source: "AlayaRenderer-Flash" (aitrends.kr), key contributions and
 * technical details: older history is kept at progressively lower
 * resolution.  Reading: per frame, the pooled cell (r, c) is the mean of the
 * source tokens in rows [r*ph, min((r+1)*ph, Gh)) x cols [c*pw, min((c+1)*pw,
 * Gw)) (ceil mode); the denominator counts valid members only.
 *
 * x: [F][Gh][Gw][C], y: [F][ceil(Gh/ph)][ceil(Gw/pw)][C].
 */
void sro_pool(const double *x, double *y, long F, int Gh, int Gw, int ph, int pw, long C)
{
    const int Rh = (Gh + ph - 1) / ph, Rw = (Gw + pw - 1) / pw;
    long f;
#pragma omp parallel for schedule(static)
    for (f = 0; f < F; ++f) {
        for (int r = 0; r < Rh; ++r) {
            for (int c = 0; c < Rw; ++c) {
                double *yc = y + ((f * Rh + r) * (long)Rw + c) * C;
                const int r0 = r * ph, r1 = (r + 1) * ph < Gh ? (r + 1) * ph : Gh;
                const int c0 = c * pw, c1 = (c + 1) * pw < Gw ? (c + 1) * pw : Gw;
                const double count = (double)((r1 - r0) * (c1 - c0));
                for (long e = 0; e < C; ++e) {
                    double sum = 0.0;
                    for (int rr = r0; rr < r1; ++rr)
                        for (int cc = c0; cc < c1; ++cc)
                            sum += x[((f * Gh + rr) * (long)Gw + cc) * C + e];
                    yc[e] = sum / count;
                }
            }
        }
    }
}

/*
 * Softmax attention of nq query rows over nk key/value rows (one head).
 *
 * Source: "StreamRender-H3" (molayo1419.me), streaming context section: the
 * window is attended bidirectionally and the moving part sees the whole
 * window; "AlayaRenderer-Flash" (aitrends.kr), methodology: past chunks enter
 * self-attention as clean tokens and the style-prompt KV is added to every
 * self-attention layer.  The caller passes only the valid keys of the
 * prompt, context and chunk segments; no mask remains here.
 *
 *   s_j = scale * (q . k_j),  m = max_j s_j,  w_j = exp(s_j - m)
 *   o   = sum_j w_j v_j / sum_j w_j,          lse = m + log(sum_j w_j)
 *
 * q: [nq][D], k, v: [nk][D], o: [nq][D], lse: [nq] (may be NULL).
 * rows: optional list of nq row indices into q (NULL = rows 0..nq-1); o and
 * lse are then indexed by position in that list.
 */
void sro_attention(const double *q, const double *k, const double *v, const long *rows,
                   long nq, long nk, int D, double scale, double *o, double *lse)
{
    long t;
#pragma omp parallel
    {
        double *s = (double *)malloc(sizeof(double) * (size_t)(nk > 0 ? nk : 1));
#pragma omp for schedule(dynamic, 4)
        for (t = 0; t < nq; ++t) {
            const long i = rows ? rows[t] : t;
            const double *qi = q + i * (long)D;
            double m = -INFINITY;
            for (long j = 0; j < nk; ++j) {
                const double *kj = k + j * (long)D;
                double dot = 0.0;
                for (int d = 0; d < D; ++d) dot += qi[d] * kj[d];
                s[j] = scale * dot;
                if (s[j] > m) m = s[j];
            }
            double denom = 0.0;
            double *ot = o + t * (long)D;
            for (int d = 0; d < D; ++d) ot[d] = 0.0;
            for (long j = 0; j < nk; ++j) {
                const double w = exp(s[j] - m);
                denom += w;
                const double *vj = v + j * (long)D;
                for (int d = 0; d < D; ++d) ot[d] += w * vj[d];
            }
            for (int d = 0; d < D; ++d) ot[d] /= denom;
            if (lse) lse[t] = m + log(denom);
        }
        free(s);
    }
}

/* Number of OpenMP threads the oracle runs with (reported by the bench). */
int sro_num_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

void sro_set_num_threads(int n)
{
#ifdef _OPENMP
    if (n > 0) omp_set_num_threads(n);
#else
    (void)n;
#endif
}
