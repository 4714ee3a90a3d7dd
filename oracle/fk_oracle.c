/*
 * fk_oracle.c -- plain, slow, obviously correct CPU oracle for one exact Lloyd
 * k-means iteration.  TEST INFRASTRUCTURE ONLY: the tests, the smoke check and
 * the benchmark's CPU-baseline leg use it to check and time the CUDA library;
 * nothing in the product path links it, and it shares no code with it.
 *
 * What it computes follows "Flash-KMeans: Fast and Memory-Efficient Exact
 * K-Means" (arXiv 2603.09229), abstract: the assignment stage gives each of N
 * points its nearest of K centroids, the centroid-update stage replaces every
 * centroid by the mean of the points assigned to it, and the method is exact,
 * i.e. it reaches exactly this textbook Lloyd result.  Where the pages are
 * silent the readings are: ties go to the lowest centroid index; a centroid
 * that receives no point keeps its previous value.
 *
 * All arithmetic is fp64, points and centroids are row-major (N x D, K x D).
 * The distance is the direct difference sum_j (x_j - c_j)^2, not the expanded
 * |x|^2 + |c|^2 - 2<x,c> form the GPU uses.  Sums run in index order.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

/* Threads an OpenMP region of this library uses (1 without OpenMP). */
int oracle_num_threads(void) {
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

/* Squared Euclidean distance, written out as the definition. */
static double sqdist(const double *x, const double *c, int D) {
    double s = 0.0;
    for (int j = 0; j < D; ++j) {
        double t = x[j] - c[j];
        s += t * t;
    }
    return s;
}

/*
 * Assignment stage: labels[i] = the first k (lowest index) reaching
 * min_k |x_i - c_k|^2; mindist[i] = that minimum; second[i] (nullable) = the
 * smallest distance over all other centroids (+inf when K == 1), which the
 * parity tests use to recognise near-ties.
 */
void oracle_assign(const double *X, int64_t N, int D, const double *C, int K,
                   int32_t *labels, double *mindist, double *second) {
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < N; ++i) {
        const double *x = X + (size_t)i * (size_t)D;
        double best = INFINITY, runner = INFINITY;
        int32_t arg = 0;
        for (int k = 0; k < K; ++k) {
            double d = sqdist(x, C + (size_t)k * (size_t)D, D);
            if (d < best) {
                runner = best;
                best = d;
                arg = k;
            } else if (d < runner) {
                runner = d;
            }
        }
        labels[i] = arg;
        if (mindist) mindist[i] = best;
        if (second) second[i] = runner;
    }
}

/*
 * The two nearest centroids (soft / multi-assignment of border points,
 * Flash-GMM abstract in the FlashDiffusion page's "similar papers" sidebar):
 * label1[i] = argmin_k |x_i - c_k|^2, label2[i] = argmin over k != label1[i],
 * each the first minimum in ascending k; d1, d2 the fp64 distances.
 * K == 1: label2 = -1, d2 = +inf.
 */
void oracle_top2(const double *X, int64_t N, int D, const double *C, int K, int32_t *label1, int32_t *label2,
                 double *d1, double *d2) {
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < N; ++i) {
        const double *x = X + (size_t)i * (size_t)D;
        double best = INFINITY, runner = INFINITY;
        int32_t a1 = 0, a2 = -1;
        for (int k = 0; k < K; ++k) {
            double d = sqdist(x, C + (size_t)k * (size_t)D, D);
            if (d < best) {
                runner = best;
                a2 = k == 0 ? -1 : a1;
                best = d;
                a1 = k;
            } else if (d < runner || a2 < 0) {
                runner = d;
                a2 = k;
            }
        }
        label1[i] = a1;
        label2[i] = a2;
        if (d1) d1[i] = best;
        if (d2) d2[i] = runner;
    }
}

/*
 * Centroid-update stage: counts[k] = #{i : labels[i] == k};
 * C_out[k] = (sum of those x_i) / counts[k], or C_prev[k] when counts[k] == 0.
 * Returns 0, or -1 if a label lies outside [0, K).
 */
int oracle_update(const double *X, const int32_t *labels, int64_t N, int D, int K,
                  const double *C_prev, double *C_out, int64_t *counts) {
    double *sums = (double *)calloc((size_t)K * (size_t)D, sizeof(double));
    if (!sums) return -2;
    for (int k = 0; k < K; ++k) counts[k] = 0;
    for (int64_t i = 0; i < N; ++i) {
        int32_t k = labels[i];
        if (k < 0 || k >= K) {
            free(sums);
            return -1;
        }
        counts[k] += 1;
        const double *x = X + (size_t)i * (size_t)D;
        double *s = sums + (size_t)k * (size_t)D;
        for (int j = 0; j < D; ++j) s[j] += x[j];
    }
    for (int k = 0; k < K; ++k) {
        double *out = C_out + (size_t)k * (size_t)D;
        if (counts[k] > 0) {
            const double *s = sums + (size_t)k * (size_t)D;
            for (int j = 0; j < D; ++j) out[j] = s[j] / (double)counts[k];
        } else {
            const double *prev = C_prev + (size_t)k * (size_t)D;
            for (int j = 0; j < D; ++j) out[j] = prev[j];
        }
    }
    free(sums);
    return 0;
}

/* Squared distance of each point to its given centroid:
 * out[i] = |x_i - c_{labels[i]}|^2, the same sum as oracle_assign forms. */
void oracle_label_dist(const double *X, const int32_t *labels, int64_t N, int D, const double *C,
                       double *out) {
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < N; ++i)
        out[i] = sqdist(X + (size_t)i * (size_t)D, C + (size_t)labels[i] * (size_t)D, D);
}

/*
 * Weighted Gauss sums ("Fast Gauss Sums via Flash Attention", abstract):
 * G[i] = sum_k w[k] exp(-beta |x_i - c_k|^2), w == NULL meaning every weight
 * is 1, with the direct-difference distance.  The terms of each sign are
 * summed as a log-sum-exp, P = sum over w > 0, Q = sum over w < 0 of
 * |w| exp(-beta d): logG[i] = ln P + ln(1 - Q / P) where P > Q (NaN
 * otherwise) and G[i] = P - Q.  Either output may be NULL.
 */
static void lse_add(double *m, double *s, double e) {
    if (e == -INFINITY) return;
    if (e > *m) {
        *s = *s * exp(*m - e) + 1.0;
        *m = e;
    } else {
        *s += exp(e - *m);
    }
}

void oracle_gauss_sum(const double *X, int64_t N, int D, const double *C, int K, const double *w, double beta,
                      double *G, double *logG) {
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < N; ++i) {
        const double *x = X + (size_t)i * (size_t)D;
        double mp = -INFINITY, sp = 0.0, mq = -INFINITY, sq = 0.0;
        for (int k = 0; k < K; ++k) {
            const double wk = w ? w[k] : 1.0;
            if (wk == 0.0) continue;
            const double e = log(fabs(wk)) - beta * sqdist(x, C + (size_t)k * (size_t)D, D);
            if (wk > 0.0) lse_add(&mp, &sp, e);
            else lse_add(&mq, &sq, e);
        }
        const double lp = mp + log(sp), lq = mq + log(sq); /* -inf for an empty part */
        if (G) G[i] = exp(lp) - exp(lq);
        if (logG) logG[i] = lp > lq ? lp + log1p(-exp(lq - lp)) : NAN;
    }
}

/*
 * k-means++ seeding (Arthur and Vassilvitskii) with reproducible draws:
 * centre 0 is point floor(u[0] N); centre t is drawn with probability
 * proportional to D2(x) = min over the chosen centres of |x - c|^2, through
 * integer weights q = floor(D2 2^s) (s the largest exponent with
 * N max D2 2^s < 2^61, fixed for the D2 after the first centre): r =
 * floor(u[t] T) (at most T - 1) for the total T, and the centre is the first
 * point whose running weight exceeds r; with T = 0, point floor(u[t] N).
 * Returns 0, or -2 when memory runs out.
 */
int oracle_kmeanspp(const double *X, int64_t N, int D, int K, const double *u, int32_t *centers) {
    double *d2 = (double *)malloc((size_t)N * sizeof(double));
    if (!d2) return -2;
    int64_t f = (int64_t)floor(u[0] * (double)N);
    centers[0] = (int32_t)(f < N ? f : N - 1);
    int L = 0;
    while (((int64_t)1 << L) < N) ++L;
    int s = 0;
    for (int t = 1; t < K; ++t) {
        const double *c = X + (size_t)centers[t - 1] * (size_t)D;
        for (int64_t i = 0; i < N; ++i) {
            const double d = sqdist(X + (size_t)i * (size_t)D, c, D);
            d2[i] = (t == 1 || d < d2[i]) ? d : d2[i];
        }
        if (t == 1) {
            double m = 0.0;
            for (int64_t i = 0; i < N; ++i) m = d2[i] > m ? d2[i] : m;
            int e = 0;
            if (m > 0.0) frexp(m, &e);
            s = m > 0.0 ? 61 - e - L : 0;
        }
        int64_t T = 0;
        for (int64_t i = 0; i < N; ++i) T += (int64_t)floor(ldexp(d2[i], s));
        if (T == 0) {
            int64_t k = (int64_t)floor(u[t] * (double)N);
            centers[t] = (int32_t)(k < N ? k : N - 1);
            continue;
        }
        int64_t r = (int64_t)floor(u[t] * (double)T);
        if (r >= T) r = T - 1;
        int64_t run = 0, i = 0;
        for (; i < N; ++i) {
            run += (int64_t)floor(ldexp(d2[i], s));
            if (run > r) break;
        }
        centers[t] = (int32_t)i;
    }
    free(d2);
    return 0;
}

/* Lloyd objective J = sum_i |x_i - c_{labels[i]}|^2. */
double oracle_objective(const double *X, const int32_t *labels, int64_t N, int D,
                        const double *C) {
    double J = 0.0;
    for (int64_t i = 0; i < N; ++i)
        J += sqdist(X + (size_t)i * (size_t)D, C + (size_t)labels[i] * (size_t)D, D);
    return J;
}
