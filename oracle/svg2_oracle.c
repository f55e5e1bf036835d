/*
 * Plain, slow CPU oracle for SVG2 semantic-aware permuted sparse attention (one DiT layer).
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path may link, load or call this file: it
 * exists so that the tests, the smoke check and the benchmark's CPU-baseline leg can compare
 * the CUDA path against an obviously correct restatement of the method.  It shares no code,
 * header, table or constant with the CUDA library.
 *
 * Source of the method: "Sparse VideoGen2: Accelerate Video Generation with Sparse Attention via
 * Semantic-Aware Permutation" (wiki summary page, sections Key claims and Method; paper sections
 * 4.1-4.3, Eq. 1-2 as cited there).  Every function below names the passage it restates.
 *
 * Arithmetic: inputs are float32 (bf16-exact for bf16 layers); every floating-point computation
 * is done in float64, with each sum taken sequentially in ascending index order and no fused
 * multiply-add (build with -ffp-contract=off).  Where the method makes an integer decision from
 * floating point (k-means++ sampling, top-p), the decision is defined in fixed-point integers so
 * that it is reproducible; those readings are documented with each function.
 *
 * Pins (tests/test_oracle.py): Lloyd vs scikit-learn's Lloyd and fixed-point properties;
 * k-means++ sampling frequencies vs D^2 / sum D^2 from scipy distances; weights vs scipy softmax;
 * top-p vs brute force over subsets; permutation vs numpy stable argsort; sparse attention vs
 * torch scaled_dot_product_attention (float64, CPU) with an equivalent token mask, and
 * top-p = 1 equal to dense attention after unpermutation.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define TWO32 4294967296.0

/* Squared Euclidean distance in float64: sum over i = 0..d-1 of (x_i - c_i)^2, sequential. */
static double sqdist_fd(const float *x, const double *c, int d) {
    double acc = 0.0;
    for (int i = 0; i < d; ++i) {
        double diff = (double)x[i] - c[i];
        double sq = diff * diff;
        acc = acc + sq;
    }
    return acc;
}

/* Fixed-point weight of a non-negative value relative to a positive scale: floor(v / s * 2^32). */
static uint64_t fixed_weight(double v, double s) {
    if (!(s > 0.0) || !(v > 0.0)) return 0;
    double r = v / s;
    return (uint64_t)floor(r * TWO32);
}

/*
 * k-means++ seeding (wiki summary, Method (1): "run k-means++ on the Q and K activations";
 * Key claims, section 4.3).  Seeds are data rows.  The first seed is row floor(u[0] * N).  Each
 * later seed s is drawn with probability proportional to D^2(t) = min over chosen seeds of
 * ||x_t - c||^2.  Reading (the pages give no sampling procedure): D^2 is turned into fixed-point
 * weights q_t = floor(D^2(t) / M0 * 2^32), M0 = max_t D^2(t) after the first seed (D^2 only
 * decreases afterwards), U = sum q_t, target = min(floor(u[s] * U), U - 1), and the seed is the
 * first t (ascending) whose inclusive prefix sum of q exceeds target.  If U == 0 (every row
 * coincides with a seed) the seed is row floor(u[s] * N).
 * u: k uniforms in [0,1).  Outputs: seeds[k] (row indices), C[k*d] (float64 copies of the rows).
 */
int svg2o_kmeanspp(const float *X, int64_t N, int d, int k, const double *u,
                   int64_t *seeds, double *C) {
    if (N < 1 || k < 1 || d < 1) return 1;
    double *D = (double *)malloc((size_t)N * sizeof(double));
    if (!D) return 2;
    int64_t s0 = (int64_t)floor(u[0] * (double)N);
    if (s0 >= N) s0 = N - 1;
    if (s0 < 0) s0 = 0;
    seeds[0] = s0;
    for (int i = 0; i < d; ++i) C[i] = (double)X[s0 * d + i];
#pragma omp parallel for schedule(static)
    for (int64_t t = 0; t < N; ++t) D[t] = sqdist_fd(X + t * d, C, d);
    double M0 = 0.0;
    for (int64_t t = 0; t < N; ++t)
        if (D[t] > M0) M0 = D[t];
    for (int s = 1; s < k; ++s) {
        uint64_t U = 0;
        for (int64_t t = 0; t < N; ++t) U += fixed_weight(D[t], M0);
        int64_t pick;
        if (U == 0) {
            pick = (int64_t)floor(u[s] * (double)N);
            if (pick >= N) pick = N - 1;
        } else {
            uint64_t target = (uint64_t)floor(u[s] * (double)U);
            if (target > U - 1) target = U - 1;
            uint64_t run = 0;
            pick = N - 1;
            for (int64_t t = 0; t < N; ++t) {
                run += fixed_weight(D[t], M0);
                if (run > target) { pick = t; break; }
            }
        }
        seeds[s] = pick;
        double *cs = C + (int64_t)s * d;
        for (int i = 0; i < d; ++i) cs[i] = (double)X[pick * d + i];
#pragma omp parallel for schedule(static)
        for (int64_t t = 0; t < N; ++t) {
            double nd = sqdist_fd(X + t * d, cs, d);
            if (nd < D[t]) D[t] = nd;
        }
    }
    free(D);
    return 0;
}

/*
 * Lloyd assignment step (wiki summary, Method (1); Key claims, section 4.1: k-means on Q and K
 * per head).  label_t = argmin_c ||x_t - c||^2 (squared Euclidean; ties to the lowest c).
 * Also returns the smallest and second-smallest distances (used to classify near-ties).
 */
void svg2o_assign(const float *X, int64_t N, int d, const double *C, int k,
                  int32_t *labels, double *dmin1, double *dmin2) {
#pragma omp parallel for schedule(static)
    for (int64_t t = 0; t < N; ++t) {
        double best = INFINITY, second = INFINITY;
        int lab = 0;
        for (int c = 0; c < k; ++c) {
            double dist = sqdist_fd(X + t * d, C + (int64_t)c * d, d);
            if (dist < best) {
                second = best;
                best = dist;
                lab = c;
            } else if (dist < second) {
                second = dist;
            }
        }
        labels[t] = lab;
        if (dmin1) dmin1[t] = best;
        if (dmin2) dmin2[t] = second;
    }
}

/*
 * Lloyd update step: c_j = (sum of x_t with label_t = j) / count_j, summed in float64 in ascending
 * t; an empty cluster keeps its previous centroid (reading: the pages are silent).
 */
void svg2o_update(const float *X, int64_t N, int d, const int32_t *labels, int k,
                  double *C, int32_t *counts) {
    for (int c = 0; c < k; ++c) counts[c] = 0;
    for (int64_t t = 0; t < N; ++t) counts[labels[t]] += 1;
    double *sums = (double *)calloc((size_t)k * d, sizeof(double));
    if (!sums) return;
#pragma omp parallel for schedule(static)
    for (int i = 0; i < d; ++i) {
        for (int64_t t = 0; t < N; ++t) {
            double *acc = sums + (int64_t)labels[t] * d + i;
            *acc = *acc + (double)X[t * d + i];
        }
    }
    for (int c = 0; c < k; ++c) {
        if (counts[c] == 0) continue;
        for (int i = 0; i < d; ++i)
            C[(int64_t)c * d + i] = sums[(int64_t)c * d + i] / (double)counts[c];
    }
    free(sums);
}

/*
 * `iters` Lloyd iterations (assign, then update) from the centroids in C.  Outputs the final
 * centroids, the labels of the last assignment (the ones that produced those centroids) and the
 * cluster sizes under those labels.
 */
void svg2o_lloyd(const float *X, int64_t N, int d, int k, int iters, double *C,
                 int32_t *labels, int32_t *counts) {
    for (int it = 0; it < iters; ++it) {
        svg2o_assign(X, N, d, C, k, labels, NULL, NULL);
        svg2o_update(X, N, d, labels, k, C, counts);
    }
}

/*
 * Centroid-based score estimation (wiki summary, Key claims section 4.2 Eq. 1; Method (3)):
 * l_ij = (sum_m cq_im * ck_jm) * scale approximates the pre-softmax score between Q-cluster i and
 * K-cluster j; weighting by cluster size gives w_ij = count_j * exp(l_ij - max_{j': count_j'>0}
 * l_ij'), and w_ij = 0 for empty K clusters.  Row-normalising w gives softmax(l + log count).
 * The weights are materialised as float32 (reading: the selection is defined on these values).
 */
void svg2o_select_weights(const float *cq, const float *ck, const int32_t *count_k,
                          int nQ, int nK, int d, double scale, float *w) {
#pragma omp parallel for schedule(static)
    for (int i = 0; i < nQ; ++i) {
        double *l = (double *)malloc((size_t)nK * sizeof(double));
        double mx = -INFINITY;
        for (int j = 0; j < nK; ++j) {
            double acc = 0.0;
            for (int m = 0; m < d; ++m) {
                double pr = (double)cq[(int64_t)i * d + m] * (double)ck[(int64_t)j * d + m];
                acc = acc + pr;
            }
            l[j] = acc * scale;
            if (count_k[j] > 0 && l[j] > mx) mx = l[j];
        }
        for (int j = 0; j < nK; ++j)
            w[(int64_t)i * nK + j] = count_k[j] > 0 ? (float)((double)count_k[j] * exp(l[j] - mx)) : 0.0f;
        free(l);
    }
}

typedef struct { uint64_t u; int j; } topp_item;

static int topp_cmp(const void *a, const void *b) {
    const topp_item *x = (const topp_item *)a, *y = (const topp_item *)b;
    if (x->u != y->u) return x->u > y->u ? -1 : 1;   /* larger weight first */
    return (x->j > y->j) - (x->j < y->j);            /* then lower index */
}

/*
 * Top-p budget selection (wiki summary, Key claims section 4.2 Eq. 2; Method (3)): per Q cluster,
 * sort the K clusters by weight descending and keep them until the accumulated weight reaches p of
 * the row total; the cluster that crosses the target is kept.  Reading, in fixed point so that it
 * is reproducible: u_j = floor(w_j / max_j w * 2^32) for non-empty j (0 otherwise), U = sum u_j,
 * T = ceil(p * U); order j by (u_j desc, j asc) and keep the shortest prefix with sum >= T.
 * p >= 1 keeps every non-empty cluster; a row whose maximum weight is not positive keeps every
 * non-empty cluster.  mask is [nQ, nK] of 0/1.
 */
void svg2o_topp(const float *w, const int32_t *count_k, int nQ, int nK, float p, uint8_t *mask) {
#pragma omp parallel for schedule(static)
    for (int i = 0; i < nQ; ++i) {
        const float *wr = w + (int64_t)i * nK;
        uint8_t *mr = mask + (int64_t)i * nK;
        double wmax = 0.0;
        for (int j = 0; j < nK; ++j)
            if (count_k[j] > 0 && (double)wr[j] > wmax) wmax = (double)wr[j];
        if ((double)p >= 1.0 || !(wmax > 0.0)) {
            for (int j = 0; j < nK; ++j) mr[j] = count_k[j] > 0;
            continue;
        }
        topp_item *items = (topp_item *)malloc((size_t)nK * sizeof(topp_item));
        uint64_t U = 0;
        for (int j = 0; j < nK; ++j) {
            items[j].j = j;
            items[j].u = count_k[j] > 0 ? fixed_weight((double)wr[j], wmax) : 0;
            U += items[j].u;
        }
        uint64_t T = (uint64_t)ceil((double)p * (double)U);
        qsort(items, (size_t)nK, sizeof(topp_item), topp_cmp);
        for (int j = 0; j < nK; ++j) mr[j] = 0;
        uint64_t run = 0;
        for (int r = 0; r < nK; ++r) {
            mr[items[r].j] = 1;
            run += items[r].u;
            if (run >= T) break;
        }
        free(items);
    }
}

/*
 * Semantic-aware permutation (wiki summary, Key claims section 4.1; Method (2)): tokens of the
 * same cluster become contiguous.  Stable counting sort: offsets = exclusive scan of the cluster
 * sizes (k+1 entries); perm[j] = original index of permuted row j, in (label asc, index asc).
 */
void svg2o_permute(const int32_t *labels, int64_t N, int k, int32_t *perm, int32_t *offsets) {
    int64_t *cursor = (int64_t *)calloc((size_t)k + 1, sizeof(int64_t));
    for (int64_t t = 0; t < N; ++t) cursor[labels[t] + 1] += 1;
    for (int c = 0; c < k; ++c) cursor[c + 1] += cursor[c];
    for (int c = 0; c <= k; ++c) offsets[c] = (int32_t)cursor[c];
    for (int64_t t = 0; t < N; ++t) perm[cursor[labels[t]]++] = (int32_t)t;
    free(cursor);
}

/* Row gather: Xp[j] = X[perm[j]] (applies P_Q to Q, P_K to K and V). */
void svg2o_gather_rows(const float *X, const int32_t *perm, int64_t N, int d, float *Xp) {
    for (int64_t j = 0; j < N; ++j) memcpy(Xp + j * d, X + (int64_t)perm[j] * d, (size_t)d * sizeof(float));
}

/* Inverse permutation of the output rows (Method (2)): O[perm[j]] = Op[j]. */
void svg2o_unpermute(const double *Op, const int32_t *perm, int64_t N, int d, double *O) {
    for (int64_t j = 0; j < N; ++j) memcpy(O + (int64_t)perm[j] * d, Op + j * d, (size_t)d * sizeof(double));
}

/* Exact two-pass softmax attention of one query row over a list of key row ranges. */
static void attend_row(const float *q, const float *K, const float *V, int d, double scale,
                       const int64_t *lo, const int64_t *hi, int nranges, double *out) {
    double m = -INFINITY;
    for (int r = 0; r < nranges; ++r)
        for (int64_t t = lo[r]; t < hi[r]; ++t) {
            double acc = 0.0;
            for (int i = 0; i < d; ++i) acc = acc + (double)q[i] * (double)K[t * d + i];
            double s = acc * scale;
            if (s > m) m = s;
        }
    double z = 0.0;
    for (int i = 0; i < d; ++i) out[i] = 0.0;
    for (int r = 0; r < nranges; ++r)
        for (int64_t t = lo[r]; t < hi[r]; ++t) {
            double acc = 0.0;
            for (int i = 0; i < d; ++i) acc = acc + (double)q[i] * (double)K[t * d + i];
            double e = exp(acc * scale - m);
            z = z + e;
            for (int i = 0; i < d; ++i) out[i] = out[i] + e * (double)V[t * d + i];
        }
    for (int i = 0; i < d; ++i) out[i] = out[i] / z;
}

/*
 * Variable-block-size block-sparse attention (wiki summary, Key claims section 4.3 Fig. 7(b);
 * Method (4)) on permuted tensors: a query row r of Q cluster i (q_off[i] <= r < q_off[i+1])
 * attends to the keys of every selected K cluster j (mask[i*nK + j] != 0), i.e. permuted key rows
 * [k_off[j], k_off[j+1]), with the softmax taken over those keys only (reading: standard
 * block-sparse semantics).  Computes only the requested permuted rows; out is [nrows, d].
 */
void svg2o_sparse_attention_rows(const float *Qp, const float *Kp, const float *Vp, int64_t N, int d,
                                 const int32_t *q_off, const int32_t *k_off, int nQ, int nK,
                                 const uint8_t *mask, double scale, const int64_t *rows,
                                 int64_t nrows, double *out) {
    (void)N;
#pragma omp parallel for schedule(dynamic, 4)
    for (int64_t n = 0; n < nrows; ++n) {
        int64_t r = rows[n];
        int i = 0;
        while (i < nQ - 1 && !(r >= q_off[i] && r < q_off[i + 1])) ++i;
        int64_t *lo = (int64_t *)malloc((size_t)nK * sizeof(int64_t));
        int64_t *hi = (int64_t *)malloc((size_t)nK * sizeof(int64_t));
        int nr = 0;
        for (int j = 0; j < nK; ++j)
            if (mask[(int64_t)i * nK + j] && k_off[j + 1] > k_off[j]) {
                lo[nr] = k_off[j];
                hi[nr] = k_off[j + 1];
                ++nr;
            }
        attend_row(Qp + r * d, Kp, Vp, d, scale, lo, hi, nr, out + n * d);
        free(lo);
        free(hi);
    }
}

/* Dense softmax attention for the requested rows (the baseline the sparse layer approximates). */
void svg2o_dense_attention_rows(const float *Q, const float *K, const float *V, int64_t N, int d,
                                double scale, const int64_t *rows, int64_t nrows, double *out) {
#pragma omp parallel for schedule(dynamic, 4)
    for (int64_t n = 0; n < nrows; ++n) {
        int64_t lo = 0, hi = N;
        attend_row(Q + rows[n] * d, K, V, d, scale, &lo, &hi, 1, out + n * d);
    }
}

/*
 * E4M3, the 8-bit floating point format of the FP8 attention variant (the project's roadmap item
 * "Support FP8 attention", GitHub README, Open-source Plan; the format is OCP's 8-bit floating point
 * E4M3): 1 sign bit, 4 exponent bits with bias 7, 3 mantissa bits.  Exponent field 0 holds the
 * subnormals m * 2^-9; there are no infinities; S.1111.111 is NaN, so the largest finite magnitude
 * is 1.75 * 2^8 = 448.  Value of one code.
 */
double svg2o_e4m3_value(uint8_t code) {
    int e = (code >> 3) & 15, m = code & 7;
    if (e == 15 && m == 7) return NAN;
    double v = e == 0 ? ldexp((double)m, -9) : ldexp(1.0 + m / 8.0, e - 7);
    return (code & 0x80) ? -v : v;
}

/*
 * Rounding to E4M3 as the quantiser defines it: the nearest finite code, a tie going to the code
 * with the even mantissa, magnitudes beyond 448 to 448 (saturation); the sign is kept (so a
 * negative value that rounds to zero gives -0, code 0x80); NaN gives 0x7F.  Brute force over the
 * 127 finite non-negative codes, which are ordered by value.
 */
uint8_t svg2o_e4m3_round(double x) {
    if (isnan(x)) return 0x7F;
    uint8_t sign = signbit(x) ? 0x80 : 0;
    double a = fabs(x), bd = INFINITY;
    int best = 0;
    for (int c = 0; c <= 0x7E; ++c) {
        double dd = fabs(svg2o_e4m3_value((uint8_t)c) - a);
        if (dd < bd || (dd == bd && (c & 1) == 0)) {
            best = c;
            bd = dd;
        }
    }
    return (uint8_t)(sign | best);
}

/*
 * Per-plane E4M3 quantisation (reading: the pages give no scaling scheme for their FP8 attention;
 * one scale per (batch, head) plane is the plainest).  amax = max |x| over the n values, NaN
 * entries ignored; if amax > 0, inv = fl32(448 / amax) and scale = fl32(amax / 448), else inv =
 * scale = 1; codes[i] = e4m3_round(fl32(x[i] * inv)).  A code c stands for e4m3_value(c) * scale.
 * The float32 steps are float32 operations (round to nearest), as the definition states them.
 */
void svg2o_quantize_e4m3(const float *X, int64_t n, uint8_t *codes, float *scale_out) {
    float amax = 0.0f;
    for (int64_t i = 0; i < n; ++i) {
        float a = fabsf(X[i]);
        if (a > amax) amax = a;  /* false for NaN */
    }
    float inv = 1.0f, scale = 1.0f;
    if (amax > 0.0f) {
        inv = 448.0f / amax;
        scale = amax / 448.0f;
    }
    for (int64_t i = 0; i < n; ++i) {
        float y = X[i] * inv;
        codes[i] = svg2o_e4m3_round((double)y);
    }
    *scale_out = scale;
}
