/*
 * Oracle for attention-level speculation (ALSpec) decode attention.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the test suite, the package smoke check and
 * the CPU-baseline leg of the benchmark may load or run this file.  The CUDA
 * product path never links it, and nothing here is shared with the kernels.
 *
 * What it computes (Attention-Level Speculation, atlas.scime.ai summary, the
 * one-line summary and the "Approach" section; ICML 2025 poster page,
 * abstract): for one decode query per sequence, the self-attention output is
 * computed twice,
 *   - exactly, as softmax attention over every cached token, and
 *   - approximately, as softmax attention restricted to the "attention sink":
 *     the first S tokens plus the last W tokens of the cache,
 * and the approximation is accepted ("commit") when the relative L2 error of
 * the approximate output against the exact one is at most lambda, otherwise
 * it is rejected ("discard").
 *
 * Readings taken where the pages are silent:
 *   - softmax scale 1/sqrt(d) (standard scaled dot-product attention);
 *   - the sink set is the set union [0, S) u [L-W, L), each token once;
 *   - the relative L2 norm is taken per decode token over all H_q * d outputs
 *     of the layer's attention op; the comparison is "r <= lambda";
 *   - N = 0 with D = 0 gives r = 0; N = 0 with D > 0 gives r = +inf; a NaN r
 *     discards;
 *   - grouped-query attention: query head h reads KV head h / (H_q / H_kv).
 *
 * Precision: every input element is widened exactly to double (float and
 * bfloat16 are subsets of double); all arithmetic is double.  The softmax is
 * the plain two-pass form: scores, their maximum, exponentials, their sum,
 * and the weighted sum of value rows.  There is no tiling, no online
 * rescaling and no reordering beyond that definition.
 *
 * It also holds the output projection that follows attention (a plain
 * matrix-vector product per token) and its commit-gated form.
 *
 * Parity status of every function here: pinned by tests/test_oracle.py
 * (hand-derived cases in tests/golden, closed forms, invariants, a planted
 * needle, and a numpy textbook cross-check).
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#ifdef _OPENMP
#include <omp.h>
#endif

/* Element types the oracle reads.  Independent of the CUDA library's enum. */
enum { OR_F32 = 0, OR_BF16 = 1, OR_F64 = 2 };

/* Status codes. */
enum { OR_OK = 0, OR_BAD_ARG = 1, OR_NO_MEM = 2 };

static size_t elem_size(int dtype) {
    switch (dtype) {
    case OR_F32: return 4;
    case OR_BF16: return 2;
    case OR_F64: return 8;
    default: return 0;
    }
}

/* Widen element i of a typed array to double, exactly. */
static double load_elem(const void* base, int dtype, size_t i) {
    if (dtype == OR_F32) {
        return (double)((const float*)base)[i];
    }
    if (dtype == OR_F64) {
        return ((const double*)base)[i];
    }
    /* bfloat16: the upper half of an IEEE binary32 word. */
    uint32_t bits = (uint32_t)((const uint16_t*)base)[i] << 16;
    float f;
    memcpy(&f, &bits, sizeof f);
    return (double)f;
}

/* Membership of token j in the sink set of a cache holding L tokens:
 * j < S (a sink token) or j >= L - W (a recent token). */
static int in_sink_set(int j, int L, int n_sink, int window) {
    return j < n_sink || j >= L - window;
}

/*
 * Softmax attention of one query row over a subset of one KV head's tokens.
 *
 *   q       : d elements of type dtype
 *   k, v    : token-major rows, row j at element offset j*d, tokens [0, L)
 *   spec    : 0 -> every token in [0, L); 1 -> only the sink set
 *   weights : optional, L doubles; receives the softmax weight of every
 *             token (0 for tokens outside the set)
 *   out     : d doubles
 *   scores  : scratch of L doubles
 *
 * Returns the number of tokens attended.
 */
static int attend_one(int d, int L, int dtype, const void* q, const void* k,
                      const void* v, int n_sink, int window, int spec,
                      double* weights, double* out, double* scores) {
    const double scale = 1.0 / sqrt((double)d);
    int n = 0;
    double m = -INFINITY;

    /* Pass 1: scores s_j = (q . k_j) / sqrt(d) and their maximum. */
    for (int j = 0; j < L; ++j) {
        if (spec && !in_sink_set(j, L, n_sink, window)) {
            continue;
        }
        double dot = 0.0;
        for (int i = 0; i < d; ++i) {
            dot += load_elem(q, dtype, (size_t)i) *
                   load_elem(k, dtype, (size_t)j * d + i);
        }
        scores[j] = dot * scale;
        if (n == 0 || scores[j] > m) {
            m = scores[j];
        }
        ++n;
    }

    /* Pass 2: w_j = exp(s_j - m) and Z = sum_j w_j. */
    double z = 0.0;
    for (int j = 0; j < L; ++j) {
        if (spec && !in_sink_set(j, L, n_sink, window)) {
            continue;
        }
        scores[j] = exp(scores[j] - m);
        z += scores[j];
    }

    /* Pass 3: O = sum_j (w_j / Z) v_j. */
    for (int i = 0; i < d; ++i) {
        out[i] = 0.0;
    }
    for (int j = 0; j < L; ++j) {
        if (spec && !in_sink_set(j, L, n_sink, window)) {
            if (weights) {
                weights[j] = 0.0;
            }
            continue;
        }
        double p = scores[j] / z;
        if (weights) {
            weights[j] = p;
        }
        for (int i = 0; i < d; ++i) {
            out[i] += p * load_elem(v, dtype, (size_t)j * d + i);
        }
    }
    return n;
}

/*
 * One (query row, KV head) pair: both outputs and, optionally, both weight
 * vectors.  k and v point at token 0 of the head's rows.
 */
int alspec_oracle_head(int d, int L, int dtype, const void* q, const void* k,
                       const void* v, int n_sink, int window, double* o_spec,
                       double* o_exact, double* w_spec, double* w_exact) {
    if (d <= 0 || L <= 0 || !elem_size(dtype) || !q || !k || !v || !o_spec ||
        !o_exact || n_sink < 0 || window < 0 || n_sink + window <= 0) {
        return OR_BAD_ARG;
    }
    double* scores = (double*)malloc(sizeof(double) * (size_t)L);
    if (!scores) {
        return OR_NO_MEM;
    }
    attend_one(d, L, dtype, q, k, v, n_sink, window, 0, w_exact, o_exact, scores);
    attend_one(d, L, dtype, q, k, v, n_sink, window, 1, w_spec, o_spec, scores);
    free(scores);
    return OR_OK;
}

/*
 * Relative L2 of the approximation for one decode token, over n values:
 *   D = sum (O_exact - O_spec)^2, N = sum O_exact^2, r = sqrt(D / N).
 */
double alspec_oracle_rel_l2(const double* o_spec, const double* o_exact, long n) {
    double num = 0.0, den = 0.0;
    for (long i = 0; i < n; ++i) {
        double diff = o_exact[i] - o_spec[i];
        num += diff * diff;
        den += o_exact[i] * o_exact[i];
    }
    if (den == 0.0) {
        return num == 0.0 ? 0.0 : INFINITY;
    }
    return sqrt(num / den);
}

/* Commit iff r <= lambda; a NaN r never commits. */
int alspec_oracle_commit(double r, double lambda) {
    return r <= lambda ? 1 : 0;
}

/*
 * The whole decode step for a batch.
 *   q        : [B, Hq, d]
 *   k, v     : [B, Hkv, Lmax, d]
 *   seq_lens : [B], 1 <= L_b <= Lmax
 *   out_spec, out_exact : [B, Hq, d] doubles
 *   rel_l2   : [B] doubles;  commit : [B] bytes
 *   n_threads: OpenMP threads over (b, h) pairs; <= 0 uses the default.
 * Returns the thread count used, or a negative status on error.
 */
int alspec_oracle_decode(int B, int Hq, int Hkv, int d, int Lmax, int dtype,
                         const void* q, const void* k, const void* v,
                         const int32_t* seq_lens, int n_sink, int window,
                         double lambda, double* out_spec, double* out_exact,
                         double* rel_l2, uint8_t* commit, int n_threads) {
    size_t es = elem_size(dtype);
    if (B <= 0 || Hq <= 0 || Hkv <= 0 || Hq % Hkv != 0 || d <= 0 || Lmax <= 0 ||
        !es || !q || !k || !v || !seq_lens || !out_spec || !out_exact ||
        !rel_l2 || !commit || n_sink < 0 || window < 0 || n_sink + window <= 0) {
        return -OR_BAD_ARG;
    }
    for (int b = 0; b < B; ++b) {
        if (seq_lens[b] < 1 || seq_lens[b] > Lmax) {
            return -OR_BAD_ARG;
        }
    }
    const int g = Hq / Hkv;
    int used = 1;
    int failed = 0;
#ifdef _OPENMP
    if (n_threads > 0) {
        omp_set_num_threads(n_threads);
    }
#pragma omp parallel
    {
#pragma omp single
        used = omp_get_num_threads();
    }
#else
    (void)n_threads;
#endif
    const long pairs = (long)B * Hq;
#pragma omp parallel for schedule(dynamic, 1) reduction(| : failed)
    for (long p = 0; p < pairs; ++p) {
        int b = (int)(p / Hq);
        int h = (int)(p % Hq);
        int kvh = h / g;
        const char* qrow = (const char*)q + ((size_t)b * Hq + h) * d * es;
        size_t head_off = (((size_t)b * Hkv + kvh) * (size_t)Lmax) * d * es;
        int rc = alspec_oracle_head(d, seq_lens[b], dtype, qrow,
                                    (const char*)k + head_off,
                                    (const char*)v + head_off, n_sink, window,
                                    out_spec + ((size_t)b * Hq + h) * d,
                                    out_exact + ((size_t)b * Hq + h) * d, NULL,
                                    NULL);
        failed |= (rc != OR_OK);
    }
    if (failed) {
        return -OR_NO_MEM;
    }
    for (int b = 0; b < B; ++b) {
        const double* os = out_spec + (size_t)b * Hq * d;
        const double* oe = out_exact + (size_t)b * Hq * d;
        rel_l2[b] = alspec_oracle_rel_l2(os, oe, (long)Hq * d);
        commit[b] = (uint8_t)alspec_oracle_commit(rel_l2[b], lambda);
    }
    return used;
}

/*
 * Output projection that follows self-attention in a decoder layer: the
 * post-attention op that attention-level speculation runs on the
 * approximate output while the exact one is computed (atlas.scime.ai
 * summary, "Approach").  The plain definition, in double:
 *   y[b][j] = sum over i = 0 .. K-1, ascending, of x[b][i] * w[j][i]
 *   x : [B, K] doubles;  w : [N, K] of element type w_dtype (row j is output
 *   feature j);  y : [B, N] doubles.
 * Returns OR_OK or OR_BAD_ARG.
 */
int alspec_oracle_oproj(int B, int K, int N, const double* x, const void* w, int w_dtype,
                        double* y) {
    if (B <= 0 || K <= 0 || N <= 0 || !x || !w || !y || !elem_size(w_dtype)) {
        return OR_BAD_ARG;
    }
    for (int b = 0; b < B; ++b) {
        for (int j = 0; j < N; ++j) {
            double acc = 0.0;
            for (int i = 0; i < K; ++i) {
                acc += x[(size_t)b * K + i] * load_elem(w, w_dtype, (size_t)j * K + i);
            }
            y[(size_t)b * N + j] = acc;
        }
    }
    return OR_OK;
}

/*
 * The projection with commit or discard ("Approach": the speculative
 * post-attention result is kept when the check commits, otherwise the op is
 * redone on the exact attention output):
 *   y[b] = o_proj(commit[b] ? o_spec[b] : o_exact[b])
 * o_spec, o_exact : [B, K] doubles; commit : [B] bytes (non-zero = commit).
 */
int alspec_oracle_oproj_gated(int B, int K, int N, const double* o_spec, const double* o_exact,
                              const uint8_t* commit, const void* w, int w_dtype, double* y) {
    if (B <= 0 || !o_spec || !o_exact || !commit) {
        return OR_BAD_ARG;
    }
    for (int b = 0; b < B; ++b) {
        const double* x = commit[b] ? o_spec + (size_t)b * K : o_exact + (size_t)b * K;
        int rc = alspec_oracle_oproj(1, K, N, x, w, w_dtype, y + (size_t)b * N);
        if (rc != OR_OK) {
            return rc;
        }
    }
    return OR_OK;
}
