/*
 * fp64 CPU oracle for the forward pass of 3D-RoPE sparse + low-rank hybrid attention.
 *
 * TEST INFRASTRUCTURE ONLY.  This file is the slow, plain definition that the CUDA path is checked
 * against.  Only the tests, the smoke check and the benchmark's CPU-baseline leg may load it; the
 * library never does.  It shares no code, header, table or helper with the CUDA path.
 *
 * Every function works on ONE attention head of ONE batch element: row-major [L][D] arrays of fp64
 * values (the exact values of the bf16 inputs).  All arithmetic is IEEE fp64, no fast-math, in the
 * order the definitions are written.  Loops are parallelised with OpenMP only over independent
 * outputs, so results do not depend on the thread count.
 *
 * Sources (page title, section):
 *   RoLA: Rotary-Positioned Low-Rank Linear Attention for Efficient Diffusion Transformers
 *     "3 Preliminary" (full attention over L = T*H*W flattened tokens; 3D RoPE splits a head across
 *     the temporal and spatial axes and makes scores depend on relative offsets, eq. (1)),
 *     "4.1" (block-sparse attention for high-energy spikes + a low-rank branch whose global context is
 *     computed once per head at O(L r d_h)), "4.2" (the low-rank branch reuses the first r rotary
 *     coordinates in the backbone's native ordering: r/2 complete pairs, same cos/sin tensors),
 *     "4.3" (RoPE applied after the low-rank nonlinearity), "B.1" (one query-independent sum),
 *     "B.2" (geometrically spaced rotary schedule).
 *   RoPeSLR: 3D RoPE-driven Sparse-LowRank Attention for Efficient Diffusion Transformers,
 *     appendix on 3D RoPE (rotary base 10000, head dim partitioned across the t, x, y axes).
 * The block-mean-pooled selection score, relu feature map phi(x) = relu(x A) with one A of shape
 * [D][R], the normaliser phi(q).sum_j phi(k_j) + 1e-6 and the plain sum of the two branches are the
 * construction this implementation targets; readings of points the pages leave open are listed in
 * the design notes and repeated at each function below.  RoLA's ablation ("5.3", Table 6) adds two
 * options: SiLU, identity or tanh in place of relu, and the low-rank branch without its RoPE.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define ORC_EXPORT __attribute__((visibility("default")))

ORC_EXPORT int orc_version(void) { return 1; }

/* bf16 bit pattern -> exact fp64 value. */
ORC_EXPORT void orc_decode_bf16(const uint16_t* src, int64_t n, double* dst) {
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < n; ++i) {
        uint32_t u = (uint32_t)src[i] << 16;
        float f;
        memcpy(&f, &u, sizeof f);
        dst[i] = (double)f;
    }
}

/*
 * Rotary pair layout (3D RoPE, RoLA "3 Preliminary"; RoPeSLR appendix: base 10000, head dim
 * partitioned over (t, x, y)).  The D/2 coordinate pairs (2j, 2j+1) are split into consecutive
 * groups for the t, h and w axes.  Default split, in pairs: t gets c - 2*floor(c/3), h and w get
 * floor(c/3) each (c = D/2); for D = 128 that is 22/21/21 pairs = 44/42/42 dims (the Wan split).
 * Within axis a with p_a pairs (axis width d_a = 2 p_a), local pair m rotates with frequency
 * omega = theta^(-2m / d_a) (geometric schedule, RoLA "B.2").
 * split3: pairs per axis, or NULL for the default.  axis[j] in {0,1,2}, omega[j] for j < D/2.
 */
ORC_EXPORT int orc_rope_pairs(int64_t D, const int64_t* split3, double theta, int32_t* axis, double* omega) {
    int64_t c = D / 2;
    int64_t p[3];
    if (split3) {
        p[0] = split3[0]; p[1] = split3[1]; p[2] = split3[2];
    } else {
        p[1] = c / 3; p[2] = c / 3; p[0] = c - 2 * (c / 3);
    }
    if (p[0] < 0 || p[1] < 0 || p[2] < 0 || p[0] + p[1] + p[2] != c) return -1;
    int64_t j = 0;
    for (int a = 0; a < 3; ++a) {
        double da = 2.0 * (double)p[a];
        for (int64_t m = 0; m < p[a]; ++m, ++j) {
            axis[j] = a;
            omega[j] = pow(theta, -2.0 * (double)m / da);
        }
    }
    return 0;
}

/*
 * Token n of the flattened grid sits at (t, h, w) = (n / (H W), (n / W) mod H, n mod W): row-major
 * t, then h, then w (RoLA "3 Preliminary": L is the product of the temporal and spatial sizes).
 * Positions are 0-based integers plus an optional constant offset per axis (used to test shift
 * invariance).
 */
static void token_pos(int64_t n, int64_t H, int64_t W, const int64_t* off, double pos[3]) {
    int64_t t = n / (H * W);
    int64_t h = (n / W) % H;
    int64_t w = n % W;
    pos[0] = (double)(t + (off ? off[0] : 0));
    pos[1] = (double)(h + (off ? off[1] : 0));
    pos[2] = (double)(w + (off ? off[2] : 0));
}

/*
 * Rotate pairs j < npairs of every row of x [L][D] by angle pos_{axis[j]} * omega[j]:
 *   (x_2j, x_2j+1) -> (x_2j cos a - x_2j+1 sin a,  x_2j sin a + x_2j+1 cos a),
 * and copy coordinates 2*npairs .. D-1 unchanged.  npairs = D/2 is the full 3D RoPE; npairs = r/2 is
 * the rank-truncated rotation of the low-rank branch (RoLA "4.2": first r coordinates in native order).
 */
ORC_EXPORT void orc_rope_rows(const double* x, int64_t L, int64_t D, int64_t T, int64_t H, int64_t W,
                              const int64_t* off, const int32_t* axis, const double* omega, int64_t npairs,
                              double* y) {
    (void)T;
#pragma omp parallel for schedule(static)
    for (int64_t n = 0; n < L; ++n) {
        double pos[3];
        token_pos(n, H, W, off, pos);
        const double* xr = x + n * D;
        double* yr = y + n * D;
        for (int64_t j = 0; j < npairs; ++j) {
            double a = pos[axis[j]] * omega[j];
            double c = cos(a), s = sin(a);
            double x0 = xr[2 * j], x1 = xr[2 * j + 1];
            yr[2 * j] = x0 * c - x1 * s;
            yr[2 * j + 1] = x0 * s + x1 * c;
        }
        for (int64_t i = 2 * npairs; i < D; ++i) yr[i] = xr[i];
    }
}

/*
 * Block mean pooling: block beta covers tokens [beta*b, min(L, (beta+1)*b)); its mean is taken over
 * the block's real tokens (a partial last block is averaged over what it has).  xbar [nb][D].
 */
ORC_EXPORT void orc_block_means(const double* x, int64_t L, int64_t D, int64_t b, double* xbar) {
    int64_t nb = (L + b - 1) / b;
#pragma omp parallel for schedule(static)
    for (int64_t beta = 0; beta < nb; ++beta) {
        int64_t lo = beta * b, hi = lo + b < L ? lo + b : L;
        for (int64_t d = 0; d < D; ++d) {
            double s = 0.0;
            for (int64_t n = lo; n < hi; ++n) s += x[n * D + d];
            xbar[beta * D + d] = s / (double)(hi - lo);
        }
    }
}

/* Block scores s[alpha][beta] = qbar_alpha . kbar_beta (unscaled; the scale does not change ranks). */
ORC_EXPORT void orc_block_scores(const double* qbar, const double* kbar, int64_t nb, int64_t D, double* s) {
#pragma omp parallel for schedule(static)
    for (int64_t a = 0; a < nb; ++a)
        for (int64_t b = 0; b < nb; ++b) {
            double acc = 0.0;
            for (int64_t d = 0; d < D; ++d) acc += qbar[a * D + d] * kbar[b * D + d];
            s[a * nb + b] = acc;
        }
}

/* Number of kept key blocks per query block: round(kappa * nb) half up, clamped to [1, nb]. */
ORC_EXPORT int64_t orc_keep_count(double keep_frac, int64_t nb) {
    int64_t k = (int64_t)floor(keep_frac * (double)nb + 0.5);
    if (k < 1) k = 1;
    if (k > nb) k = nb;
    return k;
}

typedef struct {
    double s;
    int64_t beta;
} scored_t;

/* Order: higher score first; equal scores -> lower block index first (deterministic tie-break). */
static int cmp_score_desc(const void* pa, const void* pb) {
    const scored_t* a = (const scored_t*)pa;
    const scored_t* b = (const scored_t*)pb;
    if (a->s > b->s) return -1;
    if (a->s < b->s) return 1;
    return (a->beta < b->beta) ? -1 : (a->beta > b->beta);
}

static int cmp_i32(const void* pa, const void* pb) {
    int32_t a = *(const int32_t*)pa, b = *(const int32_t*)pb;
    return (a > b) - (a < b);
}

/*
 * Per query block alpha: K(alpha) = the first k key blocks when sorted by (score desc, index asc)
 * (top-k "spike" blocks, RoLA Fig. 2 / "4.1"), returned in ascending block order in idx [nb][k].
 * tie[alpha] = 1 when k < nb and the k-th and (k+1)-th sorted scores are within
 * 1e-6 * max(1, |s_(k)|): the selection there is numerically fragile and two correct
 * implementations may differ.
 */
ORC_EXPORT void orc_topk(const double* s, int64_t nb, int64_t k, int32_t* idx, uint8_t* tie) {
#pragma omp parallel for schedule(static)
    for (int64_t a = 0; a < nb; ++a) {
        scored_t* row = (scored_t*)malloc((size_t)nb * sizeof(scored_t));
        for (int64_t b = 0; b < nb; ++b) { row[b].s = s[a * nb + b]; row[b].beta = b; }
        qsort(row, (size_t)nb, sizeof(scored_t), cmp_score_desc);
        for (int64_t j = 0; j < k; ++j) idx[a * k + j] = (int32_t)row[j].beta;
        qsort(idx + a * k, (size_t)k, sizeof(int32_t), cmp_i32);
        uint8_t t = 0;
        if (k < nb) {
            double sk = row[k - 1].s, sk1 = row[k].s;
            double band = 1e-6 * (fabs(sk) > 1.0 ? fabs(sk) : 1.0);
            t = (sk - sk1) <= band;
        }
        tie[a] = t;
        free(row);
    }
}

/*
 * Block-sparse softmax attention (RoLA "4.1"): for each query i of block alpha, exact softmax of
 * qh_i . kh_j / sqrt(D) over the union of the kept key blocks K(alpha), then sum_j p_ij v_j.
 * Keys past L (inside a partial last block) do not exist and are not attended.
 * qblocks: list of nq query-block indices to compute; out rows of other blocks are left untouched.
 */
ORC_EXPORT void orc_sparse_attn(const double* qh, const double* kh, const double* v, int64_t L, int64_t D,
                                int64_t b, const int32_t* idx, int64_t k, const int64_t* qblocks, int64_t nq,
                                double* out) {
    double scale = 1.0 / sqrt((double)D);
#pragma omp parallel for schedule(dynamic)
    for (int64_t qi = 0; qi < nq; ++qi) {
        int64_t a = qblocks[qi];
        int64_t lo = a * b, hi = lo + b < L ? lo + b : L;
        double* logit = (double*)malloc((size_t)(k * b) * sizeof(double));
        int64_t* key = (int64_t*)malloc((size_t)(k * b) * sizeof(int64_t));
        int64_t nk = 0;
        for (int64_t j = 0; j < k; ++j) {
            int64_t beta = idx[a * k + j];
            int64_t klo = beta * b, khi = klo + b < L ? klo + b : L;
            for (int64_t n = klo; n < khi; ++n) key[nk++] = n;
        }
        for (int64_t i = lo; i < hi; ++i) {
            double m = -INFINITY;
            for (int64_t t = 0; t < nk; ++t) {
                double acc = 0.0;
                for (int64_t d = 0; d < D; ++d) acc += qh[i * D + d] * kh[key[t] * D + d];
                logit[t] = acc * scale;
                if (logit[t] > m) m = logit[t];
            }
            double denom = 0.0;
            for (int64_t t = 0; t < nk; ++t) { logit[t] = exp(logit[t] - m); denom += logit[t]; }
            for (int64_t d = 0; d < D; ++d) {
                double acc = 0.0;
                for (int64_t t = 0; t < nk; ++t) acc += logit[t] * v[key[t] * D + d];
                out[i * D + d] = acc / denom;
            }
        }
        free(logit);
        free(key);
    }
}

/*
 * Feature map phi(x) = act(x A) on the raw (pre-RoPE) rows: x [L][D], A [D][R] -> phi [L][R].
 * act: 0 relu (the benchmark's map), 1 SiLU u / (1 + e^-u), 2 identity, 3 tanh -- the activations
 * RoLA's ablation compares (RoLA "5.3", Table 6).
 */
static double orc_act(double u, int act) {
    switch (act) {
        case 1: return u / (1.0 + exp(-u));
        case 2: return u;
        case 3: return tanh(u);
        default: return u > 0.0 ? u : 0.0;
    }
}

ORC_EXPORT void orc_features(const double* x, int64_t L, int64_t D, const double* A, int64_t R, int act,
                             double* phi) {
#pragma omp parallel for schedule(static)
    for (int64_t n = 0; n < L; ++n)
        for (int64_t c = 0; c < R; ++c) {
            double acc = 0.0;
            for (int64_t d = 0; d < D; ++d) acc += x[n * D + d] * A[d * R + c];
            phi[n * R + c] = orc_act(acc, act);
        }
}

/*
 * Query-independent global summary, computed once per head (RoLA "4.1", "B.1"):
 *   S[c][e] = sum_j psik[j][c] * v[j][e]      (psik = rotated features, RoPE outside the activation)
 *   z[c]    = sum_j phik[j][c]                (unrotated features, for the normaliser)
 * over all L keys (the branch is global and unmasked).
 */
ORC_EXPORT void orc_summary(const double* psik, const double* phik, const double* v, int64_t L, int64_t R,
                            int64_t D, double* S, double* z) {
#pragma omp parallel for schedule(static)
    for (int64_t c = 0; c < R; ++c) {
        for (int64_t e = 0; e < D; ++e) {
            double acc = 0.0;
            for (int64_t j = 0; j < L; ++j) acc += psik[j * R + c] * v[j * D + e];
            S[c * D + e] = acc;
        }
        double acc = 0.0;
        for (int64_t j = 0; j < L; ++j) acc += phik[j * R + c];
        z[c] = acc;
    }
}

/*
 * Query-side readout of the low-rank branch for the given query rows:
 *   O_lr[i][e] = (sum_c psiq[i][c] S[c][e]) / (sum_c phiq[i][c] z[c] + 1e-6).
 * The numerator uses the rotated query features, the denominator the unrotated ones.
 */
ORC_EXPORT void orc_lowrank_apply(const double* psiq, const double* phiq, const double* S, const double* z,
                                  int64_t R, int64_t D, const int64_t* rows, int64_t nrows, double* out) {
#pragma omp parallel for schedule(static)
    for (int64_t t = 0; t < nrows; ++t) {
        int64_t i = rows[t];
        double den = 0.0;
        for (int64_t c = 0; c < R; ++c) den += phiq[i * R + c] * z[c];
        den += 1e-6;
        for (int64_t e = 0; e < D; ++e) {
            double num = 0.0;
            for (int64_t c = 0; c < R; ++c) num += psiq[i * R + c] * S[c * D + e];
            out[i * D + e] = num / den;
        }
    }
}

/*
 * Gated fusion of the two branches (RoLA "4.4": a token-wise scalar gate combines the sparse and the
 * global output, the sparse output's RMS is the scale reference, and a negative gate bias starts the
 * module near the sparse-only output; "E.2" names the gate parameters Wg, bg).  The pages give no
 * formula; the reading implemented here, for each query row i of one head:
 *   g_i    = 1 / (1 + exp(-(q_i . w + b)))          q_i the raw (pre-RoPE) query, w = Wg [D], b = bg
 *   rms(x) = sqrt(sum_e x[e]^2 / D)
 *   out_i  = O_s,i + g_i * O_lr,i * rms(O_s,i) / sqrt(sum_e O_lr,i[e]^2 / D + 1e-6)
 * i.e. the global output is brought to the sparse output's RMS and then gated.
 */
ORC_EXPORT void orc_gated_fusion(const double* os, const double* olr, const double* q, const double* w, double b,
                                 int64_t D, const int64_t* rows, int64_t nrows, double* out) {
#pragma omp parallel for schedule(static)
    for (int64_t t = 0; t < nrows; ++t) {
        int64_t i = rows[t];
        double logit = b;
        for (int64_t e = 0; e < D; ++e) logit += q[i * D + e] * w[e];
        double g = 1.0 / (1.0 + exp(-logit));
        double ss = 0.0, sl = 0.0;
        for (int64_t e = 0; e < D; ++e) {
            ss += os[i * D + e] * os[i * D + e];
            sl += olr[i * D + e] * olr[i * D + e];
        }
        double scale = sqrt(ss / (double)D) / sqrt(sl / (double)D + 1e-6);
        for (int64_t e = 0; e < D; ++e) out[i * D + e] = os[i * D + e] + g * olr[i * D + e] * scale;
    }
}
