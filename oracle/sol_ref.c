/*
 * Sol-Attn forward: CPU oracle.  TEST INFRASTRUCTURE ONLY.
 *
 * Only the test suite, the package's smoke check and the benchmark's CPU-baseline leg may
 * load this file's library.  The CUDA path shares no code, header or constant with it.
 *
 * Source: "Sol-Attn: Accelerating Video Generation Inference via On-the-Fly Attention
 * Sparsification" (Li et al., 2026), the routing paragraphs (proxy scores of a query against
 * key blocks, their row mean and standard deviation, the threshold tau = mu + beta*sigma with
 * one global beta) and the paragraph on the fused operator (routing, exact sparse compute and
 * an approximation of the skipped blocks inside one online-softmax pass; skipped blocks are
 * approximated rather than dropped).  Readings where the page is silent (all recorded with the
 * design notes):
 *   - tiles and blocks are 64 tokens; the last one may be partial (n_j < 64);
 *   - a block is summarised by the mean of its keys / values (k_bar_j, v_bar_j);
 *   - routing is per 64-row query tile i with proxy S_ij = (q_bar_i . k_bar_j) / sqrt(d);
 *   - sigma is the population standard deviation of the row; a block is kept iff S_ij >= tau_i;
 *     beta = -inf keeps everything, beta = +inf keeps nothing;
 *   - a skipped block j enters the softmax of row r as ONE term with logit
 *     (q_r . k_bar_j)/sqrt(d) + ln(n_j) and value v_bar_j, i.e. it adds n_j*exp(q.k_bar/sqrt d - m)
 *     to the denominator and the same weight times v_bar_j to the numerator;
 *   - no causal mask (bidirectional diffusion attention, forward only).
 *
 * Precision: routing decides an integer (the block mask), so it is evaluated in the precision
 * the GPU uses for the same decision: pooled means, q_bar and S in float32 (sequential sums in
 * ascending token / channel order, no fused multiply-add), mu and sigma accumulated in double,
 * tau and the comparison in double.  The attention itself (scores, softmax, weighted sums) is
 * evaluated in double.  Built with -O2 -ffp-contract=off, never with fast-math.
 *
 * Layouts: q, k, v are bfloat16 bit patterns [BH, N, d] (row = token); pooled arrays are
 * float32 [BH, Nk, d]; T = 64, Nk = Nq = ceil(N / T).
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define SOL_REF_T 64

static float bf16_to_f32(uint16_t h)
{
    uint32_t u = (uint32_t)h << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return f;
}

static int64_t n_blocks(int64_t N) { return (N + SOL_REF_T - 1) / SOL_REF_T; }

static int64_t block_len(int64_t N, int64_t j)
{
    int64_t lo = j * SOL_REF_T;
    int64_t hi = lo + SOL_REF_T < N ? lo + SOL_REF_T : N;
    return hi - lo;
}

/* Mean of each 64-token block of x (one call pools K or V; the same rule gives q_bar).
 * xbar[bh][j][c] = (sum_{t in block j} x[bh][t][c], float32, ascending t) * (1.0f / n_j). */
int sol_ref_pool(const uint16_t *x, int64_t BH, int64_t N, int64_t d, float *xbar)
{
    if (!x || !xbar || BH <= 0 || N <= 0 || d <= 0) return 1;
    const int64_t Nk = n_blocks(N);
#pragma omp parallel for collapse(2) schedule(static)
    for (int64_t bh = 0; bh < BH; ++bh) {
        for (int64_t j = 0; j < Nk; ++j) {
            const int64_t n = block_len(N, j);
            const float inv = 1.0f / (float)n;
            for (int64_t c = 0; c < d; ++c) {
                float s = 0.0f;
                for (int64_t t = 0; t < n; ++t)
                    s += bf16_to_f32(x[(bh * N + j * SOL_REF_T + t) * d + c]);
                xbar[(bh * Nk + j) * d + c] = s * inv;
            }
        }
    }
    return 0;
}

/* Routing for a list of query tiles ("units"; unit = bh*Nq + i).
 * For each unit: q_bar_i (float32 block mean of the tile's rows), the proxy row
 * S_ij = fl32(sum_c q_bar_i[c]*k_bar_j[c]) * scale with scale = (float)(1/sqrt(d)),
 * mu = mean_j S_ij and sigma = sqrt(mean_j (S_ij - mu)^2) in double, tau = mu + beta*sigma
 * (beta = -inf -> tau = -inf, beta = +inf -> tau = +inf), mask_ij = (S_ij >= tau).
 * Outputs (any may be NULL): proxy [nunits][Nk] float32, stats [nunits][3] double (mu, sigma,
 * tau), mask [nunits][Nk] uint8, count [nunits] int32 (number of kept blocks). */
int sol_ref_route(const uint16_t *q, const float *kbar, int64_t BH, int64_t N, int64_t d,
                  float beta, const int64_t *units, int64_t nunits,
                  float *proxy, double *stats, uint8_t *mask, int32_t *count)
{
    if (!q || !kbar || !units || BH <= 0 || N <= 0 || d <= 0 || nunits < 0) return 1;
    if (isnan(beta)) return 1;
    const int64_t Nk = n_blocks(N);
    const int64_t Nq = Nk;
    const float scale = (float)(1.0 / sqrt((double)d));
    int bad = 0;
#pragma omp parallel for schedule(dynamic, 1) reduction(| : bad)
    for (int64_t u = 0; u < nunits; ++u) {
        const int64_t bh = units[u] / Nq, i = units[u] % Nq;
        if (units[u] < 0 || bh >= BH) { bad = 1; continue; }
        float *qbar = (float *)malloc((size_t)d * sizeof(float));
        float *row = (float *)malloc((size_t)Nk * sizeof(float));
        if (!qbar || !row) { free(qbar); free(row); bad = 1; continue; }
        const int64_t n = block_len(N, i);
        const float inv = 1.0f / (float)n;
        for (int64_t c = 0; c < d; ++c) {
            float s = 0.0f;
            for (int64_t t = 0; t < n; ++t)
                s += bf16_to_f32(q[(bh * N + i * SOL_REF_T + t) * d + c]);
            qbar[c] = s * inv;
        }
        for (int64_t j = 0; j < Nk; ++j) {
            const float *kb = kbar + (bh * Nk + j) * d;
            float acc = 0.0f;
            for (int64_t c = 0; c < d; ++c) {
                float prod = qbar[c] * kb[c];
                acc = acc + prod;
            }
            row[j] = acc * scale;
        }
        double sum = 0.0;
        for (int64_t j = 0; j < Nk; ++j) sum += (double)row[j];
        const double mu = sum / (double)Nk;
        double ss = 0.0;
        for (int64_t j = 0; j < Nk; ++j) {
            const double dev = (double)row[j] - mu;
            ss += dev * dev;
        }
        const double sigma = sqrt(ss / (double)Nk);
        double tau;
        if (isinf(beta)) tau = beta < 0 ? -INFINITY : INFINITY;
        else tau = mu + (double)beta * sigma;
        int32_t cnt = 0;
        for (int64_t j = 0; j < Nk; ++j) {
            const uint8_t m = (double)row[j] >= tau ? 1 : 0;
            cnt += m;
            if (mask) mask[u * Nk + j] = m;
            if (proxy) proxy[u * Nk + j] = row[j];
        }
        if (stats) { stats[3 * u] = mu; stats[3 * u + 1] = sigma; stats[3 * u + 2] = tau; }
        if (count) count[u] = cnt;
        free(qbar);
        free(row);
    }
    return bad;
}

/* Attention output for a list of query tiles under a given block mask.
 * For row r of tile i: every token t of a kept block j contributes logit (q_r . k_t)/sqrt(d) and
 * value v_t; every skipped block j contributes one logit (q_r . k_bar_j)/sqrt(d) + ln(n_j) with
 * value v_bar_j.  out_r = sum_z e^{z - m} val_z / sum_z e^{z - m}, m = max z (plain two-pass
 * softmax, double precision).  out is [nunits][64][d] double; rows past N are left untouched. */
int sol_ref_attend(const uint16_t *q, const uint16_t *k, const uint16_t *v,
                   const float *kbar, const float *vbar, int64_t BH, int64_t N, int64_t d,
                   const int64_t *units, int64_t nunits, const uint8_t *mask, double *out)
{
    if (!q || !k || !v || !kbar || !vbar || !units || !mask || !out) return 1;
    if (BH <= 0 || N <= 0 || d <= 0 || nunits < 0) return 1;
    const int64_t Nk = n_blocks(N);
    const int64_t Nq = Nk;
    const double scale = 1.0 / sqrt((double)d);
    int bad = 0;
#pragma omp parallel for collapse(2) schedule(dynamic, 4) reduction(| : bad)
    for (int64_t u = 0; u < nunits; ++u) {
        for (int64_t r = 0; r < SOL_REF_T; ++r) {
            const int64_t bh = units[u] / Nq, i = units[u] % Nq;
            if (units[u] < 0 || bh >= BH) { bad = 1; continue; }
            const int64_t tok = i * SOL_REF_T + r;
            if (tok >= N) continue;
            const uint8_t *mrow = mask + u * Nk;
            /* one logit per exact token of a kept block, one per skipped block */
            int64_t nterms = 0;
            for (int64_t j = 0; j < Nk; ++j) nterms += mrow[j] ? block_len(N, j) : 1;
            double *z = (double *)malloc((size_t)nterms * sizeof(double));
            double *qr = (double *)malloc((size_t)d * sizeof(double));
            double *acc = (double *)calloc((size_t)d, sizeof(double));
            if (!z || !qr || !acc) { free(z); free(qr); free(acc); bad = 1; continue; }
            for (int64_t c = 0; c < d; ++c) qr[c] = (double)bf16_to_f32(q[(bh * N + tok) * d + c]);
            int64_t p = 0;
            for (int64_t j = 0; j < Nk; ++j) {
                const int64_t nj = block_len(N, j);
                if (mrow[j]) {
                    for (int64_t t = j * SOL_REF_T; t < j * SOL_REF_T + nj; ++t) {
                        const uint16_t *kt = k + (bh * N + t) * d;
                        double s = 0.0;
                        for (int64_t c = 0; c < d; ++c) s += qr[c] * (double)bf16_to_f32(kt[c]);
                        z[p++] = s * scale;
                    }
                } else {
                    const float *kb = kbar + (bh * Nk + j) * d;
                    double s = 0.0;
                    for (int64_t c = 0; c < d; ++c) s += qr[c] * (double)kb[c];
                    z[p++] = s * scale + log((double)nj);
                }
            }
            double m = -INFINITY;
            for (int64_t e = 0; e < nterms; ++e) if (z[e] > m) m = z[e];
            double den = 0.0;
            p = 0;
            for (int64_t j = 0; j < Nk; ++j) {
                const int64_t nj = block_len(N, j);
                if (mrow[j]) {
                    for (int64_t t = j * SOL_REF_T; t < j * SOL_REF_T + nj; ++t) {
                        const double w = exp(z[p++] - m);
                        const uint16_t *vt = v + (bh * N + t) * d;
                        den += w;
                        for (int64_t c = 0; c < d; ++c) acc[c] += w * (double)bf16_to_f32(vt[c]);
                    }
                } else {
                    const double w = exp(z[p++] - m);
                    const float *vb = vbar + (bh * Nk + j) * d;
                    den += w;
                    for (int64_t c = 0; c < d; ++c) acc[c] += w * (double)vb[c];
                }
            }
            double *o = out + (u * SOL_REF_T + r) * d;
            for (int64_t c = 0; c < d; ++c) o[c] = acc[c] / den;
            free(z);
            free(qr);
            free(acc);
        }
    }
    return bad;
}
