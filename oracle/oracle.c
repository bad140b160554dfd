/*
 * oracle.c -- plain, slow, fp64 CPU oracle for confidence-scheduled
 * speculative verification.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path may link, load or
 * call this file: only the tests, the smoke check and the benchmark's CPU
 * baseline use it.  It shares no source, header, table or constant with the
 * CUDA library; the two meet only through the seeded synthetic inputs.
 *
 * Sources (cited as page title + section):
 *  [P1] umans.ai, "DeepSeek V4 Pro DSpark: the model isn't ready, the
 *       architecture is": sections "Speculative decoding, briefly" and
 *       "What DSpark adds" (item "2. Verify smarter").
 *  [P2] en.5iter.com DSpark news article: sections "Guess first, then test"
 *       and "What DSpark changed is how to generate a draft".
 *  [P3] zhichai.net DSpark topic: sections "Why LLMs speak so slowly" and
 *       "Under the hood: why parallel drafts get weirder".
 *  [P4] techvisionai, "DeepSeek-V4: Breaking the Efficiency Barrier",
 *       Chapter 7 "DSpark", subsections "Confidence-Scheduled Verification"
 *       and "Deployment with vLLM".
 *  [P5] aiweekly.co, "DeepSeek DSpark accelerates V4 per-user generation
 *       60-85%".
 *  [SC11] J. Salmon, M. Moraes, R. Dror, D. Shaw, "Parallel Random Numbers:
 *       As Easy as 1, 2, 3", SC'11 -- the Philox-4x32 bijection.
 *
 * The pages state the rule in words only: the target accepts the prefix it
 * agrees with plus one token of its own [P1 "Speculative decoding, briefly"],
 * by rejection sampling on the target/draft probability ratio [P3 "Why LLMs
 * speak so slowly"], which leaves the accepted tokens distributed exactly as
 * the target's own [P1]; a rejected token gives way to one of the target's
 * choosing [P1].  Written out in symbols (the standard speculative-sampling rule):
 *   accept x_i with probability min(1, p_i(x_i) / q_i(x_i)); at the first
 *   rejection j emit a draw from norm(max(0, p_j - q_j)); if all L drafts
 *   survive emit a bonus draw from p_L.
 * The verify length L comes from prefix survival S_i = prod_{j<=i} c_j
 * [P1 "Verify smarter"; P5] cut at a load threshold tau [P2; P4 Ch.7].
 *
 * Readings where the pages are silent (each is listed in the design notes):
 *  - accept iff u < min(1, ratio), u in [0,1);
 *  - inverse CDF in token order, y = smallest v with C(v) > t, t = u * R;
 *  - one temperature T per row for both models; T == 0 means greedy
 *    (argmax, lowest index wins ties); 0 < T < 1e-6 is a data error;
 *  - the bonus is drawn from target position L (not K);
 *  - uniforms: Philox4x32-10 [SC11], key = (seed_lo, seed_hi), counter =
 *    (row_lo, pos, draw, row_hi), u = (word0 >> 8) * 2^-24; draw 0 is the
 *    accept test at position pos, draw 1 the resample/bonus at pos;
 *  - residual mass R == 0 after a rejection (only reachable through
 *    rounding): draw from p_j instead (flagged in the diagnostics);
 *  - a NULL draft array means a greedy drafter: q_i is one-hot at x_i
 *    ([P4 Ch.7 "Deployment with vLLM", draft_sample_method greedy]).
 *
 * Pins (tests/test_oracle_*.py): exact interval enumeration against the
 * target distribution, chi-square of Philox-keyed draws, greedy reduction to
 * a brute-force longest matching prefix, closed-form E[accept length],
 * schedule invariants and a hand-worked example, and Philox agreement with
 * Triton's independent Philox implementation run on the CPU.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

enum { OR_F32 = 0, OR_BF16 = 1, OR_F64 = 2 };

/* Largest number of drafts per row the window enumeration handles. */
#define OR_MAX_K 64

/* ---------------------------------------------------------------------------
 * Philox4x32-10 [SC11].  One round: two 32x32->64 multiplications of the
 * even words by the round multipliers; the high halves are XORed with the
 * odd words and the key, the low halves pass through; the words are then
 * permuted.  The key is bumped by the Weyl constants between rounds.
 * ------------------------------------------------------------------------- */
#define PHILOX_M0 0xD2511F53u
#define PHILOX_M1 0xCD9E8D57u
#define PHILOX_W0 0x9E3779B9u
#define PHILOX_W1 0xBB67AE85u

void oracle_philox4x32_10(const uint32_t ctr[4], const uint32_t key[2], uint32_t out[4])
{
    uint32_t x0 = ctr[0], x1 = ctr[1], x2 = ctr[2], x3 = ctr[3];
    uint32_t k0 = key[0], k1 = key[1];
    for (int r = 0; r < 10; ++r) {
        uint64_t p0 = (uint64_t)PHILOX_M0 * (uint64_t)x0;
        uint64_t p1 = (uint64_t)PHILOX_M1 * (uint64_t)x2;
        uint32_t hi0 = (uint32_t)(p0 >> 32), lo0 = (uint32_t)p0;
        uint32_t hi1 = (uint32_t)(p1 >> 32), lo1 = (uint32_t)p1;
        uint32_t y0 = hi1 ^ x1 ^ k0;
        uint32_t y1 = lo1;
        uint32_t y2 = hi0 ^ x3 ^ k1;
        uint32_t y3 = lo0;
        x0 = y0; x1 = y1; x2 = y2; x3 = y3;
        k0 += PHILOX_W0;
        k1 += PHILOX_W1;
    }
    out[0] = x0; out[1] = x1; out[2] = x2; out[3] = x3;
}

/* u(seed, row, pos, draw) in [0,1): the top 24 bits of word 0, scaled by
 * 2^-24, so the value is exact in both fp32 and fp64. */
double oracle_uniform(uint64_t seed, uint64_t row, uint32_t pos, uint32_t draw)
{
    uint32_t ctr[4] = { (uint32_t)row, pos, draw, (uint32_t)(row >> 32) };
    uint32_t key[2] = { (uint32_t)seed, (uint32_t)(seed >> 32) };
    uint32_t out[4];
    oracle_philox4x32_10(ctr, key, out);
    return (double)(out[0] >> 8) * (1.0 / 16777216.0);
}

/* Uniforms for n (row, pos, draw) triples; used by the statistical pins. */
void oracle_uniform_batch(uint64_t seed, const uint64_t *row, const uint32_t *pos,
                          const uint32_t *draw, int64_t n, double *out)
{
    for (int64_t k = 0; k < n; ++k) out[k] = oracle_uniform(seed, row[k], pos[k], draw[k]);
}

/* ---------------------------------------------------------------------------
 * Logit access.  bf16 is widened by placing its 16 bits in the top half of
 * an IEEE single, which is exact.
 * ------------------------------------------------------------------------- */
typedef struct { const void *p; int dtype; } vec_t;

static double zval(vec_t z, int64_t v)
{
    if (z.dtype == OR_F64) return ((const double *)z.p)[v];
    if (z.dtype == OR_F32) return (double)((const float *)z.p)[v];
    uint32_t bits = (uint32_t)((const uint16_t *)z.p)[v] << 16;
    float f;
    memcpy(&f, &bits, sizeof f);
    return (double)f;
}

static size_t elt_size(int dtype) { return dtype == OR_F64 ? 8 : dtype == OR_F32 ? 4 : 2; }

static vec_t vec_at(const void *base, int dtype, int64_t index, int V)
{
    vec_t r = { (const char *)base + (size_t)index * (size_t)V * elt_size(dtype), dtype };
    return r;
}

/* Temperature-scaled softmax statistics of one logit vector:
 * m = max_v z_v and Sigma = sum_v exp((z_v - m) / T), so that
 * p(v) = exp((z_v - m) / T) / Sigma. */
static void softmax_stats(vec_t z, int V, double T, double *m_out, double *sum_out)
{
    double m = -INFINITY;
    for (int v = 0; v < V; ++v) {
        double x = zval(z, v);
        if (x > m) m = x;
    }
    double s = 0.0;
    for (int v = 0; v < V; ++v) s += exp((zval(z, v) - m) / T);
    *m_out = m;
    *sum_out = s;
}

/* Index of the largest logit; ties go to the lowest index. */
static int argmax_first(vec_t z, int V)
{
    int best = 0;
    double bv = zval(z, 0);
    for (int v = 1; v < V; ++v) {
        double x = zval(z, v);
        if (x > bv) { bv = x; best = v; }
    }
    return best;
}

void oracle_vector_stats(const void *z, int dtype, int V, double T,
                         double *m, double *sum, int32_t *amax)
{
    vec_t zz = { z, dtype };
    if (T > 0.0) softmax_stats(zz, V, T, m, sum);
    else { *m = zval(zz, argmax_first(zz, V)); *sum = 1.0; }
    if (amax) *amax = argmax_first(zz, V);
}

/* Inverse-CDF draw in token order 0..V-1 from the unnormalised weights r:
 * R = sum_v r(v), t = u * R, y = the smallest v with C(v) = sum_{w<=v} r(w)
 * strictly greater than t.  margin = distance from t to the nearer CDF
 * boundary of the chosen token, relative to R.  If no v qualifies (R == 0,
 * or rounding put t at the total) the last v with r(v) > 0 is returned and
 * *fallback is set; -1 if every weight is zero. */
static int inverse_cdf(const double *r, int V, double u, double *margin, int *fallback)
{
    double R = 0.0;
    for (int v = 0; v < V; ++v) R += r[v];
    double t = u * R;
    double C = 0.0;
    for (int v = 0; v < V; ++v) {
        double prev = C;
        C += r[v];
        if (C > t) {
            double a = t - prev, b = C - t;
            *margin = (a < b ? a : b) / R;
            *fallback = 0;
            return v;
        }
    }
    *fallback = 1;
    *margin = 0.0;
    for (int v = V - 1; v >= 0; --v)
        if (r[v] > 0.0) return v;
    return -1;
}

/* Diagnostics written per row (double[OR_NDIAG]):
 *  [0] smallest |u_i - min(1, ratio_i)| over the tested positions 0..j
 *      (+inf when none were tested, or for greedy rows);
 *  [1] inverse-CDF margin of the correction/bonus draw, relative to R
 *      (+inf for greedy rows);
 *  [2] flags: 1 = residual mass was zero (drew from p_j), 2 = inverse-CDF
 *      fallback taken;
 *  [3] j: first rejected position, or L when every draft survived;
 *  [4] R: total mass of the distribution the final token was drawn from. */
#define OR_NDIAG 5

/*
 * One row, uniforms injected.
 *   zt: target logits [K+1, V]; zd: draft logits [K, V] or NULL (greedy
 *   drafter, q_i one-hot at x_i); x: draft tokens [K]; L: verify length;
 *   T: temperature (0 = greedy verification); u_acc[i]: accept uniform of
 *   position i; u_res[i]: resample/bonus uniform used if the final token is
 *   drawn at position i.  Writes out_tokens[0..K] (x_0..x_{a-1}, y, then -1)
 *   and returns a, the accepted length.
 */
static int verify_row(vec_t zt_row, const void *zd_base, int dtype, int K, int V,
                      const int32_t *x, int L, double T,
                      const double *u_acc, const double *u_res,
                      int32_t *out_tokens, double *diag, double *work)
{
    double d0 = INFINITY, d1 = INFINITY, flags = 0.0, Rfinal = 0.0;
    int j = L;
    int y;

    if (T == 0.0) {
        /* Greedy verification: keep x_i while it equals the target argmax;
         * the final token is the target argmax at the first mismatch (or at
         * L).  No uniforms are drawn and draft logits are not read. */
        j = L;
        for (int i = 0; i < L; ++i) {
            vec_t zt = vec_at(zt_row.p, dtype, i, V);
            if (x[i] != argmax_first(zt, V)) { j = i; break; }
        }
        y = argmax_first(vec_at(zt_row.p, dtype, j, V), V);
        Rfinal = 1.0;
    } else {
        double *r = work; /* V doubles */
        int rejected = 0;
        double mt = 0, st = 0, md = 0, sd = 0;
        for (int i = 0; i < L; ++i) {
            vec_t zt = vec_at(zt_row.p, dtype, i, V);
            softmax_stats(zt, V, T, &mt, &st);
            double logp = (zval(zt, x[i]) - mt) / T - log(st);
            double logq;
            if (zd_base) {
                vec_t zd = vec_at(zd_base, dtype, i, V);
                softmax_stats(zd, V, T, &md, &sd);
                logq = (zval(zd, x[i]) - md) / T - log(sd);
            } else {
                logq = 0.0; /* q_i(x_i) = 1 */
            }
            /* min(1, p/q) in the log domain; p == 0 rejects, q == 0 accepts. */
            double acc;
            if (logp == -INFINITY) acc = 0.0;
            else if (logq == -INFINITY) acc = 1.0;
            else acc = logp >= logq ? 1.0 : exp(logp - logq);
            double mg = fabs(u_acc[i] - acc);
            if (mg < d0) d0 = mg;
            if (u_acc[i] < acc) continue; /* accepted */
            /* First rejection at i: residual r = max(0, p_i - q_i). */
            j = i;
            rejected = 1;
            for (int v = 0; v < V; ++v) {
                double p = exp((zval(zt, v) - mt) / T) / st;
                double q;
                if (zd_base) {
                    vec_t zd = vec_at(zd_base, dtype, i, V);
                    q = exp((zval(zd, v) - md) / T) / sd;
                } else {
                    q = (v == x[i]) ? 1.0 : 0.0;
                }
                r[v] = p - q > 0.0 ? p - q : 0.0;
            }
            break;
        }
        int fb = 0;
        double mg = 0.0;
        if (rejected) {
            double R = 0.0;
            for (int v = 0; v < V; ++v) R += r[v];
            if (R == 0.0) {
                /* p_j == q_j to rounding: the rejection had probability ~0.
                 * Draw from p_j instead. */
                vec_t zt = vec_at(zt_row.p, dtype, j, V);
                for (int v = 0; v < V; ++v) r[v] = exp((zval(zt, v) - mt) / T) / st;
                flags += 1.0;
            }
        } else {
            /* Every draft survived: bonus draw from p_L. */
            vec_t zt = vec_at(zt_row.p, dtype, L, V);
            softmax_stats(zt, V, T, &mt, &st);
            for (int v = 0; v < V; ++v) r[v] = exp((zval(zt, v) - mt) / T) / st;
        }
        Rfinal = 0.0;
        for (int v = 0; v < V; ++v) Rfinal += r[v];
        y = inverse_cdf(r, V, u_res[j], &mg, &fb);
        if (fb) flags += 2.0;
        d1 = mg;
    }

    for (int i = 0; i < j; ++i) out_tokens[i] = x[i];
    out_tokens[j] = y;
    for (int i = j + 1; i <= K; ++i) out_tokens[i] = -1;
    if (diag) {
        diag[0] = d0; diag[1] = d1; diag[2] = flags; diag[3] = (double)j; diag[4] = Rfinal;
    }
    return j;
}

/* Single row with fp64 logits and injected uniforms (for exact enumeration).
 * zd may be NULL (greedy drafter).  Returns a; -1 on bad arguments. */
int oracle_verify_row_u(const double *zt, const double *zd, int K, int V,
                        const int32_t *x, int L, double T,
                        const double *u_acc, const double *u_res,
                        int32_t *out_tokens, double *diag)
{
    if (K < 0 || V <= 0 || L < 0 || L > K || !(T >= 0.0)) return -1;
    for (int i = 0; i < L; ++i) if (x[i] < 0 || x[i] >= V) return -1;
    double *work = (double *)malloc(sizeof(double) * (size_t)V);
    if (!work) return -1;
    vec_t zr = { zt, OR_F64 };
    int a = verify_row(zr, zd, OR_F64, K, V, x, L, T, u_acc, u_res, out_tokens, diag, work);
    free(work);
    return a;
}

/* Data checks shared by the batch entry point: a row is invalid when its
 * length is outside [0,K], its temperature is negative, NaN, infinite or in
 * (0, 1e-6), or a draft token it verifies lies outside [0,V).  Returns the
 * status bits (1 token, 2 length, 4 temperature). */
static int row_errors(int K, int V, const int32_t *x, int L, float T)
{
    int bits = 0;
    if (L < 0 || L > K) bits |= 2;
    if (!(T >= 0.0f) || isinf(T) || (T > 0.0f && T < 1e-6f)) bits |= 4;
    if (!(bits & 2))
        for (int i = 0; i < L; ++i)
            if (x[i] < 0 || x[i] >= V) { bits |= 1; break; }
    return bits;
}

/*
 * Batch verification with Philox-keyed uniforms.
 *   zt [B, K+1, V], zd [B, K, V] (or NULL: greedy drafter), dtype OR_F32 or
 *   OR_BF16; tokens [B, K]; lengths [B]; temperature [B]; the Philox row id
 *   of local row b is row_ids[b] if row_ids is non-NULL, else row_base + b.
 *   Outputs out_tokens [B, K+1], out_accept [B] (-1 and a row of -1 for an
 *   invalid row), diag [B, OR_NDIAG] (nullable).  Returns the OR of the
 *   status bits of all rows.  nthreads <= 0 uses the OpenMP default.
 */
int oracle_verify(const void *zt, const void *zd, int dtype, int64_t B, int K, int V,
                  const int32_t *tokens, const int32_t *lengths, const float *temperature,
                  uint64_t seed, int64_t row_base, const int64_t *row_ids,
                  int32_t *out_tokens, int32_t *out_accept, double *diag, int nthreads)
{
    int status = 0;
#ifdef _OPENMP
    if (nthreads > 0) omp_set_num_threads(nthreads);
#else
    (void)nthreads;
#endif
#pragma omp parallel reduction(| : status)
    {
        double *work = (double *)malloc(sizeof(double) * (size_t)V);
        double *u_acc = (double *)malloc(sizeof(double) * (size_t)(K + 1));
        double *u_res = (double *)malloc(sizeof(double) * (size_t)(K + 1));
#pragma omp for schedule(dynamic, 1)
        for (int64_t b = 0; b < B; ++b) {
            const int32_t *x = tokens + b * K;
            int L = lengths[b];
            float T = temperature[b];
            int32_t *ot = out_tokens + b * (K + 1);
            double *dg = diag ? diag + b * OR_NDIAG : NULL;
            int bits = row_errors(K, V, x, L, T);
            if (bits) {
                status |= bits;
                out_accept[b] = -1;
                for (int i = 0; i <= K; ++i) ot[i] = -1;
                if (dg) for (int q = 0; q < OR_NDIAG; ++q) dg[q] = NAN;
                continue;
            }
            uint64_t row = row_ids ? (uint64_t)row_ids[b] : (uint64_t)(row_base + b);
            for (int i = 0; i <= K; ++i) {
                u_acc[i] = oracle_uniform(seed, row, (uint32_t)i, 0);
                u_res[i] = oracle_uniform(seed, row, (uint32_t)i, 1);
            }
            vec_t zr = vec_at(zt, dtype, b * (K + 1), V);
            const void *zdr = zd ? vec_at(zd, dtype, b * K, V).p : NULL;
            out_accept[b] = verify_row(zr, zdr, dtype, K, V, x, L, (double)T,
                                       u_acc, u_res, ot, dg, work);
        }
        free(work); free(u_acc); free(u_res);
    }
    return status;
}

/* ---------------------------------------------------------------------------
 * Tie windows: every outcome the rule allows when floating point may move
 * each decision by a small amount.
 *
 * The fp32 kernels and this fp64 oracle can legitimately disagree on a
 * decision that sits within rounding of its threshold.  Two kinds exist:
 *  - an accept test with |u_i - min(1, ratio_i)| < w_acc, which either side
 *    may take as accept or reject;
 *  - a final draw whose target t = u * R lies within w_cdf * R of a CDF
 *    boundary, where either side may land on a neighbouring token.
 * Instead of excluding such rows, this function lists every outcome that
 * decisions inside those windows can reach, so that a result can be checked
 * to be one of them.
 *
 * Per row (T > 0), the tested positions are walked in order exactly as in
 * verify_row: a position whose test lies inside the accept window can end
 * the row there (a rejection) or let it go on (an acceptance); a position
 * outside the window takes its own decision; a clear rejection ends the
 * walk; reaching L leaves the bonus.  For every reachable accepted length a
 * the final draw is made as in verify_row (residual max(0, p_a - q_a), the
 * p_a fallback when that is zero, or p_L for the bonus) at three targets:
 * u, max(0, u - w_cdf) and u + w_cdf (scaled by R), which give y, lo and hi.
 * The CDF is monotone in the target, so every token a draw inside the window
 * can return lies in [lo, hi].  Greedy rows (T == 0) have one outcome, as in
 * verify_row, with lo = hi = y: their decisions are exact comparisons.
 *
 * alt [B, K+1, 4] int32 receives (a, y, lo, hi) per reachable a in
 * increasing a, then rows of -1.  Invalid rows get -1 everywhere and their
 * status bits, as in oracle_verify.  With w_acc = w_cdf = 0 the list holds
 * the single outcome of oracle_verify.
 * ------------------------------------------------------------------------- */
#define OR_NALT 4

/* Draw weights of the final token at position j into r[0..V): residual
 * max(0, p_j - q_j) after a rejection at j < L (p_j when that has no mass),
 * p_L when every draft survived (j == L).  Returns 1 if the zero-residual
 * fallback was taken. */
static int draw_weights(vec_t zt_row, const void *zd_base, int dtype, int V, int j, int L,
                        const int32_t *x, double T, double *r)
{
    vec_t zt = vec_at(zt_row.p, dtype, j, V);
    double mt, st;
    softmax_stats(zt, V, T, &mt, &st);
    if (j == L) {
        for (int v = 0; v < V; ++v) r[v] = exp((zval(zt, v) - mt) / T) / st;
        return 0;
    }
    double md = 0.0, sd = 1.0;
    vec_t zd = { NULL, dtype };
    if (zd_base) {
        zd = vec_at(zd_base, dtype, j, V);
        softmax_stats(zd, V, T, &md, &sd);
    }
    double R = 0.0;
    for (int v = 0; v < V; ++v) {
        double p = exp((zval(zt, v) - mt) / T) / st;
        double q = zd_base ? exp((zval(zd, v) - md) / T) / sd : (v == x[j] ? 1.0 : 0.0);
        r[v] = p - q > 0.0 ? p - q : 0.0;
        R += r[v];
    }
    if (R == 0.0) {
        for (int v = 0; v < V; ++v) r[v] = exp((zval(zt, v) - mt) / T) / st;
        return 1;
    }
    return 0;
}

static void verify_row_window(vec_t zt_row, const void *zd_base, int dtype, int K, int V,
                              const int32_t *x, int L, double T, const double *u_acc,
                              const double *u_res, double w_acc, double w_cdf,
                              int32_t *alt, double *work)
{
    for (int q = 0; q < (K + 1) * OR_NALT; ++q) alt[q] = -1;
    if (T == 0.0) {
        int j = L;
        for (int i = 0; i < L; ++i)
            if (x[i] != argmax_first(vec_at(zt_row.p, dtype, i, V), V)) { j = i; break; }
        int y = argmax_first(vec_at(zt_row.p, dtype, j, V), V);
        alt[0] = j; alt[1] = y; alt[2] = y; alt[3] = y;
        return;
    }
    int n = 0;
    int ends[OR_MAX_K + 1];
    int stopped = 0;
    for (int i = 0; i < L; ++i) {
        vec_t zt = vec_at(zt_row.p, dtype, i, V);
        double mt, st;
        softmax_stats(zt, V, T, &mt, &st);
        double logp = (zval(zt, x[i]) - mt) / T - log(st);
        double logq = 0.0;
        if (zd_base) {
            vec_t zd = vec_at(zd_base, dtype, i, V);
            double md, sd;
            softmax_stats(zd, V, T, &md, &sd);
            logq = (zval(zd, x[i]) - md) / T - log(sd);
        }
        double acc;
        if (logp == -INFINITY) acc = 0.0;
        else if (logq == -INFINITY) acc = 1.0;
        else acc = logp >= logq ? 1.0 : exp(logp - logq);
        if (fabs(u_acc[i] - acc) < w_acc) {
            ends[n++] = i;          /* may reject here, or accept and go on */
            continue;
        }
        if (u_acc[i] < acc) continue;
        ends[n++] = i;              /* clear rejection: the walk ends */
        stopped = 1;
        break;
    }
    if (!stopped) ends[n++] = L;
    for (int k = 0; k < n; ++k) {
        int j = ends[k];
        draw_weights(zt_row, zd_base, dtype, V, j, L, x, T, work);
        double mg;
        int fb;
        double ulo = u_res[j] - w_cdf;
        if (ulo < 0.0) ulo = 0.0;
        alt[k * OR_NALT + 0] = j;
        alt[k * OR_NALT + 1] = inverse_cdf(work, V, u_res[j], &mg, &fb);
        alt[k * OR_NALT + 2] = inverse_cdf(work, V, ulo, &mg, &fb);
        alt[k * OR_NALT + 3] = inverse_cdf(work, V, u_res[j] + w_cdf, &mg, &fb);
    }
}

int oracle_verify_window(const void *zt, const void *zd, int dtype, int64_t B, int K, int V,
                         const int32_t *tokens, const int32_t *lengths,
                         const float *temperature, uint64_t seed, int64_t row_base,
                         const int64_t *row_ids, double w_acc, double w_cdf, int32_t *alt,
                         int nthreads)
{
    int status = 0;
    if (K > OR_MAX_K) return -1;
#ifdef _OPENMP
    if (nthreads > 0) omp_set_num_threads(nthreads);
#else
    (void)nthreads;
#endif
#pragma omp parallel reduction(| : status)
    {
        double *work = (double *)malloc(sizeof(double) * (size_t)V);
        double *u_acc = (double *)malloc(sizeof(double) * (size_t)(K + 1));
        double *u_res = (double *)malloc(sizeof(double) * (size_t)(K + 1));
#pragma omp for schedule(dynamic, 1)
        for (int64_t b = 0; b < B; ++b) {
            const int32_t *x = tokens + b * K;
            int L = lengths[b];
            float T = temperature[b];
            int32_t *ab = alt + b * (int64_t)(K + 1) * OR_NALT;
            int bits = row_errors(K, V, x, L, T);
            if (bits) {
                status |= bits;
                for (int q = 0; q < (K + 1) * OR_NALT; ++q) ab[q] = -1;
                continue;
            }
            uint64_t row = row_ids ? (uint64_t)row_ids[b] : (uint64_t)(row_base + b);
            for (int i = 0; i <= K; ++i) {
                u_acc[i] = oracle_uniform(seed, row, (uint32_t)i, 0);
                u_res[i] = oracle_uniform(seed, row, (uint32_t)i, 1);
            }
            vec_t zr = vec_at(zt, dtype, b * (K + 1), V);
            const void *zdr = zd ? vec_at(zd, dtype, b * K, V).p : NULL;
            verify_row_window(zr, zdr, dtype, K, V, x, L, (double)T, u_acc, u_res, w_acc,
                              w_cdf, ab, work);
        }
        free(work); free(u_acc); free(u_res);
    }
    return status;
}

/* Single row with fp64 logits and injected uniforms (for the pins). */
int oracle_verify_window_row_u(const double *zt, const double *zd, int K, int V,
                               const int32_t *x, int L, double T, const double *u_acc,
                               const double *u_res, double w_acc, double w_cdf, int32_t *alt)
{
    if (K < 0 || K > OR_MAX_K || V <= 0 || L < 0 || L > K || !(T >= 0.0)) return -1;
    for (int i = 0; i < L; ++i) if (x[i] < 0 || x[i] >= V) return -1;
    double *work = (double *)malloc(sizeof(double) * (size_t)V);
    if (!work) return -1;
    vec_t zr = { zt, OR_F64 };
    verify_row_window(zr, zd, OR_F64, K, V, x, L, T, u_acc, u_res, w_acc, w_cdf, alt, work);
    free(work);
    return 0;
}

/* Normaliser export: for every vector of a [n, V] array, m and Sigma at the
 * given per-vector temperature (T == 0: m only, Sigma = 1) and the argmax. */
void oracle_stats_batch(const void *z, int dtype, int64_t n, int V, const float *T,
                        double *m, double *sum, int32_t *amax, int nthreads)
{
#ifdef _OPENMP
    if (nthreads > 0) omp_set_num_threads(nthreads);
#else
    (void)nthreads;
#endif
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t k = 0; k < n; ++k)
        oracle_vector_stats(vec_at(z, dtype, k, V).p, dtype, V, (double)T[k],
                            &m[k], &sum[k], &amax[k]);
}

/* ---------------------------------------------------------------------------
 * Schedule [P1 "Verify smarter"; P2; P4 Ch.7 "Confidence-Scheduled
 * Verification"; P5]: prefix survival S_i = prod_{j<=i} c_j along the block,
 * verify length L = the largest i with S_i >= tau (S_0 = 1, so L = 0 when
 * even the first draft falls below tau).  A NaN confidence counts as 0 and
 * confidences are clamped to [0,1], which keeps S non-increasing.
 * S_out [B,K] (nullable) receives S_1..S_K; the return value is the
 * smallest |S_i - tau| over the block (for tie accounting).
 * ------------------------------------------------------------------------- */
double oracle_schedule(const float *conf, int64_t B, int K, double tau,
                       int32_t *lengths, double *S_out)
{
    double closest = INFINITY;
    for (int64_t b = 0; b < B; ++b) {
        double S = 1.0;
        int L = 0;
        for (int i = 1; i <= K; ++i) {
            double c = (double)conf[b * K + (i - 1)];
            if (isnan(c)) c = 0.0;
            if (c < 0.0) c = 0.0;
            if (c > 1.0) c = 1.0;
            S = S * c;
            if (S_out) S_out[b * K + (i - 1)] = S;
            if (fabs(S - tau) < closest) closest = fabs(S - tau);
            if (S >= tau) L = i;
        }
        lengths[b] = L;
    }
    return closest;
}

int oracle_ndiag(void) { return OR_NDIAG; }

/* ---------------------------------------------------------------------------
 * Hardware-aware admission [P1 "What DSpark adds", item "2. Verify
 * smarter"; P3 "Under the hood"; P4 Ch.7 "Hardware-Aware Scheduling"]: the
 * verification rate (steps per second) is measured once per verify batch
 * size; at each step the candidate draft tokens of all rows are ranked by
 * prefix survival and taken one by one while the expected accepted tokens,
 * multiplied by the measured rate at the resulting batch size, still grows.
 *
 * Reading: row b always verifies its final position, so the batch holds
 * n = B + k tokens after k admissions; expected emitted tokens are
 * E(k) = B + (sum of the admitted S); f(k) = E(k) * speed[n]; candidate k+1
 * is admitted iff n + 1 is inside the table and f(k+1) > f(k).  Candidates
 * are ordered by S descending, ties by (row, position) ascending, so the
 * admitted candidates of a row form a prefix.  S is the fp64 running product
 * of the clamped confidences (NaN -> 0), as in oracle_schedule.
 * Outputs: lengths[b] = admitted candidates of row b; *tau = S of the last
 * admitted candidate (+inf if none); returns k.
 * ------------------------------------------------------------------------- */
typedef struct { double s; int idx; } cand_t;

static int cand_cmp(const void *a, const void *b)
{
    const cand_t *x = (const cand_t *)a, *y = (const cand_t *)b;
    if (x->s > y->s) return -1;
    if (x->s < y->s) return 1;
    return (x->idx > y->idx) - (x->idx < y->idx);
}

int oracle_schedule_admit(const float *conf, int B, int K, const float *speed, int n_speed,
                          int32_t *lengths, double *tau, double *fvals /* [B*K+1] nullable */)
{
    int n = B * K;
    cand_t *c = (cand_t *)malloc(sizeof(cand_t) * (size_t)(n > 0 ? n : 1));
    for (int b = 0; b < B; ++b) {
        double S = 1.0;
        for (int i = 1; i <= K; ++i) {
            double ci = (double)conf[b * K + (i - 1)];
            if (isnan(ci)) ci = 0.0;
            if (ci < 0.0) ci = 0.0;
            if (ci > 1.0) ci = 1.0;
            S = S * ci;
            c[b * K + (i - 1)].s = S;
            c[b * K + (i - 1)].idx = b * K + (i - 1);
        }
        lengths[b] = 0;
    }
    qsort(c, (size_t)n, sizeof(cand_t), cand_cmp);
    double E = (double)B;
    double f = (B < n_speed) ? E * (double)speed[B] : -INFINITY;
    if (fvals) fvals[0] = f;
    int k = 0;
    while (k < n && B + k + 1 < n_speed) {
        double E2 = E + c[k].s;
        double f2 = E2 * (double)speed[B + k + 1];
        if (fvals) fvals[k + 1] = f2;
        if (!(f2 > f)) break;
        E = E2;
        f = f2;
        lengths[c[k].idx / K] += 1;
        ++k;
    }
    *tau = k > 0 ? c[k - 1].s : INFINITY;
    free(c);
    return k;
}

/* ------------------------------------------------------------------------
 * Per-position temperature scaling of the confidence head.
 *
 * umans.ai, "DeepSeek V4 Pro DSpark: the model isn't ready, the
 * architecture is", section "What DSpark adds", item "2. Verify smarter":
 * the head's raw confidences are overconfident (3-8% expected calibration
 * error), and dividing each position's logit by its own temperature,
 * chosen on blocks kept aside from training, lowers that to about 1%.  zhichai.net DSpark topic, "Under the hood": the head
 * is calibrated by Sequential Temperature Scaling.
 *
 * Held-out data: N draft blocks, the head's logits l[n, i] (confidence =
 * sigmoid(l)) for positions i = 0..K-1, and the accepted length a[n] in
 * [0, K] seen when the block was verified (a[n] < 0 skips the block).  The
 * head predicts survival given that every earlier position survived, so
 * position i of block n is observed iff i <= a[n], and survived iff
 * i < a[n]: each position is fitted on the blocks that reached it.
 *
 * T_i minimises the binary negative log-likelihood of the observed outcomes
 * at position i under confidence sigmoid(l / T).  With beta = 1/T and
 * s = +1 (survived) or -1,
 *     NLL(beta)  = sum log(1 + exp(-s beta l))           (convex in beta)
 *     NLL'(beta) = sum -s l sigmoid(-s beta l)           (non-decreasing)
 * The minimiser over [1/tmax, 1/tmin] is the end point where NLL' does not
 * change sign there, else the root of NLL' found by bisection (80
 * halvings, past fp64 resolution).  No observed sample, or NLL' zero at both
 * ends (every observed l is 0), gives T = 1.
 *
 * ECE over every observed (n, i), 15 equal-width confidence bins (the last
 * one closed): ECE = sum over bins |sum (y - conf)| / (observed count), for
 * conf = sigmoid(l) (ece[0]) and conf = sigmoid(l / T_i) (ece[1]).
 * Returns the number of observed (n, i), or -1 on bad arguments.
 * ------------------------------------------------------------------------ */
static double sts_sigmoid(double x)
{
    if (x >= 0.0) return 1.0 / (1.0 + exp(-x));
    double e = exp(x);
    return e / (1.0 + e);
}

static double sts_deriv(const float *l, const int32_t *a, int N, int K, int i, double beta,
                        long *count)
{
    double g = 0.0;
    long c = 0;
    for (int n = 0; n < N; ++n) {
        if (a[n] < 0 || i > a[n]) continue;
        double s = (i < a[n]) ? 1.0 : -1.0;
        double x = (double)l[(size_t)n * K + i];
        g += -s * x * sts_sigmoid(-s * beta * x);
        ++c;
    }
    *count = c;
    return g;
}

#define STS_BINS 15

static void sts_ece(const float *l, const int32_t *a, int N, int K, const double *T,
                    double *out)
{
    double diff[STS_BINS];
    long cnt = 0;
    for (int m = 0; m < STS_BINS; ++m) diff[m] = 0.0;
    for (int n = 0; n < N; ++n) {
        if (a[n] < 0) continue;
        for (int i = 0; i < K && i <= a[n]; ++i) {
            double conf = sts_sigmoid((double)l[(size_t)n * K + i] / (T ? T[i] : 1.0));
            int m = (int)(conf * STS_BINS);
            if (m >= STS_BINS) m = STS_BINS - 1;
            diff[m] += ((i < a[n]) ? 1.0 : 0.0) - conf;
            ++cnt;
        }
    }
    double e = 0.0;
    for (int m = 0; m < STS_BINS; ++m) e += fabs(diff[m]);
    *out = cnt > 0 ? e / (double)cnt : 0.0;
}

long oracle_sts_fit(const float *l, const int32_t *a, int N, int K, double tmin, double tmax,
                    double *T, double *ece)
{
    if (!l || !a || !T || N < 0 || K < 1 || !(tmin > 0.0) || !(tmax > tmin)) return -1;
    long total = 0;
    for (int n = 0; n < N; ++n)
        if (a[n] >= 0) total += (a[n] < K ? a[n] + 1 : K);
    #pragma omp parallel for schedule(dynamic, 1)
    for (int i = 0; i < K; ++i) {
        long c = 0;
        const double lo0 = 1.0 / tmax, hi0 = 1.0 / tmin;
        double glo = sts_deriv(l, a, N, K, i, lo0, &c);
        if (c == 0) { T[i] = 1.0; continue; }
        double ghi = sts_deriv(l, a, N, K, i, hi0, &c);
        double beta;
        if (glo == 0.0 && ghi == 0.0) {
            beta = 1.0;
        } else if (glo >= 0.0) {
            beta = lo0;
        } else if (ghi <= 0.0) {
            beta = hi0;
        } else {
            double lo = lo0, hi = hi0;
            for (int it = 0; it < 80; ++it) {
                double mid = 0.5 * (lo + hi);
                if (sts_deriv(l, a, N, K, i, mid, &c) < 0.0) lo = mid; else hi = mid;
            }
            beta = 0.5 * (lo + hi);
        }
        T[i] = 1.0 / beta;
    }
    if (ece) {
        sts_ece(l, a, N, K, NULL, &ece[0]);
        sts_ece(l, a, N, K, T, &ece[1]);
    }
    return total;
}
