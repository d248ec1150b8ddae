/*
 * Lightning attention: plain fp64 CPU oracle.
 *
 * TEST INFRASTRUCTURE ONLY. Nothing in the product path may include, link or
 * call this file; only the tests, the package smoke check and the benchmark's
 * CPU-baseline leg use it. It shares no code, header, table or constant with
 * the CUDA library.
 *
 * What it computes (per head problem, rows contiguous [N][d], d_k = d_v = d):
 *
 *   O_i     = sum_{j <= i} lam^(i-j) (q_i . k_j) v_j                     (1)
 *   state   = sum_j lam^(N-1-j) k_j^T v_j        state[a][b], a: key, b: value
 *
 * Sources:
 *   - "MiniMax-01: Scaling Foundation Models with Lightning Attention |
 *     Summary", section 2.2 (Linear Attention): causal linear attention
 *     computed without the length-by-length matrix, with a cumulative
 *     key-value state; tiles combine an intra-tile masked product with the
 *     accumulated state of the preceding tiles. Normalization, SiLU and gating
 *     are left out of the derivation there, and are left out here.
 *   - The per-head exponential decay lam_h = exp(-s_h) is part of the
 *     operator's definition as this library states it (the summary page does
 *     not mention decay); the caller passes lam per head.
 *
 * Every function below evaluates a plain definition, with no blocking, tiling
 * or reordering: the quadratic forms loop over (i, j) directly, and the
 * recurrences step one token at a time. lam^m is taken from a table filled
 * with pow(lam, m), so that lam = 1/2 gives exact powers of two.
 *
 * A "problem" is one (sequence, head) pair. Batched entry points take arrays
 * of per-problem row offsets (in rows of d elements), lengths, decays and
 * state offsets (in d*d blocks, -1 = no state), and run problems in parallel
 * with OpenMP.
 */
#include <math.h>
#include <stdlib.h>
#include <string.h>

static double* pow_table(double lam, long n)
{
    double* t = (double*)malloc(sizeof(double) * (size_t)(n > 0 ? n : 1));
    for (long m = 0; m < n; ++m) t[m] = pow(lam, (double)m);
    return t;
}

static double dot(const double* a, const double* b, long d)
{
    double s = 0.0;
    for (long c = 0; c < d; ++c) s += a[c] * b[c];
    return s;
}

/* (1) for one problem, by the quadratic form. state may be NULL. */
void oracle_forward_one(const double* q, const double* k, const double* v,
                        double* o, double* state, long N, long d, double lam)
{
    double* pw = pow_table(lam, N);
    for (long i = 0; i < N; ++i) {
        double* oi = o + i * d;
        for (long c = 0; c < d; ++c) oi[c] = 0.0;
        for (long j = 0; j <= i; ++j) {
            double w = pw[i - j] * dot(q + i * d, k + j * d, d);
            const double* vj = v + j * d;
            for (long c = 0; c < d; ++c) oi[c] += w * vj[c];
        }
    }
    if (state) {
        for (long a = 0; a < d * d; ++a) state[a] = 0.0;
        for (long j = 0; j < N; ++j) {
            double w = pw[N - 1 - j];
            for (long a = 0; a < d; ++a) {
                double ka = w * k[j * d + a];
                for (long b = 0; b < d; ++b) state[a * d + b] += ka * v[j * d + b];
            }
        }
    }
    free(pw);
}

/* (1) continued from an incoming state S_in: the state of a prefix of tokens
 * that come before token 0 (a cached prefix, "MiniMax-01: Scaling Foundation
 * Models with Lightning Attention | Summary", section 3: inference inputs
 * whose earlier segments were already computed). Every prefix token j < 0
 * enters (1) through S_in = sum_{j<0} lam^(-1-j) k_j^T v_j, so
 *
 *   O_i   = lam^(i+1) q_i S_in + sum_{0 <= j <= i} lam^(i-j) (q_i . k_j) v_j
 *   state = lam^N S_in + sum_{0 <= j < N} lam^(N-1-j) k_j^T v_j
 *
 * The second terms are (1) over the tokens 0..N-1; the first are added here.
 * state may be NULL; N may be 0 (then state = S_in). */
void oracle_forward_from_state_one(const double* q, const double* k, const double* v,
                                   const double* state_in, double* o, double* state, long N,
                                   long d, double lam)
{
    oracle_forward_one(q, k, v, o, state, N, d, lam);
    for (long i = 0; i < N; ++i) {
        double w = pow(lam, (double)(i + 1));
        for (long b = 0; b < d; ++b) {
            double s = 0.0;
            for (long a = 0; a < d; ++a) s += q[i * d + a] * state_in[a * d + b];
            o[i * d + b] += w * s;
        }
    }
    if (state) {
        double w = pow(lam, (double)N);
        for (long a = 0; a < d * d; ++a) state[a] += w * state_in[a];
    }
}

/* (1) evaluated only at the given rows of one problem: out[r] = O_{rows[r]}. */
void oracle_forward_rows(const double* q, const double* k, const double* v,
                         const long* rows, long nrows, double* out, long d, double lam)
{
    #pragma omp parallel for schedule(dynamic)
    for (long r = 0; r < nrows; ++r) {
        long i = rows[r];
        double* oi = out + r * d;
        for (long c = 0; c < d; ++c) oi[c] = 0.0;
        for (long j = 0; j <= i; ++j) {
            double w = pow(lam, (double)(i - j)) * dot(q + i * d, k + j * d, d);
            const double* vj = v + j * d;
            for (long c = 0; c < d; ++c) oi[c] += w * vj[c];
        }
    }
}

/* Token recurrence, written independently of (1):
 *   S_t = lam S_{t-1} + k_t^T v_t,   o_t = q_t S_t   (S_{-1} = state_in or 0).
 * reverse != 0 runs it from the last token to the first instead:
 *   R_t = lam R_{t+1} + k_t^T v_t,   o_t = q_t R_t. */
void oracle_recurrence_one(const double* q, const double* k, const double* v,
                           double* o, const double* state_in, double* state_out,
                           long N, long d, double lam, int reverse)
{
    double* S = (double*)calloc((size_t)(d * d), sizeof(double));
    if (state_in) memcpy(S, state_in, sizeof(double) * (size_t)(d * d));
    for (long step = 0; step < N; ++step) {
        long t = reverse ? (N - 1 - step) : step;
        const double* kt = k + t * d;
        const double* vt = v + t * d;
        for (long a = 0; a < d; ++a)
            for (long b = 0; b < d; ++b)
                S[a * d + b] = lam * S[a * d + b] + kt[a] * vt[b];
        if (o) {
            const double* qt = q + t * d;
            double* ot = o + t * d;
            for (long b = 0; b < d; ++b) {
                double s = 0.0;
                for (long a = 0; a < d; ++a) s += qt[a] * S[a * d + b];
                ot[b] = s;
            }
        }
    }
    if (state_out) memcpy(state_out, S, sizeof(double) * (size_t)(d * d));
    free(S);
}

/* One decode step per problem (state updated in place, then read out):
 *   S <- lam S + k^T v,   o = q S. */
void oracle_decode(const double* q, const double* k, const double* v, const double* lam,
                   double* state, double* o, long nprob, long d)
{
    #pragma omp parallel for schedule(static)
    for (long p = 0; p < nprob; ++p) {
        double* S = state + p * d * d;
        const double* qp = q + p * d;
        const double* kp = k + p * d;
        const double* vp = v + p * d;
        for (long a = 0; a < d; ++a)
            for (long b = 0; b < d; ++b)
                S[a * d + b] = lam[p] * S[a * d + b] + kp[a] * vp[b];
        for (long b = 0; b < d; ++b) {
            double s = 0.0;
            for (long a = 0; a < d; ++a) s += qp[a] * S[a * d + b];
            o[p * d + b] = s;
        }
    }
}

/* Incoming state of chunk r of a sequence cut into R consecutive chunks, from
 * the chunks' local states ("MiniMax-01: Scaling Foundation Models with
 * Lightning Attention | Summary", section 3.2, LASP+: every partition
 * summarizes its keys and values locally, the summaries are gathered, and
 * each partition builds its global prefix from them). Chunk p of length n_p
 * has local state S_p (the state of its tokens alone) and decay alpha_p =
 * lam^n_p over its whole length; the state after chunks 0..r-1 is
 *
 *   S_in(r) = sum_{p<r} ( prod_{p<q<r} alpha_q ) S_p
 *
 * evaluated here as that sum, with the product taken as lam raised to the
 * total length of the chunks strictly between p and r.
 * states: [R][nprob][d][d]; lam: [nprob]; lens: [R]; out: [nprob][d][d]. */
void oracle_state_prefix(const double* states, const double* lam, const long* lens, long R,
                         long r, long nprob, long d, double* out)
{
    for (long x = 0; x < nprob; ++x) {
        double* o = out + x * d * d;
        for (long e = 0; e < d * d; ++e) o[e] = 0.0;
        for (long p = 0; p < r; ++p) {
            long between = 0;
            for (long q = p + 1; q < r; ++q) between += lens[q];
            double w = pow(lam[x], (double)between);
            const double* S = states + (p * nprob + x) * d * d;
            for (long e = 0; e < d * d; ++e) o[e] += w * S[e];
        }
    }
    (void)R;
}

/* Output normalization and gate after the operator ("MiniMax-01: Scaling
 * Foundation Models with Lightning Attention | Summary", section 2.2: the
 * linear-attention output passes through Norm, and the blocks use gating; the
 * page gives neither form). Read as an RMS normalization over all H*d
 * features of a token followed by a sigmoid gate:
 *
 *   r_{b,n}         = 1 / sqrt( (1/(H d)) sum_{h,c} O[b][h][n][c]^2 + eps )
 *   Y[b][n][h d + c] = w[h d + c] * O[b][h][n][c] * r_{b,n} * sigmoid(G[b][n][h d + c])
 *
 * O is head-major [B][H][N][d]; G, w and Y are token-major [B][N][H d]. */
void oracle_norm_gate(const double* o, const double* g, const double* w, double eps,
                      double* y, long B, long H, long N, long d)
{
    #pragma omp parallel for schedule(static)
    for (long t = 0; t < B * N; ++t) {
        long b = t / N, n = t % N;
        double ss = 0.0;
        for (long h = 0; h < H; ++h)
            for (long c = 0; c < d; ++c) {
                double x = o[((b * H + h) * N + n) * d + c];
                ss += x * x;
            }
        double r = 1.0 / sqrt(ss / (double)(H * d) + eps);
        for (long h = 0; h < H; ++h)
            for (long c = 0; c < d; ++c) {
                long f = h * d + c;
                double x = o[((b * H + h) * N + n) * d + c];
                double gate = 1.0 / (1.0 + exp(-g[t * H * d + f]));
                y[t * H * d + f] = w[f] * x * r * gate;
            }
    }
}

/* Gradients of <dO, O> for (1), each by its own quadratic sum:
 *   dQ_i = sum_{j <= i} lam^(i-j) (dO_i . v_j) k_j
 *   dK_j = sum_{i >= j} lam^(i-j) (dO_i . v_j) q_i
 *   dV_j = sum_{i >= j} lam^(i-j) (q_i . k_j) dO_i */
void oracle_backward_one(const double* dout, const double* q, const double* k, const double* v,
                         double* dq, double* dk, double* dv, long N, long d, double lam)
{
    double* pw = pow_table(lam, N);
    for (long x = 0; x < N * d; ++x) { dq[x] = 0.0; dk[x] = 0.0; dv[x] = 0.0; }
    for (long i = 0; i < N; ++i)
        for (long j = 0; j <= i; ++j) {
            double w = pw[i - j] * dot(dout + i * d, v + j * d, d);
            for (long c = 0; c < d; ++c) dq[i * d + c] += w * k[j * d + c];
        }
    for (long j = 0; j < N; ++j)
        for (long i = j; i < N; ++i) {
            double wk = pw[i - j] * dot(dout + i * d, v + j * d, d);
            double wv = pw[i - j] * dot(q + i * d, k + j * d, d);
            for (long c = 0; c < d; ++c) {
                dk[j * d + c] += wk * q[i * d + c];
                dv[j * d + c] += wv * dout[i * d + c];
            }
        }
    free(pw);
}

/* Batched drivers over problems. *_off are row offsets; st_off in d*d blocks
 * (negative = no state for that problem). */
void oracle_forward(int nprob, const long* row_off, const long* len, const long* st_off,
                    const double* lam, const double* q, const double* k, const double* v,
                    double* o, double* state, long d)
{
    #pragma omp parallel for schedule(dynamic)
    for (int p = 0; p < nprob; ++p) {
        long r = row_off[p] * d;
        double* st = (state && st_off[p] >= 0) ? state + st_off[p] * d * d : NULL;
        if (len[p] == 0) {
            if (st) for (long a = 0; a < d * d; ++a) st[a] = 0.0;
            continue;
        }
        oracle_forward_one(q + r, k + r, v + r, o + r, st, len[p], d, lam[p]);
    }
}

/* Batched (1) from incoming states: state_in and state share st_off. */
void oracle_forward_from_state(int nprob, const long* row_off, const long* len, const long* st_off,
                               const double* lam, const double* q, const double* k,
                               const double* v, const double* state_in, double* o, double* state,
                               long d)
{
    #pragma omp parallel for schedule(dynamic)
    for (int p = 0; p < nprob; ++p) {
        long r = row_off[p] * d;
        const double* si = state_in + st_off[p] * d * d;
        double* st = state ? state + st_off[p] * d * d : NULL;
        oracle_forward_from_state_one(q + r, k + r, v + r, si, o + r, st, len[p], d, lam[p]);
    }
}

void oracle_recurrence(int nprob, const long* row_off, const long* len, const long* st_off,
                       const double* lam, const double* q, const double* k, const double* v,
                       double* o, const double* state_in, double* state_out, long d, int reverse)
{
    #pragma omp parallel for schedule(dynamic)
    for (int p = 0; p < nprob; ++p) {
        long r = row_off[p] * d;
        const double* si = (state_in && st_off[p] >= 0) ? state_in + st_off[p] * d * d : NULL;
        double* so = (state_out && st_off[p] >= 0) ? state_out + st_off[p] * d * d : NULL;
        oracle_recurrence_one(q + r, k + r, v + r, o ? o + r : NULL, si, so, len[p], d, lam[p],
                              reverse);
    }
}

void oracle_backward(int nprob, const long* row_off, const long* len, const double* lam,
                     const double* dout, const double* q, const double* k, const double* v,
                     double* dq, double* dk, double* dv, long d)
{
    #pragma omp parallel for schedule(dynamic)
    for (int p = 0; p < nprob; ++p) {
        long r = row_off[p] * d;
        oracle_backward_one(dout + r, q + r, k + r, v + r, dq + r, dk + r, dv + r, len[p], d,
                            lam[p]);
    }
}
