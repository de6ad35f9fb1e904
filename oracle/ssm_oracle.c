/*
 * ssm_oracle.c -- plain, slow fp64 CPU reference of the Mamba-2 selective
 * state-space recurrence.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the tests, the package smoke check and the
 * benchmark's CPU-baseline leg may load this library.  It shares no code,
 * header, table or helper with the CUDA path.
 *
 * What it computes (the selective-SSM recurrence as stated in the note
 * "Mamba 与 Nemotron 系列模型深度调研", section "1. Selective SSM 的直觉",
 * and restated for the decode path in "逐行精读 ... modeling_nemotron_h.py",
 * section "Decode 阶段"):
 *
 *     h[p,n] <- exp(dt_t * A_h) * h[p,n] + dt_t * x_t[h,p] * B_t[g,n]
 *     y_t[h,p] = sum over n of h[p,n] * C_t[g,n]  +  D_h * x_t[h,p]
 *
 * per token t, per head h, for every (p, n) element of the [head_dim, d_state]
 * state, where A, D are per-head scalars, dt is per (token, head), x is per
 * (token, head, p) and B, C are per (token, group, n), the group of head h
 * being g(h) = h / (nheads / ngroups).  The output reads the UPDATED state.
 *
 * The prefill ("chunked SSD scan") reaches exactly this result in exact
 * arithmetic, so the oracle is the plain sequential definition: one token at a
 * time, in order, for every (sequence, head).  There is no chunking, blocking
 * or reordering here.  Everything is double precision; inputs arrive already
 * widened to double (bf16 and fp32 values convert exactly).
 */
#include <math.h>
#include <stddef.h>
#include <stdint.h>

#ifdef _OPENMP
#include <omp.h>
#endif

/* Status codes of this library (independent of the CUDA library's). */
enum { ORACLE_OK = 0, ORACLE_BAD_ARG = 1 };

int oracle_num_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

void oracle_set_num_threads(int n)
{
#ifdef _OPENMP
    if (n > 0) omp_set_num_threads(n);
#else
    (void)n;
#endif
}

/*
 * One token of the recurrence for one head.
 *   h    [P*N]  state of this (sequence, head), updated in place
 *   xv   [P]    x of this token and head
 *   bv   [N]    B of this token, in the head's group
 *   cv   [N]    C of this token, in the head's group
 *   yv   [P]    output of this token and head
 */
static void recurrence_step(int P, int N, double dt, double A, double D,
                            const double *xv, const double *bv,
                            const double *cv, double *h, double *yv)
{
    const double decay = exp(A * dt);
    for (int p = 0; p < P; ++p) {
        double *row = h + (size_t)p * N;
        double acc = 0.0;
        for (int n = 0; n < N; ++n) {
            row[n] = row[n] * decay + bv[n] * dt * xv[p];
            acc += row[n] * cv[n];
        }
        yv[p] = acc + D * xv[p];
    }
}

/*
 * Sequential scan over packed sequences.
 *
 *   nseq          number of sequences
 *   cu_seqlens    [nseq+1] token offsets (cu[0] = 0, non-decreasing)
 *   H, P, N, G    heads, head_dim, d_state, groups (H % G == 0)
 *   x   [T,H,P]   dt [T,H]   A [H]   B [T,G,N]   C [T,G,N]   D [H] or NULL
 *   state [nseq,H,P,N]  in: initial state, out: final state
 *   y   [T,H,P]   output
 *
 * Returns ORACLE_OK or ORACLE_BAD_ARG.
 */
int oracle_scan(int nseq, const int64_t *cu_seqlens, int H, int P, int N, int G,
                const double *x, const double *dt, const double *A,
                const double *B, const double *C, const double *D,
                double *state, double *y)
{
    if (nseq < 0 || H <= 0 || P <= 0 || N <= 0 || G <= 0 || H % G != 0)
        return ORACLE_BAD_ARG;
    if (nseq == 0) return ORACLE_OK;
    if (!cu_seqlens || !A || !state) return ORACLE_BAD_ARG;
    if (cu_seqlens[0] != 0) return ORACLE_BAD_ARG;
    for (int s = 0; s < nseq; ++s)
        if (cu_seqlens[s + 1] < cu_seqlens[s]) return ORACLE_BAD_ARG;
    if (cu_seqlens[nseq] > 0 && (!x || !dt || !B || !C || !y))
        return ORACLE_BAD_ARG;

    const int heads_per_group = H / G;
    const long work = (long)nseq * H;

#pragma omp parallel for schedule(dynamic, 1)
    for (long w = 0; w < work; ++w) {
        const int s = (int)(w / H);
        const int h = (int)(w % H);
        const int g = h / heads_per_group;
        double *hs = state + ((size_t)s * H + h) * (size_t)P * N;
        const double Dh = D ? D[h] : 0.0;
        for (int64_t t = cu_seqlens[s]; t < cu_seqlens[s + 1]; ++t) {
            recurrence_step(P, N, dt[(size_t)t * H + h], A[h], Dh,
                            x + ((size_t)t * H + h) * P,
                            B + ((size_t)t * G + g) * N,
                            C + ((size_t)t * G + g) * N,
                            hs,
                            y + ((size_t)t * H + h) * P);
        }
    }
    return ORACLE_OK;
}

/*
 * Single-token decode update, in place on the state (the decode path of the
 * same recurrence: one token per batch element).
 *
 *   state [batch,H,P,N]  updated in place
 *   x [batch,H,P]  dt [batch,H]  A [H]  B, C [batch,G,N]  D [H] or NULL
 *   y [batch,H,P]
 */
int oracle_state_update(int batch, int H, int P, int N, int G,
                        double *state, const double *x, const double *dt,
                        const double *A, const double *B, const double *C,
                        const double *D, double *y)
{
    if (batch < 0 || H <= 0 || P <= 0 || N <= 0 || G <= 0 || H % G != 0)
        return ORACLE_BAD_ARG;
    if (batch == 0) return ORACLE_OK;
    if (!state || !x || !dt || !A || !B || !C || !y) return ORACLE_BAD_ARG;

    const int heads_per_group = H / G;
    const long work = (long)batch * H;

#pragma omp parallel for schedule(static)
    for (long w = 0; w < work; ++w) {
        const int b = (int)(w / H);
        const int h = (int)(w % H);
        const int g = h / heads_per_group;
        recurrence_step(P, N, dt[(size_t)b * H + h], A[h], D ? D[h] : 0.0,
                        x + ((size_t)b * H + h) * P,
                        B + ((size_t)b * G + g) * N,
                        C + ((size_t)b * G + g) * N,
                        state + ((size_t)b * H + h) * (size_t)P * N,
                        y + ((size_t)b * H + h) * P);
    }
    return ORACLE_OK;
}

/*
 * Causal depthwise conv1d with optional SiLU, over packed sequences in the
 * channels-last layout ("Depthwise SiLU 卷积" of the MAX nemotron_h article,
 * section 5.4 item 2; causal_conv1d_fn / causal_conv1d_update and the conv
 * state of the modeling_nemotron_h.py walk-through, "Prefill 阶段" /
 * "Decode 阶段").  For channel c, width K, token t of a sequence:
 *
 *   pre[t][c] = bias[c] + sum_{k=0}^{K-1} w[c][k] * in[t - (K-1) + k][c]
 *   y[t][c]   = act(pre[t][c]),  act = identity or SiLU (v / (1 + exp(-v)))
 *
 * where in[t'] for t' < 0 is taken from the sequence's conv state
 * (state[s][c][K-1+t'], its K-1 most recent earlier inputs, oldest first) or
 * zero when no state is given.  Afterwards the state holds the K-1 most
 * recent inputs (earlier state entries shift in when the sequence is short).
 *
 *   x [T][dim], w [dim][K], bias [dim] or NULL, state [nseq][dim][K-1] or
 *   NULL (in/out), y [T][dim].
 */
static double conv_act(double v, int act)
{
    return act ? v / (1.0 + exp(-v)) : v;
}

int oracle_causal_conv1d(int nseq, const int64_t *cu_seqlens, int dim, int K,
                         const double *x, const double *w, const double *bias, int act,
                         double *state, double *y)
{
    if (nseq < 0 || dim <= 0 || K < 1) return ORACLE_BAD_ARG;
    if (nseq == 0) return ORACLE_OK;
    if (!cu_seqlens || !w) return ORACLE_BAD_ARG;

#pragma omp parallel for schedule(static)
    for (long sc = 0; sc < (long)nseq * dim; ++sc) {
        const int s = (int)(sc / dim), c = (int)(sc % dim);
        const int64_t t0 = cu_seqlens[s], t1 = cu_seqlens[s + 1];
        double *st = state ? state + ((size_t)s * dim + c) * (size_t)(K - 1) : NULL;
        for (int64_t t = t0; t < t1; ++t) {
            double acc = bias ? bias[c] : 0.0;
            for (int k = 0; k < K; ++k) {
                const int64_t src = t - (K - 1) + k;        /* absolute token */
                double v;
                if (src >= t0) v = x[(size_t)src * dim + c];
                else if (st) v = st[(K - 1) + (src - t0)];   /* src - t0 in [-(K-1), -1] */
                else v = 0.0;
                acc += w[(size_t)c * K + k] * v;
            }
            y[(size_t)t * dim + c] = conv_act(acc, act);
        }
        if (st && K > 1) {
            /* new state: the K-1 most recent inputs (old state entries first) */
            double win[64];
            const int64_t L = t1 - t0;
            for (int k = 0; k < K - 1; ++k) {
                const int64_t src = L - (K - 1) + k;         /* relative to t0 */
                win[k] = src >= 0 ? x[(size_t)(t0 + src) * dim + c] : st[(K - 1) + src];
            }
            for (int k = 0; k < K - 1; ++k) st[k] = win[k];
        }
    }
    return ORACLE_OK;
}

/*
 * Philox-4x32 (Salmon, Moraes, Dror, Shaw, "Parallel random numbers: as easy
 * as 1, 2, 3", SC'11), written from the paper's description: `rounds` rounds
 * of the 4x32 S-box -- the two 32x32 -> 64-bit products of counter words 0
 * and 2 with the multipliers 0xD2511F53 and 0xCD9E8D57, whose high halves are
 * xored with counter words 1 and 3 and the two key words -- with the key
 * bumped by the Weyl constants 0x9E3779B9 and 0xBB67AE85 after each round.
 */
void oracle_philox4x32(const uint32_t ctr[4], const uint32_t key[2], int rounds, uint32_t out[4])
{
    uint32_t c0 = ctr[0], c1 = ctr[1], c2 = ctr[2], c3 = ctr[3];
    uint32_t k0 = key[0], k1 = key[1];
    for (int r = 0; r < rounds; ++r) {
        const uint64_t p0 = (uint64_t)0xD2511F53u * c0;
        const uint64_t p1 = (uint64_t)0xCD9E8D57u * c2;
        const uint32_t n0 = (uint32_t)(p1 >> 32) ^ c1 ^ k0;
        const uint32_t n1 = (uint32_t)p1;
        const uint32_t n2 = (uint32_t)(p0 >> 32) ^ c3 ^ k1;
        const uint32_t n3 = (uint32_t)p0;
        c0 = n0; c1 = n1; c2 = n2; c3 = n3;
        k0 += 0x9E3779B9u;
        k1 += 0xBB67AE85u;
    }
    out[0] = c0; out[1] = c1; out[2] = c2; out[3] = c3;
}

/*
 * Stochastic rounding of an fp32 value to fp16, from its definition: with
 * lo the fp16 neighbour toward zero and s the fp16 spacing there (2^(k-10) in
 * the binade [2^k, 2^(k+1)) of the normal range, 2^-24 below 2^-14), the
 * fraction f = (|v| - lo) / s is in [0, 1); the result moves to lo + s iff
 * u < f with u = r16 / 2^16 for the element's 16 random bits r16.
 * |v| >= 65504 gives +-65504.
 */
double oracle_sr_fp16(float vf, uint32_t r16)
{
    const double v = vf;
    if (v != v) return v;
    const double a = fabs(v);
    if (a >= 65504.0) return copysign(65504.0, v);
    double s;
    if (a >= ldexp(1.0, -14)) {
        int e;
        frexp(a, &e);                 /* a in [2^(e-1), 2^e) */
        s = ldexp(1.0, e - 1 - 10);
    } else {
        s = ldexp(1.0, -24);
    }
    const double lo = floor(a / s) * s;
    const double f = (a - lo) / s;
    const double u = (double)(r16 & 0xFFFFu) / 65536.0;
    double m = lo + (u < f ? s : 0.0);
    if (m > 65504.0) m = 65504.0;
    return copysign(m, v);
}

/*
 * Round n state values to fp16 as they are written to a pool: value i is
 * pool element e = elem[i]; its 16 random bits are half (e % 2, low half
 * first) of word (e % 8) / 2 of Philox(counter = (e / 8 low, e / 8 high,
 * offset low, offset high), key = (seed low, seed high)).  The decision is
 * taken on the value rounded to fp32 (the precision the state is computed in).
 */
void oracle_round_state_f16(long n, const double *v, const int64_t *elem, uint64_t seed,
                            uint64_t offset, int rounds, double *out)
{
#pragma omp parallel for schedule(static)
    for (long i = 0; i < n; ++i) {
        const uint64_t e = (uint64_t)elem[i];
        const uint64_t q = e >> 3;
        const uint32_t ctr[4] = {(uint32_t)q, (uint32_t)(q >> 32), (uint32_t)offset,
                                 (uint32_t)(offset >> 32)};
        const uint32_t key[2] = {(uint32_t)seed, (uint32_t)(seed >> 32)};
        uint32_t w[4];
        oracle_philox4x32(ctr, key, rounds, w);
        const uint32_t word = w[(e & 7) >> 1];
        out[i] = oracle_sr_fp16((float)v[i], (e & 1) ? (word >> 16) : (word & 0xFFFFu));
    }
}
