/*
 * RDA (Raon Delta Attention) core -- plain fp64 CPU oracle.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path may link, load or call
 * this file; only the tests, the smoke check and the CPU-baseline leg of the
 * benchmark do.  It shares no code, header, table or helper with the CUDA path.
 *
 * What it computes (the definition, token by token, per sequence and head):
 *
 *   article "Raon-1 nano: half of a 3.1B model is a lookup table, and a 99M
 *   model keeps one too", section "The other 1.5B: a hybrid built to forget":
 *   the reference recurrence first decays the state, then forms the error
 *   between the value and the state's prediction for the key, then writes that
 *   error with strength beta; a separate write gate rescales the value.
 *
 *   In matrix form (math orientation, S is Dv x Dk, o = S q) this is the gated
 *   delta rule  S_t = a_t S_{t-1} (I - b_t k_t k_t^T) + b_t v_t k_t^T,
 *   o_t = scale * S_t q_t  (the output reads the post-update state).
 *
 *   Readings taken where the pages are silent:
 *     - decay is a scalar per (token, head), passed as log(alpha); the
 *       per-key-channel variant (rda_oracle_forward_channel) takes log(alpha)
 *       per (token, head, key dim) and scales column i of S (key dim i) by
 *       alpha_i: S_t = S_{t-1} diag(alpha_t) (I - b_t k_t k_t^T) + b_t v_t k_t^T,
 *       which is the scalar rule when every channel has the same alpha (the
 *       model card "tiny-random/raon-1-mini", section "Printing the model",
 *       shows decay projections f_a_proj / f_b_proj as wide as heads x key
 *       dims, and the same article names Kimi Delta Attention as what RDA
 *       modifies);
 *     - the write gate gamma multiplies v before the error is formed
 *       (NULL means gamma = 1);
 *     - scale defaults to 1 at the call sites; it multiplies the output only.
 *
 *   State storage (the article's section "The cache is small if the runtime
 *   keeps it small": one fp32 16 x 128 x 128 state per layer): the caller's
 *   buffers hold S transposed, i.e. element [i][j] of a [Dk][Dv] row-major
 *   block is S[j][i].  This oracle keeps S in fp64, math orientation, and
 *   converts at the boundary.
 *
 * Parallelism: OpenMP over independent (sequence, head) units only; within a
 * unit the loop is strictly sequential in t.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#ifdef _OPENMP
#include <omp.h>
#endif

/* One token of the recurrence on an fp64 state S[Dv][Dk] (math orientation).
 * e is scratch of length Dv.  Writes o[j*o_stride] for j < Dv when o != NULL.
 * With la_ch != NULL the decay is per key channel (la_ch[i] for column i) and
 * log_alpha is not used. */
static void rda_token(double *S, int Dk, int Dv,
                      const double *q, const double *k, const double *v,
                      double log_alpha, double beta, double gamma, double scale,
                      double *e, double *o, long o_stride, const double *la_ch)
{
    const double a = exp(log_alpha);
    /* 1. decay the state */
    if (la_ch) {
        for (int j = 0; j < Dv; ++j)
            for (int i = 0; i < Dk; ++i)
                S[(long)j * Dk + i] *= exp(la_ch[i]);
    } else {
    for (int j = 0; j < Dv; ++j)
        for (int i = 0; i < Dk; ++i)
            S[(long)j * Dk + i] *= a;
    }
    /* 2. error between the (gated) value and the decayed state's prediction */
    for (int j = 0; j < Dv; ++j) {
        double pred = 0.0;
        for (int i = 0; i < Dk; ++i)
            pred += S[(long)j * Dk + i] * k[i];
        e[j] = gamma * v[j] - pred;
    }
    /* 3. write the error along k with strength beta */
    for (int j = 0; j < Dv; ++j) {
        const double be = beta * e[j];
        for (int i = 0; i < Dk; ++i)
            S[(long)j * Dk + i] += be * k[i];
    }
    /* 4. read the updated state with q */
    if (o) {
        for (int j = 0; j < Dv; ++j) {
            double acc = 0.0;
            for (int i = 0; i < Dk; ++i)
                acc += S[(long)j * Dk + i] * q[i];
            o[(long)j * o_stride] = scale * acc;
        }
    }
}

static void load_state(double *S, const double *src, int Dk, int Dv)
{
    if (!src) {
        memset(S, 0, sizeof(double) * (size_t)Dk * Dv);
        return;
    }
    for (int i = 0; i < Dk; ++i)
        for (int j = 0; j < Dv; ++j)
            S[(long)j * Dk + i] = src[(long)i * Dv + j];
}

static void store_state(double *dst, const double *S, int Dk, int Dv)
{
    if (!dst) return;
    for (int i = 0; i < Dk; ++i)
        for (int j = 0; j < Dv; ++j)
            dst[(long)i * Dv + j] = S[(long)j * Dk + i];
}

/* Runs one (sequence, head) unit over tokens [t0, t0+len) of arrays laid out as
 * [.., T_axis, H, D] with the given token stride (in elements).  la_ch, when
 * not NULL, is the per-channel log decay [.., T_axis, H, Dk] (log_alpha is then
 * only indexed, never used). */
static void rda_unit(int Dk, int Dv, int H, int h, long t0, long len,
                     const double *q, const double *k, const double *v,
                     const double *log_alpha, const double *beta, const double *gamma,
                     const double *s0, double *sf, double *out, double scale,
                     const double *la_ch)
{
    double *S = (double *)malloc(sizeof(double) * ((size_t)Dk * Dv + Dv));
    double *e = S + (size_t)Dk * Dv;
    load_state(S, s0, Dk, Dv);
    for (long t = t0; t < t0 + len; ++t) {
        const long row = t * H + h;
        rda_token(S, Dk, Dv, q + row * Dk, k + row * Dk, v + row * Dv,
                  log_alpha[row], beta[row], gamma ? gamma[row] : 1.0, scale,
                  e, out ? out + row * Dv : NULL, 1, la_ch ? la_ch + row * Dk : NULL);
    }
    store_state(sf, S, Dk, Dv);
    free(S);
}

/* Fixed-length batch: q,k [B,T,H,Dk]; v,out [B,T,H,Dv]; log_alpha, beta,
 * gamma [B,T,H]; s0, sf [B,H,Dk,Dv] (s0, sf, gamma, out may be NULL). */
int rda_oracle_forward(int B, int T, int H, int Dk, int Dv,
                       const double *q, const double *k, const double *v,
                       const double *log_alpha, const double *beta, const double *gamma,
                       const double *s0, double *sf, double *out, double scale,
                       int num_threads)
{
    if (B < 0 || T < 0 || H <= 0 || Dk <= 0 || Dv <= 0) return 1;
    const long units = (long)B * H;
#ifdef _OPENMP
    if (num_threads > 0) omp_set_num_threads(num_threads);
#else
    (void)num_threads;
#endif
#pragma omp parallel for schedule(dynamic, 1)
    for (long u = 0; u < units; ++u) {
        const long b = u / H;
        const int h = (int)(u % H);
        const long sidx = (b * H + h) * (long)Dk * Dv;
        rda_unit(Dk, Dv, H, h, b * (long)T, T, q, k, v, log_alpha, beta, gamma,
                 s0 ? s0 + sidx : NULL, sf ? sf + sidx : NULL, out, scale, NULL);
    }
    return 0;
}

/* Fixed-length batch with per-key-channel decay: log_alpha_ch [B,T,H,Dk];
 * everything else as rda_oracle_forward. */
int rda_oracle_forward_channel(int B, int T, int H, int Dk, int Dv,
                               const double *q, const double *k, const double *v,
                               const double *log_alpha_ch, const double *beta, const double *gamma,
                               const double *s0, double *sf, double *out, double scale,
                               int num_threads)
{
    if (B < 0 || T < 0 || H <= 0 || Dk <= 0 || Dv <= 0 || !log_alpha_ch) return 1;
    const long units = (long)B * H;
#ifdef _OPENMP
    if (num_threads > 0) omp_set_num_threads(num_threads);
#else
    (void)num_threads;
#endif
#pragma omp parallel for schedule(dynamic, 1)
    for (long u = 0; u < units; ++u) {
        const long b = u / H;
        const int h = (int)(u % H);
        const long sidx = (b * H + h) * (long)Dk * Dv;
        /* log_alpha_ch doubles as the (unused) scalar array: it has a row per token */
        rda_unit(Dk, Dv, H, h, b * (long)T, T, q, k, v, log_alpha_ch, beta, gamma,
                 s0 ? s0 + sidx : NULL, sf ? sf + sidx : NULL, out, scale, log_alpha_ch);
    }
    return 0;
}

/* Packed variable-length batch: tokens of sequence n are rows
 * [cu_seqlens[n], cu_seqlens[n+1]) of q,k [total,H,Dk]; v,out [total,H,Dv];
 * log_alpha, beta, gamma [total,H]; s0, sf [N,H,Dk,Dv]. */
int rda_oracle_varlen(int N, const int32_t *cu_seqlens, int H, int Dk, int Dv,
                      const double *q, const double *k, const double *v,
                      const double *log_alpha, const double *beta, const double *gamma,
                      const double *s0, double *sf, double *out, double scale,
                      int num_threads)
{
    if (N < 0 || H <= 0 || Dk <= 0 || Dv <= 0) return 1;
    for (int n = 0; n < N; ++n)
        if (cu_seqlens[n + 1] < cu_seqlens[n]) return 1;
    const long units = (long)N * H;
#ifdef _OPENMP
    if (num_threads > 0) omp_set_num_threads(num_threads);
#else
    (void)num_threads;
#endif
#pragma omp parallel for schedule(dynamic, 1)
    for (long u = 0; u < units; ++u) {
        const int n = (int)(u / H);
        const int h = (int)(u % H);
        const long sidx = ((long)n * H + h) * (long)Dk * Dv;
        rda_unit(Dk, Dv, H, h, cu_seqlens[n], (long)cu_seqlens[n + 1] - cu_seqlens[n],
                 q, k, v, log_alpha, beta, gamma,
                 s0 ? s0 + sidx : NULL, sf ? sf + sidx : NULL, out, scale, NULL);
    }
    return 0;
}

/* One decode step for B sequences, state updated in place:
 * q,k [B,H,Dk]; v,out [B,H,Dv]; log_alpha, beta, gamma [B,H]; state [B,H,Dk,Dv]. */
int rda_oracle_decode_step(int B, int H, int Dk, int Dv,
                           const double *q, const double *k, const double *v,
                           const double *log_alpha, const double *beta, const double *gamma,
                           double *state, double *out, double scale, int num_threads)
{
    /* A decode step is the T = 1 case of the fixed-length recurrence, with the
     * final state written over the initial one. */
    if (B < 0 || H <= 0 || Dk <= 0 || Dv <= 0) return 1;
    const long units = (long)B * H;
#ifdef _OPENMP
    if (num_threads > 0) omp_set_num_threads(num_threads);
#else
    (void)num_threads;
#endif
#pragma omp parallel for schedule(dynamic, 1)
    for (long u = 0; u < units; ++u) {
        const long b = u / H;
        const int h = (int)(u % H);
        double *st = state + (b * H + h) * (long)Dk * Dv;
        rda_unit(Dk, Dv, H, h, b, 1, q, k, v, log_alpha, beta, gamma,
                 st, st, out, scale, NULL);
    }
    return 0;
}

/* Packed variable-length batch with per-key-channel decay: log_alpha_ch
 * [total,H,Dk]; everything else as rda_oracle_varlen. */
int rda_oracle_varlen_channel(int N, const int32_t *cu_seqlens, int H, int Dk, int Dv,
                              const double *q, const double *k, const double *v,
                              const double *log_alpha_ch, const double *beta, const double *gamma,
                              const double *s0, double *sf, double *out, double scale,
                              int num_threads)
{
    if (N < 0 || H <= 0 || Dk <= 0 || Dv <= 0 || !log_alpha_ch) return 1;
    for (int n = 0; n < N; ++n)
        if (cu_seqlens[n + 1] < cu_seqlens[n]) return 1;
    const long units = (long)N * H;
#ifdef _OPENMP
    if (num_threads > 0) omp_set_num_threads(num_threads);
#else
    (void)num_threads;
#endif
#pragma omp parallel for schedule(dynamic, 1)
    for (long u = 0; u < units; ++u) {
        const int n = (int)(u / H);
        const int h = (int)(u % H);
        const long sidx = ((long)n * H + h) * (long)Dk * Dv;
        rda_unit(Dk, Dv, H, h, cu_seqlens[n], (long)cu_seqlens[n + 1] - cu_seqlens[n],
                 q, k, v, log_alpha_ch, beta, gamma,
                 s0 ? s0 + sidx : NULL, sf ? sf + sidx : NULL, out, scale, log_alpha_ch);
    }
    return 0;
}

/* One decode step with per-key-channel decay: log_alpha_ch [B,H,Dk]; everything
 * else as rda_oracle_decode_step. */
int rda_oracle_decode_step_channel(int B, int H, int Dk, int Dv,
                                   const double *q, const double *k, const double *v,
                                   const double *log_alpha_ch, const double *beta, const double *gamma,
                                   double *state, double *out, double scale, int num_threads)
{
    if (B < 0 || H <= 0 || Dk <= 0 || Dv <= 0 || !log_alpha_ch) return 1;
    const long units = (long)B * H;
#ifdef _OPENMP
    if (num_threads > 0) omp_set_num_threads(num_threads);
#else
    (void)num_threads;
#endif
#pragma omp parallel for schedule(dynamic, 1)
    for (long u = 0; u < units; ++u) {
        const long b = u / H;
        const int h = (int)(u % H);
        double *st = state + (b * H + h) * (long)Dk * Dv;
        rda_unit(Dk, Dv, H, h, b, 1, q, k, v, log_alpha_ch, beta, gamma,
                 st, st, out, scale, log_alpha_ch);
    }
    return 0;
}

int rda_oracle_max_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}
