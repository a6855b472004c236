/*
 * FLARE++ mixer forward -- fp64 CPU oracle.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path may link, load or
 * call this file: only the test suite, the package's smoke check and the
 * benchmark's CPU-baseline / reference leg use it.  It shares no code, header
 * or constant with the CUDA library.
 *
 * What it computes (FLARE.py README, "FLARE++" code block, the function
 * flarepp_multihead_mixer):
 *
 *     q_dyn = SDPA(q0, k0, k0)          synthesis: M latent seeds attend over N tokens
 *     q     = q_fixed + gate * q_dyn    fixed reference plus gated synthesised term
 *     z     = SDPA(q, k, v)             encode:  N -> M
 *     y     = SDPA(k, q, z)             decode:  M -> N
 *
 * and, for the gate-free FLARE form (FLARE.py README, "FLARE" code block,
 * flare_multihead_mixer; physicsnemo issue #2024, "Fixed reference and gate":
 * with the gate closed the mixer is FLARE), the last two lines with q = q_fixed.
 *
 * SDPA(Q, K, V) is PyTorch's scaled_dot_product_attention without mask,
 * dropout or causality: out_i = sum_j softmax_j(scale * <Q_i, K_j>) V_j.
 * The FLARE++ block passes no scale, so the library default 1/sqrt(D) holds;
 * the FLARE block prints scale=1.0.  Both are reachable through the `scale`
 * argument (scale <= 0 selects 1/sqrt(D)).
 *
 * Shapes (FLARE.py README, docstring of flarepp_multihead_mixer):
 *   q0, q_fixed [H, M, D]  -- shared by every batch element (broadcast over B)
 *   gate        [H]        -- already sigmoid(g), in (0, 1); NULL = closed gate
 *   k0, k, v, y [B, H, N, D]
 *   q, z        [B, H, M, D] (returned for comparison when the pointers are non-NULL)
 * All arrays are row-major, contiguous, fp64.
 *
 * Every softmax is evaluated the plain way: one pass for the row maximum, a
 * second pass for the exponential weights and their sums, in fp64 with libm
 * exp(), in sequential order within a row.  Rows are independent, so OpenMP
 * distributes whole rows over threads; the arithmetic inside a row is not
 * reordered.  Build without -ffast-math.
 */
#include <math.h>
#include <stddef.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#ifdef _OPENMP
#include <omp.h>
#endif

/* Planted mistakes, compiled in only by the test that checks the pins catch
 * them (tests build this file with -DORACLE_PLANT=<n>).  0 = the oracle. */
#ifndef ORACLE_PLANT
#define ORACLE_PLANT 0
#endif

static double dot(const double* a, const double* b, int64_t D) {
    double s = 0.0;
    for (int64_t d = 0; d < D; ++d) s += a[d] * b[d];
    return s;
}

/* One row of SDPA: out = sum_j softmax_j(scale*<q,K_j>) V_j over j < Lk. */
static void sdpa_row(const double* q, const double* K, const double* V,
                     int64_t Lk, int64_t D, double scale, double* out) {
    int64_t Lk_used = Lk;
#if ORACLE_PLANT == 7
    if (Lk_used > 1) Lk_used -= 1;               /* drops the last key */
#endif
    double mx = -INFINITY;
    for (int64_t j = 0; j < Lk_used; ++j) {
        double s = scale * dot(q, K + j * D, D);
        if (s > mx) mx = s;
    }
    for (int64_t d = 0; d < D; ++d) out[d] = 0.0;
    double den = 0.0;
    for (int64_t j = 0; j < Lk_used; ++j) {
        double s = scale * dot(q, K + j * D, D);
#if ORACLE_PLANT == 9
        double w = exp(-(s - mx));               /* wrong sign */
#else
        double w = exp(s - mx);
#endif
        den += w;
        const double* vj = V + j * D;
        for (int64_t d = 0; d < D; ++d) out[d] += w * vj[d];
    }
#if ORACLE_PLANT == 10
    (void)den;                                   /* normalisation dropped */
#else
    for (int64_t d = 0; d < D; ++d) out[d] /= den;
#endif
}

static double resolve_scale(double scale, int64_t D) {
#if ORACLE_PLANT == 1
    (void)scale; (void)D;
    return 1.0;                                  /* scale ignored */
#else
    return scale > 0.0 ? scale : 1.0 / sqrt((double)D);
#endif
}

/* Plain SDPA on one (batch, head) slice: O[Lq,D] = SDPA(Q[Lq,D], K[Lk,D], V[Lk,D]). */
int oracle_sdpa(const double* Q, const double* K, const double* V, double* O,
                int64_t Lq, int64_t Lk, int64_t D, double scale) {
    if (!Q || !K || !V || !O || Lq < 0 || Lk < 1 || D < 1) return 1;
    const double sc = resolve_scale(scale, D);
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < Lq; ++i) sdpa_row(Q + i * D, K, V, Lk, D, sc, O + i * D);
    return 0;
}

/* Synthesis and gate (steps 1-2) for one (b, h): q[m] for all m.
 * q0_h, qf_h: the head's [M,D] slices; k0_bh: the (b,h) [N,D] slice of k0. */
static void routing_queries(const double* q0_h, const double* qf_h, double g,
                            const double* k0_bh, int64_t N, int64_t M, int64_t D,
                            double sc, int flare_mode, double* q_bh /* [M,D] */) {
    if (flare_mode) {
        memcpy(q_bh, qf_h, sizeof(double) * (size_t)(M * D));
        return;
    }
#pragma omp parallel for schedule(static)
    for (int64_t m = 0; m < M; ++m) {
        double qdyn[1024];
        double* qd = D <= 1024 ? qdyn : (double*)malloc(sizeof(double) * (size_t)D);
        sdpa_row(q0_h + m * D, k0_bh, k0_bh, N, D, sc, qd);
        for (int64_t d = 0; d < D; ++d) {
#if ORACLE_PLANT == 2
            q_bh[m * D + d] = qf_h[m * D + d] + qd[d];          /* gate dropped */
#else
            q_bh[m * D + d] = qf_h[m * D + d] + g * qd[d];
#endif
        }
        if (qd != qdyn) free(qd);
    }
}

/*
 * Full mixer.  flare_mode != 0 (or gate == NULL) gives FLARE: q = q_fixed.
 * y [B,H,N,D] is always written; q_out, z_out [B,H,M,D] when non-NULL.
 * Returns 0 on success, 1 on a bad argument, 2 on allocation failure.
 */
int oracle_flarepp(const double* q0, const double* q_fixed, const double* gate,
                   const double* k0, const double* k, const double* v, double* y,
                   double* q_out, double* z_out,
                   int64_t B, int64_t H, int64_t N, int64_t M, int64_t D,
                   double scale, int flare_mode) {
    if (!q_fixed || !k || !v || !y || B < 1 || H < 1 || N < 1 || M < 1 || D < 1) return 1;
    if (!flare_mode && gate != NULL && (!q0 || !k0)) return 1;
    const double sc = resolve_scale(scale, D);
    double* q_bh = (double*)malloc(sizeof(double) * (size_t)(M * D));
    double* z_bh = (double*)malloc(sizeof(double) * (size_t)(M * D));
    if (!q_bh || !z_bh) { free(q_bh); free(z_bh); return 2; }
    for (int64_t b = 0; b < B; ++b) {
        for (int64_t h = 0; h < H; ++h) {
            const int64_t bh = b * H + h;
            const double* k_bh = k + (bh * N) * D;
            const double* v_bh = v + (bh * N) * D;
            (void)v_bh;
            /* steps 1-2: routing queries */
            const int closed = flare_mode || gate == NULL;
            const double* qf_h = q_fixed + (h * M) * D;
#if ORACLE_PLANT == 8
            qf_h = q_fixed + ((b % H) * M) * D;      /* q_fixed indexed by batch, not head */
#endif
#if ORACLE_PLANT == 3
            const double* syn_bh = k_bh;             /* synthesis reads k instead of k0 */
#else
            const double* syn_bh = closed ? NULL : k0 + (bh * N) * D;
#endif
            routing_queries(closed ? NULL : q0 + (h * M) * D, qf_h, closed ? 0.0 : gate[h],
                            syn_bh, N, M, D, sc, closed, q_bh);
            /* step 3: encode, z = SDPA(q, k, v) */
#pragma omp parallel for schedule(static)
            for (int64_t m = 0; m < M; ++m) {
#if ORACLE_PLANT == 4
                sdpa_row(q_bh + m * D, k_bh, k_bh, N, D, sc, z_bh + m * D);   /* values = keys */
#else
                sdpa_row(q_bh + m * D, k_bh, v_bh, N, D, sc, z_bh + m * D);
#endif
            }
            /* step 4: decode, y = SDPA(k, q, z) */
#pragma omp parallel for schedule(static)
            for (int64_t n = 0; n < N; ++n) {
#if ORACLE_PLANT == 5
                sdpa_row(k_bh + n * D, z_bh, q_bh, M, D, sc, y + (bh * N + n) * D);  /* keys and values swapped */
#else
                sdpa_row(k_bh + n * D, q_bh, z_bh, M, D, sc, y + (bh * N + n) * D);
#endif
            }
            if (q_out) memcpy(q_out + (bh * M) * D, q_bh, sizeof(double) * (size_t)(M * D));
            if (z_out) memcpy(z_out + (bh * M) * D, z_bh, sizeof(double) * (size_t)(M * D));
        }
    }
    free(q_bh);
    free(z_bh);
    return 0;
}

/*
 * Sampled form for large workloads: one (b, h) slice in full for q and z,
 * and y only at the listed token indices.
 *   q0, q_fixed : [M, D] slices of head h          (q0 may be NULL in flare mode)
 *   gate_h      : the head's gate value (ignored in flare mode)
 *   k0, k, v    : [N, D] slices of (b, h)
 *   tokens      : n_tok indices in [0, N); y_out [n_tok, D]
 *   q_out, z_out: [M, D], optional
 */
int oracle_flarepp_head(const double* q0, const double* q_fixed, double gate_h,
                        const double* k0, const double* k, const double* v,
                        const int64_t* tokens, int64_t n_tok, double* y_out,
                        double* q_out, double* z_out,
                        int64_t N, int64_t M, int64_t D, double scale, int flare_mode) {
    if (!q_fixed || !k || !v || N < 1 || M < 1 || D < 1 || n_tok < 0) return 1;
    if (n_tok > 0 && (!tokens || !y_out)) return 1;
    if (!flare_mode && (!q0 || !k0)) return 1;
    for (int64_t t = 0; t < n_tok; ++t)
        if (tokens[t] < 0 || tokens[t] >= N) return 1;
    const double sc = resolve_scale(scale, D);
    double* q_h = (double*)malloc(sizeof(double) * (size_t)(M * D));
    double* z_h = (double*)malloc(sizeof(double) * (size_t)(M * D));
    if (!q_h || !z_h) { free(q_h); free(z_h); return 2; }
    /* steps 1-2 */
    routing_queries(q0, q_fixed, gate_h, k0, N, M, D, sc, flare_mode, q_h);
#pragma omp parallel for schedule(static)
    for (int64_t m = 0; m < M; ++m) sdpa_row(q_h + m * D, k, v, N, D, sc, z_h + m * D);
#pragma omp parallel for schedule(static)
    for (int64_t t = 0; t < n_tok; ++t)
        sdpa_row(k + tokens[t] * D, q_h, z_h, M, D, sc, y_out + t * D);
    if (q_out) memcpy(q_out, q_h, sizeof(double) * (size_t)(M * D));
    if (z_out) memcpy(z_out, z_h, sizeof(double) * (size_t)(M * D));
    free(q_h);
    free(z_h);
    return 0;
}

/* Threads the OpenMP runtime will use (for reporting the CPU baseline). */
int oracle_num_threads(void) {
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

int oracle_plant(void) { return ORACLE_PLANT; }
