/*
 * gdn_oracle.c -- plain fp64 CPU oracle for the gated delta rule.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path may call, link or
 * execute this file: it is used by tests/, by __graft_entry__.smoke() and by
 * the cpu_baseline / reference arm of bench.py.  It shares no code, header,
 * table or helper with the CUDA library.
 *
 * Sources (cited by page title and section):
 *   [WT]  "手撕Qwen3-Next" walkthrough (wkq9411.github.io, Code-Qwen3-Next),
 *         section 一(一)5 "应用 Gated Delta Rule":
 *           (1) chunkwise recurrence, steps a-g  (torch_chunk_gated_delta_rule)
 *           (2) token-by-token recurrence        (torch_recurrent_gated_delta_rule)
 *         and section 一(一)4 "形状调整" (GQA repeat_interleave).
 *   [PTO] PyPTO-Gym "Qwen3Next 样例" README, sections 数学公式 (formulas) and
 *         参数说明 (packed [T,N,D] tensors, act_seq_len cumulative lengths).
 *
 * Gate parametrisation ([WT] section 一(一)4 "形状调整", the lines that form
 * beta and g from the projections b and a):
 *
 *   oracle_gates       -- beta = sigmoid(b);  g = -exp(A_log) * softplus(a + dt_bias)
 *                         with softplus(x) = log(1 + exp(x)), per token and v-head.
 *
 * The layer steps around it, on the same page (NEXT to the core, same rules):
 *
 *   oracle_gated_rmsnorm -- output epilogue, [WT] 一(一)1 and 6: RMSNormGated,
 *                         y = o / sqrt(mean(o^2) + eps) * w * silu(z).
 *   oracle_causal_conv1d -- [WT] 一(一)3: causal depthwise conv1d + SiLU of the
 *                         packed q|k|v channels, with the conv_state window of
 *                         torch_causal_conv1d_update (prefill and decode).
 *
 * Two functions compute the method:
 *
 *   oracle_recurrent   -- THE DEFINITION.  Token loop of [WT] (2):
 *                           S <- S*exp(g_t);  kv = k^T S;  delta = beta_t (v_t - kv);
 *                           S <- S + k delta^T;  o_t = q^T S   (updated S),
 *                         with q,k L2-normalised (eps 1e-6 inside the sqrt,
 *                         [PTO] L2 归一化) and q scaled by 1/sqrt(Dk) ([WT] 5(1)a).
 *
 *   oracle_chunk_form  -- [WT] (1) steps a-g written out with a generic chunk
 *                         size C, in the page's order: intra-chunk quantities
 *                         for every chunk first, then the sequential chunk loop.
 *                         It exists only so the tests can pin the two forms
 *                         against each other (they agree exactly up to rounding).
 *
 * Layouts (row-major, all fp64):
 *   q, k   [T, Nqk, Dk]      v, out [T, Nv, Dv]      g, beta [T, Nv]
 *   s0, s_final [N, Nv, Dk, Dv]  (Dk rows, Dv contiguous; [WT] cache layout)
 *   cu_seqlens int32 [N+1]   sequence n owns tokens [cu[n], cu[n+1])  ([PTO])
 *   v-head h reads qk-head h / (Nv/Nqk)  ([WT] 一(一)4 repeat_interleave)
 *
 * Readings where the pages are silent or garbled:
 *   - eps sits inside the square root ([PTO] L2 归一化);
 *   - the query scale 1/sqrt(Dk) is applied after the norm ([WT] 5(1)a);
 *   - the output of token t uses the state after token t's own write ([WT] (2));
 *   - every sequence starts from s0[n] (or zeros) and has its own chunk grid
 *     starting at cu[n]; the tail chunk is zero padded ([WT] 5(1)a, F.pad).
 *
 * Return value: 0 on success, negative on a bad argument.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define ORACLE_EPS 1e-6

/* x / sqrt(sum x^2 + eps) when use_norm, times `scale`.  [PTO] 数学公式, L2 归一化. */
static void normalise(const double *x, int d, int use_norm, double scale, double *y)
{
    double ss = 0.0;
    for (int i = 0; i < d; ++i) ss += x[i] * x[i];
    double f = use_norm ? 1.0 / sqrt(ss + ORACLE_EPS) : 1.0;
    for (int i = 0; i < d; ++i) y[i] = x[i] * f * scale;
}

static int check_args(int num_seqs, const int32_t *cu, int nqk, int nv, int dk, int dv)
{
    if (num_seqs < 0 || !cu || nqk <= 0 || nv <= 0 || dk <= 0 || dv <= 0) return -1;
    if (nv % nqk != 0) return -2;
    if (cu[0] != 0) return -3;
    for (int n = 0; n < num_seqs; ++n)
        if (cu[n + 1] < cu[n]) return -3;
    return 0;
}

/* ------------------------------------------------------------------------- */
/* The definition: the token-by-token gated delta rule ([WT] 5(2)).           */
/* ------------------------------------------------------------------------- */
int oracle_recurrent(int num_seqs, const int32_t *cu_seqlens,
                     int nqk, int nv, int dk, int dv,
                     const double *q, const double *k, const double *v,
                     const double *g, const double *beta,
                     const double *s0, int qk_l2norm, double scale,
                     double *out, double *s_final)
{
    int rc = check_args(num_seqs, cu_seqlens, nqk, nv, dk, dv);
    if (rc) return rc;
    if (scale <= 0.0) scale = 1.0 / sqrt((double)dk);
    const int group = nv / nqk;
    const long pairs = (long)num_seqs * nv;

#pragma omp parallel for schedule(dynamic, 1)
    for (long p = 0; p < pairs; ++p) {
        const int n = (int)(p / nv), h = (int)(p % nv);
        const int j = h / group;                     /* qk-head of v-head h */
        double *S = (double *)malloc(sizeof(double) * (size_t)dk * dv);
        double *qh = (double *)malloc(sizeof(double) * (size_t)dk);
        double *kh = (double *)malloc(sizeof(double) * (size_t)dk);
        double *kv = (double *)malloc(sizeof(double) * (size_t)dv);
        const size_t sidx = ((size_t)n * nv + h) * (size_t)dk * dv;
        if (s0) memcpy(S, s0 + sidx, sizeof(double) * (size_t)dk * dv);
        else memset(S, 0, sizeof(double) * (size_t)dk * dv);

        for (long t = cu_seqlens[n]; t < cu_seqlens[n + 1]; ++t) {
            normalise(q + ((size_t)t * nqk + j) * dk, dk, qk_l2norm, scale, qh);
            normalise(k + ((size_t)t * nqk + j) * dk, dk, qk_l2norm, 1.0, kh);
            const double alpha = exp(g[(size_t)t * nv + h]);
            const double b = beta[(size_t)t * nv + h];
            const double *vt = v + ((size_t)t * nv + h) * dv;
            double *ot = out + ((size_t)t * nv + h) * dv;

            /* decay first: S <- S * exp(g_t) */
            for (size_t e = 0; e < (size_t)dk * dv; ++e) S[e] *= alpha;
            /* kv_c = sum_r S[r,c] k_r  (the value the key currently retrieves) */
            for (int c = 0; c < dv; ++c) kv[c] = 0.0;
            for (int r = 0; r < dk; ++r)
                for (int c = 0; c < dv; ++c) kv[c] += S[(size_t)r * dv + c] * kh[r];
            /* delta_c = beta (v_c - kv_c);  S[r,c] += k_r delta_c */
            for (int c = 0; c < dv; ++c) kv[c] = b * (vt[c] - kv[c]);
            for (int r = 0; r < dk; ++r)
                for (int c = 0; c < dv; ++c) S[(size_t)r * dv + c] += kh[r] * kv[c];
            /* o_c = sum_r S[r,c] q_r, with the updated state */
            for (int c = 0; c < dv; ++c) ot[c] = 0.0;
            for (int r = 0; r < dk; ++r)
                for (int c = 0; c < dv; ++c) ot[c] += S[(size_t)r * dv + c] * qh[r];
        }
        if (s_final) memcpy(s_final + sidx, S, sizeof(double) * (size_t)dk * dv);
        free(S); free(qh); free(kh); free(kv);
    }
    return 0;
}

/* ------------------------------------------------------------------------- */
/* Chunk form ([WT] 5(1) a-g), one chunk's intra-chunk quantities.            */
/* ------------------------------------------------------------------------- */
/*
 * Inputs for one chunk of C rows (already normalised, q already scaled, padded
 * rows all zero): kh [C,dk], v [C,dv], g [C], beta [C].
 * Outputs:
 *   gcum  [C]    inclusive cumsum of g inside the chunk          (step c)
 *   gamma [C,C]  exp(gcum_r - gcum_i) for i <= r else 0           (step c)
 *   A     [C,C]  -(k_beta K^T * gamma), strictly lower             (step d)
 *   T     [C,C]  (I - A)^-1 by the row recursion, plus I           (step d)
 *   U     [C,dv] T (v * beta)                                      (step e)
 *   W     [C,dk] T (k_beta * exp(gcum))                            (step e)
 * Any output pointer except the ones needed internally may be NULL.
 */
int oracle_chunk_prepare(int C, int dk, int dv,
                         const double *kh, const double *v,
                         const double *g, const double *beta,
                         double *gcum, double *gamma, double *A, double *T,
                         double *U, double *W)
{
    if (C <= 0 || dk <= 0 || dv <= 0 || !kh || !v || !g || !beta ||
        !gcum || !gamma || !A || !T)
        return -1;
    /* step b: k_beta = k * beta, v_beta = v * beta */
    double *kb = (double *)malloc(sizeof(double) * (size_t)C * dk);
    double *vb = (double *)malloc(sizeof(double) * (size_t)C * dv);
    for (int i = 0; i < C; ++i) {
        for (int d = 0; d < dk; ++d) kb[(size_t)i * dk + d] = kh[(size_t)i * dk + d] * beta[i];
        for (int c = 0; c < dv; ++c) vb[(size_t)i * dv + c] = v[(size_t)i * dv + c] * beta[i];
    }
    /* step c: gate cumsum (restarts at every chunk) and decay mask.
       The lower-triangle mask is taken before exp, so no exp(positive). */
    double acc = 0.0;
    for (int i = 0; i < C; ++i) { acc += g[i]; gcum[i] = acc; }
    for (int r = 0; r < C; ++r)
        for (int i = 0; i < C; ++i)
            gamma[(size_t)r * C + i] = (i <= r) ? exp(gcum[r] - gcum[i]) : 0.0;
    /* step d: A = -((k_beta K^T) * gamma) with the upper triangle and the
       diagonal set to zero. */
    for (int r = 0; r < C; ++r)
        for (int i = 0; i < C; ++i) {
            double s = 0.0;
            if (i < r) {
                for (int d = 0; d < dk; ++d) s += kb[(size_t)r * dk + d] * kh[(size_t)i * dk + d];
                s = -s * gamma[(size_t)r * C + i];
            }
            A[(size_t)r * C + i] = s;
        }
    /* step d: row recursion  Tt_i = A_i + A_i Tt_{<i}  (Tt = T - I is strictly
       lower), row by row from the second row; then T = Tt + I. */
    memcpy(T, A, sizeof(double) * (size_t)C * C);
    double *row = (double *)malloc(sizeof(double) * (size_t)C);
    for (int i = 1; i < C; ++i) {
        for (int j = 0; j < i; ++j) {
            double s = A[(size_t)i * C + j];
            for (int m = 0; m < i; ++m) s += A[(size_t)i * C + m] * T[(size_t)m * C + j];
            row[j] = s;
        }
        for (int j = 0; j < i; ++j) T[(size_t)i * C + j] = row[j];
    }
    for (int i = 0; i < C; ++i) T[(size_t)i * C + i] += 1.0;
    /* step e: U = T v_beta;  W = T (k_beta * exp(gcum))  (the diagonal
       similarity D (I+L0)^-1 D^-1 folds the decay into the right factor). */
    if (U)
        for (int r = 0; r < C; ++r)
            for (int c = 0; c < dv; ++c) {
                double s = 0.0;
                for (int i = 0; i < C; ++i) s += T[(size_t)r * C + i] * vb[(size_t)i * dv + c];
                U[(size_t)r * dv + c] = s;
            }
    if (W)
        for (int r = 0; r < C; ++r)
            for (int d = 0; d < dk; ++d) {
                double s = 0.0;
                for (int i = 0; i < C; ++i)
                    s += T[(size_t)r * C + i] * kb[(size_t)i * dk + d] * exp(gcum[i]);
                W[(size_t)r * dk + d] = s;
            }
    free(kb); free(vb); free(row);
    return 0;
}

/* ------------------------------------------------------------------------- */
/* Chunk form ([WT] 5(1) a-g) for whole packed varlen batches.                */
/* ------------------------------------------------------------------------- */
int oracle_chunk_form(int num_seqs, const int32_t *cu_seqlens,
                      int nqk, int nv, int dk, int dv, int C,
                      const double *q, const double *k, const double *v,
                      const double *g, const double *beta,
                      const double *s0, int qk_l2norm, double scale,
                      double *out, double *s_final)
{
    int rc = check_args(num_seqs, cu_seqlens, nqk, nv, dk, dv);
    if (rc) return rc;
    if (C <= 0) return -4;
    if (scale <= 0.0) scale = 1.0 / sqrt((double)dk);
    const int group = nv / nqk;
    const long pairs = (long)num_seqs * nv;

#pragma omp parallel for schedule(dynamic, 1)
    for (long p = 0; p < pairs; ++p) {
        const int n = (int)(p / nv), h = (int)(p % nv);
        const int j = h / group;
        const long t0 = cu_seqlens[n], len = cu_seqlens[n + 1] - cu_seqlens[n];
        const long nch = (len + C - 1) / C;            /* step a: pad to a multiple of C */
        const long Lp = nch * C;
        const size_t sidx = ((size_t)n * nv + h) * (size_t)dk * dv;

        /* step a: normalise, gather this head, zero-pad, scale q */
        double *Q = (double *)calloc((size_t)Lp * dk + 1, sizeof(double));
        double *K = (double *)calloc((size_t)Lp * dk + 1, sizeof(double));
        double *V = (double *)calloc((size_t)Lp * dv + 1, sizeof(double));
        double *G = (double *)calloc((size_t)Lp + 1, sizeof(double));
        double *B = (double *)calloc((size_t)Lp + 1, sizeof(double));
        for (long t = 0; t < len; ++t) {
            normalise(q + ((size_t)(t0 + t) * nqk + j) * dk, dk, qk_l2norm, scale, Q + (size_t)t * dk);
            normalise(k + ((size_t)(t0 + t) * nqk + j) * dk, dk, qk_l2norm, 1.0, K + (size_t)t * dk);
            memcpy(V + (size_t)t * dv, v + ((size_t)(t0 + t) * nv + h) * dv, sizeof(double) * dv);
            G[t] = g[(size_t)(t0 + t) * nv + h];
            B[t] = beta[(size_t)(t0 + t) * nv + h];
        }

        /* steps b-e for every chunk first */
        double *GC = (double *)malloc(sizeof(double) * ((size_t)Lp + 1));
        double *GM = (double *)malloc(sizeof(double) * ((size_t)nch * C * C + 1));
        double *Am = (double *)malloc(sizeof(double) * ((size_t)C * C));
        double *Tm = (double *)malloc(sizeof(double) * ((size_t)C * C));
        double *U = (double *)malloc(sizeof(double) * ((size_t)Lp * dv + 1));
        double *W = (double *)malloc(sizeof(double) * ((size_t)Lp * dk + 1));
        for (long c = 0; c < nch; ++c)
            oracle_chunk_prepare(C, dk, dv, K + (size_t)c * C * dk, V + (size_t)c * C * dv,
                                 G + (size_t)c * C, B + (size_t)c * C,
                                 GC + (size_t)c * C, GM + (size_t)c * C * C, Am, Tm,
                                 U + (size_t)c * C * dv, W + (size_t)c * C * dk);

        /* step f: the sequential loop over chunks, carrying S [dk, dv] */
        double *S = (double *)malloc(sizeof(double) * (size_t)dk * dv);
        double *Vn = (double *)malloc(sizeof(double) * (size_t)C * dv);
        double *P = (double *)malloc(sizeof(double) * (size_t)C * C);
        if (s0) memcpy(S, s0 + sidx, sizeof(double) * (size_t)dk * dv);
        else memset(S, 0, sizeof(double) * (size_t)dk * dv);
        for (long c = 0; c < nch; ++c) {
            const double *Qc = Q + (size_t)c * C * dk, *Kc = K + (size_t)c * C * dk;
            const double *gc = GC + (size_t)c * C, *gm = GM + (size_t)c * C * C;
            const double *Uc = U + (size_t)c * C * dv, *Wc = W + (size_t)c * C * dk;
            /* attn = (q K^T * gamma) with the strict upper triangle zeroed */
            for (int r = 0; r < C; ++r)
                for (int i = 0; i < C; ++i) {
                    double s = 0.0;
                    if (i <= r) {
                        for (int d = 0; d < dk; ++d) s += Qc[(size_t)r * dk + d] * Kc[(size_t)i * dk + d];
                        s *= gm[(size_t)r * C + i];
                    }
                    P[(size_t)r * C + i] = s;
                }
            /* v_new = U - W S */
            for (int r = 0; r < C; ++r)
                for (int x = 0; x < dv; ++x) {
                    double s = 0.0;
                    for (int d = 0; d < dk; ++d) s += Wc[(size_t)r * dk + d] * S[(size_t)d * dv + x];
                    Vn[(size_t)r * dv + x] = Uc[(size_t)r * dv + x] - s;
                }
            /* o = (q * exp(gcum)) S + attn v_new;  only valid rows are kept (step g) */
            for (int r = 0; r < C; ++r) {
                const long t = c * C + r;
                if (t >= len) break;
                double *ot = out + ((size_t)(t0 + t) * nv + h) * dv;
                const double eg = exp(gc[r]);
                for (int x = 0; x < dv; ++x) {
                    double s1 = 0.0, s2 = 0.0;
                    for (int d = 0; d < dk; ++d) s1 += Qc[(size_t)r * dk + d] * eg * S[(size_t)d * dv + x];
                    for (int i = 0; i < C; ++i) s2 += P[(size_t)r * C + i] * Vn[(size_t)i * dv + x];
                    ot[x] = s1 + s2;
                }
            }
            /* S <- S exp(g_last) + (K * exp(g_last - gcum))^T v_new */
            const double glast = gc[C - 1];
            for (int d = 0; d < dk; ++d)
                for (int x = 0; x < dv; ++x) {
                    double s = S[(size_t)d * dv + x] * exp(glast);
                    for (int i = 0; i < C; ++i)
                        s += Kc[(size_t)i * dk + d] * exp(glast - gc[i]) * Vn[(size_t)i * dv + x];
                    S[(size_t)d * dv + x] = s;
                }
        }
        if (s_final) memcpy(s_final + sidx, S, sizeof(double) * (size_t)dk * dv);
        free(Q); free(K); free(V); free(G); free(B); free(GC); free(GM); free(Am); free(Tm);
        free(U); free(W); free(S); free(Vn); free(P);
    }
    return 0;
}

/* Gate parametrisation, [WT] 一(一)4: beta = sigmoid(b), g = -exp(A_log) *
 * softplus(a + dt_bias), softplus(x) = log(1 + exp(x)).  a, b, g, beta are
 * [T, nv]; A_log, dt_bias are [nv].  softplus is evaluated as
 * max(x, 0) + log1p(exp(-|x|)), the same function without overflow. */
int oracle_gates(int64_t T, int nv, const double *a, const double *b, const double *A_log,
                 const double *dt_bias, double *g, double *beta)
{
    if (T < 0 || nv <= 0 || !a || !b || !A_log || !dt_bias || !g || !beta) return -1;
    for (int64_t t = 0; t < T; ++t) {
        for (int h = 0; h < nv; ++h) {
            const int64_t i = t * nv + h;
            const double x = a[i] + dt_bias[h];
            const double sp = (x > 0.0 ? x : 0.0) + log1p(exp(-fabs(x)));
            g[i] = -exp(A_log[h]) * sp;
            beta[i] = 1.0 / (1.0 + exp(-b[i]));
        }
    }
    return 0;
}

/* ---------------------------------------------------------------------------
 * Output epilogue: gated RMSNorm (RMSNormGated), per row of head_v_dim values.
 *
 * [WT] section 一(一)1 builds the layer's norm as RMSNormGated(head_v_dim,
 * eps) and section 一(一)6 (输出调整) applies it as norm(o, z) with o and z
 * flattened to rows of head_v_dim: "RMSNorm + Gate".  The page says this
 * norm is the ordinary RMSNorm with a gain initialised to 1; its RMSNorm code
 * (section 三, Zero-Centered RMSNorm, _norm) multiplies x by
 * rsqrt(mean(x^2) + eps).  The gate's activation is not printed: it is read
 * as SiLU, z * sigmoid(z), applied to z after the norm:
 *
 *     y = o / sqrt(mean(o^2) + eps) * w * silu(z),   silu(x) = x / (1 + exp(-x))
 *
 * o, z, y are [rows, dv]; w is [dv].
 * ------------------------------------------------------------------------- */
int oracle_gated_rmsnorm(int64_t rows, int dv, const double *o, const double *z,
                         const double *w, double eps, double *y)
{
    if (rows < 0 || dv <= 0 || !o || !z || !w || !y || !(eps >= 0.0)) return -1;
    for (int64_t r = 0; r < rows; ++r) {
        const double *orow = o + r * dv, *zrow = z + r * dv;
        double ms = 0.0;
        for (int c = 0; c < dv; ++c) ms += orow[c] * orow[c];
        ms /= (double)dv;
        const double inv = 1.0 / sqrt(ms + eps);
        for (int c = 0; c < dv; ++c) {
            const double gate = zrow[c] / (1.0 + exp(-zrow[c]));
            y[r * dv + c] = orow[c] * inv * w[c] * gate;
        }
    }
    return 0;
}

/* ---------------------------------------------------------------------------
 * Causal depthwise conv1d + SiLU over the packed q|k|v channels.
 *
 * [WT] section 一(一)3 (qkv 卷积部分): every channel is convolved on its own
 * (groups = channels) with a kernel of `ksize` taps, zero padded by ksize - 1
 * on the left and cut to the sequence length, then passed through SiLU.  Tap i
 * of channel c multiplies input t - (ksize - 1) + i (cross-correlation, as
 * torch's conv1d computes it), so tap ksize - 1 meets the current token.  The
 * decode update (torch_causal_conv1d_update) is the same computation over
 * [conv_state, x]: the window before a sequence is the cached conv_state of
 * ksize pre-convolution inputs (zeros for a fresh prefill), and the new
 * conv_state is the last ksize inputs of [window, sequence], zero filled on
 * the left when fewer exist.
 *
 *   x, y       [T, channels] (token-major)  sequence n owns tokens [cu[n], cu[n+1])
 *   w          [channels, ksize]            bias [channels] or NULL
 *   state_in   [N, channels, ksize] or NULL (zeros); state_out likewise or NULL.
 *              state_out may be state_in (updated in place).
 * ------------------------------------------------------------------------- */
int oracle_causal_conv1d(int num_seqs, const int32_t *cu, int channels, int ksize,
                         const double *x, const double *w, const double *bias,
                         const double *state_in, double *y, double *state_out)
{
    if (num_seqs < 1 || !cu || channels <= 0 || ksize < 1 || !x || !w || !y) return -1;
    if (cu[0] != 0) return -2;
    for (int n = 0; n < num_seqs; ++n)
        if (cu[n + 1] < cu[n]) return -2;
#pragma omp parallel for schedule(dynamic, 16)
    for (long p = 0; p < (long)num_seqs * channels; ++p) {
        const int n = (int)(p / channels), c = (int)(p % channels);
        const int64_t t0 = cu[n], len = (int64_t)cu[n + 1] - cu[n];
        const size_t sidx = ((size_t)n * channels + c) * ksize;
        /* extended input: the ksize-entry window, then the sequence */
        double *ext = (double *)malloc(sizeof(double) * (size_t)(ksize + len));
        for (int i = 0; i < ksize; ++i) ext[i] = state_in ? state_in[sidx + i] : 0.0;
        for (int64_t t = 0; t < len; ++t) ext[ksize + t] = x[(t0 + t) * channels + c];
        for (int64_t t = 0; t < len; ++t) {
            /* token t sits at ext[ksize + t]; tap i reads ext[ksize + t - (ksize-1) + i] */
            double pre = bias ? bias[c] : 0.0;
            for (int i = 0; i < ksize; ++i) pre += w[(size_t)c * ksize + i] * ext[t + 1 + i];
            y[(t0 + t) * channels + c] = pre / (1.0 + exp(-pre));
        }
        if (state_out)
            for (int i = 0; i < ksize; ++i) state_out[sidx + i] = ext[len + i];
        free(ext);
    }
    return 0;
}
