/*
 * gdn_oracle.c -- plain, slow, fp64 CPU oracle of the gated delta rule.
 *
 * TEST INFRASTRUCTURE ONLY.  Only tests/, __graft_entry__.smoke() and the
 * cpu_baseline / reference legs of bench.py load this library.  It shares no
 * code, header, table or helper with the CUDA library: it is compiled from this
 * file alone with gcc, and the CUDA path never links or calls it.
 *
 * What it computes (sources are web pages on Gated DeltaNet):
 *
 *   Gates ("Gated DeltaNet ... Qwen3-next", section 2.1, gate code):
 *       beta = sigmoid(b)
 *       g    = -exp(A_log) * softplus(a + dt_bias),   alpha = exp(g)
 *   (the exp(g) decay is also the one in the "QWEN3.5" Q&A page, question 2).
 *
 *   Recurrence ("Gated DeltaNet and reasoning scaffolds" research log, the
 *   third of its three update rules; the same formula is in the Gated DeltaNet /
 *   Qwen 3.5 tutorial page, section 6):
 *       S_t = S_{t-1} * ( alpha_t * (I - beta_t k_t k_t^T) ) + beta_t v_t k_t^T
 *       o_t = S_t q_t                       (output read from the updated state)
 *   with S_t a Dv x Dk matrix (S k ~ v).  The Q&A page's "incremental update"
 *   note describes the same order: decay the whole state by alpha first, then
 *   clear and write along the current key with strength beta.
 *
 * Readings where the pages are silent (each is also listed in the design notes):
 *   - storage orientation: the state crosses this interface as H = S^T, laid
 *     out [n_seqs, HV, Dk, Dv] row-major; inside, the loop works on S itself;
 *   - optional q/k L2 normalisation x / sqrt(sum x^2 + 1e-6) per token and q/k
 *     head, applied before the token is used;
 *   - optional output scale (1.0 in every workload);
 *   - grouped heads: value head h reads q/k head h / (HV / HK);
 *   - packed sequences: tokens cu_seqlens[n] .. cu_seqlens[n+1]-1 form
 *     sequence n, each with its own initial state.
 *
 *   Convolution prologue (the Qwen3-next page, section 3.1, names a depthwise
 *   separable convolution before the gated update; the tutorial page, section 6,
 *   gives its kernel size field linear_conv_kernel_dim = 4):
 *       y_t[c] = act( sum_{i=0..3} w[c][i] * x_{t-3+i}[c] )
 *   per channel c, causal, with x_{-3..-1} taken from a per-sequence state of
 *   the three previous inputs (zeros if none) and the state after the last token
 *   the three last inputs.  Readings: the taps run oldest to newest; the pages
 *   name no activation, so act is the identity or, on request, SiLU
 *   (x * sigmoid(x)).
 *
 *   Output epilogue (the Qwen3-next page, section 3.2, gives the zero-centred RMSNorm:
 *   x * rsqrt(mean(x^2) + eps) with a weight initialised to zero, so the scale is
 *   1 + weight; the GDN resource-allocation page says the output gate is usually a
 *   sigmoid applied to the attention output before the residual add):
 *       out = o * rsqrt(mean_j o_j^2 + eps) * (1 + w) * sigmoid(z)
 *   per (token, value head) over the Dv values.  Readings: eps = 1e-6; z is the gate's
 *   input, given per element; w is shared by the value heads.
 *
 * Everything is fp64.  No blocking, chunking or reordering: one token at a
 * time, exactly the formula above.  OpenMP only splits independent
 * (sequence, value head) pairs across threads.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

/* softplus(x) = log(1 + e^x), written in the overflow-free form
 * max(x, 0) + log1p(e^{-|x|}). */
static double oracle_softplus(double x) {
    return fmax(x, 0.0) + log1p(exp(-fabs(x)));
}

static double oracle_sigmoid(double x) {
    return 1.0 / (1.0 + exp(-x));
}

/* Gate computation.  a, b: [n_tokens, HV]; A_log, dt_bias: [HV];
 * outputs g, beta: [n_tokens, HV]. */
void gdn_oracle_gates(const double* a, const double* b,
                      const double* A_log, const double* dt_bias,
                      int64_t n_tokens, int64_t HV,
                      double* g, double* beta) {
    for (int64_t t = 0; t < n_tokens; ++t) {
        for (int64_t h = 0; h < HV; ++h) {
            const int64_t i = t * HV + h;
            g[i] = -exp(A_log[h]) * oracle_softplus(a[i] + dt_bias[h]);
            beta[i] = oracle_sigmoid(b[i]);
        }
    }
}

/* x <- x / sqrt(sum x^2 + 1e-6) into out (n elements). */
static void oracle_l2norm(const double* x, int64_t n, double* out) {
    double ss = 0.0;
    for (int64_t i = 0; i < n; ++i) ss += x[i] * x[i];
    const double r = 1.0 / sqrt(ss + 1e-6);
    for (int64_t i = 0; i < n; ++i) out[i] = x[i] * r;
}

/*
 * The recurrence over packed sequences.
 *   q, k : [T_total, HK, Dk]      v : [T_total, HV, Dv]
 *   g, beta : [T_total, HV]       (log-decay g, alpha = exp(g); write strength beta)
 *   h0   : [n_seqs, HV, Dk, Dv] (H = S^T) or NULL for zero initial states
 *   cu_seqlens : [n_seqs + 1], cu_seqlens[0] = 0, non-decreasing, last = T_total
 *   o    : [T_total, HV, Dv]      hT : [n_seqs, HV, Dk, Dv] (may be NULL)
 * Returns 0 on success, 1 on bad arguments, 2 on allocation failure.
 */
int gdn_oracle_recurrence(const double* q, const double* k, const double* v,
                          const double* g, const double* beta,
                          const double* h0, const int64_t* cu_seqlens,
                          int64_t n_seqs, int64_t HK, int64_t HV,
                          int64_t Dk, int64_t Dv, double scale, int l2norm,
                          double* o, double* hT, int n_threads) {
    if (!q || !k || !v || !g || !beta || !cu_seqlens || !o) return 1;
    if (n_seqs < 0 || HK <= 0 || HV <= 0 || Dk <= 0 || Dv <= 0 || HV % HK != 0) return 1;
    if (cu_seqlens[0] != 0) return 1;
    for (int64_t n = 0; n < n_seqs; ++n)
        if (cu_seqlens[n + 1] < cu_seqlens[n]) return 1;
    const int64_t group = HV / HK;
    const int64_t n_tasks = n_seqs * HV;
    int failed = 0;

#ifdef _OPENMP
    if (n_threads > 0) omp_set_num_threads(n_threads);
#pragma omp parallel for schedule(dynamic, 1) reduction(| : failed)
#endif
    for (int64_t task = 0; task < n_tasks; ++task) {
        const int64_t n = task / HV;
        const int64_t h = task % HV;
        const int64_t hk = h / group;
        double* S = (double*)malloc(sizeof(double) * (size_t)(Dv * Dk)); /* S[r][c], r<Dv, c<Dk */
        double* Sk = (double*)malloc(sizeof(double) * (size_t)Dv);
        double* qh = (double*)malloc(sizeof(double) * (size_t)Dk);
        double* kh = (double*)malloc(sizeof(double) * (size_t)Dk);
        if (!S || !Sk || !qh || !kh) {
            free(S); free(Sk); free(qh); free(kh);
            failed |= 1;
            continue;
        }
        /* S_0 = H_0^T */
        for (int64_t r = 0; r < Dv; ++r)
            for (int64_t c = 0; c < Dk; ++c)
                S[r * Dk + c] = h0 ? h0[((n * HV + h) * Dk + c) * Dv + r] : 0.0;

        for (int64_t t = cu_seqlens[n]; t < cu_seqlens[n + 1]; ++t) {
            const double* qt = q + (t * HK + hk) * Dk;
            const double* kt = k + (t * HK + hk) * Dk;
            const double* vt = v + (t * HV + h) * Dv;
            if (l2norm) {
                oracle_l2norm(qt, Dk, qh);
                oracle_l2norm(kt, Dk, kh);
            } else {
                memcpy(qh, qt, sizeof(double) * (size_t)Dk);
                memcpy(kh, kt, sizeof(double) * (size_t)Dk);
            }
            const double alpha = exp(g[t * HV + h]);
            const double bt = beta[t * HV + h];

            /* S_{t-1} k_t */
            for (int64_t r = 0; r < Dv; ++r) {
                double acc = 0.0;
                for (int64_t c = 0; c < Dk; ++c) acc += S[r * Dk + c] * kh[c];
                Sk[r] = acc;
            }
            /* S_t = S_{t-1} alpha (I - beta k k^T) + beta v k^T
             *     = alpha S_{t-1} - alpha beta (S_{t-1} k) k^T + beta v k^T   */
            for (int64_t r = 0; r < Dv; ++r)
                for (int64_t c = 0; c < Dk; ++c)
                    S[r * Dk + c] = alpha * S[r * Dk + c]
                                  - alpha * bt * Sk[r] * kh[c]
                                  + bt * vt[r] * kh[c];
            /* o_t = scale * S_t q_t */
            double* ot = o + (t * HV + h) * Dv;
            for (int64_t r = 0; r < Dv; ++r) {
                double acc = 0.0;
                for (int64_t c = 0; c < Dk; ++c) acc += S[r * Dk + c] * qh[c];
                ot[r] = scale * acc;
            }
        }
        if (hT)
            for (int64_t r = 0; r < Dv; ++r)
                for (int64_t c = 0; c < Dk; ++c)
                    hT[((n * HV + h) * Dk + c) * Dv + r] = S[r * Dk + c];
        free(S); free(Sk); free(qh); free(kh);
    }
    return failed ? 2 : 0;
}

/* Number of threads OpenMP would use (1 without OpenMP). */
/* Causal depthwise convolution of kernel 4 over B sequences of T tokens and C
 * channels.  x: [B, T, C]; w: [C, 4]; state_in: [B, C, 3] (oldest first) or NULL
 * for zeros; act 0 identity, 1 SiLU.  Outputs y: [B, T, C], state_out: [B, C, 3]. */
void gdn_oracle_conv(const double* x, const double* w, const double* state_in,
                     int64_t B, int64_t T, int64_t C, int act,
                     double* y, double* state_out) {
#pragma omp parallel for collapse(2) schedule(static)
    for (int64_t b = 0; b < B; ++b) {
        for (int64_t c = 0; c < C; ++c) {
            double win[4];   /* x_{t-3}, x_{t-2}, x_{t-1}, x_t */
            for (int i = 0; i < 3; ++i)
                win[i] = state_in ? state_in[(b * C + c) * 3 + i] : 0.0;
            for (int64_t t = 0; t < T; ++t) {
                win[3] = x[(b * T + t) * C + c];
                double acc = 0.0;
                for (int i = 0; i < 4; ++i) acc += w[c * 4 + i] * win[i];
                y[(b * T + t) * C + c] = act == 1 ? acc * oracle_sigmoid(acc) : acc;
                win[0] = win[1];
                win[1] = win[2];
                win[2] = win[3];
            }
            for (int i = 0; i < 3; ++i) state_out[(b * C + c) * 3 + i] = win[i];
        }
    }
}

/* Zero-centred RMSNorm and sigmoid gate of rows of length D.  o, z: [rows, D];
 * w: [D]; out: [rows, D]. */
void gdn_oracle_out_gate(const double* o, const double* z, const double* w, int64_t rows, int64_t D,
                         double eps, double* out) {
#pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < rows; ++r) {
        const double* x = o + r * D;
        double ss = 0.0;
        for (int64_t j = 0; j < D; ++j) ss += x[j] * x[j];
        const double inv = 1.0 / sqrt(ss / (double)D + eps);
        for (int64_t j = 0; j < D; ++j)
            out[r * D + j] = x[j] * inv * (1.0 + w[j]) * oracle_sigmoid(z[r * D + j]);
    }
}

int gdn_oracle_max_threads(void) {
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}
