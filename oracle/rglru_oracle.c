/*
 * rglru_oracle.c -- plain, sequential fp64 CPU oracle for the RG-LRU recurrent block
 * (causal depthwise conv1d on the x-branch -> RG-LRU -> multiply by GeLU of the y-branch).
 *
 * TEST INFRASTRUCTURE, NOT PRODUCT CODE.  Only tests/, __graft_entry__.smoke() and the
 * cpu_baseline / reference leg of bench.py may load this library.  It shares no code,
 * header, table or helper with the CUDA library; neither includes or calls the other.
 *
 * What it computes (sources are the pages' sections, cited by title):
 *
 *   [G] "Griffin Guide: RecurrentGemma, RG-LRU & Hybrid Attention" (aifetchly blog),
 *       section "1. Formulation of the RG-LRU Gating Mechanism": the four governing
 *       equations -- recurrence gate r_t = sigma(W_a x_t + b_a), input gate
 *       i_t = sigma(W_x x_t + b_x), dynamic diagonal decay a_t = a^(c r_t) with
 *       a = sigma(Lambda) and c = 8, state update h_t = a_t h_{t-1} + sqrt(1-a_t^2)(i_t x_t)
 *       -- plus the log-space form log a_t = -c r_t softplus(-Lambda).
 *   [V] same page, "2. The Role of Square-Root Variance Normalization".
 *   [F] same page, "3. Super-Exponential Context Preservation" (r_t = 0 freezes h).
 *   [C] same page, "1. Temporal Filtering via Separable 1D Convolutions" (width-4
 *       depthwise conv on branch 1, before the RG-LRU) and "2. Non-Linear Multiplicative
 *       Gating with GeLU" (z_t = y_t * GeLU(branch 2)).
 *   [B] same page, "3. Block-Diagonal Sharding for Zero-Communication Tensor
 *       Parallelism": W_a, W_x are block diagonal, one block per head.
 *   [L] same page, "1. PyTorch Implementation of RG-LRU and the Griffin Block": the
 *       conv output feeds the gates and the i_t * x_t product; the conv is PyTorch
 *       cross-correlation with left padding K-1 truncated to the first T outputs (so
 *       tap K-1 multiplies the current token); the (y, last_state) carry; zero state
 *       when none is given; exact-erf GeLU (F.gelu default).
 *
 * Readings where the pages are silent or disagree:
 *   - the listing clamps 1 - a^2 at 1e-7; that would contradict [F], so the oracle
 *     uses the exact sqrt(-expm1(2 log a_t)) (>= 0 because log a_t <= 0);
 *   - state h is fp64 here (fp32 on the GPU); the conv history (3 past x-branch inputs,
 *     oldest first) is part of the carried state;
 *   - a segment reset at token t empties the conv history and sets h_{t-1} := 0, then
 *     the normal update runs (equivalent to starting a new document from zero state);
 *   - W is stored per head as [in][out]: gate_o = b_o + sum_i xc_i * W[i][o].
 *
 * Arithmetic: inputs are widened exactly to fp64 (fp32 as is, bf16 by placing the 16
 * stored bits in the top half of an fp32), every operation is in fp64, in the order of
 * the definition: no blocking, fusion or reordering.
 *
 * Parity pins: every function here is pinned by tests/test_oracle_pins.py (closed form,
 * freeze, 0 < a_t < 1, variance preservation, brute-force unrolling, dense-matrix gates,
 * torch conv1d, reset = separate documents, prefill/decode and split-prefill identities,
 * GeLU spot values).
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#ifdef _OPENMP
#include <omp.h>
#endif

#define ORACLE_CONV_WIDTH 4   /* [C]: "small temporal kernel width of k = 4" */
#define ORACLE_HIST (ORACLE_CONV_WIDTH - 1)

enum { ORACLE_F32 = 0, ORACLE_BF16 = 1, ORACLE_F64 = 2 };

/* Exact fp64 value of element idx: fp32, bf16 bits, or (for the layer oracle, whose projections
 * produce fp64 activations) fp64 as is. */
static double widen(const void* p, long idx, int dtype) {
    if (dtype == ORACLE_F64) return ((const double*)p)[idx];
    if (dtype == ORACLE_F32) return (double)((const float*)p)[idx];
    uint32_t bits = ((uint32_t)((const uint16_t*)p)[idx]) << 16;
    float f;
    memcpy(&f, &bits, sizeof f);
    return (double)f;
}

/* sigma(z) = 1 / (1 + e^{-z}) [G], evaluated on the side that cannot overflow. */
static double sigmoid(double z) {
    if (z >= 0.0) return 1.0 / (1.0 + exp(-z));
    double e = exp(z);
    return e / (1.0 + e);
}

/* log sigma(Lambda) = -softplus(-Lambda) [G, log-space form], overflow-free form. */
static double log_sigmoid(double z) {
    return fmin(z, 0.0) - log1p(exp(-fabs(z)));
}

/* GeLU [C]/[L]: exact v Phi(v) = 0.5 v (1 + erf(v / sqrt 2)), evaluated as
 * 0.5 v erfc(-v / sqrt 2) (the same value without cancellation for v << 0); tanh_form
 * selects the tanh approximation 0.5 v (1 + tanh(sqrt(2/pi) (v + 0.044715 v^3))). */
double rglru_oracle_gelu(double v, int tanh_form) {
    if (tanh_form) {
        const double pi = 3.14159265358979323846;
        const double k = sqrt(2.0 / pi);
        return 0.5 * v * (1.0 + tanh(k * (v + 0.044715 * v * v * v)));
    }
    return 0.5 * v * erfc(-v / sqrt(2.0));
}

/*
 * One (batch row, head) sequence of T tokens over the head's dh channels.
 *
 *   conv_w  [4][conv_ld] fp32, base at the head's first channel; tap 3 = current token
 *   conv_b  [dh] fp32 or NULL (= 0)
 *   w_a,w_x [dh][dh] (in-major) in w_dtype (0 = fp32, 1 = bf16 bits)
 *   b_a,b_x [dh] fp32 or NULL (= 0);  lambda [dh] fp32
 *   x, y    [T][ld] in act_dtype, base at the head's first channel
 *   reset   [T] or NULL; reset[t] != 0 means token t starts a new segment
 *   h       [dh] fp64, in: state before token 0, out: state after token T-1
 *   tail    [3][tail_ld] fp64, in/out: conv history x_{t-3}, x_{t-2}, x_{t-1}
 *   out     [T][out_ld] fp64
 *   a_out   [T][dh] fp64 or NULL: the decay factors a_t (for invariant tests)
 * Returns 0, or -1 on a bad size.
 */
int rglru_oracle_prefill_unit(int T, int dh, double c, int gelu_tanh, int act_dtype,
                              const float* conv_w, long conv_ld, const float* conv_b,
                              const void* w_a, const void* w_x, int w_dtype,
                              const float* b_a, const float* b_x, const float* lambda,
                              const void* x, const void* y, long ld,
                              const uint8_t* reset,
                              double* h, double* tail, long tail_ld,
                              double* out, long out_ld, double* a_out) {
    if (T < 0 || dh <= 0) return -1;
    double* xc = (double*)malloc(sizeof(double) * (size_t)dh * 4);
    if (!xc) return -1;
    double* log_a_base = xc + dh;
    double* ga = xc + 2 * dh;
    double* gx = xc + 3 * dh;
    for (int j = 0; j < dh; ++j) log_a_base[j] = log_sigmoid((double)lambda[j]);

    for (int t = 0; t < T; ++t) {
        /* segment reset: the new document sees neither old state nor old conv inputs */
        if (reset && reset[t]) {
            for (int j = 0; j < dh; ++j) h[j] = 0.0;
            for (int k = 0; k < ORACLE_HIST; ++k)
                for (int j = 0; j < dh; ++j) tail[k * tail_ld + j] = 0.0;
        }
        /* causal depthwise conv [C][L]: xc_t = b + sum_k w[k] * x_{t-3+k} */
        for (int j = 0; j < dh; ++j) {
            double xt = widen(x, (long)t * ld + j, act_dtype);
            double acc = conv_b ? (double)conv_b[j] : 0.0;
            for (int k = 0; k < ORACLE_HIST; ++k)
                acc += (double)conv_w[k * conv_ld + j] * tail[k * tail_ld + j];
            acc += (double)conv_w[ORACLE_HIST * conv_ld + j] * xt;
            xc[j] = acc;
            for (int k = 0; k + 1 < ORACLE_HIST; ++k) tail[k * tail_ld + j] = tail[(k + 1) * tail_ld + j];
            tail[(ORACLE_HIST - 1) * tail_ld + j] = xt;
        }
        /* gate pre-activations [G][B]: gate_o = b_o + sum_i xc_i W[i][o]; every sum runs
         * over i = 0..dh-1 in order (the i loop is outside only so W is read row by row) */
        for (int o = 0; o < dh; ++o) {
            ga[o] = b_a ? (double)b_a[o] : 0.0;
            gx[o] = b_x ? (double)b_x[o] : 0.0;
        }
        for (int i = 0; i < dh; ++i) {
            const double xi = xc[i];
            for (int o = 0; o < dh; ++o) {
                ga[o] += xi * widen(w_a, (long)i * dh + o, w_dtype);
                gx[o] += xi * widen(w_x, (long)i * dh + o, w_dtype);
            }
        }
        /* gates, decay and state update [G][V], then the GeLU merge [C] */
        for (int o = 0; o < dh; ++o) {
            double r = sigmoid(ga[o]);
            double ig = sigmoid(gx[o]);
            double log_a = c * r * log_a_base[o];         /* log a_t = c r_t log sigma(Lambda) */
            double a = exp(log_a);
            double beta = sqrt(-expm1(2.0 * log_a));        /* sqrt(1 - a_t^2) */
            h[o] = a * h[o] + beta * (ig * xc[o]);
            if (a_out) a_out[(long)t * dh + o] = a;
            double yv = widen(y, (long)t * ld + o, act_dtype);
            out[(long)t * out_ld + o] = h[o] * rglru_oracle_gelu(yv, gelu_tanh);
        }
    }
    free(xc);
    return 0;
}

/*
 * Whole batch, layout [B][T][W] with W = H * dh (channel ch = head * dh + j).
 * h [B][W] and tail [B][3][W] are in/out; when h is NULL the state starts at zero and
 * the final state is discarded.  units (n_units pairs of (b, head)) restricts the work to
 * those sequences (NULL = all).  Sequences are independent [B], so they run in parallel
 * over n_threads OpenMP threads (<= 0: the runtime default); each one is sequential.
 */
int rglru_oracle_prefill(int B, int T, int H, int dh, double c, int gelu_tanh, int act_dtype,
                         const float* conv_w, const float* conv_b,
                         const void* w_a, const void* w_x,
                         const float* b_a, const float* b_x, const float* lambda,
                         const void* x, const void* y, const uint8_t* reset,
                         double* h, double* tail, double* out,
                         const int* units, int n_units, int n_threads) {
    if (B < 0 || T < 0 || H <= 0 || dh <= 0) return -1;
    const long W = (long)H * dh;
    const int total = units ? n_units : B * H;
    int status = 0;
#ifdef _OPENMP
    if (n_threads <= 0) n_threads = omp_get_max_threads();
#pragma omp parallel for schedule(dynamic, 1) num_threads(n_threads) reduction(| : status)
#endif
    for (int u = 0; u < total; ++u) {
        int b = units ? units[2 * u] : u / H;
        int hd = units ? units[2 * u + 1] : u % H;
        long ch0 = (long)hd * dh;
        double* hs = NULL;
        double* ts = NULL;
        double* hbuf = NULL;
        if (h) {
            hs = h + (long)b * W + ch0;
            ts = tail + (long)b * ORACLE_HIST * W + ch0;
        } else {
            hbuf = (double*)calloc((size_t)dh * (1 + ORACLE_HIST), sizeof(double));
            hs = hbuf;
            ts = hbuf + dh;
        }
        long wsz = (long)dh * dh;
        int rc = rglru_oracle_prefill_unit(
            T, dh, c, gelu_tanh, act_dtype, conv_w + ch0, W, conv_b ? conv_b + ch0 : NULL,
            (const char*)w_a + (size_t)hd * wsz * (act_dtype == ORACLE_F32 ? 4 : 2),
            (const char*)w_x + (size_t)hd * wsz * (act_dtype == ORACLE_F32 ? 4 : 2), act_dtype,
            b_a ? b_a + ch0 : NULL, b_x ? b_x + ch0 : NULL, lambda + ch0,
            (const char*)x + (size_t)((long)b * T * W + ch0) * (act_dtype == ORACLE_F32 ? 4 : 2),
            (const char*)y + (size_t)((long)b * T * W + ch0) * (act_dtype == ORACLE_F32 ? 4 : 2), W,
            reset ? reset + (long)b * T : NULL, hs, ts, h ? W : dh,
            out + (long)b * T * W + ch0, W, NULL);
        free(hbuf);
        status |= (rc != 0);
    }
    return status ? -1 : 0;
}

/*
 * One decode step for the whole batch: the same definition with T = 1 [L, RGLRU.step],
 * carrying h [B][W] and the conv history tail [B][3][W] (both in/out).  reset [B] or NULL:
 * reset[b] != 0 empties row b's state before the step.  x, y [B][W]; out [B][W].
 */
int rglru_oracle_decode(int B, int H, int dh, double c, int gelu_tanh, int act_dtype,
                        const float* conv_w, const float* conv_b,
                        const void* w_a, const void* w_x,
                        const float* b_a, const float* b_x, const float* lambda,
                        const void* x, const void* y, const uint8_t* reset,
                        double* h, double* tail, double* out, int n_threads) {
    if (B < 0 || H <= 0 || dh <= 0 || !h || !tail) return -1;
    const long W = (long)H * dh;
    const size_t es = act_dtype == ORACLE_F32 ? 4 : 2;
    int status = 0;
#ifdef _OPENMP
    if (n_threads <= 0) n_threads = omp_get_max_threads();
#pragma omp parallel for schedule(dynamic, 1) num_threads(n_threads) reduction(| : status)
#endif
    for (int u = 0; u < B * H; ++u) {
        int b = u / H, hd = u % H;
        long ch0 = (long)hd * dh;
        long wsz = (long)dh * dh;
        int rc = rglru_oracle_prefill_unit(
            1, dh, c, gelu_tanh, act_dtype, conv_w + ch0, W, conv_b ? conv_b + ch0 : NULL,
            (const char*)w_a + (size_t)hd * wsz * es, (const char*)w_x + (size_t)hd * wsz * es,
            act_dtype, b_a ? b_a + ch0 : NULL, b_x ? b_x + ch0 : NULL, lambda + ch0,
            (const char*)x + (size_t)((long)b * W + ch0) * es,
            (const char*)y + (size_t)((long)b * W + ch0) * es, W,
            reset ? reset + b : NULL, h + (long)b * W + ch0,
            tail + (long)b * ORACLE_HIST * W + ch0, W, out + (long)b * W + ch0, W, NULL);
        status |= (rc != 0);
    }
    return status ? -1 : 0;
}

/* ------------------------------------------------------------------------------------------
 * Backward pass of the block: the exact fp64 gradients of
 *     L = sum_t <dout_t, z_t> + <dh_final, h_{T-1}> + <dtail_final, tail_T>
 * with respect to x, y, the parameters and the initial state, for the forward defined above
 * (chain rule through the same equations; no source states them, they follow from [G], [V],
 * [C], [B], [L] and the readings above).  The per-token quantities of the forward
 * (xc_t, h_{t-1}, r_t, i_t, a_t, beta_t) are kept in full, then a reverse pass carries
 * g = dL/dh_t:
 *     g_t      = dout_t GeLU(y_t) + a_{t+1} g_{t+1}      (0 across a reset: h_{t-1} := 0)
 *     dy_t     = dout_t h_t GeLU'(y_t)
 *     dL/da_t  = g_t h_{t-1},   dL/dbeta_t = g_t i_t xc_t,   dL/di_t = g_t beta_t xc_t
 *     log a_t  = kappa r_t with kappa = c log sigma(Lambda);  da/dlog a = a,
 *     dbeta/dlog a = -a^2 / beta;  with Q = dL/da a r - dL/dbeta a^2 (r / beta):
 *     dL/dga_t = kappa (1 - r_t) Q,   dL/dLambda += c sigma(-Lambda) Q,
 *     dL/dgx_t = dL/di_t i_t (1 - i_t)
 *     dxc_t    = g_t beta_t i_t + W_a dga_t + W_x dgx_t,  dW[i][o] += xc_t[i] dg_t[o]
 * (r / beta is taken as 0 where beta = 0, its limit: r -> 0 or kappa -> 0), and the conv's
 * transpose scatters dxc_t to the inputs its window read (x, or the initial history), with
 * the final history's gradient added to the inputs it copied.
 * ------------------------------------------------------------------------------------------ */

/* W[i][o] of one head's [dh][dh] block (in-major), widened to fp64 */
static double weight_at(const void* w, int i, int o, int dh, int dtype) {
    return widen(w, (long)i * dh + o, dtype);
}

static double gelu_grad(double v, int tanh_form) {
    const double pi = 3.14159265358979323846;
    if (tanh_form) {
        const double k = sqrt(2.0 / pi);
        double th = tanh(k * (v + 0.044715 * v * v * v));
        return 0.5 * (1.0 + th) + 0.5 * v * (1.0 - th * th) * k * (1.0 + 3.0 * 0.044715 * v * v);
    }
    /* d/dv [v Phi(v)] = Phi(v) + v phi(v) */
    return 0.5 * erfc(-v / sqrt(2.0)) + v * exp(-0.5 * v * v) / sqrt(2.0 * pi);
}

/* Window value x~ of tap position s seen from token t (s in [t-3, t]): x_s when no reset lies
 * in (s, t]; for s < 0 the initial history tail0[3 + s] (0 without one). *src receives the
 * position it came from (s, or -1 for zero / reset). */
static double window_value(int t, int s, const uint8_t* reset, const void* x, long ld, int dtype,
                           const double* tail0, long tail_ld, int j, int* src) {
    for (int p = (s + 1 > 0 ? s + 1 : 0); p <= t; ++p)
        if (reset && reset[p]) { *src = -4; return 0.0; }
    *src = s;
    if (s >= 0) return widen(x, (long)s * ld + j, dtype);
    return tail0 ? tail0[(ORACLE_HIST + s) * tail_ld + j] : 0.0;
}

/*
 * One (batch row, head) sequence; arguments as rglru_oracle_prefill_unit, plus
 *   h0 [dh], tail0 [3][tail_ld] fp64 or NULL (= zero initial state)
 *   dout [T][ld] in act_dtype;  dh_final [dh], dtail_final [3][tail_ld] fp64 or NULL (= 0)
 *   dx, dy [T][ld] fp64 (written);  dh0 [dh], dtail0 [3][tail_ld] fp64 (written)
 *   dconv_w [4][conv_ld], dconv_b, db_a, db_x, dlambda [dh], dw_a, dw_x [dh][dh] fp64:
 *   this sequence's terms are ADDED (the caller sums over sequences).
 */
int rglru_oracle_backward_unit(int T, int dh, double c, int gelu_tanh, int act_dtype,
                               const float* conv_w, long conv_ld, const float* conv_b,
                               const void* w_a, const void* w_x, int w_dtype,
                               const float* b_a, const float* b_x, const float* lambda,
                               const void* x, const void* y, long ld, const uint8_t* reset,
                               const double* h0, const double* tail0, long tail_ld,
                               const void* dout, const double* dh_final, const double* dtail_final,
                               double* dx, double* dy, double* dh0, double* dtail0,
                               double* dconv_w, double* dconv_b, double* dw_a, double* dw_x,
                               double* db_a, double* db_x, double* dlambda) {
    if (T < 1 || dh <= 0) return -1;
    const size_t n = (size_t)T * dh;
    double* xc = (double*)calloc(n * 6 + (size_t)dh * 6, sizeof(double));
    if (!xc) return -1;
    double* hprev = xc + n;      /* h_{t-1} as used by the update (0 after a reset) */
    double* hcur = hprev + n;    /* h_t */
    double* rr = hcur + n;
    double* ii = rr + n;
    double* dxc = ii + n;
    double* g = dxc + n;
    double* dga = g + dh;
    double* dgx = dga + dh;
    double* kappa = dgx + dh;
    double* hs = kappa + dh;
    double* sgn = hs + dh;       /* sigma(-Lambda) */

    for (int j = 0; j < dh; ++j) {
        kappa[j] = c * log_sigmoid((double)lambda[j]);
        sgn[j] = sigmoid(-(double)lambda[j]);
        hs[j] = h0 ? h0[j] : 0.0;
    }
    /* ---- forward, keeping every per-token quantity ---- */
    for (int t = 0; t < T; ++t) {
        double* xct = xc + (size_t)t * dh;
        for (int j = 0; j < dh; ++j) {
            double acc = (conv_b != NULL) ? (double)conv_b[j] : 0.0;
            for (int k = 0; k < ORACLE_CONV_WIDTH; ++k) {
                int src;
                acc += (double)conv_w[k * conv_ld + j] *
                       window_value(t, t - ORACLE_HIST + k, reset, x, ld, act_dtype, tail0, tail_ld, j, &src);
            }
            xct[j] = acc;
        }
        for (int o = 0; o < dh; ++o) {
            double ga = b_a ? (double)b_a[o] : 0.0, gx = b_x ? (double)b_x[o] : 0.0;
            for (int i = 0; i < dh; ++i) {
                ga += xct[i] * weight_at(w_a, i, o, dh, w_dtype);
                gx += xct[i] * weight_at(w_x, i, o, dh, w_dtype);
            }
            double r = sigmoid(ga), ig = sigmoid(gx);
            double la = kappa[o] * r, a = exp(la), beta = sqrt(-expm1(2.0 * la));
            double hp = (reset && reset[t]) ? 0.0 : hs[o];
            hs[o] = a * hp + beta * (ig * xct[o]);
            rr[(size_t)t * dh + o] = r;
            ii[(size_t)t * dh + o] = ig;
            hprev[(size_t)t * dh + o] = hp;
            hcur[(size_t)t * dh + o] = hs[o];
        }
    }
    /* ---- reverse pass over the recurrence and the gates ---- */
    for (int j = 0; j < dh; ++j) g[j] = dh_final ? dh_final[j] : 0.0;
    for (int t = T - 1; t >= 0; --t) {
        const double* xct = xc + (size_t)t * dh;
        for (int o = 0; o < dh; ++o) {
            const size_t e = (size_t)t * dh + o;
            double yv = widen(y, (long)t * ld + o, act_dtype);
            double dz = widen(dout, (long)t * ld + o, act_dtype);
            g[o] += dz * rglru_oracle_gelu(yv, gelu_tanh);
            dy[(long)t * ld + o] = dz * hcur[e] * gelu_grad(yv, gelu_tanh);
            double r = rr[e], ig = ii[e];
            double la = kappa[o] * r, a = exp(la), beta = sqrt(-expm1(2.0 * la));
            double dl_da = g[o] * hprev[e];
            double dl_dbeta = g[o] * ig * xct[o];
            double dl_di = g[o] * beta * xct[o];
            double r_over_beta = beta > 0.0 ? r / beta : 0.0;
            double q = dl_da * a * r - dl_dbeta * a * a * r_over_beta;
            dga[o] = kappa[o] * (1.0 - r) * q;
            dgx[o] = dl_di * ig * (1.0 - ig);
            dlambda[o] += c * sgn[o] * q;
            db_a[o] += dga[o];
            db_x[o] += dgx[o];
            dxc[e] = g[o] * beta * ig;
        }
        for (int i = 0; i < dh; ++i) {
            double acc = 0.0;
            for (int o = 0; o < dh; ++o) {
                acc += weight_at(w_a, i, o, dh, w_dtype) * dga[o];
                acc += weight_at(w_x, i, o, dh, w_dtype) * dgx[o];
                dw_a[(long)i * dh + o] += xct[i] * dga[o];
                dw_x[(long)i * dh + o] += xct[i] * dgx[o];
            }
            dxc[(size_t)t * dh + i] += acc;
        }
        /* g becomes dL/dh_{t-1}; a reset at t cut h_{t-1} out of the update */
        for (int o = 0; o < dh; ++o) {
            double a = exp(kappa[o] * rr[(size_t)t * dh + o]);
            g[o] = (reset && reset[t]) ? 0.0 : a * g[o];
        }
    }
    for (int j = 0; j < dh; ++j) dh0[j] = g[j];
    /* ---- conv transpose: scatter dxc_t to the window inputs ---- */
    for (int t = 0; t < T; ++t)
        for (int j = 0; j < dh; ++j) dx[(long)t * ld + j] = 0.0;
    for (int k = 0; k < ORACLE_HIST; ++k)
        for (int j = 0; j < dh; ++j) dtail0[k * tail_ld + j] = 0.0;
    for (int t = 0; t < T; ++t) {
        for (int j = 0; j < dh; ++j) {
            double d = dxc[(size_t)t * dh + j];
            dconv_b[j] += d;
            for (int k = 0; k < ORACLE_CONV_WIDTH; ++k) {
                int src;
                double v = window_value(t, t - ORACLE_HIST + k, reset, x, ld, act_dtype, tail0, tail_ld, j, &src);
                dconv_w[k * conv_ld + j] += d * v;
                if (src >= 0) dx[(long)src * ld + j] += (double)conv_w[k * conv_ld + j] * d;
                else if (src > -4) dtail0[(ORACLE_HIST + src) * tail_ld + j] += (double)conv_w[k * conv_ld + j] * d;
            }
        }
    }
    /* ---- the final history is a copy of the last three window inputs seen from T-1 ---- */
    if (dtail_final) {
        for (int k = 0; k < ORACLE_HIST; ++k)
            for (int j = 0; j < dh; ++j) {
                int src;
                (void)window_value(T - 1, T - ORACLE_HIST + k, reset, x, ld, act_dtype, tail0, tail_ld, j, &src);
                double d = dtail_final[k * tail_ld + j];
                if (src >= 0) dx[(long)src * ld + j] += d;
                else if (src > -4) dtail0[(ORACLE_HIST + src) * tail_ld + j] += d;
            }
    }
    free(xc);
    return 0;
}

/*
 * Whole batch [B][T][W]; h0 [B][W], tail0 [B][3][W], dh_final [B][W], dtail_final [B][3][W]
 * fp64 or NULL; dout [B][T][W] act dtype.  Outputs fp64: dx, dy [B][T][W]; dh0 [B][W];
 * dtail0 [B][3][W]; dconv_w [4][W]; dconv_b, db_a, db_x, dlambda [W]; dw_a, dw_x [H][dh][dh]
 * (all overwritten).  Sequential over (b, head): the parameter sums run in that order.
 */
int rglru_oracle_backward(int B, int T, int H, int dh, double c, int gelu_tanh, int act_dtype,
                          const float* conv_w, const float* conv_b,
                          const void* w_a, const void* w_x,
                          const float* b_a, const float* b_x, const float* lambda,
                          const void* x, const void* y, const uint8_t* reset,
                          const double* h0, const double* tail0, const void* dout,
                          const double* dh_final, const double* dtail_final,
                          double* dx, double* dy, double* dh0, double* dtail0,
                          double* dconv_w, double* dconv_b, double* dw_a, double* dw_x,
                          double* db_a, double* db_x, double* dlambda) {
    if (B < 0 || T < 1 || H <= 0 || dh <= 0) return -1;
    const long W = (long)H * dh;
    const size_t es = act_dtype == ORACLE_F32 ? 4 : 2;
    const long wsz = (long)dh * dh;
    memset(dconv_w, 0, sizeof(double) * 4 * W);
    memset(dconv_b, 0, sizeof(double) * W);
    memset(db_a, 0, sizeof(double) * W);
    memset(db_x, 0, sizeof(double) * W);
    memset(dlambda, 0, sizeof(double) * W);
    memset(dw_a, 0, sizeof(double) * H * wsz);
    memset(dw_x, 0, sizeof(double) * H * wsz);
    for (int b = 0; b < B; ++b)
        for (int hd = 0; hd < H; ++hd) {
            long ch0 = (long)hd * dh;
            int rc = rglru_oracle_backward_unit(
                T, dh, c, gelu_tanh, act_dtype, conv_w + ch0, W, conv_b ? conv_b + ch0 : NULL,
                (const char*)w_a + (size_t)hd * wsz * es, (const char*)w_x + (size_t)hd * wsz * es,
                act_dtype, b_a ? b_a + ch0 : NULL, b_x ? b_x + ch0 : NULL, lambda + ch0,
                (const char*)x + (size_t)((long)b * T * W + ch0) * es,
                (const char*)y + (size_t)((long)b * T * W + ch0) * es, W,
                reset ? reset + (long)b * T : NULL,
                h0 ? h0 + (long)b * W + ch0 : NULL,
                tail0 ? tail0 + (long)b * ORACLE_HIST * W + ch0 : NULL, W,
                (const char*)dout + (size_t)((long)b * T * W + ch0) * es,
                dh_final ? dh_final + (long)b * W + ch0 : NULL,
                dtail_final ? dtail_final + (long)b * ORACLE_HIST * W + ch0 : NULL,
                dx + (long)b * T * W + ch0, dy + (long)b * T * W + ch0,
                dh0 + (long)b * W + ch0, dtail0 + (long)b * ORACLE_HIST * W + ch0,
                dconv_w + ch0, dconv_b + ch0, dw_a + hd * wsz, dw_x + hd * wsz,
                db_a + ch0, db_x + ch0, dlambda + ch0);
            if (rc != 0) return -1;
        }
    return 0;
}
