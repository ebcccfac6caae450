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

enum { ORACLE_F32 = 0, ORACLE_BF16 = 1 };

static double widen(const void* p, long idx, int dtype) {
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
