// backward.cu -- gradients of the RG-LRU block (CUDA cores, accurate fp32 math).
//
// For the prefill of x, y [B, T, W] from an initial state, the gradients of
//     L = <dout, out> + <dh_final, h_{T-1}> + <dtail_final, tail_T>
// with respect to x, y, every parameter and the initial state.  The forward is the one the
// pages define ("Griffin Guide: RecurrentGemma, RG-LRU & Hybrid Attention": "1. Formulation of
// the RG-LRU Gating Mechanism", "2. The Role of Square-Root Variance Normalization",
// "1. Temporal Filtering via Separable 1D Convolutions", "2. Non-Linear Multiplicative Gating
// with GeLU", "3. Block-Diagonal Sharding ..."); the pages state no backward, so these kernels
// apply the chain rule to those equations.  Four launches:
//
//   1. bwd_forward_kernel: one CTA per (row, head) runs the forward again in 32-token tiles
//      (conv, FFMA gate contraction, scan) and keeps, per token-channel, the conv output xc_t,
//      the gate pre-activations and h_{t-1} in the workspace;
//   2. bwd_reverse_kernel: one CTA per (row, head) walks the tiles backwards carrying
//      g = dL/dh_t per channel:  g_t = dout_t GeLU(y_t) + a_{t+1} g_{t+1} (0 across a reset),
//      dy_t = dout_t h_t GeLU'(y_t);  with Q = g h_{t-1} a r - g i xc a^2 (r / beta) it forms
//      dL/dga = c log sigma(Lambda) (1 - r) Q and dL/dgx = g beta xc i (1 - i), overwriting the
//      pre-activations with them; dxc = g beta i + W_a dga + W_x dgx (a per-tile FFMA
//      contraction with the weights' rows); then the conv's transpose: dx_s gathers
//      w_k dxc_{s+3-k} over the windows that read x_s (the next tile's first three dxc carried
//      across), the initial history gets the taps that read it, and the final history's
//      gradient goes to the inputs it copied.  Per-(row, channel) partial sums of dLambda, db_a,
//      db_x, dconv_b, dconv_w go to the workspace;
//   3. bwd_weight_kernel: dW[h][i][o] = sum over (b, t) of xc[i] dg[o] for both gates, a
//      16 x 16 output tile per CTA reduced over the B T tokens in a fixed order;
//   4. bwd_reduce_kernel: the partial sums over the batch rows, in row order.
//
// No atomics: every sum runs in a fixed order, so the gradients are bitwise repeatable.
// r / beta is taken as 0 where beta = 0 (r = 0, or log sigma(Lambda) = 0), its limit.
#include "common.cuh"
#include "kernels.h"

namespace rglru {

namespace {

constexpr int kThreads = 256;
constexpr int kTile = 32;
constexpr int kParts = 4 + kConvWidth;   // dLambda, db_a, db_x, dconv_b, dconv_w[4]

struct BwdArgs {
    int B, T, H, dh;
    float c;
    int gelu_tanh;
    const float* conv_w;
    const float* conv_b;
    const void* w_a;
    const void* w_x;
    const float* b_a;
    const float* b_x;
    const float* lambda;
    const void* x;
    const void* y;
    const uint8_t* reset;
    const float* h0;          // initial state h [B, W] or nullptr (zero)
    const void* tail0;        // initial conv history [B, 3, W] (act dtype) or nullptr (zero)
    const void* dout;
    const float* dh_final;    // [B, W] or nullptr
    const float* dtail_final; // [B, 3, W] or nullptr
    float* xc;                // workspace [B, T, W]
    float* hprev;             // workspace [B, T, W]: h_{t-1} as the update used it
    float* ga;                // workspace [B, T, W]: gate-a pre-activation, then dL/dga
    float* gx;                // workspace [B, T, W]: gate-x pre-activation, then dL/dgx
    float* part;              // workspace [kParts][B][W]
    rglru_grads g;
};

// d/dv [v Phi(v)] = Phi(v) + v phi(v); the tanh form's derivative for the flag
__device__ __forceinline__ float gelu_grad_acc(float v, int tanh_form) {
    if (tanh_form) {
        const float k = 0.79788456080286535588f;
        const float th = tanhf(k * (v + 0.044715f * v * v * v));
        return 0.5f * (1.0f + th) + 0.5f * v * (1.0f - th * th) * k * (1.0f + 3.0f * 0.044715f * v * v);
    }
    return 0.5f * erfcf(-v * 0.70710678118654752440f) + v * expf(-0.5f * v * v) * 0.39894228040143267794f;
}

// True when the window of token t may read position s (s in [t-3, t]): no reset in (s, t].
__device__ __forceinline__ bool window_reads(const BwdArgs& a, int b, int s, int t) {
    if (!a.reset) return true;
    for (int p = (s + 1 > 0 ? s + 1 : 0); p <= t; ++p)
        if (a.reset[(size_t)b * a.T + p]) return false;
    return true;
}

// The value the window of token t reads at position s: x_s, or the initial history for s < 0.
template <typename T>
__device__ __forceinline__ float window_value(const BwdArgs& a, int b, int s, int t, int ch, int W) {
    if (!window_reads(a, b, s, t)) return 0.0f;
    if (s >= 0) return Act<T>::load(static_cast<const T*>(a.x) + ((size_t)b * a.T + s) * W + ch);
    if (!a.tail0) return 0.0f;
    return Act<T>::load(static_cast<const T*>(a.tail0) + ((size_t)b * kHist + (kHist + s)) * W + ch);
}

// ---------------------------------------------------------------- 1. forward, kept ---------
template <typename T>
__global__ void __launch_bounds__(kThreads) bwd_forward_kernel(BwdArgs a) {
    extern __shared__ float smem[];
    const int hd = blockIdx.x, b = blockIdx.y;
    const int dh = a.dh, W = a.H * dh, ch0 = hd * dh;
    float* xc_s = smem;                      // [kTile][dh]
    float* a_s = xc_s + kTile * dh;          // [kTile][dh]
    float* u_s = a_s + kTile * dh;           // [kTile][dh]
    const T* w_a = static_cast<const T*>(a.w_a) + (size_t)hd * dh * dh;
    const T* w_x = static_cast<const T*>(a.w_x) + (size_t)hd * dh * dh;

    const int groups = kThreads / dh;
    const int o = threadIdx.x % dh, grp = threadIdx.x / dh, ch = ch0 + o;
    const bool scan_thread = threadIdx.x < dh;
    float c_lab = 0.f, ba = 0.f, bx = 0.f, hreg = 0.f;
    if (grp < groups) {
        c_lab = a.c * log_sigmoid_acc(a.lambda[ch]);
        ba = a.b_a ? a.b_a[ch] : 0.f;
        bx = a.b_x ? a.b_x[ch] : 0.f;
    }
    if (scan_thread && a.h0) hreg = a.h0[(size_t)b * W + ch];

    for (int t0 = 0; t0 < a.T; t0 += kTile) {
        const int nt = min(kTile, a.T - t0);
        for (int e = threadIdx.x; e < nt * dh; e += kThreads) {
            const int tt = e / dh, j = e % dh, t = t0 + tt, c2 = ch0 + j;
            float acc = a.conv_b ? a.conv_b[c2] : 0.f;
#pragma unroll
            for (int k = 0; k < kConvWidth; ++k)
                acc += a.conv_w[(size_t)k * W + c2] * window_value<T>(a, b, t - kHist + k, t, c2, W);
            xc_s[tt * dh + j] = acc;
            a.xc[((size_t)b * a.T + t) * W + c2] = acc;
        }
        __syncthreads();
        if (grp < groups) {
            float acc_a[kTile], acc_x[kTile];
#pragma unroll
            for (int q = 0; q < kTile; ++q) { acc_a[q] = ba; acc_x[q] = bx; }
            for (int i = 0; i < dh; ++i) {
                const float wa = Act<T>::load(w_a + (size_t)i * dh + o);
                const float wx = Act<T>::load(w_x + (size_t)i * dh + o);
#pragma unroll
                for (int q = 0; q < kTile; ++q) {
                    const int tt = grp + q * groups;
                    if (q * groups < kTile && tt < nt) {
                        const float v = xc_s[tt * dh + i];
                        acc_a[q] = fmaf(v, wa, acc_a[q]);
                        acc_x[q] = fmaf(v, wx, acc_x[q]);
                    }
                }
            }
#pragma unroll
            for (int q = 0; q < kTile; ++q) {
                const int tt = grp + q * groups;
                if (q * groups < kTile && tt < nt) {
                    const size_t e = ((size_t)b * a.T + t0 + tt) * W + ch;
                    a.ga[e] = acc_a[q];
                    a.gx[e] = acc_x[q];
                    float at, beta;
                    decay_and_beta_acc(c_lab, sigmoid_acc(acc_a[q]), &at, &beta);
                    a_s[tt * dh + o] = at;
                    u_s[tt * dh + o] = beta * (sigmoid_acc(acc_x[q]) * xc_s[tt * dh + o]);
                }
            }
        }
        __syncthreads();
        if (scan_thread) {
            for (int tt = 0; tt < nt; ++tt) {
                const size_t e = ((size_t)b * a.T + t0 + tt) * W + ch;
                const float hp = (a.reset && a.reset[(size_t)b * a.T + t0 + tt]) ? 0.f : hreg;
                a.hprev[e] = hp;
                hreg = fmaf(a_s[tt * dh + o], hp, u_s[tt * dh + o]);
            }
        }
        __syncthreads();
    }
}

// ---------------------------------------------------------------- 2. reverse pass ----------
template <typename T>
__global__ void __launch_bounds__(kThreads) bwd_reverse_kernel(BwdArgs a) {
    extern __shared__ float smem[];
    const int hd = blockIdx.x, b = blockIdx.y;
    const int dh = a.dh, W = a.H * dh, ch0 = hd * dh;
    float* dga_s = smem;                     // [kTile][dh]
    float* dgx_s = dga_s + kTile * dh;       // [kTile][dh]
    float* dxc_s = dgx_s + kTile * dh;       // [kTile][dh]
    const T* w_a = static_cast<const T*>(a.w_a) + (size_t)hd * dh * dh;
    const T* w_x = static_cast<const T*>(a.w_x) + (size_t)hd * dh * dh;
    const T* y = static_cast<const T*>(a.y);
    const T* dout = static_cast<const T*>(a.dout);

    const int groups = kThreads / dh;
    const bool scan_thread = threadIdx.x < dh;
    const int o = threadIdx.x % dh, grp = threadIdx.x / dh, ch = ch0 + o;

    // per-channel state of the scan threads
    float kappa = 0.f, c_sneg = 0.f, g = 0.f;
    float s_lam = 0.f, s_ba = 0.f, s_bx = 0.f, s_cb = 0.f, s_cw[kConvWidth] = {0.f, 0.f, 0.f, 0.f};
    float carry[kHist] = {0.f, 0.f, 0.f};    // dxc of the three tokens after the current tile
    float cw[kConvWidth] = {0.f, 0.f, 0.f, 0.f};
    if (scan_thread) {
        kappa = a.c * log_sigmoid_acc(a.lambda[ch]);
        c_sneg = a.c * sigmoid_acc(-a.lambda[ch]);
        g = a.dh_final ? a.dh_final[(size_t)b * W + ch] : 0.f;
#pragma unroll
        for (int k = 0; k < kConvWidth; ++k) cw[k] = a.conv_w[(size_t)k * W + ch];
    }
    const int ntiles = (a.T + kTile - 1) / kTile;
    for (int tile = ntiles - 1; tile >= 0; --tile) {
        const int t0 = tile * kTile, nt = min(kTile, a.T - t0);
        // ---- A. the recurrence backwards through the tile, one thread per channel
        if (scan_thread) {
            for (int tt = nt - 1; tt >= 0; --tt) {
                const int t = t0 + tt;
                const size_t e = ((size_t)b * a.T + t) * W + ch;
                const float xcv = a.xc[e], hp = a.hprev[e];
                const float r = sigmoid_acc(a.ga[e]), ig = sigmoid_acc(a.gx[e]);
                float at, beta;
                decay_and_beta_acc(kappa, r, &at, &beta);
                const float h = fmaf(at, hp, beta * (ig * xcv));
                const float yv = Act<T>::load(y + e), dz = Act<T>::load(dout + e);
                g = fmaf(dz, gelu_acc(yv, a.gelu_tanh), g);
                a.g.dy[e] = dz * h * gelu_grad_acc(yv, a.gelu_tanh);
                const float dl_da = g * hp, dl_dbeta = g * ig * xcv, dl_di = g * beta * xcv;
                const float r_over_beta = beta > 0.f ? r / beta : 0.f;
                const float q = dl_da * at * r - dl_dbeta * at * at * r_over_beta;
                const float dga = kappa * (1.0f - r) * q;
                const float dgx = dl_di * ig * (1.0f - ig);
                s_lam = fmaf(c_sneg, q, s_lam);
                s_ba += dga;
                s_bx += dgx;
                a.ga[e] = dga;
                a.gx[e] = dgx;
                dga_s[tt * dh + o] = dga;
                dgx_s[tt * dh + o] = dgx;
                dxc_s[tt * dh + o] = g * beta * ig;
                g = (a.reset && a.reset[(size_t)b * a.T + t]) ? 0.f : at * g;
            }
        }
        __syncthreads();
        // ---- B. dxc += W_a dga + W_x dgx (thread = input channel i, rows of the weights)
        //      (dga_s / dgx_s are only read here; each (token, i) of dxc_s has one writer)
        if (grp < groups) {
            const int i = o;
            float acc[kTile];
#pragma unroll
            for (int q = 0; q < kTile; ++q) acc[q] = 0.f;
            for (int oo = 0; oo < dh; ++oo) {
                const float wa = Act<T>::load(w_a + (size_t)i * dh + oo);
                const float wx = Act<T>::load(w_x + (size_t)i * dh + oo);
#pragma unroll
                for (int q = 0; q < kTile; ++q) {
                    const int tt = grp + q * groups;
                    if (q * groups < kTile && tt < nt)
                        acc[q] = fmaf(wa, dga_s[tt * dh + oo], fmaf(wx, dgx_s[tt * dh + oo], acc[q]));
                }
            }
#pragma unroll
            for (int q = 0; q < kTile; ++q) {
                const int tt = grp + q * groups;
                if (q * groups < kTile && tt < nt) dxc_s[tt * dh + i] += acc[q];
            }
        }
        __syncthreads();
        // ---- C. the conv's transpose, one thread per channel
        if (scan_thread) {
            auto dxc_at = [&](int t) -> float {     // dxc of token t >= t0 (0 past the end)
                if (t >= a.T) return 0.f;
                return t < t0 + nt ? dxc_s[(t - t0) * dh + o] : carry[t - t0 - nt];
            };
            for (int tt = 0; tt < nt; ++tt) {
                const int t = t0 + tt;
                const float d = dxc_s[tt * dh + o];
                s_cb += d;
#pragma unroll
                for (int k = 0; k < kConvWidth; ++k)
                    s_cw[k] = fmaf(d, window_value<T>(a, b, t - kHist + k, t, ch, W), s_cw[k]);
            }
            // dx_s for the tile's positions, and the initial history from the first tile
            for (int s = t0 + nt - 1; s >= (t0 == 0 ? -kHist : t0); --s) {
                float acc = 0.f;
#pragma unroll
                for (int k = 0; k < kConvWidth; ++k) {
                    const int t = s + kHist - k;              // the token whose tap k reads s
                    if (t >= 0 && t < a.T && window_reads(a, b, s, t)) acc = fmaf(cw[k], dxc_at(t), acc);
                }
                if (a.dtail_final && s >= a.T - kHist && window_reads(a, b, s, a.T - 1))
                    acc += a.dtail_final[((size_t)b * kHist + (s - (a.T - kHist))) * W + ch];
                if (s >= 0) a.g.dx[((size_t)b * a.T + s) * W + ch] = acc;
                else if (a.g.dtail0) a.g.dtail0[((size_t)b * kHist + (kHist + s)) * W + ch] = acc;
            }
            float nc[kHist];
#pragma unroll
            for (int j = 0; j < kHist; ++j) nc[j] = dxc_at(t0 + j);
#pragma unroll
            for (int j = 0; j < kHist; ++j) carry[j] = nc[j];
        }
        __syncthreads();
    }
    if (scan_thread) {
        if (a.g.dh0) a.g.dh0[(size_t)b * W + ch] = g;
        const size_t pb = (size_t)a.B * W;
        float* p = a.part + (size_t)b * W + ch;
        p[0 * pb] = s_lam;
        p[1 * pb] = s_ba;
        p[2 * pb] = s_bx;
        p[3 * pb] = s_cb;
#pragma unroll
        for (int k = 0; k < kConvWidth; ++k) p[(4 + k) * pb] = s_cw[k];
    }
}

// ---------------------------------------------------------------- 3. weight gradients -------
constexpr int kWT = 16;   // output tile
constexpr int kWK = 32;   // tokens per step
__global__ void __launch_bounds__(kWT * kWT) bwd_weight_kernel(BwdArgs a) {
    __shared__ float xs[kWK][kWT], as[kWK][kWT], gs[kWK][kWT];
    const int hd = blockIdx.z, i0 = blockIdx.y * kWT, o0 = blockIdx.x * kWT;
    const int dh = a.dh, W = a.H * dh, ch0 = hd * dh;
    const int tx = threadIdx.x, ty = threadIdx.y, tid = ty * kWT + tx;
    const long N = (long)a.B * a.T;
    float acc_a = 0.f, acc_x = 0.f;
    for (long n0 = 0; n0 < N; n0 += kWK) {
        for (int e = tid; e < kWK * kWT; e += kWT * kWT) {
            const int r = e / kWT, cc = e % kWT;
            const long n = n0 + r;
            const bool in = n < N;
            xs[r][cc] = in ? a.xc[n * W + ch0 + i0 + cc] : 0.f;
            as[r][cc] = in ? a.ga[n * W + ch0 + o0 + cc] : 0.f;
            gs[r][cc] = in ? a.gx[n * W + ch0 + o0 + cc] : 0.f;
        }
        __syncthreads();
#pragma unroll 8
        for (int r = 0; r < kWK; ++r) {
            acc_a = fmaf(xs[r][ty], as[r][tx], acc_a);
            acc_x = fmaf(xs[r][ty], gs[r][tx], acc_x);
        }
        __syncthreads();
    }
    const size_t w = (size_t)hd * dh * dh + (size_t)(i0 + ty) * dh + o0 + tx;
    a.g.dw_a[w] = acc_a;
    a.g.dw_x[w] = acc_x;
}

// ---------------------------------------------------------------- 4. batch-row sums ---------
__global__ void bwd_reduce_kernel(BwdArgs a) {
    const int W = a.H * a.dh;
    const int ch = blockIdx.x * blockDim.x + threadIdx.x;
    if (ch >= W) return;
    const size_t pb = (size_t)a.B * W;
    float s[kParts];
#pragma unroll
    for (int k = 0; k < kParts; ++k) s[k] = 0.f;
    for (int b = 0; b < a.B; ++b)
#pragma unroll
        for (int k = 0; k < kParts; ++k) s[k] += a.part[k * pb + (size_t)b * W + ch];
    a.g.dlambda[ch] = s[0];
    a.g.db_a[ch] = s[1];
    a.g.db_x[ch] = s[2];
    a.g.dconv_b[ch] = s[3];
#pragma unroll
    for (int k = 0; k < kConvWidth; ++k) a.g.dconv_w[(size_t)k * W + ch] = s[4 + k];
}

// The dynamic shared-memory limits of the four tile kernels are raised once per device, to
// their largest need (head_dim 256), before the first launch.
cudaError_t raise_bwd_smem_limits() {
    static std::mutex mu;
    static bool done[64] = {};
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    std::lock_guard<std::mutex> lock(mu);
    if (dev >= 0 && dev < 64 && done[dev]) return cudaSuccess;
    const int most = 3 * kTile * 256 * (int)sizeof(float);
    const cudaFuncAttribute attr = cudaFuncAttributeMaxDynamicSharedMemorySize;
    e = cudaFuncSetAttribute(bwd_forward_kernel<float>, attr, most);
    if (e == cudaSuccess) e = cudaFuncSetAttribute(bwd_forward_kernel<__nv_bfloat16>, attr, most);
    if (e == cudaSuccess) e = cudaFuncSetAttribute(bwd_reverse_kernel<float>, attr, most);
    if (e == cudaSuccess) e = cudaFuncSetAttribute(bwd_reverse_kernel<__nv_bfloat16>, attr, most);
    if (e == cudaSuccess && dev >= 0 && dev < 64) done[dev] = true;
    return e;
}

template <typename T>
cudaError_t launch_typed(BwdArgs& a, cudaStream_t s) {
    const int smem = 3 * kTile * a.dh * (int)sizeof(float);
    cudaError_t e = raise_bwd_smem_limits();
    if (e != cudaSuccess) return e;
    const dim3 grid(a.H, a.B);
    bwd_forward_kernel<T><<<grid, kThreads, smem, s>>>(a);
    bwd_reverse_kernel<T><<<grid, kThreads, smem, s>>>(a);
    bwd_weight_kernel<<<dim3(a.dh / kWT, a.dh / kWT, a.H), dim3(kWT, kWT), 0, s>>>(a);
    const int W = a.H * a.dh;
    bwd_reduce_kernel<<<(W + 255) / 256, 256, 0, s>>>(a);
    return cudaGetLastError();
}

struct BwdLayout {
    size_t xc, hprev, ga, gx, part, total;
};

BwdLayout bwd_layout(const rglru_dims* d) {
    auto up = [](size_t v) { return (v + 255) & ~size_t(255); };
    const size_t n = (size_t)d->batch * d->seq_len * d->heads * d->head_dim * sizeof(float);
    BwdLayout l;
    l.xc = 256;
    l.hprev = up(l.xc + n);
    l.ga = up(l.hprev + n);
    l.gx = up(l.ga + n);
    l.part = up(l.gx + n);
    l.total = up(l.part + (size_t)kParts * d->batch * d->heads * d->head_dim * sizeof(float));
    return l;
}

}  // namespace

size_t backward_workspace(const rglru_dims* d) { return bwd_layout(d).total; }

int backward_launches(const rglru_dims* d) {
    (void)d;
    return 4;
}

cudaError_t launch_backward(const rglru_dims* d, const rglru_params* p, const void* x, const void* y,
                            const uint8_t* reset, const rglru_state* st0, const void* dout,
                            const float* dh_final, const float* dtail_final, const rglru_grads* grads,
                            void* ws, size_t ws_bytes, cudaStream_t s) {
    const BwdLayout l = bwd_layout(d);
    if (l.total > ws_bytes) return cudaErrorInvalidValue;
    uint8_t* w = static_cast<uint8_t*>(ws);
    BwdArgs a;
    a.B = d->batch; a.T = d->seq_len; a.H = d->heads; a.dh = d->head_dim;
    a.c = d->c; a.gelu_tanh = d->gelu_tanh;
    a.conv_w = p->conv_w; a.conv_b = p->conv_b; a.w_a = p->w_a; a.w_x = p->w_x;
    a.b_a = p->b_a; a.b_x = p->b_x; a.lambda = p->lambda;
    a.x = x; a.y = y; a.reset = reset;
    a.h0 = st0 ? st0->h : nullptr;
    a.tail0 = st0 ? st0->conv_tail : nullptr;
    a.dout = dout; a.dh_final = dh_final; a.dtail_final = dtail_final;
    a.xc = reinterpret_cast<float*>(w + l.xc);
    a.hprev = reinterpret_cast<float*>(w + l.hprev);
    a.ga = reinterpret_cast<float*>(w + l.ga);
    a.gx = reinterpret_cast<float*>(w + l.gx);
    a.part = reinterpret_cast<float*>(w + l.part);
    a.g = *grads;
    return d->act_dtype == RGLRU_F32 ? launch_typed<float>(a, s) : launch_typed<__nv_bfloat16>(a, s);
}

}  // namespace rglru
