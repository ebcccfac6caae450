// generic.cu -- portable RG-LRU kernels (CUDA cores only, accurate fp32 math).
//
// These carry the fp32 workloads, every head_dim that the tensor-core prefill does not take,
// and the decode step.  One CTA owns one (batch row, head) sequence for the whole prefill, so
// the carry stays in registers, the initial state is read before the final state is written,
// and no workspace is needed.  The gate contraction runs on FFMA with fp32 accumulation.
//
// Arithmetic per element follows "Griffin Guide: RecurrentGemma, RG-LRU & Hybrid Attention":
// gates, decay, update ("1. Formulation of the RG-LRU Gating Mechanism"), sqrt(1 - a^2)
// ("2. The Role of Square-Root Variance Normalization"), causal width-4 conv and GeLU merge
// ("1. Temporal Filtering via Separable 1D Convolutions", "2. Non-Linear Multiplicative Gating
// with GeLU"), per-head block-diagonal gates ("3. Block-Diagonal Sharding ...").
#include "common.cuh"
#include "kernels.h"

namespace rglru {

namespace {

constexpr int kThreads = 256;
constexpr int kTile = 32;        // tokens per tile (prefill) / rows per CTA (decode: kRows)
constexpr int kRows = 8;

struct GenericArgs {
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
    float* h;          // state h or nullptr
    void* tail;        // state conv_tail or nullptr
    void* out;
};

// Conv history value x~_{t'} seen from token t of row b (t' in [t-3, t]): the raw input when
// no reset lies in (t', t]; for t' < 0 the carried tail (or 0 without a state).
template <typename T>
__device__ __forceinline__ float conv_input(const GenericArgs& a, int b, int t, int tp, int ch,
                                            int W, const T* x, const T* tail) {
    if (a.reset) {
        for (int s = (tp + 1 > 0 ? tp + 1 : 0); s <= t; ++s)
            if (a.reset[(size_t)b * a.T + s]) return 0.0f;
    }
    if (tp >= 0) return Act<T>::load(x + ((size_t)b * a.T + tp) * W + ch);
    if (!tail) return 0.0f;
    return Act<T>::load(tail + ((size_t)b * kHist + (kHist + tp)) * W + ch);
}

template <typename T>
__global__ void __launch_bounds__(kThreads) prefill_generic_kernel(GenericArgs a) {
    extern __shared__ float smem[];
    const int hd = blockIdx.x, b = blockIdx.y;
    const int dh = a.dh, W = a.H * dh, ch0 = hd * dh;
    float* xc_s = smem;                      // [kTile][dh]
    float* a_s = xc_s + kTile * dh;          // [kTile][dh]
    float* u_s = a_s + kTile * dh;           // [kTile][dh]
    const T* x = static_cast<const T*>(a.x);
    const T* y = static_cast<const T*>(a.y);
    const T* tail_in = static_cast<const T*>(a.tail);
    const T* w_a = static_cast<const T*>(a.w_a) + (size_t)hd * dh * dh;
    const T* w_x = static_cast<const T*>(a.w_x) + (size_t)hd * dh * dh;
    T* out = static_cast<T*>(a.out);

    const int groups = kThreads / dh;        // token groups in the contraction
    const int o = threadIdx.x % dh;
    const int g = threadIdx.x / dh;
    const bool scan_thread = threadIdx.x < dh;
    const int ch = ch0 + o;
    float c_lab = 0.f, ba = 0.f, bx = 0.f, hreg = 0.f;
    if (g < groups) {
        c_lab = a.c * log_sigmoid_acc(a.lambda[ch]);
        ba = a.b_a ? a.b_a[ch] : 0.f;
        bx = a.b_x ? a.b_x[ch] : 0.f;
    }
    if (scan_thread && a.h) hreg = a.h[(size_t)b * W + ch];

    for (int t0 = 0; t0 < a.T; t0 += kTile) {
        const int nt = min(kTile, a.T - t0);
        // 1. causal depthwise conv of the tile
        for (int e = threadIdx.x; e < nt * dh; e += kThreads) {
            int tt = e / dh, j = e % dh, t = t0 + tt, c2 = ch0 + j;
            float acc = a.conv_b ? a.conv_b[c2] : 0.f;
#pragma unroll
            for (int k = 0; k < kConvWidth; ++k)
                acc += a.conv_w[(size_t)k * W + c2] * conv_input<T>(a, b, t, t - kHist + k, c2, W, x, tail_in);
            xc_s[tt * dh + j] = acc;
        }
        __syncthreads();
        // 2. block-diagonal gate contraction (fp32 FFMA) and the per-element gate math
        if (g < groups) {
            float acc_a[kTile], acc_x[kTile];
#pragma unroll
            for (int q = 0; q < kTile; ++q) { acc_a[q] = ba; acc_x[q] = bx; }
            for (int i = 0; i < dh; ++i) {
                float wa = Act<T>::load(w_a + (size_t)i * dh + o);
                float wx = Act<T>::load(w_x + (size_t)i * dh + o);
#pragma unroll
                for (int q = 0; q < kTile; ++q) {
                    int tt = g + q * groups;
                    if (q * groups < kTile && tt < nt) {
                        float v = xc_s[tt * dh + i];
                        acc_a[q] = fmaf(v, wa, acc_a[q]);
                        acc_x[q] = fmaf(v, wx, acc_x[q]);
                    }
                }
            }
#pragma unroll
            for (int q = 0; q < kTile; ++q) {
                int tt = g + q * groups;
                if (q * groups < kTile && tt < nt) {
                    float r = sigmoid_acc(acc_a[q]);
                    float ig = sigmoid_acc(acc_x[q]);
                    float at, beta;
                    decay_and_beta_acc(c_lab, r, &at, &beta);
                    if (a.reset && a.reset[(size_t)b * a.T + t0 + tt]) at = 0.f;  // h_{t-1} := 0
                    a_s[tt * dh + o] = at;
                    u_s[tt * dh + o] = beta * (ig * xc_s[tt * dh + o]);
                }
            }
        }
        __syncthreads();
        // 3. sequential scan over the tile, one thread per channel, and the GeLU merge
        if (scan_thread) {
            for (int tt = 0; tt < nt; ++tt) {
                hreg = fmaf(a_s[tt * dh + o], hreg, u_s[tt * dh + o]);
                size_t idx = ((size_t)b * a.T + t0 + tt) * W + ch;
                Act<T>::store(out + idx, hreg * gelu_acc(Act<T>::load(y + idx), a.gelu_tanh));
            }
        }
        __syncthreads();
    }
    // 4. final state: h, and the last three inputs of the final segment (oldest first)
    if (a.h && scan_thread) {
        a.h[(size_t)b * W + ch] = hreg;
        T* tail = static_cast<T*>(a.tail);
        float v[kHist];
#pragma unroll
        for (int k = 0; k < kHist; ++k)
            v[k] = conv_input<T>(a, b, a.T - 1, a.T - kHist + k, ch, W, x, tail_in);
        __syncwarp();
#pragma unroll
        for (int k = 0; k < kHist; ++k)
            Act<T>::store(tail + ((size_t)b * kHist + k) * W + ch, v[k]);
    }
}

template <typename T>
__global__ void __launch_bounds__(kThreads) decode_generic_kernel(GenericArgs a) {
    extern __shared__ float smem[];
    const int hd = blockIdx.x, r0 = blockIdx.y * kRows;
    const int dh = a.dh, W = a.H * dh, ch0 = hd * dh;
    const int nr = min(kRows, a.B - r0);
    float* xc_s = smem;                                   // [kRows][dh]
    const T* x = static_cast<const T*>(a.x);
    const T* y = static_cast<const T*>(a.y);
    T* tail = static_cast<T*>(a.tail);
    const T* w_a = static_cast<const T*>(a.w_a) + (size_t)hd * dh * dh;
    const T* w_x = static_cast<const T*>(a.w_x) + (size_t)hd * dh * dh;
    T* out = static_cast<T*>(a.out);

    // 1. conv over (tail, x) and the tail shift; this CTA owns these (row, channel) entries
    for (int e = threadIdx.x; e < nr * dh; e += kThreads) {
        int rr = e / dh, j = e % dh, b = r0 + rr, c2 = ch0 + j;
        bool rst = a.reset && a.reset[b];
        float hist[kHist];
#pragma unroll
        for (int k = 0; k < kHist; ++k)
            hist[k] = rst ? 0.f : Act<T>::load(tail + ((size_t)b * kHist + k) * W + c2);
        float xv = Act<T>::load(x + (size_t)b * W + c2);
        float acc = a.conv_b ? a.conv_b[c2] : 0.f;
#pragma unroll
        for (int k = 0; k < kHist; ++k) acc += a.conv_w[(size_t)k * W + c2] * hist[k];
        acc += a.conv_w[(size_t)kHist * W + c2] * xv;
        xc_s[rr * dh + j] = acc;
        Act<T>::store(tail + ((size_t)b * kHist + 0) * W + c2, hist[1]);
        Act<T>::store(tail + ((size_t)b * kHist + 1) * W + c2, hist[2]);
        Act<T>::store(tail + ((size_t)b * kHist + 2) * W + c2, xv);
    }
    __syncthreads();
    // 2. gates, decay and state update in place
    const int groups = kThreads / dh;
    const int o = threadIdx.x % dh, g = threadIdx.x / dh, ch = ch0 + o;
    if (g >= groups) return;
    float c_lab = a.c * log_sigmoid_acc(a.lambda[ch]);
    float ba = a.b_a ? a.b_a[ch] : 0.f, bx = a.b_x ? a.b_x[ch] : 0.f;
    float acc_a[kRows], acc_x[kRows];
#pragma unroll
    for (int q = 0; q < kRows; ++q) { acc_a[q] = ba; acc_x[q] = bx; }
    for (int i = 0; i < dh; ++i) {
        float wa = Act<T>::load(w_a + (size_t)i * dh + o);
        float wx = Act<T>::load(w_x + (size_t)i * dh + o);
#pragma unroll
        for (int q = 0; q < kRows; ++q) {
            int rr = g + q * groups;
            if (q * groups < kRows && rr < nr) {
                float v = xc_s[rr * dh + i];
                acc_a[q] = fmaf(v, wa, acc_a[q]);
                acc_x[q] = fmaf(v, wx, acc_x[q]);
            }
        }
    }
#pragma unroll
    for (int q = 0; q < kRows; ++q) {
        int rr = g + q * groups;
        if (q * groups < kRows && rr < nr) {
            int b = r0 + rr;
            float r = sigmoid_acc(acc_a[q]);
            float ig = sigmoid_acc(acc_x[q]);
            float at, beta;
            decay_and_beta_acc(c_lab, r, &at, &beta);
            size_t idx = (size_t)b * W + ch;
            float hp = (a.reset && a.reset[b]) ? 0.f : a.h[idx];
            float hn = fmaf(at, hp, beta * (ig * xc_s[rr * dh + o]));
            a.h[idx] = hn;
            Act<T>::store(out + idx, hn * gelu_acc(Act<T>::load(y + idx), a.gelu_tanh));
        }
    }
}

GenericArgs make_args(const rglru_dims* d, const rglru_params* p, const void* x, const void* y,
                      const uint8_t* reset, rglru_state* st, void* out) {
    GenericArgs a;
    a.B = d->batch; a.T = d->seq_len; a.H = d->heads; a.dh = d->head_dim;
    a.c = d->c; a.gelu_tanh = d->gelu_tanh;
    a.conv_w = p->conv_w; a.conv_b = p->conv_b; a.w_a = p->w_a; a.w_x = p->w_x;
    a.b_a = p->b_a; a.b_x = p->b_x; a.lambda = p->lambda;
    a.x = x; a.y = y; a.reset = reset;
    a.h = st ? st->h : nullptr;
    a.tail = st ? st->conv_tail : nullptr;
    a.out = out;
    return a;
}

// The dynamic shared-memory limits of all four kernels are raised once, to their largest need
// (head_dim 256), so that no attribute call is made while a stream is being captured.
cudaError_t raise_smem_limits() {
    static cudaError_t once = [] {
        const int pre = 3 * kTile * 256 * (int)sizeof(float);
        const int dec = kRows * 256 * (int)sizeof(float);
        cudaError_t e = cudaFuncSetAttribute(prefill_generic_kernel<float>,
                                             cudaFuncAttributeMaxDynamicSharedMemorySize, pre);
        if (e == cudaSuccess)
            e = cudaFuncSetAttribute(prefill_generic_kernel<__nv_bfloat16>,
                                     cudaFuncAttributeMaxDynamicSharedMemorySize, pre);
        if (e == cudaSuccess)
            e = cudaFuncSetAttribute(decode_generic_kernel<float>,
                                     cudaFuncAttributeMaxDynamicSharedMemorySize, dec);
        if (e == cudaSuccess)
            e = cudaFuncSetAttribute(decode_generic_kernel<__nv_bfloat16>,
                                     cudaFuncAttributeMaxDynamicSharedMemorySize, dec);
        return e;
    }();
    return once;
}

template <typename K>
cudaError_t launch(K kernel, dim3 grid, size_t smem, cudaStream_t s, const GenericArgs& a) {
    cudaError_t e = raise_smem_limits();
    if (e != cudaSuccess) return e;
    kernel<<<grid, kThreads, smem, s>>>(a);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_prefill_generic(const rglru_dims* d, const rglru_params* p, const void* x,
                                   const void* y, const uint8_t* reset, rglru_state* st,
                                   void* out, cudaStream_t s) {
    GenericArgs a = make_args(d, p, x, y, reset, st, out);
    dim3 grid(d->heads, d->batch);
    size_t smem = (size_t)3 * kTile * d->head_dim * sizeof(float);
    if (d->act_dtype == RGLRU_F32) return launch(prefill_generic_kernel<float>, grid, smem, s, a);
    return launch(prefill_generic_kernel<__nv_bfloat16>, grid, smem, s, a);
}

cudaError_t launch_decode_generic(const rglru_dims* d, const rglru_params* p, const void* x,
                                  const void* y, const uint8_t* reset, rglru_state* st,
                                  void* out, cudaStream_t s) {
    GenericArgs a = make_args(d, p, x, y, reset, st, out);
    a.T = 1;
    dim3 grid(d->heads, (d->batch + kRows - 1) / kRows);
    size_t smem = (size_t)kRows * d->head_dim * sizeof(float);
    if (d->act_dtype == RGLRU_F32) return launch(decode_generic_kernel<float>, grid, smem, s, a);
    return launch(decode_generic_kernel<__nv_bfloat16>, grid, smem, s, a);
}

}  // namespace rglru
