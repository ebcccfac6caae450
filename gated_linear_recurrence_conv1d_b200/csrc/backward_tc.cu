// backward_tc.cu -- gradients of the RG-LRU block for bf16 activations, head_dim 256, with the
// dense contractions on the tensor cores (sm_100a).
//
// The gradients are those of backward.cu (the chain rule through the forward the pages define,
// "Griffin Guide: RecurrentGemma, RG-LRU & Hybrid Attention": "1. Formulation of the RG-LRU
// Gating Mechanism", "2. The Role of Square-Root Variance Normalization", "1. Temporal Filtering
// via Separable 1D Convolutions", "2. Non-Linear Multiplicative Gating with GeLU", "3.
// Block-Diagonal Sharding ..."), computed in these steps:
//
//   1. the tensor-core prefill in its save mode (fused_prefill.cu) runs the forward again and
//      keeps, per token-channel, the complete gate pre-activations ga, gx (fp32), h_{t-1} as the
//      update used it (fp32) and the conv output as a bf16 pair hi + lo (x = hi + lo to 2^-16);
//      its gate contraction runs on both bf16 parts of the conv output, so the pre-activations
//      are those of the fp32 conv output;
//   2. the reverse scan of g = dL/dh_t:  g_t = dout_t GeLU(y_t) + a_{t+1} g_{t+1} (0 across a
//      reset), a first-order linear recurrence run backwards, cut into chunks of kChunk tokens:
//      bwd_scan_agg_kernel gives each (row, chunk, channel) its map c -> P c + Q from the carry
//      entering the chunk's last token to the one leaving its first (P the product of the a_t,
//      Q the chunk's own contribution); bwd_scan_carry_kernel chains the maps of a row from the
//      last chunk to the first (dh_final in, dL/dh_{-1} out); bwd_scan_out_kernel walks every
//      chunk again from its carry and writes dy, the direct part of dL/dxc (g beta i) and
//      dL/dga, dL/dgx as bf16 hi / lo pairs, and per-(row, chunk) partial sums of dLambda, db_a,
//      db_x;
//   3. dL/dxc += dga W_a^T + dgx W_x^T: a tensor-core GEMM per head over the B T tokens with the
//      hi and lo parts of dga and dgx as four K ranges (gemm.cu);
//   4. bwd_convT_kernel: the conv's transpose in parallel over (row, 64-token block, channel):
//      dx_s gathers w_k dxc_{s+3-k} over the windows that read x_s, the initial history gets the
//      taps that read it, the final history's gradient goes to the inputs it copied; partial
//      sums of dconv_w, dconv_b per block;
//   5. dW[h] = sum over tokens of xc^T dg for both gates: tensor-core GEMMs with the hi / lo
//      parts (xc_hi dg_hi + xc_hi dg_lo + xc_lo dg_hi), K cut into slices whose partial sums
//      are kept apart;
//   6. bwdtc_reduce_kernel: every partial sum in a fixed order.
// No atomics: the gradients are bitwise repeatable.
#include <algorithm>

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "common.cuh"
#include "kernels.h"
#include "rglru_math.cuh"

namespace rglru {

namespace {

constexpr int DH = 256;
constexpr int kTB = 64;          // tokens per conv-transpose block
constexpr int kMaxSplits = 16;   // K slices of the weight-gradient GEMMs, at most
constexpr int kScanThreads = 128;
constexpr int kChunk = 64;       // tokens per chunk of the reverse scan
// Resident blocks per SM asked of the three streaming kernels (their register caps) and the
// conv transpose's prefetch depth, set by measurement on B200 (rg2b_bf16): more resident warps
// hide the scans' load latency better than deeper per-thread batches.
constexpr int kAggMinBlocks = 12, kOutMinBlocks = 12, kConvTMinBlocks = 4;
constexpr int kPFC = 4;          // positions a conv-transpose batch loads ahead

struct Layout {
    size_t ga, gx, hprev, dxc, xc_hi, xc_lo, dga_hi, dga_lo, dgx_hi, dgx_lo;
    size_t agg, part_scan, part_conv, dw, fwd, total;
    int ntb, nch;
};

Layout layout(const rglru_dims* d) {
    auto up = [](size_t v) { return (v + 255) & ~size_t(255); };
    const size_t W = (size_t)d->heads * d->head_dim;
    const size_t n = (size_t)d->batch * d->seq_len * W;
    Layout l;
    l.ntb = (d->seq_len + kTB - 1) / kTB;
    l.nch = (d->seq_len + kChunk - 1) / kChunk;
    size_t o = 256;
    l.ga = o;      o = up(o + n * 4);
    l.gx = o;      o = up(o + n * 4);
    l.hprev = o;   o = up(o + n * 4);
    l.dxc = o;     o = up(o + n * 4);
    l.xc_hi = o;   o = up(o + n * 2);
    l.xc_lo = o;   o = up(o + n * 2);
    l.dga_hi = o;  o = up(o + n * 2);
    l.dga_lo = o;  o = up(o + n * 2);
    l.dgx_hi = o;  o = up(o + n * 2);
    l.dgx_lo = o;  o = up(o + n * 2);
    l.agg = o;     o = up(o + 2 * (size_t)d->batch * l.nch * W * 4);
    l.part_scan = o; o = up(o + 3 * (size_t)d->batch * l.nch * W * 4);
    l.part_conv = o; o = up(o + 5 * (size_t)d->batch * l.ntb * W * 4);
    l.dw = o;      o = up(o + 2 * (size_t)kMaxSplits * d->heads * DH * DH * 4);
    l.fwd = o;     o = up(o + fused_prefill_workspace(d));
    l.total = o;
    return l;
}


// d/dv [v Phi(v)] = Phi(v) + v phi(v); the tanh form's derivative for the flag
__device__ __forceinline__ float gelu_grad(float v, int tanh_form) {
    if (tanh_form) {
        const float k = 0.79788456080286535588f;
        const float th = tanhf(k * (v + 0.044715f * v * v * v));
        return 0.5f * (1.0f + th) + 0.5f * v * (1.0f - th * th) * k * (1.0f + 3.0f * 0.044715f * v * v);
    }
    return 0.5f * erfcf(-v * 0.70710678118654752440f) + v * expf(-0.5f * v * v) * 0.39894228040143267794f;
}

// The per-token arithmetic of the reverse scan, with hardware exp2 / reciprocal (relative
// errors near 2^-22) where CUDA's accurate functions would cost several times the instructions:
//   sigma(z) = 1 / (1 + 2^(-z log2 e));
//   a = 1 + E, E = expm1(c r log sigma(Lambda)) by its series to l^5 for l >= -1/8 (no
//   cancellation as a -> 1, where the reverse recurrence carries errors of a over ~1 / (1 - a)
//   tokens), else 2^(l log2 e) - 1; beta = sqrt(1 - a^2) = sqrt(-E (2 + E));
//   GeLU = v Phi and GeLU' = Phi + v phi(v) from one exp2 and a polynomial (below; the tanh
//   form keeps tanhf).
__device__ __forceinline__ float sig_fast(float z) { return fm::rcpf(1.0f + fm::ex2f(-z * fm::kLog2e)); }

__device__ __forceinline__ void decay_beta_fast(float kappa, float r, float& at, float& beta) {
    const float E = fm::expm1_any(kappa * r);
    at = 1.0f + E;
    beta = sqrtf(-E * (2.0f + E));
}

// GeLU and its derivative with Phi from fm::phi_precise (rglru_math.cuh).
__device__ __forceinline__ void gelu_and_grad(float v, int tanh_form, float& g, float& gp) {
    if (tanh_form) {
        g = gelu_acc(v, 1);
        gp = gelu_grad(v, 1);
        return;
    }
    float e;
    const float phi_c = fm::phi_precise(v, e);
    g = v * phi_c;
    gp = fmaf(v * e, 0.39894228040143267794f, phi_c);
}


struct ScanArgs {
    int B, T, W, nch;
    float c;
    int gelu_tanh;
    const float* lambda;
    const __nv_bfloat16* y;
    const __nv_bfloat16* dout;
    const uint8_t* reset;
    const float* dh_final;
    const float* ga;
    const float* gx;
    const float* hprev;
    const __nv_bfloat16* xc_hi;
    const __nv_bfloat16* xc_lo;
    float* dy;
    float* dxc;
    __nv_bfloat16* dga_hi;
    __nv_bfloat16* dga_lo;
    __nv_bfloat16* dgx_hi;
    __nv_bfloat16* dgx_lo;
    float* dh0;
    float* agg;           // [2][B][nch][W]: P, Q of each chunk, then Q replaced by the carry into it
    float* part;          // [3][B][nch][W]: dLambda, db_a, db_x
};

// ---------------------------------------------------------------- 2. the reverse scan -------
// Thread = (row b, chunk k, channel ch); the inputs of a block of kPF tokens are loaded together
// before the block is walked, so that their latencies overlap.
constexpr int kPF = 4;

// a'_t: the factor that carries g from token t to t - 1 (a_t, or 0 where t starts a segment)
__device__ __forceinline__ float carry_factor(float kappa, float ga, bool rs) {
    const float at = 1.0f + fm::expm1_any(kappa * sig_fast(ga));
    return rs ? 0.f : at;
}

// P = prod a'_t and Q = the carry leaving the chunk's first token when none enters its last.
// Thread = (row b, chunk k, channel pair ch, ch + 1): paired loads halve the address arithmetic.
__device__ __forceinline__ float2 bf2f(const __nv_bfloat16* p) {
    return __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(p));
}

__global__ void __launch_bounds__(kScanThreads, kAggMinBlocks) bwd_scan_agg_kernel(ScanArgs a) {
    const int ch = 2 * (blockIdx.x * kScanThreads + threadIdx.x), k = blockIdx.y, b = blockIdx.z;
    if (ch >= a.W) return;
    const float kap0 = a.c * log_sigmoid_acc(a.lambda[ch]), kap1 = a.c * log_sigmoid_acc(a.lambda[ch + 1]);
    const uint8_t* rrow = a.reset ? a.reset + (size_t)b * a.T : nullptr;
    const int t0 = k * kChunk, t1 = min(a.T, t0 + kChunk);
    float P0 = 1.f, P1 = 1.f, g0 = 0.f, g1 = 0.f;
    for (int tb = t1 - kPF; tb > t0 - kPF; tb -= kPF) {
        float2 vga[kPF], vy[kPF], vdz[kPF];
        bool rs[kPF];
        const size_t eb = ((size_t)b * a.T + tb) * a.W + ch;
#pragma unroll
        for (int j = 0; j < kPF; ++j) {
            if (tb + j >= t0) {
                const size_t e = eb + (size_t)j * a.W;
                vga[j] = *reinterpret_cast<const float2*>(a.ga + e);
                vy[j] = bf2f(a.y + e);
                vdz[j] = bf2f(a.dout + e);
                rs[j] = rrow && rrow[tb + j];
            }
        }
#pragma unroll
        for (int j = kPF - 1; j >= 0; --j) {
            if (tb + j < t0) continue;
            float gl, gp;
            gelu_and_grad(vy[j].x, a.gelu_tanh, gl, gp);
            g0 = fmaf(vdz[j].x, gl, g0);
            gelu_and_grad(vy[j].y, a.gelu_tanh, gl, gp);
            g1 = fmaf(vdz[j].y, gl, g1);
            const float f0 = carry_factor(kap0, vga[j].x, rs[j]), f1 = carry_factor(kap1, vga[j].y, rs[j]);
            g0 *= f0;
            g1 *= f1;
            P0 *= f0;
            P1 *= f1;
        }
    }
    const size_t pb = (size_t)a.B * a.nch * a.W, pi = ((size_t)b * a.nch + k) * a.W + ch;
    *reinterpret_cast<float2*>(a.agg + pi) = make_float2(P0, P1);
    *reinterpret_cast<float2*>(a.agg + pb + pi) = make_float2(g0, g1);
}

// per (row, channel): the carries into every chunk, from the last chunk to the first
__global__ void __launch_bounds__(kScanThreads) bwd_scan_carry_kernel(ScanArgs a) {
    const int ch = blockIdx.x * kScanThreads + threadIdx.x, b = blockIdx.y;
    if (ch >= a.W) return;
    const size_t pb = (size_t)a.B * a.nch * a.W;
    float c = a.dh_final ? a.dh_final[(size_t)b * a.W + ch] : 0.f;
    for (int kb = a.nch - kPF; kb > -kPF; kb -= kPF) {
        float vp[kPF], vq[kPF];
#pragma unroll
        for (int j = 0; j < kPF; ++j) {
            if (kb + j >= 0) {
                const size_t pi = ((size_t)b * a.nch + kb + j) * a.W + ch;
                vp[j] = a.agg[pi];
                vq[j] = a.agg[pb + pi];
            }
        }
#pragma unroll
        for (int j = kPF - 1; j >= 0; --j) {
            if (kb + j < 0) continue;
            a.agg[pb + ((size_t)b * a.nch + kb + j) * a.W + ch] = c;
            c = fmaf(vp[j], c, vq[j]);
        }
    }
    if (a.dh0) a.dh0[(size_t)b * a.W + ch] = c;
}

// every output of a chunk, from the carry into its last token; thread = (row b, chunk k, channel
// pair ch, ch + 1), kPF2 tokens a batch
constexpr int kPF2 = 1;

struct ScanOut1 {             // the results of one token-channel
    float dy, dxc, dga, dgx, q;
};
__device__ __forceinline__ ScanOut1 scan_out_one(float kappa, float ga, float gx, float hp, float xcv, float yv,
                                                 float dz, int tanh_form, float& g) {
    const float r = sig_fast(ga), ig = sig_fast(gx);
    float at, beta;
    decay_beta_fast(kappa, r, at, beta);
    const float h = fmaf(at, hp, beta * (ig * xcv));
    float gl, gp;
    gelu_and_grad(yv, tanh_form, gl, gp);
    g = fmaf(dz, gl, g);
    ScanOut1 o;
    o.dy = dz * h * gp;
    const float dl_da = g * hp, dl_dbeta = g * ig * xcv, dl_di = g * beta * xcv;
    const float r_over_beta = beta > 0.f ? r * fm::rcpf(beta) : 0.f;
    o.q = dl_da * at * r - dl_dbeta * at * at * r_over_beta;
    o.dga = kappa * (1.0f - r) * o.q;
    o.dgx = dl_di * ig * (1.0f - ig);
    o.dxc = g * beta * ig;
    g *= at;                                             // the carry to the previous token
    return o;
}

// bf16 pair hi + lo of two fp32 values, each packed in one word
__device__ __forceinline__ void split_bf16x2(float v0, float v1, uint32_t& hi, uint32_t& lo) {
    __nv_bfloat162 h = __floats2bfloat162_rn(v0, v1);
    const float2 hf = __bfloat1622float2(h);
    __nv_bfloat162 l = __floats2bfloat162_rn(v0 - hf.x, v1 - hf.y);
    hi = *reinterpret_cast<uint32_t*>(&h);
    lo = *reinterpret_cast<uint32_t*>(&l);
}

__global__ void __launch_bounds__(kScanThreads, kOutMinBlocks) bwd_scan_out_kernel(ScanArgs a) {
    const int ch = 2 * (blockIdx.x * kScanThreads + threadIdx.x), k = blockIdx.y, b = blockIdx.z;
    if (ch >= a.W) return;
    const float kap0 = a.c * log_sigmoid_acc(a.lambda[ch]), kap1 = a.c * log_sigmoid_acc(a.lambda[ch + 1]);
    const float cs0 = a.c * sigmoid_acc(-a.lambda[ch]), cs1 = a.c * sigmoid_acc(-a.lambda[ch + 1]);
    const size_t pb = (size_t)a.B * a.nch * a.W, pi = ((size_t)b * a.nch + k) * a.W + ch;
    const float2 gin = *reinterpret_cast<const float2*>(a.agg + pb + pi);
    float g0 = gin.x, g1 = gin.y;
    float2 s_lam = make_float2(0.f, 0.f), s_ba = s_lam, s_bx = s_lam;
    const uint8_t* rrow = a.reset ? a.reset + (size_t)b * a.T : nullptr;
    const int t0 = k * kChunk, t1 = min(a.T, t0 + kChunk);
    for (int tb = t1 - kPF2; tb > t0 - kPF2; tb -= kPF2) {
        float2 vga[kPF2], vgx[kPF2], vhp[kPF2], vxh[kPF2], vxl[kPF2], vy[kPF2], vdz[kPF2];
        bool rs[kPF2];
        const size_t eb = ((size_t)b * a.T + tb) * a.W + ch;
#pragma unroll
        for (int j = 0; j < kPF2; ++j) {
            if (tb + j >= t0) {
                const size_t e = eb + (size_t)j * a.W;
                vga[j] = *reinterpret_cast<const float2*>(a.ga + e);
                vgx[j] = *reinterpret_cast<const float2*>(a.gx + e);
                vhp[j] = *reinterpret_cast<const float2*>(a.hprev + e);
                vxh[j] = bf2f(a.xc_hi + e);
                vxl[j] = bf2f(a.xc_lo + e);
                vy[j] = bf2f(a.y + e);
                vdz[j] = bf2f(a.dout + e);
                rs[j] = rrow && rrow[tb + j];
            }
        }
#pragma unroll
        for (int j = kPF2 - 1; j >= 0; --j) {
            if (tb + j < t0) continue;
            const size_t e = eb + (size_t)j * a.W;
            const ScanOut1 o0 = scan_out_one(kap0, vga[j].x, vgx[j].x, vhp[j].x, vxh[j].x + vxl[j].x, vy[j].x,
                                             vdz[j].x, a.gelu_tanh, g0);
            const ScanOut1 o1 = scan_out_one(kap1, vga[j].y, vgx[j].y, vhp[j].y, vxh[j].y + vxl[j].y, vy[j].y,
                                             vdz[j].y, a.gelu_tanh, g1);
            a.dy[e] = o0.dy;                             // caller's buffer: 4-byte aligned only
            a.dy[e + 1] = o1.dy;
            *reinterpret_cast<float2*>(a.dxc + e) = make_float2(o0.dxc, o1.dxc);
            uint32_t hi, lo;
            split_bf16x2(o0.dga, o1.dga, hi, lo);
            *reinterpret_cast<uint32_t*>(a.dga_hi + e) = hi;
            *reinterpret_cast<uint32_t*>(a.dga_lo + e) = lo;
            split_bf16x2(o0.dgx, o1.dgx, hi, lo);
            *reinterpret_cast<uint32_t*>(a.dgx_hi + e) = hi;
            *reinterpret_cast<uint32_t*>(a.dgx_lo + e) = lo;
            s_lam.x = fmaf(cs0, o0.q, s_lam.x);
            s_lam.y = fmaf(cs1, o1.q, s_lam.y);
            s_ba.x += o0.dga;
            s_ba.y += o1.dga;
            s_bx.x += o0.dgx;
            s_bx.y += o1.dgx;
            if (rs[j]) g0 = g1 = 0.f;                    // no carry across a segment start
        }
    }
    const size_t ps = (size_t)a.B * a.nch * a.W;
    *reinterpret_cast<float2*>(a.part + pi) = s_lam;
    *reinterpret_cast<float2*>(a.part + ps + pi) = s_ba;
    *reinterpret_cast<float2*>(a.part + 2 * ps + pi) = s_bx;
}

struct ConvTArgs {
    int B, T, W, ntb;
    const float* conv_w;
    const __nv_bfloat16* x;
    const __nv_bfloat16* tail0;       // [B][3][W] or nullptr
    const uint8_t* reset;
    const float* dtail_final;         // [B][3][W] or nullptr
    const float* dxc;
    float* dx;
    float* dtail0;                    // [B][3][W] or nullptr
    float* part;                      // [5][B * ntb][W]: dconv_w[4], dconv_b
};

// True when the window of token t reads position s (s in [t-3, t]): no reset in (s, t].
__device__ __forceinline__ bool window_reads(const uint8_t* rrow, int s, int t) {
    if (!rrow) return true;
    for (int p = (s + 1 > 0 ? s + 1 : 0); p <= t; ++p)
        if (rrow[p]) return false;
    return true;
}

// Thread = (row b, block of kTB positions, channels ch .. ch + 3); one walk over the block's
// positions s with the last three x and the next three dxc in registers: the parameter gradients
// of token t = s (the taps that read x_{s-3..s}) and dx_s (the taps of the tokens s..s+3 that
// read x_s).  A window reads position s for token t when no segment starts in (s, t]: L below is
// the last segment start at or before the current token.  Values are four channels as two pairs.
__device__ __forceinline__ float2 f2fma(float2 a, float2 b, float2 c) { return __ffma2_rn(a, b, c); }


// Four channels as two packed pairs.
struct F4 {
    float2 lo, hi;
};
__device__ __forceinline__ F4 f4fma(F4 x, F4 y, F4 z) { return {f2fma(x.lo, y.lo, z.lo), f2fma(x.hi, y.hi, z.hi)}; }
__device__ __forceinline__ F4 f4add(F4 x, F4 y) {
    return {make_float2(x.lo.x + y.lo.x, x.lo.y + y.lo.y), make_float2(x.hi.x + y.hi.x, x.hi.y + y.hi.y)};
}
__device__ __forceinline__ F4 f4zero() { return {make_float2(0.f, 0.f), make_float2(0.f, 0.f)}; }
__device__ __forceinline__ F4 f4_bf16x4(uint2 v) {
    return {__bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&v.x)),
            __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&v.y))};
}

__global__ void __launch_bounds__(128, kConvTMinBlocks) bwd_convT_kernel(ConvTArgs a) {
    const int ch = 4 * (blockIdx.x * 128 + threadIdx.x), tb = blockIdx.y, b = blockIdx.z;
    if (ch >= a.W) return;
    const int T = a.T;
    const int t0 = tb * kTB, t1 = min(T, t0 + kTB);
    const long long W = a.W;
    const uint8_t* rrow = a.reset ? a.reset + (size_t)b * T : nullptr;
    const size_t rowe = (size_t)b * T * W + ch;             // element (b, 0, ch)
    const uint2* xr = reinterpret_cast<const uint2*>(a.x + rowe);        // 4 bf16: 8 bytes
    const float4* dr = reinterpret_cast<const float4*>(a.dxc + rowe);
    float* dxr = a.dx + rowe;                               // caller's buffer: 4-byte aligned only
    const long long W4 = W / 4;                             // row pitch in channel quads
    F4 cw[kConvWidth];
#pragma unroll
    for (int k = 0; k < kConvWidth; ++k) {
        const float* c = a.conv_w + (size_t)k * W + ch;
        cw[k] = {make_float2(c[0], c[1]), make_float2(c[2], c[3])};
    }
    auto xval = [&](int s) -> F4 {                          // x_s, the initial history for s < 0
        if (s >= 0) return f4_bf16x4(xr[s * W4]);
        if (!a.tail0) return f4zero();
        const __nv_bfloat162* tp = reinterpret_cast<const __nv_bfloat162*>(a.tail0 + ((size_t)b * kHist + (kHist + s)) * W + ch);
        return {__bfloat1622float2(tp[0]), __bfloat1622float2(tp[1])};
    };
    auto dxcv = [&](int t) -> F4 {
        if (t < 0 || t >= T) return f4zero();
        const float4 v = dr[t * W4];
        return {make_float2(v.x, v.y), make_float2(v.z, v.w)};
    };
    auto rs = [&](int p) -> bool { return rrow && p >= 0 && p < T && rrow[p] != 0; };

    int L = -kHist - 1;                                     // no segment start within reach
    for (int p = max(0, t0 - kHist); p < t0; ++p)
        if (rs(p)) L = p;
    F4 xa = xval(t0 - 3), xb = xval(t0 - 2), xcc = xval(t0 - 1);   // x_{t-3}, x_{t-2}, x_{t-1}
    F4 s_cw[kConvWidth] = {f4zero(), f4zero(), f4zero(), f4zero()}, s_cb = f4zero();
    const int sb = tb == 0 ? -kHist : t0;                   // the first block also owns the history
    F4 d0 = dxcv(sb), d1 = dxcv(sb + 1), d2 = dxcv(sb + 2);
    bool q0 = rs(sb), q1 = rs(sb + 1), q2 = rs(sb + 2);
    // positions in batches of kPFC: the batch's loads are issued together, ahead of its arithmetic
    for (int s0 = sb; s0 < t1; s0 += kPFC) {
        F4 dn[kPFC], xn[kPFC];
        bool qn[kPFC];
#pragma unroll
        for (int j = 0; j < kPFC; ++j) {
            const int s = s0 + j;
            dn[j] = dxcv(s + 3);
            qn[j] = rs(s + 3);
            xn[j] = s >= t0 && s < t1 ? f4_bf16x4(xr[s * W4]) : f4zero();
        }
#pragma unroll
        for (int j = 0; j < kPFC; ++j) {
            const int s = s0 + j;
            if (s >= t1) break;
            const F4 d3 = dn[j];
            const bool q3 = qn[j];
            if (s >= t0) {                                  // token t = s: its four taps
                const F4 xs = xn[j];
                if (q0) L = s;
                s_cb = f4add(s_cb, d0);
                if (s - 3 >= L) s_cw[0] = f4fma(d0, xa, s_cw[0]);
                if (s - 2 >= L) s_cw[1] = f4fma(d0, xb, s_cw[1]);
                if (s - 1 >= L) s_cw[2] = f4fma(d0, xcc, s_cw[2]);
                s_cw[3] = f4fma(d0, xs, s_cw[3]);
                xa = xb; xb = xcc; xcc = xs;
            }
            // dx_s: tap k of token s + 3 - k, while no segment starts in (s, s + 3 - k]
            const bool ok1 = !q1, ok2 = ok1 && !q2, ok3 = ok2 && !q3;
            F4 acc = f4zero();
            if (ok3 && s + 3 >= 0 && s + 3 < T) acc = f4fma(cw[0], d3, acc);
            if (ok2 && s + 2 >= 0 && s + 2 < T) acc = f4fma(cw[1], d2, acc);
            if (ok1 && s + 1 >= 0 && s + 1 < T) acc = f4fma(cw[2], d1, acc);
            if (s >= 0) acc = f4fma(cw[3], d0, acc);
            if (a.dtail_final && s >= T - kHist && window_reads(rrow, s, T - 1)) {
                const float* df = a.dtail_final + ((size_t)b * kHist + (s - (T - kHist))) * W + ch;
                acc = f4add(acc, {make_float2(df[0], df[1]), make_float2(df[2], df[3])});
            }
            if (s >= 0) {
                float* o = dxr + (size_t)s * W;
                o[0] = acc.lo.x;
                o[1] = acc.lo.y;
                o[2] = acc.hi.x;
                o[3] = acc.hi.y;
            } else if (a.dtail0) {
                float* dt = a.dtail0 + ((size_t)b * kHist + (kHist + s)) * W + ch;
                dt[0] = acc.lo.x;
                dt[1] = acc.lo.y;
                dt[2] = acc.hi.x;
                dt[3] = acc.hi.y;
            }
            d0 = d1; d1 = d2; d2 = d3;
            q0 = q1; q1 = q2; q2 = q3;
        }
    }
    const size_t pb = (size_t)a.B * a.ntb * W, pi = ((size_t)b * a.ntb + tb) * W + ch;
#pragma unroll
    for (int k = 0; k < kConvWidth; ++k)
        *reinterpret_cast<float4*>(a.part + k * pb + pi) = make_float4(s_cw[k].lo.x, s_cw[k].lo.y, s_cw[k].hi.x, s_cw[k].hi.y);
    *reinterpret_cast<float4*>(a.part + 4 * pb + pi) = make_float4(s_cb.lo.x, s_cb.lo.y, s_cb.hi.x, s_cb.hi.y);
}

// ---------------------------------------------------------------- 6. fixed-order sums -------
struct ReduceArgs {
    int B, ntb, nch, W, H, splits;
    const float* part_scan;
    const float* part_conv;
    const float* dw;                  // [2][splits][H][256][256]
    rglru_grads g;
};

// Block = 32 channels x kRedGroups row groups: group g sums the partial rows i = g (mod
// kRedGroups) in order, then the groups are added in order -- a fixed order, so the sums repeat
// bitwise.
constexpr int kRedGroups = 16;
__global__ void __launch_bounds__(32 * kRedGroups) bwdtc_reduce_vec_kernel(ReduceArgs a) {
    __shared__ float red[8][kRedGroups][33];
    const int c = threadIdx.x, g = threadIdx.y;
    const int ch = blockIdx.x * 32 + c;
    float s[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
    if (ch < a.W) {
        const size_t ps = (size_t)a.B * a.nch * a.W;
        for (int i = g; i < a.B * a.nch; i += kRedGroups)
#pragma unroll
            for (int k = 0; k < 3; ++k) s[k] += a.part_scan[k * ps + (size_t)i * a.W + ch];
        const size_t pc = (size_t)a.B * a.ntb * a.W;
        for (int i = g; i < a.B * a.ntb; i += kRedGroups)
#pragma unroll
            for (int k = 0; k < 5; ++k) s[3 + k] += a.part_conv[k * pc + (size_t)i * a.W + ch];
    }
#pragma unroll
    for (int k = 0; k < 8; ++k) red[k][g][c] = s[k];
    __syncthreads();
    if (g < 8 && ch < a.W) {
        float t = 0.f;
        for (int j = 0; j < kRedGroups; ++j) t += red[g][j][c];
        if (g == 0) a.g.dlambda[ch] = t;
        else if (g == 1) a.g.db_a[ch] = t;
        else if (g == 2) a.g.db_x[ch] = t;
        else if (g < 7) a.g.dconv_w[(size_t)(g - 3) * a.W + ch] = t;
        else a.g.dconv_b[ch] = t;
    }
}

__global__ void bwdtc_reduce_w_kernel(ReduceArgs a) {
    const size_t n = (size_t)a.H * DH * DH;
    const size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (i >= n) return;
#pragma unroll
    for (int gate = 0; gate < 2; ++gate) {
        float s = 0.f;
        for (int sp = 0; sp < a.splits; ++sp) s += a.dw[((size_t)gate * a.splits + sp) * n + i];
        (gate ? a.g.dw_x : a.g.dw_a)[i] = s;
    }
}

GemmPair pair_tokens_x_weights(const __nv_bfloat16* dg, const __nv_bfloat16* w, long long tokens, int H, int W) {
    // A (m = token, k = output channel o of head h): dg[token][h * 256 + o], K-major
    // B (n = input channel i, k = o): W[h][i][o], K-major (rows h * 256 + i)
    GemmPair p{};
    p.a = dg; p.a_rows = tokens; p.a_cols = W; p.a_ld = W;
    p.a_kmajor = 1; p.a_boff_row = 0; p.a_boff_col = 0; p.a_bstep_row = 0; p.a_bstep_col = DH;
    p.b = w; p.b_rows = (long long)H * DH; p.b_cols = DH; p.b_ld = DH;
    p.b_kmajor = 1; p.b_boff_row = 0; p.b_boff_col = 0; p.b_bstep_row = DH; p.b_bstep_col = 0;
    p.K = DH;
    return p;
}

GemmPair pair_xc_dg(const __nv_bfloat16* xc, const __nv_bfloat16* dg, long long tokens, int W) {
    // A (m = input channel i, k = token): xc[token][h * 256 + i], M-major
    // B (n = output channel o, k = token): dg[token][h * 256 + o], N-major
    GemmPair p{};
    p.a = xc; p.a_rows = tokens; p.a_cols = W; p.a_ld = W;
    p.a_kmajor = 0; p.a_boff_row = 0; p.a_boff_col = 0; p.a_bstep_row = 0; p.a_bstep_col = DH;
    p.b = dg; p.b_rows = tokens; p.b_cols = W; p.b_ld = W;
    p.b_kmajor = 0; p.b_boff_row = 0; p.b_boff_col = 0; p.b_bstep_row = 0; p.b_bstep_col = DH;
    p.K = (int)((tokens + 63) / 64 * 64);   // rows past the tokens read as zeros
    return p;
}

}  // namespace

bool backward_tc_supported(const rglru_dims* d) {
    return d->act_dtype == RGLRU_BF16 && d->head_dim == DH && !(d->flags & RGLRU_FLAG_GENERIC);
}

size_t backward_tc_workspace(const rglru_dims* d) { return layout(d).total; }

int backward_tc_launches(const rglru_dims* d) {
    (void)d;
    return 11;  // prefill (memset + kernel), 3 scan kernels, GEMM, conv transpose, 2 GEMMs, 2 reductions
}

cudaError_t launch_backward_tc(const rglru_dims* d, const rglru_params* p, const void* x, const void* y,
                               const uint8_t* reset, const rglru_state* st0, const void* dout,
                               const float* dh_final, const float* dtail_final, const rglru_grads* grads,
                               void* ws, size_t ws_bytes, cudaStream_t s) {
    const Layout l = layout(d);
    if (l.total > ws_bytes) return cudaErrorInvalidValue;
    uint8_t* w = static_cast<uint8_t*>(ws);
    DeviceStatus* status = reinterpret_cast<DeviceStatus*>(w);
    const int B = d->batch, T = d->seq_len, H = d->heads, W = H * DH;
    const long long tokens = (long long)B * T;
    auto f32 = [&](size_t o) { return reinterpret_cast<float*>(w + o); };
    auto b16 = [&](size_t o) { return reinterpret_cast<__nv_bfloat16*>(w + o); };

    // 1. the forward again, keeping what the gradients need
    PrefillSave sv{};
    sv.ga = f32(l.ga); sv.gx = f32(l.gx); sv.hprev = f32(l.hprev);
    sv.xc_hi = b16(l.xc_hi); sv.xc_lo = b16(l.xc_lo);
    rglru_state st_copy{};
    rglru_state* stp = nullptr;
    if (st0) {   // the save mode reads the initial state and writes nothing back
        st_copy = *st0;
        stp = &st_copy;
    }
    cudaError_t e = launch_fused_prefill_save(d, p, x, reset, stp, &sv, w + l.fwd, ws_bytes - l.fwd, status, s);
    if (e != cudaSuccess) return e;

    // 2. the reverse scan
    ScanArgs sa{};
    sa.B = B; sa.T = T; sa.W = W; sa.nch = l.nch; sa.c = d->c; sa.gelu_tanh = d->gelu_tanh;
    sa.lambda = p->lambda; sa.y = static_cast<const __nv_bfloat16*>(y);
    sa.dout = static_cast<const __nv_bfloat16*>(dout); sa.reset = reset; sa.dh_final = dh_final;
    sa.ga = f32(l.ga); sa.gx = f32(l.gx); sa.hprev = f32(l.hprev);
    sa.xc_hi = b16(l.xc_hi); sa.xc_lo = b16(l.xc_lo);
    sa.dy = grads->dy; sa.dxc = f32(l.dxc);
    sa.dga_hi = b16(l.dga_hi); sa.dga_lo = b16(l.dga_lo); sa.dgx_hi = b16(l.dgx_hi); sa.dgx_lo = b16(l.dgx_lo);
    sa.dh0 = grads->dh0; sa.agg = f32(l.agg); sa.part = f32(l.part_scan);
    const unsigned cblk = (unsigned)((W + kScanThreads - 1) / kScanThreads);
    const unsigned cblk2 = (unsigned)((W / 2 + kScanThreads - 1) / kScanThreads);   // channel pairs
    bwd_scan_agg_kernel<<<dim3(cblk2, l.nch, B), kScanThreads, 0, s>>>(sa);
    bwd_scan_carry_kernel<<<dim3(cblk, B), kScanThreads, 0, s>>>(sa);
    bwd_scan_out_kernel<<<dim3(cblk2, l.nch, B), kScanThreads, 0, s>>>(sa);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;

    // 3. dL/dxc += dga W_a^T + dgx W_x^T (hi and lo parts of dga, dgx), in place
    const __nv_bfloat16* wa = static_cast<const __nv_bfloat16*>(p->w_a);
    const __nv_bfloat16* wx = static_cast<const __nv_bfloat16*>(p->w_x);
    GemmOperands gx{};
    gx.M = (int)tokens; gx.N = DH; gx.batch = H; gx.splits = 1; gx.npairs = 4;
    gx.p[0] = pair_tokens_x_weights(b16(l.dga_hi), wa, tokens, H, W);
    gx.p[1] = pair_tokens_x_weights(b16(l.dga_lo), wa, tokens, H, W);
    gx.p[2] = pair_tokens_x_weights(b16(l.dgx_hi), wx, tokens, H, W);
    gx.p[3] = pair_tokens_x_weights(b16(l.dgx_lo), wx, tokens, H, W);
    gx.C = f32(l.dxc); gx.c_ld = W; gx.c_bstride = DH; gx.c_split = 0;
    gx.Cadd = f32(l.dxc); gx.add_ld = W; gx.add_bstride = DH;
    gx.status = status;
    e = launch_gemm(gx, s);
    if (e != cudaSuccess) return e;

    // 4. the conv's transpose
    ConvTArgs ca{};
    ca.B = B; ca.T = T; ca.W = W; ca.ntb = l.ntb;
    ca.conv_w = p->conv_w; ca.x = static_cast<const __nv_bfloat16*>(x);
    ca.tail0 = st0 ? static_cast<const __nv_bfloat16*>(st0->conv_tail) : nullptr;
    ca.reset = reset; ca.dtail_final = dtail_final; ca.dxc = f32(l.dxc);
    ca.dx = grads->dx; ca.dtail0 = grads->dtail0; ca.part = f32(l.part_conv);
    bwd_convT_kernel<<<dim3((W + 511) / 512, l.ntb, B), 128, 0, s>>>(ca);   // 4 channels a thread
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;

    // 5. dW = xc^T dg per head and gate, K (the tokens) cut into slices so that the tiles of
    //    both gates' GEMM fill the SMs about once
    int dev = 0, sms = 148;
    if (cudaGetDevice(&dev) != cudaSuccess || cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
        return cudaGetLastError();
    const int wtiles = H;                                  // 256 x 256 output tiles (a CTA pair each) per gate
    const int splits = std::max(1, std::min(kMaxSplits, (sms / 2) / wtiles));
    for (int gate = 0; gate < 2; ++gate) {
        GemmOperands gw{};
        gw.M = DH; gw.N = DH; gw.batch = H; gw.splits = splits; gw.npairs = 3;
        const __nv_bfloat16* hi = b16(gate ? l.dgx_hi : l.dga_hi);
        const __nv_bfloat16* lo = b16(gate ? l.dgx_lo : l.dga_lo);
        gw.p[0] = pair_xc_dg(b16(l.xc_hi), hi, tokens, W);
        gw.p[1] = pair_xc_dg(b16(l.xc_hi), lo, tokens, W);
        gw.p[2] = pair_xc_dg(b16(l.xc_lo), hi, tokens, W);
        gw.C = f32(l.dw) + (size_t)gate * splits * H * DH * DH;
        gw.c_ld = DH; gw.c_bstride = (long long)DH * DH; gw.c_split = (long long)H * DH * DH;
        gw.Cadd = nullptr;
        gw.status = status;
        e = launch_gemm(gw, s);
        if (e != cudaSuccess) return e;
    }

    // 6. every partial sum, in a fixed order
    ReduceArgs ra{};
    ra.B = B; ra.ntb = l.ntb; ra.nch = l.nch; ra.W = W; ra.H = H; ra.splits = splits;
    ra.part_scan = f32(l.part_scan); ra.part_conv = f32(l.part_conv); ra.dw = f32(l.dw);
    ra.g = *grads;
    bwdtc_reduce_vec_kernel<<<(W + 31) / 32, dim3(32, kRedGroups), 0, s>>>(ra);
    const size_t nw = (size_t)H * DH * DH;
    bwdtc_reduce_w_kernel<<<(unsigned)((nw + 255) / 256), 256, 0, s>>>(ra);
    return cudaGetLastError();
}

}  // namespace rglru
