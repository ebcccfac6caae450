// fused_decode.cu -- tensor-core RG-LRU decode step for bf16 activations, head_dim 256 (sm_100a).
//
// A decode step updates every batch row by one token.  There is no recurrence across tokens
// inside a call, so the batch is the parallel dimension and the gate contraction is a plain
// GEMM per head: D[row, o] = sum_i xc[row, i] W[h][i][o] with M = rows, N = output channels,
// K = 256 input channels.  Two launches:
//
//   1. conv_shift_kernel: per (row, 8 channels) the width-4 causal conv over the carried
//      history and the new input, written as bf16 into workspace scratch (it is the tensor-core
//      operand), and the history shifted in place (oldest out, x in).  A row with reset[b] set
//      starts from an empty history.
//   2. decode_gates_kernel: a CTA per (head, 128-row tile, 64-channel tile).  TMA brings the
//      128 x 256 conv tile (K-major, 128-byte swizzle) and the 256 x 64 slices of W_a, W_x
//      (as stored: output channel contiguous, i.e. MN-major for the MMA) into shared memory;
//      one thread issues tcgen05.mma (M = 128, N = 64, K = 256 per gate) into TMEM; 8 epilogue
//      warps (thread = row, 32 channels each) read the accumulators, apply the gates, update
//      the fp32 state h in place and write out = h * GeLU(y) with 16-byte vector accesses.
//
// The element-wise arithmetic is that of the prefill kernel (fused_prefill.cu): one tanh per
// gate, expm1 of the log-decay by its series near zero, sqrt(1 - a^2) without cancellation,
// GeLU in its tanh form fitted to y Phi(y).  Sources ("Griffin Guide: RecurrentGemma, RG-LRU &
// Hybrid Attention"): "1. Formulation of the RG-LRU Gating Mechanism", "2. The Role of
// Square-Root Variance Normalization", "1. Temporal Filtering via Separable 1D Convolutions",
// "2. Non-Linear Multiplicative Gating with GeLU", "3. Block-Diagonal Sharding for
// Zero-Communication Tensor Parallelism", and the listing's RGLRU.step.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "common.cuh"
#include "kernels.h"
#include "sm100.cuh"

namespace rglru {

// shared with fused_prefill.cu (host side)
namespace tc {
bool make_map_2d_sw128(CUtensorMap* m, const void* base, uint64_t inner, uint64_t outer, uint64_t row_bytes,
                       uint32_t box_inner, uint32_t box_outer);
}

namespace dec {

using namespace sm100;

constexpr int DH = 256;
constexpr int MT = 128;                 // rows per CTA (MMA M, TMEM lanes)
constexpr int NT = 64;                  // output channels per CTA (MMA N)
constexpr int KSTEPS = DH / 16;
constexpr int kWarpMma = 8, kWarpTma = 9;     // warps 0-7: epilogue (4 lane quarters x 2 channel halves)
constexpr int kThreads = 10 * 32;

constexpr uint32_t A_BYTES = MT * DH * 2;            // 65536: 4 K-blocks of 128 rows x 128 B
constexpr uint32_t A_KBLK = MT * 128;                // 16384
constexpr uint32_t B_BYTES = DH * NT * 2;            // 32768 per gate: 256 K-rows x 128 B
constexpr uint32_t OFF_A = 0;
constexpr uint32_t OFF_BA = OFF_A + A_BYTES;
constexpr uint32_t OFF_BX = OFF_BA + B_BYTES;
constexpr uint32_t OFF_CONST = OFF_BX + B_BYTES;     // hk, b_a / 2, b_x / 2 per channel: 3 x 64 fp32
constexpr uint32_t OFF_BAR = OFF_CONST + 3 * NT * 4;
constexpr uint32_t OFF_MISC = OFF_BAR + 32;
constexpr uint32_t SMEM_BYTES = OFF_MISC + 32 + 1024;
constexpr uint32_t TMEM_COLS = 128;                  // D_a [0,64), D_x [64,128)

struct Args {
    int B, H, mtiles;
    float c;
    int gelu_tanh;
    unsigned long long timeout_ns;
    const float* b_a;
    const float* b_x;
    const float* lambda;
    const uint8_t* reset;
    const __nv_bfloat16* y;
    float* h;
    __nv_bfloat16* out;
    DeviceStatus* status;
};

__device__ __forceinline__ float bf16lo(uint32_t v) { return __uint_as_float(v << 16); }
__device__ __forceinline__ float bf16hi(uint32_t v) { return __uint_as_float(v & 0xFFFF0000u); }
__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
    __nv_bfloat162 p = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t*>(&p);
}
__device__ __forceinline__ float sqrt_approx(float x) {
    float r;
    asm("sqrt.approx.ftz.f32 %0, %1;" : "=f"(r) : "f"(x));
    return r;
}

// Shared-memory matrix descriptor for an MN-major operand in the 128-byte swizzle layout: rows
// of 128 B (64 bf16 along N) for consecutive K, 8-row atoms of 1024 B stacked along K at the
// stride byte offset (1024 B); the leading byte offset (between 64-wide N atoms) is unused for
// N = 64.  Same bit fields as desc_k_sw128.
__device__ __forceinline__ uint64_t desc_mn_sw128(uint32_t smem_addr) {
    uint64_t d = 0;
    d |= (uint64_t)((smem_addr >> 4) & 0x3FFF);
    d |= (uint64_t)(B_BYTES >> 4) << 16;
    d |= (uint64_t)(1024 >> 4) << 32;
    d |= (uint64_t)1 << 46;
    d |= (uint64_t)2 << 61;
    return d;
}

// Instruction descriptor: fp32 accumulator, bf16 A (K-major) and B (MN-major), M x N.
__host__ __device__ constexpr uint32_t idesc_bf16_f32_bmn(int M, int N) {
    return (1u << 4) | (1u << 7) | (1u << 10) | (1u << 16) | ((uint32_t)(N >> 3) << 17) |
           ((uint32_t)(M >> 4) << 24);
}

__device__ bool wait_bounded(uint32_t bar, uint32_t parity, const Args& a, volatile int* abort, unsigned where) {
    if (mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = globaltimer_ns();
    for (;;) {
        if (mbar_try_wait_sleep(bar, parity, 20000u)) return true;
        if (*abort) return false;
        if (globaltimer_ns() - t0 > a.timeout_ns) {
            latch_status(a.status, RGLRU_ERR_TIMEOUT, where, blockIdx.x, parity);
            *abort = 1;
            return false;
        }
    }
}

// ---------------------------------------------------------------- 1. conv + history shift --
__global__ void __launch_bounds__(256)
conv_shift_kernel(const __nv_bfloat16* __restrict__ x, __nv_bfloat16* tail, const float* __restrict__ conv_w,
                  const float* __restrict__ conv_b, const uint8_t* __restrict__ reset, __nv_bfloat16* xc, int B, int W) {
    // the gate kernel that follows may start its set-up now: it waits for this grid before it
    // reads the conv output
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    const int groups = W / 8;
    const long long idx = (long long)blockIdx.x * blockDim.x + threadIdx.x;
    if (idx >= (long long)B * groups) return;
    const int b = (int)(idx / groups), c8 = (int)(idx % groups) * 8;
    const size_t row = (size_t)b * W + c8;
    __nv_bfloat16* tl = tail + (size_t)b * kHist * W + c8;
    const uint4 xv = *reinterpret_cast<const uint4*>(x + row);
    uint4 t0 = make_uint4(0, 0, 0, 0), t1 = t0, t2 = t0;
    if (!(reset && reset[b])) {
        t0 = *reinterpret_cast<const uint4*>(tl);
        t1 = *reinterpret_cast<const uint4*>(tl + W);
        t2 = *reinterpret_cast<const uint4*>(tl + 2 * W);
    }
    // taps k = 0..3 (oldest .. current) and the bias of these 8 channels, 16-byte loads
    float wk[kConvWidth][8], bias[8];
#pragma unroll
    for (int k = 0; k < kConvWidth; ++k) {
        const float4 w0 = *reinterpret_cast<const float4*>(conv_w + (size_t)k * W + c8);
        const float4 w1 = *reinterpret_cast<const float4*>(conv_w + (size_t)k * W + c8 + 4);
        wk[k][0] = w0.x; wk[k][1] = w0.y; wk[k][2] = w0.z; wk[k][3] = w0.w;
        wk[k][4] = w1.x; wk[k][5] = w1.y; wk[k][6] = w1.z; wk[k][7] = w1.w;
    }
    if (conv_b) {
        const float4 b0 = *reinterpret_cast<const float4*>(conv_b + c8);
        const float4 b1 = *reinterpret_cast<const float4*>(conv_b + c8 + 4);
        bias[0] = b0.x; bias[1] = b0.y; bias[2] = b0.z; bias[3] = b0.w;
        bias[4] = b1.x; bias[5] = b1.y; bias[6] = b1.z; bias[7] = b1.w;
    } else {
#pragma unroll
        for (int e = 0; e < 8; ++e) bias[e] = 0.f;
    }
    const uint32_t* px = reinterpret_cast<const uint32_t*>(&xv);
    const uint32_t* p0 = reinterpret_cast<const uint32_t*>(&t0);
    const uint32_t* p1 = reinterpret_cast<const uint32_t*>(&t1);
    const uint32_t* p2 = reinterpret_cast<const uint32_t*>(&t2);
    uint4 o;
    uint32_t* po = reinterpret_cast<uint32_t*>(&o);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        float r[2];
#pragma unroll
        for (int e = 0; e < 2; ++e) {
            const int c = 2 * i + e;
            const float v0 = e ? bf16hi(p0[i]) : bf16lo(p0[i]);
            const float v1 = e ? bf16hi(p1[i]) : bf16lo(p1[i]);
            const float v2 = e ? bf16hi(p2[i]) : bf16lo(p2[i]);
            const float v3 = e ? bf16hi(px[i]) : bf16lo(px[i]);
            float acc = fmaf(wk[0][c], v0, bias[c]);
            acc = fmaf(wk[1][c], v1, acc);
            acc = fmaf(wk[2][c], v2, acc);
            r[e] = fmaf(wk[3][c], v3, acc);
        }
        po[i] = pack_bf16x2(r[0], r[1]);
    }
    *reinterpret_cast<uint4*>(xc + row) = o;
    *reinterpret_cast<uint4*>(tl) = t1;
    *reinterpret_cast<uint4*>(tl + W) = t2;
    *reinterpret_cast<uint4*>(tl + 2 * W) = xv;
}

// ---------------------------------------------------------------- 2. gates + state update --
__global__ void __launch_bounds__(kThreads, 1)
decode_gates_kernel(const __grid_constant__ CUtensorMap map_xc, const __grid_constant__ CUtensorMap map_wa,
                    const __grid_constant__ CUtensorMap map_wx, const Args a) {
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const uint32_t sbase = smem_u32(smem);
    const uint32_t bar_full = sbase + OFF_BAR, bar_acc = sbase + OFF_BAR + 8;
    volatile uint32_t* tmem_base_s = reinterpret_cast<volatile uint32_t*>(smem + OFF_MISC);
    volatile int* abort = reinterpret_cast<volatile int*>(smem + OFF_MISC + 16);
    float* s_hk = reinterpret_cast<float*>(smem + OFF_CONST);
    float* s_ba = s_hk + NT;
    float* s_bx = s_ba + NT;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    // CTA -> (head, row tile, channel tile); channel tiles of a head are adjacent
    const int nt = blockIdx.x % (DH / NT);
    const int mt = (blockIdx.x / (DH / NT)) % a.mtiles;
    const int head = blockIdx.x / ((DH / NT) * a.mtiles);
    const int W = a.H * DH;
    const int ch0 = head * DH + nt * NT;                  // first global channel of the tile

    if (threadIdx.x == 0) {
        mbar_init(bar_full, 1);
        mbar_init(bar_acc, 1);
        *abort = 0;
        fence_barrier_init();
    }
    if (threadIdx.x < NT) {
        const int ch = ch0 + threadIdx.x;
        s_hk[threadIdx.x] = 0.5f * a.c * log_sigmoid_acc(a.lambda[ch]);
        s_ba[threadIdx.x] = a.b_a ? 0.5f * a.b_a[ch] : 0.f;
        s_bx[threadIdx.x] = a.b_x ? 0.5f * a.b_x[ch] : 0.f;
    }
    if (warp == kWarpMma) {
        tmem_alloc(smem_u32((const void*)tmem_base_s), TMEM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_base_s;

    if (warp == kWarpTma) {
        if (lane == 0) {
            prefetch_tensormap(&map_xc);
            prefetch_tensormap(&map_wa);
            prefetch_tensormap(&map_wx);
            mbar_arrive_expect_tx(bar_full, A_BYTES + 2 * B_BYTES);
            for (int kb = 0; kb < DH / 64; ++kb) {
                tma_load_2d(sbase + OFF_BA + kb * 8192, &map_wa, nt * NT, head * DH + kb * 64, bar_full);
                tma_load_2d(sbase + OFF_BX + kb * 8192, &map_wx, nt * NT, head * DH + kb * 64, bar_full);
            }
            // the conv output is written by the preceding conv kernel (a no-op without a
            // programmatic launch dependency)
            asm volatile("griddepcontrol.wait;" ::: "memory");
            for (int kb = 0; kb < DH / 64; ++kb)
                tma_load_2d(sbase + OFF_A + kb * A_KBLK, &map_xc, head * DH + kb * 64, mt * MT, bar_full);
            // never leave the CTA with a bulk copy still writing its shared memory
            const uint64_t t0 = globaltimer_ns();
            while (!mbar_try_wait_sleep(bar_full, 0, 20000u) && globaltimer_ns() - t0 < a.timeout_ns) {
            }
        }
    } else if (warp == kWarpMma) {
        if (lane == 0) {
            const uint32_t idesc = idesc_bf16_f32_bmn(MT, NT);
            if (wait_bounded(bar_full, 0, a, abort, 1)) {
                tc_fence_after();
#pragma unroll 1
                for (int g = 0; g < 2; ++g) {
                    const uint32_t bsm = sbase + (g ? OFF_BX : OFF_BA);
#pragma unroll
                    for (int ks = 0; ks < KSTEPS; ++ks) {
                        const uint64_t ad = desc_k_sw128(sbase + OFF_A + (ks >> 2) * A_KBLK + (ks & 3) * 32);
                        const uint64_t bd = desc_mn_sw128(bsm + ks * 16 * 128);
                        mma_ss(tmem + g * NT, ad, bd, idesc, ks > 0 ? 1u : 0u);
                    }
                }
            }
            mma_commit(bar_acc);     // also when the load failed: the epilogue must not wait forever
        }
    } else {
        // ================================ epilogue ============================================
        const int q = warp & 3, cg = warp >> 2;           // lane quarter, 32-channel half of the tile
        const int r = q * 32 + lane;                      // row within the tile
        const int b = mt * MT + r;
        const bool valid = b < a.B;
        const float gk1 = a.gelu_tanh ? 2.0f * 0.79788456080286535588f : 2.0f * 0.79879267f;
        const float gk3 = a.gelu_tanh ? 8.0f * 0.044715f * 0.79788456080286535588f : 8.0f * 0.03528805f;
        // this row's state and y while the tensor cores run (rows past the batch read nothing)
        const bool rst = valid && a.reset && a.reset[b];
        const size_t off = (size_t)(valid ? b : 0) * W + ch0 + cg * 32;
        float* hp = a.h + off;
        const __nv_bfloat16* yp = a.y + off;
        __nv_bfloat16* op = a.out + off;
        float4 hq[8];
        uint4 yq[4];
#pragma unroll
        for (int i = 0; i < 8; ++i)
            hq[i] = (valid && !rst) ? *reinterpret_cast<const float4*>(hp + 4 * i) : make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
        for (int i = 0; i < 4; ++i) yq[i] = valid ? *reinterpret_cast<const uint4*>(yp + 8 * i) : make_uint4(0, 0, 0, 0);
        // uniform across the warp: the TMEM loads below are warp-collective
        const bool ok = __all_sync(0xffffffffu, wait_bounded(bar_acc, 0, a, abort, 2));
        tc_fence_after();
        const uint32_t taddr = tmem + ((uint32_t)(q * 32) << 16) + cg * 32;
        const int cbase = nt * NT + cg * 32;              // channel within the head
#pragma unroll
        for (int v = 0; v < 4; ++v) {                     // 8 channels per step
            float ga[8], gx[8];
            tmem_ld8(taddr + v * 8, ga);
            tmem_ld8(taddr + NT + v * 8, gx);
            tmem_wait_ld();
            if (!(ok && valid)) continue;
            // conv output of this row: a 16-byte chunk of the swizzled A tile
            const int cl = cbase + v * 8;
            const uint32_t aoff = (uint32_t)(cl >> 6) * A_KBLK + (uint32_t)(r >> 3) * 1024 + (uint32_t)(r & 7) * 128 +
                                  ((uint32_t)(((cl & 63) >> 3) ^ (r & 7)) << 4);
            const uint4 xq = *reinterpret_cast<const uint4*>(smem + OFF_A + aoff);
            float hv[8];
            const float4 h0 = hq[2 * v], h1 = hq[2 * v + 1];
            hv[0] = h0.x; hv[1] = h0.y; hv[2] = h0.z; hv[3] = h0.w;
            hv[4] = h1.x; hv[5] = h1.y; hv[6] = h1.z; hv[7] = h1.w;
            const uint32_t* xw = reinterpret_cast<const uint32_t*>(&xq);
            const uint32_t* yw = reinterpret_cast<const uint32_t*>(&yq[v]);
            uint32_t ow[4];
#pragma unroll
            for (int e2 = 0; e2 < 4; ++e2) {
                float o[2];
#pragma unroll
                for (int e1 = 0; e1 < 2; ++e1) {
                    const int e = 2 * e2 + e1;
                    const int jc = cg * 32 + v * 8 + e;   // column within the tile
                    const float xcv = e1 ? bf16hi(xw[e2]) : bf16lo(xw[e2]);
                    const float yv = e1 ? bf16hi(yw[e2]) : bf16lo(yw[e2]);
                    const float hk = s_hk[jc];
                    const float da = fmaf(ga[e], 0.5f, s_ba[jc]);
                    const float dx = fmaf(gx[e], 0.5f, s_bx[jc]);
                    const float l = fmaf(tanh_approx(da), hk, hk);
                    float em;
                    if (l > -0.125f) {
                        float pp = fmaf(l, 1.0f / 24.0f, 1.0f / 6.0f);
                        pp = fmaf(l, pp, 0.5f);
                        pp = fmaf(l, pp, 1.0f);
                        em = l * pp;
                    } else {
                        em = ex2_approx(l * 1.4426950408889634f) - 1.0f;
                    }
                    const float at = 1.0f + em;
                    const float bh = sqrt_approx(em * fmaf(em, -0.25f, -0.5f));
                    const float w = bh * xcv;
                    const float u = fmaf(w, tanh_approx(dx), w);
                    const float hn = fmaf(at, hv[e], u);
                    hv[e] = hn;
                    const float hy = 0.5f * yv;
                    const float t = tanh_approx(hy * fmaf(hy * hy, gk3, gk1));
                    const float m = hn * hy;
                    o[e1] = fmaf(m, t, m);
                }
                ow[e2] = pack_bf16x2(o[0], o[1]);
            }
            *reinterpret_cast<float4*>(hp + v * 8) = make_float4(hv[0], hv[1], hv[2], hv[3]);
            *reinterpret_cast<float4*>(hp + v * 8 + 4) = make_float4(hv[4], hv[5], hv[6], hv[7]);
            *reinterpret_cast<uint4*>(op + v * 8) = make_uint4(ow[0], ow[1], ow[2], ow[3]);
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == kWarpMma) {
        tc_fence_after();
        tmem_dealloc(tmem, TMEM_COLS);
    }
}

}  // namespace dec

bool fused_decode_supported(const rglru_dims* d) {
    return d->act_dtype == RGLRU_BF16 && d->head_dim == dec::DH && !(d->flags & RGLRU_FLAG_GENERIC);
}

size_t fused_decode_workspace(const rglru_dims* d) {
    const size_t W = (size_t)d->heads * d->head_dim;
    return 256 + (((size_t)d->batch * W * 2 + 255) & ~size_t(255));
}

int fused_decode_launches(const rglru_dims* d) {
    (void)d;
    return 2;
}

cudaError_t launch_fused_decode(const rglru_dims* d, const rglru_params* p, const void* x, const void* y,
                                const uint8_t* reset, rglru_state* st, void* out, void* ws, size_t ws_bytes,
                                cudaStream_t s) {
    using namespace dec;
    if (fused_decode_workspace(d) > ws_bytes) return cudaErrorInvalidValue;
    const int B = d->batch, H = d->heads, W = H * DH;
    __nv_bfloat16* xc = reinterpret_cast<__nv_bfloat16*>(static_cast<uint8_t*>(ws) + 256);
    {
        const long long n = (long long)B * (W / 8);
        const int threads = 256;
        const long long blocks = (n + threads - 1) / threads;
        conv_shift_kernel<<<(unsigned)blocks, threads, 0, s>>>(static_cast<const __nv_bfloat16*>(x),
                                                               static_cast<__nv_bfloat16*>(st->conv_tail), p->conv_w,
                                                               p->conv_b, reset, xc, B, W);
        cudaError_t e = cudaGetLastError();
        if (e != cudaSuccess) return e;
    }
    CUtensorMap mxc, mwa, mwx;
    if (!tc::make_map_2d_sw128(&mxc, xc, W, B, (uint64_t)W * 2, 64, MT) ||
        !tc::make_map_2d_sw128(&mwa, p->w_a, DH, (uint64_t)H * DH, DH * 2, NT, 64) ||
        !tc::make_map_2d_sw128(&mwx, p->w_x, DH, (uint64_t)H * DH, DH * 2, NT, 64))
        return cudaErrorInvalidValue;
    cudaError_t e = set_smem_once(decode_gates_kernel, (int)SMEM_BYTES);
    if (e != cudaSuccess) return e;
    Args a;
    a.B = B; a.H = H; a.mtiles = (B + MT - 1) / MT;
    a.c = d->c; a.gelu_tanh = d->gelu_tanh;
    a.timeout_ns = 1000000000ull;
    a.b_a = p->b_a; a.b_x = p->b_x; a.lambda = p->lambda; a.reset = reset;
    a.y = static_cast<const __nv_bfloat16*>(y);
    a.h = st->h;
    a.out = static_cast<__nv_bfloat16*>(out);
    a.status = reinterpret_cast<DeviceStatus*>(ws);
    // programmatic dependent launch: this kernel's set-up (barriers, TMEM, constants, weight
    // tiles, state prefetch) overlaps the conv kernel; it waits for it before loading the conv
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)(H * a.mtiles * (DH / NT)));
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = SMEM_BYTES;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    e = cudaLaunchKernelEx(&cfg, decode_gates_kernel, mxc, mwa, mwx, a);
    if (e != cudaSuccess) return e;
    return cudaGetLastError();
}

}  // namespace rglru
