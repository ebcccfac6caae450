// fused_prefill.cu -- tensor-core RG-LRU prefill for bf16 activations, head_dim 256 (sm_100a).
//
// One kernel does the whole block (conv -> gates -> decay -> scan -> GeLU merge -> state):
//
//   * a persistent CTA owns one (head, 128-channel half) "group" for its whole life; its
//     block-diagonal gate weights W_a[h][:, half], W_x[h][:, half], pre-scaled by 1/2 (exact
//     in bf16), are written once into tensor memory (TMEM) and used as the A operand of
//     tcgen05.mma (TS form), so shared memory only holds streamed tiles;
//   * work items are (batch row, 32-token chunk) of the group, handed out by a per-group
//     atomic ticket so every CTA of a group stays busy and an item's predecessors are always
//     held by running CTAs; 4 stages of shared-memory tiles and of TMEM accumulators are in
//     flight per CTA;
//   * warp roles: an x producer (TMA: x tile with a 3-token halo, and the ticket), a y producer
//     (TMA: y tile, paced by a slot handshake with the x producer and by the out store of the
//     stage's previous item), 8 conv warps (a channel half and a quarter of the chunk's tokens
//     each; a lane convolves 4 channels with 8-byte shared-memory loads and writes them as the
//     bf16 B operand in the 128-byte swizzled K-major layout), 2 MMA issuer threads (even / odd
//     items; D = W^T/2 . xc^T for both gates, K = 256 in 16 steps; the epilogue adds the halved
//     gate biases, so a stage needs no re-arming between items), and 4 epilogue groups of 4
//     warps, group g owning TMEM stage g;
//   * transposed orientation: a TMEM lane is an output channel and the 32 columns are tokens,
//     so an epilogue thread owns one channel and runs the diagonal scan along its registers
//     (no shuffles); its first pass leaves the running (prod a, local h) of every token in
//     TMEM, so once the carry C is known the second pass is h_t = P_t C + h_t^loc;
//   * chunks of one sequence handled by different CTAs chain through a look-back in the spirit
//     of Merrill & Garland ("Single-pass Parallel Prefix Scan with Decoupled Look-back", 2016):
//     after its first pass a chunk publishes its aggregate (prod a, local h) per channel; its
//     carry is the inclusive state of an anchor chunk (every 4th chunk of the row) followed by
//     the aggregates of the chunks in between, applied in a fixed order so the result does not
//     depend on timing.  Each published value is one 64-bit word that shows whether it has been
//     written, so a reader polls the data itself: one round of independent loads per attempt,
//     no separate flag.  Every wait is bounded by %globaltimer; on expiry the kernel latches
//     RGLRU_ERR_TIMEOUT in the workspace status word and drains.
//
// Element-wise arithmetic (one transcendental per gate, one square root, one for GeLU):
//   D_a = (g_a + b_a) / 2, D_x = (g_x + b_x) / 2 (the MMA gives g / 2, the epilogue adds b / 2);
//   r_t = (1 + tanh D_a) / 2 and l_t = c r_t log sigma(Lambda) = hK (1 + tanh D_a) with
//   hK = c log sigma(Lambda) / 2;  E = expm1(l_t) = l(1 + l/2 + l^2/6) (|l| <= 1/8: the
//   truncation, summed over the ~1/|l| tokens a decay acts on, stays below 1e-4), a_t = 1 + E,
//   sqrt(1 - a_t^2) / 2 = sqrt(E (-E/4 - 1/2)) (no cancellation near a_t = 1);
//   i_t x_t sqrt(1 - a^2) = w (1 + tanh D_x) with w = x_t sqrt(1 - a^2) / 2;
//   GeLU(y) = y (1 + tanh(y (k1 + k3 y^2))) / 2, k1 / k3 fitted to the exact y Phi(y)
//   (|error in Phi| <= 1.5e-4; the tanh form of the flag uses k1 = sqrt(2/pi), k3 = 0.044715 k1).
// Channels with |c log sigma(Lambda)| > 1/8, resets and a ragged last chunk take a general path.
//
// Arithmetic follows "Griffin Guide: RecurrentGemma, RG-LRU & Hybrid Attention": recurrence /
// input gates, a_t = a^(c r_t) in log space, h_t = a_t h_{t-1} + sqrt(1 - a_t^2)(i_t x_t)
// ("1. Formulation of the RG-LRU Gating Mechanism"), the width-4 conv before the RG-LRU and
// the GeLU merge ("1. Temporal Filtering via Separable 1D Convolutions", "2. Non-Linear
// Multiplicative Gating with GeLU"), per-head block-diagonal gates ("3. Block-Diagonal
// Sharding for Zero-Communication Tensor Parallelism").  The conv output feeding the MMA and
// the i_t * x_t product is rounded to bf16 (the tensor-core operand); state and all
// element-wise math stay in fp32.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <mutex>
#include <type_traits>

#include "common.cuh"
#include "kernels.h"
#include "sm100.cuh"

namespace rglru {
namespace tc {

using namespace sm100;

constexpr int DH = 256;                 // head dim (K of the gate contraction)
constexpr int HALF = 128;               // output channels per CTA (= TMEM lanes = MMA M)
constexpr int L = 32;                   // tokens per chunk (= MMA N)
constexpr int XROWS = L + kHist;        // x tile rows incl. the 3-token halo
constexpr int KSTEPS = DH / 16;         // MMA K steps
constexpr int STAGES = 4;               // x / B / y tiles and TMEM accumulator slots
constexpr int SLOTS = 16;               // ring of item ids, indexed by iteration (> the producers' lag)
constexpr int kBlk = 8;                 // tokens per TMEM load block in the epilogue
constexpr int kConvTok = L / 4;         // tokens per conv warp

// warp roles: 0-7 conv (channel half = warp % 2, token quarter = warp / 2), 8-23 epilogue (TMEM
// lane quarter = warp % 4, group = stage = (warp - 8) / 4), 24 x producer (x tiles and
// tickets), 25 y producer, 26-27 MMA issuers (even / odd items: one thread issues the tensor
// core instructions of an item, and one alone cannot keep up).
constexpr int kConvWarps = 8, kEpiGroups = STAGES, kEpiGroup = 4, kEpiWarps = kEpiGroups * kEpiGroup;
constexpr int kWarpEpi0 = 8, kWarpProdX = 24, kWarpProdY = 25, kWarpMma = 26, kMmaWarps = 2;
constexpr int kThreads = 28 * 32;

constexpr uint32_t X_BYTES = XROWS * DH * 2;      // 17920
constexpr uint32_t Y_BYTES = L * HALF * 2;        // 8192
constexpr uint32_t B_BYTES = L * DH * 2;          // 16384 (4 K-blocks of L x 128 B)
constexpr uint32_t KBLK_BYTES = L * 128;          // one 64-wide K block

// shared memory map (offsets from a 1024-aligned base)
constexpr uint32_t OFF_B = 0;                                   // STAGES x B_BYTES
constexpr uint32_t OFF_X = OFF_B + STAGES * B_BYTES;            // STAGES x X_BYTES
constexpr uint32_t OFF_Y = OFF_X + STAGES * X_BYTES;            // STAGES x Y_BYTES
constexpr uint32_t OFF_BAR = OFF_Y + STAGES * Y_BYTES;
constexpr int NBAR = 11 * STAGES + 2;
constexpr uint32_t OFF_MISC = OFF_BAR + NBAR * 8;               // item-id ring
constexpr uint32_t OFF_TMEMP = OFF_MISC + SLOTS * 4;            // TMEM base address
constexpr uint32_t OFF_ABORT = OFF_TMEMP + 16;                  // abort flag
constexpr uint32_t SMEM_BYTES = OFF_ABORT + 16 + 1024;         // + slack for 1024 alignment
static_assert(2 * HALF * DH * 2 <= OFF_Y, "weight staging reuses the B and x tiles");

// TMEM columns: [0,128) A = W_a^T / 2 (bf16 pairs), [128,256) A = W_x^T / 2, then per stage
// 2L = 64 columns: D_a [0,L) and D_x [L,2L); the first pass overwrites them with P and H.
constexpr uint32_t TMEM_COLS = 512;
constexpr uint32_t TM_A = 0, TM_D = 256, TM_SLOT = 2 * L;
static_assert(TM_D + STAGES * TM_SLOT <= TMEM_COLS, "TMEM budget");
static_assert(SMEM_BYTES <= 232448, "shared memory budget");

constexpr unsigned FLAG_AGG = 1, FLAG_INCL = 2;
constexpr int LBW = 4;                  // look-back block: anchors every LBW chunks
// A published look-back word is 64 bits, written by one relaxed store, and says itself whether it
// has been written (the workspace starts zeroed): an aggregate is (prod a with its sign bit set,
// local h) -- prod a is never negative -- and an anchor's inclusive state is (h, -1).
constexpr uint32_t kReadyBit = 0x80000000u;

struct Args {
    int B, T, H, NC, items;          // items = B * NC per group
    int groups;                      // 2 * H
    int base, extra;                 // CTAs per group: base (+1 for the first `extra` groups)
    float c;
    int gelu_tanh;
    unsigned flags;
    unsigned long long timeout_ns;
    const float* conv_w;
    const float* conv_b;
    const __nv_bfloat16* w_a;
    const __nv_bfloat16* w_x;
    const float* b_a;
    const float* b_x;
    const float* lambda;
    const uint8_t* reset;
    float* h_state;                  // nullptr: zero initial state, no write-back
    __nv_bfloat16* tail_state;
    const __nv_bfloat16* tail_old;   // the conv history as the call found it (a copy), or nullptr
    DeviceStatus* status;
    unsigned* counters;              // [groups] tickets
    unsigned* lb_flags;              // [groups][items][4]
    int NA;                          // anchors per row: ceil(NC / LBW)
    uint64_t* lb_agg;                // [groups][items][128] aggregate words
    uint64_t* lb_incl;               // [groups][B * NA][128] anchor inclusive-state words
};

struct Bars {
    uint32_t x_full[STAGES], x_empty[STAGES], y_full[STAGES], y_empty[STAGES], b_full[STAGES],
        b_empty[STAGES], acc_full[STAGES], acc_empty[STAGES], out_ready[STAGES], slot_full[STAGES],
        slot_free[STAGES], w_ready, mma_done;
};

__device__ __forceinline__ Bars make_bars(uint32_t base) {
    Bars b;
    uint32_t o = base;
    auto next = [&]() { uint32_t r = o; o += 8; return r; };
    for (int s = 0; s < STAGES; ++s) {
        b.x_full[s] = next(); b.x_empty[s] = next(); b.y_full[s] = next(); b.y_empty[s] = next();
        b.b_full[s] = next(); b.b_empty[s] = next(); b.acc_full[s] = next(); b.acc_empty[s] = next();
        b.out_ready[s] = next(); b.slot_full[s] = next(); b.slot_free[s] = next();
    }
    b.w_ready = next();
    b.mma_done = next();
    return b;
}

// Context of the bounded waits: they give up after timeout_ns, or as soon as another thread of
// the grid has latched a failure, so that every role drains instead of hanging.
struct WaitCtx {
    DeviceStatus* status;
    unsigned long long timeout_ns;
    volatile int* abort;
};

__device__ __noinline__ bool wait_bar_slow(uint32_t bar, uint32_t parity, WaitCtx w, unsigned where) {
    const uint64_t t0 = globaltimer_ns();
    for (;;) {
        if (mbar_try_wait_sleep(bar, parity, 100000u)) return true;   // sleeps up to 100 us
        if (*w.abort) return false;
        if (*(volatile unsigned*)&w.status->code != 0) {
            *w.abort = 1;
            return false;
        }
        if (globaltimer_ns() - t0 > w.timeout_ns) {
            latch_status(w.status, RGLRU_ERR_TIMEOUT, where, blockIdx.x, parity);
            *w.abort = 1;
            return false;
        }
    }
}

__device__ __forceinline__ bool wait_bar(uint32_t bar, uint32_t parity, WaitCtx w, unsigned where) {
    if (mbar_try_wait(bar, parity)) return true;
    return wait_bar_slow(bar, parity, w, where);
}

// The same wait for a warp whose lanes then run warp-collective instructions: every lane waits,
// and the outcome is made uniform, so that the warp never splits on a timeout.
__device__ __forceinline__ bool wait_bar_warp(uint32_t bar, uint32_t parity, WaitCtx w, unsigned where) {
    return __all_sync(0xffffffffu, wait_bar(bar, parity, w, where));
}

// Bounded wait for a look-back flag to reach at least `want`; returns the flag (0 on failure).
__device__ __noinline__ unsigned wait_flag(const unsigned* f, unsigned want, WaitCtx w, unsigned where) {
    unsigned v = ld_acquire_gpu(f);
    if (v >= want) return v;
    const uint64_t t0 = globaltimer_ns();
    for (uint32_t i = 1;; ++i) {
        __nanosleep(128);
        v = ld_acquire_gpu(f);
        if (v >= want) return v;
        if ((i & 15) == 0) {
            if (*w.abort || *(volatile unsigned*)&w.status->code != 0) {
                *w.abort = 1;
                return 0;
            }
            if (globaltimer_ns() - t0 > w.timeout_ns) {
                latch_status(w.status, RGLRU_ERR_TIMEOUT, where, blockIdx.x, 0);
                *w.abort = 1;
                return 0;
            }
        }
    }
}

__device__ __forceinline__ uint32_t b_tile_offset(int t, int k) {
    // element (token t, channel k) of the 128-byte swizzled K-major B tile
    const int kb = k >> 6, kk = k & 63;
    const int chunk = (kk >> 3) ^ (t & 7);
    return kb * KBLK_BYTES + (t >> 3) * 1024 + (t & 7) * 128 + chunk * 16 + (kk & 7) * 2;
}

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

// Packed helpers (two tokens per instruction on the fp32x2 path of sm_100).
__device__ __forceinline__ float2 f2(float v) { return make_float2(v, v); }
__device__ __forceinline__ float2 fma2(float2 a, float2 b, float2 c) { return __ffma2_rn(a, b, c); }
__device__ __forceinline__ float2 mul2(float2 a, float2 b) { return __fmul2_rn(a, b); }
__device__ __forceinline__ float2 add2(float2 a, float2 b) { return __fadd2_rn(a, b); }
__device__ __forceinline__ float2 tanh2(float2 v) { return make_float2(tanh_approx(v.x), tanh_approx(v.y)); }
__device__ __forceinline__ float2 sqrt2(float2 v) { return make_float2(sqrt_approx(v.x), sqrt_approx(v.y)); }

// TMEM block load / store of kBlk consecutive columns (32 lanes x 32 bits)
__device__ __forceinline__ void tmem_ldb(uint32_t taddr, float (&v)[kBlk]) { tmem_ld8(taddr, v); }
__device__ __forceinline__ void tmem_stbf(uint32_t taddr, const float (&v)[kBlk]) { tmem_st8f(taddr, v); }

// Fast path of gates + decay + normalised input for two tokens of a channel with
// |c log sigma(Lambda)| <= 1/8 (so |l| <= 1/8).  In: D_a, D_x (pre-scaled gate
// pre-activations), xc (the bf16-rounded conv output).  Out: a_t and u_t = sqrt(1-a^2) i x.
__device__ __forceinline__ void gates_pair(float2 da, float2 dx, float2 hk, float2 xc, float2& a, float2& u) {
    const float2 ta = tanh2(da);
    const float2 l = fma2(ta, hk, hk);                                  // c r log sigma(Lambda)
    float2 p = fma2(l, f2(1.0f / 6.0f), f2(0.5f));
    p = fma2(l, p, f2(1.0f));
    const float2 e = mul2(l, p);                                        // expm1(l)
    a = add2(e, f2(1.0f));
    const float2 q = fma2(e, f2(-0.25f), f2(-0.5f));
    const float2 bh = sqrt2(mul2(e, q));                                // sqrt(1 - a^2) / 2
    const float2 ti = tanh2(dx);
    const float2 w = mul2(bh, xc);
    u = fma2(w, ti, w);                                                 // sqrt(1-a^2) i x
}

// General path of one token: any |c log sigma(Lambda)|.
__device__ __forceinline__ void gates_one(float da, float dx, float hk, float xc, float& a, float& u) {
    const float l = fmaf(tanh_approx(da), hk, hk);
    float e;
    if (l > -0.125f) {
        float p = fmaf(l, 1.0f / 24.0f, 1.0f / 6.0f);
        p = fmaf(l, p, 0.5f);
        p = fmaf(l, p, 1.0f);
        e = l * p;
    } else {
        e = ex2_approx(l * 1.4426950408889634f) - 1.0f;
    }
    a = 1.0f + e;
    const float bh = sqrt_approx(e * fmaf(e, -0.25f, -0.5f));
    const float w = bh * xc;
    u = fmaf(w, tanh_approx(dx), w);
}

// out = h * GeLU(y) for two tokens, GeLU(y) = (y/2)(1 + tanh(w(y))), w = (y/2)(K1 + K3 (y/2)^2).
__device__ __forceinline__ float2 merge_pair(float2 h, float2 y, float k1, float k3) {
    const float2 hy = mul2(y, f2(0.5f));
    const float2 s = mul2(hy, hy);
    const float2 w = mul2(hy, fma2(s, f2(k3), f2(k1)));
    const float2 t = tanh2(w);
    const float2 m = mul2(h, hy);
    return fma2(m, t, m);
}

// Bit j of the result = reset[t0 + j] != 0 for the L tokens of a chunk (0 past the end).
__device__ __forceinline__ uint64_t chunk_reset_mask(const uint8_t* row, int t0, int T, int lane) {
    uint64_t m = 0;
#pragma unroll
    for (int h = 0; h < L; h += 32) {
        const bool r = t0 + h + lane < T && row[t0 + h + lane] != 0;
        m |= (uint64_t)__ballot_sync(0xffffffffu, r) << h;
    }
    return m;
}

// A lane's 4 channels of one token (conv window entries), fp32.
struct Vec4 {
    float2 v[2];
};
__device__ __forceinline__ Vec4 unpack4(uint2 r) {
    Vec4 o;
    o.v[0] = make_float2(bf16lo(r.x), bf16hi(r.x));
    o.v[1] = make_float2(bf16lo(r.y), bf16hi(r.y));
    return o;
}
__device__ __forceinline__ uint2 pack4(const Vec4& h) {
    return make_uint2(pack_bf16x2(h.v[0].x, h.v[0].y), pack_bf16x2(h.v[1].x, h.v[1].y));
}
__device__ __forceinline__ Vec4 zero4() {
    Vec4 o;
    o.v[0] = o.v[1] = make_float2(0.f, 0.f);
    return o;
}

// The conv of one warp's kConvTok tokens (j0 + jj, jj < kConvTok) for a lane's 4 channels, written
// as bf16 into the B tile.  RST: the chunk has segment starts (bit jj of rm: token j0 + jj starts
// one, so the history before it is dropped); LAST: the row's last token (jlast, relative to j0)
// is in this range and the window after it is kept in fw (the conv history of the row).
template <bool RST, bool LAST>
__device__ __forceinline__ void conv_tokens(const uint8_t* xtw, uint8_t* btw, uint32_t cchunk, uint32_t rm, int jlast,
                                            const float2 (&w)[kConvWidth][2], const float2 (&cb)[2], Vec4& h0, Vec4& h1,
                                            Vec4& h2, uint2 (&fw)[3]) {
#pragma unroll
    for (int jj = 0; jj < kConvTok; ++jj) {
        const Vec4 xv = unpack4(*reinterpret_cast<const uint2*>(xtw + (jj + kHist) * DH * 2));
        if (RST && ((rm >> jj) & 1u)) h0 = h1 = h2 = zero4();
        uint2 o;
        float2 y = fma2(w[0][0], h0.v[0], cb[0]);
        y = fma2(w[1][0], h1.v[0], y);
        y = fma2(w[2][0], h2.v[0], y);
        y = fma2(w[3][0], xv.v[0], y);
        o.x = pack_bf16x2(y.x, y.y);
        y = fma2(w[0][1], h0.v[1], cb[1]);
        y = fma2(w[1][1], h1.v[1], y);
        y = fma2(w[2][1], h2.v[1], y);
        y = fma2(w[3][1], xv.v[1], y);
        o.y = pack_bf16x2(y.x, y.y);
        *reinterpret_cast<uint2*>(btw + (jj >> 3) * 1024 + (jj & 7) * 128 + ((cchunk ^ (jj & 7)) << 4)) = o;
        h0 = h1; h1 = h2; h2 = xv;
        if (LAST && jj == jlast) { fw[0] = pack4(h0); fw[1] = pack4(h1); fw[2] = pack4(h2); }
    }
}

__global__ void __launch_bounds__(kThreads, 1)
fused_prefill_kernel(const __grid_constant__ CUtensorMap map_x, const __grid_constant__ CUtensorMap map_y,
                     const __grid_constant__ CUtensorMap map_out, const Args a) {
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const uint32_t sbase = smem_u32(smem);
    const Bars bars = make_bars(sbase + OFF_BAR);
    volatile int* slot = reinterpret_cast<volatile int*>(smem + OFF_MISC);        // [SLOTS]
    volatile uint32_t* tmem_base_s = reinterpret_cast<volatile uint32_t*>(smem + OFF_TMEMP);
    volatile int* abort = reinterpret_cast<volatile int*>(smem + OFF_ABORT);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    // ---- group of this CTA -----------------------------------------------------------------
    int group;
    {
        const int cta = blockIdx.x, big = a.extra * (a.base + 1);
        group = cta < big ? cta / (a.base + 1) : a.extra + (cta - big) / a.base;
    }
    const int head = group >> 1, half = group & 1;
    const int W = a.H * DH;
    const size_t lb_base = (size_t)group * a.items;
    const size_t lb_base_a = (size_t)group * a.B * a.NA;     // anchors of the group

    // ---- set-up ------------------------------------------------------------------------------
    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(bars.x_full[s], 1);
            mbar_init(bars.x_empty[s], kConvWarps);
            mbar_init(bars.y_full[s], 1);
            mbar_init(bars.y_empty[s], 1);
            mbar_init(bars.b_full[s], kConvWarps);
            mbar_init(bars.b_empty[s], 1 + kEpiGroup);
            mbar_init(bars.acc_full[s], 1);
            mbar_init(bars.acc_empty[s], kEpiGroup);
            mbar_init(bars.out_ready[s], kEpiGroup);
            mbar_init(bars.slot_full[s], 1);
            mbar_init(bars.slot_free[s], 1);
        }
        mbar_init(bars.w_ready, kEpiWarps);
        mbar_init(bars.mma_done, kMmaWarps);
        *abort = 0;
        fence_barrier_init();
        fence_proxy_async_smem();
    }
    if (warp == kWarpMma) {
        tmem_alloc(smem_u32((const void*)tmem_base_s), TMEM_COLS);
        tmem_relinquish();
    }
    if (warp == kWarpProdX && lane == 0) {
        prefetch_tensormap(&map_x);
        prefetch_tensormap(&map_y);
        prefetch_tensormap(&map_out);
    }
    // stage this CTA's gate weights W_g[head][i][half*128 + o] / 2 (o contiguous) in shared
    // memory with coalesced 16-byte loads: gate a at byte 0, gate x at byte 65536 (B and x
    // tiles are still unused); halving a bf16 is exact
    if (warp < kConvWarps + kEpiWarps) {
        const int tid = threadIdx.x;                       // 0..383
        for (int e = tid; e < 2 * DH * (HALF / 8); e += (kConvWarps + kEpiWarps) * 32) {
            const int g = e / (DH * (HALF / 8)), r = e % (DH * (HALF / 8));
            const int i = r / (HALF / 8), o8 = r % (HALF / 8);
            const __nv_bfloat16* src = (g ? a.w_x : a.w_a) + ((size_t)head * DH + i) * DH + half * HALF + o8 * 8;
            uint4 v = __ldg(reinterpret_cast<const uint4*>(src));
            uint32_t* vv = reinterpret_cast<uint32_t*>(&v);
#pragma unroll
            for (int k = 0; k < 4; ++k) vv[k] = pack_bf16x2(0.5f * bf16lo(vv[k]), 0.5f * bf16hi(vv[k]));
            *reinterpret_cast<uint4*>(smem + g * (HALF * DH * 2) + (i * HALF + o8 * 8) * 2) = v;
        }
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_base_s;
    const WaitCtx wc{a.status, a.timeout_ns, abort};

    if (warp >= kWarpEpi0 && warp < kWarpEpi0 + kEpiWarps) {
        // weights -> TMEM A operand: lane m, column j holds (W[2j][m], W[2j+1][m]); group 0 of
        // each lane quarter writes gate a, group 1 gate x.
        const int q = warp & 3, g = (warp - kWarpEpi0) >> 2, m = q * 32 + lane;
        const unsigned short* ws = reinterpret_cast<const unsigned short*>(smem + (g & 1) * (HALF * DH * 2)) + m;
#pragma unroll 1
        for (int j0 = 0; j0 < (g < 2 ? DH / 2 : 0); j0 += 16) {
            uint32_t r[16];
#pragma unroll
            for (int j = 0; j < 16; ++j) {
                const int i = 2 * (j0 + j);
                r[j] = (uint32_t)ws[i * HALF] | ((uint32_t)ws[(i + 1) * HALF] << 16);
            }
            tmem_st16(tmem + ((uint32_t)(q * 32) << 16) + TM_A + g * 128 + j0, r);
        }
        tmem_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(bars.w_ready);
    }
    __syncthreads();   // the staging area is free again before any TMA load lands in it

    if (warp == kWarpProdX) {
        if (lane == 0) {
            // ============================ x producer (and tickets) ============================
            int issued[STAGES] = {};
            for (int n = 0;; ++n) {
                const int st = n % STAGES;
                const uint32_t ph = (n / STAGES) & 1;
                if (!wait_bar(bars.x_empty[st], ph ^ 1, wc, 1)) break;
                // the y producer has taken the id of iteration n - STAGES: it never lags further
                if (!wait_bar(bars.slot_free[st], ph ^ 1, wc, 19)) break;
                int k = (int)atomicAdd(&a.counters[group], 1u);
                if (k >= a.items) {
                    // terminal item for the stage-n group and for the next STAGES-1 groups
                    for (int i = 0; i < STAGES; ++i) slot[(n + i) & (SLOTS - 1)] = -1;
                    mbar_arrive(bars.slot_full[st]);
                    mbar_arrive(bars.x_full[st]);
                    issued[st] = 0;   // that phase completing implies the earlier load landed
                    break;
                }
                slot[n & (SLOTS - 1)] = k;
                mbar_arrive(bars.slot_full[st]);
                const int b = k / a.NC, c = k % a.NC;
                mbar_arrive_expect_tx(bars.x_full[st], X_BYTES);
                tma_load_3d(sbase + OFF_X + st * X_BYTES, &map_x, head * DH, c * L - kHist, b,
                            bars.x_full[st]);
                issued[st] = n + 1;
            }
            // never leave the CTA with a bulk copy still writing its shared memory
            for (int st = 0; st < STAGES; ++st)
                if (issued[st]) {
                    const int n = issued[st] - 1;
                    const uint64_t t0 = globaltimer_ns();
                    while (!mbar_try_wait_sleep(bars.x_full[st], (n / STAGES) & 1, 100000u) &&
                           globaltimer_ns() - t0 < a.timeout_ns) {
                    }
                }
        }
    } else if (warp == kWarpProdY) {
        if (lane == 0) {
            // ============================ y producer ==========================================
            int issued[STAGES] = {};
            for (int n = 0;; ++n) {
                const int st = n % STAGES;
                const uint32_t ph = (n / STAGES) & 1;
                if (!wait_bar(bars.slot_full[st], ph, wc, 15)) break;
                const int k = slot[n & (SLOTS - 1)];
                mbar_arrive(bars.slot_free[st]);
                if (k < 0) break;
                if (!wait_bar(bars.y_empty[st], ph ^ 1, wc, 2)) break;
                const int b = k / a.NC, c = k % a.NC;
                mbar_arrive_expect_tx(bars.y_full[st], Y_BYTES);
                tma_load_3d(sbase + OFF_Y + st * Y_BYTES, &map_y, head * DH + half * HALF, c * L, b,
                            bars.y_full[st]);
                issued[st] = n + 1;
            }
            for (int st = 0; st < STAGES; ++st)
                if (issued[st]) {
                    const int n = issued[st] - 1;
                    const uint64_t t0 = globaltimer_ns();
                    while (!mbar_try_wait_sleep(bars.y_full[st], (n / STAGES) & 1, 100000u) &&
                           globaltimer_ns() - t0 < a.timeout_ns) {
                    }
                }
        }
    } else if (warp >= kWarpMma && warp < kWarpMma + kMmaWarps) {
        // ================================ MMA issuers ==========================================
        // issuer i takes the items n = i (mod kMmaWarps); at the end of the work each one hands
        // the terminal item to the epilogue groups of its own next iterations
        if (lane == 0) {
            const uint32_t idesc = idesc_bf16_f32(HALF, L);
            bool ok = wait_bar(bars.w_ready, 0, wc, 3);
            tc_fence_after();
            for (int n = warp - kWarpMma; ok; n += kMmaWarps) {
                const int st = n % STAGES;
                const uint32_t ph = (n / STAGES) & 1;
                if (!wait_bar(bars.b_full[st], ph, wc, 4)) break;
                if (!wait_bar(bars.acc_empty[st], ph ^ 1, wc, 5)) break;
                if (slot[n & (SLOTS - 1)] < 0) {
                    // hand the terminal item to the groups of iterations n, n + kMmaWarps, ...:
                    // group st now, each other one once it has released its previous item (so
                    // that no phase is skipped)
                    mbar_arrive(bars.acc_full[st]);
                    for (int i = kMmaWarps; i < STAGES; i += kMmaWarps) {
                        const int s2 = (n + i) % STAGES;
                        const uint32_t ph2 = ((n + i) / STAGES) & 1;
                        if (wait_bar(bars.acc_empty[s2], ph2 ^ 1, wc, 17)) mbar_arrive(bars.acc_full[s2]);
                    }
                    break;
                }
                tc_fence_after();
                // descriptor of K step ks = the stage's base descriptor + the step's byte offset / 16
                const uint64_t bd0 = desc_k_sw128(sbase + OFF_B + st * B_BYTES);
                const uint32_t d0 = tmem + TM_D + st * TM_SLOT;
#pragma unroll
                for (int ks = 0; ks < KSTEPS; ++ks) {
                    const uint64_t bd = bd0 + (uint64_t)((((ks >> 2) * KBLK_BYTES) + (ks & 3) * 32) >> 4);
                    const uint32_t acc = ks > 0 ? 1u : 0u;
                    mma_ts(d0, tmem + TM_A + ks * 8, bd, idesc, acc);
                    mma_ts(d0 + L, tmem + TM_A + 128 + ks * 8, bd, idesc, acc);
                }
                mma_commit(bars.acc_full[st]);
                mma_commit(bars.b_empty[st]);
            }
            // every MMA this thread issued has finished before TMEM is released
            mma_commit(bars.mma_done);
            const uint64_t t0 = globaltimer_ns();
            while (!mbar_try_wait_sleep(bars.mma_done, 0, 100000u) && globaltimer_ns() - t0 < a.timeout_ns) {
            }
        }
    } else if (warp < kConvWarps) {
        // ================================ conv warps ==========================================
        // warp w convolves channels [128 (w % 2), +128) of the head for the tokens
        // [8 (w / 2), +8) of the chunk; lane l 4 channels (8 bytes of a B-tile row)
        const int chh = warp & 1;
        const int j0 = (warp >> 1) * kConvTok;
        const int cl = chh * HALF + lane * 4;             // channel within the head
        const int chg = head * DH + cl;                   // global channel
        float2 w[kConvWidth][2];
#pragma unroll
        for (int k = 0; k < kConvWidth; ++k)
#pragma unroll
            for (int i = 0; i < 2; ++i)
                w[k][i] = make_float2(a.conv_w[(size_t)k * W + chg + 2 * i], a.conv_w[(size_t)k * W + chg + 2 * i + 1]);
        float2 cb[2];
#pragma unroll
        for (int i = 0; i < 2; ++i)
            cb[i] = a.conv_b ? make_float2(a.conv_b[chg + 2 * i], a.conv_b[chg + 2 * i + 1]) : make_float2(0.f, 0.f);
        const bool own_tail = chh == half;               // this CTA writes these tail channels
        // B-tile byte offset of (token t, channel cl): kb * KBLK + (t / 8) * 1024 + (t % 8) * 128
        //   + ((chunk ^ (t % 8)) * 16) + sub, chunk / sub = 16-byte chunk / byte within it
        const uint32_t kb_off = (uint32_t)(cl >> 6) * KBLK_BYTES + ((cl & 7) * 2);
        const uint32_t cchunk = (cl & 63) >> 3;
        for (int n = 0;; ++n) {
            const int st = n % STAGES;
            const uint32_t ph = (n / STAGES) & 1;
            if (!wait_bar_warp(bars.x_full[st], ph, wc, 6)) break;
            if (!wait_bar_warp(bars.b_empty[st], ph ^ 1, wc, 7)) break;
            const int k = slot[n & (SLOTS - 1)];
            if (k < 0) {
                // every MMA issuer meets the end of the work at its own next iteration
                __syncwarp();
                if (lane == 0)
                    for (int i = 0; i < kMmaWarps; ++i) mbar_arrive(bars.b_full[(n + i) % STAGES]);
                break;
            }
            const int b = k / a.NC, c = k % a.NC, t0 = c * L;
            const int nt = min(L, a.T - t0);
            const uint8_t* rrow = a.reset ? a.reset + (size_t)b * a.T : nullptr;
            const uint64_t rmask = rrow ? chunk_reset_mask(rrow, t0, a.T, lane) : 0ull;
            const uint8_t* xt = smem + OFF_X + st * X_BYTES + cl * 2;
            uint8_t* bt = smem + OFF_B + st * B_BYTES + kb_off;
            auto xrow = [&](int r) {                      // x tile row r = token t0 - 3 + r
                return unpack4(*reinterpret_cast<const uint2*>(xt + r * DH * 2));
            };
            Vec4 h0, h1, h2;                              // window x_{t-3}, x_{t-2}, x_{t-1}
            if (c == 0 && j0 == 0) {
                if (a.tail_old) {
                    const __nv_bfloat16* tl = a.tail_old + (size_t)b * kHist * W + chg;
                    h0 = unpack4(*reinterpret_cast<const uint2*>(tl));
                    h1 = unpack4(*reinterpret_cast<const uint2*>(tl + W));
                    h2 = unpack4(*reinterpret_cast<const uint2*>(tl + 2 * W));
                } else {
                    h0 = h1 = h2 = zero4();
                }
            } else {
                h0 = xrow(j0);
                h1 = xrow(j0 + 1);
                h2 = xrow(j0 + 2);
                if (rrow) {
                    // a segment that starts at token j0-1 (j0-2) empties the older history
                    const int p1 = t0 + j0 - 1, p2 = t0 + j0 - 2;
                    if (p1 < a.T && rrow[p1]) h0 = h1 = zero4();
                    if (p2 >= 0 && p2 < a.T && rrow[p2]) h0 = zero4();
                }
            }
            uint2 fw[3];                                  // final window (the tail of the row), bf16
            const bool has_last = nt - 1 >= j0 && nt - 1 < j0 + kConvTok;
            const uint32_t rm = (uint32_t)(rmask >> j0);
            const uint8_t* xtw = xt + j0 * DH * 2;
            uint8_t* btw = bt + (j0 >> 3) * 1024;
            const int jlast = nt - 1 - j0;
            if (rm == 0) {
                if (has_last) conv_tokens<false, true>(xtw, btw, cchunk, rm, jlast, w, cb, h0, h1, h2, fw);
                else conv_tokens<false, false>(xtw, btw, cchunk, rm, jlast, w, cb, h0, h1, h2, fw);
            } else {
                if (has_last) conv_tokens<true, true>(xtw, btw, cchunk, rm, jlast, w, cb, h0, h1, h2, fw);
                else conv_tokens<true, false>(xtw, btw, cchunk, rm, jlast, w, cb, h0, h1, h2, fw);
            }
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) {
                mbar_arrive(bars.x_empty[st]);
                mbar_arrive(bars.b_full[st]);
            }
            // final conv history of the sequence.  Both channel-half groups of the head read the
            // old history (each convolves all 256 input channels), from the copy taken before the
            // launch, so the state buffer is only written, by the group that owns the channels,
            // as soon as the row's last token is convolved: no CTA waits for another here.
            if (a.tail_state && c == a.NC - 1 && has_last && own_tail) {
                __nv_bfloat16* tl = a.tail_state + (size_t)b * kHist * W + chg;
#pragma unroll
                for (int r = 0; r < 3; ++r) *reinterpret_cast<uint2*>(tl + (size_t)r * W) = fw[r];
            }
        }
    } else if (warp < kWarpEpi0 + kEpiWarps) {
        // ================================ epilogue groups ======================================
        const int q = warp & 3;                          // TMEM lane quarter
        const int eg = (warp - kWarpEpi0) >> 2;          // group = TMEM stage it owns
        const int st = eg;
        const int m = q * 32 + lane;                     // local output channel = TMEM lane
        const int chl = half * HALF + m;                 // channel within the head
        const int ch = head * DH + chl;                  // global channel
        const uint32_t lane_off = (uint32_t)(q * 32) << 16;
        const float hk = 0.5f * a.c * log_sigmoid_acc(a.lambda[ch]);   // l_t = hk (1 + tanh D_a)
        const bool small_range = hk >= -0.0625f;
        const float2 hk2 = f2(hk);
        const int tanh_form = a.gelu_tanh;
        // GeLU(y) = (y/2)(1 + tanh((y/2)(K1 + K3 (y/2)^2)))
        const float gk1 = tanh_form ? 2.0f * 0.79788456080286535588f : 2.0f * 0.79879267f;
        const float gk3 = tanh_form ? 8.0f * 0.044715f * 0.79788456080286535588f : 8.0f * 0.03528805f;
        const float2 ba2 = f2(a.b_a ? 0.5f * a.b_a[ch] : 0.f);     // gate biases, halved
        const float2 bx2 = f2(a.b_x ? 0.5f * a.b_x[ch] : 0.f);
        const bool withhold_hook = (a.flags & RGLRU_FLAG_TEST_WITHHOLD) && group == 0;
        const uint8_t* bt = smem + OFF_B + st * B_BYTES;
        uint8_t* yt = smem + OFF_Y + st * Y_BYTES + 2 * m;
        const uint32_t dcol = tmem + lane_off + TM_D + st * TM_SLOT;
        // B-tile byte offsets of this channel for tokens 0..7 (token t: boff[t & 7] + (t >> 3) * 1024)
        uint32_t boff[8];
#pragma unroll
        for (int r = 0; r < 8; ++r) boff[r] = b_tile_offset(r, chl);
        auto xc_at = [&](int t) {
            return __uint_as_float((uint32_t)*reinterpret_cast<const unsigned short*>(bt + boff[t & 7] + (t >> 3) * 1024) << 16);
        };

        for (int n = eg;; n += STAGES) {
            const uint32_t ph = (n / STAGES) & 1;
            if (!wait_bar_warp(bars.acc_full[st], ph, wc, 9)) break;
            const int k = slot[n & (SLOTS - 1)];
            if (k < 0) break;
            tc_fence_after();
            const int b = k / a.NC, c = k % a.NC, t0 = c * L;
            const int nt = min(L, a.T - t0);
            const uint8_t* rrow = a.reset ? a.reset + (size_t)b * a.T : nullptr;
            const uint64_t rmask = rrow ? chunk_reset_mask(rrow, t0, a.T, lane) : 0ull;
            const size_t kb_item = lb_base + (size_t)b * a.NC;       // first chunk of this row
            const bool withhold = withhold_hook && k == 0;
            unsigned* myflag = a.lb_flags + (lb_base + k) * 4 + q;

            // ---- pass 1: gates, decay and normalised input; TMEM keeps the running product of
            //      the decays P_t and the running local state H_t (from zero) of every token
            float aggA = 1.f, aggH = 0.f;
            const bool fast = nt == L && __all_sync(0xffffffffu, small_range);
            // RST: the chunk has segment starts (a separate copy, so chunks without any pay nothing)
            auto pass1_fast = [&](auto rst) {
#pragma unroll 1
                for (int j0 = 0; j0 < L; j0 += kBlk) {
                    float da[kBlk], dx[kBlk];
                    tmem_ldb(dcol + j0, da);
                    tmem_ldb(dcol + L + j0, dx);
                    tmem_wait_ld();
#pragma unroll
                    for (int j = 0; j < kBlk; j += 2) {
                        float2 at, u;
                        gates_pair(add2(make_float2(da[j], da[j + 1]), ba2), add2(make_float2(dx[j], dx[j + 1]), bx2), hk2,
                                   make_float2(xc_at(j0 + j), xc_at(j0 + j + 1)), at, u);
                        if constexpr (decltype(rst)::value) {             // h_{t-1} := 0 at a reset
                            if ((rmask >> (j0 + j)) & 1ull) at.x = 0.f;
                            if ((rmask >> (j0 + j + 1)) & 1ull) at.y = 0.f;
                        }
                        aggH = fmaf(at.x, aggH, u.x);
                        aggA *= at.x;
                        da[j] = aggA;
                        dx[j] = aggH;
                        aggH = fmaf(at.y, aggH, u.y);
                        aggA *= at.y;
                        da[j + 1] = aggA;
                        dx[j + 1] = aggH;
                    }
                    tmem_stbf(dcol + j0, da);
                    tmem_stbf(dcol + L + j0, dx);
                }
            };
            if (fast) {
                if (rmask) pass1_fast(std::true_type{});
                else pass1_fast(std::false_type{});
            } else {
#pragma unroll 1
                for (int j0 = 0; j0 < L; j0 += kBlk) {
                    float da[kBlk], dx[kBlk];
                    tmem_ldb(dcol + j0, da);
                    tmem_ldb(dcol + L + j0, dx);
                    tmem_wait_ld();
#pragma unroll
                    for (int j = 0; j < kBlk; ++j) {
                        const int t = j0 + j;
                        float at, u;
                        gates_one(da[j] + ba2.x, dx[j] + bx2.x, hk, xc_at(t), at, u);
                        if ((rmask >> t) & 1ull) at = 0.f;                 // h_{t-1} := 0
                        if (t >= nt) { at = 1.f; u = 0.f; }                // padding: identity
                        aggH = fmaf(at, aggH, u);
                        aggA *= at;
                        da[j] = aggA;
                        dx[j] = aggH;
                    }
                    tmem_stbf(dcol + j0, da);
                    tmem_stbf(dcol + L + j0, dx);
                }
            }
            // the B tile (xc) is no longer read by this warp
            __syncwarp();
            if (lane == 0) mbar_arrive(bars.b_empty[st]);
            if (c > 0 && !withhold)                      // chunk aggregate, as early as possible
                st_relaxed_gpu_u64(a.lb_agg + (lb_base + k) * HALF + m,
                                   ((uint64_t)__float_as_uint(aggH) << 32) | (__float_as_uint(aggA) | kReadyBit));

            // ---- carry: initial state for the first chunk, else the look-back
            float carry = 0.f;
            if (c == 0) {
                carry = a.h_state ? a.h_state[(size_t)b * W + ch] : 0.f;
            } else {
                // fixed association, so results do not depend on timing: the anchor is the
                // nearest earlier chunk whose index is a multiple of LBW; carry = the anchor's
                // inclusive state, then the aggregates of the chunks in between, in order
                const int anc = ((c - 1) / LBW) * LBW;
                const int nagg = c - 1 - anc;                       // < LBW
                const uint64_t* wi = a.lb_incl + (lb_base_a + (size_t)b * a.NA + anc / LBW) * HALF + m;
                const uint64_t* wa = a.lb_agg + (kb_item + anc + 1) * HALF + m;
                const uint64_t tw = globaltimer_ns();
                for (uint32_t it = 0;; ++it) {
                    // every word of this channel's look-back in one batch of independent loads;
                    // the combine stays in chunk order, padding entries are the identity (1, 0)
                    uint64_t g[LBW];
                    g[0] = ld_relaxed_gpu_u64(wi);
#pragma unroll
                    for (int i = 1; i < LBW; ++i)
                        g[i] = i <= nagg ? ld_relaxed_gpu_u64(wa + (size_t)(i - 1) * HALF)
                                         : (uint64_t)(__float_as_uint(1.0f) | kReadyBit);
                    bool okl = (uint32_t)(g[0] >> 32) & kReadyBit;
#pragma unroll
                    for (int i = 1; i < LBW; ++i) okl = okl && ((uint32_t)g[i] & kReadyBit);
                    if (__all_sync(0xffffffffu, okl)) {
                        float hc = __uint_as_float((uint32_t)g[0]);
#pragma unroll
                        for (int i = 1; i < LBW; ++i)
                            hc = fmaf(__uint_as_float((uint32_t)g[i] & ~kReadyBit), hc, __uint_as_float((uint32_t)(g[i] >> 32)));
                        carry = hc;
                        break;
                    }
                    __nanosleep(64);
                    if ((it & 15) == 15) {
                        int give_up = 0;
                        if (lane == 0) {
                            if (*abort || *(volatile unsigned*)&a.status->code != 0) give_up = 1;
                            else if (globaltimer_ns() - tw > a.timeout_ns) {
                                latch_status(a.status, RGLRU_ERR_TIMEOUT, 10, blockIdx.x, (unsigned)k);
                                give_up = 1;
                            }
                            if (give_up) *abort = 1;
                        }
                        if (__shfl_sync(0xffffffffu, give_up, 0)) break;
                    }
                }
            }
            const float incl = fmaf(aggA, carry, aggH);             // state after the chunk
            if (c % LBW == 0 && !withhold) {             // only anchors' inclusive states are read
                st_relaxed_gpu_u64(a.lb_incl + (lb_base_a + (size_t)b * a.NA + c / LBW) * HALF + m,
                                   ((uint64_t)0xBF800000u << 32) | __float_as_uint(incl));
                if (c == 0) {
                    // the row's first chunk has read the old state and history: the flag that the
                    // writers of the final state and history wait for
                    __syncwarp();
                    if (lane == 0) st_release_gpu(myflag, FLAG_INCL);
                }
            }
            // final state of the row, once its first chunk has read the old one
            if (a.h_state && c == a.NC - 1) {
                bool okw = true;
                if (c > 0) {
                    unsigned f = 0;
                    if (lane == 0) f = wait_flag(a.lb_flags + kb_item * 4 + q, FLAG_INCL, wc, 11);
                    okw = __shfl_sync(0xffffffffu, f, 0) != 0;
                }
                if (okw) a.h_state[(size_t)b * W + ch] = incl;
            }

            // ---- pass 2: h_t = P_t C + H_t (no serial chain), merged with GeLU(y_t)
            if (!wait_bar_warp(bars.y_full[st], ph, wc, 16)) break;
            tmem_wait_st();
            {
                const float2 cv = f2(carry);
#pragma unroll 1
                for (int j0 = 0; j0 < L; j0 += kBlk) {
                    float pv[kBlk], hv[kBlk];
                    tmem_ldb(dcol + j0, pv);
                    tmem_ldb(dcol + L + j0, hv);
                    tmem_wait_ld();
#pragma unroll
                    for (int j = 0; j < kBlk; j += 2) {
                        const int t = j0 + j;
                        unsigned short* y0 = reinterpret_cast<unsigned short*>(yt + t * HALF * 2);
                        unsigned short* y1 = reinterpret_cast<unsigned short*>(yt + (t + 1) * HALF * 2);
                        const float2 yv = make_float2(__uint_as_float((uint32_t)*y0 << 16), __uint_as_float((uint32_t)*y1 << 16));
                        const float2 hh = fma2(make_float2(pv[j], pv[j + 1]), cv, make_float2(hv[j], hv[j + 1]));
                        const float2 o = merge_pair(hh, yv, gk1, gk3);
                        const uint32_t ob = pack_bf16x2(o.x, o.y);
                        *y0 = (unsigned short)(ob & 0xFFFFu);
                        *y1 = (unsigned short)(ob >> 16);
                    }
                }
            }
            // hand the accumulator stage back to the MMA
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(bars.acc_empty[st]);

            // ---- out tile -> global (TMA store clips the ragged tail)
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) mbar_arrive(bars.out_ready[st]);
            if (q == 0 && lane == 0) {
                if (wait_bar(bars.out_ready[st], ph, wc, 12)) {
                    tma_store_3d(&map_out, sbase + OFF_Y + st * Y_BYTES, head * DH + half * HALF, t0, b);
                    bulk_commit();
                    bulk_wait_read0();
                }
                mbar_arrive(bars.y_empty[st]);
            }
        }
        // no tensor-memory access of this warp may still be in flight when TMEM is released
        tmem_wait_st();
        tmem_wait_ld();
        if (q == 0 && lane == 0) bulk_wait0();
    }

    // ---- teardown: all tensor-core work has drained (MMA thread waited on mma_done) ----------
    tc_fence_before();
    __syncthreads();
    if (warp == kWarpMma) {
        tc_fence_after();
        tmem_dealloc(tmem, TMEM_COLS);
    }
}

// --------------------------------------------------------------------------- host side ------

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
    static EncodeTiledFn fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(p);
    });
    return fn;
}

bool make_map_3d(CUtensorMap* m, const void* base, int W, int T, int B, int box_c, int box_t) {
    EncodeTiledFn f = encode_fn();
    if (!f) return false;
    cuuint64_t dims[3] = {(cuuint64_t)W, (cuuint64_t)T, (cuuint64_t)B};
    cuuint64_t strides[2] = {(cuuint64_t)W * 2, (cuuint64_t)T * W * 2};
    cuuint32_t box[3] = {(cuuint32_t)box_c, (cuuint32_t)box_t, 1};
    cuuint32_t estr[3] = {1, 1, 1};
    return f(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// 2-D map [outer][inner] of bf16 with a row pitch of row_bytes, box inner x outer, 128-byte
// swizzle (box_inner * 2 must be 128), out-of-range elements read as zero.
// 2-D map (inner x outer elements of bf16 or fp32, rows row_bytes apart) whose box rows are
// exactly 128 bytes, loaded and stored in the 128-byte swizzle
bool make_map_2d_sw128_elem(CUtensorMap* m, const void* base, uint32_t elem_bytes, uint64_t inner, uint64_t outer,
                            uint64_t row_bytes, uint32_t box_inner, uint32_t box_outer) {
    EncodeTiledFn f = encode_fn();
    if (!f || (elem_bytes != 2 && elem_bytes != 4) || box_inner * elem_bytes != 128) return false;
    cuuint64_t dims[2] = {(cuuint64_t)inner, (cuuint64_t)outer};
    cuuint64_t strides[1] = {(cuuint64_t)row_bytes};
    cuuint32_t box[2] = {box_inner, box_outer};
    cuuint32_t estr[2] = {1, 1};
    const CUtensorMapDataType t = elem_bytes == 2 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT32;
    return f(m, t, 2, const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
             CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}
bool make_map_2d_sw128(CUtensorMap* m, const void* base, uint64_t inner, uint64_t outer, uint64_t row_bytes,
                       uint32_t box_inner, uint32_t box_outer) {
    return make_map_2d_sw128_elem(m, base, 2, inner, outer, row_bytes, box_inner, box_outer);
}

struct Plan {
    int NC, items, groups, ctas, base, extra;
    int NA;
    size_t off_counters, off_flags, off_agg, off_incl, off_tail, total;
};

Plan make_plan(const rglru_dims* d, int sms) {
    Plan p{};
    p.NC = (d->seq_len + L - 1) / L;
    p.items = d->batch * p.NC;
    p.groups = 2 * d->heads;
    p.ctas = p.groups >= sms ? p.groups : sms;
    p.base = p.ctas / p.groups;
    p.extra = p.ctas % p.groups;
    auto up = [](size_t v) { return (v + 255) & ~size_t(255); };
    p.off_counters = 256;
    p.off_flags = up(p.off_counters + (size_t)p.groups * 4);
    p.off_agg = up(p.off_flags + (size_t)p.groups * p.items * 16);
    p.NA = (p.NC + LBW - 1) / LBW;
    p.off_incl = up(p.off_agg + (size_t)p.groups * p.items * HALF * 8);
    p.off_tail = up(p.off_incl + (size_t)p.groups * d->batch * p.NA * HALF * 8);
    p.total = up(p.off_tail + (size_t)d->batch * kHist * d->heads * DH * sizeof(__nv_bfloat16));
    return p;
}

}  // namespace tc

bool fused_prefill_supported(const rglru_dims* d) {
    return d->act_dtype == RGLRU_BF16 && d->head_dim == tc::DH && !(d->flags & RGLRU_FLAG_GENERIC);
}

// The workspace layout is sized for the largest grid the kernel may use (one CTA per SM up to
// 1024 SMs, so the size does not depend on the device); only the parts in use are touched.
size_t fused_prefill_workspace(const rglru_dims* d) { return tc::make_plan(d, 1024).total; }

int fused_prefill_launches(const rglru_dims* d) {
    (void)d;
    return 2;   // one memset of the tickets / look-back words, one kernel (plus a copy of the
                // conv history when a state is given: not a kernel)
}

cudaError_t launch_fused_prefill(const rglru_dims* d, const rglru_params* p, const void* x, const void* y,
                                 const uint8_t* reset, rglru_state* st, void* out, void* ws, size_t ws_bytes,
                                 cudaStream_t s) {
    using namespace tc;
    int dev = 0, sms = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    if (e != cudaSuccess) return e;
    if (sms > 1024) sms = 1024;
    Plan pl = make_plan(d, sms);
    if (pl.total > ws_bytes) return cudaErrorInvalidValue;
    const int W = d->heads * d->head_dim;
    CUtensorMap mx, my, mo;
    if (!make_map_3d(&mx, x, W, d->seq_len, d->batch, DH, XROWS) ||
        !make_map_3d(&my, y, W, d->seq_len, d->batch, HALF, L) ||
        !make_map_3d(&mo, out, W, d->seq_len, d->batch, HALF, L))
        return cudaErrorInvalidValue;
    e = set_smem_once(fused_prefill_kernel, (int)SMEM_BYTES);
    if (e != cudaSuccess) return e;

    uint8_t* w = static_cast<uint8_t*>(ws);
    Args a;
    a.B = d->batch; a.T = d->seq_len; a.H = d->heads; a.NC = pl.NC; a.items = pl.items;
    a.groups = pl.groups; a.base = pl.base; a.extra = pl.extra;
    a.c = d->c; a.gelu_tanh = d->gelu_tanh; a.flags = d->flags;
    a.timeout_ns = (d->flags & RGLRU_FLAG_TEST_WITHHOLD) ? 2000000ull : 1000000000ull;
    a.conv_w = p->conv_w; a.conv_b = p->conv_b;
    a.w_a = static_cast<const __nv_bfloat16*>(p->w_a); a.w_x = static_cast<const __nv_bfloat16*>(p->w_x);
    a.b_a = p->b_a; a.b_x = p->b_x; a.lambda = p->lambda; a.reset = reset;
    a.h_state = st ? st->h : nullptr;
    a.tail_state = st ? static_cast<__nv_bfloat16*>(st->conv_tail) : nullptr;
    a.status = reinterpret_cast<DeviceStatus*>(w);
    a.counters = reinterpret_cast<unsigned*>(w + pl.off_counters);
    a.lb_flags = reinterpret_cast<unsigned*>(w + pl.off_flags);
    a.NA = pl.NA;
    a.lb_agg = reinterpret_cast<uint64_t*>(w + pl.off_agg);
    a.lb_incl = reinterpret_cast<uint64_t*>(w + pl.off_incl);
    // tickets, flags and look-back words all start at zero ("not written")
    const size_t clear = pl.off_tail - pl.off_counters;
    e = cudaMemsetAsync(w + pl.off_counters, 0, clear, s);
    if (e != cudaSuccess) return e;
    // the conv history as this call finds it: the kernel reads the copy and writes the state
    a.tail_old = nullptr;
    if (a.tail_state) {
        const size_t tail_bytes = (size_t)d->batch * kHist * W * sizeof(__nv_bfloat16);
        e = cudaMemcpyAsync(w + pl.off_tail, a.tail_state, tail_bytes, cudaMemcpyDeviceToDevice, s);
        if (e != cudaSuccess) return e;
        a.tail_old = reinterpret_cast<const __nv_bfloat16*>(w + pl.off_tail);
    }
    fused_prefill_kernel<<<pl.ctas, kThreads, SMEM_BYTES, s>>>(mx, my, mo, a);
    return cudaGetLastError();
}

}  // namespace rglru
