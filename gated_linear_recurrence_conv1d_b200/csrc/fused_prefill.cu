// fused_prefill.cu -- tensor-core RG-LRU prefill for bf16 activations, head_dim 256 (sm_100a).
//
// One kernel does the whole block (conv -> gates -> decay -> scan -> GeLU merge -> state):
//
//   * a cluster of two CTAs owns one head for its whole life; CTA r of the pair owns the
//     output channels [128 r, 128 r + 128) of the head.  Its block-diagonal gate weights
//     W_a[h][:, half], W_x[h][:, half], pre-scaled by 1/2 (exact in bf16), sit in tensor memory
//     (TMEM) as the A operand of tcgen05.mma (TS form), with the halved gate biases as one
//     more K step (a bf16 hi / lo pair against a constant column of ones), so the gate
//     pre-activations leave the MMA complete;
//   * work items are (batch row, 32-token chunk) of the head, handed out by a per-head atomic
//     ticket that the pair's first CTA takes and passes to its sibling through distributed
//     shared memory, so both CTAs of a pair work on the same item.  Tickets run across the rows
//     first (item k = chunk k / B of row k % B), so the chunk before an item usually finished a
//     few items earlier;
//   * every CTA convolves only its own 128 channels, once: the conv warps write the result in
//     fp32 for the epilogue (the i_t x_t term of the update) and rounded to bf16 as its half of
//     the MMA's B operand, into their own shared memory and, with plain remote stores, into the
//     sibling's; the gate MMA of each CTA then contracts all 256 input channels of the head;
//   * warp roles: an x producer (tickets, TMA of the CTA's x channels with a 3-token halo), a y
//     producer (TMA of the y tile), 2 conv warps (16 tokens each; a lane convolves 4 channels
//     with packed fp32x2 FMAs), one MMA issuer (D = (W/2)^T . xc^T for both gates, M = 128
//     channels, N = 32 tokens, K = 256 + the bias step) and 3 epilogue groups of 4 warps, group
//     g taking the items n = g (mod 3); 3 stages of shared-memory tiles and TMEM accumulators;
//   * transposed orientation: a TMEM lane is an output channel and the 32 columns are tokens,
//     so an epilogue thread owns one channel.  Its first pass turns the gate pre-activations
//     into a_t and the normalised input u_t and scans tokens t and t + 16 side by side (two
//     independent 16-token scans in the two halves of packed fp32x2 registers), keeping the
//     running (prod a, local h) of every token in registers and releasing the TMEM stage at
//     once; once the carry C into the chunk is known its second pass is h_t = P_t C + H_t (no
//     serial chain) times GeLU(y_t), written in place of y and stored by TMA;
//   * chunks of one sequence handled by different pairs chain through a look-back in the
//     spirit of Merrill & Garland ("Single-pass Parallel Prefix Scan with Decoupled Look-back",
//     2016): after its first pass a chunk publishes its aggregate (prod a, local h) per channel;
//     its carry is the inclusive state of an anchor chunk (every LBW-th chunk of the row)
//     followed by the aggregates of the chunks in between, applied in a fixed order so the
//     result does not depend on timing.  Each published value is one 64-bit word that shows
//     whether it has been written, so a reader polls the data itself.  Every wait is bounded by
//     %globaltimer; on expiry the kernel latches RGLRU_ERR_TIMEOUT in the workspace status word
//     and drains.
//
// Element-wise arithmetic (one transcendental per gate, one square root, one for GeLU):
//   D_a = (g_a + b_a) / 2, D_x = (g_x + b_x) / 2 straight from the MMA;
//   r_t = (1 + tanh D_a) / 2 and l_t = c r_t log sigma(Lambda) = hK (1 + tanh D_a) with
//   hK = c log sigma(Lambda) / 2;  E = expm1(l_t) by its series to l^4 for |l| <= 1/8 (the
//   channels with |c log sigma(Lambda)| <= 1/8), by ex2 otherwise; a_t = 1 + E;
//   sqrt(1 - a_t^2) / 4 = sqrt(E (-E/16 - 1/8)) (no cancellation near a_t = 1);
//   u_t / 2 = i_t x_t sqrt(1 - a_t^2) / 2 = w (1 + tanh D_x) with w = x_t sqrt(1 - a^2) / 4,
//   x_t the fp32 conv output; the scan runs on h / 2 (P starts at 1/2), so that the merge is
//   out = (h/2) y (1 + tanh(y (k1 + k3 y^2))) with k1 / k3 fitted to the exact y Phi(y)
//   (|error in Phi| <= 1.5e-4; the tanh form of the flag uses k1 = sqrt(2/pi), k3 = 0.044715 k1).
//
// Arithmetic follows "Griffin Guide: RecurrentGemma, RG-LRU & Hybrid Attention": recurrence /
// input gates, a_t = a^(c r_t) in log space, h_t = a_t h_{t-1} + sqrt(1 - a_t^2)(i_t x_t)
// ("1. Formulation of the RG-LRU Gating Mechanism"), the width-4 conv before the RG-LRU and
// the GeLU merge ("1. Temporal Filtering via Separable 1D Convolutions", "2. Non-Linear
// Multiplicative Gating with GeLU"), per-head block-diagonal gates ("3. Block-Diagonal
// Sharding for Zero-Communication Tensor Parallelism").  Only the tensor-core operand of the
// gate contraction is rounded to bf16; the conv output entering the update, the state and
// all element-wise math stay in fp32.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <mutex>

#include "common.cuh"
#include "kernels.h"
#include "rglru_math.cuh"
#include "sm100.cuh"
#include "tma_maps.h"

namespace rglru {
namespace tc {

using namespace sm100;
using namespace fm;

constexpr int DH = 256;                 // head dim (K of the gate contraction)
constexpr int HALF = 128;               // output channels per CTA (= TMEM lanes = MMA M)
constexpr int L = 32;                   // tokens per chunk (= MMA N)
constexpr int HL = L / 2;               // the two interleaved scans of a chunk
constexpr int XROWS = L + kHist;        // x tile rows incl. the 3-token halo
constexpr int KSTEPS = DH / 16;         // MMA K steps over the input channels
constexpr int G = 3;                    // stages = epilogue groups
constexpr int RING = 16;                // ring of item ids (> the producers' lead over every consumer)
constexpr int kConvTok = 16;            // tokens per conv warp
// The gate contraction takes the fp32 conv output as an fp16 hi + lo pair (two MMAs per K step):
// fp16 alone (2^-12 relative) leaves gate errors that the recurrence carries to the bf16 bar.
constexpr bool kSplitGate = true;

// warp roles: 0-1 conv (tokens [16w, 16w + 16)), 2-13 epilogue (TMEM lane quarter = warp % 4,
// group = (warp - 2) / 4; each group also loads the y tiles of its own items), 14 x producer
// (tickets and x tiles), 15 MMA.
// 16 warps = 4 per SM sub-partition, each with 128 registers a thread: the epilogue keeps the 64
// running (prod a, h) values of its chunk in registers.
constexpr int kConvWarps = 2, kEpiGroup = 4, kEpiWarps = G * kEpiGroup;
constexpr int kWarpEpi0 = kConvWarps, kWarpProd = kWarpEpi0 + kEpiWarps;
constexpr int kWarpMma = kWarpProd + 1;
constexpr int kThreads = (kWarpMma + 1) * 32;   // 512

constexpr uint32_t KBLK_BYTES = L * 128;               // one 64-channel K block of the B tile
constexpr uint32_t B_BYTES = 4 * KBLK_BYTES;           // [32 tokens x 256 channels] fp16, 128B swizzle
constexpr uint32_t X_BYTES = XROWS * HALF * 2;         // 8960: [35 tokens x 128 channels] bf16
constexpr uint32_t X_STRIDE = 9216;
constexpr uint32_t XC_BYTES = L * HALF * 4;            // [32 tokens x 128 channels] fp32 conv output
constexpr uint32_t Y_BYTES = L * HALF * 2;             // [32 tokens x 128 channels] bf16, y then out

// shared memory map (offsets from a 1024-aligned base)
constexpr uint32_t OFF_B = 0;
constexpr uint32_t OFF_BLO = OFF_B + G * B_BYTES;               // fp16(xc - fp16(xc))
constexpr uint32_t OFF_X = OFF_BLO + G * B_BYTES;
constexpr uint32_t OFF_XC = OFF_X + G * X_STRIDE;
constexpr uint32_t OFF_Y = OFF_XC + G * XC_BYTES;
constexpr uint32_t OFF_BAR = OFF_Y + G * Y_BYTES;
constexpr int NBAR = 11 * G + 2 * RING + 2;
constexpr uint32_t OFF_SLOT = (OFF_BAR + NBAR * 8 + 15) & ~15u;   // slot[RING], mailbox[RING]
constexpr uint32_t OFF_TMEMP = OFF_SLOT + 2 * RING * 4;
constexpr uint32_t OFF_ABORT = OFF_TMEMP + 16;
constexpr uint32_t SMEM_BYTES = OFF_ABORT + 16 + 1024;           // + slack for 1024 alignment
static_assert(OFF_BLO % 1024 == 0 && B_BYTES % 1024 == 0, "swizzled MMA operands");
static_assert(OFF_X % 128 == 0 && X_STRIDE % 128 == 0 && OFF_Y % 128 == 0, "TMA destinations");
static_assert(2 * HALF * DH * 2 <= OFF_BAR, "weight staging reuses the stage tiles");
static_assert(SMEM_BYTES <= 232448, "shared memory budget");

// TMEM columns: [0,128) A = W_a^T (fp16 pairs), [128,256) A = W_x^T, then per stage 2L = 64
// columns: D_a [0,L) and D_x [L,2L) (the bias-free contractions).
constexpr uint32_t TMEM_COLS = 512;
constexpr uint32_t TM_WA = 0, TM_WX = 128, TM_D = 256, TM_SLOT = 2 * L;
static_assert(TM_D + G * TM_SLOT <= TMEM_COLS, "TMEM budget");

constexpr int LBW = 4;                  // look-back block: anchors every LBW chunks
// A published look-back word is 64 bits, written by one relaxed store, and says itself whether it
// has been written (the workspace starts zeroed): an aggregate is (prod a with its sign bit set,
// local h) -- prod a is never negative -- and an anchor's inclusive state is (h, -1).
constexpr uint32_t kReadyBit = 0x80000000u;

struct Args {
    int B, T, H, NC, items;          // items = B * NC per head
    int base, extra;                 // clusters per head: base (+1 for the first `extra` heads)
    int NA;                          // anchors per row: ceil(NC / LBW)
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
    unsigned* counters;              // [H] tickets
    uint64_t* lb_agg;                // [2H][items][128] aggregate words
    uint64_t* lb_incl;               // [2H][B * NA][128] anchor inclusive-state words
    // save mode (the forward again for the gradients): [B, T, W] outputs instead of out
    float* sv_ga;                    // complete gate pre-activations
    float* sv_gx;
    float* sv_hprev;                 // h_{t-1} as the update used it
    __nv_bfloat16* sv_xc_hi;         // the fp32 conv output as bf16 hi + lo
    __nv_bfloat16* sv_xc_lo;
};

// mbarrier addresses, computed (a runtime-indexed array of them would live in local memory):
// per stage s 11 barriers, then the two rings of RING, then w_ready and mma_done
struct Bars {
    uint32_t base;
    __device__ __forceinline__ uint32_t at(int s, int kind) const { return base + (uint32_t)(s * 11 + kind) * 8u; }
    __device__ __forceinline__ uint32_t x_full(int s) const { return at(s, 0); }
    __device__ __forceinline__ uint32_t x_empty(int s) const { return at(s, 1); }
    __device__ __forceinline__ uint32_t y_full(int s) const { return at(s, 2); }
    __device__ __forceinline__ uint32_t y_empty(int s) const { return at(s, 3); }
    __device__ __forceinline__ uint32_t half_done(int s) const { return at(s, 4); }
    __device__ __forceinline__ uint32_t b_full(int s) const { return at(s, 5); }
    __device__ __forceinline__ uint32_t b_empty(int s) const { return at(s, 6); }
    __device__ __forceinline__ uint32_t xc_empty(int s) const { return at(s, 7); }
    __device__ __forceinline__ uint32_t acc_full(int s) const { return at(s, 8); }
    __device__ __forceinline__ uint32_t acc_empty(int s) const { return at(s, 9); }
    __device__ __forceinline__ uint32_t out_ready(int s) const { return at(s, 10); }
    __device__ __forceinline__ uint32_t tk(int i) const { return base + (uint32_t)(11 * G + i) * 8u; }
    __device__ __forceinline__ uint32_t tk_mail(int i) const { return base + (uint32_t)(11 * G + RING + i) * 8u; }
    __device__ __forceinline__ uint32_t w_ready() const { return base + (uint32_t)(11 * G + 2 * RING) * 8u; }
    __device__ __forceinline__ uint32_t mma_done() const { return base + (uint32_t)(11 * G + 2 * RING + 1) * 8u; }
};

// Context of the bounded waits: they give up after timeout_ns, or as soon as another thread of
// the grid has latched a failure, so that every role drains instead of hanging.
struct WaitCtx {
    DeviceStatus* status;
    unsigned long long timeout_ns;
    volatile int* abort;
};

__device__ __noinline__ bool wait_bar_slow(uint32_t bar, uint32_t parity, WaitCtx w, unsigned where, bool cluster) {
    const uint64_t t0 = globaltimer_ns();
    for (;;) {
        if (cluster ? mbar_try_wait_cluster(bar, parity) : mbar_try_wait_sleep(bar, parity, 100000u)) return true;
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
        if (cluster) __nanosleep(256);
    }
}

__device__ __forceinline__ bool wait_bar(uint32_t bar, uint32_t parity, WaitCtx w, unsigned where) {
    if (mbar_try_wait(bar, parity)) return true;
    return wait_bar_slow(bar, parity, w, where, false);
}
// for barriers that other CTAs of the cluster arrive on (their writes are acquired at cluster scope)
__device__ __forceinline__ bool wait_bar_cl(uint32_t bar, uint32_t parity, WaitCtx w, unsigned where) {
    if (mbar_try_wait_cluster(bar, parity)) return true;
    return wait_bar_slow(bar, parity, w, where, true);
}

// The same wait for a warp whose lanes then run warp-collective instructions: every lane waits,
// and the outcome is made uniform, so that the warp never splits on a timeout.
__device__ __forceinline__ bool wait_bar_warp(uint32_t bar, uint32_t parity, WaitCtx w, unsigned where) {
    return __all_sync(0xffffffffu, wait_bar(bar, parity, w, where));
}

__device__ __forceinline__ float bf16lo(uint32_t v) { return __uint_as_float(v << 16); }
__device__ __forceinline__ float bf16hi(uint32_t v) { return __uint_as_float(v & 0xFFFF0000u); }
__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
    __nv_bfloat162 p = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t*>(&p);
}
__device__ __forceinline__ uint32_t pack_f16x2(float lo, float hi) {
    __half2 p = __floats2half2_rn(lo, hi);
    return *reinterpret_cast<uint32_t*>(&p);
}
__device__ __forceinline__ float f16lo(uint32_t v) { return __half2float(__ushort_as_half((unsigned short)(v & 0xFFFFu))); }
__device__ __forceinline__ float f16hi(uint32_t v) { return __half2float(__ushort_as_half((unsigned short)(v >> 16))); }

// A lane's 4 channels of one token, fp32.
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

// Bit j of the result = reset[t0 + j] != 0 for the L tokens of a chunk (0 past the end).
__device__ __forceinline__ uint32_t chunk_reset_mask(const uint8_t* row, int t0, int T, int lane) {
    const bool r = t0 + lane < T && row[t0 + lane] != 0;
    return __ballot_sync(0xffffffffu, r);
}

// The conv of one warp's kConvTok tokens (j0 + jj) for a lane's 4 channels: fp32 into the xc
// tile, fp16 into this CTA's and the sibling's B tile.  RST: the chunk has segment starts (bit
// jj of rm: token j0 + jj starts one, so the history before it is dropped); LAST: the row's
// last token (jlast, relative to j0) is in this range and the window after it is kept in fw.
template <bool RST, bool LAST, bool LO>
__device__ __forceinline__ void conv_tokens(const uint8_t* xtw, uint8_t* btw, uint32_t btw_peer, float4* xcw,
                                            uint32_t cchunk, uint32_t rm, int jlast, const float2 (&w)[kConvWidth][2],
                                            const float2 (&cb)[2], Vec4& h0, Vec4& h1, Vec4& h2, uint2 (&fw)[3]) {
#pragma unroll
    for (int jj = 0; jj < kConvTok; ++jj) {
        const Vec4 xv = unpack4(*reinterpret_cast<const uint2*>(xtw + (jj + kHist) * HALF * 2));
        if (RST && ((rm >> jj) & 1u)) h0 = h1 = h2 = zero4();
        float2 y0 = fma2(w[0][0], h0.v[0], cb[0]);
        y0 = fma2(w[1][0], h1.v[0], y0);
        y0 = fma2(w[2][0], h2.v[0], y0);
        y0 = fma2(w[3][0], xv.v[0], y0);
        float2 y1 = fma2(w[0][1], h0.v[1], cb[1]);
        y1 = fma2(w[1][1], h1.v[1], y1);
        y1 = fma2(w[2][1], h2.v[1], y1);
        y1 = fma2(w[3][1], xv.v[1], y1);
        xcw[jj * (HALF / 4)] = make_float4(y0.x, y0.y, y1.x, y1.y);
        const uint2 o = make_uint2(pack_f16x2(y0.x, y0.y), pack_f16x2(y1.x, y1.y));
        const uint32_t off = (jj >> 3) * 1024 + (jj & 7) * 128 + ((cchunk ^ (jj & 7)) << 4);
        *reinterpret_cast<uint2*>(btw + off) = o;
        st_cluster_v2(btw_peer + off, o);
        if constexpr (LO) {                // the rounding residue, as a second fp16 operand
            const uint2 lo = make_uint2(pack_f16x2(y0.x - f16lo(o.x), y0.y - f16hi(o.x)),
                                        pack_f16x2(y1.x - f16lo(o.y), y1.y - f16hi(o.y)));
            *reinterpret_cast<uint2*>(btw + (OFF_BLO - OFF_B) + off) = lo;
            st_cluster_v2(btw_peer + (OFF_BLO - OFF_B) + off, lo);
        }
        h0 = h1; h1 = h2; h2 = xv;
        if (LAST && jj == jlast) { fw[0] = pack4(h0); fw[1] = pack4(h1); fw[2] = pack4(h2); }
    }
}

// Per-channel constants of the epilogue: nb_g = -b_g log2 e (the gate biases, folded into the
// scaling FMA) and K = c log sigma(Lambda).
struct ChanK {
    float2 nba, nbx, K;
};

// First pass of an epilogue thread over its channel's 32 tokens: tokens j and j + 16 side by
// side.  P[j], H[j] receive the running prod a and local h of both scans (zero carry in).
// RST: zero a_t at segment starts (bit t of rm); GEN: any decay range, ragged chunk (tokens
// t >= nt are the identity a = 1, u = 0).
template <bool RST, bool GEN>
__device__ __forceinline__ void pass1(uint32_t dcol, const float* xcs, const ChanK& ck, uint32_t rm, int nt,
                                      float2 (&P)[HL], float2 (&H)[HL]) {
    float2 p = f2(1.0f), hc = f2(0.0f);
#pragma unroll
    for (int blk = 0; blk < HL / 4; ++blk) {
        float da0[4], da1[4], dx0[4], dx1[4];
        tmem_ld4(dcol + 4 * blk, da0);
        tmem_ld4(dcol + HL + 4 * blk, da1);
        tmem_ld4(dcol + L + 4 * blk, dx0);
        tmem_ld4(dcol + L + HL + 4 * blk, dx1);
        float x0[4], x1[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            x0[i] = xcs[(4 * blk + i) * HALF];
            x1[i] = xcs[(HL + 4 * blk + i) * HALF];
        }
        tmem_wait_ld();
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const int j = 4 * blk + i;
            float2 a, u;
            gates2<!GEN>(make_float2(da0[i], da1[i]), make_float2(dx0[i], dx1[i]), ck.nba, ck.nbx, ck.K,
                         make_float2(x0[i], x1[i]), a, u);
            if constexpr (RST) {                                  // h_{t-1} := 0 at a segment start
                if ((rm >> j) & 1u) a.x = 0.f;
                if ((rm >> (j + HL)) & 1u) a.y = 0.f;
            }
            if constexpr (GEN) {                                  // past the end: identity
                if (j >= nt) { a.x = 1.f; u.x = 0.f; }
                if (j + HL >= nt) { a.y = 1.f; u.y = 0.f; }
            }
            hc = fma2(a, hc, u);
            p = mul2(p, a);
            P[j] = p;
            H[j] = hc;
        }
    }
}

// Save-mode first pass: the same two scans with accurate fp32 math (CUDA's expf / sqrtf), writing
// the complete gate pre-activations (with their biases) and the conv output (as a bf16 hi + lo
// pair) of every token of the chunk to the save arrays (e0: element of token 0).
__device__ __forceinline__ void pass1_save(uint32_t dcol, const float* xcs, float kappa, float ba, float bx, uint32_t rm,
                                           int nt, const Args& a, size_t e0, int W, float2 (&P)[HL], float2 (&H)[HL]) {
    float2 p = f2(1.0f), hc = f2(0.0f);
#pragma unroll
    for (int blk = 0; blk < HL / 4; ++blk) {
        float da0[4], da1[4], dx0[4], dx1[4];
        tmem_ld4(dcol + 4 * blk, da0);
        tmem_ld4(dcol + HL + 4 * blk, da1);
        tmem_ld4(dcol + L + 4 * blk, dx0);
        tmem_ld4(dcol + L + HL + 4 * blk, dx1);
        float x0[4], x1[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            x0[i] = xcs[(4 * blk + i) * HALF];
            x1[i] = xcs[(HL + 4 * blk + i) * HALF];
        }
        tmem_wait_ld();
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const int j = 4 * blk + i;
            const float das[2] = {da0[i], da1[i]}, dxs[2] = {dx0[i], dx1[i]}, xs[2] = {x0[i], x1[i]};
            float av[2], uv[2];
#pragma unroll
            for (int hf = 0; hf < 2; ++hf) {
                const int t = j + hf * HL;
                const float ga = das[hf] + ba, gx = dxs[hf] + bx;
                const float r = sigmoid_acc(ga), ig = sigmoid_acc(gx);
                float at, beta;
                decay_and_beta_acc(kappa, r, &at, &beta);
                float u = beta * (ig * xs[hf]);
                if ((rm >> t) & 1u) at = 0.f;                 // h_{t-1} := 0 at a segment start
                if (t < nt) {
                    const size_t e = e0 + (size_t)t * W;
                    a.sv_ga[e] = ga;
                    a.sv_gx[e] = gx;
                    const __nv_bfloat16 hi = __float2bfloat16_rn(xs[hf]);
                    a.sv_xc_hi[e] = hi;
                    a.sv_xc_lo[e] = __float2bfloat16_rn(xs[hf] - __bfloat162float(hi));
                } else {                                      // past the end: identity
                    at = 1.f;
                    u = 0.f;
                }
                av[hf] = at;
                uv[hf] = u;
            }
            const float2 a2 = make_float2(av[0], av[1]);
            hc = fma2(a2, hc, make_float2(uv[0], uv[1]));
            p = mul2(p, a2);
            P[j] = p;
            H[j] = hc;
        }
    }
}

// Second pass: h_t = P_t C + H_t (no serial chain; cc = the carries into both halves) times
// GeLU(y_t), written in place of y.
template <bool TANH>
__device__ __forceinline__ void pass2(unsigned short* yt, float2 cc, const float2 (&P)[HL], const float2 (&H)[HL]) {
#pragma unroll
    for (int j = 0; j < HL; ++j) {
        unsigned short* y0 = yt + j * HALF;
        unsigned short* y1 = yt + (j + HL) * HALF;
        const float2 yv = make_float2(__uint_as_float((uint32_t)*y0 << 16), __uint_as_float((uint32_t)*y1 << 16));
        const float2 hh = fma2(P[j], cc, H[j]);
        const float2 g = TANH ? gelu_tanh2(yv) : gelu_erf2(yv);
        const float2 o = mul2(hh, g);
        const uint32_t ob = pack_bf16x2(o.x, o.y);
        *y0 = (unsigned short)(ob & 0xFFFFu);
        *y1 = (unsigned short)(ob >> 16);
    }
}

template <bool SAVE>
__global__ void __launch_bounds__(kThreads, 1)
fused_prefill_kernel(const __grid_constant__ CUtensorMap map_x, const __grid_constant__ CUtensorMap map_y,
                     const __grid_constant__ CUtensorMap map_out, const Args a) {
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const uint32_t sbase = smem_u32(smem);
    const Bars bars{sbase + OFF_BAR};
    volatile int* slot = reinterpret_cast<volatile int*>(smem + OFF_SLOT);            // [RING]
    volatile int* mailbox = reinterpret_cast<volatile int*>(smem + OFF_SLOT + RING * 4);
    volatile uint32_t* tmem_base_s = reinterpret_cast<volatile uint32_t*>(smem + OFF_TMEMP);
    volatile int* abort = reinterpret_cast<volatile int*>(smem + OFF_ABORT);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t rank = cluster_ctarank(), peer = rank ^ 1u;

    // ---- head of this pair -------------------------------------------------------------------
    int head;
    {
        const int cl = blockIdx.x >> 1, big = a.extra * (a.base + 1);
        head = cl < big ? cl / (a.base + 1) : a.extra + (cl - big) / a.base;
    }
    const int grp = head * 2 + (int)rank;             // look-back group: (head, channel half)
    const int W = a.H * DH;
    const size_t lb_base = (size_t)grp * a.items;
    const size_t lb_base_a = (size_t)grp * a.B * a.NA;

    // ---- set-up ------------------------------------------------------------------------------
    if (threadIdx.x == 0) {
        for (int s = 0; s < G; ++s) {
            mbar_init(bars.x_full(s), 1);
            mbar_init(bars.x_empty(s), kConvWarps);
            mbar_init(bars.y_full(s), 1);
            mbar_init(bars.half_done(s), kConvWarps);
            mbar_init(bars.b_full(s), kConvWarps);          // the sibling's conv warps
            mbar_init(bars.b_empty(s), 2);                  // both CTAs' MMAs
            mbar_init(bars.xc_empty(s), kEpiGroup);
            mbar_init(bars.acc_full(s), 1);
            mbar_init(bars.acc_empty(s), kEpiGroup);
            mbar_init(bars.out_ready(s), kEpiGroup);
        }
        for (int i = 0; i < RING; ++i) {
            mbar_init(bars.tk(i), 1);
            mbar_init(bars.tk_mail(i), 1);
        }
        mbar_init(bars.w_ready(), kEpiWarps);
        mbar_init(bars.mma_done(), 1);
        *abort = 0;
        fence_barrier_init();
        fence_proxy_async_smem();
    }
    if (warp == kWarpMma) {
        tmem_alloc(smem_u32((const void*)tmem_base_s), TMEM_COLS);
        tmem_relinquish();
    }
    if (warp == kWarpProd && lane == 0) {
        prefetch_tensormap(&map_x);
        prefetch_tensormap(&map_y);
        prefetch_tensormap(&map_out);
    }
    // stage this CTA's gate weights W_g[head][i][rank*128 + o] (o contiguous) in shared memory as
    // fp16 with coalesced 16-byte loads: gate a at byte 0, gate x at byte 65536 (the stage tiles
    // are still unused).  bf16 -> fp16 is exact for 2^-14 <= |w| < 65504; smaller magnitudes
    // round to the fp16 grid of 2^-24, larger ones saturate the gate as their exact value does.
    if (warp < kConvWarps + kEpiWarps) {
        const int tid = threadIdx.x;
        for (int e = tid; e < 2 * DH * (HALF / 8); e += (kConvWarps + kEpiWarps) * 32) {
            const int g = e / (DH * (HALF / 8)), r = e % (DH * (HALF / 8));
            const int i = r / (HALF / 8), o8 = r % (HALF / 8);
            const __nv_bfloat16* src = (g ? a.w_x : a.w_a) + ((size_t)head * DH + i) * DH + rank * HALF + o8 * 8;
            uint4 v = __ldg(reinterpret_cast<const uint4*>(src));
            uint32_t* vv = reinterpret_cast<uint32_t*>(&v);
#pragma unroll
            for (int k = 0; k < 4; ++k) vv[k] = pack_f16x2(bf16lo(vv[k]), bf16hi(vv[k]));
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
        // each lane quarter writes gate a, group 1 gate x
        const int q = warp & 3, g = (warp - kWarpEpi0) >> 2, m = q * 32 + lane;
        const uint32_t lane_off = (uint32_t)(q * 32) << 16;
        if (g < 2) {
            const unsigned short* ws = reinterpret_cast<const unsigned short*>(smem + g * (HALF * DH * 2)) + m;
#pragma unroll 1
            for (int j0 = 0; j0 < DH / 2; j0 += 16) {
                uint32_t r[16];
#pragma unroll
                for (int j = 0; j < 16; ++j) {
                    const int i = 2 * (j0 + j);
                    r[j] = (uint32_t)ws[i * HALF] | ((uint32_t)ws[(i + 1) * HALF] << 16);
                }
                tmem_st16(tmem + lane_off + (g ? TM_WX : TM_WA) + j0, r);
            }
        }
        tmem_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(bars.w_ready());
    }
    __syncthreads();   // the staging area is free again before any tile lands in it
    cluster_sync();    // both CTAs' barriers are initialised before any remote arrive targets them

    int mma_items = 0;   // items whose MMAs this CTA issued (the MMA thread's count)

    if (warp == kWarpProd) {
        if (lane == 0) {
            // ============================ x producer (and tickets) ============================
            const uint32_t peer_mail = map_to_rank(smem_u32((const void*)mailbox), peer);
            int issued[G] = {};
            for (int n = 0;; ++n) {
                const int st = n % G;
                const uint32_t ph = (n / G) & 1;
                if (!wait_bar(bars.x_empty(st), ph ^ 1, wc, 1)) break;
                int k;
                if (rank == 0) {
                    k = (int)atomicAdd(&a.counters[head], 1u);
                    if (k >= a.items) k = -1;
                    st_cluster_u32(peer_mail + (n % RING) * 4, (uint32_t)k);
                    mbar_arrive_cluster(map_to_rank(bars.tk_mail(n % RING), peer));
                } else {
                    if (!wait_bar_cl(bars.tk_mail(n % RING), (n / RING) & 1, wc, 2)) break;
                    k = mailbox[n % RING];
                }
                if (k < 0) {
                    // terminal item for the roles of iteration n and of the next G-1 iterations
                    // (every epilogue group's y loader looks one item past its last, so each of
                    // the G slots gets its ticket arrival)
                    for (int i = 0; i < G; ++i) slot[(n + i) % RING] = -1;
                    for (int i = 0; i < G; ++i) mbar_arrive(bars.tk((n + i) % RING));
                    mbar_arrive(bars.x_full(st));
                    issued[st] = 0;   // that phase completing implies the earlier load landed
                    break;
                }
                slot[n % RING] = k;
                mbar_arrive(bars.tk(n % RING));
                const int b = k % a.B, c = k / a.B;
                mbar_arrive_expect_tx(bars.x_full(st), X_BYTES);
                tma_load_3d(sbase + OFF_X + st * X_STRIDE, &map_x, head * DH + (int)rank * HALF, c * L - kHist, b,
                            bars.x_full(st));
                issued[st] = n + 1;
            }
            // never leave the CTA with a bulk copy still writing its shared memory
            for (int st = 0; st < G; ++st)
                if (issued[st]) {
                    const int n = issued[st] - 1;
                    const uint64_t t0 = globaltimer_ns();
                    while (!mbar_try_wait_sleep(bars.x_full(st), (n / G) & 1, 100000u) &&
                           globaltimer_ns() - t0 < a.timeout_ns) {
                    }
                }
        }
    } else if (warp == kWarpMma) {
        // ================================ MMA issuer ===========================================
        // the whole warp runs the loop (its waits and branches are warp-uniform) and one elected
        // lane issues: the instructions' operands then stay uniform, and consecutive MMAs issue
        // at the tensor pipe's rate
        const uint32_t idesc = idesc_f16_f32(HALF, L);
        const uint32_t tm = __shfl_sync(0xffffffffu, tmem, 0);
        bool ok = wait_bar_warp(bars.w_ready(), 0, wc, 5);
        tc_fence_after();
        for (int n = 0; ok; ++n) {
            const int st = n % G;
            const uint32_t ph = (n / G) & 1;
            if (!wait_bar_warp(bars.half_done(st), ph, wc, 6)) break;
            if (__shfl_sync(0xffffffffu, slot[n % RING], 0) < 0) {
                // hand the terminal item to the epilogue groups of iterations n .. n + G - 1,
                // each once it has released its previous item (so that no phase is skipped)
                for (int i = 0; i < G; ++i) {
                    const int n2 = n + i, s2 = n2 % G;
                    if (n2 >= G && !wait_bar_warp(bars.acc_empty(s2), ((n2 - G) / G) & 1, wc, 7)) break;
                    if (lane == 0) mbar_arrive(bars.acc_full(s2));
                }
                break;
            }
            if (!__all_sync(0xffffffffu, wait_bar_cl(bars.b_full(st), ph, wc, 8))) break;   // the sibling's half
            if (!wait_bar_warp(bars.acc_empty(st), ph ^ 1, wc, 9)) break;
            tc_fence_after();
            // K step ks: descriptor = the stage's base descriptor + the step's byte offset / 16;
            // the conv output's fp16 hi and lo parts
            const uint32_t d0 = tm + TM_D + st * TM_SLOT;
            if (elect_one()) {
#pragma unroll
                for (int part = 0; part < (SAVE || kSplitGate ? 2 : 1); ++part) {
                    const uint64_t bd0 = desc_k_sw128(sbase + (part ? OFF_BLO : OFF_B) + st * B_BYTES);
#pragma unroll
                    for (int ks = 0; ks < KSTEPS; ++ks) {
                        const uint64_t bd = bd0 + (uint64_t)((((ks >> 2) * KBLK_BYTES) + (ks & 3) * 32) >> 4);
                        const uint32_t acc = (part > 0 || ks > 0) ? 1u : 0u;
                        mma_ts(d0, tm + TM_WA + ks * 8, bd, idesc, acc);
                        mma_ts(d0 + L, tm + TM_WX + ks * 8, bd, idesc, acc);
                    }
                }
                mma_commit(bars.acc_full(st));
                mma_commit(bars.b_empty(st));
                mma_commit_cluster(map_to_rank(bars.b_empty(st), peer));
            }
            __syncwarp();
            mma_items = n + 1;
        }
        // every MMA this warp issued has finished before TMEM is released
        if (elect_one()) mma_commit(bars.mma_done());
        __syncwarp();
        if (lane == 0) {
            uint64_t t0 = globaltimer_ns();
            while (!mbar_try_wait_sleep(bars.mma_done(), 0, 100000u) && globaltimer_ns() - t0 < a.timeout_ns) {
            }
            // and the sibling's MMAs of the last items have told this CTA so (their commits
            // arrive on this CTA's b_empty): nothing remote is left in flight at the exit
            for (int i = mma_items - G < 0 ? 0 : mma_items - G; i < mma_items; ++i) {
                t0 = globaltimer_ns();
                while (!mbar_try_wait_cluster(bars.b_empty(i % G), (i / G) & 1) && globaltimer_ns() - t0 < a.timeout_ns) {
                    __nanosleep(256);
                }
            }
        }
        __syncwarp();
    } else if (warp < kConvWarps) {
        // ================================ conv warps ==========================================
        // warp w convolves this CTA's 128 channels for the tokens [16w, 16w + 16) of the chunk;
        // lane l 4 channels (8 bytes of a B-tile row)
        const int j0 = warp * kConvTok;
        const int cl = (int)rank * HALF + lane * 4;       // channel within the head
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
        // B-tile byte offset of (token t, channel cl): kb * KBLK + (t / 8) * 1024 + (t % 8) * 128
        //   + ((chunk ^ (t % 8)) * 16) + sub, chunk / sub = 16-byte chunk / byte within it
        const uint32_t kb_off = (uint32_t)(cl >> 6) * KBLK_BYTES + ((cl & 7) * 2);
        const uint32_t cchunk = (cl & 63) >> 3;
        const uint32_t peer_b = map_to_rank(sbase + OFF_B, peer);
        for (int n = 0;; ++n) {
            const int st = n % G;
            const uint32_t ph = (n / G) & 1;
            if (!wait_bar_warp(bars.x_full(st), ph, wc, 10)) break;
            if (!wait_bar_warp(bars.b_empty(st), ph ^ 1, wc, 11)) break;    // both MMAs of the stage's last item
            if (!wait_bar_warp(bars.xc_empty(st), ph ^ 1, wc, 12)) break;   // its epilogue has read xc
            const int k = slot[n % RING];
            if (k < 0) {
                __syncwarp();
                if (lane == 0) mbar_arrive(bars.half_done(st));   // the MMA issuer meets the end here
                break;
            }
            const int b = k % a.B, c = k / a.B, t0 = c * L;
            const int nt = min(L, a.T - t0);
            const uint8_t* rrow = a.reset ? a.reset + (size_t)b * a.T : nullptr;
            const uint32_t rmask = rrow ? chunk_reset_mask(rrow, t0, a.T, lane) : 0u;
            const uint8_t* xt = smem + OFF_X + st * X_STRIDE + lane * 8;
            auto xrow = [&](int r) {                      // x tile row r = token t0 - 3 + r
                return unpack4(*reinterpret_cast<const uint2*>(xt + r * HALF * 2));
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
            const uint32_t rm = rmask >> j0;
            const uint8_t* xtw = xt + j0 * HALF * 2;
            const uint32_t boff = st * B_BYTES + kb_off + (j0 >> 3) * 1024;
            uint8_t* btw = smem + OFF_B + boff;
            const uint32_t btw_peer = peer_b + boff;
            float4* xcw = reinterpret_cast<float4*>(smem + OFF_XC + st * XC_BYTES) + j0 * (HALF / 4) + lane;
            const int jlast = nt - 1 - j0;
            if ((rm & 0xFFFFu) == 0) {
                if (has_last) conv_tokens<false, true, SAVE || kSplitGate>(xtw, btw, btw_peer, xcw, cchunk, rm, jlast, w, cb, h0, h1, h2, fw);
                else conv_tokens<false, false, SAVE || kSplitGate>(xtw, btw, btw_peer, xcw, cchunk, rm, jlast, w, cb, h0, h1, h2, fw);
            } else {
                if (has_last) conv_tokens<true, true, SAVE || kSplitGate>(xtw, btw, btw_peer, xcw, cchunk, rm, jlast, w, cb, h0, h1, h2, fw);
                else conv_tokens<true, false, SAVE || kSplitGate>(xtw, btw, btw_peer, xcw, cchunk, rm, jlast, w, cb, h0, h1, h2, fw);
            }
            // the MMAs (async proxy) of both CTAs read what this warp wrote
            fence_proxy_async_smem();
            fence_proxy_async_cluster();
            __syncwarp();
            if (lane == 0) {
                mbar_arrive(bars.x_empty(st));
                mbar_arrive(bars.half_done(st));
                mbar_arrive_cluster(map_to_rank(bars.b_full(st), peer));
            }
            // final conv history of the sequence (this CTA's channels), as soon as the row's
            // last token is convolved: the conv read the copy taken before the launch
            if (!SAVE && a.tail_state && c == a.NC - 1 && has_last) {
                __nv_bfloat16* tl = a.tail_state + (size_t)b * kHist * W + chg;
#pragma unroll
                for (int r = 0; r < 3; ++r) *reinterpret_cast<uint2*>(tl + (size_t)r * W) = fw[r];
            }
        }
    } else if (warp < kWarpEpi0 + kEpiWarps) {
        // ================================ epilogue groups ======================================
        const int q = warp & 3;                          // TMEM lane quarter
        const int eg = (warp - kWarpEpi0) >> 2;          // group = stage it owns
        const int st = eg;
        const int m = q * 32 + lane;                     // local output channel = TMEM lane
        const int ch = head * DH + (int)rank * HALF + m; // global channel
        const uint32_t lane_off = (uint32_t)(q * 32) << 16;
        const float kappa = a.c * log_sigmoid_acc(a.lambda[ch]);       // log a_t = kappa r_t
        const float ba = a.b_a ? a.b_a[ch] : 0.0f, bx = a.b_x ? a.b_x[ch] : 0.0f;
        const ChanK ck{f2(-ba * kLog2e), f2(-bx * kLog2e), f2(kappa)};
        // the series for expm1 serves every token of a warp whose channels all decay slowly
        const bool warp_small = __all_sync(0xffffffffu, kappa >= -0.125f);
        const int tanh_form = a.gelu_tanh;
        const bool withhold_hook = (a.flags & RGLRU_FLAG_TEST_WITHHOLD) && grp == 0;
        const float* xcs = reinterpret_cast<const float*>(smem + OFF_XC + st * XC_BYTES) + m;
        unsigned short* yt = reinterpret_cast<unsigned short*>(smem + OFF_Y + st * Y_BYTES) + m;
        const uint32_t dcol = tmem + lane_off + TM_D + st * TM_SLOT;
        // y tile of the group's item m into its stage, by one thread, once the ticket of m is
        // known and the stage's previous out tile has been read by its store; false: no load
        // (the end, or a failed wait)
        const bool y_loader = !SAVE && q == 0 && lane == 0;
        auto load_y = [&](int m) -> bool {
            if (!wait_bar(bars.tk(m % RING), (m / RING) & 1, wc, 3)) return false;
            const int km = slot[m % RING];
            if (km < 0) return false;
            mbar_arrive_expect_tx(bars.y_full(st), Y_BYTES);
            tma_load_3d(sbase + OFF_Y + st * Y_BYTES, &map_y, head * DH + (int)rank * HALF, (km / a.B) * L, km % a.B,
                        bars.y_full(st));
            return true;
        };
        int y_pending = -1;                              // item whose y load is in flight, or -1
        if (y_loader && load_y(eg)) y_pending = eg;

        for (int n = eg;; n += G) {
            const uint32_t ph = (n / G) & 1;
            if (!wait_bar_warp(bars.acc_full(st), ph, wc, 13)) break;
            const int k = slot[n % RING];
            if (k < 0) break;
            if (!wait_bar_warp(bars.half_done(st), ph, wc, 14)) break;     // the xc tile is written
            tc_fence_after();
            const int b = k % a.B, c = k / a.B, t0 = c * L;
            const int nt = min(L, a.T - t0);
            const uint8_t* rrow = a.reset ? a.reset + (size_t)b * a.T : nullptr;
            const uint32_t rmask = rrow ? chunk_reset_mask(rrow, t0, a.T, lane) : 0u;
            const size_t kb_item = lb_base + (size_t)b * a.NC;       // first chunk of this row
            const bool withhold = withhold_hook && k == 0;

            // ---- pass 1: gates, decay and normalised input, both scans; the TMEM stage and the
            //      xc tile are released as soon as they have been read
            float2 P[HL], H[HL];
            if constexpr (SAVE) {
                pass1_save(dcol, xcs, kappa, ba, bx, rmask, nt, a, ((size_t)b * a.T + t0) * W + ch, W, P, H);
            } else if (nt == L && warp_small) {
                if (rmask) pass1<true, false>(dcol, xcs, ck, rmask, nt, P, H);
                else pass1<false, false>(dcol, xcs, ck, rmask, nt, P, H);
            } else {
                pass1<true, true>(dcol, xcs, ck, rmask, nt, P, H);
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) {
                mbar_arrive(bars.acc_empty(st));
                mbar_arrive(bars.xc_empty(st));
            }
            // the chunk's aggregate: prod a over the chunk and its local h
            const float aggA = P[HL - 1].x * P[HL - 1].y;
            const float aggH = fmaf(P[HL - 1].y, H[HL - 1].x, H[HL - 1].y);
            if (c > 0 && !withhold)                      // as early as possible
                st_relaxed_gpu_u64(a.lb_agg + (kb_item + c) * HALF + m,
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
                    uint64_t gw[LBW];
                    gw[0] = ld_relaxed_gpu_u64(wi);
#pragma unroll
                    for (int i = 1; i < LBW; ++i)
                        gw[i] = i <= nagg ? ld_relaxed_gpu_u64(wa + (size_t)(i - 1) * HALF)
                                          : (uint64_t)(__float_as_uint(1.0f) | kReadyBit);
                    bool okl = (uint32_t)(gw[0] >> 32) & kReadyBit;
#pragma unroll
                    for (int i = 1; i < LBW; ++i) okl = okl && ((uint32_t)gw[i] & kReadyBit);
                    if (__all_sync(0xffffffffu, okl)) {
                        float hc = __uint_as_float((uint32_t)gw[0]);
#pragma unroll
                        for (int i = 1; i < LBW; ++i)
                            hc = fmaf(__uint_as_float((uint32_t)gw[i] & ~kReadyBit), hc, __uint_as_float((uint32_t)(gw[i] >> 32)));
                        carry = hc;
                        break;
                    }
                    __nanosleep(64);
                    if ((it & 15) == 15) {
                        int give_up = 0;
                        if (lane == 0) {
                            if (*abort || *(volatile unsigned*)&a.status->code != 0) give_up = 1;
                            else if (globaltimer_ns() - tw > a.timeout_ns) {
                                latch_status(a.status, RGLRU_ERR_TIMEOUT, 15, blockIdx.x, (unsigned)k);
                                give_up = 1;
                            }
                            if (give_up) *abort = 1;
                        }
                        if (__shfl_sync(0xffffffffu, give_up, 0)) break;
                    }
                }
            }
            const float incl = fmaf(aggA, carry, aggH);             // state after the chunk
            if (c % LBW == 0 && !withhold)                          // only anchors' states are read
                st_relaxed_gpu_u64(a.lb_incl + (lb_base_a + (size_t)b * a.NA + c / LBW) * HALF + m,
                                   ((uint64_t)0xBF800000u << 32) | __float_as_uint(incl));
            // final state of the row: its carry chain passed through the first chunk, which
            // read the old state before publishing, so the old value is no longer needed
            if (!SAVE && a.h_state && c == a.NC - 1) a.h_state[(size_t)b * W + ch] = incl;

            if constexpr (SAVE) {
                // ---- save-mode second pass: h_{t-1} of every token (0 at a segment start)
                const float c1 = fmaf(P[HL - 1].x, carry, H[HL - 1].x);          // state after token 15
                const float2 cc = make_float2(carry, c1);
                float2 prev = cc;
                const size_t e0 = ((size_t)b * a.T + t0) * W + ch;
#pragma unroll
                for (int j = 0; j < HL; ++j) {
                    const float hp0 = ((rmask >> j) & 1u) ? 0.f : prev.x;
                    const float hp1 = ((rmask >> (j + HL)) & 1u) ? 0.f : prev.y;
                    if (j < nt) a.sv_hprev[e0 + (size_t)j * W] = hp0;
                    if (j + HL < nt) a.sv_hprev[e0 + (size_t)(j + HL) * W] = hp1;
                    prev = fma2(P[j], cc, H[j]);
                }
                continue;
            }

            // ---- pass 2: h_t = P_t C + H_t (no serial chain), merged with GeLU(y_t)
            if (!wait_bar_warp(bars.y_full(st), ph, wc, 16)) break;
            if (y_loader) y_pending = -1;
            {
                const float c1 = fmaf(P[HL - 1].x, carry, H[HL - 1].x);          // state after token 15
                const float2 cc = make_float2(carry, c1);
                if (tanh_form) pass2<true>(yt, cc, P, H);
                else pass2<false>(yt, cc, P, H);
            }

            // ---- out tile -> global (TMA store clips the ragged tail)
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) mbar_arrive(bars.out_ready(st));
            if (q == 0 && lane == 0) {
                if (wait_bar(bars.out_ready(st), ph, wc, 17)) {
                    tma_store_3d(&map_out, sbase + OFF_Y + st * Y_BYTES, head * DH + (int)rank * HALF, t0, b);
                    bulk_commit();
                    bulk_wait_read0();                   // the tile is free for the next y
                    if (load_y(n + G)) y_pending = n + G;
                }
            }
        }
        // no tensor-memory access of this warp may still be in flight when TMEM is released, and
        // no bulk copy may still write this CTA's shared memory when it exits
        tmem_wait_ld();
        if (q == 0 && lane == 0) {
            bulk_wait0();
            if (y_pending >= 0) {
                const uint64_t t0 = globaltimer_ns();
                while (!mbar_try_wait_sleep(bars.y_full(st), (y_pending / G) & 1, 100000u) &&
                       globaltimer_ns() - t0 < a.timeout_ns) {
                }
            }
        }
    }

    // ---- teardown: all tensor-core work has drained (the MMA thread waited on mma_done) ------
    tc_fence_before();
    __syncthreads();
    cluster_sync();    // no remote store, arrive or commit is left in flight towards either CTA
    if (warp == kWarpMma) {
        tc_fence_after();
        tmem_dealloc(tmem, TMEM_COLS);
    }
}

// --------------------------------------------------------------------------- host side ------

struct Plan {
    int NC, items, NA;
    size_t off_counters, off_agg, off_incl, off_tail, total;
};

Plan make_plan(const rglru_dims* d) {
    Plan p{};
    p.NC = (d->seq_len + L - 1) / L;
    p.items = d->batch * p.NC;
    p.NA = (p.NC + LBW - 1) / LBW;
    auto up = [](size_t v) { return (v + 255) & ~size_t(255); };
    const size_t groups = 2 * (size_t)d->heads;
    p.off_counters = 256;
    p.off_agg = up(p.off_counters + (size_t)d->heads * 4);
    p.off_incl = up(p.off_agg + groups * p.items * HALF * 8);
    p.off_tail = up(p.off_incl + groups * d->batch * p.NA * HALF * 8);
    p.total = up(p.off_tail + (size_t)d->batch * kHist * d->heads * DH * sizeof(__nv_bfloat16));
    return p;
}

// Clusters of two that fit on the device at once (1 CTA per SM), looked up once per device.
cudaError_t max_pairs(int dev, int* out) {
    static std::mutex mu;
    static int cache[64] = {};
    if (dev >= 0 && dev < 64) {
        std::lock_guard<std::mutex> lock(mu);
        if (cache[dev] > 0) {
            *out = cache[dev];
            return cudaSuccess;
        }
    }
    cudaLaunchConfig_t cfg = {};
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.gridDim = dim3(2, 1, 1);
    cfg.blockDim = dim3(kThreads, 1, 1);
    cfg.dynamicSmemBytes = SMEM_BYTES;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    int n = 0;
    cudaError_t e = cudaOccupancyMaxActiveClusters(&n, fused_prefill_kernel<false>, &cfg);
    if (e != cudaSuccess) return e;
    if (n < 1) n = 1;
    if (dev >= 0 && dev < 64) {
        std::lock_guard<std::mutex> lock(mu);
        cache[dev] = n;
    }
    *out = n;
    return cudaSuccess;
}

}  // namespace tc

bool fused_prefill_supported(const rglru_dims* d) {
    return d->act_dtype == RGLRU_BF16 && d->head_dim == tc::DH && !(d->flags & RGLRU_FLAG_GENERIC);
}

size_t fused_prefill_workspace(const rglru_dims* d) { return tc::make_plan(d).total; }

int fused_prefill_launches(const rglru_dims* d) {
    (void)d;
    return 2;   // one memset of the tickets / look-back words, one kernel (plus a copy of the
                // conv history when a state is given: not a kernel)
}

namespace tc {

// Both modes: the regular prefill (out, state written back) and the save mode (the forward again
// for the gradients: the save arrays instead of out, the state only read; `status` replaces the
// workspace's own status word).
template <bool SAVE>
cudaError_t launch_impl(const rglru_dims* d, const rglru_params* p, const void* x, const void* y,
                        const uint8_t* reset, const rglru_state* st, void* out, const PrefillSave* sv, void* ws,
                        size_t ws_bytes, DeviceStatus* status, cudaStream_t s) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    Plan pl = make_plan(d);
    if (pl.total > ws_bytes) return cudaErrorInvalidValue;
    const int W = d->heads * d->head_dim;
    CUtensorMap mx, my, mo;
    if (!make_map_3d(&mx, x, W, d->seq_len, d->batch, HALF, XROWS)) return cudaErrorInvalidValue;
    if (SAVE) {
        my = mx;   // y and out are not touched in the save mode
        mo = mx;
    } else if (!make_map_3d(&my, y, W, d->seq_len, d->batch, HALF, L) ||
               !make_map_3d(&mo, out, W, d->seq_len, d->batch, HALF, L)) {
        return cudaErrorInvalidValue;
    }
    e = set_smem_once(fused_prefill_kernel<SAVE>, (int)SMEM_BYTES);
    if (e != cudaSuccess) return e;
    int pairs = 0;
    e = max_pairs(dev, &pairs);
    if (e != cudaSuccess) return e;
    // every head gets at least one pair; with more pairs than heads, all of them stay busy
    // (a pair only takes a ticket when it is running, so pairs that wait for an SM are harmless)
    const int nclusters = pairs > d->heads ? pairs : d->heads;

    uint8_t* w = static_cast<uint8_t*>(ws);
    Args a{};
    a.B = d->batch; a.T = d->seq_len; a.H = d->heads; a.NC = pl.NC; a.items = pl.items; a.NA = pl.NA;
    a.base = nclusters / d->heads; a.extra = nclusters % d->heads;
    a.c = d->c; a.gelu_tanh = d->gelu_tanh; a.flags = d->flags;
    a.timeout_ns = (d->flags & RGLRU_FLAG_TEST_WITHHOLD) ? 2000000ull : 1000000000ull;
    a.conv_w = p->conv_w; a.conv_b = p->conv_b;
    a.w_a = static_cast<const __nv_bfloat16*>(p->w_a); a.w_x = static_cast<const __nv_bfloat16*>(p->w_x);
    a.b_a = p->b_a; a.b_x = p->b_x; a.lambda = p->lambda; a.reset = reset;
    a.h_state = st ? st->h : nullptr;
    a.tail_state = st ? static_cast<__nv_bfloat16*>(st->conv_tail) : nullptr;
    a.status = status ? status : reinterpret_cast<DeviceStatus*>(w);
    a.counters = reinterpret_cast<unsigned*>(w + pl.off_counters);
    a.lb_agg = reinterpret_cast<uint64_t*>(w + pl.off_agg);
    a.lb_incl = reinterpret_cast<uint64_t*>(w + pl.off_incl);
    if (SAVE) {
        a.sv_ga = sv->ga; a.sv_gx = sv->gx; a.sv_hprev = sv->hprev;
        a.sv_xc_hi = sv->xc_hi; a.sv_xc_lo = sv->xc_lo;
    }
    // tickets and look-back words all start at zero ("not written")
    e = cudaMemsetAsync(w + pl.off_counters, 0, pl.off_tail - pl.off_counters, s);
    if (e != cudaSuccess) return e;
    // the conv history as this call finds it: the kernel reads the copy and writes the state
    a.tail_old = nullptr;
    if (a.tail_state) {
        const size_t tail_bytes = (size_t)d->batch * kHist * W * sizeof(__nv_bfloat16);
        e = cudaMemcpyAsync(w + pl.off_tail, a.tail_state, tail_bytes, cudaMemcpyDeviceToDevice, s);
        if (e != cudaSuccess) return e;
        a.tail_old = reinterpret_cast<const __nv_bfloat16*>(w + pl.off_tail);
    }
    cudaLaunchConfig_t cfg = {};
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.gridDim = dim3(2 * nclusters, 1, 1);
    cfg.blockDim = dim3(kThreads, 1, 1);
    cfg.dynamicSmemBytes = SMEM_BYTES;
    cfg.stream = s;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, fused_prefill_kernel<SAVE>, mx, my, mo, a);
}

}  // namespace tc

cudaError_t launch_fused_prefill(const rglru_dims* d, const rglru_params* p, const void* x, const void* y,
                                 const uint8_t* reset, rglru_state* st, void* out, void* ws, size_t ws_bytes,
                                 cudaStream_t s) {
    return tc::launch_impl<false>(d, p, x, y, reset, st, out, nullptr, ws, ws_bytes, nullptr, s);
}

cudaError_t launch_fused_prefill_save(const rglru_dims* d, const rglru_params* p, const void* x,
                                      const uint8_t* reset, const rglru_state* st, const PrefillSave* sv, void* ws,
                                      size_t ws_bytes, DeviceStatus* status, cudaStream_t s) {
    return tc::launch_impl<true>(d, p, x, nullptr, reset, st, nullptr, sv, ws, ws_bytes, status, s);
}

}  // namespace rglru
