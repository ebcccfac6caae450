// fused_prefill.cu -- tensor-core RG-LRU prefill for bf16 activations, head_dim 256 (sm_100a).
//
// One kernel does the whole block (conv -> gates -> decay -> scan -> GeLU merge -> state):
//
//   * a CTA owns one half of one head -- the output channels [128 r, 128 r + 128) of head h,
//     a "group" (h, r) -- for its whole life; the groups share the SMs evenly.  Its block-diagonal
//     gate weights W_a[h][:, half], W_x[h][:, half] sit in tensor memory (TMEM) as the A operand
//     of tcgen05.mma (TS form); the gate biases enter later, as the addends of the epilogue's
//     scaling FMAs;
//   * work items are (batch row, 32-token chunk), handed out by a per-group atomic ticket.
//     Tickets run across the rows first (item k = chunk k / B of row k % B), so the chunk before
//     an item usually finished a few items earlier;
//   * every CTA convolves all 256 input channels of its head for its item (the gate contraction
//     needs them as K; the other half of the head does the same for its own output channels, so
//     the two never wait on each other): the conv warps write the result as the MMA's B operand
//     -- a bf16 pair hi + lo per value, hi = the fp32 value truncated, lo = its remainder rounded,
//     so that hi + lo is the fp32 value to 2^-16 -- and, for the CTA's own 128 channels, in fp32
//     for the epilogue (the i_t x_t term of the update);
//   * warp roles: an x producer (tickets and the TMA of the [35 tokens x 256 channels] x tile
//     with its 3-token halo), one MMA warp (D = W^T . xc^T for both gates, M = 128 channels, N =
//     32 tokens, K = 256 x 2 parts; an elected lane issues), 3 groups of 4 warps, group g taking
//     the items n = g (mod 3): it convolves its next item (a lane 8 channels x 8 tokens with
//     packed fp32x2 FMAs) and runs the epilogue of its current one, and a store warp that writes
//     each finished out tile by TMA and loads the stage's next y tile; 3 stages of shared-memory
//     tiles, 4 TMEM accumulator slots;
//   * transposed orientation: a TMEM lane is an output channel and the 32 columns are tokens,
//     so an epilogue thread owns one channel.  Its first pass turns the gate contractions into
//     a_t and the normalised input u_t, 8 tokens at a time, writes them back over the stage's
//     TMEM columns and accumulates the chunk's aggregate (prod a, local h from a zero carry);
//     once the carry into the chunk is known its second pass runs h_t = a_t h_{t-1} + u_t from
//     it, times GeLU(y_t), written in place of y and stored by TMA;
//   * chunks of one sequence handled by different CTAs chain through a look-back in the spirit
//     of Merrill & Garland ("Single-pass Parallel Prefix Scan with Decoupled Look-back", 2016):
//     after its first pass a chunk publishes its aggregate per channel; its carry is the
//     inclusive state of an anchor chunk (every LBW-th chunk of the row) followed by the
//     aggregates of the chunks in between, applied in a fixed order so the result does not depend
//     on timing.  Each published value is one 64-bit word that shows whether it has been
//     written, so a reader polls the data itself.  Every wait is bounded by %globaltimer; on
//     expiry the kernel latches RGLRU_ERR_TIMEOUT in the workspace status word and drains.
//
// Element-wise arithmetic: rglru_math.cuh (gates by ex2 and a reciprocal, expm1 of the
// log-decay by its series where |c log sigma(Lambda)| <= 1/8, sqrt(1 - a^2) i_t by one rsqrt,
// GeLU by a fitted tail polynomial and one ex2).
//
// Arithmetic follows "Griffin Guide: RecurrentGemma, RG-LRU & Hybrid Attention": recurrence /
// input gates, a_t = a^(c r_t) in log space, h_t = a_t h_{t-1} + sqrt(1 - a_t^2)(i_t x_t)
// ("1. Formulation of the RG-LRU Gating Mechanism"), the width-4 conv before the RG-LRU and
// the GeLU merge ("1. Temporal Filtering via Separable 1D Convolutions", "2. Non-Linear
// Multiplicative Gating with GeLU"), per-head block-diagonal gates ("3. Block-Diagonal
// Sharding for Zero-Communication Tensor Parallelism").  The conv output entering the update,
// the state and all element-wise math stay in fp32.
#include <cuda.h>
#include <cuda_bf16.h>
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
constexpr int XROWS = L + kHist;        // x tile rows incl. the 3-token halo
constexpr int KSTEPS = DH / 16;         // MMA K steps over the input channels
constexpr int G = 3;                    // stages = epilogue groups
constexpr int RING = 16;                // ring of item ids (> the producer's lead over every consumer)
constexpr int kConvTok = 8;             // tokens per warp of a group's conv
constexpr int kConvBatch = 4;           // x rows a conv lane loads ahead of their arithmetic
// The gate contraction takes the fp32 conv output as a bf16 pair hi + lo (two MMAs per K step):
// a single 16-bit operand leaves gate errors that the recurrence carries to the bf16 bar.
constexpr bool kSplitGate = true;

// warp roles: 0-11 three groups of 4 (TMEM lane quarter = warp % 4, group = warp / 4): a group
// convolves its next item and runs the epilogue of its current one; 12 x producer (tickets and x
// tiles), 13 MMA, 14 out stores and y loads.  15 warps: at most 4 per SM sub-partition, so 128
// registers a thread.
constexpr int kEpiGroup = 4, kEpiWarps = G * kEpiGroup;
constexpr int kWarpProd = kEpiWarps, kWarpMma = kWarpProd + 1, kWarpStore = kWarpMma + 1;
constexpr int kThreads = (kWarpStore + 1) * 32;   // 480
constexpr int kSlots = 4;               // TMEM accumulator slots (item n uses slot n % 4)

constexpr uint32_t KBLK_BYTES = L * 128;               // one 64-channel K block of the B tile
constexpr uint32_t B_BYTES = 4 * KBLK_BYTES;           // [32 tokens x 256 channels] bf16, 128B swizzle
constexpr uint32_t X_BYTES = XROWS * DH * 2;           // 17920: [35 tokens x 256 channels] bf16
constexpr uint32_t X_STRIDE = X_BYTES;
constexpr uint32_t XC_BYTES = L * HALF * 4;            // [32 tokens x 128 channels] fp32 conv output
constexpr uint32_t Y_BYTES = L * HALF * 2;             // [32 tokens x 128 channels] bf16, y then out

// shared memory map (offsets from a 1024-aligned base)
constexpr uint32_t OFF_B = 0;                          // bf16 hi parts
constexpr uint32_t OFF_BLO = OFF_B + G * B_BYTES;      // bf16 lo parts
constexpr uint32_t OFF_X = OFF_BLO + G * B_BYTES;
constexpr uint32_t OFF_XC = OFF_X + G * X_STRIDE;
constexpr uint32_t OFF_Y = OFF_XC + G * XC_BYTES;
constexpr uint32_t OFF_CW = OFF_Y + G * Y_BYTES;       // conv taps [4][256] and bias [256] of the head, fp32
constexpr uint32_t OFF_BAR = OFF_CW + 5 * DH * 4;
constexpr int kBarsPerStage = 6;
constexpr int NBAR = kBarsPerStage * G + kSlots + RING + 2;
constexpr uint32_t OFF_SLOT = (OFF_BAR + NBAR * 8 + 15) & ~15u;   // slot[RING]
constexpr uint32_t OFF_TMEMP = OFF_SLOT + RING * 4;
constexpr uint32_t OFF_ABORT = OFF_TMEMP + 16;
constexpr uint32_t SMEM_BYTES = OFF_ABORT + 16 + 1024;           // + slack for 1024 alignment
static_assert(OFF_BLO % 1024 == 0 && B_BYTES % 1024 == 0, "swizzled MMA operands");
static_assert(OFF_X % 128 == 0 && X_STRIDE % 128 == 0 && OFF_Y % 128 == 0, "TMA destinations");
static_assert(OFF_CW % 16 == 0, "16-byte loads of the conv taps");
static_assert(2 * HALF * DH * 2 <= OFF_BAR, "weight staging reuses the stage tiles");
static_assert(SMEM_BYTES <= 232448, "shared memory budget");

// TMEM columns: [0,128) A = W_a^T (bf16 pairs), [128,256) A = W_x^T, then per slot 2L = 64
// columns: D_a [0,L) and D_x [L,2L) (the bias-free contractions), which the epilogue's first
// pass overwrites with a_t and u_t for its second.  Four slots for three groups: the MMA of an
// item does not wait for the second pass of the item three before it.
constexpr uint32_t TMEM_COLS = 512;
constexpr uint32_t TM_WA = 0, TM_WX = 128, TM_D = 256, TM_SLOT = 2 * L;
static_assert(TM_D + kSlots * TM_SLOT <= TMEM_COLS, "TMEM budget");

constexpr int LBW = 4;                  // look-back block: anchors every LBW chunks
// A published look-back word is 64 bits, written by one relaxed store, and says itself whether it
// has been written (the workspace starts zeroed): an aggregate is (prod a with its sign bit set,
// local h) -- prod a is never negative -- and an anchor's inclusive state is (h, -1).
constexpr uint32_t kReadyBit = 0x80000000u;

struct Args {
    int B, T, H, NC, items;          // items = B * NC per head
    int base, extra;                 // CTAs per group (head, half): base (+1 for the first `extra` groups)
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
    unsigned* counters;              // [2H] tickets, one per group
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
// per stage (= group) s 6 barriers, per TMEM slot its release, the ticket ring, w_ready, mma_done
struct Bars {
    uint32_t base;
    __device__ __forceinline__ uint32_t at(int s, int kind) const {
        return base + (uint32_t)(s * kBarsPerStage + kind) * 8u;
    }
    __device__ __forceinline__ uint32_t x_full(int s) const { return at(s, 0); }
    __device__ __forceinline__ uint32_t x_empty(int s) const { return at(s, 1); }     // the conv read the x tile
    __device__ __forceinline__ uint32_t y_full(int s) const { return at(s, 2); }
    __device__ __forceinline__ uint32_t conv_done(int s) const { return at(s, 3); }   // the B tile is written
    __device__ __forceinline__ uint32_t acc_full(int s) const { return at(s, 4); }    // the item's MMA is done
    __device__ __forceinline__ uint32_t out_ready(int s) const { return at(s, 5); }
    __device__ __forceinline__ uint32_t slot_free(int i) const { return base + (uint32_t)(kBarsPerStage * G + i) * 8u; }
    __device__ __forceinline__ uint32_t tk(int i) const { return base + (uint32_t)(kBarsPerStage * G + kSlots + i) * 8u; }
    __device__ __forceinline__ uint32_t w_ready() const {
        return base + (uint32_t)(kBarsPerStage * G + kSlots + RING) * 8u;
    }
    __device__ __forceinline__ uint32_t mma_done() const {
        return base + (uint32_t)(kBarsPerStage * G + kSlots + RING + 1) * 8u;
    }
};

// named barrier of one group's 4 warps (ids 1..3; 0 is __syncthreads)
__device__ __forceinline__ void group_sync(int g) {
    asm volatile("bar.sync %0, %1;" ::"r"(1 + g), "n"(kEpiGroup * 32) : "memory");
}

// Context of the bounded waits: they give up after timeout_ns, or as soon as another thread of
// the CTA or the grid has latched a failure, so that every role drains instead of hanging.
struct WaitCtx {
    DeviceStatus* status;
    unsigned long long timeout_ns;
    volatile int* abort;
};

__device__ __noinline__ bool wait_bar_slow(uint32_t bar, uint32_t parity, WaitCtx w, unsigned where) {
    const uint64_t t0 = globaltimer_ns();
    for (;;) {
        if (mbar_try_wait_sleep(bar, parity, 100000u)) return true;
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

__device__ __forceinline__ float bf16lo(uint32_t v) { return __uint_as_float(v << 16); }
__device__ __forceinline__ float bf16hi(uint32_t v) { return __uint_as_float(v & 0xFFFF0000u); }
__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
    __nv_bfloat162 p = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t*>(&p);
}

// 4 channels of one token, fp32 pairs.
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

// bf16 hi (truncation) of two fp32 values, packed, and their fp32 remainders
__device__ __forceinline__ uint32_t trunc_bf16x2(float2 v) {
    return __byte_perm(__float_as_uint(v.x), __float_as_uint(v.y), 0x7632);
}
__device__ __forceinline__ float2 rem_bf16(float2 v) {
    return make_float2(v.x - __uint_as_float(__float_as_uint(v.x) & 0xFFFF0000u),
                       v.y - __uint_as_float(__float_as_uint(v.y) & 0xFFFF0000u));
}

// The conv of kConvTok tokens (j0 + jj) for 4 of a lane's channels: the bf16 pair
// hi + lo into the B tiles (bhi: the 8 bytes of these channels in the lane's 16-byte column of K
// block / chunk; row offsets added here), and for a lane of the CTA's own half (xcw != nullptr)
// fp32 into the xc tile.  x rows are loaded kConvBatch at a time ahead of their arithmetic.
// RST: the chunk has segment starts (bit jj of rm: token j0 + jj starts one, so the history
// before it is dropped); LAST: the row's last token (jlast, relative to j0) is in this range and
// the window after it (resets applied) is kept in fw.
template <bool RST, bool LAST>
__device__ __forceinline__ void conv_tokens(const uint8_t* xtw, uint8_t* bhi, float4* xcw, uint32_t cchunk, uint32_t rm,
                                            int jlast, const float2 (&w)[kConvWidth][2], const float2 (&cb)[2],
                                            Vec4& h0, Vec4& h1, Vec4& h2, uint2 (&fw)[3]) {
#pragma unroll
    for (int jb = 0; jb < kConvTok; jb += kConvBatch) {
        uint2 xr[kConvBatch];
#pragma unroll
        for (int i = 0; i < kConvBatch; ++i) xr[i] = *reinterpret_cast<const uint2*>(xtw + (jb + i + kHist) * DH * 2);
#pragma unroll
        for (int i = 0; i < kConvBatch; ++i) {
            const int jj = jb + i;
            const Vec4 xv = unpack4(xr[i]);
            if (RST && ((rm >> jj) & 1u)) h0 = h1 = h2 = zero4();
            float2 y[2];
#pragma unroll
            for (int p = 0; p < 2; ++p) {
                float2 acc = fma2(w[0][p], h0.v[p], cb[p]);
                acc = fma2(w[1][p], h1.v[p], acc);
                acc = fma2(w[2][p], h2.v[p], acc);
                y[p] = fma2(w[3][p], xv.v[p], acc);
            }
            if (xcw) xcw[jj * (HALF / 4)] = make_float4(y[0].x, y[0].y, y[1].x, y[1].y);
            const uint2 o = make_uint2(trunc_bf16x2(y[0]), trunc_bf16x2(y[1]));
            const float2 r0 = rem_bf16(y[0]), r1 = rem_bf16(y[1]);
            const uint2 lo = make_uint2(pack_bf16x2(r0.x, r0.y), pack_bf16x2(r1.x, r1.y));
            const uint32_t off = (jj >> 3) * 1024 + (jj & 7) * 128 + ((cchunk ^ (jj & 7)) << 4);
            *reinterpret_cast<uint2*>(bhi + off) = o;
            *reinterpret_cast<uint2*>(bhi + (OFF_BLO - OFF_B) + off) = lo;
            h0 = h1; h1 = h2; h2 = xv;
            if (LAST && jj == jlast) { fw[0] = pack4(h0); fw[1] = pack4(h1); fw[2] = pack4(h2); }
        }
    }
}

// Per-channel constants of the epilogue: nb_g = -b_g log2 e (the gate biases, folded into the
// scaling FMA) and K = c log sigma(Lambda).
struct ChanK {
    float2 nba, nbx, K;
};

constexpr int kBT = 8;                  // tokens per batch of the epilogue passes

// First pass of an epilogue thread over its channel's 32 tokens, 8 at a time (all loads of a
// batch issued before its arithmetic): gates, decay and normalised input of every token, written
// back over the token's TMEM columns (a_t in D_a's, u_t in D_x's), and the chunk's aggregate
// (prod a, local h from a zero carry).  RST: zero a_t at segment starts (bit t of rm); GEN: any
// decay range, ragged chunk (tokens t >= nt are the identity a = 1, u = 0).
template <bool RST, bool GEN>
__device__ __forceinline__ void pass1(uint32_t dcol, const float* xcs, const ChanK& ck, uint32_t rm, int nt,
                                      float& aggA, float& aggH) {
    float A = 1.0f, Hc = 0.0f;
#pragma unroll 1
    for (int t0 = 0; t0 < L; t0 += kBT) {
        float da[kBT], dx[kBT], xc[kBT];
        tmem_ld8(dcol + t0, da);
        tmem_ld8(dcol + L + t0, dx);
#pragma unroll
        for (int i = 0; i < kBT; ++i) xc[i] = xcs[(t0 + i) * HALF];
        tmem_wait_ld();
        float av[kBT], uv[kBT];
#pragma unroll
        for (int i = 0; i < kBT; i += 2) {
            float2 a2, u2;
            gates2<!GEN>(make_float2(da[i], da[i + 1]), make_float2(dx[i], dx[i + 1]), ck.nba, ck.nbx, ck.K,
                         make_float2(xc[i], xc[i + 1]), a2, u2);
            av[i] = a2.x; av[i + 1] = a2.y;
            uv[i] = u2.x; uv[i + 1] = u2.y;
        }
#pragma unroll
        for (int i = 0; i < kBT; ++i) {
            const int t = t0 + i;
            if (RST && ((rm >> t) & 1u)) av[i] = 0.f;       // h_{t-1} := 0 at a segment start
            if (GEN && t >= nt) { av[i] = 1.f; uv[i] = 0.f; }   // past the end: identity
            Hc = fmaf(av[i], Hc, uv[i]);
            A *= av[i];
        }
        tmem_st8f(dcol + t0, av);
        tmem_st8f(dcol + L + t0, uv);
    }
    tmem_wait_st();
    aggA = A;
    aggH = Hc;
}

// Save-mode first pass: the same arithmetic (any decay range), also writing the complete gate
// pre-activations (with their biases) and the conv output (as a bf16 hi + lo pair) of every token
// of the chunk to the save arrays (e0: element of token 0).
__device__ __forceinline__ void pass1_save(uint32_t dcol, const float* xcs, const ChanK& ck, float ba, float bx,
                                           uint32_t rm, int nt, const Args& a, size_t e0, int W, float& aggA,
                                           float& aggH) {
    float A = 1.0f, Hc = 0.0f;
#pragma unroll 1
    for (int t0 = 0; t0 < L; t0 += kBT) {
        float da[kBT], dx[kBT], xc[kBT];
        tmem_ld8(dcol + t0, da);
        tmem_ld8(dcol + L + t0, dx);
#pragma unroll
        for (int i = 0; i < kBT; ++i) xc[i] = xcs[(t0 + i) * HALF];
        tmem_wait_ld();
        float av[kBT], uv[kBT];
#pragma unroll
        for (int i = 0; i < kBT; i += 2) {
            float2 a2, u2;
            gates2<false>(make_float2(da[i], da[i + 1]), make_float2(dx[i], dx[i + 1]), ck.nba, ck.nbx, ck.K,
                          make_float2(xc[i], xc[i + 1]), a2, u2);
            av[i] = a2.x; av[i + 1] = a2.y;
            uv[i] = u2.x; uv[i + 1] = u2.y;
        }
#pragma unroll
        for (int i = 0; i < kBT; ++i) {
            const int t = t0 + i;
            if ((rm >> t) & 1u) av[i] = 0.f;                  // h_{t-1} := 0 at a segment start
            if (t < nt) {
                const size_t e = e0 + (size_t)t * W;
                a.sv_ga[e] = da[i] + ba;
                a.sv_gx[e] = dx[i] + bx;
                const __nv_bfloat16 hi = __float2bfloat16_rn(xc[i]);
                a.sv_xc_hi[e] = hi;
                a.sv_xc_lo[e] = __float2bfloat16_rn(xc[i] - __bfloat162float(hi));
            } else {                                          // past the end: identity
                av[i] = 1.f;
                uv[i] = 0.f;
            }
            Hc = fmaf(av[i], Hc, uv[i]);
            A *= av[i];
        }
        tmem_st8f(dcol + t0, av);
        tmem_st8f(dcol + L + t0, uv);
    }
    tmem_wait_st();
    aggA = A;
    aggH = Hc;
}

// Second pass: h_t = a_t h_{t-1} + u_t from the carry, times GeLU(y_t), written in place of y.
template <bool TANH>
__device__ __forceinline__ void pass2(uint32_t dcol, unsigned short* yt, float carry) {
    float h = carry;
#pragma unroll 1
    for (int t0 = 0; t0 < L; t0 += kBT) {
        float av[kBT], uv[kBT], g[kBT];
        tmem_ld8(dcol + t0, av);
        tmem_ld8(dcol + L + t0, uv);
#pragma unroll
        for (int i = 0; i < kBT; ++i) g[i] = __uint_as_float((uint32_t)yt[(t0 + i) * HALF] << 16);
        tmem_wait_ld();
#pragma unroll
        for (int i = 0; i < kBT; i += 2) {
            const float2 gg = TANH ? gelu_tanh2(make_float2(g[i], g[i + 1])) : gelu_erf2(make_float2(g[i], g[i + 1]));
            g[i] = gg.x;
            g[i + 1] = gg.y;
        }
#pragma unroll
        for (int i = 0; i < kBT; i += 2) {
            const float h0 = fmaf(av[i], h, uv[i]);
            h = fmaf(av[i + 1], h0, uv[i + 1]);
            const uint32_t ob = pack_bf16x2(h0 * g[i], h * g[i + 1]);
            yt[(t0 + i) * HALF] = (unsigned short)(ob & 0xFFFFu);
            yt[(t0 + i + 1) * HALF] = (unsigned short)(ob >> 16);
        }
    }
}

// Save-mode second pass: h_{t-1} of every token as the update used it (0 at a segment start).
__device__ __forceinline__ void pass2_save(uint32_t dcol, float carry, uint32_t rm, int nt, const Args& a, size_t e0,
                                           int W) {
    float h = carry;
#pragma unroll 1
    for (int t0 = 0; t0 < L; t0 += kBT) {
        float av[kBT], uv[kBT];
        tmem_ld8(dcol + t0, av);
        tmem_ld8(dcol + L + t0, uv);
        tmem_wait_ld();
#pragma unroll
        for (int i = 0; i < kBT; ++i) {
            const int t = t0 + i;
            if (t < nt) a.sv_hprev[e0 + (size_t)t * W] = ((rm >> t) & 1u) ? 0.f : h;
            h = fmaf(av[i], h, uv[i]);
        }
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
    volatile uint32_t* tmem_base_s = reinterpret_cast<volatile uint32_t*>(smem + OFF_TMEMP);
    volatile int* abort = reinterpret_cast<volatile int*>(smem + OFF_ABORT);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    // ---- group (head, half) of this CTA -------------------------------------------------------
    int grp;
    {
        const int cta = blockIdx.x, big = a.extra * (a.base + 1);
        grp = cta < big ? cta / (a.base + 1) : a.extra + (cta - big) / a.base;
    }
    const int head = grp >> 1, half = grp & 1;
    const int W = a.H * DH;
    const size_t lb_base = (size_t)grp * a.items;
    const size_t lb_base_a = (size_t)grp * a.B * a.NA;

    // ---- set-up ------------------------------------------------------------------------------
    if (threadIdx.x == 0) {
        for (int s = 0; s < G; ++s) {
            mbar_init(bars.x_full(s), 1);
            mbar_init(bars.x_empty(s), 1);
            mbar_init(bars.y_full(s), 1);
            mbar_init(bars.conv_done(s), 1);
            mbar_init(bars.acc_full(s), 1);
            mbar_init(bars.out_ready(s), kEpiGroup);
        }
        for (int i = 0; i < kSlots; ++i) mbar_init(bars.slot_free(i), kEpiGroup);
        for (int i = 0; i < RING; ++i) mbar_init(bars.tk(i), 1);
        mbar_init(bars.w_ready(), kEpiWarps);
        mbar_init(bars.mma_done(), 1);
        *abort = 0;
        fence_barrier_init();
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
    // stage this CTA's gate weights W_g[head][i][half*128 + o] (o contiguous, bf16 as given) in
    // shared memory with coalesced 16-byte loads: gate a at byte 0, gate x at byte 65536 (the
    // stage tiles are still unused)
    if (warp < kEpiWarps) {
        const int tid = threadIdx.x;
        for (int e = tid; e < 2 * DH * (HALF / 8); e += kEpiWarps * 32) {
            const int g = e / (DH * (HALF / 8)), r = e % (DH * (HALF / 8));
            const int i = r / (HALF / 8), o8 = r % (HALF / 8);
            const __nv_bfloat16* src = (g ? a.w_x : a.w_a) + ((size_t)head * DH + i) * DH + half * HALF + o8 * 8;
            const uint4 v = __ldg(reinterpret_cast<const uint4*>(src));
            *reinterpret_cast<uint4*>(smem + g * (HALF * DH * 2) + (i * HALF + o8 * 8) * 2) = v;
        }
        // the conv taps and bias of the head's 256 channels (the conv of every item reads them)
        float* cw = reinterpret_cast<float*>(smem + OFF_CW);
        for (int e = tid; e < 5 * DH; e += kEpiWarps * 32) {
            const int k = e / DH, c = e % DH;
            cw[e] = k < kConvWidth ? a.conv_w[(size_t)k * W + head * DH + c] : (a.conv_b ? a.conv_b[head * DH + c] : 0.f);
        }
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_base_s;
    const WaitCtx wc{a.status, a.timeout_ns, abort};

    if (warp < kEpiWarps) {
        // weights -> TMEM A operand: lane m, column j holds (W[2j][m], W[2j+1][m]); group 0 of
        // each lane quarter writes gate a, group 1 gate x
        const int q = warp & 3, g = warp >> 2, m = q * 32 + lane;
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

    if (warp == kWarpProd) {
        if (lane == 0) {
            // ============================ x producer (and tickets) ============================
            int issued[G] = {};
            for (int n = 0;; ++n) {
                const int st = n % G;
                const uint32_t ph = (n / G) & 1;
                if (!wait_bar(bars.x_empty(st), ph ^ 1, wc, 1)) break;
                int k = (int)atomicAdd(&a.counters[grp], 1u);
                if (k >= a.items) k = -1;
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
                tma_load_3d(sbase + OFF_X + st * X_STRIDE, &map_x, head * DH, c * L - kHist, b, bars.x_full(st));
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
        const uint32_t idesc = idesc_bf16_f32(HALF, L);
        const uint32_t tm = __shfl_sync(0xffffffffu, tmem, 0);
        bool ok = wait_bar_warp(bars.w_ready(), 0, wc, 5);
        tc_fence_after();
        for (int n = 0; ok; ++n) {
            const int st = n % G, sl = n % kSlots;
            // the item's B tile (its group's conv); the terminal item ends the loop
            if (!wait_bar_warp(bars.conv_done(st), (n / G) & 1, wc, 6)) break;
            if (__shfl_sync(0xffffffffu, slot[n % RING], 0) < 0) break;
            if (!wait_bar_warp(bars.slot_free(sl), ((n / kSlots) & 1) ^ 1, wc, 9)) break;
            tc_fence_after();
            // K step ks: descriptor = the stage's base descriptor + the step's byte offset / 16;
            // the conv output's bf16 hi and lo parts
            const uint32_t d0 = tm + TM_D + sl * TM_SLOT;
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
            }
            __syncwarp();
        }
        // every MMA this warp issued has finished before TMEM is released
        if (elect_one()) mma_commit(bars.mma_done());
        __syncwarp();
        if (lane == 0) {
            const uint64_t t0 = globaltimer_ns();
            while (!mbar_try_wait_sleep(bars.mma_done(), 0, 100000u) && globaltimer_ns() - t0 < a.timeout_ns) {
            }
        }
        __syncwarp();
    } else if (warp < kEpiWarps) {
        // ================================ groups: conv, epilogue, y loads =====================
        const int q = warp & 3;                          // TMEM lane quarter; conv tokens [8q, 8q + 8)
        const int eg = warp >> 2;                        // group = stage it owns (items n = eg mod 3)
        const int st = eg;
        const int m = q * 32 + lane;                     // local output channel = TMEM lane
        const int ch = head * DH + half * HALF + m;      // global channel
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

        // ---- the conv of item n (its x tile landed in this group's stage): lane l convolves the
        //      channels [8l, 8l + 8) of the head, 4 at a time, for the tokens [8q, 8q + 8): the
        //      bf16 pair hi + lo into the B tiles, fp32 into the xc tile for this CTA's half;
        //      false: item n is the end (nothing to convolve) or a wait failed
        const int j0 = q * kConvTok;
        const int cl = lane * 8;                          // channel within the head
        const bool own = (cl >> 7) == half;               // one of this CTA's output channels
        const uint32_t cchunk = (uint32_t)(lane & 7);
        const uint32_t kb_off = (uint32_t)(lane >> 3) * KBLK_BYTES + (uint32_t)(j0 >> 3) * 1024;
        auto conv_item = [&](int n) -> bool {
            if (!wait_bar_warp(bars.tk(n % RING), (n / RING) & 1, wc, 20)) return false;
            const int k = slot[n % RING];
            if (k < 0) {
                // the MMA warp meets the end at this item (groups that find the end later arrive
                // on phases no one waits for)
                if (q == 0 && lane == 0) mbar_arrive(bars.conv_done(st));
                return false;
            }
            if (!wait_bar_warp(bars.x_full(st), (n / G) & 1, wc, 10)) return false;
            const int b = k % a.B, c = k / a.B, t0 = c * L;
            const int nt = min(L, a.T - t0);
            const uint8_t* rrow = a.reset ? a.reset + (size_t)b * a.T : nullptr;
            const uint32_t rmask = rrow ? chunk_reset_mask(rrow, t0, a.T, lane) : 0u;
            const bool has_last = nt - 1 >= j0 && nt - 1 < j0 + kConvTok;
            const bool write_tail = !SAVE && a.tail_state && c == a.NC - 1 && has_last && own;
            const uint32_t rm = rmask >> j0;
            const int jlast = nt - 1 - j0;
#pragma unroll 1
            for (int pp = 0; pp < 2; ++pp) {
                // channels cl + 4 p4 .. + 3; lanes of odd K blocks take the halves the other way
                // round, so that lanes 8 apart never meet in a bank
                const int p4 = pp ^ ((lane >> 3) & 1);
                const int chg = head * DH + cl + 4 * p4;  // global channel
                float2 w[kConvWidth][2];
                const float* cwp = reinterpret_cast<const float*>(smem + OFF_CW) + cl + 4 * p4;
#pragma unroll
                for (int k2 = 0; k2 < kConvWidth; ++k2) {
                    const float4 v = *reinterpret_cast<const float4*>(cwp + k2 * DH);
                    w[k2][0] = make_float2(v.x, v.y);
                    w[k2][1] = make_float2(v.z, v.w);
                }
                float2 cb[2];
                {
                    const float4 v = *reinterpret_cast<const float4*>(cwp + kConvWidth * DH);
                    cb[0] = make_float2(v.x, v.y);
                    cb[1] = make_float2(v.z, v.w);
                }
                const uint8_t* xt = smem + OFF_X + st * X_STRIDE + lane * 16 + 8 * p4;
                auto xrow = [&](int r) {                  // x tile row r = token t0 - 3 + r
                    return unpack4(*reinterpret_cast<const uint2*>(xt + r * DH * 2));
                };
                Vec4 h0, h1, h2;                          // window x_{t-3}, x_{t-2}, x_{t-1}
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
                const uint8_t* xtw = xt + j0 * DH * 2;
                uint8_t* bhi = smem + OFF_B + st * B_BYTES + kb_off + 8 * p4;
                float4* xcw = own ? reinterpret_cast<float4*>(smem + OFF_XC + st * XC_BYTES) + j0 * (HALF / 4) +
                                        (((cl & (HALF - 1)) + 4 * p4) >> 2)
                                  : nullptr;
                uint2 fw[3];                              // final window (the tail of the row), bf16
                if ((rm & 0xFFu) == 0 && !has_last)
                    conv_tokens<false, false>(xtw, bhi, xcw, cchunk, rm, jlast, w, cb, h0, h1, h2, fw);
                else
                    conv_tokens<true, true>(xtw, bhi, xcw, cchunk, rm, jlast, w, cb, h0, h1, h2, fw);
                // final conv history of the sequence (this CTA's channels), as soon as the row's
                // last token is convolved: the conv read the copy taken before the launch
                if (write_tail) {
                    __nv_bfloat16* tl = a.tail_state + (size_t)b * kHist * W + chg;
#pragma unroll
                    for (int r = 0; r < kHist; ++r) *reinterpret_cast<uint2*>(tl + (size_t)r * W) = fw[r];
                }
            }
            // the MMA (async proxy) reads what the group wrote; the x tile is free
            fence_proxy_async_smem();
            group_sync(eg);
            if (q == 0 && lane == 0) {
                mbar_arrive(bars.x_empty(st));
                mbar_arrive(bars.conv_done(st));
            }
            return true;
        };

        int n = eg;
        bool have = conv_item(n);
        while (have) {
            const uint32_t ph = (n / G) & 1;
            const int sl = n % kSlots;
            const uint32_t dcol = tmem + lane_off + TM_D + sl * TM_SLOT;
            if (!wait_bar_warp(bars.acc_full(st), ph, wc, 13)) break;
            tc_fence_after();
            const int k = slot[n % RING];
            const int b = k % a.B, c = k / a.B, t0 = c * L;
            const int nt = min(L, a.T - t0);
            const uint8_t* rrow = a.reset ? a.reset + (size_t)b * a.T : nullptr;
            const uint32_t rmask = rrow ? chunk_reset_mask(rrow, t0, a.T, lane) : 0u;
            const size_t kb_item = lb_base + (size_t)b * a.NC;       // first chunk of this row
            const bool withhold = withhold_hook && k == 0;

            // ---- pass 1: gates, decay and normalised input into the TMEM slot, the chunk's
            //      aggregate (prod a over the chunk, its local h)
            float aggA, aggH;
            const size_t e0 = ((size_t)b * a.T + t0) * W + ch;
            if constexpr (SAVE) {
                pass1_save(dcol, xcs, ck, ba, bx, rmask, nt, a, e0, W, aggA, aggH);
            } else if (nt == L && warp_small) {
                if (rmask) pass1<true, false>(dcol, xcs, ck, rmask, nt, aggA, aggH);
                else pass1<false, false>(dcol, xcs, ck, rmask, nt, aggA, aggH);
            } else {
                pass1<true, true>(dcol, xcs, ck, rmask, nt, aggA, aggH);
            }
            if (c > 0 && !withhold)                      // as early as possible
                st_relaxed_gpu_u64(a.lb_agg + (kb_item + c) * HALF + m,
                                   ((uint64_t)__float_as_uint(aggH) << 32) | (__float_as_uint(aggA) | kReadyBit));

            // ---- the conv of the group's next item, while the chunks before this one finish
            //      (the whole group has read this item's xc tile first)
            group_sync(eg);
            const bool have_next = conv_item(n + G);

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
                pass2_save(dcol, carry, rmask, nt, a, e0, W);
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(bars.slot_free(sl));
            } else {
                // ---- pass 2: h_t from the carry, merged with GeLU(y_t)
                if (!wait_bar_warp(bars.y_full(st), ph, wc, 16)) break;
                if (tanh_form) pass2<true>(dcol, yt, carry);
                else pass2<false>(dcol, yt, carry);
                // the TMEM slot is read: the MMA of a later item may overwrite it
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(bars.slot_free(sl));

                // ---- the out tile is complete: the store warp writes it and loads the next y
                fence_proxy_async_smem();
                __syncwarp();
                if (lane == 0) mbar_arrive(bars.out_ready(st));
            }
            n += G;
            have = have_next;
        }
        // no tensor-memory access of this warp may still be in flight when TMEM is released
        tmem_wait_ld();
    } else if (warp == kWarpStore) {
        // ================================ out stores and y loads ==============================
        // one thread serves the three stages: as a stage's item completes its second pass, its
        // out tile goes to global memory by TMA (which clips the ragged tail) and, once the tile
        // has been read, the y tile of the stage's next item comes in -- so that no epilogue
        // warp waits for a store
        if (!SAVE && lane == 0) {
            int nxt[G], kb[G];                           // stage's item and its (row, chunk), or -1
            bool done[G];
            int pending_y[G];                            // item whose y load is in flight, or -1
            auto issue_y = [&](int st, int m) -> bool {  // y of item m into stage st; false: the end
                if (!wait_bar(bars.tk(m % RING), (m / RING) & 1, wc, 30)) return false;
                const int km = slot[m % RING];
                if (km < 0) return false;
                mbar_arrive_expect_tx(bars.y_full(st), Y_BYTES);
                tma_load_3d(sbase + OFF_Y + st * Y_BYTES, &map_y, head * DH + half * HALF, (km / a.B) * L, km % a.B,
                            bars.y_full(st));
                kb[st] = km;
                pending_y[st] = m;
                return true;
            };
            int live = 0;
            for (int st = 0; st < G; ++st) {
                nxt[st] = st;
                pending_y[st] = -1;
                done[st] = !issue_y(st, st);
                live += done[st] ? 0 : 1;
            }
            uint64_t t_last = globaltimer_ns();
            while (live > 0) {
                bool progress = false;
                for (int st = 0; st < G; ++st) {
                    if (done[st]) continue;
                    const int m = nxt[st];
                    if (!mbar_try_wait(bars.out_ready(st), (m / G) & 1)) continue;
                    progress = true;
                    pending_y[st] = -1;                  // its second pass consumed the y tile
                    tma_store_3d(&map_out, sbase + OFF_Y + st * Y_BYTES, head * DH + half * HALF,
                                 (kb[st] / a.B) * L, kb[st] % a.B);
                    bulk_commit();
                    bulk_wait_read0();                   // the tile is free for the next y
                    nxt[st] = m + G;
                    if (!issue_y(st, m + G)) {
                        done[st] = true;
                        --live;
                    }
                }
                if (progress) {
                    t_last = globaltimer_ns();
                } else {
                    __nanosleep(64);
                    if (*abort || *(volatile unsigned*)&a.status->code != 0) break;
                    if (globaltimer_ns() - t_last > a.timeout_ns) {
                        latch_status(a.status, RGLRU_ERR_TIMEOUT, 31, blockIdx.x, (unsigned)live);
                        *abort = 1;
                        break;
                    }
                }
            }
            // no bulk copy may still read or write this CTA's shared memory when it exits
            bulk_wait0();
            const uint64_t t0w = globaltimer_ns();
            for (int st = 0; st < G; ++st)
                if (pending_y[st] >= 0)
                    while (!mbar_try_wait_sleep(bars.y_full(st), (pending_y[st] / G) & 1, 100000u) &&
                           globaltimer_ns() - t0w < a.timeout_ns) {
                    }
        }
    }

    // ---- teardown: all tensor-core work has drained (the MMA warp waited on mma_done) ------
    tc_fence_before();
    __syncthreads();
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
    p.off_agg = up(p.off_counters + groups * 4);
    p.off_incl = up(p.off_agg + groups * p.items * HALF * 8);
    p.off_tail = up(p.off_incl + groups * d->batch * p.NA * HALF * 8);
    p.total = up(p.off_tail + (size_t)d->batch * kHist * d->heads * DH * sizeof(__nv_bfloat16));
    return p;
}

// CTAs that fit on the device at once (1 per SM), looked up once per device.
cudaError_t max_ctas(int dev, int* out) {
    static std::mutex mu;
    static int cache[64] = {};
    if (dev >= 0 && dev < 64) {
        std::lock_guard<std::mutex> lock(mu);
        if (cache[dev] > 0) {
            *out = cache[dev];
            return cudaSuccess;
        }
    }
    int per_sm = 0, sms = 0;
    cudaError_t e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, fused_prefill_kernel<false>, kThreads,
                                                                  SMEM_BYTES);
    if (e != cudaSuccess) return e;
    e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    if (e != cudaSuccess) return e;
    int n = per_sm * sms;
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
    if (!make_map_3d(&mx, x, W, d->seq_len, d->batch, DH, XROWS)) return cudaErrorInvalidValue;
    if (SAVE) {
        my = mx;   // y and out are not touched in the save mode
        mo = mx;
    } else if (!make_map_3d(&my, y, W, d->seq_len, d->batch, HALF, L) ||
               !make_map_3d(&mo, out, W, d->seq_len, d->batch, HALF, L)) {
        return cudaErrorInvalidValue;
    }
    e = set_smem_once(fused_prefill_kernel<SAVE>, (int)SMEM_BYTES);
    if (e != cudaSuccess) return e;
    e = set_smem_once(fused_prefill_kernel<false>, (int)SMEM_BYTES);   // the occupancy query's kernel
    if (e != cudaSuccess) return e;
    int ctas = 0;
    e = max_ctas(dev, &ctas);
    if (e != cudaSuccess) return e;
    // every group (head, half) gets at least one CTA; with more CTAs than groups, all of them stay
    // busy (a CTA only takes a ticket when it is running, so CTAs that wait for an SM are harmless)
    const int groups = 2 * d->heads;
    const int nctas = ctas > groups ? ctas : groups;

    uint8_t* w = static_cast<uint8_t*>(ws);
    Args a{};
    a.B = d->batch; a.T = d->seq_len; a.H = d->heads; a.NC = pl.NC; a.items = pl.items; a.NA = pl.NA;
    a.base = nctas / groups; a.extra = nctas % groups;
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
    cfg.gridDim = dim3(nctas, 1, 1);
    cfg.blockDim = dim3(kThreads, 1, 1);
    cfg.dynamicSmemBytes = SMEM_BYTES;
    cfg.stream = s;
    cfg.attrs = nullptr;
    cfg.numAttrs = 0;
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
