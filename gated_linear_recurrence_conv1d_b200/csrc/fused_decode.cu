// fused_decode.cu -- tensor-core RG-LRU decode step for bf16 activations, head_dim 256 (sm_100a).
//
// A decode step updates every batch row by one token.  There is no recurrence across tokens
// inside a call, so the batch is the parallel dimension and the gate contraction is a plain
// GEMM per head: D[row, o] = sum_i xc[row, i] W[h][i][o] with M = rows, N = output channels,
// K = 256 input channels.  One launch; a cluster of 4 CTAs per (head, 128-row tile), CTA r
// owning the 64 channels [64 r, 64 r + 64) of the head:
//
//   * conv: update thread (row, 16 channels) convolves its channels of CTA r's 64 (the width-4
//     causal conv over the carried history and the new input), shifts their history in place
//     (oldest out, x in; a row with reset[b] set starts from an empty history), keeps the fp32
//     result in its TMEM lane for the state update, and writes it as a bf16 pair -- hi = the
//     fp32 value truncated, lo = the remainder rounded, hi + lo = the value to 2^-16 -- into
//     K-block r of the CTA's two 128 x 256 operand tiles (K-major, 128-byte swizzle); one thread
//     then copies the two 16 KB blocks into the same place of the three sibling CTAs' tiles
//     through distributed shared memory (bulk copies that complete on the siblings' mbarrier),
//     so every channel is convolved once and only by the CTA that owns its history;
//   * gates: TMA brings the 256 x 64 slices W_a[h][:, 64 r], W_x[h][:, 64 r] (bf16 as stored:
//     output channel contiguous, i.e. MN-major for the MMA) side by side, one N = 128 operand;
//     an elected lane of the MMA warp issues tcgen05.mma (M = 128, N = 128, K = 16 each, bf16
//     operands, fp32 accumulation) on both parts of the conv output into TMEM, K block by K
//     block as the blocks become ready (its own first);
//   * update: TMA brings the y tile of the CTA; the update threads compute GeLU(y) while the
//     MMAs run, read their h from global memory, then the accumulators, apply the gates and
//     write h back and out into the shared tile, which TMA stores (rows past the batch are
//     clipped by the tensor map).
//
// The element-wise arithmetic is rglru_math.cuh's (shared with the prefill): gates by ex2 and a
// reciprocal, expm1 of the log-decay by its series near zero, sqrt(1 - a^2) i_t by one rsqrt,
// GeLU by a fitted tail polynomial and one ex2.  Sources ("Griffin Guide: RecurrentGemma, RG-LRU &
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
#include "rglru_math.cuh"
#include "sm100.cuh"
#include "tma_maps.h"

namespace rglru {

namespace dec {

using namespace sm100;
using namespace fm;

constexpr int DH = 256;
constexpr int MT = 128;                 // rows per CTA (MMA M, TMEM lanes)
constexpr int NT = 64;                  // output channels per CTA (MMA N)
constexpr int KSTEPS = DH / 16;
constexpr int kEpiWarps = 16;                 // 4 lane quarters x 4 quarters of the tile's channels
constexpr int kWarpMma = kEpiWarps, kWarpTma = kEpiWarps + 1;
constexpr int kThreads = (kEpiWarps + 2) * 32;
constexpr int kEpiThreads = kEpiWarps * 32;
constexpr int kEpiCh = NT / (kEpiWarps / 4);  // channels per update thread (16)

constexpr uint32_t A_BYTES = MT * DH * 2;            // 65536: 4 K-blocks of 128 rows x 128 B
constexpr uint32_t A_KBLK = MT * 128;                // 16384
constexpr uint32_t B_BYTES = DH * NT * 2;            // 32768 per gate: 256 K-rows x 128 B
constexpr uint32_t Y_BYTES = MT * NT * 2;            // y tile (then out): 128 rows x 64 bf16
constexpr uint32_t OFF_A = 0;                        // conv output, bf16 hi part
constexpr uint32_t OFF_ALO = OFF_A + A_BYTES;        // and lo part (xc - hi)
constexpr uint32_t OFF_BA = OFF_ALO + A_BYTES;
constexpr uint32_t OFF_BX = OFF_BA + B_BYTES;        // right after W_a: one N = 128 operand
// Before the weights arrive, their 64 KB hold the conv's inputs, staged by TMA in the 128-byte
// swizzle: x [128 rows][64 channels] bf16 and the history [128 rows][3][64 channels] bf16.
constexpr uint32_t X_ST_BYTES = MT * NT * 2;          // 16384
constexpr uint32_t OFF_XST = OFF_BA;
constexpr uint32_t OFF_TST = OFF_BA + X_ST_BYTES;     // 49152 bytes of history
static_assert(X_ST_BYTES * (1 + kHist) == 2 * B_BYTES, "staging fills the weight tile");
constexpr uint32_t OFF_Y = OFF_BX + B_BYTES;
constexpr uint32_t OFF_CONST = OFF_Y + Y_BYTES;      // K, -b_a log2 e, -b_x log2 e per channel: 3 x 64 fp32
constexpr uint32_t OFF_CONV = OFF_CONST + 3 * NT * 4; // conv taps [4][64] and bias [64], fp32
constexpr uint32_t OFF_BAR = OFF_CONV + 5 * NT * 4;
constexpr uint32_t OFF_MISC = OFF_BAR + 72;
constexpr int kClusterSize = DH / NT;                 // CTAs of a (head, row tile)
constexpr uint32_t SMEM_BYTES = OFF_MISC + 32 + 1024;
static_assert(SMEM_BYTES <= 232448, "shared memory budget");
// TMEM: D_a [0,64), D_x [64,128), the fp32 conv output [128,192) (lane = row)
constexpr uint32_t TMEM_COLS = 256;
constexpr uint32_t TM_XC = 2 * NT;

struct Args {
    int B, H, mtiles;
    float* h;                         // [B][W] state, read and written in place
    const __nv_bfloat16* x;
    __nv_bfloat16* tail;
    const float* conv_w;
    const float* conv_b;
    float c;
    int gelu_tanh;
    int withhold;                     // test hook: CTA 0 keeps its conv block from its siblings
    unsigned long long timeout_ns;
    const float* b_a;
    const float* b_x;
    const float* lambda;
    const uint8_t* reset;
    DeviceStatus* status;
};

__device__ __forceinline__ float bf16lo(uint32_t v) { return __uint_as_float(v << 16); }
__device__ __forceinline__ float bf16hi(uint32_t v) { return __uint_as_float(v & 0xFFFF0000u); }
__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
    __nv_bfloat162 p = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t*>(&p);
}
// bf16 hi part (truncation) of two fp32 values, packed; the remainder v - hi is exact in fp32
__device__ __forceinline__ uint32_t trunc_bf16x2(float lo, float hi) {
    return __byte_perm(__float_as_uint(lo), __float_as_uint(hi), 0x7632);
}

// Shared-memory matrix descriptor for an MN-major operand in the 128-byte swizzle layout: rows
// of 128 B (64 bf16 along N) for consecutive K, 8-row atoms of 1024 B stacked along K at the
// stride byte offset (1024 B); the leading byte offset is the distance between 64-wide N atoms,
// here from the W_a slice to the W_x slice, so that one N = 128 operand covers both gates.
// Same bit fields as desc_k_sw128.
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
    return (1u << 4) | (1u << 7) | (1u << 10) | (1u << 16) | ((uint32_t)(N >> 3) << 17) | ((uint32_t)(M >> 4) << 24);
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

// 16-byte chunk c of line l of a tile in the 128-byte swizzle
__device__ __forceinline__ uint32_t sw128(uint32_t l, uint32_t c) { return l * 128 + ((c ^ (l & 7)) << 4); }

__global__ void __launch_bounds__(kThreads, 1)
decode_fused_kernel(const __grid_constant__ CUtensorMap map_wa, const __grid_constant__ CUtensorMap map_wx,
                    const __grid_constant__ CUtensorMap map_y, const __grid_constant__ CUtensorMap map_out,
                    const __grid_constant__ CUtensorMap map_x, const __grid_constant__ CUtensorMap map_tail,
                    const __grid_constant__ CUtensorMap map_h, const Args a) {
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const uint32_t sbase = smem_u32(smem);
    const uint32_t bar_w = sbase + OFF_BAR, bar_acc = sbase + OFF_BAR + 16;
    const uint32_t bar_y = sbase + OFF_BAR + 24;      // y tile
    const uint32_t bar_x = sbase + OFF_BAR + 8;       // the conv's staged inputs
    const uint32_t bar_st = sbase + OFF_BAR + 64;     // the staging has been read: the weights may come
    // K block j of the operand tile: convolved here (j = rank) or copied in by CTA j
    auto bar_k = [&](int j) { return sbase + OFF_BAR + 32 + 8 * (uint32_t)j; };
    volatile uint32_t* tmem_base_s = reinterpret_cast<volatile uint32_t*>(smem + OFF_MISC);
    volatile int* abort = reinterpret_cast<volatile int*>(smem + OFF_MISC + 16);
    float* s_K = reinterpret_cast<float*>(smem + OFF_CONST);
    float* s_nba = s_K + NT;
    float* s_nbx = s_nba + NT;
    float* s_cw = reinterpret_cast<float*>(smem + OFF_CONV);   // [4][64]
    float* s_cb = s_cw + 4 * NT;                                 // [64]

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    // cluster = (head, row tile); rank = channel tile (blockIdx.x = (head * mtiles + mt) * 4 + rank)
    const int nt = (int)cluster_ctarank();
    const int mt = (blockIdx.x / kClusterSize) % a.mtiles;
    const int head = blockIdx.x / (kClusterSize * a.mtiles);
    const int W = a.H * DH;
    const int ch0 = head * DH + nt * NT;                  // first global channel of the tile

    // let the next step's CTAs start their set-up; they read nothing of ours before their wait
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    if (threadIdx.x == 0) {
        mbar_init(bar_w, 1);
        mbar_init(bar_x, 1);
        mbar_init(bar_st, 1);
        mbar_init(bar_acc, 1);
        mbar_init(bar_y, 1);
        for (int j = 0; j < kClusterSize; ++j) mbar_init(bar_k(j), 1);
        *abort = 0;
        fence_barrier_init();
        for (int j = 0; j < kClusterSize; ++j)
            if (j != nt) mbar_arrive_expect_tx(bar_k(j), 2 * A_KBLK);   // completed by CTA j's copies
    }
    if (warp == kWarpMma) {
        tmem_alloc(smem_u32((const void*)tmem_base_s), TMEM_COLS);
        tmem_relinquish();
    }
    if (warp == kWarpTma && lane == 0) {
        prefetch_tensormap(&map_wa);
        prefetch_tensormap(&map_wx);
        prefetch_tensormap(&map_y);
        prefetch_tensormap(&map_out);
        prefetch_tensormap(&map_x);
        prefetch_tensormap(&map_tail);
        prefetch_tensormap(&map_h);
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_base_s;
    // every CTA of the cluster has initialised its barriers before any copy targets them
    cluster_sync();
    // everything above overlaps the previous kernel of the stream; global memory only from here
    asm volatile("griddepcontrol.wait;" ::: "memory");

    if (warp == kWarpTma) {
        if (lane == 0) {
            // the conv's inputs of this tile (rows past the batch read as zeros), then its y
            mbar_arrive_expect_tx(bar_x, (1 + kHist) * X_ST_BYTES);
            tma_load_2d(sbase + OFF_XST, &map_x, ch0, mt * MT, bar_x);
            tma_load_3d(sbase + OFF_TST, &map_tail, ch0, 0, mt * MT, bar_x);
            mbar_arrive_expect_tx(bar_y, Y_BYTES);
            tma_load_2d(sbase + OFF_Y, &map_y, ch0, mt * MT, bar_y);
            // the weights, into the staging area once the conv has read it
            const uint64_t t0 = globaltimer_ns();
            bool staged = false;
            while (!(staged = mbar_try_wait_sleep(bar_st, 0, 20000u)) && globaltimer_ns() - t0 < a.timeout_ns) {
            }
            if (staged) {
                mbar_arrive_expect_tx(bar_w, 2 * B_BYTES);
                for (int kb = 0; kb < DH / 64; ++kb) {
                    tma_load_2d(sbase + OFF_BA + kb * 8192, &map_wa, nt * NT, head * DH + kb * 64, bar_w);
                    tma_load_2d(sbase + OFF_BX + kb * 8192, &map_wx, nt * NT, head * DH + kb * 64, bar_w);
                }
            }
            // never leave the CTA with a bulk copy still writing its shared memory (the staged
            // inputs, the weight tiles, or a sibling's conv block, whose completion also ends the
            // sibling's reads)
            while (!mbar_try_wait_sleep(bar_x, 0, 20000u) && globaltimer_ns() - t0 < a.timeout_ns) {
            }
            while (staged && !mbar_try_wait_sleep(bar_w, 0, 20000u) && globaltimer_ns() - t0 < a.timeout_ns) {
            }
            for (int j = 0; j < kClusterSize; ++j)
                while (!mbar_try_wait_sleep(bar_k(j), 0, 20000u) && globaltimer_ns() - t0 < a.timeout_ns) {
                }
            while (!mbar_try_wait_sleep(bar_y, 0, 20000u) && globaltimer_ns() - t0 < a.timeout_ns) {
            }
        }
    } else if (warp == kWarpMma) {
        // the whole warp follows the waits; one elected lane issues (warp-uniform operands)
        const uint32_t idesc = idesc_bf16_f32_bmn(MT, 2 * NT);   // D_a | D_x
        const uint32_t tm = __shfl_sync(0xffffffffu, tmem, 0);
        // K blocks in the order they become ready: this CTA's own first, then the siblings'
        // (CTA j sends its block to j + 1, j + 2, j + 3 in turn, so CTA nt - 1's arrives first)
        bool ok = __all_sync(0xffffffffu, wait_bounded(bar_w, 0, a, abort, 1));
        uint32_t accum = 0;
        for (int i = 0; i < kClusterSize && ok; ++i) {
            const int j = (nt - i + kClusterSize) % kClusterSize;
            ok = __all_sync(0xffffffffu, wait_bounded(bar_k(j), 0, a, abort, 3));
            if (!ok) break;
            tc_fence_after();
            if (elect_one()) {
#pragma unroll
                for (int part = 0; part < 2; ++part)          // the conv output's hi and lo parts
#pragma unroll
                    for (int kk = 0; kk < KSTEPS / kClusterSize; ++kk) {
                        const int ks = j * 4 + kk;
                        const uint64_t ad = desc_k_sw128(sbase + (part ? OFF_ALO : OFF_A) + j * A_KBLK + kk * 32);
                        const uint64_t bd = desc_mn_sw128(sbase + OFF_BA + ks * 16 * 128);
                        mma_ss(tm, ad, bd, idesc, (accum | (uint32_t)kk | (uint32_t)part) ? 1u : 0u);
                    }
            }
            __syncwarp();
            accum = 1;
        }
        if (elect_one()) mma_commit(bar_acc);     // also when a wait failed: the update must not wait forever
        __syncwarp();
        // every MMA issued here has completed before TMEM can be released (bounded by time only,
        // so that an aborted step still drains its tensor-core work)
        if (lane == 0) {
            const uint64_t t0 = globaltimer_ns();
            while (!mbar_try_wait_sleep(bar_acc, 0, 20000u) && globaltimer_ns() - t0 < a.timeout_ns) {
            }
        }
        __syncwarp();
    } else {
        // ================================ update threads =======================================
        // thread = row r of the tile (= TMEM lane r), channels [16 cg, 16 cg + 16) of its 64: it
        // convolves them, keeps their fp32 conv output in its TMEM lane, and later updates them
        const int q = warp & 3, cg = warp >> 2;           // lane quarter, channel quarter of the tile
        const int r = q * 32 + lane;                      // row within the tile
        const int b = mt * MT + r;
        const bool live = b < a.B;
        const int bs = live ? b : 0;                      // rows past the batch: any valid row
        const uint32_t sw = (uint32_t)(r & 7);
        const int cbase = ch0 + cg * kEpiCh;
        const uint32_t lane_off = (uint32_t)(q * 32) << 16;
        const uint32_t xcol = tmem + lane_off + TM_XC + cg * kEpiCh;
        if (threadIdx.x < NT) {                           // per-channel constants
            // every load first: a shared-memory store between two of them would order them
            const int ch = ch0 + threadIdx.x;
            const float lam = a.lambda[ch];
            const float ba = a.b_a ? a.b_a[ch] : 0.f;
            const float bx = a.b_x ? a.b_x[ch] : 0.f;
            const float cb0 = a.conv_b ? a.conv_b[ch] : 0.f;
            float cwv[kConvWidth];
#pragma unroll
            for (int k = 0; k < kConvWidth; ++k) cwv[k] = a.conv_w[(size_t)k * W + ch];
#pragma unroll
            for (int k = 0; k < kConvWidth; ++k) s_cw[k * NT + threadIdx.x] = cwv[k];
            s_cb[threadIdx.x] = cb0;
            s_K[threadIdx.x] = a.c * log_sigmoid_acc(lam);
            s_nba[threadIdx.x] = -ba * kLog2e;
            s_nbx[threadIdx.x] = -bx * kLog2e;
        }
        const bool rst = live && a.reset && a.reset[b];
        // the conv's inputs from the staged tiles: x and the three past inputs of this thread's
        // row and 16 channels (16-byte chunks 2 cg, 2 cg + 1 of their 128-byte lines)
        const bool ok_x = wait_bounded(bar_x, 0, a, abort, 6);
        uint4 xv[2], t0[2], t1[2], t2[2];
#pragma unroll
        for (int v = 0; v < 2; ++v) {
            const uint32_t c = (uint32_t)(2 * cg + v);
            xv[v] = *reinterpret_cast<const uint4*>(smem + OFF_XST + sw128((uint32_t)r, c));
            t0[v] = *reinterpret_cast<const uint4*>(smem + OFF_TST + sw128((uint32_t)(r * kHist + 0), c));
            t1[v] = *reinterpret_cast<const uint4*>(smem + OFF_TST + sw128((uint32_t)(r * kHist + 1), c));
            t2[v] = *reinterpret_cast<const uint4*>(smem + OFF_TST + sw128((uint32_t)(r * kHist + 2), c));
        }
        asm volatile("bar.sync 1, %0;" ::"n"(kEpiThreads) : "memory");
        if (rst) {                                        // an empty history
#pragma unroll
            for (int v = 0; v < 2; ++v) t0[v] = t1[v] = t2[v] = make_uint4(0, 0, 0, 0);
        }
        // the new history (oldest out, x in) over the staged one, stored by TMA after the conv
#pragma unroll
        for (int v = 0; v < 2; ++v) {
            const uint32_t c = (uint32_t)(2 * cg + v);
            *reinterpret_cast<uint4*>(smem + OFF_TST + sw128((uint32_t)(r * kHist + 0), c)) = t1[v];
            *reinterpret_cast<uint4*>(smem + OFF_TST + sw128((uint32_t)(r * kHist + 1), c)) = t2[v];
            *reinterpret_cast<uint4*>(smem + OFF_TST + sw128((uint32_t)(r * kHist + 2), c)) = xv[v];
        }

        // ================================ conv of this CTA's channels ==========================
        {
            const float* cwp = s_cw + cg * kEpiCh;
            const float* cbp = s_cb + cg * kEpiCh;
#pragma unroll
            for (int v = 0; v < 2; ++v) {
                const uint32_t* px = reinterpret_cast<const uint32_t*>(&xv[v]);
                const uint32_t* p0 = reinterpret_cast<const uint32_t*>(&t0[v]);
                const uint32_t* p1 = reinterpret_cast<const uint32_t*>(&t1[v]);
                const uint32_t* p2 = reinterpret_cast<const uint32_t*>(&t2[v]);
                uint32_t ohi[4], olo[4], xo[8];
#pragma unroll
                for (int e2 = 0; e2 < 4; ++e2) {
                    float rr[2];
#pragma unroll
                    for (int e1 = 0; e1 < 2; ++e1) {
                        const int j = v * 8 + 2 * e2 + e1;
                        const float v0 = e1 ? bf16hi(p0[e2]) : bf16lo(p0[e2]);
                        const float v1 = e1 ? bf16hi(p1[e2]) : bf16lo(p1[e2]);
                        const float v2 = e1 ? bf16hi(p2[e2]) : bf16lo(p2[e2]);
                        const float v3 = e1 ? bf16hi(px[e2]) : bf16lo(px[e2]);
                        float acc = fmaf(cwp[j], v0, cbp[j]);
                        acc = fmaf(cwp[NT + j], v1, acc);
                        acc = fmaf(cwp[2 * NT + j], v2, acc);
                        acc = fmaf(cwp[3 * NT + j], v3, acc);
                        rr[e1] = acc;
                        xo[2 * e2 + e1] = __float_as_uint(acc);
                    }
                    ohi[e2] = trunc_bf16x2(rr[0], rr[1]);
                    olo[e2] = pack_bf16x2(rr[0] - bf16lo(ohi[e2]), rr[1] - bf16hi(ohi[e2]));
                }
                // row r, 16-byte chunk (2 cg + v) of this CTA's K block (128-byte swizzle)
                const uint32_t so = nt * A_KBLK + (uint32_t)(r >> 3) * 1024 + sw * 128 + ((((uint32_t)(cg * 2 + v)) ^ sw) << 4);
                *reinterpret_cast<uint4*>(smem + OFF_A + so) = make_uint4(ohi[0], ohi[1], ohi[2], ohi[3]);
                *reinterpret_cast<uint4*>(smem + OFF_ALO + so) = make_uint4(olo[0], olo[1], olo[2], olo[3]);
                tmem_st8(xcol + v * 8, xo);
            }
            tmem_wait_st();
            // the blocks are complete: make them visible to the tensor core and the bulk copies,
            // then hand them to this CTA's MMA and to the three siblings
            fence_proxy_async_smem();
            asm volatile("bar.sync 1, %0;" ::"n"(kEpiThreads) : "memory");
            if (threadIdx.x == 0) {
                mbar_arrive(bar_k(nt));
                for (int rk = 1; rk < kClusterSize && !(a.withhold && blockIdx.x == 0); ++rk) {
                    const uint32_t peer = (uint32_t)((nt + rk) % kClusterSize);
#pragma unroll
                    for (int part = 0; part < 2; ++part) {
                        const uint32_t blk = sbase + (part ? OFF_ALO : OFF_A) + nt * A_KBLK;
                        dsmem_copy(map_to_rank(blk, peer), blk, A_KBLK, map_to_rank(bar_k(nt), peer));
                    }
                }
                // the new history of the tile's rows (rows past the batch are clipped); once the
                // store has read the staging area, the weights may take its place
                if (ok_x && !*abort) {
                    tma_store_3d(&map_tail, sbase + OFF_TST, ch0, 0, mt * MT);
                    bulk_commit();
                    bulk_wait_read0();
                }
                mbar_arrive(bar_st);
            }
        }

        // ================================ update ===============================================
        // the state of this thread's row and channels (its latency overlaps the exchange)
        float hv[kEpiCh];
        {
            const float4* hp = reinterpret_cast<const float4*>(a.h + (size_t)bs * W + cbase);
#pragma unroll
            for (int i = 0; i < kEpiCh / 4; ++i) {
                const float4 v = hp[i];
                hv[4 * i] = v.x; hv[4 * i + 1] = v.y; hv[4 * i + 2] = v.z; hv[4 * i + 3] = v.w;
            }
        }
        // GeLU(y) while the siblings' blocks arrive and the tensor cores run
        const bool ok_y = __all_sync(0xffffffffu, wait_bounded(bar_y, 0, a, abort, 4));
        float gg[kEpiCh];
#pragma unroll
        for (int v = 0; v < kEpiCh / 8; ++v) {
            const uint4 yq = *reinterpret_cast<const uint4*>(smem + OFF_Y + (uint32_t)r * 128 +
                                                             ((((uint32_t)(cg * 2 + v)) ^ sw) << 4));
            const uint32_t* yw = reinterpret_cast<const uint32_t*>(&yq);
#pragma unroll
            for (int e = 0; e < 8; ++e)
                gg[v * 8 + e] = gelu1((e & 1) ? bf16hi(yw[e >> 1]) : bf16lo(yw[e >> 1]), a.gelu_tanh);
        }
        if (rst) {                                        // the state restarts from zero
#pragma unroll
            for (int i = 0; i < kEpiCh; ++i) hv[i] = 0.f;
        }
        // uniform across the warp: the TMEM loads below are warp-collective
        const bool acc_ok = wait_bounded(bar_acc, 0, a, abort, 2);
        const bool ok = __all_sync(0xffffffffu, ok_x && ok_y && acc_ok);
        tc_fence_after();
        const uint32_t taddr = tmem + lane_off + cg * kEpiCh;
#pragma unroll
        for (int v = 0; v < kEpiCh / 8; ++v) {            // 8 channels per step
            float ga[8], gx[8], xc[8];
            tmem_ld8(taddr + v * 8, ga);
            tmem_ld8(taddr + NT + v * 8, gx);
            tmem_ld8(xcol + v * 8, xc);
            tmem_wait_ld();
            if (!ok) continue;
            const int c8 = cg * 2 + v;                    // 8-channel chunk of the tile
            const uint32_t yo = OFF_Y + (uint32_t)r * 128 + (((uint32_t)c8 ^ sw) << 4);   // out, in the place of y
            uint32_t ow[4];
#pragma unroll
            for (int e2 = 0; e2 < 4; ++e2) {
                const int e = 2 * e2;
                const int jc = c8 * 8 + e;                // column within the tile (even)
                float2 at, u;
                gates2<false>(make_float2(ga[e], ga[e + 1]), make_float2(gx[e], gx[e + 1]),
                              *reinterpret_cast<const float2*>(s_nba + jc), *reinterpret_cast<const float2*>(s_nbx + jc),
                              *reinterpret_cast<const float2*>(s_K + jc), make_float2(xc[e], xc[e + 1]), at, u);
                const float2 hn = fma2(at, make_float2(hv[v * 8 + e], hv[v * 8 + e + 1]), u);
                hv[v * 8 + e] = hn.x;
                hv[v * 8 + e + 1] = hn.y;
                const float2 o = mul2(hn, make_float2(gg[v * 8 + e], gg[v * 8 + e + 1]));
                ow[e2] = pack_bf16x2(o.x, o.y);
            }
            *reinterpret_cast<uint4*>(smem + yo) = make_uint4(ow[0], ow[1], ow[2], ow[3]);
        }
        // the state into the operand tile's space (the MMAs that read it are done): two boxes
        // of [128 rows x 32 channels] fp32 in the 128-byte swizzle, box cg / 2, chunks
        // 4 (cg % 2) .. 4 (cg % 2) + 3 of the row's line
#pragma unroll
        for (int i = 0; i < kEpiCh / 4; ++i)
            *reinterpret_cast<float4*>(smem + OFF_A + (uint32_t)(cg >> 1) * (MT * 128) +
                                       sw128((uint32_t)r, (uint32_t)(4 * (cg & 1) + i))) =
                make_float4(hv[4 * i], hv[4 * i + 1], hv[4 * i + 2], hv[4 * i + 3]);
        // the out and state tiles are complete: store them (rows past the batch are clipped)
        fence_proxy_async_smem();
        asm volatile("bar.sync 1, %0;" ::"n"(kEpiThreads) : "memory");
        if (threadIdx.x == 0) {
            if (!*abort) {                                // (every failed wait has set it)
                tma_store_2d(&map_out, sbase + OFF_Y, ch0, mt * MT);
                tma_store_2d(&map_h, sbase + OFF_A, ch0, mt * MT);
                tma_store_2d(&map_h, sbase + OFF_A + MT * 128, ch0 + NT / 2, mt * MT);
                bulk_commit();
            }
            bulk_wait0();                                 // every store of this CTA has completed
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == kWarpMma) {
        tc_fence_after();
        tmem_dealloc(tmem, TMEM_COLS);
    }
    // no CTA leaves while a sibling's copy may still read its shared memory or write into it
    cluster_sync();
}

}  // namespace dec

bool fused_decode_supported(const rglru_dims* d) {
    return d->act_dtype == RGLRU_BF16 && d->head_dim == dec::DH && !(d->flags & RGLRU_FLAG_GENERIC);
}

size_t fused_decode_workspace(const rglru_dims* d) {
    (void)d;
    return 256;   // the status word
}

int fused_decode_launches(const rglru_dims* d) {
    (void)d;
    return 1;
}

cudaError_t launch_fused_decode(const rglru_dims* d, const rglru_params* p, const void* x, const void* y,
                                const uint8_t* reset, rglru_state* st, void* out, void* ws, size_t ws_bytes,
                                cudaStream_t s) {
    using namespace dec;
    if (fused_decode_workspace(d) > ws_bytes) return cudaErrorInvalidValue;
    const int B = d->batch, H = d->heads;
    const uint64_t W = (uint64_t)H * DH;
    CUtensorMap mwa, mwx, my, mo, mx, mt, mh;
    if (!tc::make_map_2d_sw128(&mx, x, W, (uint64_t)B, W * 2, NT, MT) ||
        !tc::make_map_2d_sw128_elem(&mh, st->h, 4, W, (uint64_t)B, W * 4, NT / 2, MT) ||
        !tc::make_map_3d_box_sw128(&mt, st->conv_tail, W, kHist, (uint64_t)B, NT, kHist, MT) ||
        !tc::make_map_2d_sw128(&mwa, p->w_a, DH, W, DH * 2, NT, 64) ||
        !tc::make_map_2d_sw128(&mwx, p->w_x, DH, W, DH * 2, NT, 64) ||
        !tc::make_map_2d_sw128_elem(&my, y, 2, W, (uint64_t)B, W * 2, NT, MT) ||
        !tc::make_map_2d_sw128_elem(&mo, out, 2, W, (uint64_t)B, W * 2, NT, MT))
        return cudaErrorInvalidValue;
    cudaError_t e = set_smem_once(decode_fused_kernel, (int)SMEM_BYTES);
    if (e != cudaSuccess) return e;
    Args a;
    a.B = B; a.H = H; a.mtiles = (B + MT - 1) / MT;
    a.h = st->h;
    a.x = static_cast<const __nv_bfloat16*>(x);
    a.tail = static_cast<__nv_bfloat16*>(st->conv_tail);
    a.conv_w = p->conv_w; a.conv_b = p->conv_b;
    a.c = d->c; a.gelu_tanh = d->gelu_tanh;
    a.withhold = (d->flags & RGLRU_FLAG_TEST_WITHHOLD) != 0;
    a.timeout_ns = a.withhold ? 2000000ull : 1000000000ull;
    a.b_a = p->b_a; a.b_x = p->b_x; a.lambda = p->lambda; a.reset = reset;
    a.status = reinterpret_cast<DeviceStatus*>(ws);
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)(H * a.mtiles * kClusterSize));
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = SMEM_BYTES;
    cfg.stream = s;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = kClusterSize;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    // the set-up of this step may overlap the tail of the stream's previous kernel
    attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[1].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 2;
    e = cudaLaunchKernelEx(&cfg, decode_fused_kernel, mwa, mwx, my, mo, mx, mt, mh, a);
    if (e != cudaSuccess) return e;
    return cudaGetLastError();
}

}  // namespace rglru
