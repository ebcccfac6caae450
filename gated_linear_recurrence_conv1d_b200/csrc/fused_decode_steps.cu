// fused_decode_steps.cu -- persistent multi-step RG-LRU decode for bf16 activations, head_dim 256
// (sm_100a): S successive single-token steps of every row in one launch, the state on chip.
//
// The decode step of fused_decode.cu, run for S steps by one persistent kernel:
//
//   * a cluster of 4 CTAs per (head, 128-row tile), CTA r owning the 64 channels [64 r, 64 r + 64)
//     of the head, for the whole launch.  The gate-weight slices W_a[h][:, 64 r], W_x[h][:, 64 r]
//     are loaded into shared memory once and converted there to fp16 (exact for 2^-14 <= |w| <
//     65504);
//   * a thread owns one row (its TMEM lane) and 16 of the CTA's channels: their state h (fp32)
//     stays in registers from the first step to the last, their conv history (the last three x
//     inputs, bf16) and the fp32 conv output of a step in its TMEM lane, so the state never goes
//     back to HBM between steps -- per step only x, y and out move (6 bytes per row-channel);
//     x is read straight into registers two steps ahead, y arrives by TMA, out leaves by TMA;
//   * per step: the conv of step s + 1 is written as K-block r of the CTA's two 128 x 256 fp16
//     operand tiles (the conv output's hi part and its residue lo = xc - hi) and copied into the
//     three siblings' tiles through distributed shared memory; an elected lane of the MMA warp
//     issues tcgen05.mma (M = 128 rows, N = 64 channels x 2 gates, K = 256, both parts) into one
//     of two TMEM accumulators; the update of step s reads the other accumulator, so that the
//     conv, the exchange and the MMAs of step s + 1 overlap the update of step s.  The operand
//     tiles are rewritten only once all four MMAs of the cluster that read them are done (their
//     commits arrive on every CTA of the cluster);
//   * continuous batching: reset[s][b] != 0 empties row b's state (h and history) before step s,
//     so a slot can start a new sequence at any step.
//
// The element-wise arithmetic is rglru_math.cuh's, as in the single step and the prefill; the
// conv output entering the update stays fp32.  Sources ("Griffin Guide: RecurrentGemma, RG-LRU &
// Hybrid Attention"): "1. Formulation of the RG-LRU Gating Mechanism", "2. The Role of
// Square-Root Variance Normalization", "1. Temporal Filtering via Separable 1D Convolutions",
// "2. Non-Linear Multiplicative Gating with GeLU", the listing's RGLRU.step (one token, state in
// and out) and the decode-latency chart of "Production Benchmarks" (a recurrent state of fixed
// size per sequence).
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "common.cuh"
#include "kernels.h"
#include "rglru_math.cuh"
#include "sm100.cuh"
#include "tma_maps.h"

namespace rglru {
namespace dms {

using namespace sm100;
using namespace fm;

constexpr int DH = 256;
constexpr int MT = 128;                       // rows per CTA (MMA M, TMEM lanes)
constexpr int NT = 64;                        // output channels per CTA
constexpr int kCluster = DH / NT;             // 4 CTAs per (head, row tile)
constexpr int KSTEPS = DH / 16;
constexpr int kUpdWarps = 16;                 // 4 lane quarters x 4 channel quarters
constexpr int kUpdThreads = kUpdWarps * 32;
constexpr int kWarpMma = kUpdWarps, kWarpTma = kUpdWarps + 1;
constexpr int kThreads = (kUpdWarps + 2) * 32;
constexpr int kCh = NT / (kUpdWarps / 4);     // channels per thread (16)
constexpr int NBUF = 2;                       // TMEM accumulators and conv-output buffers

constexpr uint32_t A_KBLK = MT * 128;         // 16384: one 64-channel K block of the operand
constexpr uint32_t A_BYTES = 4 * A_KBLK;
constexpr uint32_t W_BYTES = DH * NT * 2;     // 32768 per gate: 256 K-rows x 128 B (MN-major)
constexpr uint32_t T_BYTES = MT * NT * 2;     // 16384: the y (then out) tile [128 rows x 64 ch], 128B swizzle
constexpr uint32_t OFF_A = 0;                 // conv output, fp16 hi part
constexpr uint32_t OFF_ALO = OFF_A + A_BYTES; // and its lo part
constexpr uint32_t OFF_WA = OFF_ALO + A_BYTES;
constexpr uint32_t OFF_WX = OFF_WA + W_BYTES;          // right after W_a: one N = 128 operand
constexpr uint32_t OFF_Y = OFF_WX + W_BYTES;
constexpr uint32_t OFF_CONST = OFF_Y + T_BYTES;        // K, -b_a log2 e, -b_x log2 e, conv w [4], conv b: 8 x 64 fp32
constexpr uint32_t OFF_BAR = OFF_CONST + 8 * NT * 4;
constexpr int NBAR = 16;
constexpr uint32_t OFF_MISC = OFF_BAR + NBAR * 8;
constexpr uint32_t SMEM_BYTES = OFF_MISC + 32 + 1024;
static_assert(SMEM_BYTES <= 232448, "shared memory budget");
// TMEM: two accumulators of D_a [0,64) | D_x [64,128); the fp32 conv outputs of two steps
// (64 columns each); the conv history, 24 columns (3 rows x 8 words of bf16 pairs) per channel
// quarter
constexpr uint32_t TMEM_COLS = 512;
constexpr uint32_t TM_XC = NBUF * (2 * NT);
constexpr uint32_t TM_HIST = TM_XC + NBUF * NT;
static_assert(TM_HIST + 4 * 24 <= TMEM_COLS, "TMEM budget");

struct Args {
    int B, H, mtiles, S;
    const __nv_bfloat16* x;           // [S][B][W]
    const float* conv_w;
    const float* conv_b;
    float c;
    int gelu_tanh;
    unsigned long long timeout_ns;
    const float* b_a;
    const float* b_x;
    const float* lambda;
    const uint8_t* reset;             // [S][B] or nullptr
    float* h;                         // [B][W] in / out
    __nv_bfloat16* tail;              // [B][3][W] in / out
    DeviceStatus* status;
};

// barriers: w (bf16 weights landed), w16 (converted), y_full, y_empty, k[4] (K-block j of the
// operand tiles for the current step), own (this CTA's blocks written), a_free (all four MMAs of
// a step done), acc_full[2], acc_empty[2], mma_done
struct Bars {
    uint32_t base;
    __device__ __forceinline__ uint32_t w() const { return base; }
    __device__ __forceinline__ uint32_t w16() const { return base + 8u; }
    __device__ __forceinline__ uint32_t y_full() const { return base + 16u; }
    __device__ __forceinline__ uint32_t y_empty() const { return base + 24u; }
    __device__ __forceinline__ uint32_t k(int j) const { return base + 8u * (4 + j); }
    __device__ __forceinline__ uint32_t own() const { return base + 8u * 8; }
    __device__ __forceinline__ uint32_t a_free() const { return base + 8u * 9; }
    __device__ __forceinline__ uint32_t acc_full(int i) const { return base + 8u * (10 + i); }
    __device__ __forceinline__ uint32_t acc_empty(int i) const { return base + 8u * (12 + i); }
    __device__ __forceinline__ uint32_t mma_done() const { return base + 8u * 14; }
};

// AND of `p` over the update threads (named barrier 1): they leave the step loop together, so
// that none of them waits at the step's closing barrier for one that has gone
__device__ __forceinline__ bool upd_all(bool p) {
    uint32_t r;
    asm volatile(
        "{\n\t.reg .pred pi, po;\n\t"
        "setp.ne.u32 pi, %1, 0;\n\t"
        "bar.red.and.pred po, 1, %2, pi;\n\t"
        "selp.u32 %0, 1, 0, po;\n\t}"
        : "=r"(r)
        : "r"((uint32_t)p), "n"(kUpdThreads)
        : "memory");
    return r != 0;
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

// TMEM 32x32b loads / stores of raw 32-bit words
__device__ __forceinline__ void tmem_ld8u(uint32_t taddr, uint32_t (&r)[8]) {
    asm volatile("tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0, %1, %2, %3, %4, %5, %6, %7}, [%8];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7])
                 : "r"(taddr)
                 : "memory");
}

// Shared-memory descriptor of the MN-major weight operand (128-byte swizzle): rows of 128 B (64
// values along N) for consecutive K, 8-row atoms of 1024 B along K; the leading byte offset jumps
// from the W_a slice to the W_x slice so that one N = 128 operand covers both gates.
__device__ __forceinline__ uint64_t desc_mn_sw128(uint32_t smem_addr) {
    uint64_t d = 0;
    d |= (uint64_t)((smem_addr >> 4) & 0x3FFF);
    d |= (uint64_t)(W_BYTES >> 4) << 16;
    d |= (uint64_t)(1024 >> 4) << 32;
    d |= (uint64_t)1 << 46;
    d |= (uint64_t)2 << 61;
    return d;
}
// fp32 accumulator, fp16 A (K-major) and B (MN-major), M x N
__host__ __device__ constexpr uint32_t idesc_bmn(int M, int N) {
    return (1u << 4) | (1u << 16) | ((uint32_t)(N >> 3) << 17) | ((uint32_t)(M >> 4) << 24);
}

__device__ __noinline__ bool wait_slow(uint32_t bar, uint32_t parity, const Args& a, volatile int* abort, unsigned where,
                                       bool cluster) {
    const uint64_t t0 = globaltimer_ns();
    for (;;) {
        if (cluster ? mbar_try_wait_cluster(bar, parity) : mbar_try_wait_sleep(bar, parity, 20000u)) return true;
        if (*abort) return false;
        if (*(volatile unsigned*)&a.status->code != 0) {
            *abort = 1;
            return false;
        }
        if (globaltimer_ns() - t0 > a.timeout_ns) {
            latch_status(a.status, RGLRU_ERR_TIMEOUT, where, blockIdx.x, parity);
            *abort = 1;
            return false;
        }
        if (cluster) __nanosleep(128);
    }
}
__device__ __forceinline__ bool wait_b(uint32_t bar, uint32_t parity, const Args& a, volatile int* abort, unsigned where) {
    if (mbar_try_wait(bar, parity)) return true;
    return wait_slow(bar, parity, a, abort, where, false);
}
__device__ __forceinline__ bool wait_cl(uint32_t bar, uint32_t parity, const Args& a, volatile int* abort, unsigned where) {
    if (mbar_try_wait_cluster(bar, parity)) return true;
    return wait_slow(bar, parity, a, abort, where, true);
}
// warp-uniform outcome, so that a timeout never splits a warp before warp-collective instructions
__device__ __forceinline__ bool wait_w(uint32_t bar, uint32_t parity, const Args& a, volatile int* abort, unsigned where) {
    return __all_sync(0xffffffffu, wait_b(bar, parity, a, abort, where));
}
__device__ __forceinline__ bool wait_wcl(uint32_t bar, uint32_t parity, const Args& a, volatile int* abort,
                                         unsigned where) {
    return __all_sync(0xffffffffu, wait_cl(bar, parity, a, abort, where));
}

__global__ void __launch_bounds__(kThreads, 1)
decode_steps_kernel(const __grid_constant__ CUtensorMap map_wa, const __grid_constant__ CUtensorMap map_wx,
                    const __grid_constant__ CUtensorMap map_y, const __grid_constant__ CUtensorMap map_out,
                    const Args a) {
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const uint32_t sbase = smem_u32(smem);
    const Bars bars{sbase + OFF_BAR};
    volatile uint32_t* tmem_base_s = reinterpret_cast<volatile uint32_t*>(smem + OFF_MISC);
    volatile int* abort = reinterpret_cast<volatile int*>(smem + OFF_MISC + 16);
    float* s_K = reinterpret_cast<float*>(smem + OFF_CONST);
    float* s_nba = s_K + NT;
    float* s_nbx = s_nba + NT;
    float* s_cw = s_nbx + NT;                                  // [4][64]
    float* s_cb = s_cw + 4 * NT;                               // [64]

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    // cluster = (head, row tile); rank = channel tile (blockIdx.x = (head * mtiles + mt) * 4 + rank)
    const int nt = (int)cluster_ctarank();
    const int mt = (blockIdx.x / kCluster) % a.mtiles;
    const int head = blockIdx.x / (kCluster * a.mtiles);
    const int W = a.H * DH;
    const int ch0 = head * DH + nt * NT;                       // first global channel of the tile
    const int S = a.S;

    if (threadIdx.x == 0) {
        mbar_init(bars.w(), 1);
        mbar_init(bars.w16(), 1);
        mbar_init(bars.y_full(), 1);
        mbar_init(bars.y_empty(), 1);
        for (int j = 0; j < kCluster; ++j) mbar_init(bars.k(j), 1);
        mbar_init(bars.own(), kUpdWarps);
        mbar_init(bars.a_free(), kCluster);
        for (int i = 0; i < NBUF; ++i) {
            mbar_init(bars.acc_full(i), 1);
            mbar_init(bars.acc_empty(i), kUpdWarps);
        }
        mbar_init(bars.mma_done(), 1);
        *abort = 0;
        fence_barrier_init();
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
    }
    if (threadIdx.x < NT) {                                    // per-channel constants
        const int ch = ch0 + threadIdx.x;
        s_K[threadIdx.x] = a.c * log_sigmoid_acc(a.lambda[ch]);
        s_nba[threadIdx.x] = a.b_a ? -a.b_a[ch] * kLog2e : 0.f;
        s_nbx[threadIdx.x] = a.b_x ? -a.b_x[ch] * kLog2e : 0.f;
#pragma unroll
        for (int k = 0; k < kConvWidth; ++k) s_cw[k * NT + threadIdx.x] = a.conv_w[(size_t)k * W + ch];
        s_cb[threadIdx.x] = a.conv_b ? a.conv_b[ch] : 0.f;
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_base_s;
    // every CTA of the cluster has initialised its barriers before any copy or arrive targets them
    cluster_sync();

    if (warp == kWarpTma) {
        if (lane == 0) {
            // ============================ loads: the weights once, y every step ===============
            mbar_arrive_expect_tx(bars.w(), 2 * W_BYTES);
            for (int kb = 0; kb < DH / 64; ++kb) {
                tma_load_2d(sbase + OFF_WA + kb * 8192, &map_wa, nt * NT, head * DH + kb * 64, bars.w());
                tma_load_2d(sbase + OFF_WX + kb * 8192, &map_wx, nt * NT, head * DH + kb * 64, bars.w());
            }
            int last_y = -1;
            for (int s = 0; s < S; ++s) {
                // the tile is free once the out store of step s - 1 has read it
                if (!wait_b(bars.y_empty(), (s & 1) ^ 1, a, abort, 2)) break;
                mbar_arrive_expect_tx(bars.y_full(), T_BYTES);
                tma_load_3d(sbase + OFF_Y, &map_y, ch0, mt * MT, s, bars.y_full());
                last_y = s;
            }
            // never leave the CTA with a bulk copy still writing its shared memory
            const uint64_t t0 = globaltimer_ns();
            while (!mbar_try_wait_sleep(bars.w(), 0, 20000u) && globaltimer_ns() - t0 < a.timeout_ns) {
            }
            if (last_y >= 0)
                while (!mbar_try_wait_sleep(bars.y_full(), last_y & 1, 20000u) && globaltimer_ns() - t0 < a.timeout_ns) {
                }
        }
    } else if (warp == kWarpMma) {
        // ================================ MMA and the exchange ================================
        // the whole warp follows the waits; one elected lane issues copies, MMAs and commits
        const uint32_t idesc = idesc_bmn(MT, 2 * NT);         // D_a | D_x
        const uint32_t tm = __shfl_sync(0xffffffffu, tmem, 0);
        bool ok = wait_w(bars.w16(), 0, a, abort, 3);
        int issued = 0;
        for (int s = 0; s < S && ok; ++s) {
            const uint32_t ph = s & 1;
            // this step's blocks from the three siblings complete on k(j) by their bytes
            if (elect_one())
                for (int j = 0; j < kCluster; ++j)
                    if (j != nt) mbar_arrive_expect_tx(bars.k(j), 2 * A_KBLK);
            __syncwarp();
            // this CTA's blocks: written by its update threads (which waited until every MMA
            // of the previous step, here and in the siblings, had finished reading the tiles)
            if (!wait_w(bars.own(), ph, a, abort, 4)) break;
            if (elect_one())
                for (int r = 1; r < kCluster; ++r) {
                    const uint32_t peer = (uint32_t)((nt + r) % kCluster);
#pragma unroll
                    for (int part = 0; part < 2; ++part) {
                        const uint32_t blk = sbase + (part ? OFF_ALO : OFF_A) + nt * A_KBLK;
                        dsmem_copy(map_to_rank(blk, peer), blk, A_KBLK, map_to_rank(bars.k(nt), peer));
                    }
                }
            __syncwarp();
            const int bi = s % NBUF;
            if (s >= NBUF && !wait_w(bars.acc_empty(bi), ((s - NBUF) / NBUF) & 1, a, abort, 5)) break;
            tc_fence_after();
            const uint32_t d = tm + bi * (2 * NT);
            for (int i = 0; i < kCluster && ok; ++i) {
                // own block first, then in arrival order (CTA j sends to j + 1, j + 2, j + 3)
                const int j = (nt - i + kCluster) % kCluster;
                if (j != nt && !wait_wcl(bars.k(j), ph, a, abort, 6)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                if (elect_one()) {
#pragma unroll
                    for (int part = 0; part < 2; ++part)
#pragma unroll
                        for (int kk = 0; kk < KSTEPS / kCluster; ++kk) {
                            const int ks = j * 4 + kk;
                            const uint64_t ad = desc_k_sw128(sbase + (part ? OFF_ALO : OFF_A) + j * A_KBLK + kk * 32);
                            const uint64_t bd = desc_mn_sw128(sbase + OFF_WA + ks * 16 * 128);
                            mma_ss(d, ad, bd, idesc, (i > 0 || kk > 0 || part > 0) ? 1u : 0u);
                        }
                }
                __syncwarp();
            }
            if (!ok) break;
            if (elect_one()) {
                mma_commit(bars.acc_full(bi));
                // the operand tiles of every CTA may be rewritten once all four MMAs are done
                for (int j = 0; j < kCluster; ++j) mma_commit_cluster(map_to_rank(bars.a_free(), (uint32_t)j));
            }
            __syncwarp();
            issued = s + 1;
        }
        // no tensor-core work and no incoming commit left in flight at the exit
        if (elect_one()) mma_commit(bars.mma_done());
        __syncwarp();
        if (lane == 0) {
            const uint64_t t0 = globaltimer_ns();
            while (!mbar_try_wait_sleep(bars.mma_done(), 0, 20000u) && globaltimer_ns() - t0 < a.timeout_ns) {
            }
            if (issued > 0)
                while (!mbar_try_wait_cluster(bars.a_free(), (issued - 1) & 1) && globaltimer_ns() - t0 < a.timeout_ns) {
                    __nanosleep(128);
                }
        }
        __syncwarp();
    } else {
        // ================================ update threads =======================================
        // thread = row r of the tile (its TMEM lane), channels [16 cg, 16 cg + 16) of its 64
        const int q = warp & 3, cg = warp >> 2;
        const int r = q * 32 + lane;
        const int b = mt * MT + r;
        const bool live = b < a.B;
        const uint32_t sw = (uint32_t)(r & 7);
        const int cbase = ch0 + cg * kCh;
        const uint32_t lane_off = (uint32_t)(q * 32) << 16;
        const uint32_t xcol = tmem + lane_off + TM_XC + cg * kCh;        // + (s & 1) NT
        const uint32_t hcol = tmem + lane_off + TM_HIST + cg * 24;       // 3 rows x 8 words
        // state: h in registers; the conv history (3 x 16 bf16) into the thread's TMEM lane
        float hv[kCh];
#pragma unroll
        for (int i = 0; i < kCh; ++i) hv[i] = 0.f;
#pragma unroll
        for (int row = 0; row < kHist; ++row) {
            uint32_t hist[8];
#pragma unroll
            for (int i = 0; i < 8; ++i) hist[i] = 0u;
            if (live) {
                const uint4* tp = reinterpret_cast<const uint4*>(a.tail + ((size_t)b * kHist + row) * W + cbase);
                const uint4 v0 = tp[0], v1 = tp[1];
                hist[0] = v0.x; hist[1] = v0.y; hist[2] = v0.z; hist[3] = v0.w;
                hist[4] = v1.x; hist[5] = v1.y; hist[6] = v1.z; hist[7] = v1.w;
            }
            tmem_st8(hcol + 8 * row, hist);
        }
        tmem_wait_st();
        if (live) {
            const float4* hp = reinterpret_cast<const float4*>(a.h + (size_t)b * W + cbase);
#pragma unroll
            for (int i = 0; i < kCh / 4; ++i) {
                const float4 v = hp[i];
                hv[4 * i] = v.x; hv[4 * i + 1] = v.y; hv[4 * i + 2] = v.z; hv[4 * i + 3] = v.w;
            }
        }
        // conv taps and bias of the thread's channels stay in shared memory (warp-wide broadcasts)
        const float* cwp = s_cw + cg * kCh;
        const float* cbp = s_cb + cg * kCh;
        const uint32_t own_blk = nt * A_KBLK;

        // x of step s for the thread's row and channels (zeros past the batch or the steps)
        auto load_x = [&](int s, uint4 (&xv)[2]) {
            if (live && s < S) {
                const uint4* xp = reinterpret_cast<const uint4*>(a.x + ((size_t)s * a.B + b) * W + cbase);
                xv[0] = xp[0];
                xv[1] = xp[1];
            } else {
                xv[0] = xv[1] = make_uint4(0, 0, 0, 0);
            }
        };

        // the weight slices to fp16, in place (an element-wise pass: the layout does not matter)
        {
            const bool okw = wait_b(bars.w(), 0, a, abort, 11);
            if (okw) {
                uint4* wt = reinterpret_cast<uint4*>(smem + OFF_WA);
#pragma unroll 4
                for (int i = threadIdx.x; i < (int)(2 * W_BYTES / 16); i += kUpdThreads) {
                    uint4 v = wt[i];
                    v.x = pack_f16x2(bf16lo(v.x), bf16hi(v.x));
                    v.y = pack_f16x2(bf16lo(v.y), bf16hi(v.y));
                    v.z = pack_f16x2(bf16lo(v.z), bf16hi(v.z));
                    v.w = pack_f16x2(bf16lo(v.w), bf16hi(v.w));
                    wt[i] = v;
                }
            }
            fence_proxy_async_smem();
            asm volatile("bar.sync 1, %0;" ::"n"(kUpdThreads) : "memory");
            if (threadIdx.x == 0) mbar_arrive(bars.w16());    // also after a failed wait: the MMA warp drains
        }

        // conv of step s from x (xv): history reset, the result in fp32 into TMEM buffer s % 2 and
        // as an fp16 hi + lo pair into this CTA's K blocks of the operand tiles; the history shifts
        auto conv_step = [&](int s, const uint4 (&xv)[2]) -> bool {
            if (s > 0 && !wait_wcl(bars.a_free(), (s - 1) & 1, a, abort, 8)) return false;
            uint32_t th[3][8];                                // history rows 0..2 (oldest first)
            tmem_ld8u(hcol, th[0]);
            tmem_ld8u(hcol + 8, th[1]);
            tmem_ld8u(hcol + 16, th[2]);
            tmem_wait_ld();
            if (live && a.reset && a.reset[(size_t)s * a.B + b]) {
#pragma unroll
                for (int row = 0; row < kHist; ++row)
#pragma unroll
                    for (int i = 0; i < 8; ++i) th[row][i] = 0u;
            }
#pragma unroll
            for (int v = 0; v < 2; ++v) {
                const uint32_t* px = reinterpret_cast<const uint32_t*>(&xv[v]);
                uint32_t ohi[4], olo[4], xo[8];
#pragma unroll
                for (int e2 = 0; e2 < 4; ++e2) {
                    float rr[2];
#pragma unroll
                    for (int e1 = 0; e1 < 2; ++e1) {
                        const int j = v * 8 + 2 * e2 + e1;
                        const int wi = v * 4 + e2;                // word of the 16-channel row
                        const float v0 = e1 ? bf16hi(th[0][wi]) : bf16lo(th[0][wi]);
                        const float v1 = e1 ? bf16hi(th[1][wi]) : bf16lo(th[1][wi]);
                        const float v2 = e1 ? bf16hi(th[2][wi]) : bf16lo(th[2][wi]);
                        const float v3 = e1 ? bf16hi(px[e2]) : bf16lo(px[e2]);
                        float acc = fmaf(cwp[j], v0, cbp[j]);
                        acc = fmaf(cwp[NT + j], v1, acc);
                        acc = fmaf(cwp[2 * NT + j], v2, acc);
                        acc = fmaf(cwp[3 * NT + j], v3, acc);
                        rr[e1] = acc;
                        xo[2 * e2 + e1] = __float_as_uint(acc);
                    }
                    ohi[e2] = pack_f16x2(rr[0], rr[1]);
                    olo[e2] = pack_f16x2(rr[0] - f16lo(ohi[e2]), rr[1] - f16hi(ohi[e2]));
                }
                // row r, 16-byte chunk (2 cg + v) of this CTA's K blocks (128-byte swizzle)
                const uint32_t so = own_blk + (uint32_t)(r >> 3) * 1024 + sw * 128 + ((((uint32_t)(cg * 2 + v)) ^ sw) << 4);
                *reinterpret_cast<uint4*>(smem + OFF_A + so) = make_uint4(ohi[0], ohi[1], ohi[2], ohi[3]);
                *reinterpret_cast<uint4*>(smem + OFF_ALO + so) = make_uint4(olo[0], olo[1], olo[2], olo[3]);
                tmem_st8(xcol + (uint32_t)(s & 1) * (uint32_t)NT + v * 8, xo);
            }
            // the history: oldest out, x in
            tmem_st8(hcol, th[1]);
            tmem_st8(hcol + 8, th[2]);
            const uint32_t nx[8] = {xv[0].x, xv[0].y, xv[0].z, xv[0].w, xv[1].x, xv[1].y, xv[1].z, xv[1].w};
            tmem_st8(hcol + 16, nx);
            tmem_wait_st();
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) mbar_arrive(bars.own());
            return true;
        };

        uint4 xa[2], xb[2];                                   // x of the next two convs
        bool ok;
        {
            uint4 x0[2];
            load_x(0, x0);
            load_x(1, xa);
            load_x(2, xb);
            ok = conv_step(0, x0);
        }
        for (int s = 0; s < S; ++s) {
            const int bi = s % NBUF;
            // the accumulators of step s are complete; the conv of step s + 1 goes first
            ok = ok && wait_w(bars.acc_full(bi), (s / NBUF) & 1, a, abort, 9);
            if (ok) tc_fence_after();
            if (ok && s + 1 < S) {
                ok = conv_step(s + 1, xa);
                xa[0] = xb[0];
                xa[1] = xb[1];
                load_x(s + 3, xb);
            }
            ok = ok && wait_w(bars.y_full(), s & 1, a, abort, 10);
            if (!upd_all(ok)) break;
            // update of step s
            const bool rst = live && a.reset && a.reset[(size_t)s * a.B + b];
            if (rst) {
#pragma unroll
                for (int i = 0; i < kCh; ++i) hv[i] = 0.f;
            }
            const uint32_t taddr = tmem + lane_off + bi * (2 * NT) + cg * kCh;
#pragma unroll
            for (int v = 0; v < 2; ++v) {
                float ga[8], gx[8], xc[8];
                tmem_ld8(taddr + v * 8, ga);
                tmem_ld8(taddr + NT + v * 8, gx);
                tmem_ld8(xcol + (uint32_t)(s & 1) * (uint32_t)NT + v * 8, xc);
                tmem_wait_ld();
                if (v == 1) {                                 // the accumulators are read
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(bars.acc_empty(bi));
                }
                const uint32_t yo = OFF_Y + (uint32_t)r * 128 + ((((uint32_t)(cg * 2 + v)) ^ sw) << 4);
                const uint4 yq = *reinterpret_cast<const uint4*>(smem + yo);
                const uint32_t* yw = reinterpret_cast<const uint32_t*>(&yq);
                uint32_t ow[4];
#pragma unroll
                for (int e2 = 0; e2 < 4; ++e2) {
                    float o[2];
#pragma unroll
                    for (int e1 = 0; e1 < 2; ++e1) {
                        const int e = v * 8 + 2 * e2 + e1;
                        const int jc = cg * kCh + e;              // column within the tile
                        float at, u;
                        gates1<false>(ga[2 * e2 + e1], gx[2 * e2 + e1], s_nba[jc], s_nbx[jc], s_K[jc],
                                      xc[2 * e2 + e1], at, u);
                        const float hn = fmaf(at, hv[e], u);
                        hv[e] = hn;
                        o[e1] = hn * gelu1(e1 ? bf16hi(yw[e2]) : bf16lo(yw[e2]), a.gelu_tanh);
                    }
                    ow[e2] = pack_bf16x2(o[0], o[1]);
                }
                *reinterpret_cast<uint4*>(smem + yo) = make_uint4(ow[0], ow[1], ow[2], ow[3]);
            }
            // out tile of step s -> global (rows past the batch are clipped by the map)
            fence_proxy_async_smem();
            asm volatile("bar.sync 1, %0;" ::"n"(kUpdThreads) : "memory");
            if (threadIdx.x == 0) {
                tma_store_3d(&map_out, sbase + OFF_Y, ch0, mt * MT, s);
                bulk_commit();
                bulk_wait_read0();
                mbar_arrive(bars.y_empty());
            }
        }
        if (threadIdx.x == 0) bulk_wait0();
        // the state after the last step (or where a failure stopped the loop: the status says so)
        uint32_t th[3][8];
        tmem_ld8u(hcol, th[0]);
        tmem_ld8u(hcol + 8, th[1]);
        tmem_ld8u(hcol + 16, th[2]);
        tmem_wait_ld();
        if (live) {
            float4* hp = reinterpret_cast<float4*>(a.h + (size_t)b * W + cbase);
#pragma unroll
            for (int i = 0; i < kCh / 4; ++i)
                hp[i] = make_float4(hv[4 * i], hv[4 * i + 1], hv[4 * i + 2], hv[4 * i + 3]);
#pragma unroll
            for (int row = 0; row < kHist; ++row) {
                uint4* tp = reinterpret_cast<uint4*>(a.tail + ((size_t)b * kHist + row) * W + cbase);
                tp[0] = make_uint4(th[row][0], th[row][1], th[row][2], th[row][3]);
                tp[1] = make_uint4(th[row][4], th[row][5], th[row][6], th[row][7]);
            }
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

}  // namespace dms

bool fused_decode_steps_supported(const rglru_dims* d) {
    return d->act_dtype == RGLRU_BF16 && d->head_dim == dms::DH && !(d->flags & RGLRU_FLAG_GENERIC);
}

cudaError_t launch_fused_decode_steps(const rglru_dims* d, const rglru_params* p, const void* x, const void* y,
                                      const uint8_t* reset, int steps, rglru_state* st, void* out, void* ws,
                                      size_t ws_bytes, cudaStream_t s) {
    using namespace dms;
    if (ws_bytes < 256) return cudaErrorInvalidValue;
    const int B = d->batch, H = d->heads;
    const int W = H * DH;
    CUtensorMap mwa, mwx, my, mo;
    if (!tc::make_map_2d_sw128(&mwa, p->w_a, DH, (uint64_t)W, DH * 2, NT, 64) ||
        !tc::make_map_2d_sw128(&mwx, p->w_x, DH, (uint64_t)W, DH * 2, NT, 64) ||
        !tc::make_map_3d_sw128(&my, y, W, B, steps, NT, MT) || !tc::make_map_3d_sw128(&mo, out, W, B, steps, NT, MT))
        return cudaErrorInvalidValue;
    cudaError_t e = set_smem_once(decode_steps_kernel, (int)SMEM_BYTES);
    if (e != cudaSuccess) return e;
    Args a;
    a.B = B; a.H = H; a.mtiles = (B + MT - 1) / MT; a.S = steps;
    a.x = static_cast<const __nv_bfloat16*>(x);
    a.conv_w = p->conv_w; a.conv_b = p->conv_b;
    a.c = d->c; a.gelu_tanh = d->gelu_tanh;
    a.timeout_ns = 1000000000ull;
    a.b_a = p->b_a; a.b_x = p->b_x; a.lambda = p->lambda; a.reset = reset;
    a.h = st->h;
    a.tail = static_cast<__nv_bfloat16*>(st->conv_tail);
    a.status = reinterpret_cast<DeviceStatus*>(ws);
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)(H * a.mtiles * kCluster));
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = SMEM_BYTES;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = kCluster;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, decode_steps_kernel, mwa, mwx, my, mo, a);
}

}  // namespace rglru
