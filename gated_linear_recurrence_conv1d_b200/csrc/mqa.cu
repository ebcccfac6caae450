// mqa.cu -- Griffin's local sliding-window multi-query attention on sm_100a (bf16, head_dim 256).
//
// "Griffin Guide: RecurrentGemma, RG-LRU & Hybrid Attention", "2. Local Sliding-Window
// Multi-Query Attention (MQA)" and "3. Bounding the Key-Value Cache Footprint"; the "Griffin"
// notes, "Local Attention Path":  H query heads share one key head and one value head; token t
// attends to N(t) = {i : t - w < i <= t}:  y_t = sum_{i in N(t)} softmax_i(s q_t . k_i) v_i, with
// rotary position embeddings on queries and keys; decoding keeps the last w keys / values in a
// ring buffer (slot = position mod w).  RoPE turns the pairs (j, j + d/2) by p base^(-2j/d).
//
//   * mqa_rope_kernel: rotates q and k (angles in fp64, reduced mod 2 pi, then fp32 sine and
//     cosine) into bf16 copies; copies the last w rotated keys and values into the ring cache;
//   * mqa_prefill_kernel: one CTA per (row, head, 128 queries), in the manner of
//     FlashAttention: the query tile sits in TMEM as the A operand (TS form); per 64-key tile of
//     the window, S = Q K^T (tcgen05.mma, M = 128, N = 64, K = 256) goes to one of two TMEM
//     buffers; 4 softmax warps (thread = query) mask the window, take exp2 against a running
//     reference maximum that moves only when the maximum grows by more than 2^8 (then the
//     accumulator is rescaled), write P in bf16 to shared memory; O += P V (M = 128, N = 256,
//     K = 64) accumulates in TMEM; the S of the next tile overlaps the softmax of this one;
//   * mqa_decode_kernel: one token per row against the ring, persistent: the ring's slots are cut
//     into tiles of 128 and a row's tiles into parts; per tile S^T = K Q^T and O^T = V^T P^T run
//     on the tensor cores (the H heads of a row form the MMA's N) while the next tiles stream in
//     by TMA, the softmax on 4 warps; each part leaves (max, sum, sum of p v) per head, and
//     mqa_merge_kernel combines the parts (the three kernels chained by programmatic dependent
//     launch).
#include <algorithm>

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <math.h>
#include <stdint.h>

#include "common.cuh"
#include "kernels.h"
#include "sm100.cuh"
#include "tma_maps.h"

namespace rglru {
namespace mq {

using namespace sm100;

constexpr int D = 256;                 // head dim (the tensor-core path)
constexpr int BQ = 128;                // queries per CTA (MMA M)
constexpr int BKV = 64;                // keys per tile (MMA N of S, K of P V)
constexpr int kRopeMaxH = 16;          // query heads a row may have
constexpr float kLog2e = 1.4426950408889634f;

// ---------------------------------------------------------------- rotary embedding ----------
struct RopeArgs {
    int B, T, H, w, pos0;
    float base;
    const __nv_bfloat16* q;            // [B, T, H, d]
    const __nv_bfloat16* k;            // [B, T, d]
    const __nv_bfloat16* v;            // [B, T, d]
    __nv_bfloat16* q_rot;
    __nv_bfloat16* k_rot;
    __nv_bfloat16* cache;              // [B][2][w][d] or nullptr
};

// sine and cosine of an angle given in fp64: reduced mod 2 pi in fp64, then fp32
__device__ __forceinline__ void sincos_of(double ang, float& s, float& c) {
    const double two_pi = 6.283185307179586476925286766559;
    sincosf((float)fmod(ang, two_pi), &s, &c);
}

// thread = (row b, token t, j < d/2) over the H query heads and the key: the inputs first
// (independent loads), then one angle, its sine and cosine for all of them
__global__ void __launch_bounds__(D / 2) mqa_rope_kernel(RopeArgs a) {
    const int j = threadIdx.x;                       // 0 .. d/2 - 1
    const int t = blockIdx.x, b = blockIdx.y, H = a.H;
    const int p = a.pos0 + t;
    const size_t qrow = ((size_t)b * a.T + t) * H * D;
    const size_t ke = ((size_t)b * a.T + t) * D;
    float x1[kRopeMaxH], x2[kRopeMaxH];
#pragma unroll
    for (int h = 0; h < kRopeMaxH; ++h)
        if (h < H) {
            x1[h] = __bfloat162float(__ldg(a.q + qrow + h * D + j));
            x2[h] = __bfloat162float(__ldg(a.q + qrow + h * D + j + D / 2));
        }
    const float k1 = __bfloat162float(__ldg(a.k + ke + j)), k2 = __bfloat162float(__ldg(a.k + ke + j + D / 2));
    const double ang = (double)p * pow((double)a.base, -2.0 * j / D);
    float sn, cs;
    sincos_of(ang, sn, cs);
#pragma unroll
    for (int h = 0; h < kRopeMaxH; ++h)
        if (h < H) {
            a.q_rot[qrow + h * D + j] = __float2bfloat16_rn(x1[h] * cs - x2[h] * sn);
            a.q_rot[qrow + h * D + j + D / 2] = __float2bfloat16_rn(x2[h] * cs + x1[h] * sn);
        }
    const __nv_bfloat16 r1 = __float2bfloat16_rn(k1 * cs - k2 * sn), r2 = __float2bfloat16_rn(k2 * cs + k1 * sn);
    a.k_rot[ke + j] = r1;
    a.k_rot[ke + j + D / 2] = r2;
    if (a.cache && t >= a.T - a.w) {                 // the last w positions stay for decoding
        const int slot = p % a.w;
        __nv_bfloat16* ck = a.cache + ((size_t)b * 2 * a.w + slot) * D;
        __nv_bfloat16* cv = a.cache + ((size_t)b * 2 * a.w + a.w + slot) * D;
        ck[j] = r1;
        ck[j + D / 2] = r2;
        cv[j] = a.v[ke + j];
        cv[j + D / 2] = a.v[ke + j + D / 2];
    }
}

// one decode token per row at position pos[b]: q_rot [B, H, d]; the rotated key and the value
// go into ring slot pos mod w
struct RopeDecArgs {
    int B, H, w;
    float base;
    const int* pos;
    const __nv_bfloat16* q;            // [B, H, d]
    const __nv_bfloat16* k;            // [B, d]
    const __nv_bfloat16* v;
    __nv_bfloat16* q_rot;
    __nv_bfloat16* cache;              // [B][2][w][d]
};

__global__ void __launch_bounds__(D / 2) mqa_rope_decode_kernel(RopeDecArgs a) {
    // the attention kernel may start its set-up now; it waits for this grid before reading
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    const int j = threadIdx.x, b = blockIdx.x, H = a.H;
    // every input of the thread first (independent loads), then one angle for all of them
    const __nv_bfloat16* qb = a.q + (size_t)b * H * D;
    float x1[kRopeMaxH], x2[kRopeMaxH];
#pragma unroll
    for (int h = 0; h < kRopeMaxH; ++h)
        if (h < H) {
            x1[h] = __bfloat162float(__ldg(qb + h * D + j));
            x2[h] = __bfloat162float(__ldg(qb + h * D + j + D / 2));
        }
    const float k1 = __bfloat162float(__ldg(a.k + (size_t)b * D + j));
    const float k2 = __bfloat162float(__ldg(a.k + (size_t)b * D + j + D / 2));
    const __nv_bfloat16 v1 = __ldg(a.v + (size_t)b * D + j), v2 = __ldg(a.v + (size_t)b * D + j + D / 2);
    const int p = __ldg(a.pos + b);
    const double ang = (double)p * pow((double)a.base, -2.0 * j / D);
    float sn, cs;
    sincos_of(ang, sn, cs);
    __nv_bfloat16* qr = a.q_rot + (size_t)b * H * D;
#pragma unroll
    for (int h = 0; h < kRopeMaxH; ++h)
        if (h < H) {
            qr[h * D + j] = __float2bfloat16_rn(x1[h] * cs - x2[h] * sn);
            qr[h * D + j + D / 2] = __float2bfloat16_rn(x2[h] * cs + x1[h] * sn);
        }
    const int slot = p % a.w;
    __nv_bfloat16* ck = a.cache + ((size_t)b * 2 * a.w + slot) * D;
    __nv_bfloat16* cv = a.cache + ((size_t)b * 2 * a.w + a.w + slot) * D;
    ck[j] = __float2bfloat16_rn(k1 * cs - k2 * sn);
    ck[j + D / 2] = __float2bfloat16_rn(k2 * cs + k1 * sn);
    cv[j] = v1;
    cv[j + D / 2] = v2;
}

// ---------------------------------------------------------------- prefill attention ---------
struct PrefArgs {
    int B, T, H, w;
    float scale_log2;                  // score scale * log2(e)
    __nv_bfloat16* out;                // [B, T, H, d]
    DeviceStatus* status;
    unsigned long long timeout_ns;
};

constexpr uint32_t Q_BYTES = BQ * D * 2;             // 65536, row-major staging of the query tile
constexpr uint32_t KT_BYTES = BKV * D * 2;           // 32768: 4 K-blocks of [64 keys x 128 B]
constexpr uint32_t VT_BYTES = BKV * D * 2;           // 32768: 4 atoms of [64 keys x 64 d] (MN-major)
constexpr uint32_t P_BYTES = BQ * BKV * 2;           // 16384: [128 queries x 64 keys], 128B swizzle
constexpr uint32_t OFF_Q = 0;
constexpr uint32_t OFF_K = OFF_Q + Q_BYTES;          // 2 stages
constexpr uint32_t OFF_V = OFF_K + 2 * KT_BYTES;     // 2 stages
constexpr uint32_t OFF_P = OFF_V + 2 * VT_BYTES;     // 2 buffers (tile parity)
constexpr uint32_t OFF_BAR = OFF_P + 2 * P_BYTES;
constexpr uint32_t SMEM_BYTES = OFF_BAR + 256 + 1024;
static_assert(SMEM_BYTES <= 232448, "shared memory budget");
// TMEM: [0,128) Q (A operand, bf16 pairs), [128,256) S double buffer, [256,512) O (fp32)
constexpr uint32_t TM_Q = 0, TM_S = 128, TM_O = 256;
constexpr int kSmWarps = 4, kWarpTma = 4, kWarpMma = 5, kThreads = 6 * 32;

struct Bars {
    uint32_t base;
    __device__ __forceinline__ uint32_t q_full() const { return base; }
    __device__ __forceinline__ uint32_t q_tmem() const { return base + 8; }
    __device__ __forceinline__ uint32_t k_full(int i) const { return base + 16 + 8u * i; }
    __device__ __forceinline__ uint32_t k_empty(int i) const { return base + 32 + 8u * i; }
    __device__ __forceinline__ uint32_t v_full(int i) const { return base + 48 + 8u * i; }
    __device__ __forceinline__ uint32_t v_empty(int i) const { return base + 64 + 8u * i; }
    __device__ __forceinline__ uint32_t s_full(int i) const { return base + 80 + 8u * i; }
    __device__ __forceinline__ uint32_t s_free(int i) const { return base + 96 + 8u * i; }
    __device__ __forceinline__ uint32_t p_full(int i) const { return base + 112 + 8u * i; }
    __device__ __forceinline__ uint32_t o_done(int i) const { return base + 128 + 8u * i; }   // P V on buffer i finished
    __device__ __forceinline__ uint32_t mma_done() const { return base + 144; }
};

__device__ __noinline__ bool wait_slow(uint32_t bar, uint32_t parity, const PrefArgs& a, volatile int* abort, unsigned where) {
    const uint64_t t0 = globaltimer_ns();
    for (;;) {
        if (mbar_try_wait_sleep(bar, parity, 20000u)) return true;
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
    }
}
__device__ __forceinline__ bool wait_b(uint32_t bar, uint32_t parity, const PrefArgs& a, volatile int* abort, unsigned where) {
    if (mbar_try_wait(bar, parity)) return true;
    return wait_slow(bar, parity, a, abort, where);
}

// MN-major (128-byte swizzle) descriptor of the V tile: 4 atoms of 64 d-columns, 8192 B apart
__device__ __forceinline__ uint64_t desc_v(uint32_t smem_addr) {
    uint64_t d = 0;
    d |= (uint64_t)((smem_addr >> 4) & 0x3FFF);
    d |= (uint64_t)(8192 >> 4) << 16;
    d |= (uint64_t)(1024 >> 4) << 32;
    d |= (uint64_t)1 << 46;
    d |= (uint64_t)2 << 61;
    return d;
}
__device__ __forceinline__ uint32_t idesc_mk(int n, int b_mn) {
    return (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)b_mn << 16) | ((uint32_t)(n >> 3) << 17) |
           ((uint32_t)(BQ >> 4) << 24);
}

__global__ void __launch_bounds__(kThreads, 1)
mqa_prefill_kernel(const __grid_constant__ CUtensorMap map_q, const __grid_constant__ CUtensorMap map_k,
                   const __grid_constant__ CUtensorMap map_v, const PrefArgs a) {
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const uint32_t sbase = smem_u32(smem);
    const Bars bars{sbase + OFF_BAR};
    volatile uint32_t* tmem_base_s = reinterpret_cast<volatile uint32_t*>(smem + OFF_BAR + 160);
    volatile int* abort = reinterpret_cast<volatile int*>(smem + OFF_BAR + 176);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    // blockIdx.x = query tile, y = head, z = row
    const int t0 = blockIdx.x * BQ, h = blockIdx.y, b = blockIdx.z;
    const int q_last = min(a.T, t0 + BQ) - 1;
    const int k_lo = max(0, t0 - a.w + 1);                // first key any query of the tile sees
    const int j0 = k_lo / BKV, j1 = q_last / BKV;         // key tiles [j0, j1]
    const int ntiles = j1 - j0 + 1;

    if (threadIdx.x == 0) {
        mbar_init(bars.q_full(), 1);
        mbar_init(bars.q_tmem(), kSmWarps);
        for (int i = 0; i < 2; ++i) {
            mbar_init(bars.k_full(i), 1);
            mbar_init(bars.k_empty(i), 1);
            mbar_init(bars.v_full(i), 1);
            mbar_init(bars.v_empty(i), 1);
            mbar_init(bars.s_full(i), 1);
            mbar_init(bars.s_free(i), kSmWarps);
            mbar_init(bars.p_full(i), kSmWarps);
            mbar_init(bars.o_done(i), 1);
        }
        mbar_init(bars.mma_done(), 1);
        *abort = 0;
        fence_barrier_init();
    }
    if (warp == kWarpMma) {
        tmem_alloc(smem_u32((const void*)tmem_base_s), 512);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_base_s;

    if (warp == kWarpTma) {
        if (lane == 0) {
            // query tile: rows (b, t0 .. t0 + 127, head h) of the [B T H, d] rotated queries
            mbar_arrive_expect_tx(bars.q_full(), Q_BYTES);
            for (int kb = 0; kb < D / 64; ++kb)
                tma_load_3d(sbase + OFF_Q + kb * (BQ * 128), &map_q, kb * 64, h, b * a.T + t0, bars.q_full());
            for (int j = 0; j < ntiles; ++j) {
                const int s = j & 1;
                const int key0 = (j0 + j) * BKV;
                if (!wait_b(bars.k_empty(s), ((j >> 1) & 1) ^ 1, a, abort, 1)) break;
                mbar_arrive_expect_tx(bars.k_full(s), KT_BYTES);
                for (int kb = 0; kb < D / 64; ++kb)
                    tma_load_2d(sbase + OFF_K + s * KT_BYTES + kb * (BKV * 128), &map_k, kb * 64, b * a.T + key0,
                                bars.k_full(s));
                if (!wait_b(bars.v_empty(s), ((j >> 1) & 1) ^ 1, a, abort, 2)) break;
                mbar_arrive_expect_tx(bars.v_full(s), VT_BYTES);
                for (int dn = 0; dn < D / 64; ++dn)
                    tma_load_2d(sbase + OFF_V + s * VT_BYTES + dn * 8192, &map_v, dn * 64, b * a.T + key0,
                                bars.v_full(s));
            }
            // no bulk copy may still be writing shared memory at the exit
            const uint64_t tt = globaltimer_ns();
            for (int j = ntiles - 2; j < ntiles; ++j)
                if (j >= 0)
                    while (!(mbar_try_wait(bars.k_full(j & 1), (j >> 1) & 1) &&
                             mbar_try_wait(bars.v_full(j & 1), (j >> 1) & 1)) &&
                           globaltimer_ns() - tt < a.timeout_ns) {
                    }
            while (!mbar_try_wait(bars.q_full(), 0) && globaltimer_ns() - tt < a.timeout_ns) {
            }
        }
    } else if (warp == kWarpMma) {
        // the whole warp follows the waits; one elected lane issues (warp-uniform operands)
        const uint32_t id_s = idesc_mk(BKV, 0), id_o = idesc_mk(D, 1);
        const uint32_t tm = __shfl_sync(0xffffffffu, tmem, 0);
        auto wait_w = [&](uint32_t bar, uint32_t par, unsigned where) {
            return __all_sync(0xffffffffu, wait_b(bar, par, a, abort, where));
        };
        bool ok = wait_w(bars.q_tmem(), 0, 3);
        tc_fence_after();
        for (int j = 0; ok && j <= ntiles; ++j) {
            if (j < ntiles) {                                // S_j = Q K_j^T
                const int s = j & 1;
                if (!wait_w(bars.k_full(s), (j >> 1) & 1, 4)) break;
                if (!wait_w(bars.s_free(s), ((j >> 1) & 1) ^ 1, 5)) break;
                tc_fence_after();
                const uint32_t ds = tm + TM_S + s * BKV;
                if (elect_one()) {
#pragma unroll
                    for (int ks = 0; ks < D / 16; ++ks) {
                        const uint64_t bd = desc_k_sw128(sbase + OFF_K + s * KT_BYTES + (ks >> 2) * (BKV * 128) + (ks & 3) * 32);
                        mma_ts(ds, tm + TM_Q + ks * 8, bd, id_s, ks > 0 ? 1u : 0u);
                    }
                    mma_commit(bars.s_full(s));
                    mma_commit(bars.k_empty(s));
                }
                __syncwarp();
            }
            if (j >= 1) {                                    // O += P_{j-1} V_{j-1}
                const int jj = j - 1, s = jj & 1;             // P and V buffers of tile jj
                if (!wait_w(bars.p_full(s), (jj >> 1) & 1, 6)) break;
                if (!wait_w(bars.v_full(s), (jj >> 1) & 1, 7)) break;
                tc_fence_after();
                if (elect_one()) {
#pragma unroll
                    for (int ks = 0; ks < BKV / 16; ++ks) {
                        const uint64_t ad = desc_k_sw128(sbase + OFF_P + s * P_BYTES + ks * 32);
                        const uint64_t bd = desc_v(sbase + OFF_V + s * VT_BYTES + ks * 2048);
                        mma_ss(tm + TM_O, ad, bd, id_o, (jj > 0 || ks > 0) ? 1u : 0u);
                    }
                    mma_commit(bars.o_done(s));
                    mma_commit(bars.v_empty(s));
                }
                __syncwarp();
            }
        }
        // every MMA of this warp has finished before TMEM is released
        if (elect_one()) mma_commit(bars.mma_done());
        __syncwarp();
        if (lane == 0) {
            const uint64_t tt = globaltimer_ns();
            while (!mbar_try_wait_sleep(bars.mma_done(), 0, 20000u) && globaltimer_ns() - tt < a.timeout_ns) {
            }
        }
        __syncwarp();
    } else {
        // ================================ softmax warps: thread = query row ==================
        const int q = warp, r = q * 32 + lane;
        const int t = t0 + r;
        const uint32_t lane_off = (uint32_t)(q * 32) << 16;
        // the query tile: shared memory (K-major rows of 128 B per 64-wide block) -> TMEM A
        bool ok = __all_sync(0xffffffffu, wait_b(bars.q_full(), 0, a, abort, 8));
        if (ok) {
#pragma unroll 1
            for (int kb = 0; kb < D / 64; ++kb) {
                // row r of block kb: 128 bytes, 16-byte chunks swizzled by (r & 7)
                uint32_t rr[32];
                const uint8_t* row = smem + OFF_Q + kb * (BQ * 128) + (r >> 3) * 1024 + (r & 7) * 128;
#pragma unroll
                for (int c = 0; c < 8; ++c) {
                    const uint4 v = *reinterpret_cast<const uint4*>(row + ((c ^ (r & 7)) << 4));
                    rr[4 * c] = v.x; rr[4 * c + 1] = v.y; rr[4 * c + 2] = v.z; rr[4 * c + 3] = v.w;
                }
                uint32_t lo[16], hi[16];
#pragma unroll
                for (int i = 0; i < 16; ++i) { lo[i] = rr[i]; hi[i] = rr[16 + i]; }
                tmem_st16(tmem + lane_off + TM_Q + kb * 32, lo);
                tmem_st16(tmem + lane_off + TM_Q + kb * 32 + 16, hi);
            }
            tmem_wait_st();
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(bars.q_tmem());

        float m_ref = -INFINITY, l = 0.f;                     // log2-domain reference max, sum
        const int lo_key = max(0, t - a.w + 1);
        int pv_issued = 0;                                    // P V products handed to the MMA
        for (int j = 0; ok && j < ntiles; ++j) {
            const int s = j & 1;
            ok = __all_sync(0xffffffffu, wait_b(bars.s_full(s), (j >> 1) & 1, a, abort, 9));
            if (!ok) break;
            tc_fence_after();
            const int key0 = (j0 + j) * BKV;
            float sv[BKV];
#pragma unroll
            for (int c = 0; c < BKV; c += 16) {
                float tmp[16];
                tmem_ld16(tmem + lane_off + TM_S + s * BKV + c, tmp);
#pragma unroll
                for (int i = 0; i < 16; ++i) sv[c + i] = tmp[i];
            }
            tmem_wait_ld();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(bars.s_free(s));
            // scores stay unscaled (scale > 0: the maximum commutes with it); a tile inside every
            // query's window (the same for the whole CTA) needs no mask
            float mx = -INFINITY;
            if (key0 >= t0 + BQ - a.w && key0 + BKV - 1 <= t0) {
#pragma unroll
                for (int i = 0; i < BKV; ++i) mx = fmaxf(mx, sv[i]);
            } else {
#pragma unroll
                for (int i = 0; i < BKV; ++i) {
                    const int key = key0 + i;
                    const bool in = t < a.T && key >= lo_key && key <= t;
                    sv[i] = in ? sv[i] : -INFINITY;
                    mx = fmaxf(mx, sv[i]);
                }
            }
            mx *= a.scale_log2;
            // the reference maximum moves (and the accumulator is rescaled) only when the
            // tile's maximum passes it by more than 8 (a factor 256 in P)
            const bool move = mx > m_ref + 8.0f;
            const bool any_move = __any_sync(0xffffffffu, move);
            const float m_new = move ? mx : m_ref;
            // P buffer s was last read by the P V of tile j - 2; O may be rescaled only once the
            // P V of tile j - 1 (and so every earlier one) is complete
            if (pv_issued >= 2) {
                const int jj = pv_issued - 2;                 // == j - 2
                ok = __all_sync(0xffffffffu, wait_b(bars.o_done(jj & 1), (jj >> 1) & 1, a, abort, 10));
                if (!ok) break;
            }
            if (any_move && pv_issued > 0) {
                const int jj = pv_issued - 1;
                ok = __all_sync(0xffffffffu, wait_b(bars.o_done(jj & 1), (jj >> 1) & 1, a, abort, 12));
                if (!ok) break;
            }
            tc_fence_after();
            if (any_move && pv_issued > 0) {
                const float f = (move && m_ref != -INFINITY) ? exp2f(m_ref - m_new) : 1.0f;
#pragma unroll 1
                for (int c = 0; c < D; c += 16) {
                    float o[16];
                    tmem_ld16(tmem + lane_off + TM_O + c, o);
                    tmem_wait_ld();
#pragma unroll
                    for (int i = 0; i < 16; ++i) o[i] *= f;
                    tmem_st16f(tmem + lane_off + TM_O + c, o);
                }
                tmem_wait_st();
                l *= f;
            }
            m_ref = m_new;
            // P in bf16: row r, 64 keys = 128 bytes, 16-byte chunks swizzled by (r & 7)
            // (m_ref is -inf only while every score so far, this tile's included, is masked: then
            // the exponent is -inf and p = 0)
            uint8_t* prow = smem + OFF_P + s * P_BYTES + (r >> 3) * 1024 + (r & 7) * 128;
            const float neg_m = m_ref == -INFINITY ? 0.f : -m_ref;
#pragma unroll
            for (int c = 0; c < 8; ++c) {
                float p[8];
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                    p[i] = ex2_approx(fmaf(sv[8 * c + i], a.scale_log2, neg_m));
                    l += p[i];
                }
                uint4 pk;
                __nv_bfloat162 t0v = __floats2bfloat162_rn(p[0], p[1]), t1v = __floats2bfloat162_rn(p[2], p[3]);
                __nv_bfloat162 t2v = __floats2bfloat162_rn(p[4], p[5]), t3v = __floats2bfloat162_rn(p[6], p[7]);
                pk.x = *reinterpret_cast<uint32_t*>(&t0v); pk.y = *reinterpret_cast<uint32_t*>(&t1v);
                pk.z = *reinterpret_cast<uint32_t*>(&t2v); pk.w = *reinterpret_cast<uint32_t*>(&t3v);
                *reinterpret_cast<uint4*>(prow + ((c ^ (r & 7)) << 4)) = pk;
            }
            fence_proxy_async_smem();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(bars.p_full(s));
            ++pv_issued;
        }
        // the last P V, then out = O / l
        if (ok && pv_issued > 0) {
            const int jj = pv_issued - 1;                     // the last P V (every earlier one is done too)
            ok = __all_sync(0xffffffffu, wait_b(bars.o_done(jj & 1), (jj >> 1) & 1, a, abort, 11));
        }
        if (ok) {
            tc_fence_after();
            const float inv = l > 0.f ? 1.0f / l : 0.f;
            __nv_bfloat16* orow = a.out + (((size_t)b * a.T + t) * a.H + h) * D;
#pragma unroll 1
            for (int c = 0; c < D; c += 16) {
                float o[16];
                tmem_ld16(tmem + lane_off + TM_O + c, o);
                tmem_wait_ld();
                if (t < a.T) {
                    uint32_t pk[8];
#pragma unroll
                    for (int i = 0; i < 8; ++i) {
                        __nv_bfloat162 p2 = __floats2bfloat162_rn(o[2 * i] * inv, o[2 * i + 1] * inv);
                        pk[i] = *reinterpret_cast<uint32_t*>(&p2);
                    }
                    *reinterpret_cast<uint4*>(orow + c) = make_uint4(pk[0], pk[1], pk[2], pk[3]);
                    *reinterpret_cast<uint4*>(orow + c + 8) = make_uint4(pk[4], pk[5], pk[6], pk[7]);
                }
            }
        }
        tmem_wait_ld();
    }
    tc_fence_before();
    __syncthreads();
    if (warp == kWarpMma) {
        tc_fence_after();
        tmem_dealloc(tmem, 512);
    }
}

// ---------------------------------------------------------------- decode ---------------------
// One token per row against its ring.  The window is a set: softmax over it does not depend on
// the order of its keys, and the ring holds exactly the window -- slots [0, n), n = min(pos + 1,
// w) (slot = position mod w, keys cached after their rotation) -- so the slots are cut into
// tiles of 128 and the tiles of a row into parts ("items") of up to kTilesMax consecutive tiles.
// A persistent CTA takes items blockIdx.x, + gridDim.x, ... and streams their tiles:
//   * a TMA warp brings each tile's keys [128 slots x 256 d], then its values, into a ring of
//     three 64 KB buffers (the row's rotated queries [16 x 256] come with an item's first keys;
//     heads past H read other data, whose columns are never used), 128-byte swizzle;
//   * an MMA warp issues S^T = K Q^T (M = 128 slots, N = 16 heads, K = 256: a TMEM lane is a
//     slot) for tile i, then O^T = V^T P^T (M = 128 d-columns x 2, N = 16, K = 128 slots; V^T is
//     the value tile read MN-major) for tile i - 1, so that the scores of the next tile overlap
//     the softmax of this one; S and O^T are double-buffered in TMEM, P in shared memory;
//   * 4 warps (thread = slot) mask the slots past n, take per head the tile's maximum and sum
//     (shuffles, then across the warps), write p = 2^(s - m) in bf16 as the B operand of the
//     value MMA (value rows past n are zeroed first: an unfilled slot may hold anything), then
//     read tile i - 1's O^T (thread = d-column) and fold it into the item's running (max, sum,
//     sum of p v) per head; an item's last tile writes them for the merge.
// The step reads the ring once (2 w d bf16 per row): it is bound by HBM.
constexpr int kTile = 128;             // slots per tile (the MMA's M)
constexpr int kMaxH = 16;              // heads (the MMA's N), padded
static_assert(kMaxH == kRopeMaxH, "one bound on the heads of a row");
constexpr int kTilesMax = 4;           // tiles per item, at most
constexpr int kNBuf = 3;               // 64 KB tile buffers
constexpr uint32_t KV_BYTES = kTile * D * 2;          // 65536: 4 boxes of [128 slots x 64 d]
constexpr uint32_t QD_BYTES = kMaxH * D * 2;          // 8192: 4 boxes of [16 heads x 64 d]
constexpr uint32_t PD_BYTES = kMaxH * kTile * 2;      // 4096: 2 K blocks of [16 heads x 64 slots]
constexpr uint32_t D_OFF_KV = 0;
constexpr uint32_t D_OFF_Q = D_OFF_KV + kNBuf * KV_BYTES;   // 2 buffers (item parity)
constexpr uint32_t D_OFF_P = D_OFF_Q + 2 * QD_BYTES;        // 2 buffers (tile parity)
constexpr uint32_t D_OFF_RED = D_OFF_P + 2 * PD_BYTES;      // [2][4 warps][16] fp32: maxima, sums
constexpr uint32_t D_OFF_BAR = D_OFF_RED + 2 * 4 * kMaxH * 4;
constexpr uint32_t D_SMEM_BYTES = D_OFF_BAR + 256 + 1024;
static_assert(D_SMEM_BYTES <= 232448, "shared memory budget");
// TMEM: S^T [0, 32) (two buffers of 16 columns), O^T [32, 96) (two buffers of 2 x 16)
constexpr uint32_t D_TM_S = 0, D_TM_O = 32, D_TMEM_COLS = 128;
constexpr int kDecThreads = 6 * 32;    // 4 softmax / epilogue warps, a TMA warp, an MMA warp

struct DecArgs {
    int B, H, w, nsplit, tiles;        // nsplit items per row of `tiles` tiles (the last ragged)
    float scale;
    const int* pos;                    // [B]
    float* part_m;                     // [B][nsplit][H], natural-log units
    float* part_l;
    float* part_o;                     // [B][nsplit][H][d]
    DeviceStatus* status;
    unsigned long long timeout_ns;
};

struct DBars {
    uint32_t base;
    __device__ __forceinline__ uint32_t kv_full(int i) const { return base + 8u * i; }
    __device__ __forceinline__ uint32_t kv_empty(int i) const { return base + 24u + 8u * i; }
    __device__ __forceinline__ uint32_t s_full(int i) const { return base + 48u + 8u * i; }
    __device__ __forceinline__ uint32_t p_full(int i) const { return base + 64u + 8u * i; }   // P written, V rows zeroed
    __device__ __forceinline__ uint32_t o_full(int i) const { return base + 80u + 8u * i; }
    __device__ __forceinline__ uint32_t o_empty(int i) const { return base + 96u + 8u * i; }  // O^T read
    __device__ __forceinline__ uint32_t mma_done() const { return base + 112u; }
};

// An item of the stream: row b, its tiles [t0, t0 + nt) (slot 128 t0 first), cnt valid slots.
struct DecItem {
    int b, sp, s0, cnt, nt;
};
__device__ __forceinline__ DecItem dec_item(const DecArgs& a, int j) {
    DecItem it;
    it.b = j / a.nsplit;
    it.sp = j % a.nsplit;
    it.s0 = it.sp * a.tiles * kTile;
    const int n = min(a.pos[it.b] + 1, a.w);
    it.cnt = max(0, min(n, it.s0 + a.tiles * kTile) - it.s0);
    it.nt = (it.cnt + kTile - 1) / kTile;
    return it;
}

__device__ __noinline__ bool dwait_slow(uint32_t bar, uint32_t parity, const DecArgs& a, volatile int* abort,
                                        unsigned where) {
    const uint64_t t0 = globaltimer_ns();
    for (;;) {
        if (mbar_try_wait_sleep(bar, parity, 20000u)) return true;
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
    }
}
__device__ __forceinline__ bool dwait(uint32_t bar, uint32_t parity, const DecArgs& a, volatile int* abort,
                                      unsigned where) {
    if (mbar_try_wait(bar, parity)) return true;
    return dwait_slow(bar, parity, a, abort, where);
}

// Named barrier 1 over the 4 softmax warps, returning the AND of v over their threads.
__device__ __forceinline__ bool bar_and_128(bool v) {
    uint32_t r;
    asm volatile(
        "{\n\t.reg .pred p, q;\n\t"
        "setp.ne.u32 q, %1, 0;\n\t"
        "barrier.red.and.pred p, 1, 128, q;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(r)
        : "r"((uint32_t)v)
        : "memory");
    return r != 0;
}

// MN-major (128-byte swizzle) descriptor of the value tile read as V^T: atoms of 64 d-columns,
// each [128 slots x 128 B], 16384 B apart
__device__ __forceinline__ uint64_t desc_vt(uint32_t smem_addr) {
    uint64_t d = 0;
    d |= (uint64_t)((smem_addr >> 4) & 0x3FFF);
    d |= (uint64_t)(16384 >> 4) << 16;
    d |= (uint64_t)(1024 >> 4) << 32;
    d |= (uint64_t)1 << 46;
    d |= (uint64_t)2 << 61;
    return d;
}
// fp32 accumulator, bf16 operands, A K-major (a_mn = 0) or MN-major (1), B K-major, M 128, N 16
__device__ __forceinline__ uint32_t idesc_dec(int a_mn) {
    return (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)a_mn << 15) | ((uint32_t)(kMaxH >> 3) << 17) |
           ((uint32_t)(kTile >> 4) << 24);
}

__global__ void __launch_bounds__(kDecThreads, 1)
mqa_decode_kernel(const __grid_constant__ CUtensorMap map_q, const __grid_constant__ CUtensorMap map_kv,
                  const DecArgs a) {
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const uint32_t sbase = smem_u32(smem);
    const DBars bars{sbase + D_OFF_BAR};
    volatile uint32_t* tmem_base_s = reinterpret_cast<volatile uint32_t*>(smem + D_OFF_BAR + 128);
    volatile int* abort = reinterpret_cast<volatile int*>(smem + D_OFF_BAR + 144);
    float* red = reinterpret_cast<float*>(smem + D_OFF_RED);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int H = a.H, nitems = a.B * a.nsplit;
    if (threadIdx.x == 0) {
        for (int i = 0; i < kNBuf; ++i) {
            mbar_init(bars.kv_full(i), 1);
            mbar_init(bars.kv_empty(i), 1);
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(bars.s_full(i), 1);
            mbar_init(bars.p_full(i), 4);
            mbar_init(bars.o_full(i), 1);
            mbar_init(bars.o_empty(i), 4);
        }
        mbar_init(bars.mma_done(), 1);
        *abort = 0;
        fence_barrier_init();
    }
    if (warp == 5) {
        tmem_alloc(smem_u32((const void*)tmem_base_s), D_TMEM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_base_s;
    // the rotated queries and the new ring slot come from the rotation kernel
    asm volatile("griddepcontrol.wait;" ::: "memory");

    if (warp == 4) {
        // ============================ TMA: per tile its keys, then its values =================
        if (lane == 0) {
            uint32_t L = 0;                                   // loads issued
            bool ok = true;
            for (int j = blockIdx.x; ok && j < nitems; j += gridDim.x) {
                const DecItem it = dec_item(a, j);
                const int krow0 = it.b * 2 * a.w + it.s0;
                const int jl = (j - (int)blockIdx.x) / (int)gridDim.x;   // item number within this CTA
                for (int ti = 0; ok && ti < it.nt; ++ti) {
                    for (int kv = 0; ok && kv < 2; ++kv, ++L) {
                        const int buf = (int)(L % kNBuf);
                        const uint32_t use = L / kNBuf;
                        if (use > 0 && !(ok = dwait(bars.kv_empty(buf), (use - 1) & 1, a, abort, 1))) break;
                        const bool q = kv == 0 && ti == 0;
                        mbar_arrive_expect_tx(bars.kv_full(buf), KV_BYTES + (q ? QD_BYTES : 0u));
                        const int row = krow0 + ti * kTile + (kv ? a.w : 0);
                        for (int kb = 0; kb < D / 64; ++kb)
                            tma_load_2d(sbase + D_OFF_KV + buf * KV_BYTES + kb * (kTile * 128), &map_kv, kb * 64, row,
                                        bars.kv_full(buf));
                        if (q)
                            for (int kb = 0; kb < D / 64; ++kb)
                                tma_load_2d(sbase + D_OFF_Q + (jl & 1) * QD_BYTES + kb * (kMaxH * 128), &map_q, kb * 64,
                                            it.b * H, bars.kv_full(buf));
                    }
                }
            }
            // no bulk copy may still be writing shared memory at the exit: the last loads
            // (up to kNBuf of them) have landed
            const uint64_t t0 = globaltimer_ns();
            for (uint32_t l = L > kNBuf ? L - kNBuf : 0; l < L; ++l)
                while (!mbar_try_wait(bars.kv_full(l % kNBuf), (l / kNBuf) & 1) &&
                       globaltimer_ns() - t0 < a.timeout_ns) {
                }
        }
    } else if (warp == 5) {
        // ============================ MMA: S^T of tile i, then O^T of tile i - 1 ==============
        const uint32_t tm = __shfl_sync(0xffffffffu, tmem, 0);
        auto wait_w = [&](uint32_t bar, uint32_t par, unsigned where) {
            return __all_sync(0xffffffffu, dwait(bar, par, a, abort, where));
        };
        bool ok = true;
        uint32_t i = 0;                                       // tiles whose S^T is issued
        auto issue_pv = [&](uint32_t t) -> bool {             // O^T of tile t (V: load 2 t + 1)
            const uint32_t lv = 2 * t + 1, buf = lv % kNBuf;
            if (!wait_w(bars.p_full(t & 1), (t >> 1) & 1, 3)) return false;
            if (!wait_w(bars.kv_full(buf), (lv / kNBuf) & 1, 4)) return false;
            if (t >= 2 && !wait_w(bars.o_empty(t & 1), ((t >> 1) - 1) & 1, 5)) return false;
            tc_fence_after();
            if (elect_one()) {
#pragma unroll
                for (int hh = 0; hh < 2; ++hh)                 // d-columns [128 hh, 128 hh + 128)
#pragma unroll
                    for (int kk = 0; kk < kTile / 16; ++kk) {
                        const uint64_t ad = desc_vt(sbase + D_OFF_KV + buf * KV_BYTES + (2 * hh) * (kTile * 128) + kk * 2048);
                        const uint64_t bd = desc_k_sw128(sbase + D_OFF_P + (t & 1) * PD_BYTES + (kk >> 2) * (kMaxH * 128) +
                                                         (kk & 3) * 32);
                        mma_ss(tm + D_TM_O + (t & 1) * 32 + hh * kMaxH, ad, bd, idesc_dec(1), kk > 0 ? 1u : 0u);
                    }
                mma_commit(bars.o_full(t & 1));
                mma_commit(bars.kv_empty(buf));
            }
            __syncwarp();
            return true;
        };
        for (int j = blockIdx.x; ok && j < nitems; j += gridDim.x) {
            const DecItem it = dec_item(a, j);
            const int jl = (j - (int)blockIdx.x) / (int)gridDim.x;
            for (int ti = 0; ok && ti < it.nt; ++ti, ++i) {
                const uint32_t lk = 2 * i, buf = lk % kNBuf;
                if (!(ok = wait_w(bars.kv_full(buf), (lk / kNBuf) & 1, 2))) break;
                tc_fence_after();
                if (elect_one()) {
#pragma unroll
                    for (int ks = 0; ks < D / 16; ++ks) {
                        const uint64_t ad = desc_k_sw128(sbase + D_OFF_KV + buf * KV_BYTES + (ks >> 2) * (kTile * 128) + (ks & 3) * 32);
                        const uint64_t bd = desc_k_sw128(sbase + D_OFF_Q + (jl & 1) * QD_BYTES + (ks >> 2) * (kMaxH * 128) +
                                                         (ks & 3) * 32);
                        mma_ss(tm + D_TM_S + (i & 1) * kMaxH, ad, bd, idesc_dec(0), ks > 0 ? 1u : 0u);
                    }
                    mma_commit(bars.s_full(i & 1));
                    mma_commit(bars.kv_empty(buf));
                }
                __syncwarp();
                if (i > 0) ok = issue_pv(i - 1);
            }
        }
        if (ok && i > 0) ok = issue_pv(i - 1);
        // every MMA issued here has completed before TMEM is released (also after a failed wait)
        if (elect_one()) mma_commit(bars.mma_done());
        __syncwarp();
        if (lane == 0) {
            const uint64_t t0 = globaltimer_ns();
            while (!mbar_try_wait(bars.mma_done(), 0) && globaltimer_ns() - t0 < a.timeout_ns) {
            }
        }
        __syncwarp();
    } else {
        // ============================ softmax of tile i, then the output of tile i - 1 ========
        const uint32_t lane_off = (uint32_t)(warp * 32) << 16;
        const int r = warp * 32 + lane;                  // slot within a tile (TMEM lane), then d-column
        const float sc = a.scale * 1.4426950408889634f;
        // empty items (a part of the ring past the window): an empty part for the merge
        for (int j = blockIdx.x; j < nitems; j += gridDim.x) {
            const DecItem it = dec_item(a, j);
            if (it.nt > 0) continue;
            const size_t pb = ((size_t)it.b * a.nsplit + it.sp) * H;
            for (int e = threadIdx.x; e < H * D; e += 128) a.part_o[pb * D + e] = 0.f;
            if (threadIdx.x < H) {
                a.part_m[pb + threadIdx.x] = -INFINITY;
                a.part_l[pb + threadIdx.x] = 0.f;
            }
        }
        float M[kMaxH], acc0[kMaxH], acc1[kMaxH], mt[kMaxH];   // item's running max, O; tile's max
        float Lh = 0.f, lt = 0.f;                         // item's running sum, tile's (head r < H)
        bool ok = true;
        uint32_t i = 0;
        int pend_b = -1, pend_sp = 0;                     // item of tile i - 1 and whether it ends it
        bool pend_last = false, pend_first = false;
        // fold tile t's O^T into the item's running values; write them at the item's end
        auto epilogue = [&](uint32_t t) -> bool {
            if (!__all_sync(0xffffffffu, dwait(bars.o_full(t & 1), (t >> 1) & 1, a, abort, 7))) return false;
            tc_fence_after();
            float o0[kMaxH], o1[kMaxH];
            tmem_ld16(tmem + lane_off + D_TM_O + (t & 1) * 32, o0);
            tmem_ld16(tmem + lane_off + D_TM_O + (t & 1) * 32 + kMaxH, o1);
            tmem_wait_ld();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(bars.o_empty(t & 1));
            if (pend_first) {
#pragma unroll
                for (int h = 0; h < kMaxH; ++h) {
                    M[h] = mt[h];
                    acc0[h] = o0[h];
                    acc1[h] = o1[h];
                }
                Lh = lt;
            } else {
                float fo_l = 1.f, fn_l = 1.f;
#pragma unroll
                for (int h = 0; h < kMaxH; ++h) {
                    const float mn = fmaxf(M[h], mt[h]);
                    const float fo = mn == -INFINITY ? 0.f : ex2_approx(M[h] - mn);
                    const float fn = mn == -INFINITY ? 0.f : ex2_approx(mt[h] - mn);
                    acc0[h] = fmaf(acc0[h], fo, o0[h] * fn);
                    acc1[h] = fmaf(acc1[h], fo, o1[h] * fn);
                    M[h] = mn;
                    if (h == r) {
                        fo_l = fo;
                        fn_l = fn;
                    }
                }
                Lh = fmaf(Lh, fo_l, lt * fn_l);
            }
            if (pend_last) {
                const size_t pb = ((size_t)pend_b * a.nsplit + pend_sp) * H;
#pragma unroll
                for (int h = 0; h < kMaxH; ++h)
                    if (h < H) {
                        a.part_o[(pb + h) * D + r] = acc0[h];
                        a.part_o[(pb + h) * D + 128 + r] = acc1[h];
                    }
                if (r < H) {
                    float mh = M[0];
#pragma unroll
                    for (int h = 1; h < kMaxH; ++h)
                        if (h == r) mh = M[h];
                    a.part_m[pb + r] = mh * 0.69314718055994531f;   // natural units
                    a.part_l[pb + r] = Lh;
                }
            }
            return true;
        };
        // The 4 warps meet at named barriers that also AND a flag across them, so that they leave
        // the loop together when any wait failed (a warp that stayed would wait forever).
        bool stop = false;                                // the same in all 4 warps
        for (int j = blockIdx.x; !stop && j < nitems; j += gridDim.x) {
            const DecItem it = dec_item(a, j);
            for (int ti = 0; ti < it.nt; ++ti, ++i) {
                const int cnt = min(kTile, it.cnt - ti * kTile);   // valid slots of the tile
                const bool valid = r < cnt;
                ok = ok && __all_sync(0xffffffffu, dwait(bars.s_full(i & 1), (i >> 1) & 1, a, abort, 6));
                float s[kMaxH];
                if (ok) {
                    tc_fence_after();
                    tmem_ld16(tmem + lane_off + D_TM_S + (i & 1) * kMaxH, s);
                    tmem_wait_ld();
                    // per head: the tile's maximum (in units of log2), across the lanes, then the warps
#pragma unroll
                    for (int h = 0; h < kMaxH; ++h) {
                        float v = valid && h < H ? s[h] * sc : -INFINITY;
                        s[h] = v;
#pragma unroll
                        for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
                        if (lane == 0) red[warp * kMaxH + h] = v;
                    }
                }
                if (!bar_and_128(ok)) {
                    stop = true;
                    break;
                }
                float m[kMaxH];
#pragma unroll
                for (int h = 0; h < kMaxH; ++h)
                    m[h] = fmaxf(fmaxf(red[h], red[kMaxH + h]), fmaxf(red[2 * kMaxH + h], red[3 * kMaxH + h]));
                // p = 2^(s - m) (0 past the window and for padded heads), in bf16 as the B operand
                // [16 heads x 128 slots]: row h, slot r at K block r / 64, 16-byte chunk (r % 64) / 8
                uint8_t* pbuf = smem + D_OFF_P + (i & 1) * PD_BYTES;
                const uint32_t pcol = (uint32_t)(r >> 6) * (kMaxH * 128) + (uint32_t)(r & 7) * 2;
                const uint32_t pch = (uint32_t)((r & 63) >> 3);
#pragma unroll
                for (int h = 0; h < kMaxH; ++h) {
                    const float p = s[h] == -INFINITY ? 0.f : ex2_approx(s[h] - m[h]);
                    *reinterpret_cast<__nv_bfloat16*>(pbuf + pcol + (uint32_t)h * 128 + ((pch ^ (uint32_t)(h & 7)) << 4)) =
                        __float2bfloat16_rn(p);
                    float v = p;
#pragma unroll
                    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
                    if (lane == 0) red[4 * kMaxH + warp * kMaxH + h] = v;
                }
                // value rows of slots past the window (the item's last tile only): zero, once
                // the values have landed (the MMA multiplies them by p = 0)
                if (cnt < kTile) {
                    const uint32_t lv = 2 * i + 1;
                    ok = __all_sync(0xffffffffu, dwait(bars.kv_full(lv % kNBuf), (lv / kNBuf) & 1, a, abort, 8));
                    if (ok && !valid) {
                        uint8_t* vt = smem + D_OFF_KV + (lv % kNBuf) * KV_BYTES + r * 128;
#pragma unroll
                        for (int kb = 0; kb < D / 64; ++kb)
#pragma unroll
                            for (int c = 0; c < 8; ++c)
                                *reinterpret_cast<uint4*>(vt + kb * (kTile * 128) + c * 16) = make_uint4(0, 0, 0, 0);
                    }
                }
                fence_proxy_async_smem();
                tc_fence_before();
                if (!bar_and_128(ok)) {
                    stop = true;
                    break;
                }
                if (lane == 0) mbar_arrive(bars.p_full(i & 1));
                // the previous tile's output (a failed wait there reaches the next barrier as
                // ok = false), then this tile's statistics take its place
                if (i > 0) ok = epilogue(i - 1);
#pragma unroll
                for (int h = 0; h < kMaxH; ++h) mt[h] = m[h];
                lt = 0.f;
                if (r < H) lt = red[4 * kMaxH + r] + red[5 * kMaxH + r] + red[6 * kMaxH + r] + red[7 * kMaxH + r];
                pend_b = it.b;
                pend_sp = it.sp;
                pend_first = ti == 0;
                pend_last = ti == it.nt - 1;
            }
        }
        if (!stop && ok && i > 0) ok = epilogue(i - 1);
    }
    // the merge may be scheduled once every CTA is past its work (it waits for this grid)
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    tc_fence_before();
    __syncthreads();
    if (warp == 5) {
        tc_fence_after();
        tmem_dealloc(tmem, D_TMEM_COLS);
    }
}

struct MergeArgs {
    int B, H, nsplit;
    const float* part_m;
    const float* part_l;
    const float* part_o;
    __nv_bfloat16* out;                // [B, H, d]
};

// Block = (head, row), thread = 4 d-columns: few enough threads that all are resident at once,
// each with its loads of the parts in flight together.
constexpr int kMergeThreads = D / 4;
__global__ void __launch_bounds__(kMergeThreads) mqa_merge_kernel(MergeArgs a) {
    asm volatile("griddepcontrol.wait;" ::: "memory");   // the parts of the attention kernel
    const int h = blockIdx.x, b = blockIdx.y, c = threadIdx.x;
    const size_t rb = (size_t)b * a.nsplit * a.H + h;   // part s of (b, h): rb + s H
    float mx = -INFINITY;
    for (int s = 0; s < a.nsplit; ++s) mx = fmaxf(mx, a.part_m[rb + (size_t)s * a.H]);
    float l = 0.f;
    float4 o = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int s = 0; s < a.nsplit; ++s) {
        const size_t ps = rb + (size_t)s * a.H;
        const float m = a.part_m[ps];
        if (m == -INFINITY) continue;
        const float f = expf(m - mx);
        l = fmaf(a.part_l[ps], f, l);
        const float4 v = reinterpret_cast<const float4*>(a.part_o + ps * D)[c];
        o = make_float4(fmaf(v.x, f, o.x), fmaf(v.y, f, o.y), fmaf(v.z, f, o.z), fmaf(v.w, f, o.w));
    }
    const float il = l > 0.f ? 1.0f / l : 0.f;
    const __nv_bfloat162 lo = __floats2bfloat162_rn(o.x * il, o.y * il), hi = __floats2bfloat162_rn(o.z * il, o.w * il);
    uint2 pk;
    pk.x = *reinterpret_cast<const uint32_t*>(&lo);
    pk.y = *reinterpret_cast<const uint32_t*>(&hi);
    *reinterpret_cast<uint2*>(a.out + ((size_t)b * a.H + h) * D + 4 * c) = pk;
}

}  // namespace mq

// --------------------------------------------------------------------------- host side ------

bool mqa_supported(const rglru_mqa_dims* d) {
    return d->head_dim == mq::D && d->q_heads >= 1 && d->q_heads <= mq::kMaxH && d->window >= 1;
}

namespace {
struct MqaLayout {
    size_t q_rot, k_rot, part_m, part_l, part_o, total;
    int nsplit, per;
};
MqaLayout mqa_layout(const rglru_mqa_dims* d, bool decode) {
    auto up = [](size_t v) { return (v + 255) & ~size_t(255); };
    MqaLayout l{};
    const size_t T = decode ? 1 : (size_t)d->seq_len;
    size_t o = 256;
    l.q_rot = o; o = up(o + (size_t)d->batch * T * d->q_heads * mq::D * 2);
    l.k_rot = o; o = up(o + (size_t)d->batch * T * mq::D * 2);
    l.per = mq::kTile;
    l.nsplit = (d->window + l.per - 1) / l.per;       // the most parts a row is cut into
    l.part_m = o; o = up(o + (size_t)d->batch * l.nsplit * d->q_heads * 4);
    l.part_l = o; o = up(o + (size_t)d->batch * l.nsplit * d->q_heads * 4);
    l.part_o = o; o = up(o + (size_t)d->batch * l.nsplit * d->q_heads * mq::D * 4);
    l.total = o;
    return l;
}
}  // namespace

size_t mqa_workspace(const rglru_mqa_dims* d, bool decode) { return mqa_layout(d, decode).total; }

cudaError_t launch_mqa_prefill(const rglru_mqa_dims* d, const void* q, const void* k, const void* v, int pos0,
                               void* out, void* cache, void* ws, size_t ws_bytes, cudaStream_t s) {
    using namespace mq;
    const MqaLayout l = mqa_layout(d, false);
    if (l.total > ws_bytes) return cudaErrorInvalidValue;
    uint8_t* w = static_cast<uint8_t*>(ws);
    const int B = d->batch, T = d->seq_len, H = d->q_heads;
    RopeArgs ra{};
    ra.B = B; ra.T = T; ra.H = H; ra.w = d->window; ra.pos0 = pos0; ra.base = d->rope_base;
    ra.q = static_cast<const __nv_bfloat16*>(q); ra.k = static_cast<const __nv_bfloat16*>(k);
    ra.v = static_cast<const __nv_bfloat16*>(v);
    ra.q_rot = reinterpret_cast<__nv_bfloat16*>(w + l.q_rot);
    ra.k_rot = reinterpret_cast<__nv_bfloat16*>(w + l.k_rot);
    ra.cache = static_cast<__nv_bfloat16*>(cache);
    mqa_rope_kernel<<<dim3(T, B), D / 2, 0, s>>>(ra);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    // tensor maps: queries as a 3-D [B T rows][H][d] tensor (box 64 x 1 head x 128 rows),
    // keys and values as 2-D [B T rows][d] (box 64 x 64 rows), all in the 128-byte swizzle
    CUtensorMap mqm, mkm, mvm;
    if (!tc::make_map_3d_box_sw128(&mqm, ra.q_rot, D, (uint64_t)H, (uint64_t)B * T, 64, 1, BQ) ||
        !tc::make_map_2d_sw128(&mkm, ra.k_rot, D, (uint64_t)B * T, D * 2, 64, BKV) ||
        !tc::make_map_2d_sw128(&mvm, v, D, (uint64_t)B * T, D * 2, 64, BKV))
        return cudaErrorInvalidValue;
    e = set_smem_once(mqa_prefill_kernel, (int)SMEM_BYTES);
    if (e != cudaSuccess) return e;
    PrefArgs pa{};
    pa.B = B; pa.T = T; pa.H = H; pa.w = d->window;
    pa.scale_log2 = d->scale * kLog2e;
    pa.out = static_cast<__nv_bfloat16*>(out);
    pa.status = reinterpret_cast<DeviceStatus*>(w);
    pa.timeout_ns = 1000000000ull;
    mqa_prefill_kernel<<<dim3((T + BQ - 1) / BQ, H, B), kThreads, SMEM_BYTES, s>>>(mqm, mkm, mvm, pa);
    return cudaGetLastError();
}

cudaError_t launch_mqa_decode(const rglru_mqa_dims* d, const void* q, const void* k, const void* v, const int* pos,
                              void* cache, void* out, void* ws, size_t ws_bytes, cudaStream_t s) {
    using namespace mq;
    const MqaLayout l = mqa_layout(d, true);
    if (l.total > ws_bytes) return cudaErrorInvalidValue;
    uint8_t* w = static_cast<uint8_t*>(ws);
    const int B = d->batch, H = d->q_heads;
    RopeDecArgs ra{};
    ra.B = B; ra.H = H; ra.w = d->window; ra.base = d->rope_base; ra.pos = pos;
    ra.q = static_cast<const __nv_bfloat16*>(q); ra.k = static_cast<const __nv_bfloat16*>(k);
    ra.v = static_cast<const __nv_bfloat16*>(v);
    ra.q_rot = reinterpret_cast<__nv_bfloat16*>(w + l.q_rot);
    ra.cache = static_cast<__nv_bfloat16*>(cache);
    mqa_rope_decode_kernel<<<B, D / 2, 0, s>>>(ra);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    // the rotated queries as a 2-D [B H rows][d] tensor (box 64 x 16 rows: a row's heads, padded
    // with the next row's or with zeros), the ring as 2-D [B 2 w rows][d] (box 64 x 128 slots)
    CUtensorMap mqm, mkv;
    if (!tc::make_map_2d_sw128(&mqm, ra.q_rot, D, (uint64_t)B * H, D * 2, 64, kMaxH) ||
        !tc::make_map_2d_sw128(&mkv, ra.cache, D, (uint64_t)B * 2 * d->window, D * 2, 64, kTile))
        return cudaErrorInvalidValue;
    e = set_smem_once(mqa_decode_kernel, (int)D_SMEM_BYTES);
    if (e != cudaSuccess) return e;
    int dev = 0, sms = 0;
    if ((e = cudaGetDevice(&dev)) != cudaSuccess) return e;
    if ((e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess) return e;
    // tiles per item: up to kTilesMax while the items still give every SM about two
    const int tiles_row = (d->window + kTile - 1) / kTile;
    const int tpi = std::max(1, std::min(kTilesMax, (int)(((long long)B * tiles_row) / (2LL * sms))));
    DecArgs da{};
    da.B = B; da.H = H; da.w = d->window; da.tiles = tpi; da.nsplit = (tiles_row + tpi - 1) / tpi;
    da.scale = d->scale;
    da.pos = pos;
    da.part_m = reinterpret_cast<float*>(w + l.part_m);
    da.part_l = reinterpret_cast<float*>(w + l.part_l);
    da.part_o = reinterpret_cast<float*>(w + l.part_o);
    da.status = reinterpret_cast<DeviceStatus*>(w);
    da.timeout_ns = 1000000000ull;
    // the attention and merge kernels are programmatic dependents of the kernel before them:
    // each one's launch and set-up overlap its predecessor's run
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)std::min(B * da.nsplit, sms));
    cfg.blockDim = dim3(kDecThreads);
    cfg.dynamicSmemBytes = D_SMEM_BYTES;
    cfg.stream = s;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    e = cudaLaunchKernelEx(&cfg, mqa_decode_kernel, mqm, mkv, da);
    if (e != cudaSuccess) return e;
    MergeArgs ma{};
    ma.B = B; ma.H = H; ma.nsplit = da.nsplit;
    ma.part_m = da.part_m; ma.part_l = da.part_l; ma.part_o = da.part_o;
    ma.out = static_cast<__nv_bfloat16*>(out);
    cudaLaunchConfig_t mcfg = {};
    mcfg.gridDim = dim3(H, B);
    mcfg.blockDim = dim3(kMergeThreads);
    mcfg.stream = s;
    mcfg.attrs = attr;
    mcfg.numAttrs = 1;
    return cudaLaunchKernelEx(&mcfg, mqa_merge_kernel, ma);
}

}  // namespace rglru
