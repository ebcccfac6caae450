// gemm.cu -- batched bf16 GEMM on the 5th-generation tensor cores (sm_100a) for the dense
// contractions around the recurrence: the transposed gate contraction and the weight gradient
// of the backward pass.
//
//   C[b][m][n] (fp32) = sum over the operand pairs p of sum_k A_p[b][m][k] B_p[b][k][n]
//                       (+ Cadd[b][m][n]),  for m < M, n < N;
// with up to four operand pairs (K ranges accumulated into one C: both gates, or the hi and lo
// bf16 parts of an fp32 operand) and an
// optional split of K into `splits` slices whose partial sums go to separate C slices (a
// reduction in fixed order follows, so results are bitwise repeatable).
//
//   * A is [M x K] "K-major" (k contiguous: element (m, k) at a_row[m] + k) or "M-major" (m
//     contiguous: element (m, k) at k * ld + m); B likewise N x K, "K-major" or "N-major".  The
//     operands are read by TMA in 128-byte swizzled tiles straight from the caller's tensors
//     (2-D maps; the batch index adds a fixed row or column offset);
//   * a persistent pair of CTAs (a 2-CTA cluster on neighbouring SMs) walks output tiles of
//     256 x 256 (batch, m-tile, n-tile, k-slice) with tcgen05.mma.cta_group::2 (M = 256, N = 256,
//     K = 16 per instruction): each CTA holds half of A (128 rows) and half of B (128 columns)
//     of every 64-wide K block, two K blocks to a stage of a 3-stage ring (64 KB a stage: the
//     loads and the MMAs of a stage share one barrier round trip), so a CTA moves 2/3 of the
//     bytes a 128 x 256 tile would for the same flops and has more of them in flight; the
//     leader CTA's MMA warp issues for both, its commits arrive on both CTAs' barriers, and
//     its ring barriers count both CTAs' TMA bytes (the partner's loads complete on the
//     leader's barrier).  Each CTA's accumulator half (its 128 rows x 256 columns, two TMEM
//     buffers) is read by its 8 epilogue warps (two per TMEM lane quadrant, 128 columns each)
//     32 columns at a time through a swizzled shared-memory tile, so that Cadd is read and C
//     written in whole 128-byte row segments; they hand the buffer back to the leader.
//   * no multicast loads: each CTA's TMA reads only its own halves.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <mutex>

#include "common.cuh"
#include "kernels.h"
#include "sm100.cuh"
#include "tma_maps.h"

namespace rglru {
namespace gm {

using namespace sm100;

constexpr int BM = 128, BN = 256, BK = 64;         // BM rows per CTA (256 per pair), BN columns
constexpr int BNH = BN / 2;                        // B columns a CTA loads
constexpr int KPS = 2;                             // 64-wide K blocks per ring stage
constexpr int STAGES = 3;
constexpr uint32_t TILE_A = BM * BK * 2;           // 16384: a CTA's half of A for one K block
constexpr uint32_t TILE_B = BNH * BK * 2;          // 16384
constexpr uint32_t STAGE_BYTES = KPS * (TILE_A + TILE_B);   // [A blocks][B blocks]
constexpr uint32_t OFF_BAR = STAGES * STAGE_BYTES;
// per epilogue warp, a [32 rows x 32 columns] fp32 staging tile (rows of 128 B, 16-byte chunks
// XOR-swizzled by the row): the warp's accumulator rows go in row by row and come out as whole
// 128-byte row segments, so that global loads and stores are coalesced
constexpr uint32_t OFF_STG = OFF_BAR + 256;
constexpr uint32_t STG_BYTES = 32 * 32 * 4;
constexpr uint32_t SMEM_BYTES = OFF_STG + 8 * STG_BYTES + 1024;
static_assert(SMEM_BYTES <= 232448, "shared memory budget");
constexpr int kEpiWarps = 8, kWarpTma = 8, kWarpMma = 9;   // two epilogue warps per TMEM lane quadrant
constexpr int kThreads = 10 * 32;
constexpr uint32_t TMEM_COLS = 2 * BN;
constexpr int kMaxPairs = 4;

struct Pair {
    int K;               // K of this pair (a multiple of 64)
    int a_kmajor;        // 1: A (m, k) at row m, column k of its map; 0: row k, column m
    int b_kmajor;        // 1: B (n, k) at row n, column k;             0: row k, column n
    int a_boff_row, a_boff_col, a_bstep_row, a_bstep_col;   // A's map coordinates: boff + b * bstep
    int b_boff_row, b_boff_col, b_bstep_row, b_bstep_col;
};

struct Args {
    int M, N, batch, splits, npairs;
    int interleave;      // every pair has the same K: their K blocks alternate
    int mt, nt;          // tiles along M and N
    Pair p[kMaxPairs];
    float* C;            // C[split][b][m][n] at C + split * c_split + b * c_bstride + m * c_ld + n
    long long c_ld, c_bstride, c_split;
    const float* Cadd;   // same indexing without the split, or nullptr (only with splits == 1)
    long long add_ld, add_bstride;
    __nv_bfloat16* C16;  // if set: C is written here as bf16 (round to nearest even) instead
    DeviceStatus* status;
    unsigned long long timeout_ns;
};

// K blocks of one output tile: when every pair has the same K, block kb is block kb / npairs of
// pair kb % npairs (the pairs interleaved, so that an operand shared by two pairs -- the hi part
// of xc against both parts of dg -- is read twice within a few blocks and the second read hits
// L2); otherwise the blocks of pair 0, then those of pair 1, ...  Cut into `splits` equal slices
// (the last may be shorter).
struct KPlan {
    int total, per;      // blocks in all, blocks per slice
};
__host__ __device__ inline KPlan kplan(const Args& a) {
    KPlan k;
    k.total = 0;
    for (int i = 0; i < a.npairs; ++i) k.total += a.p[i].K / BK;
    k.per = (k.total + a.splits - 1) / a.splits;
    return k;
}
// the pair of K block kb and the block's index within that pair
__device__ __forceinline__ int pair_of(const Args& a, int kb, int& local) {
    if (a.interleave) {
        local = kb / a.npairs;
        return kb % a.npairs;
    }
    int i = 0;
    while (i + 1 < a.npairs && kb >= a.p[i].K / BK) {
        kb -= a.p[i].K / BK;
        ++i;
    }
    local = kb;
    return i;
}

__device__ __noinline__ bool wait_slow(uint32_t bar, uint32_t parity, const Args& a, volatile int* abort, unsigned where) {
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
__device__ __forceinline__ bool wait_b(uint32_t bar, uint32_t parity, const Args& a, volatile int* abort, unsigned where) {
    if (mbar_try_wait(bar, parity)) return true;
    return wait_slow(bar, parity, a, abort, where);
}

// Shared-memory descriptors (128-byte swizzle) of a 128- or 256-row, 64-wide tile: K-major (rows
// of 128 B = 64 K, 8-row atoms 1024 B apart) or MN-major (64-wide MN atoms of 64 K-rows each,
// 8192 B apart; 8-row K groups 1024 B apart)
__device__ __forceinline__ uint64_t desc_mn_sw128(uint32_t smem_addr) {
    uint64_t d = 0;
    d |= (uint64_t)((smem_addr >> 4) & 0x3FFF);
    d |= (uint64_t)(8192 >> 4) << 16;
    d |= (uint64_t)(1024 >> 4) << 32;
    d |= (uint64_t)1 << 46;
    d |= (uint64_t)2 << 61;
    return d;
}
// instruction descriptor: fp32 accumulator, bf16 A and B, their majorness, M (the pair's 256
// rows) x N
__device__ __forceinline__ uint32_t idesc(int a_mn, int b_mn) {
    return (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)a_mn << 15) | ((uint32_t)b_mn << 16) |
           ((uint32_t)(BN >> 3) << 17) | ((uint32_t)((2 * BM) >> 4) << 24);
}

// ---- the CTA pair: every tcgen05 instruction of this kernel is of cta_group::2
__device__ __forceinline__ void tmem_alloc_pair(uint32_t dst_smem, uint32_t ncols) {
    asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(dst_smem), "r"(ncols)
                 : "memory");
}
__device__ __forceinline__ void tmem_relinquish_pair() {
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc_pair(uint32_t taddr, uint32_t ncols) {
    asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}
// D (both CTAs' TMEM) (+)= A (both CTAs' halves) * B (both CTAs' halves)^T
__device__ __forceinline__ void mma_ss_pair(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t id,
                                            uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
        "l"(a_desc), "l"(b_desc), "r"(id), "r"(accumulate)
        : "memory");
}
// arrive on the mbarrier at this shared address in both CTAs of the pair once every prior MMA
// of this thread completes
__device__ __forceinline__ void mma_commit_pair(uint32_t bar) {
    asm volatile(
        "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64 [%0], %1;" ::"r"(bar),
        "h"((uint16_t)3)
        : "memory");
}
// a tile of this CTA's half into its own shared memory, its bytes counted on the leader's
// barrier (a shared::cluster address)
__device__ __forceinline__ void tma_load_2d_pair(uint32_t dst, const CUtensorMap* map, int c0, int c1, uint32_t bar) {
    asm volatile(
        "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%2, %3}], [%4];" ::"r"(dst),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(c0), "r"(c1), "r"(bar)
        : "memory");
}
// waits on barriers that other CTAs of the pair arrive on (cluster-scope acquire)
__device__ __noinline__ bool wait_slow_c(uint32_t bar, uint32_t parity, const Args& a, volatile int* abort,
                                        unsigned where) {
    const uint64_t t0 = globaltimer_ns();
    for (uint32_t it = 0;; ++it) {
        if (mbar_try_wait_cluster(bar, parity)) return true;
        if (it > 64) __nanosleep(200);
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
__device__ __forceinline__ bool wait_c(uint32_t bar, uint32_t parity, const Args& a, volatile int* abort, unsigned where) {
    if (mbar_try_wait_cluster(bar, parity)) return true;
    return wait_slow_c(bar, parity, a, abort, where);
}

// NP: the number of operand pairs (a compile-time constant, so that the producer's per-pair
// selections fold away for a single pair)
template <int NP>
__global__ void __launch_bounds__(kThreads, 1)
gemm_kernel(const __grid_constant__ CUtensorMap ma0, const __grid_constant__ CUtensorMap mb0,
            const __grid_constant__ CUtensorMap ma1, const __grid_constant__ CUtensorMap mb1,
            const __grid_constant__ CUtensorMap ma2, const __grid_constant__ CUtensorMap mb2,
            const __grid_constant__ CUtensorMap ma3, const __grid_constant__ CUtensorMap mb3, const Args a) {
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const uint32_t sbase = smem_u32(smem);
    const uint32_t bar0 = sbase + OFF_BAR;
    auto full = [&](int s) { return bar0 + 8u * s; };
    auto empty = [&](int s) { return bar0 + 8u * (STAGES + s); };
    auto acc_full = [&](int i) { return bar0 + 8u * (2 * STAGES + i); };
    auto acc_empty = [&](int i) { return bar0 + 8u * (2 * STAGES + 2 + i); };
    const uint32_t mma_done = bar0 + 8u * (2 * STAGES + 4);
    volatile uint32_t* tmem_base_s = reinterpret_cast<volatile uint32_t*>(smem + OFF_BAR + 8 * (2 * STAGES + 5));
    volatile int* abort = reinterpret_cast<volatile int*>(smem + OFF_BAR + 8 * (2 * STAGES + 5) + 16);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t rank = cluster_ctarank();             // 0: the leader, which issues the MMAs
    const int pair = blockIdx.x >> 1, npair = gridDim.x >> 1;

    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(full(s), 1);                       // the leader's arrival + both CTAs' bytes
            mbar_init(empty(s), 1);
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(acc_full(i), 1);
            mbar_init(acc_empty(i), 2 * kEpiWarps);      // the epilogue warps of both CTAs
        }
        mbar_init(mma_done, 1);
        *abort = 0;
        fence_barrier_init();
    }
    if (warp == kWarpMma) {
        tmem_alloc_pair(smem_u32((const void*)tmem_base_s), TMEM_COLS);
        tmem_relinquish_pair();
    }
    if (warp == kWarpTma && lane == 0) {
        prefetch_tensormap(&ma0);
        prefetch_tensormap(&mb0);
        if (NP > 1) {
            prefetch_tensormap(&ma1);
            prefetch_tensormap(&mb1);
        }
        if (NP > 2) {
            prefetch_tensormap(&ma2);
            prefetch_tensormap(&mb2);
        }
        if (NP > 3) {
            prefetch_tensormap(&ma3);
            prefetch_tensormap(&mb3);
        }
    }
    tc_fence_before();
    __syncthreads();
    cluster_sync();                                      // both CTAs' barriers exist before any remote arrival
    tc_fence_after();
    const uint32_t tmem = *tmem_base_s;
    const KPlan kp = kplan(a);
    const int ntiles = a.batch * a.mt * a.nt * a.splits;

    auto tile_of = [&](int t, int& b, int& m0, int& n0, int& sp) {
        sp = t % a.splits;
        t /= a.splits;
        const int ni = t % a.nt;
        t /= a.nt;
        const int mi = t % a.mt;
        b = t / a.mt;
        m0 = mi * (2 * BM);
        n0 = ni * BN;
    };

    // the operand pairs share their majorness (checked on the host): one instruction descriptor,
    // and descriptor steps per K step of 16 -- 32 bytes along a K-major row, or 16 K-rows (2048
    // bytes) of an MN-major tile, i.e. 2 or 128 in the descriptor's address field
    const bool akm = a.p[0].a_kmajor != 0, bkm = a.p[0].b_kmajor != 0;
    const uint32_t id = idesc(akm ? 0 : 1, bkm ? 0 : 1);
    const uint64_t a_step = akm ? 2 : 128, b_step = bkm ? 2 : 128;
    // (pair, block within the pair) of K block kb, then advanced one block at a time
    auto advance = [&](int& pi, int& local) {
        if (a.interleave) {
            if (++pi == NP) {
                pi = 0;
                ++local;
            }
        } else if (++local == a.p[pi].K / BK) {
            local = 0;
            ++pi;
        }
    };

    if (warp == kWarpTma) {
        if (lane == 0) {
            // this CTA's halves: A rows [m0 + 128 rank, + 128), B columns [n0 + 128 rank, + 128);
            // their bytes complete on the leader's full barrier, which the leader arms for both
            const int rb = (int)rank * BM;
            const uint32_t fb0 = map_to_rank(full(0), 0);
            int s = 0;
            uint32_t ph = 0;
            int issued = 0;
            bool ok = true;
            for (int t = pair; t < ntiles && ok; t += npair) {
                int b, m0, n0, sp;
                tile_of(t, b, m0, n0, sp);
                const int k_beg = sp * kp.per, k_end = min(kp.total, k_beg + kp.per);
                // the tile's operand coordinates per pair (selected by value: no indexed arrays)
                int ar[NP], ac[NP], br[NP], bc[NP];
#pragma unroll
                for (int i = 0; i < NP; ++i) {
                    ar[i] = a.p[i].a_boff_row + b * a.p[i].a_bstep_row + (akm ? m0 + rb : 0);
                    ac[i] = a.p[i].a_boff_col + b * a.p[i].a_bstep_col + (akm ? 0 : m0 + rb);
                    br[i] = a.p[i].b_boff_row + b * a.p[i].b_bstep_row + (bkm ? n0 + rb : 0);
                    bc[i] = a.p[i].b_boff_col + b * a.p[i].b_bstep_col + (bkm ? 0 : n0 + rb);
                }
                int pi = 0, local = 0;
                if (k_beg < k_end) pi = pair_of(a, k_beg, local);
                for (int kb = k_beg; kb < k_end; kb += KPS) {
                    if (!wait_c(empty(s), ph ^ 1, a, abort, 1)) {
                        ok = false;
                        break;
                    }
                    const int nb = min(KPS, k_end - kb);     // K blocks in this stage
                    const uint32_t fb = fb0 + 8u * s;
                    if (rank == 0) mbar_arrive_expect_tx(full(s), 2u * (uint32_t)nb * (TILE_A + TILE_B));
#pragma unroll
                    for (int j = 0; j < KPS; ++j) {
                        if (j >= nb) break;
                        const int k0 = local * BK;
                        const CUtensorMap* ma = &ma0;
                        const CUtensorMap* mb = &mb0;
                        int arr = ar[0], acc_ = ac[0], brr = br[0], bcc = bc[0];
#pragma unroll
                        for (int i = 1; i < NP; ++i)
                            if (pi == i) {
                                ma = i == 1 ? &ma1 : i == 2 ? &ma2 : &ma3;
                                mb = i == 1 ? &mb1 : i == 2 ? &mb2 : &mb3;
                                arr = ar[i];
                                acc_ = ac[i];
                                brr = br[i];
                                bcc = bc[i];
                            }
                        const uint32_t sa = sbase + s * STAGE_BYTES + j * TILE_A;
                        const uint32_t sb = sbase + s * STAGE_BYTES + KPS * TILE_A + j * TILE_B;
                        if (akm) {
                            tma_load_2d_pair(sa, ma, acc_ + k0, arr, fb);
                        } else {
                            tma_load_2d_pair(sa, ma, acc_, arr + k0, fb);
                            tma_load_2d_pair(sa + 8192, ma, acc_ + 64, arr + k0, fb);
                        }
                        if (bkm) {
                            tma_load_2d_pair(sb, mb, bcc + k0, brr, fb);
                        } else {
                            tma_load_2d_pair(sb, mb, bcc, brr + k0, fb);
                            tma_load_2d_pair(sb + 8192, mb, bcc + 64, brr + k0, fb);
                        }
                        advance(pi, local);
                    }
                    ++issued;
                    if (++s == STAGES) {
                        s = 0;
                        ph ^= 1;
                    }
                }
            }
            // never leave the pair with a bulk copy still writing shared memory: the leader sees
            // every load of both CTAs land on its barriers (the partner waits for it below)
            if (rank == 0) {
                const uint64_t t0 = globaltimer_ns();
                for (int i = issued - STAGES; i < issued; ++i)
                    if (i >= 0)
                        while (!mbar_try_wait_cluster(full(i % STAGES), (i / STAGES) & 1) &&
                               globaltimer_ns() - t0 < a.timeout_ns) {
                        }
            }
        }
    } else if (warp == kWarpMma) {
        // the leader's warp follows the waits (warp-uniform control flow); one elected lane
        // issues for the pair.  The partner's warp only waits for the pair's last MMA.
        const uint32_t tm = __shfl_sync(0xffffffffu, tmem, 0);
        if (rank == 0) {
            int s = 0, tc = 0;
            uint32_t ph = 0;
            bool ok = true;
            const uint64_t da0 = akm ? desc_k_sw128(sbase) : desc_mn_sw128(sbase);
            const uint64_t db0 = bkm ? desc_k_sw128(sbase + KPS * TILE_A) : desc_mn_sw128(sbase + KPS * TILE_A);
            for (int t = pair; t < ntiles && ok; t += npair, ++tc) {
                int b, m0, n0, sp;
                tile_of(t, b, m0, n0, sp);
                const int k_beg = sp * kp.per, k_end = min(kp.total, k_beg + kp.per);
                const int ai = tc & 1;
                if (!__all_sync(0xffffffffu, wait_c(acc_empty(ai), ((tc >> 1) & 1) ^ 1, a, abort, 2))) break;
                tc_fence_after();
                const uint32_t d = tm + ai * BN;
                for (int kb = k_beg; kb < k_end; kb += KPS) {
                    if (!__all_sync(0xffffffffu, wait_c(full(s), ph, a, abort, 3))) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const int nb = min(KPS, k_end - kb);
                    if (elect_one()) {
                        // block j of stage s: the stage base's descriptor plus the byte offset / 16;
                        // the same offsets address the partner's halves
#pragma unroll
                        for (int j = 0; j < KPS; ++j) {
                            if (j >= nb) break;
                            const uint64_t ad = da0 + (uint64_t)((s * STAGE_BYTES + j * TILE_A) >> 4);
                            const uint64_t bd = db0 + (uint64_t)((s * STAGE_BYTES + j * TILE_B) >> 4);
#pragma unroll
                            for (int kk = 0; kk < BK / 16; ++kk)
                                mma_ss_pair(d, ad + kk * a_step, bd + kk * b_step, id,
                                            (kb > k_beg || j > 0 || kk > 0) ? 1u : 0u);
                        }
                        mma_commit_pair(empty(s));
                    }
                    __syncwarp();
                    if (++s == STAGES) {
                        s = 0;
                        ph ^= 1;
                    }
                }
                if (!ok) break;
                if (elect_one()) mma_commit_pair(acc_full(ai));
                __syncwarp();
            }
            // every MMA has finished (in both CTAs' TMEM) before TMEM is released
            if (elect_one()) mma_commit_pair(mma_done);
            __syncwarp();
        }
        if (lane == 0) {
            const uint64_t t0 = globaltimer_ns();
            while (!mbar_try_wait_cluster(mma_done, 0) && globaltimer_ns() - t0 < a.timeout_ns) {
            }
        }
        __syncwarp();
    } else {
        // ================================ epilogue: thread = row of the tile ==================
        // warp w reads lane quadrant w % 4 (the TMEM lanes a warp may access) and the columns
        // [128 (w / 4), 128 (w / 4) + 128) of this CTA's 128 rows of the tile
        const int q = warp & 3;
        const int cb = (warp >> 2) * (BN / 2);
        int tc = 0;
        for (int t = pair; t < ntiles; t += npair, ++tc) {
            int b, m0, n0, sp;
            tile_of(t, b, m0, n0, sp);
            m0 += (int)rank * BM;                        // this CTA's rows
            const int ai = tc & 1;
            if (!__all_sync(0xffffffffu, wait_c(acc_full(ai), (tc >> 1) & 1, a, abort, 4))) break;
            tc_fence_after();
            // a K slice without blocks (more slices than K blocks) contributes zeros: its
            // accumulator was never written
            const bool no_k = sp * kp.per >= kp.total;
            uint8_t* stg = smem + OFF_STG + (uint32_t)warp * STG_BYTES;
            const long long tbase = sp * a.c_split + b * a.c_bstride;
            const long long abase = b * a.add_bstride;
#pragma unroll 1
            for (int c0 = cb; c0 < cb + BN / 2; c0 += 32) {
                float v0[16], v1[16];
                if (no_k) {
#pragma unroll
                    for (int j = 0; j < 16; ++j) v0[j] = v1[j] = 0.f;
                } else {
                    const uint32_t ta = tmem + ((uint32_t)(q * 32) << 16) + ai * BN + c0;
                    tmem_ld16(ta, v0);
                    tmem_ld16(ta + 16, v1);
                    tmem_wait_ld();
                }
                // row `lane` of the warp's 32 rows into the staging tile
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    *reinterpret_cast<float4*>(stg + lane * 128 + ((j ^ (lane & 7)) << 4)) =
                        make_float4(v0[4 * j], v0[4 * j + 1], v0[4 * j + 2], v0[4 * j + 3]);
                    *reinterpret_cast<float4*>(stg + lane * 128 + (((j + 4) ^ (lane & 7)) << 4)) =
                        make_float4(v1[4 * j], v1[4 * j + 1], v1[4 * j + 2], v1[4 * j + 3]);
                }
                __syncwarp();
                // out as 4 rows x 32 columns per step: lane = (row 4 i + lane / 8, 4 columns); every
                // Cadd load is issued before any store (C may be Cadd itself, accumulated in place)
                float4 add[8];
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                    const int m = m0 + q * 32 + 4 * i + (lane >> 3), n = n0 + c0 + 4 * (lane & 7);
                    add[i] = a.Cadd && m < a.M && n < a.N
                                 ? *reinterpret_cast<const float4*>(a.Cadd + abase + (long long)m * a.add_ld + n)
                                 : make_float4(0.f, 0.f, 0.f, 0.f);
                }
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                    const int rr = 4 * i + (lane >> 3), cc = lane & 7;
                    float4 o = *reinterpret_cast<const float4*>(stg + rr * 128 + ((cc ^ (rr & 7)) << 4));
                    const int m = m0 + q * 32 + rr, n = n0 + c0 + 4 * cc;
                    if (m < a.M && n < a.N) {                // N is a multiple of 16: n + 3 < N too
                        const long long off = tbase + (long long)m * a.c_ld + n;
                        if (a.C16) {
                            __nv_bfloat162 p0 = __floats2bfloat162_rn(o.x, o.y), p1 = __floats2bfloat162_rn(o.z, o.w);
                            *reinterpret_cast<uint2*>(a.C16 + off) =
                                make_uint2(*reinterpret_cast<uint32_t*>(&p0), *reinterpret_cast<uint32_t*>(&p1));
                        } else {
                            o.x += add[i].x; o.y += add[i].y; o.z += add[i].z; o.w += add[i].w;
                            *reinterpret_cast<float4*>(a.C + off) = o;
                        }
                    }
                }
                __syncwarp();
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive_cluster(map_to_rank(acc_empty(ai), 0));   // the leader's barrier
        }
        tmem_wait_ld();
    }
    // no CTA of the pair leaves while the other may still reach its shared memory or TMEM
    tc_fence_before();
    __syncthreads();
    cluster_sync();
    if (warp == kWarpMma) {
        tc_fence_after();
        tmem_dealloc_pair(tmem, TMEM_COLS);
    }
}

// one 2-D bf16 map over a [rows x cols] row-major tensor (row pitch ld elements), box 64 x box_rows
bool map_2d(CUtensorMap* m, const void* base, long long rows, long long cols, long long ld, int box_rows) {
    return tc::make_map_2d_sw128(m, base, (uint64_t)cols, (uint64_t)rows, (uint64_t)ld * 2, 64, (uint32_t)box_rows);
}

}  // namespace gm

size_t gemm_smem_bytes() { return gm::SMEM_BYTES; }

// See kernels.h for the operand description.
cudaError_t launch_gemm(const GemmOperands& g, cudaStream_t s) {
    using namespace gm;
    if (g.npairs < 1 || g.npairs > kMaxPairs || g.M <= 0 || g.N <= 0 || g.batch <= 0 || g.splits <= 0) return cudaErrorInvalidValue;
    if (g.N % 16 != 0 || (g.splits > 1 && g.Cadd)) return cudaErrorInvalidValue;
    CUtensorMap maps[2 * kMaxPairs];
    Args a{};
    a.M = g.M; a.N = g.N; a.batch = g.batch; a.splits = g.splits; a.npairs = g.npairs;
    a.mt = (g.M + 2 * BM - 1) / (2 * BM); a.nt = (g.N + BN - 1) / BN;
    for (int i = 0; i < kMaxPairs; ++i) {
        const GemmPair& gp = g.p[i < g.npairs ? i : 0];
        if (gp.K <= 0 || gp.K % BK != 0) return cudaErrorInvalidValue;
        // a CTA's half of an operand tile: K-major, 128 rows of 64 K; MN-major, 64 K-rows of 2 x 64
        if (!map_2d(&maps[2 * i], gp.a, gp.a_rows, gp.a_cols, gp.a_ld, gp.a_kmajor ? BM : BK) ||
            !map_2d(&maps[2 * i + 1], gp.b, gp.b_rows, gp.b_cols, gp.b_ld, gp.b_kmajor ? BNH : BK))
            return cudaErrorInvalidValue;
        a.p[i].K = gp.K;
        a.p[i].a_kmajor = gp.a_kmajor; a.p[i].b_kmajor = gp.b_kmajor;
        a.p[i].a_boff_row = gp.a_boff_row; a.p[i].a_boff_col = gp.a_boff_col;
        a.p[i].a_bstep_row = gp.a_bstep_row; a.p[i].a_bstep_col = gp.a_bstep_col;
        a.p[i].b_boff_row = gp.b_boff_row; a.p[i].b_boff_col = gp.b_boff_col;
        a.p[i].b_bstep_row = gp.b_bstep_row; a.p[i].b_bstep_col = gp.b_bstep_col;
    }
    a.interleave = 1;
    for (int i = 1; i < g.npairs; ++i) {
        if (g.p[i].K != g.p[0].K) a.interleave = 0;
        if (g.p[i].a_kmajor != g.p[0].a_kmajor || g.p[i].b_kmajor != g.p[0].b_kmajor) return cudaErrorInvalidValue;
    }
    a.C = g.C; a.c_ld = g.c_ld; a.c_bstride = g.c_bstride; a.c_split = g.c_split;
    a.Cadd = g.Cadd; a.add_ld = g.add_ld; a.add_bstride = g.add_bstride;
    a.C16 = g.C16;
    if (a.C16 && (a.Cadd || g.splits > 1 || g.c_ld % 8 != 0)) return cudaErrorInvalidValue;
    a.status = g.status;
    a.timeout_ns = 1000000000ull;
    void (*kern)(CUtensorMap, CUtensorMap, CUtensorMap, CUtensorMap, CUtensorMap, CUtensorMap, CUtensorMap,
                 CUtensorMap, Args) = g.npairs == 1   ? gemm_kernel<1>
                                      : g.npairs == 2 ? gemm_kernel<2>
                                      : g.npairs == 3 ? gemm_kernel<3>
                                                      : gemm_kernel<4>;
    cudaError_t e = set_smem_once(kern, (int)SMEM_BYTES);
    if (e != cudaSuccess) return e;
    // pairs of CTAs (2-CTA clusters), as many as can be resident at once, each walking tiles
    cudaLaunchConfig_t cfg = {};
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = SMEM_BYTES;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    static std::mutex mu;
    static int max_pairs[kMaxPairs][64] = {};
    int dev = 0;
    if ((e = cudaGetDevice(&dev)) != cudaSuccess) return e;
    int pairs = 0;
    {
        std::lock_guard<std::mutex> lock(mu);
        if (dev >= 0 && dev < 64) pairs = max_pairs[g.npairs - 1][dev];
    }
    if (pairs <= 0) {
        cfg.gridDim = dim3(2);
        if ((e = cudaOccupancyMaxActiveClusters(&pairs, kern, &cfg)) != cudaSuccess) return e;
        if (pairs <= 0) return cudaErrorLaunchOutOfResources;
        std::lock_guard<std::mutex> lock(mu);
        if (dev >= 0 && dev < 64) max_pairs[g.npairs - 1][dev] = pairs;
    }
    const int ntiles = a.batch * a.mt * a.nt * a.splits;
    cfg.gridDim = dim3(2u * (unsigned)(ntiles < pairs ? ntiles : pairs));
    return cudaLaunchKernelEx(&cfg, kern, maps[0], maps[1], maps[2], maps[3], maps[4], maps[5], maps[6], maps[7], a);
}

}  // namespace rglru
