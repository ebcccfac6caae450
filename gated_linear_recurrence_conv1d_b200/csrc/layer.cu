// layer.cu -- the recurrent block with its neighbouring projections (bf16, head_dim 256):
//
//   x = u W_in_x,  y = u W_in_y    (linear_x / linear_y: model width D -> LRU width W)
//   z = block(x, y)                 (conv -> RG-LRU -> z = h GeLU(y): fused_prefill.cu)
//   out = z W_out                   (linear_out: W -> D)
//
// following the listing "1. PyTorch Implementation of RG-LRU and the Griffin Block"
// (RecurrentBlock.forward: proj_in_1, proj_in_2, proj_out) of "Griffin Guide: RecurrentGemma,
// RG-LRU & Hybrid Attention", its sections "1. Temporal Filtering via Separable 1D Convolutions"
// (the D -> D_RNN projection before the conv) and "2. Non-Linear Multiplicative Gating with
// GeLU" (the output projection), and the module names of the TransformerLens RecurrentGemma
// bridge (linear_x, linear_y, conv_1d, rg_lru, linear_out).  The three projections run on the
// tensor-core GEMM of gemm.cu (fp32 accumulation, bf16 results); x, y and z are bf16 tensors
// of the workspace, so the block sees exactly what rglru_block_prefill would be given.
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "common.cuh"
#include "kernels.h"

namespace rglru {

namespace {

struct LayerLayout {
    size_t x, y, z, total;
};

LayerLayout layer_layout(const rglru_dims* d) {
    auto up = [](size_t v) { return (v + 255) & ~size_t(255); };
    const size_t n = (size_t)d->batch * d->seq_len * d->heads * d->head_dim * 2;
    LayerLayout l;
    size_t o = up(fused_prefill_workspace(d));   // the block's workspace first: one status word
    l.x = o; o = up(o + n);
    l.y = o; o = up(o + n);
    l.z = o; o = up(o + n);
    l.total = o;
    return l;
}

// out[M x N] (bf16) = act[M x K] (bf16, row-major) . w[K x N] (bf16, row-major)
GemmOperands projection(const void* act, long long M, int K, const void* w, int N, __nv_bfloat16* out,
                        DeviceStatus* status) {
    GemmOperands g{};
    g.M = (int)M; g.N = N; g.batch = 1; g.splits = 1; g.npairs = 1;
    GemmPair& p = g.p[0];
    p.a = act; p.a_rows = M; p.a_cols = K; p.a_ld = K; p.a_kmajor = 1;       // (m, k) at row m, column k
    p.b = w; p.b_rows = K; p.b_cols = N; p.b_ld = N; p.b_kmajor = 0;         // (n, k) at row k, column n
    p.K = K;
    g.C16 = out; g.c_ld = N;
    g.status = status;
    return g;
}

}  // namespace

bool layer_supported(const rglru_dims* d, int model_dim) {
    return fused_prefill_supported(d) && model_dim > 0 && model_dim % 64 == 0;
}

size_t layer_workspace(const rglru_dims* d) { return layer_layout(d).total; }

int layer_launches(const rglru_dims* d) {
    return 3 + fused_prefill_launches(d);   // three projection GEMMs and the block
}

cudaError_t launch_layer(const rglru_dims* d, const rglru_params* p, int model_dim, const void* w_in_x,
                         const void* w_in_y, const void* w_out, const void* u, const uint8_t* reset,
                         rglru_state* st, void* out, void* ws, size_t ws_bytes, cudaStream_t s) {
    const LayerLayout l = layer_layout(d);
    if (l.total > ws_bytes) return cudaErrorInvalidValue;
    uint8_t* w = static_cast<uint8_t*>(ws);
    DeviceStatus* status = reinterpret_cast<DeviceStatus*>(w);
    const long long M = (long long)d->batch * d->seq_len;
    const int W = d->heads * d->head_dim, D = model_dim;
    __nv_bfloat16* x = reinterpret_cast<__nv_bfloat16*>(w + l.x);
    __nv_bfloat16* y = reinterpret_cast<__nv_bfloat16*>(w + l.y);
    __nv_bfloat16* z = reinterpret_cast<__nv_bfloat16*>(w + l.z);
    cudaError_t e = launch_gemm(projection(u, M, D, w_in_x, W, x, status), s);
    if (e == cudaSuccess) e = launch_gemm(projection(u, M, D, w_in_y, W, y, status), s);
    if (e == cudaSuccess) e = launch_fused_prefill(d, p, x, y, reset, st, z, ws, l.x, s);
    if (e == cudaSuccess) e = launch_gemm(projection(z, M, W, w_out, D, static_cast<__nv_bfloat16*>(out), status), s);
    return e;
}

}  // namespace rglru
