// kernels.h -- launchers of the RG-LRU kernels (internal to librglru.so).
#pragma once

#include <cuda_runtime.h>

#include "common.cuh"
#include <cuda_bf16.h>

#include "rglru.h"

namespace rglru {

// Portable kernels (any supported head_dim, fp32 or bf16); need no workspace.
cudaError_t launch_prefill_generic(const rglru_dims* d, const rglru_params* p, const void* x,
                                   const void* y, const uint8_t* reset, rglru_state* st,
                                   void* out, cudaStream_t s);
cudaError_t launch_decode_generic(const rglru_dims* d, const rglru_params* p, const void* x,
                                  const void* y, const uint8_t* reset, rglru_state* st,
                                  void* out, cudaStream_t s);

// Tensor-core prefill (bf16, head_dim 256): tcgen05 MMA with TMEM operands, TMA tiles and a
// decoupled look-back across time chunks.  Needs the workspace fused_prefill_workspace().
bool fused_prefill_supported(const rglru_dims* d);
size_t fused_prefill_workspace(const rglru_dims* d);
int fused_prefill_launches(const rglru_dims* d);
cudaError_t launch_fused_prefill(const rglru_dims* d, const rglru_params* p, const void* x, const void* y,
                                 const uint8_t* reset, rglru_state* st, void* out, void* ws, size_t ws_bytes,
                                 cudaStream_t s);

// The same kernel's save mode, the forward again for the gradients (backward_tc.cu): the gate
// contraction runs on the conv output's bf16 hi and lo parts, the element-wise math is accurate,
// and instead of out it writes per token-channel the complete gate pre-activations, h_{t-1} as
// the update used it (0 at a segment start) and the conv output as a bf16 hi + lo pair; the
// state is only read.  `status` receives device-side failures.
struct PrefillSave {
    float* ga;
    float* gx;
    float* hprev;
    __nv_bfloat16* xc_hi;
    __nv_bfloat16* xc_lo;
};
cudaError_t launch_fused_prefill_save(const rglru_dims* d, const rglru_params* p, const void* x,
                                      const uint8_t* reset, const rglru_state* st, const PrefillSave* sv, void* ws,
                                      size_t ws_bytes, DeviceStatus* status, cudaStream_t s);

// Tensor-core backward (backward_tc.cu): bf16, head_dim 256.
bool backward_tc_supported(const rglru_dims* d);
size_t backward_tc_workspace(const rglru_dims* d);
int backward_tc_launches(const rglru_dims* d);
cudaError_t launch_backward_tc(const rglru_dims* d, const rglru_params* p, const void* x, const void* y,
                               const uint8_t* reset, const rglru_state* st0, const void* dout,
                               const float* dh_final, const float* dtail_final, const rglru_grads* grads,
                               void* ws, size_t ws_bytes, cudaStream_t s);

// The block with its projections (layer.cu): x = u W_in_x, y = u W_in_y, block, out = z W_out,
// bf16, head_dim 256, model width a multiple of 64.
bool layer_supported(const rglru_dims* d, int model_dim);
size_t layer_workspace(const rglru_dims* d);
int layer_launches(const rglru_dims* d);
cudaError_t launch_layer(const rglru_dims* d, const rglru_params* p, int model_dim, const void* w_in_x,
                         const void* w_in_y, const void* w_out, const void* u, const uint8_t* reset,
                         rglru_state* st, void* out, void* ws, size_t ws_bytes, cudaStream_t s);

// Local sliding-window MQA (mqa.cu): bf16, head_dim 256.
bool mqa_supported(const rglru_mqa_dims* d);
size_t mqa_workspace(const rglru_mqa_dims* d, bool decode);
cudaError_t launch_mqa_prefill(const rglru_mqa_dims* d, const void* q, const void* k, const void* v, int pos0,
                               void* out, void* cache, void* ws, size_t ws_bytes, cudaStream_t s);
cudaError_t launch_mqa_decode(const rglru_mqa_dims* d, const void* q, const void* k, const void* v, const int* pos,
                              void* cache, void* out, void* ws, size_t ws_bytes, cudaStream_t s);

// Tensor-core decode step (bf16, head_dim 256): one launch of 4-CTA clusters (conv + history
// shift per channel quarter, conv blocks shared over distributed shared memory, tcgen05 gates,
// the state update).  Needs the workspace fused_decode_workspace() (the status word).
bool fused_decode_supported(const rglru_dims* d);
size_t fused_decode_workspace(const rglru_dims* d);
int fused_decode_launches(const rglru_dims* d);
cudaError_t launch_fused_decode(const rglru_dims* d, const rglru_params* p, const void* x, const void* y,
                                const uint8_t* reset, rglru_state* st, void* out, void* ws, size_t ws_bytes,
                                cudaStream_t s);

// Persistent multi-step decode (bf16, head_dim 256): `steps` single-token steps in one launch of
// 4-CTA clusters, the state kept in registers between steps.  Needs a 256-byte workspace.
bool fused_decode_steps_supported(const rglru_dims* d);
cudaError_t launch_fused_decode_steps(const rglru_dims* d, const rglru_params* p, const void* x, const void* y,
                                      const uint8_t* reset, int steps, rglru_state* st, void* out, void* ws,
                                      size_t ws_bytes, cudaStream_t s);

// Batched bf16 GEMM on the tensor cores (gemm.cu): C[split][b][m][n] (fp32) = sum over pairs p of
// sum_k A_p(m, k) B_p(k, n) (+ Cadd[b][m][n]).  Operand A of pair p is read from a row-major bf16
// tensor of a_rows x a_cols (pitch a_ld elements): K-major A holds (m, k) at row
// r0 + m, column c0 + k; M-major A at row r0 + k, column c0 + m, with r0 = a_boff_row +
// b * a_bstep_row and c0 = a_boff_col + b * a_bstep_col for batch b; B likewise with n
// (K-major: row r0 + n, column c0 + k; N-major: row r0 + k, column c0 + n).  K of every pair is
// a multiple of 64, N a multiple of 16; K is cut into `splits` slices written to separate C
// slices (C + split * c_split), and Cadd is only allowed without a split.
struct GemmPair {
    const void* a;
    long long a_rows, a_cols, a_ld;
    int a_kmajor, a_boff_row, a_boff_col, a_bstep_row, a_bstep_col;
    const void* b;
    long long b_rows, b_cols, b_ld;
    int b_kmajor, b_boff_row, b_boff_col, b_bstep_row, b_bstep_col;
    int K;
};
struct GemmOperands {
    int M, N, batch, splits, npairs;   // npairs <= 4
    GemmPair p[4];
    float* C;
    long long c_ld, c_bstride, c_split;
    const float* Cadd;
    long long add_ld, add_bstride;
    __nv_bfloat16* C16;       // if set, C is written here as bf16 instead (no Cadd, no split)
    DeviceStatus* status;
};
size_t gemm_smem_bytes();
cudaError_t launch_gemm(const GemmOperands& g, cudaStream_t s);

// Backward pass of the prefill (CUDA cores, fp32, any supported shape): four launches.
size_t backward_workspace(const rglru_dims* d);
int backward_launches(const rglru_dims* d);
cudaError_t launch_backward(const rglru_dims* d, const rglru_params* p, const void* x, const void* y,
                            const uint8_t* reset, const rglru_state* st0, const void* dout,
                            const float* dh_final, const float* dtail_final, const rglru_grads* grads,
                            void* ws, size_t ws_bytes, cudaStream_t s);

}  // namespace rglru
