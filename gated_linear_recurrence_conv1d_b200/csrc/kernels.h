// kernels.h -- launchers of the RG-LRU kernels (internal to librglru.so).
#pragma once

#include <cuda_runtime.h>

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

// Tensor-core decode step (bf16, head_dim 256): one launch of 4-CTA clusters (conv + history
// shift per channel quarter, conv blocks shared over distributed shared memory, tcgen05 gates,
// the state update).  Needs the workspace fused_decode_workspace() (the status word).
bool fused_decode_supported(const rglru_dims* d);
size_t fused_decode_workspace(const rglru_dims* d);
int fused_decode_launches(const rglru_dims* d);
cudaError_t launch_fused_decode(const rglru_dims* d, const rglru_params* p, const void* x, const void* y,
                                const uint8_t* reset, rglru_state* st, void* out, void* ws, size_t ws_bytes,
                                cudaStream_t s);

// Backward pass of the prefill (CUDA cores, fp32, any supported shape): four launches.
size_t backward_workspace(const rglru_dims* d);
int backward_launches(const rglru_dims* d);
cudaError_t launch_backward(const rglru_dims* d, const rglru_params* p, const void* x, const void* y,
                            const uint8_t* reset, const rglru_state* st0, const void* dout,
                            const float* dh_final, const float* dtail_final, const rglru_grads* grads,
                            void* ws, size_t ws_bytes, cudaStream_t s);

}  // namespace rglru
