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

}  // namespace rglru
