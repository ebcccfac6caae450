// api.cu -- the C ABI of librglru.so: host-side validation, workspace sizing, dispatch.
//
// Every check runs on the host before anything is enqueued; a failed check returns its code
// and launches nothing.  Device-side conditions are latched in the workspace status word.
#include <cuda_runtime.h>
#include <stdint.h>

#include <mutex>

#include "common.cuh"
#include "kernels.h"
#include "rglru.h"

namespace rglru {

// Unique id of the calling thread's current context (cuCtxGetId, reached through the runtime's
// driver entry point so that the library needs no link against libcuda).  0 when unavailable.
unsigned long long current_context_id() {
    typedef int (*GetCurrentFn)(void**);
    typedef int (*GetIdFn)(void*, unsigned long long*);
    static GetCurrentFn get_current = nullptr;
    static GetIdFn get_id = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            get_current = reinterpret_cast<GetCurrentFn>(p);
        p = nullptr;
        if (cudaGetDriverEntryPoint("cuCtxGetId", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            get_id = reinterpret_cast<GetIdFn>(p);
    });
    void* ctx = nullptr;
    unsigned long long id = 0;
    if (!get_current || !get_id || get_current(&ctx) != 0 || !ctx || get_id(ctx, &id) != 0) return 0;
    return id;
}


cudaError_t set_smem_limit(const void* kernel, int bytes) {
    struct Entry {
        const void* fn;
        unsigned long long ctx;
        int bytes;
    };
    static std::mutex mu;
    static Entry done[256];
    static int n = 0;
    const unsigned long long ctx = current_context_id();
    std::lock_guard<std::mutex> lock(mu);
    if (ctx != 0)
        for (int i = 0; i < n; ++i)
            if (done[i].fn == kernel && done[i].ctx == ctx && done[i].bytes == bytes) return cudaSuccess;
    cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
    if (e != cudaSuccess || ctx == 0) return e;
    int slot = -1;
    for (int i = 0; i < n && slot < 0; ++i)
        if (done[i].fn == kernel) slot = i;          // a kernel keeps one entry: its latest context
    if (slot < 0) slot = n < 256 ? n++ : 255;
    done[slot] = Entry{kernel, ctx, bytes};
    return cudaSuccess;
}

}  // namespace rglru

using rglru::current_context_id;

namespace {

constexpr size_t kStatusBytes = 256;   // status word area at the start of every workspace

bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

size_t act_size(int dtype) { return dtype == RGLRU_F32 ? 4 : 2; }

rglru_status check_dims(const rglru_dims* d, bool prefill) {
    if (!d) return RGLRU_ERR_INVALID_ARG;
    if (d->batch <= 0 || d->heads <= 0 || d->head_dim <= 0) return RGLRU_ERR_INVALID_ARG;
    if (prefill && d->seq_len <= 0) return RGLRU_ERR_INVALID_ARG;
    if (d->act_dtype != RGLRU_F32 && d->act_dtype != RGLRU_BF16) return RGLRU_ERR_INVALID_ARG;
    if (!(d->c > 0.0f) || d->c != d->c) return RGLRU_ERR_INVALID_ARG;
    if (d->gelu_tanh != 0 && d->gelu_tanh != 1) return RGLRU_ERR_INVALID_ARG;
    if (d->conv_width != rglru::kConvWidth) return RGLRU_ERR_UNSUPPORTED;
    if (d->head_dim % 16 != 0 || d->head_dim > 256) return RGLRU_ERR_UNSUPPORTED;
    const long long W = (long long)d->heads * d->head_dim;
    if ((W * (long long)act_size(d->act_dtype)) % 16 != 0) return RGLRU_ERR_UNSUPPORTED;
    // every [B, T, W] index must fit comfortably in 63 bits; grid dims in 31 bits
    if (d->heads > 65535 || d->batch > (1 << 30)) return RGLRU_ERR_UNSUPPORTED;
    if (prefill && (long long)d->batch * d->seq_len * W > (1LL << 40)) return RGLRU_ERR_UNSUPPORTED;
    return RGLRU_OK;
}

rglru_status check_params(const rglru_params* p) {
    if (!p || !p->conv_w || !p->w_a || !p->w_x || !p->lambda) return RGLRU_ERR_INVALID_ARG;
    if (!aligned(p->conv_w, 4) || !aligned(p->lambda, 4)) return RGLRU_ERR_INVALID_ARG;
    if ((p->conv_b && !aligned(p->conv_b, 4)) || (p->b_a && !aligned(p->b_a, 4)) ||
        (p->b_x && !aligned(p->b_x, 4)))
        return RGLRU_ERR_INVALID_ARG;
    if (!aligned(p->w_a, 16) || !aligned(p->w_x, 16)) return RGLRU_ERR_INVALID_ARG;
    return RGLRU_OK;
}

rglru_status check_state(const rglru_state* s) {
    if (!s || !s->h || !s->conv_tail) return RGLRU_ERR_INVALID_ARG;
    if (!aligned(s->h, 4) || !aligned(s->conv_tail, 16)) return RGLRU_ERR_INVALID_ARG;
    return RGLRU_OK;
}

rglru_status check_io(const void* x, const void* y, const void* out) {
    if (!x || !y || !out) return RGLRU_ERR_INVALID_ARG;
    if (!aligned(x, 16) || !aligned(y, 16) || !aligned(out, 16)) return RGLRU_ERR_INVALID_ARG;
    if (out == x || out == y) return RGLRU_ERR_INVALID_ARG;
    return RGLRU_OK;
}

rglru_status check_workspace(void* ws, size_t bytes, size_t need) {
    if (!ws || bytes < need) return RGLRU_ERR_WORKSPACE;
    if (!aligned(ws, 256)) return RGLRU_ERR_INVALID_ARG;
    return RGLRU_OK;
}

// CUDA error behind the calling thread's most recent RGLRU_ERR_CUDA
thread_local cudaError_t t_last_cuda_error = cudaSuccess;

rglru_status cuda_status(cudaError_t e) {
    if (e == cudaSuccess) return RGLRU_OK;
    t_last_cuda_error = e;
    cudaGetLastError();   // clear a sticky launch-configuration error for the caller
    return RGLRU_ERR_CUDA;
}

// Scratch of rglru_block_prefill_noalloc: a fixed area in the library's device image, for
// callers that cannot allocate device memory.  In host code `g_noalloc_scratch` names a host
// shadow, not device memory, so kernels only ever receive the address that
// cudaGetSymbolAddress returns for the current device.
__device__ __align__(256) unsigned char g_noalloc_scratch[RGLRU_NOALLOC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;

// Device address of the static scratch in the calling thread's current context, looked up with
// cudaGetSymbolAddress the first time a device is used and again whenever that device's
// context has changed since (a cudaDeviceReset destroys the primary context, the module is
// loaded anew in the next one and the area moves); cached per device with the context's
// unique id.  Without a context id the address is looked up on every call.
cudaError_t noalloc_scratch(void** addr) {
    static std::mutex mu;
    static void* cache[kMaxDevices] = {};
    static unsigned long long cache_ctx[kMaxDevices] = {};
    int dev = -1;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
    const unsigned long long ctx = current_context_id();   // 0 before the context exists
    std::lock_guard<std::mutex> lock(mu);
    if (!cache[dev] || ctx == 0 || cache_ctx[dev] != ctx) {
        void* p = nullptr;
        e = cudaGetSymbolAddress(&p, g_noalloc_scratch);     // creates the context if needed
        if (e != cudaSuccess) return e;
        if (!p) return cudaErrorInvalidSymbol;
        cache[dev] = p;
        cache_ctx[dev] = current_context_id();
    }
    *addr = cache[dev];
    return cudaSuccess;
}

}  // namespace

extern "C" {

int rglru_abi_version(void) { return RGLRU_ABI_VERSION; }

const char* rglru_status_string(rglru_status s) {
    switch (s) {
        case RGLRU_OK: return "RGLRU_OK";
        case RGLRU_ERR_INVALID_ARG: return "RGLRU_ERR_INVALID_ARG: null, misaligned or out-of-range argument";
        case RGLRU_ERR_UNSUPPORTED: return "RGLRU_ERR_UNSUPPORTED: shape outside the supported set";
        case RGLRU_ERR_WORKSPACE: return "RGLRU_ERR_WORKSPACE: workspace missing or too small";
        case RGLRU_ERR_CUDA: return "RGLRU_ERR_CUDA: a CUDA runtime call or launch failed";
        case RGLRU_ERR_TIMEOUT: return "RGLRU_ERR_TIMEOUT: a bounded device-side wait expired";
        case RGLRU_ERR_DEVICE: return "RGLRU_ERR_DEVICE: a device-side consistency check failed";
    }
    return "RGLRU_ERR_UNKNOWN";
}

rglru_status rglru_state_init(const rglru_dims* dims, rglru_state* state, void* stream) {
    rglru_status st = check_dims(dims, false);
    if (st != RGLRU_OK) return st;
    if ((st = check_state(state)) != RGLRU_OK) return st;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const size_t W = (size_t)dims->heads * dims->head_dim;
    cudaError_t e = cudaMemsetAsync(state->h, 0, (size_t)dims->batch * W * sizeof(float), s);
    if (e == cudaSuccess)
        e = cudaMemsetAsync(state->conv_tail, 0,
                            (size_t)dims->batch * rglru::kHist * W * act_size(dims->act_dtype), s);
    return cuda_status(e);
}

size_t rglru_prefill_workspace_size(const rglru_dims* dims) {
    if (check_dims(dims, true) != RGLRU_OK) return 0;
    if (rglru::fused_prefill_supported(dims)) return rglru::fused_prefill_workspace(dims);
    return kStatusBytes;
}

size_t rglru_decode_workspace_size(const rglru_dims* dims) {
    if (check_dims(dims, false) != RGLRU_OK) return 0;
    if (rglru::fused_decode_supported(dims)) return rglru::fused_decode_workspace(dims);
    return kStatusBytes;
}

rglru_status rglru_block_prefill(const rglru_dims* dims, const rglru_params* params,
                                 const void* x, const void* y, const uint8_t* reset,
                                 rglru_state* state, void* out, void* workspace,
                                 size_t workspace_bytes, void* stream) {
    rglru_status st = check_dims(dims, true);
    if (st != RGLRU_OK) return st;
    if ((st = check_params(params)) != RGLRU_OK) return st;
    if ((st = check_io(x, y, out)) != RGLRU_OK) return st;
    if (state && (st = check_state(state)) != RGLRU_OK) return st;
    if ((st = check_workspace(workspace, workspace_bytes, rglru_prefill_workspace_size(dims))) != RGLRU_OK)
        return st;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (rglru::fused_prefill_supported(dims))
        return cuda_status(rglru::launch_fused_prefill(dims, params, x, y, reset, state, out, workspace,
                                                       workspace_bytes, s));
    return cuda_status(rglru::launch_prefill_generic(dims, params, x, y, reset, state, out, s));
}

rglru_status rglru_block_decode(const rglru_dims* dims, const rglru_params* params,
                                const void* x, const void* y, const uint8_t* reset,
                                rglru_state* state, void* out, void* workspace,
                                size_t workspace_bytes, void* stream) {
    rglru_status st = check_dims(dims, false);
    if (st != RGLRU_OK) return st;
    if ((st = check_params(params)) != RGLRU_OK) return st;
    if ((st = check_io(x, y, out)) != RGLRU_OK) return st;
    if ((st = check_state(state)) != RGLRU_OK) return st;
    if ((st = check_workspace(workspace, workspace_bytes, rglru_decode_workspace_size(dims))) != RGLRU_OK)
        return st;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    // the tensor-core step reads and writes h with 16-byte vectors
    if (rglru::fused_decode_supported(dims) && aligned(state->h, 16))
        return cuda_status(rglru::launch_fused_decode(dims, params, x, y, reset, state, out, workspace,
                                                      workspace_bytes, s));
    return cuda_status(rglru::launch_decode_generic(dims, params, x, y, reset, state, out, s));
}

size_t rglru_decode_steps_workspace_size(const rglru_dims* dims, int steps) {
    if (check_dims(dims, false) != RGLRU_OK || steps <= 0) return 0;
    return kStatusBytes;
}

rglru_status rglru_block_decode_steps(const rglru_dims* dims, const rglru_params* params, const void* x,
                                      const void* y, const uint8_t* reset, int steps, rglru_state* state,
                                      void* out, void* workspace, size_t workspace_bytes, void* stream) {
    rglru_status st = check_dims(dims, false);
    if (st != RGLRU_OK) return st;
    if (steps <= 0) return RGLRU_ERR_INVALID_ARG;
    if ((long long)steps * dims->batch * dims->heads * dims->head_dim > (1LL << 40)) return RGLRU_ERR_UNSUPPORTED;
    if ((st = check_params(params)) != RGLRU_OK) return st;
    if ((st = check_io(x, y, out)) != RGLRU_OK) return st;
    if ((st = check_state(state)) != RGLRU_OK) return st;
    if ((st = check_workspace(workspace, workspace_bytes, rglru_decode_steps_workspace_size(dims, steps))) != RGLRU_OK)
        return st;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    // the persistent kernel keeps h in registers and moves it with 16-byte vectors
    if (rglru::fused_decode_steps_supported(dims) && aligned(state->h, 16))
        return cuda_status(rglru::launch_fused_decode_steps(dims, params, x, y, reset, steps, state, out, workspace,
                                                            workspace_bytes, s));
    // other shapes: one portable step after another, in stream order
    const size_t step_elems = (size_t)dims->batch * dims->heads * dims->head_dim;
    const size_t es = act_size(dims->act_dtype);
    for (int k = 0; k < steps; ++k) {
        const size_t off = (size_t)k * step_elems * es;
        cudaError_t e = rglru::launch_decode_generic(
            dims, params, static_cast<const char*>(x) + off, static_cast<const char*>(y) + off,
            reset ? reset + (size_t)k * dims->batch : nullptr, state, static_cast<char*>(out) + off, s);
        if (e != cudaSuccess) return cuda_status(e);
    }
    return RGLRU_OK;
}

rglru_status rglru_decode_steps_plan(const rglru_dims* dims, int steps, int* kernel, int* launches) {
    rglru_status st = check_dims(dims, false);
    if (st != RGLRU_OK) return st;
    if (steps <= 0 || !kernel || !launches) return RGLRU_ERR_INVALID_ARG;
    const bool tc = rglru::fused_decode_steps_supported(dims);
    *kernel = tc ? RGLRU_KERNEL_TENSOR : RGLRU_KERNEL_GENERIC;
    *launches = tc ? 1 : steps;
    return RGLRU_OK;
}

size_t rglru_layer_workspace_size(const rglru_dims* dims) {
    if (check_dims(dims, true) != RGLRU_OK) return 0;
    return rglru::layer_workspace(dims);
}

rglru_status rglru_layer_forward(const rglru_dims* dims, const rglru_params* params, const rglru_projections* proj,
                                 const void* u, const uint8_t* reset, rglru_state* state, void* out,
                                 void* workspace, size_t workspace_bytes, void* stream) {
    rglru_status st = check_dims(dims, true);
    if (st != RGLRU_OK) return st;
    if ((st = check_params(params)) != RGLRU_OK) return st;
    if (!proj || !proj->w_in_x || !proj->w_in_y || !proj->w_out) return RGLRU_ERR_INVALID_ARG;
    if (!aligned(proj->w_in_x, 16) || !aligned(proj->w_in_y, 16) || !aligned(proj->w_out, 16))
        return RGLRU_ERR_INVALID_ARG;
    if (proj->model_dim <= 0) return RGLRU_ERR_INVALID_ARG;
    if (!u || !out || !aligned(u, 16) || !aligned(out, 16) || u == out) return RGLRU_ERR_INVALID_ARG;
    if (state && (st = check_state(state)) != RGLRU_OK) return st;
    if (!rglru::layer_supported(dims, proj->model_dim)) return RGLRU_ERR_UNSUPPORTED;
    if ((long long)dims->batch * dims->seq_len * proj->model_dim > (1LL << 40)) return RGLRU_ERR_UNSUPPORTED;
    if ((st = check_workspace(workspace, workspace_bytes, rglru_layer_workspace_size(dims))) != RGLRU_OK) return st;
    return cuda_status(rglru::launch_layer(dims, params, proj->model_dim, proj->w_in_x, proj->w_in_y, proj->w_out, u,
                                           reset, state, out, workspace, workspace_bytes,
                                           static_cast<cudaStream_t>(stream)));
}

rglru_status rglru_layer_plan(const rglru_dims* dims, const rglru_projections* proj, int* kernel, int* launches) {
    rglru_status st = check_dims(dims, true);
    if (st != RGLRU_OK) return st;
    if (!proj || !kernel || !launches) return RGLRU_ERR_INVALID_ARG;
    if (!rglru::layer_supported(dims, proj->model_dim)) return RGLRU_ERR_UNSUPPORTED;
    *kernel = RGLRU_KERNEL_TENSOR;
    *launches = rglru::layer_launches(dims);
    return RGLRU_OK;
}

static rglru_status check_mqa(const rglru_mqa_dims* d, bool decode) {
    if (!d || d->batch <= 0 || d->q_heads <= 0 || d->head_dim <= 0 || d->window <= 0) return RGLRU_ERR_INVALID_ARG;
    if (!decode && d->seq_len <= 0) return RGLRU_ERR_INVALID_ARG;
    if (!(d->scale > 0.0f) || !(d->rope_base > 0.0f)) return RGLRU_ERR_INVALID_ARG;
    if (!rglru::mqa_supported(d)) return RGLRU_ERR_UNSUPPORTED;
    if (!decode && (long long)d->batch * d->seq_len * d->q_heads * d->head_dim > (1LL << 40)) return RGLRU_ERR_UNSUPPORTED;
    if (d->batch > (1 << 16) || (!decode && d->seq_len > (1 << 30))) return RGLRU_ERR_UNSUPPORTED;
    return RGLRU_OK;
}

size_t rglru_mqa_workspace_size(const rglru_mqa_dims* dims, int decode) {
    if (check_mqa(dims, decode != 0) != RGLRU_OK) return 0;
    return rglru::mqa_workspace(dims, decode != 0);
}

rglru_status rglru_mqa_prefill(const rglru_mqa_dims* dims, const void* q, const void* k, const void* v, int pos0,
                               void* out, void* cache, void* workspace, size_t workspace_bytes, void* stream) {
    rglru_status st = check_mqa(dims, false);
    if (st != RGLRU_OK) return st;
    if (!q || !k || !v || !out || !aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(out, 16))
        return RGLRU_ERR_INVALID_ARG;
    if (out == q || out == k || out == v || pos0 < 0) return RGLRU_ERR_INVALID_ARG;
    if (cache && !aligned(cache, 16)) return RGLRU_ERR_INVALID_ARG;
    if ((st = check_workspace(workspace, workspace_bytes, rglru_mqa_workspace_size(dims, 0))) != RGLRU_OK) return st;
    return cuda_status(rglru::launch_mqa_prefill(dims, q, k, v, pos0, out, cache, workspace, workspace_bytes,
                                                 static_cast<cudaStream_t>(stream)));
}

rglru_status rglru_mqa_decode(const rglru_mqa_dims* dims, const void* q, const void* k, const void* v,
                              const int* pos, void* cache, void* out, void* workspace, size_t workspace_bytes,
                              void* stream) {
    rglru_status st = check_mqa(dims, true);
    if (st != RGLRU_OK) return st;
    if (!q || !k || !v || !out || !pos || !cache) return RGLRU_ERR_INVALID_ARG;
    if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(out, 16) || !aligned(cache, 16) ||
        !aligned(pos, 4))
        return RGLRU_ERR_INVALID_ARG;
    if (out == q || out == k || out == v) return RGLRU_ERR_INVALID_ARG;
    if ((st = check_workspace(workspace, workspace_bytes, rglru_mqa_workspace_size(dims, 1))) != RGLRU_OK) return st;
    return cuda_status(rglru::launch_mqa_decode(dims, q, k, v, pos, cache, out, workspace, workspace_bytes,
                                                static_cast<cudaStream_t>(stream)));
}

size_t rglru_backward_workspace_size(const rglru_dims* dims) {
    if (check_dims(dims, true) != RGLRU_OK) return 0;
    if (rglru::backward_tc_supported(dims)) return rglru::backward_tc_workspace(dims);
    return rglru::backward_workspace(dims);
}

rglru_status rglru_block_backward(const rglru_dims* dims, const rglru_params* params,
                                  const void* x, const void* y, const uint8_t* reset,
                                  const rglru_state* state0, const void* dout,
                                  const float* dh_final, const float* dtail_final,
                                  const rglru_grads* grads, void* workspace,
                                  size_t workspace_bytes, void* stream) {
    rglru_status st = check_dims(dims, true);
    if (st != RGLRU_OK) return st;
    if ((st = check_params(params)) != RGLRU_OK) return st;
    if (!x || !y || !dout || !aligned(x, 16) || !aligned(y, 16) || !aligned(dout, 16)) return RGLRU_ERR_INVALID_ARG;
    if (state0 && (st = check_state(state0)) != RGLRU_OK) return st;
    if ((dh_final && !aligned(dh_final, 4)) || (dtail_final && !aligned(dtail_final, 4))) return RGLRU_ERR_INVALID_ARG;
    if (!grads || !grads->dx || !grads->dy || !grads->dconv_w || !grads->dconv_b || !grads->dw_a ||
        !grads->dw_x || !grads->db_a || !grads->db_x || !grads->dlambda)
        return RGLRU_ERR_INVALID_ARG;
    const void* outs[] = {grads->dx, grads->dy, grads->dh0, grads->dtail0, grads->dconv_w, grads->dconv_b,
                          grads->dw_a, grads->dw_x, grads->db_a, grads->db_x, grads->dlambda};
    for (const void* o : outs) {
        if (o && !aligned(o, 4)) return RGLRU_ERR_INVALID_ARG;
        if (o && (o == x || o == y || o == dout)) return RGLRU_ERR_INVALID_ARG;
    }
    if ((st = check_workspace(workspace, workspace_bytes, rglru_backward_workspace_size(dims))) != RGLRU_OK)
        return st;
    if (rglru::backward_tc_supported(dims))
        return cuda_status(rglru::launch_backward_tc(dims, params, x, y, reset, state0, dout, dh_final, dtail_final,
                                                     grads, workspace, workspace_bytes,
                                                     static_cast<cudaStream_t>(stream)));
    return cuda_status(rglru::launch_backward(dims, params, x, y, reset, state0, dout, dh_final, dtail_final,
                                              grads, workspace, workspace_bytes,
                                              static_cast<cudaStream_t>(stream)));
}

rglru_status rglru_block_prefill_noalloc(const rglru_dims* dims, const rglru_params* params,
                                         const void* x, const void* y, const uint8_t* reset,
                                         rglru_state* state, void* out, void* status_out,
                                         void* stream) {
    rglru_status st = check_dims(dims, true);
    if (st != RGLRU_OK) return st;
    if ((st = check_params(params)) != RGLRU_OK) return st;
    if ((st = check_io(x, y, out)) != RGLRU_OK) return st;
    if (state && (st = check_state(state)) != RGLRU_OK) return st;
    if (status_out && !aligned(status_out, 16)) return RGLRU_ERR_INVALID_ARG;
    const size_t need = rglru_prefill_workspace_size(dims);
    if (need == 0 || need > RGLRU_NOALLOC_SCRATCH_BYTES) return RGLRU_ERR_WORKSPACE;
    void* scratch = nullptr;
    cudaError_t e = noalloc_scratch(&scratch);
    if (e != cudaSuccess) return cuda_status(e);
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    // the area keeps the previous call's contents: the status word must start at zero (the
    // kernels clear their own tickets and flags)
    e = cudaMemsetAsync(scratch, 0, sizeof(rglru::DeviceStatus), s);
    if (e != cudaSuccess) return cuda_status(e);
    if (rglru::fused_prefill_supported(dims))
        e = rglru::launch_fused_prefill(dims, params, x, y, reset, state, out, scratch,
                                        RGLRU_NOALLOC_SCRATCH_BYTES, s);
    else
        e = rglru::launch_prefill_generic(dims, params, x, y, reset, state, out, s);
    if (e == cudaSuccess && status_out)
        e = cudaMemcpyAsync(status_out, scratch, sizeof(rglru::DeviceStatus), cudaMemcpyDeviceToDevice, s);
    return cuda_status(e);
}

rglru_status rglru_prefill_plan(const rglru_dims* dims, int* kernel, int* launches) {
    rglru_status st = check_dims(dims, true);
    if (st != RGLRU_OK) return st;
    if (!kernel || !launches) return RGLRU_ERR_INVALID_ARG;
    const bool tc = rglru::fused_prefill_supported(dims);
    *kernel = tc ? RGLRU_KERNEL_TENSOR : RGLRU_KERNEL_GENERIC;
    *launches = tc ? rglru::fused_prefill_launches(dims) : 1;
    return RGLRU_OK;
}

rglru_status rglru_decode_plan(const rglru_dims* dims, int* kernel, int* launches) {
    rglru_status st = check_dims(dims, false);
    if (st != RGLRU_OK) return st;
    if (!kernel || !launches) return RGLRU_ERR_INVALID_ARG;
    const bool tc = rglru::fused_decode_supported(dims);
    *kernel = tc ? RGLRU_KERNEL_TENSOR : RGLRU_KERNEL_GENERIC;
    *launches = tc ? rglru::fused_decode_launches(dims) : 1;
    return RGLRU_OK;
}

rglru_status rglru_backward_plan(const rglru_dims* dims, int* kernel, int* launches) {
    rglru_status st = check_dims(dims, true);
    if (st != RGLRU_OK) return st;
    if (!kernel || !launches) return RGLRU_ERR_INVALID_ARG;
    const bool tc = rglru::backward_tc_supported(dims);
    *kernel = tc ? RGLRU_KERNEL_TENSOR : RGLRU_KERNEL_GENERIC;
    *launches = tc ? rglru::backward_tc_launches(dims) : rglru::backward_launches(dims);
    return RGLRU_OK;
}

rglru_status rglru_read_device_status(void* workspace, size_t workspace_bytes, void* stream) {
    if (!workspace || workspace_bytes < sizeof(rglru::DeviceStatus) || !aligned(workspace, 256))
        return RGLRU_ERR_INVALID_ARG;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    rglru::DeviceStatus host{};
    cudaError_t e = cudaMemcpyAsync(&host, workspace, sizeof host, cudaMemcpyDeviceToHost, s);
    if (e == cudaSuccess) e = cudaStreamSynchronize(s);
    if (e == cudaSuccess) e = cudaMemsetAsync(workspace, 0, sizeof host, s);
    if (e == cudaSuccess) e = cudaStreamSynchronize(s);
    if (e != cudaSuccess) return cuda_status(e);
    if (host.code == 0) return RGLRU_OK;
    if (host.code == RGLRU_ERR_TIMEOUT) return RGLRU_ERR_TIMEOUT;
    return RGLRU_ERR_DEVICE;
}

}  // extern "C"

int rglru_last_cuda_error(const char** name) {
    if (name) *name = cudaGetErrorName(t_last_cuda_error);
    return (int)t_last_cuda_error;
}
