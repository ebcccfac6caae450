/*
 * rglru.h -- C ABI of the B200 (sm_100a) RG-LRU recurrent-block library (librglru.so).
 *
 * The block, per batch row b, head h, channel ch = h * head_dim + j and token t:
 *
 *   xc_t  = conv_b + sum_{k=0..3} conv_w[k] * x~_{t-3+k}          causal depthwise conv
 *   r_t   = sigmoid(xc_t(head) @ W_a[h] + b_a)                     recurrence gate
 *   i_t   = sigmoid(xc_t(head) @ W_x[h] + b_x)                     input gate
 *   log a_t = c * r_t * log sigmoid(Lambda)                        dynamic diagonal decay
 *   h_t   = a_t * h_{t-1} + sqrt(1 - a_t^2) * (i_t * xc_t)          diagonal linear scan
 *   out_t = h_t * GeLU(y_t)                                         multiplicative merge
 *
 * Sources ("Griffin Guide: RecurrentGemma, RG-LRU & Hybrid Attention"): the four governing
 * equations and the log-space decay in "1. Formulation of the RG-LRU Gating Mechanism"; the
 * sqrt(1 - a^2) factor in "2. The Role of Square-Root Variance Normalization"; the width-4
 * depthwise conv before the RG-LRU in "1. Temporal Filtering via Separable 1D Convolutions";
 * the GeLU merge in "2. Non-Linear Multiplicative Gating with GeLU"; per-head block-diagonal
 * W_a / W_x in "3. Block-Diagonal Sharding for Zero-Communication Tensor Parallelism"; the
 * conv padding (left K-1, truncated to T), the carried (y, last_state) and the zero initial
 * state in the listing "1. PyTorch Implementation of RG-LRU and the Griffin Block"
 * (RGLRU.forward / RGLRU.step / RecurrentBlock.forward).
 *
 * Conventions shared by every entry point
 *   - All tensor pointers are DEVICE pointers owned by the caller; the library allocates no
 *     memory, keeps no per-call state on the host and never synchronises unless stated.
 *   - Work is enqueued on `stream` (a cudaStream_t; NULL = the legacy default stream) in
 *     stream order; outputs are valid once the stream reaches that point.
 *   - Arguments are validated on the host before anything is launched; on any error nothing
 *     is launched and no output is touched.
 *   - Layouts are row-major.  W = heads * head_dim.  Activations ("act dtype": fp32 or bf16)
 *       x, y, out        [B, T, W]  (prefill)   /  [B, W]  (decode)
 *       w_a, w_x         [heads, head_dim(in), head_dim(out)], act dtype:
 *                        gate_o = b_o + sum_i xc_i * W[h][i][o]
 *       conv_w           [4, W] fp32, tap-major, tap 3 multiplies the current token
 *       conv_b, b_a, b_x [W] fp32, each may be NULL (= zeros)
 *       lambda           [W] fp32 (a = sigmoid(lambda))
 *       reset            [B, T] uint8 (prefill) / [B] (decode) or NULL; nonzero = that
 *                        token starts a new segment (document): the conv history is emptied
 *                        and h_{t-1} := 0 before the normal update
 *       state.h          [B, W] fp32;  state.conv_tail [B, 3, W] act dtype: the last three
 *                        x-branch inputs (pre-conv) of the current segment, oldest first
 *   - x, y, out, w_a, w_x, conv_tail must be 16-byte aligned; fp32 parameter vectors and
 *     state.h must be 4-byte aligned.  Outputs must not alias inputs (the state is in/out).
 *   - Supported shapes: conv_width == 4; head_dim a multiple of 16 in [16, 256]; batch >= 1;
 *     seq_len >= 1 (prefill); heads >= 1; W * sizeof(act) a multiple of 16.
 *   - GeLU is exact, v * Phi(v), unless dims.gelu_tanh = 1 selects the tanh approximation.
 *   - There is no CPU fallback: without a usable CUDA device every launching call returns
 *     RGLRU_ERR_CUDA.
 */
#ifndef RGLRU_H
#define RGLRU_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define RGLRU_ABI_VERSION 1

#if defined(__GNUC__)
#define RGLRU_API __attribute__((visibility("default")))
#else
#define RGLRU_API
#endif

typedef enum { RGLRU_F32 = 0, RGLRU_BF16 = 1 } rglru_dtype;

typedef enum {
    RGLRU_OK = 0,
    RGLRU_ERR_INVALID_ARG = 1,  /* NULL / misaligned pointer, non-positive size, bad enum */
    RGLRU_ERR_UNSUPPORTED = 2,  /* valid but outside the supported shapes above */
    RGLRU_ERR_WORKSPACE = 3,    /* workspace NULL or smaller than the queried size */
    RGLRU_ERR_CUDA = 4,         /* a CUDA runtime call or launch failed */
    RGLRU_ERR_TIMEOUT = 5,      /* device side: a bounded wait expired (see read_device_status) */
    RGLRU_ERR_DEVICE = 6        /* device side: an internal consistency check failed */
} rglru_status;

/* Problem description.  `flags` is 0 in normal use; bit RGLRU_FLAG_GENERIC forces the
 * portable (non-tensor-core) kernels, bit RGLRU_FLAG_TEST_WITHHOLD makes the fused prefill
 * kernel withhold the carry of its first time chunk, and the tensor-core decode step's first
 * CTA withhold its conv block from the other CTAs of its cluster, so that their bounded waits
 * expire after 2 ms (a test hook for the timeout path; outputs and state are then undefined). */
typedef struct {
    int batch;        /* B */
    int seq_len;      /* T (prefill); ignored by decode */
    int heads;        /* H */
    int head_dim;     /* dh */
    int conv_width;   /* must be 4 */
    int act_dtype;    /* rglru_dtype of x, y, out, w_a, w_x, conv_tail */
    float c;          /* decay scale c (8 on the pages) */
    int gelu_tanh;    /* 0 = exact GeLU, 1 = tanh approximation */
    unsigned flags;
} rglru_dims;

#define RGLRU_FLAG_GENERIC 1u
#define RGLRU_FLAG_TEST_WITHHOLD 2u

typedef struct {
    const float* conv_w;  /* [4, W] */
    const float* conv_b;  /* [W] or NULL */
    const void* w_a;      /* [H, dh, dh] act dtype */
    const void* w_x;      /* [H, dh, dh] act dtype */
    const float* b_a;     /* [W] or NULL */
    const float* b_x;     /* [W] or NULL */
    const float* lambda;  /* [W] */
} rglru_params;

typedef struct {
    float* h;          /* [B, W] fp32 */
    void* conv_tail;   /* [B, 3, W] act dtype */
} rglru_state;

/* Gradients written by rglru_block_backward (device pointers, fp32, overwritten).  dx, dy:
 * [B, T, W]; dh0: [B, W] and dtail0: [B, 3, W] (the initial state's gradient; either may be
 * NULL when not wanted); dconv_w [4, W]; dconv_b, db_a, db_x, dlambda [W]; dw_a, dw_x
 * [H, dh, dh] in the layout of w_a, w_x.  Gradients of absent biases are still written. */
typedef struct {
    float* dx;
    float* dy;
    float* dh0;
    float* dtail0;
    float* dconv_w;
    float* dconv_b;
    float* dw_a;
    float* dw_x;
    float* db_a;
    float* db_x;
    float* dlambda;
} rglru_grads;

/* Zero-fills state->h and state->conv_tail (the listing's "no prev_state" start).
 * Enqueued on `stream`.  Errors: INVALID_ARG (NULL/misaligned), CUDA. */
RGLRU_API rglru_status rglru_state_init(const rglru_dims* dims, rglru_state* state, void* stream);

/* Bytes of device workspace rglru_block_prefill needs for `dims` (0 on invalid dims).
 * The workspace is scratch owned by the caller; it must be 256-byte aligned, it may be
 * reused across calls on the same stream, and two calls in flight at once (on different
 * streams) need different workspaces.  Its first 16 bytes hold the device status word. */
RGLRU_API size_t rglru_prefill_workspace_size(const rglru_dims* dims);

/* Full-sequence prefill: out = block(x, y) over T tokens for every row.
 *   state == NULL: start from zero state, final state discarded.
 *   state != NULL: start from *state, and overwrite *state with the state after token T-1
 *                  (h_{T-1} and the last three x inputs of the final segment).
 * Follows RGLRU.forward / RecurrentBlock.forward of the listing, with the conv's history
 * taken from conv_tail instead of zero padding when a state is given.
 * Errors: INVALID_ARG, UNSUPPORTED, WORKSPACE, CUDA (host side, nothing launched).  Device
 * side conditions (TIMEOUT, DEVICE) are latched in the workspace status word: read them
 * with rglru_read_device_status. */
RGLRU_API rglru_status rglru_block_prefill(const rglru_dims* dims, const rglru_params* params,
                                 const void* x, const void* y, const uint8_t* reset,
                                 rglru_state* state, void* out,
                                 void* workspace, size_t workspace_bytes, void* stream);

/* Bytes of device workspace rglru_block_decode needs (at least 16: the status word). */
RGLRU_API size_t rglru_decode_workspace_size(const rglru_dims* dims);

/* One single-token decode step for every row (RGLRU.step of the listing, plus the conv):
 * conv over conv_tail[0..2] and x, gates, state update in place, out = h * GeLU(y), then the
 * conv history shifts left by one and appends x.  reset[b] != 0 empties row b's state first.
 * state is required (in/out).  dims.seq_len is ignored.  Errors as for prefill. */
RGLRU_API rglru_status rglru_block_decode(const rglru_dims* dims, const rglru_params* params,
                                const void* x, const void* y, const uint8_t* reset,
                                rglru_state* state, void* out,
                                void* workspace, size_t workspace_bytes, void* stream);

/* Persistent multi-step decode: `steps` successive single-token decode steps of every row in one
 * call (RGLRU.step of the listing, plus the conv, applied steps times), for a batch of decode
 * slots under continuous batching.
 *   x, y, out  [steps, B, W] act dtype: the token of step s for row b at [s][b][:]
 *   reset      [steps, B] uint8 or NULL: reset[s][b] != 0 empties row b's state (h and the conv
 *              history) before step s, so a slot can take a new sequence at any step
 *   state      required, in/out: the state before step 0, overwritten with the state after the
 *              last step
 * Results equal `steps` calls of rglru_block_decode in order (up to the rounding of the
 * arithmetic).  The tensor-core path (bf16, head_dim 256, state->h 16-byte aligned) is one
 * launch that keeps the state of every row on chip from the first step to the last, so only x,
 * y and out move per step; other shapes run the portable step kernel once per step.
 * Workspace: rglru_decode_steps_workspace_size bytes (the status word).  Errors as for
 * rglru_block_decode, and INVALID_ARG when steps <= 0. */
RGLRU_API size_t rglru_decode_steps_workspace_size(const rglru_dims* dims, int steps);
RGLRU_API rglru_status rglru_block_decode_steps(const rglru_dims* dims, const rglru_params* params,
                                                const void* x, const void* y, const uint8_t* reset,
                                                int steps, rglru_state* state, void* out,
                                                void* workspace, size_t workspace_bytes, void* stream);
/* How rglru_block_decode_steps runs for `dims` and `steps`: *kernel as for the other plans,
 * *launches = 1 on the tensor-core path, `steps` otherwise. */
RGLRU_API rglru_status rglru_decode_steps_plan(const rglru_dims* dims, int steps, int* kernel, int* launches);

/* The projections on either side of the block (the listing's RecurrentBlock.forward:
 * proj_in_1 / proj_in_2 / proj_out; linear_x / linear_y / linear_out in RecurrentGemma):
 *   model_dim  D, a multiple of 64
 *   w_in_x     [D, W] act dtype: x = u @ w_in_x    (the conv / RG-LRU branch)
 *   w_in_y     [D, W] act dtype: y = u @ w_in_y    (the GeLU branch)
 *   w_out      [W, D] act dtype: out = z @ w_out   (z = h * GeLU(y), the block's output) */
typedef struct {
    int model_dim;
    const void* w_in_x;
    const void* w_in_y;
    const void* w_out;
} rglru_projections;

/* Bytes of device workspace rglru_layer_forward needs for `dims` (0 on invalid dims): the
 * block's prefill workspace and the x, y, z activations [B, T, W] in the act dtype. */
RGLRU_API size_t rglru_layer_workspace_size(const rglru_dims* dims);

/* The recurrent block with its projections, for a whole sequence:
 *   u [B, T, D] act dtype  ->  out [B, T, D] act dtype
 *   x = u w_in_x, y = u w_in_y, z = rglru_block_prefill(x, y, reset, state), out = z w_out.
 * The projections run on the tensor cores with fp32 accumulation and bf16 results; x, y and z
 * live in the workspace.  reset / state as for rglru_block_prefill.  Supported: bf16, head_dim
 * 256, model_dim a multiple of 64 (else UNSUPPORTED).  Errors as for rglru_block_prefill; the
 * device status word is the workspace's first 16 bytes. */
RGLRU_API rglru_status rglru_layer_forward(const rglru_dims* dims, const rglru_params* params,
                                           const rglru_projections* proj, const void* u,
                                           const uint8_t* reset, rglru_state* state, void* out,
                                           void* workspace, size_t workspace_bytes, void* stream);
/* *kernel = RGLRU_KERNEL_TENSOR and *launches = the operations one rglru_layer_forward call
 * enqueues (three projection GEMMs and the block's), or UNSUPPORTED. */
RGLRU_API rglru_status rglru_layer_plan(const rglru_dims* dims, const rglru_projections* proj, int* kernel,
                                        int* launches);

/* ---- Griffin's second temporal-mixing block: local sliding-window multi-query attention ----
 * ("Griffin Guide: RecurrentGemma, RG-LRU & Hybrid Attention", "2. Local Sliding-Window
 * Multi-Query Attention (MQA)" and "3. Bounding the Key-Value Cache Footprint"; "Griffin"
 * notes, "Local Attention Path").  q_heads query heads share one key and one value head; token
 * t attends to the positions N(t) = {i : t - window < i <= t} of its own sequence:
 *     y_t = sum_{i in N(t)} softmax_i(scale * q_t . k_i) v_i,
 * with rotary position embeddings on q and k: the pairs (j, j + head_dim/2) of position p turn
 * by p * rope_base^(-2j / head_dim).  All tensors bf16, row-major; head_dim 256, 1 <= q_heads
 * <= 16, window >= 1 (else UNSUPPORTED).  Device pointers owned by the caller, work on `stream`.
 * The ring cache of a row holds, for position p, its rotated key in slot p mod window and its
 * value in the same slot of the value half: [B][2][window][head_dim]. */
typedef struct {
    int batch;        /* B */
    int seq_len;      /* T (prefill); ignored by decode */
    int q_heads;      /* H */
    int head_dim;     /* d, 256 */
    int window;       /* w */
    float scale;      /* score scale > 0, e.g. 1 / sqrt(head_dim) */
    float rope_base;  /* e.g. 10000 */
} rglru_mqa_dims;

/* Workspace bytes of rglru_mqa_prefill (decode = 0) or rglru_mqa_decode (decode = 1); 0 on
 * invalid dims.  256-byte aligned, first 16 bytes: the device status word. */
RGLRU_API size_t rglru_mqa_workspace_size(const rglru_mqa_dims* dims, int decode);

/* Prefill: q [B, T, H, d], k, v [B, T, d] at positions pos0 .. pos0 + T - 1 -> out
 * [B, T, H, d].  The window is restricted to the T tokens given.  cache: NULL, or the ring
 * cache [B][2][w][d], which receives the last min(T, w) rotated keys and values.  The score
 * contraction and the weighted sum run on the tensor cores (bf16 operands, fp32 accumulation).
 * Errors: INVALID_ARG, UNSUPPORTED, WORKSPACE, CUDA. */
RGLRU_API rglru_status rglru_mqa_prefill(const rglru_mqa_dims* dims, const void* q, const void* k,
                                         const void* v, int pos0, void* out, void* cache,
                                         void* workspace, size_t workspace_bytes, void* stream);

/* One decode token per row: q [B, H, d], k, v [B, d] at position pos[b] (a device int32 array
 * [B]); the rotated key and the value are written into slot pos[b] mod w of the row's ring, then
 * the token attends to the positions max(0, pos - w + 1) .. pos, all of which must have been
 * written by earlier prefill or decode calls.  out [B, H, d].  Errors as rglru_mqa_prefill. */
RGLRU_API rglru_status rglru_mqa_decode(const rglru_mqa_dims* dims, const void* q, const void* k,
                                        const void* v, const int* pos, void* cache, void* out,
                                        void* workspace, size_t workspace_bytes, void* stream);

/* Prefill for callers that cannot allocate device memory.  The pages have no counterpart:
 * this is a deployment variant of rglru_block_prefill, not a step of the method.
 *
 * Some callers cannot call cudaMalloc at all -- an engine whose device memory is one pool
 * carved up before serving starts, a plugin inside a host that owns every allocation, code
 * that runs where an allocation would synchronise the device.  They cannot provide the
 * workspace rglru_block_prefill asks for.  This entry point computes exactly what
 * rglru_block_prefill computes (same kernels, same arguments minus the workspace) and
 * takes its scratch from a fixed area that the library reserves statically on the device:
 *   - size RGLRU_NOALLOC_SCRATCH_BYTES; a problem whose rglru_prefill_workspace_size(dims)
 *     exceeds it is rejected with RGLRU_ERR_WORKSPACE before anything is enqueued;
 *   - the area is part of the library's device image: it stays reserved on every device that
 *     has loaded it (with CUDA's default lazy loading: from this entry point's first call on
 *     that device) until the process exits;
 *   - the first call on each device looks up the area's device address (with that device
 *     current), so make that first call before any stream capture; the lookup is repeated
 *     when the device's context has changed since (after a cudaDeviceReset the area is
 *     reloaded at another address), so the first call after such a reset must also come
 *     before any capture;
 *   - all calls share the one area and it keeps the previous call's contents; each call
 *     clears what must start at zero (its status word and the kernel's tickets and flags);
 *     two calls that overlap on the GPU (different streams, or concurrent host threads) race
 *     on it and give undefined results, so serialise them.
 * status_out: NULL, or a 16-byte, 16-byte aligned device buffer owned by the caller; after
 * the kernel the device status word (code, where, info0, info1 as 32-bit words) is copied
 * into it in stream order, so that a device-side TIMEOUT / DEVICE condition can be read
 * (rglru_read_device_status decodes it when the buffer is 256-byte aligned).
 * Besides what rglru_prefill_plan counts for rglru_block_prefill, each call enqueues one
 * more memset (its status word) and, when status_out is given, one device-to-device copy.
 * Nothing here calls cudaMalloc, cudaFree or any allocating routine.
 * Errors: as rglru_block_prefill (INVALID_ARG, UNSUPPORTED, CUDA), and WORKSPACE when the
 * problem does not fit the static area. */
#define RGLRU_NOALLOC_SCRATCH_BYTES ((size_t)16 << 20)
RGLRU_API rglru_status rglru_block_prefill_noalloc(const rglru_dims* dims,
                                 const rglru_params* params, const void* x, const void* y,
                                 const uint8_t* reset, rglru_state* state, void* out,
                                 void* status_out, void* stream);

/* Bytes of device workspace rglru_block_backward needs (0 on invalid dims): the status word,
 * four fp32 [B, T, W] arrays of per-token forward terms and eight fp32 [B, W] partial sums. */
RGLRU_API size_t rglru_backward_workspace_size(const rglru_dims* dims);

/* Backward pass of the prefill (the pages give the forward only; this is its chain rule,
 * training being the pages' other use of the block): with out, h_{T-1} and the final conv
 * history tail_T those of rglru_block_prefill(dims, params, x, y, reset, state0 copy), writes
 * the gradients of
 *     L = <dout, out> + <dh_final, h_{T-1}> + <dtail_final, tail_T>
 * with respect to x, y, every parameter and the initial state into *grads.
 *   x, y, dout [B, T, W] act dtype; reset [B, T] or NULL, as for the prefill.
 *   state0: the state the forward started from, or NULL for zero (not modified).
 *   dh_final [B, W], dtail_final [B, 3, W] fp32, or NULL for zero.
 * CUDA cores, fp32 arithmetic; the forward is recomputed, so only its inputs are needed.
 * Outputs must not alias inputs.  Errors as for rglru_block_prefill (host side, nothing
 * launched on error). */
RGLRU_API rglru_status rglru_block_backward(const rglru_dims* dims, const rglru_params* params,
                                            const void* x, const void* y, const uint8_t* reset,
                                            const rglru_state* state0, const void* dout,
                                            const float* dh_final, const float* dtail_final,
                                            const rglru_grads* grads, void* workspace,
                                            size_t workspace_bytes, void* stream);

/* How a call with `dims` runs (rglru_block_prefill, rglru_block_decode, rglru_block_backward):
 * *kernel receives RGLRU_KERNEL_GENERIC (CUDA-core kernels) or RGLRU_KERNEL_TENSOR (tcgen05 /
 * TMEM kernels), *launches the number of operations one call enqueues (the tensor-core prefill
 * counts its workspace memset with its kernel; its copy of a given conv history is not
 * counted).  The choice depends on dims only (the library targets sm_100a alone).
 * Errors: INVALID_ARG / UNSUPPORTED exactly as the corresponding call would return them. */
#define RGLRU_KERNEL_GENERIC 0
#define RGLRU_KERNEL_TENSOR 1
RGLRU_API rglru_status rglru_prefill_plan(const rglru_dims* dims, int* kernel, int* launches);
RGLRU_API rglru_status rglru_decode_plan(const rglru_dims* dims, int* kernel, int* launches);
RGLRU_API rglru_status rglru_backward_plan(const rglru_dims* dims, int* kernel, int* launches);

/* Synchronises `stream`, reads and clears the device status word at the start of
 * `workspace`, and returns RGLRU_OK, RGLRU_ERR_TIMEOUT or RGLRU_ERR_DEVICE (or
 * INVALID_ARG / CUDA for a bad argument or a failed copy). */
RGLRU_API rglru_status rglru_read_device_status(void* workspace, size_t workspace_bytes, void* stream);

/* Static, human-readable name of a status code. */
RGLRU_API const char* rglru_status_string(rglru_status status);

/* The CUDA runtime error (cudaError_t value) behind the calling host thread's most recent
 * RGLRU_ERR_CUDA, 0 if it has had none; *name (when name is not NULL) receives the runtime's
 * static name of that error.  Diagnostic only: it does not clear the value. */
RGLRU_API int rglru_last_cuda_error(const char** name);

/* RGLRU_ABI_VERSION of the built library. */
RGLRU_API int rglru_abi_version(void);

#ifdef __cplusplus
}
#endif

#endif /* RGLRU_H */
