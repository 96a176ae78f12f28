/*
 * moe_decode.h -- C ABI of the B200 (sm_100a) MoE decode-layer library.
 *
 * One call of moe_decode_step runs one decode step of a Kimi-K3-style
 * mixture-of-experts layer (or a stack of such layers) for a batch of 1..64
 * tokens on one GPU:
 *
 *   h      = residual_in + W_o . attn_out             o_proj fused with the residual
 *   x      = h * rstd(h) * gamma                       RMSNorm, eps from the config
 *   logits = W_r . x                                   router, fp32 accumulation
 *   idx    = top-k of logits (descending, ties to the lower expert index)
 *   gate   = softmax over the k selected logits
 *   out    = bf16(h + sum_j gate_j * W_down[e_j] . (silu(W_g[e_j] x) * W_u[e_j] x))
 *
 * Sources: "vLLM speeds up Kimi K3 up to 1.9x on NVIDIA GB300 with
 * agent-assisted kernels", section "How the specialised decode path works"
 * (16 of 896 experts active per token; kernels chosen by batch size, small-
 * matrix kernels at batch one or two and split-K above; the attention output
 * projection fused with the residual step; a side kernel that prefetches the
 * next layer's weights because decode is bound by weight reads); "vLLM and
 * NVIDIA use coding agents to nearly double Kimi K3 decode speed, then rethink
 * how to review it" (23 -> 13 kernels per layer); "vLLM tests a fast-track
 * review model with Kimi K3's specialized decode path", section "Why the
 * review model matters" (unsupported configurations are rejected at startup).
 * The RMSNorm, softmax gates renormalised over the selected experts, SwiGLU
 * experts and the bf16 output are the layer's stated configuration.
 *
 * Conventions
 *   - All functions return 0 (MOE_OK) or a negative MOE_ERR_* code; nothing is
 *     thrown across the ABI.  moe_decode_strerror names a code.
 *   - Pointers marked "device" are CUDA device pointers on the handle's device;
 *     "host" pointers are CPU memory (pinned memory makes copies asynchronous).
 *   - Tensors are dense row-major; bf16 tensors are raw 16-bit bf16 values.
 *   - Weights are borrowed: the caller owns them and must keep them alive and
 *     unchanged for the handle's lifetime.  The handle owns its workspace and
 *     its captured CUDA graphs.
 *   - Streams are cudaStream_t values passed as void*; NULL is the legacy
 *     default stream.
 */
#ifndef MOE_DECODE_H
#define MOE_DECODE_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define MOE_API __attribute__((visibility("default")))
#else
#define MOE_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

enum {
  MOE_OK = 0,
  MOE_ERR_INVALID_ARG = -1,        /* null/ill-formed argument, batch out of range */
  MOE_ERR_UNSUPPORTED_CONFIG = -2, /* shapes or device outside the supported set  */
  MOE_ERR_ALIGNMENT = -3,          /* a pointer is not 16-byte aligned              */
  MOE_ERR_OOM = -4,                /* workspace allocation failed                   */
  MOE_ERR_CUDA = -5,               /* a CUDA runtime call failed                    */
  MOE_ERR_DEVICE_TIMEOUT = -6,     /* a kernel's bounded wait ran out               */
  MOE_ERR_DEVICE_BOUNDS = -7,      /* a kernel met an out-of-range index and skipped it */
  MOE_ERR_SCRATCH_LIMIT = -8       /* moe_decode_step_static: scratch need above MOE_STATIC_SCRATCH_BYTES */
};

/* Layer shapes and options, fixed at create time.
 *   d          hidden size (RMSNorm width, router and expert input)  64 <= d <= 8192, d % 64 == 0
 *   d_o        o_proj input width (heads x head_dim)                 64 <= d_o <= 8192, d_o % 64 == 0
 *   n_experts  E, routed experts                                     k <= E <= 1024
 *   top_k      k, experts per token                                  1 <= k <= 32
 *   inter      I, SwiGLU intermediate size per expert                32 <= I <= 512, I % 32 == 0
 *   max_batch  largest batch passed to step                          1 <= max_batch <= 64
 *   n_layers   layers run back to back by one step (residual chains)  1 <= n_layers <= 64
 *   rms_eps    RMSNorm epsilon (> 0; the layer uses 1e-6)
 *   enable_prefetch  1: layer l prefetches into L2 what layer l+1 reads first (its
 *                    router matrix, RMSNorm scale and the leading 16 MB of its W_o,
 *                    split by the CTA that reads them), issued once layer l's own
 *                    router rows are in flight; no extra kernel
 *   force_variant    0: kernels by batch size (B = 1: one fused layer kernel; B = 2 to 4
 *                    with B * top_k <= 64: o_proj, router, small-M expert kernel; above:
 *                    o_proj, router, gate/up, down);
 *                    1: at B = 1 too the three small-batch kernels (testing);
 *                    2: the large-batch kernels at every batch size (testing);
 *                    3: at B <= 2 the layer kernel whose expert phase is ordered by
 *                       per-expert counters instead of a grid barrier (testing)           */
typedef struct {
  int d, d_o, n_experts, top_k, inter, max_batch, n_layers;
  float rms_eps;
  int enable_prefetch;
  int force_variant;
} moe_decode_config;

/* One layer's weights (device, bf16, row-major [out][in], 16-byte aligned):
 *   w_o        [d][d_o]
 *   gamma      [d]
 *   w_router   [n_experts][d]
 *   w_gate_up  [n_experts][2*inter][d]   rows 0..inter-1 gate, inter..2*inter-1 up
 *   w_down     [n_experts][d][inter]                                                 */
typedef struct {
  const void *w_o, *gamma, *w_router, *w_gate_up, *w_down;
} moe_decode_layer_weights;

typedef struct moe_decode_handle moe_decode_handle;

/* Validates the config against the supported set (sm_100 device, the limits
 * above, 16-byte aligned non-null weights for every layer) and rejects
 * anything else with MOE_ERR_UNSUPPORTED_CONFIG / MOE_ERR_ALIGNMENT /
 * MOE_ERR_INVALID_ARG.  Allocates the workspace on the current device.
 * weights points to n_layers structs (host memory, copied).  stream is used
 * for the workspace initialisation, which completes before create returns.
 * On success *out receives the handle; on failure *out is set to NULL. */
MOE_API int moe_decode_create(const moe_decode_config* cfg, const moe_decode_layer_weights* weights,
                      void* stream, moe_decode_handle** out);

/* Runs one step for `batch` tokens (1 <= batch <= max_batch), asynchronously
 * on `stream`.  All buffers are device memory, 16-byte aligned:
 *   attn_out     [n_layers][batch][d_o] bf16   layer l's attention output
 *   residual_in  [batch][d] bf16               residual entering layer 0
 *   out          [batch][d] bf16               output of the last layer
 *   topk_idx     [n_layers][batch][top_k] int32, or NULL
 *   topk_gate    [n_layers][batch][top_k] fp32, or NULL
 * Layer l+1's residual is layer l's bf16 output (held in the workspace).
 * The step replays a CUDA graph captured for (batch, these five addresses);
 * the first step with a new tuple captures one (milliseconds; do it before
 * timing).  Outputs are valid once `stream` has been synchronised.  A device
 * error from this or an earlier step is reported by moe_decode_sync_status.
 * Concurrent steps on one handle share its workspace and must be serialised. */
MOE_API int moe_decode_step(moe_decode_handle* h, int batch, const void* attn_out,
                    const void* residual_in, void* out, int32_t* topk_idx, float* topk_gate,
                    void* stream);

/* Same step with HOST buffers (same shapes as moe_decode_step): gathers the
 * inputs into a handle-owned pinned buffer, moves them to handle-owned device
 * buffers in one copy, runs the step, moves the outputs back in one copy,
 * synchronises `stream` and scatters them into the caller's buffers (any host
 * memory, pinned or not).  topk_idx / topk_gate may be NULL.  The first call
 * allocates the staging (device and pinned host memory for max_batch tokens);
 * MOE_ERR_OOM if that fails. */
MOE_API int moe_decode_step_host(moe_decode_handle* h, int batch, const void* attn_out_host,
                         const void* residual_in_host, void* out_host, int32_t* topk_idx_host,
                         float* topk_gate_host, void* stream);

/* Synchronises `stream` and returns MOE_ERR_DEVICE_TIMEOUT / MOE_ERR_DEVICE_BOUNDS
 * if a kernel of an earlier step recorded one (the record is then cleared),
 * MOE_ERR_CUDA on a CUDA error, else MOE_OK. */
MOE_API int moe_decode_sync_status(moe_decode_handle* h, void* stream);

/* Makes the device error reporting run, without a fault, so that callers and tests can
 * check their handling of it.  Launches on `stream` one small kernel that uses the same
 * bounded-wait and index-check code as the step's kernels:
 *   what = 1  an mbarrier wait that nothing completes and a grid barrier that one arrival
 *             short can never open, each giving up after limit_ns nanoseconds; the next
 *             moe_decode_sync_status returns MOE_ERR_DEVICE_TIMEOUT;
 *   what = 2  an expert index one past the end, clamped and skipped; the next
 *             moe_decode_sync_status returns MOE_ERR_DEVICE_BOUNDS.
 * 0 < limit_ns <= 10,000,000 (10 ms); anything else is MOE_ERR_INVALID_ARG.  The record
 * stays in the handle's error word until moe_decode_sync_status reads and clears it; steps
 * in between run normally.  Returns MOE_OK once launched, MOE_ERR_CUDA if the launch fails. */
MOE_API int moe_decode_check_error_path(moe_decode_handle* h, int what, unsigned long long limit_ns,
                                        void* stream);

/* Intermediates of the most recent step's LAST layer, for tests:
 *   which = 0  h      [batch][d]          fp32
 *           1  rstd   [batch]             fp32
 *           2  x      [batch][d]          fp32
 *           3  logits [batch][n_experts]  fp32
 * Copies min(bytes, size) bytes into dst (device) on `stream`. */
MOE_API int moe_decode_get_intermediate(moe_decode_handle* h, int which, void* dst, size_t bytes,
                                void* stream);

/* Kernel launches in one step of `batch` tokens (graph nodes that run this
 * library's kernels), or a negative error code. */
MOE_API int moe_decode_kernels_per_step(moe_decode_handle* h, int batch);

/* Runs one step eagerly (no graph, no programmatic overlap between kernels) on
 * `stream` with a CUDA event pair around every kernel, synchronises, and writes
 * each kernel's duration in milliseconds, in launch order, to kernel_ms (host,
 * max_kernels entries) and a short kernel name id to kernel_id (host, or NULL):
 * 1 o_proj+residual+RMS, 2 router+top-k (and the next layer's L2 prefetch),
 * 3 small-M expert kernel (gate/up and down), 4 large-batch gate/up, 5 large-batch
 * down+combine, 6 fused batch <= 2 layer kernel (all of a layer).  Same buffers as
 * moe_decode_step.  Returns the number of kernels timed (or a negative code). */
MOE_API int moe_decode_profile_step(moe_decode_handle* h, int batch, const void* attn_out,
                                    const void* residual_in, void* out, int32_t* topk_idx,
                                    float* topk_gate, void* stream, float* kernel_ms,
                                    int* kernel_id, int max_kernels);

/* Capacity of the static scratch array used by moe_decode_step_static (1.5 MiB per device). */
#define MOE_STATIC_SCRATCH_BYTES (1536u * 1024u)

/* One layer step for batch 1 or 2 that allocates no device memory.  The pages have no
 * counterpart of this entry point; it exists for callers that may not allocate when they
 * run a step (an engine that has reserved nearly all device memory for its own pool, a
 * process under a hard memory cap).
 * It runs the same kernels as moe_decode_step's batch <= 2 path, launched directly on
 * `stream` (no graph, no handle), with every intermediate in one static device array of
 * MOE_STATIC_SCRATCH_BYTES that is part of the loaded library (one per device).
 *   cfg          layer shapes as for moe_decode_create (host, checked against the same
 *                supported set); n_layers must be 1 and force_variant 0, 1 or 3 (as in
 *                moe_decode_step: 1 the three small-batch kernels at batch 1 too, 3 the
 *                counter-ordered layer kernel); enable_prefetch is ignored
 *   w            the layer's weights (host struct of device pointers, as for create)
 *   batch        1 or 2, and <= cfg->max_batch
 *   attn_out     [batch][d_o] bf16, residual_in [batch][d] bf16, out [batch][d] bf16 (device)
 *   topk_idx     [batch][top_k] int32 or NULL; topk_gate [batch][top_k] fp32 or NULL (device)
 *   err_word     device uint32 (4-byte aligned) or NULL: receives this call's kernel error
 *                bits (0 none, 1 a bounded wait ran out, 2 an index out of range)
 * Errors: MOE_ERR_INVALID_ARG / MOE_ERR_UNSUPPORTED_CONFIG / MOE_ERR_ALIGNMENT as for
 * create and step; MOE_ERR_SCRATCH_LIMIT when the scratch for (cfg, batch) exceeds
 * MOE_STATIC_SCRATCH_BYTES (e.g. force_variant 3 with n_experts = 1024 at batch 2 on 148 SMs,
 * whose split-K router partial sums, SMs x n_experts x batch floats, take 1.2 MB of the 1.7 MB
 * needed); nothing is launched then.  MOE_ERR_CUDA on a failed CUDA call.
 * The first call on each device, with that device current, looks up the array's address
 * (cudaGetSymbolAddress) and sets kernel attributes; make that first call before any stream
 * capture begins.  Each call zeroes the barrier counters and error word at the head of the
 * array before its kernels run; nothing else needs a starting value.
 * All calls on a device share the array: calls whose executions overlap (different streams,
 * or threads without ordering) race on it and corrupt each other's results.  Outputs are
 * valid once `stream` has been synchronised. */
MOE_API int moe_decode_step_static(const moe_decode_config* cfg, const moe_decode_layer_weights* w, int batch,
                                   const void* attn_out, const void* residual_in, void* out,
                                   int32_t* topk_idx, float* topk_gate, uint32_t* err_word, void* stream);

/* Frees the graphs and the workspace; weights are not touched.  NULL is a no-op. */
MOE_API int moe_decode_destroy(moe_decode_handle* h);

MOE_API const char* moe_decode_strerror(int code);

#ifdef __cplusplus
}
#endif

#endif /* MOE_DECODE_H */
