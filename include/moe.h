/*
 * moe.h -- C ABI of a B200 (sm_100a) implementation of a Grok-1-style sparse
 * mixture-of-experts SwiGLU FFN layer: the forward pass (bf16 and fp32, with a
 * weight-streaming path for small batches and an int8-weight path), its
 * backward pass for training, and the row exchange helpers of multi-rank use.
 *
 * The operation follows the page "How does Grok-1 use a mixture-of-experts
 * design?" (n4n.ai):
 *   - section "The high-level architecture", GrokMoELayer.forward: router
 *     logits over 8 experts, top-2, softmax over the two selected logits,
 *     dispatch to the experts and weighted combine back to token order;
 *   - section "Routing: top-2 without auxiliary loss", grok_router_forward and
 *     the paragraph after it: router weight stored [E, hidden], capacity factor
 *     (1.25 in training; no dropping at inference);
 *   - section "Expert implementation: SwiGLU at scale", SwiGLUExpert and
 *     FusedSwiGLUExpert: y = W_down(silu(W_gate x) * W_up x), no bias.
 * and the page "Let Grok spill the beans on Grok", whose feature list states
 * that the layer output is the weighted sum of the active experts' outputs.
 *
 * Readings where the pages leave a step open:
 *   capacity = ceil(capacity_factor * T * top_k / E), computed in double in that
 *   order (+INFINITY: no drop); overflow is dropped lowest token index first;
 *   routing weights are not renormalised after a drop; a token with both
 *   assignments dropped outputs zero; equal logits rank the lower expert first.
 *
 * Conventions for every entry point:
 *   - Pointers named *_host are host memory; every other buffer pointer is
 *     device memory owned by the caller.  The library never allocates or frees
 *     device memory (moe_dispatch_noalloc uses one fixed array inside the
 *     library) and keeps no pointer after a call returns.
 *   - Tensors are dense row-major.  Buffers must be 16-byte aligned.
 *   - Work is enqueued on `stream` (a cudaStream_t); calls return before the
 *     GPU finishes, except moe_layer_forward_host, moe_layer_forward_host_batches
 *     and moe_get_device_error.
 *   - Argument errors are reported synchronously, before anything is launched:
 *     MOE_ERR_INVALID_ARG (null pointer, bad size, misalignment),
 *     MOE_ERR_UNSUPPORTED (E != 8, top_k != 2, d or f not a multiple of 128
 *     for bf16 / 64 for fp32), MOE_ERR_WORKSPACE (workspace too small).
 *     A failed launch returns MOE_ERR_CUDA.  Inputs are never modified.
 *   - Checks made by the kernels themselves (an expert index outside [0, E),
 *     a slot outside the buffers, inconsistent offsets, a pipeline wait that
 *     timed out) do not trap: the offending element is skipped and a device
 *     error word is set, read back with moe_get_device_error().
 *   - T == 0 is valid and launches nothing.
 */
#ifndef SPARSE_MOE_LAYER_07_B200_MOE_H
#define SPARSE_MOE_LAYER_07_B200_MOE_H

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

/* Same type as cudaStream_t; NULL is the legacy default stream. */
typedef struct CUstream_st* moe_stream_t;

typedef enum {
  MOE_OK = 0,
  MOE_ERR_INVALID_ARG = 1,
  MOE_ERR_UNSUPPORTED = 2,
  MOE_ERR_WORKSPACE = 3,
  MOE_ERR_CUDA = 4,
  MOE_ERR_DEVICE_CHECK = 5,
  MOE_ERR_TIMEOUT = 6
} moe_status_t;

/* Storage and arithmetic type of x, the weights and out.
 * MOE_F32:  fp32 everywhere (hidden activation H in fp32).
 * MOE_BF16: bf16 storage, fp32 accumulation, H rounded once to bf16. */
typedef enum { MOE_F32 = 0, MOE_BF16 = 1 } moe_dtype_t;

/* Bits of the device error word. */
#define MOE_DEVERR_EXPERT_INDEX 0x1 /* an expert id outside [0, E) */
#define MOE_DEVERR_SLOT_INDEX 0x2   /* a slot outside [0, T*top_k) */
#define MOE_DEVERR_OFFSETS 0x4      /* expert offsets not monotone or too large */
#define MOE_DEVERR_TIMEOUT 0x8      /* a pipeline wait ran past its limit */

/* Layer hyper-parameters ("GrokMoELayer" in the architecture section:
 * num_experts 8, top_k 2, hidden_size, expert_dim). */
typedef struct {
  int64_t T;              /* tokens = batch * seq_len */
  int64_t d;              /* hidden_size */
  int64_t f;              /* expert_dim */
  int32_t E;              /* num_experts; must be 8 */
  int32_t top_k;          /* must be 2 */
  double capacity_factor; /* > 0; +INFINITY means no drop */
  int32_t dtype;          /* moe_dtype_t */
  int32_t reserved;       /* must be 0 */
} moe_config_t;

/* Length of the stats array written by moe_layer_forward (int32):
 * [0, E) counts_raw, [E, 2E) counts_kept, [2E, 3E+1) offsets, [3E+1] dropped. */
#define MOE_STATS_LEN(E) (3 * (E) + 2)

/* Version of this ABI (incremented on incompatible change). */
MOE_API int32_t moe_abi_version(void);

/* Human-readable name of a status code (static string). */
MOE_API const char* moe_status_string(moe_status_t status);

/* Per-expert capacity min(T, ceil(capacity_factor * T * top_k / E)) (T when the
 * factor is +INFINITY; no expert can receive more than T assignments), as used
 * by moe_dispatch; -1 for an invalid config.
 * Definition: capacity paragraph of "Routing: top-2 without auxiliary loss". */
MOE_API int64_t moe_capacity(const moe_config_t* cfg);

/* Bytes of device workspace needed by moe_dispatch (per-block histograms). */
MOE_API size_t moe_dispatch_workspace_size(const moe_config_t* cfg);

/* Bytes of device workspace needed by moe_expert_ffn / moe_expert_down. */
MOE_API size_t moe_expert_ffn_workspace_size(const moe_config_t* cfg);

/* Bytes of device workspace needed by moe_layer_forward and
 * moe_layer_forward_host (all intermediates); 0 for an invalid config. */
MOE_API size_t moe_workspace_size(const moe_config_t* cfg);

/* Router and top-2 ("Routing: top-2 without auxiliary loss",
 * grok_router_forward; "The high-level architecture", forward):
 *   logits[t, e] = sum_i x[t, i] * w_router[e, i]  (+ logit_bias[e])
 *   topk_idx[t, 0..1] = the two largest logits, descending, ties to lower e
 *   topk_w[t, j]      = softmax over the two selected logits
 * x [T, d] and w_router [E, d] in cfg->dtype; accumulation in fp32.
 * logit_bias [E] fp32 or NULL; logits [T, E] fp32 or NULL (not written);
 * topk_idx [T, 2] int32; topk_w [T, 2] fp32. */
MOE_API moe_status_t moe_router_topk(const moe_config_t* cfg, const void* x, const void* w_router,
                             const float* logit_bias, float* logits, int32_t* topk_idx,
                             float* topk_w, moe_stream_t stream);

/* Capacity-factor dispatch (the "_apply_capacity" and grouping steps of
 * grok_router_forward / _dispatch_and_combine):
 *   counts_raw[e]  = number of assignments routed to e
 *   rank(t, e)     = number of tokens t' < t routed to e
 *   kept iff rank < capacity;   counts_kept[e] = min(counts_raw[e], capacity)
 *   offsets        = exclusive prefix sum of counts_kept (E + 1 entries)
 *   slot_of[t, j]  = offsets[e] + rank for a kept assignment, else -1
 *   perm[slot] = t,  row_scale[slot] = topk_w[t, j]
 *   x_perm[slot, :] = x[perm[slot], :]   (skipped when x_perm is NULL)
 * perm, row_scale: [T*2] (the first offsets[E] entries are written);
 * slot_of [T, 2]; x_perm [T*2, d] in cfg->dtype.  ws: moe_dispatch_workspace_size
 * bytes of scratch.  Deterministic: no atomics decide any output. */
MOE_API moe_status_t moe_dispatch(const moe_config_t* cfg, const void* x, const int32_t* topk_idx,
                          const float* topk_w, int32_t* counts_raw, int32_t* counts_kept,
                          int32_t* offsets, int32_t* perm, int32_t* slot_of, float* row_scale,
                          void* x_perm, void* ws, size_t ws_bytes, moe_stream_t stream);

/* A batch split into token shards, one per rank, under the global capacity rule
 * ("Routing: top-2 without auxiliary loss": capacity from the whole batch,
 * overflow dropped lowest token index first, the shards in rank order forming
 * the token order).  moe_route_counts writes counts[e] = assignments routed to
 * expert e by this shard (device int32 [E]).  After every shard's counts are
 * gathered in shard order into shard_counts [n_shards, E] (device int32; one
 * all-gather of E integers per rank), moe_dispatch_shard computes what
 * moe_dispatch computes for this shard with
 *   kept iff prior[e] + rank(t, e) < capacity,  prior[e] = sum over earlier shards
 * and counts_kept[e] = min(counts_raw[e], max(capacity - prior[e], 0)).
 * capacity is the global one (moe_capacity of the whole batch's config);
 * cfg->T is this shard's token count.  Deterministic, no atomics. */
MOE_API moe_status_t moe_route_counts(const moe_config_t* cfg, const int32_t* topk_idx, int32_t* counts,
                              moe_stream_t stream);
MOE_API moe_status_t moe_dispatch_shard(const moe_config_t* cfg, int64_t capacity, const int32_t* shard_counts,
                                int32_t n_shards, int32_t shard, const void* x, const int32_t* topk_idx,
                                const float* topk_w, int32_t* counts_raw, int32_t* counts_kept,
                                int32_t* offsets, int32_t* perm, int32_t* slot_of, float* row_scale,
                                void* x_perm, void* ws, size_t ws_bytes, moe_stream_t stream);

/* Row gather, dst[i, :] = src[idx[i], :] for i < n: rows of row_bytes bytes
 * (a multiple of 16), src holding n_src rows (device memory; idx device int32).
 * Used to regroup rows between the expert-major order of a rank's own experts
 * and the rank-major order of an all-to-all exchange (expert parallelism,
 * "Expert parallelism vs. tensor parallelism", moe_layer_ep_forward).  An
 * index outside [0, n_src) skips its row and sets MOE_DEVERR_SLOT_INDEX. */
MOE_API moe_status_t moe_gather_rows(const void* src, int64_t n_src, const int32_t* idx, int64_t n,
                             int64_t row_bytes, void* dst, moe_stream_t stream);

/* SwiGLU expert FFN over the grouped rows ("Expert implementation: SwiGLU at
 * scale", SwiGLUExpert / FusedSwiGLUExpert), for each expert e and each row r
 * in [offsets[e], offsets[e+1]):
 *   h[r, :] = silu(x_perm[r, :] @ w_gate[e]) * (x_perm[r, :] @ w_up[e])
 *   y[r, :] = row_scale[r] * (h[r, :] @ w_down[e])      (row_scale NULL: 1)
 * w_gate, w_up [E, d, f]; w_down [E, f, d]; x_perm [T*2, d]; h [T*2, f], all in
 * cfg->dtype; y [T*2, d] fp32.  offsets is the device array from moe_dispatch.
 * bf16 runs on the tensor cores with fp32 accumulation; h is rounded once. */
MOE_API moe_status_t moe_expert_ffn(const moe_config_t* cfg, const void* x_perm, const int32_t* offsets,
                            const void* w_gate, const void* w_up, const void* w_down,
                            const float* row_scale, void* h, float* y, void* ws, size_t ws_bytes,
                            moe_stream_t stream);

/* The two halves of moe_expert_ffn, for callers that time or overlap them:
 * gate/up with the fused SwiGLU epilogue (writes h), and down (writes y). */
MOE_API moe_status_t moe_expert_gate_up(const moe_config_t* cfg, const void* x_perm, const int32_t* offsets,
                                const void* w_gate, const void* w_up, void* h, moe_stream_t stream);
MOE_API moe_status_t moe_expert_down(const moe_config_t* cfg, const void* h, const int32_t* offsets,
                             const void* w_down, const float* row_scale, float* y, void* ws,
                             size_t ws_bytes, moe_stream_t stream);

/* Down projection with the combine fused (bf16 only, the tensor-core kernels
 * for batches above the weight-streaming size; d a multiple of 256):
 *   out[t, :] = sum over kept slots r of token t of row_scale[r] * (h[r, :] @ w_down[e])
 * in fp32, rounded once to cfg->dtype: moe_expert_down followed by moe_combine
 * with weights_applied = 1, bit for bit, without the y buffer (the down
 * epilogue adds each row into an fp32 sum by token; with two terms per token
 * the sum does not depend on their order).  h, offsets from moe_dispatch /
 * moe_expert_gate_up; perm, row_scale from moe_dispatch; out [T, d] in
 * cfg->dtype; ws: device scratch of moe_expert_down_combine_workspace_size(cfg)
 * bytes (the fp32 sums).  MOE_ERR_UNSUPPORTED outside that scope (fp32,
 * d % 256 != 0, or T * top_k <= 64 * E, where the weight-streaming kernels
 * run instead).  moe_layer_forward uses this path in its scope. */
MOE_API size_t moe_expert_down_combine_workspace_size(const moe_config_t* cfg);
MOE_API moe_status_t moe_expert_down_combine(const moe_config_t* cfg, const void* h, const int32_t* offsets,
                                     const void* w_down, const float* row_scale, const int32_t* perm, void* out,
                                     void* ws, size_t ws_bytes, moe_stream_t stream);

/* Weighted combine back to token order ("The high-level architecture",
 * _dispatch_and_combine; weighted sum of the active experts' outputs):
 *   out[t, :] = sum over j = 0, 1 with slot_of[t, j] >= 0 of
 *               s_j * y[slot_of[t, j], :]      (fp32, j = 0 first)
 * with s_j = 1 when weights_applied != 0 (y already carries the routing
 * weight) and s_j = topk_w[t, j] otherwise.  out [T, d] in cfg->dtype
 * (rounded once); a token with no kept assignment gets zeros. */
MOE_API moe_status_t moe_combine(const moe_config_t* cfg, const float* y, const int32_t* slot_of,
                         const float* topk_w, int32_t weights_applied, void* out,
                         moe_stream_t stream);

/* The whole layer forward: router -> dispatch -> expert FFN -> combine.
 * x [T, d]; w_router [E, d]; w_gate/w_up [E, d, f]; w_down [E, f, d]; out [T, d];
 * logit_bias [E] fp32 or NULL; stats: device int32[MOE_STATS_LEN(E)] or NULL.
 * ws: moe_workspace_size(cfg) bytes of device scratch, owned by the caller. */
MOE_API moe_status_t moe_layer_forward(const moe_config_t* cfg, const void* x, const void* w_router,
                               const float* logit_bias, const void* w_gate, const void* w_up,
                               const void* w_down, void* out, int32_t* stats, void* ws,
                               size_t ws_bytes, moe_stream_t stream);

/* moe_layer_forward with x and out in host memory: copies x_host to the device
 * (inside ws), runs the layer, copies the result to out_host and waits for the
 * stream.  Weights, logit_bias and ws are device memory.  Page-locked host
 * buffers make the copies asynchronous with respect to other work. */
MOE_API moe_status_t moe_layer_forward_host(const moe_config_t* cfg, const void* x_host, const void* w_router,
                                    const float* logit_bias, const void* w_gate, const void* w_up,
                                    const void* w_down, void* out_host, void* ws, size_t ws_bytes,
                                    moe_stream_t stream);

/* Bytes of device workspace needed by moe_layer_forward_host_batches:
 * moe_workspace_size plus a second x and out staging slot; 0 for an invalid
 * config. */
MOE_API size_t moe_workspace_size_host_batches(const moe_config_t* cfg);

/* The layer over n_batches independent batches of cfg->T tokens held in host
 * memory (one layer call per batch, as moe_layer_forward_host computes it),
 * with the copies overlapped with the compute: while batch i computes on
 * `stream`, batch i+1 is copied in and batch i-1 copied out on two streams of
 * the library's own, through two staging slots in ws.  Every batch's result is
 * bit-identical to moe_layer_forward on the same x.  The pages define one
 * forward call ("The high-level architecture", forward); this entry point only
 * schedules many of them, it adds no arithmetic.
 * x_host[i]: host [T, d] in cfg->dtype; out_host[i]: host [T, d]; both arrays
 * hold n_batches pointers; entries may repeat (a repeated out_host buffer ends
 * with the last batch written to it).  Page-locked buffers are needed for the
 * copies to overlap.  Weights, logit_bias and ws are device memory; ws holds
 * moe_workspace_size_host_batches(cfg) bytes.  The work is ordered after the
 * work already in `stream`; the call returns when every out_host[i] is filled.
 * n_batches == 0 does nothing.  The two copy streams and their seven events
 * are created on a device's first call and kept until the process exits
 * (re-created after a context reset); no device memory is allocated.  Calls on
 * one device from several host threads take turns (each call holds that
 * device's copy streams until it returns). */
MOE_API moe_status_t moe_layer_forward_host_batches(const moe_config_t* cfg, int64_t n_batches,
                                            const void* const* x_host, const void* w_router,
                                            const float* logit_bias, const void* w_gate, const void* w_up,
                                            const void* w_down, void* const* out_host, void* ws,
                                            size_t ws_bytes, moe_stream_t stream);

/* Training: the forward pass that keeps what the backward needs, and the
 * backward pass.  The pages describe the forward only; the backward is the
 * derivative of that forward with the routing decisions (top-2 choice and
 * capacity mask) held fixed: the gradient reaches the router through the
 * softmax over the two selected logits ("Routing: top-2 without auxiliary
 * loss"), and the experts through "Expert implementation: SwiGLU at scale".
 * For L = sum(out * dout):
 *   dx [T, d] (cfg->dtype), dw_router [E, d], dbias [E] (or NULL),
 *   dw_gate, dw_up [E, d, f], dw_down [E, f, d]: fp32, overwritten.
 * bf16 only, d and f multiples of 256 (MOE_ERR_UNSUPPORTED otherwise).
 * ws: moe_workspace_size_train(cfg) bytes; moe_layer_forward_train fills it
 * (routing, grouped rows, H and the pre-activations G, U) and computes the
 * same out as moe_layer_forward; moe_layer_backward reads it (same cfg, x and
 * weights) and may be called again on it.  Every reduction has a fixed order:
 * results do not depend on scheduling. */
MOE_API size_t moe_workspace_size_train(const moe_config_t* cfg);
MOE_API moe_status_t moe_layer_forward_train(const moe_config_t* cfg, const void* x, const void* w_router,
                                     const float* logit_bias, const void* w_gate, const void* w_up,
                                     const void* w_down, void* out, void* ws, size_t ws_bytes,
                                     moe_stream_t stream);
MOE_API moe_status_t moe_layer_backward(const moe_config_t* cfg, const void* x, const void* w_router,
                                const void* w_gate, const void* w_up, const void* w_down, const void* dout,
                                void* dx, float* dw_router, float* dbias, float* dw_gate, float* dw_up,
                                float* dw_down, void* ws, size_t ws_bytes, moe_stream_t stream);

/* 8-bit expert weights ("Benchmarking xAI's Grok-1", section "Grok-1: In
 * Practice": the released weights were quantised; "Let Grok spill the beans
 * on Grok": 8-bit quantisation; the pages give no scheme).  Weight-only,
 * symmetric, one scale per output channel, every decision in IEEE fp32:
 *   scale[e, n] = max_k |w[e, k, n]| / 127
 *   q[e, k, n]  = clamp(rint(w[e, k, n] / scale[e, n]), -127, 127)  (0 if scale = 0)
 * w: bf16 [E, K, N] (cfg->dtype must be MOE_BF16); q: int8 [E, K, N];
 * scale: fp32 [E, N].  N must be a multiple of 64.  Gate and up are [E, d, f]
 * (channel = f), down is [E, f, d] (channel = d). */
MOE_API moe_status_t moe_quantize_int8(const moe_config_t* cfg, const void* w, int64_t K, int64_t N, int8_t* q,
                                       float* scale, moe_stream_t stream);

/* moe_expert_ffn with int8 expert weights, on the int8 tensor cores.
 * Every weight is q * scale (per output channel, from moe_quantize_int8);
 * every activation row entering a GEMM (rows of x_perm, then rows of H) is
 * held as a 15-bit code with a per-row scale (finer than bf16):
 *   s_r = max_k |v_k| / 32512,  c_k = clamp(rint(v_k / s_r), -32512, 32512)
 * split exactly as c = 256 * hi + lo into two int8 planes, so every MMA is an
 * exact int8 x int8 -> int32 product and the expert output is
 *   s_w[n] * s_r * (256 * acc_hi + acc_lo)   (fp32).
 * H is formed in fp32 and re-coded the same way before the down projection.
 * Built for the weight-streaming regime (few tokens per expert; the weights
 * are the MMA's M operand and tokens its N operand, 32 per tile).
 * ws: moe_expert_ffn_w8_workspace_size bytes, laid out (256-byte aligned) as
 * x codes hi [T*2, d] int8 | lo [T*2, d] int8 | scale [T*2] fp32 | H [T*2, f]
 * fp32 | H codes hi [T*2, f] | lo [T*2, f] | scale [T*2] | K-split partial
 * outputs [s, T*2, d] fp32 (s up to 8 when T*2 <= 64*E, else 1; summed in
 * split order into y);
 * y [T*2, d] fp32.  d must be a multiple of 256 (the down pass covers 256
 * output channels per tile). */
MOE_API size_t moe_expert_ffn_w8_workspace_size(const moe_config_t* cfg);
MOE_API moe_status_t moe_expert_ffn_w8(const moe_config_t* cfg, const void* x_perm, const int32_t* offsets,
                                       const int8_t* q_gate, const float* s_gate, const int8_t* q_up,
                                       const float* s_up, const int8_t* q_down, const float* s_down,
                                       const float* row_scale, float* y, void* ws, size_t ws_bytes,
                                       moe_stream_t stream);

/* Workspace of moe_layer_forward_w8: moe_workspace_size plus the scratch of
 * moe_expert_ffn_w8. */
MOE_API size_t moe_workspace_size_w8(const moe_config_t* cfg);

/* moe_layer_forward with int8 expert weights (router weight stays bf16). */
MOE_API moe_status_t moe_layer_forward_w8(const moe_config_t* cfg, const void* x, const void* w_router,
                                          const float* logit_bias, const int8_t* q_gate, const float* s_gate,
                                          const int8_t* q_up, const float* s_up, const int8_t* q_down,
                                          const float* s_down, void* out, int32_t* stats, void* ws,
                                          size_t ws_bytes, moe_stream_t stream);

/* Largest T accepted by moe_dispatch_noalloc. */
#define MOE_NOALLOC_MAX_TOKENS (1 << 20)

/* moe_dispatch without a caller-provided workspace and without allocating,
 * for callers that cannot allocate device memory: plug-ins hosted by a runtime
 * that owns all device memory and gives them no workspace, and latency-critical
 * loops that cannot afford cudaMalloc's implicit device-wide synchronisation.
 * The pages have no counterpart to this entry point (it concerns memory
 * management only); it computes exactly what moe_dispatch computes, with the
 * same arguments minus ws/ws_bytes.
 * Its scratch (per-block expert histograms) is a fixed device array inside
 * the library, 128 KiB held by every GPU that loads the library until the
 * process exits.  T > MOE_NOALLOC_MAX_TOKENS returns MOE_ERR_UNSUPPORTED.  All
 * calls share that array: calls that overlap on the GPU (e.g. on two streams)
 * race.  The array keeps the last call's contents; each call writes every
 * entry it reads, so nothing needs clearing.  The first call on a device looks
 * up the array's device address with that device current and caches it for
 * the current context; after cudaDeviceReset (a new context) the next call
 * looks it up again.  Make the first call on a device, and the first after a
 * reset, before any stream capture.  No cudaMalloc, cudaFree or allocating
 * routine is called. */
MOE_API moe_status_t moe_dispatch_noalloc(const moe_config_t* cfg, const void* x, const int32_t* topk_idx,
                                          const float* topk_w, int32_t* counts_raw, int32_t* counts_kept,
                                          int32_t* offsets, int32_t* perm, int32_t* slot_of,
                                          float* row_scale, void* x_perm, moe_stream_t stream);

/* Check of the bounded waits every pipelined kernel uses: one block waits on an
 * mbarrier that nothing completes, giving up after limit_ns nanoseconds
 * (1 us .. 1 s) and setting MOE_DEVERR_TIMEOUT in the device error word, as a
 * kernel whose pipeline stalled would.  The context stays usable; read the bit
 * with moe_get_device_error. */
MOE_API moe_status_t moe_check_bounded_wait(int64_t limit_ns, moe_stream_t stream);

/* Tile shape of the bf16 tensor-core grouped GEMMs (gate/up and down of the
 * expert FFN, prefill sizes), a process-wide setting:
 *   MOE_TILES_AUTO   the shape measured fastest on B200 (the default; single
 *                    CTAs for every shape timed so far);
 *   MOE_TILES_SINGLE one CTA per 128-row x N tile (M = 128 MMAs, M = 64 on an
 *                    expert's last block of at most 64 rows);
 *   MOE_TILES_PAIR   a cluster of two CTAs per 256-row tile (one 2-SM MMA of
 *                    M = 256 spanning both SMs; an expert's last block is
 *                    computed in full).
 * Both shapes compute every output element with the same K-ordered fp32
 * accumulation, so results do not depend on the mode.  Returns the previous
 * mode in *previous (may be NULL); MOE_ERR_INVALID_ARG for an unknown mode.
 * Calls already enqueued keep the shape they were launched with. */
#define MOE_TILES_AUTO 0
#define MOE_TILES_SINGLE 1
#define MOE_TILES_PAIR 2
MOE_API moe_status_t moe_set_gemm_tiles(int32_t mode, int32_t* previous);

/* Router utilisation over many calls ("How does Grok-1 use a
 * mixture-of-experts design?", section "Training dynamics: expert
 * specialization": assignments per expert normalised so that a balanced router
 * gives 1.0 for every expert).  Adds stats[0..E) (the counts_raw a layer call
 * wrote into its stats array) into the running int64 counts[E] and writes
 * utilization[e] = counts[e] * E / sum(counts) (all 0 while the sum is 0),
 * summed in expert order.  All three are device arrays owned by the caller;
 * counts must start at zero for a new statistic.  1 <= E <= 64, else
 * MOE_ERR_INVALID_ARG.  One small kernel on `stream`. */
MOE_API moe_status_t moe_expert_utilization(const int32_t* stats, int32_t E, int64_t* counts, float* utilization,
                                            moe_stream_t stream);

/* Phase timing of the training pair, for measurement; the pages have no
 * counterpart.  While enabled (moe_profile_phases(1), a process-wide setting),
 * moe_layer_forward_train and moe_layer_backward record a pair of CUDA events
 * on the call's stream around each of their kernels (events are created on
 * first use and reused; nothing is recorded while disabled, the default).
 * moe_profile_read waits for every recorded event, writes for each phase p < n
 * the summed milliseconds ms[p] and the number of calls calls[p] since the
 * previous read, and then forgets them.  ms and calls hold n entries (either
 * may be NULL); n may be smaller than MOE_PHASE_COUNT.  At most 65536 event
 * pairs are kept between reads; later ones are not recorded.  Returns
 * MOE_ERR_CUDA if an event cannot be created or read. */
#define MOE_PHASE_FWD_ROUTER 0   /* router logits + top-2 + softmax */
#define MOE_PHASE_FWD_DISPATCH 1 /* histogram, scan, stable rank */
#define MOE_PHASE_FWD_GATHER 2   /* x rows grouped by expert */
#define MOE_PHASE_FWD_GATE_UP 3  /* gate/up + SwiGLU, G and U kept */
#define MOE_PHASE_FWD_DOWN 4     /* down x routing weight */
#define MOE_PHASE_FWD_COMBINE 5  /* weighted sum back to token order */
#define MOE_PHASE_BWD_GATHER 6   /* dout by slot, routing-weighted copy */
#define MOE_PHASE_BWD_DH 7       /* dH with the SwiGLU derivative -> dG, dU */
#define MOE_PHASE_BWD_ZERO 8     /* fp32 dx accumulator cleared */
#define MOE_PHASE_BWD_DX 9       /* dx = dG W_gate^T + dU W_up^T by token */
#define MOE_PHASE_BWD_ROUTER 10  /* router backward, dx rounding */
#define MOE_PHASE_BWD_WG_DOWN 11 /* dW_down */
#define MOE_PHASE_BWD_WG_GATE 12 /* dW_gate */
#define MOE_PHASE_BWD_WG_UP 13   /* dW_up */
#define MOE_PHASE_COUNT 14
MOE_API moe_status_t moe_profile_phases(int32_t enable);
MOE_API moe_status_t moe_profile_read(float* ms, int32_t* calls, int32_t n);

/* Expert parallelism over peer memory ("Expert parallelism vs. tensor
 * parallelism", moe_layer_ep_forward: dispatch to the ranks owning the chosen
 * experts, expert FFN, combine back on the source rank), with the exchanges
 * written by the kernels themselves instead of two all-to-alls: the dispatch
 * kernel stores each kept row straight into the owner's grouped buffer, and
 * the owner's down projection adds routing_weight * (h @ W_down) straight into
 * the source rank's fp32 sums.  Rank q owns experts [q*E/W, (q+1)*E/W).
 *
 * moe_ep_peers_t lists every rank's exchange buffers as device addresses valid
 * in the calling process (its own allocations, or other ranks' allocations
 * mapped with moe_peer_import).  With R = world * T * top_k (every kept row of
 * every rank may go to one owner) and T the tokens of every rank:
 *   x_grp[q]  [R, d] cfg->dtype  rows rank q receives, its experts in order,
 *                                each expert's rows by source rank, then in
 *                                the source's kept order
 *   src[q]    [R] int32          source of each of those rows: p * T + t
 *   scale[q]  [R] fp32           routing weight of each of those rows
 *   sums[p]   [T, d] fp32        rank p's output sums, by token
 * One step, on every rank, in this order (the caller puts a barrier across
 * the ranks at each |, e.g. a one-element NCCL all-reduce on the stream):
 *   moe_router_topk, moe_dispatch (x_perm NULL), table = every rank's
 *   counts_kept, moe_ep_dispatch_peers | moe_ep_expert_ffn_peers |
 *   moe_ep_combine_peers.
 * The result on rank p equals moe_layer_forward on rank p's tokens bit for bit
 * in the fused down + combine scope (bf16, d a multiple of 256, top_k 2; every
 * row's products and its two-term fp32 sum do not depend on which rows share a
 * tile or on the order of the two adds).  world in {1, 2, 4, 8} (dividing E =
 * 8) and world * T <= 2^30, else MOE_ERR_UNSUPPORTED / MOE_ERR_INVALID_ARG;
 * x_grp and sums 16-byte aligned, src and scale 4-byte aligned, none NULL for
 * q < world (MOE_ERR_INVALID_ARG). */
#define MOE_EP_MAX_WORLD 8
typedef struct moe_ep_peers_t {
  int32_t world;
  int32_t rank;
  void* x_grp[MOE_EP_MAX_WORLD];
  int32_t* src[MOE_EP_MAX_WORLD];
  float* scale[MOE_EP_MAX_WORLD];
  float* sums[MOE_EP_MAX_WORLD];
} moe_ep_peers_t;

/* Zeroes sums[rank], then stores each of this rank's kept rows x[perm[r], :]
 * (with src and scale) into x_grp of the expert's owner, and writes this rank's
 * grouped offsets as an owner, grp_offsets [E + 1] (experts of other ranks
 * empty).  table [world, E] int32 (device): row p = counts_kept of rank p;
 * offsets, perm, row_scale: this rank's moe_dispatch outputs; x [T, d].  One
 * kernel.  A table inconsistent with offsets (this rank's row differs, a
 * negative count, more rows for an owner than its buffers hold) sets
 * MOE_DEVERR_OFFSETS, and the call then stores nothing (sums included) and
 * writes grp_offsets as all zeros.  An out-of-range perm entry sets
 * MOE_DEVERR_SLOT_INDEX and skips that row.  The stores (like the adds of
 * moe_ep_expert_ffn_peers) become visible to the other ranks when the kernel
 * completes, so the barrier must be ordered after the call on `stream` (a
 * collective, an event or a host wait), not run concurrently with it. */
MOE_API moe_status_t moe_ep_dispatch_peers(const moe_config_t* cfg, const moe_ep_peers_t* peers,
                                           const int32_t* table, const void* x, const int32_t* offsets,
                                           const int32_t* perm, const float* row_scale, int32_t* grp_offsets,
                                           moe_stream_t stream);

/* This rank's experts over the rows it received: h = silu(x_grp W_gate) *
 * (x_grp W_up) ([R, f] cfg->dtype, caller's scratch), then for each row
 * sums[p][t, :] += scale * (h W_down) with p * T + t = src of the row (vector
 * fp32 atomics into the source's buffer).  grp_offsets from
 * moe_ep_dispatch_peers; weights [E, d, f] / [E, f, d] (only this rank's
 * experts are read). */
MOE_API moe_status_t moe_ep_expert_ffn_peers(const moe_config_t* cfg, const moe_ep_peers_t* peers,
                                             const int32_t* grp_offsets, const void* w_gate, const void* w_up,
                                             const void* w_down, void* h, moe_stream_t stream);

/* out [T, d] (cfg->dtype) = sums[rank] rounded once. */
MOE_API moe_status_t moe_ep_combine_peers(const moe_config_t* cfg, const moe_ep_peers_t* peers, void* out,
                                          moe_stream_t stream);

/* Peer mappings for moe_ep_peers_t (CUDA IPC).  moe_peer_export describes the
 * device allocation holding `ptr` (any address inside a cudaMalloc block) so
 * that another process can map it: moe_peer_import maps it into the calling
 * process (peer access enabled on first use) and returns the address that
 * corresponds to `ptr`; moe_peer_release unmaps it (pass the imported address
 * and its handle).  A handle cannot be imported by the process that exported
 * it (use the address itself there).  MOE_ERR_CUDA when the runtime refuses
 * (e.g. memory not from cudaMalloc). */
typedef struct moe_peer_handle_t {
  uint8_t ipc[64];
  uint64_t offset;
} moe_peer_handle_t;
MOE_API moe_status_t moe_peer_export(const void* ptr, moe_peer_handle_t* handle);
MOE_API moe_status_t moe_peer_import(const moe_peer_handle_t* handle, void** ptr);
MOE_API moe_status_t moe_peer_release(void* ptr, const moe_peer_handle_t* handle);

/* Waits for the current device, returns the device error word (MOE_DEVERR_*
 * bits, 0 when clean) in *code, and clears it when `clear` is non-zero.
 * Returns MOE_ERR_DEVICE_CHECK when the word is non-zero, else MOE_OK. */
MOE_API moe_status_t moe_get_device_error(int32_t* code, int32_t clear);

#ifdef __cplusplus
}
#endif

#endif /* SPARSE_MOE_LAYER_07_B200_MOE_H */
