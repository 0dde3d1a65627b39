/*
 * rtv.h -- C ABI of a B200 (sm_100a) implementation of the flow-matching
 * action-expert suffix loop of a Pi0/DM0.5-class VLA, and of FLASH parallel
 * verification.
 *
 * Pages (cited by title and section):
 *   [DM0.5] "DM0.5: high-performance embodied VLA and OpenDM reading guide"
 *           sec. 5.1 prefix encoded once into a per-layer KV cache,
 *           sec. 5.2 action expert (action_in_proj, time_mlp_in/out, prefix
 *           KV access, action_out_proj -> velocity), sec. 5.3 flow matching
 *           and Euler sampling (diffusion_steps = 10, action chunk),
 *           sec. 6.1 fixed image-count / static I/O contract, sec. 6.5
 *           startup graph capture with static addresses, one replay, step
 *           count fixed at capture.
 *   [FLASH] "Realtime-VLA FLASH" sec. 02 (interpolate, predict, rebuild the
 *           endpoint, compare), sec. 03.1 (draft model: one Gemma block and
 *           a linear action head over learnable action queries and the
 *           current image features, about 110M parameters), sec. 03.2
 *           (accept the prefix below delta at every verification time; zero
 *           length -> full path), sec. 03.3 (gripper switch -> full path).
 *
 * Conventions shared by every call:
 *   - Matrices are row-major [out][in].  Activations and actions are fp32.
 *   - Work is enqueued on the caller's stream and is asynchronous; outputs
 *     are valid once that stream has completed.  Calls on one context must
 *     not run concurrently from several host threads.
 *   - Errors detectable on the host return at once and enqueue nothing.
 *     Errors raised by kernels (a bounded wait that gave up, a non-finite
 *     result) set bits of a device status word, read by rtv_device_status.
 *   - No exception or abort crosses this boundary.  rtv_last_error gives a
 *     one-line description of the last failure on the context.
 *   - Pointers are owned by the caller unless stated.  The library copies
 *     what it keeps (weights, prefix KV) into memory it owns.
 */
#ifndef RTV_H
#define RTV_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

struct CUstream_st;
/* A CUDA stream (cudaStream_t).  NULL means the legacy default stream. */
typedef struct CUstream_st* rtv_stream;

typedef enum {
  RTV_OK = 0,
  RTV_ERR_ARG = 1,         /* null pointer, bad enum, bad name or size        */
  RTV_ERR_SHAPE = 2,       /* shape differs from the config or exceeds a max  */
  RTV_ERR_STATE = 3,       /* call order: e.g. denoise before load/prefix     */
  RTV_ERR_CUDA = 4,        /* a CUDA runtime call failed                      */
  RTV_ERR_OOM = 5,         /* device allocation failed                        */
  RTV_ERR_TIMEOUT = 6,     /* a device-side bounded wait gave up              */
  RTV_ERR_NUMERIC = 7,     /* non-finite value detected on the device        */
  RTV_ERR_UNSUPPORTED = 8  /* valid request the library does not implement   */
} rtv_status;

typedef enum { RTV_F32 = 0, RTV_BF16 = 1, RTV_FP8_E4M3 = 2, RTV_SAME = 3 } rtv_dtype;

typedef enum {
  RTV_MASK_BIDIR = 0,      /* every suffix token sees the prefix and its whole suffix */
  RTV_MASK_PI0_BLOCK = 1   /* the state token does not see the action tokens          */
} rtv_suffix_mask;

/* How the flow time t enters the expert ([DM0.5] 5.2 names time_mlp_in/out
 * and a per-layer time modulator; the forms are readings of the pages). */
typedef enum {
  RTV_TIME_ADD = 0,      /* c(t) = W_to swish(W_ti e(t) + b_ti) + b_to added to every action token     */
  RTV_TIME_CONCAT = 1,   /* Pi0: action token = W_to swish(W_ti [W_ai x + b_ai ; e(t)] + b_ti) + b_to  */
  RTV_TIME_ADARMS = 2    /* DM0.5: per layer, (scale, shift, gate) of each norm's branch from c(t)     */
} rtv_time_cond;

/* Device status bits (rtv_device_status). */
#define RTV_DEV_TIMEOUT  0x1u   /* a bounded spin-wait in a kernel gave up   */
#define RTV_DEV_NUMERIC  0x2u   /* a NaN/Inf reached the action output       */
#define RTV_DEV_BOUNDS   0x4u   /* a kernel's own index check refused work   */

/* Verification flags ([FLASH] 03.2-03.3). */
#define RTV_FLAG_ZERO_ACCEPT      0x1u  /* accepted length 0 -> full path               */
#define RTV_FLAG_SWITCH           0x2u  /* gripper sign switch in the candidate chunk  */
#define RTV_FLAG_SWITCH_IN_PREFIX 0x4u  /* a switch lies inside the accepted prefix    */

/*
 * Expert shape and settings.  [DM0.5] 5.2: a Gemma-style action expert of
 * n_layers layers, hidden width `width`, grouped-query attention with
 * n_q_heads query heads sharing n_kv_heads key/value heads of head_dim, a
 * gated (GeGLU) MLP of mlp_dim; a suffix of one state token (state_dim) and
 * chunk_len action tokens (action_dim) attends to a cached prefix of up to
 * max_prefix_len tokens per layer.
 *
 * dtype (RTV_F32 or RTV_BF16) is the storage and tensor-core input type of
 * the weight matrices and of the prefix KV; biases and norm gains are fp32.
 * mlp_dtype: RTV_SAME, or RTV_FP8_E4M3 for gate/up/down weights stored in
 * E4M3 with one fp32 scale per output row ([DM0.5] 6.3), with dtype
 * RTV_BF16 only (bf16 activations, fp32 accumulation; the E4M3 values are
 * widened to bf16 exactly).  A shape the tensor-core path does not take
 * returns RTV_ERR_UNSUPPORTED from rtv_create for an FP8 MLP.
 * rope_theta 0 disables rotary embedding.  barrier_timeout_ns bounds every
 * device-side wait (0 = library default, 100 ms).  time_cond selects how the
 * flow time conditions the expert (rtv_time_cond); with RTV_TIME_ADARMS,
 * layer l's norms become x / rms(x) * (1 + scale) + shift for every suffix
 * token and its two branches are multiplied by their gates, where
 * (scale_a, shift_a, gate_a, scale_m, shift_m, gate_m) =
 * layers.l.time_mod.w . c(t) + layers.l.time_mod.b, in that order.
 */
typedef struct {
  int n_layers, width, n_q_heads, n_kv_heads, head_dim, mlp_dim;
  int action_dim, state_dim, chunk_len;
  int max_prefix_len, max_batch, max_taus;
  int dtype;
  int mlp_dtype;
  int suffix_mask;
  float rms_eps;
  float rope_theta;
  long long barrier_timeout_ns;
  int time_cond;       /* rtv_time_cond (RTV_TIME_ADD = 0 by default)                       */
} rtv_expert_config;

/*
 * One named parameter for rtv_load_expert.  `data` points to host memory
 * (is_device = 0) or device memory (is_device = 1) holding a dense
 * row-major array of `shape` in `dtype`.  Names and shapes (w = width,
 * A = action_dim, Sd = state_dim, F = mlp_dim, Q = n_q_heads*head_dim,
 * KV = n_kv_heads*head_dim, l = layer index):
 *   state_proj.w [w][Sd]  state_proj.b [w]
 *   action_in_proj.w [w][A]  action_in_proj.b [w]
 *   time_mlp_in.w [w][w]  time_mlp_in.b [w]  time_mlp_out.w [w][w]  time_mlp_out.b [w]
 *   layers.l.attn_norm.g [w]  layers.l.q_proj.w [Q][w]  layers.l.k_proj.w [KV][w]
 *   layers.l.v_proj.w [KV][w] layers.l.o_proj.w [w][Q]  layers.l.mlp_norm.g [w]
 *   layers.l.gate_proj.w [F][w]  layers.l.up_proj.w [F][w]  layers.l.down_proj.w [w][F]
 *   layers.l.gate_proj.s [F]  layers.l.up_proj.s [F]  layers.l.down_proj.s [w]
 *        (fp32 per-row scales, only with mlp_dtype = RTV_FP8_E4M3)
 *   final_norm.g [w]  action_out_proj.w [A][w]  action_out_proj.b [A]
 * With time_cond RTV_TIME_CONCAT, time_mlp_in.w is [w][2w] (its first w
 * columns read the action embedding, the last w the sinusoid e(t)).  With
 * RTV_TIME_ADARMS, every layer has layers.l.time_mod.w [6w][w] and
 * layers.l.time_mod.b [6w] instead of layers.l.attn_norm.g and mlp_norm.g.
 * Matrices must be given in the config dtype (or RTV_FP8_E4M3 for the MLP
 * when mlp_dtype says so); vectors in RTV_F32.
 */
typedef struct {
  const char* name;
  const void* data;
  int dtype;
  int ndim;
  long long shape[4];
  int is_device;
} rtv_tensor;

typedef struct rtv_ctx rtv_ctx;

/* Create a context on CUDA device `cuda_device`; allocates the static
 * buffers for the config's maxima.  *out is NULL on failure. */
rtv_status rtv_create(const rtv_expert_config* cfg, int cuda_device, rtv_ctx** out);

/* Copy and pack the expert's parameters ([DM0.5] 5.2).  Every name listed
 * above must appear exactly once.  Synchronous; the caller keeps ownership
 * of the inputs and may free them on return. */
rtv_status rtv_load_expert(rtv_ctx* ctx, const rtv_tensor* params, int n_params);

/* Install the prefix KV cache ([DM0.5] 5.1): `kv` is a device or host array
 * [n_layers][2][batch][prefix_len][n_kv_heads][head_dim] in the config dtype
 * (index 0 = keys, already rotated; 1 = values).  It is copied on `stream`
 * into library-owned memory of fixed address (the static-address contract
 * of [DM0.5] 6.5).  prefix_len <= max_prefix_len, batch <= max_batch. */
rtv_status rtv_set_prefix_kv(rtv_ctx* ctx, const void* kv, int prefix_len, int batch, rtv_stream stream);

/* Install the prefix KV cache without allocating any device memory.  No
 * counterpart in the pages: this is a service for callers that cannot call
 * cudaMalloc while running (a real-time control loop that must not block on
 * the allocator, or a process whose device memory belongs to another
 * allocator or a fixed budget).  Same arguments and result as
 * rtv_set_prefix_kv; a host-resident `kv` is staged one layer at a time
 * through a fixed 4 MiB array in device global memory that the library
 * declares statically (every GPU that loads the library holds it until the
 * process exits).  Returns RTV_ERR_SHAPE when one layer's keys and values
 * (2 * batch * prefix_len * n_kv_heads * head_dim elements) exceed 4 MiB,
 * and RTV_ERR_ARG for device memory of another GPU (device memory of the
 * context's GPU is read in place; host and managed memory are staged).
 * The first call on a device looks up the array's device address, which may
 * make the driver load the library's module and reserve the array then
 * (lazy module loading): make that first call at set-up time, before any
 * stream capture.  All calls share the array and it keeps the last call's
 * contents: calls whose work overlaps on the GPU (other streams or other
 * contexts on the same device) race on it, so serialise them.  While the
 * copy runs the context holds no prefix: if the call fails part-way,
 * denoise and verify return RTV_ERR_STATE until a prefix is installed.
 * Calls no cudaMalloc, cudaFree or allocating library routine. */
rtv_status rtv_set_prefix_kv_static(rtv_ctx* ctx, const void* kv, int prefix_len, int batch, rtv_stream stream);

/* Denoise ([DM0.5] 5.3): from noise x_1 = noise [batch][H][A], run n_steps
 * Euler steps x <- x - (1/n_steps) * v(x, t_k), t_k = 1 - k/n_steps, and
 * write the action chunk [batch][H][A] to actions_out.  state is
 * [batch][Sd].  batch is the one given to rtv_set_prefix_kv.  Each pointer
 * may be device or host memory (host copies are enqueued on `stream`).
 * The first call for a given (n_steps, batch, prefix_len) captures a CUDA
 * graph (not on `stream`); later calls replay it. */
rtv_status rtv_denoise(rtv_ctx* ctx, const float* noise, const float* state, int n_steps,
                       float* actions_out, rtv_stream stream);

/* FLASH verification ([FLASH] 02, 03.2, 03.3) of one draft chunk against
 * the prefix of batch element 0: for each tau_i (host array of n_taus
 * values in [0,1]) form X_i = tau_i*noise + (1-tau_i)*draft, evaluate the
 * expert once on all X_i together (each sees the prefix and its own
 * suffix), rebuild A_i = X_i - tau_i*v_i, take d_i[h] = ||A_i[h] - draft[h]||_2
 * and accept the longest prefix with d_i[h] < delta for every i.
 * draft, noise [H][A], state [Sd]: device or host.  Outputs (device or
 * host): *accepted_len (int32), *flags (RTV_FLAG_*), dist [n_taus][H] fp32
 * or NULL.  gripper_dim in [0, A) selects the gripper action dimension. */
rtv_status rtv_verify(rtv_ctx* ctx, const float* draft, const float* noise, const float* state,
                      const float* taus, int n_taus, float delta, int gripper_dim,
                      int* accepted_len, unsigned* flags, float* dist, rtv_stream stream);

/* Synchronise the context's device work and report the device status word
 * (RTV_DEV_* bits); the word is cleared after it is read.  Returns
 * RTV_ERR_TIMEOUT / RTV_ERR_NUMERIC when the matching bit was set. */
rtv_status rtv_device_status(rtv_ctx* ctx, unsigned* bits);

/* Last error message of the context (never NULL; "" when none). */
const char* rtv_last_error(rtv_ctx* ctx);

/* Human-readable name of the kernel path a context uses ("tcgen05", "simt"). */
const char* rtv_path_name(rtv_ctx* ctx);

/* Number of kernel launches one call makes: of the graph captured for
 * rtv_denoise(n_steps = n, current prefix batch) when is_verify = 0, or of
 * rtv_verify(n_taus = n) when is_verify = 1.  -1 if that graph has not been
 * captured yet.  Diagnostic; enqueues nothing. */
int rtv_graph_kernel_count(rtv_ctx* ctx, int n, int is_verify);

/* Release every resource of the context.  NULL is accepted. */
void rtv_destroy(rtv_ctx* ctx);


/* ------------------------------------------------------------------------
 * FLASH draft model ([FLASH] 03.1) and dual-path round ([FLASH] 03).
 *
 * The draft model is one Gemma block and a linear action head.  The image
 * features of one observation (n_vis tokens of `width`) are followed by
 * n_queries learnable action queries; the block (RMSNorm with gain 1+g,
 * q/k/v projections, RoPE at positions 0..n_vis+n_queries-1, softmax
 * attention in which every row sees every row, o_proj + residual, RMSNorm,
 * GeGLU MLP + residual) runs once, and the head maps each query row to one
 * action: chunk[h] = action_head.w . x[n_vis + h] + action_head.b.
 * ------------------------------------------------------------------------ */
typedef struct {
  int width, n_q_heads, n_kv_heads, head_dim, mlp_dim;
  int n_queries;      /* H: action queries = rows of the candidate chunk (1..64)  */
  int action_dim;     /* A                                                        */
  int max_vis;        /* largest n_vis a call may pass                            */
  int max_batch;      /* largest batch a call may pass                            */
  int dtype;          /* RTV_F32 | RTV_BF16: weight matrices and image features   */
  float rms_eps;
  float rope_theta;   /* 0 disables rotary embedding                              */
  long long barrier_timeout_ns;   /* 0 = library default (100 ms)                 */
} rtv_draft_config;

typedef struct rtv_draft rtv_draft;

/* Create a draft model on CUDA device `cuda_device`; allocates its static
 * buffers for the maxima.  width must be a multiple of 128.  *out is NULL on
 * failure.  Returns RTV_ERR_ARG on a bad config, RTV_ERR_CUDA on a bad
 * device, RTV_ERR_OOM when the buffers do not fit. */
rtv_status rtv_draft_create(const rtv_draft_config* cfg, int cuda_device, rtv_draft** out);

/* Copy and pack the draft parameters (rtv_tensor as for rtv_load_expert;
 * w = width, F = mlp_dim, Q = n_q_heads*head_dim, KV = n_kv_heads*head_dim,
 * H = n_queries, A = action_dim):
 *   action_queries [H][w] (RTV_F32)
 *   attn_norm.g [w]  q_proj.w [Q][w]  k_proj.w [KV][w]  v_proj.w [KV][w]
 *   o_proj.w [w][Q]  mlp_norm.g [w]  gate_proj.w [F][w]  up_proj.w [F][w]
 *   down_proj.w [w][F]  action_head.w [A][w]  action_head.b [A]
 * Matrices in the config dtype, vectors in RTV_F32; every name exactly once.
 * Synchronous.  A missing, duplicate or unknown name, or a wrong dtype
 * returns RTV_ERR_ARG and a wrong shape RTV_ERR_SHAPE, before anything is
 * allocated; a second load returns RTV_ERR_STATE. */
rtv_status rtv_draft_load(rtv_draft* d, const rtv_tensor* params, int n_params);

/* Candidate chunks chunk_out [batch][H][A] (fp32) from the image features
 * vis [batch][n_vis][width] (config dtype), each batch element on its own.
 * vis and chunk_out may be device or host memory (host copies are enqueued
 * on `stream`).  n_vis <= max_vis, batch <= max_batch.  Asynchronous; the
 * first call for a given (n_vis, batch) captures a CUDA graph (not on
 * `stream`), later calls replay it.  Before rtv_draft_load: RTV_ERR_STATE;
 * null pointers: RTV_ERR_ARG; sizes out of range: RTV_ERR_SHAPE; nothing is
 * enqueued on an error.  Device-side errors go to the status word
 * (rtv_draft_device_status). */
rtv_status rtv_draft_forward(rtv_draft* d, const void* vis, int n_vis, int batch, float* chunk_out,
                             rtv_stream stream);

/* One FLASH round for one observation ([FLASH] 03): draft the chunk from
 * vis [n_vis][width], verify it with the expert `ctx` (as rtv_verify, with
 * noise [H][A], state [Sd], taus, delta, gripper_dim), and when the verdict
 * is a fallback (accepted length 0 or a gripper switch) run the full path,
 * rtv_denoise(ctx, noise, state, n_steps), from the same noise.  Writes the
 * chunk [H][A] to actions_out (the draft, or the denoised chunk), and to
 * host memory *accepted_len, *flags (RTV_FLAG_*) and *used_full (1 = the
 * full path ran).  The expert's prefix KV must be installed with batch 1;
 * its chunk_len and action_dim must equal the draft's n_queries and
 * action_dim.  Synchronous: returns once actions_out holds the chunk.
 * Errors: null pointers or a draft on another device RTV_ERR_ARG, shape
 * mismatches or a prefix of batch > 1 RTV_ERR_SHAPE, and whatever
 * rtv_draft_forward, rtv_verify or rtv_denoise return (their message is
 * copied to rtv_draft_last_error). */
rtv_status rtv_flash_round(rtv_ctx* ctx, rtv_draft* d, const void* vis, int n_vis, const float* noise,
                           const float* state, const float* taus, int n_taus, float delta, int gripper_dim,
                           int n_steps, float* actions_out, int* accepted_len, unsigned* flags, int* used_full,
                           rtv_stream stream);

/* As rtv_device_status, for the draft model's kernels. */
rtv_status rtv_draft_device_status(rtv_draft* d, unsigned* bits);

/* Last error message of the draft model (never NULL). */
const char* rtv_draft_last_error(rtv_draft* d);

/* Kernel path of the draft model ("tcgen05", "simt"). */
const char* rtv_draft_path_name(rtv_draft* d);

/* Kernel launches of one rtv_draft_forward(n_vis, batch); -1 before its
 * graph has been captured. */
int rtv_draft_kernel_count(rtv_draft* d, int n_vis, int batch);

/* Release every resource of the draft model.  NULL is accepted. */
void rtv_draft_destroy(rtv_draft* d);

/* ------------------------------------------------------------------------
 * VLM prefill ([DM0.5] 5.1: the prefix is encoded once into a per-layer KV
 * cache; 6.5: one graph replay per request).
 *
 * A Gemma-style stack over the prefix embeddings of one observation (n_tokens
 * rows of `width`): RMSNorm with gain 1+g, q/k/v projections, RoPE at
 * positions 0..n_tokens-1, softmax attention in which every prefix token
 * sees every prefix token, o_proj + residual, RMSNorm, GeGLU MLP + residual.
 * Layer l's keys (after RoPE) and values become the expert's cached prefix
 * of layer l, so the stack has the expert's n_layers, n_kv_heads and
 * head_dim.  The last layer's attention output and MLP are not computed.
 * bf16 only (tensor-core path).
 * ------------------------------------------------------------------------ */
typedef struct {
  int n_layers, width, n_q_heads, n_kv_heads, head_dim, mlp_dim;
  int max_tokens;     /* largest n_tokens a call may pass (<= 960)                */
  int dtype;          /* RTV_BF16                                                 */
  float rms_eps;
  float rope_theta;   /* 0 disables rotary embedding                              */
  long long barrier_timeout_ns;   /* 0 = library default (100 ms)                 */
} rtv_prefill_config;

typedef struct rtv_prefill rtv_prefill;

/* Create a prefill stack on CUDA device `cuda_device`.  width must be a
 * multiple of 128.  Returns RTV_ERR_UNSUPPORTED for RTV_F32 or a shape the
 * tensor-core path does not take.  *out is NULL on failure. */
rtv_status rtv_prefill_create(const rtv_prefill_config* cfg, int cuda_device, rtv_prefill** out);

/* Copy and pack the stack's parameters: for every layer l the names of
 * rtv_load_expert's layers (layers.l.attn_norm.g, layers.l.q_proj.w, ...,
 * layers.l.down_proj.w), matrices in bf16, gains in RTV_F32.  Synchronous.
 * Name, dtype and shape errors as for rtv_draft_load. */
rtv_status rtv_prefill_load(rtv_prefill* p, const rtv_tensor* params, int n_params);

/* Run the stack over emb [n_tokens][width] (bf16, device or host) and
 * install the result as the prefix KV cache of the expert `ctx` (batch 1,
 * prefix_len = n_tokens), as rtv_set_prefix_kv would.  The expert must be a
 * bf16 tensor-core context with the stack's n_layers, n_kv_heads and
 * head_dim, and n_tokens <= its max_prefix_len.  Asynchronous on `stream`;
 * the first call for a given n_tokens captures a CUDA graph.  Before both
 * loads: RTV_ERR_STATE; a mismatched expert or n_tokens out of range:
 * RTV_ERR_SHAPE; an expert off the tensor-core path: RTV_ERR_UNSUPPORTED;
 * nothing is enqueued on an error. */
rtv_status rtv_prefill_kv(rtv_prefill* p, rtv_ctx* ctx, const void* emb, int n_tokens, rtv_stream stream);

/* Prefill followed by rtv_denoise(ctx, noise, state, n_steps) for one
 * observation (batch 1), captured as ONE CUDA graph per (n_tokens, n_steps)
 * and replayed: emb [n_tokens][width] bf16, noise [H][A], state [Sd],
 * actions_out [H][A]; each device or host memory.  Leaves the prefix
 * installed in ctx.  Asynchronous on `stream`. */
rtv_status rtv_prefill_denoise(rtv_prefill* p, rtv_ctx* ctx, const void* emb, int n_tokens, const float* noise,
                               const float* state, int n_steps, float* actions_out, rtv_stream stream);

/* As rtv_device_status, for the stack's kernels. */
rtv_status rtv_prefill_device_status(rtv_prefill* p, unsigned* bits);

/* Last error message of the prefill stack (never NULL). */
const char* rtv_prefill_last_error(rtv_prefill* p);

/* Kernel launches of the graph captured for (n_tokens, n_steps); n_steps 0
 * is rtv_prefill_kv's graph.  -1 before it has been captured. */
int rtv_prefill_kernel_count(rtv_prefill* p, int n_tokens, int n_steps);

/* Release every resource of the prefill stack.  NULL is accepted.  The
 * stack keeps the graphs it captured for an expert context (they address
 * that context's buffers): destroy the stack before, or together with, every
 * expert it has served, and do not pass it a context created after one of
 * those was destroyed. */
void rtv_prefill_destroy(rtv_prefill* p);

#ifdef __cplusplus
}
#endif

#endif /* RTV_H */
