// Tensor-core (tcgen05) path of the bf16 expert: interface used by the runtime.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "../../include/rtv.h"

struct rtv_ctx;

namespace rtv {

struct ModTables;

// Decide whether the config can use the tensor-core path and allocate its
// state; sets ctx->use_fast.  Returns an error only on a CUDA failure.
rtv_status fast_create(rtv_ctx* ctx);
// Pack the loaded parameters into the tensor-core layouts.
rtv_status fast_load(rtv_ctx* ctx, const rtv_tensor* params, int n_params);
bool fast_supports_prefix(rtv_ctx* ctx, int prefix_len);
// Whether the tensor-core attention serves a prefix of P keys (else the warp-MMA one).
bool fast_tc_attention(const rtv_ctx* ctx, int P);
// Refresh the tensor-core layouts of the cached prefix after ctx->prefix_kv changed.
rtv_status fast_prefix_update(rtv_ctx* ctx, int batch, int prefix_len, cudaStream_t st);
// Step boundary over G suffixes: output head (Euler update of ctx->x, or the
// velocity into ctx->v when velocity_only) and/or the suffix embedding of the
// next evaluation into ctx->h with time condition rows c (stride c_stride).
// g0 (group stride g0_stride), when set, replaces the first layer's
// attention-norm gain in the embedding's norm input.
rtv_status fast_step(rtv_ctx* ctx, int G, bool do_head, bool do_embed, float dt, const float* c, int c_stride,
                     int state_stride, bool velocity_only, cudaStream_t st, const float* g0 = nullptr,
                     int g0_stride = 0);
// Layer 0 of a bare block whose suffix rows are weights, not inputs (the
// FLASH draft's learnable action queries): their q and suffix K/V tiles and
// residual rows depend on the weights and the RoPE positions only, so they
// are computed once (fast_block_fold) and read in place of a QKV projection.
struct FoldedQueries {
  __nv_bfloat16* qt = nullptr;    // [G][Hq/2][128][D] tiled q of the head pairs
  __nv_bfloat16* kts = nullptr;   // [G][Hkv][64][D] tiled suffix keys
  __nv_bfloat16* vts = nullptr;   // [G][Hkv][D][64] tiled suffix values (transposed)
  float* h0 = nullptr;            // [G*S][width] residual rows the O projection adds to
};
// The expert's layers over G suffixes (residual stream ctx->h); mod set for
// RTV_TIME_ADARMS; fold set: layer 0 reads its query rows' tiles and
// residual from fold and launches no QKV projection (tensor-core attention only).
rtv_status fast_layers(rtv_ctx* ctx, int G, int P, int prefix_batch_stride, const float* rope_cs,
                       const float* rope_sn, cudaStream_t st, const ModTables* mod = nullptr,
                       const FoldedQueries* fold = nullptr);
// Bytes of the four FoldedQueries buffers for G suffix groups.
void folded_sizes(const rtv_ctx* ctx, int G, size_t bytes[4]);
// Bare block: fill f for G suffixes whose residual rows are rows[t % n_src_rows]
// (RMSNorm, layer 0's QKV projection with RoPE from rope_cs / rope_sn), with a
// prefix of P keys.  Uses the context's scratch; enqueued on st.
rtv_status fast_block_fold(rtv_ctx* ctx, const float* rows, int n_src_rows, int G, int P, const float* rope_cs,
                           const float* rope_sn, const FoldedQueries& f, cudaStream_t st);
// The first layer's norm input of the residual rows of G suffixes, from ctx->h.
rtv_status fast_norm_rows(rtv_ctx* ctx, int G, cudaStream_t st);
// Bare block (ctx->block_only), layer 0: keys and values of n_vis tokens per
// batch element given as bf16 rows vis [batch][n_vis][width] (RMSNorm, K/V
// projection, RoPE at positions 0..n_vis-1), written into the cached prefix,
// whose tensor-core tiles are refreshed.  hb_vis (bf16, tiled over
// round_up(batch*n_vis, 16) rows) and ssp_vis ([batch*n_vis][width/128]) are
// scratch of the caller.
rtv_status fast_block_prefix(rtv_ctx* ctx, const __nv_bfloat16* vis, int n_vis, int batch, __nv_bfloat16* hb_vis,
                             float* ssp_vis, const float* rope_cs, const float* rope_sn, cudaStream_t st);
// Bare block: residual stream of G suffixes set to rows[t % n_src_rows]
// (fp32, [n_src_rows][width]) with the first norm's inputs.
rtv_status fast_block_embed(rtv_ctx* ctx, const float* rows, int n_src_rows, int G, cudaStream_t st);
// Prefill (pre: a bare block stack whose suffix is a group of 64 query rows):
// the stack over P tokens given as bf16 embeddings emb [P][width], writing
// every layer's keys (RoPE at positions 0..P-1) and values into the prefix
// cache of the expert ex (batch element 0) and its tensor-core tiles; the
// last layer computes keys and values only.  rope_cs / rope_sn: [P][D/2].
rtv_status fast_prefill(rtv_ctx* pre, rtv_ctx* ex, const __nv_bfloat16* emb, int P, const float* rope_cs,
                        const float* rope_sn, cudaStream_t st);
void fast_destroy(rtv_ctx* ctx);
// Read-only view of the tensor-core layouts another kernel family reuses
// (packed weights, transposed embeddings, prefix tiles); false without them.
struct FastViews {
  const __nv_bfloat16 *w_qkv, *w_o, *w_gu, *w_down, *w_aiT, *w_spT, *pkt, *pvt;
  int ntile_max, num_sms;
};
bool fast_views(const rtv_ctx* ctx, FastViews* out);
// Diagnostic phase trace (only when the RTV_TRACE environment variable is set).
void fast_arm_trace(rtv_ctx* ctx);
void fast_trace_report(rtv_ctx* ctx);

}  // namespace rtv
