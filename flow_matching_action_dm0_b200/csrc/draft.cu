// FLASH draft model and dual-path round ("Realtime-VLA FLASH", sec. 03).
//
// Sec. 03.1: the draft model is one Gemma block and a linear action head
// (about 110M parameters).  On the fast path the VLM prefill is skipped: the
// current image features and a set of learnable action queries form one
// sequence, the block runs once, and the head turns the query rows into the
// whole candidate chunk.  Sec. 03.2-03.3: the chunk is verified by the
// action expert at several flow times; a zero accepted length or a gripper
// switch sends the round to the full path (the expert's Euler denoising).
//
// The block runs as a bare one-layer context of the expert's runtime (same
// kernels, same tensor-core path): the image features play the part of the
// cached prefix -- their keys and values are computed on the device, RoPE'd
// at positions 0..V-1 and written into the context's prefix cache -- and
// the H action queries are its suffix, at positions V..V+H-1, each seeing
// every visual token and every query.  The visual rows' own outputs feed
// nothing, so only their keys and values are computed.  Every draft call
// replays one CUDA graph per (visual tokens, batch).
#include <stdio.h>
#include <stdlib.h>
#include <string.h>

#include <map>
#include <string>
#include <utility>
#include <vector>

#include "common.cuh"
#include "fastpath.h"
#include "kernels.h"
#include "runtime.h"

using namespace rtv;

struct rtv_draft {
  rtv_draft_config cfg{};
  int device = 0;
  rtv_ctx* blk = nullptr;   // the block: one layer, suffix = the H action queries
  std::string last_error;
  bool loaded = false;
  int elt = 4;
  float* queries = nullptr;   // [H][w] (allocations of the block context)
  void* head_w = nullptr;     // [A][w], config dtype
  float* head_b = nullptr;    // [A]
  void* vis_in = nullptr;     // [Bmax][Vmax][w], config dtype: the graphs' fixed input address
  float* vis_f = nullptr;     // SIMT: [Bmax*Vmax][w] fp32 copy of bf16 features
  float* vis_u = nullptr;     // SIMT: normalised features
  float* vis_kv = nullptr;    // SIMT: [Bmax*Vmax][2*KV] projected keys and values
  __nv_bfloat16* vis_hb = nullptr;   // tensor cores: tiled norm input
  float* vis_ssp = nullptr;          // tensor cores: sums of squares per 128-feature tile
  float* out = nullptr;       // [Bmax][H][A]
  std::map<std::pair<int, int>, GraphEntry> graphs;   // (n_vis, batch)
  std::vector<void*> allocs;
};

namespace {

rtv_status dfail(rtv_draft* d, rtv_status s, const std::string& msg) {
  if (d) d->last_error = msg;
  return s;
}

#define DCK(call)                                                                                  \
  do {                                                                                             \
    cudaError_t _e = (call);                                                                       \
    if (_e != cudaSuccess)                                                                         \
      return dfail(d, _e == cudaErrorMemoryAllocation ? RTV_ERR_OOM : RTV_ERR_CUDA,                \
                   std::string(#call) + ": " + cudaGetErrorString(_e));                            \
  } while (0)

#define DTRY(x)                        \
  do {                                 \
    rtv_status _s = (x);               \
    if (_s != RTV_OK) return _s;       \
  } while (0)

rtv_status dalloc(rtv_draft* d, void** p, size_t bytes, bool zero = false) {
  *p = nullptr;
  if (bytes == 0) bytes = 16;
  DCK(cudaMalloc(p, bytes));
  d->allocs.push_back(*p);
  if (zero) DCK(cudaMemset(*p, 0, bytes));
  return RTV_OK;
}

// ---------------------------------------------------------------------------
// kernels
// ---------------------------------------------------------------------------

// Action head ([FLASH] 03.1): out[t][a] = W[a] . h[t] + b[a] for every
// query row t.  CTA (t, j) takes outputs 8j..8j+7 of row t, one per warp; a
// lane reads 8 consecutive features per step (16-byte weight loads for bf16).
__device__ __forceinline__ void load8(const float* p, float v[8]) {
  const float4 a = *reinterpret_cast<const float4*>(p);
  const float4 b = *reinterpret_cast<const float4*>(p + 4);
  v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
  v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
}
__device__ __forceinline__ void load8(const __nv_bfloat16* p, float v[8]) {
  const uint4 q = *reinterpret_cast<const uint4*>(p);
  const __nv_bfloat162* h2 = reinterpret_cast<const __nv_bfloat162*>(&q);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float2 f = __bfloat1622float2(h2[i]);
    v[2 * i] = f.x;
    v[2 * i + 1] = f.y;
  }
}

template <typename WT>
__global__ void __launch_bounds__(256) draft_head_kernel(const float* __restrict__ h, const WT* __restrict__ W,
                                                         const float* __restrict__ b, float* __restrict__ out,
                                                         int w, int A) {
  const int t = blockIdx.x;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const float* hr = h + (size_t)t * w;
  const int a = (int)blockIdx.y * 8 + warp;
  if (a < A) {
    const WT* wr = W + (size_t)a * w;
    float acc = 0.f;
    for (int k = lane * 8; k < w; k += 256) {   // w is a multiple of 128
      float x[8], y[8];
      load8(hr + k, x);
      load8(wr + k, y);
#pragma unroll
      for (int i = 0; i < 8; ++i) acc = fmaf(x[i], y[i], acc);
    }
    acc = warp_sum(acc);
    if (lane == 0) out[(size_t)t * A + a] = acc + b[a];
  }
}

// Residual rows of G suffixes from the queries: h[t] = q[t % H] (SIMT path).
__global__ void broadcast_rows_kernel(const float* __restrict__ q, float* __restrict__ h, int H, int w, int T) {
  const size_t n = (size_t)T * w;
  for (size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += (size_t)gridDim.x * blockDim.x) {
    const size_t t = i / w, k = i % w;
    h[i] = q[(t % H) * w + k];
  }
}

__global__ void bf16_to_f32_kernel(const __nv_bfloat16* __restrict__ x, float* __restrict__ y, size_t n) {
  for (size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += (size_t)gridDim.x * blockDim.x)
    y[i] = __bfloat162float(x[i]);
}

// Projected keys/values of the visual rows kv [B*V][2*KV] -> the cached
// prefix of layer 0 [2][Bmax][Hkv][Pmax][D] (config dtype), keys rotated at
// positions 0..V-1 with the table cs/sn [V][D/2] (pairs d, d + D/2).
template <typename KT>
__global__ void vis_kv_store_kernel(const float* __restrict__ kv, const float* __restrict__ cs,
                                    const float* __restrict__ sn, KT* __restrict__ pk, KT* __restrict__ pv, int V,
                                    int Hkv, int D, int Pmax) {
  const int r = blockIdx.x;
  const int b = r / V, s = r % V;
  const int half = D / 2, KV = Hkv * D;
  const float* src = kv + (size_t)r * 2 * KV;
  for (int idx = threadIdx.x; idx < Hkv * half; idx += blockDim.x) {
    const int kh = idx / half, dd = idx % half;
    const float c = cs[(size_t)s * half + dd], si = sn[(size_t)s * half + dd];
    const float x1 = src[kh * D + dd], x2 = src[kh * D + dd + half];
    const size_t o = (((size_t)b * Hkv + kh) * Pmax + s) * D;
    pk[o + dd] = (KT)(x1 * c - x2 * si);
    pk[o + dd + half] = (KT)(x2 * c + x1 * si);
    pv[o + dd] = (KT)src[KV + kh * D + dd];
    pv[o + dd + half] = (KT)src[KV + kh * D + dd + half];
  }
}

// The draft forward for (V, B), enqueued on st (captured into a graph).
// fold: the query rows' layer-0 tiles and residual, computed at graph build.
template <typename WT>
rtv_status enqueue_forward(rtv_draft* d, int V, int B, const float* cs_v, const float* sn_v, const float* cs_q,
                           const float* sn_q, const FoldedQueries* fold, cudaStream_t st) {
  rtv_ctx* c = d->blk;
  const rtv_expert_config& k = c->cfg;
  const int w = k.width, H = d->cfg.n_queries, A = d->cfg.action_dim;
  const int Q = c->Q, KV = c->KV, D = k.head_dim;
  const int Tv = B * V, Tq = B * H;
  if (c->use_fast) {
    DTRY(fast_block_prefix(c, (const __nv_bfloat16*)d->vis_in, V, B, d->vis_hb, d->vis_ssp, cs_v, sn_v, st));
    if (fold) {
      DTRY(fast_layers(c, B, V, 1, cs_q, sn_q, st, nullptr, fold));
    } else {
      DTRY(fast_block_embed(c, d->queries, H, B, st));
      DTRY(fast_layers(c, B, V, 1, cs_q, sn_q, st));
    }
  } else {
    const LayerW& L = c->W.layers[0];
    const float* xf = (const float*)d->vis_in;
    if (sizeof(WT) == 2) {
      bf16_to_f32_kernel<<<256, 256, 0, st>>>((const __nv_bfloat16*)d->vis_in, d->vis_f, (size_t)Tv * w);
      xf = d->vis_f;
    }
    launch_rmsnorm(xf, L.g_attn, d->vis_u, Tv, w, k.rms_eps, st);
    launch_linear<WT>(d->vis_u, w, (const WT*)L.qkv + (size_t)Q * w, nullptr, d->vis_kv, 2 * KV, Tv, 2 * KV, w,
                      EPI_STORE, st);
    const size_t kv_layer = (size_t)k.max_batch * k.n_kv_heads * k.max_prefix_len * D;
    vis_kv_store_kernel<WT><<<Tv, 128, 0, st>>>(d->vis_kv, cs_v, sn_v, (WT*)c->prefix_kv,
                                                (WT*)c->prefix_kv + kv_layer, V, k.n_kv_heads, D,
                                                k.max_prefix_len);
    broadcast_rows_kernel<<<256, 256, 0, st>>>(d->queries, c->h, H, w, Tq);
    simt_layers<WT>(c, B, V, 1, cs_q, sn_q, st);
  }
  draft_head_kernel<WT><<<dim3(Tq, (A + 7) / 8), 256, 0, st>>>(c->h, (const WT*)d->head_w, d->head_b, d->out, w,
                                                                A);
  const cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return dfail(d, RTV_ERR_CUDA, std::string("draft launch: ") + cudaGetErrorString(e));
  return RTV_OK;
}

rtv_status build_graph(rtv_draft* d, int V, int B, GraphEntry& ge) {
  rtv_ctx* c = d->blk;
  const rtv_expert_config& k = c->cfg;
  const int D = k.head_dim, H = d->cfg.n_queries;
  cudaStream_t st = c->cap_stream;
  float* tabs[4] = {nullptr, nullptr, nullptr, nullptr};
  const size_t rows[4] = {(size_t)V, (size_t)V, (size_t)H, (size_t)H};
  for (int i = 0; i < 4; ++i) {
    DCK(cudaMalloc(&tabs[i], sizeof(float) * rows[i] * (D / 2)));
    ge.owned.push_back(tabs[i]);
  }
  // RoPE of the sequence [visual tokens ; queries]: positions 0..V-1, V..V+H-1
  launch_rope_table(tabs[0], tabs[1], V, D, 0, k.rope_theta, st);
  launch_rope_table(tabs[2], tabs[3], H, D, V, k.rope_theta, st);
  DCK(cudaGetLastError());
  // The action queries are weights: the first norm of their rows, their q, k
  // and v (RoPE at V..V+H-1) and the residual the O projection adds to depend
  // on the weights and V only, so they are computed here, once per graph, and
  // the forward starts the query rows at the attention.
  FoldedQueries fold;
  const bool folding = c->use_fast && fast_tc_attention(c, V);
  if (folding) {
    size_t bytes[4];
    folded_sizes(c, B, bytes);
    void* p[4] = {nullptr, nullptr, nullptr, nullptr};
    for (int i = 0; i < 4; ++i) {
      DCK(cudaMalloc(&p[i], bytes[i]));
      ge.owned.push_back(p[i]);
    }
    fold.qt = (__nv_bfloat16*)p[0];
    fold.kts = (__nv_bfloat16*)p[1];
    fold.vts = (__nv_bfloat16*)p[2];
    fold.h0 = (float*)p[3];
    const rtv_status s = fast_block_fold(c, d->queries, H, B, V, tabs[2], tabs[3], fold, st);
    if (s != RTV_OK) return dfail(d, s, c->last_error);
  }
  DCK(cudaStreamSynchronize(st));
  c->last_error.clear();
  DCK(cudaStreamBeginCapture(st, cudaStreamCaptureModeThreadLocal));
  const FoldedQueries* fp = folding ? &fold : nullptr;
  const rtv_status fs = k.dtype == RTV_F32
                            ? enqueue_forward<float>(d, V, B, tabs[0], tabs[1], tabs[2], tabs[3], fp, st)
                            : enqueue_forward<__nv_bfloat16>(d, V, B, tabs[0], tabs[1], tabs[2], tabs[3], fp, st);
  cudaGraph_t g = nullptr;
  const cudaError_t e1 = cudaGetLastError();
  const cudaError_t e2 = cudaStreamEndCapture(st, &g);
  if (fs != RTV_OK || e1 != cudaSuccess || e2 != cudaSuccess) {
    if (g) cudaGraphDestroy(g);
    if (fs != RTV_OK) {
      if (!c->last_error.empty()) d->last_error = c->last_error;
      return fs;
    }
    return dfail(d, RTV_ERR_CUDA, std::string("draft graph capture: ") +
                                      cudaGetErrorString(e1 != cudaSuccess ? e1 : e2));
  }
  ge.graph = g;
  ge.kernels = count_kernel_nodes(g);
  DCK(cudaGraphInstantiate(&ge.exec, g, 0));
  DCK(cudaGraphUpload(ge.exec, st));
  DCK(cudaStreamSynchronize(st));
  return RTV_OK;
}

rtv_status get_graph(rtv_draft* d, int V, int B, GraphEntry** out) {
  const auto key = std::make_pair(V, B);
  auto it = d->graphs.find(key);
  if (it != d->graphs.end()) {
    *out = &it->second;
    return RTV_OK;
  }
  GraphEntry ge;
  const rtv_status s = build_graph(d, V, B, ge);
  if (s != RTV_OK) {
    for (void* p : ge.owned) cudaFree(p);
    if (ge.exec) cudaGraphExecDestroy(ge.exec);
    if (ge.graph) cudaGraphDestroy(ge.graph);
    return s;
  }
  *out = &d->graphs.emplace(key, ge).first->second;
  return RTV_OK;
}

// Enqueue one forward whose chunk stays in d->out.
rtv_status forward_to_out(rtv_draft* d, const void* vis, int n_vis, int batch, cudaStream_t st) {
  if (!d->loaded) return dfail(d, RTV_ERR_STATE, "load the draft model first");
  if (!vis) return dfail(d, RTV_ERR_ARG, "null visual tokens");
  if (n_vis <= 0 || n_vis > d->cfg.max_vis || batch <= 0 || batch > d->cfg.max_batch)
    return dfail(d, RTV_ERR_SHAPE, "n_vis or batch out of range");
  GraphEntry* ge = nullptr;
  DTRY(get_graph(d, n_vis, batch, &ge));
  const size_t bytes = (size_t)batch * n_vis * d->cfg.width * d->elt;
  DCK(cudaMemcpyAsync(d->vis_in, vis, bytes, cudaMemcpyDefault, st));
  DCK(cudaGraphLaunch(ge->exec, st));
  return RTV_OK;
}

}  // namespace

extern "C" {

rtv_status rtv_draft_create(const rtv_draft_config* cfg, int cuda_device, rtv_draft** out) {
  if (!out) return RTV_ERR_ARG;
  *out = nullptr;
  if (!cfg) return RTV_ERR_ARG;
  const rtv_draft_config& c = *cfg;
  if (c.width <= 0 || c.width % 128 || c.n_q_heads <= 0 || c.n_kv_heads <= 0 || c.n_q_heads % c.n_kv_heads ||
      c.head_dim <= 0 || c.head_dim % 2 || c.mlp_dim <= 0 || c.n_queries <= 0 || c.n_queries > 64 ||
      c.action_dim <= 0 || c.max_vis <= 0 || c.max_batch <= 0 || !(c.rms_eps >= 0.f) || !(c.rope_theta >= 0.f))
    return RTV_ERR_ARG;
  if (c.dtype != RTV_F32 && c.dtype != RTV_BF16) return RTV_ERR_ARG;
  int ndev = 0;
  if (cudaGetDeviceCount(&ndev) != cudaSuccess || cuda_device < 0 || cuda_device >= ndev) {
    cudaGetLastError();
    return RTV_ERR_CUDA;
  }
  rtv_expert_config k{};
  k.n_layers = 1;
  k.width = c.width;
  k.n_q_heads = c.n_q_heads;
  k.n_kv_heads = c.n_kv_heads;
  k.head_dim = c.head_dim;
  k.mlp_dim = c.mlp_dim;
  k.action_dim = c.action_dim;
  k.state_dim = 1;
  k.chunk_len = c.n_queries;
  k.max_prefix_len = c.max_vis;
  k.max_batch = c.max_batch;
  k.max_taus = 0;
  k.dtype = c.dtype;
  k.mlp_dtype = c.dtype;
  k.suffix_mask = RTV_MASK_BIDIR;
  k.rms_eps = c.rms_eps;
  k.rope_theta = c.rope_theta;
  k.barrier_timeout_ns = c.barrier_timeout_ns > 0 ? c.barrier_timeout_ns : 100000000LL;
  rtv_draft* d = new rtv_draft();
  d->cfg = c;
  d->device = cuda_device;
  d->elt = c.dtype == RTV_F32 ? 4 : 2;
  DeviceGuard dg(cuda_device);
  rtv_status s = ctx_create(k, cuda_device, c.n_queries, true, &d->blk);
  const size_t w = c.width, Tv = (size_t)c.max_batch * c.max_vis, KV = (size_t)c.n_kv_heads * c.head_dim;
  auto A = [&](void** p, size_t bytes, bool zero = false) {
    if (s == RTV_OK) s = dalloc(d, p, bytes, zero);
  };
  A((void**)&d->out, (size_t)c.max_batch * c.n_queries * c.action_dim * 4);
  A(&d->vis_in, Tv * w * d->elt);
  if (s == RTV_OK && d->blk->use_fast) {
    const size_t rows = (Tv + 15) / 16 * 16;
    A((void**)&d->vis_hb, rows * w * 2, true);   // padding rows stay finite
    A((void**)&d->vis_ssp, Tv * (w / 128) * 4);
  } else if (s == RTV_OK) {
    if (c.dtype == RTV_BF16) A((void**)&d->vis_f, Tv * w * 4);
    A((void**)&d->vis_u, Tv * w * 4);
    A((void**)&d->vis_kv, Tv * 2 * KV * 4);
  }
  if (s != RTV_OK) {
    rtv_draft_destroy(d);
    return s;
  }
  *out = d;
  return RTV_OK;
}

rtv_status rtv_draft_load(rtv_draft* d, const rtv_tensor* params, int n_params) {
  if (!d) return RTV_ERR_ARG;
  if (!params || n_params <= 0) return dfail(d, RTV_ERR_ARG, "no parameters");
  if (d->loaded) return dfail(d, RTV_ERR_STATE, "draft model already loaded");
  DeviceGuard dg(d->device);
  rtv_ctx* c = d->blk;
  const long long w = d->cfg.width, H = d->cfg.n_queries, A = d->cfg.action_dim;
  c->W.layers.assign(1, LayerW());
  SlotTable slots;
  add_layer_slots(c, slots, "", c->W.layers[0]);
  // the queries and the head live in allocations of the block context
  void* q_tmp = nullptr;
  void* hw_tmp = nullptr;
  float* hb_tmp = nullptr;
  slots["action_queries"] = ParamSlot{{H, w}, RTV_F32, &q_tmp, 0, nullptr, 0};
  slots["action_head.w"] = ParamSlot{{A, w}, d->cfg.dtype, &hw_tmp, 0, nullptr, 0};
  slots["action_head.b"] = ParamSlot{{A}, RTV_F32, (void**)&hb_tmp, 0, nullptr, 0};
  const rtv_status s = load_slots(c, slots, params, n_params);
  if (s != RTV_OK) return dfail(d, s, c->last_error);
  d->queries = (float*)q_tmp;
  d->head_w = hw_tmp;
  d->head_b = hb_tmp;
  if (c->use_fast) {
    const rtv_status fs = fast_load(c, params, n_params);
    if (fs != RTV_OK) return dfail(d, fs, "packing the block for the tensor cores failed");
  }
  DCK(cudaDeviceSynchronize());
  d->loaded = true;
  return RTV_OK;
}

rtv_status rtv_draft_forward(rtv_draft* d, const void* vis, int n_vis, int batch, float* chunk_out,
                             rtv_stream stream) {
  if (!d) return RTV_ERR_ARG;
  if (!chunk_out) return dfail(d, RTV_ERR_ARG, "null output");
  DeviceGuard dg(d->device);
  cudaStream_t st = (cudaStream_t)stream;
  DTRY(forward_to_out(d, vis, n_vis, batch, st));
  DCK(cudaMemcpyAsync(chunk_out, d->out, (size_t)batch * d->cfg.n_queries * d->cfg.action_dim * sizeof(float),
                      cudaMemcpyDefault, st));
  return RTV_OK;
}

rtv_status rtv_flash_round(rtv_ctx* ctx, rtv_draft* d, const void* vis, int n_vis, const float* noise,
                           const float* state, const float* taus, int n_taus, float delta, int gripper_dim,
                           int n_steps, float* actions_out, int* accepted_len, unsigned* flags, int* used_full,
                           rtv_stream stream) {
  if (!ctx || !d) return RTV_ERR_ARG;
  if (!actions_out || !accepted_len || !flags || !used_full) return dfail(d, RTV_ERR_ARG, "null output");
  if (ctx->block_only) return dfail(d, RTV_ERR_ARG, "not an expert context");
  if (ctx->device != d->device) return dfail(d, RTV_ERR_ARG, "expert and draft model on different devices");
  if (ctx->cfg.chunk_len != d->cfg.n_queries || ctx->cfg.action_dim != d->cfg.action_dim)
    return dfail(d, RTV_ERR_SHAPE, "the draft chunk shape differs from the expert's");
  if (ctx->have_prefix && ctx->prefix_batch != 1)
    return dfail(d, RTV_ERR_SHAPE, "a round serves one observation: install a prefix of batch 1");
  DeviceGuard dg(d->device);
  cudaStream_t st = (cudaStream_t)stream;
  // fast path: draft, then verification of the chunk left in d->out
  DTRY(forward_to_out(d, vis, n_vis, 1, st));
  int acc = 0;
  unsigned fl = 0;
  rtv_status s = rtv_verify(ctx, d->out, noise, state, taus, n_taus, delta, gripper_dim, &acc, &fl, nullptr,
                            stream);
  if (s != RTV_OK) return dfail(d, s, ctx->last_error);
  DCK(cudaStreamSynchronize(st));
  const bool full = (fl & (RTV_FLAG_ZERO_ACCEPT | RTV_FLAG_SWITCH)) != 0;
  if (full) {
    // full path: Euler denoising from the same noise sample
    s = rtv_denoise(ctx, noise, state, n_steps, actions_out, stream);
    if (s != RTV_OK) return dfail(d, s, ctx->last_error);
  } else {
    DCK(cudaMemcpyAsync(actions_out, d->out, (size_t)d->cfg.n_queries * d->cfg.action_dim * sizeof(float),
                        cudaMemcpyDefault, st));
  }
  DCK(cudaStreamSynchronize(st));
  *accepted_len = acc;
  *flags = fl;
  *used_full = full ? 1 : 0;
  return RTV_OK;
}

rtv_status rtv_draft_device_status(rtv_draft* d, unsigned* bits) {
  if (!d || !bits) return RTV_ERR_ARG;
  const rtv_status s = rtv_device_status(d->blk, bits);
  if (s != RTV_OK) d->last_error = d->blk->last_error;
  return s;
}

const char* rtv_draft_last_error(rtv_draft* d) { return d ? d->last_error.c_str() : "null draft model"; }

const char* rtv_draft_path_name(rtv_draft* d) { return d ? rtv_path_name(d->blk) : ""; }

int rtv_draft_kernel_count(rtv_draft* d, int n_vis, int batch) {
  if (!d) return -1;
  auto it = d->graphs.find(std::make_pair(n_vis, batch));
  return it == d->graphs.end() ? -1 : it->second.kernels;
}

void rtv_draft_destroy(rtv_draft* d) {
  if (!d) return;
  DeviceGuard dg(d->device);
  cudaDeviceSynchronize();
  for (auto& kv : d->graphs) {
    if (kv.second.exec) cudaGraphExecDestroy(kv.second.exec);
    if (kv.second.graph) cudaGraphDestroy(kv.second.graph);
    for (void* p : kv.second.owned) cudaFree(p);
  }
  for (void* p : d->allocs) cudaFree(p);
  if (d->blk) rtv_destroy(d->blk);
  cudaGetLastError();
  delete d;
}

}  // extern "C"
