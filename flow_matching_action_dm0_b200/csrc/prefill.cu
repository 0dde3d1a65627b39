// VLM prefill writing the action expert's prefix KV cache, and prefill plus
// denoising captured as one CUDA graph.
//
// "DM0.5 reading guide" sec. 5.1: the prefix (images, text, state) is
// encoded once into a per-layer KV cache that every denoising step reads;
// sec. 6.5: a request is served by one replay of a graph captured at
// start-up.  The stack is a Gemma-style VLM with as many layers as the
// expert and the same kv heads and head_dim: layer l's keys (after RoPE at
// positions 0..P-1) and values are the expert's cached prefix of layer l.
// Every prefix token attends to every prefix token; the last layer's
// attention output and MLP feed nothing and are not computed.
//
// The stack runs as a bare block context on the tensor-core path.  Its
// projections are the expert's GEMM kernel with P token rows (tiles of about
// 128 tokens, grid z), which at 816 tokens makes them compute-bound; its
// attention is the expert's tensor-core attention with the prefix split into
// groups of 64 query rows that read the layer's keys and values from the
// expert's prefix tiles, written there by the QKV projection of that layer.
#include <stdio.h>
#include <stdlib.h>
#include <string.h>

#include <map>
#include <string>
#include <utility>
#include <vector>

#include "fastpath.h"
#include "kernels.h"
#include "runtime.h"

using namespace rtv;

struct rtv_prefill {
  rtv_prefill_config cfg{};
  int device = 0;
  rtv_ctx* blk = nullptr;   // the stack: suffix = a group of 64 query rows, groups = ceil(max_tokens / 64)
  std::string last_error;
  bool loaded = false;
  void* emb_in = nullptr;   // [max_tokens][width] bf16: the graphs' fixed input address
  // graphs by (n_tokens, n_steps): n_steps 0 = the prefill alone, else
  // prefill + denoising of the expert `owner` (one graph)
  struct Entry {
    GraphEntry ge;
    rtv_ctx* owner = nullptr;
    float* rope = nullptr;   // [2][n_tokens][D/2] cos, sin
  };
  std::map<std::pair<int, int>, Entry> graphs;
  std::vector<void*> allocs;
};

namespace {

rtv_status pfail(rtv_prefill* p, rtv_status s, const std::string& msg) {
  if (p) p->last_error = msg;
  return s;
}

#define PCK(call)                                                                                  \
  do {                                                                                             \
    cudaError_t _e = (call);                                                                       \
    if (_e != cudaSuccess)                                                                         \
      return pfail(p, _e == cudaErrorMemoryAllocation ? RTV_ERR_OOM : RTV_ERR_CUDA,                \
                   std::string(#call) + ": " + cudaGetErrorString(_e));                            \
  } while (0)

void release(rtv_prefill::Entry& en) {
  if (en.ge.exec) cudaGraphExecDestroy(en.ge.exec);
  if (en.ge.graph) cudaGraphDestroy(en.ge.graph);
  for (void* q : en.ge.owned) cudaFree(q);
  if (en.rope) cudaFree(en.rope);
}

// The expert must read exactly what the stack writes.
rtv_status check_pair(rtv_prefill* p, rtv_ctx* ex, int n_tokens) {
  if (!ex) return pfail(p, RTV_ERR_ARG, "null expert context");
  if (!p->loaded || !ex->loaded) return pfail(p, RTV_ERR_STATE, "load the prefill stack and the expert first");
  if (ex->block_only) return pfail(p, RTV_ERR_ARG, "not an expert context");
  if (ex->device != p->device) return pfail(p, RTV_ERR_ARG, "expert and prefill stack on different devices");
  const rtv_expert_config& kx = ex->cfg;
  if (kx.n_layers != p->cfg.n_layers || kx.n_kv_heads != p->cfg.n_kv_heads || kx.head_dim != p->cfg.head_dim ||
      kx.dtype != p->cfg.dtype)
    return pfail(p, RTV_ERR_SHAPE, "the expert's layers, kv heads, head_dim or dtype differ from the stack's");
  if (n_tokens <= 0 || n_tokens > p->cfg.max_tokens || n_tokens > kx.max_prefix_len)
    return pfail(p, RTV_ERR_SHAPE, "n_tokens out of range");
  if (!ex->use_fast || !p->blk->use_fast)
    return pfail(p, RTV_ERR_UNSUPPORTED, "prefill needs the tensor-core path for both");
  return RTV_OK;
}

// Capture the prefill (n_steps == 0) or prefill + denoising graph.
rtv_status get_entry(rtv_prefill* p, rtv_ctx* ex, int P, int n_steps, rtv_prefill::Entry** out) {
  const auto key = std::make_pair(P, n_steps);
  auto it = p->graphs.find(key);
  if (it != p->graphs.end() && it->second.owner == ex) {
    *out = &it->second;
    return RTV_OK;
  }
  if (it != p->graphs.end()) {   // captured for another expert
    release(it->second);
    p->graphs.erase(it);
  }
  rtv_prefill::Entry en;
  en.owner = ex;
  const int D = p->cfg.head_dim;
  cudaStream_t st = p->blk->cap_stream;
  PCK(cudaMalloc(&en.rope, sizeof(float) * 2 * (size_t)P * (D / 2)));
  float* cs = en.rope;
  float* sn = en.rope + (size_t)P * (D / 2);
  launch_rope_table(cs, sn, P, D, 0, p->cfg.rope_theta, st);
  PCK(cudaGetLastError());
  PCK(cudaStreamSynchronize(st));
  const __nv_bfloat16* emb = (const __nv_bfloat16*)p->emb_in;
  rtv_ctx* blk = p->blk;
  auto body = [blk, ex, emb, P, cs, sn](cudaStream_t s) { return fast_prefill(blk, ex, emb, P, cs, sn, s); };
  rtv_status s = RTV_OK;
  if (n_steps == 0) {
    blk->last_error.clear();
    cudaError_t e = cudaStreamBeginCapture(st, cudaStreamCaptureModeThreadLocal);
    if (e != cudaSuccess) s = pfail(p, RTV_ERR_CUDA, std::string("capture: ") + cudaGetErrorString(e));
    if (s == RTV_OK) {
      const rtv_status fs = body(st);
      cudaGraph_t g = nullptr;
      const cudaError_t e1 = cudaGetLastError();
      const cudaError_t e2 = cudaStreamEndCapture(st, &g);
      if (fs != RTV_OK || e1 != cudaSuccess || e2 != cudaSuccess) {
        if (g) cudaGraphDestroy(g);
        s = fs != RTV_OK ? pfail(p, fs, blk->last_error)
                         : pfail(p, RTV_ERR_CUDA, std::string("prefill graph capture: ") +
                                                      cudaGetErrorString(e1 != cudaSuccess ? e1 : e2));
      } else {
        en.ge.graph = g;
        if (cudaGraphInstantiate(&en.ge.exec, g, 0) != cudaSuccess || cudaGraphUpload(en.ge.exec, st) != cudaSuccess)
          s = pfail(p, RTV_ERR_CUDA, "prefill graph instantiation failed");
      }
    }
  } else {
    // the prologue runs on the expert's capture stream, inside its capture
    ex->last_error.clear();
    s = capture_denoise(ex, n_steps, P, body, en.ge);
    if (s != RTV_OK) s = pfail(p, s, !blk->last_error.empty() ? blk->last_error : ex->last_error);
  }
  if (s == RTV_OK) {
    en.ge.kernels = count_kernel_nodes(en.ge.graph);
    if (cudaStreamSynchronize(st) != cudaSuccess) s = pfail(p, RTV_ERR_CUDA, "prefill graph upload failed");
  }
  if (s != RTV_OK) {
    release(en);
    return s;
  }
  *out = &p->graphs.emplace(key, en).first->second;
  return RTV_OK;
}

rtv_status stage_embeddings(rtv_prefill* p, const void* emb, int P, cudaStream_t st) {
  if (!emb) return pfail(p, RTV_ERR_ARG, "null embeddings");
  PCK(cudaMemcpyAsync(p->emb_in, emb, (size_t)P * p->cfg.width * 2, cudaMemcpyDefault, st));
  return RTV_OK;
}

void mark_prefix(rtv_ctx* ex, int P) {
  ex->prefix_len = P;
  ex->prefix_batch = 1;
  ex->have_prefix = true;
}

}  // namespace

extern "C" {

rtv_status rtv_prefill_create(const rtv_prefill_config* cfg, int cuda_device, rtv_prefill** out) {
  if (!out) return RTV_ERR_ARG;
  *out = nullptr;
  if (!cfg) return RTV_ERR_ARG;
  const rtv_prefill_config& c = *cfg;
  if (c.n_layers <= 0 || c.width <= 0 || c.width % 128 || c.n_q_heads <= 0 || c.n_kv_heads <= 0 ||
      c.n_q_heads % c.n_kv_heads || c.head_dim <= 0 || c.head_dim % 2 || c.mlp_dim <= 0 || c.max_tokens <= 0 ||
      !(c.rms_eps >= 0.f) || !(c.rope_theta >= 0.f))
    return RTV_ERR_ARG;
  if (c.dtype != RTV_F32 && c.dtype != RTV_BF16) return RTV_ERR_ARG;
  if (c.dtype != RTV_BF16) return RTV_ERR_UNSUPPORTED;   // tensor-core path only
  int ndev = 0;
  if (cudaGetDeviceCount(&ndev) != cudaSuccess || cuda_device < 0 || cuda_device >= ndev) {
    cudaGetLastError();
    return RTV_ERR_CUDA;
  }
  constexpr int kGroup = 64;   // query rows per attention group
  rtv_expert_config k{};
  k.n_layers = c.n_layers;
  k.width = c.width;
  k.n_q_heads = c.n_q_heads;
  k.n_kv_heads = c.n_kv_heads;
  k.head_dim = c.head_dim;
  k.mlp_dim = c.mlp_dim;
  k.action_dim = 1;
  k.state_dim = 1;
  k.chunk_len = kGroup - 1;
  k.max_prefix_len = 1;                                  // the stack caches no prefix of its own
  k.max_batch = (c.max_tokens + kGroup - 1) / kGroup;   // query groups
  k.max_taus = 0;
  k.dtype = c.dtype;
  k.mlp_dtype = c.dtype;
  k.suffix_mask = RTV_MASK_BIDIR;
  k.rms_eps = c.rms_eps;
  k.rope_theta = c.rope_theta;
  k.barrier_timeout_ns = c.barrier_timeout_ns > 0 ? c.barrier_timeout_ns : 100000000LL;
  rtv_prefill* p = new rtv_prefill();
  p->cfg = c;
  p->device = cuda_device;
  DeviceGuard dg(cuda_device);
  rtv_status s = ctx_create(k, cuda_device, kGroup, true, &p->blk);
  if (s == RTV_OK && !p->blk->use_fast) s = RTV_ERR_UNSUPPORTED;
  if (s == RTV_OK) {
    if (cudaMalloc(&p->emb_in, (size_t)c.max_tokens * c.width * 2) != cudaSuccess) s = RTV_ERR_OOM;
    else p->allocs.push_back(p->emb_in);
  }
  if (s != RTV_OK) {
    rtv_prefill_destroy(p);
    return s;
  }
  *out = p;
  return RTV_OK;
}

rtv_status rtv_prefill_load(rtv_prefill* p, const rtv_tensor* params, int n_params) {
  if (!p) return RTV_ERR_ARG;
  if (!params || n_params <= 0) return pfail(p, RTV_ERR_ARG, "no parameters");
  if (p->loaded) return pfail(p, RTV_ERR_STATE, "prefill stack already loaded");
  DeviceGuard dg(p->device);
  rtv_ctx* c = p->blk;
  c->W.layers.assign(c->cfg.n_layers, LayerW());
  SlotTable slots;
  for (int l = 0; l < c->cfg.n_layers; ++l) add_layer_slots(c, slots, "layers." + std::to_string(l) + ".", c->W.layers[l]);
  rtv_status s = load_slots(c, slots, params, n_params);
  if (s != RTV_OK) return pfail(p, s, c->last_error);
  s = fast_load(c, params, n_params);
  if (s != RTV_OK) return pfail(p, s, "packing the stack for the tensor cores failed");
  PCK(cudaDeviceSynchronize());
  // only the packed tensor-core copies are read from here on
  for (LayerW& L : c->W.layers)
    for (void** m : {&L.qkv, &L.o, &L.gu, &L.down}) {
      for (auto it = c->allocs.begin(); it != c->allocs.end(); ++it)
        if (*it == *m) {
          c->allocs.erase(it);
          break;
        }
      cudaFree(*m);
      *m = nullptr;
    }
  p->loaded = true;
  return RTV_OK;
}

rtv_status rtv_prefill_kv(rtv_prefill* p, rtv_ctx* ex, const void* emb, int n_tokens, rtv_stream stream) {
  if (!p) return RTV_ERR_ARG;
  rtv_status s = check_pair(p, ex, n_tokens);
  if (s != RTV_OK) return s;
  DeviceGuard dg(p->device);
  rtv_prefill::Entry* en = nullptr;
  s = get_entry(p, ex, n_tokens, 0, &en);
  if (s != RTV_OK) return s;
  cudaStream_t st = (cudaStream_t)stream;
  s = stage_embeddings(p, emb, n_tokens, st);
  if (s != RTV_OK) return s;
  PCK(cudaGraphLaunch(en->ge.exec, st));
  mark_prefix(ex, n_tokens);
  return RTV_OK;
}

rtv_status rtv_prefill_denoise(rtv_prefill* p, rtv_ctx* ex, const void* emb, int n_tokens, const float* noise,
                               const float* state, int n_steps, float* actions_out, rtv_stream stream) {
  if (!p) return RTV_ERR_ARG;
  rtv_status s = check_pair(p, ex, n_tokens);
  if (s != RTV_OK) return s;
  if (!noise || !state || !actions_out) return pfail(p, RTV_ERR_ARG, "null pointer");
  if (n_steps <= 0 || n_steps > 64) return pfail(p, RTV_ERR_SHAPE, "n_steps must be in [1, 64]");
  if (ex->cfg.max_batch < 1) return pfail(p, RTV_ERR_SHAPE, "expert batch");
  DeviceGuard dg(p->device);
  rtv_prefill::Entry* en = nullptr;
  s = get_entry(p, ex, n_tokens, n_steps, &en);
  if (s != RTV_OK) return s;
  cudaStream_t st = (cudaStream_t)stream;
  s = stage_embeddings(p, emb, n_tokens, st);
  if (s != RTV_OK) return s;
  const size_t xb = (size_t)ex->H * ex->cfg.action_dim * sizeof(float);
  PCK(cudaMemcpyAsync(ex->x, noise, xb, cudaMemcpyDefault, st));
  PCK(cudaMemcpyAsync(ex->state, state, (size_t)ex->cfg.state_dim * sizeof(float), cudaMemcpyDefault, st));
  PCK(cudaGraphLaunch(en->ge.exec, st));
  PCK(cudaMemcpyAsync(actions_out, ex->x, xb, cudaMemcpyDefault, st));
  mark_prefix(ex, n_tokens);
  return RTV_OK;
}

rtv_status rtv_prefill_device_status(rtv_prefill* p, unsigned* bits) {
  if (!p || !bits) return RTV_ERR_ARG;
  const rtv_status s = rtv_device_status(p->blk, bits);
  if (s != RTV_OK) p->last_error = p->blk->last_error;
  return s;
}

const char* rtv_prefill_last_error(rtv_prefill* p) { return p ? p->last_error.c_str() : "null prefill stack"; }

int rtv_prefill_kernel_count(rtv_prefill* p, int n_tokens, int n_steps) {
  if (!p) return -1;
  auto it = p->graphs.find(std::make_pair(n_tokens, n_steps));
  return it == p->graphs.end() ? -1 : it->second.ge.kernels;
}

void rtv_prefill_destroy(rtv_prefill* p) {
  if (!p) return;
  DeviceGuard dg(p->device);
  cudaDeviceSynchronize();
  for (auto& kv : p->graphs) release(kv.second);
  for (void* q : p->allocs) cudaFree(q);
  if (p->blk) rtv_destroy(p->blk);
  cudaGetLastError();
  delete p;
}

}  // extern "C"
