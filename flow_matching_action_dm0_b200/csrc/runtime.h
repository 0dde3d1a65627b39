// Internal state of an rtv context.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <map>
#include <string>
#include <tuple>
#include <vector>

#include "../../include/rtv.h"

namespace rtv {

struct LayerW {
  void* qkv = nullptr;    // [Q+2KV][w]   q rows, then k rows, then v rows (simt layout)
  void* o = nullptr;      // [w][Q]
  void* gu = nullptr;     // [2F][w]      gate rows, then up rows (simt layout; E4M3 codes with an FP8 MLP)
  void* down = nullptr;   // [w][F]
  float* gu_s = nullptr;  // [2F] per-row scales of gate then up (FP8 MLP only)
  float* down_s = nullptr;   // [w] per-row scales of down (FP8 MLP only)
  float* g_attn = nullptr;
  float* g_mlp = nullptr;
};

struct ExpertW {
  void* sp_w = nullptr;  float* sp_b = nullptr;
  void* ai_w = nullptr;  float* ai_b = nullptr;
  void* ti_w = nullptr;  float* ti_b = nullptr;
  void* to_w = nullptr;  float* to_b = nullptr;
  std::vector<LayerW> layers;
  float* g_final = nullptr;
  void* ao_w = nullptr;  float* ao_b = nullptr;
};

// A captured CUDA graph with the buffers that only it uses.
struct GraphEntry {
  cudaGraph_t graph = nullptr;
  cudaGraphExec_t exec = nullptr;
  std::vector<void*> owned;
  int kernels = 0;       // kernel nodes in the graph
};

struct FastPath;  // tensor-core path state (kernels_tc.cu)

}  // namespace rtv

struct rtv_ctx {
  rtv_expert_config cfg{};
  int device = 0;
  std::string last_error;
  bool loaded = false;
  int prefix_len = 0, prefix_batch = 0;
  bool have_prefix = false;
  bool use_fast = false;   // tcgen05 path

  // derived sizes
  int S = 0, H = 0, Q = 0, KV = 0, Gmax = 0, Tmax = 0, elt = 4;

  std::vector<void*> allocs;   // everything freed in rtv_destroy
  rtv::ExpertW W;
  void* prefix_kv = nullptr;   // [L][2][Bmax][Hkv][Pmax][D], config dtype

  // activations (fp32 unless stated)
  float *h = nullptr, *u = nullptr, *qkv = nullptr, *q = nullptr, *o = nullptr, *gu = nullptr, *m = nullptr;
  float *ks = nullptr, *vs = nullptr;          // suffix K/V [Gmax][Hkv][S][D]
  float *x = nullptr, *v = nullptr, *state = nullptr;
  float *e_tmp = nullptr, *z_tmp = nullptr, *c_verify = nullptr;
  float *draft = nullptr, *eps = nullptr, *taus = nullptr, *vparams = nullptr, *dist = nullptr;
  int* accepted = nullptr;
  unsigned* flags = nullptr;
  unsigned* status = nullptr;

  cudaStream_t cap_stream = nullptr;
  std::map<std::tuple<int, int, int, int>, rtv::GraphEntry> graphs;  // (kind, n, batch/taus, prefix_len)

  rtv::FastPath* fast = nullptr;
};
