// Internal state of an rtv context.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <functional>
#include <map>
#include <string>
#include <tuple>
#include <unordered_map>
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
  void* tmod_w = nullptr;  // [6w][w] per-layer time modulator (RTV_TIME_ADARMS)
  float* tmod_b = nullptr; // [6w]
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
struct ResidentState;  // resident-kernel state (resident.cu)

// One named parameter of a load table: expected shape and dtype, and where it
// goes (its own allocation, or an offset inside a packed allocation).
struct ParamSlot {
  std::vector<long long> shape;
  int dtype;          // expected input dtype
  void** dst_ptr;     // destination pointer (allocated on load)
  size_t dst_offset;  // byte offset inside a packed destination (qkv / gu), or 0
  void** pack_base;   // packed destination base (qkv/gu) or nullptr
  size_t pack_bytes;  // total bytes of the packed destination
  bool seen = false;
};
using SlotTable = std::unordered_map<std::string, ParamSlot>;

// Makes `dev` the current device for the guard's lifetime, then restores
// the caller's device.
struct DeviceGuard {
  int prev = -1;
  explicit DeviceGuard(int dev) {
    cudaGetDevice(&prev);
    if (prev != dev) cudaSetDevice(dev);
  }
  ~DeviceGuard() {
    int cur = -1;
    cudaGetDevice(&cur);
    if (prev >= 0 && cur != prev) cudaSetDevice(prev);
  }
};

// Kernel nodes of a captured graph (-1 when the graph cannot be read).
inline int count_kernel_nodes(cudaGraph_t g) {
  size_t n = 0;
  if (cudaGraphGetNodes(g, nullptr, &n) != cudaSuccess) return -1;
  std::vector<cudaGraphNode_t> nodes(n);
  cudaGraphGetNodes(g, nodes.data(), &n);
  int k = 0;
  for (auto nd : nodes) {
    cudaGraphNodeType t;
    if (cudaGraphNodeGetType(nd, &t) == cudaSuccess && t == cudaGraphNodeTypeKernel) ++k;
  }
  return k;
}

// Per-layer time modulation tables (RTV_TIME_ADARMS), rows of all layers:
// mod [.][L][6w] = (scale_a, shift_a, gate_a, scale_m, shift_m, gate_m) of
// every layer, sbq [.][L][Q+2KV] = W_qkv . shift_a and sbg [.][L][2F] =
// W_gu . shift_m (natural row order; the shifts' share of the projections).
// group_rows 0: every suffix group reads row 0 (one flow time for the
// batch); 1: group g reads row g (one flow time per verification tau).
struct ModTables {
  const float* mod = nullptr;
  const float* sbq = nullptr;
  const float* sbg = nullptr;
  int group_rows = 0;
};

// Work captured at the head of a graph, before the denoising loop.
using GraphPrologue = std::function<rtv_status(cudaStream_t)>;

}  // namespace rtv

struct rtv_ctx {
  rtv_expert_config cfg{};
  int device = 0;
  std::string last_error;
  bool loaded = false;
  int prefix_len = 0, prefix_batch = 0;
  bool have_prefix = false;
  bool use_fast = false;   // tcgen05 path
  // A bare stack of layers (the FLASH draft model's block): no suffix
  // embedding, time condition or output head of its own.
  bool block_only = false;

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
  float* czero = nullptr;   // [w] zeros: the time condition of the variants that add none to the tokens
  // RTV_TIME_ADARMS verification tables (one row per tau): see ModTables
  float *mod_v = nullptr, *sbq_v = nullptr, *sbg_v = nullptr;
  int* accepted = nullptr;
  unsigned* flags = nullptr;
  unsigned* status = nullptr;

  cudaStream_t cap_stream = nullptr;
  std::map<std::tuple<int, int, int, int>, rtv::GraphEntry> graphs;  // (kind, n, batch/taus, prefix_len)

  rtv::FastPath* fast = nullptr;
  rtv::ResidentState* resident = nullptr;   // set when the resident kernel serves this context's shapes
};

namespace rtv {

// Allocate a context's static buffers for suffixes of S token rows and pick
// its kernel path.  The caller has validated cfg and the device.
rtv_status ctx_create(const rtv_expert_config& cfg, int cuda_device, int S, bool block_only, rtv_ctx** out);
// Entries of one layer's parameters under the name prefix p.
void add_layer_slots(rtv_ctx* ctx, SlotTable& slots, const std::string& p, LayerW& L);
// Validate a parameter list against the table (every name exactly once,
// dtype and shape), then allocate and copy.  Nothing is allocated on a bad list.
rtv_status load_slots(rtv_ctx* ctx, SlotTable& slots, const rtv_tensor* params, int n_params);
// Capture (not launch) the denoising graph of n_steps Euler steps over a
// prefix of P tokens (batch 1, tensor-core path) with `prologue` enqueued
// first, on the context's capture stream, into ge.
rtv_status capture_denoise(rtv_ctx* ctx, int n_steps, int P, const GraphPrologue& prologue, GraphEntry& ge);
// The SIMT layers over G suffixes of ctx->S rows (residual stream ctx->h).
template <typename WT>
void simt_layers(rtv_ctx* ctx, int G, int P, int prefix_batch_stride, const float* rope_cs, const float* rope_sn,
                 cudaStream_t st, const ModTables* mod = nullptr);

}  // namespace rtv
