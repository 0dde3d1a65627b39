// Installing the prefix KV cache without allocating device memory.
//
// Some callers cannot call cudaMalloc once they are running: a real-time
// robot control loop that must never block on the allocator (cudaMalloc can
// synchronise the device and its latency is unbounded), or a process whose
// device memory is owned by another allocator or a fixed budget.  For them
// rtv_set_prefix_kv_static stages a host-resident prefix cache through a
// fixed-size array in device global memory, declared at file scope below,
// instead of the temporary buffer rtv_set_prefix_kv allocates.
//
// The staging array is shared by every context and every call on a device,
// and it keeps whatever the last call left in it.  Calls whose work overlaps
// on the GPU (different streams, or different contexts on one device) race
// on it: serialise them.  The array (kStageBytes) lives in this file's
// module.  CUDA loads modules lazily, so the first call on a device -- which
// looks up the array's device address -- may be the moment the driver loads
// the module and reserves the array; that first call should therefore come
// at set-up time, before any stream capture.  From then on the device holds
// the array until the process exits and no call allocates anything.
#include <mutex>
#include <string>

#include "fastpath.h"
#include "kernels.h"
#include "runtime.h"

namespace {

// One layer's keys and values (2 * batch * prefix_len * n_kv_heads * head_dim
// elements) must fit; larger caches are refused.
constexpr size_t kStageBytes = 4u << 20;   // 4 MiB

static __device__ __align__(256) unsigned char g_prefix_stage[kStageBytes];

// Device address of g_prefix_stage, looked up once per device.  In host code
// the array's name is only a host-side stand-in for the symbol, so kernels
// and copies must be given this address instead.
std::mutex g_stage_mu;
constexpr int kMaxDevices = 256;
void* g_stage_addr[kMaxDevices] = {};

rtv_status stage_address(rtv_ctx* ctx, void** out) {
  std::lock_guard<std::mutex> lock(g_stage_mu);
  if (ctx->device < 0 || ctx->device >= kMaxDevices) return RTV_ERR_ARG;
  if (!g_stage_addr[ctx->device]) {
    void* p = nullptr;
    const cudaError_t e = cudaGetSymbolAddress(&p, g_prefix_stage);
    if (e != cudaSuccess || !p) {
      ctx->last_error = std::string("cudaGetSymbolAddress(staging array): ") + cudaGetErrorString(e);
      return RTV_ERR_CUDA;
    }
    g_stage_addr[ctx->device] = p;
  }
  *out = g_stage_addr[ctx->device];
  return RTV_OK;
}

}  // namespace

extern "C" rtv_status rtv_set_prefix_kv_static(rtv_ctx* ctx, const void* kv, int prefix_len, int batch,
                                               rtv_stream stream) {
  if (!ctx) return RTV_ERR_ARG;
  if (!kv) {
    ctx->last_error = "null prefix kv";
    return RTV_ERR_ARG;
  }
  const rtv_expert_config& k = ctx->cfg;
  if (prefix_len <= 0 || prefix_len > k.max_prefix_len || batch <= 0 || batch > k.max_batch) {
    ctx->last_error = "prefix_len or batch out of range";
    return RTV_ERR_SHAPE;
  }
  if (ctx->use_fast && !rtv::fast_supports_prefix(ctx, prefix_len)) {
    ctx->last_error = "prefix length not supported by the tensor-core path";
    return RTV_ERR_UNSUPPORTED;
  }
  const size_t elems_layer = (size_t)2 * batch * prefix_len * k.n_kv_heads * k.head_dim;
  const size_t bytes_layer = elems_layer * (size_t)ctx->elt;
  if (bytes_layer > kStageBytes) {
    ctx->last_error = "one layer of the prefix cache (" + std::to_string(bytes_layer) +
                      " bytes) exceeds the static staging array (" + std::to_string(kStageBytes) + " bytes)";
    return RTV_ERR_SHAPE;
  }
  int prev = -1;
  cudaGetDevice(&prev);
  if (prev != ctx->device) cudaSetDevice(ctx->device);
  void* stage = nullptr;
  rtv_status s = stage_address(ctx, &stage);
  cudaStream_t st = (cudaStream_t)stream;
  cudaPointerAttributes at{};
  const bool dev_mem = cudaPointerGetAttributes(&at, kv) == cudaSuccess && at.type == cudaMemoryTypeDevice;
  cudaGetLastError();
  // Device memory of this GPU is read in place by the pack kernel; another
  // GPU's memory is refused (the pack kernel would need peer access to it).
  if (s == RTV_OK && dev_mem && at.device != ctx->device) {
    ctx->last_error = "prefix kv is device memory of another GPU (" + std::to_string(at.device) + ")";
    s = RTV_ERR_ARG;
  }
  const bool on_device = dev_mem;
  // From here on the library's cache is being overwritten: until every layer
  // is installed, denoise and verify refuse to run (RTV_ERR_STATE) rather
  // than read a cache that mixes two prefixes.
  if (s == RTV_OK) ctx->have_prefix = false;
  const size_t dst_layer = (size_t)2 * k.max_batch * k.n_kv_heads * k.max_prefix_len * k.head_dim;
  for (int l = 0; l < k.n_layers && s == RTV_OK; ++l) {
    const char* src = (const char*)kv + (size_t)l * bytes_layer;
    if (!on_device) {
      // host (pageable or pinned) or managed data goes through the staging
      // array; the pack below reads it before the next layer's copy
      // overwrites it (same stream)
      const cudaError_t e = cudaMemcpyAsync(stage, src, bytes_layer, cudaMemcpyDefault, st);
      if (e != cudaSuccess) {
        ctx->last_error = std::string("cudaMemcpyAsync to the staging array: ") + cudaGetErrorString(e);
        s = RTV_ERR_CUDA;
        break;
      }
      src = (const char*)stage;
    }
    if (k.dtype == RTV_F32)
      rtv::launch_prefix_pack<float>((const float*)src, (float*)ctx->prefix_kv + (size_t)l * dst_layer, 1, batch,
                                     prefix_len, k.n_kv_heads, k.head_dim, k.max_batch, k.max_prefix_len, st);
    else
      rtv::launch_prefix_pack<__nv_bfloat16>((const __nv_bfloat16*)src,
                                             (__nv_bfloat16*)ctx->prefix_kv + (size_t)l * dst_layer, 1, batch,
                                             prefix_len, k.n_kv_heads, k.head_dim, k.max_batch, k.max_prefix_len,
                                             st);
    const cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) {
      ctx->last_error = std::string("prefix pack launch: ") + cudaGetErrorString(e);
      s = RTV_ERR_CUDA;
    }
  }
  if (s == RTV_OK && ctx->use_fast) s = rtv::fast_prefix_update(ctx, batch, prefix_len, st);
  if (prev >= 0 && prev != ctx->device) cudaSetDevice(prev);
  if (s != RTV_OK) return s;
  ctx->prefix_len = prefix_len;
  ctx->prefix_batch = batch;
  ctx->have_prefix = true;
  return RTV_OK;
}
