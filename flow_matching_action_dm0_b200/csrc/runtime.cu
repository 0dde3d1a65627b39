// C-ABI entry points and host runtime: parameter packing, static buffers,
// CUDA-graph capture per (steps, batch, prefix length) and replay.
//
// "DM0.5 reading guide", sec. 6.5: capture once at start-up with fixed
// shapes, static buffer addresses and a fixed step count, then serve each
// request as a copy into the static buffers plus one graph replay.
#include <stdio.h>
#include <stdlib.h>
#include <string.h>

#include <cmath>
#include <string>
#include <unordered_map>

#include "fastpath.h"
#include "kernels.h"
#include "resident.h"
#include "runtime.h"

using namespace rtv;

namespace rtv {

// The layers of a context over G suffixes (residual stream ctx->h, T = G*S
// rows), SIMT kernels.  [DM0.5] 5.2: RMSNorm -> q/k/v -> RoPE -> attention
// over [prefix ; own suffix] -> o_proj + residual -> RMSNorm -> GeGLU MLP +
// residual.
template <typename WT>
void simt_layers(rtv_ctx* ctx, int G, int P, int prefix_batch_stride, const float* rope_cs, const float* rope_sn,
                 cudaStream_t st, const ModTables* mod) {
  const rtv_expert_config& k = ctx->cfg;
  const int S = ctx->S, T = G * S, w = k.width, F = k.mlp_dim;
  const int Q = ctx->Q, KV = ctx->KV, D = k.head_dim;
  const size_t kv_layer = (size_t)k.max_batch * k.n_kv_heads * k.max_prefix_len * D;
  const int mgs = mod ? mod->group_rows * k.n_layers * 6 * w : 0;   // group stride of the modulation rows
  for (int l = 0; l < k.n_layers; ++l) {
    const LayerW& L = ctx->W.layers[l];
    const WT* pk = (const WT*)ctx->prefix_kv + (size_t)(2 * l) * kv_layer;
    const WT* pv = (const WT*)ctx->prefix_kv + (size_t)(2 * l + 1) * kv_layer;
    const float* ml = mod ? mod->mod + (size_t)l * 6 * w : nullptr;   // scale/shift/gate of the layer
    if (ml) launch_rmsnorm_mod(ctx->h, ml, ml + w, mgs, ctx->u, T, w, S, k.rms_eps, st);
    else launch_rmsnorm(ctx->h, L.g_attn, ctx->u, T, w, k.rms_eps, st);
    launch_linear<WT>(ctx->u, w, (const WT*)L.qkv, nullptr, ctx->qkv, Q + 2 * KV, T, Q + 2 * KV, w, EPI_STORE, st);
    launch_rope_split(ctx->qkv, rope_cs, rope_sn, ctx->q, ctx->ks, ctx->vs, T, S, k.n_q_heads, k.n_kv_heads, D, st);
    launch_attention_simt<WT>(ctx->q, pk, pv, ctx->ks, ctx->vs, ctx->o, T, S, P, k.max_prefix_len, k.n_q_heads,
                              k.n_kv_heads, D, prefix_batch_stride, k.suffix_mask, st);
    if (ml) {
      launch_linear<WT>(ctx->o, Q, (const WT*)L.o, nullptr, ctx->u, w, T, w, Q, EPI_STORE, st);
      launch_gated_add(ctx->h, ctx->u, ml + 2 * w, mgs, w, S, T, st);
      launch_rmsnorm_mod(ctx->h, ml + 3 * w, ml + 4 * w, mgs, ctx->u, T, w, S, k.rms_eps, st);
    } else {
      launch_linear<WT>(ctx->o, Q, (const WT*)L.o, nullptr, ctx->h, w, T, w, Q, EPI_ADD, st);
      launch_rmsnorm(ctx->h, L.g_mlp, ctx->u, T, w, k.rms_eps, st);
    }
    launch_linear<WT>(ctx->u, w, (const WT*)L.gu, nullptr, ctx->gu, 2 * F, T, 2 * F, w, EPI_STORE, st);
    launch_geglu(ctx->gu, ctx->m, T, F, st);
    if (ml) {
      launch_linear<WT>(ctx->m, F, (const WT*)L.down, nullptr, ctx->u, w, T, w, F, EPI_STORE, st);
      launch_gated_add(ctx->h, ctx->u, ml + 5 * w, mgs, w, S, T, st);
    } else {
      launch_linear<WT>(ctx->m, F, (const WT*)L.down, nullptr, ctx->h, w, T, w, F, EPI_ADD, st);
    }
  }
}
template void simt_layers<float>(rtv_ctx*, int, int, int, const float*, const float*, cudaStream_t,
                                 const ModTables*);
template void simt_layers<__nv_bfloat16>(rtv_ctx*, int, int, int, const float*, const float*, cudaStream_t,
                                         const ModTables*);

// Pi0's concat time MLP over the action rows of G suffixes, in place in
// ctx->h: h <- W_to swish(W_ti[:, :w] h + c1[g]) + b_to, where c1 (group
// stride c1_gs) already holds W_ti[:, w:] e(t) + b_ti.
template <typename WT>
void concat_tokens(rtv_ctx* ctx, int G, const float* c1, int c1_gs, cudaStream_t st) {
  const int w = ctx->cfg.width, S = ctx->S, T = G * S;
  launch_rows_linear<WT>(ctx->h, w, (const WT*)ctx->W.ti_w, 2 * w, c1, c1_gs, ctx->u, w, T, S, 1, S, w, w,
                         EPI_SWISH, st);
  launch_rows_linear<WT>(ctx->u, w, (const WT*)ctx->W.to_w, w, ctx->W.to_b, 0, ctx->h, w, T, S, 1, S, w, w,
                         EPI_STORE, st);
}

// Per-layer modulation rows of n flow times from their conditions c [n][w]
// (mod), and, when sbq is set, the shifts' share of the QKV and gate/up
// projections (sbq, sbg).
template <typename WT>
void mod_tables(rtv_ctx* ctx, const float* c, int n, float* mod, float* sbq, float* sbg, cudaStream_t st) {
  const rtv_expert_config& k = ctx->cfg;
  const int w = k.width, L = k.n_layers, nq = ctx->Q + 2 * ctx->KV, F2 = 2 * k.mlp_dim;
  for (int l = 0; l < L; ++l) {
    const LayerW& Lw = ctx->W.layers[l];
    launch_rows_linear<WT>(c, w, (const WT*)Lw.tmod_w, w, Lw.tmod_b, 0, mod + (size_t)l * 6 * w, L * 6 * w, n, n, 0,
                           n, 6 * w, w, EPI_STORE, st);
    if (!sbq) continue;
    launch_rows_linear<WT>(mod + (size_t)l * 6 * w + w, L * 6 * w, (const WT*)Lw.qkv, w, nullptr, 0,
                           sbq + (size_t)l * nq, L * nq, n, n, 0, n, nq, w, EPI_STORE, st);
    launch_rows_linear<WT>(mod + (size_t)l * 6 * w + 4 * w, L * 6 * w, (const WT*)Lw.gu, w, nullptr, 0,
                           sbg + (size_t)l * F2, L * F2, n, n, 0, n, F2, w, EPI_STORE, st);
  }
}

}  // namespace rtv

namespace {

rtv_status fail(rtv_ctx* c, rtv_status s, const std::string& msg) {
  if (c) c->last_error = msg;
  return s;
}

#define CK(call)                                                                                   \
  do {                                                                                             \
    cudaError_t _e = (call);                                                                       \
    if (_e != cudaSuccess)                                                                         \
      return fail(ctx, _e == cudaErrorMemoryAllocation ? RTV_ERR_OOM : RTV_ERR_CUDA,               \
                  std::string(#call) + ": " + cudaGetErrorString(_e));                             \
  } while (0)

size_t dtype_size(int dt) { return dt == RTV_F32 ? 4 : dt == RTV_BF16 ? 2 : dt == RTV_FP8_E4M3 ? 1 : 0; }

rtv_status dev_alloc(rtv_ctx* ctx, void** p, size_t bytes) {
  *p = nullptr;
  if (bytes == 0) bytes = 16;
  CK(cudaMalloc(p, bytes));
  ctx->allocs.push_back(*p);
  return RTV_OK;
}

template <typename T>
rtv_status dev_alloc_t(rtv_ctx* ctx, T** p, size_t count) {
  void* q = nullptr;
  rtv_status s = dev_alloc(ctx, &q, count * sizeof(T));
  *p = (T*)q;
  return s;
}

#define TRY(x)                         \
  do {                                 \
    rtv_status _s = (x);               \
    if (_s != RTV_OK) return _s;       \
  } while (0)

// SIMT forward of the expert over G suffixes (token rows T = G*S) and the
// output head.  Used for the fp32 expert and, on request, the bf16 expert.
template <typename WT>
void simt_expert(rtv_ctx* ctx, int G, int P, const float* c, int c_stride, int state_stride, int prefix_batch_stride,
                 const float* rope_cs, const float* rope_sn, cudaStream_t st, const float* c1 = nullptr,
                 int c1_gs = 0, const ModTables* mod = nullptr) {
  const rtv_expert_config& k = ctx->cfg;
  launch_embed<WT>(ctx->x, ctx->state, state_stride, (const WT*)ctx->W.sp_w, ctx->W.sp_b, (const WT*)ctx->W.ai_w,
                   ctx->W.ai_b, c, c_stride, ctx->h, G, k.width, ctx->S, k.action_dim, k.state_dim, st);
  if (c1) concat_tokens<WT>(ctx, G, c1, c1_gs, st);
  simt_layers<WT>(ctx, G, P, prefix_batch_stride, rope_cs, rope_sn, st, mod);
}

// c(t) = time_mlp_out(swish(time_mlp_in(e(t)))) for n times (taus or the Euler schedule).
template <typename WT>
void time_condition(rtv_ctx* ctx, const float* taus, int n, int n_steps, float* c, cudaStream_t st) {
  const int w = ctx->cfg.width;
  launch_time_embedding(taus, n, n_steps, ctx->e_tmp, w, st);
  launch_linear<WT>(ctx->e_tmp, w, (const WT*)ctx->W.ti_w, ctx->W.ti_b, ctx->z_tmp, w, n, w, w, EPI_SWISH, st);
  launch_linear<WT>(ctx->z_tmp, w, (const WT*)ctx->W.to_w, ctx->W.to_b, c, w, n, w, w, EPI_STORE, st);
}

enum { KIND_DENOISE = 0, KIND_VERIFY = 1 };

// Precompute the input-independent tables of a graph (time condition of the
// Euler schedule, RoPE table of the suffix positions, the time modulator's
// rows), then capture.
template <typename WT>
rtv_status build_graph(rtv_ctx* ctx, int kind, int n, int batch, int P, GraphEntry& ge,
                       const GraphPrologue* prologue = nullptr) {
  const rtv_expert_config& k = ctx->cfg;
  cudaStream_t st = ctx->cap_stream;
  const int S = ctx->S, D = k.head_dim, w = k.width, L = k.n_layers;
  const int nq = ctx->Q + 2 * ctx->KV, F2 = 2 * k.mlp_dim;
  const int tc = k.time_cond;
  auto table = [&](float** p, size_t count) -> rtv_status {
    CK(cudaMalloc(p, sizeof(float) * count));
    ge.owned.push_back(*p);
    return RTV_OK;
  };
  float *cs = nullptr, *sn = nullptr, *ctab = nullptr, *modtab = nullptr, *sbq = nullptr, *sbg = nullptr;
  TRY(table(&cs, (size_t)S * (D / 2)));
  TRY(table(&sn, (size_t)S * (D / 2)));
  launch_rope_table(cs, sn, S, D, P, k.rope_theta, st);
  if (kind == KIND_DENOISE) {
    // per Euler step t_k (n <= 64 rows): c(t_k) = W_to swish(W_ti e(t_k) + b_ti) + b_to; with Pi0's
    // concat MLP instead the time half of its first layer, W_ti[:, w:] e(t_k) + b_ti; with the per-layer
    // modulator also the modulation rows of every layer
    TRY(table(&ctab, (size_t)n * w));
    launch_time_embedding(nullptr, n, n, ctx->e_tmp, w, st);
    if (tc == RTV_TIME_CONCAT) {
      launch_rows_linear<WT>(ctx->e_tmp, w, (const WT*)ctx->W.ti_w + w, 2 * w, ctx->W.ti_b, 0, ctab, w, n, n, 0, n,
                             w, w, EPI_STORE, st);
    } else {
      launch_linear<WT>(ctx->e_tmp, w, (const WT*)ctx->W.ti_w, ctx->W.ti_b, ctx->z_tmp, w, n, w, w, EPI_SWISH, st);
      launch_linear<WT>(ctx->z_tmp, w, (const WT*)ctx->W.to_w, ctx->W.to_b, ctab, w, n, w, w, EPI_STORE, st);
    }
    if (tc == RTV_TIME_ADARMS) {
      TRY(table(&modtab, (size_t)n * L * 6 * w));
      if (ctx->use_fast) {
        TRY(table(&sbq, (size_t)n * L * nq));
        TRY(table(&sbg, (size_t)n * L * F2));
      }
      mod_tables<WT>(ctx, ctab, n, modtab, sbq, sbg, st);
    }
  }
  CK(cudaGetLastError());
  CK(cudaStreamSynchronize(st));
  // The resident kernel serves the plain time condition on the tensor-core
  // path when its plan fits (prepared here, outside the capture).
  const bool use_res = ctx->use_fast && tc == RTV_TIME_ADD &&
                       resident_prepare(ctx, kind == KIND_DENOISE ? batch : n, P, kind == KIND_VERIFY);

  if (ctx->use_fast) fast_arm_trace(ctx);
  CK(cudaStreamBeginCapture(st, cudaStreamCaptureModeThreadLocal));
  rtv_status fs = RTV_OK;
  auto chain = [&](rtv_status s2) {
    if (fs == RTV_OK) fs = s2;
  };
  if (prologue) chain((*prologue)(st));
  // what the embedding of a step adds to the action rows: c (RTV_TIME_ADD) or nothing
  const bool add_c = tc == RTV_TIME_ADD;
  if (kind == KIND_DENOISE) {
    const float dt = (float)(1.0 / (double)n);
    auto mod_of = [&](int step) {
      ModTables m;
      m.mod = modtab + (size_t)step * L * 6 * w;
      m.sbq = sbq ? sbq + (size_t)step * L * nq : nullptr;
      m.sbg = sbg ? sbg + (size_t)step * L * F2 : nullptr;
      m.group_rows = 0;
      return m;
    };
    if (use_res) {
      chain(resident_launch(ctx, batch, P, n, false, ctab, cs, sn, st));
    } else if (ctx->use_fast) {
      // step boundary k: head of step k-1 (k > 0) and embedding of step k (k < n)
      auto embed_tail = [&](int step) {
        if (tc == RTV_TIME_CONCAT) {
          concat_tokens<WT>(ctx, batch, ctab + (size_t)step * w, 0, st);
          chain(fast_norm_rows(ctx, batch, st));
        }
      };
      const float* g00 = tc == RTV_TIME_ADARMS ? modtab : nullptr;
      chain(fast_step(ctx, batch, false, true, dt, add_c ? ctab : ctx->czero, 0, k.state_dim, false, st, g00, 0));
      embed_tail(0);
      for (int step = 0; step < n && fs == RTV_OK; ++step) {
        ModTables m;
        if (tc == RTV_TIME_ADARMS) m = mod_of(step);
        chain(fast_layers(ctx, batch, P, 1, cs, sn, st, tc == RTV_TIME_ADARMS ? &m : nullptr));
        const bool more = step + 1 < n;
        const float* cnext = add_c ? (more ? ctab + (size_t)(step + 1) * w : ctab) : ctx->czero;
        const float* g0 = (tc == RTV_TIME_ADARMS && more) ? modtab + (size_t)(step + 1) * L * 6 * w : nullptr;
        chain(fast_step(ctx, batch, true, more, dt, cnext, 0, k.state_dim, false, st, g0, 0));
        if (more) embed_tail(step + 1);
      }
    } else {
      for (int step = 0; step < n; ++step) {
        ModTables m;
        if (tc == RTV_TIME_ADARMS) m = mod_of(step);
        simt_expert<WT>(ctx, batch, P, add_c ? ctab + (size_t)step * w : ctx->czero, 0, k.state_dim, 1, cs, sn, st,
                        tc == RTV_TIME_CONCAT ? ctab + (size_t)step * w : nullptr, 0,
                        tc == RTV_TIME_ADARMS ? &m : nullptr);
        launch_out_head<WT>(ctx->h, ctx->W.g_final, (const WT*)ctx->W.ao_w, ctx->W.ao_b, ctx->x, nullptr, dt, batch,
                            w, S, k.action_dim, k.rms_eps, ctx->status, st);
      }
    }
  } else {
    const int T = n;
    launch_verify_interp(ctx->draft, ctx->eps, ctx->taus, ctx->x, T, ctx->H * k.action_dim, st);
    // one flow time per suffix group: c(tau_i) rows (or the concat MLP's time half), and the
    // modulation rows of every layer
    if (tc == RTV_TIME_CONCAT) {
      launch_time_embedding(ctx->taus, T, 0, ctx->e_tmp, w, st);
      launch_rows_linear<WT>(ctx->e_tmp, w, (const WT*)ctx->W.ti_w + w, 2 * w, ctx->W.ti_b, 0, ctx->c_verify, w, T,
                             T, 0, T, w, w, EPI_STORE, st);
    } else {
      time_condition<WT>(ctx, ctx->taus, T, 0, ctx->c_verify, st);
    }
    ModTables m;
    if (tc == RTV_TIME_ADARMS) {
      mod_tables<WT>(ctx, ctx->c_verify, T, ctx->mod_v, ctx->use_fast ? ctx->sbq_v : nullptr,
                     ctx->use_fast ? ctx->sbg_v : nullptr, st);
      m.mod = ctx->mod_v;
      m.sbq = ctx->sbq_v;
      m.sbg = ctx->sbg_v;
      m.group_rows = 1;
    }
    const ModTables* mp = tc == RTV_TIME_ADARMS ? &m : nullptr;
    if (use_res) {
      chain(resident_launch(ctx, T, P, 1, true, ctx->c_verify, cs, sn, st));
    } else if (ctx->use_fast) {
      chain(fast_step(ctx, T, false, true, 0.f, add_c ? ctx->c_verify : ctx->czero, add_c ? w : 0, 0, false, st,
                      mp ? ctx->mod_v : nullptr, mp ? L * 6 * w : 0));
      if (tc == RTV_TIME_CONCAT) {
        concat_tokens<WT>(ctx, T, ctx->c_verify, w, st);
        chain(fast_norm_rows(ctx, T, st));
      }
      chain(fast_layers(ctx, T, P, 0, cs, sn, st, mp));
      chain(fast_step(ctx, T, true, false, 0.f, ctx->c_verify, w, 0, true, st));
    } else {
      simt_expert<WT>(ctx, T, P, add_c ? ctx->c_verify : ctx->czero, add_c ? w : 0, 0, 0, cs, sn, st,
                      tc == RTV_TIME_CONCAT ? ctx->c_verify : nullptr, w, mp);
      launch_out_head<WT>(ctx->h, ctx->W.g_final, (const WT*)ctx->W.ao_w, ctx->W.ao_b, ctx->x, ctx->v, 0.f, T, w,
                          S, k.action_dim, k.rms_eps, ctx->status, st);
    }
    launch_verify_decide(ctx->x, ctx->v, ctx->draft, ctx->taus, ctx->vparams, T, ctx->H, k.action_dim, ctx->dist,
                         ctx->accepted, ctx->flags, st);
  }
  cudaGraph_t g = nullptr;
  cudaError_t e1 = cudaGetLastError();
  cudaError_t e2 = cudaStreamEndCapture(st, &g);
  if (fs != RTV_OK) {
    if (g) cudaGraphDestroy(g);
    return fs;
  }
  if (e1 != cudaSuccess || e2 != cudaSuccess) {
    if (g) cudaGraphDestroy(g);
    return fail(ctx, RTV_ERR_CUDA, std::string("graph capture: ") +
                                       cudaGetErrorString(e1 != cudaSuccess ? e1 : e2));
  }
  ge.graph = g;
  ge.kernels = count_kernel_nodes(g);
  CK(cudaGraphInstantiate(&ge.exec, g, 0));
  CK(cudaGraphUpload(ge.exec, st));
  CK(cudaStreamSynchronize(st));
  return RTV_OK;
}

rtv_status get_graph(rtv_ctx* ctx, int kind, int n, int batch, GraphEntry** out) {
  auto key = std::make_tuple(kind, n, batch, ctx->prefix_len);
  auto it = ctx->graphs.find(key);
  if (it != ctx->graphs.end()) {
    *out = &it->second;
    return RTV_OK;
  }
  GraphEntry ge;
  rtv_status s = ctx->cfg.dtype == RTV_F32 ? build_graph<float>(ctx, kind, n, batch, ctx->prefix_len, ge)
                                           : build_graph<__nv_bfloat16>(ctx, kind, n, batch, ctx->prefix_len, ge);
  if (s != RTV_OK) {
    for (void* p : ge.owned) cudaFree(p);
    if (ge.exec) cudaGraphExecDestroy(ge.exec);
    if (ge.graph) cudaGraphDestroy(ge.graph);
    return s;
  }
  auto res = ctx->graphs.emplace(key, ge);
  *out = &res.first->second;
  return RTV_OK;
}

}  // namespace

namespace rtv {

rtv_status capture_denoise(rtv_ctx* ctx, int n_steps, int P, const GraphPrologue& prologue, GraphEntry& ge) {
  if (!ctx->use_fast || ctx->cfg.dtype != RTV_BF16)
    return fail(ctx, RTV_ERR_UNSUPPORTED, "capture with a prologue needs the tensor-core path");
  const rtv_status s = build_graph<__nv_bfloat16>(ctx, KIND_DENOISE, n_steps, 1, P, ge, &prologue);
  if (s != RTV_OK) {
    for (void* p : ge.owned) cudaFree(p);
    ge.owned.clear();
    if (ge.exec) cudaGraphExecDestroy(ge.exec);
    if (ge.graph) cudaGraphDestroy(ge.graph);
    ge.exec = nullptr;
    ge.graph = nullptr;
  }
  return s;
}

rtv_status ctx_create(const rtv_expert_config& k, int cuda_device, int S, bool block_only, rtv_ctx** out) {
  *out = nullptr;
  rtv_ctx* ctx = new rtv_ctx();
  ctx->cfg = k;
  ctx->device = cuda_device;
  ctx->block_only = block_only;
  DeviceGuard dg(cuda_device);
  ctx->S = S;
  ctx->H = S - 1;
  ctx->Q = k.n_q_heads * k.head_dim;
  ctx->KV = k.n_kv_heads * k.head_dim;
  ctx->Gmax = k.max_batch > k.max_taus ? k.max_batch : k.max_taus;
  ctx->Tmax = ctx->Gmax * ctx->S;
  ctx->elt = (int)dtype_size(k.dtype);
  const int w = k.width, F = k.mlp_dim, D = k.head_dim;
  const size_t T = ctx->Tmax;
  const int H = ctx->H > 0 ? ctx->H : 1;
  rtv_status s = RTV_OK;
  auto A = [&](float** p, size_t n) { if (s == RTV_OK) s = dev_alloc_t(ctx, p, n); };
  A(&ctx->h, T * w);
  A(&ctx->u, T * w);
  A(&ctx->qkv, T * (ctx->Q + 2 * ctx->KV));
  A(&ctx->q, T * ctx->Q);
  A(&ctx->o, T * ctx->Q);
  A(&ctx->gu, T * 2 * F);
  A(&ctx->m, T * F);
  A(&ctx->ks, (size_t)ctx->Gmax * ctx->KV * ctx->S);
  A(&ctx->vs, (size_t)ctx->Gmax * ctx->KV * ctx->S);
  A(&ctx->x, (size_t)ctx->Gmax * H * k.action_dim);
  A(&ctx->v, (size_t)ctx->Gmax * H * k.action_dim);
  A(&ctx->state, (size_t)ctx->Gmax * k.state_dim);
  const size_t rows_e = T > 64 ? T : 64;   // e/z scratch rows (>= the Euler schedule length limit)
  A(&ctx->e_tmp, rows_e * w);
  A(&ctx->z_tmp, rows_e * w);
  A(&ctx->c_verify, (size_t)(ctx->Gmax) * w);
  A(&ctx->draft, (size_t)H * k.action_dim);
  A(&ctx->eps, (size_t)H * k.action_dim);
  A(&ctx->taus, (size_t)(ctx->Gmax > 0 ? ctx->Gmax : 1));
  A(&ctx->vparams, 4);
  A(&ctx->dist, (size_t)(ctx->Gmax > 0 ? ctx->Gmax : 1) * H);
  A(&ctx->czero, (size_t)w);
  if (k.time_cond == RTV_TIME_ADARMS) {
    const size_t G1 = ctx->Gmax > 0 ? ctx->Gmax : 1, L = k.n_layers;
    A(&ctx->mod_v, G1 * L * 6 * w);
    A(&ctx->sbq_v, G1 * L * (ctx->Q + 2 * ctx->KV));
    A(&ctx->sbg_v, G1 * L * 2 * F);
  }
  if (s == RTV_OK) s = dev_alloc_t(ctx, &ctx->accepted, 1);
  if (s == RTV_OK) s = dev_alloc_t(ctx, &ctx->flags, 1);
  if (s == RTV_OK) s = dev_alloc_t(ctx, &ctx->status, 1);
  void* kvp = nullptr;
  if (s == RTV_OK)
    s = dev_alloc(ctx, &kvp, (size_t)k.n_layers * 2 * k.max_batch * k.n_kv_heads * k.max_prefix_len * D * ctx->elt);
  ctx->prefix_kv = kvp;
  if (s == RTV_OK && cudaMemset(ctx->status, 0, sizeof(unsigned)) != cudaSuccess) s = RTV_ERR_CUDA;
  if (s == RTV_OK && cudaMemset(ctx->czero, 0, sizeof(float) * w) != cudaSuccess) s = RTV_ERR_CUDA;
  if (s == RTV_OK && cudaStreamCreateWithFlags(&ctx->cap_stream, cudaStreamNonBlocking) != cudaSuccess)
    s = RTV_ERR_CUDA;
  if (s == RTV_OK && k.dtype == RTV_BF16) {
    const char* env = getenv("RTV_PATH");
    const bool want_simt = env && strcmp(env, "simt") == 0;
    if (!want_simt) s = fast_create(ctx);
    if (s == RTV_OK && ctx->use_fast) s = resident_create(ctx);
  }
  if (s == RTV_OK && k.mlp_dtype == RTV_FP8_E4M3 && !ctx->use_fast) s = RTV_ERR_UNSUPPORTED;   // no SIMT FP8
  if (s != RTV_OK) {
    rtv_destroy(ctx);
    return s;
  }
  *out = ctx;
  return RTV_OK;
}

void add_layer_slots(rtv_ctx* ctx, SlotTable& slots, const std::string& p, LayerW& L) {
  const rtv_expert_config& k = ctx->cfg;
  const long long w = k.width, F = k.mlp_dim, Q = ctx->Q, KV = ctx->KV;
  const int md = k.dtype;
  const size_t e = ctx->elt;
  if (k.time_cond == RTV_TIME_ADARMS) {
    // the per-layer time modulator replaces the two norm gains
    slots[p + "time_mod.w"] = ParamSlot{{6 * w, w}, md, &L.tmod_w, 0, nullptr, 0};
    slots[p + "time_mod.b"] = ParamSlot{{6 * w}, RTV_F32, (void**)&L.tmod_b, 0, nullptr, 0};
  } else {
    slots[p + "attn_norm.g"] = ParamSlot{{w}, RTV_F32, (void**)&L.g_attn, 0, nullptr, 0};
    slots[p + "mlp_norm.g"] = ParamSlot{{w}, RTV_F32, (void**)&L.g_mlp, 0, nullptr, 0};
  }
  const size_t qkv_bytes = (size_t)(Q + 2 * KV) * w * e;
  slots[p + "q_proj.w"] = ParamSlot{{Q, w}, md, nullptr, 0, &L.qkv, qkv_bytes};
  slots[p + "k_proj.w"] = ParamSlot{{KV, w}, md, nullptr, (size_t)Q * w * e, &L.qkv, qkv_bytes};
  slots[p + "v_proj.w"] = ParamSlot{{KV, w}, md, nullptr, (size_t)(Q + KV) * w * e, &L.qkv, qkv_bytes};
  slots[p + "o_proj.w"] = ParamSlot{{w, Q}, md, &L.o, 0, nullptr, 0};
  const int mdt = k.mlp_dtype;
  const size_t em = dtype_size(mdt);
  const size_t gu_bytes = (size_t)2 * F * w * em;
  slots[p + "gate_proj.w"] = ParamSlot{{F, w}, mdt, nullptr, 0, &L.gu, gu_bytes};
  slots[p + "up_proj.w"] = ParamSlot{{F, w}, mdt, nullptr, (size_t)F * w * em, &L.gu, gu_bytes};
  slots[p + "down_proj.w"] = ParamSlot{{w, F}, mdt, &L.down, 0, nullptr, 0};
  if (mdt == RTV_FP8_E4M3) {
    slots[p + "gate_proj.s"] = ParamSlot{{F}, RTV_F32, nullptr, 0, (void**)&L.gu_s, (size_t)2 * F * 4};
    slots[p + "up_proj.s"] = ParamSlot{{F}, RTV_F32, nullptr, (size_t)F * 4, (void**)&L.gu_s, (size_t)2 * F * 4};
    slots[p + "down_proj.s"] = ParamSlot{{w}, RTV_F32, (void**)&L.down_s, 0, nullptr, 0};
  }
}

rtv_status load_slots(rtv_ctx* ctx, SlotTable& slots, const rtv_tensor* params, int n_params) {
  // validate every entry first: nothing is allocated on a bad table
  for (int i = 0; i < n_params; ++i) {
    const rtv_tensor& t = params[i];
    if (!t.name || !t.data) return fail(ctx, RTV_ERR_ARG, "parameter with null name or data");
    auto it = slots.find(t.name);
    if (it == slots.end()) return fail(ctx, RTV_ERR_ARG, std::string("unknown parameter ") + t.name);
    ParamSlot& sl = it->second;
    if (sl.seen) return fail(ctx, RTV_ERR_ARG, std::string("duplicate parameter ") + t.name);
    if (t.dtype != sl.dtype) return fail(ctx, RTV_ERR_ARG, std::string("wrong dtype for ") + t.name);
    if (t.ndim != (int)sl.shape.size()) return fail(ctx, RTV_ERR_SHAPE, std::string("wrong rank for ") + t.name);
    for (int d = 0; d < t.ndim; ++d)
      if (t.shape[d] != sl.shape[d]) return fail(ctx, RTV_ERR_SHAPE, std::string("wrong shape for ") + t.name);
    sl.seen = true;
  }
  for (auto& kv : slots)
    if (!kv.second.seen) {
      for (auto& kv2 : slots) kv2.second.seen = false;
      return fail(ctx, RTV_ERR_ARG, "missing parameter " + kv.first);
    }

  // allocate and copy
  for (int i = 0; i < n_params; ++i) {
    const rtv_tensor& t = params[i];
    ParamSlot& sl = slots[t.name];
    size_t n = 1;
    for (long long d : sl.shape) n *= (size_t)d;
    const size_t bytes = n * dtype_size(sl.dtype);
    void* dst = nullptr;
    if (sl.pack_base) {
      if (!*sl.pack_base) TRY(dev_alloc(ctx, sl.pack_base, sl.pack_bytes));
      dst = (char*)*sl.pack_base + sl.dst_offset;
    } else {
      TRY(dev_alloc(ctx, sl.dst_ptr, bytes));
      dst = *sl.dst_ptr;
    }
    CK(cudaMemcpy(dst, t.data, bytes, cudaMemcpyDefault));
  }
  return RTV_OK;
}

}  // namespace rtv

// ===========================================================================
// C ABI
// ===========================================================================
extern "C" {

rtv_status rtv_create(const rtv_expert_config* cfg_in, int cuda_device, rtv_ctx** out) {
  if (!out) return RTV_ERR_ARG;
  *out = nullptr;
  if (!cfg_in) return RTV_ERR_ARG;
  rtv_expert_config k = *cfg_in;
  if (k.n_layers <= 0 || k.width <= 0 || k.width % 2 || k.n_q_heads <= 0 || k.n_kv_heads <= 0 ||
      k.n_q_heads % k.n_kv_heads || k.head_dim <= 0 || k.head_dim % 2 || k.mlp_dim <= 0 || k.action_dim <= 0 ||
      k.state_dim <= 0 || k.chunk_len <= 0 || k.max_prefix_len <= 0 || k.max_batch <= 0 || k.max_taus < 0 ||
      k.width < 32 || k.width % 32)
    return RTV_ERR_ARG;
  if (k.dtype != RTV_F32 && k.dtype != RTV_BF16) return RTV_ERR_ARG;
  if (k.mlp_dtype == RTV_SAME) k.mlp_dtype = k.dtype;
  // FP8 E4M3 MLP weights ride on bf16 activations (tensor-core path only)
  if (k.mlp_dtype != k.dtype && !(k.mlp_dtype == RTV_FP8_E4M3 && k.dtype == RTV_BF16)) return RTV_ERR_UNSUPPORTED;
  if (k.suffix_mask != RTV_MASK_BIDIR && k.suffix_mask != RTV_MASK_PI0_BLOCK) return RTV_ERR_ARG;
  if (k.time_cond != RTV_TIME_ADD && k.time_cond != RTV_TIME_CONCAT && k.time_cond != RTV_TIME_ADARMS)
    return RTV_ERR_ARG;
  // the modulator's shift terms are taken from the bf16/fp32 gate/up rows
  if (k.time_cond == RTV_TIME_ADARMS && k.mlp_dtype == RTV_FP8_E4M3) return RTV_ERR_UNSUPPORTED;
  if (!(k.rms_eps >= 0.f) || !(k.rope_theta >= 0.f)) return RTV_ERR_ARG;
  if (k.barrier_timeout_ns <= 0) k.barrier_timeout_ns = 100000000LL;

  int ndev = 0;
  if (cudaGetDeviceCount(&ndev) != cudaSuccess || cuda_device < 0 || cuda_device >= ndev) {
    cudaGetLastError();
    return RTV_ERR_CUDA;
  }
  return ctx_create(k, cuda_device, 1 + k.chunk_len, false, out);
}

rtv_status rtv_load_expert(rtv_ctx* ctx, const rtv_tensor* params, int n_params) {
  if (!ctx) return RTV_ERR_ARG;
  if (!params || n_params <= 0) return fail(ctx, RTV_ERR_ARG, "no parameters");
  if (ctx->loaded) return fail(ctx, RTV_ERR_STATE, "expert already loaded");
  if (ctx->block_only) return fail(ctx, RTV_ERR_STATE, "not an expert context");
  DeviceGuard dg(ctx->device);
  const rtv_expert_config& k = ctx->cfg;
  const long long w = k.width, A = k.action_dim, Sd = k.state_dim;
  const int md = k.dtype;
  ExpertW& W = ctx->W;
  W.layers.assign(k.n_layers, LayerW());

  SlotTable slots;
  auto mat = [&](const std::string& n, long long r, long long c, void** dst) {
    slots[n] = ParamSlot{{r, c}, md, dst, 0, nullptr, 0};
  };
  auto vec = [&](const std::string& n, long long r, float** dst) {
    slots[n] = ParamSlot{{r}, RTV_F32, (void**)dst, 0, nullptr, 0};
  };
  mat("state_proj.w", w, Sd, &W.sp_w);
  vec("state_proj.b", w, &W.sp_b);
  mat("action_in_proj.w", w, A, &W.ai_w);
  vec("action_in_proj.b", w, &W.ai_b);
  mat("time_mlp_in.w", w, k.time_cond == RTV_TIME_CONCAT ? 2 * w : w, &W.ti_w);
  vec("time_mlp_in.b", w, &W.ti_b);
  mat("time_mlp_out.w", w, w, &W.to_w);
  vec("time_mlp_out.b", w, &W.to_b);
  vec("final_norm.g", w, &W.g_final);
  mat("action_out_proj.w", A, w, &W.ao_w);
  vec("action_out_proj.b", A, &W.ao_b);
  for (int l = 0; l < k.n_layers; ++l)
    add_layer_slots(ctx, slots, "layers." + std::to_string(l) + ".", W.layers[l]);
  TRY(load_slots(ctx, slots, params, n_params));
  if (ctx->use_fast) TRY(fast_load(ctx, params, n_params));
  TRY(resident_load(ctx));
  CK(cudaDeviceSynchronize());
  ctx->loaded = true;
  return RTV_OK;
}

rtv_status rtv_set_prefix_kv(rtv_ctx* ctx, const void* kv, int prefix_len, int batch, rtv_stream stream) {
  if (!ctx) return RTV_ERR_ARG;
  if (!kv) return fail(ctx, RTV_ERR_ARG, "null prefix kv");
  const rtv_expert_config& k = ctx->cfg;
  if (prefix_len <= 0 || prefix_len > k.max_prefix_len || batch <= 0 || batch > k.max_batch)
    return fail(ctx, RTV_ERR_SHAPE, "prefix_len or batch out of range");
  if (ctx->use_fast && !fast_supports_prefix(ctx, prefix_len))
    return fail(ctx, RTV_ERR_UNSUPPORTED, "prefix length not supported by the tensor-core path");
  DeviceGuard dg(ctx->device);
  cudaStream_t st = (cudaStream_t)stream;
  const size_t n = (size_t)k.n_layers * 2 * batch * prefix_len * k.n_kv_heads * k.head_dim;
  const size_t bytes = n * ctx->elt;
  cudaPointerAttributes at{};
  const void* src = kv;
  void* tmp = nullptr;
  if (cudaPointerGetAttributes(&at, kv) != cudaSuccess || at.type != cudaMemoryTypeDevice) {
    cudaGetLastError();
    CK(cudaMallocAsync(&tmp, bytes, st));
    CK(cudaMemcpyAsync(tmp, kv, bytes, cudaMemcpyDefault, st));
    src = tmp;
  }
  if (k.dtype == RTV_F32)
    launch_prefix_pack<float>((const float*)src, (float*)ctx->prefix_kv, k.n_layers, batch, prefix_len,
                              k.n_kv_heads, k.head_dim, k.max_batch, k.max_prefix_len, st);
  else
    launch_prefix_pack<__nv_bfloat16>((const __nv_bfloat16*)src, (__nv_bfloat16*)ctx->prefix_kv, k.n_layers, batch,
                                      prefix_len, k.n_kv_heads, k.head_dim, k.max_batch, k.max_prefix_len, st);
  CK(cudaGetLastError());
  if (tmp) CK(cudaFreeAsync(tmp, st));
  if (ctx->use_fast) {
    const rtv_status fs = fast_prefix_update(ctx, batch, prefix_len, st);
    if (fs != RTV_OK) return fs;
  }
  ctx->prefix_len = prefix_len;
  ctx->prefix_batch = batch;
  ctx->have_prefix = true;
  return RTV_OK;
}

rtv_status rtv_denoise(rtv_ctx* ctx, const float* noise, const float* state, int n_steps, float* actions_out,
                       rtv_stream stream) {
  if (!ctx) return RTV_ERR_ARG;
  if (!noise || !state || !actions_out) return fail(ctx, RTV_ERR_ARG, "null pointer");
  if (!ctx->loaded || !ctx->have_prefix) return fail(ctx, RTV_ERR_STATE, "load the expert and the prefix first");
  if (n_steps <= 0 || n_steps > 64) return fail(ctx, RTV_ERR_SHAPE, "n_steps must be in [1, 64]");
  DeviceGuard dg(ctx->device);
  const rtv_expert_config& k = ctx->cfg;
  const int B = ctx->prefix_batch;
  cudaStream_t st = (cudaStream_t)stream;
  GraphEntry* ge = nullptr;
  TRY(get_graph(ctx, KIND_DENOISE, n_steps, B, &ge));
  const size_t xb = (size_t)B * ctx->H * k.action_dim * sizeof(float);
  CK(cudaMemcpyAsync(ctx->x, noise, xb, cudaMemcpyDefault, st));
  CK(cudaMemcpyAsync(ctx->state, state, (size_t)B * k.state_dim * sizeof(float), cudaMemcpyDefault, st));
  CK(cudaGraphLaunch(ge->exec, st));
  CK(cudaMemcpyAsync(actions_out, ctx->x, xb, cudaMemcpyDefault, st));
  if (ctx->use_fast && getenv("RTV_TRACE")) {
    fast_trace_report(ctx);
    resident_trace_report(ctx);
  }
  return RTV_OK;
}

rtv_status rtv_verify(rtv_ctx* ctx, const float* draft, const float* noise, const float* state, const float* taus,
                      int n_taus, float delta, int gripper_dim, int* accepted_len, unsigned* flags, float* dist,
                      rtv_stream stream) {
  if (!ctx) return RTV_ERR_ARG;
  if (!draft || !noise || !state || !taus || !accepted_len || !flags) return fail(ctx, RTV_ERR_ARG, "null pointer");
  if (!ctx->loaded || !ctx->have_prefix) return fail(ctx, RTV_ERR_STATE, "load the expert and the prefix first");
  const rtv_expert_config& k = ctx->cfg;
  if (n_taus <= 0 || n_taus > k.max_taus) return fail(ctx, RTV_ERR_SHAPE, "n_taus out of range");
  if (gripper_dim < 0 || gripper_dim >= k.action_dim) return fail(ctx, RTV_ERR_ARG, "gripper_dim out of range");
  if (!(delta >= 0.f)) return fail(ctx, RTV_ERR_ARG, "delta must be >= 0");
  for (int i = 0; i < n_taus; ++i)
    if (!(taus[i] >= 0.f && taus[i] <= 1.f)) return fail(ctx, RTV_ERR_ARG, "taus must lie in [0, 1]");
  DeviceGuard dg(ctx->device);
  cudaStream_t st = (cudaStream_t)stream;
  GraphEntry* ge = nullptr;
  TRY(get_graph(ctx, KIND_VERIFY, n_taus, 1, &ge));
  const size_t hb = (size_t)ctx->H * k.action_dim * sizeof(float);
  // host-side parameter block, copied by value into the static buffers
  float hp[4] = {delta, (float)gripper_dim, 0.f, 0.f};
  CK(cudaMemcpyAsync(ctx->draft, draft, hb, cudaMemcpyDefault, st));
  CK(cudaMemcpyAsync(ctx->eps, noise, hb, cudaMemcpyDefault, st));
  CK(cudaMemcpyAsync(ctx->state, state, (size_t)k.state_dim * sizeof(float), cudaMemcpyDefault, st));
  CK(cudaMemcpyAsync(ctx->taus, taus, (size_t)n_taus * sizeof(float), cudaMemcpyHostToDevice, st));
  CK(cudaMemcpyAsync(ctx->vparams, hp, sizeof(hp), cudaMemcpyHostToDevice, st));
  // copies from pageable host memory are staged before cudaMemcpyAsync returns, so the
  // stack-held parameter block may go out of scope
  CK(cudaGraphLaunch(ge->exec, st));
  CK(cudaMemcpyAsync(accepted_len, ctx->accepted, sizeof(int), cudaMemcpyDefault, st));
  CK(cudaMemcpyAsync(flags, ctx->flags, sizeof(unsigned), cudaMemcpyDefault, st));
  if (dist) CK(cudaMemcpyAsync(dist, ctx->dist, (size_t)n_taus * ctx->H * sizeof(float), cudaMemcpyDefault, st));
  if (ctx->use_fast && getenv("RTV_TRACE")) {
    fast_trace_report(ctx);
    resident_trace_report(ctx);
  }
  return RTV_OK;
}

rtv_status rtv_device_status(rtv_ctx* ctx, unsigned* bits) {
  if (!ctx || !bits) return RTV_ERR_ARG;
  DeviceGuard dg(ctx->device);
  CK(cudaDeviceSynchronize());
  unsigned v = 0;
  CK(cudaMemcpy(&v, ctx->status, sizeof(v), cudaMemcpyDeviceToHost));
  CK(cudaMemset(ctx->status, 0, sizeof(unsigned)));
  *bits = v;
  if (v & RTV_DEV_TIMEOUT) return fail(ctx, RTV_ERR_TIMEOUT, "a device-side wait gave up");
  if (v & RTV_DEV_NUMERIC) return fail(ctx, RTV_ERR_NUMERIC, "non-finite action values");
  return RTV_OK;
}

const char* rtv_last_error(rtv_ctx* ctx) { return ctx ? ctx->last_error.c_str() : "null context"; }

const char* rtv_path_name(rtv_ctx* ctx) { return ctx ? (ctx->use_fast ? "tcgen05" : "simt") : ""; }

int rtv_graph_kernel_count(rtv_ctx* ctx, int n, int is_verify) {
  if (!ctx) return -1;
  auto key = std::make_tuple(is_verify ? (int)KIND_VERIFY : (int)KIND_DENOISE, n, is_verify ? 1 : ctx->prefix_batch,
                             ctx->prefix_len);
  auto it = ctx->graphs.find(key);
  return it == ctx->graphs.end() ? -1 : it->second.kernels;
}

void rtv_destroy(rtv_ctx* ctx) {
  if (!ctx) return;
  DeviceGuard dg(ctx->device);
  cudaDeviceSynchronize();
  for (auto& kv : ctx->graphs) {
    if (kv.second.exec) cudaGraphExecDestroy(kv.second.exec);
    if (kv.second.graph) cudaGraphDestroy(kv.second.graph);
    for (void* p : kv.second.owned) cudaFree(p);
  }
  if (ctx->resident) resident_destroy(ctx);
  if (ctx->fast) fast_destroy(ctx);
  for (void* p : ctx->allocs) cudaFree(p);
  if (ctx->cap_stream) cudaStreamDestroy(ctx->cap_stream);
  cudaGetLastError();
  delete ctx;
}

}  // extern "C"
