// Host-side launchers of the action-expert kernels (internal to the library).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>

namespace rtv {

enum { EPI_STORE = 0, EPI_ADD = 1, EPI_SWISH = 2 };

void launch_time_embedding(const float* taus, int n, int n_steps, float* e, int w, cudaStream_t st);

template <typename WT>
void launch_linear(const float* x, int ldx, const WT* W, const float* bias, float* y, int ldy, int M, int N, int K,
                   int epi, cudaStream_t st);

template <typename WT>
void launch_embed(const float* x, const float* state, int state_group_stride, const WT* w_sp, const float* b_sp,
                  const WT* w_ai, const float* b_ai, const float* c, int c_group_stride, float* h, int G, int w,
                  int S, int A, int Sd, cudaStream_t st);

void launch_rmsnorm(const float* h, const float* gain, float* u, int rows, int w, float eps, cudaStream_t st);

void launch_rope_table(float* cs, float* sn, int S, int D, int P, float theta, cudaStream_t st);

void launch_rope_split(const float* qkv, const float* cs, const float* sn, float* q, float* ks, float* vs, int T,
                       int S, int Hq, int Hkv, int D, cudaStream_t st);

template <typename KT>
void launch_attention_simt(const float* q, const KT* pk, const KT* pv, const float* sk, const float* sv, float* o,
                           int T, int S, int P, int Pmax, int Hq, int Hkv, int D, int prefix_batch_stride,
                           int mask_mode, cudaStream_t st);

void launch_geglu(const float* gu, float* m, int T, int F, cudaStream_t st);

// y[t][n] = act(x[t] . W[n] + bias[t / S][n]) (EPI_ADD: +=) for rows t < T
// with t % S in [s_lo, s_hi); W rows of stride ldw; bias group stride bias_gs.
template <typename WT>
void launch_rows_linear(const float* x, int ldx, const WT* W, int ldw, const float* bias, int bias_gs, float* y,
                        int ldy, int T, int S, int s_lo, int s_hi, int N, int K, int epi, cudaStream_t st);

// u = h / rms(h) * (1 + scale[t / S]) + shift[t / S] (group stride gs).
void launch_rmsnorm_mod(const float* h, const float* scale, const float* shift, int gs, float* u, int rows, int w,
                        int S, float eps, cudaStream_t st);

// h[t] += gate[t / S] * b[t] (group stride gs).
void launch_gated_add(float* h, const float* b, const float* gate, int gs, int w, int S, int T, cudaStream_t st);

template <typename WT>
void launch_out_head(const float* h, const float* gain, const WT* w_ao, const float* b_ao, float* x, float* vout,
                     float dt, int G, int w, int S, int A, float eps, unsigned* status, cudaStream_t st);

void launch_verify_interp(const float* draft, const float* eps, const float* taus, float* x, int T, int HA,
                          cudaStream_t st);

void launch_verify_decide(const float* x, const float* v, const float* draft, const float* taus,
                          const float* params, int T, int H, int A, float* dist, int* accepted, unsigned* flags,
                          cudaStream_t st);

template <typename KT>
void launch_prefix_pack(const KT* src, KT* dst, int L, int B, int P, int Hkv, int D, int Bmax, int Pmax,
                        cudaStream_t st);

}  // namespace rtv
