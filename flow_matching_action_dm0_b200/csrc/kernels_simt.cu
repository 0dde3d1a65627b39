// SIMT (FFMA) kernels of the action expert.  They serve the fp32 expert,
// whose tolerance (1e-4 on the final actions) rules out bf16/tf32 tensor
// cores, and the steps of the bf16 expert that are not matrix products
// (suffix embedding, time conditioning, output projection + Euler step,
// verification decision).
#include <math.h>

#include <algorithm>

#include "common.cuh"
#include "kernels.h"

namespace rtv {

// ---------------------------------------------------------------------------
// Time conditioning, first half: the sinusoidal embedding e(t)
// ("DM0.5 reading guide", sec. 5.2 time_mlp_in/out).  Periods run
// geometrically from 4e-3 to 4.0; angles are taken in double precision
// because 2*pi*t/4e-3 reaches ~1.6e3 rad.
// t = taus[g] when taus != nullptr, else t = 1 - g/n_steps (the Euler times).
// ---------------------------------------------------------------------------
__global__ void time_embedding_kernel(const float* __restrict__ taus, int n_steps, float* __restrict__ e, int w) {
  const int g = blockIdx.x;
  const double t = taus ? (double)taus[g] : 1.0 - (double)g / (double)n_steps;
  const int half = w / 2;
  const double ratio = 4.0 / 4e-3;
  for (int i = threadIdx.x; i < half; i += blockDim.x) {
    const double period = 4e-3 * pow(ratio, (double)i / (double)(half - 1));
    const double ang = 2.0 * 3.14159265358979323846 * t / period;
    e[(size_t)g * w + i] = (float)sin(ang);
    e[(size_t)g * w + half + i] = (float)cos(ang);
  }
}

// ---------------------------------------------------------------------------
// y[M][N] (op)= x[M][K] . W[N][K]^T (+ bias): 64x64 output tile per block,
// 16x16 threads with 4x4 outputs each, k-tiles of 16 staged in shared memory.
// ---------------------------------------------------------------------------
template <typename WT, int EPI>
__global__ void __launch_bounds__(256) linear_kernel(const float* __restrict__ x, int ldx, const WT* __restrict__ W,
                                                     const float* __restrict__ bias, float* __restrict__ y, int ldy,
                                                     int M, int N, int K) {
  __shared__ float xs[16][68];
  __shared__ float ws[16][68];
  const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
  const int m0 = blockIdx.y * 64, n0 = blockIdx.x * 64;
  float acc[4][4];
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int j = 0; j < 4; ++j) acc[i][j] = 0.f;

  for (int k0 = 0; k0 < K; k0 += 16) {
    for (int i = threadIdx.x; i < 1024; i += 256) {
      const int r = i >> 4, c = i & 15;
      const int m = m0 + r, k = k0 + c;
      xs[c][r] = (m < M && k < K) ? x[(size_t)m * ldx + k] : 0.f;
      const int n = n0 + r;
      ws[c][r] = (n < N && k < K) ? to_f32(W[(size_t)n * K + k]) : 0.f;
    }
    __syncthreads();
#pragma unroll
    for (int kk = 0; kk < 16; ++kk) {
      float a[4], b[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) a[i] = xs[kk][ty * 4 + i];
#pragma unroll
      for (int j = 0; j < 4; ++j) b[j] = ws[kk][tx * 4 + j];
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(a[i], b[j], acc[i][j]);
    }
    __syncthreads();
  }
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int m = m0 + ty * 4 + i;
    if (m >= M) continue;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int n = n0 + tx * 4 + j;
      if (n >= N) continue;
      float v = acc[i][j] + (bias ? bias[n] : 0.f);
      float* dst = y + (size_t)m * ldy + n;
      if (EPI == EPI_ADD) *dst += v;
      else if (EPI == EPI_SWISH) *dst = swish(v);
      else *dst = v;
    }
  }
}

// ---------------------------------------------------------------------------
// Suffix embedding ("DM0.5 reading guide", sec. 5.2): token 0 of group g is
// state_proj(state_g); token 1+j is action_in_proj(x_g[j]) + c_g.
// ---------------------------------------------------------------------------
template <typename WT>
__global__ void embed_kernel(const float* __restrict__ x, const float* __restrict__ state, int state_group_stride,
                             const WT* __restrict__ w_sp, const float* __restrict__ b_sp, const WT* __restrict__ w_ai,
                             const float* __restrict__ b_ai, const float* __restrict__ c, int c_group_stride,
                             float* __restrict__ h, int w, int S, int A, int Sd) {
  __shared__ float xin[64];
  const int r = blockIdx.x;
  const int g = r / S, s = r % S;
  const float* src = s == 0 ? state + (size_t)g * state_group_stride : x + ((size_t)g * (S - 1) + (s - 1)) * A;
  const int K = s == 0 ? Sd : A;
  const WT* W = s == 0 ? w_sp : w_ai;
  for (int i = threadIdx.x; i < w; i += blockDim.x) {
    float acc = 0.f;
    for (int k0 = 0; k0 < K; k0 += 64) {
      __syncthreads();
      for (int kk = threadIdx.x; kk < 64; kk += blockDim.x) xin[kk] = (k0 + kk < K) ? src[k0 + kk] : 0.f;
      __syncthreads();
      // all weight loads of the chunk are independent: issue them together
      float wv[64];
#pragma unroll
      for (int k = 0; k < 64; ++k) wv[k] = (k0 + k < K) ? to_f32(W[(size_t)i * K + k0 + k]) : 0.f;
#pragma unroll
      for (int k = 0; k < 64; ++k)
        if (k0 + k < K) acc = fmaf(wv[k], xin[k], acc);
    }
    acc += s == 0 ? b_sp[i] : b_ai[i];
    if (s != 0) acc += c[(size_t)g * c_group_stride + i];
    h[(size_t)r * w + i] = acc;
  }
}

// RMSNorm with (1 + g) gain, one block per row.
__global__ void rmsnorm_kernel(const float* __restrict__ h, const float* __restrict__ gain, float* __restrict__ u, int w,
                               float eps) {
  __shared__ float red[32];
  const float* row = h + (size_t)blockIdx.x * w;
  float ss = 0.f;
  for (int i = threadIdx.x; i < w; i += blockDim.x) ss = fmaf(row[i], row[i], ss);
  ss = block_sum(ss, red);
  const float inv = rsqrtf(ss / (float)w + eps);
  for (int i = threadIdx.x; i < w; i += blockDim.x) u[(size_t)blockIdx.x * w + i] = row[i] * inv * (1.f + gain[i]);
}

// ---------------------------------------------------------------------------
// Rotary embedding table cos/sin[S][D/2] for suffix positions P..P+S-1,
// computed in double (angles reach ~1e3 rad).
// ---------------------------------------------------------------------------
__global__ void rope_table_kernel(float* __restrict__ cs, float* __restrict__ sn, int S, int D, int P, float theta) {
  const int half = D / 2;
  for (int idx = blockIdx.x * blockDim.x + threadIdx.x; idx < S * half; idx += gridDim.x * blockDim.x) {
    const int s = idx / half, d = idx % half;
    if (theta == 0.f) {
      cs[idx] = 1.f;
      sn[idx] = 0.f;
      continue;
    }
    const double inv_freq = pow((double)theta, -2.0 * (double)d / (double)D);
    const double ang = (double)(P + s) * inv_freq;
    cs[idx] = (float)cos(ang);
    sn[idx] = (float)sin(ang);
  }
}

// Split qkv [T][Q+2KV] into rotated q [T][Hq][D] and the suffix K/V
// [G][Hkv][S][D] of this layer.
__global__ void rope_split_kernel(const float* __restrict__ qkv, const float* __restrict__ cs,
                                  const float* __restrict__ sn, float* __restrict__ q, float* __restrict__ ks,
                                  float* __restrict__ vs, int S, int Hq, int Hkv, int D) {
  const int r = blockIdx.x;
  const int g = r / S, s = r % S;
  const int half = D / 2;
  const int ld = (Hq + 2 * Hkv) * D;
  const float* src = qkv + (size_t)r * ld;
  for (int idx = threadIdx.x; idx < (Hq + Hkv) * half; idx += blockDim.x) {
    const int head = idx / half, d = idx % half;
    const float c = cs[s * half + d], si = sn[s * half + d];
    const float x1 = src[head * D + d], x2 = src[head * D + d + half];
    const float y1 = x1 * c - x2 * si, y2 = x2 * c + x1 * si;
    if (head < Hq) {
      q[((size_t)r * Hq + head) * D + d] = y1;
      q[((size_t)r * Hq + head) * D + d + half] = y2;
    } else {
      const int kh = head - Hq;
      float* dst = ks + (((size_t)g * Hkv + kh) * S + s) * D;
      dst[d] = y1;
      dst[d + half] = y2;
    }
  }
  for (int idx = threadIdx.x; idx < Hkv * D; idx += blockDim.x) {
    const int kh = idx / D, d = idx % D;
    vs[(((size_t)g * Hkv + kh) * S + s) * D + d] = src[(Hq + Hkv) * D + idx];
  }
}

// ---------------------------------------------------------------------------
// Suffix attention over [prefix ; own suffix] ("DM0.5 reading guide",
// sec. 5.1-5.2): one block per (token row, query head); scores in shared
// memory, max-subtracted softmax in fp32.
// prefix K/V: [Bmax][Hkv][Pmax][D] of type KT; suffix K/V: [G][Hkv][S][D] fp32.
// ---------------------------------------------------------------------------
template <typename KT>
__global__ void attention_simt_kernel(const float* __restrict__ q, const KT* __restrict__ pk, const KT* __restrict__ pv,
                                      const float* __restrict__ sk, const float* __restrict__ sv, float* __restrict__ o,
                                      int S, int P, int Pmax, int Hq, int Hkv, int D, int prefix_batch_stride,
                                      int mask_mode) {
  extern __shared__ float sm[];
  float* qs = sm;            // D
  float* sc = sm + D;        // P + S
  __shared__ float red[32];
  const int r = blockIdx.x, j = blockIdx.y;
  const int g = r / S, s = r % S;
  const int kvh = (j * Hkv) / Hq;
  const int pb = g * prefix_batch_stride;
  const KT* pkh = pk + ((size_t)pb * Hkv + kvh) * Pmax * D;
  const KT* pvh = pv + ((size_t)pb * Hkv + kvh) * Pmax * D;
  const float* skh = sk + ((size_t)g * Hkv + kvh) * S * D;
  const float* svh = sv + ((size_t)g * Hkv + kvh) * S * D;
  const int nk = P + S;
  const float scale = rsqrtf((float)D);
  for (int d = threadIdx.x; d < D; d += blockDim.x) qs[d] = q[((size_t)r * Hq + j) * D + d];
  __syncthreads();
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
  for (int n = warp; n < nk; n += nw) {
    float dot = 0.f;
    if (n < P) {
      for (int d = lane; d < D; d += 32) dot = fmaf(qs[d], to_f32(pkh[(size_t)n * D + d]), dot);
    } else {
      for (int d = lane; d < D; d += 32) dot = fmaf(qs[d], skh[(size_t)(n - P) * D + d], dot);
    }
    dot = warp_sum(dot);
    const bool visible = !(mask_mode == RTV_MASK_PI0_BLOCK && s == 0 && n > P);
    if (lane == 0) sc[n] = visible ? dot * scale : -INFINITY;
  }
  __syncthreads();
  float mx = -INFINITY;
  for (int n = threadIdx.x; n < nk; n += blockDim.x) mx = fmaxf(mx, sc[n]);
  mx = warp_max(mx);
  if (lane == 0) red[warp] = mx;
  __syncthreads();
  mx = red[0];
  for (int i = 1; i < nw; ++i) mx = fmaxf(mx, red[i]);
  __syncthreads();
  float tot = 0.f;
  for (int n = threadIdx.x; n < nk; n += blockDim.x) {
    const float p = expf(sc[n] - mx);
    sc[n] = p;
    tot += p;
  }
  tot = block_sum(tot, red);
  const float inv = 1.f / tot;
  for (int d = threadIdx.x; d < D; d += blockDim.x) {
    float acc = 0.f;
    for (int n = 0; n < P; ++n) acc = fmaf(sc[n], to_f32(pvh[(size_t)n * D + d]), acc);
    for (int n = 0; n < S; ++n) acc = fmaf(sc[P + n], svh[(size_t)n * D + d], acc);
    o[((size_t)r * Hq + j) * D + d] = acc * inv;
  }
}

// Gated MLP activation: m = gelu_tanh(gate) * up, gu = [T][gate F | up F].
__global__ void geglu_kernel(const float* __restrict__ gu, float* __restrict__ m, int T, int F) {
  for (size_t idx = (size_t)blockIdx.x * blockDim.x + threadIdx.x; idx < (size_t)T * F;
       idx += (size_t)gridDim.x * blockDim.x) {
    const size_t r = idx / F, i = idx % F;
    m[idx] = gelu_tanh(gu[r * 2 * F + i]) * gu[r * 2 * F + F + i];
  }
}

// ---------------------------------------------------------------------------
// Output head ("DM0.5 reading guide", sec. 5.2-5.3): v = action_out_proj(
// RMSNorm_f(h)) for the H action rows of every group, then either the Euler
// step x <- x - dt * v (x [G][H][A], in place) or v stored to vout.
// One block per action row.  A non-finite x sets RTV_DEV_NUMERIC.
// ---------------------------------------------------------------------------
template <typename WT>
__global__ void out_head_kernel(const float* __restrict__ h, const float* __restrict__ gain,
                                const WT* __restrict__ w_ao, const float* __restrict__ b_ao, float* __restrict__ x,
                                float* __restrict__ vout, float dt, int w, int S, int A, float eps,
                                unsigned* __restrict__ status) {
  extern __shared__ float hn[];
  __shared__ float red[32];
  const int H = S - 1;
  const int g = blockIdx.x / H, j = blockIdx.x % H;
  const float* row = h + ((size_t)g * S + 1 + j) * w;
  float ss = 0.f;
  for (int i = threadIdx.x; i < w; i += blockDim.x) {
    const float v = row[i];
    hn[i] = v;
    ss = fmaf(v, v, ss);
  }
  ss = block_sum(ss, red);
  const float inv = rsqrtf(ss / (float)w + eps);
  for (int i = threadIdx.x; i < w; i += blockDim.x) hn[i] = hn[i] * inv * (1.f + gain[i]);
  __syncthreads();
  // 8 threads per output: each takes w/8 consecutive inputs (loads issued together)
  const int sub = threadIdx.x & 7;
  const int per = w / 8;
  for (int a0 = threadIdx.x >> 3; a0 < ((A + 31) / 32) * 32; a0 += blockDim.x >> 3) {
    const int a = a0;
    float dot = 0.f;
    if (a < A) {
      const WT* wr = w_ao + (size_t)a * w + sub * per;
      const float* hr = hn + sub * per;
      for (int i0 = 0; i0 < per; i0 += 32) {
        float wv[32];
#pragma unroll
        for (int i = 0; i < 32; ++i) wv[i] = (i0 + i < per) ? to_f32(wr[i0 + i]) : 0.f;
#pragma unroll
        for (int i = 0; i < 32; ++i)
          if (i0 + i < per) dot = fmaf(wv[i], hr[i0 + i], dot);
      }
    }
    dot += __shfl_xor_sync(0xffffffffu, dot, 4);
    dot += __shfl_xor_sync(0xffffffffu, dot, 2);
    dot += __shfl_xor_sync(0xffffffffu, dot, 1);
    if (sub == 0 && a < A) {
      const float v = dot + b_ao[a];
      const size_t off = ((size_t)g * H + j) * A + a;
      if (vout) {
        vout[off] = v;
      } else {
        const float xn = x[off] - dt * v;
        x[off] = xn;
        if (!isfinite(xn)) atomicOr(status, RTV_DEV_NUMERIC);
      }
    }
  }
}

// ---------------------------------------------------------------------------
// FLASH verification ("Realtime-VLA FLASH", sec. 02): X_i = tau_i eps + (1 - tau_i) D.
// ---------------------------------------------------------------------------
__global__ void verify_interp_kernel(const float* __restrict__ draft, const float* __restrict__ eps,
                                     const float* __restrict__ taus, float* __restrict__ x, int T, int HA) {
  for (int idx = blockIdx.x * blockDim.x + threadIdx.x; idx < T * HA; idx += gridDim.x * blockDim.x) {
    const int i = idx / HA, e = idx % HA;
    const float tau = taus[i];
    x[idx] = tau * eps[e] + (1.f - tau) * draft[e];
  }
}

// FLASH decision ("Realtime-VLA FLASH", sec. 02, 03.2, 03.3): rebuild
// A_i = X_i - tau_i v_i, d_i[h] = ||A_i[h] - D[h]||_2, accepted length =
// longest prefix with d_i[h] < delta for every i, gripper-switch flags.
// One block; params = {delta (float bits), gripper_dim}.
__global__ void verify_decide_kernel(const float* __restrict__ x, const float* __restrict__ v,
                                     const float* __restrict__ draft, const float* __restrict__ taus,
                                     const float* __restrict__ params, int T, int H, int A,
                                     float* __restrict__ dist, int* __restrict__ accepted,
                                     unsigned* __restrict__ flags) {
  extern __shared__ int pass_sm[];   // H ints
  const float delta = params[0];
  const int gdim = (int)params[1];
  for (int h = threadIdx.x; h < H; h += blockDim.x) pass_sm[h] = 1;
  __syncthreads();
  for (int idx = threadIdx.x; idx < T * H; idx += blockDim.x) {
    const int i = idx / H, h = idx % H;
    const float tau = taus[i];
    float ss = 0.f;
    for (int a = 0; a < A; ++a) {
      const size_t off = ((size_t)i * H + h) * A + a;
      const float ahat = x[off] - tau * v[off];
      const float diff = ahat - draft[(size_t)h * A + a];
      ss = fmaf(diff, diff, ss);
    }
    const float d = sqrtf(ss);
    dist[idx] = d;
    if (!(d < delta)) atomicAnd(&pass_sm[h], 0);
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    int n_acc = 0;
    while (n_acc < H && pass_sm[n_acc]) ++n_acc;
    unsigned f = 0;
    if (n_acc == 0) f |= RTV_FLAG_ZERO_ACCEPT;
    for (int h = 1; h < H; ++h) {
      const bool a = draft[(size_t)h * A + gdim] > 0.f, b = draft[(size_t)(h - 1) * A + gdim] > 0.f;
      if (a != b) {
        f |= RTV_FLAG_SWITCH;
        if (h < n_acc) f |= RTV_FLAG_SWITCH_IN_PREFIX;
      }
    }
    *accepted = n_acc;
    *flags = f;
  }
}

// Prefix KV [L][2][B][P][Hkv][D] -> library layout [L][2][Bmax][Hkv][Pmax][D].
template <typename KT>
__global__ void prefix_pack_kernel(const KT* __restrict__ src, KT* __restrict__ dst, int L, int B, int P, int Hkv,
                                   int D, int Bmax, int Pmax) {
  const size_t total = (size_t)L * 2 * B * P * Hkv * D;
  for (size_t idx = (size_t)blockIdx.x * blockDim.x + threadIdx.x; idx < total;
       idx += (size_t)gridDim.x * blockDim.x) {
    size_t t = idx;
    const int d = t % D; t /= D;
    const int kh = t % Hkv; t /= Hkv;
    const int p = t % P; t /= P;
    const int b = t % B; t /= B;
    const int kv = t % 2; t /= 2;
    const int l = (int)t;
    dst[(((((size_t)l * 2 + kv) * Bmax + b) * Hkv + kh) * Pmax + p) * D + d] = src[idx];
  }
}

// ---------------------------------------------------------------------------
// host launchers
// ---------------------------------------------------------------------------
// ---------------------------------------------------------------------------
// Linear map of a few rows with a per-group bias, for the time-conditioning
// variants: y[t][n] = act(sum_k x[t][k] W[n][k] + bias[g][n]) (EPI_ADD adds
// into y) for the rows t < T whose position s = t % S lies in [s_lo, s_hi),
// g = t / S; W rows have stride ldw.  A CTA takes 8 outputs (a warp each)
// and 32 rows staged in shared memory 256 inputs at a time; a lane reads 8
// consecutive weights per step (K and ldw multiples of 8).
// ---------------------------------------------------------------------------
__device__ __forceinline__ void load8w(const float* p, float v[8]) {
  const float4 a = *reinterpret_cast<const float4*>(p);
  const float4 b = *reinterpret_cast<const float4*>(p + 4);
  v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
  v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
}
__device__ __forceinline__ void load8w(const __nv_bfloat16* p, float v[8]) {
  const uint4 q = *reinterpret_cast<const uint4*>(p);
  const __nv_bfloat162* h2 = reinterpret_cast<const __nv_bfloat162*>(&q);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float2 f = __bfloat1622float2(h2[i]);
    v[2 * i] = f.x;
    v[2 * i + 1] = f.y;
  }
}

template <typename WT, int EPI>
__global__ void __launch_bounds__(256) rows_linear_kernel(const float* __restrict__ x, int ldx,
                                                          const WT* __restrict__ W, int ldw,
                                                          const float* __restrict__ bias, int bias_gs,
                                                          float* __restrict__ y, int ldy, int T, int S, int s_lo,
                                                          int s_hi, int N, int K) {
  __shared__ float xs[32][260];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int n = blockIdx.x * 8 + warp;
  const int r0 = blockIdx.y * 32;
  float acc[32];
#pragma unroll
  for (int r = 0; r < 32; ++r) acc[r] = 0.f;
  for (int k0 = 0; k0 < K; k0 += 256) {
    const int kc = min(256, K - k0);
    __syncthreads();
    for (int i = threadIdx.x; i < 32 * 256; i += 256) {
      const int r = i >> 8, kk = i & 255;
      xs[r][kk] = (r0 + r < T && kk < kc) ? x[(size_t)(r0 + r) * ldx + k0 + kk] : 0.f;
    }
    __syncthreads();
    if (n < N && lane * 8 < kc) {
      float wv[8];
      load8w(W + (size_t)n * ldw + k0 + lane * 8, wv);
#pragma unroll
      for (int r = 0; r < 32; ++r) {
        float v = acc[r];
#pragma unroll
        for (int e = 0; e < 8; ++e) v = fmaf(xs[r][lane * 8 + e], wv[e], v);
        acc[r] = v;
      }
    }
  }
  if (n >= N) return;
#pragma unroll
  for (int r = 0; r < 32; ++r) {
    float v = warp_sum(acc[r]);
    const int t = r0 + r;
    if (lane == 0 && t < T) {
      const int g = t / S, sp = t - g * S;
      if (sp >= s_lo && sp < s_hi) {
        if (bias) v += bias[(size_t)g * bias_gs + n];
        float* yp = y + (size_t)t * ldy + n;
        if (EPI == EPI_ADD) *yp += v;
        else if (EPI == EPI_SWISH) *yp = swish(v);
        else *yp = v;
      }
    }
  }
}

// Modulated RMSNorm of the per-layer time modulator: u = h / rms(h) * (1 +
// scale[g]) + shift[g] for row t of group g = t / S.
__global__ void rmsnorm_mod_kernel(const float* __restrict__ h, const float* __restrict__ scale,
                                   const float* __restrict__ shift, int gs, float* __restrict__ u, int w, int S,
                                   float eps) {
  __shared__ float red[32];
  const int t = blockIdx.x, g = t / S;
  const float* row = h + (size_t)t * w;
  float ss = 0.f;
  for (int i = threadIdx.x; i < w; i += blockDim.x) ss = fmaf(row[i], row[i], ss);
  ss = block_sum(ss, red);
  const float inv = rsqrtf(ss / (float)w + eps);
  const float* sc = scale + (size_t)g * gs;
  const float* sh = shift + (size_t)g * gs;
  for (int i = threadIdx.x; i < w; i += blockDim.x) u[(size_t)t * w + i] = row[i] * inv * (1.f + sc[i]) + sh[i];
}

// Gated residual add: h[t] += gate[g] * b[t], g = t / S.
__global__ void gated_add_kernel(float* __restrict__ h, const float* __restrict__ b, const float* __restrict__ gate,
                                 int gs, int w, int S, int T) {
  const size_t n = (size_t)T * w;
  for (size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += (size_t)gridDim.x * blockDim.x) {
    const size_t t = i / w, k = i % w;
    h[i] += gate[(t / S) * (size_t)gs + k] * b[i];
  }
}

void launch_time_embedding(const float* taus, int n, int n_steps, float* e, int w, cudaStream_t st) {
  time_embedding_kernel<<<n, 128, 0, st>>>(taus, n_steps, e, w);
}

template <typename WT>
void launch_linear(const float* x, int ldx, const WT* W, const float* bias, float* y, int ldy, int M, int N, int K,
                   int epi, cudaStream_t st) {
  dim3 grid((N + 63) / 64, (M + 63) / 64);
  if (epi == EPI_ADD) linear_kernel<WT, EPI_ADD><<<grid, 256, 0, st>>>(x, ldx, W, bias, y, ldy, M, N, K);
  else if (epi == EPI_SWISH) linear_kernel<WT, EPI_SWISH><<<grid, 256, 0, st>>>(x, ldx, W, bias, y, ldy, M, N, K);
  else linear_kernel<WT, EPI_STORE><<<grid, 256, 0, st>>>(x, ldx, W, bias, y, ldy, M, N, K);
}
template void launch_linear<float>(const float*, int, const float*, const float*, float*, int, int, int, int, int,
                                   cudaStream_t);
template void launch_linear<__nv_bfloat16>(const float*, int, const __nv_bfloat16*, const float*, float*, int, int,
                                           int, int, int, cudaStream_t);

template <typename WT>
void launch_embed(const float* x, const float* state, int state_group_stride, const WT* w_sp, const float* b_sp,
                  const WT* w_ai, const float* b_ai, const float* c, int c_group_stride, float* h, int G, int w,
                  int S, int A, int Sd, cudaStream_t st) {
  const int threads = (w % 256 == 0) ? 256 : (w % 128 == 0 ? 128 : (w % 64 == 0 ? 64 : 32));
  embed_kernel<WT><<<G * S, threads, 0, st>>>(x, state, state_group_stride, w_sp, b_sp, w_ai, b_ai, c, c_group_stride,
                                              h, w, S, A, Sd);
}
template void launch_embed<float>(const float*, const float*, int, const float*, const float*, const float*,
                                  const float*, const float*, int, float*, int, int, int, int, int, cudaStream_t);
template void launch_embed<__nv_bfloat16>(const float*, const float*, int, const __nv_bfloat16*, const float*,
                                          const __nv_bfloat16*, const float*, const float*, int, float*, int, int,
                                          int, int, int, cudaStream_t);

void launch_rmsnorm(const float* h, const float* gain, float* u, int rows, int w, float eps, cudaStream_t st) {
  rmsnorm_kernel<<<rows, 256, 0, st>>>(h, gain, u, w, eps);
}

void launch_rope_table(float* cs, float* sn, int S, int D, int P, float theta, cudaStream_t st) {
  const int n = S * (D / 2);
  rope_table_kernel<<<(n + 255) / 256, 256, 0, st>>>(cs, sn, S, D, P, theta);
}

void launch_rope_split(const float* qkv, const float* cs, const float* sn, float* q, float* ks, float* vs, int T,
                       int S, int Hq, int Hkv, int D, cudaStream_t st) {
  rope_split_kernel<<<T, 128, 0, st>>>(qkv, cs, sn, q, ks, vs, S, Hq, Hkv, D);
}

template <typename KT>
void launch_attention_simt(const float* q, const KT* pk, const KT* pv, const float* sk, const float* sv, float* o,
                           int T, int S, int P, int Pmax, int Hq, int Hkv, int D, int prefix_batch_stride,
                           int mask_mode, cudaStream_t st) {
  const size_t smem = (size_t)(D + P + S) * sizeof(float);
  attention_simt_kernel<KT><<<dim3(T, Hq), 128, smem, st>>>(q, pk, pv, sk, sv, o, S, P, Pmax, Hq, Hkv, D,
                                                            prefix_batch_stride, mask_mode);
}
template void launch_attention_simt<float>(const float*, const float*, const float*, const float*, const float*,
                                           float*, int, int, int, int, int, int, int, int, int, cudaStream_t);
template void launch_attention_simt<__nv_bfloat16>(const float*, const __nv_bfloat16*, const __nv_bfloat16*,
                                                   const float*, const float*, float*, int, int, int, int, int, int,
                                                   int, int, int, cudaStream_t);

void launch_geglu(const float* gu, float* m, int T, int F, cudaStream_t st) {
  const size_t n = (size_t)T * F;
  const int blocks = (int)((n + 255) / 256 < 4096 ? (n + 255) / 256 : 4096);
  geglu_kernel<<<blocks, 256, 0, st>>>(gu, m, T, F);
}

template <typename WT>
void launch_out_head(const float* h, const float* gain, const WT* w_ao, const float* b_ao, float* x, float* vout,
                     float dt, int G, int w, int S, int A, float eps, unsigned* status, cudaStream_t st) {
  out_head_kernel<WT><<<G * (S - 1), 256, (size_t)w * sizeof(float), st>>>(h, gain, w_ao, b_ao, x, vout, dt, w, S,
                                                                          A, eps, status);
}
template void launch_out_head<float>(const float*, const float*, const float*, const float*, float*, float*, float,
                                     int, int, int, int, float, unsigned*, cudaStream_t);
template void launch_out_head<__nv_bfloat16>(const float*, const float*, const __nv_bfloat16*, const float*, float*,
                                             float*, float, int, int, int, int, float, unsigned*, cudaStream_t);

void launch_verify_interp(const float* draft, const float* eps, const float* taus, float* x, int T, int HA,
                          cudaStream_t st) {
  verify_interp_kernel<<<(T * HA + 255) / 256, 256, 0, st>>>(draft, eps, taus, x, T, HA);
}

void launch_verify_decide(const float* x, const float* v, const float* draft, const float* taus,
                          const float* params, int T, int H, int A, float* dist, int* accepted, unsigned* flags,
                          cudaStream_t st) {
  verify_decide_kernel<<<1, 256, (size_t)H * sizeof(int), st>>>(x, v, draft, taus, params, T, H, A, dist, accepted,
                                                                flags);
}

template <typename KT>
void launch_prefix_pack(const KT* src, KT* dst, int L, int B, int P, int Hkv, int D, int Bmax, int Pmax,
                        cudaStream_t st) {
  const size_t n = (size_t)L * 2 * B * P * Hkv * D;
  const int blocks = (int)((n + 255) / 256 < 8192 ? (n + 255) / 256 : 8192);
  prefix_pack_kernel<KT><<<blocks, 256, 0, st>>>(src, dst, L, B, P, Hkv, D, Bmax, Pmax);
}
template void launch_prefix_pack<float>(const float*, float*, int, int, int, int, int, int, int, cudaStream_t);
template void launch_prefix_pack<__nv_bfloat16>(const __nv_bfloat16*, __nv_bfloat16*, int, int, int, int, int, int,
                                                int, cudaStream_t);

template <typename WT>
void launch_rows_linear(const float* x, int ldx, const WT* W, int ldw, const float* bias, int bias_gs, float* y,
                        int ldy, int T, int S, int s_lo, int s_hi, int N, int K, int epi, cudaStream_t st) {
  dim3 grid((N + 7) / 8, (T + 31) / 32);
  if (epi == EPI_ADD)
    rows_linear_kernel<WT, EPI_ADD><<<grid, 256, 0, st>>>(x, ldx, W, ldw, bias, bias_gs, y, ldy, T, S, s_lo, s_hi,
                                                          N, K);
  else if (epi == EPI_SWISH)
    rows_linear_kernel<WT, EPI_SWISH><<<grid, 256, 0, st>>>(x, ldx, W, ldw, bias, bias_gs, y, ldy, T, S, s_lo,
                                                            s_hi, N, K);
  else
    rows_linear_kernel<WT, EPI_STORE><<<grid, 256, 0, st>>>(x, ldx, W, ldw, bias, bias_gs, y, ldy, T, S, s_lo,
                                                            s_hi, N, K);
}
template void launch_rows_linear<float>(const float*, int, const float*, int, const float*, int, float*, int, int,
                                        int, int, int, int, int, int, cudaStream_t);
template void launch_rows_linear<__nv_bfloat16>(const float*, int, const __nv_bfloat16*, int, const float*, int,
                                                float*, int, int, int, int, int, int, int, int, cudaStream_t);

void launch_rmsnorm_mod(const float* h, const float* scale, const float* shift, int gs, float* u, int rows, int w,
                        int S, float eps, cudaStream_t st) {
  rmsnorm_mod_kernel<<<rows, 256, 0, st>>>(h, scale, shift, gs, u, w, S, eps);
}

void launch_gated_add(float* h, const float* b, const float* gate, int gs, int w, int S, int T, cudaStream_t st) {
  const size_t n = (size_t)T * w;
  const int blocks = (int)std::min<size_t>((n + 255) / 256, 4096);
  gated_add_kernel<<<blocks, 256, 0, st>>>(h, b, gate, gs, w, S, T);
}

}  // namespace rtv
