// Tensor-core path of the bf16 action expert on sm_100a.
//
// Per layer, five kernels chained with programmatic dependent launch (PDL):
//   QKV   RMSNorm -> q/k/v projection -> RoPE, written as bf16 q and suffix K/V
//   ATTN  split-KV grouped-query attention over [prefix KV ; suffix KV]
//   O     attention output projection, added to the fp32 residual
//   GU    RMSNorm -> gate/up projection -> gelu_tanh(gate) * up (bf16)
//   DOWN  down projection, added to the fp32 residual
// ("DM0.5 reading guide", sec. 5.2 action expert; sec. 6.4 fused suffix
// kernels: normalise/modulate -> GEMM -> activation -> write back.)
//
// The projections are weight-streaming GEMMs at M = tokens (51 per suffix):
// out[t][n] = sum_k act[t][k] W[n][k].  They are computed swapped, D = W x act^T,
// so that 128 weight rows fill the tcgen05 M dimension and the tokens (padded
// to a multiple of 16) form N.  Each CTA owns one 128-row weight tile and one
// K slice: its weight bytes are fetched by TMA (128-byte swizzle) as soon as
// the CTA starts -- before it waits on the previous kernel, since weights do
// not depend on it -- while the activation slice is staged by the CTA itself
// (fusing the RMSNorm gain and the bf16 cast).  The K slices of one tile form
// a thread-block cluster; partial accumulators are reduced deterministically
// through distributed shared memory, and the epilogue applies the deferred
// RMSNorm scale 1/rms(h) (a per-token factor that commutes with the product),
// RoPE, GeGLU or the residual add.
#include <cudaTypedefs.h>

#include <math.h>
#include <stdio.h>
#include <stdlib.h>
#include <string.h>

#include <string>

#include <algorithm>
#include <vector>

#include "common.cuh"
#include "fastpath.h"
#include "kernels.h"
#include "runtime.h"
#include "tc_ptx.cuh"

namespace rtv {

enum { GM_QKV = 0, GM_O = 1, GM_GU = 2, GM_DOWN = 3 };

struct GemmArgs {
  const float* h;             // fp32 residual stream [T][w]
  float* h_out;               // residual updated in place (O, DOWN)
  const float* gain;          // RMSNorm gain g [w]: staged activation = h * (1 + g)   (QKV, GU)
  const __nv_bfloat16* act;   // bf16 activation [T][K]                                (O, DOWN)
  __nv_bfloat16* q;           // [T][Hq][D]
  __nv_bfloat16* ks;          // suffix keys   [G][Hkv][S][D]
  __nv_bfloat16* vs;          // suffix values [G][Hkv][S][D]
  const float* rope_cs;       // [S][D/2]
  const float* rope_sn;
  __nv_bfloat16* m;           // [T][F]
  unsigned* status;
  long long timeout_ns;
  int T, n_mma, K, kslice, stages, w, S, Hq, Hkv, D, F, w_row0;
  float eps;
};

struct GemmSmem {
  int stages, stage_bytes, ring_bytes, red_off, ss_off, bar_off, total;
};

// Shared memory of one GEMM CTA: a ring of `stages` stages, each one 128x64
// weight box (16 KB) plus the matching 64-wide activation box of n_mma token
// rows; the fp32 partial tile [n_mma][128] overlays the ring once the MMAs
// are done (or follows it when larger); then per-token sums of squares and
// the mbarriers.
__host__ __device__ inline GemmSmem gemm_smem_layout(int stages, int n_mma) {
  GemmSmem s;
  s.stages = stages;
  s.stage_bytes = 16384 + n_mma * 128;
  s.ring_bytes = stages * s.stage_bytes;
  const int red_bytes = n_mma * 128 * 4;
  s.red_off = red_bytes <= s.ring_bytes ? 0 : s.ring_bytes;
  const int end_red = s.red_off + red_bytes;
  s.ss_off = s.ring_bytes > end_red ? s.ring_bytes : end_red;
  s.bar_off = s.ss_off + n_mma * 4;
  s.total = s.bar_off + (2 * stages + 1) * 8 + 16 + 1024;   // barriers, TMEM slot, alignment slack
  return s;
}

__host__ __device__ inline int tmem_cols_for(int n) {
  int c = 32;
  while (c < n) c <<= 1;
  return c;
}

__device__ __forceinline__ uint32_t dynamic_smem_size() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%dynamic_smem_size;" : "=r"(r));
  return r;
}

template <int MODE>
__global__ void __launch_bounds__(192, 1) gemm_tc_kernel(const __grid_constant__ CUtensorMap wmap, const GemmArgs a) {
  extern __shared__ uint8_t smem_raw[];
  const int n_mma = a.n_mma;
  const GemmSmem L = gemm_smem_layout(a.stages, n_mma);
  // every CTA of the grid sees the same size, so a refusal is uniform across each cluster
  if (dynamic_smem_size() < (uint32_t)L.total || a.kslice < 64 || (a.kslice & 63) || a.stages < 1 || n_mma > 256) {
    if (threadIdx.x == 0) atomicOr(a.status, RTV_DEV_BOUNDS);
    return;
  }
  uint8_t* base = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = ptx::cluster_ctarank();
  const int cs = gridDim.x;
  const int nt = blockIdx.y;
  const int nbox = a.kslice >> 6;
  const int NS = L.stages;
  const int k0 = (int)rank * a.kslice;
  float* red = (float*)(base + L.red_off);
  float* ss = (float*)(base + L.ss_off);
  uint64_t* full = (uint64_t*)(base + L.bar_off);   // weights landed + activations staged
  uint64_t* empty = full + NS;                      // MMAs of the stage completed
  uint64_t* done = empty + NS;                      // all MMAs completed
  uint32_t* tmem_slot = (uint32_t*)(done + 1);
  const uint32_t ncols = (uint32_t)tmem_cols_for(n_mma);

  if (threadIdx.x == 0) {
    for (int i = 0; i < NS; ++i) {
      ptx::mbar_init(&full[i], 2);
      ptx::mbar_init(&empty[i], 1);
    }
    ptx::mbar_init(done, 1);
    ptx::fence_mbar_init();
  }
  __syncthreads();
  ptx::pdl_launch_dependents();

  // Weights do not depend on the previous kernel: the first ring-full of
  // weight boxes is requested before anyone waits on that kernel.
  const int first = nbox < NS ? nbox : NS;
  uint64_t pol = 0;
  if (warp == 0 && lane == 0) {
    pol = ptx::policy_evict_first();
    for (int b = 0; b < first; ++b) {
      ptx::mbar_expect_tx(&full[b], 16384u);
      ptx::tma_load_2d(base + b * L.stage_bytes, &wmap, &full[b], k0 + 64 * b, a.w_row0 + nt * 128, pol);
    }
  } else if (warp == 1) {
    ptx::pdl_wait();
    ptx::tmem_alloc(tmem_slot, ncols);
    ptx::tmem_relinquish();
    ptx::tc_fence_before();
  }
  __syncthreads();   // TMEM address published; nothing above waits on another role
  ptx::tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    // ---- weight producer: remaining boxes as ring stages free up ----
    if (lane == 0) {
      for (int b = first; b < nbox; ++b) {
        const int s = b % NS, u = b / NS;
        if (!ptx::mbar_wait(&empty[s], (u - 1) & 1, a.timeout_ns)) atomicOr(a.status, RTV_DEV_TIMEOUT);
        ptx::mbar_expect_tx(&full[s], 16384u);
        ptx::tma_load_2d(base + s * L.stage_bytes, &wmap, &full[s], k0 + 64 * b, a.w_row0 + nt * 128, pol);
      }
    }
  } else if (warp == 1) {
    // ---- MMA issue: one thread ----
    if (lane == 0) {
      const uint32_t idesc = ptx::idesc_bf16_f32(128, n_mma);
      for (int b = 0; b < nbox; ++b) {
        const int s = b % NS, u = b / NS;
        if (!ptx::mbar_wait(&full[s], u & 1, a.timeout_ns)) atomicOr(a.status, RTV_DEV_TIMEOUT);
        ptx::tc_fence_after();
        const uint32_t wa = ptx::smem_u32(base + s * L.stage_bytes);
        const uint32_t aa = wa + 16384;
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) {
          const uint64_t ad = ptx::sw128_kmajor_desc(wa + kk * 32);
          const uint64_t bd = ptx::sw128_kmajor_desc(aa + kk * 32);
          ptx::umma_bf16(tmem, ad, bd, idesc, (b | kk) != 0 ? 1u : 0u);
        }
        ptx::umma_commit(&empty[s]);
      }
      ptx::umma_commit(done);
    }
  } else if (warp >= 2) {
    // ---- activation staging into the ring (K-major, 128-byte swizzle) ----
    ptx::pdl_wait();
    const int tid = threadIdx.x - 64;
    const int iters = n_mma >> 4;           // n_mma * 8 chunks per box / 128 threads
    float ss_acc[16];
#pragma unroll
    for (int i = 0; i < 16; ++i) ss_acc[i] = 0.f;
    for (int b = 0; b < nbox; ++b) {
      const int s = b % NS, u = b / NS;
      if (u > 0 && !ptx::mbar_wait(&empty[s], (u - 1) & 1, a.timeout_ns)) atomicOr(a.status, RTV_DEV_TIMEOUT);
      uint8_t* abox = base + s * L.stage_bytes + 16384;
#pragma unroll
      for (int it = 0; it < 16; ++it) {
        if (it >= iters) break;
        const int c = tid + it * 128;
        const int t = c >> 3, kc = c & 7;
        const int k = k0 + b * 64 + kc * 8;
        uint4 packed;
        if (MODE == GM_QKV || MODE == GM_GU) {
          float x[8];
          if (t < a.T) {
            const float4* hp = reinterpret_cast<const float4*>(a.h + (size_t)t * a.w + k);
            const float4 h0 = hp[0], h1 = hp[1];
            x[0] = h0.x; x[1] = h0.y; x[2] = h0.z; x[3] = h0.w; x[4] = h1.x; x[5] = h1.y; x[6] = h1.z; x[7] = h1.w;
          } else {
#pragma unroll
            for (int i = 0; i < 8; ++i) x[i] = 0.f;
          }
          const float4* gp = reinterpret_cast<const float4*>(a.gain + k);
          const float4 g0 = gp[0], g1 = gp[1];
          float ssp = 0.f;
#pragma unroll
          for (int i = 0; i < 8; ++i) ssp = fmaf(x[i], x[i], ssp);
          ss_acc[it] += ssp;
          packed.x = ptx::pack_bf16x2(x[0] * (1.f + g0.x), x[1] * (1.f + g0.y));
          packed.y = ptx::pack_bf16x2(x[2] * (1.f + g0.z), x[3] * (1.f + g0.w));
          packed.z = ptx::pack_bf16x2(x[4] * (1.f + g1.x), x[5] * (1.f + g1.y));
          packed.w = ptx::pack_bf16x2(x[6] * (1.f + g1.z), x[7] * (1.f + g1.w));
        } else {
          if (t < a.T) packed = *reinterpret_cast<const uint4*>(a.act + (size_t)t * a.K + k);
          else packed = make_uint4(0u, 0u, 0u, 0u);
        }
        *reinterpret_cast<uint4*>(abox + t * 128 + ((kc ^ (t & 7)) << 4)) = packed;
      }
      ptx::fence_proxy_async_smem();
      asm volatile("bar.sync 1, 128;" ::: "memory");
      if (tid == 0) {
        asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(ptx::smem_u32(&full[s])) : "memory");
      }
    }
    if (MODE == GM_QKV || MODE == GM_GU) {
      // per-token sum of squares of the raw residual over this K slice: the 8
      // lanes of a token row reduce in a fixed order
#pragma unroll
      for (int it = 0; it < 16; ++it) {
        if (it >= iters) break;
        float v = ss_acc[it];
        v += __shfl_xor_sync(0xffffffffu, v, 4);
        v += __shfl_xor_sync(0xffffffffu, v, 2);
        v += __shfl_xor_sync(0xffffffffu, v, 1);
        const int c = tid + it * 128;
        if ((c & 7) == 0) ss[c >> 3] = v;
      }
    }
    // ---- accumulator -> shared (feature-contiguous per token) ----
    if (!ptx::mbar_wait(done, 0, a.timeout_ns)) atomicOr(a.status, RTV_DEV_TIMEOUT);
    ptx::tc_fence_after();
    const int quarter = warp & 3;
    const int f = quarter * 32 + lane;
    for (int c = 0; c < n_mma; c += 16) {
      float v[16];
      ptx::tmem_ld_16(tmem + ((uint32_t)(quarter * 32) << 16) + (uint32_t)c, v);
#pragma unroll
      for (int i = 0; i < 16; ++i) red[(c + i) * 128 + f] = v[i];
    }
  }
  ptx::tc_fence_before();
  ptx::cluster_sync();

  // ---- cluster reduction over K slices + epilogue; rank r owns a token range ----
  if (warp >= 2) {
    const int tid = threadIdx.x - 64;
    const int p = tid & 63, half = tid >> 6;
    const int per = (a.T + cs - 1) / cs;
    const int t0 = (int)rank * per;
    const int t1 = min(a.T, t0 + per);
    uint32_t red_r[16], ss_r[16];
    const uint32_t red_a = ptx::smem_u32(red), ss_a = ptx::smem_u32(ss);
    for (int qr = 0; qr < cs; ++qr) {
      red_r[qr] = ptx::mapa(red_a, (uint32_t)qr);
      ss_r[qr] = ptx::mapa(ss_a, (uint32_t)qr);
    }
    for (int t = t0 + half; t < t1; t += 2) {
      float x1 = 0.f, x2 = 0.f, sst = 0.f;
      for (int qr = 0; qr < cs; ++qr) {
        x1 += ptx::ld_dsmem_f32(red_r[qr] + (uint32_t)((t * 128 + p) * 4));
        x2 += ptx::ld_dsmem_f32(red_r[qr] + (uint32_t)((t * 128 + p + 64) * 4));
        if (MODE == GM_QKV || MODE == GM_GU) sst += ptx::ld_dsmem_f32(ss_r[qr] + (uint32_t)(t * 4));
      }
      if (MODE == GM_O || MODE == GM_DOWN) {
        float* hr = a.h_out + (size_t)t * a.w + nt * 128;
        hr[p] += x1;
        hr[p + 64] += x2;
      } else {
        const float rs = rsqrtf(sst / (float)a.w + a.eps);
        x1 *= rs;
        x2 *= rs;
        if (MODE == GM_GU) {
          a.m[(size_t)t * a.F + nt * 64 + p] = __float2bfloat16_rn(gelu_tanh(x1) * x2);
        } else {
          const int tph = a.D >> 7;
          const int hh = nt / tph, bq = nt - hh * tph;
          const int d = 64 * bq + p, hd = a.D >> 1;
          const int g = t / a.S, s = t - g * a.S;
          float y1 = x1, y2 = x2;
          if (hh < a.Hq + a.Hkv) {
            const float c = a.rope_cs[s * hd + d], sn = a.rope_sn[s * hd + d];
            y1 = x1 * c - x2 * sn;
            y2 = x2 * c + x1 * sn;
          }
          __nv_bfloat16* dst;
          if (hh < a.Hq) dst = a.q + ((size_t)t * a.Hq + hh) * a.D;
          else if (hh < a.Hq + a.Hkv) dst = a.ks + (((size_t)g * a.Hkv + (hh - a.Hq)) * a.S + s) * a.D;
          else dst = a.vs + (((size_t)g * a.Hkv + (hh - a.Hq - a.Hkv)) * a.S + s) * a.D;
          dst[d] = __float2bfloat16_rn(y1);
          dst[d + hd] = __float2bfloat16_rn(y2);
        }
      }
    }
  }
  ptx::tc_fence_before();
  ptx::cluster_sync();   // no CTA leaves while its shared memory may still be read
  if (warp == 1) {
    ptx::tc_fence_after();
    ptx::tmem_dealloc(tmem, ncols);
  }
  // never leave with a weight copy still landing in this CTA's shared memory
  if (warp == 0 && lane == 0) {
    for (int s2 = 0; s2 < first; ++s2) ptx::mbar_wait(&full[s2], ((nbox - 1 - s2) / NS) & 1, a.timeout_ns);
  }
}

// ---------------------------------------------------------------------------
// Split-KV grouped-query attention for one (query head, suffix) per cluster:
// the cluster's CTAs take consecutive key ranges of [prefix ; own suffix],
// run a flash-style online softmax with warp-level bf16 MMAs (fp32
// accumulate), and combine their (max, sum, output) through distributed
// shared memory ("DM0.5 reading guide", sec. 5.1-5.2; reading: bidirectional
// suffix, optional Pi0 block mask for the state token).
// ---------------------------------------------------------------------------
struct AttnArgs {
  const __nv_bfloat16* q;    // [T][Hq][D]
  const __nv_bfloat16* pk;   // this layer's prefix keys   [Bmax][Hkv][Pmax][D]
  const __nv_bfloat16* pv;   // this layer's prefix values
  const __nv_bfloat16* sk;   // suffix keys   [G][Hkv][S][D]
  const __nv_bfloat16* sv;
  __nv_bfloat16* o;          // [T][Hq*D]
  unsigned* status;
  int S, P, Pmax, Hq, Hkv, pbs, mask_mode, kpc;
  float scale_log2;
};

template <int D>
__global__ void __launch_bounds__(128) attn_mma_kernel(const AttnArgs a) {
  extern __shared__ __align__(128) uint8_t sm_attn[];
  __nv_bfloat16* Qs = reinterpret_cast<__nv_bfloat16*>(sm_attn);
  __nv_bfloat16* Ks = Qs + 64 * D;
  __nv_bfloat16* Vs = Ks + 64 * D;
  float* ml = reinterpret_cast<float*>(Vs + 64 * D);   // [64][2]
  constexpr int CPR = D / 8;
  if (dynamic_smem_size() < (uint32_t)(3 * 64 * D * 2 + 64 * 2 * 4) || a.S > 64 || gridDim.x > 16) {
    if (threadIdx.x == 0) atomicOr(a.status, RTV_DEV_BOUNDS);
    return;
  }
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int rank = (int)ptx::cluster_ctarank(), nchunk = gridDim.x;
  const int j = blockIdx.y, g = blockIdx.z;
  const int kvh = (j * a.Hkv) / a.Hq;
  const int pb = g * a.pbs;
  const int nk = a.P + a.S;
  const int kb = rank * a.kpc;
  const int ke = min(nk, kb + a.kpc);
  const __nv_bfloat16* pkh = a.pk + ((size_t)pb * a.Hkv + kvh) * a.Pmax * D;
  const __nv_bfloat16* pvh = a.pv + ((size_t)pb * a.Hkv + kvh) * a.Pmax * D;
  const __nv_bfloat16* skh = a.sk + ((size_t)g * a.Hkv + kvh) * a.S * D;
  const __nv_bfloat16* svh = a.sv + ((size_t)g * a.Hkv + kvh) * a.S * D;

  ptx::pdl_launch_dependents();
  ptx::pdl_wait();

  const uint32_t qs_a = ptx::smem_u32(Qs), ks_a = ptx::smem_u32(Ks), vs_a = ptx::smem_u32(Vs);
  for (int c = tid; c < 64 * CPR; c += 128) {
    const int r = c / CPR, ch = c - r * CPR;
    const uint32_t dst = qs_a + (uint32_t)((r * D + ((ch ^ (r & 7)) << 3)) * 2);
    if (r < a.S) ptx::cp_async_16(dst, a.q + (((size_t)g * a.S + r) * a.Hq + j) * D + ch * 8);
    else *reinterpret_cast<uint4*>(reinterpret_cast<uint8_t*>(Qs) + (dst - qs_a)) = make_uint4(0, 0, 0, 0);
  }

  float o_acc[D / 8][4];
#pragma unroll
  for (int i = 0; i < D / 8; ++i) o_acc[i][0] = o_acc[i][1] = o_acc[i][2] = o_acc[i][3] = 0.f;
  float m_r[2] = {-INFINITY, -INFINITY}, l_r[2] = {0.f, 0.f};
  const int row0 = 16 * warp + (lane >> 2);

  for (int kt = kb; kt < ke; kt += 64) {
    __syncthreads();
    for (int c = tid; c < 64 * CPR; c += 128) {
      const int r = c / CPR, ch = c - r * CPR;
      const int n = kt + r;
      const uint32_t off = (uint32_t)((r * D + ((ch ^ (r & 7)) << 3)) * 2);
      if (n < ke) {
        const __nv_bfloat16* ksrc = n < a.P ? pkh + (size_t)n * D : skh + (size_t)(n - a.P) * D;
        const __nv_bfloat16* vsrc = n < a.P ? pvh + (size_t)n * D : svh + (size_t)(n - a.P) * D;
        ptx::cp_async_16(ks_a + off, ksrc + ch * 8);
        ptx::cp_async_16(vs_a + off, vsrc + ch * 8);
      } else {
        *reinterpret_cast<uint4*>(reinterpret_cast<uint8_t*>(Ks) + off) = make_uint4(0, 0, 0, 0);
        *reinterpret_cast<uint4*>(reinterpret_cast<uint8_t*>(Vs) + off) = make_uint4(0, 0, 0, 0);
      }
    }
    ptx::cp_async_wait_all();
    __syncthreads();

    // scores S = Q K^T for this warp's 16 rows x 64 keys
    float s_acc[8][4];
#pragma unroll
    for (int i = 0; i < 8; ++i) s_acc[i][0] = s_acc[i][1] = s_acc[i][2] = s_acc[i][3] = 0.f;
#pragma unroll 4
    for (int kk = 0; kk < D / 16; ++kk) {
      uint32_t af[4];
      {
        const int r = 16 * warp + (lane & 15), ch = 2 * kk + (lane >> 4);
        ptx::ldmatrix_x4(af, qs_a + (uint32_t)((r * D + ((ch ^ (r & 7)) << 3)) * 2));
      }
#pragma unroll
      for (int np = 0; np < 4; ++np) {
        uint32_t bf[4];
        const int r = 16 * np + (lane & 7) + ((lane >> 4) << 3), ch = 2 * kk + ((lane >> 3) & 1);
        ptx::ldmatrix_x4(bf, ks_a + (uint32_t)((r * D + ((ch ^ (r & 7)) << 3)) * 2));
        ptx::mma_bf16_16816(s_acc[2 * np], af, bf[0], bf[1]);
        ptx::mma_bf16_16816(s_acc[2 * np + 1], af, bf[2], bf[3]);
      }
    }
    // mask, scale, online softmax (base-2 exponent)
    float tmax[2] = {-INFINITY, -INFINITY};
#pragma unroll
    for (int nt = 0; nt < 8; ++nt) {
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int key = kt + 8 * nt + 2 * (lane & 3) + (e & 1);
        const int r = row0 + ((e >> 1) << 3);
        const bool ok = key < ke && !(a.mask_mode == RTV_MASK_PI0_BLOCK && r == 0 && key > a.P);
        const float sv = ok ? s_acc[nt][e] * a.scale_log2 : -INFINITY;
        s_acc[nt][e] = sv;
        tmax[e >> 1] = fmaxf(tmax[e >> 1], sv);
      }
    }
    float corr[2], mnew[2];
#pragma unroll
    for (int i = 0; i < 2; ++i) {
      tmax[i] = fmaxf(tmax[i], __shfl_xor_sync(0xffffffffu, tmax[i], 1));
      tmax[i] = fmaxf(tmax[i], __shfl_xor_sync(0xffffffffu, tmax[i], 2));
      mnew[i] = fmaxf(m_r[i], tmax[i]);
      corr[i] = (m_r[i] == -INFINITY) ? (mnew[i] == -INFINITY ? 1.f : 0.f) : exp2f(m_r[i] - mnew[i]);
      m_r[i] = mnew[i];
      l_r[i] *= corr[i];
    }
#pragma unroll
    for (int nt = 0; nt < 8; ++nt) {
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float mi = mnew[e >> 1];
        const float pv = (s_acc[nt][e] == -INFINITY) ? 0.f : exp2f(s_acc[nt][e] - mi);
        s_acc[nt][e] = pv;
        l_r[e >> 1] += pv;
      }
    }
#pragma unroll
    for (int i = 0; i < D / 8; ++i) {
      o_acc[i][0] *= corr[0];
      o_acc[i][1] *= corr[0];
      o_acc[i][2] *= corr[1];
      o_acc[i][3] *= corr[1];
    }
    // O += P V
#pragma unroll
    for (int kb2 = 0; kb2 < 4; ++kb2) {
      uint32_t pf[4];
      pf[0] = ptx::pack_bf16x2(s_acc[2 * kb2][0], s_acc[2 * kb2][1]);
      pf[1] = ptx::pack_bf16x2(s_acc[2 * kb2][2], s_acc[2 * kb2][3]);
      pf[2] = ptx::pack_bf16x2(s_acc[2 * kb2 + 1][0], s_acc[2 * kb2 + 1][1]);
      pf[3] = ptx::pack_bf16x2(s_acc[2 * kb2 + 1][2], s_acc[2 * kb2 + 1][3]);
#pragma unroll
      for (int dn = 0; dn < D / 16; ++dn) {
        uint32_t bf[4];
        const int r = 16 * kb2 + (lane & 7) + (((lane >> 3) & 1) << 3), ch = 2 * dn + (lane >> 4);
        ptx::ldmatrix_x4_trans(bf, vs_a + (uint32_t)((r * D + ((ch ^ (r & 7)) << 3)) * 2));
        ptx::mma_bf16_16816(o_acc[2 * dn], pf, bf[0], bf[1]);
        ptx::mma_bf16_16816(o_acc[2 * dn + 1], pf, bf[2], bf[3]);
      }
    }
  }
  ptx::cp_async_wait_all();
#pragma unroll
  for (int i = 0; i < 2; ++i) {
    l_r[i] += __shfl_xor_sync(0xffffffffu, l_r[i], 1);
    l_r[i] += __shfl_xor_sync(0xffffffffu, l_r[i], 2);
  }
  __syncthreads();
  // unnormalised partial output (fp32) over the K/V tiles, then (max, sum)
  float* ob = reinterpret_cast<float*>(Ks);   // [64][D] fp32 = 2 * 64 * D * 2 bytes
#pragma unroll
  for (int nt = 0; nt < D / 8; ++nt) {
    const int d = 8 * nt + 2 * (lane & 3);
    *reinterpret_cast<float2*>(ob + row0 * D + d) = make_float2(o_acc[nt][0], o_acc[nt][1]);
    *reinterpret_cast<float2*>(ob + (row0 + 8) * D + d) = make_float2(o_acc[nt][2], o_acc[nt][3]);
  }
  if ((lane & 3) == 0) {
    ml[row0 * 2] = m_r[0];
    ml[row0 * 2 + 1] = l_r[0];
    ml[(row0 + 8) * 2] = m_r[1];
    ml[(row0 + 8) * 2 + 1] = l_r[1];
  }
  ptx::cluster_sync();
  {
    const int rpc = (a.S + nchunk - 1) / nchunk;
    const int r0 = rank * rpc, r1 = min(a.S, r0 + rpc);
    const uint32_t ob_a = ptx::smem_u32(ob), ml_a = ptx::smem_u32(ml);
    for (int r = r0; r < r1; ++r) {
      float mq[16], lq[16];
      float mx = -INFINITY;
      for (int qr = 0; qr < nchunk; ++qr) {
        const float2 v = ptx::ld_dsmem_f32x2(ptx::mapa(ml_a, (uint32_t)qr) + (uint32_t)(r * 8));
        mq[qr] = v.x;
        lq[qr] = v.y;
        mx = fmaxf(mx, v.x);
      }
      float lsum = 0.f;
      for (int qr = 0; qr < nchunk; ++qr) {
        mq[qr] = (mq[qr] == -INFINITY) ? 0.f : exp2f(mq[qr] - mx);
        lsum += mq[qr] * lq[qr];
      }
      const float inv = 1.f / lsum;
      for (int d2 = tid; d2 < D / 2; d2 += 128) {
        float ox = 0.f, oy = 0.f;
        for (int qr = 0; qr < nchunk; ++qr) {
          const float2 v = ptx::ld_dsmem_f32x2(ptx::mapa(ob_a, (uint32_t)qr) + (uint32_t)((r * D + 2 * d2) * 4));
          ox = fmaf(mq[qr], v.x, ox);
          oy = fmaf(mq[qr], v.y, oy);
        }
        *reinterpret_cast<uint32_t*>(a.o + (((size_t)g * a.S + r) * a.Hq + j) * D + 2 * d2) =
            ptx::pack_bf16x2(ox * inv, oy * inv);
      }
    }
  }
  ptx::cluster_sync();
}

// ---------------------------------------------------------------------------
// Weight packing: gather rows of a [rows][K] bf16 matrix into a new order.
// ---------------------------------------------------------------------------
__global__ void gather_rows_kernel(const __nv_bfloat16* __restrict__ src, __nv_bfloat16* __restrict__ dst,
                                   const int* __restrict__ idx, int rows, int K) {
  const int r = blockIdx.x;
  if (r >= rows) return;
  const uint4* s = reinterpret_cast<const uint4*>(src + (size_t)idx[r] * K);
  uint4* d = reinterpret_cast<uint4*>(dst + (size_t)r * K);
  for (int i = threadIdx.x; i < K / 8; i += blockDim.x) d[i] = s[i];
}

// ===========================================================================
// host side
// ===========================================================================
struct GemmPlan {
  int n_tiles = 0, cs = 1, kslice = 0, stages = 1, smem = 0;
  bool valid = false;
};

struct FastPath {
  __nv_bfloat16 *w_qkv = nullptr, *w_o = nullptr, *w_gu = nullptr, *w_down = nullptr;
  CUtensorMap map_qkv, map_o, map_gu, map_down;
  __nv_bfloat16 *qb = nullptr, *ksb = nullptr, *vsb = nullptr, *ob = nullptr, *mb = nullptr;
  int num_sms = 148;
  int max_cluster = 8;
  int smem_cap = 112 * 1024;   // keeps two CTAs per SM so the next kernel can prefetch
  std::vector<void*> allocs;
};

namespace {

PFN_cuTensorMapEncodeTiled_v12000 get_encode() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  if (!fn) {
    cudaDriverEntryPointQueryResult q;
    void* p = nullptr;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = (PFN_cuTensorMapEncodeTiled_v12000)p;
  }
  return fn;
}

bool make_weight_map(CUtensorMap* map, const void* ptr, uint64_t rows, uint64_t K) {
  auto enc = get_encode();
  if (!enc) return false;
  cuuint64_t dims[2] = {K, rows};
  cuuint64_t strides[1] = {K * 2};
  cuuint32_t box[2] = {64, 128};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(ptr), dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

int round_up(int x, int m) { return (x + m - 1) / m * m; }

// Split of one projection over CTAs: 128-row weight tiles x K slices (one
// cluster per tile).  The smallest cluster that puts at least one CTA on
// every SM is taken, within the shared-memory and cluster-size limits.
GemmPlan plan_gemm(const FastPath* fp, int N, int K, int n_mma) {
  GemmPlan best;
  best.n_tiles = N / 128;
  for (int cs = 1; cs <= fp->max_cluster; cs <<= 1) {
    if (K % (cs * 64)) break;
    best.cs = cs;
    best.kslice = K / cs;
    if (best.n_tiles * cs >= fp->num_sms) break;
  }
  const int nbox = best.kslice / 64;
  int stages = nbox;
  while (stages > 1 && gemm_smem_layout(stages, n_mma).total > fp->smem_cap) --stages;
  best.stages = stages;
  best.smem = gemm_smem_layout(stages, n_mma).total;
  best.valid = best.kslice >= 64 && best.smem <= 227 * 1024;
  return best;
}

template <int MODE>
cudaError_t launch_gemm(const FastPath* fp, const CUtensorMap& map, const GemmArgs& a, const GemmPlan& pl,
                        cudaStream_t st) {
  auto kern = gemm_tc_kernel<MODE>;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(pl.cs, pl.n_tiles, 1);
  cfg.blockDim = dim3(192, 1, 1);
  cfg.dynamicSmemBytes = pl.smem;
  cfg.stream = st;
  cudaLaunchAttribute attrs[2];
  attrs[0].id = cudaLaunchAttributeClusterDimension;
  attrs[0].val.clusterDim.x = pl.cs;
  attrs[0].val.clusterDim.y = 1;
  attrs[0].val.clusterDim.z = 1;
  attrs[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attrs[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attrs;
  cfg.numAttrs = 2;
  GemmArgs args = a;
  args.kslice = pl.kslice;
  args.stages = pl.stages;
  return cudaLaunchKernelEx(&cfg, kern, map, args);
}

int attn_smem_bytes(int D) { return 3 * 64 * D * 2 + 64 * 2 * 4; }

// Kernel attributes are set once, outside any stream capture.
template <int MODE>
cudaError_t configure_gemm() {
  cudaError_t e = cudaFuncSetAttribute(gemm_tc_kernel<MODE>, cudaFuncAttributeMaxDynamicSharedMemorySize, 227 * 1024);
  if (e == cudaSuccess) e = cudaFuncSetAttribute(gemm_tc_kernel<MODE>, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
  return e;
}

template <int D>
cudaError_t configure_attn() {
  return cudaFuncSetAttribute(attn_mma_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, attn_smem_bytes(D));
}

template <int D>
cudaError_t launch_attn(const AttnArgs& a, int nchunk, int G, cudaStream_t st) {
  auto kern = attn_mma_kernel<D>;
  const int smem = attn_smem_bytes(D);
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(nchunk, a.Hq, G);
  cfg.blockDim = dim3(128, 1, 1);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attrs[2];
  attrs[0].id = cudaLaunchAttributeClusterDimension;
  attrs[0].val.clusterDim.x = nchunk;
  attrs[0].val.clusterDim.y = 1;
  attrs[0].val.clusterDim.z = 1;
  attrs[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attrs[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attrs;
  cfg.numAttrs = 2;
  return cudaLaunchKernelEx(&cfg, kern, a);
}

}  // namespace

rtv_status fast_create(rtv_ctx* ctx) {
  const rtv_expert_config& k = ctx->cfg;
  ctx->use_fast = false;
  const int S = ctx->S;
  const int n_mma_max = round_up(ctx->Gmax * S, 16);
  const bool shape_ok = k.dtype == RTV_BF16 && k.head_dim % 128 == 0 && (k.head_dim == 128 || k.head_dim == 256) &&
                        k.width % 128 == 0 && k.mlp_dim % 128 == 0 && (ctx->Q % 128) == 0 && S <= 64 &&
                        n_mma_max <= 256 && get_encode() != nullptr;
  if (!shape_ok) return RTV_OK;
  int dev = ctx->device;
  if (configure_gemm<GM_QKV>() != cudaSuccess || configure_gemm<GM_O>() != cudaSuccess ||
      configure_gemm<GM_GU>() != cudaSuccess || configure_gemm<GM_DOWN>() != cudaSuccess ||
      configure_attn<128>() != cudaSuccess || configure_attn<256>() != cudaSuccess) {
    cudaGetLastError();
    return RTV_ERR_CUDA;
  }
  FastPath* fp = new FastPath();
  cudaDeviceGetAttribute(&fp->num_sms, cudaDevAttrMultiProcessorCount, dev);
  // largest cluster that can be co-scheduled for the GEMM kernel
  {
    auto kern = gemm_tc_kernel<GM_DOWN>;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(16, 8, 1);
    cfg.blockDim = dim3(192, 1, 1);
    cfg.dynamicSmemBytes = 100 * 1024;
    cudaLaunchAttribute at;
    at.id = cudaLaunchAttributeClusterDimension;
    at.val.clusterDim.x = 16;
    at.val.clusterDim.y = 1;
    at.val.clusterDim.z = 1;
    cfg.attrs = &at;
    cfg.numAttrs = 1;
    int n = 0;
    if (cudaOccupancyMaxActiveClusters(&n, kern, &cfg) == cudaSuccess && n >= 8) fp->max_cluster = 16;
    cudaGetLastError();
  }
  const size_t T = ctx->Tmax;
  auto alloc = [&](void** p, size_t bytes) -> bool {
    if (cudaMalloc(p, bytes) != cudaSuccess) return false;
    fp->allocs.push_back(*p);
    return true;
  };
  bool ok = alloc((void**)&fp->qb, T * ctx->Q * 2) && alloc((void**)&fp->ob, T * ctx->Q * 2) &&
            alloc((void**)&fp->mb, T * (size_t)k.mlp_dim * 2) &&
            alloc((void**)&fp->ksb, (size_t)ctx->Gmax * ctx->KV * S * 2) &&
            alloc((void**)&fp->vsb, (size_t)ctx->Gmax * ctx->KV * S * 2);
  if (!ok) {
    for (void* p : fp->allocs) cudaFree(p);
    delete fp;
    return RTV_ERR_OOM;
  }
  ctx->fast = fp;
  ctx->use_fast = true;
  return RTV_OK;
}

bool fast_supports_prefix(rtv_ctx*, int) { return true; }

rtv_status fast_load(rtv_ctx* ctx, const rtv_tensor*, int) {
  FastPath* fp = ctx->fast;
  const rtv_expert_config& k = ctx->cfg;
  const int Lh = k.n_layers, w = k.width, F = k.mlp_dim, D = k.head_dim, Q = ctx->Q, KV = ctx->KV;
  const int HH = k.n_q_heads + 2 * k.n_kv_heads, tph = D / 128;
  const size_t nq = (size_t)(Q + 2 * KV), ngu = 2 * (size_t)F;
  auto alloc = [&](void** p, size_t bytes) -> bool {
    if (cudaMalloc(p, bytes) != cudaSuccess) return false;
    fp->allocs.push_back(*p);
    return true;
  };
  if (!(alloc((void**)&fp->w_qkv, Lh * nq * w * 2) && alloc((void**)&fp->w_o, (size_t)Lh * w * Q * 2) &&
        alloc((void**)&fp->w_gu, Lh * ngu * w * 2) && alloc((void**)&fp->w_down, (size_t)Lh * w * F * 2)))
    return RTV_ERR_OOM;
  // row orders of the packed tiles
  std::vector<int> iq(nq), igu(ngu);
  for (int nt = 0; nt < HH * tph; ++nt) {
    const int hh = nt / tph, b = nt % tph;
    for (int j = 0; j < 128; ++j)
      iq[(size_t)nt * 128 + j] = hh * D + 64 * b + (j < 64 ? j : j - 64 + D / 2);
  }
  for (int nt = 0; nt < F / 64; ++nt)
    for (int j = 0; j < 128; ++j) igu[(size_t)nt * 128 + j] = j < 64 ? 64 * nt + j : F + 64 * nt + (j - 64);
  int *d_iq = nullptr, *d_igu = nullptr;
  if (cudaMalloc(&d_iq, nq * 4) != cudaSuccess || cudaMalloc(&d_igu, ngu * 4) != cudaSuccess) return RTV_ERR_OOM;
  cudaMemcpy(d_iq, iq.data(), nq * 4, cudaMemcpyHostToDevice);
  cudaMemcpy(d_igu, igu.data(), ngu * 4, cudaMemcpyHostToDevice);
  for (int l = 0; l < Lh; ++l) {
    const LayerW& Lw = ctx->W.layers[l];
    gather_rows_kernel<<<(int)nq, 128>>>((const __nv_bfloat16*)Lw.qkv, fp->w_qkv + (size_t)l * nq * w, d_iq,
                                         (int)nq, w);
    gather_rows_kernel<<<(int)ngu, 128>>>((const __nv_bfloat16*)Lw.gu, fp->w_gu + (size_t)l * ngu * w, d_igu,
                                          (int)ngu, w);
    cudaMemcpy(fp->w_o + (size_t)l * w * Q, Lw.o, (size_t)w * Q * 2, cudaMemcpyDeviceToDevice);
    cudaMemcpy(fp->w_down + (size_t)l * w * F, Lw.down, (size_t)w * F * 2, cudaMemcpyDeviceToDevice);
  }
  cudaError_t e = cudaDeviceSynchronize();
  cudaFree(d_iq);
  cudaFree(d_igu);
  if (e != cudaSuccess) return RTV_ERR_CUDA;
  if (!make_weight_map(&fp->map_qkv, fp->w_qkv, Lh * nq, w) || !make_weight_map(&fp->map_o, fp->w_o, (size_t)Lh * w, Q) ||
      !make_weight_map(&fp->map_gu, fp->w_gu, Lh * ngu, w) ||
      !make_weight_map(&fp->map_down, fp->w_down, (size_t)Lh * w, F))
    return RTV_ERR_CUDA;
  return RTV_OK;
}

rtv_status fast_expert(rtv_ctx* ctx, int G, int P, const float* c, int c_stride, int state_stride,
                       int prefix_batch_stride, const float* rope_cs, const float* rope_sn, cudaStream_t st) {
  FastPath* fp = ctx->fast;
  const rtv_expert_config& k = ctx->cfg;
  const int S = ctx->S, T = G * S, w = k.width, F = k.mlp_dim, D = k.head_dim, Q = ctx->Q, KV = ctx->KV;
  const int n_mma = round_up(T, 16);
  const int nq = Q + 2 * KV;
  launch_embed<__nv_bfloat16>(ctx->x, ctx->state, state_stride, (const __nv_bfloat16*)ctx->W.sp_w, ctx->W.sp_b,
                              (const __nv_bfloat16*)ctx->W.ai_w, ctx->W.ai_b, c, c_stride, ctx->h, G, w, S,
                              k.action_dim, k.state_dim, st);
  const GemmPlan p_qkv = plan_gemm(fp, nq, w, n_mma);
  const GemmPlan p_o = plan_gemm(fp, w, Q, n_mma);
  const GemmPlan p_gu = plan_gemm(fp, 2 * F, w, n_mma);
  const GemmPlan p_dn = plan_gemm(fp, w, F, n_mma);
  if (!(p_qkv.valid && p_o.valid && p_gu.valid && p_dn.valid)) {
    ctx->last_error = "no tensor-core split fits this token count";
    return RTV_ERR_UNSUPPORTED;
  }
  if (getenv("RTV_LOG")) {
    const GemmPlan* pls[4] = {&p_qkv, &p_o, &p_gu, &p_dn};
    const char* nm[4] = {"qkv", "o", "gu", "down"};
    for (int i = 0; i < 4; ++i)
      fprintf(stderr, "[rtv] T=%d %s: tiles=%d cluster=%d kslice=%d stages=%d smem=%d\n", T, nm[i], pls[i]->n_tiles,
              pls[i]->cs, pls[i]->kslice, pls[i]->stages, pls[i]->smem);
    fprintf(stderr, "[rtv] attention: chunks=%d keys/chunk=%d max_cluster=%d sms=%d\n", std::min(8, P + S),
            (P + S + std::min(8, P + S) - 1) / std::min(8, P + S), fp->max_cluster, fp->num_sms);
  }

  GemmArgs base{};
  base.h = ctx->h;
  base.h_out = ctx->h;
  base.q = fp->qb;
  base.ks = fp->ksb;
  base.vs = fp->vsb;
  base.rope_cs = rope_cs;
  base.rope_sn = rope_sn;
  base.m = fp->mb;
  base.status = ctx->status;
  base.timeout_ns = k.barrier_timeout_ns;
  base.T = T;
  base.n_mma = n_mma;
  base.w = w;
  base.S = S;
  base.Hq = k.n_q_heads;
  base.Hkv = k.n_kv_heads;
  base.D = D;
  base.F = F;
  base.eps = k.rms_eps;

  const int nk = P + S;
  const int nchunk = std::min(8, nk);
  AttnArgs at{};
  at.q = fp->qb;
  at.sk = fp->ksb;
  at.sv = fp->vsb;
  at.o = fp->ob;
  at.status = ctx->status;
  at.S = S;
  at.P = P;
  at.Pmax = k.max_prefix_len;
  at.Hq = k.n_q_heads;
  at.Hkv = k.n_kv_heads;
  at.pbs = prefix_batch_stride;
  at.mask_mode = k.suffix_mask;
  at.kpc = (nk + nchunk - 1) / nchunk;
  at.scale_log2 = (float)(1.4426950408889634 / sqrt((double)D));
  const size_t kv_layer = (size_t)k.max_batch * k.n_kv_heads * k.max_prefix_len * D;

  for (int l = 0; l < k.n_layers; ++l) {
    const LayerW& Lw = ctx->W.layers[l];
    GemmArgs a = base;
    a.gain = Lw.g_attn;
    a.K = w;
    a.w_row0 = l * nq;
    cudaError_t e = launch_gemm<GM_QKV>(fp, fp->map_qkv, a, p_qkv, st);

    at.pk = (const __nv_bfloat16*)ctx->prefix_kv + (size_t)(2 * l) * kv_layer;
    at.pv = (const __nv_bfloat16*)ctx->prefix_kv + (size_t)(2 * l + 1) * kv_layer;
    if (e == cudaSuccess) e = D == 256 ? launch_attn<256>(at, nchunk, G, st) : launch_attn<128>(at, nchunk, G, st);

    a = base;
    a.act = fp->ob;
    a.K = Q;
    a.w_row0 = l * w;
    if (e == cudaSuccess) e = launch_gemm<GM_O>(fp, fp->map_o, a, p_o, st);

    a = base;
    a.gain = Lw.g_mlp;
    a.K = w;
    a.w_row0 = l * 2 * F;
    if (e == cudaSuccess) e = launch_gemm<GM_GU>(fp, fp->map_gu, a, p_gu, st);

    a = base;
    a.act = fp->mb;
    a.K = F;
    a.w_row0 = l * w;
    if (e == cudaSuccess) e = launch_gemm<GM_DOWN>(fp, fp->map_down, a, p_dn, st);
    if (e != cudaSuccess) {
      ctx->last_error = std::string("tensor-core launch: ") + cudaGetErrorString(e);
      return RTV_ERR_CUDA;
    }
  }
  return RTV_OK;
}

void fast_out_head(rtv_ctx* ctx, int G, float dt, bool velocity_only, cudaStream_t st) {
  const rtv_expert_config& k = ctx->cfg;
  launch_out_head<__nv_bfloat16>(ctx->h, ctx->W.g_final, (const __nv_bfloat16*)ctx->W.ao_w, ctx->W.ao_b, ctx->x,
                                 velocity_only ? ctx->v : nullptr, dt, G, k.width, ctx->S, k.action_dim, k.rms_eps,
                                 ctx->status, st);
}

void fast_destroy(rtv_ctx* ctx) {
  if (!ctx->fast) return;
  for (void* p : ctx->fast->allocs) cudaFree(p);
  delete ctx->fast;
  ctx->fast = nullptr;
}

}  // namespace rtv
