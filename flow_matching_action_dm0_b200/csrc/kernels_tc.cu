// Tensor-core path of the bf16 action expert on sm_100a.
//
// One Euler step of the expert is 1 + 5 * n_layers kernels, chained with
// programmatic dependent launch (PDL) inside one CUDA graph:
//   STEP  output head + Euler update of the previous step and suffix
//         embedding of this one (state_proj / action_in_proj + time condition)
//   per layer:
//   QKV   q/k/v projection of RMSNorm(h), RoPE, written as bf16 q and suffix K/V
//   ATTN  split-KV grouped-query attention over [prefix KV ; suffix KV]
//   O     attention output projection added to the fp32 residual
//   GU    gate/up projection of RMSNorm(h), gelu_tanh(gate) * up (bf16)
//   DOWN  down projection added to the fp32 residual
// ("DM0.5 reading guide", sec. 5.2 action expert, sec. 5.3 Euler sampling,
// sec. 6.4 fused suffix kernels: normalise/modulate -> GEMM -> activation ->
// write back, sec. 6.5 one graph replay.)
//
// The projections are weight-streaming GEMMs at M = tokens (51 per suffix):
// out[t][n] = sum_k act[t][k] W[n][k], computed swapped, D = W x act^T, so
// that 128 weight rows fill the tcgen05 M dimension and the tokens (padded to
// a multiple of 16) form N.  A CTA owns one 128-row weight tile and one K
// slice.  Its first ring-full of weight boxes is fetched by TMA as soon as the
// CTA starts -- before it waits on the previous kernel, since weights do not
// depend on it -- and the bf16 activation boxes follow once that kernel has
// finished.  The K slices of one weight tile form a thread-block cluster: each
// rank copies the partial sums of the tokens another rank owns into that
// rank's shared memory with one bulk copy, and the owner reduces them in rank
// order (deterministic).
//
// RMSNorm is split between producer and consumer.  A kernel that writes the
// residual h (STEP, O, DOWN) also writes the next norm's input scaled by its
// gain, bf16(h * (1 + g)), and the sum of squares of h over each 128-feature
// tile.  The consumer (QKV, GU) multiplies its accumulator by
// 1/rms(h) = rsqrt(sum of the tile sums / width + eps), a per-token factor
// that commutes with the product.
#include <cudaTypedefs.h>

#include <math.h>
#include <stdio.h>
#include <stdlib.h>
#include <string.h>

#include <algorithm>
#include <string>
#include <vector>

#include "common.cuh"
#include "fastpath.h"
#include "kernels.h"
#include "runtime.h"
#include "tc_ptx.cuh"

namespace rtv {

enum { GM_QKV = 0, GM_O = 1, GM_GU = 2, GM_DOWN = 3 };

struct GemmArgs {
  float* h;                   // fp32 residual stream [T][w] (O, DOWN add into it)
  __nv_bfloat16* hb;          // next norm's input bf16(h * (1 + g_next)) [T][w]   (written by O, DOWN)
  float* ssp;                 // sums of squares of h per 128-feature tile [T][w/128]
  const float* g_next;        // gain of the next RMSNorm, or nullptr when no norm consumer follows
  __nv_bfloat16* q;           // [T][Hq][D]
  __nv_bfloat16* ks;          // suffix keys   [G][Hkv][S][D]
  __nv_bfloat16* vs;          // suffix values [G][Hkv][S][D]
  const float* rope_cs;       // [S][D/2]
  const float* rope_sn;
  __nv_bfloat16* m;           // [T][F]
  unsigned* status;
  unsigned long long* trace;  // optional phase stamps [cta][16] (globaltimer ns), or nullptr
  long long timeout_ns;
  int T, n_mma, kslice, stages, w, S, Hq, Hkv, D, F, w_row0;
  float eps;
};

// Phase stamps of the optional trace (one row of 16 per CTA).
enum { TR_START = 0, TR_W_ISSUED, TR_PDL, TR_FIRST_FULL, TR_MMA_ISSUED, TR_DONE, TR_COPIED, TR_RECV, TR_END,
       TR_PREFETCHED, TR_ARRIVED, TR_ITER0, TR_EXIT };

struct GemmSmem {
  int stages, stage_bytes, ring_bytes, part_off, recv_off, in_off, bar_off, total;
};

// Shared memory of one GEMM CTA: a ring of `stages` stages, each a 128x64
// bf16 weight box (16 KB) and the matching 64-wide bf16 activation box of
// n_mma token rows, both K-major with the 128-byte swizzle; the fp32 partial
// tile [n_mma][128] (over the ring once the MMAs are done, when it fits);
// the receive buffer [cs * per][128] of the cluster reduction; the
// epilogue's per-token inputs [per][128] (residual rows or RoPE cos/sin);
// mbarriers.
__host__ __device__ inline GemmSmem gemm_smem_layout(int stages, int n_mma, int cs, int T) {
  GemmSmem s;
  const int per = (T + cs - 1) / cs;
  s.stages = stages;
  s.stage_bytes = 16384 + n_mma * 128;
  s.ring_bytes = stages * s.stage_bytes;
  const int part_bytes = n_mma * 512;
  s.part_off = part_bytes <= s.ring_bytes ? 0 : s.ring_bytes;
  s.recv_off = s.ring_bytes > s.part_off + part_bytes ? s.ring_bytes : s.part_off + part_bytes;
  s.in_off = s.recv_off + cs * per * 512;   // [per][128] fp32 epilogue inputs of the owned tokens
  s.bar_off = s.in_off + per * 512;
  s.total = s.bar_off + (2 * stages + 2) * 8 + 16 + 1024;   // barriers, TMEM slot, alignment slack
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

// Split cluster barrier.  Every CTA of a cluster must have started (and
// initialised its mbarriers) before anyone touches its shared memory, so all
// threads arrive at entry and wait before their first remote access.
__device__ __forceinline__ void cluster_arrive_relaxed() {
  asm volatile("barrier.cluster.arrive.relaxed.aligned;" ::: "memory");
}
__device__ __forceinline__ void cluster_arrive_release() {
  asm volatile("barrier.cluster.arrive.release.aligned;" ::: "memory");
}
__device__ __forceinline__ void cluster_wait() { asm volatile("barrier.cluster.wait.aligned;" ::: "memory"); }

// Bulk copy of `bytes` from this CTA's shared memory to another CTA's shared
// memory of the cluster; completion is counted in bytes on the destination's mbarrier.
__device__ __forceinline__ void bulk_copy_to_rank(uint32_t dst_cluster, uint32_t src_cta, uint32_t bytes,
                                                  uint32_t mbar_cluster) {
  asm volatile(
      "cp.async.bulk.shared::cluster.shared::cta.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
          dst_cluster),
      "r"(src_cta), "r"(bytes), "r"(mbar_cluster)
      : "memory");
}

template <int MODE>
__global__ void __launch_bounds__(192, 1) gemm_tc_kernel(const __grid_constant__ CUtensorMap wmap,
                                                         const __grid_constant__ CUtensorMap amap, const GemmArgs a) {
  extern __shared__ uint8_t smem_raw[];
  __shared__ float rs_s[64];
  const int n_mma = a.n_mma;
  const int cs = gridDim.x;
  const GemmSmem L = gemm_smem_layout(a.stages, n_mma, cs, a.T);
  // every CTA of the grid sees the same values, so a refusal is uniform across each cluster
  if (dynamic_smem_size() < (uint32_t)L.total || a.kslice < 64 || (a.kslice & 63) || a.stages < 1 || n_mma > 256 ||
      (n_mma & 15) || a.T > n_mma || cs > 16 || (a.T + cs - 1) / cs > 64) {
    if (threadIdx.x == 0) atomicOr(a.status, RTV_DEV_BOUNDS);
    return;
  }
  uint8_t* base = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = ptx::cluster_ctarank();
  const int nt = blockIdx.y;
  const int nbox = a.kslice >> 6;
  const int NS = L.stages;
  const int k0 = (int)rank * a.kslice;
  const int per = (a.T + cs - 1) / cs;                 // tokens owned by each rank in the reduction
  const int t_own0 = (int)rank * per;
  const int n_own = max(0, min(a.T, t_own0 + per) - t_own0);
  float* part = (float*)(base + L.part_off);           // [n_mma][128] this CTA's partial sums
  float* recv = (float*)(base + L.recv_off);           // [cs][per][128] partials of the tokens I own
  uint64_t* full = (uint64_t*)(base + L.bar_off);      // weight + activation boxes landed
  uint64_t* empty = full + NS;                         // the stage's MMAs completed
  uint64_t* done = empty + NS;                         // all MMAs completed
  uint64_t* rbar = done + 1;                           // all partials of my tokens landed
  uint32_t* tmem_slot = (uint32_t*)(rbar + 1);
  const uint32_t ncols = (uint32_t)tmem_cols_for(n_mma);
  const uint32_t act_box_bytes = (uint32_t)n_mma * 128u;
  unsigned long long* trace = a.trace ? a.trace + ((size_t)blockIdx.y * gridDim.x + blockIdx.x) * 16 : nullptr;
  if (trace && threadIdx.x == 0) trace[TR_START] = ptx::globaltimer();

  if (threadIdx.x == 0) {
    for (int i = 0; i < NS; ++i) {
      ptx::mbar_init(&full[i], 2);
      ptx::mbar_init(&empty[i], 1);
    }
    ptx::mbar_init(done, 1);
    ptx::mbar_init(rbar, 1);
    ptx::fence_mbar_init();
  }
  __syncthreads();
  cluster_arrive_relaxed();
  ptx::pdl_launch_dependents();

  // Weights do not depend on the previous kernel: the first ring-full of
  // weight boxes is requested before anyone waits on that kernel.  Nothing
  // before the __syncthreads below waits on another role.
  const int first = nbox < NS ? nbox : NS;
  uint64_t pol = 0;
  if (warp == 0) {
    if (lane == 0) {
      pol = ptx::policy_evict_first();
      for (int b = 0; b < first; ++b) {
        ptx::mbar_expect_tx(&full[b], 16384u);
        ptx::tma_load_2d(base + b * L.stage_bytes, &wmap, &full[b], k0 + 64 * b, a.w_row0 + nt * 128, pol);
      }
      if (trace) trace[TR_W_ISSUED] = ptx::globaltimer();
    }
  } else if (warp == 1) {
    ptx::tmem_alloc(tmem_slot, ncols);
    ptx::tmem_relinquish();
    ptx::tc_fence_before();
  }
  __syncthreads();   // TMEM address published
  ptx::tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  // After a bounded wait gives up, a role stops issuing copies and MMAs (so no
  // barrier ever sees an extra arrival), records the timeout, and still
  // reaches every cluster barrier.
  if (warp == 0) {
    // ---- producer: activation boxes once the previous kernel is done; remaining weight boxes ----
    if (lane == 0) {
      ptx::pdl_wait();
      if (trace) trace[TR_PDL] = ptx::globaltimer();
      for (int b = 0; b < nbox; ++b) {
        const int s = b % NS, u = b / NS;
        uint8_t* st = base + s * L.stage_bytes;
        if (b >= first) {
          if (!ptx::mbar_wait(&empty[s], (u - 1) & 1, a.timeout_ns)) {
            atomicOr(a.status, RTV_DEV_TIMEOUT);
            break;
          }
          ptx::mbar_expect_tx(&full[s], 16384u);
          ptx::tma_load_2d(st, &wmap, &full[s], k0 + 64 * b, a.w_row0 + nt * 128, pol);
        }
        ptx::mbar_expect_tx(&full[s], act_box_bytes);
        ptx::tma_load_2d_nohint(st + 16384, &amap, &full[s], k0 + 64 * b, 0);
      }
    }
  } else if (warp == 1) {
    // ---- MMA issue: one thread ----
    if (lane == 0) {
      const uint32_t idesc = ptx::idesc_bf16_f32(128, n_mma);
      for (int b = 0; b < nbox; ++b) {
        const int s = b % NS, u = b / NS;
        if (!ptx::mbar_wait(&full[s], u & 1, a.timeout_ns)) {
          atomicOr(a.status, RTV_DEV_TIMEOUT);
          break;
        }
        ptx::tc_fence_after();
        if (trace && b == 0) trace[TR_FIRST_FULL] = ptx::globaltimer();
        const uint32_t wa = ptx::smem_u32(base + s * L.stage_bytes);
        const uint32_t aa = wa + 16384u;
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) {
          const uint64_t ad = ptx::sw128_kmajor_desc(wa + kk * 32);
          const uint64_t bd = ptx::sw128_kmajor_desc(aa + kk * 32);
          ptx::umma_bf16(tmem, ad, bd, idesc, (b | kk) != 0 ? 1u : 0u);
        }
        ptx::umma_commit(&empty[s]);
      }
      ptx::umma_commit(done);
      if (trace) trace[TR_MMA_ISSUED] = ptx::globaltimer();
    }
  } else {
    // ---- epilogue warps 2..5 ----
    const int tid = threadIdx.x - 64;
    ptx::pdl_wait();   // this role reads and writes what earlier kernels produced
    if (tid == 0) ptx::mbar_expect_tx(rbar, (uint32_t)(cs * n_own * 512));
    if (!ptx::mbar_wait(done, 0, a.timeout_ns)) atomicOr(a.status, RTV_DEV_TIMEOUT);
    ptx::tc_fence_after();
    if (trace && tid == 0) trace[TR_DONE] = ptx::globaltimer();
    // accumulator -> this CTA's partial tile [token][feature]
    const int quarter = warp & 3;
    const int f = quarter * 32 + lane;
    for (int c = 0; c < n_mma; c += 32) {
      float v[32];
      if (c + 16 < n_mma) {
        ptx::tmem_ld_32(tmem + ((uint32_t)(quarter * 32) << 16) + (uint32_t)c, v);
#pragma unroll
        for (int i = 0; i < 32; ++i) part[(c + i) * 128 + f] = v[i];
      } else {
        ptx::tmem_ld_16(tmem + ((uint32_t)(quarter * 32) << 16) + (uint32_t)c, *reinterpret_cast<float(*)[16]>(v));
#pragma unroll
        for (int i = 0; i < 16; ++i) part[(c + i) * 128 + f] = v[i];
      }
    }
    ptx::tc_fence_before();
    ptx::fence_proxy_async_smem();
    asm volatile("bar.sync 1, 128;" ::: "memory");
    cluster_wait();   // entry phase: every rank has started and initialised its barriers
    if (tid == 0) {
      const uint32_t part_a = ptx::smem_u32(part), recv_a = ptx::smem_u32(recv), rbar_a = ptx::smem_u32(rbar);
      for (int r = 0; r < cs; ++r) {
        const int o0 = r * per, no = max(0, min(a.T, o0 + per) - o0);
        if (no == 0) continue;
        bulk_copy_to_rank(ptx::mapa(recv_a + (uint32_t)(rank * per * 512), (uint32_t)r),
                          part_a + (uint32_t)(o0 * 512), (uint32_t)(no * 512), ptx::mapa(rbar_a, (uint32_t)r));
      }
      if (trace) trace[TR_COPIED] = ptx::globaltimer();
    }
    // Everything the epilogue reads from global memory is requested now, in
    // parallel, while the partials are still in flight: the owned tokens'
    // residual rows of this tile (O, DOWN) or their RoPE cos/sin (QKV) go to
    // shared memory by cp.async; 1/rms of the owned tokens (QKV, GU) too.
    float* in_s = (float*)(base + L.in_off);
    const int n_wt = a.w >> 7;
    const int tph = a.D >> 7, hd = a.D >> 1;
    const int hh = nt / tph, dq0 = 64 * (nt - (nt / tph) * tph);
    const bool rope = MODE == GM_QKV && hh < a.Hq + a.Hkv;
    const uint32_t in_a = ptx::smem_u32(in_s);
    if (MODE == GM_O || MODE == GM_DOWN) {
      for (int c = tid; c < n_own * 32; c += 128) {
        const int tl = c >> 5, ch = c & 31;
        ptx::cp_async_16(in_a + (uint32_t)(c * 16), a.h + (size_t)(t_own0 + tl) * a.w + nt * 128 + ch * 4);
      }
    } else if (rope) {
      for (int c = tid; c < n_own * 32; c += 128) {
        const int tl = c >> 5, ch = c & 31;   // chunks 0-15: cos, 16-31: sin (64 floats each)
        const int s = (t_own0 + tl) % a.S;
        const float* src = (ch < 16 ? a.rope_cs : a.rope_sn) + (size_t)s * hd + dq0 + (ch & 15) * 4;
        ptx::cp_async_16(in_a + (uint32_t)(c * 16), src);
      }
    }
    if ((MODE == GM_QKV || MODE == GM_GU) && tid < n_own) {
      float sst = 0.f;
      for (int j2 = 0; j2 < n_wt; ++j2) sst += a.ssp[(size_t)(t_own0 + tid) * n_wt + j2];
      rs_s[tid] = rsqrtf(sst / (float)a.w + a.eps);
    }
    ptx::cp_async_wait_all();
    asm volatile("bar.sync 1, 128;" ::: "memory");
    if (trace && tid == 0) trace[TR_PREFETCHED] = ptx::globaltimer();
    if (!ptx::mbar_wait(rbar, 0, a.timeout_ns)) atomicOr(a.status, RTV_DEV_TIMEOUT);
    if (trace && tid == 0) trace[TR_RECV] = ptx::globaltimer();
    cluster_arrive_release();   // my incoming copies are complete
    if (trace && tid == 0) trace[TR_ARRIVED] = ptx::globaltimer();

    // ---- reduction in rank order + epilogue for the tokens this rank owns ----
    // one warp per token; lane l takes features (2l, 2l+1) and (2l+64, 2l+65)
    const int ew = warp - 2;
    const int f0 = 2 * lane;
    const int n1 = nt * 128 + f0, n2 = n1 + 64;
    float2 gn1 = make_float2(0.f, 0.f), gn2 = make_float2(0.f, 0.f);
    if ((MODE == GM_O || MODE == GM_DOWN) && a.g_next) {
      gn1 = *reinterpret_cast<const float2*>(a.g_next + n1);
      gn2 = *reinterpret_cast<const float2*>(a.g_next + n2);
    }
#pragma unroll 1
    for (int tl = ew; tl < n_own; tl += 4) {
      const int t = t_own0 + tl;
      float2 x1 = make_float2(0.f, 0.f), x2 = make_float2(0.f, 0.f);
      for (int qr = 0; qr < cs; ++qr) {
        const float* rr = recv + (qr * per + tl) * 128;
        const float2 u1 = *reinterpret_cast<const float2*>(rr + f0);
        const float2 u2 = *reinterpret_cast<const float2*>(rr + 64 + f0);
        x1.x += u1.x;
        x1.y += u1.y;
        x2.x += u2.x;
        x2.y += u2.y;
      }
      if (MODE == GM_O || MODE == GM_DOWN) {
        // residual add, then the next norm's bf16 input and this tile's sum of squares
        const float2 r1 = *reinterpret_cast<const float2*>(in_s + tl * 128 + f0);
        const float2 r2 = *reinterpret_cast<const float2*>(in_s + tl * 128 + 64 + f0);
        const float2 h1 = make_float2(r1.x + x1.x, r1.y + x1.y);
        const float2 h2 = make_float2(r2.x + x2.x, r2.y + x2.y);
        *reinterpret_cast<float2*>(a.h + (size_t)t * a.w + n1) = h1;
        *reinterpret_cast<float2*>(a.h + (size_t)t * a.w + n2) = h2;
        if (a.g_next) {
          float sq = h1.x * h1.x;
          sq = fmaf(h1.y, h1.y, sq);
          sq = fmaf(h2.x, h2.x, sq);
          sq = fmaf(h2.y, h2.y, sq);
          sq = warp_sum(sq);
          *reinterpret_cast<uint32_t*>(a.hb + (size_t)t * a.w + n1) =
              ptx::pack_bf16x2(h1.x * (1.f + gn1.x), h1.y * (1.f + gn1.y));
          *reinterpret_cast<uint32_t*>(a.hb + (size_t)t * a.w + n2) =
              ptx::pack_bf16x2(h2.x * (1.f + gn2.x), h2.y * (1.f + gn2.y));
          if (lane == 0) a.ssp[(size_t)t * n_wt + nt] = sq;
        }
      } else {
        const float rs = rs_s[tl];
        x1.x *= rs;
        x1.y *= rs;
        x2.x *= rs;
        x2.y *= rs;
        if (MODE == GM_GU) {
          *reinterpret_cast<uint32_t*>(a.m + (size_t)t * a.F + nt * 64 + f0) =
              ptx::pack_bf16x2(gelu_tanh(x1.x) * x2.x, gelu_tanh(x1.y) * x2.y);
        } else {
          const int g = t / a.S, s = t - g * a.S;
          float2 y1 = x1, y2 = x2;
          if (rope) {
            const float2 c = *reinterpret_cast<const float2*>(in_s + tl * 128 + f0);
            const float2 sn = *reinterpret_cast<const float2*>(in_s + tl * 128 + 64 + f0);
            y1 = make_float2(x1.x * c.x - x2.x * sn.x, x1.y * c.y - x2.y * sn.y);
            y2 = make_float2(x2.x * c.x + x1.x * sn.x, x2.y * c.y + x1.y * sn.y);
          }
          __nv_bfloat16* dst;
          if (hh < a.Hq) dst = a.q + ((size_t)t * a.Hq + hh) * a.D;
          else if (hh < a.Hq + a.Hkv) dst = a.ks + (((size_t)g * a.Hkv + (hh - a.Hq)) * a.S + s) * a.D;
          else dst = a.vs + (((size_t)g * a.Hkv + (hh - a.Hq - a.Hkv)) * a.S + s) * a.D;
          *reinterpret_cast<uint32_t*>(dst + dq0 + f0) = ptx::pack_bf16x2(y1.x, y1.y);
          *reinterpret_cast<uint32_t*>(dst + dq0 + f0 + hd) = ptx::pack_bf16x2(y2.x, y2.y);
        }
      }
      if (trace && tid == 0 && tl == 0) trace[TR_ITER0] = ptx::globaltimer();
    }
    if (trace && tid == 0) trace[TR_END] = ptx::globaltimer();
  }
  if (warp < 2) {
    cluster_wait();             // entry phase
    cluster_arrive_release();   // nothing incoming to wait for
  }
  cluster_wait();   // every rank's incoming copies are complete: no copy still reads my shared memory
  if (trace && threadIdx.x == 64) trace[TR_EXIT] = ptx::globaltimer();
  if (warp == 1) {
    ptx::tc_fence_after();
    ptx::tmem_dealloc(tmem, ncols);
  }
  // never leave with a copy still landing in this CTA's shared memory
  if (warp == 0 && lane == 0) {
    for (int s2 = 0; s2 < first; ++s2) ptx::mbar_wait(&full[s2], ((nbox - 1 - s2) / NS) & 1, a.timeout_ns);
  }
}

// ---------------------------------------------------------------------------
// Split-KV grouped-query attention for one (query head, suffix) per cluster
// ("DM0.5 reading guide", sec. 5.1-5.2: suffix queries over the cached prefix
// KV and the bidirectional suffix; optional Pi0 block mask for the state
// token).  The cluster's CTAs take consecutive key ranges of [prefix ; own
// suffix] in tiles of 128 keys.  In a CTA, warp w handles query rows
// 16*(w%4).. and one 64-key half of each tile with a flash-style online
// softmax on warp-level bf16 MMAs (fp32 accumulate).  The two halves are
// merged in shared memory, then every CTA pushes its (max, sum, partial
// output) rows to the rank that combines them.
// ---------------------------------------------------------------------------
struct AttnArgs {
  const __nv_bfloat16* q;    // [T][Hq][D]
  const __nv_bfloat16* pk;   // this layer's prefix keys   [Bmax][Hkv][Pmax][D]
  const __nv_bfloat16* pv;   // this layer's prefix values
  const __nv_bfloat16* sk;   // suffix keys   [G][Hkv][S][D]
  const __nv_bfloat16* sv;
  __nv_bfloat16* o;          // [T][Hq*D]
  unsigned* status;
  unsigned long long* trace; // optional phase stamps [cta][16], or nullptr
  int S, P, Pmax, Hq, Hkv, pbs, mask_mode, kpc;
  float scale_log2;
};

// Q tile, K and V tiles, receive buffers of the cluster combine (bf16 rows +
// fp32 max/sum), combine weights.
__host__ __device__ inline int attn_smem_bytes(int D, int nchunk, int rpc) {
  return 64 * D * 2 + 2 * 128 * D * 2 + nchunk * rpc * D * 2 + nchunk * rpc * 2 * 4 + rpc * (nchunk + 1) * 4;
}

template <int D>
__global__ void __launch_bounds__(256) attn_mma_kernel(const AttnArgs a) {
  extern __shared__ __align__(128) uint8_t sm_attn[];
  constexpr int CPR = D / 8;   // 16-byte chunks per row
  const int nchunk = gridDim.x;
  const int rpc = (a.S + nchunk - 1) / nchunk;   // query rows combined by each rank
  if (dynamic_smem_size() < (uint32_t)attn_smem_bytes(D, nchunk, rpc) || a.S > 64 || nchunk > 16) {
    if (threadIdx.x == 0) atomicOr(a.status, RTV_DEV_BOUNDS);
    return;
  }
  __nv_bfloat16* Qs = reinterpret_cast<__nv_bfloat16*>(sm_attn);
  __nv_bfloat16* Ks = Qs + 64 * D;
  __nv_bfloat16* Vs = Ks + 128 * D;
  __nv_bfloat16* recv = Vs + 128 * D;                      // [nchunk][rpc][D] partial outputs pushed to me
  float* recv_ml = reinterpret_cast<float*>(recv + nchunk * rpc * D);   // [nchunk][rpc][2] (running max, sum)
  float* wq_s = recv_ml + nchunk * rpc * 2;                 // [rpc][nchunk] combine weights
  float* inv_s = wq_s + rpc * nchunk;                       // [rpc] 1 / combined sum
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int rb = warp & 3, kh = warp >> 2;
  const int rank = (int)ptx::cluster_ctarank();
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

  unsigned long long* trace =
      a.trace ? a.trace + (((size_t)blockIdx.z * gridDim.y + blockIdx.y) * gridDim.x + blockIdx.x) * 16 : nullptr;
  if (trace && tid == 0) trace[0] = ptx::globaltimer();
  cluster_arrive_relaxed();
  ptx::pdl_launch_dependents();
  ptx::pdl_wait();
  if (trace && tid == 0) trace[1] = ptx::globaltimer();

  const uint32_t qs_a = ptx::smem_u32(Qs), ks_a = ptx::smem_u32(Ks), vs_a = ptx::smem_u32(Vs);
  for (int c = tid; c < 64 * CPR; c += 256) {
    const int r = c / CPR, ch = c - r * CPR;
    const uint32_t off = (uint32_t)((r * D + ((ch ^ (r & 7)) << 3)) * 2);
    if (r < a.S) ptx::cp_async_16(qs_a + off, a.q + (((size_t)g * a.S + r) * a.Hq + j) * D + ch * 8);
    else *reinterpret_cast<uint4*>(reinterpret_cast<uint8_t*>(Qs) + off) = make_uint4(0, 0, 0, 0);
  }

  float o_acc[D / 8][4];
#pragma unroll
  for (int i = 0; i < D / 8; ++i) o_acc[i][0] = o_acc[i][1] = o_acc[i][2] = o_acc[i][3] = 0.f;
  float m_r[2] = {-INFINITY, -INFINITY}, l_r[2] = {0.f, 0.f};
  const int row0 = 16 * rb + (lane >> 2);

  for (int kt = kb; kt < ke; kt += 128) {
    __syncthreads();
    for (int c = tid; c < 128 * CPR; c += 256) {
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
    if (trace && tid == 0 && kt == kb) trace[2] = ptx::globaltimer();
    const int kbase = 64 * kh;   // this warp's half of the tile
    if (kt + kbase < ke) {
      // scores S = Q K^T for this warp's 16 rows x 64 keys
      float s_acc[8][4];
#pragma unroll
      for (int i = 0; i < 8; ++i) s_acc[i][0] = s_acc[i][1] = s_acc[i][2] = s_acc[i][3] = 0.f;
#pragma unroll 4
      for (int kk = 0; kk < D / 16; ++kk) {
        uint32_t af[4];
        {
          const int r = 16 * rb + (lane & 15), ch = 2 * kk + (lane >> 4);
          ptx::ldmatrix_x4(af, qs_a + (uint32_t)((r * D + ((ch ^ (r & 7)) << 3)) * 2));
        }
#pragma unroll
        for (int np = 0; np < 4; ++np) {
          uint32_t bf[4];
          const int r = kbase + 16 * np + (lane & 7) + ((lane >> 4) << 3), ch = 2 * kk + ((lane >> 3) & 1);
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
          const int key = kt + kbase + 8 * nt + 2 * (lane & 3) + (e & 1);
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
          const float pv = (s_acc[nt][e] == -INFINITY) ? 0.f : exp2f(s_acc[nt][e] - mnew[e >> 1]);
          s_acc[nt][e] = pv;
          l_r[e >> 1] += pv;
        }
      }
      if (kt != kb) {
#pragma unroll
        for (int i = 0; i < D / 8; ++i) {
          o_acc[i][0] *= corr[0];
          o_acc[i][1] *= corr[0];
          o_acc[i][2] *= corr[1];
          o_acc[i][3] *= corr[1];
        }
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
          const int r = kbase + 16 * kb2 + (lane & 7) + (((lane >> 3) & 1) << 3), ch = 2 * dn + (lane >> 4);
          ptx::ldmatrix_x4_trans(bf, vs_a + (uint32_t)((r * D + ((ch ^ (r & 7)) << 3)) * 2));
          ptx::mma_bf16_16816(o_acc[2 * dn], pf, bf[0], bf[1]);
          ptx::mma_bf16_16816(o_acc[2 * dn + 1], pf, bf[2], bf[3]);
        }
      }
    }
  }
  ptx::cp_async_wait_all();
  if (trace && tid == 0) trace[3] = ptx::globaltimer();
#pragma unroll
  for (int i = 0; i < 2; ++i) {
    l_r[i] += __shfl_xor_sync(0xffffffffu, l_r[i], 1);
    l_r[i] += __shfl_xor_sync(0xffffffffu, l_r[i], 2);
  }
  // merge the two key halves of each row block in shared memory (K/V tiles are dead)
  __syncthreads();
  // padded row strides keep the fragment-order accesses below free of bank conflicts
  constexpr int XS = D + 8;                                      // fp32 row stride of xo
  constexpr int OS = D + 8;                                      // bf16 row stride of ob_s
  float* xo = reinterpret_cast<float*>(Ks);                      // [64 rows][XS] fp32   (K and V tiles are dead)
  __nv_bfloat16* ob_s = reinterpret_cast<__nv_bfloat16*>(xo + 64 * XS);   // [64 rows][OS] merged rows, bf16
  float* xml = reinterpret_cast<float*>(Qs);                     // [64 rows][2] (the Q tile is dead too)
  float* mml = reinterpret_cast<float*>(Qs) + 64 * 2;            // [64 rows][2] merged (max, sum)
  if (kh == 1) {
#pragma unroll
    for (int nt = 0; nt < D / 8; ++nt) {
      const int d = 8 * nt + 2 * (lane & 3);
      *reinterpret_cast<float2*>(xo + row0 * XS + d) = make_float2(o_acc[nt][0], o_acc[nt][1]);
      *reinterpret_cast<float2*>(xo + (row0 + 8) * XS + d) = make_float2(o_acc[nt][2], o_acc[nt][3]);
    }
    if ((lane & 3) == 0) {
      xml[row0 * 2] = m_r[0];
      xml[row0 * 2 + 1] = l_r[0];
      xml[(row0 + 8) * 2] = m_r[1];
      xml[(row0 + 8) * 2 + 1] = l_r[1];
    }
  }
  __syncthreads();
  if (kh == 0) {
#pragma unroll
    for (int hrow = 0; hrow < 2; ++hrow) {
      const int r = row0 + 8 * hrow;
      const float m2 = xml[r * 2], l2 = xml[r * 2 + 1];
      const float mm = fmaxf(m_r[hrow], m2);
      const float w1 = m_r[hrow] == -INFINITY ? 0.f : exp2f(m_r[hrow] - mm);
      const float w2 = m2 == -INFINITY ? 0.f : exp2f(m2 - mm);
#pragma unroll
      for (int nt = 0; nt < D / 8; ++nt) {
        const int d = 8 * nt + 2 * (lane & 3);
        const float2 o2 = *reinterpret_cast<const float2*>(xo + r * XS + d);
        *reinterpret_cast<uint32_t*>(ob_s + r * OS + d) =
            ptx::pack_bf16x2(o_acc[nt][2 * hrow] * w1 + o2.x * w2, o_acc[nt][2 * hrow + 1] * w1 + o2.y * w2);
      }
      if ((lane & 3) == 0) {
        mml[r * 2] = mm;
        mml[r * 2 + 1] = l_r[hrow] * w1 + l2 * w2;
      }
    }
  }
  __syncthreads();
  if (trace && tid == 0) trace[4] = ptx::globaltimer();
  cluster_wait();   // entry phase: every rank has started
  if (trace && tid == 0) trace[5] = ptx::globaltimer();
  // push every valid row (D bf16 = D*2 bytes) to the rank that combines it:
  // one warp per row, 16 bytes per lane
  {
    const uint32_t rcv = ptx::smem_u32(recv), rml = ptx::smem_u32(recv_ml);
    constexpr int CPRB = D / 8;   // 16-byte chunks per bf16 row
    for (int r = warp; r < a.S; r += 8) {
      const int owner = r / rpc, rl = r - owner * rpc;
      const uint32_t dst = ptx::mapa(rcv, (uint32_t)owner) + (uint32_t)((rank * rpc + rl) * D * 2);
      for (int ch = lane; ch < CPRB; ch += 32) {
        const uint4 v = *reinterpret_cast<const uint4*>(ob_s + r * OS + ch * 8);
        asm volatile("st.shared::cluster.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(dst + (uint32_t)(ch * 16)), "r"(v.x),
                     "r"(v.y), "r"(v.z), "r"(v.w)
                     : "memory");
      }
      if (lane == 0) {
        const uint32_t mdst = ptx::mapa(rml, (uint32_t)owner) + (uint32_t)((rank * rpc + rl) * 8);
        asm volatile("st.shared::cluster.v2.f32 [%0], {%1, %2};" ::"r"(mdst), "f"(mml[r * 2]), "f"(mml[r * 2 + 1])
                     : "memory");
      }
    }
  }
  if (trace && tid == 0) trace[6] = ptx::globaltimer();
  ptx::cluster_sync();
  if (trace && tid == 0) trace[7] = ptx::globaltimer();
  // combine the ranks' partials for my rows, in rank order
  const int r0 = rank * rpc, n_own = min(a.S, r0 + rpc) - r0;
  if (tid < n_own) {
    const int rl = tid;
    float mx = -INFINITY;
    for (int qr = 0; qr < nchunk; ++qr) mx = fmaxf(mx, recv_ml[(qr * rpc + rl) * 2]);
    float lsum = 0.f;
    for (int qr = 0; qr < nchunk; ++qr) {
      const float mq = recv_ml[(qr * rpc + rl) * 2];
      const float wq = mq == -INFINITY ? 0.f : exp2f(mq - mx);
      wq_s[rl * nchunk + qr] = wq;
      lsum = fmaf(wq, recv_ml[(qr * rpc + rl) * 2 + 1], lsum);
    }
    inv_s[rl] = 1.f / lsum;
  }
  __syncthreads();
  for (int idx = tid; idx < n_own * (D / 2); idx += 256) {
    const int rl = idx / (D / 2), d2 = idx - rl * (D / 2);
    float ox = 0.f, oy = 0.f;
    for (int qr = 0; qr < nchunk; ++qr) {
      const float2 v = __bfloat1622float2(
          *reinterpret_cast<const __nv_bfloat162*>(recv + (size_t)(qr * rpc + rl) * D + 2 * d2));
      ox = fmaf(wq_s[rl * nchunk + qr], v.x, ox);
      oy = fmaf(wq_s[rl * nchunk + qr], v.y, oy);
    }
    *reinterpret_cast<uint32_t*>(a.o + (((size_t)g * a.S + r0 + rl) * a.Hq + j) * D + 2 * d2) =
        ptx::pack_bf16x2(ox * inv_s[rl], oy * inv_s[rl]);
  }
  if (trace && tid == 0) trace[8] = ptx::globaltimer();
}

// ---------------------------------------------------------------------------
// Step kernel: output head of the previous Euler step and suffix embedding
// of the next ("DM0.5 reading guide", sec. 5.2 action_out_proj /
// action_in_proj / state token, sec. 5.3 Euler update x <- x - dt * v).
// One block per suffix token row; w/4 threads, 4 consecutive features each.
//   head  : v = action_out_proj(RMSNorm_final(h)) for action rows; then
//           x <- x - dt * v, or v stored to vout.
//   embed : h = state_proj(state) (token 0) or action_in_proj(x) + c (tokens
//           1..H), then the first layer's norm input bf16(h * (1 + g)) and the
//           per-128-feature sums of squares of h.
// ---------------------------------------------------------------------------
struct StepArgs {
  float* h;                       // [T][w]
  __nv_bfloat16* hb;              // [T][w]
  float* ssp;                     // [T][w/128]
  float* x;                       // [G][H][A]
  float* vout;                    // [G][H][A] or nullptr
  const float* state;             // [G or 1][Sd]
  const float* c;                 // time condition rows
  const __nv_bfloat16* w_ao;      // [A][w]
  const float* b_ao;
  const float* g_final;
  const __nv_bfloat16* w_aiT;     // [A][w]  (action_in_proj transposed)
  const float* b_ai;
  const __nv_bfloat16* w_spT;     // [Sd][w] (state_proj transposed)
  const float* b_sp;
  const float* g_attn0;           // first layer's attention-norm gain
  unsigned* status;
  int w, S, A, Sd, state_stride, c_stride, do_head, do_embed;
  float dt, eps;
};

__global__ void __launch_bounds__(256) step_kernel(const StepArgs a) {
  extern __shared__ float sm_step[];
  float* hn = sm_step;              // w
  float* xs = sm_step + a.w;        // 64: this row's input vector
  __shared__ float red[32];
  const int r = blockIdx.x;
  const int g = r / a.S, s = r - g * a.S;
  const int H = a.S - 1;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int i0 = 4 * tid;           // this thread's 4 consecutive features
  ptx::pdl_launch_dependents();
  ptx::pdl_wait();

  if (s > 0 && a.do_head) {
    const int jrow = s - 1;
    const float4 hv = *reinterpret_cast<const float4*>(a.h + (size_t)r * a.w + i0);
    float ss = hv.x * hv.x;
    ss = fmaf(hv.y, hv.y, ss);
    ss = fmaf(hv.z, hv.z, ss);
    ss = fmaf(hv.w, hv.w, ss);
    ss = block_sum(ss, red);
    const float inv = rsqrtf(ss / (float)a.w + a.eps);
    const float4 gf = *reinterpret_cast<const float4*>(a.g_final + i0);
    hn[i0] = hv.x * inv * (1.f + gf.x);
    hn[i0 + 1] = hv.y * inv * (1.f + gf.y);
    hn[i0 + 2] = hv.z * inv * (1.f + gf.z);
    hn[i0 + 3] = hv.w * inv * (1.f + gf.w);
    __syncthreads();
    // 8 threads per output, each w/8 consecutive inputs (16-byte weight loads)
    const int sub = tid & 7, per = a.w / 8;
    for (int a0 = tid >> 3; a0 < ((a.A + 31) / 32) * 32; a0 += blockDim.x >> 3) {
      float dot = 0.f;
      if (a0 < a.A) {
        const uint4* wr = reinterpret_cast<const uint4*>(a.w_ao + (size_t)a0 * a.w + sub * per);
        const float* hr = hn + sub * per;
        for (int q8 = 0; q8 < per / 8; ++q8) {
          const uint4 u = wr[q8];
          const __nv_bfloat162* b2 = reinterpret_cast<const __nv_bfloat162*>(&u);
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const float2 f2 = __bfloat1622float2(b2[e]);
            dot = fmaf(f2.x, hr[q8 * 8 + 2 * e], dot);
            dot = fmaf(f2.y, hr[q8 * 8 + 2 * e + 1], dot);
          }
        }
      }
      dot += __shfl_xor_sync(0xffffffffu, dot, 4);
      dot += __shfl_xor_sync(0xffffffffu, dot, 2);
      dot += __shfl_xor_sync(0xffffffffu, dot, 1);
      if (sub == 0 && a0 < a.A) {
        const float v = dot + a.b_ao[a0];
        const size_t off = ((size_t)g * H + jrow) * a.A + a0;
        if (a.vout) {
          a.vout[off] = v;
        } else {
          const float xn = a.x[off] - a.dt * v;
          a.x[off] = xn;
          xs[a0] = xn;
          if (!isfinite(xn)) atomicOr(a.status, RTV_DEV_NUMERIC);
        }
      }
    }
    __syncthreads();
  }
  if (!a.do_embed) return;
  // input vector of this row
  const int K = s == 0 ? a.Sd : a.A;
  if (!(s > 0 && a.do_head)) {
    const float* src = s == 0 ? a.state + (size_t)g * a.state_stride : a.x + ((size_t)g * H + (s - 1)) * a.A;
    for (int k = tid; k < K; k += blockDim.x) xs[k] = src[k];
    __syncthreads();
  }
  const __nv_bfloat16* WT = s == 0 ? a.w_spT : a.w_aiT;
  float acc[4] = {0.f, 0.f, 0.f, 0.f};
  for (int k = 0; k < K; ++k) {
    const uint2 u = *reinterpret_cast<const uint2*>(WT + (size_t)k * a.w + i0);
    const float2 f01 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&u.x));
    const float2 f23 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&u.y));
    const float xk = xs[k];
    acc[0] = fmaf(f01.x, xk, acc[0]);
    acc[1] = fmaf(f01.y, xk, acc[1]);
    acc[2] = fmaf(f23.x, xk, acc[2]);
    acc[3] = fmaf(f23.y, xk, acc[3]);
  }
  float hv[4];
  const float* bias = s == 0 ? a.b_sp : a.b_ai;
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    hv[e] = acc[e] + bias[i0 + e];
    if (s > 0) hv[e] += a.c[(size_t)g * a.c_stride + i0 + e];
  }
  *reinterpret_cast<float4*>(a.h + (size_t)r * a.w + i0) = make_float4(hv[0], hv[1], hv[2], hv[3]);
  const float4 ga = *reinterpret_cast<const float4*>(a.g_attn0 + i0);
  uint2 hbv;
  hbv.x = ptx::pack_bf16x2(hv[0] * (1.f + ga.x), hv[1] * (1.f + ga.y));
  hbv.y = ptx::pack_bf16x2(hv[2] * (1.f + ga.z), hv[3] * (1.f + ga.w));
  *reinterpret_cast<uint2*>(a.hb + (size_t)r * a.w + i0) = hbv;
  // each warp covers one 128-feature tile
  float sq = hv[0] * hv[0];
  sq = fmaf(hv[1], hv[1], sq);
  sq = fmaf(hv[2], hv[2], sq);
  sq = fmaf(hv[3], hv[3], sq);
  sq = warp_sum(sq);
  if (lane == 0) a.ssp[(size_t)r * (a.w >> 7) + warp] = sq;
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

// [rows][cols] -> [cols][rows]
__global__ void transpose_bf16_kernel(const __nv_bfloat16* __restrict__ src, __nv_bfloat16* __restrict__ dst,
                                      int rows, int cols) {
  for (int idx = blockIdx.x * blockDim.x + threadIdx.x; idx < rows * cols; idx += gridDim.x * blockDim.x) {
    const int r = idx / cols, c = idx - r * cols;
    dst[(size_t)c * rows + r] = src[idx];
  }
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
  __nv_bfloat16 *w_aiT = nullptr, *w_spT = nullptr;
  CUtensorMap map_qkv, map_o, map_gu, map_down;
  __nv_bfloat16 *qb = nullptr, *ksb = nullptr, *vsb = nullptr, *ob = nullptr, *mb = nullptr, *hb = nullptr;
  float* ssp = nullptr;
  int num_sms = 148;
  int max_cluster = 8;
  int attn_fit[17] = {0};      // co-resident clusters of attention CTAs, by cluster size
  int smem_cap = 112 * 1024;   // keeps two CTAs per SM so the next kernel can prefetch
  // optional phase trace of the four projections of layer 0 in the first Euler step
  unsigned long long* trace = nullptr;
  int trace_ctas[5] = {0, 0, 0, 0, 0};
  bool trace_armed = false;
  std::vector<void*> allocs;
};

namespace {

constexpr int kSmemOptin = 227 * 1024;
constexpr int kDynSmemMax = kSmemOptin - 2048;   // every kernel here uses < 2 KB of static shared memory

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

// 2-D row-major bf16 tensor [rows][K], box of 64 elements x box_rows rows, 128-byte swizzle.
bool make_map(CUtensorMap* map, const void* ptr, uint64_t rows, uint64_t K, uint32_t box_rows) {
  auto enc = get_encode();
  if (!enc) return false;
  cuuint64_t dims[2] = {K, rows};
  cuuint64_t strides[1] = {K * 2};
  cuuint32_t box[2] = {64, box_rows};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(ptr), dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

int round_up(int x, int m) { return (x + m - 1) / m * m; }

// Split of one projection over CTAs: 128-row weight tiles x K slices (one
// cluster per tile).  The smallest cluster that puts at least one CTA on
// every SM is taken; the ring depth is then the largest that fits the
// shared-memory budget.
GemmPlan plan_gemm(const FastPath* fp, int N, int K, int n_mma, int T) {
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
  // a grid of at most one CTA per SM may use the whole shared memory for its ring
  const int cap = best.n_tiles * best.cs <= fp->num_sms ? kDynSmemMax : fp->smem_cap;
  while (stages > 1 && gemm_smem_layout(stages, n_mma, best.cs, T).total > cap) --stages;
  best.stages = stages;
  best.smem = gemm_smem_layout(stages, n_mma, best.cs, T).total;
  best.valid = best.kslice >= 64 && best.smem <= kDynSmemMax && (T + best.cs - 1) / best.cs <= 64;
  return best;
}

template <int MODE>
cudaError_t launch_gemm(const CUtensorMap& map, const CUtensorMap& amap, const GemmArgs& a, const GemmPlan& pl,
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
  return cudaLaunchKernelEx(&cfg, kern, map, amap, args);
}

// Dynamic shared memory a kernel may request: the per-block opt-in limit
// minus room for the kernel's own static shared memory.
template <typename K>
cudaError_t configure_dyn_smem(K kern) {
  cudaFuncAttributes fa;
  cudaError_t e = cudaFuncGetAttributes(&fa, kern);
  if (e != cudaSuccess) return e;
  if (fa.sharedSizeBytes > (size_t)(kSmemOptin - kDynSmemMax)) return cudaErrorInvalidValue;
  return cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, kDynSmemMax);
}

// Kernel attributes are set once, outside any stream capture.
template <int MODE>
cudaError_t configure_gemm() {
  cudaError_t e = configure_dyn_smem(gemm_tc_kernel<MODE>);
  if (e == cudaSuccess) e = cudaFuncSetAttribute(gemm_tc_kernel<MODE>, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
  return e;
}

template <int D>
cudaError_t configure_attn() {
  cudaError_t e = configure_dyn_smem(attn_mma_kernel<D>);
  if (e == cudaSuccess) e = cudaFuncSetAttribute(attn_mma_kernel<D>, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
  return e;
}

// How many clusters of `cs` attention CTAs can run at once on this device.
template <int D>
int attn_clusters_that_fit(int cs, int S) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(cs, 1, 1);
  cfg.blockDim = dim3(256, 1, 1);
  cfg.dynamicSmemBytes = attn_smem_bytes(D, cs, (S + cs - 1) / cs);
  cudaLaunchAttribute at;
  at.id = cudaLaunchAttributeClusterDimension;
  at.val.clusterDim.x = cs;
  at.val.clusterDim.y = 1;
  at.val.clusterDim.z = 1;
  cfg.attrs = &at;
  cfg.numAttrs = 1;
  int n = 0;
  if (cudaOccupancyMaxActiveClusters(&n, attn_mma_kernel<D>, &cfg) != cudaSuccess) n = 0;
  cudaGetLastError();
  return n;
}

template <int D>
cudaError_t launch_attn(const AttnArgs& a, int nchunk, int G, cudaStream_t st) {
  auto kern = attn_mma_kernel<D>;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(nchunk, a.Hq, G);
  cfg.blockDim = dim3(256, 1, 1);
  cfg.dynamicSmemBytes = attn_smem_bytes(D, nchunk, (a.S + nchunk - 1) / nchunk);
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

cudaError_t launch_step(const StepArgs& a, int rows, cudaStream_t st) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(rows, 1, 1);
  cfg.blockDim = dim3(a.w / 4, 1, 1);
  cfg.dynamicSmemBytes = (size_t)(a.w + 64) * sizeof(float);
  cfg.stream = st;
  cudaLaunchAttribute attr;
  attr.id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr.val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = &attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, step_kernel, a);
}

// Attention split: the largest cluster (at most one rank per 32 keys) of
// which every (head, suffix) pair's cluster can run at once; ranks take
// ~equal key ranges.
int attn_chunks(const FastPath* fp, int nk, int n_clusters) {
  const int cap = std::max(1, (nk + 31) / 32);
  for (int c : {16, 12, 8, 6, 4, 2}) {
    if (c > cap) continue;
    if (fp->attn_fit[c] >= n_clusters) return c;
  }
  return std::max(1, std::min(8, cap));
}

}  // namespace

rtv_status fast_create(rtv_ctx* ctx) {
  const rtv_expert_config& k = ctx->cfg;
  ctx->use_fast = false;
  const int S = ctx->S;
  const int n_mma_max = round_up(ctx->Gmax * S, 16);
  const bool shape_ok = k.dtype == RTV_BF16 && (k.head_dim == 128 || k.head_dim == 256) && k.width % 128 == 0 &&
                        k.width <= 1024 && k.mlp_dim % 128 == 0 && (ctx->Q % 128) == 0 && S <= 64 &&
                        k.action_dim <= 64 && k.state_dim <= 64 && n_mma_max <= 256 && get_encode() != nullptr;
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
  for (int c : {2, 4, 6, 8, 12, 16})
    fp->attn_fit[c] = k.head_dim == 256 ? attn_clusters_that_fit<256>(c, S) : attn_clusters_that_fit<128>(c, S);
  const size_t T = ctx->Tmax;
  auto alloc = [&](void** p, size_t bytes) -> bool {
    if (cudaMalloc(p, bytes) != cudaSuccess) return false;
    fp->allocs.push_back(*p);
    return true;
  };
  bool ok = alloc((void**)&fp->qb, T * ctx->Q * 2) && alloc((void**)&fp->ob, T * ctx->Q * 2) &&
            alloc((void**)&fp->mb, T * (size_t)k.mlp_dim * 2) && alloc((void**)&fp->hb, T * (size_t)k.width * 2) &&
            alloc((void**)&fp->ssp, T * (size_t)(k.width / 128) * 4) &&
            alloc((void**)&fp->ksb, (size_t)ctx->Gmax * ctx->KV * S * 2) &&
            alloc((void**)&fp->vsb, (size_t)ctx->Gmax * ctx->KV * S * 2);
  if (!ok) {
    for (void* p : fp->allocs) cudaFree(p);
    delete fp;
    return RTV_ERR_OOM;
  }
  if (getenv("RTV_TRACE")) {
    if (cudaMalloc(&fp->trace, 5 * 512 * 16 * sizeof(unsigned long long)) == cudaSuccess) {
      fp->allocs.push_back(fp->trace);
      cudaMemset(fp->trace, 0, 5 * 512 * 16 * sizeof(unsigned long long));
    } else {
      fp->trace = nullptr;
    }
  }
  ctx->fast = fp;
  ctx->use_fast = true;
  return RTV_OK;
}

void fast_arm_trace(rtv_ctx* ctx) {
  if (ctx->fast && ctx->fast->trace) ctx->fast->trace_armed = true;
}

// Print the phase stamps of the last traced replay (diagnostic, RTV_TRACE set).
void fast_trace_report(rtv_ctx* ctx) {
  FastPath* fp = ctx->fast;
  if (!fp || !fp->trace || !fp->trace_ctas[0]) return;
  std::vector<unsigned long long> h(5 * 512 * 16);
  cudaDeviceSynchronize();
  cudaMemcpy(h.data(), fp->trace, h.size() * 8, cudaMemcpyDeviceToHost);
  const char* nm[5] = {"qkv", "o", "gu", "down", "attention"};
  const char* ev[2][13] = {{"start", "w_issued", "pdl", "first_full", "mma_issued", "done", "copied", "recv", "end",
                           "prefetched", "arrived", "iter0", "exit"},
                          {"start", "pdl", "tile0", "loop_end", "merged", "entry", "pushed", "synced", "end", "", "", "",
                           ""}};
  unsigned long long t_ref = ~0ull;
  for (int i = 0; i < 5; ++i)
    for (int c = 0; c < fp->trace_ctas[i]; ++c)
      if (h[((size_t)i * 512 + c) * 16]) t_ref = std::min(t_ref, h[((size_t)i * 512 + c) * 16]);
  const int order[5] = {0, 4, 1, 2, 3};
  for (int oi = 0; oi < 5; ++oi) {
    const int i = order[oi];
    fprintf(stderr, "[rtv trace] %s (%d CTAs), us after the first traced start: min / median / max\n", nm[i],
            fp->trace_ctas[i]);
    const int order_e[13] = {0, 1, 2, 3, 4, 5, 6, 9, 7, 10, 11, 8, 12};
    for (int ei = 0; ei < 13; ++ei) {
      const int e = order_e[ei];
      if (!ev[i == 4][e][0]) continue;
      std::vector<double> v;
      for (int c = 0; c < fp->trace_ctas[i]; ++c) {
        const unsigned long long t = h[((size_t)i * 512 + c) * 16 + e];
        if (t) v.push_back((double)(t - t_ref) * 1e-3);
      }
      if (v.empty()) continue;
      std::sort(v.begin(), v.end());
      fprintf(stderr, "    %-11s %8.2f %8.2f %8.2f\n", ev[i == 4][e], v.front(), v[v.size() / 2], v.back());
    }
  }
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
        alloc((void**)&fp->w_gu, Lh * ngu * w * 2) && alloc((void**)&fp->w_down, (size_t)Lh * w * F * 2) &&
        alloc((void**)&fp->w_aiT, (size_t)k.action_dim * w * 2) &&
        alloc((void**)&fp->w_spT, (size_t)k.state_dim * w * 2)))
    return RTV_ERR_OOM;
  // row orders of the packed tiles: a QKV tile holds the RoPE pairs (d, d + D/2)
  // of one head; a gate/up tile holds 64 gate rows and the matching 64 up rows
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
  transpose_bf16_kernel<<<64, 256>>>((const __nv_bfloat16*)ctx->W.ai_w, fp->w_aiT, w, k.action_dim);
  transpose_bf16_kernel<<<64, 256>>>((const __nv_bfloat16*)ctx->W.sp_w, fp->w_spT, w, k.state_dim);
  cudaError_t e = cudaDeviceSynchronize();
  cudaFree(d_iq);
  cudaFree(d_igu);
  if (e != cudaSuccess) return RTV_ERR_CUDA;
  if (!make_map(&fp->map_qkv, fp->w_qkv, Lh * nq, w, 128) || !make_map(&fp->map_o, fp->w_o, (size_t)Lh * w, Q, 128) ||
      !make_map(&fp->map_gu, fp->w_gu, Lh * ngu, w, 128) ||
      !make_map(&fp->map_down, fp->w_down, (size_t)Lh * w, F, 128))
    return RTV_ERR_CUDA;
  return RTV_OK;
}

rtv_status fast_step(rtv_ctx* ctx, int G, bool do_head, bool do_embed, float dt, const float* c, int c_stride,
                     int state_stride, bool velocity_only, cudaStream_t st) {
  FastPath* fp = ctx->fast;
  const rtv_expert_config& k = ctx->cfg;
  StepArgs a{};
  a.h = ctx->h;
  a.hb = fp->hb;
  a.ssp = fp->ssp;
  a.x = ctx->x;
  a.vout = velocity_only ? ctx->v : nullptr;
  a.state = ctx->state;
  a.c = c;
  a.w_ao = (const __nv_bfloat16*)ctx->W.ao_w;
  a.b_ao = ctx->W.ao_b;
  a.g_final = ctx->W.g_final;
  a.w_aiT = fp->w_aiT;
  a.b_ai = ctx->W.ai_b;
  a.w_spT = fp->w_spT;
  a.b_sp = ctx->W.sp_b;
  a.g_attn0 = ctx->W.layers[0].g_attn;
  a.status = ctx->status;
  a.w = k.width;
  a.S = ctx->S;
  a.A = k.action_dim;
  a.Sd = k.state_dim;
  a.state_stride = state_stride;
  a.c_stride = c_stride;
  a.do_head = do_head ? 1 : 0;
  a.do_embed = do_embed ? 1 : 0;
  a.dt = dt;
  a.eps = k.rms_eps;
  const cudaError_t e = launch_step(a, G * ctx->S, st);
  if (e != cudaSuccess) {
    ctx->last_error = std::string("step launch: ") + cudaGetErrorString(e);
    return RTV_ERR_CUDA;
  }
  return RTV_OK;
}

rtv_status fast_layers(rtv_ctx* ctx, int G, int P, int prefix_batch_stride, const float* rope_cs,
                       const float* rope_sn, cudaStream_t st) {
  FastPath* fp = ctx->fast;
  const rtv_expert_config& k = ctx->cfg;
  const int S = ctx->S, T = G * S, w = k.width, F = k.mlp_dim, D = k.head_dim, Q = ctx->Q, KV = ctx->KV;
  const int n_mma = round_up(T, 16);
  const int nq = Q + 2 * KV;
  const GemmPlan p_qkv = plan_gemm(fp, nq, w, n_mma, T);
  const GemmPlan p_o = plan_gemm(fp, w, Q, n_mma, T);
  const GemmPlan p_gu = plan_gemm(fp, 2 * F, w, n_mma, T);
  const GemmPlan p_dn = plan_gemm(fp, w, F, n_mma, T);
  const int nk = P + S;
  const int nchunk = attn_chunks(fp, nk, k.n_q_heads * G);
  if (!(p_qkv.valid && p_o.valid && p_gu.valid && p_dn.valid) ||
      attn_smem_bytes(D, nchunk, (S + nchunk - 1) / nchunk) > kDynSmemMax) {
    ctx->last_error = "no tensor-core split fits this token count";
    return RTV_ERR_UNSUPPORTED;
  }
  // activation tensor maps for this token count (rows beyond T read as zeros)
  CUtensorMap m_h, m_o, m_m;
  if (!make_map(&m_h, fp->hb, T, w, n_mma) || !make_map(&m_o, fp->ob, T, Q, n_mma) ||
      !make_map(&m_m, fp->mb, T, F, n_mma)) {
    ctx->last_error = "activation tensor map encoding failed";
    return RTV_ERR_CUDA;
  }
  if (getenv("RTV_LOG")) {
    const GemmPlan* pls[4] = {&p_qkv, &p_o, &p_gu, &p_dn};
    const char* nm[4] = {"qkv", "o", "gu", "down"};
    for (int i = 0; i < 4; ++i)
      fprintf(stderr, "[rtv] T=%d %s: tiles=%d cluster=%d kslice=%d stages=%d smem=%d\n", T, nm[i], pls[i]->n_tiles,
              pls[i]->cs, pls[i]->kslice, pls[i]->stages, pls[i]->smem);
    fprintf(stderr, "[rtv] attention: chunks=%d keys/chunk=%d smem=%d max_cluster=%d sms=%d fit(8,12,16)=%d,%d,%d\n",
            nchunk, (nk + nchunk - 1) / nchunk, attn_smem_bytes(D, nchunk, (S + nchunk - 1) / nchunk), fp->max_cluster,
            fp->num_sms, fp->attn_fit[8], fp->attn_fit[12], fp->attn_fit[16]);
  }

  GemmArgs base{};
  base.h = ctx->h;
  base.hb = fp->hb;
  base.ssp = fp->ssp;
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

  const bool tracing = fp->trace_armed && fp->trace != nullptr;
  fp->trace_armed = false;
  if (tracing) {
    fp->trace_ctas[0] = p_qkv.n_tiles * p_qkv.cs;
    fp->trace_ctas[1] = p_o.n_tiles * p_o.cs;
    fp->trace_ctas[2] = p_gu.n_tiles * p_gu.cs;
    fp->trace_ctas[3] = p_dn.n_tiles * p_dn.cs;
    fp->trace_ctas[4] = nchunk * k.n_q_heads * G;
  }
  auto tr = [&](int l, int i) -> unsigned long long* {
    return (tracing && l == 0) ? fp->trace + (size_t)i * 512 * 16 : nullptr;
  };

  for (int l = 0; l < k.n_layers; ++l) {
    const LayerW& Lw = ctx->W.layers[l];
    GemmArgs a = base;
    a.trace = tr(l, 0);
    a.w_row0 = l * nq;
    cudaError_t e = launch_gemm<GM_QKV>(fp->map_qkv, m_h, a, p_qkv, st);

    at.trace = tr(l, 4);
    at.pk = (const __nv_bfloat16*)ctx->prefix_kv + (size_t)(2 * l) * kv_layer;
    at.pv = (const __nv_bfloat16*)ctx->prefix_kv + (size_t)(2 * l + 1) * kv_layer;
    if (e == cudaSuccess) e = D == 256 ? launch_attn<256>(at, nchunk, G, st) : launch_attn<128>(at, nchunk, G, st);

    a = base;
    a.trace = tr(l, 1);
    a.w_row0 = l * w;
    a.g_next = Lw.g_mlp;
    if (e == cudaSuccess) e = launch_gemm<GM_O>(fp->map_o, m_o, a, p_o, st);

    a = base;
    a.trace = tr(l, 2);
    a.w_row0 = l * 2 * F;
    if (e == cudaSuccess) e = launch_gemm<GM_GU>(fp->map_gu, m_h, a, p_gu, st);

    a = base;
    a.trace = tr(l, 3);
    a.w_row0 = l * w;
    a.g_next = (l + 1 < k.n_layers) ? ctx->W.layers[l + 1].g_attn : nullptr;
    if (e == cudaSuccess) e = launch_gemm<GM_DOWN>(fp->map_down, m_m, a, p_dn, st);
    if (e != cudaSuccess) {
      ctx->last_error = std::string("tensor-core launch: ") + cudaGetErrorString(e);
      return RTV_ERR_CUDA;
    }
  }
  return RTV_OK;
}

void fast_destroy(rtv_ctx* ctx) {
  if (!ctx->fast) return;
  for (void* p : ctx->fast->allocs) cudaFree(p);
  delete ctx->fast;
  ctx->fast = nullptr;
}

}  // namespace rtv
