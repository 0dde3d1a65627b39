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
// slice.  Its first ring-full of weight boxes is fetched as soon as the CTA
// starts -- before it waits on the previous kernel, since weights do not
// depend on it -- and the bf16 activation boxes follow once that kernel has
// finished.  Weights and activations are stored tiled and pre-swizzled (see
// ts_offset), so every box is one contiguous bulk copy that lands in shared
// memory as a ready tensor-core operand.  The K slices of one weight tile form a thread-block cluster: each
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

// Attention mask of query rows that form a prefix attending to itself: the
// keys are the cached prefix only (internal; after the RTV_MASK_* values).
constexpr int kMaskPrefixOnly = 2;

// Element offset of (row t, column k) of a bf16 operand [rows][K] stored
// tiled and pre-swizzled: blocks of `block_rows` rows x 64 columns (128-byte
// rows, stacked densely), and inside a block the eight 16-byte chunks of row
// t permuted as chunk ^ (t % 8) -- the order in which the tensor cores' 128-byte
// swizzle reads a K-major operand.  A block copied byte for byte to a
// 1024-byte-aligned shared-memory address is therefore a ready operand tile.
// Activations use one block column per 64 inputs ([K/64][n_mma][64]);
// weights use 128-row tiles ([R/128][K/64][128][64]).
__host__ __device__ __forceinline__ size_t ts_offset(int t, int k, int block_rows) {
  return ((size_t)(k >> 6) * block_rows + t) * 64 + ((((k >> 3) & 7) ^ (t & 7)) << 3) + (k & 7);
}

// Two E4M3 codes (low byte first) -> two bf16 values, exactly: the hardware
// conversion to f16 holds every E4M3 value, and so does bf16.
__device__ __forceinline__ uint32_t e4m3x2_to_bf16x2(uint32_t two) {
  uint32_t h2;
  asm("{\n\t.reg .b16 t;\n\tcvt.u16.u32 t, %1;\n\tcvt.rn.f16x2.e4m3x2 %0, t;\n\t}" : "=r"(h2) : "r"(two));
  const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&h2));
  return ptx::pack_bf16x2(f.x, f.y);
}
__device__ __forceinline__ uint4 e4m3x8_to_bf16x8(uint2 v) {
  uint4 r;
  r.x = e4m3x2_to_bf16x2(v.x & 0xFFFFu);
  r.y = e4m3x2_to_bf16x2(v.x >> 16);
  r.z = e4m3x2_to_bf16x2(v.y & 0xFFFFu);
  r.w = e4m3x2_to_bf16x2(v.y >> 16);
  return r;
}

struct GemmArgs {
  const __nv_bfloat16* wt;    // packed weights of this projection, all layers [R/128][K/64][128][64]
  const __nv_bfloat16* act;   // bf16 input, tiled [K/64][n_mma][64]
  const uint8_t* wt8;         // FP8 E4M3 weights [R/128][K/64][128][64] bytes (GU, DOWN of an FP8 MLP), or nullptr
  const float* wscale;        // their per-row scales in packed row order, this layer
  const uint8_t* pf;          // weights of the next projection, brought into L2 while this one runs
  unsigned long long pf_bytes;
  float* h;                   // fp32 residual stream [T][w] (O, DOWN add into it)
  const float* h_in;          // O, DOWN: residual rows added to, when not h itself (nullptr: h)
  __nv_bfloat16* hb;          // next norm's input bf16(h * (1 + g_next)), tiled [w/64][n_mma][64] (written by O, DOWN)
  float* ssp;                 // sums of squares of h per 128-feature tile [T][w/128]
  const float* g_next;        // gain of the next RMSNorm, or nullptr when no norm consumer follows
  __nv_bfloat16* q;           // [T][Hq][D]
  __nv_bfloat16* ks;          // suffix keys   [G][Hkv][S][D]
  __nv_bfloat16* vs;          // suffix values [G][Hkv][S][D]
  // When qt is set, q/k/v go instead to the tensor-core attention's tiles:
  __nv_bfloat16* qt;          // q of head pairs [G][Hq/2][128 rows = 2 heads x 64][D], tiled (ts_offset, 128 rows)
  __nv_bfloat16* kts;         // suffix keys [G][Hkv][64][D], tiled (64 rows)
  __nv_bfloat16* vts;         // suffix values transposed [G][Hkv][D][64], tiled (D rows, 64 keys)
  const float* rope_cs;       // [S][D/2]
  const float* rope_sn;
  __nv_bfloat16* m;           // gelu(gate) * up, tiled [F/64][n_mma][64]
  unsigned* status;
  unsigned long long* trace;  // optional phase stamps [cta][16] (globaltimer ns), or nullptr
  long long timeout_ns;
  int T, n_mma, kslice, stages, w, S, Hq, Hkv, D, F, K, w_tile0;
  int tt;                     // token rows per CTA (a multiple of 16, <= 256); blockIdx.y picks the tile
  int nt_base;                // first 128-row weight tile of the grid within the layer (QKV: K/V tiles only)
  int kv_rows;                // row stride of ks / vs per (sequence, kv head)
  int seq;                    // QKV: tokens of one sequence -- RoPE position and ks/vs row are t % seq, the
                              // sequence t / seq (= S for suffixes; the prefix length for a prefix)
  int kv_prefix;              // QKV with qt set: keys and values still go to ks / vs rows, not to kts / vts
  // QKV writing keys and values as rows of a cached prefix (ks / vs): when
  // set, also its tensor-core tiles, keys [seq][Hkv][ntile_max][64][D] and
  // values transposed [seq][Hkv][ntile_max][D][64] (the layout the attention reads)
  __nv_bfloat16* pkt;
  __nv_bfloat16* pvt;
  int ntile_max;
  // Per-layer time modulator (each suffix group g = t / S reads its own row):
  int g_stride;               // O, DOWN: the next norm's gain is g_next + g * g_stride (0: one gain for all)
  const float* sb;            // QKV, GU: added after the 1/rms factor, sb[g * sb_stride + natural row]
  int sb_stride;
  const float* gate;          // O, DOWN: the branch is multiplied by gate[g * gate_stride + feature]
  int gate_stride;
  float eps;
};

// Phase stamps of the optional trace (one row of kTraceRow per CTA; GEMM
// rows also hold the landing time of the first 8 stages from slot 16 on).
constexpr int kTraceRow = 32;
enum { TR_START = 0, TR_W_ISSUED, TR_PDL, TR_FIRST_FULL, TR_MMA_ISSUED, TR_DONE, TR_COPIED, TR_RECV, TR_END,
       TR_PREFETCHED, TR_ARRIVED, TR_ITER0, TR_EXIT, TR_PART, TR_ENTRY };

struct GemmSmem {
  int stages, stage_bytes, ring_bytes, f8_off, part_off, recv_off, in_off, bar_off, total;
};

// Shared memory of one GEMM CTA: a ring of `stages` stages, each a 128x64
// bf16 weight box (16 KB) and the matching 64-wide bf16 activation box of
// n_mma token rows, both K-major with the 128-byte swizzle; the fp32 partial
// tile [n_mma][128] (over the ring once the MMAs are done, when it fits);
// the receive buffer [cs * per][128] of the cluster reduction; the
// epilogue's per-token inputs [per][128] (residual rows or RoPE cos/sin);
// mbarriers.
__host__ __device__ inline GemmSmem gemm_smem_layout(int stages, int n_mma, int cs, int T, bool with_in = true,
                                                     bool f8 = false) {
  GemmSmem s;
  const int per = (T + cs - 1) / cs;
  s.stages = stages;
  s.stage_bytes = 16384 + n_mma * 128;
  s.ring_bytes = stages * s.stage_bytes;
  s.f8_off = s.ring_bytes;   // FP8 weights: the E4M3 box of each stage, 8 KB, before widening
  const int core = s.ring_bytes + (f8 ? stages * 8192 : 0);
  const int part_bytes = n_mma * 512;
  s.part_off = 0;   // the partial tile overlays the ring: every MMA has completed when it is written
  if (cs == 1) {
    // a lone CTA owns every token: its partial tile is its receive buffer
    s.recv_off = s.part_off;
    s.in_off = core > part_bytes ? core : part_bytes;
  } else {
    s.recv_off = core > part_bytes ? core : part_bytes;
    s.in_off = s.recv_off + cs * per * 512;   // [per][128] fp32 epilogue inputs of the owned tokens
  }
  s.bar_off = s.in_off + (with_in ? per * 512 : 0);   // GU reads no per-token epilogue inputs
  s.total = s.bar_off + (4 * stages + 2) * 8 + 16 + 1024;   // barriers, TMEM slot, alignment slack
  return s;
}

// Limit of the waits that only drain work this CTA has already issued
// (copies and MMAs that complete without help from any other agent): after a
// timeout a CTA stops issuing, then waits this long at most for what is still
// in flight before it leaves.
constexpr long long kDrainNs = 200000000ll;

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
__device__ __forceinline__ void cluster_wait() { asm volatile("barrier.cluster.wait.aligned;" ::: "memory"); }

// Non-blocking test of the completion of phase `parity` of an mbarrier.
__device__ __forceinline__ bool mbar_test(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(ptx::smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}

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

// Warp roles of a GEMM CTA: warp 0 loads, warp 1 issues the MMAs, and
// kEpiWarps warps run the epilogue -- two per TMEM lane quarter, splitting
// the token columns -- so that its latency chains overlap.
constexpr int kEpiWarps = 8;
constexpr int kEpiThreads = 32 * kEpiWarps;
constexpr int kGemmThreads = 64 + kEpiThreads;

// (Two CTAs fit an SM by registers, so a grid a little larger than the SM
// count still runs in one wave.)
// F8: the weights are FP8 E4M3 codes (GU and DOWN of an FP8 MLP), a.wt8 set.
template <int MODE, bool F8>
__global__ void __launch_bounds__(kGemmThreads, 2) gemm_tc_kernel(const GemmArgs a) {
  extern __shared__ uint8_t smem_raw[];
  constexpr int kMaxOwn = 256;   // tokens one rank reduces and finishes
  __shared__ float rs_s[kMaxOwn];
  // Grid (K slice, token tile, weight tile): blockIdx.y takes token rows
  // [t0, t0 + n_mma) of the tiled activation layout, which has n_rows rows
  // per 64-column block (T of them real tokens); the token tiles of one
  // weight tile are adjacent in launch order, so they share its weight
  // boxes through L2.
  const int n_rows = a.n_mma;
  const int t0 = (int)blockIdx.y * a.tt;
  const int n_mma = min(a.tt, n_rows - t0);
  const int T = min(a.T - t0, n_mma);
  const int cs = gridDim.x;
  constexpr bool f8 = F8 && (MODE == GM_GU || MODE == GM_DOWN);
  const GemmSmem L = gemm_smem_layout(a.stages, n_mma, cs, T, MODE != GM_GU, f8);
  // every CTA of a cluster sees the same values, so a refusal is uniform across it
  if (dynamic_smem_size() < (uint32_t)L.total || (a.wt8 != nullptr) != f8 || a.kslice < 64 || (a.kslice & 63) ||
      a.stages < 1 || n_mma > 256 ||
      n_mma < 16 || (n_mma & 15) || (n_rows & 15) || T < 1 || T > n_mma || cs > 16 || (T + cs - 1) / cs > kMaxOwn) {
    if (threadIdx.x == 0) atomicOr(a.status, RTV_DEV_BOUNDS);
    return;
  }
  uint8_t* base = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = ptx::cluster_ctarank();
  const int nt = (int)blockIdx.z + a.nt_base;
  const int nbox = a.kslice >> 6;
  const int NS = L.stages;
  const int k0 = (int)rank * a.kslice;
  const int per = (T + cs - 1) / cs;                   // tokens owned by each rank in the reduction
  const int t_own0 = (int)rank * per;                  // (tile-local)
  const int n_own = max(0, min(T, t_own0 + per) - t_own0);
  float* part = (float*)(base + L.part_off);           // [n_mma][128] this CTA's partial sums
  float* recv = (float*)(base + L.recv_off);           // [cs][per][128] partials of the tokens I own
  // bf16: the stage's weight and activation boxes both land on wfull; FP8:
  // the weight box lands on wfull (the converters wait for it alone) and the
  // activation box on afull
  uint64_t* wfull = (uint64_t*)(base + L.bar_off);
  uint64_t* afull = wfull + NS;
  uint64_t* abar = f8 ? afull : wfull;                 // where the activation boxes land
  uint64_t* empty = afull + NS;                        // the stage's MMAs completed
  uint64_t* conv = empty + NS;                         // FP8: the stage's weights widened to bf16
  uint64_t* done = conv + NS;                          // all MMAs completed
  uint64_t* rbar = done + 1;                           // all partials of my tokens landed
  uint32_t* tmem_slot = (uint32_t*)(rbar + 1);
  const uint32_t ncols = (uint32_t)tmem_cols_for(n_mma);
  const uint32_t act_box_bytes = (uint32_t)n_mma * 128u;
  // this CTA's first weight box and first activation box
  const __nv_bfloat16* wsrc = a.wt + ((size_t)(a.w_tile0 + nt) * (a.K >> 6) + (k0 >> 6)) * 8192;
  const uint8_t* wsrc8 = f8 ? a.wt8 + ((size_t)(a.w_tile0 + nt) * (a.K >> 6) + (k0 >> 6)) * 8192 : nullptr;
  uint8_t* f8s = base + L.f8_off;                      // FP8 staging, 8 KB per stage
  const uint32_t wbox_bytes = f8 ? 8192u : 16384u;
  const __nv_bfloat16* asrc = a.act + ((size_t)(k0 >> 6) * n_rows + t0) * 64;
  const size_t trace_row = ((size_t)blockIdx.z * gridDim.y + blockIdx.y) * gridDim.x + blockIdx.x;
  unsigned long long* trace = (a.trace && trace_row < 512) ? a.trace + trace_row * kTraceRow : nullptr;
  if (trace && threadIdx.x == 0) trace[TR_START] = ptx::globaltimer();

  if (threadIdx.x == 0) {
    for (int i = 0; i < NS; ++i) {
      ptx::mbar_init(&wfull[i], f8 ? 1 : 2);
      ptx::mbar_init(&afull[i], 1);
      ptx::mbar_init(&empty[i], 1);
      ptx::mbar_init(&conv[i], kEpiWarps);
    }
    ptx::mbar_init(done, 1);
    ptx::mbar_init(rbar, 1);
    ptx::fence_mbar_init();
  }
  __syncthreads();
  cluster_arrive_relaxed();

  // Weights do not depend on the previous kernel: the first ring-full of
  // weight boxes is requested before anyone waits on that kernel.  Nothing
  // before the __syncthreads below waits on another role.
  const int first = nbox < NS ? nbox : NS;
  uint64_t pol = 0;
  if (warp == 0) {
    if (lane == 0) {
      pol = ptx::policy_evict_first();
      for (int b = 0; b < first; ++b) {
        ptx::mbar_expect_tx(&wfull[b], wbox_bytes);
        if (f8) ptx::bulk_load_hint(f8s + b * 8192, wsrc8 + (size_t)b * 8192, 8192u, &wfull[b], pol);
        else ptx::bulk_load_hint(base + b * L.stage_bytes, wsrc + (size_t)b * 8192, 16384u, &wfull[b], pol);
      }
      if (trace) trace[TR_W_ISSUED] = ptx::globaltimer();
    } else if (lane == 2 && a.pf && blockIdx.y == 0) {
      // this CTA's share of the next projection's weights, into L2 (a hint;
      // the CTAs of the first token tile split it)
      const unsigned long long n_cta = (unsigned long long)gridDim.x * gridDim.z;
      const unsigned long long share = ((a.pf_bytes + n_cta - 1) / n_cta + 15) & ~15ull;
      const unsigned long long lo = share * ((unsigned long long)blockIdx.z * gridDim.x + blockIdx.x);
      const unsigned long long hi = lo + share < a.pf_bytes ? lo + share : a.pf_bytes;
      for (unsigned long long off = lo; off < hi; off += 32768)
        ptx::prefetch_l2_bulk(a.pf + off, (uint32_t)(hi - off < 32768 ? hi - off : 32768));
    }
  } else if (warp == 1) {
    ptx::tmem_alloc(tmem_slot, ncols);
    ptx::tmem_relinquish();
    ptx::tc_fence_before();
  }
  __syncthreads();   // TMEM address published
  ptx::tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  // Dependents may launch only once this CTA holds its tensor memory: every
  // kernel here allocates before it lets the next one start, so an
  // allocation can only ever wait for CTAs of earlier kernels, which never
  // wait on later ones.
  ptx::pdl_launch_dependents();

  // After a bounded wait gives up, a role stops issuing copies and MMAs (so no
  // barrier ever sees an extra arrival), records the timeout, and still
  // reaches every cluster barrier; what it had issued is drained before exit.
  int n_issued = 0;   // lane 0: weight boxes, lane 1: activation boxes requested
  if (warp == 0) {
    // ---- producers: lane 0 streams the remaining weight boxes as stages free
    // up; lane 1 the activation boxes once the previous kernel is done (two
    // issuing threads keep more copies in flight per SM) ----
    if (lane == 0) {
      n_issued = first;
      for (int b = first; b < nbox; ++b) {
        const int s = b % NS, u = b / NS;
        if (!ptx::mbar_wait(&empty[s], (u - 1) & 1, a.timeout_ns)) {
          atomicOr(a.status, RTV_DEV_TIMEOUT);
          break;
        }
        ptx::mbar_expect_tx(&wfull[s], wbox_bytes);
        if (f8) ptx::bulk_load_hint(f8s + s * 8192, wsrc8 + (size_t)b * 8192, 8192u, &wfull[s], pol);
        else ptx::bulk_load_hint(base + s * L.stage_bytes, wsrc + (size_t)b * 8192, 16384u, &wfull[s], pol);
        n_issued = b + 1;
      }
    } else if (lane == 1) {
      ptx::pdl_wait();
      if (trace) trace[TR_PDL] = ptx::globaltimer();
      for (int b = 0; b < nbox; ++b) {
        const int s = b % NS, u = b / NS;
        if (b >= NS && !ptx::mbar_wait(&empty[s], (u - 1) & 1, a.timeout_ns)) {
          atomicOr(a.status, RTV_DEV_TIMEOUT);
          break;
        }
        ptx::mbar_expect_tx(&abar[s], act_box_bytes);
        ptx::bulk_load(base + s * L.stage_bytes + 16384, asrc + (size_t)b * n_rows * 64, act_box_bytes, &abar[s]);
        n_issued = b + 1;
      }
    }
  } else if (warp == 1) {
    // ---- MMA issue: one thread ----
    if (lane == 0) {
      const uint32_t idesc = ptx::idesc_bf16_f32(128, n_mma);
      uint64_t* wready = f8 ? conv : wfull;   // FP8: the converters have seen the stage land and widened it
      for (int b = 0; b < nbox; ++b) {
        const int s = b % NS, u = b / NS;
        if (!ptx::mbar_wait(&wready[s], u & 1, a.timeout_ns) || (f8 && !ptx::mbar_wait(&afull[s], u & 1, a.timeout_ns))) {
          atomicOr(a.status, RTV_DEV_TIMEOUT);
          break;
        }
        ptx::tc_fence_after();
        if (trace && b == 0) trace[TR_FIRST_FULL] = ptx::globaltimer();
        if (trace && b < 8) trace[16 + b] = ptx::globaltimer();
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
      // (also after a break: `done` then completes once the MMAs issued so far have)
      ptx::umma_commit(done);
      if (trace) trace[TR_MMA_ISSUED] = ptx::globaltimer();
    }
  } else {
    // ---- epilogue warps 2..9 ----
    const int tid = threadIdx.x - 64;
    // FP8 weights: per-row scales of this lane's features, and the widening
    // of every stage's E4M3 box into the bf16 operand tile.  The first
    // ring-full does not depend on the previous kernel, so it is widened
    // before waiting on that kernel; later boxes as their stages come round.
    const int f0 = 2 * lane;
    float2 ws1 = make_float2(1.f, 1.f), ws2 = make_float2(1.f, 1.f);
    bool conv_ok = true;
    auto widen = [&](int b) {
      const int s = b % NS, u = b / NS;
      if (!conv_ok) return;
      // (a warp-uniform decision: the __syncwarp below needs every lane)
      if (!__all_sync(0xffffffffu, ptx::mbar_wait(&wfull[s], u & 1, a.timeout_ns))) {
        if (lane == 0) atomicOr(a.status, RTV_DEV_TIMEOUT);
        conv_ok = false;   // the MMA warp then times out on conv[s] and stops issuing
        return;
      }
      const uint8_t* src = f8s + s * 8192;          // [128 rows][64 codes]
      uint8_t* dst = base + s * L.stage_bytes;       // [128 rows][64 bf16], 128-byte swizzle
      for (int q = tid; q < 1024; q += kEpiThreads) {
        const int r = q >> 3, c = q & 7;             // 8 codes -> one 16-byte chunk
        const uint2 codes = *reinterpret_cast<const uint2*>(src + r * 64 + c * 8);
        *reinterpret_cast<uint4*>(dst + r * 128 + ((c ^ (r & 7)) << 4)) = e4m3x8_to_bf16x8(codes);
      }
      ptx::fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) ptx::mbar_arrive(&conv[s]);
    };
    if (f8) {
      ws1 = *reinterpret_cast<const float2*>(a.wscale + nt * 128 + f0);
      ws2 = *reinterpret_cast<const float2*>(a.wscale + nt * 128 + 64 + f0);
      for (int b = 0; b < first; ++b) widen(b);
    }
    ptx::pdl_wait();   // this role reads and writes what earlier kernels produced
    if (tid == 0 && cs > 1) ptx::mbar_expect_tx(rbar, (uint32_t)(cs * n_own * 512));
    // Everything the epilogue reads from global memory depends only on earlier
    // kernels, so it is requested now, while the MMAs run: the owned tokens'
    // residual rows of this tile (O, DOWN) or their RoPE cos/sin (QKV) go to
    // shared memory by cp.async; 1/rms of the owned tokens (QKV, GU) too.
    float* in_s = (float*)(base + L.in_off);
    const int n_wt = a.w >> 7;
    const int tph = a.D >> 7, hd = a.D >> 1;
    const int hh = nt / tph, dq0 = 64 * (nt - (nt / tph) * tph);
    const bool rope = MODE == GM_QKV && hh < a.Hq + a.Hkv;
    const uint32_t in_a = ptx::smem_u32(in_s);
    if (MODE == GM_O || MODE == GM_DOWN) {
      for (int c = tid; c < n_own * 32; c += kEpiThreads) {
        const int tl = c >> 5, ch = c & 31;
        ptx::cp_async_16(in_a + (uint32_t)(c * 16),
                         (a.h_in ? a.h_in : a.h) + (size_t)(t0 + t_own0 + tl) * a.w + nt * 128 + ch * 4);
      }
    } else if (rope) {
      for (int c = tid; c < n_own * 32; c += kEpiThreads) {
        const int tl = c >> 5, ch = c & 31;   // chunks 0-15: cos, 16-31: sin (64 floats each)
        const int s = (t0 + t_own0 + tl) % a.seq;   // position in its sequence
        const float* src = (ch < 16 ? a.rope_cs : a.rope_sn) + (size_t)s * hd + dq0 + (ch & 15) * 4;
        ptx::cp_async_16(in_a + (uint32_t)(c * 16), src);
      }
    }
    // gains of the next norm for this lane's features (O, DOWN)
    const int n1 = nt * 128 + f0, n2 = n1 + 64;
    float2 gn1 = make_float2(0.f, 0.f), gn2 = make_float2(0.f, 0.f);
    if ((MODE == GM_O || MODE == GM_DOWN) && a.g_next) {
      gn1 = *reinterpret_cast<const float2*>(a.g_next + n1);
      gn2 = *reinterpret_cast<const float2*>(a.g_next + n2);
    }
    if ((MODE == GM_QKV || MODE == GM_GU) && tid < n_own) {
      float sst = 0.f;
      for (int j2 = 0; j2 < n_wt; ++j2) sst += a.ssp[(size_t)(t0 + t_own0 + tid) * n_wt + j2];
      rs_s[tid] = rsqrtf(sst / (float)a.w + a.eps);
    }
    if (f8)
      for (int b = first; b < nbox; ++b) widen(b);
    if (!ptx::mbar_wait(done, 0, a.timeout_ns)) {
      atomicOr(a.status, RTV_DEV_TIMEOUT);
      ptx::mbar_wait(done, 0, kDrainNs);   // the MMAs issued so far complete on their own
    }
    ptx::tc_fence_after();
    if (trace && tid == 0) trace[TR_DONE] = ptx::globaltimer();
    // accumulator -> this CTA's partial tile [token][feature]; the two warps
    // of a lane quarter take alternate 32-column chunks
    const int quarter = warp & 3;
    const int f = quarter * 32 + lane;
    for (int c = 32 * ((warp - 2) >> 2); c < n_mma; c += 64) {
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
    asm volatile("bar.sync 1, %0;" ::"n"(kEpiThreads) : "memory");
    if (trace && tid == 0) trace[TR_PART] = ptx::globaltimer();
    cluster_wait();   // entry phase: every rank has started and initialised its barriers
    if (trace && tid == 0) trace[TR_ENTRY] = ptx::globaltimer();
    if (cs > 1 && tid < cs) {   // one lane per destination rank
      const int r = tid;
      const uint32_t part_a = ptx::smem_u32(part), recv_a = ptx::smem_u32(recv), rbar_a = ptx::smem_u32(rbar);
      const int o0 = r * per, no = max(0, min(T, o0 + per) - o0);
      if (no > 0)
        bulk_copy_to_rank(ptx::mapa(recv_a + (uint32_t)(rank * per * 512), (uint32_t)r),
                          part_a + (uint32_t)(o0 * 512), (uint32_t)(no * 512), ptx::mapa(rbar_a, (uint32_t)r));
      if (trace && tid == 0) trace[TR_COPIED] = ptx::globaltimer();
    }
    ptx::cp_async_wait_all();
    asm volatile("bar.sync 1, %0;" ::"n"(kEpiThreads) : "memory");
    if (trace && tid == 0) trace[TR_PREFETCHED] = ptx::globaltimer();
    // (every rank sends its copies unconditionally, so a wait that runs out
    // still drains them before this CTA lets anyone leave)
    if (cs > 1 && !ptx::mbar_wait(rbar, 0, a.timeout_ns)) {
      atomicOr(a.status, RTV_DEV_TIMEOUT);
      ptx::mbar_wait(rbar, 0, kDrainNs);
    }
    if (trace && tid == 0) trace[TR_RECV] = ptx::globaltimer();
    // My incoming copies are complete (seen on rbar), so the copies that read
    // the senders' shared memory are done too; the arrive needs no ordering.
    cluster_arrive_relaxed();
    if (trace && tid == 0) trace[TR_ARRIVED] = ptx::globaltimer();

    // ---- reduction in rank order + epilogue for the tokens this rank owns ----
    // one warp per token; lane l takes features (2l, 2l+1) and (2l+64, 2l+65)
    const int ew = warp - 2;
#pragma unroll 1
    for (int tl = ew; tl < n_own; tl += kEpiWarps) {
      const int t = t0 + t_own0 + tl;   // global token row
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
      if (f8) {   // per-row scale of the FP8 weights (the split-K sum is linear in it)
        x1.x *= ws1.x;
        x1.y *= ws1.y;
        x2.x *= ws2.x;
        x2.y *= ws2.y;
      }
      if ((MODE == GM_O || MODE == GM_DOWN) && a.gate) {   // gated branch (time modulator)
        const float* gp = a.gate + (size_t)(t / a.S) * a.gate_stride;
        const float2 q1 = *reinterpret_cast<const float2*>(gp + n1);
        const float2 q2 = *reinterpret_cast<const float2*>(gp + n2);
        x1.x *= q1.x;
        x1.y *= q1.y;
        x2.x *= q2.x;
        x2.y *= q2.y;
      }
      if ((MODE == GM_O || MODE == GM_DOWN) && a.g_next && a.g_stride) {   // per-group gain of the next norm
        const float* gg = a.g_next + (size_t)(t / a.S) * a.g_stride;
        gn1 = *reinterpret_cast<const float2*>(gg + n1);
        gn2 = *reinterpret_cast<const float2*>(gg + n2);
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
          *reinterpret_cast<uint32_t*>(a.hb + ts_offset(t, n1, n_rows)) =
              ptx::pack_bf16x2(h1.x * (1.f + gn1.x), h1.y * (1.f + gn1.y));
          *reinterpret_cast<uint32_t*>(a.hb + ts_offset(t, n2, n_rows)) =
              ptx::pack_bf16x2(h2.x * (1.f + gn2.x), h2.y * (1.f + gn2.y));
          if (lane == 0) a.ssp[(size_t)t * n_wt + nt] = sq;
        }
      } else {
        const float rs = rs_s[tl];
        x1.x *= rs;
        x1.y *= rs;
        x2.x *= rs;
        x2.y *= rs;
        if (a.sb) {   // the modulator's shift carried through the projection (natural row order)
          const float* sbp = a.sb + (size_t)(t / a.S) * a.sb_stride;
          const int r1 = MODE == GM_GU ? 64 * nt + f0 : hh * a.D + dq0 + f0;
          const int r2 = MODE == GM_GU ? a.F + 64 * nt + f0 : hh * a.D + dq0 + hd + f0;
          x1.x += sbp[r1];
          x1.y += sbp[r1 + 1];
          x2.x += sbp[r2];
          x2.y += sbp[r2 + 1];
        }
        if (MODE == GM_GU) {
          *reinterpret_cast<uint32_t*>(a.m + ts_offset(t, nt * 64 + f0, n_rows)) =
              ptx::pack_bf16x2(gelu_tanh(x1.x) * x2.x, gelu_tanh(x1.y) * x2.y);
        } else {
          const int g = t / a.S, s = t - g * a.S;           // suffix group and row (q and suffix K/V tiles)
          float2 y1 = x1, y2 = x2;
          if (rope) {
            const float2 c = *reinterpret_cast<const float2*>(in_s + tl * 128 + f0);
            const float2 sn = *reinterpret_cast<const float2*>(in_s + tl * 128 + 64 + f0);
            y1 = make_float2(x1.x * c.x - x2.x * sn.x, x1.y * c.y - x2.y * sn.y);
            y2 = make_float2(x2.x * c.x + x1.x * sn.x, x2.y * c.y + x1.y * sn.y);
          }
          const int d1 = dq0 + f0, d2 = d1 + hd;
          if (a.qt && (hh < a.Hq || !a.kv_prefix)) {
            if (hh < a.Hq) {
              __nv_bfloat16* dst = a.qt + (size_t)(g * (a.Hq >> 1) + (hh >> 1)) * 128 * a.D;
              const int row = ((hh & 1) << 6) + s;
              *reinterpret_cast<uint32_t*>(dst + ts_offset(row, d1, 128)) = ptx::pack_bf16x2(y1.x, y1.y);
              *reinterpret_cast<uint32_t*>(dst + ts_offset(row, d2, 128)) = ptx::pack_bf16x2(y2.x, y2.y);
            } else if (hh < a.Hq + a.Hkv) {
              __nv_bfloat16* dst = a.kts + (size_t)(g * a.Hkv + (hh - a.Hq)) * 64 * a.D;
              *reinterpret_cast<uint32_t*>(dst + ts_offset(s, d1, 64)) = ptx::pack_bf16x2(y1.x, y1.y);
              *reinterpret_cast<uint32_t*>(dst + ts_offset(s, d2, 64)) = ptx::pack_bf16x2(y2.x, y2.y);
            } else {
              __nv_bfloat16* dst = a.vts + (size_t)(g * a.Hkv + (hh - a.Hq - a.Hkv)) * a.D * 64;
              dst[ts_offset(d1, s, a.D)] = __float2bfloat16_rn(y1.x);
              dst[ts_offset(d1 + 1, s, a.D)] = __float2bfloat16_rn(y1.y);
              dst[ts_offset(d2, s, a.D)] = __float2bfloat16_rn(y2.x);
              dst[ts_offset(d2 + 1, s, a.D)] = __float2bfloat16_rn(y2.y);
            }
          } else {
            const int sq = t / a.seq, sp = t - sq * a.seq;    // sequence and position (K/V rows)
            __nv_bfloat16* dst;
            if (hh < a.Hq) dst = a.q + ((size_t)t * a.Hq + hh) * a.D;
            else if (hh < a.Hq + a.Hkv) dst = a.ks + (((size_t)sq * a.Hkv + (hh - a.Hq)) * a.kv_rows + sp) * a.D;
            else dst = a.vs + (((size_t)sq * a.Hkv + (hh - a.Hq - a.Hkv)) * a.kv_rows + sp) * a.D;
            *reinterpret_cast<uint32_t*>(dst + d1) = ptx::pack_bf16x2(y1.x, y1.y);
            *reinterpret_cast<uint32_t*>(dst + d2) = ptx::pack_bf16x2(y2.x, y2.y);
            if (a.pkt && hh >= a.Hq) {   // the same key or value in the prefix's tiles
              const bool is_k = hh < a.Hq + a.Hkv;
              const int kh = is_k ? hh - a.Hq : hh - a.Hq - a.Hkv;
              const size_t tile = ((size_t)sq * a.Hkv + kh) * a.ntile_max + (sp >> 6);
              const int key = sp & 63;
              if (is_k) {
                __nv_bfloat16* kt = a.pkt + tile * 64 * a.D;
                *reinterpret_cast<uint32_t*>(kt + ts_offset(key, d1, 64)) = ptx::pack_bf16x2(y1.x, y1.y);
                *reinterpret_cast<uint32_t*>(kt + ts_offset(key, d2, 64)) = ptx::pack_bf16x2(y2.x, y2.y);
              } else {
                __nv_bfloat16* vt = a.pvt + tile * 64 * a.D;
                vt[ts_offset(d1, key, a.D)] = __float2bfloat16_rn(y1.x);
                vt[ts_offset(d1 + 1, key, a.D)] = __float2bfloat16_rn(y1.y);
                vt[ts_offset(d2, key, a.D)] = __float2bfloat16_rn(y2.x);
                vt[ts_offset(d2 + 1, key, a.D)] = __float2bfloat16_rn(y2.y);
              }
            }
          }
        }
      }
      if (trace && tid == 0 && tl == 0) trace[TR_ITER0] = ptx::globaltimer();
    }
    if (trace && tid == 0) trace[TR_END] = ptx::globaltimer();
  }
  if (warp < 2) {
    cluster_wait();             // entry phase
    cluster_arrive_relaxed();   // nothing incoming to wait for
  }
  cluster_wait();   // every rank's incoming copies are complete: no copy still reads my shared memory
  if (trace && threadIdx.x == 64) trace[TR_EXIT] = ptx::globaltimer();
  if (warp == 1) {
    ptx::tc_fence_after();
    ptx::tmem_dealloc(tmem, ncols);
  }
  // Never leave with a copy still landing in this CTA's shared memory: each
  // producer checks the last box it requested on every stage (copies land in
  // order of request per stage, so that is the newest phase of the stage).
  // Unless a wait ran out, every one was consumed by a completed MMA and the
  // check is a single non-blocking test; otherwise it waits for the copy.
  if (warp == 0 && lane < 2) {
    uint64_t* landed = lane == 0 ? wfull : abar;
    for (int s2 = 0; s2 < NS && s2 < n_issued; ++s2) {
      const int b_last = s2 + NS * ((n_issued - 1 - s2) / NS);
      const uint32_t par = (uint32_t)(b_last / NS) & 1;
      if (!mbar_test(&landed[s2], par) && !ptx::mbar_wait(&landed[s2], par, kDrainNs))
        atomicOr(a.status, RTV_DEV_TIMEOUT);
    }
  }
}

// ---------------------------------------------------------------------------
// Split-KV grouped-query attention for one (query head, suffix) per cluster
// ("DM0.5 reading guide", sec. 5.1-5.2: suffix queries over the cached prefix
// KV and the bidirectional suffix; optional Pi0 block mask for the state
// token).  The cluster's CTAs take consecutive key ranges of [prefix ; own
// suffix] in tiles of 64 keys; warp w of a CTA owns query rows 16w..16w+15
// and runs a flash-style online softmax over all of the CTA's keys on
// warp-level bf16 MMAs (fp32 accumulate).  Each CTA then writes its
// unnormalised partial rows and their (max, sum) to global memory (they stay
// in L2), the cluster synchronises, and every rank combines the rows it owns,
// in rank order.
// ---------------------------------------------------------------------------
struct AttnArgs {
  const __nv_bfloat16* q;    // [T][Hq][D]
  const __nv_bfloat16* pk;   // this layer's prefix keys   [Bmax][Hkv][Pmax][D]
  const __nv_bfloat16* pv;   // this layer's prefix values
  const __nv_bfloat16* sk;   // suffix keys   [G][Hkv][S][D]
  const __nv_bfloat16* sv;
  __nv_bfloat16* o;          // attention output, tiled [Hq*D/64][n_mma][64]
  __nv_bfloat16* part_o;     // partial rows [G][Hq][nchunk][64][D] (scratch)
  float* part_ml;            // their (max, sum) [G][Hq][nchunk][64][2]
  unsigned* status;
  unsigned long long* trace; // optional phase stamps [cta][kTraceRow], or nullptr
  int S, P, Pmax, Hq, Hkv, pbs, mask_mode, kpc, n_mma;
  float scale_log2;
};

// Q, K and V tiles of 64 rows; once a warp is done with the keys, its rows
// of the Q tile stage its partial rows on their way to global memory.
__host__ __device__ inline int attn_smem_bytes(int D) { return 3 * 64 * D * 2; }

template <int D>
__global__ void __launch_bounds__(128) attn_mma_kernel(const AttnArgs a) {
  extern __shared__ __align__(128) uint8_t sm_attn[];
  constexpr int CPR = D / 8;           // 16-byte chunks per row
  const int nchunk = gridDim.x;
  const int rpc = (a.S + nchunk - 1) / nchunk;   // query rows combined by each rank
  // every CTA of the grid sees the same values, so a refusal is uniform
  if (dynamic_smem_size() < (uint32_t)attn_smem_bytes(D) || a.S > 64 || nchunk > 16) {
    if (threadIdx.x == 0) atomicOr(a.status, RTV_DEV_BOUNDS);
    return;
  }
  __nv_bfloat16* Qs = reinterpret_cast<__nv_bfloat16*>(sm_attn);
  __nv_bfloat16* Ks = Qs + 64 * D;
  __nv_bfloat16* Vs = Ks + 64 * D;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
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
      (a.trace && ((size_t)blockIdx.z * gridDim.y + blockIdx.y) * gridDim.x + blockIdx.x < 512)
          ? a.trace + (((size_t)blockIdx.z * gridDim.y + blockIdx.y) * gridDim.x + blockIdx.x) * kTraceRow
          : nullptr;
  if (trace && tid == 0) trace[0] = ptx::globaltimer();
  ptx::pdl_launch_dependents();

  const uint32_t qs_a = ptx::smem_u32(Qs), ks_a = ptx::smem_u32(Ks), vs_a = ptx::smem_u32(Vs);
  // K/V rows [lo, hi) of the 64-key tile starting at kt (keys past ke read as zeros)
  auto load_kv = [&](int kt, int lo, int hi) {
    for (int c = tid; c < 64 * CPR; c += 128) {
      const int r = c / CPR, ch = c - r * CPR;
      const int n = kt + r;
      if (n < lo || n >= hi) continue;
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
  };
  // The cached prefix does not depend on the previous kernel: the first
  // tile's prefix rows are requested before waiting on it.
  const int p_end = min(a.P, ke);
  load_kv(kb, kb, p_end);
  ptx::pdl_wait();
  if (trace && tid == 0) trace[1] = ptx::globaltimer();

  for (int c = tid; c < 64 * CPR; c += 128) {
    const int r = c / CPR, ch = c - r * CPR;
    const uint32_t off = (uint32_t)((r * D + ((ch ^ (r & 7)) << 3)) * 2);
    if (r < a.S) ptx::cp_async_16(qs_a + off, a.q + (((size_t)g * a.S + r) * a.Hq + j) * D + ch * 8);
    else *reinterpret_cast<uint4*>(reinterpret_cast<uint8_t*>(Qs) + off) = make_uint4(0, 0, 0, 0);
  }

  float o_acc[D / 8][4];
#pragma unroll
  for (int i = 0; i < D / 8; ++i) o_acc[i][0] = o_acc[i][1] = o_acc[i][2] = o_acc[i][3] = 0.f;
  float m_r[2] = {-INFINITY, -INFINITY}, l_r[2] = {0.f, 0.f};
  const int row0 = 16 * warp + (lane >> 2);

  for (int kt = kb; kt < ke; kt += 64) {
    if (kt == kb) {
      load_kv(kt, p_end, kt + 64);   // suffix rows and the zero tail of the first tile
    } else {
      __syncthreads();
      load_kv(kt, kt, kt + 64);
    }
    ptx::cp_async_wait_all();
    __syncthreads();
    if (trace && tid == 0 && kt == kb) trace[2] = ptx::globaltimer();
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
        const int r = 16 * kb2 + (lane & 7) + (((lane >> 3) & 1) << 3), ch = 2 * dn + (lane >> 4);
        ptx::ldmatrix_x4_trans(bf, vs_a + (uint32_t)((r * D + ((ch ^ (r & 7)) << 3)) * 2));
        ptx::mma_bf16_16816(o_acc[2 * dn], pf, bf[0], bf[1]);
        ptx::mma_bf16_16816(o_acc[2 * dn + 1], pf, bf[2], bf[3]);
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
  // This rank's partial rows: each warp stages its 16 rows (bf16,
  // chunk-swizzled) in its own rows of the Q tile, which no other warp reads,
  // then copies the valid ones to global memory with 16-byte stores.
  __syncwarp();
#pragma unroll
  for (int nt = 0; nt < D / 8; ++nt) {
#pragma unroll
    for (int hrow = 0; hrow < 2; ++hrow) {
      const int r = row0 + 8 * hrow;
      *reinterpret_cast<uint32_t*>(Qs + r * D + ((nt ^ (r & 7)) << 3) + 2 * (lane & 3)) =
          ptx::pack_bf16x2(o_acc[nt][2 * hrow], o_acc[nt][2 * hrow + 1]);
    }
  }
  __syncwarp();
  const size_t part_base = (size_t)(g * a.Hq + j) * nchunk;   // partial slot of rank q: part_base + q
  {
    __nv_bfloat16* po = a.part_o + (part_base + rank) * 64 * D;
    for (int r = 16 * warp; r < min(a.S, 16 * warp + 16); ++r)
      for (int ch = lane; ch < CPR; ch += 32)
        *reinterpret_cast<uint4*>(po + (size_t)r * D + ch * 8) =
            *reinterpret_cast<const uint4*>(Qs + r * D + ((ch ^ (r & 7)) << 3));
    float* pml = a.part_ml + (part_base + rank) * 64 * 2;
    if ((lane & 3) == 0) {
      if (row0 < a.S) *reinterpret_cast<float2*>(pml + row0 * 2) = make_float2(m_r[0], l_r[0]);
      if (row0 + 8 < a.S) *reinterpret_cast<float2*>(pml + (row0 + 8) * 2) = make_float2(m_r[1], l_r[1]);
    }
  }
  if (trace && tid == 0) trace[4] = ptx::globaltimer();
  // release / acquire at cluster scope: every rank's partials are visible
  ptx::cluster_sync();
  if (trace && tid == 0) trace[5] = trace[6] = trace[7] = ptx::globaltimer();
  // combine: one warp per owned row; lane q < nchunk weighs rank q's partial,
  // and the D outputs of the row are taken 8 per lane, ranks summed in order.
  // All of a lane's loads are issued before any is used.
  const int r0 = rank * rpc, n_own = max(0, min(a.S, r0 + rpc) - r0);
  for (int rl = warp; rl < n_own; rl += 4) {
    const int r = r0 + rl;
    float mq = -INFINITY, lq = 0.f;
    if (lane < nchunk) {
      const float2 ml = __ldcg(reinterpret_cast<const float2*>(a.part_ml + ((part_base + lane) * 64 + r) * 2));
      mq = ml.x;
      lq = ml.y;
    }
    for (int ch0 = 0; ch0 < CPR; ch0 += 32) {
      const int ch = ch0 + lane;
      uint4 v[16];
#pragma unroll
      for (int q = 0; q < 16; ++q)
        if (q < nchunk && ch < CPR)
          v[q] = __ldcg(reinterpret_cast<const uint4*>(a.part_o + ((part_base + q) * 64 + r) * D + ch * 8));
      const float mx = warp_max(mq);
      const float wq = (lane < nchunk && mq != -INFINITY) ? exp2f(mq - mx) : 0.f;
      const float inv = 1.f / warp_sum(wq * lq);
      float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int q = 0; q < 16; ++q) {
        const float wqq = __shfl_sync(0xffffffffu, wq, q);
        if (q < nchunk && ch < CPR) {
          const __nv_bfloat162* v2 = reinterpret_cast<const __nv_bfloat162*>(&v[q]);
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const float2 f = __bfloat1622float2(v2[e]);
            acc[2 * e] = fmaf(wqq, f.x, acc[2 * e]);
            acc[2 * e + 1] = fmaf(wqq, f.y, acc[2 * e + 1]);
          }
        }
      }
      if (ch < CPR) {
        uint4 out;
        out.x = ptx::pack_bf16x2(acc[0] * inv, acc[1] * inv);
        out.y = ptx::pack_bf16x2(acc[2] * inv, acc[3] * inv);
        out.z = ptx::pack_bf16x2(acc[4] * inv, acc[5] * inv);
        out.w = ptx::pack_bf16x2(acc[6] * inv, acc[7] * inv);
        *reinterpret_cast<uint4*>(a.o + ts_offset(g * a.S + r, j * D + ch * 8, a.n_mma)) = out;
      }
    }
  }
  if (trace && tid == 0) trace[8] = ptx::globaltimer();
}

// ---------------------------------------------------------------------------
// Attention on the tensor cores, for head pairs that share a KV head
// ("DM0.5 reading guide", sec. 5.1-5.2; same computation as the kernel above).
// A cluster owns one (head pair, suffix); rank c takes key tile c of
// [prefix tiles of 64 keys ; the suffix tile].  Rows are the 2 x 64 query
// rows of the pair (rows past the suffix length are padding).
//   S = Q K^T         tcgen05, M = 128 rows, N = 64 keys, K = D  -> TMEM
//   P = exp2(S - max)  one thread per row, straight from TMEM, P -> shared memory (bf16)
//   O = P V            tcgen05, M = 128, N = D, K = 64 keys, with V^T as the K-major operand -> TMEM
// Each rank writes its unnormalised O rows and (max, sum) to global memory,
// the cluster synchronises, and every rank combines the rows it owns, in
// rank order, as in the kernel above.  Q, K and V^T arrive as tiled,
// pre-swizzled blocks (ts_offset), one bulk copy each; the prefix tiles are
// requested before waiting on the previous kernel.
// ---------------------------------------------------------------------------
struct AttnTcArgs {
  const __nv_bfloat16* qt;    // [G][Hq/2][128][D] tiled
  const __nv_bfloat16* pkt;   // this layer's prefix key tiles   [Bmax][Hkv][ntile_max][64][D]
  const __nv_bfloat16* pvt;   // this layer's prefix value tiles [Bmax][Hkv][ntile_max][D][64] (transposed)
  const __nv_bfloat16* kts;   // suffix key tiles   [G][Hkv][64][D]
  const __nv_bfloat16* vts;   // suffix value tiles [G][Hkv][D][64]
  __nv_bfloat16* o;           // attention output, tiled [Hq*D/64][n_mma][64]
  __nv_bfloat16* part_o;      // partial rows [G][Hq/2][nchunk][128][D] (scratch)
  float* part_ml;             // their (max, sum) [G][Hq/2][nchunk][128][2]
  unsigned* status;
  unsigned long long* trace;  // optional phase stamps [cta][kTraceRow], or nullptr
  long long timeout_ns;
  int S, P, Hq, Hkv, pbs, mask_mode, ntile_max, n_mma;
  // 1: the prefix tiles are written by the kernel just before this one (the
  // draft model's visual keys and values), so they are requested only after
  // the dependency wait; 0: they were written before it and are requested first
  int prefix_after_wait;
  float scale_log2;
};

// Shared memory.  Separate tiles: Q (later the staged O rows), K, V^T, P,
// with K and V^T requested before the dependency wait (145 KB at D = 256: one
// CTA per SM).  Compact: the Q tile (later V^T, then the O rows) and the K
// tile (later P) only, V^T requested once S is done (97 KB: two CTAs per SM,
// for grids larger than the SM count).  Then barriers, TMEM slot, alignment.
__host__ __device__ inline int attn_tc_smem_bytes(int D, bool compact) {
  return compact ? 128 * D * 2 + 64 * D * 2 + 64 + 1024 : 128 * D * 2 + 2 * 64 * D * 2 + 128 * 128 + 64 + 1024;
}

template <int D, bool COMPACT>
__global__ void __launch_bounds__(256, 2) attn_tc_kernel(const AttnTcArgs a) {
  extern __shared__ uint8_t sm_atc[];
  __shared__ float red_m[2][128], red_l[2][128];   // per-row partial max / sum of the two column halves
  __shared__ int s_timeout;                        // a wait of this CTA ran out: drain before leaving
  constexpr int QB = 128 * D * 2, KB = 64 * D * 2, VB = D * 64 * 2, PB = 128 * 128;
  // Tensor memory: S in columns [0, 64), then O in columns [0, D) -- the PV
  // MMA is issued only after every thread has read S.  At most D <= 256
  // columns, so two CTAs sharing an SM (two attention CTAs, which a grid
  // larger than the SM count places together, or one beside a GEMM CTA of
  // at most 256 columns; shared memory admits no third) never exceed the 512
  // columns.  An allocation can only wait for a CTA of an earlier kernel,
  // which never waits on a later one.
  constexpr uint32_t TCOLS = D;
  constexpr int CPR = D / 8;
  const int nch = gridDim.x;
  const int ntp = (a.P + 63) / 64;   // prefix tiles; rank ntp holds the suffix tile
  // every CTA of the grid sees the same values, so a refusal is uniform
  if (dynamic_smem_size() < (uint32_t)attn_tc_smem_bytes(D, COMPACT) || a.S > 64 || nch != ntp + 1 || nch > 16 ||
      ntp > a.ntile_max) {
    if (threadIdx.x == 0) atomicOr(a.status, RTV_DEV_BOUNDS);
    return;
  }
  // Compact: Q and K are read only by the S MMA; once it has completed, V^T
  // lands in the Q tile's space (its copy overlaps the softmax) and P is
  // written over K.
  uint8_t* Qs = (uint8_t*)(((uintptr_t)sm_atc + 1023) & ~(uintptr_t)1023);
  uint8_t* Ks = Qs + QB;
  uint8_t* Vs = COMPACT ? Qs : Ks + KB;
  uint8_t* Ps = COMPACT ? Ks : Vs + VB;
  static_assert(VB <= QB && PB <= KB, "V^T and P reuse the Q and K tiles");
  // 0: K (and V^T, separate tiles) landed, 1: Q landed, 2: S done, 3: O done,
  // 4: V^T landed (compact)
  uint64_t* bars = (uint64_t*)(COMPACT ? Ks + KB : Ps + PB);
  uint32_t* tslot = (uint32_t*)(bars + 5);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  // warps w and w + 4 share TMEM lanes 32(w%4).. (rows) and split the columns
  const int quarter = warp & 3, half = warp >> 2;
  const uint32_t lane_base = (uint32_t)(32 * quarter) << 16;
  const int rank = (int)ptx::cluster_ctarank();
  const int hp = blockIdx.y, g = blockIdx.z;
  const int HP = a.Hq >> 1;
  const int kvh = (2 * hp * a.Hkv) / a.Hq;
  const bool suffix_tile = rank == ntp;
  unsigned long long* trace =
      (a.trace && ((size_t)blockIdx.z * gridDim.y + blockIdx.y) * gridDim.x + blockIdx.x < 512)
          ? a.trace + (((size_t)blockIdx.z * gridDim.y + blockIdx.y) * gridDim.x + blockIdx.x) * kTraceRow
          : nullptr;
  if (trace && tid == 0) trace[0] = ptx::globaltimer();
  if (tid == 0) {
    s_timeout = 0;
    for (int i = 0; i < 5; ++i) ptx::mbar_init(&bars[i], 1);
    ptx::fence_mbar_init();
  }
  if (warp == 0) {
    ptx::tmem_alloc(tslot, TCOLS);
    ptx::tmem_relinquish();
  }
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  const uint32_t tmem = *tslot;
  ptx::pdl_launch_dependents();
  // the cached prefix does not depend on the previous kernel
  // (rank ntp holds the suffix tile, produced by the previous kernel)
  const size_t kv_tile = suffix_tile ? (size_t)g * a.Hkv + kvh
                                     : ((size_t)(g * a.pbs) * a.Hkv + kvh) * a.ntile_max + rank;
  const __nv_bfloat16* vsrc = (suffix_tile ? a.vts : a.pvt) + kv_tile * 64 * D;
  auto load_prefix_tile = [&]() {
    ptx::mbar_expect_tx(&bars[0], (uint32_t)(COMPACT ? KB : KB + VB));
    ptx::bulk_load(Ks, a.pkt + kv_tile * 64 * D, (uint32_t)KB, &bars[0]);
    if (!COMPACT) ptx::bulk_load(Vs, vsrc, (uint32_t)VB, &bars[0]);
  };
  if (tid == 0 && !suffix_tile && !a.prefix_after_wait) load_prefix_tile();
  ptx::pdl_wait();
  if (tid == 0 && !suffix_tile && a.prefix_after_wait) load_prefix_tile();
  if (trace && tid == 0) trace[1] = ptx::globaltimer();
  bool ok = true;
  if (tid == 0) {
    if (suffix_tile) {
      ptx::mbar_expect_tx(&bars[0], (uint32_t)(COMPACT ? KB : KB + VB));
      ptx::bulk_load(Ks, a.kts + kv_tile * 64 * D, (uint32_t)KB, &bars[0]);
      if (!COMPACT) ptx::bulk_load(Vs, vsrc, (uint32_t)VB, &bars[0]);
    }
    ptx::mbar_expect_tx(&bars[1], (uint32_t)QB);
    const uint8_t* qsrc = reinterpret_cast<const uint8_t*>(a.qt + (size_t)(g * HP + hp) * 128 * D);
    for (int c = 0; c < QB; c += 16384) ptx::bulk_load(Qs + c, qsrc + c, 16384u, &bars[1]);
  }
  if (tid == 0) {
    ok = ptx::mbar_wait(&bars[1], 0, a.timeout_ns) && ptx::mbar_wait(&bars[0], 0, a.timeout_ns);
    if (!ok) atomicOr(&s_timeout, 1);
    if (ok) {
      if (trace) trace[2] = ptx::globaltimer();
      ptx::tc_fence_after();
      const uint32_t idesc = ptx::idesc_bf16_f32(128, 64);
      const uint32_t qa = ptx::smem_u32(Qs), ka = ptx::smem_u32(Ks);
#pragma unroll
      for (int kb = 0; kb < D / 64; ++kb)
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)
          ptx::umma_bf16(tmem, ptx::sw128_kmajor_desc(qa + kb * 16384 + kk * 32),
                         ptx::sw128_kmajor_desc(ka + kb * 8192 + kk * 32), idesc, (kb | kk) != 0 ? 1u : 0u);
      ptx::umma_commit(&bars[2]);
    } else {
      atomicOr(a.status, RTV_DEV_TIMEOUT);
    }
  }
  __syncwarp();   // the rest of warp 0 waits here, not spinning beside the issuing lane
  // ---- softmax: a row (TMEM lane) per thread pair, 32 key columns each ----
  const int r = 32 * quarter + lane;
  const int s = r & 63;
  const bool row_valid = s < a.S;
  // (a prefix attending to itself has no suffix keys: its suffix rank adds nothing)
  const int n_keys = suffix_tile ? (a.mask_mode == kMaskPrefixOnly ? 0 : a.S) : min(64, a.P - 64 * rank);
  // the Pi0 block mask hides the action tokens of the suffix from the state token (row s == 0)
  const int n_vis = (a.mask_mode == RTV_MASK_PI0_BLOCK && suffix_tile && s == 0) ? 1 : n_keys;
  const bool s_done = ptx::mbar_wait(&bars[2], 0, a.timeout_ns);
  if (!s_done) {
    atomicOr(a.status, RTV_DEV_TIMEOUT);
    atomicOr(&s_timeout, 1);
  }
  ptx::tc_fence_after();
  // V^T into the Q tile's space: the S MMA, its only reader, has completed
  // (its copy overlaps the softmax below)
  bool v_issued = !COMPACT, pv_issued = false;   // (separate tiles: V^T came with K)
  if (COMPACT && tid == 0 && ok && s_done) {
    ptx::mbar_expect_tx(&bars[4], (uint32_t)VB);
    ptx::bulk_load(Vs, vsrc, (uint32_t)VB, &bars[4]);
    v_issued = true;
  }
  if (trace && tid == 0) trace[9] = ptx::globaltimer();
  float x[32];
  ptx::tmem_ld_32(tmem + lane_base + 32u * half, x);
  if (trace && tid == 0) trace[10] = ptx::globaltimer();
  float m4[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
  for (int e = 0; e < 32; ++e) {
    x[e] = 32 * half + e < n_vis ? x[e] * a.scale_log2 : -INFINITY;
    m4[e & 3] = fmaxf(m4[e & 3], x[e]);
  }
  red_m[half][r] = fmaxf(fmaxf(m4[0], m4[1]), fmaxf(m4[2], m4[3]));
  __syncthreads();
  const float mx = fmaxf(red_m[0][r], red_m[1][r]);
  float l4[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
  for (int e = 0; e < 32; ++e) {
    x[e] = x[e] == -INFINITY ? 0.f : exp2f(x[e] - mx);
    l4[e & 3] += x[e];
  }
  red_l[half][r] = (l4[0] + l4[1]) + (l4[2] + l4[3]);
  // P row: this thread's 32 keys = 4 chunks of 16 bytes, chunk-swizzled like a K-major operand tile
#pragma unroll
  for (int cc = 0; cc < 4; ++cc) {
    const int c = 4 * half + cc;
    uint4 v;
    v.x = ptx::pack_bf16x2(x[8 * cc], x[8 * cc + 1]);
    v.y = ptx::pack_bf16x2(x[8 * cc + 2], x[8 * cc + 3]);
    v.z = ptx::pack_bf16x2(x[8 * cc + 4], x[8 * cc + 5]);
    v.w = ptx::pack_bf16x2(x[8 * cc + 6], x[8 * cc + 7]);
    *reinterpret_cast<uint4*>(Ps + r * 128 + ((c ^ (r & 7)) << 4)) = v;
  }
  if (trace && tid == 0) trace[11] = ptx::globaltimer();
  ptx::fence_proxy_async_smem();
  ptx::tc_fence_before();
  __syncthreads();
  if (trace && tid == 0) trace[3] = ptx::globaltimer();
  const size_t part_base = (size_t)(g * HP + hp) * nch;   // slot of rank q: part_base + q
  if (half == 0 && row_valid)
    *reinterpret_cast<float2*>(a.part_ml + ((part_base + rank) * 128 + r) * 2) =
        make_float2(mx, red_l[0][r] + red_l[1][r]);
  if (tid == 0 && ok && v_issued) {
    if (!COMPACT || ptx::mbar_wait(&bars[4], 0, a.timeout_ns)) {
      ptx::tc_fence_after();
      const uint32_t idesc = ptx::idesc_bf16_f32(128, D);
      const uint32_t pa = ptx::smem_u32(Ps), va = ptx::smem_u32(Vs);
#pragma unroll
      for (int kk = 0; kk < 4; ++kk)
        ptx::umma_bf16(tmem, ptx::sw128_kmajor_desc(pa + kk * 32), ptx::sw128_kmajor_desc(va + kk * 32), idesc,
                       kk != 0 ? 1u : 0u);
      ptx::umma_commit(&bars[3]);
      pv_issued = true;
    } else {
      atomicOr(a.status, RTV_DEV_TIMEOUT);
      atomicOr(&s_timeout, 1);
    }
  }
  __syncwarp();
  if (!ptx::mbar_wait(&bars[3], 0, a.timeout_ns)) {
    atomicOr(a.status, RTV_DEV_TIMEOUT);
    atomicOr(&s_timeout, 1);
  }
  ptx::tc_fence_after();
  if (trace && tid == 0) trace[4] = ptx::globaltimer();
  // unnormalised O rows -> the Q tile's space (free since S was computed),
  // chunk-swizzled; each thread of a pair takes half of the D columns
#pragma unroll 1
  for (int cb = 0; cb < D / 64; ++cb) {
    const int col = (D / 2) * half + 32 * cb;
    float v[32];
    ptx::tmem_ld_32(tmem + lane_base + (uint32_t)col, v);
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      uint4 u;
      u.x = ptx::pack_bf16x2(v[8 * e], v[8 * e + 1]);
      u.y = ptx::pack_bf16x2(v[8 * e + 2], v[8 * e + 3]);
      u.z = ptx::pack_bf16x2(v[8 * e + 4], v[8 * e + 5]);
      u.w = ptx::pack_bf16x2(v[8 * e + 6], v[8 * e + 7]);
      const int c = col / 8 + e;   // 16-byte chunk of the row
      *reinterpret_cast<uint4*>(Qs + r * (D * 2) + ((c ^ (r & 7)) << 4)) = u;
    }
  }
  if (trace && tid == 0) trace[12] = ptx::globaltimer();
  ptx::tc_fence_before();
  __syncthreads();
  // out to global memory, one coalesced row per warp step (valid rows only)
  {
    __nv_bfloat16* po = a.part_o + (part_base + rank) * 128 * D;
    for (int rr = warp; rr < 128; rr += 8) {
      if ((rr & 63) >= a.S) continue;
      for (int c = lane; c < CPR; c += 32)
        *reinterpret_cast<uint4*>(po + (size_t)rr * D + c * 8) =
            *reinterpret_cast<const uint4*>(Qs + rr * (D * 2) + ((c ^ (rr & 7)) << 4));
    }
  }
  if (trace && tid == 0) trace[5] = ptx::globaltimer();
  // release / acquire at cluster scope: every rank's partials are visible
  ptx::cluster_sync();
  if (trace && tid == 0) trace[6] = trace[7] = ptx::globaltimer();
  constexpr int kRB = 1;   // rows per warp step (one row's 16 loads in flight keeps two CTAs per SM)
  // combine: the pair's 2*S valid rows are split evenly over the ranks; a warp
  // takes one of its rank's rows at a time and issues every load of it
  // before reducing (ranks summed in order)
  const int nvalid = 2 * a.S;
  const int rpc = (nvalid + nch - 1) / nch;
  const int v0 = rank * rpc, v1 = min(nvalid, v0 + rpc);
  for (int vb = v0 + warp; vb < v1; vb += 8 * kRB) {
    int rows[kRB];
    bool has[kRB];
#pragma unroll
    for (int u = 0; u < kRB; ++u) {
      const int vi = vb + 8 * u;
      has[u] = vi < v1;
      const int hs = has[u] ? vi / a.S : 0;
      rows[u] = has[u] ? hs * 64 + (vi - hs * a.S) : 0;
    }
    float mq[kRB], lq[kRB];
    uint4 v[kRB][16];
#pragma unroll
    for (int u = 0; u < kRB; ++u) {
      mq[u] = -INFINITY;
      lq[u] = 0.f;
    }
#pragma unroll
    for (int u = 0; u < kRB; ++u) {
      if (has[u] && lane < nch) {
        const float2 ml =
            __ldcg(reinterpret_cast<const float2*>(a.part_ml + ((part_base + lane) * 128 + rows[u]) * 2));
        mq[u] = ml.x;
        lq[u] = ml.y;
      }
#pragma unroll
      for (int q = 0; q < 16; ++q)
        if (has[u] && q < nch && lane < CPR)
          v[u][q] = __ldcg(reinterpret_cast<const uint4*>(a.part_o + ((part_base + q) * 128 + rows[u]) * D + lane * 8));
    }
    if (trace && tid == 0 && vb == v0) trace[13] = ptx::globaltimer();
#pragma unroll
    for (int u = 0; u < kRB; ++u) {
      if (!has[u]) continue;   // uniform across the warp
      const float m_all = warp_max(mq[u]);
      const float wq = (lane < nch && mq[u] != -INFINITY) ? exp2f(mq[u] - m_all) : 0.f;
      const float inv = 1.f / warp_sum(wq * lq[u]);
      float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int q = 0; q < 16; ++q) {
        const float wqq = __shfl_sync(0xffffffffu, wq, q);
        if (q < nch && lane < CPR) {
          const __nv_bfloat162* v2 = reinterpret_cast<const __nv_bfloat162*>(&v[u][q]);
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const float2 f = __bfloat1622float2(v2[e]);
            acc[2 * e] = fmaf(wqq, f.x, acc[2 * e]);
            acc[2 * e + 1] = fmaf(wqq, f.y, acc[2 * e + 1]);
          }
        }
      }
      if (lane < CPR) {
        uint4 out;
        out.x = ptx::pack_bf16x2(acc[0] * inv, acc[1] * inv);
        out.y = ptx::pack_bf16x2(acc[2] * inv, acc[3] * inv);
        out.z = ptx::pack_bf16x2(acc[4] * inv, acc[5] * inv);
        out.w = ptx::pack_bf16x2(acc[6] * inv, acc[7] * inv);
        const int j = 2 * hp + (rows[u] >> 6);
        *reinterpret_cast<uint4*>(a.o + ts_offset(g * a.S + (rows[u] & 63), j * D + lane * 8, a.n_mma)) = out;
      }
      if (trace && tid == 0 && vb == v0) trace[14 + u] = ptx::globaltimer();
    }
  }
  if (trace && tid == 0) trace[8] = ptx::globaltimer();
  // Never leave, or free the tensor memory, with a copy or an MMA of this CTA
  // still in flight (they complete on their own; after a timeout above this
  // drains them).  Every copy was requested; the MMAs only when `ok`.
  ptx::tc_fence_before();
  __syncthreads();
  if (s_timeout) {   // (uniform: read after the barrier)
    if (tid == 0) {
      // every copy and MMA issued: K, Q, S (when ok), V^T, PV
      bool drained = ptx::mbar_wait(&bars[0], 0, kDrainNs) && ptx::mbar_wait(&bars[1], 0, kDrainNs);
      if (ok) drained = drained && ptx::mbar_wait(&bars[2], 0, kDrainNs);
      if (COMPACT && v_issued) drained = drained && ptx::mbar_wait(&bars[4], 0, kDrainNs);
      if (pv_issued) drained = drained && ptx::mbar_wait(&bars[3], 0, kDrainNs);
      if (!drained) atomicOr(a.status, RTV_DEV_TIMEOUT);
    }
    __syncthreads();
  }
  if (warp == 0) {
    ptx::tc_fence_after();
    ptx::tmem_dealloc(tmem, TCOLS);
  }
}

// Prefix tiles of the tensor-core attention, from the cached prefix
// [L][2][Bmax][Hkv][Pmax][D]: keys [l][b][h][tile][64][D] and values
// transposed [l][b][h][tile][D][64], both tiled and pre-swizzled.  One thread
// per 8 consecutive features of one key.
__global__ void prefix_tile_kernel(const __nv_bfloat16* __restrict__ kv, __nv_bfloat16* __restrict__ pkt,
                                   __nv_bfloat16* __restrict__ pvt, int L, int B, int P, int Hkv, int D, int Bmax,
                                   int Pmax, int ntile_max) {
  const size_t n = (size_t)L * B * Hkv * P * (D / 8);
  for (size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += (size_t)gridDim.x * blockDim.x) {
    const int d0 = 8 * (int)(i % (D / 8));
    size_t rest = i / (D / 8);
    const int key = (int)(rest % P);
    rest /= P;
    const int h = (int)(rest % Hkv);
    rest /= Hkv;
    const int b = (int)(rest % B);
    const int l = (int)(rest / B);
    const size_t src_k = ((((size_t)l * 2 + 0) * Bmax + b) * Hkv + h) * Pmax * D + (size_t)key * D + d0;
    const size_t src_v = ((((size_t)l * 2 + 1) * Bmax + b) * Hkv + h) * Pmax * D + (size_t)key * D + d0;
    const size_t tile = (((size_t)l * Bmax + b) * Hkv + h) * ntile_max + key / 64;
    const int kr = key & 63;
    *reinterpret_cast<uint4*>(pkt + tile * 64 * D + ts_offset(kr, d0, 64)) = *reinterpret_cast<const uint4*>(kv + src_k);
    const uint4 vv = *reinterpret_cast<const uint4*>(kv + src_v);
    const __nv_bfloat16* ve = reinterpret_cast<const __nv_bfloat16*>(&vv);
    __nv_bfloat16* vt = pvt + tile * 64 * D;
#pragma unroll
    for (int e = 0; e < 8; ++e) vt[ts_offset(d0 + e, kr, D)] = ve[e];
  }
}

// ---------------------------------------------------------------------------
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
  __nv_bfloat16* hb;              // tiled [w/64][n_mma][64]
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
  const float* g_attn0;           // first layer's attention-norm gain (of group g: g_attn0 + g * g0_stride)
  unsigned* status;
  int w, S, A, Sd, state_stride, c_stride, do_head, do_embed, n_mma, g0_stride;
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
  const float4 ga = *reinterpret_cast<const float4*>(a.g_attn0 + (size_t)g * a.g0_stride + i0);
  uint2 hbv;
  hbv.x = ptx::pack_bf16x2(hv[0] * (1.f + ga.x), hv[1] * (1.f + ga.y));
  hbv.y = ptx::pack_bf16x2(hv[2] * (1.f + ga.z), hv[3] * (1.f + ga.w));
  *reinterpret_cast<uint2*>(a.hb + ts_offset(r, i0, a.n_mma)) = hbv;
  // each warp covers one 128-feature tile
  float sq = hv[0] * hv[0];
  sq = fmaf(hv[1], hv[1], sq);
  sq = fmaf(hv[2], hv[2], sq);
  sq = fmaf(hv[3], hv[3], sq);
  sq = warp_sum(sq);
  if (lane == 0) a.ssp[(size_t)r * (a.w >> 7) + warp] = sq;
}

// ---------------------------------------------------------------------------
// Weight packing: row r of the packed matrix is row idx[r] (or r) of a
// [rows][K] bf16 matrix, stored in 128-row tiles of the tiled, pre-swizzled
// layout ([rows/128][K/64][128][64], see ts_offset).
// ---------------------------------------------------------------------------
__global__ void pack_tiled_kernel(const __nv_bfloat16* __restrict__ src, __nv_bfloat16* __restrict__ dst,
                                  const int* __restrict__ idx, int rows, int K) {
  const int r = blockIdx.x;
  if (r >= rows) return;
  const uint4* s = reinterpret_cast<const uint4*>(src + (size_t)(idx ? idx[r] : r) * K);
  __nv_bfloat16* d = dst + (size_t)(r >> 7) * (K >> 6) * 8192;
  for (int i = threadIdx.x; i < K / 8; i += blockDim.x)
    *reinterpret_cast<uint4*>(d + ts_offset(r & 127, 8 * i, 128)) = s[i];
}

// FP8 weights: row r of the packed matrix is row idx[r] (or r) of a [rows][K]
// E4M3 matrix, in 128-row tiles of [K/64] boxes [128][64] bytes (the
// converters add the swizzle when they widen a box to bf16).
__global__ void pack_tiled8_kernel(const uint8_t* __restrict__ src, uint8_t* __restrict__ dst,
                                   const int* __restrict__ idx, int rows, int K) {
  const int r = blockIdx.x;
  if (r >= rows) return;
  const uint8_t* s = src + (size_t)(idx ? idx[r] : r) * K;
  uint8_t* d = dst + (size_t)(r >> 7) * (K >> 6) * 8192 + (size_t)(r & 127) * 64;
  for (int i = threadIdx.x; i < K / 16; i += blockDim.x) {
    const int k = 16 * i;
    *reinterpret_cast<uint4*>(d + (size_t)(k >> 6) * 8192 + (k & 63)) = *reinterpret_cast<const uint4*>(s + k);
  }
}

__global__ void gather_f32_kernel(const float* __restrict__ src, float* __restrict__ dst, const int* __restrict__ idx,
                                  int n) {
  for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < n; i += gridDim.x * blockDim.x) dst[i] = src[idx ? idx[i] : i];
}

// [rows][cols] -> [cols][rows]
__global__ void transpose_bf16_kernel(const __nv_bfloat16* __restrict__ src, __nv_bfloat16* __restrict__ dst,
                                      int rows, int cols) {
  for (int idx = blockIdx.x * blockDim.x + threadIdx.x; idx < rows * cols; idx += gridDim.x * blockDim.x) {
    const int r = idx / cols, c = idx - r * cols;
    dst[(size_t)c * rows + r] = src[idx];
  }
}

// ---------------------------------------------------------------------------
// Rows that enter a block from outside its residual stream (the draft
// model's image features and action queries): the first norm's input
// bf16(x * (1 + g)), tiled over n_rows token rows, and the sums of squares
// of x per 128-feature tile; with h set, also x as the fp32 residual row.
// Row t reads x row t % x_rows.  One CTA of 4 warps per row; warp j takes
// the tiles j, j + 4, ...
// ---------------------------------------------------------------------------
__device__ __forceinline__ void load4_f32(const float* p, float v[4]) {
  const float4 q = *reinterpret_cast<const float4*>(p);
  v[0] = q.x;
  v[1] = q.y;
  v[2] = q.z;
  v[3] = q.w;
}
__device__ __forceinline__ void load4_f32(const __nv_bfloat16* p, float v[4]) {
  const uint2 q = *reinterpret_cast<const uint2*>(p);
  const float2 a = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&q.x));
  const float2 b = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&q.y));
  v[0] = a.x;
  v[1] = a.y;
  v[2] = b.x;
  v[3] = b.y;
}

template <typename XT>
__global__ void __launch_bounds__(128) norm_input_kernel(const XT* __restrict__ x, int x_rows, float* __restrict__ h,
                                                         const float* __restrict__ g, __nv_bfloat16* __restrict__ hb,
                                                         float* __restrict__ ssp, int n_rows, int w) {
  const int t = blockIdx.x;
  const XT* xr = x + (size_t)(t % x_rows) * w;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int n_wt = w >> 7;
  for (int j = warp; j < n_wt; j += 4) {
    const int k = j * 128 + lane * 4;
    float v[4];
    load4_f32(xr + k, v);
    float sq = v[0] * v[0];
    sq = fmaf(v[1], v[1], sq);
    sq = fmaf(v[2], v[2], sq);
    sq = fmaf(v[3], v[3], sq);
    sq = warp_sum(sq);
    if (lane == 0) ssp[(size_t)t * n_wt + j] = sq;
    if (h) *reinterpret_cast<float4*>(h + (size_t)t * w + k) = make_float4(v[0], v[1], v[2], v[3]);
    const float4 gg = *reinterpret_cast<const float4*>(g + k);
    uint2 packed;
    packed.x = ptx::pack_bf16x2(v[0] * (1.f + gg.x), v[1] * (1.f + gg.y));
    packed.y = ptx::pack_bf16x2(v[2] * (1.f + gg.z), v[3] * (1.f + gg.w));
    *reinterpret_cast<uint2*>(hb + ts_offset(t, k, n_rows)) = packed;
  }
}

// ===========================================================================
// host side
// ===========================================================================
struct GemmPlan {
  int n_tiles = 0, cs = 1, kslice = 0, stages = 1, smem = 0;
  int n_tt = 1;   // token tiles (grid y)
  int tt = 0;     // token rows per CTA (0: the caller's)
  double cost = 0.0;
  bool valid = false;
};

struct FastPath {
  __nv_bfloat16 *w_qkv = nullptr, *w_o = nullptr, *w_gu = nullptr, *w_down = nullptr;
  __nv_bfloat16 *w_aiT = nullptr, *w_spT = nullptr;
  bool mlp_f8 = false;                                      // gate/up/down in FP8 E4M3
  uint8_t *w_gu8 = nullptr, *w_down8 = nullptr;             // their tiled codes, all layers
  float *gu_s = nullptr, *down_s = nullptr;                 // per-row scales, packed row order, all layers
  __nv_bfloat16 *qb = nullptr, *ksb = nullptr, *vsb = nullptr, *ob = nullptr, *mb = nullptr, *hb = nullptr;
  float* ssp = nullptr;
  // attention partial rows [Gmax][Hq][16][64][D] (the tensor-core kernel
  // indexes the same storage as [Gmax][Hq/2][16][128][D]) and their (max, sum)
  __nv_bfloat16* att_po = nullptr;
  float* att_pml = nullptr;
  // tensor-core attention (head pairs sharing a KV head): tiled operands
  bool tc_attn = false;
  int ntile_max = 0;                 // 64-key tiles of the longest prefix
  __nv_bfloat16 *qt = nullptr, *kts = nullptr, *vts = nullptr;   // q of head pairs, suffix K and V^T tiles
  __nv_bfloat16 *pkt = nullptr, *pvt = nullptr;                  // prefix K and V^T tiles, all layers
  int num_sms = 148;
  int max_cluster = 8;
  int gemm_fit_small[17] = {0};   // co-resident GEMM clusters by size, at the smem_cap budget (diagnostic)
  int gemm_fit_large[17] = {0};   // ... and at the whole shared memory
  int attn_fit[17] = {0};      // co-resident clusters of attention CTAs, by cluster size
  // Shared-memory budget of a GEMM grid larger than the SM count.  A kernel
  // that holds tensor memory runs one CTA per SM whatever its shared memory;
  // the budget leaves room beside it for a CTA of the attention or step kernel.
  int smem_cap = 100 * 1024;
  bool deep_single_wave = false;   // see plan_gemm (a bare block: its GEMMs have no PDL partner to leave room for)
  // Bytes of the next projection's weights one launch brings into L2 at most
  // (a projection larger than L2 is partly prefetched: its first bytes).
  unsigned long long pf_cap = 48ull << 20;
  // optional phase trace of the four projections of layer 0 in the first Euler step
  unsigned long long* trace = nullptr;
  int trace_ctas[5] = {0, 0, 0, 0, 0};
  bool trace_armed = false;
  std::vector<void*> allocs;
};

// Token tiles of a projection over n_mma rows (defined below).
void token_tiles(int n_mma, int* n_tt, int* tt);

namespace {

constexpr int kSmemOptin = 227 * 1024;
constexpr int kDynSmemMax = kSmemOptin - 2048;   // every kernel here uses < 2 KB of static shared memory

int round_up(int x, int m) { return (x + m - 1) / m * m; }

// Split of one projection over CTAs: 128-row weight tiles x K slices (one
// cluster per tile, up to 16 CTAs).  A CTA's MMAs run at a fixed rate of
// about one 64-wide box per 0.4 us whatever the token count, and a wave of
// CTAs costs a few microseconds of fixed latency (loads, exchange, epilogue),
// so the split minimises waves x (fixed + boxes per CTA).  Two CTAs share an
// SM when the ring fits the smem_cap budget (the ring is then the deepest
// that does), otherwise one (the ring the deepest that fits the whole shared
// memory); a cluster size is only usable as far as its clusters fit.  Ties
// go to the smaller cluster (less reduction traffic).
GemmPlan plan_gemm(const FastPath* fp, int N, int K, int n_mma, int T, bool with_in, bool f8 = false,
                   int n_tt = 1) {
  // (With deep_single_wave, a split whose clusters are all resident at once
  // with one CTA per SM takes the deepest ring the whole shared memory
  // holds: more weight boxes in flight per CTA, at the price of no
  // co-resident CTA of the next kernel.)
  GemmPlan best;
  best.n_tiles = N / 128;
  best.n_tt = n_tt;
  double best_cost = 1e30;
  constexpr double kFixedBoxes = 8.0;   // a wave's fixed latency, in MMA boxes (~3 us)
  for (int cs = 1; cs <= fp->max_cluster; cs <<= 1) {
    if (K % (cs * 64)) break;
    if ((T + cs - 1) / cs > 256) continue;   // tokens per rank (kMaxOwn in the kernel)
    const int nbox = K / cs / 64;
    auto total = [&](int st) { return gemm_smem_layout(st, n_mma, cs, T, with_in, f8).total; };
    int stages = nbox;
    while (stages > 1 && total(stages) > fp->smem_cap) --stages;
    int per_sm = 2;
    const bool one_wave = fp->deep_single_wave && best.n_tiles * n_tt <= fp->gemm_fit_large[cs];
    if (one_wave || total(stages) > fp->smem_cap) {
      per_sm = 1;
      stages = nbox;
      while (stages > 1 && total(stages) > kDynSmemMax) --stages;
      if (total(stages) > kDynSmemMax) continue;
    }
    const int ctas = best.n_tiles * cs * n_tt;
    const int fit = per_sm * std::max(1, fp->gemm_fit_large[cs]);   // clusters resident at once
    const int waves = std::max((ctas + per_sm * fp->num_sms - 1) / (per_sm * fp->num_sms),
                               (best.n_tiles * n_tt + fit - 1) / fit);
    const double cost = waves * (kFixedBoxes + nbox);
    if (cost < best_cost) {
      best_cost = cost;
      best.cost = cost;
      best.cs = cs;
      best.kslice = K / cs;
      best.stages = stages;
      best.smem = total(stages);
    }
  }
  best.valid = best.kslice >= 64 && best.smem > 0 && best.smem <= kDynSmemMax && (T + best.cs - 1) / best.cs <= 256;
  return best;
}

// Plan of a projection of the suffix layers over n_mma token rows (T of them
// real).  Between 65 and 256 rows the token tiling is chosen with the split:
// 1-4 tiles, each tile's cluster exchange charged by its rows (about four MMA
// boxes for every 64 rows beyond the first 64: measured, 160-row tiles made a
// three-tau verification 13% slower than 64-row ones).
GemmPlan plan_suffix(const FastPath* fp, int N, int K, int n_mma, int T, bool with_in, bool f8) {
  int n_tt0 = 1, tt0 = 16;
  token_tiles(n_mma, &n_tt0, &tt0);
  if (n_mma <= 64 || n_mma > 256) {
    GemmPlan p = plan_gemm(fp, N, K, tt0, std::min(T, tt0), with_in, f8, n_tt0);
    p.tt = tt0;
    return p;
  }
  GemmPlan best;
  double best_cost = 1e30;
  for (int n_tt = 1; n_tt <= 4; ++n_tt) {
    const int tt = round_up((n_mma + n_tt - 1) / n_tt, 16);
    if ((n_tt - 1) * tt >= n_mma) continue;   // the last tile would be empty
    GemmPlan p = plan_gemm(fp, N, K, tt, std::min(T, tt), with_in, f8, n_tt);
    if (!p.valid) continue;
    const double cost = p.cost + 4.0 * std::max(0, tt - 64) / 64.0;
    if (cost < best_cost) {
      best_cost = cost;
      best = p;
      best.tt = tt;
    }
  }
  return best;
}

template <int MODE>
cudaError_t launch_gemm(const GemmArgs& a, const GemmPlan& pl, cudaStream_t st,
                        unsigned long long pf_cap = ~0ull) {
  auto kern = a.wt8 ? gemm_tc_kernel<MODE, true> : gemm_tc_kernel<MODE, false>;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(pl.cs, pl.n_tt, pl.n_tiles);
  cfg.blockDim = dim3(kGemmThreads, 1, 1);
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
  if (pl.tt) args.tt = pl.tt;
  if (args.pf_bytes > pf_cap) args.pf_bytes = pf_cap;
  return cudaLaunchKernelEx(&cfg, kern, args);
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
  cudaError_t e = cudaSuccess;
  for (auto kern : {gemm_tc_kernel<MODE, false>, gemm_tc_kernel<MODE, true>}) {
    if (e == cudaSuccess) e = configure_dyn_smem(kern);
    if (e == cudaSuccess) e = cudaFuncSetAttribute(kern, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
  }
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
  cfg.blockDim = dim3(128, 1, 1);
  cfg.dynamicSmemBytes = attn_smem_bytes(D);
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
  cfg.blockDim = dim3(128, 1, 1);
  cfg.dynamicSmemBytes = attn_smem_bytes(D);
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

template <int D>
cudaError_t configure_attn_tc() {
  cudaError_t e = cudaSuccess;
  for (int compact = 0; compact < 2; ++compact) {
    auto kern = compact ? attn_tc_kernel<D, true> : attn_tc_kernel<D, false>;
    if (e == cudaSuccess)
      e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, attn_tc_smem_bytes(D, compact));
    if (e == cudaSuccess) e = cudaFuncSetAttribute(kern, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
  }
  return e;
}

// The compact layout when the grid is larger than the SM count (two CTAs per
// SM keep it in one wave); otherwise separate tiles, whose V^T is requested
// before the dependency wait (measured: the compact layout costs the batch-1
// chunk 2.7%, and saves 8% of a three-tau verification).
template <int D>
cudaError_t launch_attn_tc(const AttnTcArgs& a, int nchunk, int G, int num_sms, cudaStream_t st) {
  const bool compact = nchunk * (a.Hq / 2) * G > num_sms;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(nchunk, a.Hq / 2, G);
  cfg.blockDim = dim3(256, 1, 1);
  cfg.dynamicSmemBytes = attn_tc_smem_bytes(D, compact);
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
  return cudaLaunchKernelEx(&cfg, compact ? attn_tc_kernel<D, true> : attn_tc_kernel<D, false>, a);
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
  // (the step kernel, which a bare block does not use, limits the width and
  // the action and state sizes)
  const bool step_ok = ctx->block_only || (k.width <= 1024 && k.action_dim <= 64 && k.state_dim <= 64);
  const bool shape_ok = k.dtype == RTV_BF16 && (k.head_dim == 128 || k.head_dim == 256) && k.width % 128 == 0 &&
                        k.mlp_dim % 128 == 0 && (ctx->Q % 128) == 0 && S <= 64 && step_ok && n_mma_max > 0;
  if (!shape_ok) return RTV_OK;
  int dev = ctx->device;
  if (configure_gemm<GM_QKV>() != cudaSuccess || configure_gemm<GM_O>() != cudaSuccess ||
      configure_gemm<GM_GU>() != cudaSuccess || configure_gemm<GM_DOWN>() != cudaSuccess ||
      configure_attn<128>() != cudaSuccess || configure_attn<256>() != cudaSuccess ||
      configure_attn_tc<128>() != cudaSuccess || configure_attn_tc<256>() != cudaSuccess) {
    cudaGetLastError();
    return RTV_ERR_CUDA;
  }
  FastPath* fp = new FastPath();
  cudaDeviceGetAttribute(&fp->num_sms, cudaDevAttrMultiProcessorCount, dev);
  // A bare block's GEMMs leave no room for a partner kernel: two CTAs per SM
  // may take half of the SM's 228 KB each (less the per-CTA reservation and
  // static shared memory), and a one-wave split the whole of it.
  fp->deep_single_wave = ctx->block_only;
  if (ctx->block_only) fp->smem_cap = 112 * 1024;
  // co-resident GEMM clusters by cluster size, at both shared-memory budgets
  for (int cs = 1; cs <= 16; cs <<= 1) {
    for (int big = 0; big < 2; ++big) {
      cudaLaunchConfig_t cfg = {};
      cfg.gridDim = dim3(cs, 1, 1);
      cfg.blockDim = dim3(kGemmThreads, 1, 1);
      cfg.dynamicSmemBytes = big ? kDynSmemMax : fp->smem_cap;
      cudaLaunchAttribute at;
      at.id = cudaLaunchAttributeClusterDimension;
      at.val.clusterDim.x = cs;
      at.val.clusterDim.y = 1;
      at.val.clusterDim.z = 1;
      cfg.attrs = &at;
      cfg.numAttrs = 1;
      int n = 0;
      if (cudaOccupancyMaxActiveClusters(&n, gemm_tc_kernel<GM_DOWN, false>, &cfg) != cudaSuccess) n = 0;
      cudaGetLastError();
      (big ? fp->gemm_fit_large : fp->gemm_fit_small)[cs] = n;
    }
  }
  fp->max_cluster = 16;
  for (int c : {2, 4, 6, 8, 12, 16})
    fp->attn_fit[c] = k.head_dim == 256 ? attn_clusters_that_fit<256>(c, S) : attn_clusters_that_fit<128>(c, S);
  const size_t T = ctx->Tmax;
  const size_t Tp = (size_t)round_up(ctx->Tmax, 16);   // token rows of the tiled GEMM inputs
  auto alloc = [&](void** p, size_t bytes) -> bool {
    if (cudaMalloc(p, bytes) != cudaSuccess) return false;
    fp->allocs.push_back(*p);
    return cudaMemset(*p, 0, bytes) == cudaSuccess;
  };
  bool ok = alloc((void**)&fp->qb, T * ctx->Q * 2) && alloc((void**)&fp->ob, Tp * ctx->Q * 2) &&
            alloc((void**)&fp->mb, Tp * (size_t)k.mlp_dim * 2) && alloc((void**)&fp->hb, Tp * (size_t)k.width * 2) &&
            alloc((void**)&fp->ssp, T * (size_t)(k.width / 128) * 4) &&
            alloc((void**)&fp->att_po, (size_t)ctx->Gmax * k.n_q_heads * 16 * 64 * k.head_dim * 2) &&
            alloc((void**)&fp->att_pml, (size_t)ctx->Gmax * k.n_q_heads * 16 * 64 * 2 * 4) &&
            alloc((void**)&fp->ksb, (size_t)ctx->Gmax * ctx->KV * S * 2) &&
            alloc((void**)&fp->vsb, (size_t)ctx->Gmax * ctx->KV * S * 2);
  // tensor-core attention: both heads of a pair must share their KV head
  fp->tc_attn = k.n_q_heads % 2 == 0 && (k.n_q_heads / k.n_kv_heads) % 2 == 0;
  fp->ntile_max = (k.max_prefix_len + 63) / 64;
  if (ok && fp->tc_attn) {
    const size_t D = k.head_dim, Hkv = k.n_kv_heads;
    ok = alloc((void**)&fp->qt, (size_t)ctx->Gmax * (k.n_q_heads / 2) * 128 * D * 2) &&
         alloc((void**)&fp->kts, (size_t)ctx->Gmax * Hkv * 64 * D * 2) &&
         alloc((void**)&fp->vts, (size_t)ctx->Gmax * Hkv * 64 * D * 2) &&
         alloc((void**)&fp->pkt, (size_t)k.n_layers * k.max_batch * Hkv * fp->ntile_max * 64 * D * 2) &&
         alloc((void**)&fp->pvt, (size_t)k.n_layers * k.max_batch * Hkv * fp->ntile_max * 64 * D * 2);
  }
  if (!ok) {
    for (void* p : fp->allocs) cudaFree(p);
    delete fp;
    return RTV_ERR_OOM;
  }
  if (getenv("RTV_TRACE")) {
    if (cudaMalloc(&fp->trace, 5 * 512 * kTraceRow * sizeof(unsigned long long)) == cudaSuccess) {
      fp->allocs.push_back(fp->trace);
      cudaMemset(fp->trace, 0, 5 * 512 * kTraceRow * sizeof(unsigned long long));
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
  std::vector<unsigned long long> h(5 * 512 * kTraceRow);
  cudaDeviceSynchronize();
  cudaMemcpy(h.data(), fp->trace, h.size() * 8, cudaMemcpyDeviceToHost);
  const char* nm[5] = {"qkv", "o", "gu", "down", "attention"};
  const char* ev[2][15] = {{"start", "w_issued", "pdl", "first_full", "mma_issued", "done", "copied", "recv", "end",
                           "prefetched", "arrived", "iter0", "exit", "part", "entry"},
                          {"start", "pdl", "tile0", "loop_end", "merged", "entry", "pushed", "synced", "end", "s_seen",
                           "s_loaded", "p_stored", "o_staged", "cmb_issued", "cmb_row0"}};
  unsigned long long t_ref = ~0ull;
  for (int i = 0; i < 5; ++i)
    for (int c = 0; c < fp->trace_ctas[i]; ++c)
      if (h[((size_t)i * 512 + c) * kTraceRow]) t_ref = std::min(t_ref, h[((size_t)i * 512 + c) * kTraceRow]);
  const int order[5] = {0, 4, 1, 2, 3};
  for (int oi = 0; oi < 5; ++oi) {
    const int i = order[oi];
    fprintf(stderr, "[rtv trace] %s (%d CTAs), us after the first traced start: min / median / max\n", nm[i],
            fp->trace_ctas[i]);
    const int order_e[15] = {0, 1, 2, 3, 4, 5, 13, 14, 6, 9, 7, 10, 11, 8, 12};
    const int order_a[15] = {0, 1, 2, 9, 10, 11, 3, 4, 12, 5, 6, 7, 13, 14, 8};
    for (int ei = 0; ei < 15; ++ei) {
      const int e = i == 4 ? order_a[ei] : order_e[ei];
      if (!ev[i == 4][e][0]) continue;
      std::vector<double> v;
      for (int c = 0; c < fp->trace_ctas[i]; ++c) {
        const unsigned long long t = h[((size_t)i * 512 + c) * kTraceRow + e];
        if (t) v.push_back((double)(t - t_ref) * 1e-3);
      }
      if (v.empty()) continue;
      std::sort(v.begin(), v.end());
      fprintf(stderr, "    %-11s %8.2f %8.2f %8.2f\n", ev[i == 4][e], v.front(), v[v.size() / 2], v.back());
    }
    if (i != 4) {
      fprintf(stderr, "    stage landed (median):");
      for (int b = 0; b < 8; ++b) {
        std::vector<double> v;
        for (int c = 0; c < fp->trace_ctas[i]; ++c) {
          const unsigned long long t = h[((size_t)i * 512 + c) * kTraceRow + 16 + b];
          if (t) v.push_back((double)(t - t_ref) * 1e-3);
        }
        if (v.empty()) break;
        std::sort(v.begin(), v.end());
        fprintf(stderr, " %.2f", v[v.size() / 2]);
      }
      fprintf(stderr, "\n");
    }
  }
}

bool fast_supports_prefix(rtv_ctx*, int) { return true; }

bool fast_tc_attention(const rtv_ctx* ctx, int P) {
  const FastPath* fp = ctx->fast;
  const int ntp = (P + 63) / 64;
  const char* attn_env = getenv("RTV_ATTN");
  return fp && fp->tc_attn && ntp + 1 <= 16 && ntp <= fp->ntile_max && !(attn_env && strcmp(attn_env, "mma") == 0);
}

rtv_status fast_prefix_update(rtv_ctx* ctx, int batch, int prefix_len, cudaStream_t st) {
  FastPath* fp = ctx->fast;
  if (!fp || !fp->tc_attn) return RTV_OK;
  const rtv_expert_config& k = ctx->cfg;
  prefix_tile_kernel<<<4 * fp->num_sms, 256, 0, st>>>((const __nv_bfloat16*)ctx->prefix_kv, fp->pkt, fp->pvt,
                                                     k.n_layers, batch, prefix_len, k.n_kv_heads, k.head_dim,
                                                     k.max_batch, k.max_prefix_len, fp->ntile_max);
  const cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) {
    ctx->last_error = std::string("prefix tiling launch: ") + cudaGetErrorString(e);
    return RTV_ERR_CUDA;
  }
  return RTV_OK;
}

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
  fp->mlp_f8 = k.mlp_dtype == RTV_FP8_E4M3;
  if (!(alloc((void**)&fp->w_qkv, Lh * nq * w * 2) && alloc((void**)&fp->w_o, (size_t)Lh * w * Q * 2)))
    return RTV_ERR_OOM;
  if (!ctx->block_only && !(alloc((void**)&fp->w_aiT, (size_t)k.action_dim * w * 2) &&
                            alloc((void**)&fp->w_spT, (size_t)k.state_dim * w * 2)))
    return RTV_ERR_OOM;
  if (fp->mlp_f8) {
    if (!(alloc((void**)&fp->w_gu8, Lh * ngu * w) && alloc((void**)&fp->w_down8, (size_t)Lh * w * F) &&
          alloc((void**)&fp->gu_s, Lh * ngu * 4) && alloc((void**)&fp->down_s, (size_t)Lh * w * 4)))
      return RTV_ERR_OOM;
  } else if (!(alloc((void**)&fp->w_gu, Lh * ngu * w * 2) && alloc((void**)&fp->w_down, (size_t)Lh * w * F * 2))) {
    return RTV_ERR_OOM;
  }
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
    pack_tiled_kernel<<<(int)nq, 128>>>((const __nv_bfloat16*)Lw.qkv, fp->w_qkv + (size_t)l * nq * w, d_iq,
                                        (int)nq, w);
    pack_tiled_kernel<<<w, 128>>>((const __nv_bfloat16*)Lw.o, fp->w_o + (size_t)l * w * Q, nullptr, w, Q);
    if (fp->mlp_f8) {
      pack_tiled8_kernel<<<(int)ngu, 128>>>((const uint8_t*)Lw.gu, fp->w_gu8 + (size_t)l * ngu * w, d_igu, (int)ngu, w);
      pack_tiled8_kernel<<<w, 128>>>((const uint8_t*)Lw.down, fp->w_down8 + (size_t)l * w * F, nullptr, w, F);
      gather_f32_kernel<<<32, 256>>>(Lw.gu_s, fp->gu_s + (size_t)l * ngu, d_igu, (int)ngu);
      gather_f32_kernel<<<4, 256>>>(Lw.down_s, fp->down_s + (size_t)l * w, nullptr, w);
    } else {
      pack_tiled_kernel<<<(int)ngu, 128>>>((const __nv_bfloat16*)Lw.gu, fp->w_gu + (size_t)l * ngu * w, d_igu,
                                           (int)ngu, w);
      pack_tiled_kernel<<<w, 128>>>((const __nv_bfloat16*)Lw.down, fp->w_down + (size_t)l * w * F, nullptr, w, F);
    }
  }
  if (!ctx->block_only) {
    transpose_bf16_kernel<<<64, 256>>>((const __nv_bfloat16*)ctx->W.ai_w, fp->w_aiT, w, k.action_dim);
    transpose_bf16_kernel<<<64, 256>>>((const __nv_bfloat16*)ctx->W.sp_w, fp->w_spT, w, k.state_dim);
  }
  cudaError_t e = cudaDeviceSynchronize();
  cudaFree(d_iq);
  cudaFree(d_igu);
  if (e != cudaSuccess) return RTV_ERR_CUDA;
  return RTV_OK;
}

rtv_status fast_step(rtv_ctx* ctx, int G, bool do_head, bool do_embed, float dt, const float* c, int c_stride,
                     int state_stride, bool velocity_only, cudaStream_t st, const float* g0, int g0_stride) {
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
  a.g_attn0 = g0 ? g0 : ctx->W.layers[0].g_attn;
  a.g0_stride = g0 ? g0_stride : 0;
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
  a.n_mma = round_up(G * ctx->S, 16);
  const cudaError_t e = launch_step(a, G * ctx->S, st);
  if (e != cudaSuccess) {
    ctx->last_error = std::string("step launch: ") + cudaGetErrorString(e);
    return RTV_ERR_CUDA;
  }
  return RTV_OK;
}

// Token tiles of a projection over n_mma tiled rows: up to 208 rows stay one
// tile; beyond, tiles of about 128 rows keep a CTA's fp32 partial tile and
// reduction buffers (512 bytes per token row each) within shared memory.
void token_tiles(int n_mma, int* n_tt, int* tt) {
  // Up to 256 token rows, tiles of 64: a CTA's partial tile and its share of
  // the cluster exchange stay those of one suffix (measured: three-tau
  // verification at 153 rows 1.61 -> 1.42 ms, batch 4 17.8 -> 13.7 ms per
  // chunk), and the extra CTAs read the same weight boxes through L2.  Above
  // that, tiles of ~128 rows (at 816 rows 64-row tiles slow the FP8 MLP).
  if (n_mma <= 64) *n_tt = 1;
  else if (n_mma <= 256) *n_tt = (n_mma + 63) / 64;
  else *n_tt = (n_mma + 127) / 128;
  *tt = round_up((n_mma + *n_tt - 1) / *n_tt, 16);
}

rtv_status fast_block_prefix(rtv_ctx* ctx, const __nv_bfloat16* vis, int n_vis, int batch, __nv_bfloat16* hb_vis,
                             float* ssp_vis, const float* rope_cs, const float* rope_sn, cudaStream_t st) {
  FastPath* fp = ctx->fast;
  const rtv_expert_config& k = ctx->cfg;
  const int w = k.width, D = k.head_dim, KV = ctx->KV;
  const int T = batch * n_vis, n_mma = round_up(T, 16);
  int n_tt = 1, tt = 16;
  token_tiles(n_mma, &n_tt, &tt);
  const LayerW& Lw = ctx->W.layers[0];
  norm_input_kernel<__nv_bfloat16><<<T, 128, 0, st>>>(vis, T, nullptr, Lw.g_attn, hb_vis, ssp_vis, n_mma, w);
  cudaError_t e = cudaGetLastError();
  const GemmPlan p = plan_gemm(fp, 2 * KV, w, tt, std::min(T, tt), true, false, n_tt);
  if (!p.valid) {
    ctx->last_error = "no tensor-core split fits the visual-token projection";
    return RTV_ERR_UNSUPPORTED;
  }
  if (getenv("RTV_LOG"))
    fprintf(stderr, "[rtv] T=%d visual k/v: tiles=%d token_tiles=%d cluster=%d kslice=%d stages=%d smem=%d\n", T,
            p.n_tiles, p.n_tt, p.cs, p.kslice, p.stages, p.smem);
  // keys and values of the visual tokens: the K and V weight tiles of the
  // layer (the q tiles are skipped), RoPE at positions 0..n_vis-1, written
  // into the cached prefix [2][Bmax][Hkv][Pmax][D] of layer 0
  const size_t kv_layer = (size_t)k.max_batch * k.n_kv_heads * k.max_prefix_len * D;
  GemmArgs a{};
  a.wt = fp->w_qkv;
  a.act = hb_vis;
  a.ssp = ssp_vis;
  a.ks = (__nv_bfloat16*)ctx->prefix_kv;
  a.vs = a.ks + kv_layer;
  a.kv_rows = k.max_prefix_len;
  a.seq = n_vis;
  a.rope_cs = rope_cs;
  a.rope_sn = rope_sn;
  a.status = ctx->status;
  a.timeout_ns = k.barrier_timeout_ns;
  a.T = T;
  a.n_mma = n_mma;
  a.tt = tt;
  a.w = w;
  a.S = n_vis;
  a.Hq = k.n_q_heads;
  a.Hkv = k.n_kv_heads;
  a.D = D;
  a.F = k.mlp_dim;
  a.K = w;
  a.w_tile0 = 0;
  a.nt_base = ctx->Q / 128;
  a.eps = k.rms_eps;
  // the tensor-core attention's tiles of the visual keys and values straight
  // from the epilogue (no separate tiling pass over the cache)
  const bool tiles = fp->tc_attn && (n_vis + 63) / 64 <= fp->ntile_max;
  if (tiles) {
    a.pkt = fp->pkt;
    a.pvt = fp->pvt;
    a.ntile_max = fp->ntile_max;
  }
  if (e == cudaSuccess) e = launch_gemm<GM_QKV>(a, p, st);
  if (e != cudaSuccess) {
    ctx->last_error = std::string("visual-token projection launch: ") + cudaGetErrorString(e);
    return RTV_ERR_CUDA;
  }
  return tiles ? RTV_OK : fast_prefix_update(ctx, batch, n_vis, st);
}

rtv_status fast_block_embed(rtv_ctx* ctx, const float* rows, int n_src_rows, int G, cudaStream_t st) {
  FastPath* fp = ctx->fast;
  const int T = G * ctx->S;
  norm_input_kernel<float><<<T, 128, 0, st>>>(rows, n_src_rows, ctx->h, ctx->W.layers[0].g_attn, fp->hb, fp->ssp,
                                              round_up(T, 16), ctx->cfg.width);
  const cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) {
    ctx->last_error = std::string("block input launch: ") + cudaGetErrorString(e);
    return RTV_ERR_CUDA;
  }
  return RTV_OK;
}

rtv_status fast_prefill(rtv_ctx* pre, rtv_ctx* ex, const __nv_bfloat16* emb, int P, const float* rope_cs,
                        const float* rope_sn, cudaStream_t st) {
  FastPath* fp = pre->fast;
  FastPath* xp = ex->fast;
  const rtv_expert_config& k = pre->cfg;
  const rtv_expert_config& kx = ex->cfg;
  const int w = k.width, F = k.mlp_dim, D = k.head_dim, Q = pre->Q, KV = pre->KV, L = k.n_layers;
  const int S = pre->S;                       // query rows per attention group (64)
  const int G = (P + S - 1) / S;              // query groups
  const int T = P, n_mma = G * S;             // real token rows; rows of the tiled layouts
  if (!fp || !xp || !xp->tc_attn || !fp->tc_attn || G > pre->Gmax || S != 64 || (P + 63) / 64 + 1 > 16 ||
      (P + 63) / 64 > xp->ntile_max) {
    pre->last_error = "prefill shape not supported by the tensor-core path";
    return RTV_ERR_UNSUPPORTED;
  }
  int n_tt = 1, tt = 16;
  token_tiles(n_mma, &n_tt, &tt);
  const int T_tile = std::min(T, tt);
  const int nq = Q + 2 * KV;
  const GemmPlan p_qkv = plan_gemm(fp, nq, w, tt, T_tile, true, false, n_tt);
  const GemmPlan p_kv = plan_gemm(fp, 2 * KV, w, tt, T_tile, true, false, n_tt);
  const GemmPlan p_o = plan_gemm(fp, w, Q, tt, T_tile, true, false, n_tt);
  // The gate/up projection (no per-token epilogue inputs) takes token tiles
  // of up to 208 rows: more FLOPs per weight and activation byte moved
  // (measured at 816 tokens: 4 tiles of 208 rows 6.33 ms per prefill, 7 of
  // ~128 rows 6.80, 5 of 176 rows 6.58).
  auto wide = [&](int N, int K, int cap, bool with_in) {
    GemmPlan p = plan_gemm(fp, N, K, tt, T_tile, with_in, false, n_tt);
    if (n_mma > cap) {
      const int w_ntt = (n_mma + cap - 1) / cap;
      const int w_tt = round_up((n_mma + w_ntt - 1) / w_ntt, 16);
      const GemmPlan alt = plan_gemm(fp, N, K, w_tt, std::min(T, w_tt), with_in, false, w_ntt);
      if (alt.valid) {
        p = alt;
        p.tt = w_tt;
      }
    }
    return p;
  };
  const GemmPlan p_gu = wide(2 * F, w, 208, false);
  // (the down projection stays on ~128-row tiles: 208-row ones measured 6.46 ms per prefill)
  const GemmPlan p_dn = plan_gemm(fp, w, F, tt, T_tile, true, false, n_tt);
  if (!(p_qkv.valid && p_kv.valid && p_o.valid && p_gu.valid && p_dn.valid)) {
    pre->last_error = "no tensor-core split fits the prefill";
    return RTV_ERR_UNSUPPORTED;
  }
  if (getenv("RTV_LOG")) {
    const GemmPlan* pls[5] = {&p_qkv, &p_kv, &p_o, &p_gu, &p_dn};
    const char* nm[5] = {"qkv", "kv", "o", "gu", "down"};
    for (int i = 0; i < 5; ++i)
      fprintf(stderr, "[rtv] prefill T=%d %s: tiles=%d token_tiles=%d cluster=%d kslice=%d stages=%d smem=%d\n", T,
              nm[i], pls[i]->n_tiles, pls[i]->n_tt, pls[i]->cs, pls[i]->kslice, pls[i]->stages, pls[i]->smem);
  }
  // layer 0's norm input and residual from the embeddings
  norm_input_kernel<__nv_bfloat16><<<T, 128, 0, st>>>(emb, T, pre->h, pre->W.layers[0].g_attn, fp->hb, fp->ssp,
                                                       n_mma, w);
  cudaError_t e = cudaGetLastError();

  GemmArgs base{};
  base.h = pre->h;
  base.hb = fp->hb;
  base.ssp = fp->ssp;
  base.qt = fp->qt;
  base.kts = fp->kts;
  base.vts = fp->vts;
  base.rope_cs = rope_cs;
  base.rope_sn = rope_sn;
  base.m = fp->mb;
  base.status = pre->status;
  base.timeout_ns = k.barrier_timeout_ns;
  base.T = T;
  base.n_mma = n_mma;
  base.tt = tt;
  base.kv_rows = kx.max_prefix_len;
  base.seq = P;
  base.kv_prefix = 1;
  base.w = w;
  base.S = S;
  base.Hq = k.n_q_heads;
  base.Hkv = k.n_kv_heads;
  base.D = D;
  base.F = F;
  base.eps = k.rms_eps;

  AttnTcArgs atc{};
  atc.qt = fp->qt;
  atc.kts = fp->kts;
  atc.vts = fp->vts;
  atc.o = fp->ob;
  atc.part_o = fp->att_po;
  atc.part_ml = fp->att_pml;
  atc.status = pre->status;
  atc.timeout_ns = k.barrier_timeout_ns;
  atc.S = S;
  atc.P = P;
  atc.Hq = k.n_q_heads;
  atc.Hkv = k.n_kv_heads;
  atc.pbs = 0;                      // every query group reads the one prefix
  atc.mask_mode = kMaskPrefixOnly;
  atc.ntile_max = xp->ntile_max;
  atc.n_mma = n_mma;
  atc.scale_log2 = (float)(1.4426950408889634 / sqrt((double)D));
  const int ntp = (P + 63) / 64;
  const size_t kv_layer = (size_t)kx.max_batch * kx.n_kv_heads * kx.max_prefix_len * D;
  const size_t ptile_layer = (size_t)kx.max_batch * kx.n_kv_heads * xp->ntile_max * 64 * D;

  for (int l = 0; l < L && e == cudaSuccess; ++l) {
    const bool last = l == L - 1;
    __nv_bfloat16* kl = (__nv_bfloat16*)ex->prefix_kv + (size_t)(2 * l) * kv_layer;
    // q/k/v of the layer (the last layer: keys and values only, straight
    // into the expert's cache), RoPE at positions 0..P-1
    GemmArgs a = base;
    a.wt = fp->w_qkv;
    a.act = fp->hb;
    a.K = w;
    a.w_tile0 = l * nq / 128;
    a.nt_base = last ? Q / 128 : 0;
    a.ks = kl;
    a.vs = kl + kv_layer;
    a.pf = last ? nullptr : (const uint8_t*)(fp->w_o + (size_t)l * w * Q);
    a.pf_bytes = last ? 0 : (unsigned long long)w * Q * 2;
    e = launch_gemm<GM_QKV>(a, last ? p_kv : p_qkv, st, fp->pf_cap);
    // the layer's cache in the attention's tiles (the expert reads them too)
    if (e == cudaSuccess) {
      prefix_tile_kernel<<<4 * fp->num_sms, 256, 0, st>>>(kl, xp->pkt + (size_t)l * ptile_layer,
                                                         xp->pvt + (size_t)l * ptile_layer, 1, 1, P, k.n_kv_heads,
                                                         D, kx.max_batch, kx.max_prefix_len, xp->ntile_max);
      e = cudaGetLastError();
    }
    if (last) break;
    atc.pkt = xp->pkt + (size_t)l * ptile_layer;
    atc.pvt = xp->pvt + (size_t)l * ptile_layer;
    if (e == cudaSuccess)
      e = D == 256 ? launch_attn_tc<256>(atc, ntp + 1, G, fp->num_sms, st)
                   : launch_attn_tc<128>(atc, ntp + 1, G, fp->num_sms, st);

    a = base;
    a.wt = fp->w_o;
    a.act = fp->ob;
    a.K = Q;
    a.w_tile0 = l * w / 128;
    a.pf = (const uint8_t*)(fp->w_gu + (size_t)l * 2 * F * w);
    a.pf_bytes = (unsigned long long)2 * F * w * 2;
    a.g_next = pre->W.layers[l].g_mlp;
    if (e == cudaSuccess) e = launch_gemm<GM_O>(a, p_o, st, fp->pf_cap);

    a = base;
    a.wt = fp->w_gu;
    a.act = fp->hb;
    a.K = w;
    a.w_tile0 = l * 2 * F / 128;
    a.pf = (const uint8_t*)(fp->w_down + (size_t)l * w * F);
    a.pf_bytes = (unsigned long long)w * F * 2;
    if (e == cudaSuccess) e = launch_gemm<GM_GU>(a, p_gu, st, fp->pf_cap);

    a = base;
    a.wt = fp->w_down;
    a.act = fp->mb;
    a.K = F;
    a.w_tile0 = l * w / 128;
    a.pf = (const uint8_t*)(fp->w_qkv + (size_t)(l + 1) * nq * w);
    a.pf_bytes = (unsigned long long)nq * w * 2;
    a.g_next = pre->W.layers[l + 1].g_attn;
    if (e == cudaSuccess) e = launch_gemm<GM_DOWN>(a, p_dn, st, fp->pf_cap);
  }
  if (e != cudaSuccess) {
    pre->last_error = std::string("prefill launch: ") + cudaGetErrorString(e);
    return RTV_ERR_CUDA;
  }
  return RTV_OK;
}

rtv_status fast_norm_rows(rtv_ctx* ctx, int G, cudaStream_t st) {
  FastPath* fp = ctx->fast;
  const int T = G * ctx->S;
  norm_input_kernel<float><<<T, 128, 0, st>>>(ctx->h, T, nullptr, ctx->W.layers[0].g_attn, fp->hb, fp->ssp,
                                              round_up(T, 16), ctx->cfg.width);
  const cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) {
    ctx->last_error = std::string("norm input launch: ") + cudaGetErrorString(e);
    return RTV_ERR_CUDA;
  }
  return RTV_OK;
}

namespace {

// The layers (see fast_layers); with fold, layer 0 reads its q / suffix K/V
// tiles and O's residual rows from fold and launches no QKV projection; with
// qkv0_only, only layer 0's QKV projection is launched.
rtv_status layers_impl(rtv_ctx* ctx, int G, int P, int prefix_batch_stride, const float* rope_cs,
                       const float* rope_sn, cudaStream_t st, const ModTables* mod, const FoldedQueries* fold,
                       bool qkv0_only) {
  FastPath* fp = ctx->fast;
  const rtv_expert_config& k = ctx->cfg;
  const int S = ctx->S, T = G * S, w = k.width, F = k.mlp_dim, D = k.head_dim, Q = ctx->Q, KV = ctx->KV;
  const int n_mma = round_up(T, 16);   // rows of the tiled activation layout
  int n_tt = 1, tt = 16;               // default token tiles (each plan may choose its own)
  token_tiles(n_mma, &n_tt, &tt);
  const int nq = Q + 2 * KV;
  const GemmPlan p_qkv = plan_suffix(fp, nq, w, n_mma, T, true, false);
  const GemmPlan p_o = plan_suffix(fp, w, Q, n_mma, T, true, false);
  const GemmPlan p_gu = plan_suffix(fp, 2 * F, w, n_mma, T, false, fp->mlp_f8);
  const GemmPlan p_dn = plan_suffix(fp, w, F, n_mma, T, true, fp->mlp_f8);
  const int nk = P + S;
  const int nchunk = attn_chunks(fp, nk, k.n_q_heads * G);
  if (!(p_qkv.valid && p_o.valid && p_gu.valid && p_dn.valid) ||
      attn_smem_bytes(D) > kDynSmemMax || nchunk > 16) {
    ctx->last_error = "no tensor-core split fits this token count";
    return RTV_ERR_UNSUPPORTED;
  }
  if (getenv("RTV_LOG")) {
    const GemmPlan* pls[4] = {&p_qkv, &p_o, &p_gu, &p_dn};
    const char* nm[4] = {"qkv", "o", "gu", "down"};
    for (int i = 0; i < 4; ++i)
      fprintf(stderr, "[rtv] T=%d %s: tiles=%d token_tiles=%d x %d cluster=%d kslice=%d stages=%d smem=%d\n", T,
              nm[i], pls[i]->n_tiles, pls[i]->n_tt, pls[i]->tt, pls[i]->cs, pls[i]->kslice, pls[i]->stages,
              pls[i]->smem);
    fprintf(stderr, "[rtv] gemm clusters that fit (size: two-per-SM budget / whole smem):");
    for (int cs = 1; cs <= 16; cs <<= 1) fprintf(stderr, " %d: %d/%d", cs, fp->gemm_fit_small[cs], fp->gemm_fit_large[cs]);
    fprintf(stderr, "\n");
    fprintf(stderr, "[rtv] attention: chunks=%d keys/chunk=%d smem=%d max_cluster=%d sms=%d fit(8,12,16)=%d,%d,%d\n",
            nchunk, (nk + nchunk - 1) / nchunk, attn_smem_bytes(D), fp->max_cluster,
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
  base.tt = tt;
  base.kv_rows = S;
  base.seq = S;
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
  at.part_o = fp->att_po;
  at.part_ml = fp->att_pml;
  at.status = ctx->status;
  at.S = S;
  at.P = P;
  at.Pmax = k.max_prefix_len;
  at.Hq = k.n_q_heads;
  at.Hkv = k.n_kv_heads;
  at.pbs = prefix_batch_stride;
  at.mask_mode = k.suffix_mask;
  at.kpc = (nk + nchunk - 1) / nchunk;
  at.n_mma = n_mma;
  at.scale_log2 = (float)(1.4426950408889634 / sqrt((double)D));
  const size_t kv_layer = (size_t)k.max_batch * k.n_kv_heads * k.max_prefix_len * D;

  // tensor-core attention when the pair layout applies and every key tile has
  // a rank (RTV_ATTN=mma selects the warp-MMA kernel instead)
  const int ntp = (P + 63) / 64;
  const bool tc_att = fast_tc_attention(ctx, P);
  AttnTcArgs atc{};
  if (tc_att) {
    base.qt = fp->qt;
    base.kts = fp->kts;
    base.vts = fp->vts;
    atc.qt = fp->qt;
    atc.kts = fp->kts;
    atc.vts = fp->vts;
    atc.o = fp->ob;
    atc.part_o = fp->att_po;
    atc.part_ml = fp->att_pml;
    atc.status = ctx->status;
    atc.timeout_ns = k.barrier_timeout_ns;
    atc.S = S;
    atc.P = P;
    atc.Hq = k.n_q_heads;
    atc.Hkv = k.n_kv_heads;
    atc.pbs = prefix_batch_stride;
    atc.mask_mode = k.suffix_mask;
    atc.ntile_max = fp->ntile_max;
    atc.n_mma = n_mma;
    atc.scale_log2 = at.scale_log2;
    // a bare block's cached prefix (the draft's visual keys and values) is
    // written by the kernel just before the layers
    atc.prefix_after_wait = ctx->block_only ? 1 : 0;
  }
  const size_t ptile_layer = (size_t)k.max_batch * k.n_kv_heads * fp->ntile_max * 64 * D;

  const bool tracing = fp->trace_armed && fp->trace != nullptr;
  fp->trace_armed = false;
  if (tracing) {
    fp->trace_ctas[0] = std::min(512, p_qkv.n_tiles * p_qkv.cs * p_qkv.n_tt);
    fp->trace_ctas[1] = std::min(512, p_o.n_tiles * p_o.cs * p_o.n_tt);
    fp->trace_ctas[2] = std::min(512, p_gu.n_tiles * p_gu.cs * p_gu.n_tt);
    fp->trace_ctas[3] = std::min(512, p_dn.n_tiles * p_dn.cs * p_dn.n_tt);
    fp->trace_ctas[4] = std::min(512, tc_att ? (ntp + 1) * (k.n_q_heads / 2) * G : nchunk * k.n_q_heads * G);
  }
  auto tr = [&](int l, int i) -> unsigned long long* {
    return (tracing && l == 0) ? fp->trace + (size_t)i * 512 * kTraceRow : nullptr;
  };
  if ((fold || qkv0_only) && !tc_att) {
    ctx->last_error = "folded query rows need the tensor-core attention";
    return RTV_ERR_UNSUPPORTED;
  }

  // per-layer time modulator rows (RTV_TIME_ADARMS): group strides
  const int L6 = k.n_layers * 6 * w;
  const int mg = mod ? mod->group_rows : 0;
  for (int l = 0; l < k.n_layers; ++l) {
    const LayerW& Lw = ctx->W.layers[l];
    const float* ml = mod ? mod->mod + (size_t)l * 6 * w : nullptr;
    GemmArgs a = base;
    a.trace = tr(l, 0);
    if (mod) {
      a.sb = mod->sbq + (size_t)l * nq;
      a.sb_stride = mg * k.n_layers * nq;
    }
    a.wt = fp->w_qkv;
    a.act = fp->hb;
    a.K = w;
    a.w_tile0 = l * nq / 128;
    a.pf = (const uint8_t*)(fp->w_o + (size_t)l * w * Q);
    a.pf_bytes = (unsigned long long)w * Q * 2;
    const bool folded = fold && l == 0;
    cudaError_t e = folded ? cudaSuccess : launch_gemm<GM_QKV>(a, p_qkv, st, fp->pf_cap);
    if (qkv0_only) {
      if (e != cudaSuccess) {
        ctx->last_error = std::string("tensor-core launch: ") + cudaGetErrorString(e);
        return RTV_ERR_CUDA;
      }
      return RTV_OK;
    }

    if (tc_att) {
      AttnTcArgs atl = atc;
      atl.trace = tr(l, 4);
      atl.pkt = fp->pkt + (size_t)l * ptile_layer;
      atl.pvt = fp->pvt + (size_t)l * ptile_layer;
      if (folded) {
        atl.qt = fold->qt;
        atl.kts = fold->kts;
        atl.vts = fold->vts;
      }
      if (e == cudaSuccess)
        e = D == 256 ? launch_attn_tc<256>(atl, ntp + 1, G, fp->num_sms, st)
                     : launch_attn_tc<128>(atl, ntp + 1, G, fp->num_sms, st);
    } else {
      at.trace = tr(l, 4);
      at.pk = (const __nv_bfloat16*)ctx->prefix_kv + (size_t)(2 * l) * kv_layer;
      at.pv = (const __nv_bfloat16*)ctx->prefix_kv + (size_t)(2 * l + 1) * kv_layer;
      if (e == cudaSuccess) e = D == 256 ? launch_attn<256>(at, nchunk, G, st) : launch_attn<128>(at, nchunk, G, st);
    }

    a = base;
    a.trace = tr(l, 1);
    a.wt = fp->w_o;
    a.act = fp->ob;
    a.K = Q;
    a.w_tile0 = l * w / 128;
    a.pf = fp->mlp_f8 ? fp->w_gu8 + (size_t)l * 2 * F * w : (const uint8_t*)(fp->w_gu + (size_t)l * 2 * F * w);
    a.pf_bytes = (unsigned long long)2 * F * w * (fp->mlp_f8 ? 1 : 2);
    a.g_next = Lw.g_mlp;
    if (folded) a.h_in = fold->h0;
    if (mod) {
      a.gate = ml + 2 * w;
      a.gate_stride = mg * L6;
      a.g_next = ml + 3 * w;
      a.g_stride = mg * L6;
    }
    if (e == cudaSuccess) e = launch_gemm<GM_O>(a, p_o, st, fp->pf_cap);

    a = base;
    a.trace = tr(l, 2);
    a.wt = fp->w_gu;
    a.wt8 = fp->mlp_f8 ? fp->w_gu8 : nullptr;
    a.wscale = fp->mlp_f8 ? fp->gu_s + (size_t)l * 2 * F : nullptr;
    a.act = fp->hb;
    a.K = w;
    a.w_tile0 = l * 2 * F / 128;
    a.pf = fp->mlp_f8 ? fp->w_down8 + (size_t)l * w * F : (const uint8_t*)(fp->w_down + (size_t)l * w * F);
    a.pf_bytes = (unsigned long long)w * F * (fp->mlp_f8 ? 1 : 2);
    if (mod) {
      a.sb = mod->sbg + (size_t)l * 2 * F;
      a.sb_stride = mg * k.n_layers * 2 * F;
    }
    if (e == cudaSuccess) e = launch_gemm<GM_GU>(a, p_gu, st, fp->pf_cap);

    a = base;
    a.trace = tr(l, 3);
    a.wt = fp->w_down;
    a.wt8 = fp->mlp_f8 ? fp->w_down8 : nullptr;
    a.wscale = fp->mlp_f8 ? fp->down_s + (size_t)l * w : nullptr;
    a.act = fp->mb;
    a.K = F;
    a.w_tile0 = l * w / 128;
    a.pf = (const uint8_t*)(fp->w_qkv + (size_t)((l + 1) % k.n_layers) * nq * w);
    a.pf_bytes = (unsigned long long)nq * w * 2;
    a.g_next = (l + 1 < k.n_layers) ? ctx->W.layers[l + 1].g_attn : nullptr;
    if (mod) {
      a.gate = ml + 5 * w;
      a.gate_stride = mg * L6;
      a.g_next = (l + 1 < k.n_layers) ? ml + 6 * w : nullptr;   // scale_a of the next layer
      a.g_stride = mg * L6;
    }
    if (e == cudaSuccess) e = launch_gemm<GM_DOWN>(a, p_dn, st, fp->pf_cap);
    if (e != cudaSuccess) {
      ctx->last_error = std::string("tensor-core launch: ") + cudaGetErrorString(e);
      return RTV_ERR_CUDA;
    }
  }
  return RTV_OK;
}

}  // namespace

rtv_status fast_layers(rtv_ctx* ctx, int G, int P, int prefix_batch_stride, const float* rope_cs,
                       const float* rope_sn, cudaStream_t st, const ModTables* mod, const FoldedQueries* fold) {
  return layers_impl(ctx, G, P, prefix_batch_stride, rope_cs, rope_sn, st, mod, fold, false);
}

void folded_sizes(const rtv_ctx* ctx, int G, size_t bytes[4]) {
  const rtv_expert_config& k = ctx->cfg;
  const size_t D = k.head_dim;
  bytes[0] = (size_t)G * (k.n_q_heads / 2) * 128 * D * 2;    // q tiles of the head pairs
  bytes[1] = (size_t)G * k.n_kv_heads * 64 * D * 2;           // suffix key tiles
  bytes[2] = bytes[1];                                        // suffix value tiles (transposed)
  bytes[3] = (size_t)G * ctx->S * k.width * sizeof(float);    // residual rows
}

rtv_status fast_block_fold(rtv_ctx* ctx, const float* rows, int n_src_rows, int G, int P, const float* rope_cs,
                           const float* rope_sn, const FoldedQueries& f, cudaStream_t st) {
  FastPath* fp = ctx->fast;
  rtv_status s = fast_block_embed(ctx, rows, n_src_rows, G, st);
  if (s == RTV_OK) s = layers_impl(ctx, G, P, 1, rope_cs, rope_sn, st, nullptr, nullptr, true);
  if (s != RTV_OK) return s;
  size_t bytes[4];
  folded_sizes(ctx, G, bytes);
  const void* from[4] = {fp->qt, fp->kts, fp->vts, ctx->h};
  void* to[4] = {f.qt, f.kts, f.vts, f.h0};
  for (int i = 0; i < 4; ++i) {
    const cudaError_t e = cudaMemcpyAsync(to[i], from[i], bytes[i], cudaMemcpyDeviceToDevice, st);
    if (e != cudaSuccess) {
      ctx->last_error = std::string("folding the query rows: ") + cudaGetErrorString(e);
      return RTV_ERR_CUDA;
    }
  }
  return RTV_OK;
}

bool fast_views(const rtv_ctx* ctx, FastViews* out) {
  const FastPath* fp = ctx->fast;
  // (the packed weights exist only after rtv_load_expert; callers check them before use)
  if (!fp || !fp->tc_attn || !fp->pkt || ctx->cfg.mlp_dtype == RTV_FP8_E4M3) return false;
  out->w_qkv = fp->w_qkv;
  out->w_o = fp->w_o;
  out->w_gu = fp->w_gu;
  out->w_down = fp->w_down;
  out->w_aiT = fp->w_aiT;
  out->w_spT = fp->w_spT;
  out->pkt = fp->pkt;
  out->pvt = fp->pvt;
  out->ntile_max = fp->ntile_max;
  out->num_sms = fp->num_sms;
  return true;
}

void fast_destroy(rtv_ctx* ctx) {
  if (!ctx->fast) return;
  for (void* p : ctx->fast->allocs) cudaFree(p);
  delete ctx->fast;
  ctx->fast = nullptr;
}

}  // namespace rtv
