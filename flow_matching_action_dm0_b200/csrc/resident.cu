// Resident (persistent) kernel of the bf16 action expert on sm_100a.
//
// One launch runs every Euler step of a chunk ("DM0.5 reading guide",
// sec. 5.3 Euler sampling), or the one velocity evaluation of a FLASH
// verification ("Realtime-VLA FLASH", sec. 02), with one CTA per SM.  The
// work of a step is a sequence of phases separated by grid-wide barriers:
//   HE    output head + Euler update of the previous step, suffix embedding
//         (state_proj / action_in_proj + time condition) of the next one
//   per layer (sec. 5.2 action expert):
//   QKV   q/k/v projection of RMSNorm(h)
//   ATTN  attention of the suffix queries over [prefix KV ; own suffix]
//   O     attention output projection, added to the residual
//   GU    gate/up projection of RMSNorm(h)
//   DOWN  down projection of gelu_tanh(gate) * up, added to the residual
//
// Why one resident kernel: at 51 token rows every projection is bound by its
// weight bytes, and the weights do not depend on the activations.  Each CTA
// owns a fixed share of every projection (a "unit": some 128-row weight tiles
// over a range of 64-wide K boxes) for the whole launch, and warp 0 streams
// the CTA's weight boxes -- for this phase, the next, the next layer's --
// through a ring of shared-memory stages without regard to phase boundaries:
// only the ring's depth limits how far ahead it runs.  The barriers, the
// epilogues and the attention happen while the next phases' weights land.
//
// Data flow.  The projections are computed swapped (D = W x act^T on tcgen05,
// M = 128 weight rows, N = the token rows padded to 16) and split over K, so
// a unit's accumulator is a partial sum: the worker warps stage it in shared
// memory and add it into an fp32 sum in global memory (L2) with bulk
// reductions (cp.reduce.async.bulk .add.f32).  Every fp32 sum is stored
// box-major, [feature / 64][token row][64], so that the 64 features of one
// K box over all token rows are one contiguous bulk copy for the phase that
// consumes them.  That phase's prologue copies each of its boxes into shared
// memory, applies the non-linear step that follows the projection and writes
// the bf16 operand box, box by box, with the MMAs of a box starting as soon
// as it is written:
//   * RMSNorm is split: the QKV / GU prologues convert bf16(h * (1 + g)) and
//     add the sum of squares of h over their K range (the units of weight
//     tile 0 cover K exactly once); the next phase applies
//     1/rms = rsqrt(sum / width + eps), a per-token factor that commutes with
//     the projection (attention for q/k/v, DOWN prologue for gate/up).
//   * gelu_tanh(gate) * up is formed in the DOWN prologue.
//   * Attention: every CTA first turns a share of the q/k/v sums into bf16
//     operand tiles (1/rms, RoPE at the suffix position), published through
//     a counter; then each attention item -- 128 query rows against one
//     64-key tile -- copies its tiles in and runs S = Q K^T and P V on the
//     tensor cores.  A prefix tile exponentiates against a common reference
//     for its row, the Cauchy-Schwarz bound |q| max|k| / sqrt(D) on every
//     prefix score (no score exceeds it, so no term overflows; the prefix
//     keys' norms are measured at the start of the launch); the row's own
//     suffix tile uses its exact maximum.  Every key tile stores its P V rows
//     and row sums in a slot of its own (no contended additions), a second
//     counter publishes them, and every CTA combines a share of the rows --
//     the prefix slots' sum and the suffix slot, each weighted by its
//     reference -- into the O projection's bf16 operand boxes.  No
//     synchronisation among the key tiles is needed before the combine.
// The residual stream h is an fp32 sum updated in place by the O and DOWN
// reductions.  fp32 additions in the order the reductions arrive: results
// are reproducible to rounding, not bit for bit.
//
// Every spin-wait is bounded (globaltimer, barrier_timeout_ns).  A CTA whose
// wait gives up records RTV_DEV_TIMEOUT and raises an abort bit in the grid
// counters; every role then stops issuing work, waits for the copies, MMAs and
// reductions it already issued (they complete without help from other CTAs),
// frees its tensor memory and returns.  The worker warps take every decision
// to leave a phase at a barrier that reduces a predicate over all of them,
// so none of them can leave for a path whose barrier the others never reach.
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <math.h>
#include <stdio.h>
#include <stdlib.h>
#include <string.h>

#include <algorithm>
#include <map>
#include <string>
#include <tuple>
#include <vector>

#include "common.cuh"
#include "fastpath.h"
#include "kernels.h"
#include "resident.h"
#include "runtime.h"
#include "tc_ptx.cuh"

namespace rtv {

namespace {

constexpr int kRWarps = 10;                 // warp 0 weights, warp 1 MMA, warps 2..9 workers
constexpr int kRThreads = 32 * kRWarps;
constexpr int kWThreads = 256;              // worker threads
constexpr int kMaxStages = 16;
constexpr int kMaxBoxes = 16;               // K boxes of one unit
constexpr unsigned kAbortBit = 0x80000000u;
constexpr int kBox = 16384;                 // one 128 x 64 bf16 weight box
constexpr int kPlanInts = 24;               // per CTA: see the PL_* slots
constexpr int kTraceSlots = 104;            // per CTA: [12 phases][8 stamps], then the start
constexpr int kTracePhases = 12;
constexpr long long kDrainNs = 1000000000ll;   // drain waits: copies and MMAs already issued complete on their own
// Plan record of one CTA: ring stages, scratch offset and size, the unit of
// each of the four projections (first tile, tiles, first K box, K boxes;
// tiles = 0: none), the attention item (-1: none).
enum { PL_NS = 0, PL_SCR = 1, PL_SCR_BYTES = 2, PL_UNIT = 3, PL_ATT = 19 };
enum { PH_QKV = 0, PH_O = 1, PH_GU = 2, PH_DOWN = 3 };
constexpr int kTmemCols = 512;
constexpr int kAttOCol = 256;               // attention P V accumulator columns [256, 256 + D)

struct ResArgs {
  const __nv_bfloat16* wts[4]; // packed weights of QKV, O, GU, DOWN, all layers [L*R][KB][128][64]
  int R[4], KB[4];             // 128-row tiles per layer and 64-wide K boxes of each projection
  const float* g_attn;         // [L][w] attention-norm gains
  const float* g_mlp;          // [L][w] MLP-norm gains
  const __nv_bfloat16* pkt;    // prefix key tiles   [L][Bmax][Hkv][ntile_max][64][D]
  const __nv_bfloat16* pvt;    // prefix value tiles [L][Bmax][Hkv][ntile_max][D][64] (transposed)
  const float* rope_cs;        // [S][D/2]
  const float* rope_sn;
  const __nv_bfloat16* w_ao;   // [A][w]
  const float* b_ao;
  const float* g_final;
  const __nv_bfloat16* w_aiT;  // [A][w]
  const float* b_ai;
  const __nv_bfloat16* w_spT;  // [Sd][w]
  const float* b_sp;
  const float* c;              // time condition rows: c + step * c_step + g * c_group
  int c_step, c_group;
  const float* state;          // group g reads state + g * state_stride ([Sd])
  int state_stride;
  float* x;                    // [G][H][A] Euler state (verification: the interpolated X)
  float* vout;                 // [G][H][A] velocity (verification) or nullptr
  // fp32 sums, box-major [feature / 64][n_mma][64]
  float* hres;                 // residual h (w features)
  float* qkv;                  // q/k/v (packed QKV rows: box 2*tile + half)
  float* gu;                   // gate/up (packed rows: box 2*tile = gate, 2*tile + 1 = up)
  // attention, per query row gr = (g*Hq + j)*S + s
  float* att_slot;             // [ntp + 1][D/64][R_att][64] P V rows of each key tile (the last: the suffix)
  float* l_slot;               // [ntp + 1][R_att] their row sums
  float* m_ref;                // [R_att] the prefix tiles' common reference (log2 units)
  float* m_suf;                // [R_att] the suffix tile's row maximum
  __nv_bfloat16* o_att;        // attention output, the O projection's input boxes [Hq*D/64][n_mma][64] (swizzled)
  __nv_bfloat16* q_pre;        // query tiles of the prefix items [n_pg*nrt_pre][D/64][128][64]
  __nv_bfloat16* q_suf;        // query tiles of the suffix items [G*Hkv*nrt_suf][D/64][128][64]
  __nv_bfloat16* k_suf;        // suffix keys   [G*Hkv][D/64][64][64]
  __nv_bfloat16* v_suf;        // suffix values [G*Hkv][D][64] (transposed)
  float* kmax;                 // [L][Bmax*Hkv] largest prefix key norm (measured in phase 0)
  float* ss1;                  // sums of squares of h (attention norm) [n_mma]
  float* ss2;                  // (MLP norm) [n_mma]
  unsigned* bar;               // [0] grid counter, [1] attention operands written, [2] key tiles' rows written
  unsigned* status;
  unsigned long long* trace;   // [ncta][kTraceSlots] or nullptr
  const int* plan;             // [ncta][kPlanInts]
  long long timeout_ns;
  int L, w, Hq, Hkv, D, F, S, G, T, n_mma, A, Sd, P, Bmax, ntile_max, mask_mode, n_steps, verify;
  // attention geometry (see att_geometry)
  int hpk, rows_pg, nrt_pre, ntp, rows_suf, nrt_suf, n_pre, n_items, R_att;
  int col_stride;              // TMEM columns between the accumulators of a unit's tiles
  int pace_ns;                 // least time between two weight copies of a CTA (0: as fast as the ring allows)
  int dyn_smem;                // dynamic shared memory the plan assumes
  float dt, eps, scale_log2;
};

__device__ __forceinline__ unsigned ld_acquire(const unsigned* p) {
  unsigned v;
  asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}
__device__ __forceinline__ void red_release(unsigned* p, unsigned v) {
  asm volatile("red.release.gpu.global.add.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}
// dst[i] += src[i] for `bytes` of fp32 (global += shared), as one bulk operation.
__device__ __forceinline__ void bulk_reduce_add(float* dst, uint32_t src_smem, uint32_t bytes) {
  asm volatile("cp.reduce.async.bulk.global.shared::cta.bulk_group.add.f32 [%0], [%1], %2;" ::"l"(dst),
               "r"(src_smem), "r"(bytes)
               : "memory");
}
// dst = src for `bytes` (global <- shared), as one bulk operation.
__device__ __forceinline__ void bulk_store(void* dst, uint32_t src_smem, uint32_t bytes) {
  asm volatile("cp.async.bulk.global.shared::cta.bulk_group [%0], [%1], %2;" ::"l"(dst), "r"(src_smem), "r"(bytes)
               : "memory");
}
__device__ __forceinline__ void bulk_commit() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
__device__ __forceinline__ void bulk_wait_all() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }
__device__ __forceinline__ void bulk_wait_read_all() { asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory"); }
__device__ __forceinline__ void fence_async_global() { asm volatile("fence.proxy.async.global;" ::: "memory"); }
__device__ __forceinline__ void workers_sync() { asm volatile("bar.sync 1, %0;" ::"n"(kWThreads) : "memory"); }
// Barrier of the worker threads that also returns, to every one of them, the
// OR of their predicates: decisions taken after it are uniform, so no worker
// warp can leave for a path whose named barrier the others never reach.
__device__ __forceinline__ bool workers_any(bool v) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\tsetp.ne.u32 q, %1, 0;\n\tbar.red.or.pred p, 1, %2, q;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(r)
      : "r"((uint32_t)v), "n"(kWThreads)
      : "memory");
  return r != 0;
}
__device__ __forceinline__ uint32_t dyn_smem_size() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%dynamic_smem_size;" : "=r"(r));
  return r;
}

// Byte offset of the 16-byte chunk c of row t in a [rows][64] bf16 operand
// box with the tensor cores' 128-byte swizzle.
__device__ __forceinline__ uint32_t sw_chunk(int t, int c) { return (uint32_t)(t * 128 + ((c ^ (t & 7)) << 4)); }
// Element offset of (row, col) in such a box.
__device__ __forceinline__ int sw_elem(int row, int col) { return row * 64 + ((((col >> 3) ^ (row & 7))) << 3) + (col & 7); }

__device__ __forceinline__ uint4 pack8(const float* v) {
  uint4 u;
  u.x = ptx::pack_bf16x2(v[0], v[1]);
  u.y = ptx::pack_bf16x2(v[2], v[3]);
  u.z = ptx::pack_bf16x2(v[4], v[5]);
  u.w = ptx::pack_bf16x2(v[6], v[7]);
  return u;
}
__device__ __forceinline__ void ld8_smem(const float* p, float* v) {
  const float4 a = *reinterpret_cast<const float4*>(p);
  const float4 b = *reinterpret_cast<const float4*>(p + 4);
  v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
  v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
}
__device__ __forceinline__ void ld8_ro(const float* p, float* v) {
  const float4 a = __ldg(reinterpret_cast<const float4*>(p));
  const float4 b = __ldg(reinterpret_cast<const float4*>(p + 4));
  v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
  v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
}

// Shared state of the roles of one CTA.
struct Ctl {
  uint64_t full[kMaxStages];    // weight box landed
  uint64_t empty[kMaxStages];   // its MMAs completed
  uint64_t act_full[kMaxBoxes]; // activation box j of the phase written (8 worker warps arrive)
  uint64_t mma_done;            // the phase's MMAs completed
  uint64_t stg[kMaxBoxes];      // prologue staging buffer landed
  uint64_t att_ld;              // attention Q, K, V tiles landed
  uint64_t att_s;               // S = Q K^T completed
  uint64_t att_pv;              // O = P V completed
  uint64_t fin;                 // every MMA of the MMA warp completed (exit)
  uint32_t tmem;
  int abort;
};

// Bounded wait on an mbarrier phase; false when the CTA is aborting or the
// limit passed (the caller records the timeout).
__device__ __forceinline__ bool mwait(uint64_t* bar, uint32_t parity, long long limit, volatile int* abort) {
  if (ptx::mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = ptx::globaltimer();
  while (true) {
    if (ptx::mbar_try_wait(bar, parity)) return true;
    if (*abort) return false;
    if ((long long)(ptx::globaltimer() - t0) > limit) return false;
  }
}
// Wait with a fixed limit whatever the abort state: for copies and MMAs this
// CTA issued, which complete without help from other CTAs.
__device__ __forceinline__ void drain_wait(uint64_t* bar, uint32_t parity) {
  int never = 0;
  mwait(bar, parity, kDrainNs, &never);
}

__device__ __noinline__ void raise_abort(const ResArgs& a, Ctl* ctl, bool timed_out) {
  if (timed_out) atomicOr(a.status, RTV_DEV_TIMEOUT);
  ctl->abort = 1;
  atomicOr(&a.bar[0], kAbortBit);
  atomicOr(&a.bar[1], kAbortBit);
  atomicOr(&a.bar[2], kAbortBit);
}

// Wait until counter >= target (or its abort bit is set); false on abort or timeout.
__device__ __noinline__ bool counter_wait(const ResArgs& a, Ctl* ctl, const unsigned* ctr, unsigned target) {
  unsigned v = ld_acquire(ctr);
  if (v < target) {
    const uint64_t t0 = ptx::globaltimer();
    while ((v = ld_acquire(ctr)) < target) {
      if ((long long)(ptx::globaltimer() - t0) > a.timeout_ns) {
        raise_abort(a, ctl, true);
        return false;
      }
    }
  }
  if (v & kAbortBit) {
    ctl->abort = 1;
    return false;
  }
  // what other CTAs wrote (generic stores or bulk operations) before their
  // release is read next by this CTA's bulk copies too: order the async proxy
  // after the acquire
  fence_async_global();
  return true;
}

struct Unit {
  int tile0, nt, kb0, nb;
};

// ---------------------------------------------------------------------------
// Attention geometry.  Query rows are numbered globally gr = (g*Hq + j)*S + s
// (suffix group g, head j, suffix row s).  A prefix item covers 128 rows of a
// prefix group -- the heads of one kv head over the groups that read the same
// cached prefix (all taus when verifying, one batch element when denoising)
// -- against one 64-key prefix tile; a suffix item covers 128 rows of one
// (group, kv head) against that group's own suffix keys.
// ---------------------------------------------------------------------------
struct AttRow {
  int g, j, s;
};
__device__ __forceinline__ AttRow pre_row(const ResArgs& a, int pg, int i) {
  const int b = pg / a.Hkv, kvh = pg - b * a.Hkv;
  const int per_g = a.hpk * a.S;
  const int gl = i / per_g, rem = i - gl * per_g;
  const int jl = rem / a.S;
  AttRow r;
  r.g = a.verify ? gl : b;
  r.j = kvh * a.hpk + jl;
  r.s = rem - jl * a.S;
  return r;
}
__device__ __forceinline__ AttRow suf_row(const ResArgs& a, int g, int kvh, int i) {
  const int jl = i / a.S;
  AttRow r;
  r.g = g;
  r.j = kvh * a.hpk + jl;
  r.s = i - jl * a.S;
  return r;
}

// ---------------------------------------------------------------------------
// The kernel
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(kRThreads, 1) resident_kernel(const ResArgs a) {
  extern __shared__ uint8_t smem_raw[];
  __shared__ Ctl ctl;
  __shared__ float s_rs[256];        // per-token 1/rms of the phase
  __shared__ float s_ss[256];        // per-token partial sums of squares
  __shared__ float s_ca[256], s_cb[256];   // O prologue: per-token weights of the two attention sums
  __shared__ float s_red[2][128];    // attention: per-row halves (max, then sum)
  __shared__ float s_wred[8];
  __shared__ int s_gr[128];          // attention: global row index of each tile row (-1: padding)
  __shared__ unsigned s_brk[4];      // attention: rows where a run of consecutive global rows breaks
  const int cta = blockIdx.x, ncta = gridDim.x;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int* pl = a.plan + (size_t)cta * kPlanInts;
  const int NS = pl[PL_NS];
  uint8_t* base = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  uint8_t* scr = base + pl[PL_SCR];
  const int scr_bytes = pl[PL_SCR_BYTES];
  // every CTA checks the same launch-wide values, so a refusal is uniform
  if (dyn_smem_size() < (uint32_t)a.dyn_smem || NS < 2 || NS > kMaxStages || a.n_mma > 256 || a.T > a.n_mma ||
      a.S > 64 || a.D > 256 || (a.D & 127) || a.w > 4096 || a.A > 64 || a.Sd > 64 ||
      pl[PL_SCR] + scr_bytes + 1024 > a.dyn_smem) {
    if (threadIdx.x == 0) atomicOr(a.status, RTV_DEV_BOUNDS);
    return;
  }
  unsigned long long* trace = a.trace ? a.trace + (size_t)cta * kTraceSlots : nullptr;
  if (threadIdx.x == 0) {
    for (int i = 0; i < NS; ++i) {
      ptx::mbar_init(&ctl.full[i], 1);
      ptx::mbar_init(&ctl.empty[i], 1);
    }
    for (int j = 0; j < kMaxBoxes; ++j) ptx::mbar_init(&ctl.act_full[j], kWThreads / 32);
    ptx::mbar_init(&ctl.mma_done, 1);
    for (int j = 0; j < kMaxBoxes; ++j) ptx::mbar_init(&ctl.stg[j], 1);
    ptx::mbar_init(&ctl.att_ld, 1);
    ptx::mbar_init(&ctl.att_s, 1);
    ptx::mbar_init(&ctl.att_pv, 1);
    ptx::mbar_init(&ctl.fin, 1);
    ctl.abort = 0;
    ptx::fence_mbar_init();
  }
  if (warp == 1) {
    ptx::tmem_alloc(&ctl.tmem, kTmemCols);
    ptx::tmem_relinquish();
  }
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  const uint32_t tmem = ctl.tmem;
  volatile int* abort = &ctl.abort;
  const int n_evals = a.verify ? 1 : a.n_steps;

  if (warp == 0) {
    // ======================= weight producer =========================
    if (lane == 0) {
      const uint64_t pol = ptx::policy_evict_first();
      const int item = pl[PL_ATT];
      int b = 0;
      bool stop = false;
      uint64_t last_issue = 0;
      for (int step = 0; step < n_evals && !stop; ++step) {
        for (int l = 0; l < a.L && !stop; ++l) {
          // this layer's prefix key/value tiles into L2 ahead of the attention phase
          if (item >= 0 && item < a.n_pre) {
            const int kt = item % a.ntp, pg = item / (a.nrt_pre * a.ntp);
            const int pb = a.verify ? 0 : pg / a.Hkv, kvh = pg % a.Hkv;
            const size_t tile = (((size_t)l * a.Bmax + pb) * a.Hkv + kvh) * a.ntile_max + kt;
            ptx::prefetch_l2_bulk(a.pkt + tile * 64 * a.D, (uint32_t)(64 * a.D * 2));
            ptx::prefetch_l2_bulk(a.pvt + tile * 64 * a.D, (uint32_t)(64 * a.D * 2));
          }
          for (int ph = 0; ph < 4 && !stop; ++ph) {
            const int* u = pl + PL_UNIT + 4 * ph;
            if (u[1] == 0) continue;
            const __nv_bfloat16* wl = a.wts[ph] + (size_t)l * a.R[ph] * a.KB[ph] * 8192;
            for (int kb = u[2]; kb < u[2] + u[3] && !stop; ++kb) {
              for (int tt = 0; tt < u[1]; ++tt) {
                const int s = b % NS;
                if (b >= NS && !mwait(&ctl.empty[s], ((b / NS) - 1) & 1, a.timeout_ns, abort)) {
                  if (!*abort) raise_abort(a, &ctl, true);
                  stop = true;
                  break;
                }
                if (a.pace_ns > 0) {
                  // spread this SM's weight traffic over time instead of bursts
                  while ((long long)(ptx::globaltimer() - last_issue) < a.pace_ns) {
                  }
                  last_issue = ptx::globaltimer();
                }
                ptx::mbar_expect_tx(&ctl.full[s], (uint32_t)kBox);
                ptx::bulk_load_hint(base + (size_t)s * kBox, wl + ((size_t)(u[0] + tt) * a.KB[ph] + kb) * 8192,
                                    (uint32_t)kBox, &ctl.full[s], pol);
                ++b;
              }
            }
          }
        }
      }
      // never leave with a copy still landing in shared memory
      const int issued = b;
      for (int s = 0; s < NS && s < issued; ++s) {
        const int last = s + ((issued - 1 - s) / NS) * NS;
        drain_wait(&ctl.full[s], (last / NS) & 1);
      }
    }
  } else if (warp == 1) {
    // ======================= MMA issue =========================
    if (lane == 0) {
      const uint32_t idesc = ptx::idesc_bf16_f32(128, a.n_mma);
      const uint32_t act_bytes = (uint32_t)a.n_mma * 128u;
      int au[kMaxBoxes];
      for (int j = 0; j < kMaxBoxes; ++j) au[j] = 0;
      int b = 0, issued = 0;
      bool stop = false;
      for (int step = 0; step < n_evals && !stop; ++step) {
        for (int l = 0; l < a.L && !stop; ++l) {
          for (int ph = 0; ph < 4 && !stop; ++ph) {
            const int* u = pl + PL_UNIT + 4 * ph;
            if (u[1] == 0) continue;
            for (int kb = 0; kb < u[3] && !stop; ++kb) {
              // activation box kb of this phase, written by the workers
              if (!mwait(&ctl.act_full[kb], au[kb] & 1, a.timeout_ns, abort)) {
                if (!*abort) raise_abort(a, &ctl, true);
                stop = true;
                break;
              }
              ++au[kb];
              ptx::tc_fence_after();
              const uint32_t aa = ptx::smem_u32(scr + (size_t)kb * act_bytes);
              for (int tt = 0; tt < u[1]; ++tt) {
                const int s = b % NS;
                if (!mwait(&ctl.full[s], (b / NS) & 1, a.timeout_ns, abort)) {
                  if (!*abort) raise_abort(a, &ctl, true);
                  stop = true;
                  break;
                }
                ptx::tc_fence_after();
                const uint32_t wa = ptx::smem_u32(base + (size_t)s * kBox);
                const uint32_t d = tmem + (uint32_t)(tt * a.col_stride);
#pragma unroll
                for (int kk = 0; kk < 4; ++kk)
                  ptx::umma_bf16(d, ptx::sw128_kmajor_desc(wa + kk * 32), ptx::sw128_kmajor_desc(aa + kk * 32), idesc,
                                 (kb | kk) != 0 ? 1u : 0u);
                ptx::umma_commit(&ctl.empty[s]);
                ++b;
                ++issued;
              }
            }
            if (!stop) ptx::umma_commit(&ctl.mma_done);
          }
        }
      }
      // every issued MMA completes before the CTA frees its tensor memory
      if (issued > 0) {
        ptx::umma_commit(&ctl.fin);
        drain_wait(&ctl.fin, 0);
      }
    }
  } else {
    // ======================= workers =========================
    const int wt = threadIdx.x - 64;
    const int ww = wt >> 5;                    // worker warp 0..7
    const int quarter = warp & 3;              // TMEM lane quarter this warp may access
    const int half = (warp - 2) >> 2;          // which half of the columns
    const uint32_t lane_base = (uint32_t)(32 * quarter) << 16;
    const int H = a.S - 1;
    const int nbx = a.D / 64;                  // 64-dim blocks of a head
    unsigned phase_no = 0;                     // grid phases this CTA has arrived at
    int gp = 0, att_no = 0;
    int stg_use[kMaxBoxes];    // staging copies waited for, per buffer (all workers)
    int stg_iss[kMaxBoxes];    // ... issued (worker 0)
    for (int j = 0; j < kMaxBoxes; ++j) stg_use[j] = stg_iss[j] = 0;
    bool ok = true;
    // parity of the last copy / MMA this role issued on each attention barrier (-1: none)
    int pend_ld = -1, pend_s = -1, pend_pv = -1;
    // stamps of the first phases: 0 released, 1-6 phase steps, 7 arrived
    auto stamp = [&](int slot) {
      if (trace && wt == 0 && phase_no < kTracePhases) trace[phase_no * 8 + slot] = ptx::globaltimer();
    };
    // ---- grid barrier: arrive (after every worker's writes), wait ----
    auto arrive = [&]() {
      workers_sync();
      if (wt == 0) {
        bulk_wait_all();
        stamp(6);
        fence_async_global();
        red_release(&a.bar[0], 1u);
      }
      stamp(7);
      ++phase_no;
    };
    auto wait_all = [&]() -> bool {
      if (wt == 0) counter_wait(a, &ctl, &a.bar[0], phase_no * (unsigned)ncta);
      const bool stop = workers_any(*abort);
      stamp(0);
      return !stop;
    };
    auto wsum = [&](float v) -> float {
      v = warp_sum(v);
      workers_sync();
      if (lane == 0) s_wred[ww] = v;
      workers_sync();
      float t = 0.f;
#pragma unroll
      for (int i = 0; i < 8; ++i) t += s_wred[i];
      return t;
    };
    // zero this CTA's share of a buffer (n4 float4s)
    auto zero_share = [&](float* p, size_t n4) {
      const size_t per = (n4 + ncta - 1) / ncta;
      const size_t lo = per * cta, hi = min(n4, lo + per);
      for (size_t i = lo + wt; i < hi; i += kWThreads) reinterpret_cast<float4*>(p)[i] = make_float4(0.f, 0.f, 0.f, 0.f);
    };
    const size_t box_f = (size_t)a.n_mma * 64;   // floats of one box-major fp32 box
    const size_t n_qkv4 = (size_t)a.R[PH_QKV] * 2 * box_f / 4, n_gu4 = (size_t)a.R[PH_GU] * 2 * box_f / 4;

    // ---- step boundary: head of step k-1 and embedding of step k ----
    auto step_phase = [&](int k) {
      const bool do_head = k > 0, do_embed = k < n_evals;
      float* hn = reinterpret_cast<float*>(scr);      // [w]
      float* xs = hn + a.w;                            // [64]
      for (int r = cta; r < a.T; r += ncta) {
        const int g = r / a.S, s = r - g * a.S;
        if (do_head && s > 0) {
          float ss = 0.f;
          for (int f = wt * 4; f < a.w; f += kWThreads * 4) {
            const float4 hv = __ldcg(reinterpret_cast<const float4*>(a.hres + (size_t)(f >> 6) * box_f + r * 64 + (f & 63)));
            ss += hv.x * hv.x + hv.y * hv.y + hv.z * hv.z + hv.w * hv.w;
            *reinterpret_cast<float4*>(hn + f) = hv;
          }
          ss = wsum(ss);
          const float inv = rsqrtf(ss / (float)a.w + a.eps);
          for (int f = wt; f < a.w; f += kWThreads) hn[f] = hn[f] * inv * (1.f + a.g_final[f]);
          workers_sync();
          // 8 threads per output, w/8 consecutive inputs each
          const int sub = wt & 7, per = a.w / 8;
          for (int a0 = wt >> 3; a0 < ((a.A + 31) / 32) * 32; a0 += kWThreads / 8) {
            float dot = 0.f;
            if (a0 < a.A) {
              const uint4* wr = reinterpret_cast<const uint4*>(a.w_ao + (size_t)a0 * a.w + sub * per);
              const float* hr = hn + sub * per;
              for (int q8 = 0; q8 < per / 8; ++q8) {
                const uint4 u = __ldg(wr + q8);
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
              const size_t off = ((size_t)g * H + (s - 1)) * a.A + a0;
              if (a.vout) {
                a.vout[off] = v;
              } else {
                const float xn = a.x[off] - a.dt * v;
                a.x[off] = xn;
                if (!isfinite(xn)) atomicOr(a.status, RTV_DEV_NUMERIC);
              }
            }
          }
          workers_sync();
        }
        if (do_embed) {
          const int K = s == 0 ? a.Sd : a.A;
          const float* src = s == 0 ? a.state + (size_t)g * a.state_stride : a.x + ((size_t)g * H + (s - 1)) * a.A;
          for (int q = wt; q < K; q += kWThreads) xs[q] = src[q];
          workers_sync();
          const __nv_bfloat16* WT = s == 0 ? a.w_spT : a.w_aiT;
          const float* bias = s == 0 ? a.b_sp : a.b_ai;
          const float* cc = a.c + (size_t)(k < n_evals ? k : 0) * a.c_step + (size_t)g * a.c_group;
          for (int f = wt * 4; f < a.w; f += kWThreads * 4) {
            float acc[4] = {0.f, 0.f, 0.f, 0.f};
            for (int q = 0; q < K; ++q) {
              const uint2 u = __ldg(reinterpret_cast<const uint2*>(WT + (size_t)q * a.w + f));
              const float2 f01 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&u.x));
              const float2 f23 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&u.y));
              const float xk = xs[q];
              acc[0] = fmaf(f01.x, xk, acc[0]);
              acc[1] = fmaf(f01.y, xk, acc[1]);
              acc[2] = fmaf(f23.x, xk, acc[2]);
              acc[3] = fmaf(f23.y, xk, acc[3]);
            }
            float4 hv;
            hv.x = acc[0] + bias[f];
            hv.y = acc[1] + bias[f + 1];
            hv.z = acc[2] + bias[f + 2];
            hv.w = acc[3] + bias[f + 3];
            if (s > 0) {
              hv.x += cc[f];
              hv.y += cc[f + 1];
              hv.z += cc[f + 2];
              hv.w += cc[f + 3];
            }
            *reinterpret_cast<float4*>(a.hres + (size_t)(f >> 6) * box_f + r * 64 + (f & 63)) = hv;
          }
          workers_sync();
        }
      }
    };

    // ---- one projection phase of layer l ----
    auto gemm_phase = [&](int ph, int l) -> bool {
      const int* up = pl + PL_UNIT + 4 * ph;
      const Unit u{up[0], up[1], up[2], up[3]};
      if (u.nt == 0) return true;
      const uint32_t act_bytes = (uint32_t)a.n_mma * 128u;
      bool okp = true;
      if (ph == PH_O) {
        // the attention output is already bf16 operand boxes: copy them in
        if (wt == 0)
          for (int j = 0; j < u.nb; ++j) {
            ++stg_iss[j];
            ptx::mbar_expect_tx(&ctl.stg[j], act_bytes);
            ptx::bulk_load(scr + (size_t)j * act_bytes, a.o_att + (size_t)(u.kb0 + j) * box_f, act_bytes, &ctl.stg[j]);
          }
        for (int j = 0; j < u.nb; ++j) {
          const bool landed = mwait(&ctl.stg[j], stg_use[j] & 1, a.timeout_ns, abort);
          if (!landed && !*abort) raise_abort(a, &ctl, true);
          ++stg_use[j];
          if (workers_any(!landed)) {
            okp = false;
            break;
          }
          if (j == 0) stamp(1);
          __syncwarp();
          if (lane == 0) ptx::mbar_arrive(&ctl.act_full[j]);
        }
      } else {
      const bool two = ph == PH_DOWN;                     // gate and up per box
      const uint32_t part = (uint32_t)a.T * 256u;        // one input box of T rows
      const uint32_t stg_bytes = two ? 2 * part : part;
      uint8_t* stg0 = scr + (size_t)u.nb * act_bytes;
      // as many input boxes in flight at once as the scratch holds (all of them when it can)
      const int nbuf = max(1, min(u.nb, (int)((scr_bytes - u.nb * act_bytes) / stg_bytes)));
      // per-token factors
      if (ph == PH_DOWN)
        for (int t = wt; t < a.n_mma; t += kWThreads)
          s_rs[t] = t < a.T ? rsqrtf(__ldcg(a.ss2 + t) / (float)a.w + a.eps) : 0.f;
      const bool norm_side = (ph == PH_QKV || ph == PH_GU) && u.tile0 == 0;
      if (norm_side)
        for (int t = wt; t < a.n_mma; t += kWThreads) s_ss[t] = 0.f;
      // the input boxes: bulk copies of T rows x 64 features (fp32) into staging
      auto issue_copy = [&](int j) {
        const int buf = j % nbuf;
        uint8_t* dst = stg0 + (size_t)buf * stg_bytes;
        uint64_t* bar = &ctl.stg[buf];
        ++stg_iss[buf];
        ptx::mbar_expect_tx(bar, stg_bytes);
        const int kb = u.kb0 + j;
        if (ph == PH_DOWN) {
          ptx::bulk_load(dst, a.gu + (size_t)(2 * kb) * box_f, part, bar);
          ptx::bulk_load(dst + part, a.gu + (size_t)(2 * kb + 1) * box_f, part, bar);
        } else {
          ptx::bulk_load(dst, a.hres + (size_t)kb * box_f, part, bar);
        }
      };
      if (wt == 0)
        for (int j = 0; j < nbuf; ++j) issue_copy(j);
      workers_sync();
      const float* gain = ph == PH_QKV ? a.g_attn + (size_t)l * a.w : a.g_mlp + (size_t)l * a.w;
      for (int j = 0; j < u.nb; ++j) {
        const int buf = j % nbuf;
        const int kb = u.kb0 + j;
        const bool landed = mwait(&ctl.stg[buf], stg_use[buf] & 1, a.timeout_ns, abort);
        if (!landed && !*abort) raise_abort(a, &ctl, true);
        ++stg_use[buf];
        if (workers_any(!landed)) {
          okp = false;
          break;
        }
        if (j == 0) stamp(1);
        const float* sp = reinterpret_cast<const float*>(stg0 + (size_t)buf * stg_bytes);
        uint8_t* dst = scr + (size_t)j * act_bytes;
        for (int it = wt; it < a.n_mma * 8; it += kWThreads) {
          const int t = it >> 3, c = it & 7;
          float v[8];
          float sq = 0.f;
          if (t < a.T) {
            ld8_smem(sp + t * 64 + 8 * c, v);
            if (ph == PH_DOWN) {
              float upv[8];
              ld8_smem(sp + a.T * 64 + t * 64 + 8 * c, upv);
              const float r = s_rs[t];
#pragma unroll
              for (int e = 0; e < 8; ++e) v[e] = gelu_tanh(v[e] * r) * (upv[e] * r);
            } else {
              float gg[8];
              ld8_ro(gain + 64 * kb + 8 * c, gg);
#pragma unroll
              for (int e = 0; e < 8; ++e) {
                sq = fmaf(v[e], v[e], sq);
                v[e] *= 1.f + gg[e];
              }
            }
          } else {
#pragma unroll
            for (int e = 0; e < 8; ++e) v[e] = 0.f;
          }
          *reinterpret_cast<uint4*>(dst + sw_chunk(t, c)) = pack8(v);
          if (norm_side) {
            // the 8 consecutive threads of an aligned group share the token
            sq += __shfl_xor_sync(0xffffffffu, sq, 1);
            sq += __shfl_xor_sync(0xffffffffu, sq, 2);
            sq += __shfl_xor_sync(0xffffffffu, sq, 4);
            if ((lane & 7) == 0 && t < a.T) s_ss[t] += sq;   // one writer per token and box
          }
        }
        ptx::fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) ptx::mbar_arrive(&ctl.act_full[j]);
        workers_sync();   // the staging buffer is free again
        if (wt == 0 && j + nbuf < u.nb) issue_copy(j + nbuf);
      }
      if (okp && norm_side) {
        // the norm statistic of this K range (while the MMAs run)
        float* ssg = ph == PH_QKV ? a.ss1 : a.ss2;
        for (int t = wt; t < a.T; t += kWThreads) atomicAdd(ssg + t, s_ss[t]);
      }
      }
      if (!okp) return false;
      stamp(2);
      const bool done = mwait(&ctl.mma_done, gp & 1, a.timeout_ns, abort);
      if (!done && !*abort) raise_abort(a, &ctl, true);
      ++gp;
      if (workers_any(!done)) return false;
      ptx::tc_fence_after();
      stamp(3);
      // ---- epilogue: accumulator -> staging [2 halves][T][64] fp32 -> bulk add into the sums ----
      float* dst_base = ph == PH_QKV ? a.qkv : ph == PH_GU ? a.gu : a.hres;
      const uint32_t part = (uint32_t)a.T * 256u;
      const int f = quarter * 32 + lane;
      const int fh = f >> 6, fc = f & 63;
      const uint32_t ebytes = (uint32_t)a.T * 512u;
      const int ebuf = 2 * ebytes <= (uint32_t)scr_bytes ? 2 : 1;
      for (int tt = 0; tt < u.nt; ++tt) {
        float* stg = reinterpret_cast<float*>(scr + (size_t)(tt % ebuf) * ebytes);
        if (tt >= ebuf) {
          if (wt == 0) bulk_wait_read_all();   // the reductions that read this buffer are done with it
          workers_sync();
        }
        for (int c = 32 * half; c < a.n_mma; c += 64) {
          float v[32];
          const uint32_t ta = tmem + lane_base + (uint32_t)(tt * a.col_stride + c);
          if (c + 16 < a.n_mma) {
            ptx::tmem_ld_32(ta, v);
#pragma unroll
            for (int i = 0; i < 32; ++i)
              if (c + i < a.T) stg[(size_t)fh * a.T * 64 + (c + i) * 64 + fc] = v[i];
          } else {
            ptx::tmem_ld_16(ta, *reinterpret_cast<float(*)[16]>(v));
#pragma unroll
            for (int i = 0; i < 16; ++i)
              if (c + i < a.T) stg[(size_t)fh * a.T * 64 + (c + i) * 64 + fc] = v[i];
          }
        }
        ptx::fence_proxy_async_smem();
        workers_sync();
        if (tt == 0) stamp(4);
        if (wt == 0) {
          const int tile = u.tile0 + tt;
          bulk_reduce_add(dst_base + (size_t)(2 * tile) * box_f, ptx::smem_u32(stg), part);
          bulk_reduce_add(dst_base + (size_t)(2 * tile + 1) * box_f, ptx::smem_u32(stg + (size_t)a.T * 64), part);
          bulk_commit();
        }
      }
      stamp(5);
      ptx::tc_fence_before();
      return true;
    };

    // ---- attention operands: this CTA's share of the q/k/v rows -> bf16 tiles ----
    // rows rf = (g, hh, s) over hh < Hq + 2*Hkv; a row takes D/2 threads, one
    // RoPE pair (d, d + D/2) each.  Up to kOpPass rows per thread group are
    // loaded before any is used (one L2 round trip for the CTA's share).
    auto attention_operands = [&](int l) {
      constexpr int kOpPass = 4;
      const int hh_n = a.Hq + 2 * a.Hkv;
      const int n_rows = a.G * hh_n * a.S;
      const int lo = (int)((long long)n_rows * cta / ncta), hi = (int)((long long)n_rows * (cta + 1) / ncta);
      const int halfD = a.D >> 1, tph = a.D >> 7;
      const int rpp = kWThreads / halfD;                 // rows per pass: 2 (D = 256) or 4 (D = 128)
      const int dl = wt % halfD, sub = wt / halfD;
      float* s_nrm = s_red[0];                           // per-row squared norms of this round
      for (int r0 = lo; r0 < hi; r0 += rpp * kOpPass) {
        float x1[kOpPass], x2[kOpPass], cs[kOpPass], sn[kOpPass], r1[kOpPass], km[kOpPass];
        int gg[kOpPass], hhv[kOpPass], ssv[kOpPass];
        if (wt < rpp * kOpPass) s_nrm[wt] = 0.f;
#pragma unroll
        for (int p = 0; p < kOpPass; ++p) {
          const int rf = r0 + p * rpp + sub;
          hhv[p] = -1;
          if (rf < hi) {
            const int g = rf / (hh_n * a.S), rem = rf - g * hh_n * a.S;
            const int hh = rem / a.S, s = rem - hh * a.S, t = g * a.S + s;
            const int nt = hh * tph + (dl >> 6), col = dl & 63;
            gg[p] = g;
            hhv[p] = hh;
            ssv[p] = s;
            r1[p] = __ldcg(a.ss1 + t);
            x1[p] = __ldcg(a.qkv + (size_t)(2 * nt) * box_f + t * 64 + col);
            x2[p] = __ldcg(a.qkv + (size_t)(2 * nt + 1) * box_f + t * 64 + col);
            cs[p] = __ldg(a.rope_cs + (size_t)s * halfD + dl);
            sn[p] = __ldg(a.rope_sn + (size_t)s * halfD + dl);
            km[p] = hh < a.Hq ? __ldcg(a.kmax + (size_t)l * a.Bmax * a.Hkv + (a.verify ? 0 : g) * a.Hkv + hh / a.hpk)
                              : 0.f;
          }
        }
        workers_sync();   // s_nrm cleared
#pragma unroll
        for (int p = 0; p < kOpPass; ++p) {
          const int hh = hhv[p];
          float q2 = 0.f;
          if (hh >= 0) {
            const int g = gg[p], s = ssv[p];
            const float rr = rsqrtf(r1[p] / (float)a.w + a.eps);
            const float v1 = x1[p] * rr, v2 = x2[p] * rr;
            float y1 = v1, y2 = v2;
            if (hh < a.Hq + a.Hkv) {
              y1 = v1 * cs[p] - v2 * sn[p];
              y2 = v2 * cs[p] + v1 * sn[p];
            }
            const int d1 = dl, d2 = dl + halfD;
            if (hh < a.Hq) {
              const int j = hh, kvh = j / a.hpk, jl = j - kvh * a.hpk;
              const int pg = (a.verify ? 0 : g) * a.Hkv + kvh;
              const int ip = ((a.verify ? g : 0) * a.hpk + jl) * a.S + s;
              __nv_bfloat16* qp = a.q_pre + ((size_t)(pg * a.nrt_pre + ip / 128) * nbx) * 8192;
              qp[(size_t)(d1 >> 6) * 8192 + sw_elem(ip & 127, d1 & 63)] = __float2bfloat16_rn(y1);
              qp[(size_t)(d2 >> 6) * 8192 + sw_elem(ip & 127, d2 & 63)] = __float2bfloat16_rn(y2);
              const int is = jl * a.S + s;
              __nv_bfloat16* qs = a.q_suf + ((size_t)((g * a.Hkv + kvh) * a.nrt_suf + is / 128) * nbx) * 8192;
              qs[(size_t)(d1 >> 6) * 8192 + sw_elem(is & 127, d1 & 63)] = __float2bfloat16_rn(y1);
              qs[(size_t)(d2 >> 6) * 8192 + sw_elem(is & 127, d2 & 63)] = __float2bfloat16_rn(y2);
              q2 = y1 * y1 + y2 * y2;
            } else if (hh < a.Hq + a.Hkv) {
              const int kvh = hh - a.Hq;
              __nv_bfloat16* kp = a.k_suf + (size_t)(g * a.Hkv + kvh) * nbx * 4096;
              kp[(size_t)(d1 >> 6) * 4096 + sw_elem(s, d1 & 63)] = __float2bfloat16_rn(y1);
              kp[(size_t)(d2 >> 6) * 4096 + sw_elem(s, d2 & 63)] = __float2bfloat16_rn(y2);
            } else {
              const int kvh = hh - a.Hq - a.Hkv;
              __nv_bfloat16* vp = a.v_suf + (size_t)(g * a.Hkv + kvh) * a.D * 64;
              vp[sw_elem(d1, s)] = __float2bfloat16_rn(y1);
              vp[sw_elem(d2, s)] = __float2bfloat16_rn(y2);
            }
          }
          // a warp lies within one row (D/2 is a multiple of 32)
          q2 = warp_sum(q2);
          if (lane == 0 && q2 != 0.f) atomicAdd(&s_nrm[p * rpp + sub], q2);
        }
        workers_sync();
        // the query row's norm -> the prefix reference of the row (RoPE keeps the norm)
#pragma unroll
        for (int p = 0; p < kOpPass; ++p)
          if (hhv[p] >= 0 && hhv[p] < a.Hq && dl == 0)
            a.m_ref[(gg[p] * a.Hq + hhv[p]) * a.S + ssv[p]] = sqrtf(s_nrm[p * rpp + sub]) * km[p] * a.scale_log2;
        workers_sync();
      }
    };

    // ---- the attention item of layer l (after every CTA's operands) ----
    auto attention_item = [&](int l) -> bool {
      const int item = pl[PL_ATT];
      if (item < 0) return true;
      const int D = a.D, QB = 128 * D * 2, KB = 64 * D * 2;
      uint8_t* Qs = scr;            // [128][D] in D/64 blocks of 16 KB; later P [128][64]
      uint8_t* Ks = scr + QB;       // [64][D] in D/64 blocks of 8 KB
      uint8_t* Vs = Ks + KB;        // [D][64] (transposed), one block
      const bool pre = item < a.n_pre;
      int pg = 0, rt = 0, kt = 0, g = 0, kvh = 0, rts = 0, n_rows;
      if (pre) {
        kt = item % a.ntp;
        rt = (item / a.ntp) % a.nrt_pre;
        pg = item / (a.ntp * a.nrt_pre);
        kvh = pg % a.Hkv;
        n_rows = min(128, a.rows_pg - rt * 128);
      } else {
        const int si = item - a.n_pre;
        rts = si % a.nrt_suf;
        kvh = (si / a.nrt_suf) % a.Hkv;
        g = si / (a.nrt_suf * a.Hkv);
        n_rows = min(128, a.rows_suf - rts * 128);
      }
      // every CTA's operand rows are written
      if (wt == 0) counter_wait(a, &ctl, &a.bar[1], (unsigned)(att_no + 1) * (unsigned)ncta);
      if (workers_any(*abort)) return false;
      stamp(2);
      if (wt == 0) {
        ptx::mbar_expect_tx(&ctl.att_ld, (uint32_t)(QB + 2 * KB));
        if (pre) {
          const int pb = a.verify ? 0 : pg / a.Hkv;
          const size_t tile = (((size_t)l * a.Bmax + pb) * a.Hkv + kvh) * a.ntile_max + kt;
          ptx::bulk_load(Qs, a.q_pre + (size_t)(pg * a.nrt_pre + rt) * nbx * 8192, (uint32_t)QB, &ctl.att_ld);
          ptx::bulk_load(Ks, a.pkt + tile * 64 * D, (uint32_t)KB, &ctl.att_ld);
          ptx::bulk_load(Vs, a.pvt + tile * 64 * D, (uint32_t)KB, &ctl.att_ld);
        } else {
          ptx::bulk_load(Qs, a.q_suf + (size_t)((g * a.Hkv + kvh) * a.nrt_suf + rts) * nbx * 8192, (uint32_t)QB,
                         &ctl.att_ld);
          ptx::bulk_load(Ks, a.k_suf + (size_t)(g * a.Hkv + kvh) * nbx * 4096, (uint32_t)KB, &ctl.att_ld);
          ptx::bulk_load(Vs, a.v_suf + (size_t)(g * a.Hkv + kvh) * D * 64, (uint32_t)KB, &ctl.att_ld);
        }
        pend_ld = att_no & 1;
        const bool landed = mwait(&ctl.att_ld, att_no & 1, a.timeout_ns, abort);
        stamp(3);
        if (!landed) {
          if (!*abort) raise_abort(a, &ctl, true);
        } else {
          ptx::tc_fence_after();
          const uint32_t idesc = ptx::idesc_bf16_f32(128, 64);
          const uint32_t qa = ptx::smem_u32(Qs), ka = ptx::smem_u32(Ks);
          for (int kb = 0; kb < D / 64; ++kb)
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)
              ptx::umma_bf16(tmem, ptx::sw128_kmajor_desc(qa + kb * 16384 + kk * 32),
                             ptx::sw128_kmajor_desc(ka + kb * 8192 + kk * 32), idesc, (kb | kk) != 0 ? 1u : 0u);
          ptx::umma_commit(&ctl.att_s);
          pend_s = att_no & 1;
        }
      }
      // ---- softmax of a row (TMEM lane) per thread pair, 32 keys each ----
      const int r = 32 * quarter + lane;
      const bool row_valid = r < n_rows;
      AttRow rr{0, 0, 0};
      if (row_valid) rr = pre ? pre_row(a, pg, rt * 128 + r) : suf_row(a, g, kvh, rts * 128 + r);
      const int gr = (rr.g * a.Hq + rr.j) * a.S + rr.s;
      if (half == 0) s_gr[r] = row_valid ? gr : -1;
      const float mref = (pre && row_valid) ? __ldcg(a.m_ref + gr) : 0.f;
      const int n_keys = pre ? min(64, a.P - 64 * kt) : a.S;
      const int n_vis = (!pre && a.mask_mode == RTV_MASK_PI0_BLOCK && rr.s == 0) ? 1 : n_keys;
      if (workers_any(*abort)) return false;
      // row r starts a new run of consecutive global rows (or is past the valid rows)
      if (half == 0) {
        const bool brk = r > 0 && (!row_valid || s_gr[r] != s_gr[r - 1] + 1);
        const unsigned m = __ballot_sync(0xffffffffu, brk);
        if (lane == 0) s_brk[quarter] = m;
      }
      const bool s_done = mwait(&ctl.att_s, att_no & 1, a.timeout_ns, abort);
      if (!s_done && !*abort) raise_abort(a, &ctl, true);
      if (workers_any(!s_done)) return false;
      ptx::tc_fence_after();
      float x[32];
      ptx::tmem_ld_32(tmem + lane_base + 32u * half, x);
      float m_row;
      if (pre) {
        m_row = mref;   // Cauchy-Schwarz bound: every prefix score of the row is at most this
#pragma unroll
        for (int e = 0; e < 32; ++e) x[e] = (row_valid && 32 * half + e < n_vis) ? x[e] * a.scale_log2 : -INFINITY;
      } else {
        float m4[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
        for (int e = 0; e < 32; ++e) {
          x[e] = (row_valid && 32 * half + e < n_vis) ? x[e] * a.scale_log2 : -INFINITY;
          m4[e & 3] = fmaxf(m4[e & 3], x[e]);
        }
        s_red[half][r] = fmaxf(fmaxf(m4[0], m4[1]), fmaxf(m4[2], m4[3]));
        workers_sync();
        m_row = fmaxf(s_red[0][r], s_red[1][r]);
        workers_sync();   // every thread has read the maxima
      }
      float l4[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int e = 0; e < 32; ++e) {
        x[e] = x[e] == -INFINITY ? 0.f : exp2f(x[e] - m_row);
        l4[e & 3] += x[e];
      }
      s_red[half][r] = (l4[0] + l4[1]) + (l4[2] + l4[3]);
      // P row: this thread's 32 keys = 4 chunks, swizzled like a K-major operand (over the Q tile)
#pragma unroll
      for (int cc = 0; cc < 4; ++cc) *reinterpret_cast<uint4*>(Qs + sw_chunk(r, 4 * half + cc)) = pack8(x + 8 * cc);
      ptx::fence_proxy_async_smem();
      ptx::tc_fence_before();
      workers_sync();
      stamp(4);
      if (wt == 0) {
        ptx::tc_fence_after();
        const uint32_t idesc = ptx::idesc_bf16_f32(128, D);
        const uint32_t pa = ptx::smem_u32(Qs), va = ptx::smem_u32(Vs);
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)
          ptx::umma_bf16(tmem + (uint32_t)kAttOCol, ptx::sw128_kmajor_desc(pa + kk * 32),
                         ptx::sw128_kmajor_desc(va + kk * 32), idesc, kk != 0 ? 1u : 0u);
        ptx::umma_commit(&ctl.att_pv);
        pend_pv = att_no & 1;
      }
      const float l_row = s_red[0][r] + s_red[1][r];
      const int slot = pre ? kt : a.ntp;   // the suffix tile takes the last slot
      if (half == 0 && row_valid) {
        a.l_slot[(size_t)slot * a.R_att + gr] = l_row;
        if (!pre) a.m_suf[gr] = m_row;
      }
      const bool pv_done = mwait(&ctl.att_pv, att_no & 1, a.timeout_ns, abort);
      if (!pv_done && !*abort) raise_abort(a, &ctl, true);
      if (workers_any(!pv_done)) return false;
      ptx::tc_fence_after();
      stamp(5);
      // ---- P V rows -> staging [128][64] fp32 per 64-dim block -> bulk add (prefix) or store (suffix) ----
      float* dst_slot = a.att_slot + (size_t)slot * nbx * a.R_att * 64;
      for (int cb = 0; cb < D / 64; ++cb) {
        float* stg = reinterpret_cast<float*>(scr + (size_t)(cb & 1) * 32768);
        if (cb >= 2) {
          if (wt == 0) bulk_wait_read_all();
          workers_sync();
        }
        float v[32];
        ptx::tmem_ld_32(tmem + lane_base + (uint32_t)(kAttOCol + 64 * cb + 32 * half), v);
#pragma unroll
        for (int e = 0; e < 8; ++e)
          *reinterpret_cast<float4*>(stg + r * 64 + 32 * half + 4 * e) =
              make_float4(v[4 * e], v[4 * e + 1], v[4 * e + 2], v[4 * e + 3]);
        ptx::fence_proxy_async_smem();
        workers_sync();
        if (wt == 0) {
          // rows whose global indices are consecutive go in one operation: the
          // runs start where the ballots below marked a break
          int i0 = 0;
          while (i0 < n_rows) {
            int i1 = n_rows;
            for (int q = (i0 + 1) >> 5; q < 4 && q * 32 < n_rows; ++q) {
              const unsigned m = s_brk[q] & (q == ((i0 + 1) >> 5) ? ~((1u << ((i0 + 1) & 31)) - 1u) : ~0u);
              if (m) {
                i1 = min(n_rows, q * 32 + __ffs(m) - 1);
                break;
              }
            }
            bulk_store(dst_slot + ((size_t)cb * a.R_att + s_gr[i0]) * 64, ptx::smem_u32(stg + i0 * 64),
                       (uint32_t)((i1 - i0) * 256));
            i0 = i1;
          }
          bulk_commit();
        }
      }
      ptx::tc_fence_before();
      return true;
    };

    // ---- combine the key tiles' rows: every CTA a share of (row, 8 dims) ----
    // o = (2^(m_ref - M) sum_prefix P V + 2^(m_suf - M) P V_suffix) /
    //     (2^(m_ref - M) sum_prefix l + 2^(m_suf - M) l_suffix),  M = max(m_ref, m_suf),
    // written as bf16 into the O projection's input boxes.  All loads of a
    // thread are issued before any is used.
    auto attention_combine = [&]() {
      const int cpr = a.D / 8;
      const int rows = a.G * a.Hq * a.S;
      const int n_it = rows * cpr;
      const int lo = (int)((long long)n_it * cta / ncta), hi = (int)((long long)n_it * (cta + 1) / ncta);
      const size_t slot_f = (size_t)nbx * a.R_att * 64;
      for (int it = lo + wt; it < hi; it += kWThreads) {
        const int gr = it / cpr, d0 = (it - gr * cpr) * 8;
        const int cb = d0 >> 6, col = d0 & 63;
        const float mr = __ldcg(a.m_ref + gr), ms = __ldcg(a.m_suf + gr);
        float lp = 0.f, acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
#pragma unroll 4
        for (int q = 0; q < a.ntp; ++q) {
          const float* src = a.att_slot + (size_t)q * slot_f + ((size_t)cb * a.R_att + gr) * 64 + col;
          const float4 u0 = __ldcg(reinterpret_cast<const float4*>(src));
          const float4 u1 = __ldcg(reinterpret_cast<const float4*>(src + 4));
          lp += __ldcg(a.l_slot + (size_t)q * a.R_att + gr);
          acc[0] += u0.x; acc[1] += u0.y; acc[2] += u0.z; acc[3] += u0.w;
          acc[4] += u1.x; acc[5] += u1.y; acc[6] += u1.z; acc[7] += u1.w;
        }
        const float* ssrc = a.att_slot + (size_t)a.ntp * slot_f + ((size_t)cb * a.R_att + gr) * 64 + col;
        float sv[8];
        {
          const float4 u0 = __ldcg(reinterpret_cast<const float4*>(ssrc));
          const float4 u1 = __ldcg(reinterpret_cast<const float4*>(ssrc + 4));
          sv[0] = u0.x; sv[1] = u0.y; sv[2] = u0.z; sv[3] = u0.w;
          sv[4] = u1.x; sv[5] = u1.y; sv[6] = u1.z; sv[7] = u1.w;
        }
        const float ls = __ldcg(a.l_slot + (size_t)a.ntp * a.R_att + gr);
        const float M = fmaxf(mr, ms);
        const float wa = exp2f(mr - M), wb = exp2f(ms - M);
        const float den = lp * wa + ls * wb;
        if (!(den > 0.f)) atomicOr(a.status, RTV_DEV_NUMERIC);
        const float ia = wa / den, ib = wb / den;
        float o[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) o[e] = acc[e] * ia + sv[e] * ib;
        // row gr = (g * Hq + j) * S + s is token t = g * S + s of head j
        const int g = gr / (a.Hq * a.S), rem = gr - g * a.Hq * a.S;
        const int j = rem / a.S, t = g * a.S + (rem - j * a.S);
        uint8_t* box = reinterpret_cast<uint8_t*>(a.o_att + (size_t)(j * nbx + cb) * box_f);
        *reinterpret_cast<uint4*>(box + sw_chunk(t, col >> 3)) = pack8(o);
      }
    };

    // ---- the largest norm of the cached prefix keys of every layer (atomic max
    // of non-negative floats as integers; the launch's memset zeroes kmax) ----
    auto key_norms = [&]() {
      const int nb_used = a.verify ? 1 : a.G;
      const long long n_keys = (long long)a.L * nb_used * a.Hkv * a.P;
      const int lanes_per_key = a.D / 8;                 // 16 bytes each
      const int keys_per_warp = 32 / lanes_per_key;
      const long long per = (n_keys + ncta - 1) / ncta;
      const long long lo = per * cta, hi = min(n_keys, lo + per);
      // every lane of a warp runs the same number of iterations (shuffles below)
      for (long long k0 = lo + (long long)ww * keys_per_warp; k0 < hi; k0 += 8 * keys_per_warp) {
        const long long kq = k0 + lane / lanes_per_key;
        float s2 = 0.f;
        int slot = 0;
        if (kq < hi) {
          const int key = (int)(kq % a.P);
          long long rest = kq / a.P;
          const int kvh = (int)(rest % a.Hkv);
          rest /= a.Hkv;
          const int b = (int)(rest % nb_used);
          const int l = (int)(rest / nb_used);
          const size_t tile = (((size_t)l * a.Bmax + b) * a.Hkv + kvh) * a.ntile_max + key / 64;
          const int c = lane % lanes_per_key;          // 8 dims: block c / 8, chunk c % 8 of the row
          const uint4 q = __ldg(reinterpret_cast<const uint4*>(a.pkt + tile * 64 * a.D + (size_t)(c >> 3) * 4096 +
                                                               (key & 63) * 64 + (c & 7) * 8));
          const __nv_bfloat162* b2 = reinterpret_cast<const __nv_bfloat162*>(&q);
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const float2 f2 = __bfloat1622float2(b2[e]);
            s2 = fmaf(f2.x, f2.x, fmaf(f2.y, f2.y, s2));
          }
          slot = (l * a.Bmax + b) * a.Hkv + kvh;
        }
        for (int o = lanes_per_key / 2; o > 0; o >>= 1) s2 += __shfl_xor_sync(0xffffffffu, s2, o);
        if (kq < hi && lane % lanes_per_key == 0)
          atomicMax(reinterpret_cast<int*>(a.kmax) + slot, __float_as_int(sqrtf(s2)));
      }
    };

    // ======================= the phase sequence =========================
    if (trace && wt == 0) trace[kTracePhases * 8] = ptx::globaltimer();
    // phase 0: embedding of the first evaluation, the prefix keys' norms; the
    // sums the first layer adds into start at zero
    step_phase(0);
    key_norms();
    zero_share(a.qkv, n_qkv4);
    if (cta == 0)
      for (int t = wt; t < a.n_mma; t += kWThreads) a.ss1[t] = 0.f;
    arrive();
    for (int step = 0; step < n_evals && ok; ++step) {
      for (int l = 0; l < a.L && ok; ++l) {
        // QKV
        ok = wait_all() && gemm_phase(PH_QKV, l);
        if (!ok) break;
        arrive();
        // attention: operands by every CTA, then the items (the gate/up sums
        // and the MLP norm statistic of this layer start at zero)
        ok = wait_all();
        if (!ok) break;
        attention_operands(l);
        workers_sync();
        if (wt == 0) red_release(&a.bar[1], 1u);
        stamp(1);
        zero_share(a.gu, n_gu4);
        if (cta == 0)
          for (int t = wt; t < a.n_mma; t += kWThreads) a.ss2[t] = 0.f;
        ok = attention_item(l);
        if (ok) {
          // this CTA's key-tile rows are stored; then every CTA combines a share
          workers_sync();
          if (wt == 0) {
            if (pl[PL_ATT] >= 0) {
              bulk_wait_all();
              fence_async_global();
              red_release(&a.bar[2], 1u);
            }
            counter_wait(a, &ctl, &a.bar[2], (unsigned)(att_no + 1) * (unsigned)a.n_items);
          }
          ok = !workers_any(*abort);
          if (ok) attention_combine();
        }
        ++att_no;
        if (!ok) break;
        arrive();
        // O (the q/k/v sums of the next layer start at zero)
        ok = wait_all();
        if (!ok) break;
        zero_share(a.qkv, n_qkv4);
        ok = gemm_phase(PH_O, l);
        if (!ok) break;
        arrive();
        // GU
        ok = wait_all();
        if (!ok) break;
        ok = gemm_phase(PH_GU, l);
        if (!ok) break;
        arrive();
        // DOWN (the attention-norm statistic of the next layer starts at zero)
        ok = wait_all();
        if (!ok) break;
        if (cta == 0)
          for (int t = wt; t < a.n_mma; t += kWThreads) a.ss1[t] = 0.f;
        ok = gemm_phase(PH_DOWN, l);
        if (!ok) break;
        arrive();
      }
      if (!ok) break;
      // step boundary
      ok = wait_all();
      if (!ok) break;
      step_phase(step + 1);
      if (step + 1 < n_evals) arrive();
    }
    if (!ok) ctl.abort = 1;   // the MMA warp and the producer stop waiting for work that will not come
    // leave nothing in flight: reductions, and copies or MMAs this role issued
    if (wt == 0) {
      bulk_wait_all();
      if (pend_ld >= 0) drain_wait(&ctl.att_ld, pend_ld);
      if (pend_s >= 0) drain_wait(&ctl.att_s, pend_s);
      if (pend_pv >= 0) drain_wait(&ctl.att_pv, pend_pv);
      for (int b2 = 0; b2 < kMaxBoxes; ++b2)
        if (stg_iss[b2] > 0) drain_wait(&ctl.stg[b2], (stg_iss[b2] - 1) & 1);
    }
  }
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  if (warp == 1) ptx::tmem_dealloc(tmem, kTmemCols);
}

// ===========================================================================
// host side
// ===========================================================================
constexpr int kSmemOptin = 227 * 1024;
constexpr int kStaticReserve = 7 * 1024;   // the kernel's static shared memory, rounded up
constexpr int kDynSmem = kSmemOptin - kStaticReserve;

int round_up_i(int x, int m) { return (x + m - 1) / m * m; }

struct Geometry {
  int hpk, n_pg, rows_pg, nrt_pre, ntp, rows_suf, nrt_suf, n_pre, n_items, R_att;
};

// Attention items of a call: G suffix groups, prefix of P tokens; verification
// groups share the prefix of batch element 0, denoising groups each read their own.
Geometry att_geometry(const rtv_expert_config& k, int S, int G, int P, bool verify) {
  Geometry ge{};
  ge.hpk = k.n_q_heads / k.n_kv_heads;
  ge.n_pg = (verify ? 1 : G) * k.n_kv_heads;
  ge.rows_pg = (verify ? G : 1) * ge.hpk * S;
  ge.nrt_pre = (ge.rows_pg + 127) / 128;
  ge.ntp = (P + 63) / 64;
  ge.rows_suf = ge.hpk * S;
  ge.nrt_suf = (ge.rows_suf + 127) / 128;
  ge.n_pre = ge.n_pg * ge.nrt_pre * ge.ntp;
  ge.n_items = ge.n_pre + G * k.n_kv_heads * ge.nrt_suf;
  ge.R_att = round_up_i(G * k.n_q_heads * S, 4);
  return ge;
}

// One projection split into units: the weight tiles in groups of nt, each
// group's K boxes in q near-equal ranges.
std::vector<Unit> split_projection(int R, int KB, int nt, int q) {
  std::vector<Unit> v;
  for (int t0 = 0; t0 < R; t0 += nt) {
    const int n = std::min(nt, R - t0);
    for (int i = 0; i < q; ++i) {
      const int k0 = (int)((long long)KB * i / q), k1 = (int)((long long)KB * (i + 1) / q);
      if (k1 > k0) v.push_back(Unit{t0, n, k0, k1 - k0});
    }
  }
  return v;
}

struct PlanResult {
  std::vector<int> plan;
  std::string why;
  bool ok = false;
};

// Shared memory a unit needs with all of its input boxes in flight at once:
// its bf16 activation boxes plus an fp32 staging buffer per input box (T rows;
// two inputs per box for O and DOWN), or the epilogue's staging of one tile's
// partial sums if that is larger (it reuses the same space).
constexpr int kScratchTarget = 120 * 1024;   // scratch a unit may take before its inputs are pipelined instead
int unit_act(int nb, int n_mma) { return nb * n_mma * 128; }
// (the O projection's input arrives as bf16 operand boxes: no staging)
int unit_stage(int ph, int T) { return ph == PH_O ? 0 : (ph == PH_DOWN ? 2 : 1) * T * 256; }
int unit_scratch(const Unit& u, int ph, int n_mma, int T) {
  const int all = unit_act(u.nb, n_mma) + u.nb * unit_stage(ph, T);
  const int one = unit_act(u.nb, n_mma) + unit_stage(ph, T);
  return std::max(std::max(std::min(all, kScratchTarget), one), T * 512);
}

// Per-CTA plan: one unit of each projection (or none), at most one attention
// item, and the ring depth the CTA's scratch leaves (the scratch takes the
// rest, so double buffering happens where it fits).  Each projection's split
// minimises an estimate of a phase's critical path on one CTA (the first
// input copy, the MMAs at ~0.2 us per 64-wide box, and the phase's partial
// sums through the L2 reduction) among the splits with at most one unit per
// CTA.  Units go to the CTA with the fewest weight boxes so far, largest
// first, so that every SM streams a similar share of each layer's weights.
PlanResult make_plan(const int R[4], const int KB[4], int ncta, int n_mma, int T, int D, int n_items, int w) {
  PlanResult pr;
  const int att_scr = 128 * D * 2 + 2 * 64 * D * 2;   // Q, K, V^T tiles (the output staging reuses them)
  const int he_scr = round_up_i((w + 64) * 4, 1024);
  const int budget = kDynSmem - 1024 - 2 * kBox;      // scratch that still leaves two ring stages
  std::vector<std::vector<Unit>> units(4);
  for (int ph = 0; ph < 4; ++ph) {
    double best = 1e30;
    for (int nt : {1, 2, 4}) {
      if (nt * round_up_i(n_mma, 32) > kTmemCols || nt > R[ph]) continue;
      const int groups = (R[ph] + nt - 1) / nt;
      const int q = std::min(KB[ph], ncta / groups);
      if (q < 1) continue;
      const int nb = (KB[ph] + q - 1) / q;
      if (nb > kMaxBoxes || unit_scratch(Unit{0, nt, 0, nb}, ph, n_mma, T) > budget) continue;
      const int n_units = groups * q;
      // input boxes in flight at once within the scratch target; each further
      // round of copies exposes another L2 round trip (~0.9 us)
      const int nbuf = unit_stage(ph, T) == 0 ? nb
                       : std::max(1, std::min(nb, (kScratchTarget - unit_act(nb, n_mma)) / unit_stage(ph, T)));
      const int rounds = (nb + nbuf - 1) / nbuf;
      // us: input copies, MMA boxes, the phase's partial sums through L2 at ~5 TB/s
      const double cost = 0.9 * rounds + 0.2 * nt * nb + n_units * nt * T * 512.0 / 5e6;
      if (cost < best) {
        best = cost;
        units[ph] = split_projection(R[ph], KB[ph], nt, q);
      }
    }
    if (units[ph].empty() || (int)units[ph].size() > ncta) {
      pr.why = "no split of a projection fits the grid";
      return pr;
    }
  }
  if (n_items > ncta) {
    pr.why = "more attention items than CTAs";
    return pr;
  }
  pr.plan.assign((size_t)ncta * kPlanInts, 0);
  std::vector<double> load(ncta, 0.0);
  std::vector<int> scr_need(ncta, he_scr);
  // attention items on the first CTAs; their scratch holds the Q, K, V tiles,
  // so their ring is shallower: they start with a weight-box handicap
  for (int c = 0; c < ncta; ++c) {
    pr.plan[(size_t)c * kPlanInts + PL_ATT] = c < n_items ? c : -1;
    if (c < n_items) {
      load[c] = 3.0;
      scr_need[c] = std::max(scr_need[c], att_scr);
    }
  }
  const int order[4] = {PH_GU, PH_DOWN, PH_QKV, PH_O};
  for (int oi = 0; oi < 4; ++oi) {
    const int ph = order[oi];
    std::vector<Unit> us = units[ph];
    std::stable_sort(us.begin(), us.end(), [](const Unit& x, const Unit& y) { return x.nt * x.nb > y.nt * y.nb; });
    std::vector<char> taken(ncta, 0);
    for (const Unit& u : us) {
      int best = -1;
      for (int c = 0; c < ncta; ++c)
        if (!taken[c] && (best < 0 || load[c] < load[best])) best = c;
      taken[best] = 1;
      load[best] += u.nt * u.nb;
      int* p = &pr.plan[(size_t)best * kPlanInts + PL_UNIT + 4 * ph];
      p[0] = u.tile0;
      p[1] = u.nt;
      p[2] = u.kb0;
      p[3] = u.nb;
      scr_need[best] = std::max(scr_need[best], unit_scratch(u, ph, n_mma, T));
    }
  }
  for (int c = 0; c < ncta; ++c) {
    const int scr = round_up_i(scr_need[c], 1024);
    const int ns = std::min(kMaxStages, (kDynSmem - 1024 - scr) / kBox);
    if (ns < 2) {
      pr.why = "shared memory leaves fewer than two ring stages";
      return pr;
    }
    pr.plan[(size_t)c * kPlanInts + PL_NS] = ns;
    pr.plan[(size_t)c * kPlanInts + PL_SCR] = ns * kBox;
    pr.plan[(size_t)c * kPlanInts + PL_SCR_BYTES] = kDynSmem - 1024 - ns * kBox;
  }
  pr.ok = true;
  return pr;
}

}  // namespace

struct ResidentPlan {
  int* d_plan = nullptr;
  Geometry ge{};
};

// Resident-path state of a context.
struct ResidentState {
  int ncta = 0;
  int n_mma_max = 0, R_att_max = 0, qpre_tiles = 0, qsuf_tiles = 0;
  float *g_attn = nullptr, *g_mlp = nullptr;
  float *hres = nullptr, *qkv = nullptr, *gu = nullptr;
  float *att_slot = nullptr, *l_slot = nullptr, *m_ref = nullptr, *m_suf = nullptr;
  __nv_bfloat16* o_att = nullptr;
  __nv_bfloat16 *q_pre = nullptr, *q_suf = nullptr, *k_suf = nullptr, *v_suf = nullptr;
  float *ss1 = nullptr, *ss2 = nullptr;
  unsigned* bar = nullptr;        // [16] counters, then kmax (zeroed together before every launch)
  float* kmax = nullptr;
  size_t bar_bytes = 0;
  unsigned long long* trace = nullptr;
  int trace_ncta = 0;
  std::map<std::tuple<int, int, int>, ResidentPlan> plans;   // (G, P, verify)
  std::vector<void*> allocs;
};

rtv_status resident_create(rtv_ctx* ctx) {
  const rtv_expert_config& k = ctx->cfg;
  // opt-in (RTV_PATH=resident) while the layered kernels remain the faster path
  const char* env = getenv("RTV_PATH");
  if (!env || strcmp(env, "resident") != 0) return RTV_OK;
  FastViews fv;
  if (!ctx->use_fast || ctx->block_only || !fast_views(ctx, &fv)) return RTV_OK;
  const int S = ctx->S, w = k.width, D = k.head_dim;
  if (k.time_cond != RTV_TIME_ADD || (k.mlp_dtype != RTV_SAME && k.mlp_dtype != k.dtype) || S > 64 ||
      (D != 128 && D != 256) || w % 128 != 0 || w > 4096 || k.mlp_dim % 64 != 0 || k.action_dim > 64 ||
      k.state_dim > 64 || k.n_q_heads % k.n_kv_heads != 0)
    return RTV_OK;
  if (cudaFuncSetAttribute(resident_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kDynSmem) != cudaSuccess) {
    cudaGetLastError();
    return RTV_OK;
  }
  int per_sm = 0;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, resident_kernel, kRThreads, kDynSmem) != cudaSuccess ||
      per_sm < 1) {
    cudaGetLastError();
    return RTV_OK;
  }
  ResidentState* rs = new ResidentState();
  rs->ncta = fv.num_sms;
  const int Tmax = std::min(256, ctx->Tmax);
  const int Gmax = std::max(1, ctx->Gmax);
  rs->n_mma_max = round_up_i(Tmax, 16);
  rs->R_att_max = round_up_i(Gmax * k.n_q_heads * S, 4);
  const int hpk = k.n_q_heads / k.n_kv_heads;
  // query tiles: prefix groups x row tiles, for the larger of the two groupings
  const int nrt_v = (Gmax * hpk * S + 127) / 128, nrt_d = (hpk * S + 127) / 128;
  rs->qpre_tiles = std::max(k.n_kv_heads * nrt_v, Gmax * k.n_kv_heads * nrt_d);
  rs->qsuf_tiles = Gmax * k.n_kv_heads * nrt_d;
  const size_t nq = (size_t)(ctx->Q + 2 * ctx->KV);
  const size_t nbx = D / 64;
  bool ok = true;
  auto alloc = [&](void** p, size_t bytes) {
    if (!ok) return;
    if (cudaMalloc(p, bytes) != cudaSuccess) {
      ok = false;
      return;
    }
    rs->allocs.push_back(*p);
    if (cudaMemset(*p, 0, bytes) != cudaSuccess) ok = false;
  };
  const size_t nm = rs->n_mma_max;
  alloc((void**)&rs->g_attn, (size_t)k.n_layers * w * 4);
  alloc((void**)&rs->g_mlp, (size_t)k.n_layers * w * 4);
  alloc((void**)&rs->hres, (size_t)w * nm * 4);
  alloc((void**)&rs->qkv, nq * nm * 4);
  alloc((void**)&rs->gu, (size_t)2 * k.mlp_dim * nm * 4);
  const size_t n_slots = (size_t)fv.ntile_max + 1;
  alloc((void**)&rs->att_slot, n_slots * nbx * rs->R_att_max * 64 * 4);
  alloc((void**)&rs->l_slot, n_slots * rs->R_att_max * 4);
  alloc((void**)&rs->o_att, (size_t)k.n_q_heads * nbx * nm * 64 * 2);
  alloc((void**)&rs->m_ref, (size_t)rs->R_att_max * 4);
  alloc((void**)&rs->m_suf, (size_t)rs->R_att_max * 4);
  alloc((void**)&rs->q_pre, (size_t)rs->qpre_tiles * nbx * 8192 * 2);
  alloc((void**)&rs->q_suf, (size_t)rs->qsuf_tiles * nbx * 8192 * 2);
  alloc((void**)&rs->k_suf, (size_t)Gmax * k.n_kv_heads * nbx * 4096 * 2);
  alloc((void**)&rs->v_suf, (size_t)Gmax * k.n_kv_heads * D * 64 * 2);
  alloc((void**)&rs->ss1, 256 * 4);
  alloc((void**)&rs->ss2, 256 * 4);
  rs->bar_bytes = 64 + (size_t)k.n_layers * k.max_batch * k.n_kv_heads * 4;
  alloc((void**)&rs->bar, rs->bar_bytes);
  if (ok) rs->kmax = reinterpret_cast<float*>(reinterpret_cast<uint8_t*>(rs->bar) + 64);
  if (ok && getenv("RTV_TRACE")) {
    alloc((void**)&rs->trace, (size_t)rs->ncta * kTraceSlots * 8);
    rs->trace_ncta = rs->ncta;
  }
  if (!ok) {
    for (void* p : rs->allocs) cudaFree(p);
    delete rs;
    cudaGetLastError();
    return RTV_ERR_OOM;
  }
  ctx->resident = rs;
  return RTV_OK;
}

rtv_status resident_load(rtv_ctx* ctx) {
  ResidentState* rs = ctx->resident;
  if (!rs) return RTV_OK;
  const rtv_expert_config& k = ctx->cfg;
  for (int l = 0; l < k.n_layers; ++l) {
    const LayerW& Lw = ctx->W.layers[l];
    if (cudaMemcpy(rs->g_attn + (size_t)l * k.width, Lw.g_attn, k.width * 4, cudaMemcpyDeviceToDevice) != cudaSuccess ||
        cudaMemcpy(rs->g_mlp + (size_t)l * k.width, Lw.g_mlp, k.width * 4, cudaMemcpyDeviceToDevice) != cudaSuccess)
      return RTV_ERR_CUDA;
  }
  return RTV_OK;
}

bool resident_prepare(rtv_ctx* ctx, int G, int P, bool verify) {
  ResidentState* rs = ctx->resident;
  if (!rs) return false;
  const rtv_expert_config& k = ctx->cfg;
  const int S = ctx->S, T = G * S;
  FastViews fv;
  if (!fast_views(ctx, &fv) || !fv.w_qkv || !fv.w_o || !fv.w_gu || !fv.w_down || !fv.w_aiT || !fv.w_spT ||
      T > rs->n_mma_max || P < 1 || G < 1)
    return false;
  const Geometry ge = att_geometry(k, S, G, P, verify);
  if (ge.n_items > rs->ncta || ge.R_att > rs->R_att_max || ge.ntp > fv.ntile_max ||
      ge.n_pg * ge.nrt_pre > rs->qpre_tiles || G * k.n_kv_heads * ge.nrt_suf > rs->qsuf_tiles)
    return false;
  const auto key = std::make_tuple(G, P, verify ? 1 : 0);
  if (rs->plans.count(key)) return true;
  const int n_mma = round_up_i(T, 16);
  const int nq = ctx->Q + 2 * ctx->KV;
  const int R[4] = {nq / 128, k.width / 128, 2 * k.mlp_dim / 128, k.width / 128};
  const int KB[4] = {k.width / 64, ctx->Q / 64, k.width / 64, k.mlp_dim / 64};
  const PlanResult pr = make_plan(R, KB, rs->ncta, n_mma, T, k.head_dim, ge.n_items, k.width);
  if (!pr.ok) {
    if (getenv("RTV_LOG")) fprintf(stderr, "[rtv] resident plan refused: %s\n", pr.why.c_str());
    return false;
  }
  ResidentPlan rp;
  rp.ge = ge;
  if (cudaMalloc(&rp.d_plan, pr.plan.size() * 4) != cudaSuccess) {
    cudaGetLastError();
    return false;
  }
  rs->allocs.push_back(rp.d_plan);
  if (cudaMemcpy(rp.d_plan, pr.plan.data(), pr.plan.size() * 4, cudaMemcpyHostToDevice) != cudaSuccess) return false;
  if (getenv("RTV_LOG")) {
    const char* nm[4] = {"qkv", "o", "gu", "down"};
    for (int ph = 0; ph < 4; ++ph) {
      int mx = 0, n = 0;
      for (int c = 0; c < rs->ncta; ++c) {
        const int* u = &pr.plan[(size_t)c * kPlanInts + PL_UNIT + 4 * ph];
        if (u[1]) ++n;
        mx = std::max(mx, u[1] * u[3]);
      }
      fprintf(stderr, "[rtv] resident %s: %d units, at most %d boxes per CTA\n", nm[ph], n, mx);
    }
    int mn = 99, mxs = 0;
    for (int c = 0; c < rs->ncta; ++c) {
      mn = std::min(mn, pr.plan[(size_t)c * kPlanInts + PL_NS]);
      mxs = std::max(mxs, pr.plan[(size_t)c * kPlanInts + PL_NS]);
    }
    fprintf(stderr, "[rtv] resident attention items %d (prefix %d), ring stages %d..%d, T=%d\n", ge.n_items,
            ge.n_pre, mn, mxs, T);
  }
  rs->plans[key] = rp;
  return true;
}

rtv_status resident_launch(rtv_ctx* ctx, int G, int P, int n_steps, bool verify, const float* c, const float* rope_cs,
                           const float* rope_sn, cudaStream_t st) {
  ResidentState* rs = ctx->resident;
  FastViews fv;
  if (!rs || !fast_views(ctx, &fv)) return RTV_ERR_UNSUPPORTED;
  const auto it = rs->plans.find(std::make_tuple(G, P, verify ? 1 : 0));
  if (it == rs->plans.end()) return RTV_ERR_UNSUPPORTED;
  const ResidentPlan& rp = it->second;
  const rtv_expert_config& k = ctx->cfg;
  const int S = ctx->S, T = G * S;
  ResArgs a{};
  a.wts[PH_QKV] = fv.w_qkv;
  a.wts[PH_O] = fv.w_o;
  a.wts[PH_GU] = fv.w_gu;
  a.wts[PH_DOWN] = fv.w_down;
  const int nq = ctx->Q + 2 * ctx->KV;
  a.R[PH_QKV] = nq / 128;
  a.R[PH_O] = k.width / 128;
  a.R[PH_GU] = 2 * k.mlp_dim / 128;
  a.R[PH_DOWN] = k.width / 128;
  a.KB[PH_QKV] = k.width / 64;
  a.KB[PH_O] = ctx->Q / 64;
  a.KB[PH_GU] = k.width / 64;
  a.KB[PH_DOWN] = k.mlp_dim / 64;
  a.g_attn = rs->g_attn;
  a.g_mlp = rs->g_mlp;
  a.pkt = fv.pkt;
  a.pvt = fv.pvt;
  a.rope_cs = rope_cs;
  a.rope_sn = rope_sn;
  a.w_ao = (const __nv_bfloat16*)ctx->W.ao_w;
  a.b_ao = ctx->W.ao_b;
  a.g_final = ctx->W.g_final;
  a.w_aiT = fv.w_aiT;
  a.b_ai = ctx->W.ai_b;
  a.w_spT = fv.w_spT;
  a.b_sp = ctx->W.sp_b;
  a.c = c;
  a.c_step = verify ? 0 : k.width;
  a.c_group = verify ? k.width : 0;
  a.state = ctx->state;
  a.state_stride = verify ? 0 : k.state_dim;
  a.x = ctx->x;
  a.vout = verify ? ctx->v : nullptr;
  a.hres = rs->hres;
  a.qkv = rs->qkv;
  a.gu = rs->gu;
  a.att_slot = rs->att_slot;
  a.l_slot = rs->l_slot;
  a.o_att = rs->o_att;
  a.m_ref = rs->m_ref;
  a.m_suf = rs->m_suf;
  a.q_pre = rs->q_pre;
  a.q_suf = rs->q_suf;
  a.k_suf = rs->k_suf;
  a.v_suf = rs->v_suf;
  a.kmax = rs->kmax;
  a.ss1 = rs->ss1;
  a.ss2 = rs->ss2;
  a.bar = rs->bar;
  a.status = ctx->status;
  a.trace = rs->trace;
  a.plan = rp.d_plan;
  a.timeout_ns = k.barrier_timeout_ns;
  a.L = k.n_layers;
  a.w = k.width;
  a.Hq = k.n_q_heads;
  a.Hkv = k.n_kv_heads;
  a.D = k.head_dim;
  a.F = k.mlp_dim;
  a.S = S;
  a.G = G;
  a.T = T;
  a.n_mma = round_up_i(T, 16);
  a.A = k.action_dim;
  a.Sd = k.state_dim;
  a.P = P;
  a.Bmax = k.max_batch;
  a.ntile_max = fv.ntile_max;
  a.mask_mode = k.suffix_mask;
  a.n_steps = n_steps;
  a.verify = verify ? 1 : 0;
  const Geometry& ge = rp.ge;
  a.hpk = ge.hpk;
  a.rows_pg = ge.rows_pg;
  a.nrt_pre = ge.nrt_pre;
  a.ntp = ge.ntp;
  a.rows_suf = ge.rows_suf;
  a.nrt_suf = ge.nrt_suf;
  a.n_pre = ge.n_pre;
  a.n_items = ge.n_items;
  a.R_att = ge.R_att;
  a.col_stride = round_up_i(a.n_mma, 32);
  a.pace_ns = getenv("RTV_PACE_NS") ? atoi(getenv("RTV_PACE_NS")) : 0;
  a.dyn_smem = kDynSmem;
  a.dt = verify ? 0.f : (float)(1.0 / (double)n_steps);
  a.eps = k.rms_eps;
  a.scale_log2 = (float)(1.4426950408889634 / sqrt((double)k.head_dim));
  cudaError_t e = cudaMemsetAsync(rs->bar, 0, rs->bar_bytes, st);
  if (e == cudaSuccess) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(rs->ncta, 1, 1);
    cfg.blockDim = dim3(kRThreads, 1, 1);
    cfg.dynamicSmemBytes = kDynSmem;
    cfg.stream = st;
    cudaLaunchAttribute at[1];
    at[0].id = cudaLaunchAttributeCooperative;   // every CTA resident at once (grid barriers)
    at[0].val.cooperative = 1;
    cfg.attrs = at;
    cfg.numAttrs = 1;
    e = cudaLaunchKernelEx(&cfg, resident_kernel, a);
  }
  if (e != cudaSuccess) {
    ctx->last_error = std::string("resident kernel launch: ") + cudaGetErrorString(e);
    return RTV_ERR_CUDA;
  }
  return RTV_OK;
}

void resident_destroy(rtv_ctx* ctx) {
  ResidentState* rs = ctx->resident;
  if (!rs) return;
  for (void* p : rs->allocs) cudaFree(p);
  delete rs;
  ctx->resident = nullptr;
}

void resident_trace_report(rtv_ctx* ctx) {
  ResidentState* rs = ctx->resident;
  if (!rs || !rs->trace) return;
  std::vector<unsigned long long> h((size_t)rs->trace_ncta * kTraceSlots);
  cudaDeviceSynchronize();
  if (cudaMemcpy(h.data(), rs->trace, h.size() * 8, cudaMemcpyDeviceToHost) != cudaSuccess) return;
  unsigned long long t_ref = ~0ull;
  for (int c = 0; c < rs->trace_ncta; ++c)
    if (h[(size_t)c * kTraceSlots + kTracePhases * 8]) t_ref = std::min(t_ref, h[(size_t)c * kTraceSlots + kTracePhases * 8]);
  const char* ph[kTracePhases] = {"embed", "qkv0", "attn0", "o0", "gu0", "down0",
                                  "qkv1", "attn1", "o1", "gu1", "down1", "qkv2"};
  const char* ev_g[8] = {"released", "box0 in", "operands", "mma done", "staged", "reduce out", "reduce done",
                         "arrived"};
  const char* ev_a[8] = {"released", "operands", "counter", "tiles in", "softmax", "pv done", "reduce done",
                         "arrived"};
  fprintf(stderr, "[rtv trace] resident kernel, us after the first CTA started: min / median / max over CTAs\n");
  for (int p = 0; p < kTracePhases; ++p) {
    const bool att = p >= 2 && (p - 2) % 5 == 0;
    for (int e = 0; e < 8; ++e) {
      std::vector<double> v;
      for (int c = 0; c < rs->trace_ncta; ++c) {
        const unsigned long long t = h[(size_t)c * kTraceSlots + p * 8 + e];
        if (t && t_ref != ~0ull && t >= t_ref) v.push_back((double)(t - t_ref) * 1e-3);
      }
      if (v.empty()) continue;
      std::sort(v.begin(), v.end());
      fprintf(stderr, "    %-6s %-12s %8.2f %8.2f %8.2f  (%zu CTAs)\n", ph[p], att ? ev_a[e] : ev_g[e], v.front(),
              v[v.size() / 2], v.back(), v.size());
    }
  }
  cudaMemset(rs->trace, 0, h.size() * 8);
}

}  // namespace rtv
