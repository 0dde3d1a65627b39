// Resident (persistent) tensor-core kernel of the bf16 action expert:
// interface used by the runtime.
#pragma once

#include <cuda_runtime.h>

#include "../../include/rtv.h"

struct rtv_ctx;

namespace rtv {

struct ResidentState;

// Decide whether the context's shapes suit the resident kernel and allocate
// its buffers (sets ctx->resident; leaves it null when they do not suit).
// Call after fast_create.  Returns an error only when an allocation fails.
rtv_status resident_create(rtv_ctx* ctx);
// Gather the per-layer norm gains after rtv_load_expert.
rtv_status resident_load(rtv_ctx* ctx);
// Prepare (outside any stream capture) the work plan of a call over G suffix
// groups (G batch elements when denoising, G taus when verifying) with a
// prefix of P tokens; false when the resident kernel does not serve it.
bool resident_prepare(rtv_ctx* ctx, int G, int P, bool verify);
// Enqueue (or capture) one resident launch prepared by resident_prepare:
// n_steps Euler steps from ctx->x with time conditions c + step * width
// (denoise), or one velocity evaluation of the G suffixes into ctx->v with
// condition c + g * width (verify).  A memset of the launch's barrier
// counters precedes it on the same stream.  rope_cs / rope_sn: [S][D/2]
// tables of the suffix positions P..P+S-1.
rtv_status resident_launch(rtv_ctx* ctx, int G, int P, int n_steps, bool verify, const float* c,
                           const float* rope_cs, const float* rope_sn, cudaStream_t st);
void resident_destroy(rtv_ctx* ctx);
// Print the phase stamps of the last resident launch (RTV_TRACE set).
void resident_trace_report(rtv_ctx* ctx);

}  // namespace rtv
