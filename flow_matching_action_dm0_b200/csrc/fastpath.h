// Tensor-core (tcgen05) path of the bf16 expert: interface used by the runtime.
#pragma once

#include <cuda_runtime.h>

#include "../../include/rtv.h"

struct rtv_ctx;

namespace rtv {

// Decide whether the config can use the tensor-core path and allocate its
// state; sets ctx->use_fast.  Returns an error only on a CUDA failure.
rtv_status fast_create(rtv_ctx* ctx);
// Pack the loaded parameters into the tensor-core layouts.
rtv_status fast_load(rtv_ctx* ctx, const rtv_tensor* params, int n_params);
bool fast_supports_prefix(rtv_ctx* ctx, int prefix_len);
// Expert forward over G suffixes into ctx->h (same contract as the SIMT forward).
rtv_status fast_expert(rtv_ctx* ctx, int G, int P, const float* c, int c_stride, int state_stride,
                       int prefix_batch_stride, const float* rope_cs, const float* rope_sn, cudaStream_t st);
// Output head: Euler step on ctx->x (velocity_only = false) or v into ctx->v.
void fast_out_head(rtv_ctx* ctx, int G, float dt, bool velocity_only, cudaStream_t st);
void fast_destroy(rtv_ctx* ctx);

}  // namespace rtv
