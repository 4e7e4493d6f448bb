// The prefill-sized write path (lrkv_compress with more than a few new tokens
// per row): tensor-core projection, then the routing passes.
#pragma once

#include <cuda_runtime.h>

#include "lrkv.h"
#include "lrkv_common.cuh"

namespace lrkv {

// k_new, v_new [B][t_new][Hkv][d]; w: the workspace laid out as L.
lrkv_status compress_tc(const lrkv_dims& D, const lrkv_cache& C, const lrkv_bf16* k_new,
                        const lrkv_bf16* v_new, int t_new, const int32_t* t_new_b, float tau,
                        float* err_out, char* w, const WsLayout& L, cudaStream_t s);

}  // namespace lrkv
