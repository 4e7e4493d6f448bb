// Parameters of the write-path kernels (the one-launch append path).
//
// OjaKV repository README, "Method Summary": a fixed per-head basis
// (StaticPCA) and the hybrid policy that keeps tokens with a high
// reconstruction error in full rank (OjaKV).
#pragma once

#include "lrkv_common.cuh"

namespace lrkv {

struct CompressParams {
  lrkv_dims D;
  lrkv_cache C;
  const lrkv_bf16* k_new;
  const lrkv_bf16* v_new;
  int t_new;
  const int32_t* t_new_b;
  float tau;
  float* err_out;
  int32_t* ticket;    // CTAs done, zero between calls
};

}  // namespace lrkv
