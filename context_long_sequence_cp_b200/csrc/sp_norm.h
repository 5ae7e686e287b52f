// sp_norm.h — launch parameters of the sequence-parallel LayerNorm/Dropout step (internal).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cstdint>

namespace cpattn {

struct SpArgs {
  const __nv_bfloat16* partials;   // [nparts][rows][H]
  int nparts;
  int64_t part_stride;             // elements between partials (rows * H)
  const uint32_t* keep;            // keep bits, or null (no dropout)
  float inv_keep;                  // 1 / (1 - p)
  const __nv_bfloat16* residual;   // [rows][H] or null
  const float* gamma;              // [H] (with beta) when y is written
  const float* beta;
  float eps;
  __nv_bfloat16* z;                // [rows][H] or null
  __nv_bfloat16* y;                // [rows][H] or null
  int64_t rows;
  int H;
};

cudaError_t launch_sp_rs_dropout_add_ln(const SpArgs& a, cudaStream_t stream);

}  // namespace cpattn
