// attn_bwd.h — launch parameters of the attention backward kernels (internal).
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cstdint>

#include "geometry.h"

namespace cpattn {

// Row statistics of the backward, per view row (rb, h, t) stored [NR*B][Hh][T]:
// lse2 = -lse * log2(e), the negated lse in log2 units (-inf where lse is -inf,
// so that exp2(s * scale_log2 + lse2) is 0), and dvec = rowsum(dO * O).
struct BwdPreParams {
  Geometry g;
  const __nv_bfloat16* o;      // forward output, view layout [NR*B][T][Hh][D]
  const __nv_bfloat16* dout;   // upstream gradient, same layout
  const float* lse;            // natural [lse_B][lse_H][lse_S] (as cp_attn_fwd writes it)
  int lse_B, lse_H;
  int64_t lse_S;
  float* lse2;
  float* dvec;
};

// One backward kernel: the dK/dV kernel walks, for each 128-key tile, the query
// tiles that see it; the dQ kernel walks, for each 128-query tile, the key tiles
// it sees (ring order). Items are (rank*B + batch, head, tile) with the tile in
// WorkItem::qp.
struct BwdParams {
  Geometry g;
  float scale_log2;            // softmax scale * log2(e)
  float scale;                 // softmax scale (factor of dQ and dK)
  const WorkItem* items;
  const int* cta_begin;        // CTA c runs items [cta_begin[c], cta_begin[c+1])
  int n_cta;
  // Walk of (rank, tile): entries[walk_off[rank*ntiles + tile] .. walk_off[rank*ntiles + tile + 1]),
  // each pack_entry(other rank, other tile, class, 0).
  const int* walk_off;
  const uint32_t* entries;
  int ntiles;                  // 128-token tiles per rank
  const float* lse2;           // [NR*B][Hh][T] (+ 512 bytes of padding)
  const float* dvec;           // [NR*B][Hh][T] (+ 512 bytes of padding)
  __nv_bfloat16* out0;         // dK (key kernel) or dQ (query kernel), view layout
  __nv_bfloat16* out1;         // dV (key kernel)
  int* status;
  uint64_t wait_limit_ns;
};

struct BwdLaunch {
  CUtensorMap tm_q, tm_k, tm_v, tm_do;   // 4-D views (D, Hh, T, NR*B)
  BwdParams params;
};

cudaError_t launch_attn_bwd_pre(const BwdPreParams& p, int D, cudaStream_t stream);
cudaError_t launch_attn_bwd_kv(const BwdLaunch& L, int D, cudaStream_t stream);
cudaError_t launch_attn_bwd_q(const BwdLaunch& L, int D, cudaStream_t stream);

}  // namespace cpattn
