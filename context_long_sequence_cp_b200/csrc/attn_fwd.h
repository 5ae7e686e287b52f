// attn_fwd.h — launch parameters of the attention forward kernel (internal).
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cstdint>

#include "geometry.h"

namespace cpattn {

constexpr int kMaxPullRanks = 64;   // ranks a fused-pull ring launch can fetch from

struct FwdParams {
  Geometry g;
  int t_begin, t_end;          // ring steps visited: [t_begin, t_end)
  float scale_log2;            // softmax scale * log2(e)
  const WorkItem* items;       // device work list
  int n_items;
  const int* cta_begin;        // CTA c runs items [cta_begin[c], cta_begin[c+1])
  int n_cta;                   // grid size the schedule was made for
  // Precomputed key walks: the walk of query-tile pair (rq, qp) over ring step t
  // is entries[step_off[(rq*npairs + qp)*(NR+1) + t] .. step_off[... + t + 1]).
  const int* step_off;
  const uint32_t* entries;
  int npairs;
  __nv_bfloat16* o;            // fused output, view layout [NR*B][T][Hh][D]
  float* lse;                  // natural [lse_B][lse_H][lse_S]; may be null
  int lse_B, lse_H;
  int64_t lse_S;
  float* o_part;               // partial mode: [rows][D], row = (rb*T + tl)*Hh + h
  float* lse_part;             // partial mode: [rows]
  // Rank-local buffers (one ring step of one rank): q, o and the partials hold
  // row blocks from q_rb0 on (0 for the whole view), and with kv_local the k and
  // v maps hold the key rank's B row blocks only.
  int q_rb0;
  int kv_local;
  // Ring launches (partial mode): every item is a unit, a query-tile pair over
  // ring steps [unit_t0, unit_t1), whose partial goes to part
  // min(unit_t0, unit_split), part_rows rows per part; before its first load from
  // the key/value block of another rank k the producer waits until arrived[k]
  // >= arrive_target (arrived null: no wait).
  int unit_steps;
  int unit_split;
  int64_t part_rows;
  int* arrived;
  int arrive_target;
  // Fused pull (ring launches): warps 10 and 11 of every CTA copy the blocks of
  // the other ranks, in ring order from the query rank, from pull_src[2k] (K)
  // and pull_src[2k + 1] (V) into slot k of pull_k_all / pull_v_all, in chunks of
  // pull_chunk_bytes, adding 1 to arrived[k] per finished chunk; pull_chunks
  // chunks per block, K and V together (0: no pull). The launch is cooperative,
  // so every CTA whose chunks a unit waits for is resident.
  uint64_t pull_src[2 * kMaxPullRanks];
  char* pull_k_all;
  char* pull_v_all;
  int64_t pull_block_bytes;
  int pull_chunk_bytes;
  int pull_chunks;
  int* status;                 // device status word (0 = ok)
  uint64_t wait_limit_ns;      // budget of one in-kernel wait
};

struct FwdLaunch {
  CUtensorMap tm_q, tm_k, tm_v;   // 4-D views (D, Hh, T, NR*B) of q, k, v
  FwdParams params;
};

cudaError_t launch_attn_fwd(const FwdLaunch& L, int D, bool partial, cudaStream_t stream);
size_t attn_fwd_smem_bytes(int D);

// merge_permute.cu: merge of partials
cudaError_t launch_merge(int num_parts, int64_t rows, int D, const float* o_parts,
                         const float* lse_parts, __nv_bfloat16* o_out, float* lse_out,
                         cudaStream_t stream);

// merge_permute.cu: layout maps
struct PermuteArgs {
  int kind;          // 0: contiguous/zigzag token rows; 1: Ulysses head-group runs
  int direction;     // 0: forward gather, 1: inverse
  int N, B, S, H, D;
  int zigzag;
  int elem_bytes;
};
cudaError_t launch_permute(const PermuteArgs& a, const void* in, void* out, cudaStream_t stream);
cudaError_t launch_index_map(const PermuteArgs& a, int64_t* map_out, cudaStream_t stream);

// Rotary embedding parameters: theta[i] = base^(-2i/D) (fp64), i < D/2 <= 64.
struct RopeArgs {
  double theta[64];
  int64_t pos_offset;
  int D;
};
cudaError_t launch_rope_permute(const PermuteArgs& a, const RopeArgs& ra, const void* in, void* out,
                                cudaStream_t stream);

// merge_permute.cu: the bounded-wait self-test (a wait on a barrier nothing arrives on)
cudaError_t launch_wait_probe(int* status, uint64_t limit_ns, cudaStream_t stream);

}  // namespace cpattn

// api.cu: the Ulysses forward with a caller-chosen scratch buffer of at least
// cp_attn_workspace_bytes(plan, 0) bytes (used by the no-alloc entry point).
struct cp_attn_plan_s;
int cp_internal_plan_device(const cp_attn_plan_s* plan);
int cp_internal_ulysses_fwd_scratch(cp_attn_plan_s* plan, const void* q, const void* k, const void* v,
                                    void* o, float* lse, void* scratch, size_t scratch_bytes,
                                    cudaStream_t stream);
