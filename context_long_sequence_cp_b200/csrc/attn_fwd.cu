// attn_fwd.cu — context-parallel attention forward on sm_100a (tcgen05 + TMEM + TMA).
//
// What it computes (page "序列与上下文并行", section "上下文并行：注意力本身切分"):
// for every query tile of every virtual rank r, the key/value tiles of ranks
// (r + t) mod N, t = 0..N-1, are visited in that ring order and folded into one
// running online-softmax state (row max m, row sum l, unnormalised O), which is
// the incremental merge of the per-step partials; at the end O/l and the
// logsumexp m + log l are written. Scores are scaled by 1/sqrt(D) and masked
// keys are -inf (page "Tensor并行与算子拆分", section "注意力的并行化优化"); the
// causal mask uses global positions (section "工程实践" of the first page).
// Key tiles wholly above the causal diagonal are never loaded or multiplied.
// In partial mode the kernel visits a single ring step and writes that step's
// normalised fp32 (O_t, lse_t) instead.
//
// Kernel design (one CTA per SM, persistent over a work list; 12 warps):
//   warps 0-3  softmax warpgroup 0: query tile 0 of the item, one row per thread
//   warps 4-7  softmax warpgroup 1: query tile 1 of the item
//   warp  8    allocates TMEM; lane 0 issues every tcgen05.mma
//   warp  9    lane 0 issues every TMA load
//   warps 10-11 idle, except in a ring launch with a fused fetch, where they
//              copy the other ranks' key/value blocks into local slots
// TMEM (512 columns x 128 lanes): S0 [0,128) S1 [128,256) O0 [256,256+D)
// O1 [256+D, 256+2D). P (bf16, packed 2 per column) overwrites the upper 64
// columns of its S tile (the scores of keys 64-127, in registers by then), so the
// scores of keys 0-63 stay in TMEM for the rare recompute after a rescale, and
// feeds the PV product straight from TMEM.
// Shared memory: Q0, Q1 and a ring of NS key/value stages, each a 128 x D bf16
// tile stored as D/64 column blocks of 128 rows x 128 B with the 128-byte swizzle
// that TMA writes and the UMMA descriptors read.
//
// Per key tile j the MMA warp issues: PV0(j), S0(j+1), PV1(j), S1(j+1), so the
// tensor core computes one query tile's products while the other warpgroup
// runs its softmax. Rescaling of O is lazy: only when a row max grows by more
// than 2^8 (in the exp2 domain) is O multiplied in TMEM.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cstdint>
#include <cstdio>

#include "attn_fwd.h"
#include "geometry.h"
#include "sm100.cuh"

namespace cpattn {

using namespace sm100;

namespace {

constexpr int kThreads = 384;
constexpr float kRescaleThreshold = 8.0f;  // log2 units: rescale when max grows by > 256x
// P is handed to the MMA warp in two halves (keys 0-63, 64-127), so the first
// half of PV starts while the exponentials of the second half are computed.


template <int D>
struct Cfg {
  static constexpr int kTileBytes = kTile * D * 2;               // one 128 x D bf16 tile
  static constexpr int kBlocks = D / 64;                         // 128-byte column blocks
  static constexpr int kBlockBytes = kTile * 128;                // 16 KB
  static constexpr int kStages = D == 128 ? 5 : 8;
  static constexpr int kTmemCols = 512;
  static constexpr int kOCol = 256;
  static constexpr uint32_t kIdescS = idesc_bf16_f32(128, 128, 0, 0);   // Q K^T, both K-major
  static constexpr uint32_t kIdescPV = idesc_bf16_f32(128, D, 0, 1);    // P V, V is MN-major
};

template <int D>
struct alignas(1024) Smem {
  __nv_bfloat16 q[2][kTile * D];
  __nv_bfloat16 kv[Cfg<D>::kStages][kTile * D];
  uint64_t q_full, q_empty;
  uint64_t kv_full[Cfg<D>::kStages];
  uint64_t kv_empty[Cfg<D>::kStages];
  uint64_t s_full[2];
  uint64_t p_full[2][2];   // [query tile][P half]
  uint64_t o_done[2];
  uint64_t drain;
  uint32_t tmem_base;
  WaitBlock wblk;
};

// Loads a work item with a volatile access, which the compiler cannot merge with
// an earlier load of the same item.
__device__ __forceinline__ WorkItem ld_item_volatile(const WorkItem* ptr) {
  int4 v;
  asm volatile("ld.global.nc.v4.s32 {%0, %1, %2, %3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(ptr));
  return WorkItem{v.x, v.y, v.z, v.w};
}

// One CTA per SM: the dynamic shared memory request (struct + alignment slack)
// stays within the 227 KB a CTA may use.
static_assert(sizeof(Smem<128>) + 1024 <= 232448, "Smem<128> exceeds the per-CTA limit");
static_assert(sizeof(Smem<64>) + 1024 <= 232448, "Smem<64> exceeds the per-CTA limit");

__device__ __forceinline__ int lane_id() { return threadIdx.x & 31; }

template <int D>
__device__ __forceinline__ void issue_s(uint32_t tS, uint32_t q_addr, uint32_t k_addr) {
  // S = Q K^T over K = D in steps of 16: four steps per 128-byte column block.
#pragma unroll
  for (int kk = 0; kk < D / 16; ++kk) {
    const uint32_t off = (kk >> 2) * Cfg<D>::kBlockBytes + (kk & 3) * 32;
    const uint64_t a = smem_desc_sw128(q_addr + off, 16, 1024);
    const uint64_t b = smem_desc_sw128(k_addr + off, 16, 1024);
    umma_ss_elect(tS, a, b, Cfg<D>::kIdescS, kk > 0 ? 1u : 0u);
  }
}

template <int D, int KK_BEGIN, int KK_END>
__device__ __forceinline__ void issue_pv(uint32_t tO, uint32_t tP, uint32_t v_addr, bool accumulate) {
  // O (+)= P V over keys [16*KK_BEGIN, 16*KK_END) in steps of 16: P from TMEM (8
  // packed columns per step), V from shared memory as an MN-major operand (8-key
  // groups 1024 B apart, 64-column blocks kBlockBytes apart).
#pragma unroll
  for (int kk = KK_BEGIN; kk < KK_END; ++kk) {
    const uint64_t b = smem_desc_sw128(v_addr + kk * 2048, Cfg<D>::kBlockBytes, 1024);
    umma_ts_elect(tO, tP + kk * 8, b, Cfg<D>::kIdescPV, (accumulate || kk > 0) ? 1u : 0u);
  }
}

// Exponentials of one 32-column chunk c of a score row, packed to bf16 pairs and
// stored as 16 TMEM columns of P at tS + 64 + 16c (over the scores of keys
// 64-127, which are in registers by then); row-sum partials accumulate in ls.
// The scaling x = s * scale - m runs two columns per instruction (f32x2).
__device__ __forceinline__ void softmax_chunk(const float (&s)[kTile], int c, float sl2, float m_use,
                                              uint32_t tS, float (&ls)[8]) {
  uint32_t pk[16];
  const uint64_t sl2_2 = f2_pack(sl2, sl2);
  const uint64_t nm_2 = f2_pack(-m_use, -m_use);
#pragma unroll
  for (int j = 0; j < 16; ++j) {
    const int col = c * 32 + 2 * j;
    float x0, x1;
    f2_unpack(f2_fma(f2_pack(s[col], s[col + 1]), sl2_2, nm_2), x0, x1);
    const float e0 = ex2_approx(x0);
    const float e1 = ex2_approx(x1);
    ls[j & 7] += e0 + e1;
    pk[j] = pack_bf16x2(e0, e1);
  }
  tmem_st16(tS + 64 + c * 16, pk);
}

// Maximum of the 64 scores s[32c .. 32c+63], four chains of 3-input maxima.
__device__ __forceinline__ float half_max(const float (&s)[kTile], int c) {
  float m[4];
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    const int b = 32 * c + 16 * k;
    float x = max3(s[b], s[b + 1], s[b + 2]);
#pragma unroll
    for (int j = 3; j + 1 < 16; j += 2) x = max3(x, s[b + j], s[b + j + 1]);
    m[k] = fmaxf(x, s[b + 15]);
  }
  return fmaxf(max3(m[0], m[1], m[2]), m[3]);
}

}  // namespace

// Walk of an item: its precomputed key tiles over ring steps [t_begin, t_end),
// or over its own step for the units of a ring launch.
template <bool PARTIAL>
__device__ __forceinline__ void item_walk(const FwdParams& p, const WorkItem& w, int rq, int& e_begin, int& e_end) {
  const int qp = PARTIAL ? item_qp(w) : w.qp;
  const int* off = p.step_off + (rq * p.npairs + qp) * (p.g.NR + 1);
  int t0 = p.t_begin, t1 = p.t_end;
  if (PARTIAL && p.unit_steps) {
    t0 = unit_t0(w);
    t1 = unit_t1(w);
  }
  e_begin = __ldg(off + t0);
  e_end = __ldg(off + t1);
}

template <int D, bool PARTIAL>
__global__ void __launch_bounds__(kThreads, 1)
    attn_fwd_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                    const __grid_constant__ CUtensorMap tm_v, const FwdParams p) {
  using C = Cfg<D>;
  extern __shared__ uint8_t smem_raw[];
  Smem<D>& sm = *reinterpret_cast<Smem<D>*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));

  const int warp = threadIdx.x >> 5;
  const int lane = lane_id();
  const Geometry g = p.g;

  if (threadIdx.x == 0) {
    mbar_init(smem_addr(&sm.q_full), 1);
    mbar_init(smem_addr(&sm.q_empty), 1);
    for (int s = 0; s < C::kStages; ++s) {
      mbar_init(smem_addr(&sm.kv_full[s]), 1);
      mbar_init(smem_addr(&sm.kv_empty[s]), 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(smem_addr(&sm.s_full[i]), 1);
      mbar_init(smem_addr(&sm.p_full[i][0]), 128);
      mbar_init(smem_addr(&sm.p_full[i][1]), 128);
      mbar_init(smem_addr(&sm.o_done[i]), 1);
    }
    mbar_init(smem_addr(&sm.drain), 1);
    wait_block_init(sm.wblk, p.status, p.wait_limit_ns);
    fence_barrier_init();
  }
  if (warp == 8) {
    tmem_alloc(smem_addr(&sm.tmem_base), C::kTmemCols);
    tmem_relinquish();
  }
  if (warp == 9 && lane == 0) {
    prefetch_tensormap(&tm_q);
    prefetch_tensormap(&tm_k);
    prefetch_tensormap(&tm_v);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = sm.tmem_base;
  const WaitCtl ctl = wait_ctl(sm.wblk);
  const int it_end = __ldg(p.cta_begin + blockIdx.x + 1);   // this CTA's items end here

  // Every role walks the same precomputed key list of each work item.

  if (warp == 9) {
    // ------------------------------------------------------------ TMA producer
    // The whole warp runs the loop; one elected lane issues each load.
    {
      const uint64_t pol_q = l2_policy_evict_first();
      const uint64_t pol_kv = l2_policy_evict_last();
      int q_iter = 0;
      int kv_idx = 0;
      bool ok = true;
      for (int it = __ldg(p.cta_begin + blockIdx.x); it < it_end && ok; ++it) {
        const WorkItem w = p.items[it];
        const int rq = w.rb / g.B;
        const int bv = w.rb - rq * g.B;
        const int q0 = (PARTIAL ? item_qp(w) : w.qp) * kPair;
        int e_begin, e_end;
        item_walk<PARTIAL>(p, w, rq, e_begin, e_end);
        if (q_iter > 0) ok = mbar_wait(smem_addr(&sm.q_empty), (q_iter - 1) & 1, ctl);
        ok = __all_sync(0xffffffffu, ok);
        if (!ok) break;
        const uint32_t qbar = smem_addr(&sm.q_full);
        mbar_arrive_expect_tx_elect(qbar, 2 * C::kTileBytes);
        for (int i = 0; i < 2; ++i)
          for (int blk = 0; blk < C::kBlocks; ++blk)
            tma_load_4d_elect(smem_addr(&sm.q[i][0]) + blk * C::kBlockBytes, &tm_q, qbar, blk * 64, w.h,
                        q0 + i * kTile, w.rb - p.q_rb0, pol_q);
        ++q_iter;
        int waited = rq;   // the block last waited for (the own block needs no wait)
        for (int e = e_begin; e < e_end && ok; ++e) {
          const uint32_t ent = __ldg(p.entries + e);
          if (PARTIAL && p.arrived != nullptr && entry_rank(ent) != waited) {
            // first load from another rank's block: wait until all of it has arrived
            waited = entry_rank(ent);
            ok = count_wait(p.arrived + waited, p.arrive_target, ctl);
            ok = __all_sync(0xffffffffu, ok);
            if (!ok) break;
          }
          const int rbk = p.kv_local ? bv : entry_rank(ent) * g.B + bv;
          const int k0 = entry_tile(ent) * kTile;
          for (int which = 0; which < 2; ++which) {
            const int stage = kv_idx % C::kStages;
            const int round = kv_idx / C::kStages;
            if (round > 0) ok = mbar_wait(smem_addr(&sm.kv_empty[stage]), (round - 1) & 1, ctl);
            ok = __all_sync(0xffffffffu, ok);
            if (!ok) break;
            const uint32_t bar = smem_addr(&sm.kv_full[stage]);
            mbar_arrive_expect_tx_elect(bar, C::kTileBytes);
            const CUtensorMap* map = which == 0 ? &tm_k : &tm_v;
            for (int blk = 0; blk < C::kBlocks; ++blk)
              tma_load_4d_elect(smem_addr(&sm.kv[stage][0]) + blk * C::kBlockBytes, map, bar, blk * 64, w.h, k0,
                          rbk, pol_kv);
            ++kv_idx;
          }
        }
      }
      if (!ok) {
        // Abort: let every load this thread issued land before the CTA exits.
        const uint64_t lim = p.wait_limit_ns;
        for (int idx = kv_idx - C::kStages; idx < kv_idx; ++idx)
          if (idx >= 0)
            mbar_wait_drain(smem_addr(&sm.kv_full[idx % C::kStages]), (idx / C::kStages) & 1, lim);
        if (q_iter > 0) mbar_wait_drain(smem_addr(&sm.q_full), (q_iter - 1) & 1, lim);
      }
    }
  } else if (warp == 8) {
    // ------------------------------------------------------------ MMA issuer
    // The whole warp runs the loop; one elected lane issues each MMA and commit.
    {
      const uint32_t tS0 = tbase, tS1 = tbase + 128;
      const uint32_t tO0 = tbase + C::kOCol, tO1 = tbase + C::kOCol + D;
      const uint32_t q_addr0 = smem_addr(&sm.q[0][0]), q_addr1 = smem_addr(&sm.q[1][0]);
      int q_iter = 0, kv_idx = 0;
      int p_cnt0 = 0, p_cnt1 = 0;
      bool ok = true, issued = false;
      for (int it = __ldg(p.cta_begin + blockIdx.x); it < it_end && ok; ++it) {
        const WorkItem w = p.items[it];
        const int rq = w.rb / g.B;
        int e_begin, e_end;
        item_walk<PARTIAL>(p, w, rq, e_begin, e_end);
        // The last PV of each query tile signals o_done: find where they are.
        int last0 = -1, last1 = -1;
        for (int e = e_begin; e < e_end; ++e) {
          const uint32_t ent = __ldg(p.entries + e);
          if (entry_c0(ent) != kSkip) last0 = e;
          if (entry_c1(ent) != kSkip) last1 = e;
        }
        ok = mbar_wait(smem_addr(&sm.q_full), q_iter & 1, ctl);
        ok = __all_sync(0xffffffffu, ok);
        if (!ok) break;
        ++q_iter;
        tc_fence_after();
        if (e_begin == e_end) {
          umma_commit_elect(smem_addr(&sm.q_empty));
          continue;
        }
        // First key tile: its S products.
        uint32_t cur = __ldg(p.entries + e_begin);
        int kst = kv_idx % C::kStages;
        ok = mbar_wait(smem_addr(&sm.kv_full[kst]), (kv_idx / C::kStages) & 1, ctl);
        ok = __all_sync(0xffffffffu, ok);
        if (!ok) break;
        ++kv_idx;
        tc_fence_after();
        {
          const uint32_t k_addr = smem_addr(&sm.kv[kst][0]);
          if (entry_c0(cur) != kSkip) {
            issue_s<D>(tS0, q_addr0, k_addr);
            umma_commit_elect(smem_addr(&sm.s_full[0]));
          }
          if (entry_c1(cur) != kSkip) {
            issue_s<D>(tS1, q_addr1, k_addr);
            umma_commit_elect(smem_addr(&sm.s_full[1]));
          }
        }
        issued = true;
        umma_commit_elect(smem_addr(&sm.kv_empty[kst]));
        bool acc0 = false, acc1 = false;
        for (int e = e_begin; e < e_end; ++e) {
          const bool has_next = e + 1 < e_end;
          const uint32_t nxt = has_next ? __ldg(p.entries + e + 1) : 0u;
          // Both operand tiles of this step first (V of this tile, K of the next),
          // so that once P is ready the PV and the next S issue back to back.
          const int vst = kv_idx % C::kStages;
          ok = mbar_wait(smem_addr(&sm.kv_full[vst]), (kv_idx / C::kStages) & 1, ctl);
          ok = __all_sync(0xffffffffu, ok);
          if (!ok) break;
          ++kv_idx;
          int nst = 0;
          if (has_next) {
            nst = kv_idx % C::kStages;
            ok = mbar_wait(smem_addr(&sm.kv_full[nst]), (kv_idx / C::kStages) & 1, ctl);
            ok = __all_sync(0xffffffffu, ok);
            if (!ok) break;
            ++kv_idx;
          }
          tc_fence_after();
          const uint32_t v_addr = smem_addr(&sm.kv[vst][0]);
          const uint32_t nk_addr = smem_addr(&sm.kv[nst][0]);
          // Query tile 0: PV0(cur), then S0(next).
          if (entry_c0(cur) != kSkip) {
            // First half of P (keys 0-63), then the second half.
            ok = mbar_wait(smem_addr(&sm.p_full[0][0]), p_cnt0 & 1, ctl);
            ok = __all_sync(0xffffffffu, ok);
            if (!ok) break;
            tc_fence_after();
            issue_pv<D, 0, 4>(tO0, tS0 + 64, v_addr, acc0);
            ok = mbar_wait(smem_addr(&sm.p_full[0][1]), p_cnt0 & 1, ctl);
            ok = __all_sync(0xffffffffu, ok);
            if (!ok) break;
            tc_fence_after();
            issue_pv<D, 4, 8>(tO0, tS0 + 64, v_addr, true);
            ++p_cnt0;
            acc0 = true;
            if (e == last0) umma_commit_elect(smem_addr(&sm.o_done[0]));
          }
          if (has_next && entry_c0(nxt) != kSkip) {
            issue_s<D>(tS0, q_addr0, nk_addr);
            umma_commit_elect(smem_addr(&sm.s_full[0]));
          }
          // Query tile 1: PV1(cur), then S1(next).
          if (entry_c1(cur) != kSkip) {
            // First half of P (keys 0-63), then the second half.
            ok = mbar_wait(smem_addr(&sm.p_full[1][0]), p_cnt1 & 1, ctl);
            ok = __all_sync(0xffffffffu, ok);
            if (!ok) break;
            tc_fence_after();
            issue_pv<D, 0, 4>(tO1, tS1 + 64, v_addr, acc1);
            ok = mbar_wait(smem_addr(&sm.p_full[1][1]), p_cnt1 & 1, ctl);
            ok = __all_sync(0xffffffffu, ok);
            if (!ok) break;
            tc_fence_after();
            issue_pv<D, 4, 8>(tO1, tS1 + 64, v_addr, true);
            ++p_cnt1;
            acc1 = true;
            if (e == last1) umma_commit_elect(smem_addr(&sm.o_done[1]));
          }
          if (has_next && entry_c1(nxt) != kSkip) {
            issue_s<D>(tS1, q_addr1, nk_addr);
            umma_commit_elect(smem_addr(&sm.s_full[1]));
          }
          if (has_next) umma_commit_elect(smem_addr(&sm.kv_empty[nst]));
          umma_commit_elect(smem_addr(&sm.kv_empty[vst]));
          cur = nxt;
        }
        if (!ok) break;
        umma_commit_elect(smem_addr(&sm.q_empty));
      }
      if (issued) {
        // Every tensor-core op (and the arrivals of its commits) must finish before
        // TMEM is freed and the CTA exits; on the abort path too.
        umma_commit_elect(smem_addr(&sm.drain));
        mbar_wait_drain(smem_addr(&sm.drain), 0, p.wait_limit_ns);
      }
    }
  } else if (warp < 8) {
    // ------------------------------------------------------------ softmax warpgroups
    const int wg = warp >> 2;
    const int quad = warp & 3;
    const int row = quad * 32 + lane;
    const uint32_t lane_off = static_cast<uint32_t>(quad * 32) << 16;
    const uint32_t tS = tbase + lane_off + wg * 128;
    const uint32_t tO = tbase + lane_off + C::kOCol + wg * D;
    const float sl2 = p.scale_log2;
    const int cls_shift = wg == 0 ? 25 : 27;
    int s_cnt = 0, od_cnt = 0;
    bool ok = true;
    for (int it = __ldg(p.cta_begin + blockIdx.x); it < it_end && ok; ++it) {
      int64_t gq;
      bool valid;
      int e_begin, e_end;
      {
        const WorkItem w = p.items[it];
        const int rq = w.rb / g.B;
        const int tl = (PARTIAL ? item_qp(w) : w.qp) * kPair + wg * kTile + row;
        valid = tl < g.T;
        gq = global_pos(g, rq, valid ? tl : g.T - 1);
        item_walk<PARTIAL>(p, w, rq, e_begin, e_end);
      }
      float m_run = -INFINITY, l_run = 0.f;
      int ntile = 0;
      uint32_t ent = e_begin < e_end ? __ldg(p.entries + e_begin) : 0u;
      for (int e = e_begin; e < e_end; ++e) {
        const uint32_t cur = ent;
        if (e + 1 < e_end) ent = __ldg(p.entries + e + 1);   // prefetch the next entry
        const int cls = static_cast<int>((cur >> cls_shift) & 3u);
        if (cls == kSkip) continue;
        ok = mbar_wait(smem_addr(&sm.s_full[wg]), s_cnt & 1, ctl);
        ok = __all_sync(0xffffffffu, ok);
        if (!ok) break;
        ++s_cnt;
        tc_fence_after();
        const int rk = entry_rank(cur);
        const int kt = entry_tile(cur);
        float s[kTile];
        tmem_ld128(tS, reinterpret_cast<uint32_t*>(s));
        if (cls == kMasked) {
          const int lim = valid ? column_limit(g, rk, kt * kTile, gq) : 0;
#pragma unroll
          for (int j = 0; j < kTile; ++j) s[j] = j < lim ? s[j] : -INFINITY;
        }
        // Exponentials, then the row max. Rescaling is lazy (the running max
        // moves only when the scores exceed it by more than 2^8), so when every
        // row of the warp has a running max, the exponentials of keys 0-63 start
        // from it at once and the tile's own max is computed alongside them; a
        // warp with a row still at -inf takes the max of keys 0-63 first. When
        // the tile raises a row's max past the threshold (rare after a row's
        // first tiles), P of keys 0-63 and its partial sums are recomputed from
        // the scores with the new max before the MMA warp may read them.
        const float m_prev = m_run;
        const bool stale = __all_sync(0xffffffffu, m_run != -INFINITY);
        // Stale path: the exponentials do not depend on m01, so its max chain
        // overlaps them; it comes first only so the scores of keys 0-63 die early.
        const float m01 = half_max(s, 0);
        bool resc = false;
        if (!stale) {
          resc = m01 * sl2 - m_run > kRescaleThreshold;   // false while both are -inf
          if (resc) m_run = m01 * sl2;
        }
        float m_use = m_run == -INFINITY ? 0.f : m_run;
        float ls[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
        softmax_chunk(s, 0, sl2, m_use, tS, ls);
        softmax_chunk(s, 1, sl2, m_use, tS, ls);
        const float m23 = half_max(s, 2);
        const float mt = stale ? fmaxf(m01, m23) : m23;
        const bool resc_b = mt * sl2 - m_run > kRescaleThreshold;
        if (__any_sync(0xffffffffu, resc_b)) {
          if (resc_b) {
            m_run = mt * sl2;
            m_use = m_run;
            resc = true;
          }
          // Recompute P of keys 0-63 with the (possibly) new max, from their
          // scores, still intact in TMEM columns 0-63 (P is written over those
          // of keys 64-127): exact, and no value computed from a stale max is
          // ever published.
          tmem_st_wait();
          tmem_ld64(tS, *reinterpret_cast<uint32_t(*)[32]>(&s[0]), *reinterpret_cast<uint32_t(*)[32]>(&s[32]));
          if (cls == kMasked) {
            const int lim = valid ? column_limit(g, entry_rank(cur), entry_tile(cur) * kTile, gq) : 0;
#pragma unroll
            for (int j = 0; j < 64; ++j) s[j] = j < lim ? s[j] : -INFINITY;
          }
#pragma unroll
          for (int q = 0; q < 8; ++q) ls[q] = 0.f;
          softmax_chunk(s, 0, sl2, m_use, tS, ls);
          softmax_chunk(s, 1, sl2, m_use, tS, ls);
        }
        const float alpha = resc ? ex2_approx(m_prev - m_run) : 1.f;   // 0 when m_prev = -inf
        l_run *= alpha;
        if (ntile > 0 && __any_sync(0xffffffffu, resc)) {
          // O holds the previous PV products (complete: this tile's s_full was
          // committed after them) and no PV of this tile starts before p_full:
          // rescale it in place.
#pragma unroll
          for (int c = 0; c < D; c += 16) {
            uint32_t o[16];
            tmem_ld16(tO + c, o);
#pragma unroll
            for (int q = 0; q < 16; ++q) o[q] = __float_as_uint(__uint_as_float(o[q]) * alpha);
            tmem_st16(tO + c, o);
          }
        }
        tmem_st_wait();
        tc_fence_before();
        mbar_arrive(smem_addr(&sm.p_full[wg][0]));
        softmax_chunk(s, 2, sl2, m_use, tS, ls);
        softmax_chunk(s, 3, sl2, m_use, tS, ls);
        const float lsum = ((ls[0] + ls[1]) + (ls[2] + ls[3])) + ((ls[4] + ls[5]) + (ls[6] + ls[7]));
        l_run += lsum;
        tmem_st_wait();
        tc_fence_before();
        mbar_arrive(smem_addr(&sm.p_full[wg][1]));
        ++ntile;
      }
      if (!ok) break;
      // ---------------------------------------------------------- epilogue
      // The item's fields again: a fresh load, so that they are not kept live
      // across the key loop in registers the scores need.
      const WorkItem w = ld_item_volatile(p.items + it);
      const int bv = w.rb % g.B;
      const int tl = (PARTIAL ? item_qp(w) : w.qp) * kPair + wg * kTile + row;
      const int64_t row_id = (static_cast<int64_t>(w.rb - p.q_rb0) * g.T + tl) * g.Hh + w.h +
                             (PARTIAL && p.unit_steps ? min(unit_t0(w), p.unit_split) * p.part_rows : 0);
      if (ntile > 0) {
        ok = mbar_wait(smem_addr(&sm.o_done[wg]), od_cnt & 1, ctl);
        ok = __all_sync(0xffffffffu, ok);
        if (!ok) break;
        ++od_cnt;
        tc_fence_after();
        const float inv = l_run > 0.f ? 1.f / l_run : 0.f;
#pragma unroll
        for (int c = 0; c < D; c += 32) {
          uint32_t o[32];
          tmem_ld32(tO + c, o);
          if (valid) {
            if (PARTIAL) {
              float4* dst = reinterpret_cast<float4*>(p.o_part + row_id * D + c);
#pragma unroll
              for (int j = 0; j < 8; ++j)
                dst[j] = make_float4(__uint_as_float(o[4 * j]) * inv, __uint_as_float(o[4 * j + 1]) * inv,
                                     __uint_as_float(o[4 * j + 2]) * inv,
                                     __uint_as_float(o[4 * j + 3]) * inv);
            } else {
              uint4* dst = reinterpret_cast<uint4*>(p.o + row_id * D + c);
#pragma unroll
              for (int j = 0; j < 4; ++j) {
                uint4 v;
                v.x = pack_bf16x2(__uint_as_float(o[8 * j + 0]) * inv, __uint_as_float(o[8 * j + 1]) * inv);
                v.y = pack_bf16x2(__uint_as_float(o[8 * j + 2]) * inv, __uint_as_float(o[8 * j + 3]) * inv);
                v.z = pack_bf16x2(__uint_as_float(o[8 * j + 4]) * inv, __uint_as_float(o[8 * j + 5]) * inv);
                v.w = pack_bf16x2(__uint_as_float(o[8 * j + 6]) * inv, __uint_as_float(o[8 * j + 7]) * inv);
                dst[j] = v;
              }
            }
          }
        }
        if (valid) {
          const float lse = l_run > 0.f ? (m_run + __log2f(l_run)) * 0.69314718055994531f : -INFINITY;
          if (PARTIAL) {
            p.lse_part[row_id] = lse;
          } else if (p.lse != nullptr) {
            const int64_t li = (static_cast<int64_t>(bv % p.lse_B) * p.lse_H + (bv / p.lse_B) * g.Hh + w.h) *
                                   p.lse_S + gq;
            p.lse[li] = lse;
          }
        }
      } else if (valid) {
        // No allowed key at all in the visited steps: O = 0, lse = -inf.
        if (PARTIAL) {
          float4* dst = reinterpret_cast<float4*>(p.o_part + row_id * D);
          for (int j = 0; j < D / 4; ++j) dst[j] = make_float4(0.f, 0.f, 0.f, 0.f);
          p.lse_part[row_id] = -INFINITY;
        } else {
          uint4* dst = reinterpret_cast<uint4*>(p.o + row_id * D);
          for (int j = 0; j < D / 8; ++j) dst[j] = make_uint4(0, 0, 0, 0);
          if (p.lse != nullptr) {
            const int64_t li = (static_cast<int64_t>(bv % p.lse_B) * p.lse_H + (bv / p.lse_B) * g.Hh + w.h) *
                                   p.lse_S + gq;
            p.lse[li] = -INFINITY;
          }
        }
      }
    }
  }

  if constexpr (PARTIAL) {
    if (warp >= 10 && p.pull_chunks > 0) {
      // ---------------------------------------------------------- fused pull
      // Copy warps: chunk c of the (NR - 1) * pull_chunks chunks goes to copy
      // warp c mod (2 * grid), so every warp walks the blocks in ring order and
      // each block completes at about the same time on all of them.
      const int cw = static_cast<int>(blockIdx.x) * 2 + (warp - 10);
      const int ncw = static_cast<int>(gridDim.x) * 2;
      const int rank = p.q_rb0 / g.B;
      const int per_half = p.pull_chunks / 2;
      const int64_t half = p.pull_block_bytes;
      const int64_t total = static_cast<int64_t>(g.NR - 1) * p.pull_chunks;
      // The fetch streams every other block through L2 once: evict-first, so
      // that it does not displace the key/value tiles the units are reusing
      // (their TMA loads are evict-last).
      const uint64_t pol = l2_policy_evict_first();
      for (int64_t c = cw; c < total; c += ncw) {
        if (abort_raised(ctl.wb)) break;
        const int jj = static_cast<int>(c / p.pull_chunks);
        const int ci = static_cast<int>(c - static_cast<int64_t>(jj) * p.pull_chunks);
        int j = rank + 1 + jj;
        if (j >= g.NR) j -= g.NR;
        const int is_v = ci >= per_half;
        const int64_t off = static_cast<int64_t>(ci - is_v * per_half) * p.pull_chunk_bytes;
        const int64_t n = half - off < p.pull_chunk_bytes ? half - off : p.pull_chunk_bytes;
        const char* src = reinterpret_cast<const char*>(p.pull_src[2 * j + is_v]) + off;
        char* dst = (is_v ? p.pull_v_all : p.pull_k_all) + static_cast<int64_t>(j) * half + off;
        constexpr int kU = 8;   // 16-byte vectors in flight per lane
        for (int64_t i = static_cast<int64_t>(lane) * 16; i < n; i += 32 * 16 * kU) {
          uint4 r[kU];
#pragma unroll
          for (int u = 0; u < kU; ++u)
            if (i + u * 512 < n) r[u] = ld_stream_v4_policy(src + i + u * 512, pol);
#pragma unroll
          for (int u = 0; u < kU; ++u)
            if (i + u * 512 < n) st_v4_policy(dst + i + u * 512, r[u], pol);
        }
        chunk_stores_fence();
        __syncwarp();
        if (lane == 0) red_release_add(p.arrived + j, 1);
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 8) {
    tc_fence_after();
    tmem_dealloc(tbase, C::kTmemCols);
  }
}

// ---------------------------------------------------------------------- host side

namespace {

template <int D, bool PARTIAL>
cudaError_t launch_impl(const FwdLaunch& L, cudaStream_t stream) {
  const size_t smem = sizeof(Smem<D>) + 1024;
  auto kern = attn_fwd_kernel<D, PARTIAL>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  const int grid = L.params.n_cta;   // the schedule's CTA count (normally the SM count)
  if (grid <= 0) return cudaSuccess;
  // A fused-pull launch is cooperative: units wait for chunks that copy warps of
  // other CTAs bring in, so all CTAs must be resident together (one per SM).
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeCooperative;
  attr[0].val.cooperative = 1;
  cfg.attrs = attr;
  cfg.numAttrs = (PARTIAL && L.params.pull_chunks > 0) ? 1 : 0;
  return cudaLaunchKernelEx(&cfg, kern, L.tm_q, L.tm_k, L.tm_v, L.params);
}

}  // namespace

cudaError_t launch_attn_fwd(const FwdLaunch& L, int D, bool partial, cudaStream_t stream) {
  if (D == 128) return partial ? launch_impl<128, true>(L, stream) : launch_impl<128, false>(L, stream);
  if (D == 64) return partial ? launch_impl<64, true>(L, stream) : launch_impl<64, false>(L, stream);
  return cudaErrorInvalidValue;
}

size_t attn_fwd_smem_bytes(int D) {
  return D == 128 ? sizeof(Smem<128>) + 1024 : sizeof(Smem<64>) + 1024;
}

}  // namespace cpattn
