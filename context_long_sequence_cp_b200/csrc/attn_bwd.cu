// attn_bwd.cu — backward pass of the context-parallel attention: dQ, dK, dV from
// the saved logsumexp, with the same global-position causal mask and ring walk
// as the forward.
//
// The pages train long-context models (page "序列与上下文并行", opening and
// section "长上下文的显存墙") but print no backward pass; the backward of the
// method's plain softmax attention (page "Tensor并行与算子拆分", section
// "注意力的并行化优化") is its chain rule, per (batch, head):
//   P = exp(scale * Q K^T - lse),  dV = P^T dO,  dP = dO V^T,
//   Dr = rowsum(dO * O),  dS = P * (dP - Dr),  dQ = scale dS K,  dK = scale dS^T Q.
//
// Three kernels, no atomics (results are deterministic):
//   bwd_pre_kernel     per view row: nlse2 = -lse * log2(e) and Dr, stored
//                      [NR*B][Hh][T] so that a query tile's 128 values are
//                      contiguous (one bulk copy).
//   attn_bwd_kv_kernel one 128-key tile per work item; walks the query tiles
//                      that see it. TMEM (512 columns): region A [0,128) takes
//                      S^T = K Q^T and then dP^T = V dO^T of the same tile,
//                      region B [128,256) the bf16 P^T and dS^T, then dV and dK.
//                      Keys are TMEM lanes, so P^T and dS^T feed dV += P^T dO and
//                      dK += dS^T Q straight from TMEM; dO and Q are read as
//                      MN-major operands (no transpose is materialised). The next
//                      tile's S^T runs while the current P^T/dS^T are formed.
//   attn_bwd_q_kernel  one 128-query tile per work item; walks the key tiles it
//                      sees in ring order. TMEM: S = Q K^T [0,128), dP = dO V^T
//                      [128,256), dQ [256,256+D), dS double-buffered as bf16 in
//                      [384,448) and [448,512); dS (from TMEM) times K (MN-major)
//                      accumulates dQ. S and dP of the next key tile are computed
//                      while the current dS is formed. K and V come through
//                      rings of their own: V is released once dP has read it, K
//                      (3 stages at D = 128) only once dQ has, so the next tiles'
//                      loads are in flight while a tile's dS is formed.
// The dK/dV and dQ kernels recompute S and dP each (7 tile products per tile
// pair instead of 5 with an atomic dQ): the price of having no atomics.
//
// Both tile kernels use the forward's layout of roles (12 warps, one persistent
// CTA per SM): warps 0-7 two elementwise warpgroups (warpgroup w owns columns
// [64w, 64w+64) of every tile, one TMEM lane = one row per thread), warp 8 the
// MMA issuer (whole warp, elect.sync issue), warp 9 the TMA producer (same),
// warps 10-11 idle. The two warpgroups write their bf16 halves inside their own
// fp32 columns (P of columns 0-63 at [0,32), of 64-127 at [64,96)), so neither
// overwrites scores the other has not read; the accumulating MMAs read that
// layout. Every wait is bounded (CP_ERR_TIMEOUT in the plan's status word).
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cstdint>

#include "attn_bwd.h"
#include "geometry.h"
#include "sm100.cuh"

namespace cpattn {

using namespace sm100;

namespace {

constexpr int kBwdThreads = 384;
constexpr int kWarpMma = 8;
constexpr int kWarpTma = 9;
constexpr float kLog2e = 1.4426950408889634f;

template <int D>
struct BwdCfg {
  static constexpr int kTileBytes = kTile * D * 2;   // one 128 x D bf16 tile
  static constexpr int kBlocks = D / 64;             // 128-byte column blocks
  static constexpr int kBlockBytes = kTile * 128;    // 16 KB
  static constexpr int kStages = D == 128 ? 2 : 4;
  // dQ kernel: K is held from S(e) until dQ(e) has read it, V only until dP(e)
  // has, so the two have rings of their own and K the deeper one.
  static constexpr int kKStages = D == 128 ? 3 : 5;
  static constexpr int kVStages = D == 128 ? 2 : 4;
  static constexpr uint32_t kIdescS = idesc_bf16_f32(128, 128, 0, 0);   // both operands K-major
  static constexpr uint32_t kIdescAcc = idesc_bf16_f32(128, D, 0, 1);   // A from TMEM, B MN-major
};

// C = A B^T over K = D: A and B are 128 x D bf16 tiles, both K-major (the
// forward's score product form).
template <int D>
__device__ __forceinline__ void issue_nt(uint32_t tC, uint32_t a_addr, uint32_t b_addr) {
#pragma unroll
  for (int kk = 0; kk < D / 16; ++kk) {
    const uint32_t off = (kk >> 2) * BwdCfg<D>::kBlockBytes + (kk & 3) * 32;
    umma_ss_elect(tC, smem_desc_sw128(a_addr + off, 16, 1024), smem_desc_sw128(b_addr + off, 16, 1024),
                  BwdCfg<D>::kIdescS, kk > 0 ? 1u : 0u);
  }
}

// dQ (+)= dS K over the 128 keys of a tile: dS from a TMEM buffer of 64 packed
// columns (keys 16kk.. at column 8kk), K a 128 x D tile read as an MN-major operand.
template <int D>
__device__ __forceinline__ void issue_dq(uint32_t tdQ, uint32_t tBuf, uint32_t k_addr, bool accumulate) {
#pragma unroll
  for (int kk = 0; kk < 8; ++kk) {
    const uint64_t b = smem_desc_sw128(k_addr + kk * 2048, BwdCfg<D>::kBlockBytes, 1024);
    umma_ts_elect(tdQ, tBuf + kk * 8, b, BwdCfg<D>::kIdescAcc, (accumulate || kk > 0) ? 1u : 0u);
  }
}

// Two 32-column TMEM loads, one wait.
__device__ __forceinline__ void tmem_ld32x2(uint32_t ta, uint32_t tb, uint32_t (&a)[32], uint32_t (&b)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, "
      "%12, %13, %14, %15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%64];\n\t"
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%32, %33, %34, %35, %36, %37, %38, %39, %40, %41, %42, %43, "
      "%44, %45, %46, %47, %48, %49, %50, %51, %52, %53, %54, %55, %56, %57, %58, %59, %60, %61, %62, %63}, [%65];\n\t"
      "tcgen05.wait::ld.sync.aligned;"
      : "=r"(a[0]), "=r"(a[1]), "=r"(a[2]), "=r"(a[3]), "=r"(a[4]), "=r"(a[5]), "=r"(a[6]), "=r"(a[7]),
        "=r"(a[8]), "=r"(a[9]), "=r"(a[10]), "=r"(a[11]), "=r"(a[12]), "=r"(a[13]), "=r"(a[14]), "=r"(a[15]),
        "=r"(a[16]), "=r"(a[17]), "=r"(a[18]), "=r"(a[19]), "=r"(a[20]), "=r"(a[21]), "=r"(a[22]), "=r"(a[23]),
        "=r"(a[24]), "=r"(a[25]), "=r"(a[26]), "=r"(a[27]), "=r"(a[28]), "=r"(a[29]), "=r"(a[30]), "=r"(a[31]),
        "=r"(b[0]), "=r"(b[1]), "=r"(b[2]), "=r"(b[3]), "=r"(b[4]), "=r"(b[5]), "=r"(b[6]), "=r"(b[7]),
        "=r"(b[8]), "=r"(b[9]), "=r"(b[10]), "=r"(b[11]), "=r"(b[12]), "=r"(b[13]), "=r"(b[14]), "=r"(b[15]),
        "=r"(b[16]), "=r"(b[17]), "=r"(b[18]), "=r"(b[19]), "=r"(b[20]), "=r"(b[21]), "=r"(b[22]), "=r"(b[23]),
        "=r"(b[24]), "=r"(b[25]), "=r"(b[26]), "=r"(b[27]), "=r"(b[28]), "=r"(b[29]), "=r"(b[30]), "=r"(b[31])
      : "r"(ta), "r"(tb)
      : "memory");
}

// Writes a 128-byte-aligned run of D/nparts columns of a TMEM accumulator row,
// times `mul`, as bf16 to dst (or zeros when `have` is false).
template <int NCOL>
__device__ __forceinline__ void store_row_bf16(uint32_t tAcc, bool have, float mul, __nv_bfloat16* dst, bool valid) {
#pragma unroll
  for (int c = 0; c < NCOL; c += 32) {
    uint32_t r[32];
    if (have) {
      tmem_ld32(tAcc + c, r);
    } else {
#pragma unroll
      for (int q = 0; q < 32; ++q) r[q] = 0u;
    }
    if (valid) {
      uint4* d = reinterpret_cast<uint4*>(dst + c);
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        uint4 u;
        u.x = pack_bf16x2(__uint_as_float(r[8 * q + 0]) * mul, __uint_as_float(r[8 * q + 1]) * mul);
        u.y = pack_bf16x2(__uint_as_float(r[8 * q + 2]) * mul, __uint_as_float(r[8 * q + 3]) * mul);
        u.z = pack_bf16x2(__uint_as_float(r[8 * q + 4]) * mul, __uint_as_float(r[8 * q + 5]) * mul);
        u.w = pack_bf16x2(__uint_as_float(r[8 * q + 6]) * mul, __uint_as_float(r[8 * q + 7]) * mul);
        d[q] = u;
      }
    }
  }
}

// ------------------------------------------------------------------ preprocess
// One warp per view row: Dr = sum_d dO * O (fp32), and the row's lse in log2
// units, negated (so that P = exp2(fma(s, scale_log2, nlse2))), both stored
// [NR*B][Hh][T].
template <int D>
__global__ void __launch_bounds__(256) bwd_pre_kernel(const BwdPreParams p) {
  const Geometry g = p.g;
  const int lane = threadIdx.x & 31;
  const int64_t warp0 = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const int64_t nwarps = (static_cast<int64_t>(gridDim.x) * blockDim.x) >> 5;
  const int64_t rows = static_cast<int64_t>(g.NR) * g.B * g.T * g.Hh;
  // The dK/dV kernel's 512-byte copies of a ragged last query tile read up to
  // 127 values past the end of each array: zero dvec's padding, so that a masked
  // column's P = 0 times (dP - Dr) stays 0 (lse2's over-read lands in dvec).
  if (blockIdx.x == 0 && threadIdx.x < kTile) p.dvec[rows + threadIdx.x] = 0.f;
  constexpr int E = D / 32;   // elements per lane: 4 (D = 128) or 2 (D = 64)
  for (int64_t r = warp0; r < rows; r += nwarps) {
    const __nv_bfloat16* orow = p.o + r * D + lane * E;
    const __nv_bfloat16* grow = p.dout + r * D + lane * E;
    float acc = 0.f;
    if (E == 4) {
      const uint2 a = __ldg(reinterpret_cast<const uint2*>(orow));
      const uint2 b = __ldg(reinterpret_cast<const uint2*>(grow));
      const uint32_t av[2] = {a.x, a.y}, bv[2] = {b.x, b.y};
#pragma unroll
      for (int k = 0; k < 2; ++k) {
        acc = fmaf(__uint_as_float(av[k] << 16), __uint_as_float(bv[k] << 16), acc);
        acc = fmaf(__uint_as_float(av[k] & 0xffff0000u), __uint_as_float(bv[k] & 0xffff0000u), acc);
      }
    } else {
      const uint32_t a = __ldg(reinterpret_cast<const uint32_t*>(orow));
      const uint32_t b = __ldg(reinterpret_cast<const uint32_t*>(grow));
      acc = fmaf(__uint_as_float(a << 16), __uint_as_float(b << 16), acc);
      acc = fmaf(__uint_as_float(a & 0xffff0000u), __uint_as_float(b & 0xffff0000u), acc);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
    if (lane == 0) {
      const int h = static_cast<int>(r % g.Hh);
      const int64_t rt = r / g.Hh;
      const int t = static_cast<int>(rt % g.T);
      const int rb = static_cast<int>(rt / g.T);
      const int rq = rb / g.B, bv = rb - rq * g.B;
      const int64_t gq = global_pos(g, rq, t);
      const int64_t li = (static_cast<int64_t>(bv % p.lse_B) * p.lse_H + (bv / p.lse_B) * g.Hh + h) * p.lse_S + gq;
      const float l = __ldg(p.lse + li);
      const int64_t wi = (static_cast<int64_t>(rb) * g.Hh + h) * g.T + t;
      p.lse2[wi] = l == -INFINITY ? -INFINITY : -l * kLog2e;
      p.dvec[wi] = acc;
    }
  }
}

// ------------------------------------------------------------------ dK / dV
template <int D>
struct alignas(1024) KvSmem {
  __nv_bfloat16 k[kTile * D];
  __nv_bfloat16 v[kTile * D];
  __nv_bfloat16 q[BwdCfg<D>::kStages][kTile * D];
  __nv_bfloat16 dout[BwdCfg<D>::kStages][kTile * D];
  float lse2[BwdCfg<D>::kStages][kTile];
  float dvec[BwdCfg<D>::kStages][kTile];
  uint64_t kv_full, kv_empty;
  uint64_t qd_full[BwdCfg<D>::kStages], qd_empty[BwdCfg<D>::kStages];
  uint64_t s_full;      // S^T of the current tile is in region A
  uint64_t s_free;      // both warpgroups have read it (256 arrivals)
  uint64_t dp_full;     // dP^T of the current tile is in region A
  uint64_t a_free;      // both warpgroups have read it (256 arrivals)
  uint64_t b_free;      // the products of the previous tile have read region B
  uint64_t p_full[2];   // [warpgroup]: its half of P^T and dS^T is in region B
  uint64_t acc_done;
  uint64_t drain;
  WaitBlock wblk;
  uint32_t tmem_base;
};

template <int D>
struct alignas(1024) QSmem {
  __nv_bfloat16 q[kTile * D];
  __nv_bfloat16 dout[kTile * D];
  __nv_bfloat16 k[BwdCfg<D>::kKStages][kTile * D];
  __nv_bfloat16 v[BwdCfg<D>::kVStages][kTile * D];
  uint64_t q_full, q_empty;
  uint64_t k_full[BwdCfg<D>::kKStages], k_empty[BwdCfg<D>::kKStages];
  uint64_t v_full[BwdCfg<D>::kVStages], v_empty[BwdCfg<D>::kVStages];
  uint64_t s_full;
  uint64_t sdp_free;   // both warpgroups have read S and dP of the current tile
  uint64_t p_full[2];
  uint64_t acc_done;
  uint64_t drain;
  WaitBlock wblk;
  uint32_t tmem_base;
};

static_assert(sizeof(KvSmem<128>) + 1024 <= 232448, "KvSmem<128> exceeds the per-CTA limit");
static_assert(sizeof(KvSmem<64>) + 1024 <= 232448, "KvSmem<64> exceeds the per-CTA limit");
static_assert(sizeof(QSmem<128>) + 1024 <= 232448, "QSmem<128> exceeds the per-CTA limit");
static_assert(sizeof(QSmem<64>) + 1024 <= 232448, "QSmem<64> exceeds the per-CTA limit");

template <int D>
__global__ void __launch_bounds__(kBwdThreads, 1)
    attn_bwd_kv_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                       const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_do,
                       const BwdParams p) {
  using C = BwdCfg<D>;
  extern __shared__ uint8_t smem_raw[];
  KvSmem<D>& sm = *reinterpret_cast<KvSmem<D>*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const Geometry g = p.g;

  if (threadIdx.x == 0) {
    mbar_init(smem_addr(&sm.kv_full), 1);
    mbar_init(smem_addr(&sm.kv_empty), 1);
    for (int s = 0; s < C::kStages; ++s) {
      mbar_init(smem_addr(&sm.qd_full[s]), 1);
      mbar_init(smem_addr(&sm.qd_empty[s]), 1);
    }
    mbar_init(smem_addr(&sm.s_full), 1);
    mbar_init(smem_addr(&sm.s_free), 256);
    mbar_init(smem_addr(&sm.dp_full), 1);
    mbar_init(smem_addr(&sm.a_free), 256);
    mbar_init(smem_addr(&sm.b_free), 1);
    mbar_init(smem_addr(&sm.p_full[0]), 128);
    mbar_init(smem_addr(&sm.p_full[1]), 128);
    mbar_init(smem_addr(&sm.acc_done), 1);
    mbar_init(smem_addr(&sm.drain), 1);
    wait_block_init(sm.wblk, p.status, p.wait_limit_ns);
    fence_barrier_init();
  }
  if (warp == kWarpMma) {
    tmem_alloc(smem_addr(&sm.tmem_base), 512);
    tmem_relinquish();
  }
  if (warp == kWarpTma && lane == 0) {
    prefetch_tensormap(&tm_q);
    prefetch_tensormap(&tm_k);
    prefetch_tensormap(&tm_v);
    prefetch_tensormap(&tm_do);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = sm.tmem_base;
  const WaitCtl ctl = wait_ctl(sm.wblk);
  const int it_end = __ldg(p.cta_begin + blockIdx.x + 1);

  if (warp == kWarpTma) {
    // ------------------------------------------------------------ TMA producer
    const uint64_t pol_kv = l2_policy_evict_first();
    const uint64_t pol_q = l2_policy_evict_last();
    int kv_iter = 0, qd_idx = 0;
    bool ok = true;
    for (int it = __ldg(p.cta_begin + blockIdx.x); it < it_end && ok; ++it) {
      const WorkItem w = p.items[it];
      const int rk = w.rb / g.B, bv = w.rb - rk * g.B;
      const int k0 = w.qp * kTile;
      const int* off = p.walk_off + rk * p.ntiles + w.qp;
      const int e_begin = __ldg(off), e_end = __ldg(off + 1);
      if (kv_iter > 0) ok = mbar_wait(smem_addr(&sm.kv_empty), (kv_iter - 1) & 1, ctl);
      ok = __all_sync(0xffffffffu, ok);
      if (!ok) break;
      mbar_arrive_expect_tx_elect(smem_addr(&sm.kv_full), 2 * C::kTileBytes);
      for (int blk = 0; blk < C::kBlocks; ++blk) {
        tma_load_4d_elect(smem_addr(sm.k) + blk * C::kBlockBytes, &tm_k, smem_addr(&sm.kv_full), blk * 64, w.h, k0,
                          w.rb, pol_kv);
        tma_load_4d_elect(smem_addr(sm.v) + blk * C::kBlockBytes, &tm_v, smem_addr(&sm.kv_full), blk * 64, w.h, k0,
                          w.rb, pol_kv);
      }
      ++kv_iter;
      for (int e = e_begin; e < e_end; ++e) {
        const uint32_t ent = __ldg(p.entries + e);
        const int rbq = entry_rank(ent) * g.B + bv;
        const int q0 = entry_tile(ent) * kTile;
        const int st = qd_idx % C::kStages;
        const int round = qd_idx / C::kStages;
        if (round > 0) ok = mbar_wait(smem_addr(&sm.qd_empty[st]), (round - 1) & 1, ctl);
        ok = __all_sync(0xffffffffu, ok);
        if (!ok) break;
        const uint32_t bar = smem_addr(&sm.qd_full[st]);
        mbar_arrive_expect_tx_elect(bar, 2 * C::kTileBytes + 2 * kTile * 4);
        for (int blk = 0; blk < C::kBlocks; ++blk) {
          tma_load_4d_elect(smem_addr(sm.q[st]) + blk * C::kBlockBytes, &tm_q, bar, blk * 64, w.h, q0, rbq, pol_q);
          tma_load_4d_elect(smem_addr(sm.dout[st]) + blk * C::kBlockBytes, &tm_do, bar, blk * 64, w.h, q0, rbq,
                            pol_q);
        }
        const int64_t vi = (static_cast<int64_t>(rbq) * g.Hh + w.h) * g.T + q0;
        bulk_load_elect(smem_addr(sm.lse2[st]), p.lse2 + vi, kTile * 4, bar);
        bulk_load_elect(smem_addr(sm.dvec[st]), p.dvec + vi, kTile * 4, bar);
        ++qd_idx;
      }
    }
    if (!ok) {
      // Abort: every load issued lands before the CTA exits.
      const uint64_t lim = p.wait_limit_ns;
      for (int idx = qd_idx - C::kStages; idx < qd_idx; ++idx)
        if (idx >= 0) mbar_wait_drain(smem_addr(&sm.qd_full[idx % C::kStages]), (idx / C::kStages) & 1, lim);
      if (kv_iter > 0) mbar_wait_drain(smem_addr(&sm.kv_full), (kv_iter - 1) & 1, lim);
    }
  } else if (warp == kWarpMma) {
    // ------------------------------------------------------------ MMA issuer
    // TMEM: region A [0,128) holds S^T(e) and then dP^T(e) (fp32), region B
    // [128,256) holds P^T(e) at [128,192) and dS^T(e) at [192,256) (bf16), then dV
    // and dK. Per query tile e the tensor core runs S^T(e), dV/dK(e-1), dP^T(e):
    // S^T(e) once region A is free (the warpgroups have read dP^T(e-1)), dP^T(e)
    // once they have read S^T(e), the products of tile e-1 once its P^T and dS^T
    // are in region B; the warpgroups fill region B only after the products of
    // the tile before have read it (b_free).
    const uint32_t tA = tbase, tB = tbase + 128, tdV = tbase + 256, tdK = tbase + 256 + D;
    const uint32_t k_addr = smem_addr(sm.k), v_addr = smem_addr(sm.v);
    int kv_iter = 0, qd_idx = 0, p_cnt = 0, a_cnt = 0, sf_cnt = 0;
    int tiles = 0;   // tiles of this CTA so far (across items)
    bool ok = true, issued = false;
    for (int it = __ldg(p.cta_begin + blockIdx.x); it < it_end && ok; ++it) {
      const WorkItem w = p.items[it];
      const int rk = w.rb / g.B;
      const int* off = p.walk_off + rk * p.ntiles + w.qp;
      const int e_begin = __ldg(off), e_end = __ldg(off + 1);
      ok = mbar_wait(smem_addr(&sm.kv_full), kv_iter & 1, ctl);
      ok = __all_sync(0xffffffffu, ok);
      if (!ok) break;
      ++kv_iter;
      tc_fence_after();
      bool acc = false;
      int prev_st = 0;
      for (int e = e_begin; e < e_end; ++e) {
        const int nt = e - e_begin;
        const int st = qd_idx % C::kStages;
        ok = mbar_wait(smem_addr(&sm.qd_full[st]), (qd_idx / C::kStages) & 1, ctl);
        if (ok && tiles > 0) ok = mbar_wait(smem_addr(&sm.a_free), a_cnt & 1, ctl);
        ok = __all_sync(0xffffffffu, ok);
        if (!ok) break;
        ++qd_idx;
        if (tiles > 0) ++a_cnt;
        ++tiles;
        tc_fence_after();
        const uint32_t q_addr = smem_addr(sm.q[st]), do_addr = smem_addr(sm.dout[st]);
        issue_nt<D>(tA, k_addr, q_addr);   // S^T(e) = K Q^T
        umma_commit_elect(smem_addr(&sm.s_full));
        issued = true;
        if (nt > 0) {
          // Products of tile e-1 (both warpgroups' halves of P^T and dS^T). The
          // first of an item overwrites dV and dK, which the previous item's
          // epilogue read before these halves were stored.
          ok = mbar_wait(smem_addr(&sm.p_full[0]), p_cnt & 1, ctl);
          if (ok) ok = mbar_wait(smem_addr(&sm.p_full[1]), p_cnt & 1, ctl);
          ok = __all_sync(0xffffffffu, ok);
          if (!ok) break;
          ++p_cnt;
          tc_fence_after();
          const uint32_t pq = smem_addr(sm.q[prev_st]), pd = smem_addr(sm.dout[prev_st]);
          issue_dq<D>(tdV, tB, pd, acc);        // dV += P^T(e-1) dO(e-1)
          issue_dq<D>(tdK, tB + 64, pq, acc);   // dK += dS^T(e-1) Q(e-1)
          acc = true;
          umma_commit_elect(smem_addr(&sm.b_free));
          umma_commit_elect(smem_addr(&sm.qd_empty[prev_st]));
        }
        ok = mbar_wait(smem_addr(&sm.s_free), sf_cnt & 1, ctl);
        ok = __all_sync(0xffffffffu, ok);
        if (!ok) break;
        ++sf_cnt;
        tc_fence_after();
        issue_nt<D>(tA, v_addr, do_addr);   // dP^T(e) = V dO^T, over S^T(e) once read
        umma_commit_elect(smem_addr(&sm.dp_full));
        prev_st = st;
      }
      if (!ok) break;
      if (e_end > e_begin) {
        ok = mbar_wait(smem_addr(&sm.p_full[0]), p_cnt & 1, ctl);
        if (ok) ok = mbar_wait(smem_addr(&sm.p_full[1]), p_cnt & 1, ctl);
        ok = __all_sync(0xffffffffu, ok);
        if (!ok) break;
        ++p_cnt;
        tc_fence_after();
        issue_dq<D>(tdV, tB, smem_addr(sm.dout[prev_st]), acc);
        issue_dq<D>(tdK, tB + 64, smem_addr(sm.q[prev_st]), acc);
        umma_commit_elect(smem_addr(&sm.b_free));
        umma_commit_elect(smem_addr(&sm.qd_empty[prev_st]));
        umma_commit_elect(smem_addr(&sm.acc_done));
      }
      umma_commit_elect(smem_addr(&sm.kv_empty));
    }
    if (issued) {
      umma_commit_elect(smem_addr(&sm.drain));
      mbar_wait_drain(smem_addr(&sm.drain), 0, p.wait_limit_ns);
    }
  } else if (warp < 8) {
    // ------------------------------------------------------------ elementwise warpgroups
    const int wg = warp >> 2;
    const int quad = warp & 3;
    const int row = quad * 32 + lane;   // key row of the tile
    const uint32_t lane_off = static_cast<uint32_t>(quad * 32) << 16;
    const uint32_t tA = tbase + lane_off, tB = tA + 128, tdV = tA + 256, tdK = tA + 256 + D;
    const float sl2 = p.scale_log2;
    int s_cnt = 0, d_cnt = 0, b_cnt = 0, acc_cnt = 0, qd_idx = 0;
    int tiles = 0;
    bool ok = true;
    for (int it = __ldg(p.cta_begin + blockIdx.x); it < it_end && ok; ++it) {
      const WorkItem w = p.items[it];
      const int rk = w.rb / g.B;
      const int kl = w.qp * kTile + row;
      const bool valid_k = kl < g.T;
      const int64_t kpos = global_pos(g, rk, valid_k ? kl : g.T - 1);
      const int* off = p.walk_off + rk * p.ntiles + w.qp;
      const int e_begin = __ldg(off), e_end = __ldg(off + 1);
      int ntile = 0;
      for (int e = e_begin; e < e_end; ++e) {
        const uint32_t ent = __ldg(p.entries + e);
        const int st = qd_idx % C::kStages;
        // The stage's lse2 / dvec vectors come by bulk copy: wait for them directly.
        ok = mbar_wait(smem_addr(&sm.qd_full[st]), (qd_idx / C::kStages) & 1, ctl);
        ++qd_idx;
        if (ok) ok = mbar_wait(smem_addr(&sm.s_full), s_cnt & 1, ctl);
        ok = __all_sync(0xffffffffu, ok);
        if (!ok) break;
        ++s_cnt;
        tc_fence_after();
        // Allowed query columns [lo, hi) of this key row.
        int lo = 0, hi = kTile;
        if (entry_c0(ent) == kMasked) {
          const int rq = entry_rank(ent), q0 = entry_tile(ent) * kTile;
          hi = g.T - q0 < kTile ? g.T - q0 : kTile;
          if (g.causal) lo = clamp_int(static_cast<int64_t>(count_le(g, rq, kpos - 1)) - q0, 0, kTile);
          if (!valid_k) lo = hi;
        }
        const float* nl2 = sm.lse2[st];
        const float* dr = sm.dvec[st];
        // Whole tiles take the packed path: no column limits, two columns per
        // f32x2 instruction, the statistics read in pairs. The class is the same
        // for every thread of the CTA (one walk entry per tile), so the branch
        // is uniform; the TMEM stores below are outside it.
        const bool whole = entry_c0(ent) == kFull;
        // P^T of this warpgroup's 64 query columns from S^T, packed to bf16 (the
        // values dV's product uses; dS^T below is formed from the same values).
        uint32_t pk[32];
        {
          uint32_t sa[32], sb[32];
          tmem_ld32x2(tA + wg * 64, tA + wg * 64 + 32, sa, sb);
          tc_fence_before();
          mbar_arrive(smem_addr(&sm.s_free));   // region A may take dP^T
          if (whole) {
            const uint64_t sl2_2 = f2_pack(sl2, sl2);
#pragma unroll
            for (int j = 0; j < 16; ++j) {
              const int c = wg * 64 + 2 * j;
              const uint64_t na = *reinterpret_cast<const uint64_t*>(nl2 + c);
              const uint64_t nb = *reinterpret_cast<const uint64_t*>(nl2 + c + 32);
              float x0, x1, x2, x3;
              f2_unpack(f2_fma(f2_pack(__uint_as_float(sa[2 * j]), __uint_as_float(sa[2 * j + 1])), sl2_2, na), x0, x1);
              f2_unpack(f2_fma(f2_pack(__uint_as_float(sb[2 * j]), __uint_as_float(sb[2 * j + 1])), sl2_2, nb), x2, x3);
              pk[j] = pack_bf16x2(ex2_approx(x0), ex2_approx(x1));
              pk[16 + j] = pack_bf16x2(ex2_approx(x2), ex2_approx(x3));
            }
          } else {
#pragma unroll
            for (int j = 0; j < 16; ++j) {
              const int c = wg * 64 + 2 * j;
              const float p0 = (c >= lo && c < hi) ? ex2_approx(fmaf(__uint_as_float(sa[2 * j]), sl2, nl2[c])) : 0.f;
              const float p1 =
                  (c + 1 >= lo && c + 1 < hi) ? ex2_approx(fmaf(__uint_as_float(sa[2 * j + 1]), sl2, nl2[c + 1])) : 0.f;
              const float p2 =
                  (c + 32 >= lo && c + 32 < hi) ? ex2_approx(fmaf(__uint_as_float(sb[2 * j]), sl2, nl2[c + 32])) : 0.f;
              const float p3 = (c + 33 >= lo && c + 33 < hi)
                                   ? ex2_approx(fmaf(__uint_as_float(sb[2 * j + 1]), sl2, nl2[c + 33]))
                                   : 0.f;
              pk[j] = pack_bf16x2(p0, p1);
              pk[16 + j] = pack_bf16x2(p2, p3);
            }
          }
        }
        ok = mbar_wait(smem_addr(&sm.dp_full), d_cnt & 1, ctl);
        ok = __all_sync(0xffffffffu, ok);
        if (!ok) break;
        ++d_cnt;
        tc_fence_after();
        uint32_t dk[32];
        {
          uint32_t da[32], db[32];
          tmem_ld32x2(tA + wg * 64, tA + wg * 64 + 32, da, db);
          tc_fence_before();
          mbar_arrive(smem_addr(&sm.a_free));   // region A may take the next S^T
          // dS^T = P^T * (dP^T - Dr), two columns per f32x2 instruction (masked
          // columns have P = 0, so the same form serves every tile).
#pragma unroll
          for (int j = 0; j < 16; ++j) {
            const int c = wg * 64 + 2 * j;
            const uint64_t ra = *reinterpret_cast<const uint64_t*>(dr + c);
            const uint64_t rb = *reinterpret_cast<const uint64_t*>(dr + c + 32);
            const uint64_t ga = f2_sub(f2_pack(__uint_as_float(da[2 * j]), __uint_as_float(da[2 * j + 1])), ra);
            const uint64_t gb = f2_sub(f2_pack(__uint_as_float(db[2 * j]), __uint_as_float(db[2 * j + 1])), rb);
            float d0, d1, d2, d3;
            f2_unpack(f2_mul(bf16x2_to_f2(pk[j]), ga), d0, d1);
            f2_unpack(f2_mul(bf16x2_to_f2(pk[16 + j]), gb), d2, d3);
            dk[j] = pack_bf16x2(d0, d1);
            dk[16 + j] = pack_bf16x2(d2, d3);
          }
        }
        // Region B is free once the products of the previous tile have read it.
        if (tiles > 0) {
          ok = mbar_wait(smem_addr(&sm.b_free), b_cnt & 1, ctl);
          ok = __all_sync(0xffffffffu, ok);
          if (!ok) break;
          ++b_cnt;
          tc_fence_after();
        }
        ++tiles;
        tmem_st16(tB + wg * 32, pk);
        tmem_st16(tB + wg * 32 + 16, pk + 16);
        tmem_st16(tB + 64 + wg * 32, dk);
        tmem_st16(tB + 64 + wg * 32 + 16, dk + 16);
        tmem_st_wait();
        tc_fence_before();
        mbar_arrive(smem_addr(&sm.p_full[wg]));
        ++ntile;
      }
      if (!ok) break;
      // ---------------------------------------------------------- epilogue
      if (ntile > 0) {
        ok = mbar_wait(smem_addr(&sm.acc_done), acc_cnt & 1, ctl);
        ok = __all_sync(0xffffffffu, ok);
        if (!ok) break;
        ++acc_cnt;
        tc_fence_after();
      }
      const int64_t orow = ((static_cast<int64_t>(w.rb) * g.T + kl) * g.Hh + w.h) * D;
      if (wg == 0)
        store_row_bf16<D>(tdV, ntile > 0, 1.f, p.out1 + orow, valid_k);
      else
        store_row_bf16<D>(tdK, ntile > 0, p.scale, p.out0 + orow, valid_k);
      tc_fence_before();
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == kWarpMma) {
    tc_fence_after();
    tmem_dealloc(tbase, 512);
  }
}

// ------------------------------------------------------------------ dQ
template <int D>
__global__ void __launch_bounds__(kBwdThreads, 1)
    attn_bwd_q_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                      const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_do,
                      const BwdParams p) {
  using C = BwdCfg<D>;
  extern __shared__ uint8_t smem_raw[];
  QSmem<D>& sm = *reinterpret_cast<QSmem<D>*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const Geometry g = p.g;

  if (threadIdx.x == 0) {
    mbar_init(smem_addr(&sm.q_full), 1);
    mbar_init(smem_addr(&sm.q_empty), 1);
    for (int s = 0; s < C::kKStages; ++s) {
      mbar_init(smem_addr(&sm.k_full[s]), 1);
      mbar_init(smem_addr(&sm.k_empty[s]), 1);
    }
    for (int s = 0; s < C::kVStages; ++s) {
      mbar_init(smem_addr(&sm.v_full[s]), 1);
      mbar_init(smem_addr(&sm.v_empty[s]), 1);
    }
    mbar_init(smem_addr(&sm.s_full), 1);
    mbar_init(smem_addr(&sm.sdp_free), 256);
    mbar_init(smem_addr(&sm.p_full[0]), 128);
    mbar_init(smem_addr(&sm.p_full[1]), 128);
    mbar_init(smem_addr(&sm.acc_done), 1);
    mbar_init(smem_addr(&sm.drain), 1);
    wait_block_init(sm.wblk, p.status, p.wait_limit_ns);
    fence_barrier_init();
  }
  if (warp == kWarpMma) {
    tmem_alloc(smem_addr(&sm.tmem_base), 512);
    tmem_relinquish();
  }
  if (warp == kWarpTma && lane == 0) {
    prefetch_tensormap(&tm_q);
    prefetch_tensormap(&tm_k);
    prefetch_tensormap(&tm_v);
    prefetch_tensormap(&tm_do);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = sm.tmem_base;
  const WaitCtl ctl = wait_ctl(sm.wblk);
  const int it_end = __ldg(p.cta_begin + blockIdx.x + 1);

  if (warp == kWarpTma) {
    // ------------------------------------------------------------ TMA producer
    const uint64_t pol_q = l2_policy_evict_first();
    const uint64_t pol_kv = l2_policy_evict_last();
    int q_iter = 0, k_idx = 0, v_idx = 0;
    bool ok = true;
    for (int it = __ldg(p.cta_begin + blockIdx.x); it < it_end && ok; ++it) {
      const WorkItem w = p.items[it];
      const int rq = w.rb / g.B, bv = w.rb - rq * g.B;
      const int q0 = w.qp * kTile;
      const int* off = p.walk_off + rq * p.ntiles + w.qp;
      const int e_begin = __ldg(off), e_end = __ldg(off + 1);
      if (q_iter > 0) ok = mbar_wait(smem_addr(&sm.q_empty), (q_iter - 1) & 1, ctl);
      ok = __all_sync(0xffffffffu, ok);
      if (!ok) break;
      mbar_arrive_expect_tx_elect(smem_addr(&sm.q_full), 2 * C::kTileBytes);
      for (int blk = 0; blk < C::kBlocks; ++blk) {
        tma_load_4d_elect(smem_addr(sm.q) + blk * C::kBlockBytes, &tm_q, smem_addr(&sm.q_full), blk * 64, w.h, q0,
                          w.rb, pol_q);
        tma_load_4d_elect(smem_addr(sm.dout) + blk * C::kBlockBytes, &tm_do, smem_addr(&sm.q_full), blk * 64, w.h,
                          q0, w.rb, pol_q);
      }
      ++q_iter;
      for (int e = e_begin; e < e_end; ++e) {
        const uint32_t ent = __ldg(p.entries + e);
        const int rbk = entry_rank(ent) * g.B + bv;
        const int k0 = entry_tile(ent) * kTile;
        // K(e) into its ring, then V(e) into its own.
        {
          const int st = k_idx % C::kKStages;
          const int round = k_idx / C::kKStages;
          if (round > 0) ok = mbar_wait(smem_addr(&sm.k_empty[st]), (round - 1) & 1, ctl);
          ok = __all_sync(0xffffffffu, ok);
          if (!ok) break;
          const uint32_t bar = smem_addr(&sm.k_full[st]);
          mbar_arrive_expect_tx_elect(bar, C::kTileBytes);
          for (int blk = 0; blk < C::kBlocks; ++blk)
            tma_load_4d_elect(smem_addr(sm.k[st]) + blk * C::kBlockBytes, &tm_k, bar, blk * 64, w.h, k0, rbk, pol_kv);
          ++k_idx;
        }
        {
          const int st = v_idx % C::kVStages;
          const int round = v_idx / C::kVStages;
          if (round > 0) ok = mbar_wait(smem_addr(&sm.v_empty[st]), (round - 1) & 1, ctl);
          ok = __all_sync(0xffffffffu, ok);
          if (!ok) break;
          const uint32_t bar = smem_addr(&sm.v_full[st]);
          mbar_arrive_expect_tx_elect(bar, C::kTileBytes);
          for (int blk = 0; blk < C::kBlocks; ++blk)
            tma_load_4d_elect(smem_addr(sm.v[st]) + blk * C::kBlockBytes, &tm_v, bar, blk * 64, w.h, k0, rbk, pol_kv);
          ++v_idx;
        }
      }
    }
    if (!ok) {
      // Abort: let every load this thread issued land before the CTA exits.
      const uint64_t lim = p.wait_limit_ns;
      for (int idx = k_idx - C::kKStages; idx < k_idx; ++idx)
        if (idx >= 0) mbar_wait_drain(smem_addr(&sm.k_full[idx % C::kKStages]), (idx / C::kKStages) & 1, lim);
      for (int idx = v_idx - C::kVStages; idx < v_idx; ++idx)
        if (idx >= 0) mbar_wait_drain(smem_addr(&sm.v_full[idx % C::kVStages]), (idx / C::kVStages) & 1, lim);
      if (q_iter > 0) mbar_wait_drain(smem_addr(&sm.q_full), (q_iter - 1) & 1, lim);
    }
  } else if (warp == kWarpMma) {
    // ------------------------------------------------------------ MMA issuer
    // Per key tile e: S(e), dP(e) as soon as the elementwise warps have read
    // S(e-1), dP(e-1) (sdp_free); then dQ += dS(e-1) K(e-1) once dS(e-1) is in
    // its buffer (p_full). dS is double-buffered in TMEM columns [384, 512), so
    // the tensor core computes the next scores while the current dS is formed.
    // V(e)'s stage is released once dP(e) has read it (its commit follows dP),
    // K(e)'s once dQ(e) has.
    const uint32_t tS = tbase, tP2 = tbase + 128, tdQ = tbase + 256, tdS = tbase + 384;
    const uint32_t q_addr = smem_addr(sm.q), do_addr = smem_addr(sm.dout);
    int q_iter = 0, kv_idx = 0, p_cnt = 0, f_cnt = 0;
    int tiles = 0;   // tiles issued by this CTA so far (across items)
    bool ok = true, issued = false;
    for (int it = __ldg(p.cta_begin + blockIdx.x); it < it_end && ok; ++it) {
      const WorkItem w = p.items[it];
      const int rq = w.rb / g.B;
      const int* off = p.walk_off + rq * p.ntiles + w.qp;
      const int e_begin = __ldg(off), e_end = __ldg(off + 1);
      ok = mbar_wait(smem_addr(&sm.q_full), q_iter & 1, ctl);
      ok = __all_sync(0xffffffffu, ok);
      if (!ok) break;
      ++q_iter;
      tc_fence_after();
      bool acc = false;
      int prev_st = 0;
      for (int e = e_begin; e < e_end; ++e) {
        const int nt = e - e_begin;
        const int st = kv_idx % C::kKStages;
        const int vst = kv_idx % C::kVStages;
        ok = mbar_wait(smem_addr(&sm.k_full[st]), (kv_idx / C::kKStages) & 1, ctl);
        if (ok) ok = mbar_wait(smem_addr(&sm.v_full[vst]), (kv_idx / C::kVStages) & 1, ctl);
        // S and dP of the previous tile (of this or the previous item) are read.
        if (ok && tiles > 0) ok = mbar_wait(smem_addr(&sm.sdp_free), f_cnt & 1, ctl);
        ok = __all_sync(0xffffffffu, ok);
        if (!ok) break;
        ++kv_idx;
        if (tiles > 0) ++f_cnt;
        ++tiles;
        tc_fence_after();
        issue_nt<D>(tS, q_addr, smem_addr(sm.k[st]));      // S = Q K^T
        issue_nt<D>(tP2, do_addr, smem_addr(sm.v[vst]));   // dP = dO V^T
        umma_commit_elect(smem_addr(&sm.v_empty[vst]));     // V is read by dP only
        issued = true;
        if (nt > 0) {
          // dS(e-1) of both warpgroups; waited before s_full(e) is committed, so
          // no warpgroup can arrive for tile e while this wait is pending.
          ok = mbar_wait(smem_addr(&sm.p_full[0]), p_cnt & 1, ctl);
          if (ok) ok = mbar_wait(smem_addr(&sm.p_full[1]), p_cnt & 1, ctl);
          ok = __all_sync(0xffffffffu, ok);
          if (!ok) break;
          ++p_cnt;
          tc_fence_after();
          umma_commit_elect(smem_addr(&sm.s_full));
          issue_dq<D>(tdQ, tdS + ((nt - 1) & 1) * 64, smem_addr(sm.k[prev_st]), acc);
          acc = true;
          umma_commit_elect(smem_addr(&sm.k_empty[prev_st]));
        } else {
          umma_commit_elect(smem_addr(&sm.s_full));
        }
        prev_st = st;
      }
      if (!ok) break;
      if (e_end > e_begin) {
        ok = mbar_wait(smem_addr(&sm.p_full[0]), p_cnt & 1, ctl);
        if (ok) ok = mbar_wait(smem_addr(&sm.p_full[1]), p_cnt & 1, ctl);
        ok = __all_sync(0xffffffffu, ok);
        if (!ok) break;
        ++p_cnt;
        tc_fence_after();
        issue_dq<D>(tdQ, tdS + ((e_end - e_begin - 1) & 1) * 64, smem_addr(sm.k[prev_st]), acc);
        umma_commit_elect(smem_addr(&sm.k_empty[prev_st]));
        umma_commit_elect(smem_addr(&sm.acc_done));
      }
      umma_commit_elect(smem_addr(&sm.q_empty));
    }
    if (issued) {
      umma_commit_elect(smem_addr(&sm.drain));
      mbar_wait_drain(smem_addr(&sm.drain), 0, p.wait_limit_ns);
    }
  } else if (warp < 8) {
    // ------------------------------------------------------------ elementwise warpgroups
    const int wg = warp >> 2;
    const int quad = warp & 3;
    const int row = quad * 32 + lane;   // query row of the tile
    const uint32_t lane_off = static_cast<uint32_t>(quad * 32) << 16;
    const uint32_t tS = tbase + lane_off, tP2 = tS + 128, tdQ = tS + 256, tdS = tS + 384;
    const float sl2 = p.scale_log2;
    int s_cnt = 0, acc_cnt = 0;
    bool ok = true;
    for (int it = __ldg(p.cta_begin + blockIdx.x); it < it_end && ok; ++it) {
      const WorkItem w = p.items[it];
      const int rq = w.rb / g.B;
      const int tl = w.qp * kTile + row;
      const bool valid = tl < g.T;
      const int64_t gq = global_pos(g, rq, valid ? tl : g.T - 1);
      const int64_t vi = (static_cast<int64_t>(w.rb) * g.Hh + w.h) * g.T + (valid ? tl : 0);
      const float nlse2 = valid ? __ldg(p.lse2 + vi) : -INFINITY;
      const float drow = valid ? __ldg(p.dvec + vi) : 0.f;
      const int* off = p.walk_off + rq * p.ntiles + w.qp;
      const int e_begin = __ldg(off), e_end = __ldg(off + 1);
      int ntile = 0;
      for (int e = e_begin; e < e_end; ++e) {
        const uint32_t ent = __ldg(p.entries + e);
        ok = mbar_wait(smem_addr(&sm.s_full), s_cnt & 1, ctl);
        ok = __all_sync(0xffffffffu, ok);
        if (!ok) break;
        ++s_cnt;
        tc_fence_after();
        // Allowed key columns [0, lim): keys at or before the query in global
        // position, inside the key rank's T tokens (a prefix, positions grow
        // within a rank).
        int lim = kTile;
        if (entry_c0(ent) == kMasked) lim = valid ? column_limit(g, entry_rank(ent), entry_tile(ent) * kTile, gq) : 0;
        // Read this warpgroup's 64 columns of S and dP, then release them to the
        // next tile's products before computing dS.
        uint32_t sa[2][32], da[2][32];
        tmem_ld32x2(tS + wg * 64, tP2 + wg * 64, sa[0], da[0]);
        tmem_ld32x2(tS + wg * 64 + 32, tP2 + wg * 64 + 32, sa[1], da[1]);
        tc_fence_before();
        mbar_arrive(smem_addr(&sm.sdp_free));
        const uint32_t tbuf = tdS + (ntile & 1) * 64 + wg * 32;
        // Whole tiles (the class is the same for every thread of the CTA, so the
        // branch is uniform) take the packed path: two columns per f32x2
        // instruction, no column limit. The TMEM stores are outside the branch.
        const bool whole = entry_c0(ent) == kFull;
        uint32_t dk[2][16];
        if (whole) {
          const uint64_t sl2_2 = f2_pack(sl2, sl2), nl_2 = f2_pack(nlse2, nlse2), dr_2 = f2_pack(drow, drow);
#pragma unroll
          for (int cc = 0; cc < 2; ++cc)
#pragma unroll
            for (int j = 0; j < 16; ++j) {
              float x0, x1, d0, d1;
              f2_unpack(f2_fma(f2_pack(__uint_as_float(sa[cc][2 * j]), __uint_as_float(sa[cc][2 * j + 1])), sl2_2,
                               nl_2),
                        x0, x1);
              const uint64_t g2 =
                  f2_sub(f2_pack(__uint_as_float(da[cc][2 * j]), __uint_as_float(da[cc][2 * j + 1])), dr_2);
              f2_unpack(f2_mul(f2_pack(ex2_approx(x0), ex2_approx(x1)), g2), d0, d1);
              dk[cc][j] = pack_bf16x2(d0, d1);
            }
        } else {
#pragma unroll
          for (int cc = 0; cc < 2; ++cc) {
            const int col0 = wg * 64 + cc * 32;
#pragma unroll
            for (int j = 0; j < 16; ++j) {
              const int c = col0 + 2 * j;
              const bool a0 = c < lim, a1 = c + 1 < lim;
              const float p0 = a0 ? ex2_approx(fmaf(__uint_as_float(sa[cc][2 * j]), sl2, nlse2)) : 0.f;
              const float p1 = a1 ? ex2_approx(fmaf(__uint_as_float(sa[cc][2 * j + 1]), sl2, nlse2)) : 0.f;
              const float d0 = a0 ? p0 * (__uint_as_float(da[cc][2 * j]) - drow) : 0.f;
              const float d1 = a1 ? p1 * (__uint_as_float(da[cc][2 * j + 1]) - drow) : 0.f;
              dk[cc][j] = pack_bf16x2(d0, d1);
            }
          }
        }
        tmem_st16(tbuf, dk[0]);
        tmem_st16(tbuf + 16, dk[1]);
        tmem_st_wait();
        tc_fence_before();
        mbar_arrive(smem_addr(&sm.p_full[wg]));
        ++ntile;
      }
      if (!ok) break;
      if (ntile > 0) {
        ok = mbar_wait(smem_addr(&sm.acc_done), acc_cnt & 1, ctl);
        ok = __all_sync(0xffffffffu, ok);
        if (!ok) break;
        ++acc_cnt;
        tc_fence_after();
      }
      const int64_t orow = ((static_cast<int64_t>(w.rb) * g.T + tl) * g.Hh + w.h) * D;
      store_row_bf16<D / 2>(tdQ + wg * (D / 2), ntile > 0, p.scale, p.out0 + orow + wg * (D / 2), valid);
      tc_fence_before();
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == kWarpMma) {
    tc_fence_after();
    tmem_dealloc(tbase, 512);
  }
}

template <typename KernelT>
cudaError_t launch_tile_kernel(KernelT kern, size_t smem, const BwdLaunch& L, cudaStream_t stream) {
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  if (L.params.n_cta <= 0) return cudaSuccess;
  kern<<<L.params.n_cta, kBwdThreads, smem, stream>>>(L.tm_q, L.tm_k, L.tm_v, L.tm_do, L.params);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_attn_bwd_pre(const BwdPreParams& p, int D, cudaStream_t stream) {
  const int64_t rows = static_cast<int64_t>(p.g.NR) * p.g.B * p.g.T * p.g.Hh;
  if (rows == 0) return cudaSuccess;
  int dev = 0, sms = 148;
  if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  int64_t blocks = (rows + 7) / 8;
  const int64_t cap = static_cast<int64_t>(sms) * 16;
  if (blocks > cap) blocks = cap;
  if (D == 128)
    bwd_pre_kernel<128><<<static_cast<int>(blocks), 256, 0, stream>>>(p);
  else
    bwd_pre_kernel<64><<<static_cast<int>(blocks), 256, 0, stream>>>(p);
  return cudaGetLastError();
}

cudaError_t launch_attn_bwd_kv(const BwdLaunch& L, int D, cudaStream_t stream) {
  if (D == 128) return launch_tile_kernel(attn_bwd_kv_kernel<128>, sizeof(KvSmem<128>) + 1024, L, stream);
  return launch_tile_kernel(attn_bwd_kv_kernel<64>, sizeof(KvSmem<64>) + 1024, L, stream);
}

cudaError_t launch_attn_bwd_q(const BwdLaunch& L, int D, cudaStream_t stream) {
  if (D == 128) return launch_tile_kernel(attn_bwd_q_kernel<128>, sizeof(QSmem<128>) + 1024, L, stream);
  return launch_tile_kernel(attn_bwd_q_kernel<64>, sizeof(QSmem<64>) + 1024, L, stream);
}

}  // namespace cpattn
