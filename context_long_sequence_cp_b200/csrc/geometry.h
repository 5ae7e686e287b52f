// geometry.h — token positions, tile classes and work items of the context-parallel
// schedule, shared by the host planner and the device kernels.
//
// The ring (page "序列与上下文并行", section "上下文并行：注意力本身切分"): rank r at
// ring step t works on the key/value block of rank (r + t) mod NR. Under causal
// masking a query only sees keys at or before its GLOBAL position (section
// "工程实践"), so a (query tile, key tile) pair is skipped when every key lies
// after every query, computed without a mask when every key lies at or before
// every query, and masked otherwise.
//
// An attention "view" is NR ranks x B batches x T local tokens x Hh heads x D,
// stored [NR][B][T][Hh][D]. Contiguous: rank r's local token l is global r*T + l.
// Zigzag (the reading used for the pages' Z-shaped assignment): the sequence is
// 2*NR chunks of C tokens and rank r holds chunk r then chunk 2*NR-1-r, so local
// l < C is global r*C + l and local l >= C is (2*NR-1-r)*C + (l - C). In both
// cases the global position grows with the local index, which makes every tile's
// positions an increasing run and every mask a per-row column limit.
#pragma once

#include <cstdint>

#if defined(__CUDACC__)
#define CP_HD __host__ __device__ __forceinline__
#else
#define CP_HD inline
#endif

namespace cpattn {

constexpr int kTile = 128;       // query and key tile length (tokens)
constexpr int kPair = 2 * kTile; // a work item covers two consecutive query tiles

enum TileClass : int { kSkip = 0, kFull = 1, kMasked = 2 };

struct Geometry {
  int NR;      // ranks in the ring
  int B;       // batches per rank in the view
  int Hh;      // heads in the view
  int T;       // local tokens per rank
  int C;       // zigzag chunk length (T/2); T for contiguous
  int zigzag;  // 0/1
  int causal;  // 0/1
};

CP_HD int64_t global_pos(const Geometry& g, int rank, int l) {
  if (!g.zigzag) return static_cast<int64_t>(rank) * g.T + l;
  return l < g.C ? static_cast<int64_t>(rank) * g.C + l
                 : static_cast<int64_t>(2 * g.NR - 1 - rank) * g.C + (l - g.C);
}

CP_HD int clamp_int(int64_t x, int lo, int hi) {
  return x < lo ? lo : (x > hi ? hi : static_cast<int>(x));
}

// Number of local tokens of `rank` whose global position is <= p.
CP_HD int count_le(const Geometry& g, int rank, int64_t p) {
  if (!g.zigzag) return clamp_int(p - static_cast<int64_t>(rank) * g.T + 1, 0, g.T);
  const int a = clamp_int(p - static_cast<int64_t>(rank) * g.C + 1, 0, g.C);
  const int b = clamp_int(p - static_cast<int64_t>(2 * g.NR - 1 - rank) * g.C + 1, 0, g.C);
  return a + b;
}

// Class of the pair (query tile of rank rq at local q0, key tile of rank rk at local k0).
CP_HD int classify(const Geometry& g, int rq, int q0, int rk, int k0) {
  const int nq = g.T - q0 < kTile ? g.T - q0 : kTile;
  if (nq <= 0) return kSkip;
  const int nk = g.T - k0 < kTile ? g.T - k0 : kTile;
  if (g.causal) {
    const int64_t gq_max = global_pos(g, rq, q0 + nq - 1);
    const int64_t gk_min = global_pos(g, rk, k0);
    if (gk_min > gq_max) return kSkip;
    const int64_t gq_min = global_pos(g, rq, q0);
    const int64_t gk_max = global_pos(g, rk, k0 + nk - 1);
    return (gk_max <= gq_min && nk == kTile) ? kFull : kMasked;
  }
  return nk == kTile ? kFull : kMasked;
}

// Allowed key columns [0, limit) of a masked tile for a query at global position gq.
CP_HD int column_limit(const Geometry& g, int rk, int k0, int64_t gq) {
  const int nk = g.T - k0 < kTile ? g.T - k0 : kTile;
  if (!g.causal) return nk;
  return clamp_int(static_cast<int64_t>(count_le(g, rk, gq)) - k0, 0, nk);
}

// A work item: two consecutive query tiles [qp*256, qp*256+256) of one (rank, batch, head).
struct WorkItem {
  int rb;    // rank * B + batch (row block of the view)
  int h;     // head in the view
  int qp;    // query-tile pair index
  int cost;  // executed key tiles (both query tiles), used for ordering
};

// Ring launches run one rank's units: a query-tile pair over ring steps
// [t0, t1), packed as qp | t0 << 16 | t1 << 24 (steps < 256); everywhere else
// the high half of qp is zero.
CP_HD int item_qp(const WorkItem& w) { return w.qp & 0xffff; }
CP_HD int unit_t0(const WorkItem& w) { return static_cast<int>((static_cast<unsigned>(w.qp) >> 16) & 0xffu); }
CP_HD int unit_t1(const WorkItem& w) { return static_cast<int>(static_cast<unsigned>(w.qp) >> 24); }
CP_HD int pack_unit(int qp, int t0, int t1) {
  return static_cast<int>(static_cast<unsigned>(qp) | (static_cast<unsigned>(t0) << 16) |
                          (static_cast<unsigned>(t1) << 24));
}

// A precomputed key-tile entry of a work item's walk, packed in 32 bits:
// bits [0,13) key tile index, [13,25) key rank, [25,27) class of query tile 0,
// [27,29) class of query tile 1.
constexpr int kEntryTileBits = 13;
constexpr int kEntryRankBits = 12;
CP_HD uint32_t pack_entry(int rk, int kt, int c0, int c1) {
  return static_cast<uint32_t>(kt) | (static_cast<uint32_t>(rk) << kEntryTileBits) |
         (static_cast<uint32_t>(c0) << 25) | (static_cast<uint32_t>(c1) << 27);
}
CP_HD int entry_tile(uint32_t e) { return static_cast<int>(e & ((1u << kEntryTileBits) - 1)); }
CP_HD int entry_rank(uint32_t e) { return static_cast<int>((e >> kEntryTileBits) & ((1u << kEntryRankBits) - 1)); }
CP_HD int entry_c0(uint32_t e) { return static_cast<int>((e >> 25) & 3u); }
CP_HD int entry_c1(uint32_t e) { return static_cast<int>((e >> 27) & 3u); }

// Walks the key tiles one work item visits, in ring order (t = t_begin..t_end-1,
// key tiles ascending within each step), yielding the classes for both query
// tiles and skipping pairs where both are kSkip. Causal masks make skips
// monotone along a rank's tiles, so the first all-skip tile ends the step.
struct KeyTileWalk {
  Geometry g;
  int rq, qa, qb;      // query rank and the two query tile starts
  int t, t_end, kt, nkt;

  CP_HD void init(const Geometry& geo, int rank_q, int q_first, int t_begin, int t_stop) {
    g = geo;
    rq = rank_q;
    qa = q_first;
    qb = q_first + kTile;
    t = t_begin;
    t_end = t_stop;
    kt = 0;
    nkt = (geo.T + kTile - 1) / kTile;
  }

  // Next executed key tile: its rank, tile index and the two query tiles' classes.
  CP_HD bool next(int& rk, int& ktile, int& c0, int& c1) {
    while (t < t_end) {
      rk = rq + t;
      if (rk >= g.NR) rk -= g.NR;
      while (kt < nkt) {
        const int k0 = kt * kTile;
        c0 = classify(g, rq, qa, rk, k0);
        c1 = classify(g, rq, qb, rk, k0);
        if (c0 == kSkip && c1 == kSkip) break;
        ktile = kt++;
        return true;
      }
      kt = 0;
      ++t;
    }
    return false;
  }
};

}  // namespace cpattn
