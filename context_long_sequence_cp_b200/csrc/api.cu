// api.cu — the C ABI (include/cp_attn.h): plan construction, argument
// validation, TMA descriptor encoding and kernel launches.
#include <cuda.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <mutex>
#include <new>
#include <queue>
#include <utility>
#include <vector>

#include "attn_bwd.h"
#include "attn_fwd.h"
#include "sp_norm.h"
#include "cp_attn.h"
#include "geometry.h"

using namespace cpattn;

constexpr int kDefaultSmCountPlan = 148;   // B200; used when no device is visible

struct cp_attn_plan_s {
  int B, H, S, D, N, causal, layout;
  float scale;
  Geometry g;                       // attention view of the kernel
  int lse_B, lse_H;
  int64_t lse_S;
  std::vector<WorkItem> items;      // sorted work list
  std::vector<int64_t> tile_counts; // executed tile pairs per virtual rank
  WorkItem* d_items = nullptr;      // device copy of the work list
  int* d_status = nullptr;          // device status word
  int device = -1;
  // Precomputed key walks per query-tile pair (rank, qp): entries in ring order
  // and the offset of every ring step (NR + 1 offsets per pair).
  int npairs = 0;
  std::vector<int> step_off;
  std::vector<uint32_t> entries;
  int* d_step_off = nullptr;
  uint32_t* d_entries = nullptr;
  // Static schedule: CTA c runs items [cta_begin[c], cta_begin[c+1]) in order.
  int n_cta = 0;
  std::vector<int> cta_begin;
  std::vector<int64_t> cta_load;    // modelled cost per CTA (key tiles + item overhead)
  int* d_cta_begin = nullptr;
  // Backward schedules (contiguous and zigzag layouts): per key tile the query
  // tiles that see it (dK/dV kernel), per query tile the key tiles it sees (dQ
  // kernel); walks are per (rank, tile), shared by every batch and head.
  struct BwdSched {
    std::vector<WorkItem> items;
    std::vector<int> cta_begin;
    std::vector<int64_t> cta_load;
    std::vector<int> walk_off;        // NR * ntiles + 1
    std::vector<uint32_t> entries;    // pack_entry(other rank, other tile, class, 0)
    int n_cta = 0;
    WorkItem* d_items = nullptr;
    int* d_cta_begin = nullptr;
    int* d_walk_off = nullptr;
    uint32_t* d_entries = nullptr;
  };
  int ntiles = 0;
  BwdSched bwd_kv, bwd_q;
  // Rank-local ring steps (contiguous and zigzag layouts): for one rank and each
  // ring step t, that rank's items ordered and assigned to CTAs by their walk at
  // step t alone. Built for a rank on first use.
  struct RingRank {
    bool built = false;
    int nper = 0;                     // items per step: B * H * query-tile pairs
    std::vector<WorkItem> items;      // [NR][nper], step t's list at t * nper
    std::vector<int> cta_begin;       // [NR][sms + 1], step t's at t * (sms + 1)
    std::vector<int> n_cta;           // [NR]
    std::vector<int64_t> cta_load;    // [NR][sms]
    WorkItem* d_items = nullptr;
    int* d_cta_begin = nullptr;
    // The rank's whole forward as one launch: every (step, item) unit, step-major
    // and longest first within a step, assigned to CTAs in that order.
    std::vector<WorkItem> units;
    std::vector<int> unit_cta_begin;
    std::vector<int64_t> unit_cta_load;
    int unit_n_cta = 0;
    WorkItem* d_units = nullptr;
    int* d_unit_cta_begin = nullptr;
  };
  int sms = kDefaultSmCountPlan;
  std::vector<RingRank> ring;
};

namespace {

constexpr uint64_t kWaitLimitNs = 2000000000ull;   // 2 s per in-kernel wait
constexpr int64_t kPullChunkBytes = 32768;          // fused-pull copy unit
constexpr int kDefaultSmCount = kDefaultSmCountPlan;

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// 4-D view (D, Hh, T, NR*B) of a bf16 tensor stored [NR*B][T][Hh][D]; box of
// 64 x 1 x 128 x 1 elements (128 B x 128 rows) with the 128-byte swizzle.
// A rank-local buffer holds B row blocks only (row_blocks = B).
int encode_view(CUtensorMap* map, const void* base, const Geometry& g, int D, int64_t row_blocks = -1) {
  EncodeTiledFn fn = encode_fn();
  if (fn == nullptr) return CP_ERR_CUDA;
  if (row_blocks < 0) row_blocks = static_cast<int64_t>(g.NR) * g.B;
  const cuuint64_t dims[4] = {static_cast<cuuint64_t>(D), static_cast<cuuint64_t>(g.Hh),
                              static_cast<cuuint64_t>(g.T), static_cast<cuuint64_t>(row_blocks)};
  const cuuint64_t strides[3] = {static_cast<cuuint64_t>(D) * 2, static_cast<cuuint64_t>(g.Hh) * D * 2,
                                 static_cast<cuuint64_t>(g.T) * g.Hh * D * 2};
  const cuuint32_t box[4] = {64, 1, static_cast<cuuint32_t>(kTile), 1};
  const cuuint32_t estr[4] = {1, 1, 1, 1};
  CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(base), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? CP_OK : CP_ERR_CUDA;
}

// Executed key tiles of a work item (both query tiles) over ring steps [t0, t1).
void item_cost(const Geometry& g, int rq, int qp, int t0, int t1, int* c0n, int* c1n) {
  KeyTileWalk w;
  w.init(g, rq, qp * kPair, t0, t1);
  int rk, kt, c0, c1;
  *c0n = *c1n = 0;
  while (w.next(rk, kt, c0, c1)) {
    *c0n += c0 != kSkip;
    *c1n += c1 != kSkip;
  }
}

// Modelled cost of an item in executed key tiles: the tiles of its walk plus a
// fixed overhead for loading its query tiles, the first score product and the
// output write, measured at about one and a half key tiles.
constexpr int64_t kItemOverheadHalfTiles = 3;

// Assigns the sorted work list to n_cta persistent CTAs: each item, in list
// order, goes to the CTA whose modelled finish time is the earliest (ties to the
// lower index). Items therefore start in about list order (so that the items
// running together still share keys and values in L2) while the CTAs finish
// together. The list is reordered so that each CTA's items are contiguous.
// Assigns a sorted work list to n_cta persistent CTAs: each item, in list order,
// goes to the CTA whose modelled finish time is the earliest (ties to the lower
// index). Items therefore start in about list order (so that the items running
// together still share their operands in L2) while the CTAs finish together.
// The list is reordered so that each CTA's items are contiguous.
int assign_greedy(std::vector<WorkItem>& items, const std::vector<int64_t>& cost, int n_cta,
                  std::vector<int>& cta_begin, std::vector<int64_t>& cta_load) {
  const int n = static_cast<int>(items.size());
  n_cta = n < n_cta ? n : n_cta;
  cta_load.assign(n_cta, 0);
  std::vector<int> owner(n);
  using Slot = std::pair<int64_t, int>;
  std::priority_queue<Slot, std::vector<Slot>, std::greater<Slot>> free_at;
  for (int c = 0; c < n_cta; ++c) free_at.push(Slot(0, c));
  for (int i = 0; i < n; ++i) {
    const Slot s = free_at.top();
    free_at.pop();
    owner[i] = s.second;
    cta_load[s.second] = s.first + cost[i];
    free_at.push(Slot(s.first + cost[i], s.second));
  }
  std::vector<WorkItem> sorted;
  sorted.reserve(n);
  cta_begin.assign(n_cta + 1, 0);
  for (int c = 0; c < n_cta; ++c) {
    cta_begin[c] = static_cast<int>(sorted.size());
    for (int i = 0; i < n; ++i)
      if (owner[i] == c) sorted.push_back(items[i]);
  }
  cta_begin[n_cta] = n;
  items.swap(sorted);
  return n_cta;
}

// Assigns the items (already in the grouped order: items that share keys/values
// next to each other) twice: in that order and longest-first over the whole list.
// The grouped assignment is kept unless longest-first lowers the modelled finish
// time of the last CTA by more than 2%: grouping keeps the K/V of the items that
// run together shared in L2, which only balance on few items per CTA (short
// sequences, whose K/V fits in L2 anyway) should override.
template <class CostOf>
int assign_balanced(std::vector<WorkItem>& items, CostOf cost_of, int n_cta, std::vector<int>& cta_begin,
                    std::vector<int64_t>& cta_load) {
  const int n = static_cast<int>(items.size());
  std::vector<WorkItem> lpt = items;
  std::vector<int64_t> cost(n), cost_lpt(n);
  for (int i = 0; i < n; ++i) cost[i] = cost_of(items[i]);
  std::vector<int> order(n);
  for (int i = 0; i < n; ++i) order[i] = i;
  std::stable_sort(order.begin(), order.end(), [&](int a, int b) { return cost[a] > cost[b]; });
  for (int i = 0; i < n; ++i) {
    lpt[i] = items[order[i]];
    cost_lpt[i] = cost[order[i]];
  }
  std::vector<int> begin_lpt;
  std::vector<int64_t> load_lpt;
  const int n_grouped = assign_greedy(items, cost, n_cta, cta_begin, cta_load);
  const int n_lpt = assign_greedy(lpt, cost_lpt, n_cta, begin_lpt, load_lpt);
  int64_t max_grouped = 0, max_lpt = 0;
  for (int64_t l : cta_load) max_grouped = l > max_grouped ? l : max_grouped;
  for (int64_t l : load_lpt) max_lpt = l > max_lpt ? l : max_lpt;
  if (max_lpt * 100 < max_grouped * 98) {
    items.swap(lpt);
    cta_begin.swap(begin_lpt);
    cta_load.swap(load_lpt);
    return n_lpt;
  }
  return n_grouped;
}

void schedule_items(cp_attn_plan_s* p, int n_cta) {
  auto cost_of = [p](const WorkItem& w) {
    const int rq = w.rb / p->g.B;
    const int* off = p->step_off.data() + static_cast<size_t>(rq * p->npairs + w.qp) * (p->g.NR + 1);
    return 2 * static_cast<int64_t>(off[p->g.NR] - off[0]) + kItemOverheadHalfTiles;
  };
  p->n_cta = assign_balanced(p->items, cost_of, n_cta, p->cta_begin, p->cta_load);
}

// Walks and schedules of the two backward kernels. A walk entry's class is
// kFull when every (row, column) pair of the tile pair is allowed and both tiles
// are whole; otherwise kMasked (the kernels then bound the allowed columns).
void build_bwd(cp_attn_plan_s* p, int n_cta) {
  const Geometry& g = p->g;
  const int nt = (g.T + kTile - 1) / kTile;
  p->ntiles = nt;
  for (int kind = 0; kind < 2; ++kind) {   // 0: dK/dV (per key tile), 1: dQ (per query tile)
    cp_attn_plan_s::BwdSched& b = kind == 0 ? p->bwd_kv : p->bwd_q;
    b.walk_off.assign(static_cast<size_t>(g.NR) * nt + 1, 0);
    b.entries.clear();
    for (int r = 0; r < g.NR; ++r) {
      for (int tile = 0; tile < nt; ++tile) {
        b.walk_off[static_cast<size_t>(r) * nt + tile] = static_cast<int>(b.entries.size());
        for (int t = 0; t < g.NR; ++t) {
          // dK/dV: the query ranks whose ring step t reaches key rank r; dQ: the
          // key rank of step t of query rank r.
          const int other = kind == 0 ? (r - t + g.NR) % g.NR : (r + t) % g.NR;
          for (int ot = 0; ot < nt; ++ot) {
            const int rq = kind == 0 ? other : r, qt = kind == 0 ? ot : tile;
            const int rk = kind == 0 ? r : other, kt = kind == 0 ? tile : ot;
            int c = classify(g, rq, qt * kTile, rk, kt * kTile);
            if (c == kSkip) continue;
            if (c == kFull && g.T - qt * kTile < kTile) c = kMasked;   // ragged query tile
            b.entries.push_back(pack_entry(other, ot, c, 0));
          }
        }
      }
    }
    b.walk_off[static_cast<size_t>(g.NR) * nt] = static_cast<int>(b.entries.size());
    b.items.clear();
    for (int r = 0; r < g.NR; ++r)
      for (int bb = 0; bb < g.B; ++bb)
        for (int tile = 0; tile < nt; ++tile) {
          const int len = b.walk_off[static_cast<size_t>(r) * nt + tile + 1] - b.walk_off[static_cast<size_t>(r) * nt + tile];
          for (int h = 0; h < g.Hh; ++h) b.items.push_back(WorkItem{r * g.B + bb, h, tile, len});
        }
    std::stable_sort(b.items.begin(), b.items.end(), [&](const WorkItem& x, const WorkItem& y) {
      const int bx = x.rb % g.B, by = y.rb % g.B;
      if (bx != by) return bx < by;
      if (x.h / 2 != y.h / 2) return x.h / 2 < y.h / 2;
      return x.cost > y.cost;
    });
    auto cost_of = [](const WorkItem& w) { return 2 * static_cast<int64_t>(w.cost) + kItemOverheadHalfTiles; };
    b.n_cta = assign_balanced(b.items, cost_of, n_cta, b.cta_begin, b.cta_load);
  }
}

bool upload_bwd(cp_attn_plan_s::BwdSched& b) {
  const size_t ib = b.items.size() * sizeof(WorkItem), cb = b.cta_begin.size() * sizeof(int);
  const size_t wb = b.walk_off.size() * sizeof(int), eb = b.entries.size() * sizeof(uint32_t);
  return cudaMalloc(&b.d_items, ib > 0 ? ib : sizeof(WorkItem)) == cudaSuccess &&
         cudaMalloc(&b.d_cta_begin, cb) == cudaSuccess && cudaMalloc(&b.d_walk_off, wb) == cudaSuccess &&
         cudaMalloc(&b.d_entries, eb > 0 ? eb : sizeof(uint32_t)) == cudaSuccess &&
         (ib == 0 || cudaMemcpy(b.d_items, b.items.data(), ib, cudaMemcpyHostToDevice) == cudaSuccess) &&
         cudaMemcpy(b.d_cta_begin, b.cta_begin.data(), cb, cudaMemcpyHostToDevice) == cudaSuccess &&
         cudaMemcpy(b.d_walk_off, b.walk_off.data(), wb, cudaMemcpyHostToDevice) == cudaSuccess &&
         (eb == 0 || cudaMemcpy(b.d_entries, b.entries.data(), eb, cudaMemcpyHostToDevice) == cudaSuccess);
}

void free_bwd(cp_attn_plan_s::BwdSched& b) {
  if (b.d_items != nullptr) cudaFree(b.d_items);
  if (b.d_cta_begin != nullptr) cudaFree(b.d_cta_begin);
  if (b.d_walk_off != nullptr) cudaFree(b.d_walk_off);
  if (b.d_entries != nullptr) cudaFree(b.d_entries);
  b.d_items = nullptr;
  b.d_cta_begin = nullptr;
  b.d_walk_off = nullptr;
  b.d_entries = nullptr;
}

int ensure_device(cp_attn_plan_s* p) {
  if (p->d_items != nullptr) return CP_OK;
  return CP_ERR_CUDA;
}

// First step of the tail phase of a one-launch ring forward: half the steps run
// one unit per step, the rest in one unit per query-tile pair.
int ring_split(int nr) { return nr <= 2 ? nr : (nr + 1) / 2; }

// Schedules of one rank's ring steps: at step t the rank's items (every batch,
// head and query-tile pair) carry the key tiles of their walk at step t, and are
// assigned to CTAs by the whole-view list's greedy rule, longest first.
void build_ring_rank(cp_attn_plan_s* p, int r) {
  cp_attn_plan_s::RingRank& rr = p->ring[r];
  const Geometry& g = p->g;
  const int stride = p->sms + 1;
  rr.nper = g.B * g.Hh * p->npairs;
  rr.items.clear();
  rr.items.reserve(static_cast<size_t>(g.NR) * rr.nper);
  rr.cta_begin.assign(static_cast<size_t>(g.NR) * stride, 0);
  rr.cta_load.assign(static_cast<size_t>(g.NR) * p->sms, 0);
  rr.n_cta.assign(g.NR, 0);
  for (int t = 0; t < g.NR; ++t) {
    std::vector<WorkItem> items;
    items.reserve(rr.nper);
    for (int b = 0; b < g.B; ++b)
      for (int qp = 0; qp < p->npairs; ++qp) {
        const int* off = p->step_off.data() + static_cast<size_t>(r * p->npairs + qp) * (g.NR + 1);
        const int len = off[t + 1] - off[t];
        for (int h = 0; h < g.Hh; ++h) items.push_back(WorkItem{r * g.B + b, h, qp, len});
      }
    // Longest first: one step has few items per CTA (about 3.5 on 32 heads of
    // 32k tokens over 8 ranks), and one rank's key/value block stays in L2
    // whatever the order, so the order serves the balance alone.
    std::stable_sort(items.begin(), items.end(), [](const WorkItem& a, const WorkItem& b) { return a.cost > b.cost; });
    std::vector<int64_t> cost(items.size());
    for (size_t i = 0; i < items.size(); ++i) cost[i] = 2 * static_cast<int64_t>(items[i].cost) + kItemOverheadHalfTiles;
    std::vector<int> cb;
    std::vector<int64_t> load;
    rr.n_cta[t] = assign_greedy(items, cost, p->sms, cb, load);
    std::copy(cb.begin(), cb.end(), rr.cta_begin.begin() + static_cast<size_t>(t) * stride);
    std::copy(load.begin(), load.end(), rr.cta_load.begin() + static_cast<size_t>(t) * p->sms);
    rr.items.insert(rr.items.end(), items.begin(), items.end());
  }
  // One launch over all steps, in two phases. Steps [0, split) run as one unit
  // per (step, pair), step-major, while the later blocks are still arriving;
  // then each pair walks steps [split, NR) in one unit, its softmax state kept
  // on chip as in the fused kernel. split + 1 partials (NR when split = NR - 1).
  rr.units.clear();
  rr.unit_cta_begin.assign(1, 0);
  rr.unit_cta_load.clear();
  rr.unit_n_cta = 0;
  if (g.NR > 255) {   // unit steps are packed in 8 bits: no one-launch schedule
    rr.built = true;
    return;
  }
  const int split = ring_split(g.NR);
  struct U {
    WorkItem w;
    int64_t cost;
    int phase;   // the step for the first phase, split for the tail
  };
  std::vector<U> us;
  us.reserve(static_cast<size_t>(rr.nper) * (split + 1));
  for (int b = 0; b < g.B; ++b)
    for (int qp = 0; qp < p->npairs; ++qp) {
      const int* off = p->step_off.data() + static_cast<size_t>(r * p->npairs + qp) * (g.NR + 1);
      for (int h = 0; h < g.Hh; ++h) {
        for (int t = 0; t < split; ++t) {
          const int len = off[t + 1] - off[t];
          us.push_back(U{WorkItem{r * g.B + b, h, pack_unit(qp, t, t + 1), len},
                         2 * static_cast<int64_t>(len) + kItemOverheadHalfTiles, t});
        }
        if (split < g.NR) {
          const int len = off[g.NR] - off[split];
          us.push_back(U{WorkItem{r * g.B + b, h, pack_unit(qp, split, g.NR), len},
                         2 * static_cast<int64_t>(len) + kItemOverheadHalfTiles, split});
        }
      }
    }
  std::stable_sort(us.begin(), us.end(), [](const U& x, const U& y) {
    if (x.phase != y.phase) return x.phase < y.phase;
    return x.cost > y.cost;
  });
  rr.units.clear();
  std::vector<int64_t> ucost;
  for (const U& u : us) {
    rr.units.push_back(u.w);
    ucost.push_back(u.cost);
  }
  rr.unit_n_cta = assign_greedy(rr.units, ucost, p->sms, rr.unit_cta_begin, rr.unit_cta_load);
  rr.built = true;
}

void free_ring(cp_attn_plan_s::RingRank& rr) {
  for (void* ptr : {static_cast<void*>(rr.d_items), static_cast<void*>(rr.d_cta_begin),
                    static_cast<void*>(rr.d_units), static_cast<void*>(rr.d_unit_cta_begin)})
    if (ptr != nullptr) cudaFree(ptr);
  rr.d_items = nullptr;
  rr.d_cta_begin = nullptr;
  rr.d_units = nullptr;
  rr.d_unit_cta_begin = nullptr;
}

int upload_ring_rank(cp_attn_plan_s::RingRank& rr) {
  if (rr.d_items != nullptr) return CP_OK;
  const size_t ib = rr.items.size() * sizeof(WorkItem), cb = rr.cta_begin.size() * sizeof(int);
  const size_t ub = (rr.units.empty() ? 1 : rr.units.size()) * sizeof(WorkItem);
  const size_t ucb = rr.unit_cta_begin.size() * sizeof(int);
  const bool ok = cudaMalloc(&rr.d_items, ib) == cudaSuccess && cudaMalloc(&rr.d_cta_begin, cb) == cudaSuccess &&
                  cudaMalloc(&rr.d_units, ub) == cudaSuccess && cudaMalloc(&rr.d_unit_cta_begin, ucb) == cudaSuccess &&
                  cudaMemcpy(rr.d_items, rr.items.data(), ib, cudaMemcpyHostToDevice) == cudaSuccess &&
                  cudaMemcpy(rr.d_cta_begin, rr.cta_begin.data(), cb, cudaMemcpyHostToDevice) == cudaSuccess &&
                  (rr.units.empty() ||
                   cudaMemcpy(rr.d_units, rr.units.data(), ub, cudaMemcpyHostToDevice) == cudaSuccess) &&
                  cudaMemcpy(rr.d_unit_cta_begin, rr.unit_cta_begin.data(), ucb, cudaMemcpyHostToDevice) ==
                      cudaSuccess;
  if (!ok) {
    free_ring(rr);
    return CP_ERR_CUDA;
  }
  return CP_OK;
}

int launch_view(cp_attn_plan_s* p, const Geometry& g, const void* q, const void* k, const void* v, void* o,
                float* lse, float* o_part, float* lse_part, int t0, int t1, bool partial, cudaStream_t st) {
  FwdLaunch L;
  std::memset(&L, 0, sizeof(L));
  int rc;
  if ((rc = encode_view(&L.tm_q, q, g, p->D)) != CP_OK) return rc;
  if ((rc = encode_view(&L.tm_k, k, g, p->D)) != CP_OK) return rc;
  if ((rc = encode_view(&L.tm_v, v, g, p->D)) != CP_OK) return rc;
  FwdParams& P = L.params;
  P.g = g;
  P.t_begin = t0;
  P.t_end = t1;
  P.scale_log2 = p->scale * 1.4426950408889634f;
  P.items = p->d_items;
  P.n_items = static_cast<int>(p->items.size());
  P.cta_begin = p->d_cta_begin;
  P.n_cta = p->n_cta;
  P.step_off = p->d_step_off;
  P.entries = p->d_entries;
  P.npairs = p->npairs;
  P.o = static_cast<__nv_bfloat16*>(o);
  P.lse = lse;
  P.lse_B = p->lse_B;
  P.lse_H = p->lse_H;
  P.lse_S = p->lse_S;
  P.o_part = o_part;
  P.lse_part = lse_part;
  P.status = p->d_status;
  P.wait_limit_ns = kWaitLimitNs;
  return launch_attn_fwd(L, p->D, partial, st) == cudaSuccess ? CP_OK : CP_ERR_CUDA;
}

PermuteArgs permute_args(const cp_attn_plan_s* p, int direction, int elem_bytes) {
  PermuteArgs a;
  a.kind = p->layout == CP_LAYOUT_ULYSSES ? 1 : 0;
  a.direction = direction;
  a.N = p->N;
  a.B = p->B;
  a.S = p->S;
  a.H = p->H;
  a.D = p->D;
  a.zigzag = p->layout == CP_LAYOUT_ZIGZAG;
  a.elem_bytes = elem_bytes;
  return a;
}

}  // namespace

extern "C" {

int cp_attn_plan(cp_attn_plan_t* out, int B, int H, int S, int D, int N, int causal, int layout,
                 float softmax_scale) {
  if (out == nullptr) return CP_ERR_INVALID_ARG;
  *out = nullptr;
  if (B <= 0 || H <= 0 || S <= 0 || N <= 0) return CP_ERR_INVALID_ARG;
  if (causal != 0 && causal != 1) return CP_ERR_INVALID_ARG;
  if (layout < CP_LAYOUT_CONTIGUOUS || layout > CP_LAYOUT_ULYSSES) return CP_ERR_INVALID_ARG;
  if (!(softmax_scale <= 0.f || std::isfinite(softmax_scale))) return CP_ERR_INVALID_ARG;
  if (D != 64 && D != 128) return CP_ERR_UNSUPPORTED;
  if (S % N != 0) return CP_ERR_UNSUPPORTED;
  if (layout == CP_LAYOUT_ZIGZAG && S % (2 * N) != 0) return CP_ERR_UNSUPPORTED;
  if (layout == CP_LAYOUT_ULYSSES && (H % N != 0 || causal)) return CP_ERR_UNSUPPORTED;
  // int32 indexing limits of the kernels: tokens per view, view row blocks, TMA dims.
  if (static_cast<int64_t>(B) * N > (1 << 20) || static_cast<int64_t>(B) * S * H * D > (int64_t(1) << 40))
    return CP_ERR_UNSUPPORTED;
  // Packed walk entries: key rank < 2^12, key tile index < 2^13.
  if (N >= (1 << kEntryRankBits) || (static_cast<int64_t>(S) + kTile - 1) / kTile >= (1 << kEntryTileBits))
    return CP_ERR_UNSUPPORTED;

  cp_attn_plan_s* p = new (std::nothrow) cp_attn_plan_s();
  if (p == nullptr) return CP_ERR_INVALID_ARG;
  p->B = B;
  p->H = H;
  p->S = S;
  p->D = D;
  p->N = N;
  p->causal = causal;
  p->layout = layout;
  p->scale = softmax_scale > 0.f ? softmax_scale : 1.0f / std::sqrt(static_cast<float>(D));
  p->lse_B = B;
  p->lse_H = H;
  p->lse_S = S;
  Geometry& g = p->g;
  if (layout == CP_LAYOUT_ULYSSES) {
    g = Geometry{1, N * B, H / N, S, S, 0, 0};
  } else {
    g = Geometry{N, B, H, S / N, layout == CP_LAYOUT_ZIGZAG ? S / (2 * N) : S / N, layout == CP_LAYOUT_ZIGZAG,
                 causal};
  }

  // Key walks: for every (rank, query-tile pair), the executed key tiles in ring
  // order with both query tiles' classes, and where each ring step starts.
  const int npairs = (g.T + kPair - 1) / kPair;
  p->npairs = npairs;
  p->step_off.reserve(static_cast<size_t>(g.NR) * npairs * (g.NR + 1));
  for (int r = 0; r < g.NR; ++r) {
    for (int qp = 0; qp < npairs; ++qp) {
      for (int t = 0; t < g.NR; ++t) {
        p->step_off.push_back(static_cast<int>(p->entries.size()));
        KeyTileWalk w;
        w.init(g, r, qp * kPair, t, t + 1);
        int rk, kt, c0, c1;
        while (w.next(rk, kt, c0, c1)) p->entries.push_back(pack_entry(rk, kt, c0, c1));
      }
      p->step_off.push_back(static_cast<int>(p->entries.size()));
    }
  }
  if (p->entries.size() >= (size_t(1) << 31)) {
    delete p;
    return CP_ERR_UNSUPPORTED;
  }

  // Work list: every (rank, batch, head, query-tile pair) with its executed key tiles.
  p->tile_counts.assign(N, 0);
  p->items.reserve(static_cast<size_t>(g.NR) * g.B * g.Hh * npairs);
  for (int r = 0; r < g.NR; ++r) {
    for (int b = 0; b < g.B; ++b) {
      for (int qp = 0; qp < npairs; ++qp) {
        int c0, c1;
        item_cost(g, r, qp, 0, g.NR, &c0, &c1);   // same for every head
        for (int h = 0; h < g.Hh; ++h) {
          p->items.push_back(WorkItem{r * g.B + b, h, qp, c0 + c1});
          const int rank = layout == CP_LAYOUT_ULYSSES ? b / B : r;
          p->tile_counts[rank] += c0 + c1;
        }
      }
    }
  }
  // Items that read the same keys/values (same batch, heads in pairs) are kept
  // together so that the ones running at the same time share them in L2; within
  // a group the most expensive come first. Pairs of heads (rather than single
  // heads) give the schedule below enough large items late in the list to end
  // level (modelled max/mean CTA load 1.005 instead of 1.024 on 32 heads).
  std::stable_sort(p->items.begin(), p->items.end(), [&](const WorkItem& a, const WorkItem& b) {
    const int ba = a.rb % g.B, bb = b.rb % g.B;
    if (ba != bb) return ba < bb;
    if (a.h / 2 != b.h / 2) return a.h / 2 < b.h / 2;
    return a.cost > b.cost;
  });

  int ndev = 0;
  const bool have_device = cudaGetDeviceCount(&ndev) == cudaSuccess && ndev > 0;
  int sms = kDefaultSmCount;
  if (have_device) {
    cudaGetDevice(&p->device);
    if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, p->device) != cudaSuccess || sms <= 0)
      sms = kDefaultSmCount;
  }
  p->sms = sms;
  p->ring.resize(layout == CP_LAYOUT_ULYSSES ? 0 : g.NR);
  schedule_items(p, sms);
  if (layout != CP_LAYOUT_ULYSSES) build_bwd(p, sms);
  if (have_device) {
    const size_t bytes = p->items.size() * sizeof(WorkItem);
    const size_t off_bytes = p->step_off.size() * sizeof(int);
    const size_t ent_bytes = p->entries.size() * sizeof(uint32_t);
    const size_t cta_bytes = p->cta_begin.size() * sizeof(int);
    bool ok = cudaMalloc(&p->d_items, bytes > 0 ? bytes : sizeof(WorkItem)) == cudaSuccess &&
              cudaMalloc(&p->d_cta_begin, cta_bytes) == cudaSuccess &&
              cudaMemcpy(p->d_cta_begin, p->cta_begin.data(), cta_bytes, cudaMemcpyHostToDevice) == cudaSuccess &&
              cudaMalloc(&p->d_status, sizeof(int)) == cudaSuccess &&
              cudaMalloc(&p->d_step_off, off_bytes) == cudaSuccess &&
              cudaMalloc(&p->d_entries, ent_bytes > 0 ? ent_bytes : sizeof(uint32_t)) == cudaSuccess &&
              cudaMemcpy(p->d_items, p->items.data(), bytes, cudaMemcpyHostToDevice) == cudaSuccess &&
              cudaMemcpy(p->d_step_off, p->step_off.data(), off_bytes, cudaMemcpyHostToDevice) == cudaSuccess &&
              (ent_bytes == 0 ||
               cudaMemcpy(p->d_entries, p->entries.data(), ent_bytes, cudaMemcpyHostToDevice) == cudaSuccess) &&
              cudaMemset(p->d_status, 0, sizeof(int)) == cudaSuccess &&
              (layout == CP_LAYOUT_ULYSSES || (upload_bwd(p->bwd_kv) && upload_bwd(p->bwd_q)));
    if (!ok) {
      free_bwd(p->bwd_kv);
      free_bwd(p->bwd_q);
      cudaFree(p->d_items);
      cudaFree(p->d_cta_begin);
      p->d_cta_begin = nullptr;
      cudaFree(p->d_status);
      cudaFree(p->d_step_off);
      cudaFree(p->d_entries);
      p->d_items = nullptr;
      p->d_status = nullptr;
      p->d_step_off = nullptr;
      p->d_entries = nullptr;
    }
  } else {
    cudaGetLastError();   // clear the "no device" error
  }
  *out = p;
  return CP_OK;
}

int cp_attn_plan_destroy(cp_attn_plan_t plan) {
  if (plan == nullptr) return CP_OK;
  if (plan->d_items != nullptr) cudaFree(plan->d_items);
  if (plan->d_cta_begin != nullptr) cudaFree(plan->d_cta_begin);
  free_bwd(plan->bwd_kv);
  free_bwd(plan->bwd_q);
  for (auto& rr : plan->ring) free_ring(rr);
  if (plan->d_status != nullptr) cudaFree(plan->d_status);
  if (plan->d_step_off != nullptr) cudaFree(plan->d_step_off);
  if (plan->d_entries != nullptr) cudaFree(plan->d_entries);
  delete plan;
  return CP_OK;
}

int64_t cp_attn_plan_tile_counts(cp_attn_plan_t plan, int64_t* per_rank) {
  if (plan == nullptr) return CP_ERR_INVALID_ARG;
  int64_t tot = 0;
  for (int r = 0; r < plan->N; ++r) {
    if (per_rank != nullptr) per_rank[r] = plan->tile_counts[r];
    tot += plan->tile_counts[r];
  }
  return tot;
}

int64_t cp_attn_plan_num_items(cp_attn_plan_t plan) {
  if (plan == nullptr) return CP_ERR_INVALID_ARG;
  return static_cast<int64_t>(plan->items.size());
}

size_t cp_attn_bwd_workspace_bytes(cp_attn_plan_t plan) {
  if (plan == nullptr || plan->layout == CP_LAYOUT_ULYSSES) return 0;
  const int64_t rows = static_cast<int64_t>(plan->g.NR) * plan->g.B * plan->g.T * plan->g.Hh;
  return static_cast<size_t>(2 * rows * 4 + 1024);   // lse2 and dvec, plus bulk-copy over-read padding
}

int64_t cp_attn_plan_bwd_pairs(cp_attn_plan_t plan, int64_t* kv_pairs, int64_t* q_pairs) {
  if (plan == nullptr) return CP_ERR_INVALID_ARG;
  if (plan->layout == CP_LAYOUT_ULYSSES) return CP_ERR_UNSUPPORTED;
  if (kv_pairs != nullptr) *kv_pairs = static_cast<int64_t>(plan->bwd_kv.entries.size());
  if (q_pairs != nullptr) *q_pairs = static_cast<int64_t>(plan->bwd_q.entries.size());
  return static_cast<int64_t>(plan->bwd_q.entries.size());
}

int cp_attn_bwd(cp_attn_plan_t plan, const void* q, const void* k, const void* v, const void* o, const float* lse,
                const void* dout, void* dq, void* dk, void* dv, void* workspace, cp_stream_t stream) {
  if (plan == nullptr || q == nullptr || k == nullptr || v == nullptr || o == nullptr || lse == nullptr ||
      dout == nullptr || dq == nullptr || dk == nullptr || dv == nullptr || workspace == nullptr)
    return CP_ERR_INVALID_ARG;
  if (plan->layout == CP_LAYOUT_ULYSSES) return CP_ERR_UNSUPPORTED;
  if (plan->g.T % 4 != 0) return CP_ERR_UNSUPPORTED;   // 16-byte rows of the per-row statistics
  const void* ptrs[11] = {q, k, v, o, lse, dout, dq, dk, dv, workspace, nullptr};
  for (int i = 0; i < 10; ++i)
    if (!aligned16(ptrs[i])) return CP_ERR_ALIGNMENT;
  if (plan->d_items == nullptr || plan->bwd_kv.d_items == nullptr) return CP_ERR_CUDA;
  const Geometry& g = plan->g;
  const int64_t rows = static_cast<int64_t>(g.NR) * g.B * g.T * g.Hh;
  float* lse2 = static_cast<float*>(workspace);
  float* dvec = lse2 + rows;
  cudaStream_t st = static_cast<cudaStream_t>(stream);

  BwdPreParams pre;
  pre.g = g;
  pre.o = static_cast<const __nv_bfloat16*>(o);
  pre.dout = static_cast<const __nv_bfloat16*>(dout);
  pre.lse = lse;
  pre.lse_B = plan->lse_B;
  pre.lse_H = plan->lse_H;
  pre.lse_S = plan->lse_S;
  pre.lse2 = lse2;
  pre.dvec = dvec;
  if (launch_attn_bwd_pre(pre, plan->D, st) != cudaSuccess) return CP_ERR_CUDA;

  BwdLaunch L;
  std::memset(&L, 0, sizeof(L));
  int rc;
  if ((rc = encode_view(&L.tm_q, q, g, plan->D)) != CP_OK) return rc;
  if ((rc = encode_view(&L.tm_k, k, g, plan->D)) != CP_OK) return rc;
  if ((rc = encode_view(&L.tm_v, v, g, plan->D)) != CP_OK) return rc;
  if ((rc = encode_view(&L.tm_do, dout, g, plan->D)) != CP_OK) return rc;
  BwdParams& P = L.params;
  P.g = g;
  P.scale = plan->scale;
  P.scale_log2 = plan->scale * 1.4426950408889634f;
  P.ntiles = plan->ntiles;
  P.lse2 = lse2;
  P.dvec = dvec;
  P.status = plan->d_status;
  P.wait_limit_ns = kWaitLimitNs;
  P.items = plan->bwd_kv.d_items;
  P.cta_begin = plan->bwd_kv.d_cta_begin;
  P.n_cta = plan->bwd_kv.n_cta;
  P.walk_off = plan->bwd_kv.d_walk_off;
  P.entries = plan->bwd_kv.d_entries;
  P.out0 = static_cast<__nv_bfloat16*>(dk);
  P.out1 = static_cast<__nv_bfloat16*>(dv);
  if (launch_attn_bwd_kv(L, plan->D, st) != cudaSuccess) return CP_ERR_CUDA;
  P.items = plan->bwd_q.d_items;
  P.cta_begin = plan->bwd_q.d_cta_begin;
  P.n_cta = plan->bwd_q.n_cta;
  P.walk_off = plan->bwd_q.d_walk_off;
  P.entries = plan->bwd_q.d_entries;
  P.out0 = static_cast<__nv_bfloat16*>(dq);
  P.out1 = nullptr;
  if (launch_attn_bwd_q(L, plan->D, st) != cudaSuccess) return CP_ERR_CUDA;
  return CP_OK;
}

int64_t cp_attn_plan_cta_loads(cp_attn_plan_t plan, int64_t* per_cta) {
  if (plan == nullptr) return CP_ERR_INVALID_ARG;
  if (per_cta != nullptr)
    for (int c = 0; c < plan->n_cta; ++c) per_cta[c] = plan->cta_load[c];
  return plan->n_cta;
}

size_t cp_attn_workspace_bytes(cp_attn_plan_t plan, int with_partials) {
  if (plan == nullptr) return 0;
  if (plan->layout == CP_LAYOUT_ULYSSES && !with_partials)
    return 4 * static_cast<size_t>(plan->B) * plan->S * plan->H * plan->D * 2;
  return 0;
}

int cp_attn_fwd(cp_attn_plan_t plan, const void* q, const void* k, const void* v, void* o, float* lse,
                void* workspace, cp_stream_t stream) {
  if (plan == nullptr || q == nullptr || k == nullptr || v == nullptr || o == nullptr) return CP_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned16(lse) ||
      !aligned16(workspace))
    return CP_ERR_ALIGNMENT;
  int rc = ensure_device(plan);
  if (rc != CP_OK) return rc;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (plan->layout != CP_LAYOUT_ULYSSES)
    return launch_view(plan, plan->g, q, k, v, o, lse, nullptr, nullptr, 0, plan->g.NR, false, st);

  if (workspace == nullptr) return CP_ERR_WORKSPACE;
  const size_t tensor = static_cast<size_t>(plan->B) * plan->S * plan->H * plan->D * 2;
  char* ws = static_cast<char*>(workspace);
  void* gq = ws;
  void* gk = ws + tensor;
  void* gv = ws + 2 * tensor;
  void* go = ws + 3 * tensor;
  const PermuteArgs fwd = permute_args(plan, 0, 2);
  if (launch_permute(fwd, q, gq, st) != cudaSuccess || launch_permute(fwd, k, gk, st) != cudaSuccess ||
      launch_permute(fwd, v, gv, st) != cudaSuccess)
    return CP_ERR_CUDA;
  rc = launch_view(plan, plan->g, gq, gk, gv, go, lse, nullptr, nullptr, 0, 1, false, st);
  if (rc != CP_OK) return rc;
  return launch_permute(permute_args(plan, 1, 2), go, o, st) == cudaSuccess ? CP_OK : CP_ERR_CUDA;
}

int cp_attn_fwd_partials(cp_attn_plan_t plan, const void* q, const void* k, const void* v, float* o_parts,
                         float* lse_parts, void* workspace, cp_stream_t stream) {
  (void)workspace;
  if (plan == nullptr || q == nullptr || k == nullptr || v == nullptr || o_parts == nullptr ||
      lse_parts == nullptr)
    return CP_ERR_INVALID_ARG;
  if (plan->layout == CP_LAYOUT_ULYSSES) return CP_ERR_UNSUPPORTED;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o_parts) || !aligned16(lse_parts))
    return CP_ERR_ALIGNMENT;
  int rc = ensure_device(plan);
  if (rc != CP_OK) return rc;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const int64_t rows = static_cast<int64_t>(plan->B) * plan->S * plan->H;
  for (int t = 0; t < plan->N; ++t) {
    rc = launch_view(plan, plan->g, q, k, v, nullptr, nullptr, o_parts + t * rows * plan->D, lse_parts + t * rows,
                     t, t + 1, true, st);
    if (rc != CP_OK) return rc;
  }
  return CP_OK;
}

int cp_attn_ring_prepare(cp_attn_plan_t plan, int rank) {
  if (plan == nullptr) return CP_ERR_INVALID_ARG;
  if (plan->layout == CP_LAYOUT_ULYSSES) return CP_ERR_UNSUPPORTED;
  if (rank < 0 || rank >= plan->N) return CP_ERR_INVALID_ARG;
  cp_attn_plan_s::RingRank& rr = plan->ring[rank];
  if (!rr.built) build_ring_rank(plan, rank);
  if (plan->d_items == nullptr) return CP_OK;   // no device: host schedules only
  return upload_ring_rank(rr);
}

int cp_attn_ring_num_parts(cp_attn_plan_t plan) {
  if (plan == nullptr) return CP_ERR_INVALID_ARG;
  if (plan->layout == CP_LAYOUT_ULYSSES) return CP_ERR_UNSUPPORTED;
  const int split = ring_split(plan->N);
  return split < plan->N ? split + 1 : plan->N;
}

int64_t cp_attn_ring_schedule(cp_attn_plan_t plan, int rank, int step, int32_t* items, int64_t* cta_loads) {
  if (plan == nullptr) return CP_ERR_INVALID_ARG;
  if (plan->layout == CP_LAYOUT_ULYSSES) return CP_ERR_UNSUPPORTED;
  if (rank < 0 || rank >= plan->N || step < -1 || step >= plan->N) return CP_ERR_INVALID_ARG;
  cp_attn_plan_s::RingRank& rr = plan->ring[rank];
  if (!rr.built) build_ring_rank(plan, rank);
  if (step == -1) {   // the one-launch schedule of cp_attn_fwd_ring
    const int n_cta = rr.unit_n_cta;
    if (items != nullptr)
      for (int c = 0; c < n_cta; ++c)
        for (int i = rr.unit_cta_begin[c]; i < rr.unit_cta_begin[c + 1]; ++i) {
          int32_t* o = items + static_cast<size_t>(i) * 5;
          o[0] = rr.units[i].rb;
          o[1] = rr.units[i].h;
          o[2] = rr.units[i].qp;
          o[3] = rr.units[i].cost;
          o[4] = c;
        }
    if (cta_loads != nullptr)
      for (int c = 0; c < n_cta; ++c) cta_loads[c] = rr.unit_cta_load[c];
    return static_cast<int64_t>(rr.units.size());
  }
  const int stride = plan->sms + 1;
  const int* cb = rr.cta_begin.data() + static_cast<size_t>(step) * stride;
  const WorkItem* it = rr.items.data() + static_cast<size_t>(step) * rr.nper;
  const int n_cta = rr.n_cta[step];
  if (items != nullptr)
    for (int c = 0; c < n_cta; ++c)
      for (int i = cb[c]; i < cb[c + 1]; ++i) {
        int32_t* o = items + static_cast<size_t>(i) * 5;
        o[0] = it[i].rb;
        o[1] = it[i].h;
        o[2] = it[i].qp;
        o[3] = it[i].cost;
        o[4] = c;
      }
  if (cta_loads != nullptr)
    for (int c = 0; c < n_cta; ++c) cta_loads[c] = rr.cta_load[static_cast<size_t>(step) * plan->sms + c];
  return rr.nper;
}

int cp_attn_fwd_ring_step(cp_attn_plan_t plan, int rank, int step, const void* q, const void* k, const void* v,
                          float* o_part, float* lse_part, cp_stream_t stream) {
  if (plan == nullptr || q == nullptr || k == nullptr || v == nullptr || o_part == nullptr || lse_part == nullptr)
    return CP_ERR_INVALID_ARG;
  if (plan->layout == CP_LAYOUT_ULYSSES) return CP_ERR_UNSUPPORTED;
  if (rank < 0 || rank >= plan->N || step < 0 || step >= plan->N) return CP_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o_part) || !aligned16(lse_part))
    return CP_ERR_ALIGNMENT;
  int rc = ensure_device(plan);
  if (rc != CP_OK) return rc;
  if ((rc = cp_attn_ring_prepare(plan, rank)) != CP_OK) return rc;
  const cp_attn_plan_s::RingRank& rr = plan->ring[rank];
  const Geometry& g = plan->g;
  FwdLaunch L;
  std::memset(&L, 0, sizeof(L));
  if ((rc = encode_view(&L.tm_q, q, g, plan->D, g.B)) != CP_OK) return rc;
  if ((rc = encode_view(&L.tm_k, k, g, plan->D, g.B)) != CP_OK) return rc;
  if ((rc = encode_view(&L.tm_v, v, g, plan->D, g.B)) != CP_OK) return rc;
  FwdParams& P = L.params;
  P.g = g;
  P.t_begin = step;
  P.t_end = step + 1;
  P.scale_log2 = plan->scale * 1.4426950408889634f;
  P.items = rr.d_items + static_cast<size_t>(step) * rr.nper;
  P.n_items = rr.nper;
  P.cta_begin = rr.d_cta_begin + static_cast<size_t>(step) * (plan->sms + 1);
  P.n_cta = rr.n_cta[step];
  P.step_off = plan->d_step_off;
  P.entries = plan->d_entries;
  P.npairs = plan->npairs;
  P.o_part = o_part;
  P.lse_part = lse_part;
  P.q_rb0 = rank * g.B;
  P.kv_local = 1;
  P.status = plan->d_status;
  P.wait_limit_ns = kWaitLimitNs;
  return launch_attn_fwd(L, plan->D, true, static_cast<cudaStream_t>(stream)) == cudaSuccess ? CP_OK : CP_ERR_CUDA;
}

}  // extern "C"

namespace {

// One rank's whole ring forward in one launch. Three arrival modes: pulling (the
// kernel's copy warps fetch the other blocks and count their chunks in arrived),
// external (arrived[j] >= 1 is set by the caller's own transfer) and resident
// (arrived NULL: every slot already holds its block, no wait).
int ring_launch(cp_attn_plan_t plan, int rank, const void* q, void* k_all, void* v_all, const void* const* pull_k,
                const void* const* pull_v, int* arrived, bool external, float* o_parts, float* lse_parts,
                cp_stream_t stream) {
  if (plan == nullptr || q == nullptr || k_all == nullptr || v_all == nullptr || o_parts == nullptr ||
      lse_parts == nullptr)
    return CP_ERR_INVALID_ARG;
  if (plan->layout == CP_LAYOUT_ULYSSES) return CP_ERR_UNSUPPORTED;
  if (rank < 0 || rank >= plan->N) return CP_ERR_INVALID_ARG;
  if ((pull_k == nullptr) != (pull_v == nullptr)) return CP_ERR_INVALID_ARG;
  const bool pull = pull_k != nullptr && plan->N > 1;
  if (pull && arrived == nullptr) return CP_ERR_INVALID_ARG;
  // Without pull sources a wait on arrived counts is only made on request: a
  // stale arrived buffer passed by mistake would otherwise stall every unit
  // until its wait runs out.
  if (!pull && !external && arrived != nullptr) return CP_ERR_INVALID_ARG;
  if (external && arrived == nullptr) return CP_ERR_INVALID_ARG;
  if (pull && plan->N > kMaxPullRanks) return CP_ERR_UNSUPPORTED;
  if (plan->N > 255) return CP_ERR_UNSUPPORTED;   // unit steps are packed in 8 bits
  if (!aligned16(q) || !aligned16(k_all) || !aligned16(v_all) || !aligned16(o_parts) || !aligned16(lse_parts) ||
      (reinterpret_cast<uintptr_t>(arrived) & 3u))
    return CP_ERR_ALIGNMENT;
  const Geometry& g = plan->g;
  FwdLaunch L;
  std::memset(&L, 0, sizeof(L));
  FwdParams& P = L.params;
  const int64_t block_bytes = static_cast<int64_t>(g.B) * g.T * g.Hh * plan->D * 2;
  if (pull) {
    for (int j = 0; j < plan->N; ++j) {
      if (j == rank) continue;
      if (pull_k[j] == nullptr || pull_v[j] == nullptr) return CP_ERR_INVALID_ARG;
      if (!aligned16(pull_k[j]) || !aligned16(pull_v[j])) return CP_ERR_ALIGNMENT;
      P.pull_src[2 * j] = reinterpret_cast<uint64_t>(pull_k[j]);
      P.pull_src[2 * j + 1] = reinterpret_cast<uint64_t>(pull_v[j]);
    }
    const int64_t chunk = block_bytes < kPullChunkBytes ? block_bytes : kPullChunkBytes;
    const int64_t per_half = (block_bytes + chunk - 1) / chunk;
    if (2 * per_half > (int64_t(1) << 30)) return CP_ERR_UNSUPPORTED;
    P.pull_k_all = static_cast<char*>(k_all);
    P.pull_v_all = static_cast<char*>(v_all);
    P.pull_block_bytes = block_bytes;
    P.pull_chunk_bytes = static_cast<int>(chunk);
    P.pull_chunks = static_cast<int>(2 * per_half);
  }
  int rc = ensure_device(plan);
  if (rc != CP_OK) return rc;
  if ((rc = cp_attn_ring_prepare(plan, rank)) != CP_OK) return rc;
  const cp_attn_plan_s::RingRank& rr = plan->ring[rank];
  if ((rc = encode_view(&L.tm_q, q, g, plan->D, g.B)) != CP_OK) return rc;
  if ((rc = encode_view(&L.tm_k, k_all, g, plan->D)) != CP_OK) return rc;
  if ((rc = encode_view(&L.tm_v, v_all, g, plan->D)) != CP_OK) return rc;
  P.g = g;
  P.t_begin = 0;
  P.t_end = g.NR;
  P.scale_log2 = plan->scale * 1.4426950408889634f;
  P.items = rr.d_units;
  P.n_items = static_cast<int>(rr.units.size());
  P.cta_begin = rr.d_unit_cta_begin;
  P.n_cta = rr.unit_n_cta;
  P.step_off = plan->d_step_off;
  P.entries = plan->d_entries;
  P.npairs = plan->npairs;
  P.o_part = o_parts;
  P.lse_part = lse_parts;
  P.q_rb0 = rank * g.B;
  P.kv_local = 0;
  P.unit_steps = 1;
  P.unit_split = ring_split(g.NR);
  P.part_rows = static_cast<int64_t>(g.B) * g.T * g.Hh;
  P.arrived = arrived;
  P.arrive_target = pull ? P.pull_chunks : 1;
  P.status = plan->d_status;
  P.wait_limit_ns = kWaitLimitNs;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (pull && cudaMemsetAsync(arrived, 0, sizeof(int) * plan->N, st) != cudaSuccess) return CP_ERR_CUDA;
  return launch_attn_fwd(L, plan->D, true, st) == cudaSuccess ? CP_OK : CP_ERR_CUDA;
}

}  // namespace

extern "C" {

int cp_attn_fwd_ring(cp_attn_plan_t plan, int rank, const void* q, void* k_all, void* v_all,
                     const void* const* pull_k, const void* const* pull_v, int* arrived, float* o_parts,
                     float* lse_parts, cp_stream_t stream) {
  return ring_launch(plan, rank, q, k_all, v_all, pull_k, pull_v, arrived, false, o_parts, lse_parts, stream);
}

int cp_attn_fwd_ring_external(cp_attn_plan_t plan, int rank, const void* q, void* k_all, void* v_all,
                              int* arrived, float* o_parts, float* lse_parts, cp_stream_t stream) {
  return ring_launch(plan, rank, q, k_all, v_all, nullptr, nullptr, arrived, true, o_parts, lse_parts, stream);
}

int cp_merge_partials(int num_parts, int64_t rows, int D, const float* o_parts, const float* lse_parts,
                      void* o_out, float* lse_out, cp_stream_t stream) {
  if (num_parts < 1 || num_parts > 64 || rows < 0) return CP_ERR_INVALID_ARG;
  if (D != 64 && D != 128) return CP_ERR_UNSUPPORTED;
  if (rows > 0 && (o_parts == nullptr || lse_parts == nullptr || o_out == nullptr)) return CP_ERR_INVALID_ARG;
  if (!aligned16(o_parts) || !aligned16(o_out) || (reinterpret_cast<uintptr_t>(lse_parts) & 3u) ||
      (reinterpret_cast<uintptr_t>(lse_out) & 3u))
    return CP_ERR_ALIGNMENT;
  return launch_merge(num_parts, rows, D, o_parts, lse_parts, static_cast<__nv_bfloat16*>(o_out), lse_out,
                      static_cast<cudaStream_t>(stream)) == cudaSuccess
             ? CP_OK
             : CP_ERR_CUDA;
}

int cp_layout_permute(cp_attn_plan_t plan, int direction, const void* in, void* out, int elem_bytes,
                      cp_stream_t stream) {
  if (plan == nullptr || in == nullptr || out == nullptr) return CP_ERR_INVALID_ARG;
  if (direction != 0 && direction != 1) return CP_ERR_INVALID_ARG;
  if (elem_bytes != 2 && elem_bytes != 4) return CP_ERR_INVALID_ARG;
  if (!aligned16(in) || !aligned16(out)) return CP_ERR_ALIGNMENT;
  const PermuteArgs a = permute_args(plan, direction, elem_bytes);
  const int64_t unit_elems =
      a.kind == 0 ? static_cast<int64_t>(plan->H) * plan->D : static_cast<int64_t>(plan->H / plan->N) * plan->D;
  if ((unit_elems * elem_bytes) % 16 != 0) return CP_ERR_UNSUPPORTED;
  int ndev = 0;
  if (cudaGetDeviceCount(&ndev) != cudaSuccess || ndev == 0) return CP_ERR_CUDA;
  return launch_permute(a, in, out, static_cast<cudaStream_t>(stream)) == cudaSuccess ? CP_OK : CP_ERR_CUDA;
}

int cp_rope_permute(cp_attn_plan_t plan, const void* in, void* out, double base, int64_t pos_offset,
                    cp_stream_t stream) {
  if (plan == nullptr || in == nullptr || out == nullptr) return CP_ERR_INVALID_ARG;
  if (!(base > 1.0) || !std::isfinite(base)) return CP_ERR_INVALID_ARG;
  if (pos_offset < 0 || pos_offset > (int64_t(1) << 31) - plan->S) return CP_ERR_INVALID_ARG;
  if (!aligned16(in) || !aligned16(out)) return CP_ERR_ALIGNMENT;
  if (plan->D % 8 != 0 || plan->D > 128 || 256 % plan->D != 0) return CP_ERR_UNSUPPORTED;
  int ndev = 0;
  if (cudaGetDeviceCount(&ndev) != cudaSuccess || ndev == 0) return CP_ERR_CUDA;
  RopeArgs ra;
  std::memset(&ra, 0, sizeof(ra));
  for (int i = 0; i < plan->D / 2; ++i) ra.theta[i] = std::pow(base, -2.0 * i / plan->D);
  ra.pos_offset = pos_offset;
  ra.D = plan->D;
  return launch_rope_permute(permute_args(plan, 0, 2), ra, in, out, static_cast<cudaStream_t>(stream)) == cudaSuccess
             ? CP_OK
             : CP_ERR_CUDA;
}

int cp_sp_rs_dropout_add_ln(const void* partials, int nparts, int64_t rows, int H, const uint32_t* keep_bits,
                            float p, const void* residual, const float* gamma, const float* beta, float eps,
                            void* z_out, void* y_out, cp_stream_t stream) {
  if (partials == nullptr || nparts < 1 || rows < 0) return CP_ERR_INVALID_ARG;
  if (H < 8 || H > 8192 || H % 8 != 0) return CP_ERR_UNSUPPORTED;
  if (keep_bits != nullptr && !(p >= 0.f && p < 1.f)) return CP_ERR_INVALID_ARG;
  if ((gamma == nullptr) != (beta == nullptr)) return CP_ERR_INVALID_ARG;
  if (y_out != nullptr && gamma == nullptr) return CP_ERR_INVALID_ARG;
  if (z_out == nullptr && y_out == nullptr) return CP_ERR_INVALID_ARG;
  if (y_out != nullptr && !(eps > 0.f)) return CP_ERR_INVALID_ARG;
  if (!aligned16(partials) || (residual != nullptr && !aligned16(residual)) || (gamma != nullptr && !aligned16(gamma)) ||
      (beta != nullptr && !aligned16(beta)) || (z_out != nullptr && !aligned16(z_out)) ||
      (y_out != nullptr && !aligned16(y_out)) ||
      (keep_bits != nullptr && (reinterpret_cast<uintptr_t>(keep_bits) & 3u) != 0))
    return CP_ERR_ALIGNMENT;
  int ndev = 0;
  if (cudaGetDeviceCount(&ndev) != cudaSuccess || ndev == 0) return CP_ERR_CUDA;
  SpArgs a;
  a.partials = static_cast<const __nv_bfloat16*>(partials);
  a.nparts = nparts;
  a.part_stride = rows * H;
  a.keep = keep_bits;
  a.inv_keep = keep_bits != nullptr ? 1.f / (1.f - p) : 1.f;
  a.residual = static_cast<const __nv_bfloat16*>(residual);
  a.gamma = gamma;
  a.beta = beta;
  a.eps = eps;
  a.z = static_cast<__nv_bfloat16*>(z_out);
  a.y = static_cast<__nv_bfloat16*>(y_out);
  a.rows = rows;
  a.H = H;
  return launch_sp_rs_dropout_add_ln(a, static_cast<cudaStream_t>(stream)) == cudaSuccess ? CP_OK : CP_ERR_CUDA;
}

int64_t cp_layout_index_map_len(cp_attn_plan_t plan) {
  if (plan == nullptr) return CP_ERR_INVALID_ARG;
  return plan->layout == CP_LAYOUT_ULYSSES ? static_cast<int64_t>(plan->N) * plan->B * plan->S
                                           : static_cast<int64_t>(plan->B) * plan->S;
}

int cp_layout_index_map(cp_attn_plan_t plan, int64_t* map_out, cp_stream_t stream) {
  if (plan == nullptr || map_out == nullptr) return CP_ERR_INVALID_ARG;
  if (!aligned16(map_out)) return CP_ERR_ALIGNMENT;
  int ndev = 0;
  if (cudaGetDeviceCount(&ndev) != cudaSuccess || ndev == 0) return CP_ERR_CUDA;
  return launch_index_map(permute_args(plan, 0, 2), map_out, static_cast<cudaStream_t>(stream)) == cudaSuccess
             ? CP_OK
             : CP_ERR_CUDA;
}

int cp_attn_check(cp_attn_plan_t plan, cp_stream_t stream) {
  if (plan == nullptr) return CP_ERR_INVALID_ARG;
  if (plan->d_status == nullptr) return CP_ERR_CUDA;
  if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess) return CP_ERR_CUDA;
  int status = 0;
  if (cudaMemcpy(&status, plan->d_status, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess) return CP_ERR_CUDA;
  if (status != 0) {
    cudaMemset(plan->d_status, 0, sizeof(int));
    return status;
  }
  return cudaGetLastError() == cudaSuccess ? CP_OK : CP_ERR_CUDA;
}

const char* cp_status_string(int status) {
  switch (status) {
    case CP_OK: return "ok";
    case CP_ERR_INVALID_ARG: return "invalid argument";
    case CP_ERR_UNSUPPORTED: return "unsupported shape or layout";
    case CP_ERR_ALIGNMENT: return "device pointer not 16-byte aligned";
    case CP_ERR_CUDA: return "CUDA error or no device";
    case CP_ERR_TIMEOUT: return "in-kernel wait timed out";
    case CP_ERR_WORKSPACE: return "workspace missing or too small";
    default: return "unknown status";
  }
}

int cp_debug_wait_timeout_probe(cp_attn_plan_t plan, int timeout_us, cp_stream_t stream) {
  if (plan == nullptr || timeout_us < 1 || timeout_us > 1000000) return CP_ERR_INVALID_ARG;
  if (plan->d_status == nullptr) return CP_ERR_CUDA;
  return launch_wait_probe(plan->d_status, static_cast<uint64_t>(timeout_us) * 1000ull,
                           static_cast<cudaStream_t>(stream)) == cudaSuccess
             ? CP_OK
             : CP_ERR_CUDA;
}

}  // extern "C"

// The device a plan was made on (-1 without a device).
int cp_internal_plan_device(const cp_attn_plan_s* plan) { return plan == nullptr ? -1 : plan->device; }

// Ulysses forward on a caller-chosen scratch buffer: the same launches as the
// Ulysses branch of cp_attn_fwd, with the head-group copies placed in `scratch`.
int cp_internal_ulysses_fwd_scratch(cp_attn_plan_s* plan, const void* q, const void* k, const void* v, void* o,
                                    float* lse, void* scratch, size_t scratch_bytes, cudaStream_t st) {
  if (plan == nullptr || q == nullptr || k == nullptr || v == nullptr || o == nullptr) return CP_ERR_INVALID_ARG;
  if (plan->layout != CP_LAYOUT_ULYSSES) return CP_ERR_UNSUPPORTED;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned16(lse) || !aligned16(scratch))
    return CP_ERR_ALIGNMENT;
  const size_t tensor = static_cast<size_t>(plan->B) * plan->S * plan->H * plan->D * 2;
  if (scratch == nullptr || scratch_bytes < 4 * tensor) return CP_ERR_WORKSPACE;
  int rc = ensure_device(plan);
  if (rc != CP_OK) return rc;
  char* ws = static_cast<char*>(scratch);
  void* gq = ws;
  void* gk = ws + tensor;
  void* gv = ws + 2 * tensor;
  void* go = ws + 3 * tensor;
  const PermuteArgs fwd = permute_args(plan, 0, 2);
  if (launch_permute(fwd, q, gq, st) != cudaSuccess || launch_permute(fwd, k, gk, st) != cudaSuccess ||
      launch_permute(fwd, v, gv, st) != cudaSuccess)
    return CP_ERR_CUDA;
  rc = launch_view(plan, plan->g, gq, gk, gv, go, lse, nullptr, nullptr, 0, 1, false, st);
  if (rc != CP_OK) return rc;
  return launch_permute(permute_args(plan, 1, 2), go, o, st) == cudaSuccess ? CP_OK : CP_ERR_CUDA;
}
