// vkv_chunk_attn: argument checks, work schedule, TMA descriptors, launch.
#include <algorithm>
#include <cmath>
#include <cstdlib>
#include <cstring>
#include <deque>
#include <functional>
#include <map>
#include <memory>
#include <mutex>
#include <queue>
#include <string>
#include <vector>

#include "vkv_attn_kernel.cuh"

static_assert(sizeof(vkv::AttnParams) <= 32764, "kernel parameter space");

namespace vkv {

namespace {

// ---------------------------------------------------------------------------
// schedule: units of one or two 128-row query tiles, balanced over the SMs
// ---------------------------------------------------------------------------
struct Plan {
  int n_ctas = 0;
  std::vector<int> cta_begin;
  std::vector<uint32_t> units;
  // key-axis pieces (empty when no unit is split)
  std::vector<int> cta_piece0;
  std::vector<uint2> pieces;
  int n_slots = 0;
  // the split units, for the combine kernel: unit code, first slot | piece count << 16
  std::vector<uint32_t> split_code, split_slots;
};

struct Cand {
  uint32_t code;
  double cost;
};

// Time of a one-tile unit relative to a two-tile unit over the same keys.  A
// lone tile cannot hide its softmax behind another tile's MMAs, so it costs
// almost as much as a pair (measured on B200: 0.9 balances the dense, ragged
// and block-sparse schedules best; VKV_SINGLE_COST overrides it).
double single_tile_cost() {
  static double c = [] {
    const char* e = std::getenv("VKV_SINGLE_COST");
    double v = e ? std::atof(e) : 0.0;
    return (v > 0.05 && v <= 1.0) ? v : 0.9;
  }();
  return c;
}

// One-tile units of the block-sparse kernel that selects for itself: their key
// steps alternate between the two softmax warpgroups (VKV_KX=0 turns this off;
// the other instantiations keep lone tiles on one warpgroup, whose code this
// would slow down by a few per cent), so that a lone tile overlaps
// two softmax passes as a pair does.  Such a unit costs kx_rate() of its steps
// plus the fixed cost of a unit, above one half because each of its K/V tiles
// feeds one query tile instead of two, so its loads run twice as fast per
// product and its ring holds half as many steps (measured on B200: 0.65
// balances K = 9 to 144 best; VKV_KX_RATE overrides it).
bool kx_enabled() {
  static bool on = [] {
    const char* e = std::getenv("VKV_KX");
    return !(e && e[0] == '0');
  }();
  return on;
}

double kx_rate() {
  static double c = [] {
    const char* e = std::getenv("VKV_KX_RATE");
    double v = e ? std::atof(e) : 0.0;
    return (v > 0.05 && v <= 1.0) ? v : 0.65;
  }();
  return c;
}

// Longest-processing-time assignment of `units` to `g` CTAs; returns makespan.
double lpt(std::vector<Cand>& units, int g, Plan* out) {
  std::stable_sort(units.begin(), units.end(), [](const Cand& a, const Cand& b) { return a.cost > b.cost; });
  using E = std::pair<double, int>;
  std::priority_queue<E, std::vector<E>, std::greater<E>> heap;
  for (int c = 0; c < g; ++c) heap.push({0.0, c});
  std::vector<std::vector<uint32_t>> per(out ? g : 0);
  double mk = 0;
  for (const Cand& u : units) {
    E e = heap.top();
    heap.pop();
    e.first += u.cost;
    mk = std::max(mk, e.first);
    if (out) per[e.second].push_back(u.code);
    heap.push(e);
  }
  if (out) {
    out->n_ctas = g;
    out->cta_begin.assign(g + 1, 0);
    out->units.clear();
    for (int c = 0; c < g; ++c) {
      out->cta_begin[c] = (int)out->units.size();
      out->units.insert(out->units.end(), per[c].begin(), per[c].end());
    }
    out->cta_begin[g] = (int)out->units.size();
    out->cta_piece0.assign(g + 1, 0);
    out->pieces.clear();
    out->n_slots = 0;
    out->split_code.clear();
    out->split_slots.clear();
  }
  return mk;
}

constexpr uint32_t kPieceBit = 1u << 12;

inline uint32_t unit_code(int s, int tile0, bool two) {
  return ((uint32_t)s << 14) | (two ? (1u << 13) : 0u) | (uint32_t)tile0;
}

// Fixed cost of a unit (Q load, first product, epilogue) and of a piece (the
// same plus its partial in the workspace and a share of the combine), in key
// steps; pieces are at least kMinPieceSteps long (kMinPieceStepsSparse for the
// short units of BLOCK_SPARSE).
constexpr double kUnitOverhead = 2.0;
constexpr double kPieceOverhead = 4.0;
constexpr int kMinPieceSteps = 16;
#ifndef VKV_MIN_PIECE_SPARSE
#define VKV_MIN_PIECE_SPARSE 24
#endif
constexpr int kMinPieceStepsSparse = VKV_MIN_PIECE_SPARSE;
#ifndef VKV_HEAD_MAJOR
#define VKV_HEAD_MAJOR 1
#endif
#ifndef VKV_SPLIT_GAIN
#define VKV_SPLIT_GAIN 0.97
#endif
constexpr double kSplitGain = VKV_SPLIT_GAIN;  // a split schedule is used below this makespan ratio

// Schedule with key-axis pieces: each unit onto the least loaded CTA against a
// capacity T = slack * (total cost / CTAs).  A unit that does not fit the least
// loaded CTA is cut: the piece that fills that CTA up to T stays there, and the
// rest of its key steps is placed next (cut again if needed, at most
// kMaxPiecesPerUnit pieces).  The best of a few slacks is kept.  steps[s] is the
// key-step count of sequence s.
//
// Order of placement.  head_major: units in sequence order, each sequence's
// tiles in order, and the rest of a cut unit right after its piece.  With equal
// unit costs this deals the units out in waves, so the CTAs working on one
// head's query tiles (its odd last tile included) run at the same time and its
// K/V is read from DRAM about once; only the last wave is cut into pieces.
// Otherwise longest first (for unequal costs: ragged caches), the rest of a cut
// unit going back into the queue by its cost.  whole_singles: one-tile units are
// never cut (their steps alternate between the warpgroups, which a piece does not do).
bool split_plan(int n_seq, int T, const std::vector<double>& pair_cost, const std::vector<double>& one_cost,
                const std::vector<int>& steps, const std::vector<int>& steps1, int min_steps, int n_sm,
                bool head_major, bool whole_singles, Plan* out, double* mk_out) {
  struct Item {
    double cost;
    uint32_t code;
    int S;       // steps of the whole unit
    int j0, j1;  // steps still to place
    double rate;
    int k;       // pieces already cut from this unit
    int unit;    // index of the unit (for its piece list)
    bool cut;    // may be cut into pieces
  };
  auto cmp = [](const Item& a, const Item& b) {
    if (a.cost != b.cost) return a.cost < b.cost;  // max-heap on cost
    return a.unit > b.unit;                        // then the earlier unit
  };
  std::vector<Item> base;
  for (int s = 0; s < n_seq; ++s) {
    for (int i = 0; i < T / 2; ++i)
      base.push_back({pair_cost[s], unit_code(s, 2 * i, true), steps[s], 0, steps[s], 1.0, 0, 0, true});
    if (T & 1)
      base.push_back(
          {one_cost[s], unit_code(s, T - 1, false), steps1[s], 0, steps1[s], 0.0, 0, 0, !whole_singles});
  }
  if (base.empty() || (long long)base.size() > kMaxUnits) return false;
  double tot = 0, lb_piece = 0;
  for (size_t i = 0; i < base.size(); ++i) {
    base[i].unit = (int)i;
    base[i].rate = base[i].cost / (base[i].S + kUnitOverhead);
    tot += base[i].cost;
    // no CTA can finish before a unit cut into the most pieces allowed
    const int most = base[i].cut ? std::max(1, std::min(kMaxPiecesPerUnit, base[i].S / min_steps)) : 1;
    lb_piece = std::max(lb_piece, base[i].rate * ((double)base[i].S / most + kPieceOverhead));
  }
  const int g = n_sm;
  const double lb = std::max(tot / g, lb_piece);
  double best = 1e300;
  using E = std::pair<double, int>;
  // capacities from the lower bound up by 0.25 % steps to +10 %, then a few coarser ones
  std::vector<double> slacks;
  for (int i = 0; i <= 40; ++i) slacks.push_back(1.0 + 0.0025 * i);
  for (double x : {1.15, 1.2, 1.3, 1.4}) slacks.push_back(x);
  for (double slack : slacks) {
    const double cap = lb * slack;
    std::priority_queue<Item, std::vector<Item>, decltype(cmp)> q(cmp, head_major ? std::vector<Item>() : base);
    std::deque<Item> fifo;
    if (head_major) fifo.assign(base.begin(), base.end());
    std::priority_queue<E, std::vector<E>, std::greater<E>> heap;
    for (int c = 0; c < g; ++c) heap.push({0.0, c});
    // per CTA: (unit index, j0, j1) in placement order; j1 < 0 marks a whole unit
    std::vector<std::vector<std::pair<int, std::pair<int, int>>>> lists(g);
    std::vector<int> n_cut(base.size(), 0);
    while (head_major ? !fifo.empty() : !q.empty()) {
      Item it;
      if (head_major) {
        it = fifo.front();
        fifo.pop_front();
      } else {
        it = q.top();
        q.pop();
      }
      E e = heap.top();
      heap.pop();
      const bool whole_unit = it.k == 0;
      int n = it.j1 - it.j0;
      if (e.first + it.cost > cap && it.cut && it.k < kMaxPiecesPerUnit - 1 && it.S <= 0xFFFF) {
        int fit = (int)((cap - e.first) / it.rate - kPieceOverhead);
        // leave at least a minimum piece for the rest rather than overfilling this CTA
        if (fit >= min_steps && n - fit < min_steps) fit = n - min_steps;
        if (fit >= min_steps && n - fit >= min_steps) n = fit;
      }
      if (n == it.j1 - it.j0) {
        // the rest of the unit in one go
        e.first += it.cost;
        lists[e.second].push_back({it.unit, {whole_unit ? 0 : it.j0, whole_unit ? -1 : it.j1}});
        if (!whole_unit) ++n_cut[it.unit];
      } else {
        e.first += it.rate * (n + kPieceOverhead);
        lists[e.second].push_back({it.unit, {it.j0, it.j0 + n}});
        ++n_cut[it.unit];
        Item rest = it;
        rest.j0 = it.j0 + n;
        rest.k = it.k + 1;
        rest.cost = it.rate * (rest.j1 - rest.j0 + kPieceOverhead);
        if (head_major)
          fifo.push_front(rest);
        else
          q.push(rest);
      }
      heap.push(e);
    }
    double mk = 0;
    while (!heap.empty()) {
      mk = std::max(mk, heap.top().first);
      heap.pop();
    }
    // slots: the pieces of a unit get consecutive slots, numbered in j0 order
    std::vector<int> slot0(base.size(), -1);
    int n_slots = 0, n_pieces = 0, n_units = 0;
    for (size_t i = 0; i < base.size(); ++i)
      if (n_cut[i] > 0) {
        slot0[i] = n_slots;
        n_slots += n_cut[i];
        n_pieces += n_cut[i];
      }
    for (int c = 0; c < g; ++c) n_units += (int)lists[c].size();
    int n_split = 0;
    for (size_t i = 0; i < base.size(); ++i) n_split += n_cut[i] > 0 ? 1 : 0;
    if (n_pieces > kMaxPieces || n_units > kMaxUnits || n_slots > 0xFFFF || n_split > kMaxSplitUnits) continue;
    if (!(mk < best)) continue;
    best = mk;
    // piece index of a cut = its rank among the unit's cuts by j0
    std::vector<std::vector<int>> starts(base.size());
    for (int c = 0; c < g; ++c)
      for (const auto& e : lists[c])
        if (e.second.second >= 0) starts[e.first].push_back(e.second.first);
    for (auto& v : starts) std::sort(v.begin(), v.end());
    out->n_ctas = g;
    out->cta_begin.assign(g + 1, 0);
    out->cta_piece0.assign(g + 1, 0);
    out->units.clear();
    out->pieces.clear();
    for (int c = 0; c < g; ++c) {
      out->cta_begin[c] = (int)out->units.size();
      out->cta_piece0[c] = (int)out->pieces.size();
      for (const auto& e : lists[c]) {
        const Item& b = base[e.first];
        if (e.second.second < 0) {
          out->units.push_back(b.code);
          continue;
        }
        const auto& v = starts[e.first];
        const int idx = (int)(std::lower_bound(v.begin(), v.end(), e.second.first) - v.begin());
        out->units.push_back(b.code | kPieceBit);
        out->pieces.push_back(make_uint2((uint32_t)e.second.first | ((uint32_t)e.second.second << 16),
                                         (uint32_t)slot0[e.first] | ((uint32_t)idx << 16) |
                                             ((uint32_t)n_cut[e.first] << 24)));
      }
    }
    out->cta_begin[g] = (int)out->units.size();
    out->cta_piece0[g] = (int)out->pieces.size();
    out->n_slots = n_slots;
    out->split_code.clear();
    out->split_slots.clear();
    for (size_t i = 0; i < base.size(); ++i)
      if (n_cut[i] > 0) {
        out->split_code.push_back(base[i].code);
        out->split_slots.push_back((uint32_t)slot0[i] | ((uint32_t)n_cut[i] << 16));
      }
  }
  if (best >= 1e299) return false;
  *mk_out = best;
  return true;
}

// pair_cost[s] / single_cost[s]: estimated cost of a 2-tile / 1-tile unit of sequence s.
// steps / steps1 (empty: unknown) give the key steps of sequence s's 2-tile /
// 1-tile units; with them the schedule may split units along the key axis,
// into pieces of at least min_steps, when that shortens it by 12 % or more.
bool make_plan(int n_seq, int T, const std::vector<double>& pair_cost, const std::vector<double>& one_cost,
               const std::vector<int>& steps, const std::vector<int>& steps1, int min_steps, int n_sm,
               bool head_major, bool whole_singles, Plan* plan) {
  // sequences by decreasing pair cost: their pairs are split first
  std::vector<int> order(n_seq);
  for (int s = 0; s < n_seq; ++s) order[s] = s;
  std::stable_sort(order.begin(), order.end(), [&](int a, int b) { return pair_cost[a] > pair_cost[b]; });
  const int pairs_per_seq = T / 2;
  const long long n_pairs = (long long)n_seq * pairs_per_seq;
  auto build = [&](long long n_split, std::vector<Cand>& u) {
    u.clear();
    long long split = 0;
    for (int oi = 0; oi < n_seq; ++oi) {
      const int s = order[oi];
      for (int i = 0; i < pairs_per_seq; ++i) {
        if (split < n_split) {
          u.push_back({unit_code(s, 2 * i, false), one_cost[s]});
          u.push_back({unit_code(s, 2 * i + 1, false), one_cost[s]});
          ++split;
        } else {
          u.push_back({unit_code(s, 2 * i, true), pair_cost[s]});
        }
      }
      if (T & 1) u.push_back({unit_code(s, T - 1, false), one_cost[s]});
    }
  };
  std::vector<long long> cands = {0};
  for (int k = 1; k <= 32; ++k) cands.push_back((long long)k * n_sm / 8);
  // and the splits that leave exactly k * n_sm units (k units per SM when the costs are equal)
  const long long n_odd = (T & 1) ? n_seq : 0;
  for (int k = 1; k <= 16; ++k) {
    const long long c = (long long)k * n_sm - n_pairs - n_odd;
    if (c > 0 && c < n_pairs) cands.push_back(c);
  }
  cands.push_back(n_pairs);
  double best = 1e300;
  long long best_split = 0;
  std::vector<Cand> u;
  for (long long c : cands) {
    if (c > n_pairs) continue;
    build(c, u);
    if ((long long)u.size() > kMaxUnits) continue;
    const int g = (int)std::min<long long>(n_sm, (long long)u.size());
    const double mk = lpt(u, g, nullptr);
    if (mk < best * 0.999) {
      best = mk;
      best_split = c;
    }
  }
  if (!steps.empty()) {
    Plan sp;
    double mk_split = 1e300;
    // compared with the whole-unit makespan in the same cost terms (a split plan
    // always uses n_sm CTAs); pieces add a workspace fill, partial stores and the
    // combine launch, so a split must model a few per cent of gain (measured on
    // B200: the Wan-14B shape, modelled 11 % shorter, ran 5-8 % faster split)
    if (split_plan(n_seq, T, pair_cost, one_cost, steps, steps1, min_steps, n_sm, head_major, whole_singles, &sp,
                   &mk_split) &&
        mk_split < kSplitGain * best) {
      *plan = std::move(sp);
      return true;
    }
  }
  if (best >= 1e299) return false;
  build(best_split, u);
  const int g = (int)std::min<long long>(n_sm, (long long)u.size());
  lpt(u, g, plan);
  return true;
}

std::mutex g_plan_mu;
std::map<std::string, std::shared_ptr<Plan>> g_plans;

std::shared_ptr<Plan> get_plan(const std::string& key, int n_seq, int T, const std::vector<double>& pc,
                               const std::vector<double>& oc, const std::vector<int>& steps,
                               const std::vector<int>& steps1, int min_steps, int n_sm, bool head_major,
                               bool whole_singles) {
  {
    std::lock_guard<std::mutex> lk(g_plan_mu);
    auto it = g_plans.find(key);
    if (it != g_plans.end()) return it->second;
  }
  auto plan = std::make_shared<Plan>();
  if (!make_plan(n_seq, T, pc, oc, steps, steps1, min_steps, n_sm, head_major, whole_singles, plan.get()))
    return nullptr;
  std::lock_guard<std::mutex> lk(g_plan_mu);
  if (g_plans.size() > 256) g_plans.clear();
  g_plans[key] = plan;
  return plan;
}

template <int D, bool SP, bool PC, bool FS>
bool set_smem_attr_t(int dev) {
  static std::mutex mu;
  static unsigned long long done = 0;
  std::lock_guard<std::mutex> lk(mu);
  if (done & (1ull << dev)) return true;
  const void* fn = reinterpret_cast<const void*>(chunk_attn_kernel<D, SP, PC, FS>);
  cudaFuncAttributes fa;
  if (cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, AttnCfg<D>::SMEM_BYTES) !=
          cudaSuccess ||
      cudaFuncGetAttributes(&fa, fn) != cudaSuccess) {
    cudaGetLastError();
    return false;
  }
  // the warpgroup register split needs every register the launch provides
  if (fa.numRegs < kRegsLaunchNeeded) return false;
  done |= 1ull << dev;
  return true;
}

// Sets the shared-memory size of the instantiation and launches it.
template <int D, bool SP, bool PC, bool FS = false>
vkv_status launch_attn_t(int dev, const AttnParams& P, cudaStream_t st) {
  if (!set_smem_attr_t<D, SP, PC, FS>(dev)) return VKV_ERR_CUDA;
  chunk_attn_kernel<D, SP, PC, FS><<<P.n_ctas, 384, AttnCfg<D>::SMEM_BYTES, st>>>(P);
  return cudaGetLastError() == cudaSuccess ? VKV_OK : VKV_ERR_CUDA;
}

template <int D>
vkv_status launch_attn_d(int dev, bool sp, bool pc, const AttnParams& P, cudaStream_t st) {
  if (sp && P.kbar) return launch_attn_t<D, true, false, true>(dev, P, st);
  if (sp) return pc ? launch_attn_t<D, true, true>(dev, P, st) : launch_attn_t<D, true, false>(dev, P, st);
  return pc ? launch_attn_t<D, false, true>(dev, P, st) : launch_attn_t<D, false, false>(dev, P, st);
}

bool dims_ok_for_tma(const vkv_tensor& t, int B, int L, int H, int d) {
  const long long lim = 1ll << 39;  // strides below 2^40 bytes
  return std::llabs(t.sb) < lim && std::llabs(t.st) < lim && std::llabs(t.sh) < lim && B > 0 && L > 0 &&
         H > 0 && d > 0 && t.st > 0 && (H == 1 || t.sh > 0) && (B == 1 || t.sb > 0);
}

// (d, H, L, B) map with strides (sh, st, sb); size-1 axes get a natural stride.
bool encode_bhld(CUtensorMap* tm, const vkv_tensor& t, int B, int L, int H, int d, uint32_t box_rows) {
  const uint64_t dims[4] = {(uint64_t)d, (uint64_t)H, (uint64_t)L, (uint64_t)B};
  const uint64_t sh = (H == 1) ? (uint64_t)d * 2 : (uint64_t)t.sh * 2;
  const uint64_t st = (uint64_t)t.st * 2;
  const uint64_t sb = (B == 1) ? st * (uint64_t)L : (uint64_t)t.sb * 2;
  const uint64_t strides[3] = {sh, st, sb};
  const uint32_t box[4] = {64, 1, box_rows, 1};
  return encode_tmap_bf16_4d(tm, t.ptr, dims, strides, box);
}

bool encode_flat(CUtensorMap* tm, const vkv_tensor& t, int rows, int d) {
  const uint64_t dims[4] = {(uint64_t)d, 1, (uint64_t)rows, 1};
  const uint64_t st = (uint64_t)t.st * 2;
  const uint64_t strides[3] = {(uint64_t)d * 2, st, st * (uint64_t)rows};
  const uint32_t box[4] = {64, 1, 64, 1};
  return encode_tmap_bf16_4d(tm, t.ptr, dims, strides, box);
}

bool out_ok(const vkv_tensor& t) {
  return t.ptr != nullptr && tensor_aligned(t);
}

// The piece combine kernel behind the attention grid (programmatic dependent
// launch: its blocks wait for the whole attention grid with griddepcontrol.wait).
vkv_status launch_combine(const AttnParams& P, const Plan& plan, int d, cudaStream_t st) {
  auto c = std::make_unique<CombineParams>();
  std::memset(c.get(), 0, sizeof(CombineParams));
  c->mode = P.mode;
  c->H = P.H;
  c->Lq = P.Lq;
  c->n_qblk = P.n_qblk;
  c->nbr = P.mode == VKV_MODE_SEGMENTS ? P.n_branches : 1;
  c->qblk_order = P.qblk_order;
  c->ws_o = P.ws_o;
  c->ws_l = P.ws_l;
  for (int br = 0; br < VKV_MAX_BRANCHES; ++br) {
    c->o[br] = P.o[br];
    c->o_sb[br] = P.o_sb[br];
    c->o_st[br] = P.o_st[br];
    c->o_sh[br] = P.o_sh[br];
    c->lse[br] = P.lse[br];
  }
  c->om = P.om;
  c->om_sb = P.om_sb;
  c->om_st = P.om_st;
  c->om_sh = P.om_sh;
  c->lsem = P.lsem;
  c->n_units = (int)plan.split_code.size();
  std::copy(plan.split_code.begin(), plan.split_code.end(), c->code);
  std::copy(plan.split_slots.begin(), plan.split_slots.end(), c->slots);
  const int rows_per_block = 256 / (d / 8);
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)(c->n_units * 2 * (128 / rows_per_block)));
  cfg.blockDim = dim3(256);
  cfg.dynamicSmemBytes = 0;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  const cudaError_t e = d == 128 ? cudaLaunchKernelEx(&cfg, piece_combine_kernel<128>, *c)
                                 : cudaLaunchKernelEx(&cfg, piece_combine_kernel<64>, *c);
  return e == cudaSuccess ? VKV_OK : VKV_ERR_CUDA;
}

}  // namespace

}  // namespace vkv

namespace vkv {
namespace {

// Bytes of the piece workspace: partial LSEs, then partial outputs (256-aligned).
struct WsLayout {
  size_t l_off, o_off, bytes;
};

WsLayout ws_layout(int n_slots, int nbr, int d) {
  auto al = [](size_t x) { return (x + 255) & ~(size_t)255; };
  WsLayout w;
  w.l_off = 0;
  w.o_off = al((size_t)n_slots * 2 * nbr * 128 * sizeof(float));
  w.bytes = n_slots > 0 ? w.o_off + (size_t)n_slots * 2 * nbr * 128 * d * sizeof(float) : 0;
  return w;
}

// Checks the arguments and builds the kernel parameters and the schedule.
// check_ptrs = false (workspace size query): only the host-side fields are read.
vkv_status attn_setup(const vkv_attn_args* a, bool check_ptrs, bool want_split, AttnParams* P,
                      std::shared_ptr<Plan>* plan_out, int* dev_out, int n_sm_override = 0) {
  if (!a) return VKV_ERR_NULL;
  const int mode = a->mode;
  if (mode != VKV_MODE_SEGMENTS && mode != VKV_MODE_BLOCK_SPARSE && mode != VKV_MODE_RAGGED)
    return VKV_ERR_UNSUPPORTED;
  if (a->d != 64 && a->d != 128) return VKV_ERR_UNSUPPORTED;
  if (a->B <= 0 || a->H <= 0 || a->Lq <= 0 || a->Lkv < 0) return VKV_ERR_SHAPE;
  if (!(a->scale > 0.f) || !std::isfinite(a->scale)) return VKV_ERR_SHAPE;
  const int B = a->B, H = a->H, Lq = a->Lq, Lkv = a->Lkv, d = a->d;
  const long long n_seq = (long long)B * H;
  const int T = (Lq + 127) / 128;
  if (n_seq >= (1ll << 18) || T > 4096) return VKV_ERR_UNSUPPORTED;
  if (check_ptrs) {
    if (!a->q.ptr || !a->k.ptr || !a->v.ptr) return VKV_ERR_NULL;
    if (!tensor_aligned(a->q) || !tensor_aligned(a->k) || !tensor_aligned(a->v)) return VKV_ERR_ALIGN;
    if (!dims_ok_for_tma(a->q, B, Lq, H, d)) return VKV_ERR_SHAPE;
  }

  std::memset(P, 0, sizeof(AttnParams));
  P->mode = mode;
  P->B = B;
  P->H = H;
  P->Lq = Lq;
  P->Lkv = Lkv;
  P->d = d;
  P->scale_log2 = a->scale * 1.4426950408889634f;
  P->err = a->err_word;

  int nb = 1;
  std::vector<double> pc(n_seq), oc(n_seq);
  std::vector<int> steps, steps1;  // key steps of 2-tile / 1-tile units, when units may be split
  int min_steps = kMinPieceSteps;
  const double c1 = single_tile_cost();
  std::string key;
  if (mode == VKV_MODE_SEGMENTS) {
    nb = a->n_branches;
    if (nb < 1 || nb > 2) return VKV_ERR_SHAPE;
    if (Lkv <= 0) return VKV_ERR_SHAPE;
    if (check_ptrs && (!dims_ok_for_tma(a->k, B, Lkv, H, d) || !dims_ok_for_tma(a->v, B, Lkv, H, d)))
      return VKV_ERR_SHAPE;
    P->n_branches = nb;
    int nf = 0, total = 0;
    for (int br = 0; br < nb; ++br) {
      const int ns = a->n_segs[br];
      if (ns < 0 || ns > VKV_MAX_SEGMENTS) return VKV_ERR_SHAPE;
      if (ns > 0 && !a->segs[br]) return VKV_ERR_NULL;
      bool first = true;
      int stp = 0;
      for (int i = 0; i < ns; ++i) {
        const vkv_segment sg = a->segs[br][i];
        if (sg.start < 0 || sg.len < 0 || (long long)sg.start + sg.len > Lkv) return VKV_ERR_RANGE;
        if (sg.len == 0) continue;
        P->flat_start[nf] = sg.start;
        P->flat_len[nf] = sg.len;
        P->flat_branch[nf] = br;
        P->flat_first[nf] = first ? 1 : 0;
        P->flat_step0[nf] = total + stp;
        first = false;
        stp += (sg.len + 127) / 128;
        ++nf;
      }
      P->branch_steps[br] = stp;
      total += stp;
    }
    P->n_flat = nf;
    P->total_steps = total;
    for (long long s = 0; s < n_seq; ++s) {
      pc[s] = total + 2.0;
      oc[s] = c1 * (total + 2.0);
    }
    if (want_split) steps.assign(n_seq, total);
    key = "S" + std::to_string(n_seq) + "/" + std::to_string(T) + "/" + std::to_string(total);
  } else if (mode == VKV_MODE_BLOCK_SPARSE) {
    if (a->block != 64) return VKV_ERR_UNSUPPORTED;
    if (Lkv <= 0) return VKV_ERR_SHAPE;
    if (check_ptrs && (!dims_ok_for_tma(a->k, B, Lkv, H, d) || !dims_ok_for_tma(a->v, B, Lkv, H, d)))
      return VKV_ERR_SHAPE;
    if (a->n_persist < 0 || a->topk < 0 || a->n_win_blk < 0 || a->window_blk0 < 0) return VKV_ERR_SHAPE;
    if (a->n_win_blk > 1024 || a->topk > a->n_win_blk) return VKV_ERR_SHAPE;
    if ((long long)(a->window_blk0 + a->n_win_blk) * 64 > Lkv) return VKV_ERR_RANGE;
    if (a->n_persist + std::min(a->n_win_blk, 4 * a->topk) > kMaxListEntries) return VKV_ERR_UNSUPPORTED;
    // selection in the kernel (window block means given): whole units, at least one
    // block per query block, a window that fits the kernel's ranking keys
    const bool fs = a->kbar != nullptr;
    if (fs && (a->topk < 1 || a->n_win_blk > kFsMaxWin)) return VKV_ERR_SHAPE;
    if (fs) want_split = false;
    if (check_ptrs && ((a->n_persist > 0 && !a->persist_idx) || (a->topk > 0 && !a->sel_idx && !fs)))
      return VKV_ERR_NULL;
    if (check_ptrs && fs && (reinterpret_cast<uintptr_t>(a->kbar) & 15)) return VKV_ERR_ALIGN;
    if (fs) {
      P->kbar = a->kbar;
      P->sel_out = a->sel_out;
      P->qp = reinterpret_cast<const __nv_bfloat16*>(a->q.ptr);
      P->q_sb = a->q.sb;
      P->q_st = a->q.st;
      P->q_sh = a->q.sh;
    }
    P->n_persist = a->n_persist;
    P->topk = a->topk;
    P->window_blk0 = a->window_blk0;
    P->n_win_blk = a->n_win_blk;
    P->n_qblk = (Lq + 63) / 64;
    P->n_blocks_total = Lkv / 64;
    P->persist_idx = a->persist_idx;
    P->sel_idx = a->sel_idx;
    P->qblk_order = a->qblk_order;
    // expected key tiles of a unit: persistent blocks + the union of its query blocks'
    // selections (two blocks per tile); a grouped order keeps the union near one selection
    const bool grouped = a->qblk_order != nullptr;
    const double u4 = std::min<double>(a->n_win_blk, (grouped ? 1.5 : 4.0) * a->topk);
    const double u2 = std::min<double>(a->n_win_blk, (grouped ? 1.25 : 2.0) * a->topk);
    const double sp = (a->n_persist + u4) * 0.5 + 2.0;
    const double s1 = (a->n_persist + u2) * 0.5 + 2.0;
    P->kx = (fs && kx_enabled()) ? 1 : 0;
    const double s1_cost = P->kx ? kx_rate() * (a->n_persist + u2) * 0.5 + kUnitOverhead : c1 * s1;
    for (long long s = 0; s < n_seq; ++s) {
      pc[s] = sp;
      oc[s] = s1_cost;
    }
    // pieces are cut in these estimated steps and scaled on the device to the
    // unit's real step count
    P->sp_est[0] = (int)std::ceil((a->n_persist + u2) * 0.5);
    P->sp_est[1] = (int)std::ceil((a->n_persist + u4) * 0.5);
    if (want_split) {
      steps.assign(n_seq, P->sp_est[1]);
      steps1.assign(n_seq, P->sp_est[0]);
    }
    key = "B" + std::to_string(n_seq) + "/" + std::to_string(T) + "/" + std::to_string(a->n_persist) + "/" +
          std::to_string(a->topk) + "/" + std::to_string(a->n_win_blk) + (grouped ? "/g" : "/n") + (fs ? "/fs" : "") + (P->kx ? "/kx" : "");
  } else {
    if (check_ptrs && !a->cu_seqlens) return VKV_ERR_NULL;
    if (Lkv <= 0) return VKV_ERR_SHAPE;
    if (check_ptrs && (a->k.st <= 0 || a->v.st <= 0 || (a->k.st % 8) || (a->v.st % 8))) return VKV_ERR_SHAPE;
    if (a->cu_seqlens_host) {
      const int32_t* cu = a->cu_seqlens_host;
      if (cu[0] < 0) return VKV_ERR_RANGE;
      for (long long s = 0; s < n_seq; ++s)
        if (cu[s + 1] < cu[s] || cu[s + 1] > Lkv) return VKV_ERR_RANGE;
      key = "R" + std::to_string(n_seq) + "/" + std::to_string(T);
      if (want_split) steps.resize(n_seq);
      for (long long s = 0; s < n_seq; ++s) {
        const int stp = (cu[s + 1] - cu[s] + 127) / 128;
        pc[s] = stp + 2.0;
        oc[s] = c1 * (stp + 2.0);
        if (want_split) steps[s] = stp;
        key += "," + std::to_string(stp);
      }
    } else {
      for (long long s = 0; s < n_seq; ++s) {
        pc[s] = 1.0;
        oc[s] = c1;
      }
      key = "R" + std::to_string(n_seq) + "/" + std::to_string(T) + "/u";
    }
    P->cu_seqlens = a->cu_seqlens;
  }
  if (check_ptrs) {
    const int nout = (mode == VKV_MODE_SEGMENTS) ? nb : 1;
    for (int br = 0; br < nout; ++br) {
      if (!a->lse[br]) return VKV_ERR_NULL;
      if (!out_ok(a->o[br])) return a->o[br].ptr ? VKV_ERR_ALIGN : VKV_ERR_NULL;
      P->o[br] = reinterpret_cast<__nv_bfloat16*>(a->o[br].ptr);
      P->o_sb[br] = a->o[br].sb;
      P->o_st[br] = a->o[br].st;
      P->o_sh[br] = a->o[br].sh;
      P->lse[br] = a->lse[br];
    }
    if (mode == VKV_MODE_SEGMENTS && nb == 2 && a->o_merged.ptr) {
      if (!a->lse_merged) return VKV_ERR_NULL;
      if (!out_ok(a->o_merged)) return VKV_ERR_ALIGN;
      P->om = reinterpret_cast<__nv_bfloat16*>(a->o_merged.ptr);
      P->om_sb = a->o_merged.sb;
      P->om_st = a->o_merged.st;
      P->om_sh = a->o_merged.sh;
      P->lsem = a->lse_merged;
    }
  }

  int dev = 0;
  const int n_sm = n_sm_override > 0 ? n_sm_override : device_sm_count(&dev);
  if (n_sm <= 0) return VKV_ERR_CUDA;
  const int g_max = std::min(n_sm, kMaxCtas);
  key += "@" + std::to_string(g_max) + ":" + std::to_string(c1) + (steps.empty() ? "" : "/split");
  if (mode == VKV_MODE_BLOCK_SPARSE) min_steps = kMinPieceStepsSparse;
  if (steps1.empty()) steps1 = steps;
  // equal unit costs (every mode but ragged): units dealt out head by head
  const bool head_major = VKV_HEAD_MAJOR && mode != VKV_MODE_RAGGED;
  std::shared_ptr<Plan> plan =
      get_plan(key, (int)n_seq, T, pc, oc, steps, steps1, min_steps, g_max, head_major, P->kx != 0);
  if (!plan) return VKV_ERR_UNSUPPORTED;
  P->n_ctas = plan->n_ctas;
  std::copy(plan->cta_begin.begin(), plan->cta_begin.end(), P->cta_begin);
  std::copy(plan->cta_piece0.begin(), plan->cta_piece0.end(), P->cta_piece0);
  std::copy(plan->pieces.begin(), plan->pieces.end(), P->pieces);
  std::copy(plan->units.begin(), plan->units.end(), P->units);
  *plan_out = plan;
  *dev_out = dev;
  return VKV_OK;
}

}  // namespace
}  // namespace vkv

using namespace vkv;

extern "C" size_t vkv_chunk_attn_workspace_size(const vkv_attn_args* a) {
  if (!a) return 0;
  auto P = std::make_unique<AttnParams>();
  std::shared_ptr<Plan> plan;
  int dev = 0;
  if (attn_setup(a, false, true, P.get(), &plan, &dev) != VKV_OK) return 0;
  const int nbr = a->mode == VKV_MODE_SEGMENTS ? a->n_branches : 1;
  return ws_layout(plan->n_slots, nbr, a->d).bytes;
}

extern "C" vkv_status vkv_debug_schedule(const vkv_attn_args* a, int32_t n_sm, int32_t split,
                                         vkv_schedule* out) {
  if (!a || !out || n_sm <= 0 || n_sm > kMaxCtas) return VKV_ERR_SHAPE;
  auto P = std::make_unique<AttnParams>();
  std::shared_ptr<Plan> plan;
  int dev = 0;
  const vkv_status stt = attn_setup(a, false, split != 0, P.get(), &plan, &dev, n_sm);
  if (stt != VKV_OK) return stt;
  out->n_ctas = plan->n_ctas;
  out->n_units = (int32_t)plan->units.size();
  out->n_pieces = (int32_t)plan->pieces.size();
  out->n_slots = plan->n_slots;
  if (out->cta_begin) std::copy(plan->cta_begin.begin(), plan->cta_begin.end(), out->cta_begin);
  if (out->cta_piece0) std::copy(plan->cta_piece0.begin(), plan->cta_piece0.end(), out->cta_piece0);
  if (out->units) std::copy(plan->units.begin(), plan->units.end(), out->units);
  if (out->pieces)
    for (size_t i = 0; i < plan->pieces.size(); ++i) {
      out->pieces[2 * i] = plan->pieces[i].x;
      out->pieces[2 * i + 1] = plan->pieces[i].y;
    }
  return VKV_OK;
}

extern "C" vkv_status vkv_chunk_attn(const vkv_attn_args* a, vkv_stream_t stream) {
  if (!a) return VKV_ERR_NULL;
  const bool want_split = a->workspace != nullptr;
  auto P = std::make_unique<AttnParams>();
  std::shared_ptr<Plan> plan;
  int dev = 0;
  const vkv_status stt = attn_setup(a, true, want_split, P.get(), &plan, &dev);
  if (stt != VKV_OK) return stt;
#ifdef VKV_TEST_AIDS
  P->withhold_first_copy = take_withhold_request() ? 1 : 0;
#endif
  const int mode = a->mode, B = a->B, H = a->H, Lq = a->Lq, Lkv = a->Lkv, d = a->d;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  if (plan->n_slots > 0) {
    const int nbr = mode == VKV_MODE_SEGMENTS ? a->n_branches : 1;
    const WsLayout w = ws_layout(plan->n_slots, nbr, d);
    if (a->workspace_bytes < w.bytes) return VKV_ERR_WORKSPACE;
    if (reinterpret_cast<uintptr_t>(a->workspace) & 255) return VKV_ERR_ALIGN;
    uint8_t* ws = reinterpret_cast<uint8_t*>(a->workspace);
    P->ws_l = reinterpret_cast<float*>(ws + w.l_off);
    P->ws_o = reinterpret_cast<float*>(ws + w.o_off);
    // partial LSEs to NaN (all bits set), which marks a branch a piece did not reach
    if (cudaMemsetAsync(P->ws_l, 0xFF, (size_t)plan->n_slots * 2 * nbr * 128 * sizeof(float), st) != cudaSuccess)
      return VKV_ERR_CUDA;
  }

  // BLOCK_SPARSE loads a query tile as two 64-row blocks (a unit's blocks follow qblk_order)
  if (!encode_bhld(&P->tm_q, a->q, B, Lq, H, d, mode == VKV_MODE_BLOCK_SPARSE ? 64 : 128)) return VKV_ERR_CUDA;
  if (mode == VKV_MODE_RAGGED) {
    if (!encode_flat(&P->tm_k, a->k, Lkv, d) || !encode_flat(&P->tm_v, a->v, Lkv, d)) return VKV_ERR_CUDA;
  } else {
    if (!encode_bhld(&P->tm_k, a->k, B, Lkv, H, d, 64) || !encode_bhld(&P->tm_v, a->v, B, Lkv, H, d, 64))
      return VKV_ERR_CUDA;
  }
  const bool sp = mode == VKV_MODE_BLOCK_SPARSE;
  const bool pc = plan->n_slots > 0;
  const vkv_status ls = d == 128 ? launch_attn_d<128>(dev, sp, pc, *P, st) : launch_attn_d<64>(dev, sp, pc, *P, st);
  if (ls != VKV_OK || !pc) return ls;
  return launch_combine(*P, *plan, d, st);
}

#ifdef VKV_TEST_AIDS
namespace vkv {
namespace {
__global__ void exp2_poly_kernel(const float* x, float* y, int n) {
  const int i = 2 * (blockIdx.x * blockDim.x + threadIdx.x);
  if (i >= n) return;
  const float x0 = x[i], x1 = i + 1 < n ? x[i + 1] : 0.f;
  float e0, e1;
  exp2_poly2(x0, x1, e0, e1);
  y[i] = e0;
  if (i + 1 < n) y[i + 1] = e1;
}
}  // namespace
}  // namespace vkv

// Test build only (vkv_test.h): the attention softmax's FMA-pipe exp2 on n DEVICE floats.
extern "C" vkv_status vkv_debug_exp2_poly(const float* x, float* y, int32_t n, vkv_stream_t stream) {
  if (!x || !y) return VKV_ERR_NULL;
  if (n <= 0) return VKV_ERR_SHAPE;
  int dev = 0;
  if (device_sm_count(&dev) <= 0) return VKV_ERR_CUDA;
  const int pairs = (n + 1) / 2;
  vkv::exp2_poly_kernel<<<(pairs + 255) / 256, 256, 0, reinterpret_cast<cudaStream_t>(stream)>>>(x, y, n);
  return cudaGetLastError() == cudaSuccess ? VKV_OK : VKV_ERR_CUDA;
}
#endif

#ifdef VKV_TRACE
// Development only (not in the public header): copy CTA 0's pipeline timeline.
extern "C" int vkv_debug_trace(void* dst, size_t bytes) {
  cudaDeviceSynchronize();
  return (int)cudaMemcpyFromSymbol(dst, vkv::g_vkv_trace, bytes < sizeof(vkv::g_vkv_trace) ? bytes : sizeof(vkv::g_vkv_trace));
}
extern "C" int vkv_debug_trace_clear() {
  static unsigned long long zeros[2 * 28672];
  return (int)cudaMemcpyToSymbol(vkv::g_vkv_trace, zeros, sizeof(zeros));
}
#endif
