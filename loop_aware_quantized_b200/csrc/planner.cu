// LoopKV planner (host code): the plan with the fewest reads within a damage
// budget and a storage budget.
//
// "LoopKV: Loop-Aware KV Cache Compression for Serving Looped Transformers",
// section 概要: a one-time offline profile gives each (loop, layer) cell a
// predicted damage for 4-bit storage, 2-bit storage or reuse of the final
// loop's KV; damages add over cells; the planner looks for the least data
// read while predicted damage and storage each stay within a budget.  The costs per cached token and
// KV head, in quarters of head_dim bytes, are read as: Q4 stores 6 blocks
// and reads 5 plus a low-plane row for a fraction of its tokens; Q2 stores
// and reads 4; SHARE stores nothing and reads what its layer's final-loop
// cell reads.
//
// A SHARE cell's reads depend on the final-loop cell of its layer, so the
// dynamic program runs over layers: a layer's options are the assignments of
// its cells (final-loop kind x the others' kinds), its state the exact
// (damage, storage) used so far, its value the fewest reads.  Options a
// layer dominates (no better in damage, storage or reads) are dropped first.
// Reads are integers (thousandths of a quarter of head_dim bytes), so the
// comparison is exact.

#include <algorithm>
#include <climits>
#include <cmath>
#include <cstdint>
#include <vector>

#include "loopkv.h"

namespace {

constexpr int kMaxLoops = 6;
constexpr int kMaxCells = 4096;
constexpr int64_t kMaxStates = int64_t(1) << 20;
constexpr int64_t kInf = INT64_MAX;

struct Option {
  int64_t damage, reads;
  int32_t storage;    // quarters of head_dim bytes
  uint32_t code;      // kind of loop l in base-3 digit l
};

// Reads (thousandths of a quarter of head_dim bytes) and storage (quarters)
// per cached token and KV head.
int64_t reads_of(int kind, int sel_milli) { return kind == LOOPKV_Q4 ? 5000 + sel_milli : 4000; }
int32_t storage_of(int kind) { return kind == LOOPKV_Q4 ? 6 : kind == LOOPKV_Q2 ? 4 : 0; }

std::vector<Option> layer_options(const loopkv_planner_desc* d, int layer, int sel_milli) {
  const int L = d->n_loops, N = d->n_layers;
  std::vector<Option> all;
  int combos = 2;
  for (int l = 0; l + 1 < L; ++l) combos *= 3;
  for (int x = 0; x < combos; ++x) {
    // digit L-1 (final loop) in {Q4, Q2}; the others in {Q4, Q2, SHARE}
    int rest = x;
    const int fk = rest % 2;
    rest /= 2;
    Option o{0, 0, 0, 0};
    uint32_t code = 0, mul = 1;
    for (int l = 0; l < L; ++l) {
      int k;
      if (l == L - 1) {
        k = fk;
      } else {
        k = rest % 3;
        rest /= 3;
      }
      const int cell = l * N + layer;
      o.damage += d->damage[cell * 3 + k];
      o.storage += storage_of(k);
      o.reads += k == LOOPKV_SHARE ? reads_of(fk, sel_milli) : reads_of(k, sel_milli);
      code += (uint32_t)k * mul;
      mul *= 3;
    }
    o.code = code;
    all.push_back(o);
  }
  // drop dominated options (never needed by an optimum), keep a fixed order
  std::vector<Option> keep;
  for (size_t i = 0; i < all.size(); ++i) {
    bool dominated = false;
    for (size_t j = 0; j < all.size() && !dominated; ++j) {
      if (i == j) continue;
      const Option &a = all[j], &b = all[i];
      const bool le = a.damage <= b.damage && a.storage <= b.storage && a.reads <= b.reads;
      const bool lt = a.damage < b.damage || a.storage < b.storage || a.reads < b.reads;
      dominated = le && (lt || j < i);  // equal options: keep the first
    }
    if (!dominated) keep.push_back(all[i]);
  }
  return keep;
}

}  // namespace

extern "C" loopkv_status loopkv_plan_optimize(const loopkv_planner_desc* d, uint8_t* kinds_out,
                                              loopkv_plan_cost* cost) {
  if (d == nullptr || kinds_out == nullptr || d->damage == nullptr) return LOOPKV_ERR_INVALID_ARG;
  const int L = d->n_loops, N = d->n_layers;
  if (L < 1 || L > kMaxLoops || N < 1 || (int64_t)L * N > kMaxCells) return LOOPKV_ERR_INVALID_ARG;
  if (d->head_dim != 64 && d->head_dim != 128) return LOOPKV_ERR_INVALID_ARG;
  if (d->damage_budget < 0 || d->storage_budget < 0) return LOOPKV_ERR_INVALID_ARG;
  if (!(d->sel_fraction >= 0.f && d->sel_fraction <= 1.f)) return LOOPKV_ERR_INVALID_ARG;
  const int cells = L * N;
  int64_t dmg_max = 0;
  for (int c = 0; c < cells; ++c) {
    int32_t m = 0;
    for (int k = 0; k < 3; ++k) {
      if (d->damage[c * 3 + k] < 0) return LOOPKV_ERR_INVALID_ARG;
      if (k < 2 || c / N < L - 1) m = std::max(m, d->damage[c * 3 + k]);
    }
    dmg_max += m;
  }
  const int sel_milli = (int)std::lround(1000.0 * d->sel_fraction);
  const int64_t quarter = d->head_dim / 4;
  // budgets capped at what the cells can use
  const int64_t Db = std::min(d->damage_budget, dmg_max);
  const int64_t Sb = std::min(d->storage_budget / quarter, (int64_t)6 * cells);
  const int64_t S1 = Sb + 1;
  const int64_t states = (Db + 1) * S1;
  if (states > kMaxStates) return LOOPKV_ERR_UNSUPPORTED;

  std::vector<std::vector<Option>> opts(N);
  for (int n = 0; n < N; ++n) opts[n] = layer_options(d, n, sel_milli);
  std::vector<int64_t> val(states, kInf), nxt(states);
  std::vector<std::vector<uint16_t>> pick(N, std::vector<uint16_t>(states, 0));
  val[0] = 0;
  for (int n = 0; n < N; ++n) {
    std::fill(nxt.begin(), nxt.end(), kInf);
    const std::vector<Option>& os = opts[n];
    for (int64_t st = 0; st < states; ++st) {
      const int64_t v = val[st];
      if (v == kInf) continue;
      const int64_t dm = st / S1, sg = st % S1;
      for (size_t i = 0; i < os.size(); ++i) {
        const int64_t d2 = dm + os[i].damage, s2 = sg + os[i].storage;
        if (d2 > Db || s2 > Sb) continue;
        const int64_t t = d2 * S1 + s2, r = v + os[i].reads;
        if (r < nxt[t]) { nxt[t] = r; pick[n][t] = (uint16_t)i; }
      }
    }
    val.swap(nxt);
  }
  // best final state: fewest reads, then least damage, then least storage
  int64_t best = -1;
  for (int64_t st = 0; st < states; ++st) {
    if (val[st] == kInf) continue;
    if (best < 0 || val[st] < val[best]) best = st;  // scan order is (damage, storage) ascending
  }
  if (best < 0) return LOOPKV_ERR_PLAN;
  const int64_t best_reads = val[best];
  int64_t st = best;
  int64_t total_storage = 0;
  for (int n = N - 1; n >= 0; --n) {
    const Option& o = opts[n][pick[n][st]];
    uint32_t code = o.code;
    for (int l = 0; l < L; ++l) {
      kinds_out[l * N + n] = (uint8_t)(code % 3);
      code /= 3;
    }
    total_storage += o.storage;
    st = (st / S1 - o.damage) * S1 + (st % S1 - o.storage);
  }
  if (cost != nullptr) {
    cost->reads = (double)best_reads * (double)quarter / 1000.0;
    cost->damage = best / S1;
    cost->storage = total_storage * quarter;
  }
  return LOOPKV_OK;
}
