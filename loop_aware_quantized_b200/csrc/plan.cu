// Host side of the LoopKV C ABI (include/loopkv.h): plan validation, the
// canonical cache layout, the host copy of the lengths, argument checks and
// kernel launches.  No device memory is allocated here.

#include <cuda_runtime.h>

#include <cmath>
#include <cstdlib>
#include <cstring>
#include <new>
#include <vector>

#include "loopkv_internal.cuh"

using namespace loopkv;

struct loopkv_plan {
  int n_loops = 0, n_layers = 0, n_cells = 0, H = 0, D = 0, max_batch = 0;
  int group = 1;                  // query heads per KV head
  int min_split = 1;              // CTAs per decoded unit at least (the descriptor's decode_split)
  float tau = 0.f, sm_scale = 0.f;
  std::vector<uint8_t> kinds;     // [cells]
  std::vector<int32_t> cap;       // [max_batch]
  std::vector<int32_t> len;       // [cells][max_batch] host copy of the lengths
  std::vector<uint64_t> offset;   // [cells][max_batch] head-0 region offset
  std::vector<uint64_t> stride;   // [cells][max_batch] region bytes per head
  uint8_t* d_table = nullptr;
  uint8_t* d_cache = nullptr;
  size_t cache_bytes = 0;

  int src(int cell) const { return (n_loops - 1) * n_layers + cell % n_layers; }
  // positions of a unit's reference that a RES2 unit may read: the
  // quantized ones of a Q4/Q2 reference, every one of a BF16 reference
  int ref_positions(int cell, int b) const {
    const int r = src(cell);
    return kinds[r] == LOOPKV_BF16 ? L(r, b) : L(r, b) / kGroup * kGroup;
  }
  int32_t& L(int cell, int b) { return len[(size_t)cell * max_batch + b]; }
  int32_t L(int cell, int b) const { return len[(size_t)cell * max_batch + b]; }
};

namespace {

constexpr uint32_t kMagic = 0x4C4B5631u;  // "LKV1"
constexpr int kMaxCells = 4096;
constexpr int kMaxCapacity = 1 << 20;

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

loopkv_status validate_desc(const loopkv_plan_desc* d) {
  if (d == nullptr || d->capacity == nullptr || d->kinds == nullptr) return LOOPKV_ERR_INVALID_ARG;
  if (d->n_loops < 1 || d->n_layers < 1 || d->n_kv_heads < 1) return LOOPKV_ERR_PLAN;
  if ((long long)d->n_loops * d->n_layers > kMaxCells) return LOOPKV_ERR_PLAN;
  if (d->head_dim != 64 && d->head_dim != 128) return LOOPKV_ERR_PLAN;
  if (d->max_batch < 1 || d->max_batch > LOOPKV_MAX_BATCH) return LOOPKV_ERR_PLAN;
  if (d->n_kv_heads > (1 << 16)) return LOOPKV_ERR_PLAN;
  if (!(d->tau >= 0.f) || !std::isfinite(d->tau)) return LOOPKV_ERR_PLAN;
  if (!std::isfinite(d->sm_scale)) return LOOPKV_ERR_PLAN;
  if (d->q_per_kv != 0 && d->q_per_kv != 1 && d->q_per_kv != 2 && d->q_per_kv != 4)
    return LOOPKV_ERR_PLAN;
  if (d->decode_split < 0 || d->decode_split > decode_max_split() ||
      (d->decode_split & (d->decode_split - 1)) != 0)
    return LOOPKV_ERR_PLAN;
  for (int b = 0; b < d->max_batch; ++b)
    if (d->capacity[b] < 0 || d->capacity[b] > kMaxCapacity) return LOOPKV_ERR_PLAN;
  const int cells = d->n_loops * d->n_layers;
  for (int c = 0; c < cells; ++c) {
    const int k = d->kinds[c];
    if (k > LOOPKV_RES2) return LOOPKV_ERR_PLAN;
    // SHARE and RES2 read the final loop's cell of their layer, so neither
    // can sit in the final loop (whose cells are then Q4, Q2 or BF16)
    if ((k == LOOPKV_SHARE || k == LOOPKV_RES2) && c / d->n_layers == d->n_loops - 1)
      return LOOPKV_ERR_PLAN;
  }
  return LOOPKV_OK;
}

size_t cache_bytes_of(const loopkv_plan_desc* d) {
  const int cells = d->n_loops * d->n_layers;
  size_t total = 0;
  for (int c = 0; c < cells; ++c)
    for (int b = 0; b < d->max_batch; ++b)
      total += (size_t)d->n_kv_heads * unit_layout(d->kinds[c], d->head_dim, d->capacity[b]).total;
  return total;
}

loopkv_status check_cells(const loopkv_plan* p, const int32_t* h_cells, int32_t n_cells,
                          int32_t batch, CellList* out) {
  if (p == nullptr || h_cells == nullptr) return LOOPKV_ERR_INVALID_ARG;
  if (n_cells < 1 || n_cells > LOOPKV_MAX_CELLS_PER_CALL) return LOOPKV_ERR_INVALID_ARG;
  if (batch < 1 || batch > p->max_batch) return LOOPKV_ERR_INVALID_ARG;
  std::vector<char> seen(p->n_cells, 0);
  for (int i = 0; i < n_cells; ++i) {
    const int c = h_cells[i];
    if (c < 0 || c >= p->n_cells || seen[c]) return LOOPKV_ERR_INVALID_ARG;
    seen[c] = 1;
    out->cell[i] = c;
    out->out[i] = i;
  }
  return LOOPKV_OK;
}

loopkv_status from_cuda(int e) { return e == 0 ? LOOPKV_OK : LOOPKV_ERR_CUDA; }

loopkv_status decode_launch(loopkv_plan* p, const CellList& cl, int n_cells, int batch,
                            int npos_max, bool res2, const uint16_t* d_q, float* d_out,
                            float* d_lse, uint32_t* d_mask, int32_t mask_words, int32_t* d_nsel,
                            void* stream);

}  // namespace

extern "C" {

loopkv_status loopkv_plan_query(const loopkv_plan_desc* desc, loopkv_sizes* sizes) {
  if (sizes == nullptr) return LOOPKV_ERR_INVALID_ARG;
  const loopkv_status st = validate_desc(desc);
  if (st != LOOPKV_OK) return st;
  sizes->table_bytes = table_bytes(desc->n_loops * desc->n_layers, desc->max_batch);
  sizes->cache_bytes = cache_bytes_of(desc);
  return LOOPKV_OK;
}

loopkv_status loopkv_plan_load(const loopkv_plan_desc* desc, void* d_table, size_t tbytes,
                               void* d_cache, size_t cbytes, void* stream, loopkv_plan** out) {
  if (out == nullptr) return LOOPKV_ERR_INVALID_ARG;
  *out = nullptr;
  loopkv_sizes sz;
  loopkv_status st = loopkv_plan_query(desc, &sz);
  if (st != LOOPKV_OK) return st;
  if (d_table == nullptr || tbytes < sz.table_bytes || !aligned16(d_table)) return LOOPKV_ERR_INVALID_ARG;
  if (sz.cache_bytes > 0 && (d_cache == nullptr || cbytes < sz.cache_bytes ||
                             (reinterpret_cast<uintptr_t>(d_cache) & 255u) != 0))
    return LOOPKV_ERR_INVALID_ARG;

  loopkv_plan* p = new (std::nothrow) loopkv_plan();
  if (p == nullptr) return LOOPKV_ERR_INVALID_ARG;
  p->n_loops = desc->n_loops;
  p->n_layers = desc->n_layers;
  p->n_cells = desc->n_loops * desc->n_layers;
  p->H = desc->n_kv_heads;
  p->group = desc->q_per_kv > 1 ? desc->q_per_kv : 1;
  p->min_split = desc->decode_split > 1 ? desc->decode_split : 1;
  p->D = desc->head_dim;
  p->max_batch = desc->max_batch;
  p->tau = desc->tau;
  p->sm_scale = desc->sm_scale > 0.f ? desc->sm_scale : 1.0f / std::sqrt((float)desc->head_dim);
  p->kinds.assign(desc->kinds, desc->kinds + p->n_cells);
  p->cap.assign(desc->capacity, desc->capacity + p->max_batch);
  p->len.assign((size_t)p->n_cells * p->max_batch, 0);
  p->offset.resize((size_t)p->n_cells * p->max_batch);
  p->stride.resize((size_t)p->n_cells * p->max_batch);
  p->d_table = static_cast<uint8_t*>(d_table);
  p->d_cache = static_cast<uint8_t*>(d_cache);
  p->cache_bytes = sz.cache_bytes;

  std::vector<uint8_t> img(sz.table_bytes, 0);
  TableHeader* hdr = reinterpret_cast<TableHeader*>(img.data());
  hdr->status = 0;
  hdr->magic = kMagic;
  hdr->n_cells = p->n_cells;
  hdr->max_batch = p->max_batch;
  hdr->n_heads = p->H;
  hdr->head_dim = p->D;
  DevCell* cells = reinterpret_cast<DevCell*>(img.data() + table_cells_offset());
  DevSeq* seqs = reinterpret_cast<DevSeq*>(img.data() + table_seqs_offset(p->n_cells));
  size_t off = 0;
  for (int c = 0; c < p->n_cells; ++c) {
    cells[c].kind = p->kinds[c];
    cells[c].src = (p->kinds[c] == LOOPKV_SHARE || p->kinds[c] == LOOPKV_RES2) ? p->src(c) : c;
    for (int b = 0; b < p->max_batch; ++b) {
      const size_t stride = unit_layout(p->kinds[c], p->D, p->cap[b]).total;
      DevSeq& s = seqs[(size_t)c * p->max_batch + b];
      s.offset = off;
      s.stride = stride;
      s.cap = p->cap[b];
      s.len = 0;
      p->offset[(size_t)c * p->max_batch + b] = off;
      p->stride[(size_t)c * p->max_batch + b] = stride;
      off += stride * (size_t)p->H;
    }
  }
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  cudaError_t e = cudaMemcpyAsync(d_table, img.data(), img.size(), cudaMemcpyHostToDevice, s);
  if (e == cudaSuccess) e = cudaStreamSynchronize(s);
  if (e != cudaSuccess) {
    delete p;
    return LOOPKV_ERR_CUDA;
  }
  *out = p;
  return LOOPKV_OK;
}

void loopkv_plan_free(loopkv_plan* plan) { delete plan; }

loopkv_status loopkv_append(loopkv_plan* p, const int32_t* h_cells, int32_t n_cells, int32_t batch,
                            const int32_t* h_n_new, int32_t n_new_max, const uint16_t* d_k,
                            const uint16_t* d_v, void* stream) {
  CellList cl{};
  loopkv_status st = check_cells(p, h_cells, n_cells, batch, &cl);
  if (st != LOOPKV_OK) return st;
  if (h_n_new == nullptr || n_new_max < 0) return LOOPKV_ERR_INVALID_ARG;
  bool any = false;
  for (int b = 0; b < batch; ++b) {
    if (h_n_new[b] < 0 || h_n_new[b] > n_new_max) return LOOPKV_ERR_INVALID_ARG;
    any = any || h_n_new[b] > 0;
  }
  if (!any) return LOOPKV_OK;
  if (d_k == nullptr || d_v == nullptr || !aligned16(d_k) || !aligned16(d_v))
    return LOOPKV_ERR_INVALID_ARG;
  for (int i = 0; i < n_cells; ++i) {
    const int c = cl.cell[i];
    if (p->kinds[c] == LOOPKV_SHARE) continue;
    for (int b = 0; b < batch; ++b)
      if ((long long)p->L(c, b) + h_n_new[b] > p->cap[b]) return LOOPKV_ERR_CAPACITY;
  }
  for (int i = 0; i < n_cells; ++i) {
    const int c = cl.cell[i];
    if (p->kinds[c] != LOOPKV_RES2) continue;
    // the reference's groups this append quantizes against must be there
    // already (its length before this call: the kernels run side by side)
    for (int b = 0; b < batch; ++b)
      if (h_n_new[b] > 0 && res2_qtok(p->L(c, b) + h_n_new[b]) > p->ref_positions(c, b))
        return LOOPKV_ERR_INVALID_ARG;
  }
  // RES2 cells go to their own kernel: split the list, keeping each
  // cell's index in the caller's list (its input slot)
  CellList plain{}, res{};
  int n_plain = 0, n_res = 0;
  for (int i = 0; i < n_cells; ++i) {
    CellList& dst = p->kinds[cl.cell[i]] == LOOPKV_RES2 ? res : plain;
    int& k = p->kinds[cl.cell[i]] == LOOPKV_RES2 ? n_res : n_plain;
    dst.cell[k] = cl.cell[i];
    dst.out[k] = i;
    ++k;
  }
  AppendParams ap{};
  ap.table = p->d_table;
  ap.cache = p->d_cache;
  ap.k = d_k;
  ap.v = d_v;
  ap.n_cells = n_cells;
  ap.batch = batch;
  ap.n_heads = p->H;
  ap.n_new_max = n_new_max;
  for (int b = 0; b < batch; ++b) ap.n_new[b] = h_n_new[b];
  // a bulk append (many groups per unit) spreads its groups over several
  // CTAs per unit: at most ceil((n_new_max + 63) / 32) groups become due
  const int groups_max = (n_new_max + 2 * kGroup - 1) / kGroup;
  ap.chunks = (groups_max + kAppendGroupsPerCta - 1) / kAppendGroupsPerCta;
  if (ap.chunks < 1) ap.chunks = 1;
  int e = 0;
  if (n_plain > 0) {
    ap.n_cells = n_plain;
    e = launch_append(ap, plain, stream, p->D, false);
  }
  if (e == 0 && n_res > 0) {
    ap.n_cells = n_res;
    e = launch_append(ap, res, stream, p->D, true);
  }
  if (e != 0) return LOOPKV_ERR_CUDA;
  for (int i = 0; i < n_cells; ++i)
    for (int b = 0; b < batch; ++b) p->L(cl.cell[i], b) += h_n_new[b];
  return LOOPKV_OK;
}

loopkv_status loopkv_decode(loopkv_plan* p, const int32_t* h_cells, int32_t n_cells, int32_t batch,
                            const uint16_t* d_q, float* d_out, float* d_lse, uint32_t* d_mask,
                            int32_t mask_words, int32_t* d_nsel, void* stream) {
  CellList cl{};
  loopkv_status st = check_cells(p, h_cells, n_cells, batch, &cl);
  if (st != LOOPKV_OK) return st;
  if (d_q == nullptr || d_out == nullptr || !aligned16(d_q) || !aligned16(d_out))
    return LOOPKV_ERR_INVALID_ARG;
  int npos_max[2] = {0, 0};  // plain cells, RES2 cells
  CellList lists[2]{};
  int counts[2] = {0, 0};
  for (int i = 0; i < n_cells; ++i) {
    const int c = cl.cell[i];
    const bool share = p->kinds[c] == LOOPKV_SHARE;
    const bool res2 = p->kinds[c] == LOOPKV_RES2;
    const int dkind = (share || res2) ? p->kinds[p->src(c)] : p->kinds[c];
    for (int b = 0; b < batch; ++b) {
      const int n = p->L(c, b);
      if (n < 1) return LOOPKV_ERR_INVALID_ARG;
      int n_att = n, nd = n;
      if (share) {
        n_att = n - 1;
        nd = p->L(p->src(c), b);
        if (n_att > nd) return LOOPKV_ERR_INVALID_ARG;
      }
      int nq = std::min(n_att, nd / kGroup * kGroup);
      if (res2) {
        nq = res2_qtok(n);
        if (nq > p->ref_positions(c, b)) return LOOPKV_ERR_INVALID_ARG;
      }
      if (d_mask != nullptr && dkind == LOOPKV_Q4 && (nq + kGroup - 1) / kGroup > mask_words)
        return LOOPKV_ERR_INVALID_ARG;
      npos_max[res2] = std::max(npos_max[res2], n);
    }
    lists[res2].cell[counts[res2]] = c;
    lists[res2].out[counts[res2]] = i;
    ++counts[res2];
  }
  if (d_mask != nullptr && (mask_words < 0 || !aligned16(d_mask))) return LOOPKV_ERR_INVALID_ARG;
  for (int k = 0; k < 2; ++k) {
    if (counts[k] == 0) continue;
    st = decode_launch(p, lists[k], counts[k], batch, npos_max[k], k == 1, d_q, d_out, d_lse,
                       d_mask, mask_words, d_nsel, stream);
    if (st != LOOPKV_OK) return st;
  }
  return LOOPKV_OK;
}

}  // extern "C"

namespace {

// One decode launch over cells of one sort (all RES2 or none): choose the
// cluster split and the score slots, fill the parameter block, launch.
loopkv_status decode_launch(loopkv_plan* p, const CellList& cl, int n_cells, int batch,
                            int npos_max, bool res2, const uint16_t* d_q, float* d_out,
                            float* d_lse, uint32_t* d_mask, int32_t mask_words, int32_t* d_nsel,
                            void* stream) {
  // Split a unit over a cluster of CTAs when its positions do not fit one
  // CTA's score slots (per query of the group), or when the units fall short
  // of one full wave (two CTAs on each of the 148 SMs): every extra CTA of a
  // unit costs its own start, merge and reduction, which outweighs a fuller
  // last wave once the first wave is full.
  const int max_slots = decode_max_slots(p->D, p->group);
  const long long units = (long long)n_cells * batch * p->H;
  int split = 1;
  auto slots_for = [&](int s) { return ((npos_max + s - 1) / s + 31) / 32 * 32; };
  while (slots_for(split) > max_slots && split < decode_max_split()) split *= 2;
  if (slots_for(split) > max_slots) return LOOPKV_ERR_UNSUPPORTED;
  if (p->min_split > 1) {
    split = std::max(split, p->min_split);
  } else {
    while (units * split < 148 * 2 && split < decode_max_split() && npos_max / (2 * split) >= 512)
      split *= 2;
  }
  DecodeParams dp{};
  dp.table = p->d_table;
  dp.cache = p->d_cache;
  dp.q = d_q;
  dp.out = d_out;
  dp.lse = d_lse;
  dp.mask = d_mask;
  dp.nsel = d_nsel;
  dp.mask_words = mask_words;
  dp.n_cells = n_cells;
  dp.batch = batch;
  dp.n_heads = p->H;
  dp.group = p->group;
  dp.split = split;
  dp.slots = slots_for(split);
  dp.tau = p->tau;
  dp.score_scale = p->sm_scale * 1.4426950408889634f;
  return from_cuda(launch_decode(dp, cl, stream, p->D, res2));
}

}  // namespace

extern "C" {

loopkv_status loopkv_set_lengths(loopkv_plan* p, const int32_t* h_cells, int32_t n_cells,
                                 int32_t batch, const int32_t* h_len, void* stream) {
  CellList cl{};
  loopkv_status st = check_cells(p, h_cells, n_cells, batch, &cl);
  if (st != LOOPKV_OK) return st;
  if (h_len == nullptr) return LOOPKV_ERR_INVALID_ARG;
  for (int i = 0; i < n_cells; ++i) {
    const int c = cl.cell[i];
    for (int b = 0; b < batch; ++b) {
      const int nw = h_len[(size_t)i * batch + b], old = p->L(c, b);
      if (nw == 0) continue;
      if (nw < 0 || nw > old) return LOOPKV_ERR_INVALID_ARG;
      const int k = p->kinds[c];
      if ((k == LOOPKV_Q4 || k == LOOPKV_Q2) && nw < old / kGroup * kGroup && nw % kGroup != 0)
        return LOOPKV_ERR_INVALID_ARG;
      if (k == LOOPKV_SHARE && nw != old) return LOOPKV_ERR_INVALID_ARG;  // current token is gone
      // RES2: the residual-coded count must stay (its bf16 window is gone)
      if (k == LOOPKV_RES2 && res2_qtok(nw) != res2_qtok(old)) return LOOPKV_ERR_INVALID_ARG;
    }
  }
  // Residual slots of a Q4/Q2 unit cut back to a group boundary hold tokens
  // that are now quantized; the next append refills them from slot 0, which
  // is the layout's rule, so no data moves.  Lengths are patched in place.
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  for (int i = 0; i < n_cells; ++i) {
    const int c = cl.cell[i];
    for (int b = 0; b < batch; ++b) {
      const int32_t nw = h_len[(size_t)i * batch + b];
      uint8_t* dst = p->d_table + table_seqs_offset(p->n_cells) +
                     sizeof(DevSeq) * ((size_t)c * p->max_batch + b) + offsetof(DevSeq, len);
      cudaError_t e = cudaMemcpyAsync(dst, &h_len[(size_t)i * batch + b], sizeof(int32_t),
                                      cudaMemcpyHostToDevice, s);
      if (e != cudaSuccess) return LOOPKV_ERR_CUDA;
      p->L(c, b) = nw;
    }
  }
  return from_cuda(cudaStreamSynchronize(s));
}

loopkv_status loopkv_get_lengths(const loopkv_plan* p, int32_t* h_len) {
  if (p == nullptr || h_len == nullptr) return LOOPKV_ERR_INVALID_ARG;
  std::memcpy(h_len, p->len.data(), p->len.size() * sizeof(int32_t));
  return LOOPKV_OK;
}

loopkv_status loopkv_unit_region(const loopkv_plan* p, int32_t cell, int32_t seq, int32_t head,
                                 uint64_t* offset, uint64_t* bytes) {
  if (p == nullptr || offset == nullptr || bytes == nullptr) return LOOPKV_ERR_INVALID_ARG;
  if (cell < 0 || cell >= p->n_cells || seq < 0 || seq >= p->max_batch || head < 0 || head >= p->H)
    return LOOPKV_ERR_INVALID_ARG;
  const size_t i = (size_t)cell * p->max_batch + seq;
  *offset = p->offset[i] + (uint64_t)head * p->stride[i];
  *bytes = p->stride[i];
  return LOOPKV_OK;
}

loopkv_status loopkv_check(loopkv_plan* p, void* stream) {
  if (p == nullptr) return LOOPKV_ERR_INVALID_ARG;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (cudaStreamSynchronize(s) != cudaSuccess) return LOOPKV_ERR_CUDA;
  uint32_t status = 0;
  if (cudaMemcpy(&status, p->d_table, sizeof(status), cudaMemcpyDeviceToHost) != cudaSuccess)
    return LOOPKV_ERR_CUDA;
  if (status == 0) return LOOPKV_OK;
  const uint32_t zero = 0;
  if (cudaMemcpy(p->d_table, &zero, sizeof(zero), cudaMemcpyHostToDevice) != cudaSuccess)
    return LOOPKV_ERR_CUDA;
  return LOOPKV_ERR_DEVICE;
}

const char* loopkv_status_string(loopkv_status s) {
  switch (s) {
    case LOOPKV_OK: return "ok";
    case LOOPKV_ERR_INVALID_ARG: return "invalid argument";
    case LOOPKV_ERR_PLAN: return "invalid plan";
    case LOOPKV_ERR_CAPACITY: return "append exceeds a unit's capacity";
    case LOOPKV_ERR_UNSUPPORTED: return "unsupported request";
    case LOOPKV_ERR_CUDA: return "CUDA error";
    case LOOPKV_ERR_DEVICE: return "device-side inconsistency flagged";
  }
  return "unknown status";
}

}  // extern "C"
