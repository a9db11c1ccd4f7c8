// LoopKV cache append for sm_100a: quantize, split into bit planes, store.
//
// "LoopKV: Loop-Aware KV Cache Compression for Serving Looped Transformers",
// section 概要: a cell keeps 4-bit storage (read as a high and a low 2-bit
// plane), 2-bit storage, or reuses the final loop's KV.  Quantization is
// asymmetric min/max as in "KIVI: A Tuning-Free Asymmetric 2bit
// Quantization for KV Cache": keys per channel over a group of 32 tokens,
// values per token over groups of 32 channels; the fp32 steps
//   scale = (max - min) / qmax,  code = rne((x - min) / scale)
// are done with explicit round-to-nearest intrinsics (no contraction), so the
// codes are the ones any IEEE implementation of the same steps produces.
//
// One CTA per (cell, sequence, head) unit (several for a bulk append).
// New tokens fill the bf16 residual; every 32-position group that becomes
// complete is quantized by one warp through a padded shared-memory tile,
// then the remaining tokens are written to the residual.  The CTAs of a
// (cell, sequence) pair all read its old length; the last of them to finish
// stores the new one (an arrival count in the plan table), so no second
// launch is needed.

#include <cuda_runtime.h>

#include <cstdint>

#include "loopkv_internal.cuh"

namespace loopkv {
namespace {

constexpr int kAppendThreads = 128;
constexpr int kAppendWarps = kAppendThreads / 32;

// Quantize x (fp32) of a 32-value group: returns the code, given the
// group's min, scale and inv = rn(1 / scale).  scale == 0 gives 0.
// The code is rne(q) of the IEEE quotient q = rn(x - mn) / scale without a
// division per code: with a normal inv, r = rn(rn(x - mn) * inv) differs
// from q by less than 2^-23 relative, i.e. by less than 2^-19 for
// q <= 15 (q <= qmax (1 + 2^-24) since scale = rn(range / qmax)), so
// rne(r) = rne(q) unless r lies within 2^-19 of a half-integer; there (the
// test uses 2^-16) the exact quotient is taken.  r - floor(r) and its
// distance to 0.5 are exact (Sterbenz), and a NaN or infinite r falls back
// too, so the codes equal the division's for every input.
__device__ __forceinline__ uint32_t quant_code(float x, float mn, float scale, float inv, int qmax) {
  if (scale == 0.0f) return 0u;
  const float d = __fsub_rn(x, mn);
  float r = __fmul_rn(d, inv);
  const float f = __fsub_rn(r, floorf(r));
  if (!(fabsf(__fsub_rn(f, 0.5f)) > 0x1p-16f) || !(inv >= 0x1p-125f)) r = __fdiv_rn(d, scale);
  int c = __float2int_rn(r);  // round half to even
  c = c < 0 ? 0 : (c > qmax ? qmax : c);
  return (uint32_t)c;
}

// A zero range stores scale +0 whatever the signs of zero min / max.
__device__ __forceinline__ float group_scale(float mn, float mx, int qmax) {
  const float range = __fsub_rn(mx, mn);
  return range == 0.0f ? 0.0f : __fdiv_rn(range, (float)qmax);
}

__device__ __forceinline__ float canon_zero(float mn) { return mn == 0.0f ? 0.0f : mn; }

__device__ __forceinline__ float bf16f(uint16_t b) { return __uint_as_float((uint32_t)b << 16); }

// The length commit of a (cell, sequence) pair: each of its `expected` CTAs
// arrives once it is done; the last one stores n_old + n_new and resets the
// count for the next launch.  Every CTA read the old length before it
// arrived, so none of them sees the new one.
__device__ __forceinline__ void arrive_commit(DevSeq* e, int n_old, int n_new, unsigned expected) {
  __syncthreads();
  if (threadIdx.x == 0) {
    __threadfence();
    if (atomicAdd(&e->arrive, 1u) == expected - 1u) {
      e->len = n_old + n_new;
      e->arrive = 0u;
    }
  }
}

constexpr int kCodeRow = 16;  // padding bytes of a code-tile row (D + 16 bytes)

// Keys of one 32-token group: per channel over the tokens (x(t, d), fp32),
// the channel's scale and zero point into kmeta (scale[D] then zero[D]) and
// its codes into the warp's code tile ([32][D + 16] bytes).  Lane d owns
// channels d, d + 32, ...
template <int D, typename X>
__device__ __forceinline__ void quantize_key_group(X x, uint8_t* codes, float* kmeta, int qmax,
                                                   int lane) {
#pragma unroll
  for (int i = 0; i < D / 32; ++i) {
    const int d = lane + 32 * i;
    float mn = x(0, d), mx = mn;
    for (int t = 1; t < 32; ++t) {
      mn = fminf(mn, x(t, d));
      mx = fmaxf(mx, x(t, d));
    }
    const float sc = group_scale(mn, mx, qmax);
    const float inv = sc == 0.0f ? 0.0f : __frcp_rn(sc);
    for (int t = 0; t < 32; ++t)
      codes[t * (D + kCodeRow) + d] = (uint8_t)quant_code(x(t, d), mn, sc, inv, qmax);
    kmeta[d] = sc;
    kmeta[D + d] = canon_zero(mn);
  }
}

// The code tile's row of token `lane` into the group's key planes: chunk c
// of 64 channels -> 4 words per plane at hi + c * 512 + lane * 16 (lo: the
// low plane, 4-bit only; a 2-bit code goes whole into hi).
template <int D>
__device__ __forceinline__ void pack_key_planes(const uint8_t* codes, uint8_t* hi, uint8_t* lo,
                                                bool q4, int lane) {
#pragma unroll
  for (int cc = 0; cc < D / 64; ++cc) {
    uint32_t hiw[4], low[4];
#pragma unroll
    for (int w = 0; w < 4; ++w) {
      const uint4 cw = *reinterpret_cast<const uint4*>(codes + lane * (D + kCodeRow) + 64 * cc + 16 * w);
      const uint32_t bytes[4] = {cw.x, cw.y, cw.z, cw.w};
      uint32_t hv = 0, lv = 0;
#pragma unroll
      for (int j = 0; j < 16; ++j) {
        const uint32_t q = (bytes[j / 4] >> (8 * (j % 4))) & 0xFFu;
        hv |= ((q4 ? (q >> 2) : q) & 3u) << (2 * j);
        lv |= (q & 3u) << (2 * j);
      }
      hiw[w] = hv;
      low[w] = lv;
    }
    const size_t off = cc * 512 + lane * 16;
    *reinterpret_cast<uint4*>(hi + off) = make_uint4(hiw[0], hiw[1], hiw[2], hiw[3]);
    if (q4) *reinterpret_cast<uint4*>(lo + off) = make_uint4(low[0], low[1], low[2], low[3]);
  }
}

// Values of one token: per group of 32 channels (v(c), fp32 of channel c)
// the scale / zero pair and the codes, written as the token's V_hi (V_lo,
// 4-bit) words and V_meta row (channel 16w + j of a row in bits 2j..2j+1
// of word w).
template <int D, typename V>
__device__ __forceinline__ void quantize_value_row(V v, bool q4, int qmax, uint4* vh, uint4* vl,
                                                   float4* vm) {
  uint32_t hiw[D / 16], low[D / 16];
  float meta[D / 16];
#pragma unroll
  for (int j = 0; j < D / 32; ++j) {
    float mn = v(32 * j), mx = mn;
#pragma unroll
    for (int e = 1; e < 32; ++e) {
      mn = fminf(mn, v(32 * j + e));
      mx = fmaxf(mx, v(32 * j + e));
    }
    const float sc = group_scale(mn, mx, qmax);
    const float inv = sc == 0.0f ? 0.0f : __frcp_rn(sc);
    uint32_t hv0 = 0, lv0 = 0, hv1 = 0, lv1 = 0;
#pragma unroll
    for (int e = 0; e < 32; ++e) {
      const uint32_t q = quant_code(v(32 * j + e), mn, sc, inv, qmax);
      const uint32_t h = (q4 ? (q >> 2) : q) & 3u, l = q & 3u;
      if (e < 16) {
        hv0 |= h << (2 * e);
        lv0 |= l << (2 * e);
      } else {
        hv1 |= h << (2 * (e - 16));
        lv1 |= l << (2 * (e - 16));
      }
    }
    hiw[2 * j] = hv0;
    hiw[2 * j + 1] = hv1;
    low[2 * j] = lv0;
    low[2 * j + 1] = lv1;
    meta[2 * j] = sc;
    meta[2 * j + 1] = canon_zero(mn);
  }
#pragma unroll
  for (int i = 0; i < D / 64; ++i) {
    vh[i] = make_uint4(hiw[4 * i], hiw[4 * i + 1], hiw[4 * i + 2], hiw[4 * i + 3]);
    if (q4) vl[i] = make_uint4(low[4 * i], low[4 * i + 1], low[4 * i + 2], low[4 * i + 3]);
    vm[i] = make_float4(meta[4 * i], meta[4 * i + 1], meta[4 * i + 2], meta[4 * i + 3]);
  }
}

template <int D>
__global__ void __launch_bounds__(kAppendThreads)
append_kernel(const AppendParams p, const CellList cl) {
  require_ieee_subnormals();
  constexpr int TROW = D + 2;     // bf16 per padded tile row
  constexpr int CROW = D + kCodeRow;  // bytes per padded code row
  extern __shared__ __align__(16) uint8_t sm[];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  uint16_t* tk = reinterpret_cast<uint16_t*>(sm) + warp * (2 * 32 * TROW);
  uint16_t* tv = tk + 32 * TROW;
  uint8_t* codes = sm + kAppendWarps * (2 * 32 * TROW) * 2 + warp * (32 * CROW);

  const int H = p.n_heads;
  const int chunk = blockIdx.x % p.chunks;  // this CTA's share of the unit's groups / rows
  const int unit = blockIdx.x / p.chunks;
  const int h = unit % H;
  const int b = (unit / H) % p.batch;
  const int ci = unit / (H * p.batch);
  const int cell = cl.cell[ci];
  const int n_new = p.n_new[b];
  if (n_new <= 0) return;

  const TableHeader* hdr = reinterpret_cast<const TableHeader*>(p.table);
  const DevCell* cells = reinterpret_cast<const DevCell*>(p.table + table_cells_offset());
  DevSeq* seqs = reinterpret_cast<DevSeq*>(p.table + table_seqs_offset(hdr->n_cells));
  const DevCell c = cells[cell];
  DevSeq* const entry = seqs + (size_t)cell * hdr->max_batch + b;
  const DevSeq s = *entry;
  const int kind = c.kind;
  const int n_old = s.len;
  if (n_old < 0 || (kind != LOOPKV_SHARE && n_old + n_new > s.cap)) {
    // host checks make this unreachable; flag it, leave the unit and its
    // length alone (every CTA of the pair takes this branch)
    if (threadIdx.x == 0 && chunk == 0) atomicOr(reinterpret_cast<uint32_t*>(p.table), kStatusLength);
    return;
  }
  const unsigned expected = (unsigned)(H * p.chunks);
  uint8_t* base = p.cache + s.offset + (size_t)h * s.stride;
  const UnitLayout L = unit_layout(kind, D, s.cap);
  const size_t in_off = (((size_t)cl.out[ci] * p.batch + b) * H + h) * (size_t)p.n_new_max * D;
  const uint16_t* kin = p.k + in_off;
  const uint16_t* vin = p.v + in_off;

  if (kind == LOOPKV_SHARE) {
    if (chunk == 0) {
      // keep only the last appended token as the current one
      const uint4* ks = reinterpret_cast<const uint4*>(kin + (size_t)(n_new - 1) * D);
      const uint4* vs = reinterpret_cast<const uint4*>(vin + (size_t)(n_new - 1) * D);
      for (int i = threadIdx.x; i < D / 8; i += kAppendThreads) {
        reinterpret_cast<uint4*>(base + L.cur_k)[i] = ks[i];
        reinterpret_cast<uint4*>(base + L.cur_v)[i] = vs[i];
      }
    }
    arrive_commit(entry, n_old, n_new, expected);
    return;
  }
  if (kind == LOOPKV_BF16) {
    // rows split evenly over the unit's CTAs
    const int per = (n_new + p.chunks - 1) / p.chunks;
    const int t0 = chunk * per, t1 = min(n_new, t0 + per);
    uint4* kd = reinterpret_cast<uint4*>(base + L.raw_k + (size_t)n_old * D * 2);
    uint4* vd = reinterpret_cast<uint4*>(base + L.raw_v + (size_t)n_old * D * 2);
    for (size_t i = (size_t)t0 * (D / 8) + threadIdx.x; i < (size_t)max(t1, t0) * (D / 8);
         i += kAppendThreads) {
      const size_t t = i / (D / 8), cc = i % (D / 8);
      kd[i] = reinterpret_cast<const uint4*>(kin + t * D)[cc];
      vd[i] = reinterpret_cast<const uint4*>(vin + t * D)[cc];
    }
    arrive_commit(entry, n_old, n_new, expected);
    return;
  }

  const bool q4 = kind == LOOPKV_Q4;
  const int qmax = q4 ? 15 : 3;
  const int qtok0 = n_old / kGroup * kGroup;
  const int n1 = n_old + n_new;
  const int qtok1 = n1 / kGroup * kGroup;
  const uint16_t* resk = reinterpret_cast<const uint16_t*>(base + L.res_k);
  const uint16_t* resv = reinterpret_cast<const uint16_t*>(base + L.res_v);
  // this CTA's groups; only the first group reads the old residual, and it
  // is in chunk 0, which also writes the new residual afterwards
  const int gb = qtok0 / kGroup + chunk * kAppendGroupsPerCta;
  const int ge = min(qtok1 / kGroup, gb + kAppendGroupsPerCta);

  for (int g = gb + warp; g < ge; g += kAppendWarps) {
    // gather the group's 32 tokens: residual slots first, then new tokens
    for (int i = lane; i < 32 * (D / 2); i += 32) {
      const int t = i / (D / 2), cc = i % (D / 2);
      const int pos = g * kGroup + t;
      const uint32_t* ksrc;
      const uint32_t* vsrc;
      if (pos < n_old) {
        ksrc = reinterpret_cast<const uint32_t*>(resk + (size_t)(pos - qtok0) * D);
        vsrc = reinterpret_cast<const uint32_t*>(resv + (size_t)(pos - qtok0) * D);
      } else {
        ksrc = reinterpret_cast<const uint32_t*>(kin + (size_t)(pos - n_old) * D);
        vsrc = reinterpret_cast<const uint32_t*>(vin + (size_t)(pos - n_old) * D);
      }
      reinterpret_cast<uint32_t*>(tk + t * TROW)[cc] = ksrc[cc];
      reinterpret_cast<uint32_t*>(tv + t * TROW)[cc] = vsrc[cc];
    }
    __syncwarp();

    // keys: per channel over the 32 tokens
    quantize_key_group<D>([&](int t, int d) { return bf16f(tk[t * TROW + d]); }, codes,
                          reinterpret_cast<float*>(base + L.k_meta + (size_t)g * 8 * D), qmax,
                          lane);
    __syncwarp();
    pack_key_planes<D>(codes, base + L.k_hi + (size_t)g * 8 * D, base + L.k_lo + (size_t)g * 8 * D,
                       q4, lane);
    // values: lane = token, per group of 32 channels
    {
      const size_t tpos = (size_t)g * kGroup + lane;
      const uint16_t* row = tv + lane * TROW;
      quantize_value_row<D>([&](int c) { return bf16f(row[c]); }, q4, qmax,
                            reinterpret_cast<uint4*>(base + L.v_hi + tpos * (D / 4)),
                            reinterpret_cast<uint4*>(base + L.v_lo + tpos * (D / 4)),
                            reinterpret_cast<float4*>(base + L.v_meta + tpos * (D / 4)));
    }
    __syncwarp();
  }
  __syncthreads();  // flushed groups have read the old residual
  if (chunk != 0) {
    arrive_commit(entry, n_old, n_new, expected);
    return;
  }

  // remaining tokens go to the residual
  const int r_first = (qtok1 > qtok0) ? qtok1 : n_old;  // first position to write
  uint8_t* rk = base + L.res_k;
  uint8_t* rv = base + L.res_v;
  const int nres = n1 - r_first;
  for (int i = threadIdx.x; i < nres * (D / 8); i += kAppendThreads) {
    const int t = i / (D / 8), cc = i % (D / 8);
    const int pos = r_first + t;
    const int slot = pos - qtok1;
    reinterpret_cast<uint4*>(rk + (size_t)slot * D * 2)[cc] =
        reinterpret_cast<const uint4*>(kin + (size_t)(pos - n_old) * D)[cc];
    reinterpret_cast<uint4*>(rv + (size_t)slot * D * 2)[cc] =
        reinterpret_cast<const uint4*>(vin + (size_t)(pos - n_old) * D)[cc];
  }
  arrive_commit(entry, n_old, n_new, expected);
}

// The reference's stored key / value at (pos, d) dequantized in fp32, the
// way a residual is taken against it: fl(fl(scale * q) + zero) with the full
// code q of a 4-bit or 2-bit reference, the raw value of a bf16 one.
__device__ float ref_key32(const uint8_t* rb, const UnitLayout& RL, int rkind, int pos, int d,
                           int D) {
  if (rkind == LOOPKV_BF16)
    return bf16f(*reinterpret_cast<const uint16_t*>(rb + RL.raw_k + ((size_t)pos * D + d) * 2));
  const int g = pos / kGroup, t = pos % kGroup, c = d / 64, w = (d % 64) / 16, j = d % 16;
  const size_t off = (size_t)g * 8 * D + c * 512 + t * 16 + w * 4;
  uint32_t q = (*reinterpret_cast<const uint32_t*>(rb + RL.k_hi + off) >> (2 * j)) & 3u;
  if (rkind == LOOPKV_Q4)
    q = 4u * q + ((*reinterpret_cast<const uint32_t*>(rb + RL.k_lo + off) >> (2 * j)) & 3u);
  const float* meta = reinterpret_cast<const float*>(rb + RL.k_meta + (size_t)g * 8 * D);
  return __fadd_rn(__fmul_rn(meta[d], (float)q), meta[D + d]);
}

__device__ float ref_value32(const uint8_t* rb, const UnitLayout& RL, int rkind, int pos, int d,
                             int D) {
  if (rkind == LOOPKV_BF16)
    return bf16f(*reinterpret_cast<const uint16_t*>(rb + RL.raw_v + ((size_t)pos * D + d) * 2));
  const size_t row = (size_t)pos * (D / 4);
  const int w = d / 16, j = d % 16;
  uint32_t q = (*reinterpret_cast<const uint32_t*>(rb + RL.v_hi + row + w * 4) >> (2 * j)) & 3u;
  if (rkind == LOOPKV_Q4)
    q = 4u * q + ((*reinterpret_cast<const uint32_t*>(rb + RL.v_lo + row + w * 4) >> (2 * j)) & 3u);
  const float* m = reinterpret_cast<const float*>(rb + RL.v_meta + row + (d / kGroup) * 8);
  return __fadd_rn(__fmul_rn(m[0], (float)q), m[1]);
}

// Append to RES2 units (2-bit residuals against the final loop's KV:
// "ResidualQuant: KV Cache Quantization for Looped Transformers with 2-Bit
// Residuals", as summarised in the related-paper list (関連論文リスト) of the
// page "LoopVQ: Sub 1-bit KV Cache Quantization for Looped Transformers").
// One CTA per unit.  Tokens live in a 64-slot bf16 window (position t in
// slot t mod 64); residual group g is quantized when
// the unit reaches 32 (g + 2) tokens: each warp takes a group, forms the
// residuals x - r in an fp32 tile (r: the reference's stored value, read
// from its planes) and quantizes them at 2 bits exactly as a Q2 cell's
// tokens (keys per channel, values per token per 32 channels).  Window
// slots are written after every group has read them.
template <int D>
__global__ void __launch_bounds__(kAppendThreads)
append_res2_kernel(const AppendParams p, const CellList cl) {
  require_ieee_subnormals();
  constexpr int XROW = D + 1;     // fp32 per padded tile row
  constexpr int CROW = D + kCodeRow;  // bytes per padded code row
  extern __shared__ __align__(16) uint8_t sm[];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  float* xk = reinterpret_cast<float*>(sm) + warp * (2 * 32 * XROW);
  float* xv = xk + 32 * XROW;
  uint8_t* codes = sm + (size_t)kAppendWarps * (2 * 32 * XROW) * 4 + warp * (32 * CROW);

  const int H = p.n_heads;
  const int chunk = blockIdx.x % p.chunks;  // this CTA's share of the unit's groups
  const int unit = blockIdx.x / p.chunks;
  const int h = unit % H;
  const int b = (unit / H) % p.batch;
  const int ci = unit / (H * p.batch);
  const int cell = cl.cell[ci];
  const int n_new = p.n_new[b];
  if (n_new <= 0) return;

  const TableHeader* hdr = reinterpret_cast<const TableHeader*>(p.table);
  const DevCell* cells = reinterpret_cast<const DevCell*>(p.table + table_cells_offset());
  DevSeq* seqs = reinterpret_cast<DevSeq*>(p.table + table_seqs_offset(hdr->n_cells));
  const DevCell c = cells[cell];
  DevSeq* const entry = seqs + (size_t)cell * hdr->max_batch + b;
  const DevSeq s = *entry;
  const DevCell rc = cells[c.src];
  const DevSeq rs = seqs[(size_t)c.src * hdr->max_batch + b];
  const int rkind = rc.kind;
  const int n_old = s.len;
  const int n1 = n_old + n_new;
  const int q0 = res2_qtok(n_old), q1 = res2_qtok(n1);
  const int ref_pos = rkind == LOOPKV_BF16 ? rs.len : rs.len / kGroup * kGroup;
  const bool ref_ok = rkind == LOOPKV_Q4 || rkind == LOOPKV_Q2 || rkind == LOOPKV_BF16;
  if (c.kind != LOOPKV_RES2 || !ref_ok || n_old < 0 || n1 > s.cap || q1 > ref_pos) {
    // host checks make this unreachable; flag it and leave the unit alone
    if (threadIdx.x == 0 && chunk == 0) atomicOr(reinterpret_cast<uint32_t*>(p.table), kStatusLength);
    return;
  }
  const unsigned expected = (unsigned)(H * p.chunks);
  uint8_t* base = p.cache + s.offset + (size_t)h * s.stride;
  const uint8_t* rbase = p.cache + rs.offset + (size_t)h * rs.stride;
  const UnitLayout L = unit_layout(LOOPKV_RES2, D, s.cap);
  const UnitLayout RL = unit_layout(rkind, D, rs.cap);
  const size_t in_off = (((size_t)cl.out[ci] * p.batch + b) * H + h) * (size_t)p.n_new_max * D;
  const uint16_t* kin = p.k + in_off;
  const uint16_t* vin = p.v + in_off;
  const uint16_t* wk = reinterpret_cast<const uint16_t*>(base + L.res_k);
  const uint16_t* wv = reinterpret_cast<const uint16_t*>(base + L.res_v);

  // this CTA's groups; the ones that read the old window (at most two) are
  // in chunk 0, which also writes the window afterwards
  const int gb = q0 / kGroup + chunk * kAppendGroupsPerCta;
  const int ge = min(q1 / kGroup, gb + kAppendGroupsPerCta);
  for (int g = gb + warp; g < ge; g += kAppendWarps) {
    // residuals of the group's 32 tokens (window slots or new tokens)
    for (int i = lane; i < 32 * D; i += 32) {
      const int t = i / D, d = i % D;
      const int pos = g * kGroup + t;
      const uint16_t kx = pos < n_old ? wk[(size_t)(pos % kResWindow) * D + d]
                                      : kin[(size_t)(pos - n_old) * D + d];
      const uint16_t vx = pos < n_old ? wv[(size_t)(pos % kResWindow) * D + d]
                                      : vin[(size_t)(pos - n_old) * D + d];
      xk[t * XROW + d] = __fsub_rn(bf16f(kx), ref_key32(rbase, RL, rkind, pos, d, D));
      xv[t * XROW + d] = __fsub_rn(bf16f(vx), ref_value32(rbase, RL, rkind, pos, d, D));
    }
    __syncwarp();

    // keys: per channel over the 32 tokens, then values per token, at 2 bits
    quantize_key_group<D>([&](int t, int d) { return xk[t * XROW + d]; }, codes,
                          reinterpret_cast<float*>(base + L.k_meta + (size_t)g * 8 * D), 3, lane);
    __syncwarp();
    pack_key_planes<D>(codes, base + L.k_hi + (size_t)g * 8 * D, nullptr, false, lane);
    {
      const size_t tpos = (size_t)g * kGroup + lane;
      const float* row = xv + lane * XROW;
      quantize_value_row<D>([&](int c) { return row[c]; }, false, 3,
                            reinterpret_cast<uint4*>(base + L.v_hi + tpos * (D / 4)), nullptr,
                            reinterpret_cast<float4*>(base + L.v_meta + tpos * (D / 4)));
    }
    __syncwarp();
  }
  __syncthreads();  // every group has read its window slots
  if (chunk != 0) {
    arrive_commit(entry, n_old, n_new, expected);
    return;
  }

  // new tokens past the residual-coded range go to their window slots
  const int first = n_old > q1 ? n_old : q1;
  uint8_t* rk = base + L.res_k;
  uint8_t* rv = base + L.res_v;
  for (int i = threadIdx.x; i < (n1 - first) * (D / 8); i += kAppendThreads) {
    const int t = i / (D / 8), cc = i % (D / 8);
    const int pos = first + t;
    const size_t slot = (size_t)(pos % kResWindow) * D * 2;
    reinterpret_cast<uint4*>(rk + slot)[cc] =
        reinterpret_cast<const uint4*>(kin + (size_t)(pos - n_old) * D)[cc];
    reinterpret_cast<uint4*>(rv + slot)[cc] =
        reinterpret_cast<const uint4*>(vin + (size_t)(pos - n_old) * D)[cc];
  }
  arrive_commit(entry, n_old, n_new, expected);
}

template <int D>
size_t append_smem() {
  return (size_t)kAppendWarps * (2 * 32 * (D + 2) * 2 + 32 * (D + 16));
}
template <int D>
size_t append_res2_smem() {
  return (size_t)kAppendWarps * (2 * 32 * (D + 1) * 4 + 32 * (D + 16));
}

template <int D>
int launch_append_t(const AppendParams& p, const CellList& cells, cudaStream_t stream, bool res2) {
  const size_t smem = res2 ? append_res2_smem<D>() : append_smem<D>();
  auto kern = res2 ? append_res2_kernel<D> : append_kernel<D>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return (int)e;
  const long long units = (long long)p.n_cells * p.batch * p.n_heads;
  kern<<<(unsigned)(units * p.chunks), kAppendThreads, smem, stream>>>(p, cells);
  return (int)cudaGetLastError();
}

}  // namespace

int launch_append(const AppendParams& p, const CellList& cells, void* stream, int head_dim,
                  bool res2) {
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (head_dim == 64) return launch_append_t<64>(p, cells, s, res2);
  return launch_append_t<128>(p, cells, s, res2);
}

}  // namespace loopkv
