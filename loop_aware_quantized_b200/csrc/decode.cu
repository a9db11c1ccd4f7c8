// LoopKV fused decode attention for sm_100a.
//
// "LoopKV: Loop-Aware KV Cache Compression for Serving Looped Transformers",
// section 概要: each loop reads the high 2 bits of every 4-bit value and
// fetches the low 2 bits only where its own attention weights require 4-bit
// precision; one fused kernel runs the per-cell plan.
//
// One CTA (8 warps) handles a contiguous, 32-aligned range of one unit's
// attended positions for the G query heads that share the unit's KV head
// (G = 1, 2 or 4); when a unit is split over several CTAs they form a
// thread-block cluster and exchange their partial softmax statistics and
// partial outputs through distributed shared memory, so no global
// workspace is needed.  The scores of the CTA's range stay in shared memory
// between the two passes:
//   pass 1  keys: per 32-token group, each query is folded with the group's
//           per-channel key scales (qs_d = q_d * scale_d) and zero points
//           (c = sum_d q_d * zero_d), then each lane (one token) unpacks its
//           packed planes once and forms sum_d qs_d * code_d + c for every
//           query.  Scores are kept in log2 units.
//   softmax per query: the CTA's max and sum of exponentials, merged across
//           the cluster into the unit's logsumexp.
//   pass 2  values: lane = position computes p for every query and the
//           selection (some query has p >= tau; a warp ballot gives the
//           mask word of the group); lanes then work per token ((D / 64) G
//           lanes of 64 / G channels) accumulating p * scale * code in fp32
//           for every query and the per-group constant
//           p * (zero [+ 1.5 * scale]) separately; the low plane row of a
//           token is loaded only when the token is selected.
//   combine warp shuffles reduce the per-token partial outputs, shared
//           memory reduces across warps, DSMEM across the cluster.
// Each pass loads a warp's next group into registers while the current one
// is processed and requests its lines into L2 at the same time; with four
// queries per KV head the value blocks go through shared-memory staging
// buffers filled by cp.async instead (no registers to spare).  A RES2 unit
// (template flag, its own launch) runs both passes over its reference and
// adds its own 2-bit residual planes.
// No tensor cores: single-query decode is not a dense contraction; the
// kernel streams the cache once, and the ALU pipe (one logic op per code)
// is what bounds it in practice.

#include <cooperative_groups.h>
#include <cuda_runtime.h>

#include <cstdint>

#include "loopkv_internal.cuh"

namespace cg = cooperative_groups;

namespace loopkv {
namespace {

constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;
constexpr int kMaxSlots = 24576;  // score slots per CTA (96 KB)
constexpr int kMaxSplit = 8;      // portable cluster size
constexpr int kListCap = 64;      // per-warp list of selected positions awaiting their low plane

__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

__device__ __forceinline__ uint4 ldg128(const void* p) {
  return __ldg(reinterpret_cast<const uint4*>(p));
}
__device__ __forceinline__ float4 ldg128f(const void* p) {
  return __ldg(reinterpret_cast<const float4*>(p));
}

// Stream-once loads of the cache: no reuse, keep them out of L1.
__device__ __forceinline__ uint4 ld_stream(const void* p) {
  uint4 r;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
               : "l"(p));
  return r;
}

__device__ __forceinline__ uint2 ld_stream2(const void* p) {
  uint2 r;
  asm volatile("ld.global.nc.L1::no_allocate.v2.u32 {%0,%1}, [%2];" : "=r"(r.x), "=r"(r.y) : "l"(p));
  return r;
}
__device__ __forceinline__ uint32_t ld_stream1(const void* p) {
  uint32_t r;
  asm volatile("ld.global.nc.L1::no_allocate.u32 %0, [%1];" : "=r"(r) : "l"(p));
  return r;
}

// Packed fp32 pair arithmetic (sm_100): one instruction for two lanes of
// work.  Round to nearest, no flush to zero.
__device__ __forceinline__ float2 add2(float2 a, float2 b) {
  float2 d;
  asm("add.f32x2 %0, %1, %2;"
      : "=l"(reinterpret_cast<unsigned long long&>(d))
      : "l"(reinterpret_cast<unsigned long long&>(a)),
        "l"(reinterpret_cast<unsigned long long&>(b)));
  return d;
}
__device__ __forceinline__ float2 fma2(float2 a, float2 b, float2 c) {
  float2 d;
  asm("fma.rn.f32x2 %0, %1, %2, %3;"
      : "=l"(reinterpret_cast<unsigned long long&>(d))
      : "l"(reinterpret_cast<unsigned long long&>(a)),
        "l"(reinterpret_cast<unsigned long long&>(b)),
        "l"(reinterpret_cast<unsigned long long&>(c)));
  return d;
}

// Codes to floats, exactly, at one logic op per code.  A field of `bits`
// bits at bit offset `off` (off + bits <= 23) of a word, masked in place so
// that the float's exponent field stays zero, is the subnormal float
// code * 2^(off - 149): exact, with no implicit leading one to cancel.  The
// weights carry 2^(kSub - off), so every product is an ordinary normal float
// code * weight * 2^(kSub - 149); the FMA units take subnormal operands at
// full rate and the build keeps them (no flush to zero).  Keys fold
// 2^(kSub - off) into the folded query, values carry 2^kSub in their weights
// and remove 2^(off + kSub - 149) from each channel's accumulator at the end.
constexpr int kSub = 100;

template <int off, int bits>
__device__ __forceinline__ float field_f(uint32_t w) {
  static_assert(off + bits <= 23, "field must stay inside the mantissa");
  return __uint_as_float(w & (((1u << bits) - 1u) << off));
}

// 16 two-bit codes of w (code j in bits 2j..2j+1) -> 8 pairs
// (code 2i * 2^(o(2i) - 149), code 2i+1 * 2^(o(2i+1) - 149)),
// o(j) = 2j for j < 6, 2(j-6) else.
__device__ __forceinline__ void codes2_to_pairs(uint32_t w, float2 (&out)[8]) {
  const uint32_t y = w >> 12;
  out[0] = make_float2(field_f<0, 2>(w), field_f<2, 2>(w));
  out[1] = make_float2(field_f<4, 2>(w), field_f<6, 2>(w));
  out[2] = make_float2(field_f<8, 2>(w), field_f<10, 2>(w));
  out[3] = make_float2(field_f<0, 2>(y), field_f<2, 2>(y));
  out[4] = make_float2(field_f<4, 2>(y), field_f<6, 2>(y));
  out[5] = make_float2(field_f<8, 2>(y), field_f<10, 2>(y));
  out[6] = make_float2(field_f<12, 2>(y), field_f<14, 2>(y));
  out[7] = make_float2(field_f<16, 2>(y), field_f<18, 2>(y));
}
// Bit offset a two-bit code j of a word ends up at in codes2_to_pairs.
__host__ __device__ constexpr int code2_off(int j) { return j < 6 ? 2 * j : 2 * (j - 6); }

// Hi and lo planes of 16 four-bit codes -> 8 pairs (q_2m * 2^(o(m) - 149),
// q_2m+1 * 2^(o(m) - 149)), q = 4hi + lo, o(m) = 4m for m < 3, 4(m-3) else.
// The planes are merged into a word of even codes (nibble m = code 2m) and
// one of odd codes.
__device__ __forceinline__ void codes4_to_pairs(uint32_t hi, uint32_t lo, float2 (&out)[8]) {
  const uint32_t even = ((hi << 2) & 0xCCCCCCCCu) | (lo & 0x33333333u);
  const uint32_t odd = (hi & 0xCCCCCCCCu) | ((lo >> 2) & 0x33333333u);
  const uint32_t eh = even >> 12, oh = odd >> 12;
  out[0] = make_float2(field_f<0, 4>(even), field_f<0, 4>(odd));
  out[1] = make_float2(field_f<4, 4>(even), field_f<4, 4>(odd));
  out[2] = make_float2(field_f<8, 4>(even), field_f<8, 4>(odd));
  out[3] = make_float2(field_f<0, 4>(eh), field_f<0, 4>(oh));
  out[4] = make_float2(field_f<4, 4>(eh), field_f<4, 4>(oh));
  out[5] = make_float2(field_f<8, 4>(eh), field_f<8, 4>(oh));
  out[6] = make_float2(field_f<12, 4>(eh), field_f<12, 4>(oh));
  out[7] = make_float2(field_f<16, 4>(eh), field_f<16, 4>(oh));
}
__host__ __device__ constexpr int code4_off(int m) { return m < 3 ? 4 * m : 4 * (m - 3); }

// Streams run ahead of use: a warp's next group is loaded into registers
// while the current one is processed, and its lines are also requested
// into L2 (prefetch.global.L2) right after those loads.
constexpr int kAheadK = 1;
constexpr int kAheadV = 1;

__device__ __forceinline__ void prefetch_l2(const void* p) {
  asm volatile("prefetch.global.L2 [%0];" ::"l"(p));
}

// 2^k as a float, k in [-126, 127].
__device__ __forceinline__ float pow2(int k) { return __int_as_float((127 + k) << 23); }

struct Unit {
  int own_kind, data_kind;
  const uint8_t* own;   // own region (SHARE: current token)
  const uint8_t* data;  // region the attended positions live in
  UnitLayout Lo, Ld;
  int n_att;            // positions read from data
  int nq;               // leading quantized positions among them
  int qtok;             // quantized tokens stored in the data unit
  int npos;             // n_att + has_cur
  int rtok;             // RES2: positions that carry a residual (read through data)
  bool has_cur;
  bool ok;
};

// RES2: the unit's own region holds residual codes and its bf16 window,
// data is its reference (the final loop's cell of the layer).
template <bool RES2>
__device__ Unit resolve(const DecodeParams& p, int cell, int b, int h, int D) {
  Unit u{};
  const TableHeader* hdr = reinterpret_cast<const TableHeader*>(p.table);
  const DevCell* cells = reinterpret_cast<const DevCell*>(p.table + table_cells_offset());
  const DevSeq* seqs = reinterpret_cast<const DevSeq*>(p.table + table_seqs_offset(hdr->n_cells));
  const int B = hdr->max_batch;
  const DevCell oc = cells[cell];
  const DevSeq os = seqs[(size_t)cell * B + b];
  if constexpr (RES2) {
    const DevCell dc = cells[oc.src];
    const DevSeq ds = seqs[(size_t)oc.src * B + b];
    u.own_kind = oc.kind;
    u.own = p.cache + os.offset + (size_t)h * os.stride;
    u.Lo = unit_layout(LOOPKV_RES2, D, os.cap);
    u.data_kind = dc.kind;
    u.data = p.cache + ds.offset + (size_t)h * ds.stride;
    u.Ld = unit_layout(dc.kind, D, ds.cap);
    u.n_att = os.len;
    u.has_cur = false;
    u.rtok = res2_qtok(os.len);
    const bool quant = dc.kind == LOOPKV_Q4 || dc.kind == LOOPKV_Q2;
    const int ref_pos = quant ? ds.len / kGroup * kGroup : ds.len;
    u.ok = oc.kind == LOOPKV_RES2 && os.len >= 1 && os.len <= os.cap && ds.len <= ds.cap &&
           (quant || dc.kind == LOOPKV_BF16) && u.rtok <= ref_pos;
    u.qtok = quant ? u.rtok : 0;
    u.nq = u.qtok;
    u.npos = u.n_att;
    return u;
  }
  u.own_kind = oc.kind;
  u.own = p.cache + os.offset + (size_t)h * os.stride;
  u.Lo = unit_layout(oc.kind, D, os.cap);
  u.ok = os.len >= 1 && os.len <= os.cap + (oc.kind == LOOPKV_SHARE ? (1 << 30) : 0);
  if (oc.kind == LOOPKV_SHARE) {
    const DevCell dc = cells[oc.src];
    const DevSeq ds = seqs[(size_t)oc.src * B + b];
    u.data_kind = dc.kind;
    u.data = p.cache + ds.offset + (size_t)h * ds.stride;
    u.Ld = unit_layout(dc.kind, D, ds.cap);
    u.n_att = os.len - 1;
    u.has_cur = true;
    u.ok = u.ok && u.n_att <= ds.len && ds.len <= ds.cap && dc.kind != LOOPKV_SHARE;
    u.qtok = (dc.kind == LOOPKV_BF16) ? 0 : (ds.len / kGroup) * kGroup;
  } else {
    u.data_kind = oc.kind;
    u.data = u.own;
    u.Ld = u.Lo;
    u.n_att = os.len;
    u.has_cur = false;
    u.qtok = (oc.kind == LOOPKV_BF16) ? 0 : (os.len / kGroup) * kGroup;
  }
  u.nq = u.n_att < u.qtok ? u.n_att : u.qtok;
  u.npos = u.n_att + (u.has_cur ? 1 : 0);
  return u;
}

// Pointer to the bf16 key (or value) row of a raw position (RES2: positions
// past the residual-coded ones are in the unit's own window, slot pos mod 64).
template <bool RES2>
__device__ __forceinline__ const uint8_t* raw_row(const Unit& u, int pos, int D, bool value) {
  if constexpr (RES2) {
    if (pos >= u.rtok)
      return u.own + (value ? u.Lo.res_v : u.Lo.res_k) + (size_t)(pos % kResWindow) * D * 2;
  }
  if (u.has_cur && pos == u.n_att) return u.own + (value ? u.Lo.cur_v : u.Lo.cur_k);
  if (u.data_kind == LOOPKV_BF16)
    return u.data + (value ? u.Ld.raw_v : u.Ld.raw_k) + (size_t)pos * D * 2;
  return u.data + (value ? u.Ld.res_v : u.Ld.res_k) + (size_t)(pos - u.qtok) * D * 2;
}

// bf16 key row dotted with the G queries of the group (q_s: [G][D] fp32).
template <int D, int G>
__device__ __forceinline__ void dot_bf16(const uint8_t* row, const float* q_s, float (&out)[G]) {
#pragma unroll
  for (int r = 0; r < G; ++r) out[r] = 0.f;
#pragma unroll
  for (int c = 0; c < D / 8; ++c) {
    const uint4 w = ldg128(row + c * 16);
    const float k[8] = {bf16_lo(w.x), bf16_hi(w.x), bf16_lo(w.y), bf16_hi(w.y),
                        bf16_lo(w.z), bf16_hi(w.z), bf16_lo(w.w), bf16_hi(w.w)};
#pragma unroll
    for (int r = 0; r < G; ++r) {
      const float4 qa = *reinterpret_cast<const float4*>(q_s + r * D + 8 * c);
      const float4 qb = *reinterpret_cast<const float4*>(q_s + r * D + 8 * c + 4);
      float acc = out[r];
      acc = fmaf(qa.x, k[0], acc);
      acc = fmaf(qa.y, k[1], acc);
      acc = fmaf(qa.z, k[2], acc);
      acc = fmaf(qa.w, k[3], acc);
      acc = fmaf(qb.x, k[4], acc);
      acc = fmaf(qb.y, k[5], acc);
      acc = fmaf(qb.z, k[6], acc);
      acc = fmaf(qb.w, k[7], acc);
      out[r] = acc;
    }
  }
}

// Scores of one quantized token for the G queries: sum_d qs_d * code_d over
// the token's packed planes (16-byte rows h[c], l[c] of K_hi / K_lo for chunk
// c of 64 channels); the codes are converted once and serve every query.
// qs2: the warp's staged q * scale, [G][D] as float pairs.
template <int D, bool Q4, int G>
__device__ __forceinline__ void dot_codes(const uint4 (&h)[D / 64], const uint4 (&l)[D / 64],
                                          const float2* qs2, float (&dot)[G]) {
  // independent accumulators keep the fma chains short: four per query for
  // one query, fewer when the queries themselves give independent chains
  constexpr int NA = G >= 4 ? 1 : 4 / G;
  float2 acc[G][NA];
#pragma unroll
  for (int r = 0; r < G; ++r)
#pragma unroll
    for (int k = 0; k < NA; ++k) acc[r][k] = make_float2(0.f, 0.f);
#pragma unroll
  for (int c = 0; c < D / 64; ++c) {
    const uint32_t hw[4] = {h[c].x, h[c].y, h[c].z, h[c].w};
    const uint32_t lw[4] = {l[c].x, l[c].y, l[c].z, l[c].w};
#pragma unroll
    for (int w = 0; w < 4; ++w) {
      float2 v[8];
      if (Q4) codes4_to_pairs(hw[w], lw[w], v);
      else codes2_to_pairs(hw[w], v);
#pragma unroll
      for (int r = 0; r < G; ++r) {
        const float4* q4p = reinterpret_cast<const float4*>(qs2 + r * (D / 2) + 32 * c + 8 * w);
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const float4 qq = q4p[i];
          acc[r][(2 * i) % NA] = fma2(make_float2(qq.x, qq.y), v[2 * i], acc[r][(2 * i) % NA]);
          acc[r][(2 * i + 1) % NA] =
              fma2(make_float2(qq.z, qq.w), v[2 * i + 1], acc[r][(2 * i + 1) % NA]);
        }
      }
    }
  }
#pragma unroll
  for (int r = 0; r < G; ++r) {
    if constexpr (NA == 4) {
      const float2 a = add2(acc[r][0], acc[r][1]), b = add2(acc[r][2], acc[r][3]);
      dot[r] = (a.x + b.x) + (a.y + b.y);
    } else if constexpr (NA == 2) {
      const float2 a = add2(acc[r][0], acc[r][1]);
      dot[r] = a.x + a.y;
    } else {
      dot[r] = acc[r][0].x + acc[r][0].y;
    }
  }
}

// Per-lane load of one 32-token key group: the lane's token rows of the
// planes and the lane's D/32 channels of the group's scale / zero point.
template <int D>
struct KGroup {
  uint4 h[D / 64], l[D / 64];
  float sc[D / 32], zr[D / 32];
};

// Lane pointers into one group: kh -> the lane's K_hi row of chunk 0,
// lo_off -> K_lo - K_hi, km -> the lane's scales (zeros D floats further).
template <int D, bool Q4>
__device__ __forceinline__ void load_kgroup(KGroup<D>& g, const uint8_t* kh, size_t lo_off,
                                            const float* km) {
#pragma unroll
  for (int c = 0; c < D / 64; ++c) {
    g.h[c] = ld_stream(kh + c * 512);
    g.l[c] = Q4 ? ld_stream(kh + lo_off + c * 512) : make_uint4(0, 0, 0, 0);
  }
  if constexpr (D == 128) {
    const float4 a = __ldg(reinterpret_cast<const float4*>(km));
    const float4 z = __ldg(reinterpret_cast<const float4*>(km + D));
    g.sc[0] = a.x; g.sc[1] = a.y; g.sc[2] = a.z; g.sc[3] = a.w;
    g.zr[0] = z.x; g.zr[1] = z.y; g.zr[2] = z.z; g.zr[3] = z.w;
  } else {
    const float2 a = __ldg(reinterpret_cast<const float2*>(km));
    const float2 z = __ldg(reinterpret_cast<const float2*>(km + D));
    g.sc[0] = a.x; g.sc[1] = a.y;
    g.zr[0] = z.x; g.zr[1] = z.y;
  }
}

// Score one group held in registers for the G queries; s[r] = the lane's
// score for query r (or -inf past qlim).
// qf[i]: 2^(kSub - o) of the lane's channel i (o: the bit offset its code
// keeps after conversion); q_s: the group's queries [G][D].
template <int D, bool Q4, int G>
__device__ __forceinline__ void key_group(const KGroup<D>& g, const float (&qf)[D / 32],
                                          const float* q_s, float* qs, int pos, int qlim,
                                          float sscale, int lane, float (&s)[G]) {
  constexpr int CPL = D / 32;
  // fold each query into the group's key scale / zero point
  float cpart[G];
#pragma unroll
  for (int r = 0; r < G; ++r) {
    cpart[r] = 0.f;
#pragma unroll
    for (int i = 0; i < CPL; ++i) {
      const float qz = q_s[r * D + CPL * lane + i];
      qs[r * D + CPL * lane + i] = (qz * qf[i]) * g.sc[i];
      cpart[r] = fmaf(qz, g.zr[i], cpart[r]);
    }
  }
  if constexpr (G == 1) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) cpart[0] += __shfl_xor_sync(0xffffffffu, cpart[0], o);
  } else {
    // transposed butterfly: the first steps halve the queries a lane keeps
    // (lane bit 4, then bit 3), the rest sum one query over the warp; the
    // G totals are then read from the lanes that hold them
    const bool b4 = (lane & 16) != 0;
    float k;
    if constexpr (G == 2) {
      k = (b4 ? cpart[1] : cpart[0]) + __shfl_xor_sync(0xffffffffu, b4 ? cpart[0] : cpart[1], 16);
    } else {
      const float r0 = __shfl_xor_sync(0xffffffffu, b4 ? cpart[0] : cpart[2], 16);
      const float r1 = __shfl_xor_sync(0xffffffffu, b4 ? cpart[1] : cpart[3], 16);
      const float k0 = (b4 ? cpart[2] : cpart[0]) + r0;
      const float k1 = (b4 ? cpart[3] : cpart[1]) + r1;
      const bool b3 = (lane & 8) != 0;
      k = (b3 ? k1 : k0) + __shfl_xor_sync(0xffffffffu, b3 ? k0 : k1, 8);
    }
#pragma unroll
    for (int o = (G == 2 ? 8 : 4); o > 0; o >>= 1) k += __shfl_xor_sync(0xffffffffu, k, o);
#pragma unroll
    for (int r = 0; r < G; ++r)
      cpart[r] = __shfl_sync(0xffffffffu, k, G == 2 ? 16 * r : 16 * (r >> 1) + 8 * (r & 1));
  }
  __syncwarp();
#pragma unroll
  for (int r = 0; r < G; ++r) s[r] = -INFINITY;
  if (pos < qlim) {
    float dot[G];
    dot_codes<D, Q4, G>(g.h, g.l, reinterpret_cast<const float2*>(qs), dot);
#pragma unroll
    for (int r = 0; r < G; ++r) s[r] = fmaf(dot[r], pow2(149 - kSub) * sscale, cpart[r] * sscale);
  }
  __syncwarp();
}

// L2 requests for one key group by a lane with lane % 8 == 0: kh -> the
// lane's K_hi row of chunk 0 (16 lane bytes into the group's block, so the
// lanes 0, 8, 16, 24 start the chunk's four lines), km -> its scales.
template <int D, bool Q4>
__device__ __forceinline__ void prefetch_kgroup(const uint8_t* kh, size_t lo_off, const float* km) {
#pragma unroll
  for (int c = 0; c < D / 64; ++c) {
    prefetch_l2(kh + c * 512);
    if (Q4) prefetch_l2(kh + lo_off + c * 512);
  }
  // meta block: scales then zeros, D floats each; km is CPL lane floats in
  prefetch_l2(km);
  prefetch_l2(km + D);
}

// Pass 1 over the CTA's quantized key groups [b_begin, b_end), warp-strided.
// Two register buffers alternate, so the next group's loads are in flight
// while the current one is scored, without copies between them.  Scores of
// query r go to sc[r * S + pos - p0]; lmax[r] is raised to their maximum.
// ADD: the scores are added to what sc holds (a RES2 unit's residual keys
// on top of its reference's); lmax is then left alone.
template <int D, bool Q4, int G, bool ADD = false>
__device__ __forceinline__ void key_pass(const Unit& u, int b_begin, int b_end, int p0, int p1,
                                         const float* q_s, float* qs, float* sc, int S,
                                         float sscale, int warp, int lane, float (&lmax)[G]) {
  constexpr int CPL = D / 32;  // channels per lane for the q fold
  const int first = b_begin + warp;
  if (first >= b_end) return;
  // 2^(kSub - o) for the lane's channels: o is the bit offset the channel's
  // code keeps after conversion (see codes4_to_pairs / codes2_to_pairs)
  float qf[CPL];
#pragma unroll
  for (int i = 0; i < CPL; ++i) {
    const int j = (CPL * lane + i) & 15;
    qf[i] = pow2(kSub - (Q4 ? code4_off(j >> 1) : code2_off(j)));
  }
  const int qlim = min(p1, u.nq);
  constexpr size_t GB = 8 * D;                      // bytes of one group in each block
  constexpr size_t STEP = (size_t)kWarps * GB;      // a warp's stride between its groups
  const uint8_t* kh = u.data + u.Ld.k_hi + (size_t)first * GB + lane * 16;
  const size_t lo_off = u.Ld.k_lo - u.Ld.k_hi;
  const float* km = reinterpret_cast<const float*>(u.data + u.Ld.k_meta + (size_t)first * GB) +
                    CPL * lane;
  const bool pon = (lane & 7) == 0;  // lanes whose row pointers start a line
  KGroup<D> a, b;
  load_kgroup<D, Q4>(a, kh, lo_off, km);
  int bk = first;
  float s[G];
  for (;;) {
    const bool hasb = bk + kWarps < b_end;
    if (hasb) load_kgroup<D, Q4>(b, kh + STEP, lo_off, km + STEP / 4);
    if (kAheadK > 0 && pon && hasb)
      prefetch_kgroup<D, Q4>(kh + kAheadK * STEP, lo_off, km + kAheadK * STEP / 4);
    key_group<D, Q4, G>(a, qf, q_s, qs, bk * 32 + lane, qlim, sscale, lane, s);
    if (bk * 32 + lane < qlim) {
#pragma unroll
      for (int r = 0; r < G; ++r) {
        if (ADD) {
          sc[r * S + bk * 32 + lane - p0] += s[r];
        } else {
          sc[r * S + bk * 32 + lane - p0] = s[r];
          lmax[r] = fmaxf(lmax[r], s[r]);
        }
      }
    }
    if (!hasb) break;
    bk += kWarps;
    kh += STEP;
    km += STEP / 4;
    const bool hasa = bk + kWarps < b_end;
    if (hasa) load_kgroup<D, Q4>(a, kh + STEP, lo_off, km + STEP / 4);
    if (kAheadK > 0 && pon && hasa)
      prefetch_kgroup<D, Q4>(kh + kAheadK * STEP, lo_off, km + kAheadK * STEP / 4);
    key_group<D, Q4, G>(b, qf, q_s, qs, bk * 32 + lane, qlim, sscale, lane, s);
    if (bk * 32 + lane < qlim) {
#pragma unroll
      for (int r = 0; r < G; ++r) {
        if (ADD) {
          sc[r * S + bk * 32 + lane - p0] += s[r];
        } else {
          sc[r * S + bk * 32 + lane - p0] = s[r];
          lmax[r] = fmaxf(lmax[r], s[r]);
        }
      }
    }
    if (!hasa) break;
    bk += kWarps;
    kh += STEP;
    km += STEP / 4;
  }
}

// ------------------------------------------------- keys of a query group
//
// With G >= 2 query heads per KV head the key scores of a 32-token group are
// a [G x D] by [D x 32] product: a dense contraction, so it goes to the
// tensor cores (mma.sync m16n8k32, s8 weight digits x u8 code bytes, s32
// accumulate), exactly, in integers.  One query keeps the FMA-pipe pass
// above (single-query decode is not a dense contraction).
//
// Weights.  For query r the folded weights qs_c = q_c * scale_c of the group
// share one power of two 2^E chosen from the warp's largest |qs|, so that
// W_c = rint(qs_c 2^E) has |W_c| < 2^26; the score is then
// (sum_c W_c code_c) 2^-E + sum_c q_c zero_c.
//
// Codes.  The hi / lo planes of a 16-channel word merge into two nibble
// words (byte b of the even word holds channels 4b (low nibble) and 4b + 2
// (high), the odd word channels 4b + 1 and 4b + 3): one byte carries two
// codes, c_lo + 16 c_hi.  With X = 16 W(c_lo's channel) and
// Y = W(c_hi's channel) - 16 W(c_lo's channel),
//   byte * X + (byte & 0xF0) * Y = 16 (c_lo W_lo + c_hi W_hi),
// so two products into one accumulator cover both codes without unpacking
// them.  X and Y are split into four signed base-256 digits (byte p of
// v + 0x80808080 as u8, minus 128; exact for |v| < 0x7F7F7F7F, and
// |X|, |Y| < 17 * 2^26).
//
// Tile.  A (16 x 32, s8): row r holds digit d of query q, r = 2q + (d & 1) +
// 8 (d >> 1), so lane group g (rows g and g + 8) holds digits d0 = g & 1 and
// d0 + 2 of query g >> 1.  B (32 x 8, u8): column n is token n of an 8-token
// tile; K byte 4t' + b (b < 4) of K tile kt is byte b of the even word of
// plane word W = (D / 64) t' + kt, K byte 16 + 4t' + b the same of its odd
// word.  D (16 x 8, s32) rows and columns follow A and B.  A lane (g, t)
// loads the plane words W(kt, t) of tokens g + 8j, j = 0..3 (the B
// fragments of the four token tiles), and after the products combines its
// two digits, then the digit pair of lanes g and g ^ 1: it ends with the
// sums of query g >> 1 for tokens 8 (2p + (g & 1)) + 2t + {0, 1}, p = 0, 1.

__device__ __forceinline__ void mma_s8u8(int (&c)[4], const uint32_t (&a)[4], uint32_t b0,
                                         uint32_t b1) {
  asm("mma.sync.aligned.m16n8k32.row.col.s32.s8.u8.s32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+r"(c[0]), "+r"(c[1]), "+r"(c[2]), "+r"(c[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

__device__ __forceinline__ void mma_u8s8(int (&c)[4], const uint32_t (&a)[4], uint32_t b0,
                                         uint32_t b1) {
  asm("mma.sync.aligned.m16n8k32.row.col.s32.u8.s8.s32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+r"(c[0]), "+r"(c[1]), "+r"(c[2]), "+r"(c[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// A lane's plane words of one key group: token g + 8j, plane word W(kt, t).
template <int D>
struct KTileMma {
  uint32_t h[4][D / 64 > 0 ? D / 64 : 1], l[4][D / 64 > 0 ? D / 64 : 1];
  float4 sc, zr;  // scales / zero points of channels 4 lane .. 4 lane + 3 (lanes < D / 4)
};

template <int D, bool Q4>
__device__ __forceinline__ void load_ktile_mma(KTileMma<D>& k, const uint8_t* kb, size_t lo_off,
                                               const float* km, bool meta) {
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    if constexpr (D == 128) {
      const uint2 hw = ld_stream2(kb + j * 128);
      k.h[j][0] = hw.x;
      k.h[j][1] = hw.y;
      if constexpr (Q4) {
        const uint2 lw = ld_stream2(kb + lo_off + j * 128);
        k.l[j][0] = lw.x;
        k.l[j][1] = lw.y;
      } else {
        k.l[j][0] = 0u;
        k.l[j][1] = 0u;
      }
    } else {
      k.h[j][0] = ld_stream1(kb + j * 128);
      k.l[j][0] = Q4 ? ld_stream1(kb + lo_off + j * 128) : 0u;
    }
  }
  if (meta) {
    k.sc = __ldg(reinterpret_cast<const float4*>(km));
    k.zr = __ldg(reinterpret_cast<const float4*>(km + D));
  } else {
    k.sc = make_float4(0.f, 0.f, 0.f, 0.f);
    k.zr = k.sc;
  }
}

// Nibble words of a 16-channel plane word pair (q = 4 hi + lo for 4-bit
// keys, q = hi for 2-bit keys).
template <bool Q4>
__device__ __forceinline__ void nibble_words(uint32_t hi, uint32_t lo, uint32_t& ev, uint32_t& od) {
  if constexpr (Q4) {
    ev = ((hi << 2) & 0xCCCCCCCCu) | (lo & 0x33333333u);
    od = (hi & 0xCCCCCCCCu) | ((lo >> 2) & 0x33333333u);
  } else {
    ev = hi & 0x33333333u;
    od = (hi >> 2) & 0x33333333u;
  }
}

// Digit d (0..3) of four biased weights, as the signed bytes of one word.
__device__ __forceinline__ uint32_t digit_word(int4 v, uint32_t sel) {
  const uint32_t lo2 = __byte_perm((uint32_t)v.x, (uint32_t)v.y, sel);
  const uint32_t hi2 = __byte_perm((uint32_t)v.z, (uint32_t)v.w, sel);
  return __byte_perm(lo2, hi2, 0x5410u) ^ 0x80808080u;
}

// Products and digits of a group for two queries, tokens in the tile's
// rows: A (16 x 32, u8) = the code bytes of 16 tokens (lane (g, t) holds the
// even and odd nibble words of plane word W(kt, t) of tokens g and g + 8 of
// the M tile), B (32 x 8, s8) = the weight digits, column n = digit n & 3 of
// query n >> 2.  Every row and column is used, so two queries take half the
// products of the query-digit layout.  Lane (g, t) receives digits
// 2 (t & 1) and 2 (t & 1) + 1 of query t >> 1 for tokens g and g + 8; with
// lane t ^ 1 (the other two digits) it completes one token per M tile:
// token 16 mt + g + 8 (t & 1).
template <int D, bool Q4, bool ADD>
__device__ __forceinline__ void key_products_g2(const KTileMma<D>& k, const int* st,
                                                const float (&finv)[2], const float (&cpart)[2],
                                                int gpos0, int qlim, int p0, float* sc, int S,
                                                float sscale, int lane, float (&lmax)[2]) {
  constexpr int KT = D / 64 > 0 ? D / 64 : 1;
  constexpr int Q4W = D / 4;
  const int g = lane >> 2, t = lane & 3;
  const int qn = g >> 2, dn = g & 3;  // this lane's B column: digit dn of query qn
  const uint32_t sel = (uint32_t)dn | ((uint32_t)(dn + 4) << 4);
  int acc[2][4];
#pragma unroll
  for (int mt = 0; mt < 2; ++mt)
#pragma unroll
    for (int i = 0; i < 4; ++i) acc[mt][i] = 0;
#pragma unroll
  for (int kt = 0; kt < KT; ++kt) {
    const int W = (D / 64 > 0 ? D / 64 : 1) * t + kt;
    const int4 xe = *reinterpret_cast<const int4*>(st + (0 * 2 + qn) * Q4W + 4 * W);
    const int4 xo = *reinterpret_cast<const int4*>(st + (1 * 2 + qn) * Q4W + 4 * W);
    const int4 ye = *reinterpret_cast<const int4*>(st + (2 * 2 + qn) * Q4W + 4 * W);
    const int4 yo = *reinterpret_cast<const int4*>(st + (3 * 2 + qn) * Q4W + 4 * W);
    const uint32_t bx0 = digit_word(xe, sel), bx1 = digit_word(xo, sel);
    const uint32_t by0 = digit_word(ye, sel), by1 = digit_word(yo, sel);
#pragma unroll
    for (int mt = 0; mt < 2; ++mt) {
      uint32_t e0, o0, e1, o1;
      nibble_words<Q4>(k.h[2 * mt][kt], k.l[2 * mt][kt], e0, o0);          // token g + 16 mt
      nibble_words<Q4>(k.h[2 * mt + 1][kt], k.l[2 * mt + 1][kt], e1, o1);  // token g + 8 + 16 mt
      const uint32_t ax[4] = {e0, e1, o0, o1};
      const uint32_t ay[4] = {e0 & 0xF0F0F0F0u, e1 & 0xF0F0F0F0u, o0 & 0xF0F0F0F0u,
                              o1 & 0xF0F0F0F0u};
      mma_u8s8(acc[mt], ax, bx0, bx1);
      mma_u8s8(acc[mt], ay, by0, by1);
    }
  }
  __syncwarp();  // the staging is read; the next group may overwrite it
  // columns 2t, 2t + 1: digits d1 = 2 (t & 1) and d1 + 1 of query t >> 1
  const int d1 = 2 * (t & 1);
  const float f0 = __int_as_float((127 + 8 * d1 - 4) << 23);   // 2^(8 d1) / 16
  const float f1 = __int_as_float((127 + 8 * d1 + 4) << 23);   // 2^(8 (d1 + 1)) / 16
  const bool up = (t & 1) != 0;
  const int qq = t >> 1;
  const float fs = (qq ? finv[1] : finv[0]) * sscale;
  const float cs = (qq ? cpart[1] : cpart[0]) * sscale;
  float mx = -INFINITY;
#pragma unroll
  for (int mt = 0; mt < 2; ++mt) {
    const float vg = fmaf((float)acc[mt][1], f1, (float)acc[mt][0] * f0);   // row g
    const float vg8 = fmaf((float)acc[mt][3], f1, (float)acc[mt][2] * f0);  // row g + 8
    // lanes t, t ^ 1 hold the other digit pair of the same query: the
    // lower one completes row g, the upper one row g + 8
    const float tot = (up ? vg8 : vg) + __shfl_xor_sync(0xffffffffu, up ? vg : vg8, 1);
    const int pos = gpos0 + 16 * mt + g + (up ? 8 : 0);
    if (pos < qlim) {
      const float sv = fmaf(tot, fs, cs);
      float* dst = sc + qq * S + pos - p0;
      if (ADD) *dst += sv;
      else *dst = sv;
      mx = fmaxf(mx, sv);
    }
  }
  if (!ADD) {
    if (qq) lmax[1] = fmaxf(lmax[1], mx);
    else lmax[0] = fmaxf(lmax[0], mx);
  }
}

// Scores of one group held in registers for the G queries.  st: the warp's
// staging of the biased weights, [4 arrays][G][D / 4] ints (X even, X odd,
// Y even, Y odd).  Writes (ADD: adds) the scores of positions below qlim
// into sc[r * S + pos - p0] and raises lmax[r].
template <int D, bool Q4, int G, bool ADD>
__device__ __forceinline__ void key_group_mma(const KTileMma<D>& k, const float* q_s, int* st,
                                              int gpos0, int qlim, int p0, float* sc, int S,
                                              float sscale, int lane, float (&lmax)[G]) {
  constexpr int KT = D / 64 > 0 ? D / 64 : 1;
  constexpr int Q4W = D / 4;  // weights per array and query
  const int g = lane >> 2, t = lane & 3;
  const bool fold = lane < D / 4;
  // ---- fold each query into the group's scales: integer weights
  float cpart[G], finv[G];
#pragma unroll
  for (int r = 0; r < G; ++r) {
    const float4 qv = fold ? *reinterpret_cast<const float4*>(q_s + r * D + 4 * lane)
                           : make_float4(0.f, 0.f, 0.f, 0.f);
    const float w0 = qv.x * k.sc.x, w1 = qv.y * k.sc.y, w2 = qv.z * k.sc.z, w3 = qv.w * k.sc.w;
    cpart[r] = fmaf(qv.w, k.zr.w, fmaf(qv.z, k.zr.z, fmaf(qv.y, k.zr.y, qv.x * k.zr.x)));
    const float amax = fmaxf(fmaxf(fabsf(w0), fabsf(w1)), fmaxf(fabsf(w2), fabsf(w3)));
    const uint32_t mbits = __reduce_max_sync(0xffffffffu, __float_as_uint(amax));
    const int fexp = min(279 - (int)(mbits >> 23), 253);  // max |w| 2^(fexp - 127) < 2^26
    const float F = __int_as_float(fexp << 23);
    finv[r] = __int_as_float((254 - fexp) << 23);
    if (fold) {
      const int i0 = __float2int_rn(w0 * F), i1 = __float2int_rn(w1 * F);
      const int i2 = __float2int_rn(w2 * F), i3 = __float2int_rn(w3 * F);
      constexpr uint32_t kBias = 0x80808080u;
      st[(0 * G + r) * Q4W + lane] = (int)((uint32_t)(16 * i0) + kBias);       // X even
      st[(1 * G + r) * Q4W + lane] = (int)((uint32_t)(16 * i1) + kBias);       // X odd
      st[(2 * G + r) * Q4W + lane] = (int)((uint32_t)(i2 - 16 * i0) + kBias);  // Y even
      st[(3 * G + r) * Q4W + lane] = (int)((uint32_t)(i3 - 16 * i1) + kBias);  // Y odd
    }
  }
  // zero-point terms: sum over the warp, every lane gets all G totals
  {
    const bool b4 = (lane & 16) != 0;
    float kk;
    if constexpr (G == 2) {
      kk = (b4 ? cpart[1] : cpart[0]) + __shfl_xor_sync(0xffffffffu, b4 ? cpart[0] : cpart[1], 16);
    } else {
      const float r0 = __shfl_xor_sync(0xffffffffu, b4 ? cpart[0] : cpart[2], 16);
      const float r1 = __shfl_xor_sync(0xffffffffu, b4 ? cpart[1] : cpart[3], 16);
      const float k0 = (b4 ? cpart[2] : cpart[0]) + r0;
      const float k1 = (b4 ? cpart[3] : cpart[1]) + r1;
      const bool b3 = (lane & 8) != 0;
      kk = (b3 ? k1 : k0) + __shfl_xor_sync(0xffffffffu, b3 ? k0 : k1, 8);
    }
#pragma unroll
    for (int o = (G == 2 ? 8 : 4); o > 0; o >>= 1) kk += __shfl_xor_sync(0xffffffffu, kk, o);
#pragma unroll
    for (int r = 0; r < G; ++r)
      cpart[r] = __shfl_sync(0xffffffffu, kk, G == 2 ? 16 * r : 16 * (r >> 1) + 8 * (r & 1));
  }
  __syncwarp();
  if constexpr (G == 2) {
    key_products_g2<D, Q4, ADD>(k, st, finv, cpart, gpos0, qlim, p0, sc, S, sscale, lane, lmax);
    return;
  }
  // ---- products: lane group g holds digits d0, d0 + 2 of query qg
  const int qg = g >> 1, d0 = g & 1;
  const bool qok = qg < G;
  const uint32_t sel_lo = (uint32_t)d0 | ((uint32_t)(d0 + 4) << 4);
  const uint32_t sel_hi = (uint32_t)(d0 + 2) | ((uint32_t)(d0 + 6) << 4);
  int acc[4][4];
#pragma unroll
  for (int j = 0; j < 4; ++j)
#pragma unroll
    for (int i = 0; i < 4; ++i) acc[j][i] = 0;
#pragma unroll
  for (int kt = 0; kt < KT; ++kt) {
    const int W = (D / 64 > 0 ? D / 64 : 1) * t + kt;
    uint32_t ax[4] = {0u, 0u, 0u, 0u}, ay[4] = {0u, 0u, 0u, 0u};
    if (qok) {
      const int qq = qg < G ? qg : 0;
      const int4 xe = *reinterpret_cast<const int4*>(st + (0 * G + qq) * Q4W + 4 * W);
      const int4 xo = *reinterpret_cast<const int4*>(st + (1 * G + qq) * Q4W + 4 * W);
      const int4 ye = *reinterpret_cast<const int4*>(st + (2 * G + qq) * Q4W + 4 * W);
      const int4 yo = *reinterpret_cast<const int4*>(st + (3 * G + qq) * Q4W + 4 * W);
      ax[0] = digit_word(xe, sel_lo);  // row g: even bytes
      ax[1] = digit_word(xe, sel_hi);  // row g + 8
      ax[2] = digit_word(xo, sel_lo);  // row g: odd bytes
      ax[3] = digit_word(xo, sel_hi);
      ay[0] = digit_word(ye, sel_lo);
      ay[1] = digit_word(ye, sel_hi);
      ay[2] = digit_word(yo, sel_lo);
      ay[3] = digit_word(yo, sel_hi);
    }
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      uint32_t ev, od;
      nibble_words<Q4>(k.h[j][kt], k.l[j][kt], ev, od);
      mma_s8u8(acc[j], ax, ev, od);
      mma_s8u8(acc[j], ay, ev & 0xF0F0F0F0u, od & 0xF0F0F0F0u);
    }
  }
  __syncwarp();  // the staging is read; the next group may overwrite it
  // ---- digits: rows g (digit d0) and g + 8 (d0 + 2), then lanes g, g ^ 1
  const float flo = __int_as_float((127 + 8 * d0 - 4) << 23);   // 2^(8 d0) / 16
  const float fhi = __int_as_float((127 + 8 * d0 + 12) << 23);  // 2^(8 (d0 + 2)) / 16
  float v[4][2];
#pragma unroll
  for (int j = 0; j < 4; ++j)
#pragma unroll
    for (int c = 0; c < 2; ++c) v[j][c] = fmaf((float)acc[j][c + 2], fhi, (float)acc[j][c] * flo);
  float w[2][2];
#pragma unroll
  for (int pp = 0; pp < 2; ++pp)
#pragma unroll
    for (int c = 0; c < 2; ++c) {
      const float keep = d0 ? v[2 * pp + 1][c] : v[2 * pp][c];
      const float send = d0 ? v[2 * pp][c] : v[2 * pp + 1][c];
      w[pp][c] = keep + __shfl_xor_sync(0xffffffffu, send, 4);
    }
  if (!qok) return;
  float fsel = finv[0], csel = cpart[0];
#pragma unroll
  for (int r = 1; r < G; ++r) {
    fsel = qg == r ? finv[r] : fsel;
    csel = qg == r ? cpart[r] : csel;
  }
  const float fs = fsel * sscale, cs = csel * sscale;
  float mx = -INFINITY;
#pragma unroll
  for (int pp = 0; pp < 2; ++pp)
#pragma unroll
    for (int c = 0; c < 2; ++c) {
      const int pos = gpos0 + 8 * (2 * pp + d0) + 2 * t + c;
      if (pos < qlim) {
        const float sv = fmaf(w[pp][c], fs, cs);
        float* dst = sc + qg * S + pos - p0;
        if (ADD) *dst += sv;
        else *dst = sv;
        mx = fmaxf(mx, sv);
      }
    }
  if (!ADD) {
#pragma unroll
    for (int r = 0; r < G; ++r)
      if (qg == r) lmax[r] = fmaxf(lmax[r], mx);
  }
}

// L2 requests for one key group in the tensor-core layout (see key_pass_mma).
template <int D, bool Q4>
__device__ __forceinline__ void prefetch_kgroup_mma(const uint8_t* kb, size_t lo_off, const float* km,
                                                    bool pon_k, bool pon_m) {
  if (pon_k) {
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      prefetch_l2(kb + j * 128);
      if (Q4) prefetch_l2(kb + lo_off + j * 128);
    }
  }
  if (pon_m) {
    prefetch_l2(km);
    prefetch_l2(km + D);
  }
}

// Pass 1 for a query group on the tensor cores: as key_pass, with the
// warp's q * scale rows (G * D floats) as the weight staging.
template <int D, bool Q4, int G, bool ADD = false>
__device__ __forceinline__ void key_pass_mma(const Unit& u, int b_begin, int b_end, int p0, int p1,
                                             const float* q_s, float* qs, float* sc, int S,
                                             float sscale, int warp, int lane, float (&lmax)[G]) {
  static_assert(G == 2 || G == 4, "query groups of 2 or 4");
  const int first = b_begin + warp;
  if (first >= b_end) return;
  const int qlim = min(p1, u.nq);
  const int g = lane >> 2, t = lane & 3;
  const bool meta = lane < D / 4;
  constexpr size_t GB = 8 * D;                  // bytes of one group in each block
  constexpr size_t STEP = (size_t)kWarps * GB;  // a warp's stride between its groups
  const size_t lane_off = (D == 128) ? (size_t)(t >> 1) * 512 + g * 16 + (t & 1) * 8
                                     : (size_t)g * 16 + t * 4;
  const uint8_t* kb = u.data + u.Ld.k_hi + (size_t)first * GB + lane_off;
  const size_t lo_off = u.Ld.k_lo - u.Ld.k_hi;
  const float* km = reinterpret_cast<const float*>(u.data + u.Ld.k_meta + (size_t)first * GB) +
                    (meta ? 4 * lane : 0);
  int* st = reinterpret_cast<int*>(qs);
  // L2 requests for a group ahead of the register loads: the lanes whose
  // plane pointers start a 128-byte line request the four token rows of
  // their chunk (K_hi, K_lo), every eighth meta lane its scale and zero lines
  const bool pon_k = g == 0 && (t & 1) == 0 && (D == 128 || t == 0);
  const bool pon_m = meta && (lane & 7) == 0;
  if constexpr (G == 4) {
    // one tile buffer: the registers the second one would hold go to the
    // value pass; the L2 requests two groups ahead cover the loads' latency
    for (int bk = first; bk < b_end; bk += kWarps, kb += STEP, km += STEP / 4) {
      KTileMma<D> a;
      load_ktile_mma<D, Q4>(a, kb, lo_off, km, meta);
      if (kAheadK > 0 && bk + 2 * kWarps < b_end)
        prefetch_kgroup_mma<D, Q4>(kb + 2 * STEP, lo_off, km + 2 * STEP / 4, pon_k, pon_m);
      key_group_mma<D, Q4, G, ADD>(a, q_s, st, bk * 32, qlim, p0, sc, S, sscale, lane, lmax);
    }
    return;
  }
  KTileMma<D> a, b;
  load_ktile_mma<D, Q4>(a, kb, lo_off, km, meta);
  int bk = first;
  for (;;) {
    const bool hasb = bk + kWarps < b_end;
    if (hasb) load_ktile_mma<D, Q4>(b, kb + STEP, lo_off, km + STEP / 4, meta);
    // L2 requests two groups ahead of the register loads (one ahead, the
    // same group as those loads, measured 1 % slower at two queries)
    if (kAheadK > 0 && bk + 2 * kWarps < b_end)
      prefetch_kgroup_mma<D, Q4>(kb + 2 * STEP, lo_off, km + 2 * STEP / 4, pon_k, pon_m);
    key_group_mma<D, Q4, G, ADD>(a, q_s, st, bk * 32, qlim, p0, sc, S, sscale, lane, lmax);
    if (!hasb) break;
    bk += kWarps;
    kb += STEP;
    km += STEP / 4;
    const bool hasa = bk + kWarps < b_end;
    if (hasa) load_ktile_mma<D, Q4>(a, kb + STEP, lo_off, km + STEP / 4, meta);
    if (kAheadK > 0 && bk + 2 * kWarps < b_end)
      prefetch_kgroup_mma<D, Q4>(kb + 2 * STEP, lo_off, km + 2 * STEP / 4, pon_k, pon_m);
    key_group_mma<D, Q4, G, ADD>(b, q_s, st, bk * 32, qlim, p0, sc, S, sscale, lane, lmax);
    if (!hasa) break;
    bk += kWarps;
    kb += STEP;
    km += STEP / 4;
  }
}

// A lane's share of a token's value row in pass 2: with G queries per KV
// head, LPT = (D / 64) * G lanes share a token and each holds CH = 64 / G
// channels for every query (G * CH / 2 = 32 accumulator pairs): NW plane
// words, NGRP 32-channel value groups.
template <int G>
struct VShare {
  static constexpr int CH = 64 / G;
  static constexpr int NW = CH / 16;
  static constexpr int NGRP = CH >= 32 ? CH / 32 : 1;
};


// Asynchronous 16-byte copies global -> shared (L1 bypassed), in groups
// that a thread waits for; the warp then syncs before reading them.
__device__ __forceinline__ void cp_async16(void* dst, const void* src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;"
               ::"r"((uint32_t)__cvta_generic_to_shared(dst)), "l"(src)
               : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory"); }

// One 32-token value block into a warp's staging buffer: the block's V_hi
// rows ([32][D / 4] bytes), then its V_meta rows (the same size).  Both are
// contiguous in the cache and 16-byte aligned.
template <int D>
__device__ __forceinline__ void stage_vblock(uint8_t* st, const Unit& u, int bk, int lane) {
  constexpr int BB = 8 * D;  // bytes of one block of a value plane / of value meta
  const uint8_t* hi = u.data + u.Ld.v_hi + (size_t)bk * BB;
  const uint8_t* me = u.data + u.Ld.v_meta + (size_t)bk * BB;
#pragma unroll
  for (int i = lane; i < BB / 16; i += 32) {
    cp_async16(st + 16 * i, hi + 16 * i);
    cp_async16(st + BB + 16 * i, me + 16 * i);
  }
}

// NW plane words of a value row (16 NW bytes, 16-byte aligned for NW = 4).
template <int NW>
__device__ __forceinline__ void load_words(uint32_t (&w)[NW], const uint8_t* p) {
  if constexpr (NW == 4) {
    const uint4 x = ld_stream(p);
    w[0] = x.x; w[1] = x.y; w[2] = x.z; w[3] = x.w;
  } else if constexpr (NW == 2) {
    const uint2 x = ld_stream2(p);
    w[0] = x.x; w[1] = x.y;
  } else {
    w[0] = ld_stream1(p);
  }
}

// (scale, zero) of NGRP value groups of a meta row.
template <int NGRP>
__device__ __forceinline__ void load_meta(float (&m)[2 * NGRP], const uint8_t* p) {
  if constexpr (NGRP == 2) {
    const float4 x = ldg128f(p);
    m[0] = x.x; m[1] = x.y; m[2] = x.z; m[3] = x.w;
  } else {
    const float2 x = __ldg(reinterpret_cast<const float2*>(p));
    m[0] = x.x; m[1] = x.y;
  }
}

// The same words and (scale, zero) pairs from a staged block in shared memory.
template <int NW>
__device__ __forceinline__ void lds_words(uint32_t (&w)[NW], const uint8_t* p) {
  if constexpr (NW == 4) {
    const uint4 x = *reinterpret_cast<const uint4*>(p);
    w[0] = x.x; w[1] = x.y; w[2] = x.z; w[3] = x.w;
  } else if constexpr (NW == 2) {
    const uint2 x = *reinterpret_cast<const uint2*>(p);
    w[0] = x.x; w[1] = x.y;
  } else {
    w[0] = *reinterpret_cast<const uint32_t*>(p);
  }
}
template <int NGRP>
__device__ __forceinline__ void lds_meta(float (&m)[2 * NGRP], const uint8_t* p) {
  if constexpr (NGRP == 2) {
    const float4 x = *reinterpret_cast<const float4*>(p);
    m[0] = x.x; m[1] = x.y; m[2] = x.z; m[3] = x.w;
  } else {
    const float2 x = *reinterpret_cast<const float2*>(p);
    m[0] = x.x; m[1] = x.y;
  }
}

// Value accumulation of the lane's share of one quantized token row:
// acc[r] += a[r][group] * code * 2^(o - 149) per channel, one conversion per
// code for all G queries; the per-channel power of two is removed once at
// the end.
template <int G>
__device__ __forceinline__ void value_codes(float2 (&acc)[G][32 / G],
                                            const uint32_t (&w)[VShare<G>::NW],
                                            const float (&a)[G][VShare<G>::NGRP]) {
  constexpr int NW = VShare<G>::NW;
#pragma unroll
  for (int wi = 0; wi < NW; ++wi) {
    float2 v[8];
    codes2_to_pairs(w[wi], v);
    constexpr int kPerGroup = 2;  // 16-channel words per 32-channel group
#pragma unroll
    for (int r = 0; r < G; ++r) {
      const float aw = a[r][wi / kPerGroup];
      const float2 aa = make_float2(aw, aw);
#pragma unroll
      for (int i = 0; i < 8; ++i) acc[r][8 * wi + i] = fma2(aa, v[i], acc[r][8 * wi + i]);
    }
  }
}

// bf16 value row (the lane's CH channels) with weight pt[r] per query, in the
// accumulators' scaled representation (channel j of a 16-channel word
// carries 2^(o(j) + kSub - 149)).
template <int G>
__device__ __forceinline__ void value_raw(float2 (&acc)[G][32 / G], const uint8_t* row,
                                          const float (&pt)[G]) {
  constexpr int CH = VShare<G>::CH;
#pragma unroll
  for (int c = 0; c < CH / 8; ++c) {
    const uint4 w = ldg128(row + c * 16);
    const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const int pair = 4 * c + k;          // channels 2*pair, 2*pair+1 of the lane's share
      const int j = (2 * pair) & 15;       // position inside the 16-channel word
      const float2 x = make_float2(bf16_lo(ws[k]), bf16_hi(ws[k]));
#pragma unroll
      for (int r = 0; r < G; ++r) {
        const float2 wt = make_float2(pt[r] * pow2(code2_off(j) + kSub - 149),
                                      pt[r] * pow2(code2_off(j + 1) + kSub - 149));
        acc[r][pair] = fma2(wt, x, acc[r][pair]);
      }
    }
  }
}

// Low planes of queued selected positions: acc[r] += p_r * scale * lo, TPI
// positions per warp iteration (LPT lanes per position).  fs[r] turns the
// stored exponential of query r into p_r * 2^kSub.
template <int D, int G, int LPT>
__device__ __forceinline__ void low_planes(float2 (&acc)[G][32 / G], const Unit& u,
                                           const int* list, int n, const float* sc, int S,
                                           int p0, const float (&fs)[G], int lane) {
  using VS = VShare<G>;
  constexpr int TPI = 32 / LPT;
  const int hf = lane % LPT;
  for (int k0 = 0; k0 < n; k0 += TPI) {
    const int kk = k0 + lane / LPT;
    if (kk < n) {
      const int tpos = list[kk];
      uint32_t lw[VS::NW];
      float m[2 * VS::NGRP];
      load_words<VS::NW>(lw, u.data + u.Ld.v_lo + (size_t)tpos * (D / 4) + hf * (VS::CH / 4));
      load_meta<VS::NGRP>(m, u.data + u.Ld.v_meta + (size_t)tpos * (D / 4) + (hf * VS::CH / 32) * 8);
      float a[G][VS::NGRP];
#pragma unroll
      for (int r = 0; r < G; ++r) {
        const float pt = sc[r * S + tpos - p0] * fs[r];
#pragma unroll
        for (int gi = 0; gi < VS::NGRP; ++gi) a[r][gi] = pt * m[2 * gi];
      }
      value_codes<G>(acc, lw, a);
    }
  }
  __syncwarp();
}

// One CTA per (unit, split) for a group of G query heads sharing the unit's
// KV head.  DENSE_LO: tau <= 0, every 4-bit token takes its low plane (read
// densely in the value loop); otherwise low planes come from the
// selected-position list.
template <int D, int G, bool DENSE_LO, bool RES2>
__global__ void __launch_bounds__(kThreads, 2)
decode_kernel(const DecodeParams p, const CellList cl) {
  require_ieee_subnormals();
  using VS = VShare<G>;
  const int S = p.slots;  // score slots per query
  extern __shared__ __align__(16) float smem[];
  float* q_s = smem;                                  // [G][D]
  float* qs_all = q_s + G * D;                        // [kWarps][G][D]
  float* red = qs_all + kWarps * G * D;               // [kWarps][G][D]
  float* o_s = red + kWarps * G * D;                  // [G][D]
  float* misc = o_s + G * D;                          // [128]
  int* lst = reinterpret_cast<int*>(misc + 128);      // [kWarps][kListCap] selected positions
  uint32_t* mask_s = reinterpret_cast<uint32_t*>(lst + kWarps * kListCap);  // [S / 32]
  float* sc = reinterpret_cast<float*>(mask_s + S / 32);                    // [G][S]

  const int split = p.split;
  const int rank = blockIdx.x % split;
  const int unit_id = blockIdx.x / split;
  const int H = p.n_heads;
  const int h = unit_id % H;
  const int b = (unit_id / H) % p.batch;
  const int ci = unit_id / (H * p.batch);
  const int cell = cl.cell[ci];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  // outputs (and queries) sit at the cell's index in the caller's list
  const size_t uidx = ((size_t)cl.out[ci] * p.batch + b) * H + h;

  const Unit u = resolve<RES2>(p, cell, b, h, D);
  if (!u.ok) {
    // Host checks make this unreachable; flag it and leave the outputs alone.
    // Every CTA of the cluster takes this branch together (same unit).
    if (tid == 0 && rank == 0)
      atomicOr(reinterpret_cast<uint32_t*>(const_cast<uint8_t*>(p.table)), kStatusLength);
    return;
  }
  const int chunk = ((u.npos + split - 1) / split + 31) / 32 * 32;
  const int p0 = rank * chunk;
  const int p1 = min(u.npos, p0 + chunk);
  if (chunk > S) {
    if (tid == 0 && rank == 0)
      atomicOr(reinterpret_cast<uint32_t*>(const_cast<uint8_t*>(p.table)), kStatusRange);
    return;
  }

  // the group's queries -> fp32 shared
  const uint16_t* qg = p.q + uidx * G * D;
  for (int d = tid; d < G * D; d += kThreads) q_s[d] = __uint_as_float((uint32_t)qg[d] << 16);
  __syncthreads();

  const bool quant = u.data_kind == LOOPKV_Q4 || u.data_kind == LOOPKV_Q2;
  const bool q4 = u.data_kind == LOOPKV_Q4;
  float* qs = qs_all + warp * G * D;
  const float sscale = p.score_scale;
  const int blk0 = p0 / 32;
  const int blk1 = (p1 + 31) / 32;
  const int nqb = quant ? (u.nq + 31) / 32 : 0;     // blocks holding quantized positions
  const int qend = min(blk1, nqb);

  // ------------------------------------------------------------- pass 1
  float lmax[G];
#pragma unroll
  for (int r = 0; r < G; ++r) lmax[r] = -INFINITY;
  if constexpr (G == 1) {
    if (q4) key_pass<D, true, G>(u, blk0, qend, p0, p1, q_s, qs, sc, S, sscale, warp, lane, lmax);
    else if (quant) key_pass<D, false, G>(u, blk0, qend, p0, p1, q_s, qs, sc, S, sscale, warp, lane, lmax);
  } else {
    if (q4) key_pass_mma<D, true, G>(u, blk0, qend, p0, p1, q_s, qs, sc, S, sscale, warp, lane, lmax);
    else if (quant)
      key_pass_mma<D, false, G>(u, blk0, qend, p0, p1, q_s, qs, sc, S, sscale, warp, lane, lmax);
  }
  // the warp's first value block is requested now, ahead of the softmax merge
  constexpr int LPT = (D / 64) * G;  // lanes per token in pass 2
  constexpr int TPI = 32 / LPT;      // tokens per warp iteration in pass 2
  const int hf = lane % LPT;
  const size_t vrow = D / 4;  // bytes per token of a value plane / value meta
  const int qlim = min(p1, u.nq);
  const size_t trow = ((size_t)(blk0 + warp) * 32 + lane / LPT) * vrow;
  const uint8_t* vh = u.data + u.Ld.v_hi + trow + hf * (VS::CH / 4);
  const uint8_t* vm = u.data + u.Ld.v_meta + trow + (hf * VS::CH / 32) * 8;
  constexpr size_t VSTEP = (size_t)kWarps * 32 * (D / 4);
  auto full_block = [&](int bk) { return (bk + 1) * 32 <= qlim; };
  // Up to two queries per KV head: the next block's rows wait in registers.
  // Four have no registers to spare: their blocks go through shared-memory
  // staging buffers (below).
  constexpr bool kRegNext = G <= 2;
  constexpr int NB = kRegNext ? LPT : 1;
  uint32_t nh[NB][VS::NW];
  float nm[NB][2 * VS::NGRP];
  if (kRegNext && blk0 + warp < blk1 && full_block(blk0 + warp)) {
#pragma unroll
    for (int it = 0; it < NB; ++it) {
      load_words<VS::NW>(nh[it], vh + it * TPI * vrow);
      load_meta<VS::NGRP>(nm[it], vm + it * TPI * vrow);
    }
  }
  // Four queries per KV head: full blocks go through two staging buffers
  // in shared memory, the next block's copy in flight while the current one
  // is used.  The buffers are the warp's own q * scale rows (free after
  // pass 1) and its rows of the final reduction (unused until then).
  uint8_t* const stg0 = reinterpret_cast<uint8_t*>(qs);
  uint8_t* const stg1 = reinterpret_cast<uint8_t*>(red + warp * G * D);
  static_assert(kRegNext || 16 * D <= 4 * G * D, "a staged value block must fit a warp's rows");
  int sti = 0;
  auto stage_first = [&]() {
    if (!kRegNext) {
      if (blk0 + warp < blk1 && full_block(blk0 + warp)) stage_vblock<D>(stg0, u, blk0 + warp, lane);
      cp_async_commit();
    }
  };
  if constexpr (!RES2) stage_first();
  // bf16 positions: residual, raw cells, the SHARE current token, a RES2
  // unit's window (and its bf16 reference's positions)
  for (int pos = max(p0, u.nq) + 32 * warp + lane; pos < p1; pos += 32 * kWarps) {
    float s[G];
    dot_bf16<D, G>(raw_row<RES2>(u, pos, D, false), q_s, s);
#pragma unroll
    for (int r = 0; r < G; ++r) {
      sc[r * S + pos - p0] = s[r] * sscale;
      lmax[r] = fmaxf(lmax[r], s[r] * sscale);
    }
  }
  if constexpr (RES2) {
    // residual keys: sc += sm_scale * <q, d^> over the residual-coded
    // positions (written above by the same threads: the same warp-strided
    // blocks, lane = token), then the maximum over the finished scores
    Unit ur = u;
    ur.data = u.own;
    ur.Ld = u.Lo;
    ur.data_kind = LOOPKV_Q2;
    ur.nq = u.rtok;
    if constexpr (G == 1)
      key_pass<D, false, G, true>(ur, blk0, min(blk1, u.rtok / 32), p0, p1, q_s, qs, sc, S, sscale,
                                  warp, lane, lmax);
    else
      key_pass_mma<D, false, G, true>(ur, blk0, min(blk1, u.rtok / 32), p0, p1, q_s, qs, sc, S,
                                      sscale, warp, lane, lmax);
    __syncthreads();
#pragma unroll
    for (int r = 0; r < G; ++r) {
      lmax[r] = -INFINITY;
      for (int i = tid; i < p1 - p0; i += kThreads) lmax[r] = fmaxf(lmax[r], sc[r * S + i]);
    }
    stage_first();  // the staging buffer is the q * scale rows the residual pass used
  }
#pragma unroll
  for (int r = 0; r < G; ++r) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) lmax[r] = fmaxf(lmax[r], __shfl_xor_sync(0xffffffffu, lmax[r], o));
    if (lane == 0) misc[warp * G + r] = lmax[r];
  }
  __syncthreads();
  float m_r[G];
#pragma unroll
  for (int r = 0; r < G; ++r) {
    m_r[r] = misc[r];
#pragma unroll
    for (int w = 1; w < kWarps; ++w) m_r[r] = fmaxf(m_r[r], misc[w * G + r]);
  }

  // exponentials relative to the CTA max, and their sum, per query
  float lsum[G];
#pragma unroll
  for (int r = 0; r < G; ++r) {
    lsum[r] = 0.f;
    for (int i = tid; i < p1 - p0; i += kThreads) {
      const float e = exp2f(sc[r * S + i] - m_r[r]);
      sc[r * S + i] = e;
      lsum[r] += e;
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) lsum[r] += __shfl_xor_sync(0xffffffffu, lsum[r], o);
    if (lane == 0) misc[32 + warp * G + r] = lsum[r];
  }
  __syncthreads();
  float l_r[G];
#pragma unroll
  for (int r = 0; r < G; ++r) {
    l_r[r] = 0.f;
#pragma unroll
    for (int w = 0; w < kWarps; ++w) l_r[r] += misc[32 + w * G + r];
    if (p1 <= p0) { m_r[r] = -INFINITY; l_r[r] = 0.f; }
  }

  // merge across the cluster: the unit's logsumexp per query (log2 units)
  float M[G], L[G];
#pragma unroll
  for (int r = 0; r < G; ++r) { M[r] = m_r[r]; L[r] = l_r[r]; }
  if (split > 1) {
    cg::cluster_group cluster = cg::this_cluster();
    if (tid == 0) {
#pragma unroll
      for (int r = 0; r < G; ++r) { misc[64 + r] = m_r[r]; misc[72 + r] = l_r[r]; }
    }
    cluster.sync();
#pragma unroll
    for (int r = 0; r < G; ++r) {
      M[r] = -INFINITY;
      for (int k = 0; k < split; ++k) M[r] = fmaxf(M[r], cluster.map_shared_rank(misc, k)[64 + r]);
      L[r] = 0.f;
      for (int k = 0; k < split; ++k) {
        const float* rm = cluster.map_shared_rank(misc, k);
        if (rm[72 + r] > 0.f) L[r] += rm[72 + r] * exp2f(rm[64 + r] - M[r]);
      }
    }
  }
  float f[G], fsub[G];  // e -> p, and p * 2^kSub for the low planes
#pragma unroll
  for (int r = 0; r < G; ++r) {
    f[r] = (l_r[r] > 0.f) ? exp2f(m_r[r] - M[r]) / L[r] : 0.f;
    fsub[r] = f[r] * pow2(kSub);
  }
  const float tau = p.tau;

  // ------------------------------------------------------------- pass 2
  float2 acc[G][32 / G];
#pragma unroll
  for (int r = 0; r < G; ++r)
#pragma unroll
    for (int i = 0; i < 32 / G; ++i) acc[r][i] = make_float2(0.f, 0.f);
  float gc[G][VS::NGRP];  // per-group constants of the lane's value groups, per query
#pragma unroll
  for (int r = 0; r < G; ++r)
#pragma unroll
    for (int gi = 0; gi < VS::NGRP; ++gi) gc[r][gi] = 0.f;
  int nsel = 0;
  // 4-bit high plane: weight 4 * p * scale; its missing low bits read as 1.5,
  // i.e. + 1.5 * p * scale = 0.375 * (4 * p * scale) per unselected token
  // (the value weights carry 2^kSub for the code conversion; mid_unsel takes
  // it back out for the constants)
  const float hmul = (q4 ? 4.f : 1.f) * pow2(kSub);
  const float mid_unsel = q4 ? 0.375f * pow2(-kSub) : 0.f;
  // tau <= 0 selects every 4-bit token: the low planes are read with the high
  // ones in this loop instead of through the selected-position list
  const bool dense_lo = DENSE_LO && q4;
  const size_t lo_off = u.Ld.v_lo - u.Ld.v_hi;
  // one token-row share of a full or partial block, for every query
  auto token_share = [&](const uint32_t (&hw)[VS::NW], const float (&mt)[2 * VS::NGRP],
                         const float (&pt)[G], float mid, const uint8_t* lo_row) {
    float a[G][VS::NGRP];
    if constexpr (G == 1) {
#pragma unroll
      for (int gi = 0; gi < VS::NGRP; ++gi) {
        a[0][gi] = (hmul * pt[0]) * mt[2 * gi];
        gc[0][gi] = fmaf(mid, a[0][gi], fmaf(pt[0], mt[2 * gi + 1], gc[0][gi]));
      }
    } else {
      // the group's weight scale and constant, once for every query:
      // a_r = p_r * (hmul * scale) (hmul a power of two: the same product),
      // constant p_r * (zero + mid * hmul * scale)
#pragma unroll
      for (int gi = 0; gi < VS::NGRP; ++gi) {
        const float hs = hmul * mt[2 * gi];
        const float zc = fmaf(mid * hmul, mt[2 * gi], mt[2 * gi + 1]);
#pragma unroll
        for (int r = 0; r < G; ++r) {
          a[r][gi] = pt[r] * hs;
          gc[r][gi] = fmaf(pt[r], zc, gc[r][gi]);
        }
      }
    }
    value_codes<G>(acc, hw, a);
    if (dense_lo) {
      uint32_t lw[VS::NW];
      load_words<VS::NW>(lw, lo_row);
#pragma unroll
      for (int r = 0; r < G; ++r)
#pragma unroll
        for (int gi = 0; gi < VS::NGRP; ++gi) a[r][gi] *= 0.25f;
      value_codes<G>(acc, lw, a);
    }
  };
  for (int bk = blk0 + warp; bk < blk1; bk += kWarps, vh += VSTEP, vm += VSTEP) {
    const int pos = bk * 32 + lane;
    const bool active = pos < p1;
    float pw[G];
    bool any = false;
#pragma unroll
    for (int r = 0; r < G; ++r) {
      pw[r] = active ? sc[r * S + pos - p0] * f[r] : 0.f;
      any = any || pw[r] >= tau;
    }
    const bool sel = q4 && pos < qlim && any;
    const uint32_t ballot = __ballot_sync(0xffffffffu, sel);
    nsel += __popc(ballot);
    if (lane == 0) {
      mask_s[bk - blk0] = ballot;
      if (p.mask != nullptr && q4 && bk < nqb) p.mask[uidx * p.mask_words + bk] = ballot;
    }
    if (kRegNext && full_block(bk)) {
      // a full quantized block: rows arrived with the previous iteration
      uint32_t hw[LPT][VS::NW];
      float mt[LPT][2 * VS::NGRP];
#pragma unroll
      for (int it = 0; it < NB; ++it) {
#pragma unroll
        for (int k = 0; k < VS::NW; ++k) hw[it][k] = nh[it][k];
#pragma unroll
        for (int k = 0; k < 2 * VS::NGRP; ++k) mt[it][k] = nm[it][k];
      }
      if (bk + kWarps < blk1 && full_block(bk + kWarps)) {
#pragma unroll
        for (int it = 0; it < NB; ++it) {
          load_words<VS::NW>(nh[it], vh + VSTEP + it * TPI * vrow);
          load_meta<VS::NGRP>(nm[it], vm + VSTEP + it * TPI * vrow);
        }
        // vh sits 16 lane bytes into the block's rows when G = 1, so lanes
        // with lane % 8 == 0 start its lines
        if (G == 1 && kAheadV > 0 && (lane & 7) == 0) {
#pragma unroll
          for (int c = 0; c < D / 64; ++c) {
            prefetch_l2(vh + kAheadV * VSTEP + c * 512);
            prefetch_l2(vm + kAheadV * VSTEP + c * 512);
          }
        }
      }
#pragma unroll
      for (int it = 0; it < LPT; ++it) {
        const int tk = it * TPI + lane / LPT;
        float pt[G];
#pragma unroll
        for (int r = 0; r < G; ++r) pt[r] = __shfl_sync(0xffffffffu, pw[r], tk);
        const float mid = ((ballot >> tk) & 1u) ? 0.f : mid_unsel;
        token_share(hw[it], mt[it], pt, mid, vh + lo_off + it * TPI * vrow);
      }
    } else if (!kRegNext && full_block(bk)) {
      // a full quantized block from its staging buffer; the next full block
      // is copied into the other one meanwhile
      const uint8_t* cur = sti ? stg1 : stg0;
      if (bk + kWarps < blk1 && full_block(bk + kWarps))
        stage_vblock<D>(sti ? stg0 : stg1, u, bk + kWarps, lane);
      cp_async_commit();
      cp_async_wait<1>();
      __syncwarp();
#pragma unroll
      for (int it = 0; it < LPT; ++it) {
        const int tk = it * TPI + lane / LPT;
        float pt[G];
#pragma unroll
        for (int r = 0; r < G; ++r) pt[r] = __shfl_sync(0xffffffffu, pw[r], tk);
        uint32_t hwv[VS::NW];
        float mtv[2 * VS::NGRP];
        lds_words<VS::NW>(hwv, cur + tk * vrow + hf * (VS::CH / 4));
        lds_meta<VS::NGRP>(mtv, cur + 8 * D + tk * vrow + (hf * VS::CH / 32) * 8);
        const float mid = ((ballot >> tk) & 1u) ? 0.f : mid_unsel;
        token_share(hwv, mtv, pt, mid, vh + lo_off + it * TPI * vrow);
      }
      __syncwarp();  // the buffer is refilled two blocks on
      sti ^= 1;
    } else {
      // partial block: quantized tokens below qlim, bf16 ones up to p1
#pragma unroll
      for (int it = 0; it < LPT; ++it) {
        const int tk = it * TPI + lane / LPT;
        float pt[G];
#pragma unroll
        for (int r = 0; r < G; ++r) pt[r] = __shfl_sync(0xffffffffu, pw[r], tk);
        const int tpos = bk * 32 + tk;
        if (tpos < qlim) {
          uint32_t hwv[VS::NW];
          float mtv[2 * VS::NGRP];
          load_words<VS::NW>(hwv, vh + it * TPI * vrow);
          load_meta<VS::NGRP>(mtv, vm + it * TPI * vrow);
          const float mid = ((ballot >> tk) & 1u) ? 0.f : mid_unsel;
          token_share(hwv, mtv, pt, mid, vh + lo_off + it * TPI * vrow);
        } else if (tpos < p1) {
          value_raw<G>(acc, raw_row<RES2>(u, tpos, D, true) + hf * VS::CH * 2, pt);
        }
      }
    }
  }
  if (!kRegNext) cp_async_wait<0>();  // nothing stays in flight into the reduction rows
  if constexpr (RES2) {
    // residual values: acc += p * (scale * code + zero) of the unit's own
    // 2-bit residual rows, every residual-coded position (full blocks)
    const uint8_t* rvh = u.own + u.Lo.v_hi;
    const uint8_t* rvm = u.own + u.Lo.v_meta;
    const float rmul = pow2(kSub);
    for (int bk = blk0 + warp; bk < min(blk1, u.rtok / 32); bk += kWarps) {
      float pw[G];
#pragma unroll
      for (int r = 0; r < G; ++r) pw[r] = sc[r * S + bk * 32 + lane - p0] * f[r];
#pragma unroll
      for (int it = 0; it < LPT; ++it) {
        const int tk = it * TPI + lane / LPT;
        float pt[G];
#pragma unroll
        for (int r = 0; r < G; ++r) pt[r] = __shfl_sync(0xffffffffu, pw[r], tk);
        const size_t row = (size_t)(bk * 32 + tk) * vrow;
        uint32_t hw[VS::NW];
        float mt[2 * VS::NGRP];
        load_words<VS::NW>(hw, rvh + row + hf * (VS::CH / 4));
        load_meta<VS::NGRP>(mt, rvm + row + (hf * VS::CH / 32) * 8);
        float a[G][VS::NGRP];
#pragma unroll
        for (int r = 0; r < G; ++r)
#pragma unroll
          for (int gi = 0; gi < VS::NGRP; ++gi) {
            a[r][gi] = (rmul * pt[r]) * mt[2 * gi];
            gc[r][gi] = fmaf(pt[r], mt[2 * gi + 1], gc[r][gi]);
          }
        value_codes<G>(acc, hw, a);
      }
    }
  }
  // low planes of the selected tokens: acc += p * scale * lo.  The warp
  // gathers its selected positions into a list and processes them TPI at a
  // time, so the cost follows the number of selected tokens.
  if (q4 && !dense_lo) {
    __syncwarp();  // the warp reads only the mask words its own lane 0 wrote
    int* my = lst + warp * kListCap;
    int nlist = 0;
    for (int bk = blk0 + warp; bk < qend; bk += kWarps) {
      const uint32_t word = mask_s[bk - blk0];
      if (word == 0u) continue;
      const int cnt = __popc(word);
      if (nlist + cnt > kListCap) {
        low_planes<D, G, LPT>(acc, u, my, nlist, sc, S, p0, fsub, lane);
        nlist = 0;
      }
      if ((word >> lane) & 1u) my[nlist + __popc(word & ((1u << lane) - 1u))] = bk * 32 + lane;
      nlist += cnt;
      __syncwarp();
    }
    if (nlist > 0) low_planes<D, G, LPT>(acc, u, my, nlist, sc, S, p0, fsub, lane);
  }
  // undo the per-channel 2^o of the code conversion, add the per-group
  // constants, then reduce over the lanes that share a channel range
#pragma unroll
  for (int r = 0; r < G; ++r)
#pragma unroll
    for (int i = 0; i < 32 / G; ++i) {
      const int j = (2 * i) & 15;
      const float gcon = gc[r][(2 * i) / 32];
      acc[r][i].x = fmaf(acc[r][i].x, pow2(149 - kSub - code2_off(j)), gcon);
      acc[r][i].y = fmaf(acc[r][i].y, pow2(149 - kSub - code2_off(j + 1)), gcon);
    }
  {
    // transposed butterfly over the TPI lanes with the same lane % LPT: each
    // step keeps half of the values (the upper half where the step's lane
    // bit is set) and adds the partner's copy of them, so the lane ends with
    // NVL consecutive sums of the flattened [G][CH] slice, from index
    // 2 (lane - lane % LPT) on
    constexpr int NV = G * VS::CH;    // 64
    constexpr int NVL = 2 * LPT;      // = NV / TPI
    float v[NV];
#pragma unroll
    for (int r = 0; r < G; ++r)
#pragma unroll
      for (int i = 0; i < VS::CH / 2; ++i) {
        v[r * VS::CH + 2 * i] = acc[r][i].x;
        v[r * VS::CH + 2 * i + 1] = acc[r][i].y;
      }
#pragma unroll
    for (int o = 16; o >= LPT; o >>= 1) {
      const int half = NV * o / 32;
      const bool up = (lane & o) != 0;
#pragma unroll
      for (int j = 0; j < half; ++j) {
        const float keep = up ? v[j + half] : v[j];
        const float send = up ? v[j] : v[j + half];
        v[j] = keep + __shfl_xor_sync(0xffffffffu, send, o);
      }
    }
    const int base = 2 * (lane - hf);  // flattened index of v[0]
    float* dst = red + (warp * G + base / VS::CH) * D + hf * VS::CH + base % VS::CH;
    if constexpr (NVL == 2) {
      *reinterpret_cast<float2*>(dst) = make_float2(v[0], v[1]);
    } else {
#pragma unroll
      for (int k = 0; k < NVL / 4; ++k)
        reinterpret_cast<float4*>(dst)[k] = make_float4(v[4 * k], v[4 * k + 1], v[4 * k + 2], v[4 * k + 3]);
    }
  }
  if (lane == 0) misc[80 + warp] = __int_as_float(nsel);
  __syncthreads();
  for (int d = tid; d < G * D; d += kThreads) {
    float o = 0.f;
#pragma unroll
    for (int w = 0; w < kWarps; ++w) o += red[w * G * D + d];
    o_s[d] = o;
  }
  if (tid == 0) {
    int t = 0;
    for (int w = 0; w < kWarps; ++w) t += __float_as_int(misc[80 + w]);
    misc[88] = __int_as_float(t);
  }
  __syncthreads();

  if (split > 1) {
    cg::cluster_group cluster = cg::this_cluster();
    cluster.sync();
    if (rank == 0) {
      for (int d = tid; d < G * D; d += kThreads) {
        float o = 0.f;
        for (int k = 0; k < split; ++k) o += cluster.map_shared_rank(o_s, k)[d];
        p.out[uidx * G * D + d] = o;
      }
      if (tid == 0) {
        int t = 0;
        for (int k = 0; k < split; ++k) t += __float_as_int(cluster.map_shared_rank(misc, k)[88]);
        if (p.nsel) p.nsel[uidx] = t;
        if (p.lse) {
#pragma unroll
          for (int r = 0; r < G; ++r) p.lse[uidx * G + r] = (M[r] + log2f(L[r])) * 0.69314718055994531f;
        }
      }
    }
    cluster.sync();  // keep every CTA's shared memory alive until rank 0 has read it
  } else {
    for (int d = tid; d < G * D; d += kThreads) p.out[uidx * G * D + d] = o_s[d];
    if (tid == 0) {
      if (p.nsel) p.nsel[uidx] = __float_as_int(misc[88]);
      if (p.lse) {
#pragma unroll
        for (int r = 0; r < G; ++r) p.lse[uidx * G + r] = (M[r] + log2f(L[r])) * 0.69314718055994531f;
      }
    }
  }
}

// Shared memory of one CTA for S score slots per query.
template <int D, int G>
constexpr size_t decode_smem(int S) {
  return sizeof(float) * ((size_t)G * D * (2 + 2 * kWarps) + 128 + kWarps * kListCap + S / 32 +
                          (size_t)G * S);
}

template <int D, int G, bool DENSE_LO, bool RES2>
int launch_decode_t(const DecodeParams& p, const CellList& cells, cudaStream_t stream) {
  const size_t smem = decode_smem<D, G>(p.slots);
  cudaError_t e = cudaFuncSetAttribute(decode_kernel<D, G, DENSE_LO, RES2>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return (int)e;
  const long long units = (long long)p.n_cells * p.batch * p.n_heads;
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = dim3((unsigned)(units * p.split), 1, 1);
  cfg.blockDim = dim3(kThreads, 1, 1);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  int nattr = 0;
  if (p.split > 1) {
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = p.split;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    nattr = 1;
  }
  cfg.attrs = attr;
  cfg.numAttrs = nattr;
  e = cudaLaunchKernelEx(&cfg, decode_kernel<D, G, DENSE_LO, RES2>, p, cells);
  return (int)e;
}

template <int D, int G, bool RES2>
int launch_decode_g(const DecodeParams& p, const CellList& cells, cudaStream_t s) {
  const bool dense = !(p.tau > 0.f);
  return dense ? launch_decode_t<D, G, true, RES2>(p, cells, s)
               : launch_decode_t<D, G, false, RES2>(p, cells, s);
}

template <int D, bool RES2>
int launch_decode_d(const DecodeParams& p, const CellList& cells, cudaStream_t s) {
  if (p.group == 2) return launch_decode_g<D, 2, RES2>(p, cells, s);
  if (p.group == 4) return launch_decode_g<D, 4, RES2>(p, cells, s);
  return launch_decode_g<D, 1, RES2>(p, cells, s);
}

// Largest score slots per query that keep two CTAs on an SM (at most
// kMaxSlots in all), for a group of G queries.
template <int D, int G>
constexpr int max_slots_g() {
  constexpr size_t kBudget = 113 * 1024;  // bytes of shared memory per CTA for two CTAs per SM
  constexpr size_t fixed = decode_smem<D, G>(0);
  constexpr size_t per_query = (kBudget - fixed) / sizeof(float);  // G * S + S / 32 <= this
  constexpr size_t s = per_query * 32 / (32 * G + 1) / 32 * 32;
  return (int)(s * G > (size_t)kMaxSlots ? kMaxSlots / G : s);
}

}  // namespace

int decode_max_slots(int head_dim, int group) {
  if (head_dim == 64)
    return group == 4 ? max_slots_g<64, 4>() : group == 2 ? max_slots_g<64, 2>() : max_slots_g<64, 1>();
  return group == 4 ? max_slots_g<128, 4>() : group == 2 ? max_slots_g<128, 2>() : max_slots_g<128, 1>();
}
int decode_max_split() { return kMaxSplit; }

int launch_decode(const DecodeParams& p, const CellList& cells, void* stream, int head_dim,
                  bool res2) {
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (head_dim == 64) return res2 ? launch_decode_d<64, true>(p, cells, s) : launch_decode_d<64, false>(p, cells, s);
  return res2 ? launch_decode_d<128, true>(p, cells, s) : launch_decode_d<128, false>(p, cells, s);
}

}  // namespace loopkv
