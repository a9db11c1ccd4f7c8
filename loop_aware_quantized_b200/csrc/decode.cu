// LoopKV fused decode attention for sm_100a.
//
// "LoopKV: Loop-Aware KV Cache Compression for Serving Looped Transformers",
// section 概要: each loop reads the high 2 bits of every 4-bit value and
// fetches the low 2 bits only where its own attention weights require 4-bit
// precision; one fused kernel runs the per-cell plan.
//
// One CTA (8 warps) handles a contiguous, 32-aligned range of one unit's
// attended positions; when a unit is split over several CTAs they form a
// thread-block cluster and exchange their partial softmax statistics and
// partial outputs through distributed shared memory, so no global
// workspace is needed.  The scores of the CTA's range stay in shared memory
// between the two passes:
//   pass 1  keys: per 32-token group, q is folded with the group's per-channel
//           key scales (qs_d = q_d * scale_d) and zero points
//           (c = sum_d q_d * zero_d), then each lane (one token) forms
//           sum_d qs_d * code_d + c from its packed planes.  Scores are kept
//           in log2 units.
//   softmax the CTA's max and sum of exponentials, merged across the cluster
//           into the unit's logsumexp.
//   pass 2  values: lane = position computes p and the selection p >= tau
//           (a warp ballot gives the mask word of the group); lanes then
//           work per token (64 channels per lane) accumulating
//           p * scale * code in fp32 and the per-group constant
//           p * (zero [+ 1.5 * scale]) separately; the low plane row of a
//           token is loaded only when the token is selected.
//   combine warp shuffles reduce the per-token partial outputs, shared
//           memory reduces across warps, DSMEM across the cluster.
// No tensor cores: one query per KV head makes this a stream over the
// cache, bound by HBM bandwidth.

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
  bool has_cur;
  bool ok;
};

__device__ Unit resolve(const DecodeParams& p, int cell, int b, int h, int D) {
  Unit u{};
  const TableHeader* hdr = reinterpret_cast<const TableHeader*>(p.table);
  const DevCell* cells = reinterpret_cast<const DevCell*>(p.table + table_cells_offset());
  const DevSeq* seqs = reinterpret_cast<const DevSeq*>(p.table + table_seqs_offset(hdr->n_cells));
  const int B = hdr->max_batch;
  const DevCell oc = cells[cell];
  const DevSeq os = seqs[(size_t)cell * B + b];
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

// Pointer to the bf16 key (or value) row of a raw position.
__device__ __forceinline__ const uint8_t* raw_row(const Unit& u, int pos, int D, bool value) {
  if (u.has_cur && pos == u.n_att) return u.own + (value ? u.Lo.cur_v : u.Lo.cur_k);
  if (u.data_kind == LOOPKV_BF16)
    return u.data + (value ? u.Ld.raw_v : u.Ld.raw_k) + (size_t)pos * D * 2;
  return u.data + (value ? u.Ld.res_v : u.Ld.res_k) + (size_t)(pos - u.qtok) * D * 2;
}

template <int D>
__device__ __forceinline__ float dot_bf16(const uint8_t* row, const float* q_s) {
  float acc = 0.f;
#pragma unroll
  for (int c = 0; c < D / 8; ++c) {
    const uint4 w = ldg128(row + c * 16);
    const float4 qa = *reinterpret_cast<const float4*>(q_s + 8 * c);
    const float4 qb = *reinterpret_cast<const float4*>(q_s + 8 * c + 4);
    acc = fmaf(qa.x, bf16_lo(w.x), acc);
    acc = fmaf(qa.y, bf16_hi(w.x), acc);
    acc = fmaf(qa.z, bf16_lo(w.y), acc);
    acc = fmaf(qa.w, bf16_hi(w.y), acc);
    acc = fmaf(qb.x, bf16_lo(w.z), acc);
    acc = fmaf(qb.y, bf16_hi(w.z), acc);
    acc = fmaf(qb.z, bf16_lo(w.w), acc);
    acc = fmaf(qb.w, bf16_hi(w.w), acc);
  }
  return acc;
}

// Score of one quantized token: sum_d qs_d * code_d over the token's packed
// planes (16-byte rows h[c], l[c] of K_hi / K_lo for chunk c of 64 channels).
template <int D, bool Q4>
__device__ __forceinline__ float dot_codes(const uint4 (&h)[D / 64], const uint4 (&l)[D / 64],
                                           const float2* qs2) {
  // four independent accumulators keep the fma chain short
  float2 acc[4];
#pragma unroll
  for (int k = 0; k < 4; ++k) acc[k] = make_float2(0.f, 0.f);
#pragma unroll
  for (int c = 0; c < D / 64; ++c) {
    const uint32_t hw[4] = {h[c].x, h[c].y, h[c].z, h[c].w};
    const uint32_t lw[4] = {l[c].x, l[c].y, l[c].z, l[c].w};
#pragma unroll
    for (int w = 0; w < 4; ++w) {
      float2 v[8];
      if (Q4) codes4_to_pairs(hw[w], lw[w], v);
      else codes2_to_pairs(hw[w], v);
      const float4* q4p = reinterpret_cast<const float4*>(qs2 + 32 * c + 8 * w);
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const float4 qq = q4p[i];
        acc[(2 * i) & 3] = fma2(make_float2(qq.x, qq.y), v[2 * i], acc[(2 * i) & 3]);
        acc[(2 * i + 1) & 3] = fma2(make_float2(qq.z, qq.w), v[2 * i + 1], acc[(2 * i + 1) & 3]);
      }
    }
  }
  const float2 a = add2(acc[0], acc[1]), b = add2(acc[2], acc[3]);
  return (a.x + b.x) + (a.y + b.y);
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

// Score one group held in registers; returns the lane's score (or -inf).
template <int D, bool Q4>
__device__ __forceinline__ float key_group(const KGroup<D>& g, const float (&qv)[D / 32],
                                           const float (&qz)[D / 32], float* qs, int pos,
                                           int qlim, float sscale,
                                           int lane) {
  constexpr int CPL = D / 32;
  // fold q into the group's key scale / zero point
  float cpart = 0.f;
#pragma unroll
  for (int i = 0; i < CPL; ++i) {
    qs[CPL * lane + i] = qv[i] * g.sc[i];
    cpart = fmaf(qz[i], g.zr[i], cpart);
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) cpart += __shfl_xor_sync(0xffffffffu, cpart, o);
  __syncwarp();
  float s = -INFINITY;
  if (pos < qlim) {
    const float dot = dot_codes<D, Q4>(g.h, g.l, reinterpret_cast<const float2*>(qs));
    s = fmaf(dot, pow2(149 - kSub) * sscale, cpart * sscale);
  }
  __syncwarp();
  return s;
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
// while the current one is scored, without copies between them.
template <int D, bool Q4>
__device__ __forceinline__ float key_pass(const Unit& u, int b_begin, int b_end, int p0, int p1,
                                          const float* q_s, float* qs, float* sc, float sscale,
                                          int warp, int lane) {
  constexpr int CPL = D / 32;  // channels per lane for the q fold
  float lmax = -INFINITY;
  const int first = b_begin + warp;
  if (first >= b_end) return lmax;
  // q of the lane's channels, times 2^-o: o is the bit offset the channel's
  // code keeps after conversion (see codes4_to_pairs / codes2_to_pairs)
  float qv[CPL], qz[CPL];
#pragma unroll
  for (int i = 0; i < CPL; ++i) {
    const int j = (CPL * lane + i) & 15;
    qz[i] = q_s[CPL * lane + i];
    qv[i] = qz[i] * pow2(kSub - (Q4 ? code4_off(j >> 1) : code2_off(j)));
  }
  const int qlim = min(p1, u.nq);
  constexpr size_t G = 8 * D;                       // bytes of one group in each block
  constexpr size_t STEP = (size_t)kWarps * G;       // a warp's stride between its groups
  const uint8_t* kh = u.data + u.Ld.k_hi + (size_t)first * G + lane * 16;
  const size_t lo_off = u.Ld.k_lo - u.Ld.k_hi;
  const float* km = reinterpret_cast<const float*>(u.data + u.Ld.k_meta + (size_t)first * G) +
                    CPL * lane;
  const bool pon = (lane & 7) == 0;  // lanes whose row pointers start a line
  KGroup<D> a, b;
  load_kgroup<D, Q4>(a, kh, lo_off, km);
  int bk = first;
  for (;;) {
    const bool hasb = bk + kWarps < b_end;
    if (hasb) load_kgroup<D, Q4>(b, kh + STEP, lo_off, km + STEP / 4);
    if (kAheadK > 0 && pon && hasb) prefetch_kgroup<D, Q4>(kh + kAheadK * STEP, lo_off, km + kAheadK * STEP / 4);
    float s = key_group<D, Q4>(a, qv, qz, qs, bk * 32 + lane, qlim, sscale, lane);
    if (bk * 32 + lane < qlim) { sc[bk * 32 + lane - p0] = s; lmax = fmaxf(lmax, s); }
    if (!hasb) break;
    bk += kWarps;
    kh += STEP;
    km += STEP / 4;
    const bool hasa = bk + kWarps < b_end;
    if (hasa) load_kgroup<D, Q4>(a, kh + STEP, lo_off, km + STEP / 4);
    if (kAheadK > 0 && pon && hasa) prefetch_kgroup<D, Q4>(kh + kAheadK * STEP, lo_off, km + kAheadK * STEP / 4);
    s = key_group<D, Q4>(b, qv, qz, qs, bk * 32 + lane, qlim, sscale, lane);
    if (bk * 32 + lane < qlim) { sc[bk * 32 + lane - p0] = s; lmax = fmaxf(lmax, s); }
    if (!hasa) break;
    bk += kWarps;
    kh += STEP;
    km += STEP / 4;
  }
  return lmax;
}

// Value accumulation of one quantized token half-row (64 channels): acc +=
// (a_j) * code * 2^o for the lane's two 32-channel groups (a0 for words 0-1,
// a1 for words 2-3); the 2^o of each channel is removed once at the end.
__device__ __forceinline__ void value_codes(float2 (&acc)[32], const uint4 hw4, float a0, float a1) {
  const uint32_t hw[4] = {hw4.x, hw4.y, hw4.z, hw4.w};
#pragma unroll
  for (int w = 0; w < 4; ++w) {
    float2 v[8];
    codes2_to_pairs(hw[w], v);
    const float a = (w < 2) ? a0 : a1;
    const float2 aa = make_float2(a, a);
#pragma unroll
    for (int i = 0; i < 8; ++i) acc[8 * w + i] = fma2(aa, v[i], acc[8 * w + i]);
  }
}

// bf16 value row (64 channels) with weight pt, in the accumulators' scaled
// representation (channel j of a 16-channel word carries 2^o(j)).
__device__ __forceinline__ void value_raw(float2 (&acc)[32], const uint8_t* row, float pt) {
#pragma unroll
  for (int c = 0; c < 8; ++c) {
    const uint4 w = ldg128(row + c * 16);
    const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const int pair = 4 * c + k;          // channels 2*pair, 2*pair+1
      const int j = (2 * pair) & 15;       // position inside the 16-channel word
      const float2 wt = make_float2(pt * pow2(code2_off(j) + kSub - 149),
                                    pt * pow2(code2_off(j + 1) + kSub - 149));
      acc[pair] = fma2(wt, make_float2(bf16_lo(ws[k]), bf16_hi(ws[k])), acc[pair]);
    }
  }
}

// Low planes of queued selected positions: acc += p * scale * lo, TPI
// positions per warp iteration (LPT lanes per position, 64 channels each).
template <int D, int LPT>
__device__ __forceinline__ void low_planes(float2 (&acc)[32], const Unit& u, const int* list,
                                           int n, const float* sc, int p0, float f, int lane) {
  constexpr int TPI = 32 / LPT;
  const int hf = lane % LPT;
  for (int k0 = 0; k0 < n; k0 += TPI) {
    const int kk = k0 + lane / LPT;
    if (kk < n) {
      const int tpos = list[kk];
      const float pt = sc[tpos - p0] * f;
      const uint4 lw = ld_stream(u.data + u.Ld.v_lo + (size_t)tpos * (D / 4) + hf * 16);
      const float4 m4 = ldg128f(u.data + u.Ld.v_meta + (size_t)tpos * (D / 4) + hf * 16);
      value_codes(acc, lw, pt * m4.x, pt * m4.z);
    }
  }
  __syncwarp();
}

// DENSE_LO: tau <= 0, every 4-bit token takes its low plane (read densely in
// the value loop); otherwise low planes come from the selected-position list.
template <int D, bool DENSE_LO>
__global__ void __launch_bounds__(kThreads, 2)
decode_kernel(const DecodeParams p, const CellList cl) {
  extern __shared__ __align__(16) float smem[];
  float* q_s = smem;                                  // [D]
  float* qs_all = q_s + D;                            // [kWarps][D]
  float* red = qs_all + kWarps * D;                   // [kWarps][D]
  float* o_s = red + kWarps * D;                      // [D]
  float* misc = o_s + D;                              // [64]
  int* lst = reinterpret_cast<int*>(misc + 64);       // [kWarps][kListCap] selected positions
  uint32_t* mask_s = reinterpret_cast<uint32_t*>(lst + kWarps * kListCap);  // [slots / 32]
  float* sc = reinterpret_cast<float*>(mask_s + p.slots / 32);        // [slots]

  const int split = p.split;
  const int rank = blockIdx.x % split;
  const int unit_id = blockIdx.x / split;
  const int H = p.n_heads;
  const int h = unit_id % H;
  const int b = (unit_id / H) % p.batch;
  const int ci = unit_id / (H * p.batch);
  const int cell = cl.cell[ci];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const size_t uidx = ((size_t)ci * p.batch + b) * H + h;

  const Unit u = resolve(p, cell, b, h, D);
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
  if (chunk > p.slots) {
    if (tid == 0 && rank == 0)
      atomicOr(reinterpret_cast<uint32_t*>(const_cast<uint8_t*>(p.table)), kStatusRange);
    return;
  }

  // query -> fp32 shared
  const uint16_t* qg = p.q + uidx * D;
  for (int d = tid; d < D; d += kThreads) q_s[d] = __uint_as_float((uint32_t)qg[d] << 16);
  __syncthreads();

  const bool quant = u.data_kind == LOOPKV_Q4 || u.data_kind == LOOPKV_Q2;
  const bool q4 = u.data_kind == LOOPKV_Q4;
  float* qs = qs_all + warp * D;
  const float sscale = p.score_scale;
  const int blk0 = p0 / 32;
  const int blk1 = (p1 + 31) / 32;
  const int nqb = quant ? (u.nq + 31) / 32 : 0;     // blocks holding quantized positions
  const int qend = min(blk1, nqb);

  // ------------------------------------------------------------- pass 1
  float lmax = -INFINITY;
  if (q4) lmax = key_pass<D, true>(u, blk0, qend, p0, p1, q_s, qs, sc, sscale, warp, lane);
  else if (quant)
    lmax = key_pass<D, false>(u, blk0, qend, p0, p1, q_s, qs, sc, sscale, warp, lane);
  // the warp's first value block is requested now, ahead of the softmax merge
  constexpr int LPT = D / 64;       // lanes per token in pass 2 (64 channels per lane)
  constexpr int TPI = 32 / LPT;     // tokens per warp iteration in pass 2
  const int hf = lane % LPT;
  const size_t vrow = D / 4;  // bytes per token of a value plane / value meta
  const int qlim = min(p1, u.nq);
  const size_t row0 = ((size_t)(blk0 + warp) * 32 + lane / LPT) * vrow + hf * 16;
  const uint8_t* vh = u.data + u.Ld.v_hi + row0;
  const uint8_t* vm = u.data + u.Ld.v_meta + row0;
  constexpr size_t VSTEP = (size_t)kWarps * 32 * (D / 4);
  auto full_block = [&](int bk) { return (bk + 1) * 32 <= qlim; };
  uint4 nh[LPT];
  float4 nm[LPT];
  if (blk0 + warp < blk1 && full_block(blk0 + warp)) {
#pragma unroll
    for (int it = 0; it < LPT; ++it) {
      nh[it] = ld_stream(vh + it * TPI * vrow);
      nm[it] = ldg128f(vm + it * TPI * vrow);
    }
  }
  // bf16 positions: residual, raw cells, the SHARE current token
  for (int pos = max(p0, u.nq) + 32 * warp + lane; pos < p1; pos += 32 * kWarps) {
    const float s = dot_bf16<D>(raw_row(u, pos, D, false), q_s) * sscale;
    sc[pos - p0] = s;
    lmax = fmaxf(lmax, s);
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) lmax = fmaxf(lmax, __shfl_xor_sync(0xffffffffu, lmax, o));
  if (lane == 0) misc[warp] = lmax;
  __syncthreads();
  float m_r = misc[0];
#pragma unroll
  for (int w = 1; w < kWarps; ++w) m_r = fmaxf(m_r, misc[w]);

  // exponentials relative to the CTA max, and their sum
  float lsum = 0.f;
  for (int i = tid; i < p1 - p0; i += kThreads) {
    const float e = exp2f(sc[i] - m_r);
    sc[i] = e;
    lsum += e;
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) lsum += __shfl_xor_sync(0xffffffffu, lsum, o);
  __syncthreads();  // everyone has read misc[]
  if (lane == 0) misc[8 + warp] = lsum;
  __syncthreads();
  float l_r = 0.f;
#pragma unroll
  for (int w = 0; w < kWarps; ++w) l_r += misc[8 + w];
  if (p1 <= p0) { m_r = -INFINITY; l_r = 0.f; }

  // merge across the cluster: unit logsumexp (log2 units)
  float M = m_r, L = l_r;
  if (split > 1) {
    cg::cluster_group cluster = cg::this_cluster();
    if (tid == 0) { misc[16] = m_r; misc[17] = l_r; }
    cluster.sync();
    M = -INFINITY;
    for (int r = 0; r < split; ++r) M = fmaxf(M, cluster.map_shared_rank(misc, r)[16]);
    L = 0.f;
    for (int r = 0; r < split; ++r) {
      const float* rm = cluster.map_shared_rank(misc, r);
      if (rm[17] > 0.f) L += rm[17] * exp2f(rm[16] - M);
    }
  }
  const float f = (l_r > 0.f) ? exp2f(m_r - M) / L : 0.f;  // e -> p
  const float tau = p.tau;

  // ------------------------------------------------------------- pass 2
  float2 acc[32];
#pragma unroll
  for (int i = 0; i < 32; ++i) acc[i] = make_float2(0.f, 0.f);
  float g0 = 0.f, g1 = 0.f;  // per-group constants of the lane's two 32-channel groups
  int nsel = 0;
  // 4-bit high plane: weight 4 * p * scale; its missing low bits read as 1.5,
  // i.e. + 1.5 * p * scale = 0.375 * (4 * p * scale) per unselected token
  // (the value weights carry 2^kSub for the code conversion; mid_unsel takes
  // it back out for the constants)
  const float hmul = (q4 ? 4.f : 1.f) * pow2(kSub);
  const float mid_unsel = q4 ? 0.375f * pow2(-kSub) : 0.f;
  const float fsub = f * pow2(kSub);  // e -> p * 2^kSub for the low planes
  // tau <= 0 selects every 4-bit token: the low planes are read with the high
  // ones in this loop instead of through the selected-position list
  const bool dense_lo = DENSE_LO && q4;
  const size_t lo_off = u.Ld.v_lo - u.Ld.v_hi;
  for (int bk = blk0 + warp; bk < blk1; bk += kWarps, vh += VSTEP, vm += VSTEP) {
    const int pos = bk * 32 + lane;
    const bool active = pos < p1;
    const float pw = active ? sc[pos - p0] * f : 0.f;
    const bool sel = q4 && pos < qlim && pw >= tau;
    const uint32_t ballot = __ballot_sync(0xffffffffu, sel);
    nsel += __popc(ballot);
    if (lane == 0) {
      mask_s[bk - blk0] = ballot;
      if (p.mask != nullptr && q4 && bk < nqb) p.mask[uidx * p.mask_words + bk] = ballot;
    }
    if (full_block(bk)) {
      // a full quantized block: rows arrived with the previous iteration
      uint4 hw[LPT];
      float4 mt[LPT];
#pragma unroll
      for (int it = 0; it < LPT; ++it) { hw[it] = nh[it]; mt[it] = nm[it]; }
      if (bk + kWarps < blk1 && full_block(bk + kWarps)) {
#pragma unroll
        for (int it = 0; it < LPT; ++it) {
          nh[it] = ld_stream(vh + VSTEP + it * TPI * vrow);
          nm[it] = ldg128f(vm + VSTEP + it * TPI * vrow);
        }
        if (kAheadV > 0 && (lane & 7) == 0) {
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
        const float pt = __shfl_sync(0xffffffffu, pw, tk);
        const float mid = ((ballot >> tk) & 1u) ? 0.f : mid_unsel;
        const float a0 = (hmul * pt) * mt[it].x, a1 = (hmul * pt) * mt[it].z;
        g0 = fmaf(mid, a0, fmaf(pt, mt[it].y, g0));
        g1 = fmaf(mid, a1, fmaf(pt, mt[it].w, g1));
        value_codes(acc, hw[it], a0, a1);
        if (dense_lo)
          value_codes(acc, ld_stream(vh + lo_off + it * TPI * vrow), 0.25f * a0, 0.25f * a1);
      }
    } else {
      // partial block: quantized tokens below qlim, bf16 ones up to p1
#pragma unroll
      for (int it = 0; it < LPT; ++it) {
        const int tk = it * TPI + lane / LPT;
        const float pt = __shfl_sync(0xffffffffu, pw, tk);
        const int tpos = bk * 32 + tk;
        if (tpos < qlim) {
          const uint4 hwv = ld_stream(vh + it * TPI * vrow);
          const float4 mtv = ldg128f(vm + it * TPI * vrow);
          const float mid = ((ballot >> tk) & 1u) ? 0.f : mid_unsel;
          const float a0 = (hmul * pt) * mtv.x, a1 = (hmul * pt) * mtv.z;
          g0 = fmaf(mid, a0, fmaf(pt, mtv.y, g0));
          g1 = fmaf(mid, a1, fmaf(pt, mtv.w, g1));
          value_codes(acc, hwv, a0, a1);
          if (dense_lo)
            value_codes(acc, ld_stream(vh + lo_off + it * TPI * vrow), 0.25f * a0, 0.25f * a1);
        } else if (tpos < p1) {
          value_raw(acc, raw_row(u, tpos, D, true) + hf * 128, pt);
        }
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
        low_planes<D, LPT>(acc, u, my, nlist, sc, p0, fsub, lane);
        nlist = 0;
      }
      if ((word >> lane) & 1u) my[nlist + __popc(word & ((1u << lane) - 1u))] = bk * 32 + lane;
      nlist += cnt;
      __syncwarp();
    }
    if (nlist > 0) low_planes<D, LPT>(acc, u, my, nlist, sc, p0, fsub, lane);
  }
  // undo the per-channel 2^o of the code conversion, add the per-group
  // constants, then reduce over the lanes that share a channel half
#pragma unroll
  for (int i = 0; i < 32; ++i) {
    const int j = (2 * i) & 15;
    acc[i].x = fmaf(acc[i].x, pow2(149 - kSub - code2_off(j)), i < 16 ? g0 : g1);
    acc[i].y = fmaf(acc[i].y, pow2(149 - kSub - code2_off(j + 1)), i < 16 ? g0 : g1);
  }
#pragma unroll
  for (int i = 0; i < 32; ++i) {
#pragma unroll
    for (int o = 16; o >= LPT; o >>= 1) {
      acc[i].x += __shfl_xor_sync(0xffffffffu, acc[i].x, o);
      acc[i].y += __shfl_xor_sync(0xffffffffu, acc[i].y, o);
    }
  }
  if (lane < LPT) {
#pragma unroll
    for (int i = 0; i < 32; ++i)
      reinterpret_cast<float2*>(red + warp * D + lane * 64)[i] = acc[i];
  }
  if (lane == 0) misc[24 + warp] = __int_as_float(nsel);
  __syncthreads();
  for (int d = tid; d < D; d += kThreads) {
    float o = 0.f;
#pragma unroll
    for (int w = 0; w < kWarps; ++w) o += red[w * D + d];
    o_s[d] = o;
  }
  if (tid == 0) {
    int t = 0;
    for (int w = 0; w < kWarps; ++w) t += __float_as_int(misc[24 + w]);
    misc[32] = __int_as_float(t);
  }
  __syncthreads();

  if (split > 1) {
    cg::cluster_group cluster = cg::this_cluster();
    cluster.sync();
    if (rank == 0) {
      for (int d = tid; d < D; d += kThreads) {
        float o = 0.f;
        for (int r = 0; r < split; ++r) o += cluster.map_shared_rank(o_s, r)[d];
        p.out[uidx * D + d] = o;
      }
      if (tid == 0) {
        int t = 0;
        for (int r = 0; r < split; ++r) t += __float_as_int(cluster.map_shared_rank(misc, r)[32]);
        if (p.nsel) p.nsel[uidx] = t;
        if (p.lse) p.lse[uidx] = (M + log2f(L)) * 0.69314718055994531f;
      }
    }
    cluster.sync();  // keep every CTA's shared memory alive until rank 0 has read it
  } else {
    for (int d = tid; d < D; d += kThreads) p.out[uidx * D + d] = o_s[d];
    if (tid == 0) {
      if (p.nsel) p.nsel[uidx] = __float_as_int(misc[32]);
      if (p.lse) p.lse[uidx] = (M + log2f(L)) * 0.69314718055994531f;
    }
  }
}

template <int D>
size_t decode_smem(int slots) {
  return sizeof(float) * (size_t)(D + 2 * kWarps * D + D + 64 + kWarps * kListCap + slots / 32 + slots);
}

template <int D, bool DENSE_LO>
int launch_decode_t(const DecodeParams& p, const CellList& cells, cudaStream_t stream) {
  const size_t smem = decode_smem<D>(p.slots);
  cudaError_t e = cudaFuncSetAttribute(decode_kernel<D, DENSE_LO>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)smem);
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
  e = cudaLaunchKernelEx(&cfg, decode_kernel<D, DENSE_LO>, p, cells);
  return (int)e;
}

}  // namespace

int decode_max_slots(int) { return kMaxSlots; }
int decode_max_split() { return kMaxSplit; }

int launch_decode(const DecodeParams& p, const CellList& cells, void* stream, int head_dim) {
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const bool dense = !(p.tau > 0.f);
  if (head_dim == 64) return dense ? launch_decode_t<64, true>(p, cells, s) : launch_decode_t<64, false>(p, cells, s);
  return dense ? launch_decode_t<128, true>(p, cells, s) : launch_decode_t<128, false>(p, cells, s);
}

}  // namespace loopkv
