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
//           key scales into integer weights under one power of two, and
//           integer tensor-core products (mma.sync, u8 codes x s8 weight
//           digits) give sum_d qs_d * code_d exactly; the zero points add
//           c = sum_d q_d * zero_d.  Scores are kept in log2 units.
//   softmax the CTA's max and sum of exponentials, merged across the cluster
//           into the unit's logsumexp.
//   pass 2  values: p and the selection p >= tau per block (a warp ballot
//           gives the mask word); the high planes of the quantized blocks
//           go through integer tensor-core products against the weights
//           hmul * p * scale (channel-major planes, contraction over
//           tokens), the per-group constants p * (zero [+ 1.5 * scale])
//           are summed in fp32; the low planes of the selected tokens and
//           the bf16 positions are accumulated in fp32, lane = 64 channels
//           of a token, so a low-plane row is read only when selected.
//   combine warp shuffles reduce the per-token partial outputs, shared
//           memory reduces across warps, DSMEM across the cluster.
// The kernel streams the cache once: HBM bandwidth and memory latency bound
// it, with the per-code arithmetic on the tensor cores.

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
// bits at bit offset `off` (off + bits <= 23) of a word w becomes the float
// 2^23 + code * 2^off: the word's field is placed in the mantissa of a float
// whose exponent word `expo` (the bits of 2^23) arrives in a register, so the
// mask is the logic op's only immediate.  Subtracting 2^23 (exact) leaves
// code * 2^off; the power of two is folded into the weights (keys) or
// removed from the accumulators at the end (values).
template <int off, int bits>
__device__ __forceinline__ float field_f(uint32_t w, uint32_t expo) {
  static_assert(off + bits <= 23, "field must stay inside the mantissa");
  return __uint_as_float((w & (((1u << bits) - 1u) << off)) | expo);
}

// 16 two-bit codes of w (code j in bits 2j..2j+1) -> 8 pairs
// (code 2i * 2^o(2i), code 2i+1 * 2^o(2i+1)), o(j) = 2j for j < 6, 2(j-6) else.
__device__ __forceinline__ void codes2_to_pairs(uint32_t w, uint32_t expo, float2 neg,
                                                float2 (&out)[8]) {
  const uint32_t y = w >> 12;
  out[0] = add2(make_float2(field_f<0, 2>(w, expo), field_f<2, 2>(w, expo)), neg);
  out[1] = add2(make_float2(field_f<4, 2>(w, expo), field_f<6, 2>(w, expo)), neg);
  out[2] = add2(make_float2(field_f<8, 2>(w, expo), field_f<10, 2>(w, expo)), neg);
  out[3] = add2(make_float2(field_f<0, 2>(y, expo), field_f<2, 2>(y, expo)), neg);
  out[4] = add2(make_float2(field_f<4, 2>(y, expo), field_f<6, 2>(y, expo)), neg);
  out[5] = add2(make_float2(field_f<8, 2>(y, expo), field_f<10, 2>(y, expo)), neg);
  out[6] = add2(make_float2(field_f<12, 2>(y, expo), field_f<14, 2>(y, expo)), neg);
  out[7] = add2(make_float2(field_f<16, 2>(y, expo), field_f<18, 2>(y, expo)), neg);
}
// Bit offset a two-bit code j of a word ends up at in codes2_to_pairs.
__host__ __device__ constexpr int code2_off(int j) { return j < 6 ? 2 * j : 2 * (j - 6); }

// 2^-k as a float, k in [0, 126].
__device__ __forceinline__ float pow2_neg(int k) { return __int_as_float((127 - k) << 23); }

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

// ---------------------------------------------------------------- keys
//
// Key scores with integer tensor-core products (mma.sync m16n8k32, u8 x s8,
// s32 accumulate).  For a 32-token group the folded weights qs_d = q_d *
// scale_d share one power of two 2^E chosen from the group's largest |qs|,
// W_d = rint(qs_d * 2^E) with |W_d| < 2^26, so sum_d W_d * code_d is exact
// in integers and the score is that sum * 2^-E + sum_d q_d * zero_d.
//
// A operand (16 tokens x 32 bytes): the hi / lo planes of a 16-channel word
// merge into two nibble words (even channels, odd channels); a byte of a
// nibble word holds two codes, c_lo + 16 c_hi.  Two products cover both
// codes without unpacking them: A_X = the nibble word against X = W(c_lo's
// channel), A_Y = (nibble word & 0xF0F0F0F0) = 16 c_hi against
// Y = W(c_hi's channel) - 16 W(c_lo's channel); then
//   A_X . X + (A_Y . Y) / 16 = sum c_lo W_lo + sum c_hi W_hi.
// B operand (32 bytes x 8 columns): X and Y as four signed base-256 digits
// each, X's digits in columns 0-3 and Y's in columns 4-7; the X product
// sees Y's columns as zero and the Y product X's, so both accumulate into
// one fragment.  Digits: b_p = byte p of (W + 0x80808080) read as u8, minus
// 128 (exact for |W| < 0x7F7F7F7F).
//
// Lane (g, t) = (lane / 4, lane % 4) holds tokens g + 8j (j = 0..3) of the
// group: M tile j / 2, row g or g + 8.  K tile kt takes from lane t the
// plane word w = (D / 64) t + kt of each of its tokens (16 channels), so a
// K tile is 64 channels and a lane's words are contiguous in a row.

__device__ __forceinline__ void mma_u8s8(int (&c)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                         uint32_t a3, uint32_t b0, uint32_t b1) {
  asm("mma.sync.aligned.m16n8k32.row.col.s32.u8.s8.s32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+r"(c[0]), "+r"(c[1]), "+r"(c[2]), "+r"(c[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
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

// Streams run ahead of use: the next group of a warp is loaded into
// registers while the current one is processed, and the lines of the group
// kAheadK / kAheadV groups ahead (0: none; 1 is the group being loaded) are
// requested into L2, one 128-byte line per lane; kPreV value groups of each
// warp are requested before the softmax.  Distances 1 measured fastest.
constexpr int kAheadK = 1;
constexpr int kAheadV = 1;
constexpr int kPreV = 2;

__device__ __forceinline__ void prefetch_l2(const void* p) {
  asm volatile("prefetch.global.L2 [%0];" ::"l"(p));
}

// One lane's share of a 32-token key group.
template <int D>
struct KTile {
  uint32_t h[4][D / 64], l[4][D / 64];  // token g + 8j: the lane's plane words
  float4 sc, zr;                        // scale / zero of channels 4 lane .. 4 lane + 3
};

// kb -> the lane's K_hi words of token g; lo_off = K_lo - K_hi; km -> the
// lane's four scales (zeros D floats further); meta: the lane folds channels.
template <int D, bool Q4>
__device__ __forceinline__ void load_ktile(KTile<D>& k, const uint8_t* kb, size_t lo_off,
                                           const float* km, bool meta) {
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    if constexpr (D == 128) {
      const uint2 hw = ld_stream2(kb + j * 128);
      k.h[j][0] = hw.x; k.h[j][1] = hw.y;
      if (Q4) {
        const uint2 lw = ld_stream2(kb + lo_off + j * 128);
        k.l[j][0] = lw.x; k.l[j][1] = lw.y;
      } else {
        k.l[j][0] = 0u; k.l[j][1] = 0u;
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

// Nibble words of a 16-channel plane word: byte b of `ev` holds the codes of
// channels 4b (low nibble) and 4b + 2 (high), byte b of `od` channels 4b + 1
// and 4b + 3.  q = 4 hi + lo for 4-bit keys, q = hi for 2-bit keys.
template <bool Q4>
__device__ __forceinline__ void nibble_words(uint32_t hi, uint32_t lo, uint32_t& ev, uint32_t& od) {
  if (Q4) {
    ev = ((hi << 2) & 0xCCCCCCCCu) | (lo & 0x33333333u);
    od = (hi & 0xCCCCCCCCu) | ((lo >> 2) & 0x33333333u);
  } else {
    ev = hi & 0x33333333u;
    od = (hi >> 2) & 0x33333333u;
  }
}

// Scores one group; stores the scores of positions below qlim into sc and
// returns their max.  stage: the warp's 64 * (D / 64) ints of staging.
template <int D, bool Q4>
__device__ __forceinline__ float key_group(const KTile<D>& k, float4 qv, int* stage, int gpos0,
                                           int qlim, int p0, float* sc, float sscale, int lane) {
  constexpr int KT = D / 64;
  const int g = lane >> 2, t = lane & 3;
  // fold q into the scales; the zero-point term
  const float q0 = qv.x * k.sc.x, q1 = qv.y * k.sc.y, q2 = qv.z * k.sc.z, q3 = qv.w * k.sc.w;
  float cpart = fmaf(qv.w, k.zr.w, fmaf(qv.z, k.zr.z, fmaf(qv.y, k.zr.y, qv.x * k.zr.x)));
  // the group's power of two: max|qs| * F < 2^26
  const float amax = fmaxf(fmaxf(fabsf(q0), fabsf(q1)), fmaxf(fabsf(q2), fabsf(q3)));
  const uint32_t mbits = __reduce_max_sync(0xffffffffu, __float_as_uint(amax));
  const int fexp = min(279 - (int)(mbits >> 23), 253);
  const float F = __int_as_float(fexp << 23);
  const float Finv = __int_as_float((254 - fexp) << 23);
  const int w0 = __float2int_rn(q0 * F), w1 = __float2int_rn(q1 * F);
  const int w2 = __float2int_rn(q2 * F), w3 = __float2int_rn(q3 * F);
  if (lane < D / 4) {
    // channels 4 lane + {0,1,2,3}: byte (lane % 4) of plane word lane / 4
    const int w = lane >> 2, b = lane & 3;
    const int base = (w % KT) * 16 + (w / KT) * 4 + b;
    constexpr uint32_t kBias = 0x80808080u;
    stage[base] = (int)((uint32_t)w0 + kBias);                       // X, even word
    stage[base + 16 * KT] = (int)((uint32_t)(w2 - 16 * w0) + kBias);  // Y, even word
    stage[base + 32 * KT] = (int)((uint32_t)w1 + kBias);             // X, odd word
    stage[base + 48 * KT] = (int)((uint32_t)(w3 - 16 * w1) + kBias);  // Y, odd word
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) cpart += __shfl_xor_sync(0xffffffffu, cpart, o);
  __syncwarp();
  // B fragments: column g, bytes k = 4t..4t+3 (b0) and 16+4t.. (b1)
  const uint32_t pl = (uint32_t)(g & 3);
  const uint32_t selp = pl | ((pl + 4u) << 4) | (pl << 8) | ((pl + 4u) << 12);
  const uint32_t mx = g < 4 ? 0xFFFFFFFFu : 0u;
  uint32_t bx[KT][2], by[KT][2];
#pragma unroll
  for (int kt = 0; kt < KT; ++kt) {
#pragma unroll
    for (int part = 0; part < 2; ++part) {
      const int4 iv = *reinterpret_cast<const int4*>(
          stage + ((part * 2 + (g >> 2)) * KT + kt) * 16 + t * 4);
      const uint32_t lo2 = __byte_perm((uint32_t)iv.x, (uint32_t)iv.y, selp);
      const uint32_t hi2 = __byte_perm((uint32_t)iv.z, (uint32_t)iv.w, selp);
      const uint32_t dg = __byte_perm(lo2, hi2, 0x5410u) ^ 0x80808080u;
      bx[kt][part] = dg & mx;
      by[kt][part] = dg & ~mx;
    }
  }
  // products: fragment j / 2 holds tokens g + 8 (j & ~1) and g + 8 (j | 1)
  int acc[2][4];
#pragma unroll
  for (int mt = 0; mt < 2; ++mt) {
#pragma unroll
    for (int i = 0; i < 4; ++i) acc[mt][i] = 0;
#pragma unroll
    for (int kt = 0; kt < KT; ++kt) {
      uint32_t e0, o0, e1, o1;
      nibble_words<Q4>(k.h[2 * mt][kt], k.l[2 * mt][kt], e0, o0);
      nibble_words<Q4>(k.h[2 * mt + 1][kt], k.l[2 * mt + 1][kt], e1, o1);
      mma_u8s8(acc[mt], e0, e1, o0, o1, bx[kt][0], bx[kt][1]);
      mma_u8s8(acc[mt], e0 & 0xF0F0F0F0u, e1 & 0xF0F0F0F0u, o0 & 0xF0F0F0F0u, o1 & 0xF0F0F0F0u,
               by[kt][0], by[kt][1]);
    }
  }
  // lane t holds digit columns 2t, 2t+1: X digits 0-1, 2-3 (t = 0, 1), Y
  // digits 0-1, 2-3 (t = 2, 3); weight them and sum over the quad
  const float fac = (t == 0) ? 1.f : (t == 1) ? 65536.f : (t == 2) ? 0.0625f : 4096.f;
  float r[4];
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const int* c = acc[j >> 1] + 2 * (j & 1);
    r[j] = (float)(c[0] + (c[1] << 8)) * fac;
  }
  // reduce-scatter over the quad: lane t ends with row rho(t) = {0, 2, 1, 3}[t]
  const bool odd = t & 1;
  float k0 = odd ? r[2] : r[0], k1 = odd ? r[3] : r[1];
  const float s0 = odd ? r[0] : r[2], s1 = odd ? r[1] : r[3];
  k0 += __shfl_xor_sync(0xffffffffu, s0, 1);
  k1 += __shfl_xor_sync(0xffffffffu, s1, 1);
  const bool up = t & 2;
  float tot = up ? k1 : k0;
  tot += __shfl_xor_sync(0xffffffffu, up ? k0 : k1, 2);
  const int rho = (odd ? 2 : 0) + (up ? 1 : 0);
  const int pos = gpos0 + g + 8 * rho;
  float lmax = -INFINITY;
  if (pos < qlim) {
    const float s = fmaf(tot, Finv * sscale, cpart * sscale);
    sc[pos - p0] = s;
    lmax = s;
  }
  return lmax;
}

// Pass 1 over the CTA's quantized key groups [b_begin, b_end), warp-strided.
// Two register buffers alternate, so the next group's loads are in flight
// while the current one is scored.  Staging alternates between two halves
// of the warp's area so one __syncwarp per group suffices.
template <int D, bool Q4>
__device__ __forceinline__ float key_pass(const Unit& u, int b_begin, int b_end, int p0, int p1,
                                          const float* q_s, int* stage, float* sc, float sscale,
                                          int warp, int lane) {
  float lmax = -INFINITY;
  const int first = b_begin + warp;
  if (first >= b_end) return lmax;
  const bool meta = lane < D / 4;
  const float4 qv = meta ? *reinterpret_cast<const float4*>(q_s + 4 * lane)
                         : make_float4(0.f, 0.f, 0.f, 0.f);
  const int qlim = min(p1, u.nq);
  const int g = lane >> 2, t = lane & 3;
  constexpr size_t G = 8 * D;                  // bytes of one group in each block
  constexpr size_t STEP = (size_t)kWarps * G;  // a warp's stride between its groups
  constexpr int SH = 64 * (D / 64);            // ints of one staging half
  const size_t lane_off = (D == 128) ? (size_t)(t >> 1) * 512 + g * 16 + (t & 1) * 8
                                     : (size_t)g * 16 + t * 4;
  const uint8_t* kb = u.data + u.Ld.k_hi + (size_t)first * G + lane_off;
  const size_t lo_off = u.Ld.k_lo - u.Ld.k_hi;
  const float* km = reinterpret_cast<const float*>(u.data + u.Ld.k_meta + (size_t)first * G) +
                    (meta ? 4 * lane : 0);
  // L2 prefetch: lane -> line (lane % (D / 16)) of block K_hi, K_lo or K_meta
  constexpr int LINES = D / 16;
  const int pblk = lane / LINES;
  const bool pon = pblk < (Q4 ? 3 : 2);
  const uint8_t* pf = u.data + (pblk == 0 ? u.Ld.k_hi : (Q4 && pblk == 1) ? u.Ld.k_lo : u.Ld.k_meta) +
                      (size_t)(lane % LINES) * 128;
  KTile<D> a, b;
  load_ktile<D, Q4>(a, kb, lo_off, km, meta);
  int bk = first;
  for (;;) {
    const bool hasb = bk + kWarps < b_end;
    if (hasb) load_ktile<D, Q4>(b, kb + STEP, lo_off, km + STEP / 4, meta);
    if (kAheadK > 0 && pon && bk + kAheadK * kWarps < b_end)
      prefetch_l2(pf + (size_t)(bk + kAheadK * kWarps) * G);
    lmax = fmaxf(lmax, key_group<D, Q4>(a, qv, stage, bk * 32, qlim, p0, sc, sscale, lane));
    if (!hasb) break;
    bk += kWarps;
    kb += STEP;
    km += STEP / 4;
    const bool hasa = bk + kWarps < b_end;
    if (hasa) load_ktile<D, Q4>(a, kb + STEP, lo_off, km + STEP / 4, meta);
    if (kAheadK > 0 && pon && bk + kAheadK * kWarps < b_end)
      prefetch_l2(pf + (size_t)(bk + kAheadK * kWarps) * G);
    lmax = fmaxf(lmax, key_group<D, Q4>(b, qv, stage + SH, bk * 32, qlim, p0, sc, sscale, lane));
    if (!hasa) break;
    bk += kWarps;
    kb += STEP;
    km += STEP / 4;
  }
  return lmax;
}

// Value accumulation of one quantized token half-row (64 channels): acc +=
// (a_j) * code * 2^o for the lane's two 32-channel groups (a0 for words 0-1,
// a1 for words 2-3); the 2^o of each channel is removed once at the end.
__device__ __forceinline__ void value_codes(float2 (&acc)[32], const uint4 hw4, float a0, float a1,
                                            uint32_t expo, float2 neg) {
  const uint32_t hw[4] = {hw4.x, hw4.y, hw4.z, hw4.w};
#pragma unroll
  for (int w = 0; w < 4; ++w) {
    float2 v[8];
    codes2_to_pairs(hw[w], expo, neg, v);
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
      const float2 wt = make_float2(pt * (float)(1u << code2_off(j)),
                                    pt * (float)(1u << code2_off(j + 1)));
      acc[pair] = fma2(wt, make_float2(bf16_lo(ws[k]), bf16_hi(ws[k])), acc[pair]);
    }
  }
}

// Low planes of queued selected positions: acc += p * scale * lo, TPI
// positions per warp iteration (LPT lanes per position, 64 channels each).
template <int D, int LPT>
__device__ __forceinline__ void low_planes(float2 (&acc)[32], const Unit& u, const int* list,
                                           int n, const float* sc, int p0, float f,
                                           uint32_t expo, float2 neg, int lane) {
  constexpr int TPI = 32 / LPT;
  const int hf = lane % LPT;
  for (int k0 = 0; k0 < n; k0 += TPI) {
    const int kk = k0 + lane / LPT;
    if (kk < n) {
      const int tpos = list[kk];
      const float pt = sc[tpos - p0] * f;
      const uint4 lw = ld_stream(u.data + u.Ld.v_lo + (size_t)tpos * (D / 4) + hf * 16);
      const float4 m4 = ldg128f(u.data + u.Ld.v_meta + (size_t)tpos * (D / 4) + hf * 16);
      value_codes(acc, lw, pt * m4.x, pt * m4.z, expo, neg);
    }
  }
  __syncwarp();
}

// ---------------------------------------------------------------- values
//
// High planes of the quantized value blocks on the tensor cores
// (mma.sync m16n8k16, u8 x s8, s32 accumulate):
//   out_c += sum_T a_{T,G} * hi_{T,c},  a_{T,G} = hmul * p_T * scale_{T,G},
// G = c / 32 the channel's value group.  M = 16 channels, K = 16 bytes = the
// 32 tokens of a group (two codes per byte), N = 8 digit columns.  Lane
// (g, t) supplies channels 8i + g (i = 0..D/8-1) of tokens 16 (t >> 1) ..
// 16 (t >> 1) + 15, whose words are contiguous in the group's channel-major
// block.  Even t takes the codes at bits 0-1 / 4-5 of each byte (tokens 4b
// and 4b + 2 of the half), odd t those at bits 2-3 / 6-7 (tokens 4b + 1 and
// 4b + 3, at four times their value); the weights of even-t bytes carry the
// factor 4 instead, so every product comes out 4x and no code is shifted.
// Byte k = 4t + b pairs tokens T_lo = 16 (t >> 1) + 4b + (t & 1) and
// T_hi = T_lo + 2, with X = w(T_lo), Y = w(T_hi) - 16 w(T_lo) as for the keys.
//
// The integer weights share one power of two per channel group for the whole
// pass, so the products accumulate in int32 across groups.  It is chosen from
// hmul * f * max(scale) of the first group (p <= f for every token) with two
// bits of headroom, and chosen again, after folding the accumulators into
// fp32, only when a later group's weights outgrow it.

__device__ __forceinline__ void mma16_u8s8(int (&c)[4], uint32_t a0, uint32_t a1, uint32_t b0) {
  asm("mma.sync.aligned.m16n8k16.row.col.s32.u8.s8.s32 {%0,%1,%2,%3}, {%4,%5}, {%6}, "
      "{%0,%1,%2,%3};"
      : "+r"(c[0]), "+r"(c[1]), "+r"(c[2]), "+r"(c[3])
      : "r"(a0), "r"(a1), "r"(b0));
}

// One lane's share of a 32-token value group.
template <int D>
struct VTile {
  uint4 w[D / 32];  // high-plane words i = 0..D/8-1 (channel 8i + g)
  float4 m[D / 64];  // meta row of token `lane`: (scale, zero) x D/32
};

template <int D>
__device__ __forceinline__ void load_vtile(VTile<D>& v, const uint8_t* vh, const float* vm) {
#pragma unroll
  for (int i = 0; i < D / 32; ++i) v.w[i] = ld_stream(vh + 16 * i);
#pragma unroll
  for (int i = 0; i < D / 64; ++i) v.m[i] = __ldg(reinterpret_cast<const float4*>(vm) + i);
}

__device__ __forceinline__ uint32_t word_of(const uint4& q, int j) {
  return j == 0 ? q.x : j == 1 ? q.y : j == 2 ? q.z : q.w;
}

// The lane's 128-byte line of group 0 for L2 prefetches of the value high
// plane (lanes 0 .. D/16 - 1) and value meta (the next D/16 lanes), else null;
// group i's line is 8 D i bytes further.
template <int D>
__device__ __forceinline__ const uint8_t* vgroup_line(const Unit& u, int lane) {
  constexpr int LINES = D / 16;
  if (lane >= 2 * LINES) return nullptr;
  return u.data + (lane < LINES ? u.Ld.v_hi : u.Ld.v_meta) + (size_t)(lane % LINES) * 128;
}

// Pass over the warp's quantized blocks [b_begin, b_end) (warp-strided).
// vo[G]: lane (g, t)'s total for channel 32 G + 8 t + g (scaled by 2^o = 1);
// cst[G]: the lane's share (token = lane) of sum_T p_T (zero + mid scale).
template <int D>
__device__ __forceinline__ void value_high_pass(const Unit& u, int b_begin, int b_end, int p0,
                                                int qlim, int blk0, const float* sc,
                                                const uint32_t* mask_s, float f, float hmul,
                                                float mid_unsel, int* stage, float (&vo)[D / 32],
                                                float (&cst)[D / 32], int warp, int lane) {
  constexpr int NG = D / 32;
  const int first = b_begin + warp;
  if (first >= b_end) return;
  const int g = lane >> 2, t = lane & 3;
  // consumer side: operand masks, B column digit, digit weights of columns 2t, 2t+1
  const uint32_t m1 = (t & 1) ? 0xCCCCCCCCu : 0x33333333u;
  const uint32_t m2 = (t & 1) ? 0xC0C0C0C0u : 0x30303030u;
  const uint32_t pl = (uint32_t)(g & 3);
  const uint32_t selp = pl | ((pl + 4u) << 4) | (pl << 8) | ((pl + 4u) << 12);
  const uint32_t mx = g < 4 ? 0xFFFFFFFFu : 0u;
  const float fac = ((t == 0) ? 1.f : (t == 1) ? 65536.f : (t == 2) ? 0.0625f : 4096.f) * 0.25f;
  // producer side: lane = token T; T_lo lanes (T % 4 < 2) stage the X / Y pair
  const float mtok = (lane & 1) ? 1.f : 4.f;
  const float hm = hmul * mtok;
  const float mid_m = mid_unsel / mtok;
  const bool tlo = (lane & 2) == 0;
  const int kslot = (2 * (lane >> 4) + (lane & 1)) * 4 + ((lane >> 2) & 3);
  constexpr uint32_t kBias = 0x80808080u;

  int acc[NG][2][4];
#pragma unroll
  for (int G = 0; G < NG; ++G)
#pragma unroll
    for (int i = 0; i < 8; ++i) acc[G][i >> 2][i & 3] = 0;
  float F[NG];
#pragma unroll
  for (int G = 0; G < NG; ++G) F[G] = 0.f;
  bool fresh = true;

  auto flush = [&]() {
#pragma unroll
    for (int G = 0; G < NG; ++G) {
      const float sG = fac * __int_as_float((254 - (int)(__float_as_uint(F[G]) >> 23)) << 23);
#pragma unroll
      for (int mt = 0; mt < 2; ++mt) {
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          float x = fmaf((float)acc[G][mt][2 * h + 1], 256.f, (float)acc[G][mt][2 * h]) * sG;
          x += __shfl_xor_sync(0xffffffffu, x, 1);
          x += __shfl_xor_sync(0xffffffffu, x, 2);
          if (2 * mt + h == t) vo[G] += x;
          acc[G][mt][2 * h] = 0;
          acc[G][mt][2 * h + 1] = 0;
        }
      }
    }
  };

  auto body = [&](const VTile<D>& v, int bk, int* st) {
    const int pos = bk * 32 + lane;
    const bool valid = pos < qlim;
    const float pw = valid ? sc[pos - p0] * f : 0.f;
    const bool sel = (mask_s[bk - blk0] >> lane) & 1u;
    const float hp = hm * pw;
    const float mid = sel ? 0.f : mid_m;
    float a[NG];
    int w[NG];
    int wmax = 0;
#pragma unroll
    for (int G = 0; G < NG; ++G) {
      const float4 mm = v.m[G >> 1];
      const float s = (G & 1) ? mm.z : mm.x, z = (G & 1) ? mm.w : mm.y;
      a[G] = hp * s;
      cst[G] = fmaf(mid, a[G], fmaf(pw, z, cst[G]));
      w[G] = __float2int_rn(a[G] * F[G]);
      wmax = max(wmax, w[G]);
    }
    if (__any_sync(0xffffffffu, fresh || wmax >= (1 << 26))) {
      if (!fresh) flush();
#pragma unroll
      for (int G = 0; G < NG; ++G) {
        const float4 mm = v.m[G >> 1];
        const float s = valid ? ((G & 1) ? mm.z : mm.x) : 0.f;
        const uint32_t smax = __reduce_max_sync(0xffffffffu, __float_as_uint(s));
        const float x = hmul * f * __uint_as_float(smax);
        const int fexp = min(275 - (int)(__float_as_uint(x) >> 23), 253);
        F[G] = __int_as_float(fexp << 23);
        w[G] = __float2int_rn(a[G] * F[G]);
      }
      fresh = false;
    }
#pragma unroll
    for (int G = 0; G < NG; ++G) {
      const int wp = __shfl_down_sync(0xffffffffu, w[G], 2);
      if (tlo) {
        st[G * 32 + kslot] = (int)((uint32_t)w[G] + kBias);
        st[G * 32 + 16 + kslot] = (int)((uint32_t)(wp - 16 * w[G]) + kBias);
      }
    }
    __syncwarp();
#pragma unroll
    for (int G = 0; G < NG; ++G) {
      const int4 iv = *reinterpret_cast<const int4*>(st + G * 32 + (g >> 2) * 16 + 4 * t);
      const uint32_t lo2 = __byte_perm((uint32_t)iv.x, (uint32_t)iv.y, selp);
      const uint32_t hi2 = __byte_perm((uint32_t)iv.z, (uint32_t)iv.w, selp);
      const uint32_t dg = __byte_perm(lo2, hi2, 0x5410u) ^ 0x80808080u;
      const uint32_t bx = dg & mx, by = dg & ~mx;
#pragma unroll
      for (int mt = 0; mt < 2; ++mt) {
        const int i0 = 4 * G + 2 * mt;
        const uint32_t w0 = word_of(v.w[i0 >> 2], i0 & 3);
        const uint32_t w1 = word_of(v.w[i0 >> 2], (i0 & 3) + 1);
        mma16_u8s8(acc[G][mt], w0 & m1, w1 & m1, bx);
        mma16_u8s8(acc[G][mt], w0 & m2, w1 & m2, by);
      }
    }
  };

  constexpr size_t GB = 8 * D;                        // bytes of a group's high-plane block
  constexpr size_t VSTEP = (size_t)kWarps * GB;       // a warp's stride between its groups
  constexpr size_t MSTEP = (size_t)kWarps * 32 * (D / 16);  // same, in meta floats
  const uint8_t* vh = u.data + u.Ld.v_hi + (size_t)first * GB + (size_t)(g * 2 + (t >> 1)) * (D / 2);
  const float* vm = reinterpret_cast<const float*>(u.data + u.Ld.v_meta) +
                    ((size_t)first * 32 + lane) * (D / 16);
  const uint8_t* pf = vgroup_line<D>(u, lane);
  VTile<D> va, vb;
  load_vtile<D>(va, vh, vm);
  int bk = first;
  for (;;) {
    const bool hasb = bk + kWarps < b_end;
    if (hasb) load_vtile<D>(vb, vh + VSTEP, vm + MSTEP);
    if (kAheadV > 0 && pf != nullptr && bk + kAheadV * kWarps < b_end)
      prefetch_l2(pf + (size_t)(bk + kAheadV * kWarps) * GB);
    body(va, bk, stage);
    if (!hasb) break;
    bk += kWarps;
    vh += VSTEP;
    vm += MSTEP;
    const bool hasa = bk + kWarps < b_end;
    if (hasa) load_vtile<D>(va, vh + VSTEP, vm + MSTEP);
    if (kAheadV > 0 && pf != nullptr && bk + kAheadV * kWarps < b_end)
      prefetch_l2(pf + (size_t)(bk + kAheadV * kWarps) * GB);
    body(vb, bk, stage + NG * 32);
    if (!hasa) break;
    bk += kWarps;
    vh += VSTEP;
    vm += MSTEP;
  }
  flush();
}

// tau <= 0 selects every 4-bit token: the low-plane list pass then covers
// them all.
template <int D>
__global__ void __launch_bounds__(kThreads, 2)
decode_kernel(const DecodeParams p, const CellList cl) {
  extern __shared__ __align__(16) float smem[];
  float* q_s = smem;                                  // [D]
  float* kstage = q_s + D;                            // [kWarps][D] key-weight staging, pass 1
  float* red = kstage + kWarps * D;                   // [kWarps][D] (pass 1 staging continues here)
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
  int* stage = reinterpret_cast<int*>(kstage) + warp * 2 * D;  // 2 D ints per warp
  const float sscale = p.score_scale;
  const int blk0 = p0 / 32;
  const int blk1 = (p1 + 31) / 32;
  const int nqb = quant ? (u.nq + 31) / 32 : 0;     // blocks holding quantized positions
  const int qend = min(blk1, nqb);

  // ------------------------------------------------------------- pass 1
  float lmax = -INFINITY;
  const uint32_t expo = p.code_expo;
  const float2 neg = make_float2(p.code_neg, p.code_neg);
  if (q4) lmax = key_pass<D, true>(u, blk0, qend, p0, p1, q_s, stage, sc, sscale, warp, lane);
  else if (quant) lmax = key_pass<D, false>(u, blk0, qend, p0, p1, q_s, stage, sc, sscale, warp, lane);
  // the warp's first value groups go to L2 ahead of the softmax merge
  if (quant) {
    const uint8_t* pf = vgroup_line<D>(u, lane);
    if (pf != nullptr)
      for (int j = 0; j < kPreV; ++j)
        if (blk0 + warp + j * kWarps < qend) prefetch_l2(pf + (size_t)(blk0 + warp + j * kWarps) * 8 * D);
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
  const int qlim = min(p1, u.nq);
  // selection: p >= tau on the quantized 4-bit positions, a ballot per block
  int nsel = 0;
  for (int bk = blk0 + warp; bk < blk1; bk += kWarps) {
    const int pos = bk * 32 + lane;
    const float pw = pos < p1 ? sc[pos - p0] * f : 0.f;
    const bool sel = q4 && pos < qlim && pw >= tau;
    const uint32_t ballot = __ballot_sync(0xffffffffu, sel);
    nsel += __popc(ballot);
    if (lane == 0) {
      mask_s[bk - blk0] = ballot;
      if (p.mask != nullptr && q4 && bk < nqb) p.mask[uidx * p.mask_words + bk] = ballot;
    }
  }
  __syncwarp();  // the warp reads back only the mask words its own lane 0 wrote

  // high planes on the tensor cores.  A 4-bit high plane has weight
  // 4 * p * scale; its missing low bits read as 1.5, i.e. + 1.5 * p * scale =
  // 0.375 * (4 * p * scale) per unselected token, folded into the constants.
  float vo[D / 32], cst[D / 32];
#pragma unroll
  for (int i = 0; i < D / 32; ++i) { vo[i] = 0.f; cst[i] = 0.f; }
  if (quant)
    value_high_pass<D>(u, blk0, qend, p0, qlim, blk0, sc, mask_s, f, q4 ? 4.f : 1.f,
                       q4 ? 0.375f : 0.f, stage, vo, cst, warp, lane);

  // fp32 part, lane = 64 channels of a token: bf16 positions (residual, raw
  // cells, the SHARE current token) and the low planes of selected tokens
  constexpr int LPT = D / 64;       // lanes per token (64 channels per lane)
  constexpr int TPI = 32 / LPT;     // tokens per warp iteration
  const int hf = lane % LPT;
  float2 acc[32];
#pragma unroll
  for (int i = 0; i < 32; ++i) acc[i] = make_float2(0.f, 0.f);
  const int raw0 = max(p0, u.nq);
  if (raw0 < p1) {
    for (int bk = max(blk0, raw0 / 32) + warp; bk < blk1; bk += kWarps) {
      const int pos = bk * 32 + lane;
      const float pw = pos < p1 ? sc[pos - p0] * f : 0.f;
#pragma unroll
      for (int it = 0; it < LPT; ++it) {
        const int tk = it * TPI + lane / LPT;
        const float pt = __shfl_sync(0xffffffffu, pw, tk);
        const int tpos = bk * 32 + tk;
        if (tpos >= raw0 && tpos < p1) value_raw(acc, raw_row(u, tpos, D, true) + hf * 128, pt);
      }
    }
  }
  // low planes of the selected tokens: acc += p * scale * lo.  The warp
  // gathers its selected positions into a list and processes them TPI at a
  // time, so the cost follows the number of selected tokens.
  if (q4) {
    int* my = lst + warp * kListCap;
    int nlist = 0;
    for (int bk = blk0 + warp; bk < qend; bk += kWarps) {
      const uint32_t word = mask_s[bk - blk0];
      if (word == 0u) continue;
      const int cnt = __popc(word);
      if (nlist + cnt > kListCap) {
        low_planes<D, LPT>(acc, u, my, nlist, sc, p0, f, expo, neg, lane);
        nlist = 0;
      }
      if ((word >> lane) & 1u) my[nlist + __popc(word & ((1u << lane) - 1u))] = bk * 32 + lane;
      nlist += cnt;
      __syncwarp();
    }
    if (nlist > 0) low_planes<D, LPT>(acc, u, my, nlist, sc, p0, f, expo, neg, lane);
  }
  // undo the per-channel 2^o of the fp32 part's code conversion, then reduce
  // over the lanes that share a channel half
#pragma unroll
  for (int i = 0; i < 32; ++i) {
    const int j = (2 * i) & 15;
    acc[i].x *= pow2_neg(code2_off(j));
    acc[i].y *= pow2_neg(code2_off(j + 1));
  }
#pragma unroll
  for (int i = 0; i < 32; ++i) {
#pragma unroll
    for (int o = 16; o >= LPT; o >>= 1) {
      acc[i].x += __shfl_xor_sync(0xffffffffu, acc[i].x, o);
      acc[i].y += __shfl_xor_sync(0xffffffffu, acc[i].y, o);
    }
  }
#pragma unroll
  for (int i = 0; i < D / 32; ++i)
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) cst[i] += __shfl_xor_sync(0xffffffffu, cst[i], o);
  __syncthreads();  // every warp is done with its staging, which spans red
  if (lane < LPT) {
#pragma unroll
    for (int i = 0; i < 32; ++i)
      reinterpret_cast<float2*>(red + warp * D + lane * 64)[i] = acc[i];
  }
  __syncwarp();
  // the tensor-core part and the per-group constants: lane (g, t) owns
  // channel 32 G + 8 t + g of each value group G
#pragma unroll
  for (int i = 0; i < D / 32; ++i) red[warp * D + 32 * i + 8 * (lane & 3) + (lane >> 2)] += vo[i] + cst[i];
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

template <int D>
int launch_decode_t(const DecodeParams& p, const CellList& cells, cudaStream_t stream) {
  const size_t smem = decode_smem<D>(p.slots);
  cudaError_t e = cudaFuncSetAttribute(decode_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
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
  e = cudaLaunchKernelEx(&cfg, decode_kernel<D>, p, cells);
  return (int)e;
}

}  // namespace

int decode_max_slots(int) { return kMaxSlots; }
int decode_max_split() { return kMaxSplit; }

int launch_decode(const DecodeParams& p, const CellList& cells, void* stream, int head_dim) {
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (head_dim == 64) return launch_decode_t<64>(p, cells, s);
  return launch_decode_t<128>(p, cells, s);
}

}  // namespace loopkv
