// LoopVQ decode for sm_100a: attention over a KV cache coded by cross-loop
// codebooks.
//
// "LoopVQ: Sub 1-bit KV Cache Quantization for Looped Transformers",
// section 概要: a vector quantizer codes channels of several loop steps
// jointly at 0.5 bits per element.  Here one byte indexes a 256-entry
// codebook whose entries hold 4 channels of a token across the L loops of
// its layer (loop-major); decoding loop l reads slice [4l, 4l + 4) of each
// indexed entry (the format is spelled out in include/loopkv.h).
//
// One CTA (8 warps) per (layer, sequence, KV head, split); splits of a long
// sequence form a thread-block cluster and merge through DSMEM.
//   table   T[e][c] = <q_g, entry_e's loop slice> for channel group
//           g = c mod (D/4), over 32 columns c (each group once at D = 128,
//           twice at D = 64): the query is folded into the codebook once,
//           so a token's score is D/4 shared-memory lookups;
//   pass 1  lane = token.  At step k a lane reads group (lane ^ k) mod (D/4)
//           of its token from column lane ^ k: the 32 lanes of a warp then
//           touch 32 different columns, i.e. 32 different banks, whatever
//           the indices are (a table laid out by group would put a warp's 32
//           random entries of one group on random banks).  Each lane
//           permutes its token's D/4 index bytes by its lane number once, so
//           the byte step k needs sits at a fixed register position, and the
//           address is a byte permute and one logic op:
//           (e << 8) | (4 lane ^ 4 k); scores stay in shared memory (log2
//           units);
//   softmax the CTA's max and sum of exponentials, merged over the cluster;
//   pass 2  the same walk adds p_t into a histogram over the value codebook
//           laid out like the table: p_t as a fixed-point integer (units of
//           2^-31) with integer shared-memory atomics, which are native,
//           order-independent and exact; the bins of a (group, entry) are
//           summed over its columns afterwards; every bin holds at most the
//           sum of all weights (1), and each token's rounding (<= 2^-32)
//           lands in one bin, so an output moves by at most n 2^-32 times
//           the largest codebook magnitude;
//   output  out[4g + i] = 2^-31 sum_e W[g][e] * entry_e[4l + i].
// Shared memory is 256-byte rows: row e holds the 32 table (histogram)
// columns of entry e in its first half and 32 score slots in its second, so
// an entry's row offset is its index byte moved up one byte (no shift).  The
// codebooks' loop slices (256 x 16 bytes) are copied to shared memory once
// (the key slice before the table build, the value slice while the
// histogram fills), so neither the table build nor the output sum waits on
// L2 inside its loop.
// The index streams are read once (D/2 bytes per token at D = 128: 32 key
// and 32 value bytes); the work per token is D/2 shared-memory accesses,
// one bank-conflict-free wavefront per warp instruction.  A CTA holds 70 KB
// of shared memory and 80 registers, so three CTAs share an SM: the kernel
// waits on index loads, and the extra warps hide that latency.

#include <cooperative_groups.h>
#include <cuda_runtime.h>

#include <cmath>
#include <cstdint>

#include "loopkv_internal.cuh"

namespace cg = cooperative_groups;

namespace loopkv {
namespace {

constexpr int kVqThreads = 256;
constexpr int kVqWarps = kVqThreads / 32;
constexpr int kVqSub = 4;        // channels per sub-vector
constexpr int kEntries = 256;    // codebook entries (one byte)
constexpr int kCols = 32;         // table / histogram columns: column c is group c mod (D/4)
constexpr int kVqSlots = 8448;   // score slots per CTA (16K + a few hundred tokens in a cluster of two)
constexpr int kVqMaxSplit = 8;   // portable cluster size

struct VqParams {
  const uint8_t* idx_k;
  const uint8_t* idx_v;
  const float* cb_k;
  const float* cb_v;
  const uint16_t* q;
  float* out;
  float* lse;
  int32_t batch, H, L, cap, loop, split;
  float score_scale;  // sm_scale * log2(e)
  int32_t len[LOOPKV_MAX_BATCH];
};

// L2 requests for the index rows a warp reads kVqAhead iterations from now
// (the register loads cover only the next one): 64 tokens x D/4 bytes, one
// 128-byte line per lane.
constexpr int kVqAhead = 2;
__device__ __forceinline__ void prefetch_l2(const void* p) {
  asm volatile("prefetch.global.L2 [%0];" ::"l"(p));
}

// 16-byte asynchronous copy global -> shared (L1 bypassed).
__device__ __forceinline__ void cp_async16(void* dst, const void* src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;"
               ::"r"((uint32_t)__cvta_generic_to_shared(dst)), "l"(src)
               : "memory");
}
__device__ __forceinline__ void cp_async_wait_all() {
  asm volatile("cp.async.commit_group;\ncp.async.wait_group 0;" ::: "memory");
}

__device__ __forceinline__ uint4 ld_idx(const uint8_t* p) {
  uint4 r;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
               : "l"(p));
  return r;
}

// The D/4 indices of a token as D/16 words, permuted by r = lane mod (D/4):
// byte p of the result (byte p & 3 of word p >> 2) is index p ^ r of the
// token.  At D = 128 the word permutation's top bit is the choice of which
// 16-byte half to load first; its other two bits are conditional swaps of
// word pairs, and one byte permute per word applies r & 3.
template <int D>
__device__ __forceinline__ void load_xored(uint32_t (&w)[D / 16], const uint8_t* row, int lane) {
  constexpr int NW = D / 16;
  const int r = lane & (D / 4 - 1);
  const int a = r >> 2;
  if constexpr (D == 128) {
    const int first = (a >> 2) & 1;
    const uint4 x = ld_idx(row + 16 * first);
    const uint4 y = ld_idx(row + 16 * (first ^ 1));
    w[0] = x.x; w[1] = x.y; w[2] = x.z; w[3] = x.w;
    w[4] = y.x; w[5] = y.y; w[6] = y.z; w[7] = y.w;
  } else {
    const uint4 x = ld_idx(row);
    w[0] = x.x; w[1] = x.y; w[2] = x.z; w[3] = x.w;
  }
#pragma unroll
  for (int s = 1; s <= 2; s <<= 1) {
    const bool take = (a & s) != 0;
    uint32_t t[NW];
#pragma unroll
    for (int i = 0; i < NW; ++i) t[i] = take ? w[i ^ s] : w[i];
#pragma unroll
    for (int i = 0; i < NW; ++i) w[i] = t[i];
  }
  const int b = r & 3;
  const uint32_t sel = (uint32_t)(b | ((1 ^ b) << 4) | ((2 ^ b) << 8) | ((3 ^ b) << 12));
#pragma unroll
  for (int i = 0; i < NW; ++i) w[i] = __byte_perm(w[i], 0u, sel);
}

// Shared-memory rows are 256 bytes: row e holds the 32 table (or
// histogram) columns of entry e in its first 128 bytes and score slots
// 32 e .. 32 e + 31 in its second 128.  Byte offset of entry e's row
// (e << 8), e the index in byte k & 3 of a word: one byte permute.
constexpr int kRow = 256;
constexpr int kRowSlots = kEntries * 32;  // score slots held in the rows
__device__ __forceinline__ uint32_t entry_row(uint32_t word, int k) {
  return __byte_perm(word, 0u, 0x4404u | ((k & 3) << 4));
}
// Score slot s: in the second half of row s / 32, else in the overflow.
__device__ __forceinline__ float* slot(char* rows, float* over, int s) {
  return s < kRowSlots ? reinterpret_cast<float*>(rows + ((s >> 5) << 8) + 128 + ((s & 31) << 2))
                       : over + (s - kRowSlots);
}

template <int D>
__global__ void __launch_bounds__(kVqThreads, 3)
vq_decode_kernel(const VqParams p) {
  require_ieee_subnormals();
  constexpr int GR = D / kVqSub;  // channel groups
  extern __shared__ __align__(16) float sm[];
  char* rows = reinterpret_cast<char*>(sm);  // [kEntries][kRow]: table / histogram, score slots
  float* q_s = sm + kEntries * kRow / 4;     // [D]
  float* misc = q_s + D;                     // [64]
  float* over = misc + 64;                   // [kVqSlots - kRowSlots] score slots, then partials
  float* cbs = over + (kVqSlots - kRowSlots);  // [kEntries][4]: a codebook's loop slice

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int split = p.split;
  const int rank = blockIdx.x % split;
  const int unit = blockIdx.x / split;
  const int h = unit % p.H;
  const int b = (unit / p.H) % p.batch;
  const int layer = unit / (p.H * p.batch);
  const int n = p.len[b];
  const int chunk = ((n + split - 1) / split + 31) / 32 * 32;  // <= kVqSlots (host check)
  const int p0 = rank * chunk;
  const int p1 = min(n, p0 + chunk);
  const size_t uidx = ((size_t)layer * p.batch + b) * p.H + h;
  const int W = p.L * kVqSub;  // floats per codebook entry
  const size_t cbo = ((size_t)layer * p.H + h) * kEntries * W + (size_t)p.loop * kVqSub;
  const float* cbk = p.cb_k + cbo;
  const float* cbv = p.cb_v + cbo;

  static_assert(kVqThreads == kEntries, "one thread per codebook entry stages its slice");
  cp_async16(cbs + kVqSub * tid, cbk + (size_t)tid * W);
  for (int d = tid; d < D; d += kVqThreads) q_s[d] = __uint_as_float((uint32_t)p.q[uidx * D + d] << 16);
  cp_async_wait_all();
  __syncthreads();
  // T[e][c] = sum_i q[4g + i] * entry_e[4 loop + i], g = c mod GR (thread = column)
  for (int i = tid; i < kEntries * kCols; i += kVqThreads) {
    const int e = i / kCols, g = (i % kCols) % GR;
    const float4 c4 = *reinterpret_cast<const float4*>(cbs + kVqSub * e);
    const float* qq = q_s + kVqSub * g;
    float a = qq[0] * c4.x;
    a = fmaf(qq[1], c4.y, a);
    a = fmaf(qq[2], c4.z, a);
    a = fmaf(qq[3], c4.w, a);
    *reinterpret_cast<float*>(rows + e * kRow + 4 * (i % kCols)) = a;
  }
  __syncthreads();
  // step k reads column lane ^ k of row e, at byte (e << 8) | (4 lane ^ 4 k)
  const char* tb = rows;
  const uint32_t l4 = 4u * (uint32_t)lane;

  // ---------------------------------------------------------------- pass 1
  // two tokens per lane and iteration (t and t + 32): twice the independent
  // table lookups in flight per warp; the next iteration's indices are
  // loaded into registers while the current ones are used
  const uint8_t* ik = p.idx_k + uidx * (size_t)p.cap * GR;
  constexpr int STRIDE = 64 * kVqWarps;
  float lmax = -INFINITY;
  uint32_t n0[D / 16], n1[D / 16];
  if (p0 + 64 * warp + lane < p1) load_xored<D>(n0, ik + (size_t)(p0 + 64 * warp + lane) * GR, lane);
  if (p0 + 64 * warp + lane + 32 < p1)
    load_xored<D>(n1, ik + (size_t)(p0 + 64 * warp + lane + 32) * GR, lane);
  for (int base = p0 + 64 * warp; base < p1; base += STRIDE) {
    const int t0 = base + lane, t1 = t0 + 32;
    uint32_t w0[D / 16], w1[D / 16];
#pragma unroll
    for (int k = 0; k < D / 16; ++k) {
      w0[k] = n0[k];
      w1[k] = n1[k];
    }
    if (t0 + STRIDE < p1) load_xored<D>(n0, ik + (size_t)(t0 + STRIDE) * GR, lane);
    if (t1 + STRIDE < p1) load_xored<D>(n1, ik + (size_t)(t1 + STRIDE) * GR, lane);
    if (lane * 128 < 64 * GR && base + kVqAhead * STRIDE + lane * 128 / GR < p1)
      prefetch_l2(ik + (size_t)(base + kVqAhead * STRIDE) * GR + lane * 128);
    float a0 = 0.f, a1 = 0.f, b0 = 0.f, b1 = 0.f;
    if (t1 < p1) {
#pragma unroll
      for (int k = 0; k < GR; k += 2) {
        a0 += *reinterpret_cast<const float*>(tb + (entry_row(w0[k >> 2], k) | (l4 ^ (4u * k))));
        b0 += *reinterpret_cast<const float*>(tb + (entry_row(w1[k >> 2], k) | (l4 ^ (4u * k))));
        a1 += *reinterpret_cast<const float*>(tb + (entry_row(w0[k >> 2], k + 1) | (l4 ^ (4u * (k + 1)))));
        b1 += *reinterpret_cast<const float*>(tb + (entry_row(w1[k >> 2], k + 1) | (l4 ^ (4u * (k + 1)))));
      }
    } else if (t0 < p1) {
#pragma unroll
      for (int k = 0; k < GR; k += 2) {
        a0 += *reinterpret_cast<const float*>(tb + (entry_row(w0[k >> 2], k) | (l4 ^ (4u * k))));
        a1 += *reinterpret_cast<const float*>(tb + (entry_row(w0[k >> 2], k + 1) | (l4 ^ (4u * (k + 1)))));
      }
    }
    if (t0 < p1) {
      const float s = (a0 + a1) * p.score_scale;
      *slot(rows, over, t0 - p0) = s;
      lmax = fmaxf(lmax, s);
    }
    if (t1 < p1) {
      const float s = (b0 + b1) * p.score_scale;
      *slot(rows, over, t1 - p0) = s;
      lmax = fmaxf(lmax, s);
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) lmax = fmaxf(lmax, __shfl_xor_sync(0xffffffffu, lmax, o));
  if (lane == 0) misc[warp] = lmax;
  // the value index rows of the warp's first iterations go to L2 during the
  // softmax merge
  {
    const uint8_t* iv0 = p.idx_v + uidx * (size_t)p.cap * GR;
#pragma unroll
    for (int it = 0; it < kVqAhead; ++it) {
      const int base = p0 + 64 * warp + it * STRIDE;
      if (lane * 128 < 64 * GR && base + lane * 128 / GR < p1)
        prefetch_l2(iv0 + (size_t)base * GR + lane * 128);
    }
  }
  __syncthreads();
  float m = misc[0];
#pragma unroll
  for (int k = 1; k < kVqWarps; ++k) m = fmaxf(m, misc[k]);
  float ls = 0.f;
  for (int i = tid; i < p1 - p0; i += kVqThreads) ls += exp2f(*slot(rows, over, i) - m);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) ls += __shfl_xor_sync(0xffffffffu, ls, o);
  if (lane == 0) misc[8 + warp] = ls;
  __syncthreads();
  float l = 0.f;
#pragma unroll
  for (int k = 0; k < kVqWarps; ++k) l += misc[8 + k];
  if (p1 <= p0) {
    m = -INFINITY;
    l = 0.f;
  }
  float M = m, Lt = l;
  if (split > 1) {
    cg::cluster_group cluster = cg::this_cluster();
    if (tid == 0) {
      misc[32] = m;
      misc[33] = l;
    }
    cluster.sync();
    M = -INFINITY;
    for (int k = 0; k < split; ++k) M = fmaxf(M, cluster.map_shared_rank(misc, k)[32]);
    Lt = 0.f;
    for (int k = 0; k < split; ++k) {
      const float* rm = cluster.map_shared_rank(misc, k);
      if (rm[33] > 0.f) Lt += rm[33] * exp2f(rm[32] - M);
    }
  }
  const float inv = Lt > 0.f ? 1.f / Lt : 0.f;

  // ---------------------------------------------------------------- pass 2
  // the key table is free (every warp passed the barriers above): it becomes
  // the value histogram
  for (int i = tid; i < kEntries * kCols / 4; i += kVqThreads)
    *reinterpret_cast<uint4*>(rows + (i >> 3) * kRow + 16 * (i & 7)) = make_uint4(0u, 0u, 0u, 0u);
  // the value codebook's slice replaces the key one (read by the table build,
  // which every thread finished before the barriers above); it arrives
  // while the histogram fills
  cp_async16(cbs + kVqSub * tid, cbv + (size_t)tid * W);
  asm volatile("cp.async.commit_group;" ::: "memory");
  __syncthreads();
  char* hb = rows;
  const uint8_t* iv = p.idx_v + uidx * (size_t)p.cap * GR;
  if (p0 + 64 * warp + lane < p1) load_xored<D>(n0, iv + (size_t)(p0 + 64 * warp + lane) * GR, lane);
  if (p0 + 64 * warp + lane + 32 < p1)
    load_xored<D>(n1, iv + (size_t)(p0 + 64 * warp + lane + 32) * GR, lane);
  for (int base = p0 + 64 * warp; base < p1; base += STRIDE) {
    const int t0 = base + lane, t1 = t0 + 32;
    uint32_t w0[D / 16], w1[D / 16];
#pragma unroll
    for (int k = 0; k < D / 16; ++k) {
      w0[k] = n0[k];
      w1[k] = n1[k];
    }
    if (t0 + STRIDE < p1) load_xored<D>(n0, iv + (size_t)(t0 + STRIDE) * GR, lane);
    if (t1 + STRIDE < p1) load_xored<D>(n1, iv + (size_t)(t1 + STRIDE) * GR, lane);
    if (lane * 128 < 64 * GR && base + kVqAhead * STRIDE + lane * 128 / GR < p1)
      prefetch_l2(iv + (size_t)(base + kVqAhead * STRIDE) * GR + lane * 128);
    if (t0 < p1) {
      const uint32_t pw = __float2uint_rn(exp2f(*slot(rows, over, t0 - p0) - M) * inv * 2147483648.0f);
#pragma unroll
      for (int k = 0; k < GR; ++k)
        atomicAdd(reinterpret_cast<uint32_t*>(hb + (entry_row(w0[k >> 2], k) | (l4 ^ (4u * k)))), pw);
    }
    if (t1 < p1) {
      const uint32_t pw = __float2uint_rn(exp2f(*slot(rows, over, t1 - p0) - M) * inv * 2147483648.0f);
#pragma unroll
      for (int k = 0; k < GR; ++k)
        atomicAdd(reinterpret_cast<uint32_t*>(hb + (entry_row(w1[k >> 2], k) | (l4 ^ (4u * k)))), pw);
    }
  }
  asm volatile("cp.async.wait_group 0;" ::: "memory");
  __syncthreads();
  // out[4g + i] = sum_e W[g][e] * entry_e[4 loop + i] with W[g][e] the sum of
  // the bins of every column of group g (integers: exact); PARTS threads per
  // channel split the entries, their partial sums go to the overflow slots
  constexpr int PARTS = kVqThreads / D;
  constexpr int COPIES = kCols / GR;
  {
    const int d = tid % D, part = tid / D, g = d / kVqSub, i = d % kVqSub;
    float o = 0.f;
    for (int e = part; e < kEntries; e += PARTS) {
      uint32_t wsum = 0u;
#pragma unroll
      for (int c = 0; c < COPIES; ++c)
        wsum += *reinterpret_cast<const uint32_t*>(rows + e * kRow + 4 * (g + c * GR));
      o = fmaf((float)wsum, cbs[kVqSub * e + i], o);
    }
    over[tid] = o * 4.656612873077393e-10f;  // 2^-31
  }
  __syncthreads();
  if (tid < D) {
    float o = 0.f;
#pragma unroll
    for (int k = 0; k < PARTS; ++k) o += over[k * D + tid];
    q_s[tid] = o;  // the query is no longer needed
  }
  __syncthreads();

  if (split > 1) {
    cg::cluster_group cluster = cg::this_cluster();
    cluster.sync();
    if (rank == 0) {
      for (int d = tid; d < D; d += kVqThreads) {
        float o = 0.f;
        for (int k = 0; k < split; ++k) o += cluster.map_shared_rank(q_s, k)[d];
        p.out[uidx * D + d] = o;
      }
      if (tid == 0 && p.lse) p.lse[uidx] = (M + log2f(Lt)) * 0.69314718055994531f;
    }
    cluster.sync();  // every CTA's shared memory stays alive until rank 0 has read it
  } else {
    for (int d = tid; d < D; d += kVqThreads) p.out[uidx * D + d] = q_s[d];
    if (tid == 0 && p.lse) p.lse[uidx] = (M + log2f(Lt)) * 0.69314718055994531f;
  }
}

// Encoder: one CTA per new token of a (layer, sequence, KV head); thread e
// holds codebook entry e and computes its squared distance to the token's
// D/4 sub-vectors in the fixed fp32 order (no fused multiply-add); the
// smallest (distance, index) pair per group wins, so ties go to the lowest
// index.
struct VqEncodeParams {
  const uint16_t* x;   // [L][n_layers][batch][H][n_new][D]
  const float* cb;     // [n_layers][H][256][4 L]
  uint8_t* idx;        // [n_layers][batch][H][cap][D/4]
  int32_t n_layers, batch, H, L, cap, n_new;
  int32_t pos[LOOPKV_MAX_BATCH];
};

template <int D>
__global__ void __launch_bounds__(kEntries)
vq_encode_kernel(const VqEncodeParams p) {
  require_ieee_subnormals();
  constexpr int GR = D / kVqSub;
  __shared__ float x_s[GR][8 * kVqSub];                 // sub-vectors, loop-major
  __shared__ unsigned long long best[kEntries / 32][GR];
  const int e = threadIdx.x, lane = e & 31, warp = e >> 5;
  const int i = blockIdx.x % p.n_new;
  const int unit = blockIdx.x / p.n_new;
  const int h = unit % p.H;
  const int b = (unit / p.H) % p.batch;
  const int layer = unit / (p.H * p.batch);
  const int W = p.L * kVqSub;
  const size_t loop_stride = (size_t)p.n_layers * p.batch * p.H * p.n_new * D;
  const size_t tok = ((((size_t)layer * p.batch + b) * p.H + h) * p.n_new + i) * D;
  for (int k = e; k < p.L * D; k += kEntries) {
    const int l = k / D, d = k % D;
    x_s[d / kVqSub][l * kVqSub + d % kVqSub] =
        __uint_as_float((uint32_t)p.x[l * loop_stride + tok + d] << 16);
  }
  float c[8 * kVqSub];
  const float* ce = p.cb + (((size_t)layer * p.H + h) * kEntries + e) * W;
#pragma unroll
  for (int m = 0; m < 8 * kVqSub; ++m) c[m] = m < W ? __ldg(ce + m) : 0.f;
  __syncthreads();
  for (int j = 0; j < GR; ++j) {
    float dist = 0.f;
#pragma unroll
    for (int m = 0; m < 8 * kVqSub; ++m) {
      if (m < W) {
        const float diff = __fsub_rn(x_s[j][m], c[m]);
        dist = __fadd_rn(dist, __fmul_rn(diff, diff));
      }
    }
    // distances are >= 0, so their bit patterns order like the values
    unsigned long long key = ((unsigned long long)__float_as_uint(dist) << 32) | (unsigned)e;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      const unsigned long long other = __shfl_xor_sync(0xffffffffu, key, o);
      key = other < key ? other : key;
    }
    if (lane == 0) best[warp][j] = key;
  }
  __syncthreads();
  if (e < GR) {
    unsigned long long key = best[0][e];
#pragma unroll
    for (int w = 1; w < kEntries / 32; ++w) key = best[w][e] < key ? best[w][e] : key;
    const size_t row = (((size_t)layer * p.batch + b) * p.H + h) * p.cap + p.pos[b] + i;
    p.idx[row * GR + e] = (uint8_t)(key & 0xFFu);
  }
}

template <int D>
constexpr size_t vq_smem() {
  static_assert(kVqSlots - kRowSlots >= kVqThreads, "the overflow slots hold the partial sums");
  return (size_t)kEntries * kRow +
         sizeof(float) * ((size_t)D + 64 + (kVqSlots - kRowSlots) + kEntries * kVqSub);
}

template <int D>
int launch_vq_t(const VqParams& p, long long units, cudaStream_t stream) {
  const size_t smem = vq_smem<D>();
  cudaError_t e = cudaFuncSetAttribute(vq_decode_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)smem);
  if (e != cudaSuccess) return (int)e;
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = dim3((unsigned)(units * p.split), 1, 1);
  cfg.blockDim = dim3(kVqThreads, 1, 1);
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
  return (int)cudaLaunchKernelEx(&cfg, vq_decode_kernel<D>, p);
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

bool vq_desc_ok(const loopkv_vq_desc* d) {
  return d != nullptr && d->n_loops >= 1 && d->n_loops <= 8 && d->n_layers >= 1 &&
         d->n_kv_heads >= 1 && d->n_kv_heads <= (1 << 16) &&
         (d->head_dim == 64 || d->head_dim == 128) && d->batch >= 1 &&
         d->batch <= LOOPKV_MAX_BATCH && d->capacity >= 1 && d->capacity <= (1 << 20) &&
         std::isfinite(d->sm_scale);
}

}  // namespace
}  // namespace loopkv

using namespace loopkv;

extern "C" loopkv_status loopkv_vq_decode(const loopkv_vq_desc* d, int32_t loop, const int32_t* h_len,
                                          const uint8_t* d_idx_k, const uint8_t* d_idx_v,
                                          const float* d_cb_k, const float* d_cb_v,
                                          const uint16_t* d_q, float* d_out, float* d_lse,
                                          void* stream) {
  if (h_len == nullptr || !vq_desc_ok(d)) return LOOPKV_ERR_INVALID_ARG;
  if (loop < 0 || loop >= d->n_loops) return LOOPKV_ERR_INVALID_ARG;
  const void* ptrs[6] = {d_idx_k, d_idx_v, d_cb_k, d_cb_v, d_q, d_out};
  for (const void* ptr : ptrs)
    if (ptr == nullptr || !aligned16(ptr)) return LOOPKV_ERR_INVALID_ARG;
  if (d_lse != nullptr && (reinterpret_cast<uintptr_t>(d_lse) & 3u) != 0) return LOOPKV_ERR_INVALID_ARG;
  VqParams p{};
  int nmax = 0;
  for (int b = 0; b < d->batch; ++b) {
    if (h_len[b] < 1 || h_len[b] > d->capacity) return LOOPKV_ERR_INVALID_ARG;
    p.len[b] = h_len[b];
    nmax = h_len[b] > nmax ? h_len[b] : nmax;
  }
  const long long units = (long long)d->n_layers * d->batch * d->n_kv_heads;
  auto slots_for = [&](int s) { return ((nmax + s - 1) / s + 31) / 32 * 32; };
  int split = 1;
  while (slots_for(split) > kVqSlots && split < kVqMaxSplit) split *= 2;
  if (slots_for(split) > kVqSlots) return LOOPKV_ERR_UNSUPPORTED;
  while (units * split < 148 * 4 && split < kVqMaxSplit && nmax / (2 * split) >= 512) split *= 2;
  if (units * split >= (1LL << 31)) return LOOPKV_ERR_UNSUPPORTED;
  p.idx_k = d_idx_k;
  p.idx_v = d_idx_v;
  p.cb_k = d_cb_k;
  p.cb_v = d_cb_v;
  p.q = d_q;
  p.out = d_out;
  p.lse = d_lse;
  p.batch = d->batch;
  p.H = d->n_kv_heads;
  p.L = d->n_loops;
  p.cap = d->capacity;
  p.loop = loop;
  p.split = split;
  const float sm_scale = d->sm_scale > 0.f ? d->sm_scale : 1.0f / std::sqrt((float)d->head_dim);
  p.score_scale = sm_scale * 1.4426950408889634f;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const int e = d->head_dim == 64 ? launch_vq_t<64>(p, units, s) : launch_vq_t<128>(p, units, s);
  return e == 0 ? LOOPKV_OK : LOOPKV_ERR_CUDA;
}

extern "C" loopkv_status loopkv_vq_encode(const loopkv_vq_desc* d, const int32_t* h_pos,
                                          int32_t n_new, const uint16_t* d_x, const float* d_cb,
                                          uint8_t* d_idx, void* stream) {
  if (h_pos == nullptr || !vq_desc_ok(d) || n_new < 0) return LOOPKV_ERR_INVALID_ARG;
  if (n_new == 0) return LOOPKV_OK;
  const void* ptrs[3] = {d_x, d_cb, d_idx};
  for (const void* ptr : ptrs)
    if (ptr == nullptr || !aligned16(ptr)) return LOOPKV_ERR_INVALID_ARG;
  VqEncodeParams p{};
  for (int b = 0; b < d->batch; ++b) {
    if (h_pos[b] < 0 || (long long)h_pos[b] + n_new > d->capacity) return LOOPKV_ERR_INVALID_ARG;
    p.pos[b] = h_pos[b];
  }
  const long long blocks = (long long)d->n_layers * d->batch * d->n_kv_heads * n_new;
  if (blocks >= (1LL << 31)) return LOOPKV_ERR_UNSUPPORTED;
  p.x = d_x;
  p.cb = d_cb;
  p.idx = d_idx;
  p.n_layers = d->n_layers;
  p.batch = d->batch;
  p.H = d->n_kv_heads;
  p.L = d->n_loops;
  p.cap = d->capacity;
  p.n_new = n_new;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (d->head_dim == 64)
    vq_encode_kernel<64><<<(unsigned)blocks, kEntries, 0, s>>>(p);
  else
    vq_encode_kernel<128><<<(unsigned)blocks, kEntries, 0, s>>>(p);
  return cudaGetLastError() == cudaSuccess ? LOOPKV_OK : LOOPKV_ERR_CUDA;
}
