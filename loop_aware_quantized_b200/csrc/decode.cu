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

// Small integer (0..15) as float: exponent trick, exact.
__device__ __forceinline__ float code_f(uint32_t c) {
  return __uint_as_float(0x4B000000u | c) - 8388608.0f;
}

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
// planes (K_hi[g][chunk][token][4 words], same for K_lo).
template <int D, bool Q4>
__device__ __forceinline__ float dot_codes(const uint8_t* khi, const uint8_t* klo,
                                           const float* qs) {
  float acc = 0.f;
#pragma unroll
  for (int c = 0; c < D / 64; ++c) {
    const uint4 h = ld_stream(khi + c * 512);
    uint4 l = make_uint4(0, 0, 0, 0);
    if (Q4) l = ld_stream(klo + c * 512);
    const uint32_t hw[4] = {h.x, h.y, h.z, h.w};
    const uint32_t lw[4] = {l.x, l.y, l.z, l.w};
#pragma unroll
    for (int w = 0; w < 4; ++w) {
#pragma unroll
      for (int j4 = 0; j4 < 4; ++j4) {
        const float4 s = *reinterpret_cast<const float4*>(qs + 64 * c + 16 * w + 4 * j4);
        const float sv[4] = {s.x, s.y, s.z, s.w};
#pragma unroll
        for (int jj = 0; jj < 4; ++jj) {
          const int j = 4 * j4 + jj;
          uint32_t code = (hw[w] >> (2 * j)) & 3u;
          if (Q4) code = (code << 2) | ((lw[w] >> (2 * j)) & 3u);
          acc = fmaf(sv[jj], code_f(code), acc);
        }
      }
    }
  }
  return acc;
}

template <int D>
__global__ void __launch_bounds__(kThreads)
decode_kernel(const DecodeParams p, const CellList cl) {
  constexpr int LPT = D / 64;       // lanes per token in pass 2
  constexpr int TPI = 32 / LPT;     // tokens per warp iteration in pass 2
  extern __shared__ __align__(16) float smem[];
  float* q_s = smem;                                  // [D]
  float* qs_all = q_s + D;                            // [kWarps][D]
  float* red = qs_all + kWarps * D;                   // [kWarps][D]
  float* o_s = red + kWarps * D;                      // [D]
  float* misc = o_s + D;                              // [64]
  float* sc = misc + 64;                              // [slots]

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

  // ------------------------------------------------------------- pass 1
  float lmax = -INFINITY;
  const int blk0 = p0 / 32;
  const int blk1 = (p1 + 31) / 32;
  for (int bk = blk0 + warp; bk < blk1; bk += kWarps) {
    const int pos = bk * 32 + lane;
    const bool active = pos < p1;
    float s = -INFINITY;
    if (quant && bk * 32 < u.nq) {
      // fold q with the group's key scale / zero point
      const uint8_t* meta = u.data + u.Ld.k_meta + (size_t)bk * 8 * D;
      float cpart = 0.f;
#pragma unroll
      for (int i = 0; i < D / 32; ++i) {
        const int d = lane + 32 * i;
        const float sc_d = __ldg(reinterpret_cast<const float*>(meta) + d);
        const float z_d = __ldg(reinterpret_cast<const float*>(meta) + D + d);
        qs[d] = q_s[d] * sc_d;
        cpart = fmaf(q_s[d], z_d, cpart);
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) cpart += __shfl_xor_sync(0xffffffffu, cpart, o);
      __syncwarp();
      if (active && pos < u.nq) {
        const uint8_t* khi = u.data + u.Ld.k_hi + (size_t)bk * 8 * D + lane * 16;
        const uint8_t* klo = u.data + u.Ld.k_lo + (size_t)bk * 8 * D + lane * 16;
        const float dot = q4 ? dot_codes<D, true>(khi, klo, qs) : dot_codes<D, false>(khi, klo, qs);
        s = (dot + cpart) * sscale;
      }
      __syncwarp();
    }
    if (active && pos >= u.nq) s = dot_bf16<D>(raw_row(u, pos, D, false), q_s) * sscale;
    if (active) {
      sc[pos - p0] = s;
      lmax = fmaxf(lmax, s);
    }
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
    for (int r = 0; r < split; ++r) {
      const float* rm = cluster.map_shared_rank(misc, r);
      M = fmaxf(M, rm[16]);
    }
    L = 0.f;
    for (int r = 0; r < split; ++r) {
      const float* rm = cluster.map_shared_rank(misc, r);
      if (rm[17] > 0.f) L += rm[17] * exp2f(rm[16] - M);
    }
  }
  const float f = (l_r > 0.f) ? exp2f(m_r - M) / L : 0.f;  // e -> p
  const float tau = p.tau;

  // ------------------------------------------------------------- pass 2
  float acc[64];
#pragma unroll
  for (int i = 0; i < 64; ++i) acc[i] = 0.f;
  float g0 = 0.f, g1 = 0.f;  // per-group constants of the lane's two 32-channel groups
  int nsel = 0;
  const int hf = lane % LPT;
  const size_t vrow = D / 4;  // bytes per token of a value plane / value meta
  for (int bk = blk0 + warp; bk < blk1; bk += kWarps) {
    const int pos = bk * 32 + lane;
    const bool active = pos < p1;
    const float pw = active ? sc[pos - p0] * f : 0.f;
    const bool sel = q4 && active && pos < u.nq && pw >= tau;
    const uint32_t ballot = __ballot_sync(0xffffffffu, sel);
    nsel += __popc(ballot);
    if (p.mask != nullptr && lane == 0 && bk * 32 < u.nq && q4)
      p.mask[uidx * p.mask_words + bk] = ballot;
#pragma unroll 1
    for (int it = 0; it < LPT; ++it) {
      const int tk = it * TPI + lane / LPT;
      const int tpos = bk * 32 + tk;
      const float pt = __shfl_sync(0xffffffffu, pw, tk);
      if (tpos >= p1) continue;
      if (quant && tpos < u.nq) {
        const uint8_t* vh = u.data + u.Ld.v_hi + (size_t)tpos * vrow + hf * 16;
        const uint8_t* vm = u.data + u.Ld.v_meta + (size_t)tpos * vrow + hf * 16;
        const uint4 hw4 = ld_stream(vh);
        const float4 mt = ldg128f(vm);  // (scale, zero) of the lane's two groups
        const float ps0 = pt * mt.x, ps1 = pt * mt.z;
        const bool tsel = (ballot >> tk) & 1u;
        uint4 lw4 = make_uint4(0, 0, 0, 0);
        if (q4) {
          if (tsel) {
            lw4 = ld_stream(u.data + u.Ld.v_lo + (size_t)tpos * vrow + hf * 16);
            g0 = fmaf(pt, mt.y, g0);
            g1 = fmaf(pt, mt.w, g1);
          } else {
            g0 += fmaf(1.5f, ps0, pt * mt.y);
            g1 += fmaf(1.5f, ps1, pt * mt.w);
          }
        } else {
          g0 = fmaf(pt, mt.y, g0);
          g1 = fmaf(pt, mt.w, g1);
        }
        const uint32_t hw[4] = {hw4.x, hw4.y, hw4.z, hw4.w};
        const uint32_t lw[4] = {lw4.x, lw4.y, lw4.z, lw4.w};
#pragma unroll
        for (int w = 0; w < 4; ++w) {
          const float ps = (w < 2) ? ps0 : ps1;
#pragma unroll
          for (int j = 0; j < 16; ++j) {
            uint32_t code = (hw[w] >> (2 * j)) & 3u;
            if (q4) code = (code << 2) | ((lw[w] >> (2 * j)) & 3u);
            acc[16 * w + j] = fmaf(ps, code_f(code), acc[16 * w + j]);
          }
        }
      } else {
        const uint8_t* row = raw_row(u, tpos, D, true) + hf * 128;
#pragma unroll
        for (int c = 0; c < 8; ++c) {
          const uint4 w = ldg128(row + c * 16);
          acc[8 * c + 0] = fmaf(pt, bf16_lo(w.x), acc[8 * c + 0]);
          acc[8 * c + 1] = fmaf(pt, bf16_hi(w.x), acc[8 * c + 1]);
          acc[8 * c + 2] = fmaf(pt, bf16_lo(w.y), acc[8 * c + 2]);
          acc[8 * c + 3] = fmaf(pt, bf16_hi(w.y), acc[8 * c + 3]);
          acc[8 * c + 4] = fmaf(pt, bf16_lo(w.z), acc[8 * c + 4]);
          acc[8 * c + 5] = fmaf(pt, bf16_hi(w.z), acc[8 * c + 5]);
          acc[8 * c + 6] = fmaf(pt, bf16_lo(w.w), acc[8 * c + 6]);
          acc[8 * c + 7] = fmaf(pt, bf16_hi(w.w), acc[8 * c + 7]);
        }
      }
    }
  }
  // per-group constants, then reduce over the lanes that share a channel half
#pragma unroll
  for (int i = 0; i < 32; ++i) acc[i] += g0;
#pragma unroll
  for (int i = 32; i < 64; ++i) acc[i] += g1;
#pragma unroll
  for (int i = 0; i < 64; ++i) {
#pragma unroll
    for (int o = 16; o >= LPT; o >>= 1) acc[i] += __shfl_xor_sync(0xffffffffu, acc[i], o);
  }
  if (lane < LPT) {
#pragma unroll
    for (int i = 0; i < 64; ++i) red[warp * D + lane * 64 + i] = acc[i];
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
  return sizeof(float) * (size_t)(D + 2 * kWarps * D + D + 64 + slots);
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
