// GPU twin of synth/philox.py and synth/workloads.py: the seeded synthetic
// keys, values and queries, generated on the device so that inputs of
// hundreds of GB never cross PCIe.  Same counters, same fp32 round-to-nearest
// steps, same bf16 rounding as the host generator, hence the same bits.
//
// Philox4x32-10: Salmon, Moraes, Dror and Shaw, "Parallel Random Numbers: As
// Easy as 1, 2, 3" (SC'11).  This file holds no LoopKV arithmetic.

#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cstdint>

namespace {

constexpr uint32_t kStreamK = 1, kStreamV = 2, kStreamQNoise = 3, kStreamQPos = 4;

struct U4 {
  uint32_t x, y, z, w;
};

__device__ __forceinline__ U4 philox(uint32_t c0, uint32_t c1, uint32_t c2, uint32_t c3,
                                     uint32_t k0, uint32_t k1) {
#pragma unroll
  for (int r = 0; r < 10; ++r) {
    if (r) {
      k0 += 0x9E3779B9u;
      k1 += 0xBB67AE85u;
    }
    const uint32_t lo0 = 0xD2511F53u * c0, hi0 = __umulhi(0xD2511F53u, c0);
    const uint32_t lo1 = 0xCD9E8D57u * c2, hi1 = __umulhi(0xCD9E8D57u, c2);
    const uint32_t n0 = hi1 ^ c1 ^ k0, n1 = lo1, n2 = hi0 ^ c3 ^ k1, n3 = lo0;
    c0 = n0; c1 = n1; c2 = n2; c3 = n3;
  }
  return U4{c0, c1, c2, c3};
}

// Sum of the eight 16-bit halves, centred, times the unit-variance scale.
__device__ __forceinline__ float normal_from(U4 u, float nscale) {
  const int s = (int)((u.x & 0xFFFFu) + (u.x >> 16) + (u.y & 0xFFFFu) + (u.y >> 16) +
                      (u.z & 0xFFFFu) + (u.z >> 16) + (u.w & 0xFFFFu) + (u.w >> 16));
  return __fmul_rn((float)(s - 262140), nscale);
}

__device__ __forceinline__ uint16_t to_bf16_bits(float x) {
  return __bfloat16_as_ushort(__float2bfloat16_rn(x));
}

__device__ __forceinline__ float from_bf16_bits(uint16_t b) {
  return __uint_as_float((uint32_t)b << 16);
}

__device__ __forceinline__ uint16_t key_bits(int cell, int b, int h, uint32_t t, int d, int H, int D,
                                             const float* chscale, uint32_t seed, float nscale) {
  const U4 u = philox(t, (uint32_t)d, (uint32_t)(h + H * b), (uint32_t)cell, seed, kStreamK);
  const float z = normal_from(u, nscale);
  return to_bf16_bits(__fmul_rn(z, chscale[((size_t)cell * H + h) * D + d]));
}

__device__ __forceinline__ uint16_t value_bits(int cell, int b, int h, uint32_t t, int d, int H,
                                               uint32_t seed, float nscale) {
  const U4 u = philox(t, (uint32_t)d, (uint32_t)(h + H * b), (uint32_t)cell, seed, kStreamV);
  return to_bf16_bits(normal_from(u, nscale));
}

// Keys / values of a cell that follows a reference cell (refs[cell] >= 0):
// the reference's raw token plus 0.25 * N(0,1) of the cell's own stream
// (keys: times the cell's channel scale).
__device__ __forceinline__ uint16_t key_of(int cell, const int32_t* refs, int b, int h, uint32_t t,
                                           int d, int H, int D, const float* chscale,
                                           uint32_t seed, float nscale) {
  const int ref = refs[cell];
  if (ref < 0) return key_bits(cell, b, h, t, d, H, D, chscale, seed, nscale);
  const float kr = from_bf16_bits(key_bits(ref, b, h, t, d, H, D, chscale, seed, nscale));
  const U4 u = philox(t, (uint32_t)d, (uint32_t)(h + H * b), (uint32_t)cell, seed, kStreamK);
  const float z = __fmul_rn(__fmul_rn(normal_from(u, nscale), 0.25f),
                            chscale[((size_t)cell * H + h) * D + d]);
  return to_bf16_bits(__fadd_rn(kr, z));
}
__device__ __forceinline__ uint16_t value_of(int cell, const int32_t* refs, int b, int h,
                                             uint32_t t, int d, int H, uint32_t seed, float nscale) {
  const int ref = refs[cell];
  if (ref < 0) return value_bits(cell, b, h, t, d, H, seed, nscale);
  const float vr = from_bf16_bits(value_bits(ref, b, h, t, d, H, seed, nscale));
  const U4 u = philox(t, (uint32_t)d, (uint32_t)(h + H * b), (uint32_t)cell, seed, kStreamV);
  return to_bf16_bits(__fadd_rn(vr, __fmul_rn(normal_from(u, nscale), 0.25f)));
}

// out[c][b][h][i][d] for positions t0[b] + i, i < T.
__global__ void gen_kv_kernel(uint16_t* __restrict__ k, uint16_t* __restrict__ v,
                              const int32_t* __restrict__ cells, const int32_t* __restrict__ seqs,
                              const int32_t* __restrict__ t0, int n_cells, int batch, int H, int D,
                              int T, int table_cells, const float* __restrict__ chscale,
                              const int32_t* __restrict__ refs, uint32_t seed, float nscale) {
  const size_t total = (size_t)n_cells * batch * H * T * D;
  for (size_t i = blockIdx.x * (size_t)blockDim.x + threadIdx.x; i < total;
       i += (size_t)gridDim.x * blockDim.x) {
    const int d = (int)(i % D);
    size_t r = i / D;
    const int ti = (int)(r % T);
    r /= T;
    const int h = (int)(r % H);
    r /= H;
    const int bl = (int)(r % batch);
    const int c = (int)(r / batch);
    const int cell = cells[c], b = seqs[bl];
    if (cell < 0 || cell >= table_cells) continue;  // host passes valid ids; never index past the table
    const uint32_t t = (uint32_t)(t0[bl] + ti);
    if (k) k[i] = key_of(cell, refs, b, h, t, d, H, D, chscale, seed, nscale);
    if (v) v[i] = value_of(cell, refs, b, h, t, d, H, seed, nscale);
  }
}

// One warp per (c, b, h) query; lanes over channels.
// mode 0: sum of raw keys at 3 distinct attended positions + 0.5 * N(0,1)
// mode 1: 2 * raw key at one attended position + N(0,1)
// One warp per query: [n_cells][batch][H][g][D], query head rep < g of KV
// head h (rep 0 is the one-query stream; rep r offsets the stream words by
// r << 16, as the host generator does).
__global__ void gen_q_kernel(uint16_t* __restrict__ q, const int32_t* __restrict__ cells,
                             const int32_t* __restrict__ srcs, const int32_t* __restrict__ seqs,
                             const int32_t* __restrict__ lens, int n_cells, int batch, int H, int g,
                             int D, int mode, int table_cells, const float* __restrict__ chscale,
                             const int32_t* __restrict__ refs, uint32_t seed, float nscale) {
  const long long warp = ((long long)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (warp >= (long long)n_cells * batch * H * g) return;
  const int rep = (int)(warp % g);
  const int h = (int)((warp / g) % H);
  const int bl = (int)((warp / ((long long)g * H)) % batch);
  const int c = (int)(warp / ((long long)g * H * batch));
  const int cell = cells[c], src = srcs[c], b = seqs[bl];
  const int n = lens[c * batch + bl];
  if (cell < 0 || cell >= table_cells || src < 0 || src >= table_cells) return;
  const bool share = src != cell;
  const uint32_t rw = (uint32_t)rep << 16;
  const U4 u = philox((uint32_t)n, rw, (uint32_t)(h + H * b), (uint32_t)cell, seed, kStreamQPos);
  const uint32_t uu[3] = {u.x, u.y, u.z};
  const int want = mode == 0 ? 3 : 1;
  const int kcount = n < want ? n : want;
  int picks[3] = {0, 0, 0};
  for (int i = 0; i < kcount; ++i) {
    int r = (int)(((uint64_t)uu[i] * (uint64_t)(n - i)) >> 32);
    // skip the positions already taken, in ascending order
    int a0 = picks[0], a1 = picks[1];
    if (i == 2 && a1 < a0) { const int tmp = a0; a0 = a1; a1 = tmp; }
    if (i >= 1 && r >= a0) ++r;
    if (i >= 2 && r >= a1) ++r;
    picks[i] = r;
  }
  for (int d = lane; d < D; d += 32) {
    float key[3] = {0.f, 0.f, 0.f};
    for (int i = 0; i < kcount; ++i) {
      const int p = picks[i];
      const int kc = (share && p < n - 1) ? src : cell;
      key[i] = from_bf16_bits(key_of(kc, refs, b, h, (uint32_t)p, d, H, D, chscale, seed, nscale));
    }
    const U4 un = philox((uint32_t)n, (uint32_t)d + rw, (uint32_t)(h + H * b), (uint32_t)cell, seed,
                         kStreamQNoise);
    const float z = normal_from(un, nscale);
    float x;
    if (mode == 0) {
      float acc = 0.f;
      for (int i = 0; i < kcount; ++i) acc = __fadd_rn(acc, key[i]);
      x = __fadd_rn(acc, __fmul_rn(0.5f, z));
    } else {
      x = __fadd_rn(__fmul_rn(2.0f, key[0]), z);
    }
    q[(size_t)warp * D + d] = to_bf16_bits(x);
  }
}

// LoopVQ inputs (twins of workloads.vq_indices / vq_query).
constexpr uint32_t kStreamVqIdx = 9, kStreamVqQ = 11;

// out [n_layers][batch][H][cap][D/4] indices of tokens < T (later token
// slots untouched) of sequences seq0 .. seq0 + batch - 1; which 0 keys, 1
// values.
__global__ void gen_vq_idx_kernel(uint8_t* __restrict__ out, int n_layers, int batch, int H, int D,
                                  int cap, int T, int which, int seq0, uint32_t seed) {
  const int groups = D / 4;
  const size_t total = (size_t)n_layers * batch * H * T * groups;
  for (size_t i = blockIdx.x * (size_t)blockDim.x + threadIdx.x; i < total;
       i += (size_t)gridDim.x * blockDim.x) {
    const int j = (int)(i % groups);
    size_t r = i / groups;
    const int t = (int)(r % T);
    r /= T;
    const int h = (int)(r % H);
    r /= H;
    const int b = (int)(r % batch);
    const int layer = (int)(r / batch);
    const U4 u = philox((uint32_t)t, (uint32_t)j, (uint32_t)(h + H * (b + seq0)),
                        (uint32_t)layer | ((uint32_t)which << 16), seed, kStreamVqIdx);
    out[((((size_t)layer * batch + b) * H + h) * cap + t) * groups + j] = (uint8_t)(u.x & 255u);
  }
}

// q [n_layers][batch][H][D] of one loop, sequences seq0 ...
__global__ void gen_vq_q_kernel(uint16_t* __restrict__ q, int n_layers, int batch, int H, int D,
                                int loop, int seq0, uint32_t seed, float nscale) {
  const size_t total = (size_t)n_layers * batch * H * D;
  for (size_t i = blockIdx.x * (size_t)blockDim.x + threadIdx.x; i < total;
       i += (size_t)gridDim.x * blockDim.x) {
    const int d = (int)(i % D);
    size_t r = i / D;
    const int h = (int)(r % H);
    r /= H;
    const int b = (int)(r % batch);
    const int layer = (int)(r / batch);
    const U4 u = philox((uint32_t)d, (uint32_t)loop, (uint32_t)(h + H * (b + seq0)),
                        (uint32_t)layer, seed, kStreamVqQ);
    q[i] = to_bf16_bits(__fmul_rn(2.0f, normal_from(u, nscale)));
  }
}

// Philox4x32-10 of n (counter, key) rows: in [n][6] = c0..c3, k0, k1; out [n][4].
__global__ void philox_rows_kernel(const uint32_t* __restrict__ in, uint32_t* __restrict__ out,
                                   int n) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= n) return;
  const uint32_t* r = in + (size_t)i * 6;
  const U4 u = philox(r[0], r[1], r[2], r[3], r[4], r[5]);
  uint32_t* o = out + (size_t)i * 4;
  o[0] = u.x; o[1] = u.y; o[2] = u.z; o[3] = u.w;
}

}  // namespace

extern "C" {

// The generator's Philox4x32-10 on explicit (counter, key) rows, so it can be
// checked against the published known-answer vectors.
int synth_philox(const uint32_t* d_in, uint32_t* d_out, int n, void* stream) {
  if (n <= 0) return 0;
  philox_rows_kernel<<<(unsigned)((n + 127) / 128), 128, 0, reinterpret_cast<cudaStream_t>(stream)>>>(
      d_in, d_out, n);
  return (int)cudaGetLastError();
}

int synth_gen_vq_idx(uint8_t* out, int n_layers, int batch, int H, int D, int cap, int T,
                     int which, int seq0, uint32_t seed, void* stream) {
  const size_t total = (size_t)n_layers * batch * H * T * (D / 4);
  if (total == 0) return 0;
  if (T > cap) return -1;
  size_t blocks = (total + 255) / 256;
  if (blocks > 148 * 64) blocks = 148 * 64;
  gen_vq_idx_kernel<<<(unsigned)blocks, 256, 0, reinterpret_cast<cudaStream_t>(stream)>>>(
      out, n_layers, batch, H, D, cap, T, which, seq0, seed);
  return (int)cudaGetLastError();
}

int synth_gen_vq_q(uint16_t* q, int n_layers, int batch, int H, int D, int loop, int seq0,
                   uint32_t seed, float nscale, void* stream) {
  const size_t total = (size_t)n_layers * batch * H * D;
  if (total == 0) return 0;
  size_t blocks = (total + 255) / 256;
  if (blocks > 148 * 64) blocks = 148 * 64;
  gen_vq_q_kernel<<<(unsigned)blocks, 256, 0, reinterpret_cast<cudaStream_t>(stream)>>>(
      q, n_layers, batch, H, D, loop, seq0, seed, nscale);
  return (int)cudaGetLastError();
}


int synth_gen_kv(uint16_t* k, uint16_t* v, const int32_t* d_cells, const int32_t* d_seqs,
                 const int32_t* d_t0, int n_cells, int batch, int H, int D, int T,
                 int table_cells, const float* d_chscale, const int32_t* d_refs, uint32_t seed,
                 float nscale, void* stream) {
  const size_t total = (size_t)n_cells * batch * H * T * D;
  if (total == 0) return 0;
  const int threads = 256;
  size_t blocks = (total + threads - 1) / threads;
  if (blocks > 148 * 64) blocks = 148 * 64;
  gen_kv_kernel<<<(unsigned)blocks, threads, 0, reinterpret_cast<cudaStream_t>(stream)>>>(
      k, v, d_cells, d_seqs, d_t0, n_cells, batch, H, D, T, table_cells, d_chscale, d_refs, seed,
      nscale);
  return (int)cudaGetLastError();
}

int synth_gen_q(uint16_t* q, const int32_t* d_cells, const int32_t* d_srcs, const int32_t* d_seqs,
                const int32_t* d_lens, int n_cells, int batch, int H, int g, int D, int mode,
                int table_cells, const float* d_chscale, const int32_t* d_refs, uint32_t seed,
                float nscale, void* stream) {
  const long long warps = (long long)n_cells * batch * H * g;
  if (warps == 0) return 0;
  const int threads = 256;
  const long long blocks = (warps * 32 + threads - 1) / threads;
  gen_q_kernel<<<(unsigned)blocks, threads, 0, reinterpret_cast<cudaStream_t>(stream)>>>(
      q, d_cells, d_srcs, d_seqs, d_lens, n_cells, batch, H, g, D, mode, table_cells, d_chscale,
      d_refs, seed, nscale);
  return (int)cudaGetLastError();
}

}  // extern "C"
