// Internal definitions of the LoopKV library: the device plan table, the
// canonical unit layout (as documented in include/loopkv.h) and the kernel
// parameter blocks.  Host and device code of the library include this file;
// nothing outside the library does.
#pragma once

#include <cstddef>
#include <cstdint>

#include "loopkv.h"

namespace loopkv {

constexpr int kGroup = 32;  // tokens per key group, channels per value group
constexpr int kResWindow = 64;  // bf16 window slots of a RES2 unit

// Residual-coded positions of a RES2 unit of n tokens: group g is quantized
// once the unit holds 32 (g + 2) tokens.
inline __host__ __device__ int res2_qtok(int n) { return n >= 2 * kGroup ? (n / kGroup - 1) * kGroup : 0; }

// Status bits a kernel may set in the table's status word.
constexpr uint32_t kStatusLength = 1u;     // a length outside [0, capacity]
constexpr uint32_t kStatusShare = 2u;      // SHARE unit longer than its source allows
constexpr uint32_t kStatusRange = 4u;      // unit needs more score slots than launched

struct TableHeader {           // 256 bytes at the start of the table
  uint32_t status;             // OR of kStatus* bits, cleared by loopkv_check
  uint32_t magic;
  int32_t n_cells, max_batch, n_heads, head_dim;
  uint32_t pad[58];
};
static_assert(sizeof(TableHeader) == 256, "header size");

struct DevCell {               // 16 bytes per cell
  int32_t kind;                // loopkv_kind
  int32_t src;                 // SHARE, RES2: the final-loop cell of the same layer; else itself
  int32_t pad[2];
};

struct DevSeq {                // 32 bytes per (cell, sequence)
  uint64_t offset;             // byte offset of head 0's region from the cache base
  uint64_t stride;             // bytes of one head's region
  int32_t cap;                 // capacity in tokens
  int32_t len;                 // tokens stored
  uint32_t arrive;             // append CTAs done with this pair in the running launch (0 between)
  int32_t pad;
};
static_assert(sizeof(DevSeq) == 32, "seq entry size");

inline __host__ __device__ size_t round_up(size_t x, size_t m) { return (x + m - 1) / m * m; }

// The kernels need IEEE fp32 with subnormals kept: the quantizer must give
// the IEEE codes for subnormal inputs too, the decode turns codes into floats
// as exact subnormals, and the LoopVQ encoder decides indices by fp32
// distances.  A build that flushes subnormals to zero (-ftz=true, or
// --use_fast_math) would change results without a sign, so it does not
// build: there the compiler's __CUDA_FTZ reflection is 1, the call below
// stays in the code, and ptxas stops on the undefined function it names.
// In a correct build the branch is removed and costs nothing.
extern "C" __device__ int __nvvm_reflect(const char*);
extern "C" __device__ void loopkv_build_error_flush_to_zero_is_not_supported(void);
__device__ __forceinline__ void require_ieee_subnormals() {
  if (__nvvm_reflect("__CUDA_FTZ")) loopkv_build_error_flush_to_zero_is_not_supported();
}

inline __host__ __device__ size_t table_cells_offset() { return sizeof(TableHeader); }
inline __host__ __device__ size_t table_seqs_offset(int n_cells) {
  return round_up(sizeof(TableHeader) + sizeof(DevCell) * (size_t)n_cells, 256);
}
inline __host__ __device__ size_t table_bytes(int n_cells, int max_batch) {
  return table_seqs_offset(n_cells) + sizeof(DevSeq) * (size_t)n_cells * (size_t)max_batch;
}

// Byte offsets of the blocks inside one unit's region.
struct UnitLayout {
  size_t k_hi, k_lo, k_meta, v_hi, v_lo, v_meta, res_k, res_v;  // Q4 / Q2
  size_t cur_k, cur_v;                                           // SHARE
  size_t raw_k, raw_v;                                           // BF16
  size_t total;
};

inline __host__ __device__ UnitLayout unit_layout(int kind, int D, int cap) {
  UnitLayout L{};
  const size_t ng = (size_t)(cap / kGroup);
  const size_t block = ng * 8 * (size_t)D;  // a key plane, key meta, value plane or value meta
  const size_t res = (size_t)kGroup * D * 2;
  size_t off = 0;
  if (kind == LOOPKV_Q4 || kind == LOOPKV_Q2 || kind == LOOPKV_RES2) {
    const bool q4 = kind == LOOPKV_Q4;
    const size_t window = kind == LOOPKV_RES2 ? res * (kResWindow / kGroup) : res;
    L.k_hi = off;   off += block;
    L.k_lo = off;   off += q4 ? block : 0;
    L.k_meta = off; off += block;
    L.v_hi = off;   off += block;
    L.v_lo = off;   off += q4 ? block : 0;
    L.v_meta = off; off += block;
    L.res_k = off;  off += window;
    L.res_v = off;  off += window;
  } else if (kind == LOOPKV_SHARE) {
    L.cur_k = off;  off += round_up((size_t)D * 2, 128);
    L.cur_v = off;  off += round_up((size_t)D * 2, 128);
  } else {
    L.raw_k = off;  off += round_up((size_t)cap * D * 2, 128);
    L.raw_v = off;  off += round_up((size_t)cap * D * 2, 128);
  }
  L.total = off;
  return L;
}

// ---------------------------------------------------------------- kernels

struct CellList {
  int32_t cell[LOOPKV_MAX_CELLS_PER_CALL];
  int32_t out[LOOPKV_MAX_CELLS_PER_CALL];  // the cell's index in the caller's list (its input / output slot)
};

struct AppendParams {
  uint8_t* table;
  uint8_t* cache;
  const uint16_t* k;           // [n_cells][batch][H][n_new_max][D]
  const uint16_t* v;
  int32_t n_cells, batch, n_heads, n_new_max;
  int32_t chunks;              // CTAs per unit: a bulk append splits its groups over them
  int32_t n_new[LOOPKV_MAX_BATCH];
};

// Groups one append CTA quantizes when an append brings many (bulk build).
constexpr int kAppendGroupsPerCta = 16;

struct DecodeParams {
  const uint8_t* table;
  const uint8_t* cache;
  const uint16_t* q;           // [n_cells][batch][H][group][D]
  float* out;                  // [n_cells][batch][H][group][D]
  float* lse;                  // nullable [n_cells][batch][H][group]
  uint32_t* mask;              // nullable [n_cells][batch][H][mask_words]
  int32_t* nsel;               // nullable [n_cells][batch][H]
  int32_t mask_words;
  int32_t n_cells, batch, n_heads;
  int32_t group;               // query heads per KV head: 1, 2 or 4
  int32_t split;               // CTAs per unit (a thread-block cluster when > 1)
  int32_t slots;               // score slots per query per CTA (multiple of 32)
  float tau;
  float score_scale;           // sm_scale * log2(e): scores are kept in log2 units
};

// Launchers (decode.cu / append.cu).  Return cudaGetLastError() as int.
// res2: the cells are all RES2 (their own kernel); else none is.  cells.out[i]
// is cell i's index in the caller's list (its slot of the inputs / outputs).
int launch_append(const AppendParams& p, const CellList& cells, void* stream, int head_dim,
                  bool res2);
int launch_decode(const DecodeParams& p, const CellList& cells, void* stream, int head_dim,
                  bool res2);
int decode_max_slots(int head_dim, int group);  // largest per-query score slots per CTA
int decode_max_split();                 // largest cluster size used

}  // namespace loopkv
