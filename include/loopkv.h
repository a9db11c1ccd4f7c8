/*
 * loopkv.h - C ABI of the LoopKV decode library for NVIDIA B200 (sm_100a).
 *
 * What it computes.  "LoopKV: Loop-Aware KV Cache Compression for Serving
 * Looped Transformers", section 概要 (abstract): a looped transformer keeps
 * one KV cache per (loop, layer) cell; a plan gives every cell 4-bit storage,
 * 2-bit storage, or reuse of the final loop's KV (SHARE); a 4-bit value is
 * held as two 2-bit planes, every loop streams the upper plane, and the
 * lower plane is gathered only for the tokens that loop's softmax weights
 * mark as needing full precision; a single fused kernel executes the plan.  The abstract fixes no arithmetic; this
 * library takes these readings (the CPU oracle under oracle/ takes the same):
 *   - asymmetric min/max quantization as in "KIVI: A Tuning-Free Asymmetric
 *     2bit Quantization for KV Cache": keys per channel over groups of 32
 *     tokens, values per token over groups of 32 channels, fp32 scale =
 *     (max - min) / qmax and zero point = min, codes rounded half to even,
 *     all in IEEE fp32 without fused multiply-add; scale 0 gives codes 0;
 *   - a 4-bit code q is kept as two 2-bit planes, hi = q >> 2 and
 *     lo = q & 3; reading hi alone reconstructs scale * (4*hi + 1.5) + zero;
 *   - a value of a 4-bit cell uses hi and lo when its softmax weight
 *     p >= tau, else hi only; keys are always read at stored precision;
 *   - fewer than 32 recent tokens stay in a bf16 residual, quantized as a
 *     group the moment it holds 32;
 *   - a SHARE cell of length n attends over the final loop's stored
 *     positions [0, n-1) (same layer, sequence and head) plus its own
 *     current bf16 key and value;
 *   - softmax scale 1/sqrt(head_dim) unless given; one query per KV head,
 *     or a group of 2 or 4 sharing it (q_per_kv; see loopkv_decode).
 * LOOPKV_BF16 (raw bf16 cells) exists for ablations and checks.
 *
 * Residual cells.  "ResidualQuant: KV Cache Quantization for Looped
 * Transformers with 2-Bit Residuals", as summarised in the related-paper list
 * (関連論文リスト) of the page "LoopVQ: Sub 1-bit KV Cache Quantization for
 * Looped Transformers": the final loop's KV is a reference and the other
 * loops keep low-precision residuals against it.  A LOOPKV_RES2 cell (non-final loops only) stores, for each
 * position t, d = fl32(x - r) quantized like a LOOPKV_Q2 cell, where x is
 * its own bf16 input and r the reference's stored value at t in fp32:
 * fl32(fl32(scale * q) + zero) with the full code q of a 4-bit or 2-bit
 * reference, the raw value of a bf16 one.  The reference is the final loop's
 * cell of the same layer, sequence and head (LOOPKV_Q4, LOOPKV_Q2 or
 * LOOPKV_BF16).  A residual group g is quantized when the cell reaches
 * 32 (g + 2) tokens, so the reference, appended after it in a decode step,
 * already holds the group; the cell keeps its other tokens, 32..63 of them
 * once it has 32 (all of them before), in bf16.  Decode reads a quantized
 * position as the reference's reading (keys at stored precision, values of
 * a 4-bit reference through the tau rule with the cell's own weights) plus
 * scale * code + zero of the residual, and a bf16 position as the cell's own
 * token.
 *
 * Terms.  cells = n_loops * n_layers, indexed loop-major (cell = loop *
 * n_layers + layer).  A unit is one (cell, sequence, head).  Tokens of a
 * unit are positions 0..n-1.
 *
 * Memory.  The caller owns every device buffer (table, cache, inputs and
 * outputs) and every stream; the library allocates no device memory and
 * owns only the host-side plan handle, which holds a host copy of the
 * per-(cell, sequence) lengths.  Device pointers must be 16-byte aligned;
 * the cache must be 256-byte aligned.  Streams are passed as `void*` and
 * mean `cudaStream_t` (NULL = the legacy default stream).  bf16 data travel
 * as their 16-bit patterns (`uint16_t`).
 *
 * Errors.  Every call returns a status.  Argument, plan and capacity errors
 * are found on the host, from the host copy of the lengths, before anything
 * is launched; the device state is then untouched.  A failed launch returns
 * LOOPKV_ERR_CUDA.  Kernels never trap: an inconsistency they detect (which
 * the host checks should make impossible) sets a bit in a status word inside
 * the table, skips the affected unit, and is reported by loopkv_check().
 *
 * Asynchrony.  loopkv_append, loopkv_decode and loopkv_set_lengths only
 * enqueue work on the given stream and return.  A decode (and the LoopVQ
 * calls) can be captured into a CUDA graph and replayed any number of times.
 * An append or set_lengths updates the host copy of the lengths when it is
 * called, i.e. at capture time, while the kernels advance the device lengths
 * when they run: a graph holding appends (whole serving steps) is to be
 * replayed once after its capture, which leaves the two copies equal; a
 * second replay would leave the host copy behind.  A plan handle must not be
 * used from two host threads at once.
 *
 * Cache layout (canonical, part of the contract).  The cache is one buffer;
 * cell c, sequence b, head h owns a region at loopkv_unit_region().  With
 * capacity C tokens and NG = C / 32 (integer division) groups, a LOOPKV_Q4
 * region holds, in order, each block a multiple of 128 bytes:
 *   K_hi  [NG][D/64][32 tokens][4 words]   2-bit codes, channel 64c+16w+j of
 *                                           the token in bits 2j..2j+1 of word w
 *   K_lo  [NG][D/64][32][4]                 low planes, same arrangement
 *   K_meta[NG]{scale[D], zero[D]}           fp32, per channel of the group
 *   V_hi  [NG*32 tokens][D/16 words]        channel 16w+j in bits 2j..2j+1
 *   V_lo  [NG*32][D/16]
 *   V_meta[NG*32]{(scale, zero) x D/32}     fp32 pairs per 32 channels
 *   res_K [32][D], res_V [32][D]            bf16 residual; slot r holds
 *                                           position 32*floor(n/32) + r
 * LOOPKV_Q2 has the same blocks without K_lo and V_lo; its "hi" planes hold
 * the 2-bit codes.  LOOPKV_RES2 has the LOOPKV_Q2 blocks holding residual
 * codes, with res_K [64][D], res_V [64][D] instead: position t of its bf16
 * window in slot t mod 64.  LOOPKV_SHARE holds cur_K[D], cur_V[D] (bf16, each block
 * rounded up to 128 bytes).  LOOPKV_BF16 holds K[C][D] then V[C][D] (bf16,
 * each rounded up to 128 bytes).
 */
#ifndef LOOPKV_H_
#define LOOPKV_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  LOOPKV_OK = 0,
  LOOPKV_ERR_INVALID_ARG = 1, /* null pointer, bad size, bad cell index ... */
  LOOPKV_ERR_PLAN = 2,        /* plan descriptor is not a valid plan */
  LOOPKV_ERR_CAPACITY = 3,    /* an append would exceed a unit's capacity */
  LOOPKV_ERR_UNSUPPORTED = 4, /* valid request outside what is implemented */
  LOOPKV_ERR_CUDA = 5,        /* a CUDA call failed */
  LOOPKV_ERR_DEVICE = 6       /* a kernel flagged an inconsistency */
} loopkv_status;

typedef enum {
  LOOPKV_Q4 = 0,    /* 4-bit codes kept as hi and lo 2-bit planes */
  LOOPKV_Q2 = 1,    /* 2-bit codes */
  LOOPKV_SHARE = 2, /* reuse the final loop's KV; keeps its current token */
  LOOPKV_BF16 = 3,  /* raw bf16 (ablation / checks) */
  LOOPKV_RES2 = 4   /* 2-bit residuals against the final loop's KV */
} loopkv_kind;

/* Largest number of cells one loopkv_append / loopkv_decode call may name. */
#define LOOPKV_MAX_CELLS_PER_CALL 256
/* Largest batch (sequences) a plan may hold. */
#define LOOPKV_MAX_BATCH 256

typedef struct {
  int32_t n_loops;        /* >= 1 */
  int32_t n_layers;       /* >= 1; n_loops * n_layers <= 4096 */
  int32_t n_kv_heads;     /* >= 1 */
  int32_t head_dim;       /* 64 or 128 */
  int32_t max_batch;      /* 1 .. LOOPKV_MAX_BATCH */
  const int32_t* capacity;/* host [max_batch]: tokens each unit of sequence b
                             can hold, 0 .. 2^20 */
  const uint8_t* kinds;   /* host [n_loops * n_layers], loop-major,
                             loopkv_kind values; LOOPKV_SHARE and
                             LOOPKV_RES2 only in loops < n_loops - 1 */
  float tau;              /* low-plane threshold on the softmax weight, >= 0 */
  float sm_scale;         /* softmax scale; <= 0 means 1/sqrt(head_dim) */
  int32_t q_per_kv;       /* query heads per KV head (grouped-query
                             attention): 1, 2 or 4; 0 means 1.  The heads of
                             a group share the KV head's reads; see
                             loopkv_decode for their selection. */
  int32_t decode_split;   /* CTAs (a thread-block cluster) per decoded unit:
                             0 lets the library choose (enough score slots
                             for the longest unit of a call, more while a
                             call's CTAs fall short of one full wave of two
                             per SM); 1, 2, 4 or
                             8 asks for at least that many.  The results do
                             not depend on it beyond fp32 rounding order. */
} loopkv_plan_desc;

typedef struct {
  size_t table_bytes; /* device plan table: the plan's device state (cells,
                         per-(cell, sequence) regions and lengths, the
                         appends' arrival counts, the status word) */
  size_t cache_bytes; /* device KV cache in the canonical layout */
} loopkv_sizes;

typedef struct loopkv_plan loopkv_plan; /* opaque host handle */

/* Validate a plan and report the device memory it needs.
 * Errors: LOOPKV_ERR_INVALID_ARG (null), LOOPKV_ERR_PLAN (bad kinds, SHARE
 * in the final loop, head_dim not 64/128, sizes out of range). */
loopkv_status loopkv_plan_query(const loopkv_plan_desc* desc, loopkv_sizes* sizes);

/* Bind a plan to caller-allocated device memory.  Writes the plan table to
 * d_table (table_bytes >= the queried size) on `stream` and sets every
 * length to 0.  The cache contents need no initialisation.  The descriptor's
 * host arrays are copied; the handle keeps the pointers d_table and d_cache,
 * which must stay valid until loopkv_plan_free.  On success *out receives a
 * new handle. */
loopkv_status loopkv_plan_load(const loopkv_plan_desc* desc, void* d_table, size_t table_bytes,
                               void* d_cache, size_t cache_bytes, void* stream,
                               loopkv_plan** out);

/* Release the host handle (device memory stays the caller's). NULL is a no-op. */
void loopkv_plan_free(loopkv_plan* plan);

/* Append tokens: the LoopKV cache update (quantize, split into bit planes,
 * store).  For every listed cell c = h_cells[i], sequence b < batch and head
 * h, tokens t < h_n_new[b] of
 *     d_k, d_v: bf16 [n_cells][batch][n_kv_heads][n_new_max][head_dim]
 * become positions len+t of the unit (len = the unit's length before the
 * call).  Q4/Q2 cells: tokens enter the bf16 residual; each time it holds 32
 * tokens they are quantized as one group (keys per channel, values per token
 * per 32 channels) into the planes.  SHARE cells keep only the last appended
 * token as their current key and value.  BF16 cells store tokens raw.
 * RES2 cells keep tokens in their bf16 window and quantize residual group g
 * once they hold 32 (g + 2) tokens, reading the reference's group g; the
 * reference must hold that group before the call (its length before the
 * call is what counts, so a call may append a RES2 cell and its reference
 * together).  Lengths grow by h_n_new[b].  h_cells: distinct cell indices;
 * h_n_new: host [batch], each 0 .. n_new_max.
 * Errors (nothing launched): LOOPKV_ERR_INVALID_ARG (also: a RES2 append
 * whose reference does not yet hold a group it needs), LOOPKV_ERR_CAPACITY
 * (len + n_new > capacity for a non-SHARE unit). */
loopkv_status loopkv_append(loopkv_plan* plan, const int32_t* h_cells, int32_t n_cells,
                            int32_t batch, const int32_t* h_n_new, int32_t n_new_max,
                            const uint16_t* d_k, const uint16_t* d_v, void* stream);

/* Decode attention: the fused LoopKV read of the plan.  For every listed
 * cell c = h_cells[i], sequence b < batch, KV head h and query head r <
 * g = q_per_kv of h's group, with queries
 *     d_q: bf16 [n_cells][batch][n_kv_heads][g][head_dim]
 * computes over the unit's attended positions (its own n tokens; for a SHARE
 * unit of length n, the final loop's stored positions [0, n-1) and its own
 * current token; for a RES2 unit its n tokens, the residual-coded ones read
 * through the reference) the scores sm_scale * <q_r, k>, with keys dequantized at
 * their stored precision, each query's softmax p_r, the selection of the
 * 4-bit quantized positions where some query of the group has p_r >= tau
 * (one query: p >= tau; the KV head's low plane is read once for the whole
 * group, and every query of the group uses what was read), and
 *     d_out: fp32 [n_cells][batch][n_kv_heads][g][head_dim] = sum_t p_r,t v_t
 * with v_t at 4-bit precision where selected, high plane only otherwise,
 * 2-bit, or bf16 as stored.  Optional outputs (NULL to skip):
 *     d_lse : fp32 [n_cells][batch][n_kv_heads][g], natural-log logsumexp
 *     d_mask: uint32 [n_cells][batch][n_kv_heads][mask_words]; bit j of
 *             word w = position 32w+j was selected; words
 *             0 .. ceil(nq/32)-1 are written, nq = 4-bit positions attended
 *     d_nsel: int32 [n_cells][batch][n_kv_heads], number of selected positions
 * Every unit must hold n >= 1 tokens; a SHARE unit needs its source to hold
 * at least n-1; a RES2 unit needs its reference to hold its residual-coded
 * positions.  SHARE units read the source as it is stored when the kernel
 * runs (decode a loop before appending to the final loop for serving order).
 * RES2 cells run in a second launch on the same stream.
 * Errors (nothing launched): LOOPKV_ERR_INVALID_ARG, LOOPKV_ERR_UNSUPPORTED
 * (a unit longer than the kernel's limit). */
loopkv_status loopkv_decode(loopkv_plan* plan, const int32_t* h_cells, int32_t n_cells,
                            int32_t batch, const uint16_t* d_q, float* d_out, float* d_lse,
                            uint32_t* d_mask, int32_t mask_words, int32_t* d_nsel,
                            void* stream);

/* Set the lengths of (cell, sequence) pairs: h_len is host [n_cells][batch]
 * for the listed cells.  Allowed per unit: 0 (reset), or any value that
 * keeps every stored position valid: new <= old and, for Q4/Q2 cells,
 * new >= 32*floor(old/32) (drop residual tokens only) or new a multiple of
 * 32 (drop whole groups); SHARE cells: new == old (only the current
 * token is kept, so a SHARE unit can only be reset); RES2 cells: new keeps
 * the same residual-coded count 32 * max(0, floor(n/32) - 1) (drop window
 * tokens only).  For rollback and reuse of sequence slots.
 * Errors: LOOPKV_ERR_INVALID_ARG. */
loopkv_status loopkv_set_lengths(loopkv_plan* plan, const int32_t* h_cells, int32_t n_cells,
                                 int32_t batch, const int32_t* h_len, void* stream);

/* Host copy of the lengths: h_len receives [n_loops*n_layers][max_batch]. */
loopkv_status loopkv_get_lengths(const loopkv_plan* plan, int32_t* h_len);

/* Byte offset (from the cache base) and size of the region of unit
 * (cell, seq, head) in the canonical layout. */
loopkv_status loopkv_unit_region(const loopkv_plan* plan, int32_t cell, int32_t seq,
                                 int32_t head, uint64_t* offset, uint64_t* bytes);

/* Wait for `stream`, then read and clear the device status word.
 * Returns LOOPKV_ERR_DEVICE if a kernel flagged an inconsistency. */
loopkv_status loopkv_check(loopkv_plan* plan, void* stream);

/* Static description of a status code. */
const char* loopkv_status_string(loopkv_status status);

/* ---- Planner ------------------------------------------------------------
 * "LoopKV: Loop-Aware KV Cache Compression for Serving Looped Transformers",
 * section 概要: a one-time offline profile gives every (loop, layer) cell a
 * predicted damage for 4-bit storage, 2-bit storage and reuse of the final
 * loop's KV (SHARE); damages add over cells; the planner looks for the plan
 * with the least data read whose predicted damage and storage each stay
 * within a budget.  The pages fix nothing
 * else; this library reads it as follows.  Per cached token and KV head:
 *   Q4    stores 6 blocks of D/4 bytes (K hi/lo/meta, V hi/lo/meta) and reads
 *         5 of them plus a low-plane row for a fraction sel_fraction of its
 *         tokens;
 *   Q2    stores and reads 4 blocks;
 *   SHARE stores nothing per token and reads what the final-loop cell of its
 *         layer reads (its own read of that KV); not allowed in the final loop.
 * Among the plans within both budgets the one with the fewest reads wins,
 * then the least damage, then the least storage (ties beyond that: any).
 * Exact: a dynamic program over layers whose options are the 2 * 3^(L-1)
 * assignments of a layer's cells, over (damage, storage) states. */
typedef struct {
  int32_t n_loops;         /* 1 .. 6 */
  int32_t n_layers;        /* >= 1; n_loops * n_layers <= 4096 */
  int32_t head_dim;        /* 64 or 128 */
  const int32_t* damage;   /* host [n_loops * n_layers][3], loop-major cells:
                              predicted damage of Q4, Q2 and SHARE in integer
                              profile units, >= 0 (SHARE ignored in the final
                              loop) */
  int64_t damage_budget;   /* >= 0: total damage allowed */
  int64_t storage_budget;  /* >= 0: bytes per cached token and KV head,
                              summed over the cells */
  float sel_fraction;      /* [0, 1]: expected fraction of 4-bit tokens whose
                              low plane is read; counted in thousandths */
} loopkv_planner_desc;

typedef struct {
  double reads;            /* bytes read per decode step per cached token and
                              KV head, summed over the cells */
  int64_t damage;          /* total predicted damage */
  int64_t storage;         /* bytes per cached token and KV head */
} loopkv_plan_cost;

/* Choose every cell's storage (kinds_out: host [n_loops * n_layers],
 * loop-major loopkv_kind values, ready for loopkv_plan_desc.kinds) and
 * report the plan's cost (cost may be NULL).  Host only; no device work.
 * Errors: LOOPKV_ERR_INVALID_ARG (null pointers, negative values, sizes out
 * of range), LOOPKV_ERR_PLAN (no plan fits the budgets; kinds_out untouched),
 * LOOPKV_ERR_UNSUPPORTED (more than 2^20 (damage, storage) states after the
 * budgets are capped at what the cells can use). */
loopkv_status loopkv_plan_optimize(const loopkv_planner_desc* desc, uint8_t* kinds_out,
                                   loopkv_plan_cost* cost);

/* ---- LoopVQ decode --------------------------------------------------------
 * "LoopVQ: Sub 1-bit KV Cache Quantization for Looped Transformers", section
 * 概要 (abstract): a vector quantizer codes channels of several loop steps
 * jointly (0.5 bits per element), with codebooks fine-tuned offline.  The
 * abstract fixes no format; this library reads it as follows (the CPU
 * oracle takes the same readings):
 *   - a sub-vector is 4 consecutive channels of one token (group j: channels
 *     4j .. 4j+3) across the n_loops loops of its layer, loop-major (element
 *     (l, i) at 4l + i); one byte indexes a 256-entry codebook, so one byte
 *     codes 4 * n_loops elements (0.5 bits per element at 4 loops);
 *   - one key codebook and one value codebook per (layer, KV head), fp32
 *     entries [256][4 * n_loops], shared by sequences and channel groups
 *     (trained offline: inputs here);
 *   - decoding loop l reads slice [4l, 4l + 4) of each indexed entry as the
 *     token's channels of group j; scores sm_scale * <q, k>, softmax, and
 *     out = sum_t p_t v_t in fp32;
 *   - every position [0, len[b]) of a unit is coded.
 * Shapes: idx_k, idx_v uint8 [n_layers][batch][n_kv_heads][capacity][D/4]
 * (a token's D/4 indices contiguous); cb_k, cb_v fp32
 * [n_layers][n_kv_heads][256][4 * n_loops]; q bf16 [n_layers][batch]
 * [n_kv_heads][D]; out fp32, same shape; lse fp32 [n_layers][batch]
 * [n_kv_heads] (natural log) or NULL.  All device pointers 16-byte aligned;
 * the caller owns them. */
typedef struct {
  int32_t n_loops;     /* loops coded jointly, 1 .. 8 */
  int32_t n_layers;    /* layers decoded by one call, >= 1 */
  int32_t n_kv_heads;  /* >= 1 */
  int32_t head_dim;    /* 64 or 128 */
  int32_t batch;       /* sequences, 1 .. LOOPKV_MAX_BATCH */
  int32_t capacity;    /* token stride of the index arrays, 1 .. 2^20 */
  float sm_scale;      /* <= 0 means 1/sqrt(head_dim) */
} loopkv_vq_desc;

/* Decode loop `loop` (0 .. n_loops-1) of every (layer, sequence, KV head)
 * over positions [0, h_len[b]) (host [batch], each 1 .. capacity).  Enqueued
 * on `stream`.  Errors (nothing launched): LOOPKV_ERR_INVALID_ARG (null or
 * misaligned pointers, sizes out of range), LOOPKV_ERR_UNSUPPORTED (a
 * sequence longer than 8 CTAs of score slots), LOOPKV_ERR_CUDA. */
loopkv_status loopkv_vq_decode(const loopkv_vq_desc* desc, int32_t loop, const int32_t* h_len,
                               const uint8_t* d_idx_k, const uint8_t* d_idx_v,
                               const float* d_cb_k, const float* d_cb_v, const uint16_t* d_q,
                               float* d_out, float* d_lse, void* stream);

/* Encode n_new tokens of every (layer, sequence, KV head) once every loop
 * has produced them: d_x bf16 [n_loops][n_layers][batch][n_kv_heads][n_new]
 * [head_dim] holds each token's keys (or values) in every loop; its D/4
 * codebook indices go to positions h_pos[b] .. h_pos[b] + n_new - 1 of
 * d_idx [n_layers][batch][n_kv_heads][capacity][D/4], using d_cb (the key
 * or the value codebooks, shapes as for loopkv_vq_decode).  Per group: the
 * entry nearest to the sub-vector in squared Euclidean distance, computed
 * in fp32 as sum over m = 0 .. 4 n_loops - 1 (in that order) of
 * fl(fl(x_m - c_m)^2) without fused multiply-add; ties go to the lowest
 * index.  Call once for keys and once for values.  Errors (nothing
 * launched): LOOPKV_ERR_INVALID_ARG (null or misaligned pointers, sizes,
 * positions outside the capacity). */
loopkv_status loopkv_vq_encode(const loopkv_vq_desc* desc, const int32_t* h_pos, int32_t n_new,
                               const uint16_t* d_x, const float* d_cb, uint8_t* d_idx,
                               void* stream);

#ifdef __cplusplus
}
#endif

#endif /* LOOPKV_H_ */
