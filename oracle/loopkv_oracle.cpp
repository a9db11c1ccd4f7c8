// LoopKV oracle: a plain, slow, single-threaded CPU restatement of what the
// LoopKV decode path computes.  TEST INFRASTRUCTURE ONLY: the tests, the
// smoke check and the benchmark's CPU-baseline leg may call it; the product
// path never does.  It shares no code, header, table or constant with the
// CUDA library.
//
// Source of the method: "LoopKV: Loop-Aware KV Cache Compression for Serving
// Looped Transformers", section 概要 (the abstract):
//   * each (loop, layer) cell keeps 4-bit codes, 2-bit codes, or reuses the
//     final loop's KV (SHARE);
//   * a 4-bit value is held as two 2-bit planes: every loop takes the upper
//     plane, and the lower plane only for tokens whose weights in that loop
//     call for 4-bit precision.
// The abstract leaves the arithmetic open; this file takes these readings:
//   R1 asymmetric min/max quantization as in "KIVI: A Tuning-Free Asymmetric
//      2bit Quantization for KV Cache": keys per channel over a group of 32
//      tokens, values per token over groups of 32 channels, fp32 scale and
//      zero point (zero = group minimum), codes rounded half-to-even;
//   R2 the IEEE fp32 operations that produce a code are fixed:
//      scale = (max - min) / qmax, code = rne((x - min) / scale), no fused
//      multiply-add, -0 zero point stored as +0, scale 0 => all codes 0;
//   R3 a 4-bit code q splits as hi = q >> 2 (high plane), lo = q & 3 (low
//      plane); a high-plane-only read reconstructs 4*hi + 1.5;
//   R4 a token of a 4-bit cell whose softmax weight p >= tau gets hi+lo, all
//      others hi only; keys are always read at stored precision;
//   R5 fewer than 32 recent tokens stay in a bf16 residual; the residual is
//      quantized as a group the moment it holds 32 tokens;
//   R6 a SHARE cell of length n attends over the final loop's stored
//      positions [0, n-1) plus its own current bf16 key and value;
//   R7 softmax scale 1/sqrt(D) unless given;
//   R8 several query heads may share a KV head (grouped-query attention):
//      each head has its own scores, softmax and output; a token's low
//      plane is fetched for the group when any head's weight reaches tau,
//      and every head of the group reconstructs that token with it (the
//      selection is the union over the group's heads).
// "ResidualQuant: KV Cache Quantization for Looped Transformers with 2-Bit
// Residuals", as summarised in the related-paper list (関連論文リスト) of the
// page "LoopVQ: Sub 1-bit KV Cache Quantization for Looped Transformers":
// the final loop's KV state is the reference and the other loops keep
// low-precision residuals against it.
// Readings for that cell kind (RES2):
//   R9  a RES2 cell sits in a non-final loop; its reference is the final
//       loop's cell of the same layer, sequence and head, stored as 4-bit,
//       2-bit or bf16.  For a position t the residual is d = x - r, where x
//       is the cell's own bf16 input and r the reference's stored value at t
//       dequantized in fp32 (r = fl(fl(scale * q) + zero) with the full code
//       q, no fused multiply-add; the raw value for a bf16 reference), and d
//       = fl(x - r).  Residuals are quantized like a 2-bit cell (R1, R2);
//   R10 a residual group is quantized once the cell holds the 32 tokens
//       after it too (32 (g + 2) tokens for group g), so that the reference,
//       appended later in a decode step, holds the group by then; the cell
//       keeps its last 32..63 tokens (all of them below 32) in bf16;
//   R11 a quantized position reads r^ + d^: r^ the reference's reading as
//       the cell's own decode takes it (keys at stored precision; a 4-bit
//       reference's values through the tau rule of R4 with the cell's own
//       weights), d^ = scale * code + zero of the residual; bf16 positions
//       read the cell's own token.
// "LoopVQ: Sub 1-bit KV Cache Quantization for Looped Transformers",
// section 概要 (the abstract): a vector quantizer codes channels of several
// loop steps jointly, at 0.5 bits per element, with codebooks fine-tuned
// offline.  Readings for its decode (the codebooks are inputs here):
//   V1  a sub-vector is c consecutive channels of one token (channels
//       c*j .. c*j+c-1, group j) across the L loops of its layer, loop-major
//       (element (l, i) at l*c + i); one byte indexes a 256-entry codebook,
//       so L*c = 16 elements per byte is 0.5 bits per element at L = 4, c = 4;
//   V2  one codebook per (layer, KV head) for keys and one for values,
//       shared by the sequences and the channel groups, fp32 entries;
//   V3  decoding loop l reads slice [l*c, l*c + c) of each indexed entry as
//       the token's channels of group j; softmax attention as in R7;
//   V4  every position of a unit is coded (the op attends over coded
//       tokens only);
//   V5  encoding a token picks, per group, the entry nearest to its
//       sub-vector in squared Euclidean distance, computed in fp32 as
//       sum over m = 0 .. 4L-1 (in that order) of fl(fl(x_m - c_m)^2), no
//       fused multiply-add; ties go to the lowest index.
// All attention arithmetic is fp64 (dequantized values, scores, softmax,
// weighted sum).  Quantization is fp32 because the codes are defined by it.
//
// Build: g++ -O2 -std=c++17 -ffp-contract=off -fno-fast-math -shared -fPIC
// (no contraction and no fast-math, so the fp32 steps are the IEEE ones).

#include <algorithm>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <vector>

namespace {

constexpr int kG = 32;  // group size (R1)

enum Kind { KIND_Q4 = 0, KIND_Q2 = 1, KIND_SHARE = 2, KIND_BF16 = 3, KIND_RES2 = 4 };

constexpr int kResWindow = 64;  // bf16 token slots of a RES2 cell (R10)

float bf16_to_float(uint16_t b) {
  uint32_t u = static_cast<uint32_t>(b) << 16;
  float f;
  std::memcpy(&f, &u, 4);
  return f;
}

// One group of 32 fp32 values -> codes, scale, zero (R1, R2).
void quantize_group(const float* x, int bits, uint8_t* code, float* scale,
                    float* zero) {
  const int qmax = (1 << bits) - 1;
  float mn = x[0], mx = x[0];
  for (int i = 1; i < kG; ++i) {
    if (x[i] < mn) mn = x[i];
    if (x[i] > mx) mx = x[i];
  }
  const float range = mx - mn;               // fp32, round to nearest
  const float s = range / static_cast<float>(qmax);
  for (int i = 0; i < kG; ++i) {
    if (s == 0.0f) {
      code[i] = 0;
      continue;
    }
    const float shifted = x[i] - mn;          // fp32
    const float ratio = shifted / s;          // fp32
    float r = std::nearbyint(ratio);          // default mode: half to even
    if (r < 0.0f) r = 0.0f;
    if (r > static_cast<float>(qmax)) r = static_cast<float>(qmax);
    code[i] = static_cast<uint8_t>(r);
  }
  *scale = s;
  *zero = (mn == 0.0f) ? 0.0f : mn;  // canonical +0
}

// State of one (cell, sequence, head) unit after some appends.
struct Unit {
  int kind = 0, D = 0, cap = 0, n = 0;
  // KIND_Q4 / KIND_Q2: quantized groups and the bf16 residual (R5).
  std::vector<uint8_t> kq;   // [qtok][D] key codes
  std::vector<float> ks, kz; // [qtok/32][D] per-channel key scale, zero
  std::vector<uint8_t> vq;   // [qtok][D] value codes
  std::vector<float> vs, vz; // [qtok][D/32] per-token value scale, zero
  std::vector<uint16_t> rk, rv;  // residual [R][D] bf16 bits
  // KIND_BF16 and KIND_RES2: every token raw (RES2 derives its residual
  // codes from these and its reference, R9).
  std::vector<uint16_t> bk, bv;  // [n][D]
  // KIND_SHARE: the current token only.
  std::vector<uint16_t> ck, cv;  // [D]

  int qtok() const {
    if (kind == KIND_RES2) return n / kG >= 2 ? (n / kG - 1) * kG : 0;  // R10
    return (kind == KIND_Q4 || kind == KIND_Q2) ? n - residual() : 0;
  }
  int residual() const { return static_cast<int>(rk.size()) / D; }
  int bits() const { return kind == KIND_Q4 ? 4 : 2; }

  void flush_group() {
    // keys: per channel over the 32 residual tokens
    const int g = static_cast<int>(ks.size()) / D;
    const size_t tok0 = kq.size() / D;
    kq.resize((tok0 + kG) * D);
    vq.resize((tok0 + kG) * D);
    ks.resize((g + 1) * D);
    kz.resize((g + 1) * D);
    vs.resize((tok0 + kG) * (D / kG));
    vz.resize((tok0 + kG) * (D / kG));
    float x[kG];
    uint8_t c[kG];
    for (int d = 0; d < D; ++d) {
      for (int i = 0; i < kG; ++i) x[i] = bf16_to_float(rk[i * D + d]);
      quantize_group(x, bits(), c, &ks[g * D + d], &kz[g * D + d]);
      for (int i = 0; i < kG; ++i) kq[(tok0 + i) * D + d] = c[i];
    }
    // values: per token over groups of 32 channels
    for (int i = 0; i < kG; ++i) {
      for (int j = 0; j < D / kG; ++j) {
        for (int e = 0; e < kG; ++e) x[e] = bf16_to_float(rv[i * D + j * kG + e]);
        const size_t t = tok0 + i;
        quantize_group(x, bits(), c, &vs[t * (D / kG) + j], &vz[t * (D / kG) + j]);
        for (int e = 0; e < kG; ++e) vq[t * D + j * kG + e] = c[e];
      }
    }
    rk.clear();
    rv.clear();
  }

  // Append one token (bf16 bits) following R5 / R6.
  void append_token(const uint16_t* k, const uint16_t* v) {
    if (kind == KIND_SHARE) {
      ck.assign(k, k + D);
      cv.assign(v, v + D);
    } else if (kind == KIND_BF16 || kind == KIND_RES2) {
      bk.insert(bk.end(), k, k + D);
      bv.insert(bv.end(), v, v + D);
    } else {
      rk.insert(rk.end(), k, k + D);
      rv.insert(rv.end(), v, v + D);
      if (residual() == kG) flush_group();
    }
    ++n;
  }
};

// Quantized residual state of a RES2 unit against its reference (R9, R10):
// the same arrays a 2-bit cell keeps, for the positions below own.qtok().
struct ResState {
  int qtok = 0;
  std::vector<uint8_t> kq, vq;
  std::vector<float> ks, kz, vs, vz;
};

bool reference_ok(const Unit& own, const Unit* ref) {
  if (ref == nullptr || ref->D != own.D) return false;
  if (ref->kind == KIND_Q4 || ref->kind == KIND_Q2) return ref->qtok() >= own.qtok();
  if (ref->kind == KIND_BF16) return ref->n >= own.qtok();
  return false;
}

// The reference's stored key / value at (pos, d) in fp32 (R9).
float ref_key32(const Unit& ref, int pos, int d) {
  const int D = ref.D;
  if (ref.kind == KIND_BF16) return bf16_to_float(ref.bk[static_cast<size_t>(pos) * D + d]);
  const int gr = pos / kG;
  const float q = static_cast<float>(ref.kq[static_cast<size_t>(pos) * D + d]);
  const float prod = ref.ks[gr * D + d] * q;
  return prod + ref.kz[gr * D + d];
}
float ref_value32(const Unit& ref, int pos, int d) {
  const int D = ref.D;
  if (ref.kind == KIND_BF16) return bf16_to_float(ref.bv[static_cast<size_t>(pos) * D + d]);
  const size_t j = static_cast<size_t>(pos) * (D / kG) + d / kG;
  const float q = static_cast<float>(ref.vq[static_cast<size_t>(pos) * D + d]);
  const float prod = ref.vs[j] * q;
  return prod + ref.vz[j];
}

ResState residual_state(const Unit& own, const Unit& ref) {
  const int D = own.D;
  ResState st;
  st.qtok = own.qtok();
  const int ng = st.qtok / kG;
  st.kq.resize(static_cast<size_t>(st.qtok) * D);
  st.vq.resize(static_cast<size_t>(st.qtok) * D);
  st.ks.resize(static_cast<size_t>(ng) * D);
  st.kz.resize(static_cast<size_t>(ng) * D);
  st.vs.resize(static_cast<size_t>(st.qtok) * (D / kG));
  st.vz.resize(static_cast<size_t>(st.qtok) * (D / kG));
  float x[kG];
  uint8_t c[kG];
  for (int g = 0; g < ng; ++g) {
    // keys: per channel over the group's 32 tokens
    for (int d = 0; d < D; ++d) {
      for (int i = 0; i < kG; ++i) {
        const int pos = g * kG + i;
        const float xi = bf16_to_float(own.bk[static_cast<size_t>(pos) * D + d]);
        x[i] = xi - ref_key32(ref, pos, d);
      }
      quantize_group(x, 2, c, &st.ks[g * D + d], &st.kz[g * D + d]);
      for (int i = 0; i < kG; ++i) st.kq[static_cast<size_t>(g * kG + i) * D + d] = c[i];
    }
  }
  // values: per token over groups of 32 channels
  for (int pos = 0; pos < st.qtok; ++pos) {
    for (int j = 0; j < D / kG; ++j) {
      for (int e = 0; e < kG; ++e) {
        const int d = j * kG + e;
        const float xi = bf16_to_float(own.bv[static_cast<size_t>(pos) * D + d]);
        x[e] = xi - ref_value32(ref, pos, d);
      }
      const size_t t = static_cast<size_t>(pos) * (D / kG) + j;
      quantize_group(x, 2, c, &st.vs[t], &st.vz[t]);
      for (int e = 0; e < kG; ++e) st.vq[static_cast<size_t>(pos) * D + j * kG + e] = c[e];
    }
  }
  return st;
}

size_t round128(size_t x) { return (x + 127) / 128 * 128; }

// Canonical per-unit region layout (the one the CUDA library writes).
// Offsets in bytes from the start of the unit's region.
struct Layout {
  size_t k_hi = 0, k_lo = 0, k_meta = 0, v_hi = 0, v_lo = 0, v_meta = 0;
  size_t res_k = 0, res_v = 0, cur_k = 0, cur_v = 0, raw_k = 0, raw_v = 0;
  size_t total = 0;
};

Layout make_layout(int kind, int D, int cap) {
  Layout L;
  const size_t ng = static_cast<size_t>(cap / kG);
  const size_t kblock = ng * 8 * D;           // one key plane or key meta
  const size_t vblock = ng * kG * (D / 4);    // one value plane or value meta
  const size_t rblock = static_cast<size_t>(kG) * D * 2;
  size_t off = 0;
  if (kind == KIND_Q4 || kind == KIND_Q2 || kind == KIND_RES2) {
    L.k_hi = off; off += round128(kblock);
    if (kind == KIND_Q4) { L.k_lo = off; off += round128(kblock); }
    L.k_meta = off; off += round128(kblock);
    L.v_hi = off; off += round128(vblock);
    if (kind == KIND_Q4) { L.v_lo = off; off += round128(vblock); }
    L.v_meta = off; off += round128(vblock);
    const size_t window = (kind == KIND_RES2) ? rblock * (kResWindow / kG) : rblock;
    L.res_k = off; off += window;
    L.res_v = off; off += window;
  } else if (kind == KIND_SHARE) {
    L.cur_k = off; off += round128(static_cast<size_t>(D) * 2);
    L.cur_v = off; off += round128(static_cast<size_t>(D) * 2);
  } else {
    L.raw_k = off; off += round128(static_cast<size_t>(cap) * D * 2);
    L.raw_v = off; off += round128(static_cast<size_t>(cap) * D * 2);
  }
  L.total = off;
  return L;
}

void put_bytes(uint8_t* out, uint8_t* valid, size_t off, const void* src, size_t n) {
  std::memcpy(out + off, src, n);
  std::memset(valid + off, 1, n);
}

}  // namespace

extern "C" {

// ---- quantizer -------------------------------------------------------------
void orc_quantize_group(const float* x, int bits, uint8_t* code, float* scale,
                        float* zero) {
  quantize_group(x, bits, code, scale, zero);
}

// ---- unit state ------------------------------------------------------------
void* orc_unit_new(int kind, int D, int cap) {
  if (kind < 0 || kind > 4 || (D != 64 && D != 128) || cap < 0) return nullptr;
  Unit* u = new Unit();
  u->kind = kind;
  u->D = D;
  u->cap = cap;
  return u;
}

void orc_unit_free(void* p) { delete static_cast<Unit*>(p); }

int orc_unit_len(const void* p) { return static_cast<const Unit*>(p)->n; }

// Append n_new tokens given as bf16 bits [n_new][D] each.  Returns 0, or -1
// when the capacity would be exceeded (nothing is appended then).
int orc_unit_append(void* p, const uint16_t* k, const uint16_t* v, int n_new) {
  Unit* u = static_cast<Unit*>(p);
  if (n_new < 0) return -1;
  if (u->kind != KIND_SHARE && u->n + n_new > u->cap) return -1;
  for (int t = 0; t < n_new; ++t)
    u->append_token(k + static_cast<size_t>(t) * u->D, v + static_cast<size_t>(t) * u->D);
  return 0;
}

// Quantized state, for tests: key codes [qtok][D], key scale/zero [qtok/32][D],
// value codes [qtok][D], value scale/zero [qtok][D/32].  Any pointer may be
// null.  src: the reference unit of a RES2 unit (else ignored); the codes of
// a RES2 unit are its residual codes.  Returns qtok, or -1 when a RES2 unit's
// reference is missing or does not hold its quantized positions.
int orc_unit_export(const void* p, const void* src, uint8_t* kq, float* ks, float* kz,
                    uint8_t* vq, float* vs, float* vz) {
  const Unit* u = static_cast<const Unit*>(p);
  ResState rs;
  const ResState* st = nullptr;
  if (u->kind == KIND_RES2) {
    if (!reference_ok(*u, static_cast<const Unit*>(src))) return -1;
    rs = residual_state(*u, *static_cast<const Unit*>(src));
    st = &rs;
  }
  const std::vector<uint8_t>& ukq = st ? st->kq : u->kq;
  const std::vector<float>& uks = st ? st->ks : u->ks;
  const std::vector<float>& ukz = st ? st->kz : u->kz;
  const std::vector<uint8_t>& uvq = st ? st->vq : u->vq;
  const std::vector<float>& uvs = st ? st->vs : u->vs;
  const std::vector<float>& uvz = st ? st->vz : u->vz;
  if (kq) std::copy(ukq.begin(), ukq.end(), kq);
  if (ks) std::copy(uks.begin(), uks.end(), ks);
  if (kz) std::copy(ukz.begin(), ukz.end(), kz);
  if (vq) std::copy(uvq.begin(), uvq.end(), vq);
  if (vs) std::copy(uvs.begin(), uvs.end(), vs);
  if (vz) std::copy(uvz.begin(), uvz.end(), vz);
  return u->qtok();
}

size_t orc_region_bytes(int kind, int D, int cap) { return make_layout(kind, D, cap).total; }

// Write the unit's bytes in the canonical layout; valid[i] = 1 for every byte
// the layout defines at the unit's current length (unused groups and residual
// slots stay 0 in both arrays).  src: a RES2 unit's reference (else ignored).
// Returns 0, or -1 on a size mismatch or a missing / short reference.
int orc_unit_serialize(const void* p, const void* src, uint8_t* out, uint8_t* valid,
                       size_t bytes) {
  const Unit* u = static_cast<const Unit*>(p);
  const int D = u->D;
  const Layout L = make_layout(u->kind, D, u->cap);
  if (bytes != L.total) return -1;
  if (u->kind == KIND_RES2 && !reference_ok(*u, static_cast<const Unit*>(src))) return -1;
  std::memset(out, 0, bytes);
  std::memset(valid, 0, bytes);
  if (u->kind == KIND_SHARE) {
    if (u->n > 0) {
      put_bytes(out, valid, L.cur_k, u->ck.data(), D * 2);
      put_bytes(out, valid, L.cur_v, u->cv.data(), D * 2);
    }
    return 0;
  }
  if (u->kind == KIND_BF16) {
    put_bytes(out, valid, L.raw_k, u->bk.data(), u->bk.size() * 2);
    put_bytes(out, valid, L.raw_v, u->bv.data(), u->bv.size() * 2);
    return 0;
  }
  const bool q4 = u->kind == KIND_Q4;
  const bool res2 = u->kind == KIND_RES2;
  ResState rs;
  if (res2) rs = residual_state(*u, *static_cast<const Unit*>(src));
  const std::vector<uint8_t>& ukq = res2 ? rs.kq : u->kq;
  const std::vector<float>& uks = res2 ? rs.ks : u->ks;
  const std::vector<float>& ukz = res2 ? rs.kz : u->kz;
  const std::vector<uint8_t>& uvq = res2 ? rs.vq : u->vq;
  const std::vector<float>& uvs = res2 ? rs.vs : u->vs;
  const std::vector<float>& uvz = res2 ? rs.vz : u->vz;
  const int ngq = u->qtok() / kG;
  for (int g = 0; g < ngq; ++g) {
    // key planes: [g][chunk of 64 channels][token][4 words of 16 codes]
    for (int c = 0; c < D / 64; ++c) {
      for (int t = 0; t < kG; ++t) {
        for (int w = 0; w < 4; ++w) {
          uint32_t hi = 0, lo = 0;
          for (int j = 0; j < 16; ++j) {
            const int d = 64 * c + 16 * w + j;
            const uint32_t q = ukq[static_cast<size_t>(g * kG + t) * D + d];
            const uint32_t plane_hi = q4 ? (q >> 2) : q;
            hi |= (plane_hi & 3u) << (2 * j);
            lo |= (q & 3u) << (2 * j);
          }
          const size_t off = static_cast<size_t>(g) * 8 * D + c * 512 + t * 16 + w * 4;
          put_bytes(out, valid, L.k_hi + off, &hi, 4);
          if (q4) put_bytes(out, valid, L.k_lo + off, &lo, 4);
        }
      }
    }
    // key meta: scale[D] then zero[D]
    put_bytes(out, valid, L.k_meta + static_cast<size_t>(g) * 8 * D, &uks[g * D], 4 * D);
    put_bytes(out, valid, L.k_meta + static_cast<size_t>(g) * 8 * D + 4 * D, &ukz[g * D], 4 * D);
  }
  for (int t = 0; t < u->qtok(); ++t) {
    // value planes: [token][D/16 words]
    for (int w = 0; w < D / 16; ++w) {
      uint32_t hi = 0, lo = 0;
      for (int j = 0; j < 16; ++j) {
        const uint32_t q = uvq[static_cast<size_t>(t) * D + 16 * w + j];
        const uint32_t plane_hi = q4 ? (q >> 2) : q;
        hi |= (plane_hi & 3u) << (2 * j);
        lo |= (q & 3u) << (2 * j);
      }
      const size_t off = static_cast<size_t>(t) * (D / 4) + w * 4;
      put_bytes(out, valid, L.v_hi + off, &hi, 4);
      if (q4) put_bytes(out, valid, L.v_lo + off, &lo, 4);
    }
    // value meta: (scale_j, zero_j) pairs
    for (int j = 0; j < D / kG; ++j) {
      const size_t off = static_cast<size_t>(t) * (D / 4) + j * 8;
      put_bytes(out, valid, L.v_meta + off, &uvs[t * (D / kG) + j], 4);
      put_bytes(out, valid, L.v_meta + off + 4, &uvz[t * (D / kG) + j], 4);
    }
  }
  if (res2) {
    // bf16 window: position t in slot t mod 64 (R10)
    for (int t = u->qtok(); t < u->n; ++t) {
      const size_t slot = static_cast<size_t>(t % kResWindow) * D * 2;
      put_bytes(out, valid, L.res_k + slot, &u->bk[static_cast<size_t>(t) * D], D * 2);
      put_bytes(out, valid, L.res_v + slot, &u->bv[static_cast<size_t>(t) * D], D * 2);
    }
    return 0;
  }
  for (int r = 0; r < u->residual(); ++r) {
    put_bytes(out, valid, L.res_k + static_cast<size_t>(r) * D * 2, &u->rk[r * D], D * 2);
    put_bytes(out, valid, L.res_v + static_cast<size_t>(r) * D * 2, &u->rv[r * D], D * 2);
  }
  return 0;
}

// ---- decode ----------------------------------------------------------------
// Decode one unit for a group of g query heads that share its keys and
// values (R8; g = 1 is plain one-query decode).  own: the unit; src: the final
// loop's unit of the same layer, sequence and head when own is SHARE (else
// ignored).  q: bf16 bits [g][D].  sm_scale <= 0 means 1/sqrt(D).
// Outputs: out[g][D]; lse[g] (natural log); mask words, one per 32 positions
// of the data cell's quantized range, bit j of word w = position 32w+j
// selected by some head (only when the data cell is 4-bit); *nsel (selected
// positions).  *n_mask_words receives the number of mask words written;
// weights[g][npos] (nullable) receives every head's softmax weight of every
// attended position, own current last.
// sel_override (nullable; mask words in the layout of `mask`): a 4-bit
// position where some head's weight lies within band of tau is selected
// when its bit there is set and not selected otherwise, instead of by the
// comparison p >= tau.  A kernel working in fp32 may decide such a position
// either way; passing its choice gives the output that choice implies, so
// the outputs can then be compared at the full tolerance.  Positions outside
// the band are always decided by the comparison.
// Returns 0, or -1 on invalid input (no positions, SHARE without a source,
// SHARE longer than its source allows, g < 1).
int orc_decode_group(const void* own_p, const void* src_p, const uint16_t* q, int g,
                     double tau, double sm_scale, double band, double* out, double* lse,
                     uint32_t* mask, int* n_mask_words, int* nsel,
                     const uint32_t* sel_override, double* weights) {
  const Unit* own = static_cast<const Unit*>(own_p);
  const Unit* src = static_cast<const Unit*>(src_p);
  const int D = own->D;
  if (g < 1) return -1;
  const Unit* data = own;
  int n_att = own->n;
  const bool share = own->kind == KIND_SHARE;
  const bool res2 = own->kind == KIND_RES2;
  ResState rs;
  if (res2) {
    // the reference's reading plus the residual below qtok (R11)
    if (!reference_ok(*own, src)) return -1;
    rs = residual_state(*own, *src);
    data = src;
  }
  if (share) {
    if (src == nullptr || src->kind == KIND_SHARE || src->D != D) return -1;
    data = src;
    n_att = own->n - 1;  // R6
    if (own->n < 1 || n_att > src->n) return -1;
  }
  if (n_att + (share ? 1 : 0) < 1) return -1;
  if (sm_scale <= 0.0) sm_scale = 1.0 / std::sqrt(static_cast<double>(D));

  std::vector<double> qd(static_cast<size_t>(g) * D);
  for (int i = 0; i < g * D; ++i) qd[i] = static_cast<double>(bf16_to_float(q[i]));

  const bool quant = data->kind == KIND_Q4 || data->kind == KIND_Q2;
  // quantized positions of the data cell; for RES2 those that carry a residual
  const int qtok = res2 ? rs.qtok : (quant ? data->qtok() : 0);
  const int npos = n_att + (share ? 1 : 0);

  // dequantized key of a position (fp64)
  std::vector<double> khat(D);
  auto key_of = [&](int pos) {
    if (res2 && pos >= qtok) {
      for (int d = 0; d < D; ++d) khat[d] = bf16_to_float(own->bk[static_cast<size_t>(pos) * D + d]);
      return;
    }
    if (share && pos == n_att) {
      for (int d = 0; d < D; ++d) khat[d] = bf16_to_float(own->ck[d]);
    } else if (data->kind == KIND_BF16) {
      for (int d = 0; d < D; ++d) khat[d] = bf16_to_float(data->bk[static_cast<size_t>(pos) * D + d]);
    } else if (pos < qtok) {
      const int gr = pos / kG;
      for (int d = 0; d < D; ++d)
        khat[d] = static_cast<double>(data->ks[gr * D + d]) *
                      data->kq[static_cast<size_t>(pos) * D + d] +
                  static_cast<double>(data->kz[gr * D + d]);
    } else {
      const int r = pos - qtok;
      for (int d = 0; d < D; ++d) khat[d] = bf16_to_float(data->rk[static_cast<size_t>(r) * D + d]);
    }
    if (res2) {
      const int gr = pos / kG;
      for (int d = 0; d < D; ++d)
        khat[d] += static_cast<double>(rs.ks[gr * D + d]) * rs.kq[static_cast<size_t>(pos) * D + d] +
                   static_cast<double>(rs.kz[gr * D + d]);
    }
  };

  // scores and softmax, per head
  std::vector<double> p(static_cast<size_t>(g) * npos);
  std::vector<double> s(npos);
  for (int h = 0; h < g; ++h) {
    const double* qh = &qd[static_cast<size_t>(h) * D];
    double smax = -INFINITY;
    for (int pos = 0; pos < npos; ++pos) {
      key_of(pos);
      double acc = 0.0;
      for (int d = 0; d < D; ++d) acc += qh[d] * khat[d];
      s[pos] = sm_scale * acc;
      smax = std::max(smax, s[pos]);
    }
    double sum = 0.0;
    for (int pos = 0; pos < npos; ++pos) sum += std::exp(s[pos] - smax);
    const double l = smax + std::log(sum);
    for (int pos = 0; pos < npos; ++pos) p[static_cast<size_t>(h) * npos + pos] = std::exp(s[pos] - l);
    lse[h] = l;
  }
  if (weights) std::copy(p.begin(), p.end(), weights);

  // selection over the 4-bit quantized positions: any head (R4, R8)
  const bool q4 = data->kind == KIND_Q4;
  const int nq_att = q4 ? std::min(n_att, qtok) : 0;
  const int nwords = (nq_att + kG - 1) / kG;
  for (int w = 0; w < nwords; ++w) mask[w] = 0;
  int count = 0;
  std::vector<char> sel(npos, 0), near(npos, 0);
  for (int pos = 0; pos < nq_att; ++pos) {
    for (int h = 0; h < g; ++h) {
      const double ph = p[static_cast<size_t>(h) * npos + pos];
      if (ph >= tau) sel[pos] = 1;
      if (std::fabs(ph - tau) <= band) near[pos] = 1;
    }
    if (sel_override && near[pos]) sel[pos] = (sel_override[pos / kG] >> (pos % kG)) & 1u;
    if (sel[pos]) {
      mask[pos / kG] |= 1u << (pos % kG);
      ++count;
    }
  }
  *n_mask_words = nwords;
  *nsel = count;

  // weighted values, per head
  for (int i = 0; i < g * D; ++i) out[i] = 0.0;
  for (int pos = 0; pos < npos; ++pos) {
    for (int d = 0; d < D; ++d) {
      double v;
      if (res2 && pos >= qtok) {
        v = bf16_to_float(own->bv[static_cast<size_t>(pos) * D + d]);
      } else if (share && pos == n_att) {
        v = bf16_to_float(own->cv[d]);
      } else if (data->kind == KIND_BF16) {
        v = bf16_to_float(data->bv[static_cast<size_t>(pos) * D + d]);
      } else if (pos < qtok) {
        const int j = d / kG;
        const double sc = data->vs[static_cast<size_t>(pos) * (D / kG) + j];
        const double ze = data->vz[static_cast<size_t>(pos) * (D / kG) + j];
        const int code = data->vq[static_cast<size_t>(pos) * D + d];
        if (q4) {
          const int hi = code >> 2, lo = code & 3;
          const double low_part = sel[pos] ? static_cast<double>(lo) : 1.5;  // R3
          v = sc * (4.0 * hi + low_part) + ze;
        } else {
          v = sc * code + ze;
        }
      } else {
        v = bf16_to_float(data->rv[static_cast<size_t>(pos - qtok) * D + d]);
      }
      if (res2 && pos < qtok) {
        const size_t j = static_cast<size_t>(pos) * (D / kG) + d / kG;
        v += static_cast<double>(rs.vs[j]) * rs.vq[static_cast<size_t>(pos) * D + d] +
             static_cast<double>(rs.vz[j]);
      }
      for (int h = 0; h < g; ++h) {
        const double ph = p[static_cast<size_t>(h) * npos + pos];
        out[static_cast<size_t>(h) * D + d] += ph * v;
      }
    }
  }
  return 0;
}

// One query head (g = 1): q bf16 bits [D], out[D], *lse, sel_override and
// weights[npos] as in orc_decode_group.
int orc_decode(const void* own_p, const void* src_p, const uint16_t* q,
               double tau, double sm_scale, double band, double* out,
               double* lse, uint32_t* mask, int* n_mask_words, int* nsel,
               const uint32_t* sel_override, double* weights) {
  return orc_decode_group(own_p, src_p, q, 1, tau, sm_scale, band, out, lse, mask,
                          n_mask_words, nsel, sel_override, weights);
}

// ---- LoopVQ decode ----------------------------------------------------------
// One unit, one loop (V1-V4).  idx_k, idx_v: [n][D/c] codebook indices;
// cb_k, cb_v: [256][L*c] entries; q: bf16 bits [D]; sm_scale <= 0 means
// 1/sqrt(D).  out[D] (fp64) and *lse (natural log).  Returns 0, or -1 on
// invalid sizes (n < 1, loop outside [0, L), c not dividing D).
int orc_vq_decode(int n_loops, int D, int c, int n, int loop, const uint8_t* idx_k,
                  const uint8_t* idx_v, const float* cb_k, const float* cb_v, const uint16_t* q,
                  double sm_scale, double* out, double* lse) {
  if (n < 1 || n_loops < 1 || loop < 0 || loop >= n_loops || c < 1 || D % c != 0) return -1;
  if (sm_scale <= 0.0) sm_scale = 1.0 / std::sqrt(static_cast<double>(D));
  const int groups = D / c, width = n_loops * c;
  // the loop's channels of an indexed entry (V1, V3)
  auto entry = [&](const float* cb, int e, int d) {
    const int i = d % c;
    return static_cast<double>(cb[static_cast<size_t>(e) * width + loop * c + i]);
  };
  std::vector<double> s(n);
  double smax = -INFINITY;
  for (int t = 0; t < n; ++t) {
    double acc = 0.0;
    for (int d = 0; d < D; ++d) {
      const int e = idx_k[static_cast<size_t>(t) * groups + d / c];
      acc += static_cast<double>(bf16_to_float(q[d])) * entry(cb_k, e, d);
    }
    s[t] = sm_scale * acc;
    smax = std::max(smax, s[t]);
  }
  double sum = 0.0;
  for (int t = 0; t < n; ++t) sum += std::exp(s[t] - smax);
  const double l = smax + std::log(sum);
  *lse = l;
  for (int d = 0; d < D; ++d) out[d] = 0.0;
  for (int t = 0; t < n; ++t) {
    const double p = std::exp(s[t] - l);
    for (int d = 0; d < D; ++d) {
      const int e = idx_v[static_cast<size_t>(t) * groups + d / c];
      out[d] += p * entry(cb_v, e, d);
    }
  }
  return 0;
}

// One token's codebook indices (V1, V5).  x: bf16 bits [n_loops][D], the
// token's keys (or values) in every loop of its layer; cb: [256][L*c];
// idx_out: [D/c].  Returns 0, or -1 on invalid sizes.
int orc_vq_encode(int n_loops, int D, int c, const uint16_t* x, const float* cb,
                  uint8_t* idx_out) {
  if (n_loops < 1 || c < 1 || D % c != 0) return -1;
  const int width = n_loops * c;
  std::vector<float> sub(width);
  for (int j = 0; j < D / c; ++j) {
    for (int l = 0; l < n_loops; ++l)
      for (int i = 0; i < c; ++i)
        sub[l * c + i] = bf16_to_float(x[static_cast<size_t>(l) * D + j * c + i]);
    int best = 0;
    float best_d = INFINITY;
    for (int e = 0; e < 256; ++e) {
      float dist = 0.0f;
      for (int m = 0; m < width; ++m) {
        const float diff = sub[m] - cb[static_cast<size_t>(e) * width + m];
        const float sq = diff * diff;
        dist = dist + sq;
      }
      if (dist < best_d) {
        best_d = dist;
        best = e;
      }
    }
    idx_out[j] = static_cast<uint8_t>(best);
  }
  return 0;
}

// ---- planner ---------------------------------------------------------------
// The plan with the fewest reads within a damage budget and a storage budget,
// by trying every assignment (small instances only).  "LoopKV: Loop-Aware KV
// Cache Compression for Serving Looped Transformers", section 概要: an offline
// profile gives each (loop, layer) cell a predicted damage for 4-bit storage,
// 2-bit storage and reuse of the final loop's KV (damages add); the planner
// searches for the least data read while predicted damage and storage each
// stay within a budget.  Readings:
//   P1 per cached token and KV head, a 4-bit cell stores its six blocks
//      (K hi/lo/meta, V hi/lo/meta: 6 x D/4 bytes) and reads five of them plus
//      the low-plane row of a selected fraction sel of its tokens
//      (5 + sel quarters of D bytes); a 2-bit cell stores and reads four
//      blocks; a SHARE cell stores nothing per token and reads what its
//      layer's final-loop cell reads (its own separate read of that KV);
//   P2 damages are integers (the profile's units) and add over cells;
//   P3 among the assignments within both budgets the lowest total reads
//      wins, then the lowest damage, then the lowest storage.
// Units: storage in quarters of D bytes; reads in thousandths of a quarter
// of D bytes, sel_milli = round(1000 sel).  damage: [cells][3] (Q4, Q2,
// SHARE), loop-major cells.  kinds_out: loop-major, 0 = Q4, 1 = Q2,
// 2 = SHARE.  Returns 0, or -1 when no assignment fits (or bad input).
int orc_plan_brute(int n_loops, int n_layers, const int32_t* damage, int64_t damage_budget,
                   int64_t storage_budget_q, int sel_milli, uint8_t* kinds_out,
                   int64_t* best_reads, int64_t* best_damage, int64_t* best_storage) {
  const int L = n_loops, N = n_layers, cells = L * N;
  if (L < 1 || N < 1 || cells > 16) return -1;
  auto options = [&](int c) { return (c / N == L - 1) ? 2 : 3; };  // no SHARE in the final loop
  std::vector<int> choice(cells, 0);
  bool found = false;
  int64_t br = 0, bd = 0, bs = 0;
  std::vector<uint8_t> best(cells, 0);
  for (;;) {
    int64_t rd = 0, dm = 0, st = 0;
    for (int c = 0; c < cells; ++c) {
      const int k = choice[c];
      dm += damage[c * 3 + k];
      if (k == 0) { st += 6; rd += 5000 + sel_milli; }
      else if (k == 1) { st += 4; rd += 4000; }
      else {
        const int fk = choice[(L - 1) * N + c % N];  // the layer's final-loop cell
        rd += fk == 0 ? 5000 + sel_milli : 4000;
      }
    }
    if (dm <= damage_budget && st <= storage_budget_q) {
      bool better = !found || rd < br || (rd == br && (dm < bd || (dm == bd && st < bs)));
      if (better) {
        found = true; br = rd; bd = dm; bs = st;
        for (int c = 0; c < cells; ++c) best[c] = static_cast<uint8_t>(choice[c]);
      }
    }
    int c = 0;
    while (c < cells) {
      if (++choice[c] < options(c)) break;
      choice[c] = 0;
      ++c;
    }
    if (c == cells) break;
  }
  if (!found) return -1;
  for (int c = 0; c < cells; ++c) kinds_out[c] = best[c];
  *best_reads = br; *best_damage = bd; *best_storage = bs;
  return 0;
}

}  // extern "C"
