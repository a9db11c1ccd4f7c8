"""Plant one mistake at a time in a copy of the CPU oracle and check that the
pins catch it.  Shows the pins would notice a dropped term, a wrong sign,
index or operand, or a wrong constant.  CPU only; the planted copies are
compiled into a temporary directory and never touch the real oracle."""

import ctypes
import os
import subprocess
import tempfile

import pytest

from oracle import build as obuild
from oracle import oracle as orc
from tests import oracle_pins

# (name, text in the oracle, replacement)
MUTANTS = [
    ("qmax off by one", "const int qmax = (1 << bits) - 1;", "const int qmax = (1 << bits);"),
    ("offset by max", "const float shifted = x[i] - mn;", "const float shifted = x[i] - mx;"),
    ("truncate", "float r = std::nearbyint(ratio);", "float r = std::floor(ratio);"),
    ("zero sign kept", "*zero = (mn == 0.0f) ? 0.0f : mn;", "*zero = mn;"),
    ("value axis transposed", "x[e] = bf16_to_float(rv[i * D + j * kG + e]);",
     "x[e] = bf16_to_float(rv[e * D + j * kG + i]);"),
    ("late flush", "if (residual() == kG) flush_group();",
     "if (residual() == kG + 1) flush_group();"),
    ("code order reversed", "hi |= (plane_hi & 3u) << (2 * j);",
     "hi |= (plane_hi & 3u) << (2 * (15 - j));"),
    ("key index shifted", "for (int d = 0; d < D; ++d) acc += qh[d] * khat[d];",
     "for (int d = 0; d < D; ++d) acc += qh[d] * khat[(d + 1) % D];"),
    ("softmax not normalised", "p[static_cast<size_t>(h) * npos + pos] = std::exp(s[pos] - l);",
     "p[static_cast<size_t>(h) * npos + pos] = std::exp(s[pos] - smax);"),
    ("share reads its own slot", "n_att = own->n - 1;  // R6", "n_att = own->n;  // R6"),
    ("high plane weight", "v = sc * (4.0 * hi + low_part) + ze;",
     "v = sc * (2.0 * hi + low_part) + ze;"),
    ("high-plane midpoint", "sel[pos] ? static_cast<double>(lo) : 1.5",
     "sel[pos] ? static_cast<double>(lo) : 2.0"),
    ("zero point dropped", "v = sc * code + ze;", "v = sc * code;"),
    ("tie not selected", "if (ph >= tau) sel[pos] = 1;", "if (ph > tau) sel[pos] = 1;"),
    ("override outside the band", "if (sel_override && near[pos]) sel[pos]",
     "if (sel_override) sel[pos]"),
    ("override ignored", "if (sel_override && near[pos]) sel[pos]",
     "if (sel_override && near[pos] && false) sel[pos]"),
    ("selection from one head only", "if (ph >= tau) sel[pos] = 1;",
     "if (ph >= tau && h == 0) sel[pos] = 1;"),
    ("query heads share one query", "const double* qh = &qd[static_cast<size_t>(h) * D];",
     "const double* qh = &qd[0];"),
    ("sign of zero point", "static_cast<double>(data->kz[gr * D + d]);",
     "-static_cast<double>(data->kz[gr * D + d]);"),
    ("planner: SHARE in the final loop", "return (c / N == L - 1) ? 2 : 3;",
     "return 3;"),
    ("planner: SHARE reads nothing", "rd += fk == 0 ? 5000 + sel_milli : 4000;", "rd += 0;"),
    ("planner: damage tie-break dropped", "(rd == br && (dm < bd || (dm == bd && st < bs)))",
     "(rd == br && st < bs)"),
    ("residual against the reference's high plane",
     "const float q = static_cast<float>(ref.kq[static_cast<size_t>(pos) * D + d]);",
     "const float q = static_cast<float>(ref.kq[static_cast<size_t>(pos) * D + d] & 12);"),
    ("value residual against the reference's high plane",
     "const float q = static_cast<float>(ref.vq[static_cast<size_t>(pos) * D + d]);",
     "const float q = static_cast<float>(ref.vq[static_cast<size_t>(pos) * D + d] & 12);"),
    ("residual window not deferred",
     "if (kind == KIND_RES2) return n / kG >= 2 ? (n / kG - 1) * kG : 0;",
     "if (kind == KIND_RES2) return n / kG * kG;"),
    ("key residual codes dropped", "khat[d] += static_cast<double>(rs.ks[gr * D + d])",
     "khat[d] += 0.0 * static_cast<double>(rs.ks[gr * D + d])"),
    ("value residual codes dropped", "v += static_cast<double>(rs.vs[j])",
     "v += 0.0 * static_cast<double>(rs.vs[j])"),
    ("vq loop slice interleaved", "cb[static_cast<size_t>(e) * width + loop * c + i]",
     "cb[static_cast<size_t>(e) * width + i * n_loops + loop]"),
    ("vq values read the key indices", "const int e = idx_v[static_cast<size_t>(t) * groups + d / c];",
     "const int e = idx_k[static_cast<size_t>(t) * groups + d / c];"),
    ("vq group of a channel", "const int e = idx_k[static_cast<size_t>(t) * groups + d / c];",
     "const int e = idx_k[static_cast<size_t>(t) * groups + d % groups];"),
    ("vq encode keeps the farthest entry", "if (dist < best_d) {", "if (dist > best_d || e == 0) {"),
    ("vq encode ties to the highest index", "if (dist < best_d) {", "if (dist <= best_d) {"),
    ("vq encode reads one loop only", "sub[l * c + i] = bf16_to_float(x[static_cast<size_t>(l) * D + j * c + i]);",
     "sub[l * c + i] = bf16_to_float(x[j * c + i]);"),
    ("residual window slot not modulo 64",
     "const size_t slot = static_cast<size_t>(t % kResWindow) * D * 2;",
     "const size_t slot = static_cast<size_t>(t - u->qtok()) * D * 2;"),
    ("softmax scale 1/D", "sm_scale = 1.0 / std::sqrt(static_cast<double>(D));",
     "sm_scale = 1.0 / static_cast<double>(D);"),
    ("lse without the running max", "const double l = smax + std::log(sum);",
     "const double l = std::log(sum);"),
    ("bf16 residual keys read the values",
     "khat[d] = bf16_to_float(data->rk[static_cast<size_t>(r) * D + d]);",
     "khat[d] = bf16_to_float(data->rv[static_cast<size_t>(r) * D + d]);"),
    ("SHARE current value read from its key", "v = bf16_to_float(own->cv[d]);",
     "v = bf16_to_float(own->ck[d]);"),
    ("mask bits in reverse order", "mask[pos / kG] |= 1u << (pos % kG);",
     "mask[pos / kG] |= 1u << (kG - 1 - pos % kG);"),
    ("vq scores skip the softmax scale", "    s[t] = sm_scale * acc;", "    s[t] = acc;"),
    ("vq value weights unnormalised", "const double p = std::exp(s[t] - l);",
     "const double p = std::exp(s[t] - smax);"),
    ("vq encode distance without the square", "const float sq = diff * diff;",
     "const float sq = std::fabs(diff);"),
    ("planner: storage budget ignored", "if (dm <= damage_budget && st <= storage_budget_q) {",
     "if (dm <= damage_budget) {"),
    ("division by the scale's reciprocal", "const float ratio = shifted / s;          // fp32",
     "const float ratio = shifted * (1.0f / s);  // fp32"),
    ("scale over 2^bits steps", "const float s = range / static_cast<float>(qmax);",
     "const float s = range / static_cast<float>(qmax + 1);"),
    ("residual reference dequantized with one rounding",
     "  const float prod = ref.ks[gr * D + d] * q;\n  return prod + ref.kz[gr * D + d];",
     "  return static_cast<float>(static_cast<double>(ref.ks[gr * D + d]) * q + ref.kz[gr * D + d]);"),
    ("value meta pair stored zero first",
     "      put_bytes(out, valid, L.v_meta + off, &uvs[t * (D / kG) + j], 4);\n"
     "      put_bytes(out, valid, L.v_meta + off + 4, &uvz[t * (D / kG) + j], 4);",
     "      put_bytes(out, valid, L.v_meta + off + 4, &uvs[t * (D / kG) + j], 4);\n"
     "      put_bytes(out, valid, L.v_meta + off, &uvz[t * (D / kG) + j], 4);"),
    ("key meta stored zeros first",
     "put_bytes(out, valid, L.k_meta + static_cast<size_t>(g) * 8 * D, &uks[g * D], 4 * D);",
     "put_bytes(out, valid, L.k_meta + static_cast<size_t>(g) * 8 * D + 4 * D, &uks[g * D], 4 * D);"),
    ("key plane rows a word apart", "c * 512 + t * 16 + w * 4;", "c * 512 + t * 4 + w * 16;"),
    ("planner: 2-bit reads priced as 4-bit", "else if (k == 1) { st += 4; rd += 4000; }",
     "else if (k == 1) { st += 4; rd += 5000; }"),
]


def _compile(src_text, path):
    cpp = path + ".cpp"
    with open(cpp, "w") as f:
        f.write(src_text)
    subprocess.check_call(["g++", *obuild.FLAGS, cpp, "-o", path])


@pytest.mark.parametrize("name,old,new", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_pins_catch_mutant(name, old, new, monkeypatch):
    src = open(obuild.SRC).read()
    assert src.count(old) >= 1, "mutation site not found: %s" % name
    mutated = src.replace(old, new, 1)
    with tempfile.TemporaryDirectory() as tmp:
        lib = os.path.join(tmp, "libmutant.so")
        _compile(mutated, lib)
        monkeypatch.setattr(orc, "_lib", None)
        monkeypatch.setattr(obuild, "build", lambda force=False: lib)
        failed = []
        for pin in oracle_pins.ALL_PINS:
            try:
                pin()
            except Exception as e:  # AssertionError or a rejected input
                failed.append((pin.__name__, type(e).__name__))
        monkeypatch.setattr(orc, "_lib", None)
    assert failed, "planted mistake %r passed every pin" % name


def test_real_oracle_passes_all_pins():
    orc._lib = None
    for pin in oracle_pins.ALL_PINS:
        pin()
    assert isinstance(orc._load(), ctypes.CDLL)
