"""Pins that tie the CPU oracle to facts outside itself.

Each ``pin_*`` function raises AssertionError when the oracle disagrees with
a hand-worked example, a closed form, brute force, or a textbook attention
routine (``torch.nn.functional.scaled_dot_product_attention`` in fp64) on a
special case the LoopKV decode reduces to.  ``test_oracle_pins.py`` runs them
against the oracle; ``test_oracle_mutants.py`` runs them against copies of the
oracle with a mistake planted, each of which must fail at least one pin.

Method: "LoopKV: Loop-Aware KV Cache Compression for Serving Looped
Transformers", section 概要; quantizer as in "KIVI: A Tuning-Free Asymmetric
2bit Quantization for KV Cache" (keys per channel, values per token, groups
of 32, asymmetric min/max, round half to even).
"""

import numpy as np
import torch

from oracle import oracle as orc
from synth import philox as px

G = 32


def bf16(x):
    return px.float_to_bf16_bits(np.asarray(x, np.float32))


def f32(bits):
    return px.bf16_bits_to_float(bits)


def sdpa(q, k, v, scale):
    """Textbook softmax attention in fp64 (library routine)."""
    q = torch.tensor(np.asarray(q, np.float64)).view(1, 1, 1, -1)
    k = torch.tensor(np.asarray(k, np.float64))[None, None]
    v = torch.tensor(np.asarray(v, np.float64))[None, None]
    return torch.nn.functional.scaled_dot_product_attention(q, k, v, scale=scale).view(-1).numpy()


def rng_bits(seed, shape, scale=1.0):
    """Seeded bf16 bit patterns from the shared input generator."""
    n = int(np.prod(shape))
    u = px.philox4x32(np.arange(n, dtype=np.uint32), 0, 0, 0, seed, 99)
    z = px.normal_from_bits(*u).reshape(shape) * np.float32(scale)
    return bf16(z)


# ------------------------------------------------------------ quantizer pins

def pin_quantize_q2_ties():
    # range [0, 3] at 2 bits: scale 1, zero 0; 0.5 -> 0 and 2.5 -> 2 (ties to
    # even), 1.5 -> 2.
    x = np.zeros(G, np.float32)
    x[:7] = [0.0, 3.0, 0.5, 1.5, 2.5, 1.0, 2.0]
    code, s, z = orc.quantize_group(x, 2)
    assert s == np.float32(1.0) and z == np.float32(0.0), (s, z)
    assert list(code[:7]) == [0, 3, 0, 2, 2, 1, 2], code[:7]
    assert (code[7:] == 0).all()


def pin_quantize_q4_ties():
    # range [0, 15] at 4 bits: scale 1; 7.5 -> 8, 8.5 -> 8, 0.25 -> 0, 14.75 -> 15
    x = np.zeros(G, np.float32)
    x[:16] = np.arange(16)
    x[16:20] = [7.5, 8.5, 0.25, 14.75]
    code, s, z = orc.quantize_group(x, 4)
    assert s == np.float32(1.0) and z == np.float32(0.0)
    assert list(code[:16]) == list(range(16))
    assert list(code[16:20]) == [8, 8, 0, 15], code[16:20]


def pin_quantize_fp32_scale():
    # group {-1, 1, 0...} at 4 bits: scale = fl32(2/15) = 0.13333334, and
    # (0 - (-1)) / scale = 7.4999995 in fp32, so 0 maps to code 7 (the exact
    # ratio 7.5 would give 8): the division uses the stored fp32 scale.
    x = np.zeros(G, np.float32)
    x[0], x[1] = -1.0, 1.0
    code, s, z = orc.quantize_group(x, 4)
    assert s == np.float32(2.0) / np.float32(15.0)
    assert z == np.float32(-1.0)
    assert code[0] == 0 and code[1] == 15 and (code[2:] == 7).all(), code


def pin_quantize_division_is_correctly_rounded():
    # The ratio is one IEEE fp32 division (x - min) / scale, rounded once,
    # then rounded half to even.  4 bits, group {0, 1.125, 0.5625, 0...}:
    # scale = fl32(1.125 / 15) = 0.0750000030 (just above 0.075), and
    # 0.5625 / 0.0750000030 = 7.49999970..., whose nearest fp32 is 7.49999952
    # (7.5 is 2.98e-7 away, 7.49999952 only 1.79e-7), so the code is 7; a
    # multiply by the rounded reciprocal lands on 7.5 and gives 8.
    # 2 bits, group {0, 1.625, 0.8125, 0...}: scale = fl32(1.625 / 3) =
    # 0.541666687, and 0.8125 / 0.541666687 = 1.49999995..., whose nearest
    # fp32 is 1.5 (a tie, so code 2); the reciprocal path gives 1.49999988 -> 1.
    x = np.zeros(G, np.float32)
    x[1], x[2] = 1.125, 0.5625
    code, s, z = orc.quantize_group(x, 4)
    assert s == np.float32(1.125) / np.float32(15.0) and z == 0.0
    assert code[0] == 0 and code[1] == 15 and code[2] == 7, code[:3]
    x[1], x[2] = 1.625, 0.8125
    code, s, z = orc.quantize_group(x, 2)
    assert s == np.float32(1.625) / np.float32(3.0)
    assert code[0] == 0 and code[1] == 3 and code[2] == 2, code[:3]


def pin_quantize_degenerate():
    # constant group: scale 0, all codes 0, zero = the constant
    x = np.full(G, 3.25, np.float32)
    code, s, z = orc.quantize_group(x, 4)
    assert s == 0.0 and z == np.float32(3.25) and (code == 0).all()
    # a group of signed zeros stores a +0 zero point
    x = np.full(G, -0.0, np.float32)
    code, s, z = orc.quantize_group(x, 2)
    assert s == 0.0 and (code == 0).all() and np.signbit(z) == False  # noqa: E712


def pin_quantize_brute_force():
    # every code is a nearest grid point of zero + scale * q, q in [0, qmax];
    # the extremes map to 0 and qmax; reconstruction error <= scale / 2.
    for bits in (2, 4):
        qmax = (1 << bits) - 1
        for seed in range(40):
            scale_in = [0.01, 1.0, 37.0, 1e-3][seed % 4]
            x = f32(rng_bits(1000 + seed, (G,), scale_in)) + np.float32(seed % 3)
            code, s, z = orc.quantize_group(x, bits)
            xd = x.astype(np.float64)
            assert z == x.min() or (z == 0 and x.min() == 0)
            assert abs(float(s) * qmax - (xd.max() - xd.min())) <= 4e-7 * (xd.max() - xd.min()) + 1e-30
            grid = float(z) + float(s) * np.arange(qmax + 1)
            err = np.abs(xd[:, None] - grid[None, :])
            best = err.min(axis=1)
            mine = err[np.arange(G), code.astype(int)]
            assert (mine <= best + 1e-6 * max(float(s), 1e-30)).all(), (bits, seed)
            assert (mine <= float(s) / 2 * (1 + 1e-6) + 1e-30).all()
            assert code[np.argmin(x)] == 0 and code[np.argmax(x)] == qmax


# ------------------------------------------------------- append / layout pins

def pin_pack_worked_example():
    # One 4-bit group, D = 64.  Key channel d (0..15) holds d at token 0, 0 at
    # token 1 and 15 at token 2, so its codes over the group are d, 0, 15.
    # Value token t holds channels 0..15 = 0..15 and channels 16..31 = 15.
    # Codes 0..15 on channels 0..15 pack to high word 0xFFAA5500 and low word
    # 0xE4E4E4E4 (code j in bits 2j..2j+1).
    D = 64
    k = np.zeros((G, D), np.float32)
    k[0, :16] = np.arange(16)
    k[2, :16] = 15.0
    v = np.zeros((G, D), np.float32)
    v[:, :16] = np.arange(16)
    v[:, 16:32] = 15.0
    u = orc.OracleUnit(orc.KIND_Q4, D, 64)
    u.append(bf16(k), bf16(v))
    out, valid = u.serialize()
    words = out.view(np.uint32)
    kblock = (64 // G) * 8 * D
    vblock = (64 // G) * G * (D // 4)
    # key planes: group 0, chunk 0, token 0, word 0
    assert words[0] == 0xFFAA5500, hex(words[0])
    assert words[kblock // 4] == 0xE4E4E4E4, hex(words[kblock // 4])
    # key meta: scale[D] then zero[D]; channel 3 spans [0, 15] -> scale 1
    meta = out[2 * kblock: 3 * kblock].view(np.float32)
    assert meta[3] == 1.0 and meta[D + 3] == 0.0
    # value planes: token 0 words 0 and 1
    vh = (3 * kblock) // 4
    vl = (3 * kblock + vblock) // 4
    assert words[vh] == 0xFFAA5500 and words[vh + 1] == 0xFFFFFFFF
    assert words[vl] == 0xE4E4E4E4 and words[vl + 1] == 0xFFFFFFFF
    # value meta: (scale, zero) pairs per 32 channels of token 0
    vm = out[3 * kblock + 2 * vblock: 3 * kblock + 2 * vblock + 16].view(np.float32)
    assert vm[0] == 1.0 and vm[1] == 0.0
    # one filled group: three key blocks and three value blocks of it
    assert valid.sum() == 3 * 8 * D + 3 * G * (D // 4)


def pin_axes():
    # Keys are quantized per channel over tokens and values per token over
    # channels: with every channel of token t equal to t, each key channel
    # spans [0, 31] (scale fl32(31/15)) while each value group is constant
    # (scale 0, zero = t).
    D = 64
    x = np.repeat(np.arange(G, dtype=np.float32)[:, None], D, axis=1)
    u = orc.OracleUnit(orc.KIND_Q4, D, 64)
    u.append(bf16(x), bf16(x))
    st = u.export()
    assert st["qtok"] == G
    assert (st["ks"] == np.float32(31.0) / np.float32(15.0)).all()
    assert (st["kz"] == 0).all()
    assert (st["vs"] == 0).all() and (st["vz"][:, 0] == np.arange(G)).all()
    assert (st["kq"][:, 0] == np.rint(np.arange(G) / (np.float32(31.0) / np.float32(15.0)))).all()


def pin_flush_and_bulk():
    # The residual flushes exactly when it holds 32 tokens, and appending one
    # token at a time gives the same bytes as one bulk append.
    D = 64
    k = rng_bits(7, (100, D))
    v = rng_bits(8, (100, D))
    a = orc.OracleUnit(orc.KIND_Q4, D, 128)
    for t in range(100):
        a.append(k[t:t + 1], v[t:t + 1])
        qtok = a.export()["qtok"]
        assert qtok == (t + 1) // G * G, (t, qtok)
    b = orc.OracleUnit(orc.KIND_Q4, D, 128)
    b.append(k[:45], v[:45])
    b.append(k[45:], v[45:])
    assert a.n == b.n == 100
    oa, va = a.serialize()
    ob, vb = b.serialize()
    assert (oa == ob).all() and (va == vb).all()
    # capacity is enforced
    c = orc.OracleUnit(orc.KIND_Q2, D, 64)
    c.append(k[:64], v[:64])
    try:
        c.append(k[:1], v[:1])
    except ValueError:
        pass
    else:
        raise AssertionError("capacity not enforced")


# ------------------------------------------------------------------ decode pins

def dequant_keys(st, res_k):
    """Keys of a quantized unit as the decode must see them (stored precision)."""
    qtok = st["qtok"]
    g = np.arange(qtok) // G
    kk = st["ks"][g].astype(np.float64) * st["kq"] + st["kz"][g].astype(np.float64)
    return np.concatenate([kk, f32(res_k).astype(np.float64)]) if len(res_k) else kk


def dequant_values(st, res_v, mode):
    """Values: mode 'full' (all code bits), 'hi' (high plane + 1.5), 'q2'."""
    qtok = st["qtok"]
    D = st["vq"].shape[1]
    s = np.repeat(st["vs"].astype(np.float64), G, axis=1)[:, :D]
    z = np.repeat(st["vz"].astype(np.float64), G, axis=1)[:, :D]
    c = st["vq"].astype(np.float64)
    if mode == "hi":
        c = 4.0 * (st["vq"] >> 2) + 1.5
    vv = s * c + z
    return np.concatenate([vv, f32(res_v).astype(np.float64)]) if len(res_v) else vv


def _unit(kind, D, n, seed, cap=None, kscale=1.0):
    k = rng_bits(seed, (n, D), kscale)
    v = rng_bits(seed + 1, (n, D))
    u = orc.OracleUnit(kind, D, cap or (n + 64))
    u.append(k, v)
    return u, k, v


def pin_bf16_is_textbook():
    D = 64
    for n in (1, 5, 50):
        u, k, v = _unit(orc.KIND_BF16, D, n, 20 + n)
        q = rng_bits(30 + n, (D,), 2.0)
        r = orc.decode(u, q, tau=0.01)
        ref = sdpa(f32(q), f32(k), f32(v), 1 / np.sqrt(D))
        assert np.abs(r.out - ref).max() < 1e-12, np.abs(r.out - ref).max()
        assert abs(r.weights.sum() - 1.0) < 1e-12
        assert r.nsel == 0 and len(r.mask) == 0


def pin_tau_zero_is_full_4bit():
    D = 64
    n = 70  # two groups and 6 residual tokens
    u, k, v = _unit(orc.KIND_Q4, D, n, 40)
    st = u.export()
    q = rng_bits(41, (D,), 2.0)
    r = orc.decode(u, q, tau=0.0)
    ref = sdpa(f32(q), dequant_keys(st, k[64:]), dequant_values(st, v[64:], "full"),
               1 / np.sqrt(D))
    assert np.abs(r.out - ref).max() < 1e-12
    assert r.nsel == 64 and list(r.mask) == [0xFFFFFFFF, 0xFFFFFFFF]


def pin_tau_above_one_is_high_plane():
    D = 64
    n = 70
    u, k, v = _unit(orc.KIND_Q4, D, n, 42)
    st = u.export()
    q = rng_bits(43, (D,), 2.0)
    r = orc.decode(u, q, tau=1.5)
    ref = sdpa(f32(q), dequant_keys(st, k[64:]), dequant_values(st, v[64:], "hi"),
               1 / np.sqrt(D))
    assert np.abs(r.out - ref).max() < 1e-12
    assert r.nsel == 0 and (r.mask == 0).all()


def pin_q2_is_plain_dequant():
    D = 128
    n = 96 + 31
    u, k, v = _unit(orc.KIND_Q2, D, n, 44)
    st = u.export()
    q = rng_bits(45, (D,), 2.0)
    r = orc.decode(u, q, tau=0.0)
    ref = sdpa(f32(q), dequant_keys(st, k[96:]), dequant_values(st, v[96:], "full"),
               1 / np.sqrt(D))
    assert np.abs(r.out - ref).max() < 1e-12
    assert r.nsel == 0


def pin_share_reads_final_loop():
    # A SHARE unit of length n attends over the source's positions [0, n-1)
    # as the source stores them, plus its own current token.
    D = 64
    for n_src, n_own in ((100, 90), (100, 101), (96, 97), (64, 40), (5, 3)):
        src, ks_, vs_ = _unit(orc.KIND_Q4, D, n_src, 50 + n_own)
        own = orc.OracleUnit(orc.KIND_SHARE, D, 0)
        kown = rng_bits(60 + n_own, (n_own, D))
        vown = rng_bits(61 + n_own, (n_own, D))
        own.append(kown, vown)
        assert own.n == n_own
        st = src.export()
        qtok = st["qtok"]
        kk = dequant_keys(st, ks_[qtok:])[: n_own - 1]
        vv = dequant_values(st, vs_[qtok:], "full")[: n_own - 1]
        keys = np.concatenate([kk, f32(kown[-1:]).astype(np.float64)])
        vals = np.concatenate([vv, f32(vown[-1:]).astype(np.float64)])
        q = rng_bits(70 + n_own, (D,), 2.0)
        r = orc.decode(own, q, tau=0.0, src=src)
        ref = sdpa(f32(q), keys, vals, 1 / np.sqrt(D))
        assert np.abs(r.out - ref).max() < 1e-12, (n_src, n_own)
        assert r.nsel == min(n_own - 1, qtok)
    # a SHARE unit cannot read past the source's length
    src, _, _ = _unit(orc.KIND_Q4, D, 10, 80)
    own = orc.OracleUnit(orc.KIND_SHARE, D, 0)
    own.append(rng_bits(81, (12, D)), rng_bits(82, (12, D)))
    try:
        orc.decode(own, rng_bits(83, (D,)), tau=0.0, src=src)
    except ValueError:
        pass
    else:
        raise AssertionError("SHARE past its source accepted")


def _mask_bits(words, n):
    """Selection per position [n] from mask words (bit j of word w = 32w + j)."""
    out = np.zeros(n, bool)
    for w, word in enumerate(np.asarray(words, np.uint64)):
        for j in range(32):
            if 32 * w + j < n and (int(word) >> j) & 1:
                out[32 * w + j] = True
    return out


def pin_group_query_heads():
    # Grouped-query decode: each head of the group has its own softmax and
    # output; the low planes fetched for the group are the ones any head
    # selects, and every head reconstructs those tokens at 4 bits.  So, head
    # by head: the weights and lse equal a one-query decode, the mask is the
    # union of the heads' own masks, and the output differs from the
    # one-query decode by exactly p * scale * (lo - 1.5) summed over the
    # tokens selected by other heads only.
    D = 64
    u, k, v = _unit(orc.KIND_Q4, D, 150, 90)
    kf = f32(k)
    q = np.stack([bf16(3.0 * kf[t]) for t in (10, 70, 100)])   # peaks on three tokens
    tau = 0.01
    r = orc.decode_group(u, q, tau)
    st = u.export()
    qtok = st["qtok"]
    lo = (st["vq"].astype(np.int64) & 3) - 1.5                     # [qtok][D]
    sc = np.repeat(st["vs"].astype(np.float64), G, axis=1)        # [qtok][D]
    grp = _mask_bits(r.mask, qtok)
    union = np.zeros_like(r.mask)
    nsel_heads = []
    for h in range(q.shape[0]):
        one = orc.decode(u, q[h], tau)
        assert np.array_equal(r.weights[h], one.weights) and r.lse[h] == one.lse
        union |= one.mask
        nsel_heads.append(one.nsel)
        extra = grp & ~_mask_bits(one.mask, qtok)
        delta = (r.weights[h][:qtok, None] * sc * lo * extra[:, None]).sum(0)
        assert np.abs(r.out[h] - one.out - delta).max() < 1e-12, h
    assert np.array_equal(r.mask, union)
    assert r.nsel == int(grp.sum()) and r.nsel > max(nsel_heads)
    # tau = 0 (every token) and tau > 1 (none) leave nothing to share
    for t in (0.0, 2.0):
        r2 = orc.decode_group(u, q, t)
        for h in range(q.shape[0]):
            assert np.array_equal(r2.out[h], orc.decode(u, q[h], t).out)
    # a group of one head is the one-query decode
    r1, o1 = orc.decode_group(u, q[:1], tau), orc.decode(u, q[0], tau)
    assert np.array_equal(r1.out[0], o1.out) and np.array_equal(r1.mask, o1.mask)
    assert r1.nsel == o1.nsel and np.array_equal(r1.weights[0], o1.weights)
    # SHARE units group the same way over the final loop's positions
    own = orc.OracleUnit(orc.KIND_SHARE, D, 0)
    own.append(rng_bits(95, (120, D)), rng_bits(96, (120, D)))
    rs = orc.decode_group(own, q, tau, src=u)
    for h in range(q.shape[0]):
        assert np.array_equal(rs.weights[h], orc.decode(own, q[h], tau, src=u).weights)


def pin_selection_override():
    # A position whose weight is within the band of tau takes the selection
    # the caller passes; with tau set to one position's own weight, turning
    # that position off moves each output channel by exactly
    # p * scale * (1.5 - lo) (its value falls back to the high-plane
    # midpoint), clears its mask bit and lowers the count by one.  Bits of
    # positions outside the band are ignored.
    D = 64
    u, k, v = _unit(orc.KIND_Q4, D, 150, 90)
    kf = f32(k)
    q = bf16(2.0 * kf[37])
    base = orc.decode(u, q, 0.5)
    t = int(np.argsort(base.weights[:128])[-3])       # a quantized position, not the peak
    tau = float(base.weights[t])
    r = orc.decode(u, q, tau)
    sel = _mask_bits(r.mask, 128)
    assert sel[t] and r.nsel == int(sel.sum())
    ov = r.mask.copy()
    ov[t // G] &= ~np.uint32(1 << (t % G))
    far = int(np.nonzero(sel & (np.abs(r.weights[:128] - tau) > 1e-6))[0][0])   # selected, outside the band
    ov[far // G] &= ~np.uint32(1 << (far % G))
    o = orc.decode(u, q, tau, sel_override=ov)
    st = u.export()
    lo = (st["vq"][t].astype(np.int64) & 3).astype(np.float64)
    sc = np.repeat(st["vs"][t].astype(np.float64), G)
    expect = r.out + r.weights[t] * sc * (1.5 - lo)
    assert np.abs(o.out - expect).max() < 1e-12
    assert o.nsel == r.nsel - 1 and np.array_equal(o.weights, r.weights)
    want = r.mask.copy()
    want[t // G] &= ~np.uint32(1 << (t % G))
    assert np.array_equal(o.mask, want)
    # the same through a group of one head, and no override changes nothing
    g = orc.decode_group(u, q[None], tau, sel_override=ov)
    assert np.array_equal(g.out[0], o.out) and np.array_equal(g.mask, o.mask)
    assert np.array_equal(orc.decode(u, q, tau, sel_override=r.mask).out, r.out)


def pin_planner_worked_example():
    # Two loops x two layers, D-quarter units.  Damage [Q4, Q2, SHARE] per
    # cell (loop-major): c0 [1,5,3], c1 [2,6,4], c2 [0,3,0], c3 [1,2,0] (the
    # final loop may not SHARE however cheap it looks).  Reads per cell: Q4
    # 5000, Q2 4000, SHARE = its layer's final cell's; storage Q4 6, Q2 4,
    # SHARE 0.
    dm = np.array([[1, 5, 3], [2, 6, 4], [0, 3, 0], [1, 2, 0]])
    # unlimited: final cells 2-bit (4000 each), c0 and c1 SHARE them (4000
    # each, damage 3 and 4 < their own 2-bit 5 and 6): reads 16000, damage
    # 3 + 4 + 3 + 2 = 12, storage 8
    k, r, d, s = orc.plan_brute(2, 2, dm, 100, 100, 0)
    assert list(k) == [2, 2, 1, 1] and (r, d, s) == (16000, 12, 8)
    # damage budget 4: only all-4-bit fits (damage 1 + 2 + 0 + 1)
    k, r, d, s = orc.plan_brute(2, 2, dm, 4, 100, 0)
    assert list(k) == [0, 0, 0, 0] and (r, d, s) == (20000, 4, 24)
    # a selected fraction of 0.25 adds 250 per 4-bit cell, also to a SHARE
    # cell whose final cell is 4-bit
    k, r, d, s = orc.plan_brute(2, 2, dm, 4, 100, 250)
    assert r == 4 * 5250
    # damage budget 9, storage 14: both layers at 8000 reads (final 2-bit +
    # SHARE) cost damage 12; layer 1 can keep that (damage 2 + 4 = 6) if
    # layer 0 stays within 3: its final cell 4-bit + c0 SHARE (0 + 3, reads
    # 10000, storage 6).  The alternative (layer 0 at 8000, layer 1 all
    # 4-bit, damage 6 + 3) needs storage 4 + 12 = 16.  So reads 18000,
    # damage 9, storage 10.
    k, r, d, s = orc.plan_brute(2, 2, dm, 9, 14, 0)
    assert list(k) == [2, 2, 0, 1] and (r, d, s) == (18000, 9, 10)
    # nothing has zero damage in c0
    assert orc.plan_brute(2, 2, dm, 0, 100, 0) is None
    # equal reads are settled by damage before storage: with c1's SHARE at
    # damage 9, c1 keeps its own 2-bit (6) although SHARE would store nothing
    dm2 = dm.copy()
    dm2[1, 2] = 9
    k, r, d, s = orc.plan_brute(2, 2, dm2, 100, 100, 0)
    assert list(k) == [2, 1, 1, 1] and (r, d, s) == (16000, 3 + 6 + 3 + 2, 12)


def pin_high_plane_worked_example():
    # 32 tokens with equal keys (key scale 0, so every weight is 1/32).  Each
    # value token is 0 on channel 0, 15 on channel 1, 13 on channel 2 and 0
    # elsewhere in its first 32 channels: scale 1, zero 0, channel 2 code 13 =
    # (hi 3, lo 1).  Full precision gives 13; high plane only gives 13.5.
    # Channel 1 (code 15 = hi 3, lo 3) reads 13.5 from the high plane alone,
    # channel 0 (code 0) reads 1.5.
    D = 64
    k = np.full((G, D), 0.5, np.float32)
    v = np.zeros((G, D), np.float32)
    v[:, 1], v[:, 2] = 15.0, 13.0
    u = orc.OracleUnit(orc.KIND_Q4, D, 64)
    u.append(bf16(k), bf16(v))
    q = bf16(np.ones(D, np.float32))
    hi_only = orc.decode(u, q, tau=0.5)
    full = orc.decode(u, q, tau=0.01)
    assert abs(hi_only.out[2] - 13.5) < 1e-12 and abs(full.out[2] - 13.0) < 1e-12
    assert abs(hi_only.out[1] - 13.5) < 1e-12 and abs(hi_only.out[0] - 1.5) < 1e-12
    assert abs(full.out[1] - 15.0) < 1e-12 and abs(full.out[0]) < 1e-12
    assert hi_only.nsel == 0 and full.nsel == G
    # equal scores: lse = s + log(32) with s = sum(q * 0.5) / sqrt(D)
    s = 0.5 * D / np.sqrt(D)
    assert abs(full.lse - (s + np.log(G))) < 1e-12
    assert np.allclose(full.weights, 1.0 / G, atol=1e-15)


def pin_mask_properties():
    # N_sel <= floor(1/tau); the selected set shrinks as tau grows; a token is
    # selected exactly when its weight reaches tau (ties included).
    D = 128
    n = 32 * 20 + 7
    u, _, _ = _unit(orc.KIND_Q4, D, n, 90, kscale=3.0)
    q = rng_bits(91, (D,), 3.0)
    prev = None
    for tau in (0.0005, 0.001, 0.002, 0.005, 0.01, 0.05, 0.2):
        r = orc.decode(u, q, tau=tau)
        assert r.nsel <= int(np.floor(1.0 / tau) + 1e-9)
        assert abs(r.weights.sum() - 1.0) < 1e-12
        bits = np.unpackbits(r.mask.view(np.uint8), bitorder="little")[: n // G * G]
        assert bits.sum() == r.nsel
        if prev is not None:
            assert ((bits & ~prev) == 0).all()
        prev = bits
    r = orc.decode(u, q, tau=0.0)
    w = r.weights[5]
    r2 = orc.decode(u, q, tau=float(w))
    assert (r2.mask[0] >> 5) & 1 == 1


# --------------------------------------------------------- residual (RES2) pins
# "ResidualQuant: KV Cache Quantization for Looped Transformers with 2-Bit
# Residuals", as summarised in the related-paper list (関連論文リスト) of the
# page "LoopVQ: Sub 1-bit KV Cache Quantization for Looped Transformers": the
# final loop's KV is the reference and the other loops store 2-bit
# residuals against it.

def pin_residual_deferred_window():
    # A residual group is quantized once the 32 tokens after it are in, so
    # the bf16 window keeps 32..63 tokens (all of them below 32):
    # qtok(n) = 32 * max(0, floor(n / 32) - 1).
    D = 64
    ref, _, _ = _unit(orc.KIND_BF16, D, 200, 300)
    k = rng_bits(301, (200, D))
    v = rng_bits(302, (200, D))
    a = orc.OracleUnit(orc.KIND_RES2, D, 256)
    for t in range(200):
        a.append(k[t:t + 1], v[t:t + 1])
        n = t + 1
        assert a.export(src=ref)["qtok"] == max(0, n // G - 1) * G, n
    b = orc.OracleUnit(orc.KIND_RES2, D, 256)
    b.append(k[:77], v[:77])
    b.append(k[77:], v[77:])
    oa, va = a.serialize(src=ref)
    ob, vb = b.serialize(src=ref)
    assert (oa == ob).all() and (va == vb).all()


def pin_residual_worked_example():
    # bf16 reference r = 1 everywhere; the cell's token t < 32 is r + (t mod 4)
    # on every channel, so every residual is t mod 4: key channels span [0, 3]
    # over a group (scale 1, zero 0, codes t mod 4), each value group of
    # token t is constant (scale 0, zero t mod 4, codes 0).  Layout as a
    # 2-bit cell plus a 64-slot bf16 window (position t in slot t mod 64).
    D = 64
    n = 70
    ones = np.ones((n, D), np.float32)
    ref = orc.OracleUnit(orc.KIND_BF16, D, 128)
    ref.append(bf16(ones), bf16(ones))
    x = 1.0 + (np.arange(n) % 4)[:, None] * np.ones((1, D), np.float32)
    x[32:] = np.arange(32, n)[:, None]  # window tokens: distinct rows
    u = orc.OracleUnit(orc.KIND_RES2, D, 128)
    u.append(bf16(x), bf16(x))
    st = u.export(src=ref)
    assert st["qtok"] == 32
    assert (st["ks"] == 1.0).all() and (st["kz"] == 0.0).all()
    assert (st["kq"] == (np.arange(32) % 4)[:, None]).all()
    assert (st["vs"] == 0.0).all() and (st["vq"] == 0).all()
    assert (st["vz"][:, 0] == np.arange(32) % 4).all()
    out, valid = u.serialize(src=ref)
    words = out.view(np.uint32)
    kblock = (128 // G) * 8 * D
    vblock = (128 // G) * G * (D // 4)
    # key plane, group 0, chunk 0: token t's word 0 is (t mod 4) * 0x55555555
    for t in range(4):
        assert words[t * 4] == (t % 4) * 0x55555555, (t, hex(words[t * 4]))
    # window: K rows after k_hi, k_meta, v_hi, v_meta; position 64 -> slot 0,
    # position 33 -> slot 33
    res_k = 2 * kblock + 2 * vblock
    row = out[res_k: res_k + 2 * D].view(np.uint16)
    assert (row == bf16(x[64])).all()
    row = out[res_k + 33 * 2 * D: res_k + 34 * 2 * D].view(np.uint16)
    assert (row == bf16(x[33])).all()
    # defined bytes: one group of K (plane + meta), 32 V rows (plane + meta),
    # 38 window tokens of K and V
    assert valid.sum() == 2 * 8 * D + 2 * G * (D // 4) + 2 * 38 * 2 * D
    # the zero residual of an identical cell reads back the reference exactly
    same = orc.OracleUnit(orc.KIND_RES2, D, 128)
    same.append(bf16(ones), bf16(ones))
    z = same.export(src=ref)
    assert (z["ks"] == 0).all() and (z["kz"] == 0).all() and (z["vz"] == 0).all()


def pin_residual_reference_rounding():
    # r, the reference's stored value in fp32, is fl(fl(scale * code) + zero):
    # the two roundings of a 4-bit dequantization.  Worked case: a reference
    # key channel spanning [-2.71875, 2.953125] (both exact in bf16) has scale
    # fl32(5.671875 / 15) = 0.378125012; its top code 15 gives
    # fl(15 * 0.378125012) = 5.671875 (the product 5.67187518 lies 1.8e-7
    # from it), and 5.671875 - 2.71875 = 2.953125 exactly, where one rounding
    # of the exact 2.95312518 would give 2.95312524.  A residual cell whose
    # keys are 0 on that channel stores d = -r, so its residual group's zero
    # point (the group minimum) is -2.953125.
    D = 64
    n = 64   # the residual group 0 is quantized once the cell holds 64 tokens
    zeros = np.zeros((n, D), np.float32)
    kr = zeros.copy()
    kr[0, 0], kr[1, 0] = -2.71875, 2.953125
    ref = orc.OracleUnit(orc.KIND_Q4, D, 128)
    ref.append(bf16(kr), bf16(zeros))
    st_ref = ref.export()
    assert st_ref["ks"][0, 0] == np.float32(5.671875) / np.float32(15.0)
    assert st_ref["kz"][0, 0] == np.float32(-2.71875) and st_ref["kq"][1, 0] == 15
    u = orc.OracleUnit(orc.KIND_RES2, D, 128)
    u.append(bf16(zeros), bf16(zeros))
    st = u.export(src=ref)
    assert st["qtok"] == 32
    assert st["kz"][0, 0] == np.float32(-2.953125), repr(st["kz"][0, 0])


def _ref32(st, pos, keys):
    """The reference's stored value in fp32: fl(fl(scale * code) + zero)."""
    g = pos // G
    if keys:
        return (st["ks"][g] * st["kq"][pos].astype(np.float32)) + st["kz"][g]
    s = np.repeat(st["vs"][pos], G)
    z = np.repeat(st["vz"][pos], G)
    return (s * st["vq"][pos].astype(np.float32)) + z


def pin_residual_reconstructs():
    # Against a 4-bit reference: (a) every quantized position reconstructs
    # its own input within half a residual step, (b) decode is textbook
    # attention over r^ + d^ (reference keys at stored precision, reference
    # values through the tau rule) and the cell's own bf16 window tokens.
    D = 64
    n = 3 * G + 13
    ref, _, _ = _unit(orc.KIND_Q4, D, n + 5, 310)
    k = rng_bits(311, (n, D), 1.0)
    v = rng_bits(312, (n, D))
    u = orc.OracleUnit(orc.KIND_RES2, D, 160)
    u.append(k, v)
    rs = ref.export()
    st = u.export(src=ref)
    qtok = st["qtok"]
    assert qtok == 2 * G
    kx = f32(k).astype(np.float32)
    vx = f32(v).astype(np.float32)
    for pos in range(qtok):
        g = pos // G
        kr = _ref32(rs, pos, True).astype(np.float64)
        kh = kr + st["ks"][g].astype(np.float64) * st["kq"][pos] + st["kz"][g]
        assert (np.abs(kx[pos] - kh) <= st["ks"][g] * 0.5000005 + 1e-6).all(), pos
        vr = _ref32(rs, pos, False).astype(np.float64)
        vs = np.repeat(st["vs"][pos], G).astype(np.float64)
        vh = vr + vs * st["vq"][pos] + np.repeat(st["vz"][pos], G)
        assert (np.abs(vx[pos] - vh) <= vs * 0.5000005 + 1e-6).all(), pos
    gi = np.arange(qtok) // G
    kref = rs["ks"][gi].astype(np.float64) * rs["kq"][:qtok] + rs["kz"][gi]
    kres = st["ks"][gi].astype(np.float64) * st["kq"] + st["kz"][gi]
    keys = np.concatenate([kref + kres, kx[qtok:].astype(np.float64)])
    vs = np.repeat(st["vs"].astype(np.float64), G, axis=1)
    vres = vs * st["vq"] + np.repeat(st["vz"].astype(np.float64), G, axis=1)
    rvs = np.repeat(rs["vs"][:qtok].astype(np.float64), G, axis=1)
    rvz = np.repeat(rs["vz"][:qtok].astype(np.float64), G, axis=1)
    q = rng_bits(313, (D,), 2.0)
    for tau, mode in ((0.0, "full"), (1.5, "hi")):
        c = rs["vq"][:qtok].astype(np.float64)
        if mode == "hi":
            c = 4.0 * (rs["vq"][:qtok] >> 2) + 1.5
        vals = np.concatenate([rvs * c + rvz + vres, vx[qtok:].astype(np.float64)])
        r = orc.decode(u, q, tau=tau, src=ref)
        want = sdpa(f32(q), keys, vals, 1 / np.sqrt(D))
        assert np.abs(r.out - want).max() < 1e-12, (tau, np.abs(r.out - want).max())
        assert r.nsel == (qtok if tau == 0.0 else 0)


def pin_residual_reference_checks():
    # No reference, a reference that does not yet hold the quantized
    # positions, and a SHARE reference are all rejected.
    D = 64
    u = orc.OracleUnit(orc.KIND_RES2, D, 128)
    u.append(rng_bits(320, (70, D)), rng_bits(321, (70, D)))
    q = rng_bits(322, (D,))
    short, _, _ = _unit(orc.KIND_Q4, D, 40, 323)   # holds one group; u needs 32 quantized
    ok, _, _ = _unit(orc.KIND_Q4, D, 64, 324)
    sh = orc.OracleUnit(orc.KIND_SHARE, D, 0)
    sh.append(rng_bits(325, (3, D)), rng_bits(326, (3, D)))
    orc.decode(u, q, tau=0.01, src=ok)
    orc.decode(u, q, tau=0.01, src=short)   # 32 quantized reference positions suffice
    tiny, _, _ = _unit(orc.KIND_Q4, D, 31, 327)
    for bad in (None, tiny, sh):
        try:
            orc.decode(u, q, tau=0.01, src=bad)
        except ValueError:
            continue
        raise AssertionError("residual unit accepted a bad reference")


# ------------------------------------------------------------ LoopVQ pins
# "LoopVQ: Sub 1-bit KV Cache Quantization for Looped Transformers", section
# 概要: channels of several loop steps are coded jointly by a codebook.

def _vq_exact(D, L, c, n, seed):
    """A codebook that holds every (token, group) sub-vector of raw per-loop
    keys and values exactly, and the indices that pick them."""
    groups = D // c
    assert n * groups == 256
    K = f32(rng_bits(seed, (L, n, D)))
    V = f32(rng_bits(seed + 1, (L, n, D)))
    perm = np.argsort(f32(rng_bits(seed + 2, (256,))), kind="stable")  # a shuffle of the entries
    cb_k = np.zeros((256, L * c), np.float32)
    cb_v = np.zeros((256, L * c), np.float32)
    idx_k = np.zeros((n, groups), np.uint8)
    idx_v = np.zeros((n, groups), np.uint8)
    for t in range(n):
        for j in range(groups):
            e, ev = t * groups + j, int(perm[t * groups + j])
            idx_k[t, j], idx_v[t, j] = e, ev
            for l in range(L):
                cb_k[e, l * c:(l + 1) * c] = K[l, t, j * c:(j + 1) * c]
                cb_v[ev, l * c:(l + 1) * c] = V[l, t, j * c:(j + 1) * c]
    return K, V, cb_k, cb_v, idx_k, idx_v


def pin_vq_exact_codebook():
    # With a codebook that holds each sub-vector exactly, decoding loop l is
    # textbook attention over loop l's raw keys and values (every loop, two
    # head dims, values indexed through a shuffled codebook).
    for D, L, c, n in ((64, 4, 4, 16), (128, 2, 8, 16)):
        K, V, cb_k, cb_v, idx_k, idx_v = _vq_exact(D, L, c, n, 400 + D)
        q = rng_bits(401 + D, (D,), 2.0)
        for loop in range(L):
            out, lse = orc.vq_decode(idx_k, idx_v, cb_k, cb_v, q, loop, L)
            want = sdpa(f32(q), K[loop].astype(np.float64), V[loop].astype(np.float64),
                        1 / np.sqrt(D))
            assert np.abs(out - want).max() < 1e-12, (D, loop, np.abs(out - want).max())


def pin_vq_uniform_keys():
    # Every key entry reads the same vector at loop 2: all scores equal, so
    # lse = s + ln n and the output is the plain mean of the value slices.
    D, L, c, n = 64, 4, 4, 40
    rng = np.random.default_rng(5)
    cb_k = rng.standard_normal((256, L * c)).astype(np.float32)
    kvec = rng.standard_normal(c).astype(np.float32)
    cb_k[:, 2 * c:3 * c] = kvec
    cb_v = rng.standard_normal((256, L * c)).astype(np.float32)
    idx_k = rng.integers(0, 256, (n, D // c)).astype(np.uint8)
    idx_v = rng.integers(0, 256, (n, D // c)).astype(np.uint8)
    q = rng_bits(410, (D,), 1.0)
    out, lse = orc.vq_decode(idx_k, idx_v, cb_k, cb_v, q, 2, L)
    s = float(np.dot(f32(q).astype(np.float64), np.tile(kvec.astype(np.float64), D // c))) / np.sqrt(D)
    assert abs(lse - (s + np.log(n))) < 1e-12
    vals = cb_v[idx_v][:, :, 2 * c:3 * c].reshape(n, D).astype(np.float64)
    assert np.abs(out - vals.mean(axis=0)).max() < 1e-12


def pin_vq_encode_nearest():
    # (a) a codebook holding every sub-vector exactly gives back their indices
    # (distance 0); (b) on random data the chosen entry's distance, in fp64,
    # is the brute-force minimum up to fp32 rounding; (c) equal entries: the
    # lowest index wins.
    D, L, c, n = 64, 4, 4, 16
    K, V, cb_k, cb_v, idx_k, idx_v = _vq_exact(D, L, c, n, 420)
    for t in range(n):
        x = bf16(K[:, t, :])
        assert (orc.vq_encode(x, cb_k) == idx_k[t]).all(), t
    rng = np.random.default_rng(11)
    cb = rng.standard_normal((256, L * c)).astype(np.float32)
    for t in range(8):
        x = rng_bits(430 + t, (L, 128))
        idx = orc.vq_encode(x, cb)
        xf = f32(x).astype(np.float64)
        for j in range(32):
            sub = xf[:, 4 * j:4 * j + 4].reshape(-1)
            dist = ((cb.astype(np.float64) - sub[None, :]) ** 2).sum(axis=1)
            assert dist[idx[j]] <= dist.min() * (1 + 1e-5) + 1e-9, (t, j)
    x = rng_bits(440, (L, 64))
    first = int(orc.vq_encode(x, cb)[0])
    assert 0 < first < 255, first      # (this seed's pick leaves room on both sides)
    cb2 = cb.copy()
    cb2[255] = cb2[first]              # a later duplicate of the chosen entry
    assert orc.vq_encode(x, cb2)[0] == first
    cb3 = cb.copy()
    cb3[0] = cb3[first]                # an earlier duplicate wins
    assert orc.vq_encode(x, cb3)[0] == 0


ALL_PINS = [
    pin_quantize_q2_ties,
    pin_quantize_q4_ties,
    pin_quantize_fp32_scale,
    pin_quantize_division_is_correctly_rounded,
    pin_quantize_degenerate,
    pin_quantize_brute_force,
    pin_pack_worked_example,
    pin_axes,
    pin_flush_and_bulk,
    pin_bf16_is_textbook,
    pin_tau_zero_is_full_4bit,
    pin_tau_above_one_is_high_plane,
    pin_q2_is_plain_dequant,
    pin_share_reads_final_loop,
    pin_high_plane_worked_example,
    pin_mask_properties,
    pin_group_query_heads,
    pin_selection_override,
    pin_planner_worked_example,
    pin_residual_deferred_window,
    pin_residual_worked_example,
    pin_residual_reference_rounding,
    pin_residual_reconstructs,
    pin_residual_reference_checks,
    pin_vq_exact_codebook,
    pin_vq_uniform_keys,
    pin_vq_encode_nearest,
]
