"""Seeded synthetic workloads for the LoopKV decode path (host side).

A workload fixes the cell grid (loops x layers), heads, head dim, batch,
per-sequence lengths, the per-cell storage plan and tau, and the recipe of
every raw key, value and query.  Every value is a pure function of
(seed, stream, counters) through Philox4x32-10 (``philox.py``), so the GPU
twin in ``csrc/synth.cu`` produces the same bits and either side can
regenerate any slice.  No LoopKV arithmetic lives here.

Cells are indexed loop-major: cell = loop * n_layers + layer.  The final loop
is loop n_loops - 1; a SHARE cell at (loop, layer) reuses cell
(n_loops - 1, layer).

Recipes (the shapes follow a 1.4B-parameter looped model at 4K-16K context):
  keys    "lognormal": N(0,1) times a per-(cell, head, channel) factor
          exp(N(0,1)); "outlier": N(0,1), with 4 channels per (cell, head)
          scaled by 10.
  values  N(0,1).
  Cells stored as 2-bit residuals against the final loop (RES2) follow their
  reference: each raw key is the reference cell's raw key plus 0.25 * N(0,1)
  times the cell's own channel factor, each raw value the reference's value
  plus 0.25 * N(0,1) (the loops of a looped model keep close KV states).
  queries "sum3": the sum of the raw keys at 3 distinct random attended
          positions plus 0.5 * N(0,1); "peaked": 2 * the raw key at one random
          attended position plus N(0,1).  Attended positions of a SHARE unit
          of length n are the final loop's positions [0, n-1) and its own
          position n-1.
N(0,1) is the Irwin-Hall stand-in of ``philox.normal_from_bits``.  Sums and
products are fp32 round-to-nearest, then rounded once to bf16.
"""

import dataclasses

import numpy as np

from . import philox as px

Q4, Q2, SHARE, BF16, RES2 = 0, 1, 2, 3, 4
KIND_NAMES = {Q4: "Q4", Q2: "Q2", SHARE: "SHARE", BF16: "BF16", RES2: "RES2"}

# Philox key word 1 selects the stream; key word 0 is the workload seed.
STREAM_K, STREAM_V, STREAM_QNOISE, STREAM_QPOS = 1, 2, 3, 4
STREAM_CHSCALE, STREAM_PLAN, STREAM_LEN, STREAM_OUTLIER = 5, 6, 7, 8
STREAM_VQ_IDX, STREAM_VQ_CB, STREAM_VQ_Q = 9, 10, 11


@dataclasses.dataclass
class Workload:
    name: str
    n_loops: int
    n_layers: int
    n_heads: int
    head_dim: int
    batch: int
    seed: int
    kinds: np.ndarray        # uint8 [cells], loop-major
    tau: float
    lengths: np.ndarray      # int32 [batch]: tokens cached per cell after the build
    capacity: np.ndarray     # int32 [batch]
    key_dist: str            # "lognormal" | "outlier"
    query_mode: str          # "sum3" | "peaked"
    chscale: np.ndarray      # float32 [cells, heads, head_dim]
    description: str = ""

    @property
    def n_cells(self):
        return self.n_loops * self.n_layers

    def source_cell(self, cell):
        """Cell whose KV a SHARE cell reuses: the final loop, same layer."""
        return (self.n_loops - 1) * self.n_layers + cell % self.n_layers

    def data_cell(self, cell):
        return self.source_cell(cell) if self.kinds[cell] == SHARE else cell

    def token_ref(self, cell):
        """Cell whose raw tokens a residual cell's tokens follow, else -1."""
        return self.source_cell(cell) if self.kinds[cell] == RES2 else -1

    def cells_of_loop(self, loop):
        return list(range(loop * self.n_layers, (loop + 1) * self.n_layers))


# ---------------------------------------------------------------- raw streams

def _unit_word(wl, b, h):
    return np.uint32(h + wl.n_heads * b)


def raw_keys(wl, cell, b, h, t0, t1):
    """bf16 bits [t1-t0, D] of the raw keys of (cell, b, h) at positions t0..t1-1."""
    D = wl.head_dim
    t = np.arange(t0, t1, dtype=np.uint32)[:, None]
    d = np.arange(D, dtype=np.uint32)[None, :]
    u = px.philox4x32(t, d, _unit_word(wl, b, h), np.uint32(cell), wl.seed, STREAM_K)
    z = px.normal_from_bits(*u)
    ref = wl.token_ref(cell)
    if ref >= 0:
        kr = px.bf16_bits_to_float(raw_keys(wl, ref, b, h, t0, t1))
        noise = ((z * np.float32(0.25)).astype(np.float32) * wl.chscale[cell, h][None, :])
        return px.float_to_bf16_bits((kr + noise.astype(np.float32)).astype(np.float32))
    x = (z * wl.chscale[cell, h][None, :]).astype(np.float32)
    return px.float_to_bf16_bits(x)


def raw_values(wl, cell, b, h, t0, t1):
    """bf16 bits [t1-t0, D] of the raw values of (cell, b, h)."""
    D = wl.head_dim
    t = np.arange(t0, t1, dtype=np.uint32)[:, None]
    d = np.arange(D, dtype=np.uint32)[None, :]
    u = px.philox4x32(t, d, _unit_word(wl, b, h), np.uint32(cell), wl.seed, STREAM_V)
    z = px.normal_from_bits(*u)
    ref = wl.token_ref(cell)
    if ref >= 0:
        vr = px.bf16_bits_to_float(raw_values(wl, ref, b, h, t0, t1))
        return px.float_to_bf16_bits((vr + (z * np.float32(0.25)).astype(np.float32)).astype(np.float32))
    return px.float_to_bf16_bits(z)


def query_positions(wl, cell, b, h, n, rep=0):
    """Attended positions the query of a unit of length n is built from.

    rep: query head of the KV head's group (0 for one query per KV head)."""
    u = px.philox4x32(np.uint32(n), np.uint32(rep << 16), _unit_word(wl, b, h), np.uint32(cell),
                      wl.seed, STREAM_QPOS)
    u = [int(x) for x in u]
    want = 3 if wl.query_mode == "sum3" else 1
    k = min(want, n)
    picks = []
    for i in range(k):
        r = int(px.uniform_index(np.uint32(u[i]), n - i))
        for p in sorted(picks):  # skip the positions already taken
            if r >= p:
                r += 1
        picks.append(r)
    return picks


def query(wl, cell, b, h, n, rep=0):
    """bf16 bits [D] of the query of unit (cell, b, h) when it holds n tokens.

    rep: query head of the KV head's group; rep 0 is the one-query stream."""
    D = wl.head_dim
    share = wl.kinds[cell] == SHARE
    keys = []
    for p in query_positions(wl, cell, b, h, n, rep):
        src = wl.source_cell(cell) if (share and p < n - 1) else cell
        keys.append(px.bf16_bits_to_float(raw_keys(wl, src, b, h, p, p + 1)[0]))
    d = np.arange(D, dtype=np.uint32) + np.uint32(rep << 16)
    u = px.philox4x32(np.uint32(n), d, _unit_word(wl, b, h), np.uint32(cell), wl.seed,
                      STREAM_QNOISE)
    z = px.normal_from_bits(*u)
    if wl.query_mode == "sum3":
        acc = np.zeros(D, np.float32)
        for kv in keys:
            acc = (acc + kv).astype(np.float32)
        x = (acc + (np.float32(0.5) * z).astype(np.float32)).astype(np.float32)
    else:
        x = ((np.float32(2.0) * keys[0]).astype(np.float32) + z).astype(np.float32)
    return px.float_to_bf16_bits(x)


def query_group(wl, cell, b, h, n, g):
    """bf16 bits [g][D]: the queries of the g query heads sharing KV head h."""
    return np.stack([query(wl, cell, b, h, n, rep=r) for r in range(g)])


# ------------------------------------------------------------------ tables

def _permutation(seed, n, purpose):
    u = px.philox4x32(np.arange(n, dtype=np.uint32), np.uint32(purpose), 0, 0, seed,
                      STREAM_PLAN)[0]
    return np.argsort(u.astype(np.int64) * 4096 + np.arange(n), kind="stable")


def percent_plan(seed, n_loops, n_layers, pct_q4, pct_share, final_all_q4=False):
    """Seeded plan with round(pct * cells) Q4 and SHARE cells, the rest Q2.

    SHARE cells are drawn from the non-final loops only.  With final_all_q4
    the final loop is all Q4 and the percentages apply to the other loops.
    """
    cells = n_loops * n_layers
    kinds = np.full(cells, Q2, np.uint8)
    nonfinal = np.arange((n_loops - 1) * n_layers)
    if final_all_q4:
        kinds[(n_loops - 1) * n_layers:] = Q4
        pool = nonfinal
        n_share = int(round(pct_share * len(pool)))
        n_q4 = int(round(pct_q4 * len(pool)))
        perm = pool[_permutation(seed, len(pool), 1)]
        kinds[perm[:n_share]] = SHARE
        kinds[perm[n_share:n_share + n_q4]] = Q4
        return kinds
    n_share = int(round(pct_share * cells))
    n_q4 = int(round(pct_q4 * cells))
    perm = nonfinal[_permutation(seed, len(nonfinal), 1)]
    kinds[perm[:n_share]] = SHARE
    rest = np.array([c for c in range(cells) if kinds[c] != SHARE])
    rest = rest[_permutation(seed, len(rest), 2)]
    kinds[rest[:n_q4]] = Q4
    return kinds


def lognormal_chscale(seed, cells, H, D):
    d = np.arange(D, dtype=np.uint32)[None, None, :]
    h = np.arange(H, dtype=np.uint32)[None, :, None]
    c = np.arange(cells, dtype=np.uint32)[:, None, None]
    z = px.normal_from_bits(*px.philox4x32(d, h, c, 0, seed, STREAM_CHSCALE))
    return np.exp(z.astype(np.float64)).astype(np.float32)


def outlier_chscale(seed, cells, H, D, n_out=4, factor=10.0):
    out = np.ones((cells, H, D), np.float32)
    d = np.arange(D, dtype=np.uint32)
    for c in range(cells):
        for h in range(H):
            u = px.philox4x32(d, np.uint32(h), np.uint32(c), 0, seed, STREAM_OUTLIER)[0]
            idx = np.argsort(u.astype(np.int64) * 256 + d, kind="stable")[:n_out]
            out[c, h, idx] = factor
    return out


def round_up(x, m):
    return (np.asarray(x) + m - 1) // m * m


# --------------------------------------------------------------- the configs

def make(config, **over):
    """Workload for config 0, 1, 2, "2r", "3a".."3d" or 4; keyword args override fields."""
    config = str(config)
    if config == "0":
        # plan given as [[Q4, Q2], [SHARE, Q4]] indexed [layer][loop]
        kinds = np.array([Q4, SHARE, Q2, Q4], np.uint8)  # loop-major
        wl = Workload("tiny", 2, 2, 2, 64, 1, 0, kinds, 0.01,
                      np.array([256], np.int32), np.array([256 + 64], np.int32),
                      "lognormal", "sum3", lognormal_chscale(0, 4, 2, 64),
                      "2 loops x 2 layers, batch 1, 2 heads, D 64, 256 tokens")
    elif config == "1":
        kinds = percent_plan(1, 4, 24, 0.5, 0.2)
        wl = Workload("single-4k", 4, 24, 16, 128, 1, 1, kinds, 0.005,
                      np.array([4096 + 17], np.int32), round_up([4096 + 17 + 64], 32).astype(np.int32),
                      "lognormal", "sum3", lognormal_chscale(1, 96, 16, 128),
                      "4x24 cells, 16 heads, D 128, batch 1, 4096 + 17 tokens")
    elif config in ("2", "2r") or config.startswith("3"):
        kinds = percent_plan(2, 4, 24, 0.35, 0.30, final_all_q4=True)
        tau = 0.002
        name = "batched-16k"
        if config == "2r":
            # the SHARE cells of the plan stored as 2-bit residuals instead
            kinds = np.where(kinds == SHARE, RES2, kinds).astype(np.uint8)
            name = "batched-16k-residual"
        if config.startswith("3"):
            sub = config[1:]
            if sub == "a":
                kinds, tau = np.full(96, Q4, np.uint8), 0.0
            elif sub == "b":
                kinds = np.full(96, Q4, np.uint8)
            elif sub == "c":
                kinds = np.full(96, Q2, np.uint8)
            elif sub == "d":
                kinds = np.full(96, BF16, np.uint8)
            else:
                raise ValueError(config)
            name = "ablation-" + sub
        wl = Workload(name, 4, 24, 16, 128, 32, 2, kinds, tau,
                      np.full(32, 16384, np.int32), np.full(32, 16384 + 64, np.int32),
                      "outlier", "peaked", outlier_chscale(2, 96, 16, 128),
                      "4x24 cells, 16 heads, D 128, batch 32, 16384 tokens")
    elif config == "4":
        B = 64
        u = px.philox4x32(np.arange(B, dtype=np.uint32), 0, 0, 0, 4, STREAM_LEN)
        ctx = 1024 + px.uniform_index(u[0], 16384 - 1024 + 1)
        res = px.uniform_index(u[1], 32)
        lengths = (ctx // 32 * 32 + res).astype(np.int32)
        kinds = percent_plan(4, 4, 32, 0.40, 0.25)
        wl = Workload("ragged-append", 4, 32, 32, 128, B, 4, kinds, 0.003, lengths,
                      round_up(lengths + 64, 32).astype(np.int32),
                      "lognormal", "sum3", lognormal_chscale(4, 128, 32, 128),
                      "4x32 cells, 32 heads, D 128, batch 64, ragged 1K-16K")
    else:
        raise ValueError("unknown config %r" % config)
    for k, v in over.items():
        setattr(wl, k, v)
    return wl


def unit_length(wl, cell, b):
    """Tokens a unit of this cell holds after the build (all cells alike)."""
    return int(wl.lengths[b])


def custom(n_loops, n_layers, n_heads, head_dim, kinds, lengths, capacity, tau, seed=9,
           key_dist="lognormal", query_mode="sum3"):
    """A small workload with an explicit plan and lengths (edge-case tests).

    All arguments are plain values or tuples so the spec can be hashed and
    sent to worker processes.
    """
    cells = n_loops * n_layers
    if key_dist == "lognormal":
        ch = lognormal_chscale(seed, cells, n_heads, head_dim)
    else:
        ch = outlier_chscale(seed, cells, n_heads, head_dim)
    return Workload("custom", n_loops, n_layers, n_heads, head_dim, len(lengths), seed,
                    np.array(kinds, np.uint8), float(tau), np.array(lengths, np.int32),
                    np.array(capacity, np.int32), key_dist, query_mode, ch, "edge case")


# ------------------------------------------------------- LoopVQ workloads
# Codebook-coded caches for the LoopVQ decode ("LoopVQ: Sub 1-bit KV Cache
# Quantization for Looped Transformers"): per (layer, sequence, KV head,
# token) D/4 key and D/4 value indices, uniform over the 256 entries; per
# (layer, KV head) a key and a value codebook of N(0,1) entries [256][4 L];
# queries 2 * N(0,1).  which: 0 keys, 1 values.

@dataclasses.dataclass
class VqWorkload:
    name: str
    n_loops: int
    n_layers: int
    n_heads: int
    head_dim: int
    batch: int
    seed: int
    lengths: np.ndarray      # int32 [batch]: coded tokens per unit
    capacity: int            # token stride of the index arrays
    description: str = ""

    @property
    def n_cells(self):
        return self.n_loops * self.n_layers


def make_vq(config="vq16k", **over):
    """LoopVQ workload: "vq16k" (the batched 16K shape) or "vqsmall"."""
    if config == "vq16k":
        wl = VqWorkload("vq-batched-16k", 4, 24, 16, 128, 32, 12, np.full(32, 16384, np.int32),
                        16384, "4 loops x 24 layers, 16 KV heads, D 128, batch 32, 16384 coded tokens")
    elif config == "vqsmall":
        wl = VqWorkload("vq-small", 4, 2, 2, 128, 3, 13, np.array([1, 33, 700], np.int32), 704,
                        "4 loops x 2 layers, 2 KV heads, D 128, batch 3, ragged")
    else:
        raise ValueError("unknown LoopVQ config %r" % config)
    for k, v in over.items():
        setattr(wl, k, v)
    return wl


def vq_indices(wl, which, layer, b, h, t0, t1):
    """uint8 [t1 - t0, D/4]: codebook indices of tokens t0..t1-1 of a unit."""
    groups = wl.head_dim // 4
    t = np.arange(t0, t1, dtype=np.uint32)[:, None]
    j = np.arange(groups, dtype=np.uint32)[None, :]
    u = px.philox4x32(t, j, np.uint32(h + wl.n_heads * b), np.uint32(layer | (which << 16)),
                      wl.seed, STREAM_VQ_IDX)
    return (u[0] & np.uint32(255)).astype(np.uint8)


def vq_codebook(wl, which, layer, h):
    """fp32 [256, 4 * n_loops]: the key (which 0) or value (1) codebook."""
    e = np.arange(256, dtype=np.uint32)[:, None]
    k = np.arange(4 * wl.n_loops, dtype=np.uint32)[None, :]
    u = px.philox4x32(e, k, np.uint32(h), np.uint32(layer | (which << 16)), wl.seed, STREAM_VQ_CB)
    return px.normal_from_bits(*u)


def vq_query(wl, loop, layer, b, h):
    """bf16 bits [D]: the query of (loop, layer, sequence, KV head)."""
    d = np.arange(wl.head_dim, dtype=np.uint32)
    u = px.philox4x32(d, np.uint32(loop), np.uint32(h + wl.n_heads * b), np.uint32(layer), wl.seed,
                      STREAM_VQ_Q)
    z = px.normal_from_bits(*u)
    return px.float_to_bf16_bits((np.float32(2.0) * z).astype(np.float32))
