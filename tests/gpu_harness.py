"""Build LoopKV caches for the seeded workloads on the GPU and compare sampled
units with the CPU oracle.  Used by the ``-m gpu`` tests and by the smoke
check; never by the library."""

import numpy as np

from tests import parity as P
from synth import workloads as W


def make_plan(wl, seqs, decode_split=0):
    from loop_aware_quantized_b200 import Plan
    return Plan(wl.n_loops, wl.n_layers, wl.n_heads, wl.head_dim, wl.capacity[seqs], wl.kinds,
                wl.tau, decode_split=decode_split)


def build_cache(wl, plan, gen, seqs, lengths, cells=None, chunk_tokens=None):
    """Append every token of [0, lengths[b]) to each cell (one call per cell).

    The final loop's cells go first: a RES2 cell quantizes its residuals
    against them, so they must hold the tokens before it does."""
    cells = list(range(wl.n_cells)) if cells is None else list(cells)
    cells.sort(key=lambda c: c // wl.n_layers != wl.n_loops - 1)
    T = int(max(lengths))
    kbuf = vbuf = None
    for c in cells:
        kbuf, vbuf = gen.kv([c], seqs, np.zeros(len(seqs), np.int32), T, k=kbuf, v=vbuf)
        plan.append([c], kbuf, vbuf, n_new=np.asarray(lengths, np.int32))
    return kbuf, vbuf


def decode_all(wl, plan, gen, seqs, cells, lens, device, with_mask=True):
    """Decode `cells` for queries of units with lengths lens[c][b]; host copies of outputs."""
    import torch
    q = gen.queries(cells, seqs, lens)
    n = (len(cells), len(seqs), wl.n_heads)
    out = torch.empty(n + (wl.head_dim,), dtype=torch.float32, device=device)
    lse = torch.empty(n, dtype=torch.float32, device=device)
    nsel = torch.empty(n, dtype=torch.int32, device=device)
    mw = int(wl.capacity.max()) // 32 + 1
    mask = torch.zeros(n + (mw,), dtype=torch.int32, device=device) if with_mask else None
    plan.decode(cells, q, out=out, lse=lse, mask=mask, nsel=nsel)
    torch.cuda.synchronize()
    return dict(q=q.view(torch.int16).cpu().numpy().view(np.uint16), out=out.cpu().numpy(),
                lse=lse.cpu().numpy(), nsel=nsel.cpu().numpy(),
                mask=None if mask is None else mask.cpu().numpy().view(np.uint32))


def sample_units(wl, cells, seqs, n, seed):
    """Up to n (ci, bl, h) units, covering every kind present, seeded."""
    rng = np.random.default_rng(seed)
    by_kind = {}
    for ci, c in enumerate(cells):
        by_kind.setdefault(int(wl.kinds[c]), []).append(ci)
    units = []
    kinds = sorted(by_kind)
    for i in range(n):
        ci = int(rng.choice(by_kind[kinds[i % len(kinds)]]))
        units.append((ci, int(rng.integers(len(seqs))), int(rng.integers(wl.n_heads))))
    return sorted(set(units))


def compare(config, wl, plan, res, cells, seqs, units, own_len, src_len, pool, check_bytes=True):
    """Oracle-check sampled units.  own_len / src_len: fn(cell, b_global) -> tokens."""
    jobs = []
    for ci, bl, h in units:
        c, b = cells[ci], seqs[bl]
        jobs.append((config, c, b, h, own_len(c, b), src_len(c, b), check_bytes))
    refs = pool.map(P.oracle_unit_job, jobs)
    stats = []
    for (ci, bl, h), job, ref in zip(units, jobs, refs):
        tag = "cfg%s cell%d b%d h%d (%s)" % (config, job[1], job[2], h, W.KIND_NAMES[ref["kind"]])
        assert (res["q"][ci, bl, h] == ref["q"]).all(), tag + ": device query differs from host"
        mask = None if res["mask"] is None else res["mask"][ci, bl, h]
        st = P.check_unit(tag, ref, res["out"][ci, bl, h], lse=res["lse"][ci, bl, h], mask=mask,
                          nsel=res["nsel"][ci, bl, h], tau=wl.tau)
        if check_bytes:
            P.check_bytes(tag, ref, plan.unit_bytes(job[1], bl, h).cpu().numpy())
        stats.append(st)
    return stats
