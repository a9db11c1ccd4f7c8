"""One decode step of a looped model in serving order, on a loaded ``Plan``.

A looped transformer runs loop 0 over all layers, then loop 1, and so on; the
final loop's KV is what SHARE cells reuse ("LoopKV: Loop-Aware KV Cache
Compression for Serving Looped Transformers", section 概要).  So for one new
token the cache sees: append + decode for the cells of the non-final loops
(their SHARE units read the final loop's positions < n-1, all stored by the
previous step), then append + decode for the final loop.  Batching all cells
of a phase into one launch is the throughput form of that order.

Only library calls (``Plan.append``, ``Plan.decode``) are issued here.
"""

import numpy as np


def phases(n_loops, n_layers):
    """Cell lists of the two phases: non-final loops, then the final loop."""
    nonfinal = np.arange((n_loops - 1) * n_layers, dtype=np.int32)
    final = np.arange((n_loops - 1) * n_layers, n_loops * n_layers, dtype=np.int32)
    return [c for c in (nonfinal, final) if c.size]


def decode_step(plan, phase_cells, q, k_new, v_new, out, lse=None, mask=None, nsel=None,
                n_new=None, stream=None, events=None):
    """Append one token per (cell, sequence, head) and decode, phase by phase.

    For phase i: q[i] bf16 [cells, batch, H, D], k_new[i] / v_new[i] bf16
    [cells, batch, H, 1, D], out[i] fp32 [cells, batch, H, D] (lse, mask,
    nsel optional lists of the same arity).  ``events`` (optional) is a list
    of (start, end) CUDA event pairs recorded around each decode launch.
    """
    for i, cells in enumerate(phase_cells):
        plan.append(cells, k_new[i], v_new[i], n_new=n_new, stream=stream)
        if events is not None:
            events[i][0].record(stream)
        plan.decode(cells, q[i], out=out[i], lse=None if lse is None else lse[i],
                    mask=None if mask is None else mask[i],
                    nsel=None if nsel is None else nsel[i], stream=stream)
        if events is not None:
            events[i][1].record(stream)
