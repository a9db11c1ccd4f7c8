"""Device-side generation of the synthetic workloads (``csrc/synth.cu``).

Produces the same bits as ``workloads.raw_keys`` / ``raw_values`` / ``query``
on the host.  Torch provides the device buffers.
"""

import ctypes
import os

import numpy as np

from . import philox as px
from . import workloads as W

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libloopkv_synth.so")
_lib = None


def _ok(rc):
    """A generator call's status: 0, -1 for a range the output cannot hold, or
    the CUDA error its launch returned."""
    if rc != 0:
        raise RuntimeError("synthetic input generator failed with status %d" % rc)


def _load():
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError("libloopkv_synth.so is missing; run `python synth/build.py`")
        lib = ctypes.CDLL(LIB_PATH)
        P, I = ctypes.c_void_p, ctypes.c_int
        lib.synth_gen_kv.argtypes = [P, P, P, P, P, I, I, I, I, I, I, P, P, ctypes.c_uint32,
                                     ctypes.c_float, P]
        lib.synth_gen_kv.restype = I
        lib.synth_gen_q.argtypes = [P, P, P, P, P, I, I, I, I, I, I, I, P, P, ctypes.c_uint32,
                                    ctypes.c_float, P]
        lib.synth_gen_q.restype = I
        lib.synth_gen_vq_idx.argtypes = [P, I, I, I, I, I, I, I, I, ctypes.c_uint32, P]
        lib.synth_gen_vq_idx.restype = I
        lib.synth_gen_vq_q.argtypes = [P, I, I, I, I, I, I, ctypes.c_uint32, ctypes.c_float, P]
        lib.synth_gen_vq_q.restype = I
        lib.synth_philox.argtypes = [P, P, I, P]
        lib.synth_philox.restype = I
        _lib = lib
    return _lib


def _p(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def philox_rows(rows, device="cuda"):
    """The device generator's Philox4x32-10 of (c0, c1, c2, c3, k0, k1) rows ->
    uint32 [n][4] (host array)."""
    import torch
    a = np.ascontiguousarray(rows, dtype=np.uint32).reshape(-1, 6)
    d_in = torch.from_numpy(a.view(np.int32)).to(device)
    d_out = torch.empty((a.shape[0], 4), dtype=torch.int32, device=device)
    _ok(_load().synth_philox(_p(d_in), _p(d_out), a.shape[0], None))
    torch.cuda.synchronize()
    return d_out.cpu().numpy().view(np.uint32)


class DeviceGenerator:
    """Generates a workload's raw keys, values and queries on a CUDA device."""

    def __init__(self, wl, device="cuda"):
        import torch
        self.wl = wl
        self.device = torch.device(device)
        self.chscale = torch.from_numpy(np.ascontiguousarray(wl.chscale)).to(self.device)
        # per cell: the reference cell a residual cell's tokens follow, else -1
        self.refs = self._i32([wl.token_ref(c) for c in range(wl.n_cells)])
        self.nscale = float(px.NORMAL_SCALE)

    def _i32(self, a):
        import torch
        return torch.from_numpy(np.ascontiguousarray(a, dtype=np.int32)).to(self.device)

    def kv(self, cells, seqs, t0, T, k=None, v=None, stream=None):
        """bf16 [n_cells, len(seqs), H, T, D] keys and values at positions t0[b] + i."""
        import torch
        wl = self.wl
        shape = (len(cells), len(seqs), wl.n_heads, T, wl.head_dim)
        if k is None:
            k = torch.empty(shape, dtype=torch.bfloat16, device=self.device)
        if v is None:
            v = torch.empty(shape, dtype=torch.bfloat16, device=self.device)
        s = torch.cuda.current_stream() if stream is None else stream
        # the index tensors must outlive the launch (a freed block is reused
        # by the next allocation before the kernel runs)
        d_cells, d_seqs, d_t0 = self._i32(cells), self._i32(seqs), self._i32(t0)
        rc = _load().synth_gen_kv(_p(k), _p(v), _p(d_cells), _p(d_seqs), _p(d_t0), len(cells),
                                  len(seqs), wl.n_heads, wl.head_dim, T, wl.n_cells,
                                  _p(self.chscale), _p(self.refs),
                                  wl.seed, self.nscale, ctypes.c_void_p(s.cuda_stream))
        s.synchronize()
        del d_cells, d_seqs, d_t0
        _ok(rc)
        return k, v

    def queries(self, cells, seqs, lens, out=None, stream=None, g=1):
        """bf16 [n_cells, len(seqs), H, D] (g = 1) or [n_cells, len(seqs), H, g, D]
        (g query heads per KV head); lens [n_cells, len(seqs)] = unit lengths."""
        import torch
        wl = self.wl
        srcs = [wl.data_cell(c) for c in cells]
        shape = (len(cells), len(seqs), wl.n_heads) + ((g,) if g > 1 else ()) + (wl.head_dim,)
        if out is None:
            out = torch.empty(shape, dtype=torch.bfloat16, device=self.device)
        mode = 0 if wl.query_mode == "sum3" else 1
        s = torch.cuda.current_stream() if stream is None else stream
        d_cells, d_srcs, d_seqs = self._i32(cells), self._i32(srcs), self._i32(seqs)
        d_lens = self._i32(np.asarray(lens).reshape(-1))
        rc = _load().synth_gen_q(_p(out), _p(d_cells), _p(d_srcs), _p(d_seqs), _p(d_lens),
                                 len(cells), len(seqs), wl.n_heads, g, wl.head_dim, mode,
                                 wl.n_cells, _p(self.chscale), _p(self.refs), wl.seed, self.nscale,
                                 ctypes.c_void_p(s.cuda_stream))
        s.synchronize()
        del d_cells, d_srcs, d_seqs, d_lens
        _ok(rc)
        return out


def host_kv(wl, cell, b, h, t0, t1):
    """Host twin: (keys, values) bf16 bits [t1 - t0, D]."""
    return W.raw_keys(wl, cell, b, h, t0, t1), W.raw_values(wl, cell, b, h, t0, t1)


class VqDeviceGenerator:
    """LoopVQ inputs on a CUDA device (same bits as the host generator).

    seq0: global id of the first sequence (ranks of a multi-GPU run serve
    disjoint sequences)."""

    def __init__(self, wl, device="cuda", seq0=0):
        import torch
        self.wl = wl
        self.seq0 = int(seq0)
        self.device = torch.device(device)
        self.nscale = float(px.NORMAL_SCALE)

    def indices(self, which, T=None, out=None):
        """uint8 [n_layers, batch, H, capacity, D/4]; tokens < T filled."""
        import torch
        wl = self.wl
        T = wl.capacity if T is None else T
        shape = (wl.n_layers, wl.batch, wl.n_heads, wl.capacity, wl.head_dim // 4)
        if out is None:
            out = torch.zeros(shape, dtype=torch.uint8, device=self.device)
        s = torch.cuda.current_stream()
        rc = _load().synth_gen_vq_idx(_p(out), wl.n_layers, wl.batch, wl.n_heads, wl.head_dim,
                                      wl.capacity, int(T), int(which), self.seq0, wl.seed,
                                      ctypes.c_void_p(s.cuda_stream))
        s.synchronize()
        _ok(rc)
        return out

    def codebooks(self, which):
        """fp32 [n_layers, H, 256, 4 * n_loops] from the host generator (small)."""
        import torch
        wl = self.wl
        cb = np.stack([np.stack([W.vq_codebook(wl, which, layer, h) for h in range(wl.n_heads)])
                       for layer in range(wl.n_layers)])
        return torch.from_numpy(np.ascontiguousarray(cb)).to(self.device)

    def queries(self, loop, out=None):
        """bf16 [n_layers, batch, H, D] of one loop."""
        import torch
        wl = self.wl
        shape = (wl.n_layers, wl.batch, wl.n_heads, wl.head_dim)
        if out is None:
            out = torch.empty(shape, dtype=torch.bfloat16, device=self.device)
        s = torch.cuda.current_stream()
        rc = _load().synth_gen_vq_q(_p(out), wl.n_layers, wl.batch, wl.n_heads, wl.head_dim,
                                    int(loop), self.seq0, wl.seed, self.nscale,
                                    ctypes.c_void_p(s.cuda_stream))
        s.synchronize()
        _ok(rc)
        return out
