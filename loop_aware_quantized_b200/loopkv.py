"""Python binding of the LoopKV C ABI (``include/loopkv.h``).

Argument marshalling only: every step of append and decode runs in the CUDA
library ``libloopkv.so`` built in-tree for sm_100a.  PyTorch supplies device
memory and streams.  Importing this module on a machine where the library is
missing raises immediately; there is no other code path.

Low-level functions carry the C names (``loopkv_plan_query``,
``loopkv_append`` ...) and take raw pointers; ``Plan`` wraps a plan handle
together with the torch tensors that hold its table and cache.
"""

import ctypes
import os

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libloopkv.so")

LOOPKV_Q4, LOOPKV_Q2, LOOPKV_SHARE, LOOPKV_BF16, LOOPKV_RES2 = 0, 1, 2, 3, 4
LOOPKV_MAX_CELLS_PER_CALL = 256
LOOPKV_MAX_BATCH = 256

STATUS = {
    0: "LOOPKV_OK",
    1: "LOOPKV_ERR_INVALID_ARG",
    2: "LOOPKV_ERR_PLAN",
    3: "LOOPKV_ERR_CAPACITY",
    4: "LOOPKV_ERR_UNSUPPORTED",
    5: "LOOPKV_ERR_CUDA",
    6: "LOOPKV_ERR_DEVICE",
}


class LoopKVError(RuntimeError):
    def __init__(self, status, where):
        self.status = status
        super().__init__("%s: %s (%s)" % (where, STATUS.get(status, status),
                                          loopkv_status_string(status)))


class loopkv_plan_desc(ctypes.Structure):
    _fields_ = [
        ("n_loops", ctypes.c_int32),
        ("n_layers", ctypes.c_int32),
        ("n_kv_heads", ctypes.c_int32),
        ("head_dim", ctypes.c_int32),
        ("max_batch", ctypes.c_int32),
        ("capacity", ctypes.POINTER(ctypes.c_int32)),
        ("kinds", ctypes.POINTER(ctypes.c_uint8)),
        ("tau", ctypes.c_float),
        ("sm_scale", ctypes.c_float),
        ("q_per_kv", ctypes.c_int32),
        ("decode_split", ctypes.c_int32),
    ]


class loopkv_planner_desc(ctypes.Structure):
    _fields_ = [
        ("n_loops", ctypes.c_int32),
        ("n_layers", ctypes.c_int32),
        ("head_dim", ctypes.c_int32),
        ("damage", ctypes.POINTER(ctypes.c_int32)),
        ("damage_budget", ctypes.c_int64),
        ("storage_budget", ctypes.c_int64),
        ("sel_fraction", ctypes.c_float),
    ]


class loopkv_plan_cost(ctypes.Structure):
    _fields_ = [("reads", ctypes.c_double), ("damage", ctypes.c_int64), ("storage", ctypes.c_int64)]


class loopkv_vq_desc(ctypes.Structure):
    _fields_ = [
        ("n_loops", ctypes.c_int32),
        ("n_layers", ctypes.c_int32),
        ("n_kv_heads", ctypes.c_int32),
        ("head_dim", ctypes.c_int32),
        ("batch", ctypes.c_int32),
        ("capacity", ctypes.c_int32),
        ("sm_scale", ctypes.c_float),
    ]


class loopkv_sizes(ctypes.Structure):
    _fields_ = [("table_bytes", ctypes.c_size_t), ("cache_bytes", ctypes.c_size_t)]


def _load():
    if not os.path.exists(LIB_PATH):
        raise ImportError(
            "libloopkv.so is missing (%s); build it with "
            "`python loop_aware_quantized_b200/build.py`" % LIB_PATH)
    lib = ctypes.CDLL(LIB_PATH)
    P = ctypes.c_void_p
    I32 = ctypes.c_int32
    st = ctypes.c_int
    sig = {
        "loopkv_plan_query": (st, [ctypes.POINTER(loopkv_plan_desc), ctypes.POINTER(loopkv_sizes)]),
        "loopkv_plan_load": (st, [ctypes.POINTER(loopkv_plan_desc), P, ctypes.c_size_t, P,
                                  ctypes.c_size_t, P, ctypes.POINTER(P)]),
        "loopkv_plan_free": (None, [P]),
        "loopkv_append": (st, [P, P, I32, I32, P, I32, P, P, P]),
        "loopkv_decode": (st, [P, P, I32, I32, P, P, P, P, I32, P, P]),
        "loopkv_set_lengths": (st, [P, P, I32, I32, P, P]),
        "loopkv_get_lengths": (st, [P, P]),
        "loopkv_unit_region": (st, [P, I32, I32, I32, ctypes.POINTER(ctypes.c_uint64),
                                    ctypes.POINTER(ctypes.c_uint64)]),
        "loopkv_check": (st, [P, P]),
        "loopkv_status_string": (ctypes.c_char_p, [ctypes.c_int]),
        "loopkv_plan_optimize": (st, [ctypes.POINTER(loopkv_planner_desc), P,
                                      ctypes.POINTER(loopkv_plan_cost)]),
        "loopkv_vq_decode": (st, [ctypes.POINTER(loopkv_vq_desc), I32, P, P, P, P, P, P, P, P,
                                  P]),
        "loopkv_vq_encode": (st, [ctypes.POINTER(loopkv_vq_desc), P, I32, P, P, P, P]),
    }
    for name, (res, args) in sig.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    return lib


_lib = _load()


# ----------------------------------------------------------- C-named calls

def loopkv_status_string(status):
    return _lib.loopkv_status_string(int(status)).decode()


def loopkv_plan_query(desc):
    sizes = loopkv_sizes()
    ref = None if desc is None else ctypes.byref(desc)
    return _lib.loopkv_plan_query(ref, ctypes.byref(sizes)), sizes


def loopkv_plan_load(desc, d_table, table_bytes, d_cache, cache_bytes, stream):
    handle = ctypes.c_void_p()
    rc = _lib.loopkv_plan_load(ctypes.byref(desc), d_table, table_bytes, d_cache, cache_bytes,
                               stream, ctypes.byref(handle))
    return rc, handle


def loopkv_plan_free(handle):
    _lib.loopkv_plan_free(handle)


def loopkv_append(handle, h_cells, n_cells, batch, h_n_new, n_new_max, d_k, d_v, stream):
    return _lib.loopkv_append(handle, h_cells, n_cells, batch, h_n_new, n_new_max, d_k, d_v,
                              stream)


def loopkv_decode(handle, h_cells, n_cells, batch, d_q, d_out, d_lse, d_mask, mask_words,
                  d_nsel, stream):
    return _lib.loopkv_decode(handle, h_cells, n_cells, batch, d_q, d_out, d_lse, d_mask,
                              mask_words, d_nsel, stream)


def loopkv_vq_decode(desc, loop, h_len, d_idx_k, d_idx_v, d_cb_k, d_cb_v, d_q, d_out, d_lse,
                     stream):
    ref = None if desc is None else ctypes.byref(desc)
    return _lib.loopkv_vq_decode(ref, loop, h_len, d_idx_k, d_idx_v, d_cb_k, d_cb_v, d_q, d_out,
                                 d_lse, stream)


def loopkv_vq_encode(desc, h_pos, n_new, d_x, d_cb, d_idx, stream):
    ref = None if desc is None else ctypes.byref(desc)
    return _lib.loopkv_vq_encode(ref, h_pos, n_new, d_x, d_cb, d_idx, stream)


def loopkv_plan_optimize(desc, kinds_out):
    cost = loopkv_plan_cost()
    ref = None if desc is None else ctypes.byref(desc)
    return _lib.loopkv_plan_optimize(ref, kinds_out, ctypes.byref(cost)), cost


def loopkv_set_lengths(handle, h_cells, n_cells, batch, h_len, stream):
    return _lib.loopkv_set_lengths(handle, h_cells, n_cells, batch, h_len, stream)


def loopkv_get_lengths(handle, h_len):
    return _lib.loopkv_get_lengths(handle, h_len)


def loopkv_unit_region(handle, cell, seq, head):
    off = ctypes.c_uint64()
    nbytes = ctypes.c_uint64()
    rc = _lib.loopkv_unit_region(handle, cell, seq, head, ctypes.byref(off), ctypes.byref(nbytes))
    return rc, off.value, nbytes.value


def loopkv_check(handle, stream):
    return _lib.loopkv_check(handle, stream)


# ------------------------------------------------------------------ helpers

def _np_ptr(a):
    return a.ctypes.data_as(ctypes.c_void_p)


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream_handle(stream):
    import torch
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def _check(rc, where):
    if rc != 0:
        raise LoopKVError(rc, where)


def _invalid(where, what):
    return LoopKVError(1, "%s: %s" % (where, what))


def _need(t, where, name, dtypes, shape=None, ndim=None, device=None, optional=False):
    """Check a tensor argument before its pointer reaches the library: a
    contiguous CUDA tensor of one of ``dtypes``, with ``shape`` (or ``ndim``
    dimensions) and on ``device`` when given.  The library sees only pointers,
    so these are the checks it cannot make; a failure raises LoopKVError
    with LOOPKV_ERR_INVALID_ARG and launches nothing."""
    import torch
    if t is None:
        if optional:
            return
        raise _invalid(where, "%s is required" % name)
    if not isinstance(t, torch.Tensor):
        raise _invalid(where, "%s must be a torch tensor, not %s" % (name, type(t).__name__))
    if not t.is_cuda:
        raise _invalid(where, "%s must be on a CUDA device, not %s" % (name, t.device))
    if device is not None and t.device != device:
        raise _invalid(where, "%s is on %s, expected %s" % (name, t.device, device))
    if t.dtype not in dtypes:
        raise _invalid(where, "%s must be %s, not %s" % (
            name, " or ".join(str(d) for d in dtypes), t.dtype))
    if not t.is_contiguous():
        raise _invalid(where, "%s must be contiguous" % name)
    if ndim is not None and t.dim() != ndim:
        raise _invalid(where, "%s must have %d dimensions, not %d" % (name, ndim, t.dim()))
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise _invalid(where, "%s must have shape %s, not %s" % (
            name, tuple(shape), tuple(t.shape)))


def _host_ints(a, where, name, size):
    a = np.ascontiguousarray(a, dtype=np.int32)
    if a.size != size:
        raise _invalid(where, "%s must hold %d values, not %d" % (name, size, a.size))
    return a


def _int_dtypes():
    import torch
    u32 = getattr(torch, "uint32", None)
    return (torch.int32,) if u32 is None else (torch.int32, u32)


def make_desc(n_loops, n_layers, n_kv_heads, head_dim, capacity, kinds, tau, sm_scale=0.0,
              q_per_kv=1, decode_split=0):
    """Build a loopkv_plan_desc; returns (desc, keepalive arrays)."""
    cap = np.ascontiguousarray(capacity, dtype=np.int32)
    kinds = np.ascontiguousarray(kinds, dtype=np.uint8)
    d = loopkv_plan_desc()
    d.n_loops, d.n_layers, d.n_kv_heads, d.head_dim = n_loops, n_layers, n_kv_heads, head_dim
    d.max_batch = int(cap.size)
    d.capacity = cap.ctypes.data_as(ctypes.POINTER(ctypes.c_int32))
    d.kinds = kinds.ctypes.data_as(ctypes.POINTER(ctypes.c_uint8))
    d.tau = float(tau)
    d.sm_scale = float(sm_scale)
    d.q_per_kv = int(q_per_kv)
    d.decode_split = int(decode_split)
    return d, (cap, kinds)


def query_sizes(n_loops, n_layers, n_kv_heads, head_dim, capacity, kinds, tau=0.0, q_per_kv=1):
    """(table_bytes, cache_bytes) a plan needs; raises LoopKVError if invalid."""
    d, keep = make_desc(n_loops, n_layers, n_kv_heads, head_dim, capacity, kinds, tau,
                        q_per_kv=q_per_kv)
    rc, sizes = loopkv_plan_query(d)
    _check(rc, "loopkv_plan_query")
    return int(sizes.table_bytes), int(sizes.cache_bytes)


class Plan:
    """A loaded LoopKV plan with its device table and cache (torch tensors)."""

    def __init__(self, n_loops, n_layers, n_kv_heads, head_dim, capacity, kinds, tau,
                 sm_scale=0.0, device="cuda", stream=None, q_per_kv=1, cache_guard=0,
                 decode_split=0):
        """cache_guard: extra bytes allocated after the cache (not given to the
        library), so tests can check that nothing is written past its end.
        decode_split: CTAs per decoded unit at least (0: the library chooses)."""
        import torch
        self.n_loops, self.n_layers = n_loops, n_layers
        self.n_cells = n_loops * n_layers
        self.n_heads, self.head_dim = n_kv_heads, head_dim
        self.capacity = np.ascontiguousarray(capacity, dtype=np.int32)
        self.max_batch = int(self.capacity.size)
        self.kinds = np.ascontiguousarray(kinds, dtype=np.uint8)
        self.tau = float(tau)
        self.q_per_kv = int(q_per_kv)
        d, keep = make_desc(n_loops, n_layers, n_kv_heads, head_dim, self.capacity, self.kinds,
                            tau, sm_scale, q_per_kv, decode_split)
        rc, sizes = loopkv_plan_query(d)
        _check(rc, "loopkv_plan_query")
        self.table_bytes, self.cache_bytes = int(sizes.table_bytes), int(sizes.cache_bytes)
        self.table = torch.empty(self.table_bytes, dtype=torch.uint8, device=device)
        self.cache = torch.empty(max(self.cache_bytes, 256) + int(cache_guard), dtype=torch.uint8,
                                 device=device)
        self._handle = None
        rc, h = loopkv_plan_load(d, _ptr(self.table), self.table_bytes, _ptr(self.cache),
                                 self.cache_bytes, _stream_handle(stream))
        _check(rc, "loopkv_plan_load")
        self._handle = h

    def close(self):
        if getattr(self, "_handle", None):
            loopkv_plan_free(self._handle)
            self._handle = None

    def __del__(self):
        self.close()

    @property
    def handle(self):
        return self._handle

    def source_cell(self, cell):
        return (self.n_loops - 1) * self.n_layers + cell % self.n_layers

    def append(self, cells, k, v, n_new=None, stream=None):
        """k, v: bf16 [n_cells, batch, H, n_new_max, D] on the device."""
        import torch
        where = "Plan.append"
        cells = np.ascontiguousarray(cells, dtype=np.int32).reshape(-1)
        dev = self.cache.device
        _need(k, where, "k", (torch.bfloat16,), ndim=5, device=dev)
        nc, batch, H, nmax, D = k.shape
        if nc != cells.size or H != self.n_heads or D != self.head_dim:
            raise _invalid(where, "k has shape %s; expected (%d cells, batch, %d heads, n_new_max, "
                                  "%d)" % (tuple(k.shape), cells.size, self.n_heads, self.head_dim))
        _need(v, where, "v", (torch.bfloat16,), shape=k.shape, device=dev)
        if n_new is None:
            n_new = np.full(batch, nmax, np.int32)
        n_new = _host_ints(n_new, where, "n_new", batch)
        rc = loopkv_append(self._handle, _np_ptr(cells), int(cells.size), int(batch),
                           _np_ptr(n_new), int(nmax), _ptr(k), _ptr(v), _stream_handle(stream))
        _check(rc, "loopkv_append")

    def decode(self, cells, q, out=None, lse=None, mask=None, nsel=None, stream=None):
        """q: bf16 [n_cells, batch, H, D] on the device, or [n_cells, batch, H,
        q_per_kv, D] for a plan with several query heads per KV head; returns
        out (fp32, same shape).  lse: [n_cells, batch, H(, q_per_kv)]; mask
        and nsel are per KV head."""
        import torch
        where = "Plan.decode"
        cells = np.ascontiguousarray(cells, dtype=np.int32).reshape(-1)
        dev = self.cache.device
        _need(q, where, "q", (torch.bfloat16,), device=dev)
        g = self.q_per_kv
        batch = q.shape[1] if q.dim() > 1 else -1
        want = (cells.size, batch, self.n_heads, g, self.head_dim)
        if tuple(q.shape) != want and (g > 1 or tuple(q.shape) != want[:3] + want[4:]):
            raise _invalid(where, "q has shape %s; expected (cells %d, batch, KV heads %d, "
                                  "query heads %d, head dim %d)%s" % (
                                      tuple(q.shape), cells.size, self.n_heads, g, self.head_dim,
                                      ", the query-head axis optional" if g == 1 else ""))
        nc, H = cells.size, self.n_heads
        if out is None:
            out = torch.empty(q.shape, dtype=torch.float32, device=q.device)
        _need(out, where, "out", (torch.float32,), shape=q.shape, device=dev)
        _need(lse, where, "lse", (torch.float32,), shape=q.shape[:-1], device=dev, optional=True)
        _need(nsel, where, "nsel", (torch.int32,), shape=(nc, batch, H), device=dev,
              optional=True)
        _need(mask, where, "mask", _int_dtypes(), ndim=4, device=dev, optional=True)
        if mask is not None and tuple(mask.shape[:3]) != (nc, batch, H):
            raise _invalid(where, "mask has shape %s; expected (%d, %d, %d, words)" % (
                tuple(mask.shape), nc, batch, H))
        mask_words = 0 if mask is None else int(mask.shape[-1])
        rc = loopkv_decode(self._handle, _np_ptr(cells), int(cells.size), int(batch), _ptr(q),
                           _ptr(out), _ptr(lse), _ptr(mask), mask_words, _ptr(nsel),
                           _stream_handle(stream))
        _check(rc, "loopkv_decode")
        return out

    def set_lengths(self, cells, lengths, stream=None):
        cells = np.ascontiguousarray(cells, dtype=np.int32).reshape(-1)
        lengths = np.ascontiguousarray(lengths, dtype=np.int32)
        batch = lengths.shape[-1] if lengths.ndim else 0
        if lengths.size != cells.size * batch:
            raise _invalid("Plan.set_lengths", "lengths must be [cells][batch], got shape %s for "
                                               "%d cells" % (lengths.shape, cells.size))
        rc = loopkv_set_lengths(self._handle, _np_ptr(cells), int(cells.size), int(batch),
                                _np_ptr(lengths), _stream_handle(stream))
        _check(rc, "loopkv_set_lengths")

    def lengths(self):
        out = np.zeros((self.n_cells, self.max_batch), np.int32)
        _check(loopkv_get_lengths(self._handle, _np_ptr(out)), "loopkv_get_lengths")
        return out

    def unit_region(self, cell, seq, head):
        rc, off, nbytes = loopkv_unit_region(self._handle, cell, seq, head)
        _check(rc, "loopkv_unit_region")
        return off, nbytes

    def unit_bytes(self, cell, seq, head):
        """Device bytes of a unit's region (a uint8 view into the cache)."""
        off, nbytes = self.unit_region(cell, seq, head)
        return self.cache[off:off + nbytes]

    def check(self, stream=None):
        _check(loopkv_check(self._handle, _stream_handle(stream)), "loopkv_check")


def plan_optimize(n_loops, n_layers, head_dim, damage, damage_budget, storage_budget,
                  sel_fraction=0.0):
    """Plan every cell (loop-major kinds) to minimize reads within a damage and
    a storage budget.  damage: int [n_loops * n_layers, 3] (Q4, Q2, SHARE);
    storage_budget: bytes per cached token and KV head.  Returns (kinds,
    {"reads", "damage", "storage"}); raises LoopKVError when nothing fits."""
    dmg = np.ascontiguousarray(damage, dtype=np.int32)
    if dmg.size != 3 * n_loops * n_layers:
        raise _invalid("plan_optimize", "damage must be [%d cells][3], got shape %s" % (
            n_loops * n_layers, dmg.shape))
    dmg = dmg.reshape(-1, 3)
    d = loopkv_planner_desc()
    d.n_loops, d.n_layers, d.head_dim = n_loops, n_layers, head_dim
    d.damage = dmg.ctypes.data_as(ctypes.POINTER(ctypes.c_int32))
    d.damage_budget, d.storage_budget = int(damage_budget), int(storage_budget)
    d.sel_fraction = float(sel_fraction)
    kinds = np.zeros(n_loops * n_layers, np.uint8)
    rc, cost = loopkv_plan_optimize(d, _np_ptr(kinds))
    _check(rc, "loopkv_plan_optimize")
    return kinds, {"reads": cost.reads, "damage": int(cost.damage), "storage": int(cost.storage)}


def vq_decode(loop, lengths, idx_k, idx_v, cb_k, cb_v, q, out=None, lse=None, sm_scale=0.0,
              stream=None):
    """LoopVQ decode of loop ``loop`` for every (layer, sequence, KV head).

    idx_k / idx_v: uint8 [n_layers, batch, H, capacity, D/4]; cb_k / cb_v:
    fp32 [n_layers, H, 256, 4 * n_loops]; q: bf16 [n_layers, batch, H, D];
    lengths: host [batch] coded tokens.  Returns out (fp32, q's shape)."""
    import torch
    where = "vq_decode"
    _need(q, where, "q", (torch.bfloat16,), ndim=4)
    dev = q.device
    n_layers, batch, H, D = q.shape
    _need(idx_k, where, "idx_k", (torch.uint8,), ndim=5, device=dev)
    cap = idx_k.shape[3]
    if tuple(idx_k.shape) != (n_layers, batch, H, cap, D // 4) or D % 4:
        raise _invalid(where, "idx_k has shape %s; expected (%d, %d, %d, capacity, %d)" % (
            tuple(idx_k.shape), n_layers, batch, H, D // 4))
    _need(idx_v, where, "idx_v", (torch.uint8,), shape=idx_k.shape, device=dev)
    _need(cb_k, where, "cb_k", (torch.float32,), ndim=4, device=dev)
    if tuple(cb_k.shape[:3]) != (n_layers, H, 256) or cb_k.shape[3] % 4:
        raise _invalid(where, "cb_k has shape %s; expected (%d, %d, 256, 4 * loops)" % (
            tuple(cb_k.shape), n_layers, H))
    _need(cb_v, where, "cb_v", (torch.float32,), shape=cb_k.shape, device=dev)
    if out is None:
        out = torch.empty(q.shape, dtype=torch.float32, device=dev)
    _need(out, where, "out", (torch.float32,), shape=q.shape, device=dev)
    _need(lse, where, "lse", (torch.float32,), shape=q.shape[:-1], device=dev, optional=True)
    d = loopkv_vq_desc(cb_k.shape[3] // 4, n_layers, H, D, batch, cap, float(sm_scale))
    lengths = _host_ints(lengths, where, "lengths", batch)
    rc = loopkv_vq_decode(d, int(loop), _np_ptr(lengths), _ptr(idx_k), _ptr(idx_v), _ptr(cb_k),
                          _ptr(cb_v), _ptr(q), _ptr(out), _ptr(lse), _stream_handle(stream))
    _check(rc, "loopkv_vq_decode")
    return out


def vq_encode(positions, x, cb, idx, stream=None):
    """LoopVQ encoder: x bf16 [n_loops, n_layers, batch, H, n_new, D] (each
    token in every loop of its layer) -> codebook indices written into idx
    (uint8 [n_layers, batch, H, capacity, D/4]) at positions[b] + i, using cb
    (fp32 [n_layers, H, 256, 4 * n_loops]).  Returns idx."""
    import torch
    where = "vq_encode"
    _need(x, where, "x", (torch.bfloat16,), ndim=6)
    dev = x.device
    L, n_layers, batch, H, n_new, D = x.shape
    _need(idx, where, "idx", (torch.uint8,), ndim=5, device=dev)
    if tuple(idx.shape) != (n_layers, batch, H, idx.shape[3], D // 4) or D % 4:
        raise _invalid(where, "idx has shape %s; expected (%d, %d, %d, capacity, %d)" % (
            tuple(idx.shape), n_layers, batch, H, D // 4))
    _need(cb, where, "cb", (torch.float32,), shape=(n_layers, H, 256, 4 * L), device=dev)
    d = loopkv_vq_desc(L, n_layers, H, D, batch, idx.shape[3], 0.0)
    positions = _host_ints(positions, where, "positions", batch)
    rc = loopkv_vq_encode(d, _np_ptr(positions), int(n_new), _ptr(x), _ptr(cb), _ptr(idx),
                          _stream_handle(stream))
    _check(rc, "loopkv_vq_encode")
    return idx
